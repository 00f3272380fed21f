// Split-KV GQA decode for the low-rank form: shared basis + per-layer int8 residual.
//
// Per token t of layer l (pair p), the pages' reconstruction ("DepthWeave-KV:
// Smarter KV Cache Compression by Sharing Across Layers and Adapting Per Token",
// Core Mechanism: shared basis plus a per-layer low-rank quantised residual at a
// per-token rank) reads
//   K~_t = C_K[t] B_K + s_K[t] (U_K[t] masked to i < r_t) R_K        (same for V).
// Rebuilding K~_t costs 2 * 48 * d multiply-adds per token, far more than the
// ~165 bytes the token costs to read, so the projections are absorbed into the
// query and the output instead (exact in real arithmetic):
//   score_t = C_K[t] . (B_K q) + s_K[t] * (U_K[t] . (R_K q))
//   c^ = sum_t p_t C_V[t],   u^ = sum_t p_t s_V[t] U_V[t],   o = (c^ B_V + u^ R_V) / sum_t p_t
// This is the "basis lookup, residual dequantisation and attention projection in
// a single pass" the DepthWeave pages describe, restated for sm_100a:
//   - TMA streams coefficient tiles (64/128-B swizzle) and int8 code tiles per warp;
//   - q~ = B_K q and q^ = R_K q are split into bf16 hi + lo halves so the score
//     MMAs (mma.sync m16n8k16) keep ~16 bits of the fp32 projection;
//   - int8 codes convert exactly to bf16 B operands, masked by the token's rank;
//   - c^ and u^ accumulate in fp32 MMA accumulators; one projection per CTA.
#include "kvs_device.cuh"

namespace kvs {
namespace {

constexpr int NW = 4;
constexpr int RM = 16;

template <int RB>
struct CoefLayout {
    // bytes of one token row, TMA box inner width (elements), halves per row
    static constexpr int ROW = RB * 2;
    static constexpr int BOX = RB < 64 ? RB : 64;
    static constexpr int HALVES = RB / BOX;
    // byte offset of 16-B chunk c of token row t in a tile of TT rows
    template <int TT>
    __device__ static __forceinline__ uint32_t off(int t, int c) {
        if (RB == 32) return static_cast<uint32_t>(t * 64 + (((c ^ (t >> 1)) & 3) << 4));
        return static_cast<uint32_t>((c >> 3) * (TT * 128) + t * 128 + ((((c & 7) ^ t) & 7) << 4));
    }
};

template <int D, int RB, int TT, int NSW>
struct LrCfg {
    using L = CoefLayout<RB>;
    static constexpr int COEF_BYTES = TT * RB * 2;
    static constexpr int U_BYTES = TT * RM;
    static constexpr int STAGE_BYTES = 2 * COEF_BYTES + 2 * U_BYTES;
    static constexpr int RING_BYTES = NW * NSW * STAGE_BYTES;
    // per-warp scratch of per-token s_K, s_V (fp32) and rank (int)
    static constexpr int TOK_BYTES = NW * TT * 3 * 4;
    static constexpr int PD = RB + RM;    // coefficient-space partial width
    static constexpr int COMBINE_FLOATS = NW * 16 * PD + 2 * NW * 16 + 32 + 16 * PD + 16 * D + MAX_GROUP * MAX_SPLITS + 64;
    static constexpr int QPROJ_FLOATS = 16 * PD;
    static constexpr int BODY0 = RING_BYTES > COMBINE_FLOATS * 4 ? RING_BYTES : COMBINE_FLOATS * 4;
    static constexpr int SMEM = BODY0 + TOK_BYTES + QPROJ_FLOATS * 4 + 1024;
    static_assert(TT % 16 == 0 && COEF_BYTES % 1024 == 0, "tile shape");
};

__device__ __forceinline__ uint32_t pack_i8_bf16(int a, int b) {
    return pack_bf16(static_cast<float>(a), static_cast<float>(b));
}

template <int D, int RB, int TT, int NSW>
__global__ void __launch_bounds__(NW * 32)
decode_lowrank_kernel(const __grid_constant__ CUtensorMap tmCK, const __grid_constant__ CUtensorMap tmCV,
                      const __grid_constant__ CUtensorMap tmUK, const __grid_constant__ CUtensorMap tmUV,
                      const DecodeArgs a) {
    using C = LrCfg<D, RB, TT, NSW>;
    using LY = typename C::L;
    extern __shared__ uint8_t smem_dyn[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
    float* tok = reinterpret_cast<float*>(smem + C::BODY0);                    // [NW][3][TT]
    float* qproj = tok + NW * TT * 3;                                          // [16][RB + RM]
    __shared__ __align__(8) uint64_t bars[NW * NSW + 1];

    const int split = blockIdx.x;
    const int j = blockIdx.y;
    const int b = blockIdx.z;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int g = a.g;
    const int ntiles = (a.T + TT - 1) / TT;
    const int tile0 = split * a.tiles_per_split;
    const int tile1 = min(tile0 + a.tiles_per_split, ntiles);
    const int crow = (a.pair * a.B + b) * a.Hkv + j;        // coefficient row in [P*B*Hkv]
    const int urow = b * a.Hkv + j;                         // code row within the layer's [B*Hkv]
    const size_t tokrow = static_cast<size_t>(b * a.Hkv + j) * a.T;   // s_K / s_V row start
    const uint8_t* rank_row = a.rank + static_cast<size_t>(b) * a.T;

    if (threadIdx.x == 0) {
        for (int i = 0; i < NW * NSW + 1; ++i) mbar_init(&bars[i], 1);
        mbar_init_fence();
    }
    // ---- q~ = B_K q and q^ = R_K q for the g heads (fp32, into shared memory)
    {
        const uint16_t* qb = reinterpret_cast<const uint16_t*>(a.q) +
                             (static_cast<size_t>(b) * a.Hq + static_cast<size_t>(j) * g) * D;
        const uint16_t* Bk = reinterpret_cast<const uint16_t*>(a.basis_k) + static_cast<size_t>(j) * RB * D;
        const uint16_t* Rk = reinterpret_cast<const uint16_t*>(a.r_k) + static_cast<size_t>(j) * RM * D;
        for (int idx = threadIdx.x; idx < 16 * C::PD; idx += blockDim.x) {
            const int h = idx / C::PD;
            const int i = idx % C::PD;
            float acc = 0.f;
            if (h < g) {
                const uint16_t* row = i < RB ? Bk + static_cast<size_t>(i) * D : Rk + static_cast<size_t>(i - RB) * D;
                for (int e = 0; e < D; e += 2) {
                    const uint32_t bw = *reinterpret_cast<const uint32_t*>(row + e);
                    const uint32_t qw = *reinterpret_cast<const uint32_t*>(qb + h * D + e);
                    acc += bf16_lo(bw) * bf16_lo(qw);
                    acc += bf16_hi(bw) * bf16_hi(qw);
                }
            }
            qproj[idx] = acc;
        }
    }
    __syncthreads();
    if (a.stall && threadIdx.x == 0) mbar_wait_bounded(&bars[NW * NSW], 0, a.stall_limit, a.err);

    // A fragments: rows = heads; q~ (RB wide) and q^ (16 wide), each as bf16 hi + lo
    uint32_t qc_hi[RB / 16][4], qc_lo[RB / 16][4], qu_hi[4], qu_lo[4];
    {
        const int h0 = lane >> 2;
        const int cq = 2 * (lane & 3);
        auto frag = [&](int col0, uint32_t (&hi)[4], uint32_t (&lo)[4]) {
            const int cols[4] = {col0 + cq, col0 + cq, col0 + 8 + cq, col0 + 8 + cq};
            const int rows[4] = {h0, h0 + 8, h0, h0 + 8};
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const float x0 = qproj[rows[r] * C::PD + cols[r]];
                const float x1 = qproj[rows[r] * C::PD + cols[r] + 1];
                hi[r] = pack_bf16(x0, x1);
                lo[r] = pack_bf16(x0 - bf16_lo(hi[r]), x1 - bf16_hi(hi[r]));
            }
        };
#pragma unroll
        for (int kk = 0; kk < RB / 16; ++kk) frag(kk * 16, qc_hi[kk], qc_lo[kk]);
        frag(RB, qu_hi, qu_lo);
    }

    float cacc[RB / 8][4];
    float uacc[2][4];
#pragma unroll
    for (int i = 0; i < RB / 8; ++i) cacc[i][0] = cacc[i][1] = cacc[i][2] = cacc[i][3] = 0.f;
#pragma unroll
    for (int i = 0; i < 2; ++i) uacc[i][0] = uacc[i][1] = uacc[i][2] = uacc[i][3] = 0.f;
    float m0 = NEG_INF, m1 = NEG_INF, l0 = 0.f, l1 = 0.f;

    uint8_t* ring = smem + warp * NSW * C::STAGE_BYTES;
    uint64_t* wb = &bars[warp * NSW];
    float* tks = tok + warp * TT * 3;     // [3][TT]: s_K, s_V, rank
    const int span = tile1 - tile0;
    const int my_n = span > warp ? (span - warp + NW - 1) / NW : 0;

    auto issue = [&](int k) {
        const int t = tile0 + warp + k * NW;
        const int s = k % NSW;
        uint8_t* st = ring + s * C::STAGE_BYTES;
        mbar_arrive_expect_tx(&wb[s], C::STAGE_BYTES);
#pragma unroll
        for (int h = 0; h < LY::HALVES; ++h) {
            tma_load_3d(st + h * TT * 128, &tmCK, h * 64, t * TT, crow, &wb[s]);
            tma_load_3d(st + C::COEF_BYTES + h * TT * 128, &tmCV, h * 64, t * TT, crow, &wb[s]);
        }
        tma_load_3d(st + 2 * C::COEF_BYTES, &tmUK, 0, t * TT, urow, &wb[s]);
        tma_load_3d(st + 2 * C::COEF_BYTES + C::U_BYTES, &tmUV, 0, t * TT, urow, &wb[s]);
    };
    // per-token scales and ranks of a tile, loaded by the lanes (tokens lane, lane+32, ...)
    constexpr int TPL = TT / 32;
    float pf_sk[TPL], pf_sv[TPL], pf_r[TPL];
    auto prefetch = [&](int k) {
        const int t0 = (tile0 + warp + k * NW) * TT;
#pragma unroll
        for (int u = 0; u < TPL; ++u) {
            const int t = t0 + lane + 32 * u;
            if (t < a.T) {
                pf_sk[u] = __half2float(__ushort_as_half(__ldg(a.s_k + tokrow + t)));
                pf_sv[u] = __half2float(__ushort_as_half(__ldg(a.s_v + tokrow + t)));
                pf_r[u] = static_cast<float>(__ldg(rank_row + t));
            } else {
                pf_sk[u] = 0.f; pf_sv[u] = 0.f; pf_r[u] = 0.f;
            }
        }
    };
    if (lane == 0) {
        for (int k = 0; k < min(NSW, my_n); ++k) issue(k);
    }
    if (my_n > 0) prefetch(0);
    __syncwarp();

    for (int k = 0; k < my_n; ++k) {
        const int s = k % NSW;
        // publish this tile's per-token values, start fetching the next tile's
        __syncwarp();
#pragma unroll
        for (int u = 0; u < TPL; ++u) {
            tks[lane + 32 * u] = pf_sk[u];
            tks[TT + lane + 32 * u] = pf_sv[u];
            tks[2 * TT + lane + 32 * u] = pf_r[u];
        }
        if (k + 1 < my_n) prefetch(k + 1);
        __syncwarp();
        const bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(&wb[s], (k / NSW) & 1, a.wait_limit, a.err));
        if (!ok) {
            const int issued = min(my_n, k + NSW);
            for (int kk = k + 1; kk < issued; ++kk) mbar_wait_bounded(&wb[kk % NSW], (kk / NSW) & 1, a.wait_limit, a.err);
            break;
        }
        const int t = tile0 + warp + k * NW;
        const uint32_t ckb = smem_u32(ring + s * C::STAGE_BYTES);
        const uint32_t cvb = ckb + C::COEF_BYTES;
        const uint8_t* ukp = ring + s * C::STAGE_BYTES + 2 * C::COEF_BYTES;
        const uint8_t* uvp = ukp + C::U_BYTES;

        float sc[TT / 8][4];
        float su[TT / 8][4];
#pragma unroll
        for (int nb = 0; nb < TT / 8; ++nb) {
            sc[nb][0] = sc[nb][1] = sc[nb][2] = sc[nb][3] = 0.f;
            su[nb][0] = su[nb][1] = su[nb][2] = su[nb][3] = 0.f;
        }
        // ---- basis part of the scores: C_K q~ (hi and lo)
#pragma unroll
        for (int kk2 = 0; kk2 < RB / 32; ++kk2) {
            const int c = kk2 * 4 + (lane >> 3);
#pragma unroll
            for (int nb = 0; nb < TT / 8; ++nb) {
                const int row = nb * 8 + (lane & 7);
                uint32_t r0, r1, r2, r3;
                ldsm_x4(ckb + LY::template off<TT>(row, c), r0, r1, r2, r3);
                mma_bf16(sc[nb], qc_hi[2 * kk2], r0, r1);
                mma_bf16(sc[nb], qc_lo[2 * kk2], r0, r1);
                mma_bf16(sc[nb], qc_hi[2 * kk2 + 1], r2, r3);
                mma_bf16(sc[nb], qc_lo[2 * kk2 + 1], r2, r3);
            }
        }
        // ---- residual part: U_K (masked to the token's rank) q^
#pragma unroll
        for (int nb = 0; nb < TT / 8; ++nb) {
            const int tt = nb * 8 + (lane >> 2);
            const int r = static_cast<int>(tks[2 * TT + tt]);
            const int i0 = 2 * (lane & 3);
            const int8_t* up = reinterpret_cast<const int8_t*>(ukp + tt * RM);
            const uint32_t b0 = pack_i8_bf16(i0 < r ? up[i0] : 0, i0 + 1 < r ? up[i0 + 1] : 0);
            const uint32_t b1 = pack_i8_bf16(i0 + 8 < r ? up[i0 + 8] : 0, i0 + 9 < r ? up[i0 + 9] : 0);
            mma_bf16(su[nb], qu_hi, b0, b1);
            mma_bf16(su[nb], qu_lo, b0, b1);
        }
        // ---- scores, mask, online softmax
        const int tb = 2 * (lane & 3);
        float mx0 = NEG_INF, mx1 = NEG_INF;
#pragma unroll
        for (int nb = 0; nb < TT / 8; ++nb) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int tt = nb * 8 + tb + (i & 1);
                float v = (sc[nb][i] + tks[tt] * su[nb][i]) * a.scale_log2;
                if (t * TT + tt >= a.T) v = NEG_INF;
                sc[nb][i] = v;
                if (i < 2) mx0 = fmaxf(mx0, v); else mx1 = fmaxf(mx1, v);
            }
        }
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
        const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
        const float ref0 = mn0 == NEG_INF ? 0.f : mn0;
        const float ref1 = mn1 == NEG_INF ? 0.f : mn1;
        const float cr0 = exp2f(m0 - ref0), cr1 = exp2f(m1 - ref1);
        m0 = mn0;
        m1 = mn1;
        l0 *= cr0;
        l1 *= cr1;
#pragma unroll
        for (int i = 0; i < RB / 8; ++i) { cacc[i][0] *= cr0; cacc[i][1] *= cr0; cacc[i][2] *= cr1; cacc[i][3] *= cr1; }
#pragma unroll
        for (int i = 0; i < 2; ++i) { uacc[i][0] *= cr0; uacc[i][1] *= cr0; uacc[i][2] *= cr1; uacc[i][3] *= cr1; }

#pragma unroll
        for (int kk = 0; kk < TT / 16; ++kk) {
            float p[2][4];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                p[u][0] = exp2f(sc[2 * kk + u][0] - ref0);
                p[u][1] = exp2f(sc[2 * kk + u][1] - ref0);
                p[u][2] = exp2f(sc[2 * kk + u][2] - ref1);
                p[u][3] = exp2f(sc[2 * kk + u][3] - ref1);
            }
            uint32_t pa[4], pv[4];
            pa[0] = pack_bf16(p[0][0], p[0][1]);
            pa[1] = pack_bf16(p[0][2], p[0][3]);
            pa[2] = pack_bf16(p[1][0], p[1][1]);
            pa[3] = pack_bf16(p[1][2], p[1][3]);
            l0 += (bf16_lo(pa[0]) + bf16_hi(pa[0])) + (bf16_lo(pa[2]) + bf16_hi(pa[2]));
            l1 += (bf16_lo(pa[1]) + bf16_hi(pa[1])) + (bf16_lo(pa[3]) + bf16_hi(pa[3]));
            // p * s_V for the residual accumulation
            const int ta = kk * 16 + tb;                 // tokens ta, ta+1 and ta+8, ta+9
            const float sv0 = tks[TT + ta], sv1 = tks[TT + ta + 1];
            const float sv8 = tks[TT + ta + 8], sv9 = tks[TT + ta + 9];
            pv[0] = pack_bf16(p[0][0] * sv0, p[0][1] * sv1);
            pv[1] = pack_bf16(p[0][2] * sv0, p[0][3] * sv1);
            pv[2] = pack_bf16(p[1][0] * sv8, p[1][1] * sv9);
            pv[3] = pack_bf16(p[1][2] * sv8, p[1][3] * sv9);
            // c^ += P C_V
            const int mtx = lane >> 3;
            const int row = (2 * kk + (mtx & 1)) * 8 + (lane & 7);
#pragma unroll
            for (int cb2 = 0; cb2 < RB / 16; ++cb2) {
                const int c = 2 * cb2 + (mtx >> 1);
                uint32_t r0, r1, r2, r3;
                ldsm_x4_t(cvb + LY::template off<TT>(row, c), r0, r1, r2, r3);
                mma_bf16(cacc[2 * cb2], pa, r0, r1);
                mma_bf16(cacc[2 * cb2 + 1], pa, r2, r3);
            }
            // u^ += (P s_V) U_V, codes masked to each token's rank
            const int r0t = static_cast<int>(tks[2 * TT + ta]), r1t = static_cast<int>(tks[2 * TT + ta + 1]);
            const int r8t = static_cast<int>(tks[2 * TT + ta + 8]), r9t = static_cast<int>(tks[2 * TT + ta + 9]);
            const int8_t* uv = reinterpret_cast<const int8_t*>(uvp);
#pragma unroll
            for (int nbi = 0; nbi < 2; ++nbi) {
                const int i = nbi * 8 + (lane >> 2);
                const uint32_t b0 = pack_i8_bf16(i < r0t ? uv[ta * RM + i] : 0, i < r1t ? uv[(ta + 1) * RM + i] : 0);
                const uint32_t b1 = pack_i8_bf16(i < r8t ? uv[(ta + 8) * RM + i] : 0, i < r9t ? uv[(ta + 9) * RM + i] : 0);
                mma_bf16(uacc[nbi], pv, b0, b1);
            }
        }
        __syncwarp();
        if (lane == 0 && k + NSW < my_n) {
            fence_proxy_async();
            issue(k + NSW);
        }
    }
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);

    // ---- merge warps in coefficient space, project once, finish the split
    __syncthreads();
    constexpr int PD = C::PD;
    float* comb = reinterpret_cast<float*>(smem);   // [NW][16][PD]
    float* comb_m = comb + NW * 16 * PD;
    float* comb_l = comb_m + NW * 16;
    float* fin_m = comb_l + NW * 16;
    float* fin_l = fin_m + 16;
    float* fin_c = fin_l + 16;                      // [16][PD]
    float* fin_o = fin_c + 16 * PD;                 // [16][D]
    float* scratch = fin_o + 16 * D;
    {
        const int h0 = lane >> 2;
        const int e0 = 2 * (lane & 3);
#pragma unroll
        for (int cb = 0; cb < RB / 8; ++cb) {
            float* p0 = comb + (warp * 16 + h0) * PD + cb * 8 + e0;
            float* p1 = comb + (warp * 16 + h0 + 8) * PD + cb * 8 + e0;
            p0[0] = cacc[cb][0]; p0[1] = cacc[cb][1];
            p1[0] = cacc[cb][2]; p1[1] = cacc[cb][3];
        }
#pragma unroll
        for (int ub = 0; ub < 2; ++ub) {
            float* p0 = comb + (warp * 16 + h0) * PD + RB + ub * 8 + e0;
            float* p1 = comb + (warp * 16 + h0 + 8) * PD + RB + ub * 8 + e0;
            p0[0] = uacc[ub][0]; p0[1] = uacc[ub][1];
            p1[0] = uacc[ub][2]; p1[1] = uacc[ub][3];
        }
        if ((lane & 3) == 0) {
            comb_m[warp * 16 + h0] = m0;
            comb_m[warp * 16 + h0 + 8] = m1;
            comb_l[warp * 16 + h0] = l0;
            comb_l[warp * 16 + h0 + 8] = l1;
        }
    }
    __syncthreads();
    if (threadIdx.x < g) {
        const int h = threadIdx.x;
        float M = NEG_INF;
        for (int ww = 0; ww < NW; ++ww) M = fmaxf(M, comb_m[ww * 16 + h]);
        float L = 0.f;
        for (int ww = 0; ww < NW; ++ww) L += exp2f(comb_m[ww * 16 + h] - M) * comb_l[ww * 16 + h];
        fin_m[h] = M;
        fin_l[h] = L;
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < g * PD; idx += blockDim.x) {
        const int h = idx / PD;
        float acc = 0.f;
#pragma unroll
        for (int ww = 0; ww < NW; ++ww) acc += exp2f(comb_m[ww * 16 + h] - fin_m[h]) * comb[(ww * 16 + h) * PD + (idx % PD)];
        fin_c[idx] = acc;
    }
    __syncthreads();
    {
        const uint16_t* Bv = reinterpret_cast<const uint16_t*>(a.basis_v) + static_cast<size_t>(j) * RB * D;
        const uint16_t* Rv = reinterpret_cast<const uint16_t*>(a.r_v) + static_cast<size_t>(j) * RM * D;
        for (int idx = threadIdx.x; idx < g * D; idx += blockDim.x) {
            const int h = idx / D;
            const int e = idx % D;
            float acc = 0.f;
            for (int i = 0; i < RB; ++i) acc += fin_c[h * PD + i] * bf16_lo(Bv[static_cast<size_t>(i) * D + e]);
            for (int i = 0; i < RM; ++i) acc += fin_c[h * PD + RB + i] * bf16_lo(Rv[static_cast<size_t>(i) * D + e]);
            fin_o[idx] = acc;
        }
    }
    __syncthreads();
    finish_split(a, D, b, j, split, fin_m, fin_l, fin_o, scratch);
}

template <int D, int RB, int TT, int NSW>
cudaError_t launch_one(const DecodeArgs& a, const CUtensorMap* maps, cudaStream_t st) {
    using C = LrCfg<D, RB, TT, NSW>;
    auto kern = decode_lowrank_kernel<D, RB, TT, NSW>;
    static bool attr_done = false;
    if (!attr_done) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
        if (e != cudaSuccess) return e;
        attr_done = true;
    }
    dim3 grid(a.splits, a.Hkv, a.B);
    kern<<<grid, NW * 32, C::SMEM, st>>>(maps[0], maps[1], maps[2], maps[3], a);
    return cudaGetLastError();
}

template <int D, int RB, int TT, int NSW>
int occupancy_of() {
    using C = LrCfg<D, RB, TT, NSW>;
    auto kern = decode_lowrank_kernel<D, RB, TT, NSW>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, NW * 32, C::SMEM) != cudaSuccess) return 1;
    return n > 0 ? n : 1;
}

// token tile and stages per warp by basis rank (the full-rank basis only serves tests)
template <int RB>
struct LrShape {
    static constexpr int TT = RB == 128 ? 32 : 64;
    static constexpr int NSW = RB == 128 ? 1 : 2;
};

template <int D, int RB>
int occ() { return occupancy_of<D, RB, LrShape<RB>::TT, LrShape<RB>::NSW>(); }

template <int D, int RB>
cudaError_t run(const DecodeArgs& a, const CUtensorMap* maps, cudaStream_t st) {
    return launch_one<D, RB, LrShape<RB>::TT, LrShape<RB>::NSW>(a, maps, st);
}

}  // namespace

int decode_lowrank_tile(int rb) { return rb == 128 ? LrShape<128>::TT : LrShape<32>::TT; }

int decode_lowrank_occupancy(int d, int rb) {
    if (d == 64) return rb == 32 ? occ<64, 32>() : occ<64, 64>();
    return rb == 32 ? occ<128, 32>() : occ<128, 128>();
}

cudaError_t launch_decode_lowrank(int d, int rb, const DecodeArgs& a, const CUtensorMap* maps, cudaStream_t st) {
    if (d == 64) return rb == 32 ? run<64, 32>(a, maps, st) : run<64, 64>(a, maps, st);
    return rb == 32 ? run<128, 32>(a, maps, st) : run<128, 128>(a, maps, st);
}

}  // namespace kvs

// Split-KV GQA decode over a shared cache, bf16 storage, forms SINGLE and MIX.
//
// One CTA = one (split, kv head j, batch b). Four warps; each warp owns a
// private ring of NSW shared-memory stages and streams every 4th token tile of
// the split into it with TMA (128-byte swizzle), re-issuing a stage as soon as
// it has consumed it. Per tile and warp:
//   S   = Q K^T            mma.sync m16n8k16 bf16 -> fp32, the g query heads of
//                          kv head j are the M rows (padded to 16)
//   MIX S = w S1 + (1-w) S2, the two sources' scores mixed in fp32, which equals
//                          the scores against w K1 + (1-w) K2 (the convex mix of
//                          the DepthGraft source pair) up to fp32 rounding
//   online softmax in base 2 (quad shuffles for the row max)
//   O  += P V              P rounded to bf16 as the A operand; for MIX,
//                          O += bf16(w P) V1 + bf16((1-w) P) V2
// The mixed K/V never exist anywhere, in HBM or in shared memory.
// The four warps' (m, l, O) are merged in shared memory, then finish_split
// writes the output or the split partial (the last CTA merges the splits).
#include "kvs_device.cuh"

namespace kvs {
namespace {

constexpr int NW = 4;

template <int D, bool MIX, int TT, int NSW>
struct DecodeCfg {
    static constexpr int HALVES = D / 64;
    static constexpr int HALF_BYTES = TT * 128;              // [TT][64] bf16
    static constexpr int TILE_BYTES = TT * D * 2;
    static constexpr int NSRC = MIX ? 2 : 1;
    static constexpr int STAGE_BYTES = 2 * NSRC * TILE_BYTES;
    static constexpr int RING_BYTES = NW * NSW * STAGE_BYTES;
    static constexpr int COMBINE_FLOATS = NW * 16 * D + 2 * NW * 16 + 32 + 16 * D + MAX_GROUP * MAX_SPLITS + 64;
    static constexpr int BODY = RING_BYTES > COMBINE_FLOATS * 4 ? RING_BYTES : COMBINE_FLOATS * 4;
    static constexpr int SMEM = BODY + 1024;                  // slack to align the ring to 1024 B
    static_assert(TT % 16 == 0, "token tile must hold whole k16 steps");
    static_assert(HALF_BYTES % 1024 == 0, "swizzled halves must stay 1024-B aligned");
};

template <int D, bool MIX, int TT, int NSW>
__global__ void __launch_bounds__(NW * 32)
decode_bf16_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                   const DecodeArgs a) {
    using C = DecodeCfg<D, MIX, TT, NSW>;
    extern __shared__ uint8_t smem_dyn[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
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
    const int BH = a.B * a.Hkv;
    const int row0 = a.src0 * BH + b * a.Hkv + j;
    const int row1 = MIX ? a.src1 * BH + b * a.Hkv + j : 0;

    if (threadIdx.x == 0) {
        for (int i = 0; i < NW * NSW + 1; ++i) mbar_init(&bars[i], 1);
        mbar_init_fence();
    }
    __syncthreads();

    if (a.stall && threadIdx.x == 0) {
        // test hook: nothing ever arrives on the spare barrier; the bounded wait gives up
        mbar_wait_bounded(&bars[NW * NSW], 0, a.stall_limit, a.err);
    }

    // A fragments of Q (rows = the g query heads, zero rows beyond g)
    uint32_t qa[D / 16][4];
    {
        const uint16_t* qb = reinterpret_cast<const uint16_t*>(a.q) +
                             (static_cast<size_t>(b) * a.Hq + static_cast<size_t>(j) * g) * D;
        const int h0 = lane >> 2;
        const int h1 = h0 + 8;
        const int cq = 2 * (lane & 3);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
            qa[kk][0] = h0 < g ? *reinterpret_cast<const uint32_t*>(qb + h0 * D + kk * 16 + cq) : 0u;
            qa[kk][1] = h1 < g ? *reinterpret_cast<const uint32_t*>(qb + h1 * D + kk * 16 + cq) : 0u;
            qa[kk][2] = h0 < g ? *reinterpret_cast<const uint32_t*>(qb + h0 * D + kk * 16 + 8 + cq) : 0u;
            qa[kk][3] = h1 < g ? *reinterpret_cast<const uint32_t*>(qb + h1 * D + kk * 16 + 8 + cq) : 0u;
        }
    }
    const float w = MIX ? a.w[j] : 1.f;
    const float w1 = 1.f - w;

    float o[D / 8][4];
#pragma unroll
    for (int i = 0; i < D / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    float m0 = NEG_INF, m1 = NEG_INF, l0 = 0.f, l1 = 0.f;

    uint8_t* ring = smem + warp * NSW * C::STAGE_BYTES;
    uint64_t* wb = &bars[warp * NSW];
    const int span = tile1 - tile0;
    const int my_n = span > warp ? (span - warp + NW - 1) / NW : 0;

    auto issue = [&](int k) {
        const int t = tile0 + warp + k * NW;
        const int s = k % NSW;
        uint8_t* st = ring + s * C::STAGE_BYTES;
        mbar_arrive_expect_tx(&wb[s], C::STAGE_BYTES);
#pragma unroll
        for (int h = 0; h < C::HALVES; ++h) {
            tma_load_3d(st + h * C::HALF_BYTES, &tmK, h * 64, t * TT, row0, &wb[s]);
            tma_load_3d(st + C::TILE_BYTES + h * C::HALF_BYTES, &tmV, h * 64, t * TT, row0, &wb[s]);
            if (MIX) {
                tma_load_3d(st + 2 * C::TILE_BYTES + h * C::HALF_BYTES, &tmK, h * 64, t * TT, row1, &wb[s]);
                tma_load_3d(st + 3 * C::TILE_BYTES + h * C::HALF_BYTES, &tmV, h * 64, t * TT, row1, &wb[s]);
            }
        }
    };
    if (lane == 0) {
        for (int k = 0; k < min(NSW, my_n); ++k) issue(k);
    }
    __syncwarp();

    for (int k = 0; k < my_n; ++k) {
        const int s = k % NSW;
        const bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(&wb[s], (k / NSW) & 1, a.wait_limit, a.err));
        if (!ok) {
            // give the copies still in flight a bounded chance to land, then stop
            const int issued = min(my_n, k + NSW);
            for (int kk = k + 1; kk < issued; ++kk) mbar_wait_bounded(&wb[kk % NSW], (kk / NSW) & 1, a.wait_limit, a.err);
            break;
        }
        const int t = tile0 + warp + k * NW;
        const uint32_t kb = smem_u32(ring + s * C::STAGE_BYTES);
        const uint32_t vb = kb + C::TILE_BYTES;

        float sc[TT / 8][4];
        float sc2[MIX ? TT / 8 : 1][4];
#pragma unroll
        for (int nb = 0; nb < TT / 8; ++nb) {
            sc[nb][0] = sc[nb][1] = sc[nb][2] = sc[nb][3] = 0.f;
            if (MIX) sc2[nb][0] = sc2[nb][1] = sc2[nb][2] = sc2[nb][3] = 0.f;
        }
        // ---- S = Q K^T
#pragma unroll
        for (int kk2 = 0; kk2 < D / 32; ++kk2) {
            const int c = kk2 * 4 + (lane >> 3);
#pragma unroll
            for (int nb = 0; nb < TT / 8; ++nb) {
                const int row = nb * 8 + (lane & 7);
                const uint32_t off = (c >> 3) * C::HALF_BYTES + swz128(row, c & 7);
                uint32_t r0, r1, r2, r3;
                ldsm_x4(kb + off, r0, r1, r2, r3);
                mma_bf16(sc[nb], qa[2 * kk2], r0, r1);
                mma_bf16(sc[nb], qa[2 * kk2 + 1], r2, r3);
                if (MIX) {
                    ldsm_x4(kb + 2 * C::TILE_BYTES + off, r0, r1, r2, r3);
                    mma_bf16(sc2[nb], qa[2 * kk2], r0, r1);
                    mma_bf16(sc2[nb], qa[2 * kk2 + 1], r2, r3);
                }
            }
        }
        // ---- scale, mask the ragged tail, online softmax
        const int tb = t * TT + 2 * (lane & 3);
        float mx0 = NEG_INF, mx1 = NEG_INF;
#pragma unroll
        for (int nb = 0; nb < TT / 8; ++nb) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                float v = MIX ? (w * sc[nb][i] + w1 * sc2[nb][i]) : sc[nb][i];
                v *= a.scale_log2;
                if (tb + nb * 8 + (i & 1) >= a.T) v = NEG_INF;
                sc[nb][i] = v;
                if (i < 2) mx0 = fmaxf(mx0, v); else mx1 = fmaxf(mx1, v);
            }
        }
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
        const float mn0 = fmaxf(m0, mx0);
        const float mn1 = fmaxf(m1, mx1);
        const float ref0 = mn0 == NEG_INF ? 0.f : mn0;
        const float ref1 = mn1 == NEG_INF ? 0.f : mn1;
        const float cr0 = exp2f(m0 - ref0);
        const float cr1 = exp2f(m1 - ref1);
        m0 = mn0;
        m1 = mn1;
        l0 *= cr0;
        l1 *= cr1;
#pragma unroll
        for (int db = 0; db < D / 8; ++db) {
            o[db][0] *= cr0; o[db][1] *= cr0;
            o[db][2] *= cr1; o[db][3] *= cr1;
        }
        uint32_t pa[TT / 16][4];
        uint32_t pb[MIX ? TT / 16 : 1][4];
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
            if (!MIX) {
                pa[kk][0] = pack_bf16(p[0][0], p[0][1]);
                pa[kk][1] = pack_bf16(p[0][2], p[0][3]);
                pa[kk][2] = pack_bf16(p[1][0], p[1][1]);
                pa[kk][3] = pack_bf16(p[1][2], p[1][3]);
                l0 += (bf16_lo(pa[kk][0]) + bf16_hi(pa[kk][0])) + (bf16_lo(pa[kk][2]) + bf16_hi(pa[kk][2]));
                l1 += (bf16_lo(pa[kk][1]) + bf16_hi(pa[kk][1])) + (bf16_lo(pa[kk][3]) + bf16_hi(pa[kk][3]));
            } else {
                pa[kk][0] = pack_bf16(w * p[0][0], w * p[0][1]);
                pa[kk][1] = pack_bf16(w * p[0][2], w * p[0][3]);
                pa[kk][2] = pack_bf16(w * p[1][0], w * p[1][1]);
                pa[kk][3] = pack_bf16(w * p[1][2], w * p[1][3]);
                pb[kk][0] = pack_bf16(w1 * p[0][0], w1 * p[0][1]);
                pb[kk][1] = pack_bf16(w1 * p[0][2], w1 * p[0][3]);
                pb[kk][2] = pack_bf16(w1 * p[1][0], w1 * p[1][1]);
                pb[kk][3] = pack_bf16(w1 * p[1][2], w1 * p[1][3]);
                l0 += (bf16_lo(pa[kk][0]) + bf16_hi(pa[kk][0])) + (bf16_lo(pa[kk][2]) + bf16_hi(pa[kk][2])) +
                      (bf16_lo(pb[kk][0]) + bf16_hi(pb[kk][0])) + (bf16_lo(pb[kk][2]) + bf16_hi(pb[kk][2]));
                l1 += (bf16_lo(pa[kk][1]) + bf16_hi(pa[kk][1])) + (bf16_lo(pa[kk][3]) + bf16_hi(pa[kk][3])) +
                      (bf16_lo(pb[kk][1]) + bf16_hi(pb[kk][1])) + (bf16_lo(pb[kk][3]) + bf16_hi(pb[kk][3]));
            }
        }
        // ---- O += P V
#pragma unroll
        for (int kk = 0; kk < TT / 16; ++kk) {
            const int mtx = lane >> 3;
            const int row = (2 * kk + (mtx & 1)) * 8 + (lane & 7);
#pragma unroll
            for (int db2 = 0; db2 < D / 16; ++db2) {
                const int c = 2 * db2 + (mtx >> 1);
                const uint32_t off = (c >> 3) * C::HALF_BYTES + swz128(row, c & 7);
                uint32_t r0, r1, r2, r3;
                ldsm_x4_t(vb + off, r0, r1, r2, r3);
                mma_bf16(o[2 * db2], pa[kk], r0, r1);
                mma_bf16(o[2 * db2 + 1], pa[kk], r2, r3);
                if (MIX) {
                    ldsm_x4_t(vb + 2 * C::TILE_BYTES + off, r0, r1, r2, r3);
                    mma_bf16(o[2 * db2], pb[kk], r0, r1);
                    mma_bf16(o[2 * db2 + 1], pb[kk], r2, r3);
                }
            }
        }
        __syncwarp();
        if (lane == 0 && k + NSW < my_n) {
            fence_proxy_async();
            issue(k + NSW);
        }
        __syncwarp();
    }
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);

    // ---- merge the four warps (reusing the ring; every copy issued has been consumed)
    __syncthreads();
    float* comb_o = reinterpret_cast<float*>(smem);   // [NW][16][D]
    float* comb_m = comb_o + NW * 16 * D;             // [NW][16]
    float* comb_l = comb_m + NW * 16;                 // [NW][16]
    float* fin_m = comb_l + NW * 16;                  // [16]
    float* fin_l = fin_m + 16;                        // [16]
    float* fin_o = fin_l + 16;                        // [16][D]
    float* scratch = fin_o + 16 * D;                  // merge scratch
    {
        const int h0 = lane >> 2;
        const int e0 = 2 * (lane & 3);
#pragma unroll
        for (int db = 0; db < D / 8; ++db) {
            float* r0p = comb_o + (warp * 16 + h0) * D + db * 8 + e0;
            float* r1p = comb_o + (warp * 16 + h0 + 8) * D + db * 8 + e0;
            r0p[0] = o[db][0]; r0p[1] = o[db][1];
            r1p[0] = o[db][2]; r1p[1] = o[db][3];
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
    for (int idx = threadIdx.x; idx < g * D; idx += blockDim.x) {
        const int h = idx / D;
        const int e = idx % D;
        float acc = 0.f;
#pragma unroll
        for (int ww = 0; ww < NW; ++ww) acc += exp2f(comb_m[ww * 16 + h] - fin_m[h]) * comb_o[(ww * 16 + h) * D + e];
        fin_o[idx] = acc;
    }
    __syncthreads();
    finish_split(a, D, b, j, split, fin_m, fin_l, fin_o, scratch);
}

template <int D, bool MIX, int TT, int NSW>
cudaError_t launch_one(const CUtensorMap& tmK, const CUtensorMap& tmV, const DecodeArgs& a, cudaStream_t st) {
    using C = DecodeCfg<D, MIX, TT, NSW>;
    auto kern = decode_bf16_kernel<D, MIX, TT, NSW>;
    static bool attr_done = false;
    if (!attr_done) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
        if (e != cudaSuccess) return e;
        attr_done = true;
    }
    dim3 grid(a.splits, a.Hkv, a.B);
    kern<<<grid, NW * 32, C::SMEM, st>>>(tmK, tmV, a);
    return cudaGetLastError();
}

template <int D, bool MIX, int TT, int NSW>
int occupancy() {
    using C = DecodeCfg<D, MIX, TT, NSW>;
    auto kern = decode_bf16_kernel<D, MIX, TT, NSW>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, NW * 32, C::SMEM) != cudaSuccess) return 1;
    return n > 0 ? n : 1;
}

template <int D, bool MIX, int TT, int NSW>
TileShape shape_of() {
    return {TT, NSW, DecodeCfg<D, MIX, TT, NSW>::SMEM};
}

// tile shapes: tokens per tile, stages per warp
#define KVS_SHAPE_64_SINGLE 32, 3
#define KVS_SHAPE_64_MIX 16, 3
#define KVS_SHAPE_128_SINGLE 16, 3
#define KVS_SHAPE_128_MIX 16, 2

}  // namespace

TileShape decode_bf16_shape(int d, bool mix) {
    if (d == 64 && !mix) return shape_of<64, false, KVS_SHAPE_64_SINGLE>();
    if (d == 64 && mix) return shape_of<64, true, KVS_SHAPE_64_MIX>();
    if (d == 128 && !mix) return shape_of<128, false, KVS_SHAPE_128_SINGLE>();
    return shape_of<128, true, KVS_SHAPE_128_MIX>();
}

int decode_bf16_ctas_per_sm(int d, bool mix) {
    if (d == 64 && !mix) return occupancy<64, false, KVS_SHAPE_64_SINGLE>();
    if (d == 64 && mix) return occupancy<64, true, KVS_SHAPE_64_MIX>();
    if (d == 128 && !mix) return occupancy<128, false, KVS_SHAPE_128_SINGLE>();
    return occupancy<128, true, KVS_SHAPE_128_MIX>();
}

cudaError_t launch_decode_bf16(int d, bool mix, const CUtensorMap& tmK, const CUtensorMap& tmV,
                               const DecodeArgs& a, cudaStream_t st) {
    if (d == 64 && !mix) return launch_one<64, false, KVS_SHAPE_64_SINGLE>(tmK, tmV, a, st);
    if (d == 64 && mix) return launch_one<64, true, KVS_SHAPE_64_MIX>(tmK, tmV, a, st);
    if (d == 128 && !mix) return launch_one<128, false, KVS_SHAPE_128_SINGLE>(tmK, tmV, a, st);
    return launch_one<128, true, KVS_SHAPE_128_MIX>(tmK, tmV, a, st);
}

}  // namespace kvs

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
//   - TMA streams coefficient tiles (64/128-B swizzle) per warp, and bulk copies
//     bring each 32-token group's used code bytes (group-packed codes);
//   - q~ = B_K q and q^ = R_K q are split into bf16 hi + lo halves so the score
//     MMAs (mma.sync m16n8k16) keep ~16 bits of the fp32 projection;
//   - tokens are the MMA's M rows and the g heads its N columns (S^T = C q~^T),
//     so a group of up to 8 heads wastes nothing on padding; P^T reaches the
//     PV MMAs through an in-register transpose (movmatrix);
//   - int8 codes convert exactly to f16 operands, masked by the token's rank;
//   - c^ and u^ accumulate in fp32 MMA accumulators; split partials stay in this
//     coefficient space and the CTA that merges a unit projects it once;
//   - when the entropy is asked for, the online softmax also carries
//     z = sum 2^(s - m) (m - s) through the warp and split merges (a separate
//     compiled instance), so entropy and peak need no pass over the scores.
#include "kvs_quant.cuh"

namespace kvs {
namespace {

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

template <int D, int RB, int TT, int NSW, int NW>
struct LrCfg {
    using L = CoefLayout<RB>;
    static constexpr int COEF_BYTES = TT * RB * 2;
    static constexpr int U_BYTES = TT * RM;
    // every TMA destination in shared memory starts on a 128-byte boundary
    static constexpr int ALIGN128(int x) { return (x + 127) / 128 * 128; }
    static constexpr int OFF_UK = 2 * COEF_BYTES;
    static constexpr int OFF_UV = OFF_UK + ALIGN128(U_BYTES);
    // keeps swizzled tiles aligned (the word-wise code reads may run up to 20 bytes past a
    // stage's V codes: into the next stage, or the buffers that follow the ring)
    static constexpr int STAGE_BYTES = ((OFF_UV + U_BYTES + 1023) / 1024) * 1024;
    static_assert(COEF_BYTES % 128 == 0 && OFF_UK % 128 == 0 && OFF_UV % 128 == 0,
                  "TMA destinations must be 128-byte aligned");
    static constexpr int RING_BYTES = NW * NSW * STAGE_BYTES;
    // per-warp scratch of per-token s_K, s_V (fp32) and rank (int)
    static constexpr int TOK_BYTES = NW * TT * 3 * 4;
    // per-warp f16 copies of the tile's K and V codes, masked to each token's rank:
    // [K | V][TT][16] halves, rows of 32 B whose two 16-B halves swap on every 4th row
    static constexpr int CVT_BYTES = NW * 2 * TT * 32;
    static constexpr int PD = RB + RM;    // coefficient-space partial width
    static constexpr int COMBINE_FLOATS = NW * 16 * PD + 4 * NW * 16 + 64 + 16 * PD + 16 * D + 4 * MAX_GROUP * MAX_SPLITS + 64;
    static constexpr int QPROJ_FLOATS = 16 * PD;
    // staging: B_K [RB][D] + R_K [RM][D] (bf16), the query rows [<=16][D], then B_V + R_V
    static constexpr int STAGE_FACTORS = (RB + RM) * D * 2;
    static constexpr int OFF_VFAC = STAGE_FACTORS + 16 * D * 2;
    static constexpr int STAGE_BYTES_TOTAL = OFF_VFAC + STAGE_FACTORS;
    static constexpr int BODY0 = RING_BYTES > COMBINE_FLOATS * 4 ? RING_BYTES : COMBINE_FLOATS * 4;
    static constexpr int SMEM = BODY0 + TOK_BYTES + CVT_BYTES + QPROJ_FLOATS * 4 + STAGE_BYTES_TOTAL + 1024;
    static_assert(TT % 16 == 0 && COEF_BYTES % 1024 == 0, "tile shape");
    static_assert(SMEM + 4096 <= 227 * 1024, "shared memory (dynamic + the kernel's static arrays)");
    static_assert(BODY0 % 16 == 0, "the split merge stages partials by bulk copy after the body");
};

// Writes out = (c^ B_V + u^ R_V) / l from the merged coefficient-space sums v [g][RB + 16].
template <int D, int RB>
struct EmitProject {
    const DecodeArgs& a;
    size_t head0;
    const uint16_t* Bv;     // [RB][D] bf16 in shared memory
    const uint16_t* Rv;     // [16][D] bf16 in shared memory
    __device__ void operator()(const float* v, const float* l, const float* lx, const float* m, const float* z) const {
        constexpr int PDV = RB + RM;
        for (int idx = threadIdx.x; idx < a.g * D; idx += blockDim.x) {
            const int h = idx / D;
            const int e = idx % D;
            float acc = 0.f;
#pragma unroll 8
            for (int i = 0; i < RB; ++i) acc += v[h * PDV + i] * bf16_lo(Bv[i * D + e]);
#pragma unroll
            for (int i = 0; i < RM; ++i) acc += v[h * PDV + RB + i] * bf16_lo(Rv[i * D + e]);
            a.out[(head0 + h) * D + e] = l[h] > 0.f ? acc / l[h] : 0.f;
        }
        if (a.lse != nullptr && threadIdx.x < a.g) a.lse[head0 + threadIdx.x] = lse_of(m[threadIdx.x], lx[threadIdx.x]);
        emit_entropy_peak(a, head0, lx, z);
    }
};

// int8 pair (low byte = first) -> bf16 pair, each byte kept only if its flag is set
__device__ __forceinline__ uint32_t i8pair_bf16(uint32_t w16, bool keep0, bool keep1) {
    const int x0 = keep0 ? static_cast<int>(static_cast<int8_t>(w16 & 0xffu)) : 0;
    const int x1 = keep1 ? static_cast<int>(static_cast<int8_t>((w16 >> 8) & 0xffu)) : 0;
    return pack_bf16(static_cast<float>(x0), static_cast<float>(x1));
}

// ENT: the launch asks for the entropy; only then does the softmax carry z (a separate
// instantiation, so the plain decode loop carries nothing for it)
template <int D, int RB, int TT, int NSW, int NW, int NH, bool ENT>
__global__ void __launch_bounds__(NW * 32, 1)
decode_lowrank_kernel(const __grid_constant__ CUtensorMap tmCK, const __grid_constant__ CUtensorMap tmCV,
                      const DecodeArgs a) {
    using C = LrCfg<D, RB, TT, NSW, NW>;
    using LY = typename C::L;
    constexpr int MT = TT / 16;
    constexpr int NB = NH / 8;
    extern __shared__ uint8_t smem_dyn[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
    float* tok = reinterpret_cast<float*>(smem + C::BODY0);                    // [NW][3][TT]: s_K, s_V, rank
    uint8_t* cvt = reinterpret_cast<uint8_t*>(tok + NW * TT * 3);              // [NW][K | V][TT][16] f16
    float* qproj = reinterpret_cast<float*>(cvt + C::CVT_BYTES);               // [16][RB + RM]
    uint8_t* stagebuf = reinterpret_cast<uint8_t*>(qproj + C::QPROJ_FLOATS);   // K factors, q rows, V factors
    uint8_t* vfac = stagebuf + C::OFF_VFAC;
    __shared__ __align__(8) uint64_t bars[NW * NSW + 1];
    __shared__ __align__(8) uint64_t fac_bar[2];    // [0]: B_K, R_K, q   [1]: B_V, R_V

    const int split = blockIdx.x;
    const int j = blockIdx.y;
    const int b = blockIdx.z;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int g = a.g;
    const int tile0 = split * a.tiles_per_split;
    // the sequence's own tokens; with per-sequence lengths they are read where the first
    // tiles are requested (before the dependent-launch wait only under kv_early)
    int tlen = a.T;
    int tile1 = tile0;
    const int crow = (a.pair * a.B + b) * a.Hkv + j;        // coefficient row in [P*B*Hkv]
    const int urow = b * a.Hkv + j;                         // code row within the layer's [B*Hkv]
    const size_t tokrow = static_cast<size_t>(b * a.Hkv + j) * a.T;   // s_K / s_V row start
    const uint8_t* rank_row = a.rank + static_cast<size_t>(b) * a.T;

    const uint16_t* qsrc = reinterpret_cast<const uint16_t*>(a.q) +
                           (static_cast<size_t>(b) * a.Hq + static_cast<size_t>(j) * g) * D;
    if (threadIdx.x == 0) {
        prefetch_tmap(&tmCK);
        prefetch_tmap(&tmCV);
        for (int i = 0; i < NW * NSW + 1; ++i) mbar_init(&bars[i], 1);
        mbar_init(&fac_bar[0], 1);
        mbar_init(&fac_bar[1], 1);
        mbar_init_fence();
    }
    __syncthreads();   // every warp's ring barriers are initialised before any warp issues
    uint8_t* ring = smem + warp * NSW * C::STAGE_BYTES;
    uint64_t* wb = &bars[warp * NSW];
    int my_n = 0;
    auto set_range = [&] {
        tlen = seq_len(a, b);
        tile1 = min(tile0 + a.tiles_per_split, (tlen + TT - 1) / TT);
        const int span = tile1 - tile0;
        my_n = span > warp ? (span - warp + NW - 1) / NW : 0;
    };

    // A tile's stage: its coefficients by TMA first (lane 0), then, once the tile's ranks
    // are known, the used bytes of its code groups by bulk copy; the second step arrives.
    auto issue_coef = [&](int k) {
        const int t = tile0 + warp + k * NW;
        const int s = k % NSW;
        uint8_t* st = ring + s * C::STAGE_BYTES;
        mbar_expect_tx(&wb[s], 2 * C::COEF_BYTES);
#pragma unroll
        for (int h = 0; h < LY::HALVES; ++h) {
            tma_load_3d(st + h * TT * 128, &tmCK, h * 64, t * TT, crow, &wb[s]);
            tma_load_3d(st + C::COEF_BYTES + h * TT * 128, &tmCV, h * 64, t * TT, crow, &wb[s]);
        }
    };
    // per-token scales and ranks of a tile, loaded by the lanes (tokens lane, lane+32, ...);
    // lane u-th token of the tile's code group u
    constexpr int TPL = TT / 32;
    static_assert(TT % CODE_GROUP == 0 && CODE_GROUP == 32, "code groups of 32 tokens, one per lane set");
    // whole warp: the tile's code-group sizes (pad16 of the summed code lengths) from
    // its ranks, then lane 0 requests them
    auto issue_codes = [&](int k, const unsigned (&rr)[TPL]) {
        const int t = tile0 + warp + k * NW;
        const int s = k % NSW;
        unsigned gb[TPL], total = 0;
#pragma unroll
        for (int u = 0; u < TPL; ++u) {
            gb[u] = (__reduce_add_sync(0xffffffffu, static_cast<unsigned>(code_len(rr[u]))) + 15u) & ~15u;
            total += gb[u];
        }
        if (lane == 0) {
            uint8_t* st = ring + s * C::STAGE_BYTES;
            mbar_arrive_expect_tx(&wb[s], 2 * total);
#pragma unroll
            for (int u = 0; u < TPL; ++u) {
                if (gb[u] == 0) continue;
                const size_t g0 = (static_cast<size_t>(urow) * a.T + static_cast<size_t>(t) * TT + u * 32) * RM;
                bulk_load(st + C::OFF_UK + u * 32 * RM, a.u_k + g0, gb[u], &wb[s]);
                bulk_load(st + C::OFF_UV + u * 32 * RM, a.u_v + g0, gb[u], &wb[s]);
            }
        }
    };
    // ranks of the tokens of tile k this lane stands for (0 past the sequence)
    auto ranks_of = [&](int k, unsigned (&rr)[TPL]) {
        const int t0 = (tile0 + warp + k * NW) * TT;
#pragma unroll
        for (int u = 0; u < TPL; ++u) {
            const int tt = t0 + lane + 32 * u;
            rr[u] = tt < tlen ? static_cast<unsigned>(__ldg(rank_row + tt)) : 0u;
        }
    };
    // raw 16-bit scales and 8-bit ranks: converted only when published, a tile later, so
    // nothing waits on these loads until then
    unsigned pf_sk[TPL], pf_sv[TPL], pf_r[TPL];
    auto prefetch = [&](int k) {
        const int t0 = (tile0 + warp + k * NW) * TT;
#pragma unroll
        for (int u = 0; u < TPL; ++u) {
            const int t = t0 + lane + 32 * u;
            if (t < tlen) {
                pf_sk[u] = __ldg(a.s_k + tokrow + t);
                pf_sv[u] = __ldg(a.s_v + tokrow + t);
                pf_r[u] = __ldg(rank_row + t);
            } else {
                pf_sk[u] = 0u; pf_sv[u] = 0u; pf_r[u] = 0u;
            }
        }
    };
    // Cache reads only (bases, residual factors, this warp's first tiles and scales).
    // Under a dependent launch the kernel ahead on the stream may still be running; with
    // kv_early the caller has promised that it writes none of the cache, so these are
    // requested before the wait. The query and everything written come after it.
    auto request_cache = [&] {
        if (threadIdx.x == 0) {
            mbar_arrive_expect_tx(&fac_bar[0], C::STAGE_FACTORS + g * D * 2);   // q lands on it too
            bulk_load(stagebuf, static_cast<const uint16_t*>(a.basis_k) + static_cast<size_t>(j) * RB * D,
                      RB * D * 2, &fac_bar[0]);
            bulk_load(stagebuf + RB * D * 2, static_cast<const uint16_t*>(a.r_k) + static_cast<size_t>(j) * RM * D,
                      RM * D * 2, &fac_bar[0]);
            mbar_arrive_expect_tx(&fac_bar[1], C::STAGE_FACTORS);
            bulk_load(vfac, static_cast<const uint16_t*>(a.basis_v) + static_cast<size_t>(j) * RB * D, RB * D * 2,
                      &fac_bar[1]);
            bulk_load(vfac + RB * D * 2, static_cast<const uint16_t*>(a.r_v) + static_cast<size_t>(j) * RM * D,
                      RM * D * 2, &fac_bar[1]);
        }
        const int first = min(NSW, my_n);
        if (lane == 0) {
            for (int k = 0; k < first; ++k) issue_coef(k);
        }
        unsigned r0[NSW][TPL];
#pragma unroll
        for (int k = 0; k < NSW; ++k)
            if (k < first) ranks_of(k, r0[k]);
#pragma unroll
        for (int k = 0; k < NSW; ++k)
            if (k < first) issue_codes(k, r0[k]);
        __syncwarp();
        if (my_n > 0) prefetch(0);
    };
    if (a.kv_early) {
        set_range();
        request_cache();
    }
    grid_dep_wait();
    if (threadIdx.x == 0) grid_dep_launch();
    if (!a.kv_early) {
        set_range();
        request_cache();
    }
    float* srow = a.sscore != nullptr ? a.sscore + (static_cast<size_t>(b) * a.Hq + static_cast<size_t>(j) * g) * a.T
                                      : nullptr;
    if (threadIdx.x == 0) bulk_load(stagebuf + C::STAGE_FACTORS, qsrc, g * D * 2, &fac_bar[0]);
    for (int idx = g * C::PD + threadIdx.x; idx < 16 * C::PD; idx += blockDim.x) qproj[idx] = 0.f;
    // ---- q~ = B_K q and q^ = R_K q for the g heads: one thread per output; lane l starts
    // its walk over d at pair l, so the 32 lanes of a warp read 32 different banks
    mbar_wait_bounded(&fac_bar[0], 0, a.wait_limit, a.err);
    {
        constexpr int W = D / 2;   // bf16 pairs per row
        const uint32_t* fac = reinterpret_cast<const uint32_t*>(stagebuf);   // basis rows, then factor rows
        const uint32_t* qs = reinterpret_cast<const uint32_t*>(stagebuf + C::STAGE_FACTORS);
        // two adjacent lanes per output (each half of d) when the block has the threads
        const int halves = 2 * g * C::PD <= static_cast<int>(blockDim.x) ? 2 : 1;
        const int WP = W / halves;
        const int total = g * C::PD * halves;
        // whole warps run each pass (the pair sum is a shuffle); lanes past the end idle
        for (int t = threadIdx.x; t < ((total + 31) & ~31); t += blockDim.x) {
            const bool valid = t < total;
            const int idx = valid ? t / halves : 0;
            const int w0 = (t % halves) * WP;
            const uint32_t* row = fac + (idx % C::PD) * W;
            const uint32_t* qr = qs + (idx / C::PD) * W;
            float acc0 = 0.f, acc1 = 0.f, acc2 = 0.f, acc3 = 0.f;
#pragma unroll 4
            for (int k = 0; k < WP; k += 2) {
                const int wa = w0 + ((k + lane) & (WP - 1));
                const int wb = w0 + ((k + 1 + lane) & (WP - 1));
                const uint32_t ba = row[wa], qa = qr[wa];
                const uint32_t bb = row[wb], qb = qr[wb];
                acc0 = fmaf(bf16_lo(ba), bf16_lo(qa), acc0);
                acc1 = fmaf(bf16_hi(ba), bf16_hi(qa), acc1);
                acc2 = fmaf(bf16_lo(bb), bf16_lo(qb), acc2);
                acc3 = fmaf(bf16_hi(bb), bf16_hi(qb), acc3);
            }
            float acc = (acc0 + acc1) + (acc2 + acc3);
            if (halves == 2) acc += __shfl_xor_sync(0xffffffffu, acc, 1);
            if (valid && t % halves == 0) qproj[idx] = acc;
        }
    }
    __syncthreads();
    if (a.stall && threadIdx.x == 0) mbar_wait_bounded(&bars[NW * NSW], 0, a.stall_limit, a.err);

    // B fragments of q~^T (RB rows, bf16 hi + lo) and q^^T (16 rows, f16 hi + lo): each
    // projection keeps about 16 (bf16) or 22 (f16) bits; column = head nb*8 + lane/4
    uint32_t qch[RB / 16][NB][2], qcl[RB / 16][NB][2], quh[NB][2], qul[NB][2];
    {
        const int cq = 2 * (lane & 3);
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) {
            const int h = nb * 8 + (lane >> 2);
            auto frag = [&](int col, uint32_t& hi, uint32_t& lo) {
                const float x0 = qproj[h * C::PD + col];
                const float x1 = qproj[h * C::PD + col + 1];
                hi = pack_bf16(x0, x1);
                lo = pack_bf16(x0 - bf16_lo(hi), x1 - bf16_hi(hi));
            };
#pragma unroll
            for (int ks = 0; ks < RB / 16; ++ks) {
                frag(ks * 16 + cq, qch[ks][nb][0], qcl[ks][nb][0]);
                frag(ks * 16 + 8 + cq, qch[ks][nb][1], qcl[ks][nb][1]);
            }
            auto frag16 = [&](int col, uint32_t& hi, uint32_t& lo) {
                const float x0 = qproj[h * C::PD + col];
                const float x1 = qproj[h * C::PD + col + 1];
                hi = pack_f16(x0, x1);
                const __half2 hv = *reinterpret_cast<const __half2*>(&hi);
                lo = pack_f16(x0 - __low2float(hv), x1 - __high2float(hv));
            };
            frag16(RB + cq, quh[nb][0], qul[nb][0]);
            frag16(RB + 8 + cq, quh[nb][1], qul[nb][1]);
        }
    }

    // accumulators c^^T (RB rows) and u^^T (16 rows), columns = heads
    float oc[RB / 16][NB][4];
    float ou[NB][4];
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) {
#pragma unroll
        for (int i = 0; i < RB / 16; ++i) oc[i][nb][0] = oc[i][nb][1] = oc[i][nb][2] = oc[i][nb][3] = 0.f;
        ou[nb][0] = ou[nb][1] = ou[nb][2] = ou[nb][3] = 0.f;
    }
    float mrow[NB][2], lrow[NB][2], lxrow[NB][2];
    float zrow[NB][2];                    // sums of 2^(s - m) (m - s), for the entropy when asked for
    constexpr bool want_z = ENT;
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) {
        mrow[nb][0] = mrow[nb][1] = NEG_INF;
        lrow[nb][0] = lrow[nb][1] = lxrow[nb][0] = lxrow[nb][1] = 0.f;
        zrow[nb][0] = zrow[nb][1] = 0.f;
    }

    float* tks = tok + warp * TT * 3;     // [3][TT]: s_K, s_V, rank
    int* tkr = reinterpret_cast<int*>(tks + 2 * TT);
    uint8_t* cvk = cvt + warp * 2 * TT * 32;   // this warp's f16 K codes [TT][16]
    uint8_t* cvv = cvk + TT * 32;              //                  V codes [TT][16]
    // byte offset of the 16-B half `seg` (channels 8 seg .. 8 seg + 7) of token row t
    auto cvt_off = [](int t, int seg) { return static_cast<uint32_t>(t * 32 + ((seg ^ ((t >> 2) & 1)) << 4)); };


    const int mi = lane >> 3;
    const int ri = lane & 7;
    const int q4 = lane & 3;
    for (int k = 0; k < my_n; ++k) {
        const int s = k % NSW;
        // publish this tile's per-token values, start fetching the next tile's
        __syncwarp();
#pragma unroll
        for (int u = 0; u < TPL; ++u) {
            tks[lane + 32 * u] = __half2float(__ushort_as_half(static_cast<unsigned short>(pf_sk[u])));
            tks[TT + lane + 32 * u] = __half2float(__ushort_as_half(static_cast<unsigned short>(pf_sv[u])));
            tkr[lane + 32 * u] = static_cast<int>(pf_r[u]);
        }
        // where each token's codes start in its group: the exclusive scan of the group's
        // code lengths (lane = token), while the tile is still landing
        int code_off[TPL];
#pragma unroll
        for (int u = 0; u < TPL; ++u) {
            const int kl = code_len(pf_r[u]);
            int o = kl;
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                const int n = __shfl_up_sync(0xffffffffu, o, d);
                if (lane >= d) o += n;
            }
            code_off[u] = o - kl;
        }
        if (k + 1 < my_n) prefetch(k + 1);
        // ranks of the tile requested at the end of this one (loaded here, a register
        // that no later iteration carries: a load still in flight across the loop's
        // back edge made the whole step 2.2 us per layer slower)
        unsigned nr[TPL];
        if (k + NSW < my_n) ranks_of(k + NSW, nr);
        __syncwarp();
        const bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(&wb[s], (k / NSW) & 1, a.wait_limit, a.err));
        if (!ok) {
            const int issued = min(my_n, k + NSW);
            for (int kk = k + 1; kk < issued; ++kk) mbar_wait_bounded(&wb[kk % NSW], (kk / NSW) & 1, a.wait_limit, a.err);
            break;
        }
        const int t = tile0 + warp + k * NW;
        if (a.lens != nullptr && (t + 1) * TT > tlen) {
            // V coefficients past the sequence (the K side is masked by score)
            if (RB == 32)
                zero_tile_rows(ring + s * C::STAGE_BYTES + C::COEF_BYTES, 64, 1, 0, tlen - t * TT, TT, lane);
            else
                zero_tile_rows(ring + s * C::STAGE_BYTES + C::COEF_BYTES, 128, LY::HALVES, TT * 128, tlen - t * TT, TT,
                               lane);
            __syncwarp();
        }
        const uint32_t ckb = smem_u32(ring + s * C::STAGE_BYTES);
        const uint32_t cvb = ckb + C::COEF_BYTES;
        const uint8_t* ukp = ring + s * C::STAGE_BYTES + C::OFF_UK;
        const uint8_t* uvp = ring + s * C::STAGE_BYTES + C::OFF_UV;
        // the tile's int8 codes -> f16, masked to each token's rank: lane = token row
#pragma unroll
        for (int u = 0; u < TPL; ++u) {
            const int tr = lane + 32 * u;
            const int r = tkr[tr];
            const uint4 wk = codes_at(ukp + u * 32 * RM + code_off[u]);
            const uint4 wv = codes_at(uvp + u * 32 * RM + code_off[u]);
            uint32_t m0, m1, m2, m3;
            rank_keep4(r, m0, m1, m2, m3);
            uint4 k0, k1, v0, v1;
            i8x4_f16(wk.x, m0, k0.x, k0.y);
            i8x4_f16(wk.y, m1, k0.z, k0.w);
            i8x4_f16(wk.z, m2, k1.x, k1.y);
            i8x4_f16(wk.w, m3, k1.z, k1.w);
            i8x4_f16(wv.x, m0, v0.x, v0.y);
            i8x4_f16(wv.y, m1, v0.z, v0.w);
            i8x4_f16(wv.z, m2, v1.x, v1.y);
            i8x4_f16(wv.w, m3, v1.z, v1.w);
            *reinterpret_cast<uint4*>(cvk + cvt_off(tr, 0)) = k0;
            *reinterpret_cast<uint4*>(cvk + cvt_off(tr, 1)) = k1;
            *reinterpret_cast<uint4*>(cvv + cvt_off(tr, 0)) = v0;
            *reinterpret_cast<uint4*>(cvv + cvt_off(tr, 1)) = v1;
        }
        __syncwarp();

        float sc[MT][NB][4];
        float su[MT][NB][4];
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int nb = 0; nb < NB; ++nb) {
                sc[mt][nb][0] = sc[mt][nb][1] = sc[mt][nb][2] = sc[mt][nb][3] = 0.f;
                su[mt][nb][0] = su[mt][nb][1] = su[mt][nb][2] = su[mt][nb][3] = 0.f;
            }
        // ---- basis part of the scores: C_K q~^T (hi and lo)
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
            const int row = mt * 16 + (mi & 1) * 8 + ri;
#pragma unroll
            for (int ks = 0; ks < RB / 16; ++ks) {
                uint32_t af[4];
                ldsm_x4(ckb + LY::template off<TT>(row, ks * 2 + (mi >> 1)), af[0], af[1], af[2], af[3]);
#pragma unroll
                for (int nb = 0; nb < NB; ++nb) {
                    mma_bf16(sc[mt][nb], af, qch[ks][nb][0], qch[ks][nb][1]);
                    mma_bf16(sc[mt][nb], af, qcl[ks][nb][0], qcl[ks][nb][1]);
                }
            }
        }
        // ---- residual part: U_K (f16 codes masked to each token's rank) q^^T
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
            const int row = mt * 16 + (mi & 1) * 8 + ri;
            uint32_t af[4];
            ldsm_x4(smem_u32(cvk) + cvt_off(row, mi >> 1), af[0], af[1], af[2], af[3]);
#pragma unroll
            for (int nb = 0; nb < NB; ++nb) {
                mma_f16(su[mt][nb], af, quh[nb][0], quh[nb][1]);
                mma_f16(su[mt][nb], af, qul[nb][0], qul[nb][1]);
            }
        }
        // ---- scores, mask, online softmax per head; P^T and (P s_V)^T by movmatrix
        uint32_t pb[MT][NB][2], pvb[MT][NB][2];
        const bool tail = (t + 1) * TT > tlen;       // only the last tile holds tokens past the sequence
        const int lim = tlen - t * TT;
        float skr[MT][2];                            // s_K of this lane's two rows per m tile
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
            skr[mt][0] = tks[mt * 16 + (lane >> 2)];
            skr[mt][1] = tks[mt * 16 + (lane >> 2) + 8];
        }
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) {
            float mx0 = NEG_INF, mx1 = NEG_INF;
#pragma unroll
            for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    sc[mt][nb][i] = fmaf(skr[mt][i >> 1], su[mt][nb][i], sc[mt][nb][i]);   // raw score
            if (tail) {
#pragma unroll
                for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        if (mt * 16 + (lane >> 2) + (i >> 1) * 8 >= lim) sc[mt][nb][i] = NEG_INF;
            }
            if (srow != nullptr) {
                // keep the scores of the tile's valid tokens for the attention statistics
                const int h0 = nb * 8 + 2 * q4;
#pragma unroll
                for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int h = h0 + (i & 1);
                        const int r = mt * 16 + (lane >> 2) + (i >> 1) * 8;
                        if (h < g && r < lim) srow[static_cast<size_t>(h) * a.T + t * TT + r] = __fmul_rn(sc[mt][nb][i], a.scale_log2);
                    }
            }
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                mx0 = fmaxf(mx0, fmaxf(sc[mt][nb][0], sc[mt][nb][2]));
                mx1 = fmaxf(mx1, fmaxf(sc[mt][nb][1], sc[mt][nb][3]));
            }
#pragma unroll
            for (int off = 4; off < 32; off <<= 1) {
                mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
                mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
            }
            // the row max in the scaled (log2) domain: scaling by a positive factor and
            // rounding are monotonic, so this is the max of the scaled scores
            mx0 = __fmul_rn(mx0, a.scale_log2);
            mx1 = __fmul_rn(mx1, a.scale_log2);
            const float mn0 = fmaxf(mrow[nb][0], mx0), mn1 = fmaxf(mrow[nb][1], mx1);
            const float ref0 = mn0 == NEG_INF ? 0.f : mn0;
            const float ref1 = mn1 == NEG_INF ? 0.f : mn1;
            const float cr0 = ex2_approx(mrow[nb][0] - ref0), cr1 = ex2_approx(mrow[nb][1] - ref1);
            if (want_z) {
                // z moves to the new reference with the unscaled lx (see kvs_device.cuh)
                zrow[nb][0] = cr0 * fmaf(lxrow[nb][0], mrow[nb][0] == NEG_INF ? 0.f : ref0 - mrow[nb][0], zrow[nb][0]);
                zrow[nb][1] = cr1 * fmaf(lxrow[nb][1], mrow[nb][1] == NEG_INF ? 0.f : ref1 - mrow[nb][1], zrow[nb][1]);
            }
            mrow[nb][0] = mn0;
            mrow[nb][1] = mn1;
            lrow[nb][0] *= cr0;
            lrow[nb][1] *= cr1;
            lxrow[nb][0] *= cr0;
            lxrow[nb][1] *= cr1;
#pragma unroll
            for (int i = 0; i < RB / 16; ++i) { oc[i][nb][0] *= cr0; oc[i][nb][2] *= cr0; oc[i][nb][1] *= cr1; oc[i][nb][3] *= cr1; }
            ou[nb][0] *= cr0; ou[nb][2] *= cr0; ou[nb][1] *= cr1; ou[nb][3] *= cr1;
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                const int ta = mt * 16 + (lane >> 2);
                const float x0 = fmaf(sc[mt][nb][0], a.scale_log2, -ref0);
                const float x1 = fmaf(sc[mt][nb][1], a.scale_log2, -ref1);
                const float x2 = fmaf(sc[mt][nb][2], a.scale_log2, -ref0);
                const float x3 = fmaf(sc[mt][nb][3], a.scale_log2, -ref1);
                const float p0 = ex2_approx(x0);
                const float p1 = ex2_approx(x1);
                const float p2 = ex2_approx(x2);
                const float p3 = ex2_approx(x3);
                const uint32_t lo = pack_bf16(p0, p1), hi = pack_bf16(p2, p3);
                lrow[nb][0] += bf16_lo(lo) + bf16_lo(hi);
                lrow[nb][1] += bf16_hi(lo) + bf16_hi(hi);
                lxrow[nb][0] += p0 + p2;
                lxrow[nb][1] += p1 + p3;
                if (want_z) {
                    // p (ref - s); a masked token (x = -inf, p = 0) adds 0
                    zrow[nb][0] = fmaf(p0, -fmaxf(x0, -3.0e38f), fmaf(p2, -fmaxf(x2, -3.0e38f), zrow[nb][0]));
                    zrow[nb][1] = fmaf(p1, -fmaxf(x1, -3.0e38f), fmaf(p3, -fmaxf(x3, -3.0e38f), zrow[nb][1]));
                }
                pb[mt][nb][0] = movmatrix_t(lo);
                pb[mt][nb][1] = movmatrix_t(hi);
                const float sva = tks[TT + ta], svb = tks[TT + ta + 8];
                pvb[mt][nb][0] = movmatrix_t(pack_f16(p0 * sva, p1 * sva));
                pvb[mt][nb][1] = movmatrix_t(pack_f16(p2 * svb, p3 * svb));
            }
        }
        // ---- c^^T += C_V^T P^T
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
            const int row = mt * 16 + (mi >> 1) * 8 + ri;
#pragma unroll
            for (int ct = 0; ct < RB / 16; ++ct) {
                uint32_t af[4];
                ldsm_x4_t(cvb + LY::template off<TT>(row, ct * 2 + (mi & 1)), af[0], af[1], af[2], af[3]);
#pragma unroll
                for (int nb = 0; nb < NB; ++nb) mma_bf16(oc[ct][nb], af, pb[mt][nb][0], pb[mt][nb][1]);
            }
        }
        // ---- u^^T += U_V^T (P s_V)^T: the f16 codes (masked to each token's rank) read
        // transposed, channels as rows and tokens as k
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
            const int row = mt * 16 + (mi >> 1) * 8 + ri;
            uint32_t af[4];
            ldsm_x4_t(smem_u32(cvv) + cvt_off(row, mi & 1), af[0], af[1], af[2], af[3]);
#pragma unroll
            for (int nb = 0; nb < NB; ++nb) mma_f16(ou[nb], af, pvb[mt][nb][0], pvb[mt][nb][1]);
        }
        __syncwarp();
        if (k + NSW < my_n) {
            if (lane == 0) {
                fence_proxy_async();
                issue_coef(k + NSW);
            }
            issue_codes(k + NSW, nr);
        }
    }
#pragma unroll
    for (int nb = 0; nb < NB; ++nb)
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) {
            lrow[nb][0] += __shfl_xor_sync(0xffffffffu, lrow[nb][0], off);
            lrow[nb][1] += __shfl_xor_sync(0xffffffffu, lrow[nb][1], off);
            lxrow[nb][0] += __shfl_xor_sync(0xffffffffu, lxrow[nb][0], off);
            lxrow[nb][1] += __shfl_xor_sync(0xffffffffu, lxrow[nb][1], off);
            zrow[nb][0] += __shfl_xor_sync(0xffffffffu, zrow[nb][0], off);
            zrow[nb][1] += __shfl_xor_sync(0xffffffffu, zrow[nb][1], off);
        }

    // ---- merge warps in coefficient space, project once, finish the split
    // (the code-conversion buffers, written through the generic proxy in the loop, later
    // receive the unit's partials by bulk copy)
    fence_proxy_async();
    __syncthreads();
    constexpr int PD = C::PD;
    float* comb = reinterpret_cast<float*>(smem);   // [NW][16][PD]
    float* comb_m = comb + NW * 16 * PD;
    float* comb_l = comb_m + NW * 16;
    float* comb_lx = comb_l + NW * 16;
    float* comb_z = comb_lx + NW * 16;
    float* fin_m = comb_z + NW * 16;
    float* fin_l = fin_m + 16;
    float* fin_lx = fin_l + 16;
    float* fin_z = fin_lx + 16;
    float* fin_c = fin_z + 16;                      // [16][PD]
    float* fin_o = fin_c + 16 * PD;                 // [16][D]
    float* scratch = fin_o + 16 * D;
    {
        const int e0 = lane >> 2;
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) {
            const int h0 = nb * 8 + 2 * q4;
#pragma unroll
            for (int ct = 0; ct < RB / 16; ++ct) {
                comb[(warp * 16 + h0) * PD + ct * 16 + e0] = oc[ct][nb][0];
                comb[(warp * 16 + h0) * PD + ct * 16 + e0 + 8] = oc[ct][nb][2];
                comb[(warp * 16 + h0 + 1) * PD + ct * 16 + e0] = oc[ct][nb][1];
                comb[(warp * 16 + h0 + 1) * PD + ct * 16 + e0 + 8] = oc[ct][nb][3];
            }
            comb[(warp * 16 + h0) * PD + RB + e0] = ou[nb][0];
            comb[(warp * 16 + h0) * PD + RB + e0 + 8] = ou[nb][2];
            comb[(warp * 16 + h0 + 1) * PD + RB + e0] = ou[nb][1];
            comb[(warp * 16 + h0 + 1) * PD + RB + e0 + 8] = ou[nb][3];
            if (lane < 4) {
                comb_m[warp * 16 + h0] = mrow[nb][0];
                comb_m[warp * 16 + h0 + 1] = mrow[nb][1];
                comb_l[warp * 16 + h0] = lrow[nb][0];
                comb_l[warp * 16 + h0 + 1] = lrow[nb][1];
                comb_lx[warp * 16 + h0] = lxrow[nb][0];
                comb_lx[warp * 16 + h0 + 1] = lxrow[nb][1];
                comb_z[warp * 16 + h0] = zrow[nb][0];
                comb_z[warp * 16 + h0 + 1] = zrow[nb][1];
            }
        }
    }
    __syncthreads();
    // one weight 2^(m_w - M) per (warp, head), so the vector combine is FMAs only
    __shared__ float fac[NW][16];
    if (threadIdx.x < g) {
        const int h = threadIdx.x;
        float M = NEG_INF;
        for (int ww = 0; ww < NW; ++ww) M = fmaxf(M, comb_m[ww * 16 + h]);
        float L = 0.f, LX = 0.f, Z = 0.f;
        for (int ww = 0; ww < NW; ++ww) {
            const float m = comb_m[ww * 16 + h];
            const float f = merge_factor(m, M);
            fac[ww][h] = f;
            L += f * comb_l[ww * 16 + h];
            LX += f * comb_lx[ww * 16 + h];
            Z += merged_z(f, m, M, comb_lx[ww * 16 + h], comb_z[ww * 16 + h]);
        }
        fin_m[h] = M;
        fin_l[h] = L;
        fin_lx[h] = LX;
        fin_z[h] = Z;
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < g * PD; idx += blockDim.x) {
        const int h = idx / PD;
        float acc = 0.f;
        // a warp without tokens left its slot unset: skip it, never 0 * x
#pragma unroll
        for (int ww = 0; ww < NW; ++ww)
            if (fac[ww][h] != 0.f) acc = fmaf(fac[ww][h], comb[(ww * 16 + h) * PD + (idx % PD)], acc);
        fin_c[idx] = acc;
    }
    __syncthreads();
    // partials stay in coefficient space (RB + 16 values per head); the CTA that
    // finishes the unit projects once: o = (c^ B_V + u^ R_V) / l
    mbar_wait_bounded(&fac_bar[1], 0, a.wait_limit, a.err);
    const uint16_t* Bv = reinterpret_cast<const uint16_t*>(vfac);
    const EmitProject<D, RB> emit{a, static_cast<size_t>(b) * a.Hq + static_cast<size_t>(j) * g, Bv, Bv + RB * D};
    const int unit = b * a.Hkv + j;
    // the per-token and code-conversion buffers are free now: they stage the unit's partials
    finish_unit<(PD > D ? PD : D)>(a, PD, unit, split, a.splits, static_cast<long long>(unit) * a.splits, fin_m, fin_l,
                                   fin_lx, fin_z, fin_c, scratch,
                reinterpret_cast<uint8_t*>(tok), C::TOK_BYTES + C::CVT_BYTES, emit);
}

template <int D, int RB, int TT, int NSW, int NW, int NH, bool ENT>
cudaError_t launch_ent(const DecodeArgs& a, const CUtensorMap* maps, cudaStream_t st) {
    using C = LrCfg<D, RB, TT, NSW, NW>;
    auto kern = decode_lowrank_kernel<D, RB, TT, NSW, NW, NH, ENT>;
    static std::atomic<unsigned long long> attr_done{0};
    cudaError_t e = once_per_device(attr_done, [&] {
        return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    });
    if (e != cudaSuccess) return e;
    dim3 grid(a.splits, a.Hkv, a.B);
    return launch_kernel(kern, grid, dim3(NW * 32), C::SMEM, st, a.pdl != 0, maps[0], maps[1], a);
}

template <int D, int RB, int TT, int NSW, int NW, int NH>
cudaError_t launch_nh(const DecodeArgs& a, const CUtensorMap* maps, cudaStream_t st) {
    return a.entropy != nullptr ? launch_ent<D, RB, TT, NSW, NW, NH, true>(a, maps, st)
                                : launch_ent<D, RB, TT, NSW, NW, NH, false>(a, maps, st);
}

template <int D, int RB, int TT, int NSW, int NW>
cudaError_t launch_one(const DecodeArgs& a, const CUtensorMap* maps, cudaStream_t st) {
    return a.g <= 8 ? launch_nh<D, RB, TT, NSW, NW, 8>(a, maps, st) : launch_nh<D, RB, TT, NSW, NW, 16>(a, maps, st);
}

template <int D, int RB, int TT, int NSW, int NW>
int occupancy_of() {
    using C = LrCfg<D, RB, TT, NSW, NW>;
    auto kern = decode_lowrank_kernel<D, RB, TT, NSW, NW, 8, false>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, NW * 32, C::SMEM) != cudaSuccess) return 1;
    return n > 0 ? n : 1;
}

// token tile, stages per warp and warps per CTA by basis rank (the 64 and full-rank
// bases only serve tests). Rb = 32 defaults: the fastest of a measured sweep on the
// 64K-token workload (µs per layer in the replayed step): 12 warps with two 32-token
// stages each 25.7; 16 warps x 1 stage 27.5; 8 x 2 and 8 x 3 27.0; 8 warps x one
// 64-token stage 28.5 (and earlier: 18 to 20 warps x 1 stage slower than 16).
#ifndef KVS_LR_TT
#define KVS_LR_TT 32
#endif

#ifndef KVS_LR_NSW
#define KVS_LR_NSW 2
#endif
#ifndef KVS_LR_NW
#define KVS_LR_NW 12
#endif
template <int RB>
struct LrShape {
    static constexpr int TT = RB == 32 ? KVS_LR_TT : 32;
    static constexpr int NSW = RB == 32 ? KVS_LR_NSW : 1;
    static constexpr int NW = RB == 32 ? KVS_LR_NW : (RB == 128 ? 4 : 16);
};

template <int D, int RB>
int occ() { return occupancy_of<D, RB, LrShape<RB>::TT, LrShape<RB>::NSW, LrShape<RB>::NW>(); }

template <int D, int RB>
cudaError_t run(const DecodeArgs& a, const CUtensorMap* maps, cudaStream_t st) {
    return launch_one<D, RB, LrShape<RB>::TT, LrShape<RB>::NSW, LrShape<RB>::NW>(a, maps, st);
}

}  // namespace

int decode_lowrank_tile(int rb) { return rb == 32 ? LrShape<32>::TT : (rb == 64 ? LrShape<64>::TT : LrShape<128>::TT); }

int decode_lowrank_occupancy(int d, int rb) {
    if (d == 64) return rb == 32 ? occ<64, 32>() : occ<64, 64>();
    return rb == 32 ? occ<128, 32>() : occ<128, 128>();
}

cudaError_t launch_decode_lowrank(int d, int rb, const DecodeArgs& a, const CUtensorMap* maps, cudaStream_t st) {
    if (d == 64) return rb == 32 ? run<64, 32>(a, maps, st) : run<64, 64>(a, maps, st);
    return rb == 32 ? run<128, 32>(a, maps, st) : run<128, 128>(a, maps, st);
}

}  // namespace kvs

// Split-KV GQA decode over a shared cache, bf16 storage, forms SINGLE and MIX.
//
// Balanced split scheduling: the (batch, kv head) units' token tiles form one
// flat list of units * n_t tiles that is cut into G equal ranges, one per CTA.
// By default G is a whole number of CTAs per unit, as many as are resident at
// once, so no range crosses a unit (the STRADDLE = false instance); any other G
// is handled too, a range then covering at most two units. Each unit's partial
// results merge in the last CTA to finish it. When the entropy is asked for, the
// online softmax also carries z = sum 2^(s - m) (m - s) through every merge (the
// ENT instance), so entropy and peak need no pass over the scores.
// Inside a CTA, NW warps each own a private ring of NSW shared-memory stages
// and stream every NW-th tile of the range into it with TMA (128-byte swizzle),
// re-issuing a stage as soon as it is consumed. Per tile and warp, with the
// tokens as the MMA's M rows and the g query heads of the kv head as its N
// columns (a group of up to 8 heads wastes nothing on padding):
//   S^T = K Q^T            mma.sync m16n8k16 bf16 -> fp32
//   MIX S^T = w S1^T + (1-w) S2^T, the two sources' scores mixed in fp32, which
//                          equals the scores against w K1 + (1-w) K2 (the convex
//                          mix of the DepthGraft source pair) up to fp32 rounding
//   online softmax per head in base 2 (max over tokens by shuffles across lanes)
//   P^T: the S^T accumulator rounded to bf16 and transposed in registers
//        (movmatrix) into the B operand of
//   O^T += V^T P^T         for MIX, O^T += V1^T bf16(w P)^T + V2^T bf16((1-w) P)^T
// The mixed K/V never exist anywhere, in HBM or in shared memory.
#include "kvs_device.cuh"

namespace kvs {
namespace {

template <int D, bool MIX, int TT, int NSW, int NW>
struct DecodeCfg {
    static constexpr int HALVES = D / 64;
    static constexpr int HALF_BYTES = TT * 128;              // [TT][64] bf16
    static constexpr int TILE_BYTES = TT * D * 2;
    static constexpr int NSRC = MIX ? 2 : 1;
    static constexpr int STAGE_BYTES = 2 * NSRC * TILE_BYTES;
    static constexpr int RING_BYTES = NW * NSW * STAGE_BYTES;
    static constexpr int COMBINE_FLOATS = NW * 16 * D + 4 * NW * 16 + 64 + 16 * D + 4 * MAX_GROUP * MAX_SPLITS + 64;
    static constexpr int MERGE_STAGE_OFF = ((COMBINE_FLOATS * 4 + 1023) / 1024) * 1024;   // free smem for the merge
    static constexpr int BODY = RING_BYTES > COMBINE_FLOATS * 4 ? RING_BYTES : COMBINE_FLOATS * 4;
    // per-warp state of the first unit when a warp's tiles cross into the second one
    static constexpr int SAVE_FLOATS = NW * (16 * D + 64);
    static constexpr int SMEM = BODY + SAVE_FLOATS * 4 + 1024;  // + slack to align the ring to 1024 B
    static constexpr int SMEM_ALIGNED = BODY + 1024;             // grids whose ranges never straddle
    static_assert(TT % 16 == 0, "token tile must hold whole m16 tiles");
    static_assert(HALF_BYTES % 1024 == 0, "swizzled halves must stay 1024-B aligned");
};

// ENT: the launch asks for the entropy; only then does the softmax carry z (a separate
// instantiation, so the plain decode loop carries nothing for it)
template <int D, bool MIX, int TT, int NSW, int NW, int NH, bool STRADDLE, bool ENT>
__global__ void __launch_bounds__(NW * 32, 1)
decode_bf16_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                   const DecodeArgs a) {
    using C = DecodeCfg<D, MIX, TT, NSW, NW>;
    constexpr int MT = TT / 16;      // m16 token tiles per tile
    constexpr int NB = NH / 8;       // n8 head blocks
    extern __shared__ uint8_t smem_dyn[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
    float* save = reinterpret_cast<float*>(smem + C::BODY);    // [NW][16][D] O, then [NW][64]: m, l, lx, z
    __shared__ __align__(8) uint64_t bars[NW * NSW + 1];
    __shared__ int fin_unit[NW], sav_unit[NW];

    const int cta = blockIdx.x;
    const int G = gridDim.x;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int g = a.g;
    const long long W = static_cast<long long>(a.units) * a.n_t;
    const long long tb = (static_cast<long long>(cta) * W + G - 1) / G;
    const long long te = (static_cast<long long>(cta + 1) * W + G - 1) / G;
    const int cap_span = static_cast<int>(te - tb);        // tiles of the range in store capacity
    const int u_first = static_cast<int>(tb / a.n_t);
    const int u_last = static_cast<int>((te - 1) / a.n_t);
    const int BH = a.B * a.Hkv;
    // token tiles of unit u's own sequence
    auto unit_tiles = [&](int u) { return (seq_len(a, u / a.Hkv) + TT - 1) / TT; };
    // A range inside one unit is clipped to the unit's sequence; a range that may cross
    // units keeps its tiles and skips those past their sequence one by one.
    int span = cap_span;

    if (threadIdx.x == 0) {
        prefetch_tmap(&tmK);
        prefetch_tmap(&tmV);
        for (int i = 0; i < NW * NSW + 1; ++i) mbar_init(&bars[i], 1);
        mbar_init_fence();
    }
    __syncthreads();

    uint8_t* ring = smem + warp * NSW * C::STAGE_BYTES;
    uint64_t* wb = &bars[warp * NSW];
    int my_n = 0;
    // with per-sequence lengths the range depends on them: read them where the first
    // tiles are requested (before the dependent-launch wait only under kv_early)
    auto set_range = [&] {
        if (!STRADDLE && a.lens != nullptr) {
            const long long u_end = static_cast<long long>(u_first) * a.n_t + unit_tiles(u_first);
            span = te <= u_end ? cap_span : (u_end > tb ? static_cast<int>(u_end - tb) : 0);
        }
        my_n = span > warp ? (span - warp + NW - 1) / NW : 0;
    };
    // (unit, tile) of this warp's first tile; later tiles step by NW without dividing
    const long long g0 = tb + warp;
    const int u_w0 = static_cast<int>(g0 / a.n_t);
    const int t_w0 = static_cast<int>(g0 - static_cast<long long>(u_w0) * a.n_t);
    auto advance = [&](int& u, int& t) {
        t += NW;
        while (t >= a.n_t) {
            t -= a.n_t;
            ++u;
        }
    };
    int iu = u_w0, it = t_w0;        // next tile to issue

    auto issue = [&](int k) {
        (void)k;
        const int u = iu;
        const int t = it;
        advance(iu, it);
        const int row0 = a.src0 * BH + u;
        const int row1 = MIX ? a.src1 * BH + u : 0;
        const int s = k % NSW;
        uint8_t* st = ring + s * C::STAGE_BYTES;
        if (STRADDLE && a.lens != nullptr && t >= unit_tiles(u)) {
            mbar_arrive(&wb[s]);      // a tile past its sequence: the stage completes empty
            return;
        }
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
    // Under a dependent launch everything up to grid_dep_wait overlaps the previous
    // kernel's tail. Inputs, workspace and counters are touched only after it; with
    // kv_early the caller has promised that no kernel ahead on the stream writes the
    // cache, so the first ring stages are already requested before the wait.
    if (a.kv_early) {
        set_range();
        if (lane == 0) {
            for (int k = 0; k < min(NSW, my_n); ++k) issue(k);
        }
        __syncwarp();
    }
    grid_dep_wait();
    if (threadIdx.x == 0) grid_dep_launch();
    if (!a.kv_early) {
        set_range();
        if (lane == 0) {
            for (int k = 0; k < min(NSW, my_n); ++k) issue(k);
        }
        __syncwarp();
    }

    if (a.stall && threadIdx.x == 0) {
        // test hook: nothing ever arrives on the spare barrier; the bounded wait gives up
        mbar_wait_bounded(&bars[NW * NSW], 0, a.stall_limit, a.err);
    }

    uint32_t qb[D / 16][NB][2];      // B fragments of Q^T: column n = head nb*8 + lane/4
    float o[D / 16][NB][4];          // O^T: rows = channels, columns = heads nb*8 + 2(lane%4) (+1)
    float mrow[NB][2], lrow[NB][2];  // softmax statistics of those two heads
    float lxrow[NB][2];              // sums of the unrounded weights (for the lse)
    float zrow[NB][2];               // sums of 2^(s - m) (m - s) (for the entropy, when asked for)
    constexpr bool want_z = ENT;
    float w = 1.f, w1 = 0.f;
    int tlen = a.T;                  // tokens of the current unit's sequence
    float* srow = nullptr;           // the current unit's kept scores [g][T], if requested
    auto begin_unit = [&](int u) {
        const int b = u / a.Hkv;
        const int j = u % a.Hkv;
        const uint16_t* qg = reinterpret_cast<const uint16_t*>(a.q) +
                             (static_cast<size_t>(b) * a.Hq + static_cast<size_t>(j) * g) * D;
        const int cq = 2 * (lane & 3);
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) {
            const int h = nb * 8 + (lane >> 2);
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
                qb[ks][nb][0] = h < g ? *reinterpret_cast<const uint32_t*>(qg + h * D + ks * 16 + cq) : 0u;
                qb[ks][nb][1] = h < g ? *reinterpret_cast<const uint32_t*>(qg + h * D + ks * 16 + 8 + cq) : 0u;
            }
            mrow[nb][0] = mrow[nb][1] = NEG_INF;
            lrow[nb][0] = lrow[nb][1] = 0.f;
            lxrow[nb][0] = lxrow[nb][1] = 0.f;
            zrow[nb][0] = zrow[nb][1] = 0.f;
#pragma unroll
            for (int i = 0; i < D / 16; ++i) o[i][nb][0] = o[i][nb][1] = o[i][nb][2] = o[i][nb][3] = 0.f;
        }
        w = MIX ? a.w[j] : 1.f;
        w1 = 1.f - w;
        tlen = seq_len(a, b);
        srow = a.sscore != nullptr ? a.sscore + (static_cast<size_t>(b) * a.Hq + static_cast<size_t>(j) * g) * a.T
                                   : nullptr;
    };
    // write this warp's statistics and O^T for heads < g: O to dst_o [16][D], m, l, lx, z
    // to dst_ml [64]
    auto store_state = [&](float* dst_o, float* dst_ml) {
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
        const int e0 = lane >> 2;
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) {
            const int h0 = nb * 8 + 2 * (lane & 3);
#pragma unroll
            for (int dt = 0; dt < D / 16; ++dt) {
                if (h0 < g) {
                    dst_o[h0 * D + dt * 16 + e0] = o[dt][nb][0];
                    dst_o[h0 * D + dt * 16 + e0 + 8] = o[dt][nb][2];
                }
                if (h0 + 1 < g) {
                    dst_o[(h0 + 1) * D + dt * 16 + e0] = o[dt][nb][1];
                    dst_o[(h0 + 1) * D + dt * 16 + e0 + 8] = o[dt][nb][3];
                }
            }
            if (lane < 4) {
                dst_ml[h0] = mrow[nb][0];
                dst_ml[h0 + 1] = mrow[nb][1];
                dst_ml[16 + h0] = lrow[nb][0];
                dst_ml[16 + h0 + 1] = lrow[nb][1];
                dst_ml[32 + h0] = lxrow[nb][0];
                dst_ml[32 + h0 + 1] = lxrow[nb][1];
                dst_ml[48 + h0] = zrow[nb][0];
                dst_ml[48 + h0 + 1] = zrow[nb][1];
            }
        }
    };


    int cur_u = -1, saved_u = -1;
    const int mi = lane >> 3;        // ldmatrix: which 8x8 matrix this lane addresses
    const int ri = lane & 7;         //           and which row of it
    int u = u_w0, t = t_w0;          // tile being consumed
    if (!STRADDLE && my_n > 0) {
        // the CTA's range lies inside one unit
        begin_unit(u_first);
        cur_u = u_first;
    }
    for (int k = 0; k < my_n; ++k, advance(u, t)) {
        if (STRADDLE && u != cur_u) {
            if (cur_u >= 0) {
                store_state(save + warp * 16 * D, save + NW * 16 * D + warp * 64);
                saved_u = cur_u;
            }
            begin_unit(u);
            cur_u = u;
        }
        const int s = k % NSW;
        const bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(&wb[s], (k / NSW) & 1, a.wait_limit, a.err));
        if (!ok) {
            // give the copies still in flight a bounded chance to land, then stop
            const int issued = min(my_n, k + NSW);
            for (int kk = k + 1; kk < issued; ++kk) mbar_wait_bounded(&wb[kk % NSW], (kk / NSW) & 1, a.wait_limit, a.err);
            break;
        }
        if (STRADDLE && t * TT >= tlen) {
            // a tile past the sequence: its stage completed empty; hand it on
            __syncwarp();
            if (lane == 0 && k + NSW < my_n) issue(k + NSW);
            __syncwarp();
            continue;
        }
        if (a.lens != nullptr && (t + 1) * TT > tlen) {
            uint8_t* vt = ring + s * C::STAGE_BYTES + C::TILE_BYTES;
            zero_tile_rows(vt, 128, C::HALVES, C::HALF_BYTES, tlen - t * TT, TT, lane);
            if (MIX) zero_tile_rows(vt + 2 * C::TILE_BYTES, 128, C::HALVES, C::HALF_BYTES, tlen - t * TT, TT, lane);
            __syncwarp();
        }
        const uint32_t kb = smem_u32(ring + s * C::STAGE_BYTES);
        const uint32_t vb = kb + C::TILE_BYTES;

        float sc[MT][NB][4];
        float sc2[MIX ? MT : 1][NB][4];
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int nb = 0; nb < NB; ++nb) {
                sc[mt][nb][0] = sc[mt][nb][1] = sc[mt][nb][2] = sc[mt][nb][3] = 0.f;
                if (MIX) sc2[mt][nb][0] = sc2[mt][nb][1] = sc2[mt][nb][2] = sc2[mt][nb][3] = 0.f;
            }
        // ---- S^T = K Q^T
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
            const int row = mt * 16 + (mi & 1) * 8 + ri;
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
                const int c = ks * 2 + (mi >> 1);
                const uint32_t off = (c >> 3) * C::HALF_BYTES + swz128(row, c & 7);
                uint32_t af[4];
                ldsm_x4(kb + off, af[0], af[1], af[2], af[3]);
#pragma unroll
                for (int nb = 0; nb < NB; ++nb) mma_bf16(sc[mt][nb], af, qb[ks][nb][0], qb[ks][nb][1]);
                if (MIX) {
                    ldsm_x4(kb + 2 * C::TILE_BYTES + off, af[0], af[1], af[2], af[3]);
#pragma unroll
                    for (int nb = 0; nb < NB; ++nb) mma_bf16(sc2[mt][nb], af, qb[ks][nb][0], qb[ks][nb][1]);
                }
            }
        }
        // ---- scale, mask the ragged tail, online softmax per head, P^T by movmatrix
        uint32_t pb[MT][NB][2];
        uint32_t pb2[MIX ? MT : 1][NB][2];
        const bool tail = (t + 1) * TT > tlen;       // only the last tile holds tokens past the sequence
        const int lim = tlen - t * TT - (lane >> 2);  // rows r of this lane are valid iff r < lim
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) {
            float mx0 = NEG_INF, mx1 = NEG_INF;
#pragma unroll
            for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    // raw (unscaled) scores: every operation written out, so every compiled
                    // copy of this loop gives the same bits
                    if (MIX) sc[mt][nb][i] = fmaf(w, sc[mt][nb][i], __fmul_rn(w1, sc2[mt][nb][i]));
            if (tail) {
#pragma unroll
                for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        if (mt * 16 + (i >> 1) * 8 >= lim) sc[mt][nb][i] = NEG_INF;
            }
            if (srow != nullptr) {
                // keep the scores of the tile's valid tokens for the attention statistics
                const int h0 = nb * 8 + 2 * (lane & 3);
#pragma unroll
                for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int h = h0 + (i & 1);
                        const int r = mt * 16 + (i >> 1) * 8;
                        if (h < g && r < lim) srow[static_cast<size_t>(h) * a.T + t * TT + (lane >> 2) + r] = __fmul_rn(sc[mt][nb][i], a.scale_log2);
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
            const float mn0 = fmaxf(mrow[nb][0], mx0);
            const float mn1 = fmaxf(mrow[nb][1], mx1);
            const float ref0 = mn0 == NEG_INF ? 0.f : mn0;
            const float ref1 = mn1 == NEG_INF ? 0.f : mn1;
            const float cr0 = ex2_approx(mrow[nb][0] - ref0);
            const float cr1 = ex2_approx(mrow[nb][1] - ref1);
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
            for (int dt = 0; dt < D / 16; ++dt) {
                o[dt][nb][0] *= cr0; o[dt][nb][2] *= cr0;
                o[dt][nb][1] *= cr1; o[dt][nb][3] *= cr1;
            }
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                const float x0 = fmaf(sc[mt][nb][0], a.scale_log2, -ref0);
                const float x1 = fmaf(sc[mt][nb][1], a.scale_log2, -ref1);
                const float x2 = fmaf(sc[mt][nb][2], a.scale_log2, -ref0);
                const float x3 = fmaf(sc[mt][nb][3], a.scale_log2, -ref1);
                const float p0 = ex2_approx(x0);
                const float p1 = ex2_approx(x1);
                const float p2 = ex2_approx(x2);
                const float p3 = ex2_approx(x3);
                lxrow[nb][0] += p0 + p2;
                lxrow[nb][1] += p1 + p3;
                if (want_z) {
                    // p (ref - s); a masked token (x = -inf, p = 0) adds 0
                    zrow[nb][0] = fmaf(p0, -fmaxf(x0, -3.0e38f), fmaf(p2, -fmaxf(x2, -3.0e38f), zrow[nb][0]));
                    zrow[nb][1] = fmaf(p1, -fmaxf(x1, -3.0e38f), fmaf(p3, -fmaxf(x3, -3.0e38f), zrow[nb][1]));
                }
                if (!MIX) {
                    const uint32_t lo = pack_bf16(p0, p1), hi = pack_bf16(p2, p3);
                    lrow[nb][0] += bf16_lo(lo) + bf16_lo(hi);
                    lrow[nb][1] += bf16_hi(lo) + bf16_hi(hi);
                    pb[mt][nb][0] = movmatrix_t(lo);
                    pb[mt][nb][1] = movmatrix_t(hi);
                } else {
                    const uint32_t lo = pack_bf16(w * p0, w * p1), hi = pack_bf16(w * p2, w * p3);
                    const uint32_t lo2 = pack_bf16(w1 * p0, w1 * p1), hi2 = pack_bf16(w1 * p2, w1 * p3);
                    lrow[nb][0] += (bf16_lo(lo) + bf16_lo(hi)) + (bf16_lo(lo2) + bf16_lo(hi2));
                    lrow[nb][1] += (bf16_hi(lo) + bf16_hi(hi)) + (bf16_hi(lo2) + bf16_hi(hi2));
                    pb[mt][nb][0] = movmatrix_t(lo);
                    pb[mt][nb][1] = movmatrix_t(hi);
                    pb2[mt][nb][0] = movmatrix_t(lo2);
                    pb2[mt][nb][1] = movmatrix_t(hi2);
                }
            }
        }
        // ---- O^T += V^T P^T
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
            const int row = mt * 16 + (mi >> 1) * 8 + ri;
#pragma unroll
            for (int dt = 0; dt < D / 16; ++dt) {
                const int c = dt * 2 + (mi & 1);
                const uint32_t off = (c >> 3) * C::HALF_BYTES + swz128(row, c & 7);
                uint32_t af[4];
                ldsm_x4_t(vb + off, af[0], af[1], af[2], af[3]);
#pragma unroll
                for (int nb = 0; nb < NB; ++nb) mma_bf16(o[dt][nb], af, pb[mt][nb][0], pb[mt][nb][1]);
                if (MIX) {
                    ldsm_x4_t(vb + 2 * C::TILE_BYTES + off, af[0], af[1], af[2], af[3]);
#pragma unroll
                    for (int nb = 0; nb < NB; ++nb) mma_bf16(o[dt][nb], af, pb2[mt][nb][0], pb2[mt][nb][1]);
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

    // ---- merge the NW warps per unit (reusing the ring; every copy issued has been consumed)
    __syncthreads();
    (void)t;
    float* comb_o = reinterpret_cast<float*>(smem);   // [NW][16][D]
    float* comb_ml = comb_o + NW * 16 * D;            // [NW][64]: m[16], l[16], lx[16], z[16]
    float* fin_m = comb_ml + NW * 64;                 // [16]
    float* fin_l = fin_m + 16;                        // [16]
    float* fin_lx = fin_l + 16;                       // [16]
    float* fin_z = fin_lx + 16;                       // [16]
    float* fin_o = fin_z + 16;                        // [16][D]
    float* scratch = fin_o + 16 * D;                  // merge scratch
    if (cur_u >= 0) store_state(comb_o + warp * 16 * D, comb_ml + warp * 64);
    if (lane == 0) {
        fin_unit[warp] = cur_u;
        sav_unit[warp] = saved_u;
    }
    __syncthreads();
    const float* save_o = save;
    const float* save_ml = save + NW * 16 * D;
    // every CTA whose range meets a unit takes part in its merge, also with no tokens of it
    for (int uu = u_first; uu <= u_last && cap_span > 0; ++uu) {
        const int u = uu;
        // the warps' contributions to unit u: final states, and states saved at a unit switch;
        // one weight 2^(m_w - M) per (warp, head), so the vector combine is FMAs only
        __shared__ float fac_f[NW][16], fac_s[NW][16];
        if (threadIdx.x < g) {
            const int h = threadIdx.x;
            float M = NEG_INF;
            for (int ww = 0; ww < NW; ++ww) {
                if (fin_unit[ww] == u) M = fmaxf(M, comb_ml[ww * 64 + h]);
                if (STRADDLE && sav_unit[ww] == u) M = fmaxf(M, save_ml[ww * 64 + h]);
            }
            // a warp without a state for u left its slots as they were (ring data, or an
            // earlier kernel's shared memory, NaN included): never read them, not even as 0 * x
            float L = 0.f, LX = 0.f, Z = 0.f;
            for (int ww = 0; ww < NW; ++ww) {
                float ff = 0.f;
                if (fin_unit[ww] == u) {
                    const float* st = comb_ml + ww * 64;
                    const float mf = st[h];
                    if (mf != NEG_INF) {
                        ff = ex2_approx(mf - M);
                        L = fmaf(ff, st[16 + h], L);
                        LX = fmaf(ff, st[32 + h], LX);
                        Z += merged_z(ff, mf, M, st[32 + h], st[48 + h]);
                    }
                }
                fac_f[ww][h] = ff;
                if (STRADDLE) {
                    float fs = 0.f;
                    if (sav_unit[ww] == u) {
                        const float* st = save_ml + ww * 64;
                        const float ms = st[h];
                        if (ms != NEG_INF) {
                            fs = ex2_approx(ms - M);
                            L = fmaf(fs, st[16 + h], L);
                            LX = fmaf(fs, st[32 + h], LX);
                            Z += merged_z(fs, ms, M, st[32 + h], st[48 + h]);
                        }
                    }
                    fac_s[ww][h] = fs;
                }
            }
            fin_m[h] = M;
            fin_l[h] = L;
            fin_lx[h] = LX;
            fin_z[h] = Z;
        }
        __syncthreads();
        for (int idx = threadIdx.x; idx < g * D; idx += blockDim.x) {
            const int h = idx / D;
            const int e = idx % D;
            float acc = 0.f;
#pragma unroll
            for (int ww = 0; ww < NW; ++ww) {
                // a warp without a state for u left whatever its slot held: skip it, never 0 * x
                const float ff = fac_f[ww][h];
                if (ff != 0.f) acc = fmaf(ff, comb_o[(ww * 16 + h) * D + e], acc);
                if (STRADDLE) {
                    const float fs = fac_s[ww][h];
                    if (fs != 0.f) acc = fmaf(fs, save_o[(ww * 16 + h) * D + e], acc);
                }
            }
            fin_o[idx] = acc;
        }
        __syncthreads();
        // partials of unit u: one per CTA whose range meets it, CTAs c_first .. c_last
        const int c_first = static_cast<int>((static_cast<long long>(u) * G) / a.units);
        const int c_last = static_cast<int>(((static_cast<long long>(u + 1) * a.n_t - 1) * G) / W);
        const EmitPlain emit{a, D, static_cast<size_t>(u / a.Hkv) * a.Hq + static_cast<size_t>(u % a.Hkv) * g};
        finish_unit(a, D, u, cta - c_first, c_last - c_first + 1, static_cast<long long>(u) + c_first, fin_m, fin_l,
                    fin_lx, fin_z, fin_o, scratch, smem + C::MERGE_STAGE_OFF,
                    C::BODY > C::MERGE_STAGE_OFF ? C::BODY - C::MERGE_STAGE_OFF : 0, emit);
        __syncthreads();
    }
}

template <int D, bool MIX, int TT, int NSW, int NW, int NH, bool STRADDLE, bool ENT>
cudaError_t launch_ent(const CUtensorMap& tmK, const CUtensorMap& tmV, const DecodeArgs& a, cudaStream_t st) {
    using C = DecodeCfg<D, MIX, TT, NSW, NW>;
    auto kern = decode_bf16_kernel<D, MIX, TT, NSW, NW, NH, STRADDLE, ENT>;
    constexpr int smem = STRADDLE ? C::SMEM : C::SMEM_ALIGNED;
    static std::atomic<unsigned long long> attr_done{0};
    cudaError_t e = once_per_device(attr_done, [&] {
        return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    });
    if (e != cudaSuccess) return e;
    return launch_kernel(kern, dim3(a.splits), dim3(NW * 32), smem, st, a.pdl != 0, tmK, tmV, a);
}

template <int D, bool MIX, int TT, int NSW, int NW, int NH, bool STRADDLE>
cudaError_t launch_nh(const CUtensorMap& tmK, const CUtensorMap& tmV, const DecodeArgs& a, cudaStream_t st) {
    return a.entropy != nullptr ? launch_ent<D, MIX, TT, NSW, NW, NH, STRADDLE, true>(tmK, tmV, a, st)
                                : launch_ent<D, MIX, TT, NSW, NW, NH, STRADDLE, false>(tmK, tmV, a, st);
}

template <int D, bool MIX, int TT, int NSW, int NW>
cudaError_t launch_one(const CUtensorMap& tmK, const CUtensorMap& tmV, const DecodeArgs& a, cudaStream_t st) {
    // with a whole number m of CTAs per unit, CTA u*m starts exactly at unit u's first
    // tile (ceil(u*m*W/G) = u*n_t), so no range crosses a unit boundary
    const bool aligned = a.splits % a.units == 0;
    if (aligned)
        return a.g <= 8 ? launch_nh<D, MIX, TT, NSW, NW, 8, false>(tmK, tmV, a, st)
                        : launch_nh<D, MIX, TT, NSW, NW, 16, false>(tmK, tmV, a, st);
    return a.g <= 8 ? launch_nh<D, MIX, TT, NSW, NW, 8, true>(tmK, tmV, a, st)
                    : launch_nh<D, MIX, TT, NSW, NW, 16, true>(tmK, tmV, a, st);
}

template <int D, bool MIX, int TT, int NSW, int NW>
int occupancy() {
    using C = DecodeCfg<D, MIX, TT, NSW, NW>;
    // the default grid is unit-aligned, so its CTAs carry no straddle save area
    auto kern = decode_bf16_kernel<D, MIX, TT, NSW, NW, 8, false, false>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_ALIGNED);
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, NW * 32, C::SMEM_ALIGNED) != cudaSuccess) return 1;
    return n > 0 ? n : 1;
}

template <int D, bool MIX, int TT, int NSW, int NW>
TileShape shape_of() {
    return {TT, NSW, DecodeCfg<D, MIX, TT, NSW, NW>::SMEM};
}

// tile shapes: tokens per tile (TT), stages per warp (NSW) and warps per CTA (NW) for each variant
#ifndef KVS_TT_64S
#define KVS_TT_64S 64
#endif
#ifndef KVS_NSW_64S
#define KVS_NSW_64S 3
#endif
#ifndef KVS_TT_64M
#define KVS_TT_64M 32
#endif
#ifndef KVS_NSW_64M
#define KVS_NSW_64M 2
#endif
#ifndef KVS_TT_128S
#define KVS_TT_128S 32
#endif
#ifndef KVS_NSW_128S
#define KVS_NSW_128S 2
#endif
#ifndef KVS_TT_128M
#define KVS_TT_128M 16
#endif
#ifndef KVS_NSW_128M
#define KVS_NSW_128M 2
#endif
#ifndef KVS_NW_64S
#define KVS_NW_64S 4
#endif
#ifndef KVS_NW_64M
#define KVS_NW_64M 4
#endif
#ifndef KVS_NW_128S
#define KVS_NW_128S 4
#endif
#ifndef KVS_NW_128M
#define KVS_NW_128M 4
#endif
#define KVS_SHAPE_64_SINGLE KVS_TT_64S, KVS_NSW_64S, KVS_NW_64S
#define KVS_SHAPE_64_MIX KVS_TT_64M, KVS_NSW_64M, KVS_NW_64M
#define KVS_SHAPE_128_SINGLE KVS_TT_128S, KVS_NSW_128S, KVS_NW_128S
#define KVS_SHAPE_128_MIX KVS_TT_128M, KVS_NSW_128M, KVS_NW_128M

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

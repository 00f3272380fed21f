// Causal prefill over a shared cache on the 5th-generation tensor cores (tcgen05 + TMEM).
//
// One CTA = two 128-row query tiles of one head (rows q0 .. q0+255), sharing every
// K/V tile it streams. TMEM holds both tiles' scores S0, S1 and outputs O0, O1.
// Warp roles, by warpgroup (each moves its register budget with setmaxnreg first):
//   warpgroups 0, 1  softmax of query tile 0 / 1, one thread per query row: the
//                 whole S row from TMEM in one round trip, causal mask on diagonal
//                 tiles only, online softmax in base 2 with a lazy max (O rescaled
//                 in TMEM only when a row max grows by more than 2^8), P as bf16
//                 written back over the row's S columns; epilogue O / l -> bf16
//                 through shared memory and a TMA store
//   last warpgroup  one warp TMA producer (Q0, Q1 once, then K/V tiles: a 2-stage
//                 ring; two-source layers: a 3-stage ring for the first source and a
//                 2-stage ring for the second, which the mixers free as soon as they
//                 have read it), one warp TMEM owner and MMA issuer (one thread),
//                 in the order S0_j, S1_j, PV0_j, S0_{j+1}, PV1_j, S1_{j+1}, ... so
//                 that the tensor core computes one tile's product while the other
//                 tile's softmax runs:  S = Q K^T  (A, B from shared memory)
//                                       O += P V  (A = P straight from TMEM, B = V from shared)
//   warpgroup 2 (two-source layers only) mixers: K~ = w K1 + (1-w) K2 and the
//                 same for V, in fp32, rounded once to bf16, written in place over
//                 the first source's tile, so the MMA reads the mixed operand and
//                 the mixed K/V never reach HBM ("DepthGraft: Structural
//                 Regularization through Hierarchical Cross-Layer KV
//                 Reconstruction", Abstract: deep-layer KV rebuilt from a
//                 shallow/middle source pair; the convex mix is this library's reading).
// Every mbarrier wait is bounded; a wait that runs out records KVS_ETIMEOUT,
// makes the other waits of the CTA give up, and the CTA still frees its TMEM.
#include <type_traits>

#include "tc_sm100.cuh"

namespace kvs {
namespace {

constexpr int BM = 128;   // rows per query tile
constexpr int NQ = 2;     // query tiles per CTA
constexpr int NS_MAX = 3;   // K/V stages of the first-source ring, at most
#ifndef KVS_PF_MIXERS
#define KVS_PF_MIXERS 128
#endif

template <int D, bool MIX>
struct PfCfg {
    static constexpr int BN = MIX ? 64 : 128;
    static constexpr int HALVES = D / 64;
    static constexpr int NSRC = MIX ? 2 : 1;
    static constexpr int Q_BYTES = BM * D * 2;     // one query tile
    static constexpr int TILE = BN * D * 2;        // one K or V tile
    static constexpr int HALF_T = BN * 128;        // one 64-column half of it
    // ring A: [K | V] (the first source, mixed in place on two-source layers), NS stages;
    // ring B (two-source layers): [K2 | V2], NSB stages, freed by the mixers as soon as
    // they have read it, so the copies of the second source run ahead of the MMA
    static constexpr int NS = MIX ? 3 : 2;
    static constexpr int NSB = MIX ? 2 : 0;
    static constexpr int STAGE = 2 * TILE;
    static constexpr int SMEM = NQ * Q_BYTES + (NS + NSB) * STAGE + 1024;
    static_assert(NS <= NS_MAX, "ring A depth");
    static_assert(SMEM <= 227 * 1024, "shared memory");
    static constexpr uint32_t TMEM_COLS = 512;     // S0 | S1 | O0 | O1
    // warpgroups: 0, 1 softmax; MIX: 2 mixers, 3 TMA + MMA (+2 idle); single: 2 TMA + MMA (+2 idle)
    // (one mixer warpgroup measured faster than two: mix layers 619 -> 629 TFLOP/s, the
    // mixers still run ahead, and the softmax threads get 184 registers instead of 152)
    static constexpr int MIXERS = KVS_PF_MIXERS;            // mixer threads (whole warpgroups)
    static constexpr int THREADS = MIX ? 384 + MIXERS : 384;
    static constexpr int W_MIX = 8;
    static constexpr int W_TMA = MIX ? 8 + MIXERS / 32 : 8, W_MMA = W_TMA + 1;
    // per-thread registers after the split (setmaxnreg): the softmax threads hold a whole
    // S row; the sum over the block must not exceed what the block was launched with
    static constexpr int LAUNCH_REGS = MIX ? (MIXERS == 128 ? 128 : 96) : 168;
    static constexpr int REG_SOFTMAX = MIX ? (MIXERS == 128 ? 184 : 152) : 216;
    static constexpr int REG_MIXER = 56;
    static constexpr int REG_CTRL = 64;
    static constexpr int REG_SUM = 2 * 128 * REG_SOFTMAX + (MIX ? MIXERS * REG_MIXER : 0) + 128 * REG_CTRL;
    static_assert(REG_SUM <= THREADS * LAUNCH_REGS, "register split exceeds the launch allocation");
    static_assert(2 * BN + 2 * D <= 512, "TMEM budget");
};

struct Sync {
    uint64_t q_full;
    uint64_t kv_full[NS_MAX];
    uint64_t kv_ready[NS_MAX];
    uint64_t kv_empty[NS_MAX];
    uint64_t kvb_full[2];
    uint64_t kvb_empty[2];
    uint64_t s_full[NQ];
    uint64_t p_full[NQ];
    uint64_t o_full;
    uint32_t tmem_base;
    volatile int abort;
};

// bounded wait that also gives up at once when another thread of the CTA already timed out
__device__ __forceinline__ void wait_cta(Sync& sy, uint64_t* bar, unsigned parity, long long limit, unsigned* err) {
    if (mbar_try_wait(bar, parity)) return;
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity)) {
        if (sy.abort) return;
        if (clock64() - t0 > limit) {
            atomicOr(err, ERR_TIMEOUT);
            sy.abort = 1;
            return;
        }
    }
}

// 2^x on the FMA pipe, for a share of the softmax exponentials so that the MUFU unit
// (16 results per clock per SM, the same rate as the tensor core's bf16 products need
// at BN = D = 128) is not the bottleneck. Range reduction: x = j + f with j = rint(x)
// taken by the 1.5 * 2^23 rounding shift and f in [-1/2, 1/2]; 2^f from a degree-3
// polynomial whose coefficients are a relative-error minimax fit on that interval
// (iteratively reweighted least squares; largest relative error 7.6e-5, well below the
// bf16 rounding of P); 2^j added to the exponent field. x >= -125 keeps the result a
// normal float; inputs below that return 2^-125 instead of a smaller value.
// KVS_PF_EMU_PAIRS (pairs of every 16 that take this path) is 0 by default: on the
// d = 128 causal prefill every share from 3/16 to 9/16 measured slower, the issue
// slots and FMA/ALU pipes rather than MUFU bounding this kernel's softmax.
#ifndef KVS_PF_EMU_PAIRS
#define KVS_PF_EMU_PAIRS 0
#endif
constexpr int EMU_PAIRS = KVS_PF_EMU_PAIRS;
constexpr float EXP2_C0 = 0.9999281764030457f;
constexpr float EXP2_C1 = 0.6932609677314758f;
constexpr float EXP2_C2 = 0.24260950088500977f;
constexpr float EXP2_C3 = 0.05517100542783737f;
__device__ __forceinline__ float exp2_fma(float x) {
    x = fmaxf(x, -125.f);
    const float t = x + 12582912.f;
    const float f = x - (t - 12582912.f);
    const float p = fmaf(fmaf(fmaf(EXP2_C3, f, EXP2_C2), f, EXP2_C1), f, EXP2_C0);
    return __int_as_float(__float_as_int(p) + (__float_as_int(t) << 23));
}

// number of K/V tiles a query tile whose first row is qbase needs
__device__ __forceinline__ int kv_tiles(int qbase, int S, int BN) {
    if (qbase >= S) return 0;
    return (min(qbase + BM, S) - 1) / BN + 1;
}

template <int D, bool MIX>
__global__ void __launch_bounds__(PfCfg<D, MIX>::THREADS, 1)
prefill_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
               const PrefillArgs a) {
    using C = PfCfg<D, MIX>;
    constexpr int BN = C::BN;
    extern __shared__ uint8_t smem_dyn[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
    uint8_t* sQ = smem;                                  // [NQ][HALVES][BM][64]
    uint8_t* sKV = smem + NQ * C::Q_BYTES;               // ring A [NS][K | V]
    uint8_t* sKV2 = sKV + C::NS * C::STAGE;              // ring B [NSB][K2 | V2] (two-source layers)
    constexpr int NS = C::NS;
    constexpr int NSB = C::NSB;
    __shared__ __align__(8) Sync sy;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int n_ct = (a.S + NQ * BM - 1) / (NQ * BM);
    const int ct = n_ct - 1 - static_cast<int>(blockIdx.z);    // heaviest query tiles first
    const int h = blockIdx.x;
    const int b = blockIdx.y;
    const int jkv = h / a.g;
    const int q0 = ct * NQ * BM;
    int nq[NQ];
#pragma unroll
    for (int i = 0; i < NQ; ++i) nq[i] = kv_tiles(q0 + i * BM, a.S, BN);
    const int n_kv = nq[NQ - 1] > nq[0] ? nq[NQ - 1] : nq[0];

    if (threadIdx.x == 0) {
        prefetch_tmap(&tmQ);
        prefetch_tmap(&tmK);
        prefetch_tmap(&tmV);
        prefetch_tmap(&tmO);
        mbar_init(&sy.q_full, 1);
        for (int s = 0; s < NSB; ++s) {
            mbar_init(&sy.kvb_full[s], 1);
            mbar_init(&sy.kvb_empty[s], C::MIXERS);
        }
        for (int s = 0; s < NS; ++s) {
            mbar_init(&sy.kv_full[s], 1);
            mbar_init(&sy.kv_ready[s], C::MIXERS);
            mbar_init(&sy.kv_empty[s], 1);
        }
        for (int i = 0; i < NQ; ++i) {
            mbar_init(&sy.s_full[i], 1);
            mbar_init(&sy.p_full[i], 128);
        }
        mbar_init(&sy.o_full, 1);
        sy.abort = 0;
        mbar_init_fence();
    }
    if (warp == C::W_MMA) {
        tc::alloc(&sy.tmem_base, C::TMEM_COLS);
        tc::relinquish();
    }
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = sy.tmem_base;
    // TMEM columns: S_i at i * BN, O_i at 2 * BN + i * D
    auto tS = [&](int i) { return tmem + static_cast<uint32_t>(i * BN); };
    auto tO = [&](int i) { return tmem + static_cast<uint32_t>(2 * BN + i * D); };

    // Warpgroup roles. Each branch first moves its per-thread register budget
    // (setmaxnreg, executed by all four warps of the warpgroup), so the softmax threads
    // can hold a whole S row; the budgets add up to at most the launch allocation.
    const int wg = warp >> 2;
    if (wg < NQ) {
        tc::reg_inc<C::REG_SOFTMAX>();
        // ------------------------------------------------------------ softmax, one warpgroup per query tile
        const int qi = warp >> 2;
        const int wq = warp & 3;                         // lane quadrant of TMEM this warp may access
        const int row = wq * 32 + lane;
        const int qpos = q0 + qi * BM + row;
        const uint32_t lane_base = static_cast<uint32_t>(wq * 32) << 16;
        const uint32_t sS = tS(qi) + lane_base;
        const uint32_t sO = tO(qi) + lane_base;
        const int n_my = nq[qi];
        const int diag0 = (q0 + qi * BM) / BN;
        float m_used = NEG_INF;
        float l = 0.f;
        // one K/V tile of this row; MASKED (diagonal tiles only) zeroes the columns past qpos
        auto step = [&](auto mask_tag, int j) {
            constexpr bool MASKED = decltype(mask_tag)::value;
            const int lim = qpos - j * BN;               // column c is visible iff c <= lim
            // the whole row of S in one TMEM round trip
            uint32_t r[BN / 32][32];
#pragma unroll
            for (int c = 0; c < BN / 32; ++c) tc::ld32(sS + c * 32, r[c]);
            tc::wait_ld();
            if (MASKED) {
#pragma unroll
                for (int c = 0; c < BN / 32; ++c)
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        if (c * 32 + i > lim) r[c][i] = __float_as_uint(NEG_INF);
            }
            // row max of the raw (unscaled) scores over four independent chains
            float mx[4] = {NEG_INF, NEG_INF, NEG_INF, NEG_INF};
#pragma unroll
            for (int c = 0; c < BN / 32; ++c)
#pragma unroll
                for (int i = 0; i < 32; i += 2)
                    mx[(i >> 1) & 3] = fmaxf(mx[(i >> 1) & 3], fmaxf(__uint_as_float(r[c][i]), __uint_as_float(r[c][i + 1])));
            const float mt = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * a.scale_log2;
            // lazy max: rescale O only when the row max grew by more than 2^8; the TMEM
            // load/store is warp-collective, so the warp rescales if any row needs it
            float corr = 1.f;
            if (m_used == NEG_INF) {
                m_used = mt;
            } else if (mt > m_used + 8.f) {
                corr = tc::ex2(m_used - mt);
                m_used = mt;
            }
            if (__any_sync(0xffffffffu, corr != 1.f)) {
                l *= corr;
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t o32[32];
                    tc::ld32(sO + c * 32, o32);
                    tc::wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) o32[i] = __float_as_uint(__uint_as_float(o32[i]) * corr);
                    tc::st32(sO + c * 32, o32);
                }
            }
            // P = 2^(s * scale - m) as bf16, packed two per column over the row's first BN/2
            // S columns (every S value is in registers already); masked columns hold -inf,
            // whose exponential is 0. EMU_PAIRS of every 16 pairs take the FMA-pipe exponential.
            const float nm = -m_used;
            float ls[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int c = 0; c < BN / 32; ++c) {
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float x0 = fmaf(__uint_as_float(r[c][2 * i]), a.scale_log2, nm);
                    const float x1 = fmaf(__uint_as_float(r[c][2 * i + 1]), a.scale_log2, nm);
                    float p0, p1;
                    if (i < EMU_PAIRS) {
                        p0 = exp2_fma(x0);
                        p1 = exp2_fma(x1);
                        if (MASKED && c * 32 + 2 * i > lim) p0 = 0.f;
                        if (MASKED && c * 32 + 2 * i + 1 > lim) p1 = 0.f;
                    } else {
                        p0 = tc::ex2(x0);
                        p1 = tc::ex2(x1);
                    }
                    ls[i & 3] += p0 + p1;
                    pk[i] = pack_bf16(p0, p1);
                }
                tc::st16(sS + c * 16, pk);
            }
            l += (ls[0] + ls[1]) + (ls[2] + ls[3]);
        };
        for (int j = 0; j < n_my; ++j) {
            wait_cta(sy, &sy.s_full[qi], j & 1, a.wait_limit, a.err);
            tc::fence_after();
            if (j >= diag0)
                step(std::true_type{}, j);
            else
                step(std::false_type{}, j);
            tc::wait_st();
            tc::fence_before();
            mbar_arrive(&sy.p_full[qi]);
        }
        // ------------------------------------------------------------ epilogue through shared memory
        if (n_my > 0) {
            wait_cta(sy, &sy.o_full, 0, a.wait_limit, a.err);
            tc::fence_after();
            const float inv = 1.f / l;
            uint8_t* so = sQ + qi * C::Q_BYTES;          // this tile's Q buffer is free now
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t r[32];
                tc::ld32(sO + c * 32, r);
                tc::wait_ld();
#pragma unroll
                for (int i = 0; i < 32; i += 8) {
                    uint4 v;
                    v.x = pack_bf16(__uint_as_float(r[i]) * inv, __uint_as_float(r[i + 1]) * inv);
                    v.y = pack_bf16(__uint_as_float(r[i + 2]) * inv, __uint_as_float(r[i + 3]) * inv);
                    v.z = pack_bf16(__uint_as_float(r[i + 4]) * inv, __uint_as_float(r[i + 5]) * inv);
                    v.w = pack_bf16(__uint_as_float(r[i + 6]) * inv, __uint_as_float(r[i + 7]) * inv);
                    const int chunk = (c * 32 + i) >> 3;          // 16-B chunk of the row
                    *reinterpret_cast<uint4*>(so + (chunk >> 3) * (BM * 128) + swz128(row, chunk & 7)) = v;
                }
            }
            if (a.lse != nullptr && qpos < a.S)
                a.lse[static_cast<size_t>(b * a.Hq + h) * a.S + qpos] = (m_used + log2f(l)) * LN2_F;
            fence_proxy_async();
            named_sync(1 + qi, 128);
            if (row == 0) {
#pragma unroll
                for (int hh = 0; hh < C::HALVES; ++hh)
                    tma_store_3d(&tmO, so + hh * BM * 128, hh * 64, q0 + qi * BM, b * a.Hq + h);
                bulk_commit();
                bulk_wait_read0();
            }
        }
    } else if (MIX && wg >= C::W_MIX / 4 && wg < C::W_MIX / 4 + C::MIXERS / 128) {
        tc::reg_dec<C::REG_MIXER>();
        // ------------------------------------------------------------ mixers (two-source layers)
        const int t = threadIdx.x - 32 * C::W_MIX;
        const float w = a.w[jkv];
        const float w1 = 1.f - w;
        for (int j = 0; j < n_kv; ++j) {
            const int s = j % NS;
            const int sb = j % (NSB > 0 ? NSB : 1);
            wait_cta(sy, &sy.kv_full[s], (j / NS) & 1, a.wait_limit, a.err);
            wait_cta(sy, &sy.kvb_full[sb], (j / (NSB > 0 ? NSB : 1)) & 1, a.wait_limit, a.err);
            uint4* dst = reinterpret_cast<uint4*>(sKV + s * C::STAGE);                    // K1 | V1
            const uint4* src = reinterpret_cast<const uint4*>(sKV2 + sb * C::STAGE);     // K2 | V2
            // 16-B chunks of K1|V1 and K2|V2, four per thread in flight before any is mixed
            constexpr int NIT = 2 * C::TILE / 16 / C::MIXERS;
            static_assert(NIT % 4 == 0, "mixer batches");
#pragma unroll
            for (int it0 = 0; it0 < NIT; it0 += 4) {
                uint4 x[4], y[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    x[u] = dst[t + (it0 + u) * C::MIXERS];
                    y[u] = src[t + (it0 + u) * C::MIXERS];
                }
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    uint4 r;
                    r.x = pack_bf16(w * bf16_lo(x[u].x) + w1 * bf16_lo(y[u].x), w * bf16_hi(x[u].x) + w1 * bf16_hi(y[u].x));
                    r.y = pack_bf16(w * bf16_lo(x[u].y) + w1 * bf16_lo(y[u].y), w * bf16_hi(x[u].y) + w1 * bf16_hi(y[u].y));
                    r.z = pack_bf16(w * bf16_lo(x[u].z) + w1 * bf16_lo(y[u].z), w * bf16_hi(x[u].z) + w1 * bf16_hi(y[u].z));
                    r.w = pack_bf16(w * bf16_lo(x[u].w) + w1 * bf16_lo(y[u].w), w * bf16_hi(x[u].w) + w1 * bf16_hi(y[u].w));
                    dst[t + (it0 + u) * C::MIXERS] = r;
                }
            }
            fence_proxy_async();
            mbar_arrive(&sy.kv_ready[s]);
            mbar_arrive(&sy.kvb_empty[sb]);   // ring B slot read: the next copy may land
        }
    } else {
        tc::reg_dec<C::REG_CTRL>();
        if (warp == C::W_TMA) {
            // ------------------------------------------------------------ TMA producer
            if (lane == 0) {
                mbar_arrive_expect_tx(&sy.q_full, NQ * C::Q_BYTES);
#pragma unroll
                for (int i = 0; i < NQ; ++i)
#pragma unroll
                    for (int hh = 0; hh < C::HALVES; ++hh)
                        tma_load_3d(sQ + i * C::Q_BYTES + hh * BM * 128, &tmQ, hh * 64, q0 + i * BM, b * a.Hq + h,
                                    &sy.q_full);
                const int BH = a.B * a.Hkv;
                const int r0 = a.src0 * BH + b * a.Hkv + jkv;
                const int r1 = a.src1 * BH + b * a.Hkv + jkv;
                for (int j = 0; j < n_kv; ++j) {
                    const int s = j % NS;
                    if (MIX) {
                        // the second source first: its ring is freed by the mixers, not the MMA
                        const int sb = j % NSB;
                        if (j >= NSB) wait_cta(sy, &sy.kvb_empty[sb], ((j / NSB) - 1) & 1, a.wait_limit, a.err);
                        if (sy.abort) break;
                        uint8_t* st2 = sKV2 + sb * C::STAGE;
                        mbar_arrive_expect_tx(&sy.kvb_full[sb], C::STAGE);
#pragma unroll
                        for (int hh = 0; hh < C::HALVES; ++hh) {
                            tma_load_3d(st2 + hh * C::HALF_T, &tmK, hh * 64, j * BN, r1, &sy.kvb_full[sb]);
                            tma_load_3d(st2 + C::TILE + hh * C::HALF_T, &tmV, hh * 64, j * BN, r1, &sy.kvb_full[sb]);
                        }
                    }
                    if (j >= NS) wait_cta(sy, &sy.kv_empty[s], ((j / NS) - 1) & 1, a.wait_limit, a.err);
                    if (sy.abort) break;
                    uint8_t* st = sKV + s * C::STAGE;
                    mbar_arrive_expect_tx(&sy.kv_full[s], C::STAGE);
#pragma unroll
                    for (int hh = 0; hh < C::HALVES; ++hh) {
                        tma_load_3d(st + hh * C::HALF_T, &tmK, hh * 64, j * BN, r0, &sy.kv_full[s]);
                        tma_load_3d(st + C::TILE + hh * C::HALF_T, &tmV, hh * 64, j * BN, r0, &sy.kv_full[s]);
                    }
                }
                if (sy.abort) {
                    // let copies still in flight land before the CTA's shared memory goes away
                    const int first = n_kv > NS ? n_kv - NS : 0;
                    for (int j = first; j < n_kv; ++j) {
                        const long long t0 = clock64();
                        while (!mbar_try_wait(&sy.kv_full[j % NS], (j / NS) & 1) && clock64() - t0 < a.wait_limit) {
                        }
                    }
                    if (MIX) {
                        const int firstb = n_kv > NSB ? n_kv - NSB : 0;
                        for (int j = firstb; j < n_kv; ++j) {
                            const long long t0 = clock64();
                            while (!mbar_try_wait(&sy.kvb_full[j % NSB], (j / NSB) & 1) &&
                                   clock64() - t0 < a.wait_limit) {
                            }
                        }
                    }
                }
            }
        } else if (warp == C::W_MMA) {
            // ------------------------------------------------------------ MMA issuer
            if (lane == 0) {
                constexpr uint32_t idS = tc::idesc_bf16(BM, BN, false, false);
                constexpr uint32_t idO = tc::idesc_bf16(BM, D, false, true);
                // descriptors: one base per operand tile, then the start-address field
                // (address >> 4, in the low bits) advanced by a constant per K step
                auto issue_s = [&](int i, int j) {          // S_i = Q_i K_j^T
                    const uint64_t qd = tc::smem_desc(smem_u32(sQ + i * C::Q_BYTES), 16, 1024, tc::LAYOUT_SW128);
                    const uint64_t kd = tc::smem_desc(smem_u32(sKV + (j % NS) * C::STAGE), 16, 1024, tc::LAYOUT_SW128);
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        // 16 bf16 along K inside the 128-B row, then the next 64-column half
                        const uint32_t off = (kk & 3) * 32;
                        const uint64_t ad = qd + (((kk >> 2) * (BM * 128) + off) >> 4);
                        const uint64_t bd = kd + (((kk >> 2) * C::HALF_T + off) >> 4);
                        tc::mma_ss(tS(i), ad, bd, idS, kk > 0 ? 1u : 0u);
                    }
                    tc::commit(&sy.s_full[i]);
                };
                auto issue_pv = [&](int i, int j) {         // O_i += P_i V_j, P_i read from TMEM
                    wait_cta(sy, &sy.p_full[i], j & 1, a.wait_limit, a.err);
                    tc::fence_after();
                    const uint64_t vd =
                        tc::smem_desc(smem_u32(sKV + (j % NS) * C::STAGE + C::TILE), C::HALF_T, 1024, tc::LAYOUT_SW128);
#pragma unroll
                    for (int kk = 0; kk < BN / 16; ++kk)
                        tc::mma_ts(tO(i), tS(i) + kk * 8, vd + ((kk * 16 * 128) >> 4), idO, (j > 0 || kk > 0) ? 1u : 0u);
                };
                auto wait_kv = [&](int j) {
                    wait_cta(sy, MIX ? &sy.kv_ready[j % NS] : &sy.kv_full[j % NS], (j / NS) & 1, a.wait_limit, a.err);
                    tc::fence_after();
                };
                wait_cta(sy, &sy.q_full, 0, a.wait_limit, a.err);
                wait_kv(0);
                if (nq[0] > 0) issue_s(0, 0);
                if (nq[1] > 0) issue_s(1, 0);
                for (int j = 0; j < n_kv && !sy.abort; ++j) {
                    const bool next = j + 1 < n_kv;
                    if (j < nq[0]) issue_pv(0, j);
                    if (next) wait_kv(j + 1);
                    if (next && j + 1 < nq[0]) issue_s(0, j + 1);
                    if (j < nq[1]) issue_pv(1, j);
                    tc::commit(&sy.kv_empty[j % NS]);
                    if (next && j + 1 < nq[1]) issue_s(1, j + 1);
                }
                tc::commit(&sy.o_full);
            }
        }
    }

    tc::fence_before();
    __syncthreads();
    if (warp == C::W_MMA) {
        tc::fence_after();
        tc::dealloc(tmem, C::TMEM_COLS);
    }
}

template <int D, bool MIX>
cudaError_t launch_one(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& to,
                       const PrefillArgs& a, cudaStream_t st) {
    using C = PfCfg<D, MIX>;
    auto kern = prefill_kernel<D, MIX>;
    static std::atomic<unsigned long long> attr_done{0};
    cudaError_t e = once_per_device(attr_done, [&] {
        cudaError_t r = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
        if (r != cudaSuccess) return r;
        // the register split assumes the block is launched with LAUNCH_REGS per thread;
        // with fewer, the softmax warps' setmaxnreg.inc could never be satisfied
        cudaFuncAttributes fa;
        r = cudaFuncGetAttributes(&fa, kern);
        if (r != cudaSuccess) return r;
        return fa.numRegs * C::THREADS < C::REG_SUM ? cudaErrorInvalidConfiguration : cudaSuccess;
    });
    if (e != cudaSuccess) return e;
    dim3 grid(a.Hq, a.B, (a.S + NQ * BM - 1) / (NQ * BM));
    kern<<<grid, C::THREADS, C::SMEM, st>>>(tq, tk, tv, to, a);
    return cudaGetLastError();
}

}  // namespace

int prefill_kv_tile(int d, bool mix) {
    (void)d;
    return mix ? PfCfg<128, true>::BN : PfCfg<128, false>::BN;
}

cudaError_t launch_prefill(int d, bool mix, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                           const CUtensorMap& to, const PrefillArgs& a, cudaStream_t st) {
    if (d == 64) return mix ? launch_one<64, true>(tq, tk, tv, to, a, st) : launch_one<64, false>(tq, tk, tv, to, a, st);
    return mix ? launch_one<128, true>(tq, tk, tv, to, a, st) : launch_one<128, false>(tq, tk, tv, to, a, st);
}

}  // namespace kvs

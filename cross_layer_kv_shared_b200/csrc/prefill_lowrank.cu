// Causal prefill of a low-rank layer on the 5th-generation tensor cores (tcgen05 + TMEM).
//
// A layer pair shares a low-rank basis and each layer adds a quantised low-rank
// residual at a per-token rank ("DepthWeave-KV: Smarter KV Cache Compression by
// Sharing Across Layers and Adapting Per Token", Core Mechanism; "DepthWeave-KV:
// Token-Adaptive Cross-Layer Residual Factorization for Long-Context KV Cache
// Compression", Detailed Explanation: basis lookup, dequantisation and attention
// projection fused, with little memory traffic). Rebuilding K~, V~ per token would
// cost 2 x 48 x d multiply-adds per token; instead the projections are absorbed,
// exactly in real arithmetic:
//   q'_i  = [B_K q_i | R_K q_i | 0]                      (64 values, the pre-pass below)
//   k'_t  = [C_K[t]  | s_K[t] U_K[t] (first r_t) | 0]    (built per tile in shared memory)
//   v'_t  = [C_V[t]  | s_V[t] U_V[t] (first r_t) | 0]
//   S = Q' K'^T,  O' = P V'  (64 columns, tcgen05),  o_i = O'_i [B_V; R_V] / l_i
// so both contractions run at width 64 instead of d. The kernel follows the
// two-source prefill: one CTA = two 128-row query tiles of one head; warpgroups 0, 1
// run the softmax of one query tile each (one thread per row, P written back into
// TMEM as bf16 and read from there by the PV product) and the epilogue
// o = O' W / l; warpgroup 2 converts each raw tile (coefficients by TMA, int8
// codes by TMA, per-token scales and ranks by plain loads) into the K', V' operands;
// the last warpgroup has the TMA producer and the MMA issuer. Every wait is bounded.
#include <type_traits>

#include "kvs_quant.cuh"
#include "tc_sm100.cuh"

namespace kvs {
namespace {

constexpr int BM = 128;     // rows per query tile
constexpr int NQ = 2;       // query tiles per CTA
// tokens per K/V tile: 128 measured 4 % faster than 64 on the 4K-token DepthWeave
// prefill (half as many S/P handoffs per token; ring depth and registers rebalanced)
#ifndef KVS_LR_PF_BN
#define KVS_LR_PF_BN 128
#endif
constexpr int BN = KVS_LR_PF_BN;
static_assert(BN == 64 || BN == 128, "K/V tile of 64 or 128 tokens");
constexpr int RB = 32;      // basis rank
constexpr int RM = 16;      // residual slots
constexpr int QW = LR_QW;   // operand width: RB + RM padded to one 128-byte swizzle row

template <int D>
struct LrPfCfg {
    static constexpr int Q_BYTES = BM * QW * 2;        // one projected query tile [128][64] bf16
    static constexpr int OP_TILE = BN * QW * 2;        // one K' or V' tile [BN][64] bf16
    static constexpr int NS = BN == 128 ? 2 : 3;       // ring A: [K' | V'] stages (built by the converters)
    static constexpr int STAGE_A = 2 * OP_TILE;
    // ring B: raw tiles [C_K | C_V | U_K | U_V], filled by TMA, freed by the converters
    static constexpr int NSB = BN == 128 ? 2 : 4;
    static constexpr int C_BYTES = BN * RB * 2;        // [BN][32] bf16, unswizzled 64-byte rows
    static constexpr int U_BYTES = BN * RM;            // [BN][16] int8
    static constexpr int STAGE_B = 2 * C_BYTES + 2 * U_BYTES;
    static constexpr int W_BYTES = (RB + RM) * D * 2;  // [B_V; R_V] bf16
    static constexpr int OUT_TILE = BM * D * 2;        // one output tile, 64-column swizzled halves
    static constexpr int OFF_A = NQ * Q_BYTES;
    static constexpr int OFF_B = OFF_A + NS * STAGE_A;
    static constexpr int OFF_W = OFF_B + NSB * STAGE_B;
    static constexpr int OFF_OUT = ((OFF_W + W_BYTES + 1023) / 1024) * 1024;
    static constexpr int SMEM = OFF_OUT + NQ * OUT_TILE + 1024;
    static_assert(OFF_A % 1024 == 0 && OFF_B % 1024 == 0 && STAGE_A % 1024 == 0 && STAGE_B % 128 == 0 &&
                      C_BYTES % 128 == 0 && OFF_W % 16 == 0,
                  "TMA destinations 128-byte aligned, swizzled tiles 1024-byte aligned");
    static_assert(SMEM <= 227 * 1024, "shared memory");
    static constexpr uint32_t TMEM_COLS = BN == 128 ? 512 : 256;   // S0 | S1 | O'0 | O'1
    // converter threads: one warpgroup, each thread a whole token row of K' or V' (two
    // warpgroups that split each row measured 8% slower over the layer: more threads
    // contending for the shared-memory pipes and fewer registers for softmax)
    static constexpr int CONV = 128;
    static constexpr int THREADS = 384 + CONV;
    static constexpr int W_CONV = 8;
    static constexpr int W_TMA = 8 + CONV / 32, W_MMA = W_TMA + 1;
    static constexpr int LAUNCH_REGS = 128;
    // with 128-token tiles each converter thread builds two rows: registers move from
    // the softmax (which then holds at most 64 scores of a row at a time) to the converters
    static constexpr int REG_SOFTMAX = BN == 128 ? 168 : 184;
    static constexpr int REG_CONV = BN == 128 ? 112 : 72;
    static constexpr int REG_CTRL = 64;
    static constexpr int REG_SUM = 2 * 128 * REG_SOFTMAX + CONV * REG_CONV + 128 * REG_CTRL;
    static_assert(REG_SUM <= THREADS * LAUNCH_REGS, "register split exceeds the launch allocation");
};

struct LrSync {
    uint64_t q_full;
    uint64_t w_full;
    uint64_t raw_full[4];
    uint64_t raw_empty[4];
    uint64_t op_ready[3];
    uint64_t op_empty[3];
    uint64_t s_full[NQ];
    uint64_t p_full[NQ];
    uint64_t o_full;
    uint32_t tmem_base;
    volatile int abort;
};

__device__ __forceinline__ void wait_lr(LrSync& sy, uint64_t* bar, unsigned parity, long long limit, unsigned* err) {
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

__device__ __forceinline__ int tiles_for(int qbase, int S) {
    if (qbase >= S) return 0;
    return (min(qbase + BM, S) - 1) / BN + 1;
}

template <int D>
__global__ void __launch_bounds__(LrPfCfg<D>::THREADS, 1)
prefill_lowrank_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmO,
                       const __grid_constant__ CUtensorMap tmCK, const __grid_constant__ CUtensorMap tmCV,
                       const __grid_constant__ CUtensorMap tmUK, const __grid_constant__ CUtensorMap tmUV,
                       const PrefillLrArgs a) {
    using C = LrPfCfg<D>;
    constexpr int NS = C::NS, NSB = C::NSB;
    extern __shared__ uint8_t smem_dyn[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
    uint8_t* sQ = smem;                          // [NQ][128][64] swizzled
    uint8_t* sA = smem + C::OFF_A;               // ring A [NS][K' | V'], each [BN][64] swizzled
    uint8_t* sB = smem + C::OFF_B;               // ring B [NSB][C_K | C_V | U_K | U_V]
    uint8_t* sW = smem + C::OFF_W;               // [B_V; R_V] [48][D] bf16
    uint8_t* sOut = smem + C::OFF_OUT;           // [NQ][D / 64][128][64] swizzled
    __shared__ __align__(8) LrSync sy;
    __shared__ int conv_len[2][BN];              // code lengths of a tile's tokens (converters)

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
    for (int i = 0; i < NQ; ++i) nq[i] = tiles_for(q0 + i * BM, a.S);
    const int n_kv = nq[NQ - 1] > nq[0] ? nq[NQ - 1] : nq[0];

    if (threadIdx.x == 0) {
        prefetch_tmap(&tmQ);
        prefetch_tmap(&tmO);
        prefetch_tmap(&tmCK);
        prefetch_tmap(&tmCV);
        prefetch_tmap(&tmUK);
        prefetch_tmap(&tmUV);
        mbar_init(&sy.q_full, 1);
        mbar_init(&sy.w_full, 1);
        for (int s = 0; s < NSB; ++s) {
            mbar_init(&sy.raw_full[s], 1);
            mbar_init(&sy.raw_empty[s], C::CONV);
        }
        for (int s = 0; s < NS; ++s) {
            mbar_init(&sy.op_ready[s], C::CONV);
            mbar_init(&sy.op_empty[s], 1);
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
    auto tS = [&](int i) { return tmem + static_cast<uint32_t>(i * BN); };
    auto tO = [&](int i) { return tmem + static_cast<uint32_t>(NQ * BN + i * QW); };

    const int wg = warp >> 2;
    if (wg < NQ) {
        tc::reg_inc<C::REG_SOFTMAX>();
        // ------------------------------------------------------------ softmax and epilogue, one warpgroup per query tile
        const int qi = wg;
        const int wq = warp & 3;
        const int row = wq * 32 + lane;
        const int qpos = q0 + qi * BM + row;
        const uint32_t lane_base = static_cast<uint32_t>(wq * 32) << 16;
        const uint32_t sS = tS(qi) + lane_base;
        const uint32_t sO = tO(qi) + lane_base;
        const int n_my = nq[qi];
        const int diag0 = (q0 + qi * BM) / BN;
        float m_used = NEG_INF;
        float l = 0.f;
        // one tile of S in groups of 64 columns (two 32-column TMEM loads each): with BN =
        // 128 the row max is taken over both groups first and each group is loaded again
        // for its weights, so a row never holds more than 64 scores in registers
        constexpr int G64 = BN / 64;
        auto load_group = [&](auto mask_tag, int gi, int lim, uint32_t (&r)[2][32]) {
            constexpr bool MASKED = decltype(mask_tag)::value;
#pragma unroll
            for (int c = 0; c < 2; ++c) tc::ld32(sS + gi * 64 + c * 32, r[c]);
            tc::wait_ld();
            if (MASKED) {
#pragma unroll
                for (int c = 0; c < 2; ++c)
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        if (gi * 64 + c * 32 + i > lim) r[c][i] = __float_as_uint(NEG_INF);
            }
        };
        auto step = [&](auto mask_tag, int j) {
            const int lim = qpos - j * BN;               // column c is visible iff c <= lim
            uint32_t r[2][32];
            float mx[4] = {NEG_INF, NEG_INF, NEG_INF, NEG_INF};
#pragma unroll
            for (int gi = 0; gi < G64; ++gi) {
                load_group(mask_tag, gi, lim, r);
#pragma unroll
                for (int c = 0; c < 2; ++c)
#pragma unroll
                    for (int i = 0; i < 32; i += 2)
                        mx[(i >> 1) & 3] = fmaxf(mx[(i >> 1) & 3], fmaxf(__uint_as_float(r[c][i]), __uint_as_float(r[c][i + 1])));
            }
            const float mt = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * a.scale_log2;
            // lazy max: rescale O' only when the row max grew by more than 2^8
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
                for (int c = 0; c < QW / 32; ++c) {
                    uint32_t o32[32];
                    tc::ld32(sO + c * 32, o32);
                    tc::wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) o32[i] = __float_as_uint(__uint_as_float(o32[i]) * corr);
                    tc::st32(sO + c * 32, o32);
                }
            }
            const float nm = -m_used;
            float ls[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int gi = 0; gi < G64; ++gi) {
                if (G64 > 1) load_group(mask_tag, gi, lim, r);   // P of group 0 lands over its own S
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    uint32_t pk[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const float p0 = tc::ex2(fmaf(__uint_as_float(r[c][2 * i]), a.scale_log2, nm));
                        const float p1 = tc::ex2(fmaf(__uint_as_float(r[c][2 * i + 1]), a.scale_log2, nm));
                        ls[i & 3] += p0 + p1;
                        pk[i] = pack_bf16(p0, p1);
                    }
                    tc::st16(sS + (gi * 2 + c) * 16, pk);
                }
            }
            l += (ls[0] + ls[1]) + (ls[2] + ls[3]);
        };
        for (int j = 0; j < n_my; ++j) {
            wait_lr(sy, &sy.s_full[qi], j & 1, a.wait_limit, a.err);
            tc::fence_after();
            if (j >= diag0)
                step(std::true_type{}, j);
            else
                step(std::false_type{}, j);
            tc::wait_st();
            tc::fence_before();
            mbar_arrive(&sy.p_full[qi]);
        }
        // ------------------------------------------------------------ epilogue: o = O' [B_V; R_V] / l
        if (n_my > 0) {
            wait_lr(sy, &sy.o_full, 0, a.wait_limit, a.err);
            wait_lr(sy, &sy.w_full, 0, a.wait_limit, a.err);
            tc::fence_after();
            float ov[RB + RM];
            {
                uint32_t r0[32], r1[32];
                tc::ld32(sO, r0);
                tc::ld32(sO + 32, r1);
                tc::wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i) ov[i] = __uint_as_float(r0[i]);
#pragma unroll
                for (int i = 0; i < RM; ++i) ov[RB + i] = __uint_as_float(r1[i]);
            }
            const float inv = 1.f / l;
            uint8_t* so = sOut + qi * C::OUT_TILE;
            const uint16_t* W = reinterpret_cast<const uint16_t*>(sW);
#pragma unroll 1
            for (int e0 = 0; e0 < D; e0 += 8) {
                float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int i = 0; i < RB + RM; ++i) {
                    const uint4 w4 = *reinterpret_cast<const uint4*>(W + i * D + e0);   // same address in every lane
                    acc[0] = fmaf(ov[i], bf16_lo(w4.x), acc[0]);
                    acc[1] = fmaf(ov[i], bf16_hi(w4.x), acc[1]);
                    acc[2] = fmaf(ov[i], bf16_lo(w4.y), acc[2]);
                    acc[3] = fmaf(ov[i], bf16_hi(w4.y), acc[3]);
                    acc[4] = fmaf(ov[i], bf16_lo(w4.z), acc[4]);
                    acc[5] = fmaf(ov[i], bf16_hi(w4.z), acc[5]);
                    acc[6] = fmaf(ov[i], bf16_lo(w4.w), acc[6]);
                    acc[7] = fmaf(ov[i], bf16_hi(w4.w), acc[7]);
                }
                uint4 v;
                v.x = pack_bf16(acc[0] * inv, acc[1] * inv);
                v.y = pack_bf16(acc[2] * inv, acc[3] * inv);
                v.z = pack_bf16(acc[4] * inv, acc[5] * inv);
                v.w = pack_bf16(acc[6] * inv, acc[7] * inv);
                const int chunk = e0 >> 3;
                *reinterpret_cast<uint4*>(so + (chunk >> 3) * (BM * 128) + swz128(row, chunk & 7)) = v;
            }
            if (a.lse != nullptr && qpos < a.S)
                a.lse[static_cast<size_t>(b * a.Hq + h) * a.S + qpos] = (m_used + log2f(l)) * LN2_F;
            fence_proxy_async();
            named_sync(1 + qi, 128);
            if (row == 0) {
#pragma unroll
                for (int hh = 0; hh < D / 64; ++hh)
                    tma_store_3d(&tmO, so + hh * BM * 128, hh * 64, q0 + qi * BM, b * a.Hq + h);
                bulk_commit();
                bulk_wait_read0();
            }
        }
    } else if (wg >= C::W_CONV / 4 && wg < C::W_CONV / 4 + C::CONV / 128) {
        tc::reg_dec<C::REG_CONV>();
        // ------------------------------------------------------------ converters: raw tiles -> K', V'
        // thread t: operand m (0: K', 1: V') and token rows r0 + 64 k of the tile (whole
        // 128-byte rows)
        constexpr int RPT = BN / 64;                     // rows per thread
        const int t = threadIdx.x - 32 * C::W_CONV;
        const int m = t >> 6;
        const int r0 = t & 63;
        const size_t tok_row = (static_cast<size_t>(b) * a.Hkv + jkv) * a.T;
        const uint16_t* s_src = m == 0 ? a.s_k : a.s_v;
        // the tokens' scale bits and ranks, loaded PF tiles ahead of their use (plain loads;
        // the loop below is unrolled by PF so that no register with a load in flight moves)
        constexpr int PF = BN == 128 ? 2 : 3;     // 256 or 192 tokens ahead
        uint32_t pf_s[PF][RPT], pf_r[PF][RPT];
        auto meta = [&](int jj, uint32_t (&sb)[RPT], uint32_t (&rb)[RPT]) {
#pragma unroll
            for (int k = 0; k < RPT; ++k) {
                const int tok = jj * BN + r0 + 64 * k;
                sb[k] = 0u;
                rb[k] = 0u;
                if (jj < n_kv && tok < a.S) {            // rows past the sequence stay zero
                    sb[k] = s_src[tok_row + tok];
                    rb[k] = a.rank[static_cast<size_t>(b) * a.T + tok];
                }
            }
        };
#pragma unroll
        for (int q = 0; q < PF; ++q) meta(q, pf_s[q], pf_r[q]);
        for (int j0 = 0; j0 < n_kv; j0 += PF) {
#pragma unroll
          for (int q = 0; q < PF; ++q) {
            const int j = j0 + q;
            if (j >= n_kv) break;
            const int s = j % NS;
            const int sb = j % NSB;
            float scale[RPT];
            int rkv[RPT];
#pragma unroll
            for (int k = 0; k < RPT; ++k) {
                scale[k] = __half2float(__ushort_as_half(static_cast<unsigned short>(pf_s[q][k])));
                rkv[k] = static_cast<int>(pf_r[q][k]);
            }
            meta(j + PF, pf_s[q], pf_r[q]);
            // where a token's codes start in its 32-token code group: after the codes of
            // the group's earlier tokens (the converters exchange the tile's code lengths)
            if (m == 0) {
#pragma unroll
                for (int k = 0; k < RPT; ++k) conv_len[j & 1][r0 + 64 * k] = code_len(static_cast<unsigned>(rkv[k]));
            }
            named_sync(3, C::CONV);
            int ov[RPT];
#pragma unroll
            for (int k = 0; k < RPT; ++k) {
                const int r = r0 + 64 * k;
                ov[k] = 0;
                for (int i = r & ~31; i < r; ++i) ov[k] += conv_len[j & 1][i];
            }
            wait_lr(sy, &sy.raw_full[sb], (j / NSB) & 1, a.wait_limit, a.err);
            if (j >= NS) wait_lr(sy, &sy.op_empty[s], ((j / NS) - 1) & 1, a.wait_limit, a.err);
            const uint8_t* raw = sB + sb * C::STAGE_B;
            uint8_t* op = sA + s * C::STAGE_A + m * C::OP_TILE;
#pragma unroll
            for (int k = 0; k < RPT; ++k) {
                const int r = r0 + 64 * k;
                const int rk = rkv[k];
                const int o = ov[k];
                {
                    // chunks 0-3: the 32 coefficients, copied into the swizzled row
                    const uint4* src = reinterpret_cast<const uint4*>(raw + m * C::C_BYTES + r * (RB * 2));
#pragma unroll
                    for (int c = 0; c < 4; ++c) *reinterpret_cast<uint4*>(op + swz128(r, c)) = src[c];
                }
                {
                    // chunks 4-5: s * u for the first r_t codes (exact product, one bf16 rounding); 6-7: zero
                    const uint4 w = codes_at(raw + 2 * C::C_BYTES + m * C::U_BYTES + (r & ~31) * RM + o);
                    const uint32_t words[4] = {w.x, w.y, w.z, w.w};
                    uint32_t pk[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const int c0 = 2 * i, c1 = 2 * i + 1;
                        const int x0 = static_cast<int8_t>((words[c0 >> 2] >> (8 * (c0 & 3))) & 0xffu);
                        const int x1 = static_cast<int8_t>((words[c1 >> 2] >> (8 * (c1 & 3))) & 0xffu);
                        pk[i] = pack_bf16(c0 < rk ? static_cast<float>(x0) * scale[k] : 0.f,
                                          c1 < rk ? static_cast<float>(x1) * scale[k] : 0.f);
                    }
                    *reinterpret_cast<uint4*>(op + swz128(r, 4)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                    *reinterpret_cast<uint4*>(op + swz128(r, 5)) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
                    *reinterpret_cast<uint4*>(op + swz128(r, 6)) = make_uint4(0u, 0u, 0u, 0u);
                    *reinterpret_cast<uint4*>(op + swz128(r, 7)) = make_uint4(0u, 0u, 0u, 0u);
                }
            }
            fence_proxy_async();
            mbar_arrive(&sy.op_ready[s]);
            mbar_arrive(&sy.raw_empty[sb]);
          }
        }
    } else {
        tc::reg_dec<C::REG_CTRL>();
        if (warp == C::W_TMA) {
            // ------------------------------------------------------------ TMA producer
            if (lane == 0) {
                mbar_arrive_expect_tx(&sy.q_full, NQ * C::Q_BYTES);
#pragma unroll
                for (int i = 0; i < NQ; ++i)
                    tma_load_3d(sQ + i * C::Q_BYTES, &tmQ, 0, q0 + i * BM, b * a.Hq + h, &sy.q_full);
                mbar_arrive_expect_tx(&sy.w_full, C::W_BYTES);
                bulk_load(sW, a.basis_v + static_cast<size_t>(jkv) * RB * D, RB * D * 2, &sy.w_full);
                bulk_load(sW + RB * D * 2, a.r_v + static_cast<size_t>(jkv) * RM * D, RM * D * 2, &sy.w_full);
                const int crow = (a.pair * a.B + b) * a.Hkv + jkv;
                const int urow = b * a.Hkv + jkv;
                for (int j = 0; j < n_kv; ++j) {
                    const int sb = j % NSB;
                    if (j >= NSB) wait_lr(sy, &sy.raw_empty[sb], ((j / NSB) - 1) & 1, a.wait_limit, a.err);
                    if (sy.abort) break;
                    uint8_t* st = sB + sb * C::STAGE_B;
                    mbar_arrive_expect_tx(&sy.raw_full[sb], C::STAGE_B);
                    tma_load_3d(st, &tmCK, 0, j * BN, crow, &sy.raw_full[sb]);
                    tma_load_3d(st + C::C_BYTES, &tmCV, 0, j * BN, crow, &sy.raw_full[sb]);
                    tma_load_3d(st + 2 * C::C_BYTES, &tmUK, 0, j * BN, urow, &sy.raw_full[sb]);
                    tma_load_3d(st + 2 * C::C_BYTES + C::U_BYTES, &tmUV, 0, j * BN, urow, &sy.raw_full[sb]);
                }
                if (sy.abort) {
                    // let copies still in flight land before the CTA's shared memory goes away
                    const int first = n_kv > NSB ? n_kv - NSB : 0;
                    for (int j = first; j < n_kv; ++j) {
                        const long long t0 = clock64();
                        while (!mbar_try_wait(&sy.raw_full[j % NSB], (j / NSB) & 1) && clock64() - t0 < a.wait_limit) {
                        }
                    }
                }
                {
                    const long long t0 = clock64();
                    while (!mbar_try_wait(&sy.q_full, 0) && clock64() - t0 < a.wait_limit) {
                    }
                    const long long t1 = clock64();
                    while (!mbar_try_wait(&sy.w_full, 0) && clock64() - t1 < a.wait_limit) {
                    }
                }
            }
        } else if (warp == C::W_MMA) {
            // ------------------------------------------------------------ MMA issuer
            if (lane == 0) {
                constexpr uint32_t idS = tc::idesc_bf16(BM, BN, false, false);
                constexpr uint32_t idO = tc::idesc_bf16(BM, QW, false, true);
                // descriptors: one base per operand tile, then the start-address field
                // (address >> 4, in the low bits) advanced by a constant per K step
                auto issue_s = [&](int i, int j) {          // S_i = Q'_i K'_j^T
                    const uint64_t qd = tc::smem_desc(smem_u32(sQ + i * C::Q_BYTES), 16, 1024, tc::LAYOUT_SW128);
                    const uint64_t kd = tc::smem_desc(smem_u32(sA + (j % NS) * C::STAGE_A), 16, 1024, tc::LAYOUT_SW128);
#pragma unroll
                    for (int kk = 0; kk < QW / 16; ++kk)
                        tc::mma_ss(tS(i), qd + ((kk * 32) >> 4), kd + ((kk * 32) >> 4), idS, kk > 0 ? 1u : 0u);
                    tc::commit(&sy.s_full[i]);
                };
                auto issue_pv = [&](int i, int j) {         // O'_i += P_i V'_j, P_i from TMEM
                    wait_lr(sy, &sy.p_full[i], j & 1, a.wait_limit, a.err);
                    tc::fence_after();
                    const uint64_t vd = tc::smem_desc(smem_u32(sA + (j % NS) * C::STAGE_A + C::OP_TILE), BN * 128, 1024,
                                                      tc::LAYOUT_SW128);
#pragma unroll
                    for (int kk = 0; kk < BN / 16; ++kk)
                        tc::mma_ts(tO(i), tS(i) + kk * 8, vd + ((kk * 16 * 128) >> 4), idO, (j > 0 || kk > 0) ? 1u : 0u);
                };
                auto wait_op = [&](int j) {
                    wait_lr(sy, &sy.op_ready[j % NS], (j / NS) & 1, a.wait_limit, a.err);
                    tc::fence_after();
                };
                wait_lr(sy, &sy.q_full, 0, a.wait_limit, a.err);
                wait_op(0);
                if (nq[0] > 0) issue_s(0, 0);
                if (nq[1] > 0) issue_s(1, 0);
                for (int j = 0; j < n_kv && !sy.abort; ++j) {
                    const bool next = j + 1 < n_kv;
                    if (j < nq[0]) issue_pv(0, j);
                    if (next) wait_op(j + 1);
                    if (next && j + 1 < nq[0]) issue_s(0, j + 1);
                    if (j < nq[1]) issue_pv(1, j);
                    tc::commit(&sy.op_empty[j % NS]);
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

// ---------------------------------------------------------------- query projection pre-pass
// q'[b][h][s] = [B_K q | R_K q | 0] as bf16: per (sequence, head) a [rows x d] by [d x 48]
// product on the tensor cores (mma.sync m16n8k16, bf16 operands, fp32 accumulation),
// rounded once to bf16. Block: one (sequence, head) and 128 query rows, 16 rows per warp.
constexpr int QP_ROWS = 128;
constexpr int QP_WARPS = QP_ROWS / 16;

template <int D>
__global__ void __launch_bounds__(QP_WARPS * 32) lr_qproj_kernel(const PrefillLrArgs a) {
    constexpr int LD = D + 8;     // padded rows: the 8 rows of an ldmatrix fall on distinct banks
    __shared__ __align__(16) uint16_t W[RB + RM][LD];     // [B_K; R_K], row n = output column n
    __shared__ __align__(16) uint16_t qs[QP_ROWS][LD];
    const int h = blockIdx.x, b = blockIdx.y, r0 = blockIdx.z * QP_ROWS;
    const int j = h / a.g;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint16_t* Bk = a.basis_k + static_cast<size_t>(j) * RB * D;
    const uint16_t* Rk = a.r_k + static_cast<size_t>(j) * RM * D;
    for (int idx = tid; idx < (RB + RM) * D / 8; idx += blockDim.x) {
        const int c = idx / (D / 8), i8 = idx % (D / 8);
        const uint16_t* src = c < RB ? Bk + c * D : Rk + (c - RB) * D;
        *reinterpret_cast<uint4*>(&W[c][i8 * 8]) = *reinterpret_cast<const uint4*>(src + i8 * 8);
    }
    const size_t bh = static_cast<size_t>(b) * a.Hq + h;
    const int nrows = min(QP_ROWS, a.S - r0);
    for (int idx = tid; idx < QP_ROWS * D / 8; idx += blockDim.x) {
        const int rr = idx / (D / 8), c8 = idx % (D / 8);
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (rr < nrows) v = *reinterpret_cast<const uint4*>(a.q + (bh * a.S + r0 + rr) * D + c8 * 8);
        *reinterpret_cast<uint4*>(&qs[rr][c8 * 8]) = v;
    }
    __syncthreads();
    const int wr = warp * 16;
    if (wr >= nrows) return;
    constexpr int NT = (RB + RM) / 8;     // n8 tiles of output columns
    float acc[NT][4];
#pragma unroll
    for (int n = 0; n < NT; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
    const int mi = lane >> 3, ri = lane & 7;
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
        // A: (rows 0-7 | 8-15) x (k 0-7 | 8-15) of the warp's 16 rows
        uint32_t af[4];
        ldsm_x4(smem_u32(&qs[wr + (mi & 1) * 8 + ri][ks * 16 + (mi >> 1) * 8]), af[0], af[1], af[2], af[3]);
#pragma unroll
        for (int n = 0; n < NT; n += 2) {
            // B of two n-tiles: W rows are the output columns, contiguous in k
            uint32_t b0, b1, b2, b3;
            ldsm_x4(smem_u32(&W[(n + (mi >> 1)) * 8 + ri][ks * 16 + (mi & 1) * 8]), b0, b1, b2, b3);
            mma_bf16(acc[n], af, b0, b1);
            mma_bf16(acc[n + 1], af, b2, b3);
        }
    }
    // accumulator rows lane/4 and lane/4 + 8, columns 2 (lane % 4) and + 1 of each n-tile
    const int rw = lane >> 2, cq = 2 * (lane & 3);
#pragma unroll
    for (int half = 0; half < 2; ++half) {
        const int rr = wr + rw + half * 8;
        if (rr >= nrows) continue;
        uint16_t* dst = a.qp + (bh * a.S + r0 + rr) * QW;
#pragma unroll
        for (int n = 0; n < NT; ++n)
            *reinterpret_cast<uint32_t*>(dst + n * 8 + cq) = pack_bf16(acc[n][2 * half], acc[n][2 * half + 1]);
    }
    // the padding columns 48..63 of the warp's rows are zero
    {
        const int rr = wr + (lane >> 1);
        if (rr < nrows)
            *reinterpret_cast<uint4*>(a.qp + (bh * a.S + r0 + rr) * QW + RB + RM + (lane & 1) * 8) =
                make_uint4(0u, 0u, 0u, 0u);
    }
}

template <int D>
cudaError_t launch_lr_one(const CUtensorMap* maps, const PrefillLrArgs& a, cudaStream_t st) {
    using C = LrPfCfg<D>;
    auto kern = prefill_lowrank_kernel<D>;
    static std::atomic<unsigned long long> attr_done{0};
    cudaError_t e = once_per_device(attr_done, [&] {
        cudaError_t r = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
        if (r != cudaSuccess) return r;
        cudaFuncAttributes fa;
        r = cudaFuncGetAttributes(&fa, kern);
        if (r != cudaSuccess) return r;
        return fa.numRegs * C::THREADS < C::REG_SUM ? cudaErrorInvalidConfiguration : cudaSuccess;
    });
    if (e != cudaSuccess) return e;
    dim3 grid(a.Hq, a.B, (a.S + NQ * BM - 1) / (NQ * BM));
    kern<<<grid, C::THREADS, C::SMEM, st>>>(maps[0], maps[1], maps[2], maps[3], maps[4], maps[5], a);
    return cudaGetLastError();
}

}  // namespace

int prefill_lowrank_tile() { return BN; }

cudaError_t launch_lr_qproj(const PrefillLrArgs& a, cudaStream_t st) {
    dim3 grid(a.Hq, a.B, (a.S + QP_ROWS - 1) / QP_ROWS);
    if (a.d == 64)
        lr_qproj_kernel<64><<<grid, QP_WARPS * 32, 0, st>>>(a);
    else
        lr_qproj_kernel<128><<<grid, QP_WARPS * 32, 0, st>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_prefill_lowrank(int d, const CUtensorMap* maps, const PrefillLrArgs& a, cudaStream_t st) {
    return d == 64 ? launch_lr_one<64>(maps, a, st) : launch_lr_one<128>(maps, a, st);
}

}  // namespace kvs

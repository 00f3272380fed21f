// Causal prefill over a shared cache on the 5th-generation tensor cores (tcgen05 + TMEM).
//
// One CTA = 128 query rows of one head. Warp roles:
//   warp 0       TMA producer: Q once, then K/V tiles into a 2-stage ring
//   warp 1       TMEM owner and MMA issuer (one thread): S = Q K^T into one of two
//                TMEM S buffers, O += P V into the TMEM O accumulator
//   warps 4-7    softmax warpgroup, one thread per query row: S from TMEM,
//                causal mask, online softmax in base 2 with a lazy max (O is
//                rescaled in TMEM only when the row max grows by more than 2^8),
//                P as bf16 into shared memory (128-B swizzled, the MMA's A layout),
//                epilogue O / l -> bf16 and the log-sum-exp
//   warps 8-11   (two-source layers only) mixers: K~ = w K1 + (1-w) K2 and the
//                same for V, in fp32, rounded once to bf16, written in place over
//                the first source's tile, so the MMA reads the mixed operand and
//                the mixed K/V never reach HBM ("DepthGraft: Structural
//                Regularization through Hierarchical Cross-Layer KV
//                Reconstruction", Abstract: deep-layer KV rebuilt from a
//                shallow/middle source pair; the convex mix is this library's reading).
// Every mbarrier wait is bounded; a wait that runs out records KVS_ETIMEOUT,
// makes the other waits of the CTA give up, and the CTA still frees its TMEM.
#include "tc_sm100.cuh"

namespace kvs {
namespace {

constexpr int BM = 128;
constexpr int NS = 2;

template <int D, bool MIX>
struct PfCfg {
    static constexpr int BN = MIX ? 64 : 128;
    static constexpr int HALVES = D / 64;
    static constexpr int NSRC = MIX ? 2 : 1;
    static constexpr int Q_BYTES = BM * D * 2;
    static constexpr int TILE = BN * D * 2;        // one K or V tile
    static constexpr int HALF_T = BN * 128;        // one 64-column half of it
    static constexpr int STAGE = 2 * NSRC * TILE;
    static constexpr int P_BYTES = BM * BN * 2;
    static constexpr int SMEM = Q_BYTES + NS * STAGE + P_BYTES + 1024;
    static constexpr uint32_t TMEM_COLS = (2 * BN + D) <= 256 ? 256u : 512u;
    static constexpr int THREADS = MIX ? 384 : 256;
};

struct Sync {
    uint64_t q_full;
    uint64_t kv_full[NS];
    uint64_t kv_ready[NS];
    uint64_t kv_empty[NS];
    uint64_t s_full[2];
    uint64_t s_free[2];
    uint64_t p_full;
    uint64_t p_free;
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

template <int D, bool MIX>
__global__ void __launch_bounds__(PfCfg<D, MIX>::THREADS, 1)
prefill_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const PrefillArgs a) {
    using C = PfCfg<D, MIX>;
    constexpr int BN = C::BN;
    extern __shared__ uint8_t smem_dyn[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
    uint8_t* sQ = smem;
    uint8_t* sKV = smem + C::Q_BYTES;
    uint8_t* sP = sKV + NS * C::STAGE;
    __shared__ __align__(8) Sync sy;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int n_mt = (a.S + BM - 1) / BM;
    const int mt = n_mt - 1 - static_cast<int>(blockIdx.z);     // heaviest query tiles first
    const int h = blockIdx.x;
    const int b = blockIdx.y;
    const int jkv = h / a.g;
    const int q0 = mt * BM;
    const int q_last = min(q0 + BM, a.S) - 1;
    const int n_kv = q_last / BN + 1;
    const int diag0 = q0 / BN;

    if (threadIdx.x == 0) {
        mbar_init(&sy.q_full, 1);
        for (int s = 0; s < NS; ++s) {
            mbar_init(&sy.kv_full[s], 1);
            mbar_init(&sy.kv_ready[s], 128);
            mbar_init(&sy.kv_empty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sy.s_full[i], 1);
            mbar_init(&sy.s_free[i], 128);
        }
        mbar_init(&sy.p_full, 128);
        mbar_init(&sy.p_free, 1);
        mbar_init(&sy.o_full, 1);
        sy.abort = 0;
        mbar_init_fence();
    }
    if (warp == 1) {
        tc::alloc(&sy.tmem_base, C::TMEM_COLS);
        tc::relinquish();
    }
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = sy.tmem_base;
    const uint32_t tmem_o = tmem + 2 * BN;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            mbar_arrive_expect_tx(&sy.q_full, C::Q_BYTES);
#pragma unroll
            for (int hh = 0; hh < C::HALVES; ++hh)
                tma_load_3d(sQ + hh * BM * 128, &tmQ, hh * 64, q0, b * a.Hq + h, &sy.q_full);
            const int BH = a.B * a.Hkv;
            const int r0 = a.src0 * BH + b * a.Hkv + jkv;
            const int r1 = a.src1 * BH + b * a.Hkv + jkv;
            for (int j = 0; j < n_kv; ++j) {
                const int s = j % NS;
                if (j >= NS) wait_cta(sy, &sy.kv_empty[s], ((j / NS) - 1) & 1, a.wait_limit, a.err);
                if (sy.abort) break;
                uint8_t* st = sKV + s * C::STAGE;
                mbar_arrive_expect_tx(&sy.kv_full[s], C::STAGE);
#pragma unroll
                for (int hh = 0; hh < C::HALVES; ++hh) {
                    tma_load_3d(st + hh * C::HALF_T, &tmK, hh * 64, j * BN, r0, &sy.kv_full[s]);
                    tma_load_3d(st + C::TILE + hh * C::HALF_T, &tmV, hh * 64, j * BN, r0, &sy.kv_full[s]);
                    if (MIX) {
                        tma_load_3d(st + 2 * C::TILE + hh * C::HALF_T, &tmK, hh * 64, j * BN, r1, &sy.kv_full[s]);
                        tma_load_3d(st + 3 * C::TILE + hh * C::HALF_T, &tmV, hh * 64, j * BN, r1, &sy.kv_full[s]);
                    }
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
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idS = tc::idesc_bf16(BM, BN, false, false);
            constexpr uint32_t idO = tc::idesc_bf16(BM, D, false, true);
            const uint32_t q_addr = smem_u32(sQ);
            const uint32_t p_addr = smem_u32(sP);
            auto issue_pv = [&](int jj) {
                wait_cta(sy, &sy.p_full, jj & 1, a.wait_limit, a.err);
                tc::fence_after();
                const int s = jj % NS;
                const uint32_t v_addr = smem_u32(sKV + s * C::STAGE + C::TILE);
#pragma unroll
                for (int kk = 0; kk < BN / 16; ++kk) {
                    const uint64_t ad = tc::smem_desc(p_addr + (kk >> 2) * (BM * 128) + (kk & 3) * 32, 16, 1024,
                                                      tc::LAYOUT_SW128);
                    const uint64_t bd = tc::smem_desc(v_addr + kk * 16 * 128, C::HALF_T, 1024, tc::LAYOUT_SW128);
                    tc::mma_ss(tmem_o, ad, bd, idO, (jj > 0 || kk > 0) ? 1u : 0u);
                }
                tc::commit(&sy.p_free);
                tc::commit(&sy.kv_empty[s]);
            };
            wait_cta(sy, &sy.q_full, 0, a.wait_limit, a.err);
            for (int j = 0; j < n_kv; ++j) {
                const int s = j % NS;
                wait_cta(sy, MIX ? &sy.kv_ready[s] : &sy.kv_full[s], (j / NS) & 1, a.wait_limit, a.err);
                const int sb = j & 1;
                if (j >= 2) wait_cta(sy, &sy.s_free[sb], ((j >> 1) - 1) & 1, a.wait_limit, a.err);
                tc::fence_after();
                const uint32_t k_addr = smem_u32(sKV + s * C::STAGE);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk & 3) * 32;      // 16 bf16 along K inside the 128-B row
                    const uint64_t ad = tc::smem_desc(q_addr + (kk >> 2) * (BM * 128) + off, 16, 1024, tc::LAYOUT_SW128);
                    const uint64_t bd = tc::smem_desc(k_addr + (kk >> 2) * C::HALF_T + off, 16, 1024, tc::LAYOUT_SW128);
                    tc::mma_ss(tmem + sb * BN, ad, bd, idS, kk > 0 ? 1u : 0u);
                }
                tc::commit(&sy.s_full[sb]);
                if (j >= 1) issue_pv(j - 1);
                if (sy.abort) break;
            }
            if (!sy.abort) issue_pv(n_kv - 1);
            tc::commit(&sy.o_full);
        }
    } else if (warp >= 4 && warp < 8) {
        // ------------------------------------------------------------ softmax warpgroup
        const int row = (warp - 4) * 32 + lane;
        const int qpos = q0 + row;
        const uint32_t lane_base = static_cast<uint32_t>((warp - 4) * 32) << 16;
        float m_used = NEG_INF;
        float l = 0.f;
        for (int j = 0; j < n_kv; ++j) {
            const int sb = j & 1;
            wait_cta(sy, &sy.s_full[sb], (j >> 1) & 1, a.wait_limit, a.err);
            tc::fence_after();
            float s[BN];
#pragma unroll
            for (int c = 0; c < BN / 32; ++c) {
                uint32_t r[32];
                tc::ld32(tmem + lane_base + sb * BN + c * 32, r);
                tc::wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i) s[c * 32 + i] = __uint_as_float(r[i]);
            }
            tc::fence_before();
            mbar_arrive(&sy.s_free[sb]);
            const int k0 = j * BN;
            float mt = NEG_INF;
#pragma unroll
            for (int c = 0; c < BN; ++c) {
                float v = s[c] * a.scale_log2;
                if (j >= diag0 && k0 + c > qpos) v = NEG_INF;
                s[c] = v;
                mt = fmaxf(mt, v);
            }
            // lazy max: rescale O only when this row's max grew by more than 2^8; the
            // TMEM load/store is warp-collective, so the warp rescales if any row needs it
            float corr = 1.f;
            if (m_used == NEG_INF) {
                m_used = mt;
            } else if (mt > m_used + 8.f) {
                corr = tc::ex2(m_used - mt);
                m_used = mt;
            }
            const bool rescale = __any_sync(0xffffffffu, corr != 1.f);
            if (j >= 1) wait_cta(sy, &sy.p_free, (j - 1) & 1, a.wait_limit, a.err);
            if (rescale) {
                l *= corr;
                tc::fence_after();
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t r[32];
                    tc::ld32(tmem_o + lane_base + c * 32, r);
                    tc::wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * corr);
                    tc::st32(tmem_o + lane_base + c * 32, r);
                }
                tc::wait_st();
            }
#pragma unroll
            for (int c8 = 0; c8 < BN / 8; ++c8) {
                uint32_t pk[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    pk[i] = pack_bf16(tc::ex2(s[c8 * 8 + 2 * i] - m_used), tc::ex2(s[c8 * 8 + 2 * i + 1] - m_used));
                    l += bf16_lo(pk[i]) + bf16_hi(pk[i]);
                }
                uint8_t* dst = sP + (c8 >> 3) * (BM * 128) + swz128(row, c8 & 7);
                *reinterpret_cast<uint4*>(dst) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            }
            fence_proxy_async();
            tc::fence_before();
            mbar_arrive(&sy.p_full);
        }
        // ------------------------------------------------------------ epilogue
        wait_cta(sy, &sy.o_full, 0, a.wait_limit, a.err);
        tc::fence_after();
        const float inv = 1.f / l;
        uint16_t* orow = reinterpret_cast<uint16_t*>(a.out) + (static_cast<size_t>(b * a.Hq + h) * a.S + qpos) * D;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
            uint32_t r[32];
            tc::ld32(tmem_o + lane_base + c * 32, r);
            tc::wait_ld();
            if (qpos < a.S) {
#pragma unroll
                for (int i = 0; i < 32; i += 8) {
                    uint4 v;
                    v.x = pack_bf16(__uint_as_float(r[i]) * inv, __uint_as_float(r[i + 1]) * inv);
                    v.y = pack_bf16(__uint_as_float(r[i + 2]) * inv, __uint_as_float(r[i + 3]) * inv);
                    v.z = pack_bf16(__uint_as_float(r[i + 4]) * inv, __uint_as_float(r[i + 5]) * inv);
                    v.w = pack_bf16(__uint_as_float(r[i + 6]) * inv, __uint_as_float(r[i + 7]) * inv);
                    *reinterpret_cast<uint4*>(orow + c * 32 + i) = v;
                }
            }
        }
        if (a.lse != nullptr && qpos < a.S)
            a.lse[static_cast<size_t>(b * a.Hq + h) * a.S + qpos] = (m_used + log2f(l)) * LN2_F;
    } else if (MIX && warp >= 8) {
        // ------------------------------------------------------------ mixers (two-source layers)
        const int t = threadIdx.x - 256;
        const float w = a.w[jkv];
        const float w1 = 1.f - w;
        for (int j = 0; j < n_kv; ++j) {
            const int s = j % NS;
            wait_cta(sy, &sy.kv_full[s], (j / NS) & 1, a.wait_limit, a.err);
            uint4* dst = reinterpret_cast<uint4*>(sKV + s * C::STAGE);               // K1 | V1
            const uint4* src = reinterpret_cast<const uint4*>(sKV + s * C::STAGE + 2 * C::TILE);   // K2 | V2
            for (int idx = t; idx < 2 * C::TILE / 16; idx += 128) {
                const uint4 x = dst[idx];
                const uint4 y = src[idx];
                uint4 r;
                r.x = pack_bf16(w * bf16_lo(x.x) + w1 * bf16_lo(y.x), w * bf16_hi(x.x) + w1 * bf16_hi(y.x));
                r.y = pack_bf16(w * bf16_lo(x.y) + w1 * bf16_lo(y.y), w * bf16_hi(x.y) + w1 * bf16_hi(y.y));
                r.z = pack_bf16(w * bf16_lo(x.z) + w1 * bf16_lo(y.z), w * bf16_hi(x.z) + w1 * bf16_hi(y.z));
                r.w = pack_bf16(w * bf16_lo(x.w) + w1 * bf16_lo(y.w), w * bf16_hi(x.w) + w1 * bf16_hi(y.w));
                dst[idx] = r;
            }
            fence_proxy_async();
            mbar_arrive(&sy.kv_ready[s]);
        }
    }

    tc::fence_before();
    __syncthreads();
    if (warp == 1) {
        tc::fence_after();
        tc::dealloc(tmem, C::TMEM_COLS);
    }
}

template <int D, bool MIX>
cudaError_t launch_one(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const PrefillArgs& a,
                       cudaStream_t st) {
    using C = PfCfg<D, MIX>;
    auto kern = prefill_kernel<D, MIX>;
    static bool attr_done = false;
    if (!attr_done) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
        if (e != cudaSuccess) return e;
        attr_done = true;
    }
    dim3 grid(a.Hq, a.B, (a.S + BM - 1) / BM);
    kern<<<grid, C::THREADS, C::SMEM, st>>>(tq, tk, tv, a);
    return cudaGetLastError();
}

}  // namespace

int prefill_kv_tile(int d, bool mix) {
    (void)d;
    return mix ? PfCfg<128, true>::BN : PfCfg<128, false>::BN;
}

cudaError_t launch_prefill(int d, bool mix, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                           const PrefillArgs& a, cudaStream_t st) {
    if (d == 64) return mix ? launch_one<64, true>(tq, tk, tv, a, st) : launch_one<64, false>(tq, tk, tv, a, st);
    return mix ? launch_one<128, true>(tq, tk, tv, a, st) : launch_one<128, false>(tq, tk, tv, a, st);
}

}  // namespace kvs

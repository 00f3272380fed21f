// Device helpers for the sm_100a kernels: mbarriers, TMA, ldmatrix / mma.sync,
// bounded waits and the split-KV merge shared by every decode kernel.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "kvs_internal.h"

namespace kvs {

constexpr float LN2_F = 0.69314718055994530942f;
constexpr float NEG_INF = -__builtin_huge_valf();

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ------------------------------------------------------------------ mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, unsigned count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_init_fence() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, unsigned bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, unsigned parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait for the phase with the given parity to complete, for at most `limit`
// SM clock cycles. On expiry, record ERR_TIMEOUT in the status word and return false.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, unsigned parity, long long limit,
                                                  unsigned* err) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (clock64() - t0 > limit) {
            atomicOr(err, ERR_TIMEOUT);
            return false;
        }
    }
}

__device__ __forceinline__ void fence_proxy_async() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------------------------------------ TMA
// 3-D tiled bulk tensor load global -> shared, completion counted on `bar`.
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int c0, int c1, int c2,
                                            uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
        : "memory");
}

// Plain (untiled) bulk copy global -> shared; both addresses 16-B aligned, bytes % 16 == 0.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, unsigned bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// ------------------------------------------------------------------ tensor-core fragments
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

// D = A(16x16 bf16, row) * B(16x8 bf16, col) + D, fp32 accumulate
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }

// Byte offset of element chunk `c` (8 bf16 = 16 B) of row `row` inside a
// [rows][64] bf16 tile stored with the 128-byte TMA swizzle (tile base 1024-B aligned).
__device__ __forceinline__ uint32_t swz128(int row, int c) {
    return static_cast<uint32_t>(row * 128 + (((c ^ row) & 7) << 4));
}

// ------------------------------------------------------------------ split merge
// Every decode CTA ends here with, in shared memory, for its g query heads:
//   sm_m[h]  running max of the log2-domain scores,
//   sm_l[h]  sum of 2^(s - m) weights,
//   sm_o[h][e] un-normalised output sum_t 2^(s_t - m) V_t.
// With one split the CTA writes out = o / l and lse = (m + log2 l) ln 2.
// Otherwise it stores its partial and the last CTA of the (b, kv head) to
// arrive merges all partials: M = max m_s, l = sum 2^(m_s - M) l_s,
// o = sum 2^(m_s - M) o_s / l. That CTA resets the arrival counter to zero.
__device__ inline void finish_split(const DecodeArgs& a, int D, int b, int j, int split, const float* sm_m,
                                    const float* sm_l, const float* sm_o, float* sm_scratch /* >= g*MAX_SPLITS */) {
    const int g = a.g;
    const int tid = threadIdx.x;
    const int nthr = blockDim.x;
    const size_t head0 = static_cast<size_t>(b) * a.Hq + static_cast<size_t>(j) * g;
    if (a.splits == 1) {
        for (int idx = tid; idx < g * D; idx += nthr) {
            const int h = idx / D;
            a.out[(head0 + h) * D + (idx % D)] = sm_o[idx] / sm_l[h];
        }
        if (a.lse != nullptr && tid < g) a.lse[head0 + tid] = (sm_m[tid] + log2f(sm_l[tid])) * LN2_F;
        return;
    }
    const int PD = D + 2;
    const size_t unit = static_cast<size_t>(b) * a.Hkv + j;
    float* part = a.ws + (unit * a.splits + split) * static_cast<size_t>(g * PD);
    for (int idx = tid; idx < g * D; idx += nthr) part[(idx / D) * PD + (idx % D)] = sm_o[idx];
    if (tid < g) {
        part[tid * PD + D] = sm_m[tid];
        part[tid * PD + D + 1] = sm_l[tid];
    }
    __threadfence();
    __syncthreads();
    __shared__ unsigned s_is_last;
    if (tid == 0) {
        const unsigned prev = atomicAdd(a.counters + unit, 1u);
        s_is_last = (prev == static_cast<unsigned>(a.splits - 1)) ? 1u : 0u;
    }
    __syncthreads();
    if (!s_is_last) return;
    __threadfence();
    const float* base = a.ws + unit * a.splits * static_cast<size_t>(g * PD);
    // per-head max over splits, then per-(head, split) factors 2^(m_s - M)
    float* fac = sm_scratch;                 // [g][splits]
    float* hm = sm_scratch + g * a.splits;   // [g] max, then [g] l
    float* hl = hm + g;
    if (tid < g) {
        float M = NEG_INF;
        for (int s = 0; s < a.splits; ++s) M = fmaxf(M, __ldcg(base + (size_t)s * g * PD + tid * PD + D));
        float L = 0.f;
        for (int s = 0; s < a.splits; ++s) {
            const float ms = __ldcg(base + (size_t)s * g * PD + tid * PD + D);
            const float f = exp2f(ms - M);
            fac[tid * a.splits + s] = f;
            L += f * __ldcg(base + (size_t)s * g * PD + tid * PD + D + 1);
        }
        hm[tid] = M;
        hl[tid] = L;
    }
    __syncthreads();
    for (int idx = tid; idx < g * D; idx += nthr) {
        const int h = idx / D;
        const int e = idx % D;
        float acc = 0.f;
        for (int s = 0; s < a.splits; ++s) acc += fac[h * a.splits + s] * __ldcg(base + (size_t)s * g * PD + h * PD + e);
        a.out[(head0 + h) * D + e] = acc / hl[h];
    }
    if (a.lse != nullptr && tid < g) a.lse[head0 + tid] = (hm[tid] + log2f(hl[tid])) * LN2_F;
    if (tid == 0) a.counters[unit] = 0u;
}

}  // namespace kvs

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

// raise the transaction count of the current phase without arriving
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, unsigned bytes) {
    asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
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

// ------------------------------------------------------------------ dependent launch
// Wait until the grids this one depends on (programmatic stream serialization) have
// completed and their writes are visible; a no-op for an ordinary launch.
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
// Allow the next kernel on the stream to be scheduled once every CTA of this grid has
// signalled or exited; that kernel still waits for this grid's completion before it
// touches memory.
__device__ __forceinline__ void grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ------------------------------------------------------------------ TMA
// Start fetching a tensor map (a __grid_constant__ kernel parameter) into the
// descriptor cache, so the first copy that names it does not wait for it.
__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 3-D tiled bulk tensor load global -> shared, completion counted on `bar`.
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int c0, int c1, int c2,
                                            uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
        : "memory");
}

// 3-D tiled bulk tensor store shared -> global (rows outside the tensor are not written).
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, const void* src, int c0, int c1, int c2) {
    asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(smem_u32(src)), "r"(c0), "r"(c1), "r"(c2)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }

__device__ __forceinline__ void named_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
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

// D = A(16x16 f16, row) * B(16x8 f16, col) + D, fp32 accumulate
__device__ __forceinline__ void mma_f16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
    __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

// Four int8 codes (one 32-bit word, byte i = code i) -> two f16 pairs, exactly.
// Byte b becomes the f16 with bit pattern 0x64 | (b ^ 0x80), i.e. 1024 + 128 + code,
// which f16 holds exactly (its spacing is 1 on [1024, 2048)); subtracting 1152 leaves
// the code. Codes whose byte is cleared by `keep` come out as 0.
__device__ __forceinline__ void i8x4_f16(uint32_t word, uint32_t keep, uint32_t& h01, uint32_t& h23) {
    const uint32_t x = (word & keep) ^ 0x80808080u;
    const uint32_t lo = __byte_perm(x, 0x64646464u, 0x5140);
    const uint32_t hi = __byte_perm(x, 0x64646464u, 0x7362);
    const __half2 bias = __halves2half2(__ushort_as_half(0x6480), __ushort_as_half(0x6480));   // 1152
    const __half2 a = __hsub2(*reinterpret_cast<const __half2*>(&lo), bias);
    const __half2 b = __hsub2(*reinterpret_cast<const __half2*>(&hi), bias);
    h01 = *reinterpret_cast<const uint32_t*>(&a);
    h23 = *reinterpret_cast<const uint32_t*>(&b);
}

// Byte masks of the 16 code bytes of a token (byte i kept iff i < rank, 0 <= rank <= 16),
// as four 32-bit words: bytes 0-7 and 8-15 each from one 64-bit shift.
__device__ __forceinline__ void rank_keep4(int rank, uint32_t& m0, uint32_t& m1, uint32_t& m2, uint32_t& m3) {
    const int lo = min(rank, 8), hi = max(rank - 8, 0);
    const unsigned long long a = lo >= 8 ? ~0ull : ((1ull << (8 * lo)) - 1ull);
    const unsigned long long b = hi >= 8 ? ~0ull : ((1ull << (8 * hi)) - 1ull);
    m0 = static_cast<uint32_t>(a);
    m1 = static_cast<uint32_t>(a >> 32);
    m2 = static_cast<uint32_t>(b);
    m3 = static_cast<uint32_t>(b >> 32);
}

// Transpose an 8x8 matrix of 16-bit values held one pair per thread (thread t owns
// row t/4, columns 2(t%4), 2(t%4)+1) so that thread t owns row t/4 of the transpose.
__device__ __forceinline__ uint32_t movmatrix_t(uint32_t x) {
    uint32_t y;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
    return y;
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

// ------------------------------------------------------------------ sequence lengths
// Tokens of sequence b: lens[b] clamped to [0, T] (a value outside records ERR_RANGE),
// or every cached token without per-sequence lengths.
__device__ __forceinline__ int seq_len(const DecodeArgs& a, int b) {
    if (a.lens == nullptr) return a.T;
    const int n = a.lens[b];
    if (n < 0 || n > a.T) {
        atomicOr(a.err, ERR_RANGE);
        return n < 0 ? 0 : a.T;
    }
    return n;
}

// Zero rows [r0, rows) of a staged tile: `halves` blocks of `half_stride` bytes, each row
// `row_bytes` contiguous bytes of every block (a swizzle only permutes 16-B chunks inside
// a row). The values past a sequence's length in its last tile are whatever the cache
// holds there, and a zero weight times a NaN is still NaN, so they are cleared before
// the P.V product reads them. One warp; the caller syncs the warp afterwards.
__device__ __forceinline__ void zero_tile_rows(uint8_t* base, int row_bytes, int halves, int half_stride, int r0,
                                               int rows, int lane) {
    const int chunks = row_bytes / 16;
    const int n = (rows - r0) * chunks * halves;
    for (int i = lane; i < n; i += 32) {
        const int h = i / ((rows - r0) * chunks);
        const int rem = i % ((rows - r0) * chunks);
        *reinterpret_cast<uint4*>(base + h * half_stride + (r0 + rem / chunks) * row_bytes + (rem % chunks) * 16) =
            make_uint4(0u, 0u, 0u, 0u);
    }
}

// ------------------------------------------------------------------ split merge
// Partial layout: [unit][split][head][D + 4] floats: o[0..D), m, l, lx, z (rows stay
// 16-byte aligned so whole partial blocks can move by bulk copy). l sums the weights as
// the P.V products used them (rounded to the operand type), so o / l is a convex
// combination of the values; lx sums the unrounded fp32 weights and gives the lse;
// z = sum 2^(s - m) (m - s), kept when the entropy is asked for (0 otherwise).
//
// Entropy and peak of the attention weights p_t = 2^(s_t - lse2), lse2 = M + log2 lx,
// from the merged statistics of a head (M the largest score, every term of lx and z
// taken against it): H = -sum p ln p = ln 2 (log2 lx + z / lx), every term of z being
// non-negative (no cancellation, also for sharply peaked rows); max p = 2^(M - lse2) =
// 1 / lx. When the running max rises from m to m' a partial sum moves to the new
// reference as z' = 2^(m - m') (z + lx (m' - m)), lx' = 2^(m - m') lx.
__host__ __device__ constexpr int partial_width(int D) { return D + 4; }

// 2^x by the MUFU unit (ex2.approx, flush-to-zero): one instruction; -inf gives 0.
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
    return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    return v;
}

// Every decode CTA ends here with, in shared memory, for its g query heads:
//   sm_m[h]  running max of the log2-domain scores,
//   sm_l[h]  sum of 2^(s - m) weights as rounded for the P.V products,
//   sm_lx[h] sum of the unrounded 2^(s - m) weights,
//   sm_z[h]  sum of 2^(s - m) (m - s) (when the entropy is asked for),
//   sm_v[h][e] un-normalised accumulated vector (e < DV): the output
//            sum_t 2^(s_t - m) V_t, or the low-rank form's coefficient-space sums.
// With one partial per unit the CTA emits it at once. Otherwise it stores its
// partial and the last CTA of the unit to arrive merges all partials:
// M = max m_s, l = sum 2^(m_s - M) l_s (lx likewise), z = sum 2^(m_s - M) (z_s + lx_s
// (M - m_s)), v = sum 2^(m_s - M) v_s, then emits
// (and resets the unit's arrival counter to zero). Arrival is one acq_rel
// atomic per CTA. The last CTA bulk-copies the unit's partials (contiguous) into
// `stage` (free shared memory of `stage_bytes`, 16-B aligned) in one copy when
// they fit, in chunks otherwise (0 bytes: read them directly); one warp per head
// reduces (m, l), then every thread combines its share of the vector.
// `emit(v, l, lx, m, z)` writes the unit's outputs from v [g][DV] (shared memory),
// l[g], lx[g], m[g] and z[g]; it is called by all threads of the CTA. A unit with no
// tokens has l = 0: its outputs are 0, its lse is -inf, its entropy and peak 0.
// sm_scratch holds at least 4 * g * count floats; sm_v is reused for the merge.
__device__ __forceinline__ float lse_of(float m, float lx) {
    return lx > 0.f ? (m + log2f(lx)) * LN2_F : NEG_INF;
}

// Writes the entropy and peak of heads head0 .. head0 + g - 1 (threads 0 .. g - 1).
__device__ __forceinline__ void emit_entropy_peak(const DecodeArgs& a, size_t head0, const float* lx, const float* z) {
    if (threadIdx.x >= a.g) return;
    const float x = lx[threadIdx.x];
    if (a.entropy != nullptr) a.entropy[head0 + threadIdx.x] = x > 0.f ? (log2f(x) + z[threadIdx.x] / x) * LN2_F : 0.f;
    if (a.peak != nullptr) a.peak[head0 + threadIdx.x] = x > 0.f ? 1.f / x : 0.f;
}

// The weight a split or warp statistic (m, lx, z) carries in a merge against the common
// max M, and its z moved to that reference. A statistic with m = -inf has no tokens.
__device__ __forceinline__ float merge_factor(float m, float M) { return m != NEG_INF ? ex2_approx(m - M) : 0.f; }
__device__ __forceinline__ float merged_z(float f, float m, float M, float lx, float z) {
    return f != 0.f ? f * fmaf(lx, M - m, z) : 0.f;
}

struct EmitPlain {
    const DecodeArgs& a;
    int D;
    size_t head0;
    __device__ void operator()(const float* v, const float* l, const float* lx, const float* m, const float* z) const {
        for (int idx = threadIdx.x; idx < a.g * D; idx += blockDim.x) {
            const float lh = l[idx / D];
            a.out[(head0 + idx / D) * D + (idx % D)] = lh > 0.f ? v[idx] / lh : 0.f;
        }
        if (a.lse != nullptr && threadIdx.x < a.g) a.lse[head0 + threadIdx.x] = lse_of(m[threadIdx.x], lx[threadIdx.x]);
        emit_entropy_peak(a, head0, lx, z);
    }
};

// MAXDV bounds DV (values per head of a partial): each thread holds up to
// MAX_GROUP * MAXDV / 128 merged values, as every caller runs at least 128 threads.
template <int MAXDV = 128, typename Emit>
__device__ inline void finish_unit(const DecodeArgs& a, int DV, int unit_i, int index, int count, long long slot0,
                                   const float* sm_m, const float* sm_l, const float* sm_lx, const float* sm_z,
                                   float* sm_v, float* sm_scratch, uint8_t* stage, int stage_bytes, const Emit& emit) {
    const int g = a.g;
    const int tid = threadIdx.x;
    const int nthr = blockDim.x;
    if (count == 1) {
        emit(sm_v, sm_l, sm_lx, sm_m, sm_z);
        return;
    }
    const int PD = partial_width(DV);
    const int per = g * PD;
    const size_t unit = static_cast<size_t>(unit_i);
    float* part = a.ws + static_cast<size_t>(slot0 + index) * per;
    for (int idx = tid; idx < g * DV; idx += nthr) part[(idx / DV) * PD + (idx % DV)] = sm_v[idx];
    if (tid < g) {
        part[tid * PD + DV] = sm_m[tid];
        part[tid * PD + DV + 1] = sm_l[tid];
        part[tid * PD + DV + 2] = sm_lx[tid];
        part[tid * PD + DV + 3] = sm_z[tid];
    }
    // the last CTA reads the partials with a bulk copy (the async proxy): every writer
    // orders its own generic stores before that proxy before the arrival releases them
    asm volatile("fence.proxy.async.global;" ::: "memory");
    __syncthreads();
    __shared__ unsigned s_is_last;
    if (tid == 0) {
        // one acq_rel atomic: its release publishes this CTA's partial (ordered before it
        // by the barrier), its acquire lets the last arrival see every other partial
        unsigned prev;
        asm volatile("atom.add.acq_rel.gpu.global.u32 %0, [%1], 1;"
                     : "=r"(prev)
                     : "l"(a.counters + unit)
                     : "memory");
        s_is_last = (prev == static_cast<unsigned>(count - 1)) ? 1u : 0u;
    }
    __syncthreads();
    if (!s_is_last) return;
    const int n = count;
    const float* base = a.ws + static_cast<size_t>(slot0) * per;
    float* fm = sm_scratch;            // [n][g]: m, then the factors 2^(m - M)
    float* fl = sm_scratch + n * g;    // [n][g]: l
    float* flx = fl + n * g;           // [n][g]: lx
    float* fz = flx + n * g;           // [n][g]: z
    __shared__ float hm[MAX_GROUP], hl[MAX_GROUP], hlx[MAX_GROUP], hz[MAX_GROUP];
    __shared__ __align__(8) uint64_t mbar;
    const int chunk = stage_bytes / (per * 4);
    float* sp_buf = reinterpret_cast<float*>(stage);
    const bool one_copy = chunk >= n;  // the unit's partials are contiguous: one bulk copy
    if (chunk >= 1) {
        if (tid == 0) {
            mbar_init(&mbar, 1);
            mbar_init_fence();
            if (one_copy) {
                asm volatile("fence.proxy.async;" ::: "memory");
                mbar_arrive_expect_tx(&mbar, static_cast<unsigned>(n * per * 4));
                bulk_load(sp_buf, base, static_cast<unsigned>(n * per * 4), &mbar);
            }
        }
        __syncthreads();
    }
    // This CTA's own partial is taken from its shared memory, never read back from
    // global: its stores may not yet be what a bulk copy of the slot returns, and a
    // stale slot (an earlier launch's partial) would silently take its place.
    if (one_copy) {
        mbar_wait_bounded(&mbar, 0, a.wait_limit, a.err);
        for (int idx = tid; idx < n * g; idx += nthr) {
            const int sp = idx / g;
            const int h = idx % g;
            const bool own = sp == index;
            fm[idx] = own ? sm_m[h] : sp_buf[sp * per + h * PD + DV];
            fl[idx] = own ? sm_l[h] : sp_buf[sp * per + h * PD + DV + 1];
            flx[idx] = own ? sm_lx[h] : sp_buf[sp * per + h * PD + DV + 2];
            fz[idx] = own ? sm_z[h] : sp_buf[sp * per + h * PD + DV + 3];
        }
    } else {
        for (int idx = tid; idx < n * g; idx += nthr) {
            const int sp = idx / g;
            const int h = idx % g;
            const bool own = sp == index;
            fm[idx] = own ? sm_m[h] : __ldcg(base + static_cast<size_t>(sp) * per + h * PD + DV);
            fl[idx] = own ? sm_l[h] : __ldcg(base + static_cast<size_t>(sp) * per + h * PD + DV + 1);
            flx[idx] = own ? sm_lx[h] : __ldcg(base + static_cast<size_t>(sp) * per + h * PD + DV + 2);
            fz[idx] = own ? sm_z[h] : __ldcg(base + static_cast<size_t>(sp) * per + h * PD + DV + 3);
        }
    }
    __syncthreads();
    const int warp = tid >> 5, lane = tid & 31, nwarps = nthr >> 5;
    for (int h = warp; h < g; h += nwarps) {
        float M = NEG_INF;
        for (int sp = lane; sp < n; sp += 32) M = fmaxf(M, fm[sp * g + h]);
        M = warp_max(M);
        float L = 0.f, LX = 0.f, Z = 0.f;
        for (int sp = lane; sp < n; sp += 32) {
            // a split without tokens has m = -inf and weighs nothing (also when all do)
            const float ms = fm[sp * g + h];
            const float f = merge_factor(ms, M);
            fm[sp * g + h] = f;
            L += f * fl[sp * g + h];
            LX += f * flx[sp * g + h];
            Z += merged_z(f, ms, M, flx[sp * g + h], fz[sp * g + h]);
        }
        L = warp_sum(L);
        LX = warp_sum(LX);
        Z = warp_sum(Z);
        if (lane == 0) {
            hm[h] = M;
            hl[h] = L;
            hlx[h] = LX;
            hz[h] = Z;
        }
    }
    __syncthreads();
    constexpr int MAXO = (MAX_GROUP * MAXDV + 127) / 128;   // values per thread at >= 128 threads
    float acc[MAXO];
#pragma unroll
    for (int k = 0; k < MAXO; ++k) acc[k] = 0.f;
    if (one_copy) {
#pragma unroll
        for (int k = 0; k < MAXO; ++k) {
            const int idx = tid + k * nthr;
            if (idx < g * DV) {
                const int h = idx / DV;
                const int e = idx % DV;
                float v = 0.f;
                for (int c = 0; c < n; ++c) v += fm[c * g + h] * (c == index ? sm_v[h * DV + e] : sp_buf[c * per + h * PD + e]);
                acc[k] = v;
            }
        }
    } else if (chunk >= 1) {
        unsigned phase = 0;
        for (int s0 = 0; s0 < n; s0 += chunk) {
            const int cnt = min(chunk, n - s0);
            if (tid == 0) {
                asm volatile("fence.proxy.async;" ::: "memory");
                mbar_arrive_expect_tx(&mbar, static_cast<unsigned>(cnt * per * 4));
                bulk_load(sp_buf, base + static_cast<size_t>(s0) * per, static_cast<unsigned>(cnt * per * 4), &mbar);
            }
            mbar_wait_bounded(&mbar, phase, a.wait_limit, a.err);
            phase ^= 1u;
#pragma unroll
            for (int k = 0; k < MAXO; ++k) {
                const int idx = tid + k * nthr;
                if (idx < g * DV) {
                    const int h = idx / DV;
                    const int e = idx % DV;
                    float v = acc[k];
                    for (int c = 0; c < cnt; ++c)
                        v += fm[(s0 + c) * g + h] * (s0 + c == index ? sm_v[h * DV + e] : sp_buf[c * per + h * PD + e]);
                    acc[k] = v;
                }
            }
            __syncthreads();   // the buffer is refilled by the next chunk
        }
    } else {
#pragma unroll
        for (int k = 0; k < MAXO; ++k) {
            const int idx = tid + k * nthr;
            if (idx < g * DV) {
                const int h = idx / DV;
                const int e = idx % DV;
                float v = 0.f;
#pragma unroll 8
                for (int sp = 0; sp < n; ++sp)
                    v += fm[sp * g + h] * (sp == index ? sm_v[h * DV + e] : __ldcg(base + static_cast<size_t>(sp) * per + h * PD + e));
                acc[k] = v;
            }
        }
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < MAXO; ++k) {
        const int idx = tid + k * nthr;
        if (idx < g * DV) sm_v[idx] = acc[k];
    }
    __syncthreads();
    emit(sm_v, hl, hlx, hm, hz);
    if (tid == 0) a.counters[unit] = 0u;
}

// Split-grid kernels: CTA (split, j, b) holds partial `split` of `a.splits` for its unit.
__device__ inline void finish_split(const DecodeArgs& a, int D, int b, int j, int split, const float* sm_m,
                                    const float* sm_l, const float* sm_lx, const float* sm_z, float* sm_o,
                                    float* sm_scratch, uint8_t* stage, int stage_bytes) {
    const int unit = b * a.Hkv + j;
    const EmitPlain emit{a, D, static_cast<size_t>(b) * a.Hq + static_cast<size_t>(j) * a.g};
    finish_unit(a, D, unit, split, a.splits, static_cast<long long>(unit) * a.splits, sm_m, sm_l, sm_lx, sm_z, sm_o,
                sm_scratch, stage, stage_bytes, emit);
}

}  // namespace kvs

// Attention statistics of one decoded layer and the online router score.
//
// The rank router reads attention statistics, entropy and peak, and runs online
// during generation, per token and per step ("DepthWeave-KV: Smarter KV Cache
// Compression by Sharing Across Layers and Adapting Per Token", Core Mechanism,
// second component; Key Concepts, Token-Conditional Depth Routing). The decode
// kernels keep every valid token's log2-domain scaled score s_{h,t} for the layer;
// with the layer's lse (exact weight sums) each weight is p_{h,t} = 2^(s - lse/ln 2).
// Each thread takes one token of one sequence (all of a pass's head scores loaded at once) and writes
//   mass[j][t]  = sum over the g heads of kv head j of p_{h,t}
//   score[t]    = x / (1 + x),  x = (T_b * sum_j mass[j][t]) / Hq     (fp32, in this order)
// Tokens past the sequence get mass 0 and score 0. Per head, each block reduces its
// entropy terms p (lse2 - s) ln 2 and its largest p in shared memory and stores one
// partial; a second small kernel (one block per sequence and head) adds the partials
// in a fixed order, so entropy and peak are deterministic.
#include "kvs_device.cuh"

namespace kvs {
namespace {

constexpr int NT = 128;
constexpr int HC = 32;                        // heads per pass: all their scores loaded at once
constexpr float LOG2E_F = 1.4426950408889634f;

// Reduces 32 per-lane values across the warp in 31 shuffles (16 + 8 + 4 + 2 + 1):
// at the step of width w every lane keeps the half of its values whose index has bit
// w equal to its own lane bit, adds the partner's copy of that half and sends the
// other half. Lane i ends with the total of index i in v[0]. Sum (MAX false) or max.
template <bool MAX>
__device__ __forceinline__ float warp_transpose_reduce(float (&v)[32], int lane) {
#pragma unroll
    for (int w = 16; w >= 1; w >>= 1) {
        const bool upper = (lane & w) != 0;
#pragma unroll
        for (int k = 0; k < w; ++k) {
            const float keep = upper ? v[k + w] : v[k];
            const float send = upper ? v[k] : v[k + w];
            const float got = __shfl_xor_sync(0xffffffffu, send, w);
            v[k] = MAX ? fmaxf(keep, got) : keep + got;
        }
    }
    return v[0];
}

// G: query heads per kv head when it divides HC (the groups then never straddle a
// pass and their bookkeeping is static), 0: any g, read at run time.
template <int G>
__global__ void __launch_bounds__(NT, 4) router_stats_kernel(const StatsArgs a) {
    static_assert(G == 0 || HC % G == 0, "groups inside one pass");
    // dependent launch: the decode's scores and lse are read only after it completes;
    // the next kernel may then be scheduled while this one runs
    grid_dep_wait();
    if (threadIdx.x == 0) grid_dep_launch();
    const int b = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int n = a.T;
    if (a.lens != nullptr) {
        n = a.lens[b];
        if (n < 0 || n > a.T) {
            if (threadIdx.x == 0 && blockIdx.x == 0) atomicOr(a.err, ERR_RANGE);
            n = n < 0 ? 0 : a.T;
        }
    }
    const bool want_red = a.entropy != nullptr || a.peak != nullptr;
    static_assert(HC == 32, "one head per lane in the block reduction");
    __shared__ float red_e[NT / 32][HC], red_p[NT / 32][HC];
    __shared__ float lse2_s[HC];
    const int t = blockIdx.x * NT + threadIdx.x;         // this thread's token
    const bool live = t < n;
    const float* srow = a.sscore + static_cast<size_t>(b) * a.Hq * a.T + t;
    float* mrow = a.mass != nullptr ? a.mass + static_cast<size_t>(b) * a.Hkv * a.T + t : nullptr;
    float macc = 0.f, total = 0.f;
    int hg = 0, j = 0;                                   // run-time grouping (G == 0): head j g + hg
    for (int h0 = 0; h0 < a.Hq; h0 += HC) {
        const int hn = min(HC, a.Hq - h0);
        if (threadIdx.x < hn) lse2_s[threadIdx.x] = a.lse[static_cast<size_t>(b) * a.Hq + h0 + threadIdx.x] * LOG2E_F;
        __syncthreads();
        // every score of the pass first, all loads in flight together
        float sv[HC];
#pragma unroll
        for (int q = 0; q < HC; ++q) sv[q] = (q < hn && live) ? __ldcs(srow + static_cast<size_t>(h0 + q) * a.T) : 0.f;
        // per head: the weight p (this thread's largest weight, one token) and the entropy
        // term p (lse2 - s); reduced over the block after the pass
        float es[HC], pm[HC];
#pragma unroll
        for (int q = 0; q < HC; ++q) {
            float p = 0.f, e = 0.f;
            if (q < hn && live) {
                const float x = sv[q] - lse2_s[q];
                p = ex2_approx(x);
                e = -p * x;
            }
            es[q] = e;
            pm[q] = p;
            if (G > 0) {
                macc = q % G == 0 ? p : macc + p;
                if (q % G == G - 1 && q < hn) {          // group complete: its mass, then the total
                    const int jj = (h0 + q) / G;
                    if (mrow != nullptr && t < a.T) mrow[static_cast<size_t>(jj) * a.T] = macc;
                    total = jj == 0 ? macc : __fadd_rn(total, macc);
                }
            } else if (q < hn) {
                macc = hg == 0 ? p : macc + p;
                if (hg == a.g - 1) {
                    if (mrow != nullptr && t < a.T) mrow[static_cast<size_t>(j) * a.T] = macc;
                    total = j == 0 ? macc : __fadd_rn(total, macc);
                    hg = 0;
                    ++j;
                } else {
                    ++hg;
                }
            }
        }
        if (want_red) {
            // lane q ends with head q's warp total and largest weight
            red_e[warp][lane] = warp_transpose_reduce<false>(es, lane);
            red_p[warp][lane] = warp_transpose_reduce<true>(pm, lane);
        }
        __syncthreads();
        if (want_red && threadIdx.x < hn) {
            float e = 0.f, p = 0.f;
            for (int w = 0; w < NT / 32; ++w) {
                e += red_e[w][threadIdx.x];
                p = fmaxf(p, red_p[w][threadIdx.x]);
            }
            float* part = a.part + ((static_cast<size_t>(b) * gridDim.x + blockIdx.x) * a.Hq + h0 + threadIdx.x) * 2;
            part[0] = e;
            part[1] = p;
        }
        __syncthreads();
    }
    if (a.score != nullptr && t < a.T) {
        float x = __fmul_rn(static_cast<float>(n), total);
        x = __fdiv_rn(x, static_cast<float>(a.Hq));
        a.score[static_cast<size_t>(b) * a.T + t] = __fdiv_rn(x, __fadd_rn(1.f, x));
    }
}

// Entropy and peak of every (sequence, head) from the per-block partials: thread i adds
// blocks i, i + 256, ... in order, then a fixed tree (shuffles, the warps in order).
constexpr int NF = 256;
__global__ void __launch_bounds__(NF) router_stats_final_kernel(const StatsArgs a, int blocks) {
    grid_dep_wait();
    if (threadIdx.x == 0) grid_dep_launch();
    const int h = blockIdx.x, b = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float e = 0.f, p = 0.f;
#pragma unroll 4
    for (int blk = threadIdx.x; blk < blocks; blk += NF) {
        const float2 v = *reinterpret_cast<const float2*>(a.part + ((static_cast<size_t>(b) * blocks + blk) * a.Hq + h) * 2);
        e += v.x;
        p = fmaxf(p, v.y);
    }
    e = warp_sum(e);
    p = warp_max(p);
    __shared__ float we[NF / 32], wp[NF / 32];
    if (lane == 0) {
        we[warp] = e;
        wp[warp] = p;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        float se = 0.f, sp = 0.f;
        for (int w = 0; w < NF / 32; ++w) {
            se += we[w];
            sp = fmaxf(sp, wp[w]);
        }
        const size_t o = static_cast<size_t>(b) * a.Hq + h;
        if (a.entropy != nullptr) a.entropy[o] = se * LN2_F;
        if (a.peak != nullptr) a.peak[o] = sp;
    }
}

}  // namespace

int router_stats_blocks(int T) { return (T + NT - 1) / NT; }

int launch_router_stats(const StatsArgs& a, cudaStream_t st) {
    const int blocks = router_stats_blocks(a.T);
    // both launches are dependent launches: their start overlaps the tail of the kernel
    // ahead, and they wait for it before touching memory
    auto kern = a.g == 4 ? router_stats_kernel<4> : a.g == 8 ? router_stats_kernel<8>
              : a.g == 2 ? router_stats_kernel<2> : a.g == 16 ? router_stats_kernel<16> : router_stats_kernel<0>;
    if (launch_kernel(kern, dim3(blocks, a.B), dim3(NT), 0, st, true, a) != cudaSuccess) return -1;
    if (a.entropy == nullptr && a.peak == nullptr) return 1;
    if (launch_kernel(router_stats_final_kernel, dim3(a.Hq, a.B), dim3(NF), 0, st, true, a, blocks) != cudaSuccess)
        return -1;
    return 2;
}

}  // namespace kvs

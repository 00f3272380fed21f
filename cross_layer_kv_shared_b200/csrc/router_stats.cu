// Attention statistics of one decoded layer and the online router score.
//
// The rank router reads attention statistics, entropy and peak, and runs online
// during generation, per token and per step ("DepthWeave-KV: Smarter KV Cache
// Compression by Sharing Across Layers and Adapting Per Token", Core Mechanism,
// second component; Key Concepts, Token-Conditional Depth Routing). The decode
// kernels keep every valid token's log2-domain scaled score s_{h,t} for the layer;
// with the layer's lse (exact weight sums) each weight is p_{h,t} = 2^(s - lse/ln 2).
// Each thread takes one token of one sequence (all of a pass's head scores loaded at
// once) and writes
//   mass[j][t]  = sum over the g heads of kv head j of p_{h,t}
//   score[t]    = x / (1 + x),  x = (T_b * sum_j mass[j][t]) / Hq     (fp32, in this order)
// Tokens past the sequence get mass 0 and score 0. The per-head entropy and peak need
// no pass of their own: the decode kernels carry them through their online softmax
// and split merge.
#include "kvs_device.cuh"

namespace kvs {
namespace {

constexpr int NT = 128;
constexpr int HC = 32;                        // heads per pass: all their scores loaded at once
constexpr float LOG2E_F = 1.4426950408889634f;

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
    int n = a.T;
    if (a.lens != nullptr) {
        n = a.lens[b];
        if (n < 0 || n > a.T) {
            if (threadIdx.x == 0 && blockIdx.x == 0) atomicOr(a.err, ERR_RANGE);
            n = n < 0 ? 0 : a.T;
        }
    }
    __shared__ float lse2_s[HC];
    const int t = blockIdx.x * NT + threadIdx.x;         // this thread's token
    const bool live = t < n;
    const float* srow = a.sscore + static_cast<size_t>(b) * a.Hq * a.T + t;
    float* mrow = a.mass != nullptr ? a.mass + static_cast<size_t>(b) * a.Hkv * a.T + t : nullptr;
    float macc = 0.f, total = 0.f;
    int hg = 0, j = 0;                                   // run-time grouping (G == 0): head j g + hg
    for (int h0 = 0; h0 < a.Hq; h0 += HC) {
        const int hn = min(HC, a.Hq - h0);
        // every score of the pass first, all loads in flight together (and in flight
        // while the heads' lse values are fetched and shared)
        float sv[HC];
#pragma unroll
        for (int q = 0; q < HC; ++q) sv[q] = (q < hn && live) ? __ldcs(srow + static_cast<size_t>(h0 + q) * a.T) : 0.f;
        if (threadIdx.x < hn) lse2_s[threadIdx.x] = a.lse[static_cast<size_t>(b) * a.Hq + h0 + threadIdx.x] * LOG2E_F;
        __syncthreads();
        // the weights, summed per kv head in head order
#pragma unroll
        for (int q = 0; q < HC; ++q) {
            const float p = (q < hn && live) ? ex2_approx(sv[q] - lse2_s[q]) : 0.f;
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
        __syncthreads();   // lse2_s is rewritten by the next pass
    }
    if (a.score != nullptr && t < a.T) {
        float x = __fmul_rn(static_cast<float>(n), total);
        x = __fdiv_rn(x, static_cast<float>(a.Hq));
        a.score[static_cast<size_t>(b) * a.T + t] = __fdiv_rn(x, __fadd_rn(1.f, x));
    }
}

}  // namespace

int launch_router_stats(const StatsArgs& a, cudaStream_t st) {
    const int blocks = (a.T + NT - 1) / NT;
    // a dependent launch: its start overlaps the tail of the decode ahead, and it waits
    // for the decode before touching memory
    auto kern = a.g == 4 ? router_stats_kernel<4> : a.g == 8 ? router_stats_kernel<8>
              : a.g == 2 ? router_stats_kernel<2> : a.g == 16 ? router_stats_kernel<16> : router_stats_kernel<0>;
    return launch_kernel(kern, dim3(blocks, a.B), dim3(NT), 0, st, true, a) == cudaSuccess ? 1 : -1;
}

}  // namespace kvs

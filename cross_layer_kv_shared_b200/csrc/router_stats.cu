// Attention statistics of one decoded layer and the online router score.
//
// The rank router reads attention statistics, entropy and peak, and runs online
// during generation, per token and per step ("DepthWeave-KV: Smarter KV Cache
// Compression by Sharing Across Layers and Adapting Per Token", Core Mechanism,
// second component; Key Concepts, Token-Conditional Depth Routing). The decode
// kernels keep every valid token's log2-domain scaled score s_{h,t} for the layer;
// with the layer's lse (exact weight sums) each weight is p_{h,t} = 2^(s - lse/ln 2).
// One thread per (sequence, token) then writes
//   mass[j][t]  = sum over the g heads of kv head j of p_{h,t}
//   score[t]    = x / (1 + x),  x = (T_b * sum_j mass[j][t]) / Hq     (fp32, in this order)
// and adds each head's entropy terms p (lse2 - s) ln 2 and peak candidates p into
// the per-head outputs (warp reductions, one atomic per warp and head). Tokens past
// the sequence get mass 0 and score 0.
#include "kvs_device.cuh"

namespace kvs {
namespace {

constexpr int NT = 256;
constexpr float LOG2E_F = 1.4426950408889634f;

__global__ void __launch_bounds__(NT) router_stats_kernel(const StatsArgs a) {
    const int b = blockIdx.y;
    const int t = blockIdx.x * NT + threadIdx.x;
    const int lane = threadIdx.x & 31;
    int n = a.T;
    if (a.lens != nullptr) {
        n = a.lens[b];
        if (n < 0 || n > a.T) {
            if (threadIdx.x == 0 && blockIdx.x == 0) atomicOr(a.err, ERR_RANGE);
            n = n < 0 ? 0 : a.T;
        }
    }
    const bool in_store = t < a.T;
    const bool valid = t < n;
    const bool want_ent = a.entropy != nullptr, want_peak = a.peak != nullptr;
    float total = 0.f;
    for (int j = 0; j < a.Hkv; ++j) {
        float mj = 0.f;
        for (int hh = 0; hh < a.g; ++hh) {
            const int h = j * a.g + hh;
            const size_t bh = static_cast<size_t>(b) * a.Hq + h;
            const float lse2 = a.lse[bh] * LOG2E_F;
            float p = 0.f, e = 0.f;
            if (valid) {
                const float s = a.sscore[bh * a.T + t];
                p = exp2f(s - lse2);
                e = p * (lse2 - s);
            }
            mj += p;
            if (want_ent) {
                const float es = warp_sum(e);
                if (lane == 0 && es != 0.f) atomicAdd(a.entropy + bh, es * LN2_F);
            }
            if (want_peak) {
                const float pm = warp_max(p);
                if (lane == 0 && pm > 0.f) atomicMax(reinterpret_cast<int*>(a.peak + bh), __float_as_int(pm));
            }
        }
        if (a.mass != nullptr && in_store) a.mass[(static_cast<size_t>(b) * a.Hkv + j) * a.T + t] = mj;
        total = j == 0 ? mj : __fadd_rn(total, mj);
    }
    if (a.score != nullptr && in_store) {
        float x = __fmul_rn(static_cast<float>(n), total);
        x = __fdiv_rn(x, static_cast<float>(a.Hq));
        a.score[static_cast<size_t>(b) * a.T + t] = __fdiv_rn(x, __fadd_rn(1.f, x));
    }
}

}  // namespace

cudaError_t launch_router_stats(const StatsArgs& a, cudaStream_t st) {
    dim3 grid((a.T + NT - 1) / NT, a.B);
    router_stats_kernel<<<grid, NT, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace kvs

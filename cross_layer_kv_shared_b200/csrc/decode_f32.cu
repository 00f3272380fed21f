// Split-KV GQA decode over a shared cache, fp32 storage, forms SINGLE and MIX.
//
// CUDA-core kernel for fp32 caches (small models, tests at fp32 tolerance):
// one CTA = one (split, kv head j, batch b), 128 threads, token chunks of 64.
//   scores: one warp per token, lanes split d, warp-shuffle sum per query head;
//           a MIX layer forms K~ = w K1 + (1-w) K2 element by element in fp32
//   softmax: per-head online max/sum in base 2 over the chunk
//   output: each thread owns (head, channel) pairs and accumulates p V~.
// Ends in finish_split like the bf16 kernels.
#include "kvs_device.cuh"

namespace kvs {
namespace {

constexpr int NT = 128;
constexpr int CH = 64;

template <int D, bool MIX>
__global__ void __launch_bounds__(NT) decode_f32_kernel(const DecodeArgs a) {
    // the query rows and a chunk's scores during the stream; the split merge's scratch after it
    constexpr int STREAM_FLOATS = MAX_GROUP * D + MAX_GROUP * CH;
    constexpr int MERGE_FLOATS = 4 * MAX_GROUP * F32_MAX_SPLITS;
    __shared__ float pool[STREAM_FLOATS > MERGE_FLOATS ? STREAM_FLOATS : MERGE_FLOATS];
    float (*sq)[D] = reinterpret_cast<float (*)[D]>(pool);
    float (*ss)[CH] = reinterpret_cast<float (*)[CH]>(pool + MAX_GROUP * D);
    float* scratch = pool;
    __shared__ float sm_m[MAX_GROUP], sm_l[MAX_GROUP], sm_z[MAX_GROUP], scorr[MAX_GROUP];
    __shared__ float fin_o[MAX_GROUP * D];
    __shared__ __align__(8) uint64_t never_bar;

    const int split = blockIdx.x;
    const int j = blockIdx.y;
    const int b = blockIdx.z;
    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int g = a.g;
    constexpr int OPT = (MAX_GROUP * D + NT - 1) / NT;     // (head, channel) pairs per thread

    if (a.stall && tid == 0) {
        mbar_init(&never_bar, 1);
        mbar_init_fence();
        mbar_wait_bounded(&never_bar, 0, a.stall_limit, a.err);
    }

    const size_t row_stride = static_cast<size_t>(a.T) * D;
    const size_t BH = static_cast<size_t>(a.B) * a.Hkv;
    const float* K1 = static_cast<const float*>(a.k) + (a.src0 * BH + static_cast<size_t>(b) * a.Hkv + j) * row_stride;
    const float* V1 = static_cast<const float*>(a.v) + (a.src0 * BH + static_cast<size_t>(b) * a.Hkv + j) * row_stride;
    const float* K2 = MIX ? static_cast<const float*>(a.k) + (a.src1 * BH + static_cast<size_t>(b) * a.Hkv + j) * row_stride : K1;
    const float* V2 = MIX ? static_cast<const float*>(a.v) + (a.src1 * BH + static_cast<size_t>(b) * a.Hkv + j) * row_stride : V1;
    const float w = MIX ? a.w[j] : 1.f;
    const float w1 = 1.f - w;

    const float* qb = static_cast<const float*>(a.q) + (static_cast<size_t>(b) * a.Hq + static_cast<size_t>(j) * g) * D;
    for (int idx = tid; idx < g * D; idx += NT) sq[idx / D][idx % D] = qb[idx];
    if (tid < g) {
        sm_m[tid] = NEG_INF;
        sm_l[tid] = 0.f;
        sm_z[tid] = 0.f;
    }
    const bool want_z = a.entropy != nullptr;   // sum of 2^(s - m) (m - s), for the entropy
    float acc[OPT];
#pragma unroll
    for (int i = 0; i < OPT; ++i) acc[i] = 0.f;
    __syncthreads();

    const int t0 = split * a.tiles_per_split * CH;
    const int t1 = min(seq_len(a, b), t0 + a.tiles_per_split * CH);
    float* srow = a.sscore != nullptr
                      ? a.sscore + (static_cast<size_t>(b) * a.Hq + static_cast<size_t>(j) * g) * a.T : nullptr;
    for (int c = t0; c < t1; c += CH) {
        const int n = min(CH, t1 - c);
        for (int tt = warp; tt < n; tt += NT / 32) {
            const size_t t = static_cast<size_t>(c + tt);
            float kv[D / 32];
#pragma unroll
            for (int i = 0; i < D / 32; ++i) {
                const int e = lane + 32 * i;
                kv[i] = MIX ? w * K1[t * D + e] + w1 * K2[t * D + e] : K1[t * D + e];
            }
            for (int h = 0; h < g; ++h) {
                float part = 0.f;
#pragma unroll
                for (int i = 0; i < D / 32; ++i) part += sq[h][lane + 32 * i] * kv[i];
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
                if (lane == 0) {
                    ss[h][tt] = part * a.scale_log2;
                    if (srow != nullptr) srow[static_cast<size_t>(h) * a.T + t] = part * a.scale_log2;
                }
            }
        }
        __syncthreads();
        if (tid < g) {
            const int h = tid;
            float mx = NEG_INF;
            for (int tt = 0; tt < n; ++tt) mx = fmaxf(mx, ss[h][tt]);
            const float mn = fmaxf(sm_m[h], mx);
            const float corr = exp2f(sm_m[h] - mn);
            float sum = 0.f, zs = 0.f;
            for (int tt = 0; tt < n; ++tt) {
                const float sv = ss[h][tt];
                const float p = exp2f(sv - mn);
                ss[h][tt] = p;
                sum += p;
                if (want_z) zs = fmaf(p, mn - sv, zs);
            }
            if (want_z) sm_z[h] = fmaf(corr, sm_m[h] != NEG_INF ? fmaf(sm_l[h], mn - sm_m[h], sm_z[h]) : 0.f, zs);
            sm_l[h] = sm_l[h] * corr + sum;
            sm_m[h] = mn;
            scorr[h] = corr;
        }
        __syncthreads();
#pragma unroll
        for (int i = 0; i < OPT; ++i) {
            const int idx = tid + i * NT;
            if (idx < g * D) {
                const int h = idx / D;
                const int e = idx % D;
                float s = acc[i] * scorr[h];
                for (int tt = 0; tt < n; ++tt) {
                    const size_t t = static_cast<size_t>(c + tt);
                    const float vv = MIX ? w * V1[t * D + e] + w1 * V2[t * D + e] : V1[t * D + e];
                    s += ss[h][tt] * vv;
                }
                acc[i] = s;
            }
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < OPT; ++i) {
        const int idx = tid + i * NT;
        if (idx < g * D) fin_o[idx] = acc[i];
    }
    __syncthreads();
    // the weights are fp32 throughout: the P.V sum and the exact sum are the same
    finish_split(a, D, b, j, split, sm_m, sm_l, sm_l, sm_z, fin_o, scratch, nullptr, 0);
}

template <int D, bool MIX>
cudaError_t launch_one(const DecodeArgs& a, cudaStream_t st) {
    dim3 grid(a.splits, a.Hkv, a.B);
    decode_f32_kernel<D, MIX><<<grid, NT, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace

int decode_f32_tile() { return CH; }

cudaError_t launch_decode_f32(bool mix, int d, const DecodeArgs& a, cudaStream_t st) {
    if (d == 64) return mix ? launch_one<64, true>(a, st) : launch_one<64, false>(a, st);
    return mix ? launch_one<128, true>(a, st) : launch_one<128, false>(a, st);
}

}  // namespace kvs

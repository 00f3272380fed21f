// Write side of the low-rank form: per-token rank routing and int8 residual codes.
//
// The DepthWeave-KV pages keep a per-layer low-rank residual that is
// quantised, at a per-token rank chosen by a router ("DepthWeave-KV: Smarter KV
// Cache Compression by Sharing Across Layers and Adapting Per Token", Core
// Mechanism and Framework Shift). The rule implemented, in fp32 with correctly
// rounded operations so the integers are reproducible bit for bit:
//   r      = 0 if score < 0.7f, 8 if score < 0.9f, else 16
//   amax   = max_{i<r} |u_i|
//   scale  = fp16_rne(min(amax / 127f, 65504f))
//   code_i = clamp(rint(u_i / scale), -127, 127) for i < r, 0 otherwise
//   a zero scale gives zero codes.
// One thread per (layer, batch, kv head, token) row of 16 values, for K and V.
#include "kvs_device.cuh"

namespace kvs {
namespace {

constexpr int RM = 16;

__device__ __forceinline__ uint8_t route(float s) { return s < 0.7f ? 0 : (s < 0.9f ? 8 : 16); }

__device__ __forceinline__ void quantize_row(const float* __restrict__ u, int r, int8_t* __restrict__ codes,
                                             uint16_t* __restrict__ scale) {
    float x[RM];
    const float4* u4 = reinterpret_cast<const float4*>(u);
#pragma unroll
    for (int i = 0; i < RM / 4; ++i) {
        const float4 v = u4[i];
        x[4 * i] = v.x; x[4 * i + 1] = v.y; x[4 * i + 2] = v.z; x[4 * i + 3] = v.w;
    }
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < RM; ++i)
        if (i < r) amax = fmaxf(amax, fabsf(x[i]));
    const float s32 = fminf(__fdiv_rn(amax, 127.f), 65504.f);
    const __half s16 = __float2half_rn(s32);
    const float sf = __half2float(s16);
    uint32_t packed[RM / 4];
#pragma unroll
    for (int i = 0; i < RM / 4; ++i) packed[i] = 0u;
#pragma unroll
    for (int i = 0; i < RM; ++i) {
        int c = 0;
        if (i < r && sf > 0.f) {
            const float q = rintf(__fdiv_rn(x[i], sf));
            c = static_cast<int>(fminf(fmaxf(q, -127.f), 127.f));
        }
        packed[i / 4] |= (static_cast<uint32_t>(c) & 0xffu) << (8 * (i % 4));
    }
    *reinterpret_cast<uint4*>(codes) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
    *scale = __half_as_ushort(s16);
}

__global__ void __launch_bounds__(256) pack_residual_kernel(const PackArgs a) {
    const long long rows = a.tokens * a.Hkv;     // (l, b, h, t) rows
    for (long long idx = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; idx < rows;
         idx += static_cast<long long>(gridDim.x) * blockDim.x) {
        // idx = ((lb * Hkv) + h) * T + t with lb = l * B + b
        const long long t = idx % a.T;
        const long long lbh = idx / a.T;
        const long long h = lbh % a.Hkv;
        const long long lb = lbh / a.Hkv;
        const long long tok = lb * a.T + t;
        const uint8_t r = route(a.score[tok]);
        if (h == 0) a.rank[tok] = r;
        quantize_row(a.u_k + idx * RM, r, a.u_k8 + idx * RM, a.s_k + idx);
        quantize_row(a.u_v + idx * RM, r, a.u_v8 + idx * RM, a.s_v + idx);
    }
}

}  // namespace

cudaError_t launch_pack_residual(const PackArgs& a, cudaStream_t st) {
    const long long rows = a.tokens * a.Hkv;
    long long blocks = (rows + 255) / 256;
    if (blocks > 148LL * 32) blocks = 148LL * 32;
    if (blocks < 1) blocks = 1;
    pack_residual_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace kvs

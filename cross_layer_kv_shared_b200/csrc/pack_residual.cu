// Write side of the low-rank form: per-token rank routing and int8 residual codes for
// every cached token (the rule is in kvs_quant.cuh). One thread per (layer, batch,
// kv head, token) row of 16 values, for K and V.
#include "kvs_quant.cuh"

namespace kvs {
namespace {

constexpr int RM = QUANT_RM;

__device__ __forceinline__ void quantize_row(const float* __restrict__ u, int r, int8_t* __restrict__ codes,
                                             uint16_t* __restrict__ scale) {
    float x[RM];
    const float4* u4 = reinterpret_cast<const float4*>(u);
#pragma unroll
    for (int i = 0; i < RM / 4; ++i) {
        const float4 v = u4[i];
        x[4 * i] = v.x; x[4 * i + 1] = v.y; x[4 * i + 2] = v.z; x[4 * i + 3] = v.w;
    }
    uint32_t packed[4];
    uint16_t sc;
    quantize16(x, r, packed, sc);
    *reinterpret_cast<uint4*>(codes) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
    *scale = sc;
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
        const uint8_t r = route_rank(a.score[tok]);
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

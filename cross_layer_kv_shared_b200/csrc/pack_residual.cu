// Write side of the low-rank form: per-token rank routing and int8 residual codes for
// every cached token (the rule and the group-packed code layout are in kvs_quant.cuh).
// One warp per code group (32 tokens of one layer, sequence and kv head), for K and V.
#include "kvs_quant.cuh"

namespace kvs {
namespace {

constexpr int RM = QUANT_RM;

__device__ __forceinline__ void load_row(const float* __restrict__ u, float (&x)[RM]) {
    const float4* u4 = reinterpret_cast<const float4*>(u);
#pragma unroll
    for (int i = 0; i < RM / 4; ++i) {
        const float4 v = u4[i];
        x[4 * i] = v.x; x[4 * i + 1] = v.y; x[4 * i + 2] = v.z; x[4 * i + 3] = v.w;
    }
}

// One warp per code group of one (layer, sequence, kv head) row: lane = token. The
// group's ranks are scanned across the lanes to place each token's codes.
__global__ void __launch_bounds__(256) pack_residual_kernel(const PackArgs a) {
    const int lane = threadIdx.x & 31;
    const long long groups_per_row = (a.T + CODE_GROUP - 1) / CODE_GROUP;
    const long long tasks = a.tokens / a.T * a.Hkv * groups_per_row;   // (l, b, h, group)
    const long long warps = static_cast<long long>(gridDim.x) * (blockDim.x >> 5);
    for (long long w = blockIdx.x * static_cast<long long>(blockDim.x >> 5) + (threadIdx.x >> 5); w < tasks;
         w += warps) {
        const long long grp = w % groups_per_row;
        const long long lbh = w / groups_per_row;     // (l * B + b) * Hkv + h
        const long long h = lbh % a.Hkv;
        const long long lb = lbh / a.Hkv;
        const long long t = grp * CODE_GROUP + lane;
        const bool valid = t < a.T;
        const long long tok = lb * a.T + t;
        const long long row = lbh * a.T + t;          // (l, b, h, t) row of the inputs and scales
        const uint8_t r = valid ? route_rank(a.score[tok]) : 0;
        if (valid && h == 0) a.rank[tok] = r;
        // exclusive scan of the code lengths over the group
        const int k = code_len(r);
        int o = k;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, o, d);
            if (lane >= d) o += n;
        }
        o -= k;
        if (!valid) continue;
        const long long gbase = (lbh * a.T + grp * CODE_GROUP) * RM;   // the group's first byte
        float x[RM];
        uint32_t packed[4];
        uint16_t sc;
        load_row(a.u_k + row * RM, x);
        quantize16(x, r, packed, sc);
        store_codes(a.u_k8 + gbase + o, packed, k);
        a.s_k[row] = sc;
        load_row(a.u_v + row * RM, x);
        quantize16(x, r, packed, sc);
        store_codes(a.u_v8 + gbase + o, packed, k);
        a.s_v[row] = sc;
    }
}

}  // namespace

cudaError_t launch_pack_residual(const PackArgs& a, cudaStream_t st) {
    const long long rows = a.tokens / a.T * a.Hkv * ((a.T + CODE_GROUP - 1) / CODE_GROUP) * CODE_GROUP;
    long long blocks = (rows + 255) / 256;
    if (blocks > 148LL * 32) blocks = 148LL * 32;
    if (blocks < 1) blocks = 1;
    pack_residual_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace kvs

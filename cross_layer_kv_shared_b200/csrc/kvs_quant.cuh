// The residual quantiser of the low-rank form, shared by the packer and the append.
//
// In fp32 with correctly rounded operations, so the integers are reproducible bit for
// bit ("DepthWeave-KV: Smarter KV Cache Compression by Sharing Across Layers and
// Adapting Per Token", Core Mechanism diagram: a low-rank, quantised residual; the
// rule itself is this library's reading):
//   r      = 0 if score < 0.7f, 8 if score < 0.9f, else 16
//   amax   = max_{i<r} |u_i|
//   scale  = fp16_rne(min(amax / 127f, 65504f))
//   code_i = clamp(rint(u_i / scale), -127, 127) for i < r, 0 otherwise
//   a zero scale gives zero codes.
#pragma once

#include "kvs_device.cuh"

namespace kvs {

constexpr int QUANT_RM = 16;

// Residual code store ("group-packed"). A (layer, sequence, kv head) row of a code
// store holds T x 16 bytes. Its tokens form groups of CODE_GROUP = 32 (group g: tokens
// 32 g .. 32 g + 31, the last group possibly shorter), and group g owns the bytes
// [512 g, 512 g + 16 n_g) of the row. Inside a group the tokens' code slots follow one
// another in token order: token t takes k_t = 8 ceil(min(r_t, 16) / 8) bytes (0, 8 or
// 16) holding its first min(r_t, 16) codes and then zeros, at byte o_t of the group,
// o_t the sum of k over the group's earlier tokens (so every slot is 8-byte aligned).
// The group's other bytes are unused. A reader fetches a group's first
// pad16(sum over the group of k) bytes: the codes of rank-0 tokens are never stored,
// and a rank-8 token costs 8 bytes instead of 16.
constexpr int CODE_GROUP = 32;
__device__ __forceinline__ int code_len(unsigned r) { return r == 0u ? 0 : (r <= 8u ? 8 : 16); }

// a token's code slot (k = 0, 8 or 16 bytes, 8-byte aligned) from `packed` (code i in byte i)
__device__ __forceinline__ void store_codes(int8_t* dst, const uint32_t (&packed)[4], int k) {
    if (k >= 8) *reinterpret_cast<uint2*>(dst) = make_uint2(packed[0], packed[1]);
    if (k == 16) *reinterpret_cast<uint2*>(dst + 8) = make_uint2(packed[2], packed[3]);
}

// 16 bytes from an 8-byte aligned slot in shared memory (the bytes past the token's own
// codes belong to the next slot, or are unused, and are masked by its rank afterwards)
__device__ __forceinline__ uint4 codes_at(const uint8_t* slot) {
    const uint2 a = *reinterpret_cast<const uint2*>(slot);
    const uint2 b = *reinterpret_cast<const uint2*>(slot + 8);
    return make_uint4(a.x, a.y, b.x, b.y);
}

__device__ __forceinline__ uint8_t route_rank(float s) { return s < 0.7f ? 0 : (s < 0.9f ? 8 : 16); }

// 16 residual values at rank r -> four words of int8 codes (byte i = code i) and the fp16 scale bits
__device__ __forceinline__ void quantize16(const float (&x)[QUANT_RM], int r, uint32_t (&packed)[4], uint16_t& scale) {
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < QUANT_RM; ++i)
        if (i < r) amax = fmaxf(amax, fabsf(x[i]));
    const float s32 = fminf(__fdiv_rn(amax, 127.f), 65504.f);
    const __half s16 = __float2half_rn(s32);
    const float sf = __half2float(s16);
#pragma unroll
    for (int i = 0; i < 4; ++i) packed[i] = 0u;
#pragma unroll
    for (int i = 0; i < QUANT_RM; ++i) {
        int c = 0;
        if (i < r && sf > 0.f) {
            const float q = rintf(__fdiv_rn(x[i], sf));
            c = static_cast<int>(fminf(fmaxf(q, -127.f), 127.f));
        }
        packed[i / 4] |= (static_cast<uint32_t>(c) & 0xffu) << (8 * (i % 4));
    }
    scale = __half_as_ushort(s16);
}

}  // namespace kvs

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

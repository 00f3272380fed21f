// GPU twin of synth/philox.py: identical bits for every element (see include/kvsynth.h).
// Only seeded random numbers are made here.
#include "kvsynth.h"

#include <cuda_runtime.h>
#include <stdint.h>

namespace {

constexpr int ATANH_TERMS = 13;
constexpr int TRIG_TERMS = 14;

struct SeriesCoeffs {
    double at[ATANH_TERMS];   // 1/(2k+1)
    double sn[TRIG_TERMS];    // (-1)^k / (2k+1)!
    double cs[TRIG_TERMS];    // (-1)^k / (2k)!
};

__device__ __forceinline__ void philox4x32_10(uint32_t c[4], uint32_t k0, uint32_t k1) {
    const uint32_t M0 = 0xD2511F53u, M1 = 0xCD9E8D57u, W0 = 0x9E3779B9u, W1 = 0xBB67AE85u;
#pragma unroll
    for (int r = 0; r < 10; ++r) {
        const uint32_t hi0 = __umulhi(M0, c[0]), lo0 = M0 * c[0];
        const uint32_t hi1 = __umulhi(M1, c[2]), lo1 = M1 * c[2];
        const uint32_t n0 = hi1 ^ c[1] ^ k0, n2 = hi0 ^ c[3] ^ k1;
        c[0] = n0; c[1] = lo1; c[2] = n2; c[3] = lo0;
        k0 += W0;
        k1 += W1;
    }
}

// ln((w0 + 1) * 2^-32) by the atanh series, one IEEE fp64 operation at a time
__device__ double series_log(uint32_t w0, const SeriesCoeffs& C) {
    const uint64_t n = static_cast<uint64_t>(w0) + 1ull;
    int e = 63 - __clzll(static_cast<long long>(n));
    double m = __ddiv_rn(static_cast<double>(n), static_cast<double>(1ull << e));
    if (m > 1.4142135623730951) {
        m = __dmul_rn(m, 0.5);
        e += 1;
    }
    const double y = __ddiv_rn(__dadd_rn(m, -1.0), __dadd_rn(m, 1.0));
    const double y2 = __dmul_rn(y, y);
    double acc = C.at[ATANH_TERMS - 1];
    for (int k = ATANH_TERMS - 2; k >= 0; --k) acc = __dadd_rn(__dmul_rn(acc, y2), C.at[k]);
    const double lnm = __dmul_rn(__dmul_rn(2.0, y), acc);
    return __dadd_rn(__dmul_rn(static_cast<double>(e - 32), 0.6931471805599453), lnm);
}

__device__ void series_sincos(uint32_t w1, const SeriesCoeffs& C, double* cos_t, double* sin_t) {
    const uint32_t quad = w1 >> 30;
    const double frac = __dmul_rn(static_cast<double>(w1 & 0x3FFFFFFFu), 9.313225746154785e-10);  // 2^-30
    const double phi = __dmul_rn(frac, 1.5707963267948966);
    const double p2 = __dmul_rn(phi, phi);
    double sa = C.sn[TRIG_TERMS - 1];
    double ca = C.cs[TRIG_TERMS - 1];
    for (int k = TRIG_TERMS - 2; k >= 0; --k) {
        sa = __dadd_rn(__dmul_rn(sa, p2), C.sn[k]);
        ca = __dadd_rn(__dmul_rn(ca, p2), C.cs[k]);
    }
    const double s = __dmul_rn(phi, sa);
    const double c = ca;
    switch (quad) {
        case 0: *cos_t = c; *sin_t = s; break;
        case 1: *cos_t = -s; *sin_t = c; break;
        case 2: *cos_t = -c; *sin_t = -s; break;
        default: *cos_t = s; *sin_t = -c; break;
    }
}

__device__ __forceinline__ uint16_t f32_to_bf16_rne(float f) {
    const uint32_t u = __float_as_uint(f);
    return static_cast<uint16_t>((u + 0x7FFFu + ((u >> 16) & 1u)) >> 16);
}

__global__ void normal_kernel(void* out, int dtype, uint64_t count, uint64_t offset, uint32_t seed, uint32_t tid,
                              double scale, const SeriesCoeffs C) {
    const uint64_t first_blk = offset >> 2;
    const uint64_t last_blk = (offset + count + 3) >> 2;
    for (uint64_t blk = first_blk + blockIdx.x * static_cast<uint64_t>(blockDim.x) + threadIdx.x; blk < last_blk;
         blk += static_cast<uint64_t>(gridDim.x) * blockDim.x) {
        uint32_t c[4] = {static_cast<uint32_t>(blk), static_cast<uint32_t>(blk >> 32), 0u, 0u};
        philox4x32_10(c, seed, tid);
        double z[4];
#pragma unroll
        for (int p = 0; p < 2; ++p) {
            const double r = __dsqrt_rn(__dmul_rn(-2.0, series_log(c[2 * p], C)));
            double ct, st;
            series_sincos(c[2 * p + 1], C, &ct, &st);
            z[2 * p] = __dmul_rn(r, ct);
            z[2 * p + 1] = __dmul_rn(r, st);
        }
#pragma unroll
        for (int l = 0; l < 4; ++l) {
            const uint64_t i = blk * 4 + l;
            if (i < offset || i >= offset + count) continue;
            const float f = __double2float_rn(__dmul_rn(z[l], scale));
            if (dtype == 0)
                static_cast<float*>(out)[i - offset] = f;
            else
                static_cast<uint16_t*>(out)[i - offset] = f32_to_bf16_rne(f);
        }
    }
}

__global__ void uniform_kernel(float* out, uint64_t count, uint64_t offset, uint32_t seed, uint32_t tid) {
    const uint64_t first_blk = offset >> 2;
    const uint64_t last_blk = (offset + count + 3) >> 2;
    for (uint64_t blk = first_blk + blockIdx.x * static_cast<uint64_t>(blockDim.x) + threadIdx.x; blk < last_blk;
         blk += static_cast<uint64_t>(gridDim.x) * blockDim.x) {
        uint32_t c[4] = {static_cast<uint32_t>(blk), static_cast<uint32_t>(blk >> 32), 0u, 0u};
        philox4x32_10(c, seed, tid);
#pragma unroll
        for (int l = 0; l < 4; ++l) {
            const uint64_t i = blk * 4 + l;
            if (i < offset || i >= offset + count) continue;
            out[i - offset] = static_cast<float>(c[l] >> 8) * 5.9604644775390625e-08f;   // 2^-24
        }
    }
}

SeriesCoeffs make_coeffs() {
    SeriesCoeffs C;
    for (int k = 0; k < ATANH_TERMS; ++k) C.at[k] = 1.0 / static_cast<double>(2 * k + 1);
    double s = 1.0, c = 1.0;
    C.sn[0] = 1.0;
    C.cs[0] = 1.0;
    for (int k = 1; k < TRIG_TERMS; ++k) {
        s = s / static_cast<double>((2 * k) * (2 * k + 1));
        c = c / static_cast<double>((2 * k - 1) * (2 * k));
        C.sn[k] = (k % 2 == 0) ? s : -s;
        C.cs[k] = (k % 2 == 0) ? c : -c;
    }
    return C;
}

unsigned grid_for(uint64_t blocks) {
    uint64_t g = (blocks + 255) / 256;
    if (g > 148ull * 64) g = 148ull * 64;
    return static_cast<unsigned>(g < 1 ? 1 : g);
}

}  // namespace

extern "C" int kvsynth_normal(void* out, int dtype, uint64_t count, uint64_t offset, uint32_t seed,
                              uint32_t tensor_id, double scale, void* stream) {
    if (count == 0) return 0;
    if (out == nullptr || (dtype != 0 && dtype != 1)) return static_cast<int>(cudaErrorInvalidValue);
    static const SeriesCoeffs C = make_coeffs();
    const uint64_t blocks = ((offset + count + 3) >> 2) - (offset >> 2);
    normal_kernel<<<grid_for(blocks), 256, 0, static_cast<cudaStream_t>(stream)>>>(out, dtype, count, offset, seed,
                                                                                  tensor_id, scale, C);
    return static_cast<int>(cudaGetLastError());
}

extern "C" int kvsynth_uniform_f32(float* out, uint64_t count, uint64_t offset, uint32_t seed, uint32_t tensor_id,
                                   void* stream) {
    if (count == 0) return 0;
    if (out == nullptr) return static_cast<int>(cudaErrorInvalidValue);
    const uint64_t blocks = ((offset + count + 3) >> 2) - (offset >> 2);
    uniform_kernel<<<grid_for(blocks), 256, 0, static_cast<cudaStream_t>(stream)>>>(out, count, offset, seed,
                                                                                   tensor_id);
    return static_cast<int>(cudaGetLastError());
}

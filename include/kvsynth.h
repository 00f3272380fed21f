/*
 * kvsynth.h - seeded synthetic inputs on the GPU (libkvsynth.so).
 *
 * Fills device buffers with the same bits as the numpy generator in
 * synth/philox.py (Philox4x32-10 counter stream keyed by (seed, tensor id);
 * Box-Muller normals with series ln/sin/cos in plain IEEE fp64 operations;
 * fp32 round-to-nearest-even, then bf16 round-to-nearest-even). It holds no
 * attention arithmetic; it only makes test and benchmark inputs, shaped like
 * the workloads of the shared-KV pages, without copying gigabytes from the host.
 *
 * Element i of a tensor (flat index, counting from 0 at the tensor start) is
 * written to out[i - offset] for i in [offset, offset + count).
 * `stream` is a cudaStream_t (void*, NULL = legacy default stream); calls are
 * asynchronous. Return value: 0, or the cudaError_t of the failed launch.
 * Pointers are caller-owned device memory, aligned to the element size.
 */
#ifndef KVSYNTH_H
#define KVSYNTH_H
#include <stdint.h>
#ifdef __cplusplus
extern "C" {
#endif

/* N(0,1) * scale. dtype 0: float32 out; dtype 1: bf16 bit patterns (uint16) out. */
int kvsynth_normal(void* out, int dtype, uint64_t count, uint64_t offset, uint32_t seed, uint32_t tensor_id,
                   double scale, void* stream);

/* U[0,1) float32 with 24 random bits: (word >> 8) * 2^-24. */
int kvsynth_uniform_f32(float* out, uint64_t count, uint64_t offset, uint32_t seed, uint32_t tensor_id,
                        void* stream);

#ifdef __cplusplus
}
#endif
#endif /* KVSYNTH_H */

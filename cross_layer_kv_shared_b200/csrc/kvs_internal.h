// Internal declarations shared by the host library and the kernels of libkvshare.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

namespace kvs {

// bits of the device status word
constexpr unsigned ERR_TIMEOUT = 1u;
constexpr unsigned ERR_RANGE = 2u;     // a per-sequence length outside [0, context] (clamped)

// one split partial: o[d] (un-normalised, relative to m), m (log2 domain), l
constexpr int MAX_SPLITS = 160;
constexpr int F32_MAX_SPLITS = 128;   // the fp32 kernel merges from static shared memory
constexpr int MAX_GROUP = 16;

// Arguments of one decode launch (one layer). Pointers are already offset to the layer.
struct DecodeArgs {
    const void* q;          // [B][Hq][d] config dtype
    float* out;             // [B][Hq][d]
    float* lse;             // [B][Hq] or nullptr
    const void* k;          // store base [slots][B][Hkv][T][d] (used by the fp32 kernel)
    const void* v;
    int src0, src1;         // slots (SINGLE/MIX)
    const float* w;         // [Hkv] mix weights of this layer (device), MIX only
    int B, Hq, Hkv, T, g;   // T: tokens each store holds (row stride of the cache)
    const int* lens;        // [B] tokens of each sequence (device), or nullptr: all T
    float* sscore;          // [B][Hq][T] log2-domain scaled scores for the statistics, or nullptr
    float* entropy;         // [B][Hq] attention entropy (nats) of every head, or nullptr
    float* peak;            // [B][Hq] largest attention weight of every head, or nullptr
    int splits;             // splits per (b, kv head)            (split-grid kernels)
    int tiles_per_split;    // token tiles per split               (split-grid kernels)
    int units;              // B * Hkv                             (balanced-grid kernels)
    int n_t;                // token tiles per unit                (balanced-grid kernels)
    float scale_log2;       // softmax scale * log2(e)
    float* ws;              // split partials: [g][d + 4] each (o, m, l, lx, z)
    unsigned* counters;     // [B*Hkv] arrival counters, zero between launches
    unsigned* err;          // device status word
    long long wait_limit;   // clock cycles a bounded wait may spin
    int stall;              // test hook: one warp waits on a barrier nothing arrives on
    long long stall_limit;
    // form (c)
    int pair;               // basis pair
    const void* coef_k; const void* coef_v;     // pair's [B][Hkv][T][Rb]
    const void* basis_k; const void* basis_v;   // pair's [Hkv][Rb][d]
    const int8_t* u_k; const int8_t* u_v;       // layer's [B][Hkv][T][Rm]
    const uint16_t* s_k; const uint16_t* s_v;   // layer's [B][Hkv][T]
    const void* r_k; const void* r_v;           // layer's [Hkv][Rm][d]
    const uint8_t* rank;                        // layer's [B][T]
    int Rb, Rm;
    // launch with programmatic stream serialization: the kernel may be scheduled while
    // the previous kernel on the stream drains, and waits (griddepcontrol.wait) before
    // its first global memory access
    int pdl;
    // the caller guarantees no kernel ahead on the stream writes the cache: the first
    // K/V tiles may be requested before the wait on the previous kernel
    int kv_early;
};

// One-time set-up of a kernel on the current device (the dynamic shared-memory limit is
// a per-device function attribute): `setup()` runs the first time this kernel is
// launched on each device; `done` is the kernel's own device bit mask.
template <typename Setup>
inline cudaError_t once_per_device(std::atomic<unsigned long long>& done, Setup setup) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const unsigned long long bit = 1ull << (dev & 63);
    if (done.load(std::memory_order_acquire) & bit) return cudaSuccess;
    e = setup();
    if (e == cudaSuccess) done.fetch_or(bit, std::memory_order_acq_rel);
    return e;
}

// cudaLaunchKernelEx with the programmatic-stream-serialization attribute when `pdl`
template <typename... KArgs, typename... Args>
inline cudaError_t launch_kernel(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                                 bool pdl, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<Args&&>(args)...);
}

// Attention statistics of one decoded layer from its kept scores and lse.
struct StatsArgs {
    const float* sscore;    // [B][Hq][T] log2-domain scaled scores
    const float* lse;       // [B][Hq] natural-log lse of the layer
    const int* lens;        // [B] or nullptr
    float* mass;            // [B][Hkv][T] or nullptr
    float* score;           // [B][T] or nullptr
    unsigned* err;
    int B, Hq, Hkv, T, g;
};
// launches the per-token statistics kernel (mass and router score); returns the number
// of launches, or -1 on a launch error
int launch_router_stats(const StatsArgs& a, cudaStream_t st);

// Append of one new token to a low-rank cache (every basis pair, sequence and kv head).
constexpr int APPEND_MAX_PAIRS = 64;
struct AppendArgs {
    const uint16_t* k_new; const uint16_t* v_new;   // [L][B][Hkv][d] bf16: the token in every layer
    const float* score;                             // [L][B] router score of the token per layer
    const int* pos;                                 // [B] token index written in each sequence
    const uint16_t* basis_k; const uint16_t* basis_v;   // [P][Hkv][Rb][d]
    const uint16_t* r_k; const uint16_t* r_v;           // [L][Hkv][16][d]
    uint16_t* coef_k; uint16_t* coef_v;                 // [P][B][Hkv][T][Rb]
    int8_t* u_k; int8_t* u_v;                           // [L][B][Hkv][T][16]
    uint16_t* s_k; uint16_t* s_v;                       // [L][B][Hkv][T]
    uint8_t* rank;                                      // [L][B][T]
    unsigned* err;
    int P, B, Hkv, T, d, Rb;
    int pair_layers[2 * APPEND_MAX_PAIRS];              // the two layers of each pair (-1: unused)
};
cudaError_t launch_append_lowrank(const AppendArgs& a, cudaStream_t st);

struct PackArgs {
    const float* score; const float* u_k; const float* u_v;
    uint8_t* rank; int8_t* u_k8; int8_t* u_v8; uint16_t* s_k; uint16_t* s_v;
    long long tokens;       // L * B * T
    int Hkv, T, Rm;
};

struct PrefillArgs {
    const void* q;          // layer's [B][Hq][S][d] bf16
    void* out;              // layer's [B][Hq][S][d] bf16
    float* lse;             // layer's [B][Hq][S] or nullptr
    int src0, src1, mix;
    const float* w;         // [Hkv] (device) when mix
    int B, Hq, Hkv, S, T, g;
    float scale_log2;
    unsigned* err;
    long long wait_limit;
};

// Low-rank causal prefill of one layer (absorbed form, basis rank 32).
constexpr int LR_QW = 64;   // width of a projected query row: B_K q (32) | R_K q (16) | 0 (16)
struct PrefillLrArgs {
    const uint16_t* q;          // layer's [B][Hq][S][d] bf16
    uint16_t* qp;               // [B][Hq][S][LR_QW] bf16 projected queries (written by the pre-pass)
    float* lse;                 // layer's [B][Hq][S] or nullptr
    const uint16_t* basis_k;    // pair's [Hkv][32][d]
    const uint16_t* basis_v;
    const uint16_t* r_k;        // layer's [Hkv][16][d]
    const uint16_t* r_v;
    const uint16_t* s_k;        // layer's [B][Hkv][T] fp16
    const uint16_t* s_v;
    const uint8_t* rank;        // layer's [B][T]
    int pair;                   // basis pair (row block of the coefficient maps)
    int B, Hq, Hkv, S, T, g, d;
    float scale_log2;
    unsigned* err;
    long long wait_limit;
};
cudaError_t launch_lr_qproj(const PrefillLrArgs& a, cudaStream_t st);
// maps: Q' [B*Hq][S][64], O [B*Hq][S][d], C_K, C_V [P*B*Hkv][T][32], U_K, U_V [B*Hkv][T][16] (the layer's)
cudaError_t launch_prefill_lowrank(int d, const CUtensorMap* maps, const PrefillLrArgs& a, cudaStream_t st);
// tokens per K/V tile of the low-rank prefill: the row count of its coefficient and
// code tensor-map boxes
int prefill_lowrank_tile();

// kernel launchers (return cudaGetLastError() of the launch)
struct TileShape { int tt; int nsw; int smem; };
TileShape decode_bf16_shape(int d, bool mix);
cudaError_t launch_decode_bf16(int d, bool mix, const CUtensorMap& tmK, const CUtensorMap& tmV,
                               const DecodeArgs& a, cudaStream_t st);
int decode_bf16_ctas_per_sm(int d, bool mix);

int decode_f32_tile();
cudaError_t launch_decode_f32(bool mix, int d, const DecodeArgs& a, cudaStream_t st);

int decode_lowrank_tile(int rb);
int decode_lowrank_occupancy(int d, int rb);
// maps: coef_k, coef_v (whole [P*B*Hkv][T][Rb]); the group-packed codes come through a.u_k, a.u_v
cudaError_t launch_decode_lowrank(int d, int rb, const DecodeArgs& a, const CUtensorMap* maps, cudaStream_t st);

cudaError_t launch_pack_residual(const PackArgs& a, cudaStream_t st);

int prefill_kv_tile(int d, bool mix);
cudaError_t launch_prefill(int d, bool mix, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                           const CUtensorMap& to, const PrefillArgs& a, cudaStream_t st);

}  // namespace kvs

// One-layer bf16 decode that allocates no device memory (kvshare_decode_layer_noalloc).
//
// kvshare_decode keeps its split-KV partials and arrival counters in a
// workspace that kvshare_create allocates with cudaMalloc. Some callers cannot
// allocate at all: code running inside a captured or replayed region they do
// not own, plug-ins of a host framework whose allocator is the only one allowed
// to hand out device memory, or processes that must not grow their footprint
// after start-up. This entry point runs the same split-KV decode kernel with
// its scratch in a fixed, file-scope device array instead, so the caller only
// passes inputs and outputs.
//
// The scratch: KVS_NOALLOC_SCRATCH_BYTES (2 MiB) of device memory that every
// GPU which loads this library holds until the process exits. It holds the
// arrival counters (one per batch x kv-head unit, at most KVS_NOALLOC_MAX_UNITS),
// a status word, and the split partials. Requests with more units are rejected;
// the CTA count is lowered until the partials fit.
#include "kvshare.h"

#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstring>
#include <mutex>

#include "kvs_internal.h"

using namespace kvs;

namespace {

constexpr size_t KVS_NOALLOC_SCRATCH_BYTES = size_t(2) << 20;
constexpr int KVS_NOALLOC_MAX_UNITS = 4096;
constexpr size_t COUNTER_BYTES = KVS_NOALLOC_MAX_UNITS * sizeof(unsigned);
constexpr size_t STATUS_BYTES = 256;
constexpr size_t PARTIAL_FLOATS = (KVS_NOALLOC_SCRATCH_BYTES - COUNTER_BYTES - STATUS_BYTES) / sizeof(float);

// The scratch itself. In host code this name is only a stand-in for the
// device symbol; its device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[KVS_NOALLOC_SCRATCH_BYTES];

constexpr int MAX_DEVICES = 64;
std::mutex g_setup_mutex;
unsigned char* g_scratch_addr[MAX_DEVICES] = {};

// Device address of the scratch on the current device, looked up once per device.
cudaError_t scratch_address(int device, unsigned char** out) {
    if (device < 0 || device >= MAX_DEVICES) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (g_scratch_addr[device] == nullptr) {
        void* p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_addr[device] = static_cast<unsigned char*>(p);
    }
    *out = g_scratch_addr[device];
    return cudaSuccess;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encoder() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

bool store_map(const void* base, int D, int T, int rows, int tt, CUtensorMap* m) {
    EncodeTiledFn fn = encoder();
    if (fn == nullptr) return false;
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)T, (cuuint64_t)rows};
    cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)T * D * 2};
    cuuint32_t box[3] = {64u, (cuuint32_t)tt, 1u};
    cuuint32_t estr[3] = {1u, 1u, 1u};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool device_ptr(const void* p, uintptr_t align) {
    if (p == nullptr || (reinterpret_cast<uintptr_t>(p) & (align - 1)) != 0) return false;
    cudaPointerAttributes at;
    if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    return at.type == cudaMemoryTypeDevice || at.type == cudaMemoryTypeManaged;
}

}  // namespace

extern "C" kvshare_status kvshare_decode_layer_noalloc(const void* q, const void* k, const void* v, const float* w,
                                                       float* out, float* lse, int batch, int num_q_heads,
                                                       int num_kv_heads, int head_dim, int context, int slots,
                                                       int src0, int src1, void* stream) {
    if (batch < 1 || num_kv_heads < 1 || num_q_heads < 1 || context < 1 || slots < 1) return KVS_EINVAL;
    if (num_q_heads % num_kv_heads != 0) return KVS_EINVAL;
    if (head_dim != 64 && head_dim != 128) return KVS_EUNSUPPORTED;
    const int g = num_q_heads / num_kv_heads;
    if (g > MAX_GROUP) return KVS_EUNSUPPORTED;
    const bool mix = src1 >= 0;
    if (src0 < 0 || src0 >= slots || src1 >= slots || (mix && src1 == src0)) return KVS_EINVAL;
    const long long units = static_cast<long long>(batch) * num_kv_heads;
    if (units > KVS_NOALLOC_MAX_UNITS) return KVS_EINVAL;   // beyond the scratch's counter capacity
    if (!device_ptr(q, 16) || !device_ptr(k, 16) || !device_ptr(v, 16) || !device_ptr(out, 16)) return KVS_EINVAL;
    if (lse != nullptr && !device_ptr(lse, 4)) return KVS_EINVAL;
    if (mix && !device_ptr(w, 4)) return KVS_EINVAL;

    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return KVS_ECUDA;
    unsigned char* scratch = nullptr;
    if (scratch_address(dev, &scratch) != cudaSuccess) return KVS_ECUDA;
    unsigned* counters = reinterpret_cast<unsigned*>(scratch);
    unsigned* status = reinterpret_cast<unsigned*>(scratch + COUNTER_BYTES);
    float* partials = reinterpret_cast<float*>(scratch + COUNTER_BYTES + STATUS_BYTES);

    int sms = 148;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    // resident CTAs per SM of each kernel variant, looked up once (racing threads store
    // the same value)
    static std::atomic<int> occ[2][2];
    std::atomic<int>& occ_slot = occ[head_dim == 128][mix];
    int ctas_per_sm = occ_slot.load(std::memory_order_relaxed);
    if (ctas_per_sm == 0) {
        ctas_per_sm = decode_bf16_ctas_per_sm(head_dim, mix);
        occ_slot.store(ctas_per_sm, std::memory_order_relaxed);
    }
    const TileShape ts = decode_bf16_shape(head_dim, mix);
    // balanced grid: the units' token tiles cut into G equal ranges, one CTA each; a
    // unit spread over several CTAs keeps one partial per CTA in the array
    const int n_t = (context + ts.tt - 1) / ts.tt;
    const long long W = units * n_t;
    const long long per_unit = (static_cast<long long>(sms) * ctas_per_sm) / units;
    long long G = units * (per_unit > 1 ? per_unit : 1);
    if (G > W) G = W;
    // partial slots run up to units + G; lower G until they fit the array. With one CTA
    // per unit (G == units) no partial is written at all. On a 148-SM B200 with one
    // resident CTA per SM the default grid always fits (at most 222 slots of
    // 16 x (128 + 4) floats, 1.9 MB), so the loop guards other devices and tile shapes.
    const size_t per = static_cast<size_t>(g) * (head_dim + 4);
    while (G > units && (static_cast<size_t>(units) + G) * per > PARTIAL_FLOATS) --G;

    DecodeArgs a;
    std::memset(&a, 0, sizeof(a));
    a.q = q;
    a.out = out;
    a.lse = lse;
    a.k = k;
    a.v = v;
    a.src0 = src0;
    a.src1 = mix ? src1 : 0;
    a.w = w;
    a.B = batch;
    a.Hq = num_q_heads;
    a.Hkv = num_kv_heads;
    a.T = context;
    a.g = g;
    a.units = static_cast<int>(units);
    a.n_t = n_t;
    a.splits = static_cast<int>(G);
    a.scale_log2 = (1.0f / std::sqrt(static_cast<float>(head_dim))) * 1.4426950408889634f;
    a.ws = partials;
    a.counters = counters;
    a.err = status;
    a.wait_limit = 4000000000LL;

    CUtensorMap tmK, tmV;
    const int rows = slots * batch * num_kv_heads;
    if (!store_map(k, head_dim, context, rows, ts.tt, &tmK) || !store_map(v, head_dim, context, rows, ts.tt, &tmV))
        return KVS_ECUDA;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // the array keeps the previous call's contents: counters and status must start at zero
    if (cudaMemsetAsync(scratch, 0, COUNTER_BYTES + STATUS_BYTES, st) != cudaSuccess) return KVS_ECUDA;
    if (launch_decode_bf16(head_dim, mix, tmK, tmV, a, st) != cudaSuccess) return KVS_ECUDA;
    return KVS_OK;
}

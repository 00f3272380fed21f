// Host side of libkvshare: argument validation, layer-table resolution,
// split heuristic, TMA descriptors and kernel launches. See include/kvshare.h.
#include "kvshare.h"

#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstring>
#include <mutex>
#include <new>
#include <unordered_map>
#include <vector>

#include "kvs_internal.h"

using namespace kvs;

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
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

struct MapKey {
    const void* ptr;
    uint64_t d0, d1, d2;
    uint32_t box0, box1;
    int dtype, swizzle;
    bool operator==(const MapKey& o) const {
        return ptr == o.ptr && d0 == o.d0 && d1 == o.d1 && d2 == o.d2 && box0 == o.box0 && box1 == o.box1 &&
               dtype == o.dtype && swizzle == o.swizzle;
    }
};

struct MapKeyHash {
    size_t operator()(const MapKey& k) const {
        size_t h = reinterpret_cast<uintptr_t>(k.ptr);
        for (uint64_t v : {k.d0, k.d1, k.d2, (uint64_t)k.box0, (uint64_t)k.box1, (uint64_t)k.dtype, (uint64_t)k.swizzle})
            h = h * 1000003u ^ std::hash<uint64_t>()(v);
        return h;
    }
};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool is_device_ptr(const void* p) {
    if (p == nullptr) return false;
    cudaPointerAttributes at;
    if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    return at.type == cudaMemoryTypeDevice || at.type == cudaMemoryTypeManaged;
}

bool dev_ok(const void* p) { return p != nullptr && aligned16(p) && is_device_ptr(p); }

}  // namespace

struct kvshare_ctx {
    kvshare_config cfg{};
    int device = 0;
    int sms = 148;
    float scale = 0.f;
    std::vector<kvshare_layer> map;
    bool map_set = false;
    float* w_dev = nullptr;          // [L][Hkv]
    std::vector<float> w_host;
    float* ws = nullptr;             // split partials
    size_t ws_floats = 0;
    unsigned* counters = nullptr;    // [max_batch * Hkv]
    unsigned* err = nullptr;         // status word
    int splits_override = 0;
    int kv_overlap = 0;
    int grid_override = 0;
    std::vector<int> order;          // layer order of decode calls (a permutation of 0..L-1)
    int stall_next = 0;
    long long wait_limit = 4000000000LL;     // ~2 s of SM clock
    long long stall_limit = 20000000LL;      // ~10 ms
    uint64_t launches = 0;
    std::unordered_map<MapKey, CUtensorMap, MapKeyHash> maps;
    // kept scores of one layer for the attention statistics [max_batch][Hq][max_context]
    float* sscore = nullptr;
    // projected queries of one low-rank prefill layer [max_batch][Hq][max_context][64] bf16
    uint16_t* qp = nullptr;
    // staging for kvshare_decode_host
    void* q_stage = nullptr;
    float* out_stage = nullptr;
    float* lse_stage = nullptr;
    // kvshare_decode_host: copy streams (host to device, device to host) and events that
    // pipeline chunks of layers (copies of one chunk under the decode of another)
    static constexpr int HOST_CHUNKS = 8;
    cudaStream_t h2d = nullptr, d2h = nullptr;
    cudaEvent_t ev_start = nullptr, ev_done = nullptr;
    cudaEvent_t ev_in[HOST_CHUNKS] = {}, ev_out[HOST_CHUNKS] = {};
};

namespace {

size_t elem_size(kvshare_dtype t) { return t == KVS_F32 ? 4 : 2; }

kvshare_status cuda_status(cudaError_t e) { return e == cudaSuccess ? KVS_OK : KVS_ECUDA; }

// 3-D tiled map over [rows][T][inner] elements, box {box0, tt, 1}; rows are `pitch`
// tokens apart (0: T), so a map may end before the store does.
bool get_map(kvshare_ctx* c, const void* base, CUtensorMapDataType dt, int esize, int inner, int T, int rows,
             int box0, int tt, CUtensorMapSwizzle sw, CUtensorMap* out, int pitch = 0) {
    if (pitch == 0) pitch = T;
    MapKey key{base, (uint64_t)inner, (uint64_t)T | (static_cast<uint64_t>(pitch) << 32), (uint64_t)rows,
               (uint32_t)box0, (uint32_t)tt, (int)dt, (int)sw};
    auto it = c->maps.find(key);
    if (it != c->maps.end()) {
        *out = it->second;
        return true;
    }
    EncodeTiledFn fn = encode_fn();
    if (fn == nullptr) return false;
    CUtensorMap m;
    cuuint64_t dims[3] = {(cuuint64_t)inner, (cuuint64_t)T, (cuuint64_t)rows};
    cuuint64_t strides[2] = {(cuuint64_t)inner * esize, (cuuint64_t)pitch * inner * esize};
    cuuint32_t box[3] = {(cuuint32_t)box0, (cuuint32_t)tt, 1u};
    cuuint32_t estr[3] = {1u, 1u, 1u};
    CUresult r = fn(&m, dt, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return false;
    if (c->maps.size() >= 4096) c->maps.clear();
    c->maps.emplace(key, m);
    *out = m;
    return true;
}

// K or V store [rows][T][D] bf16, box {64, tt}, 128-B swizzle
bool get_store_map(kvshare_ctx* c, const void* base, int D, int T, int rows, int tt, CUtensorMap* out) {
    return get_map(c, base, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, D, T, rows, 64, tt, CU_TENSOR_MAP_SWIZZLE_128B, out);
}

int choose_splits(const kvshare_ctx* c, int units, int tiles, int ctas_per_sm, int g, int part_values) {
    int s;
    if (c->splits_override > 0) {
        s = c->splits_override;
    } else {
        const int resident = c->sms * ctas_per_sm;
        s = resident / units;
        if (s < 1) s = 1;
    }
    if (s > tiles) s = tiles;
    if (s > MAX_SPLITS) s = MAX_SPLITS;
    // workspace capacity: units * splits * g * (part_values + 4) floats
    const size_t per_split = static_cast<size_t>(units) * g * (part_values + 4);
    while (s > 1 && per_split * s > c->ws_floats) --s;
    if (s < 1) s = 1;
    return s;
}

kvshare_status validate_cache_common(const kvshare_ctx* c, const kvshare_cache* k) {
    if (k == nullptr) return KVS_EINVAL;
    if (k->batch < 1 || k->batch > c->cfg.max_batch) return KVS_EINVAL;
    if (k->context < 1 || k->context > c->cfg.max_context) return KVS_EINVAL;
    return KVS_OK;
}

kvshare_status check_layer_sources(const kvshare_ctx* c, const kvshare_cache* k, int l, bool* need_kv,
                                   bool* need_lr) {
    const kvshare_layer& e = c->map[l];
    if (e.kind == KVS_SRC_SINGLE || e.kind == KVS_SRC_MIX) {
        if (e.src0 < 0 || e.src0 >= k->slots) return KVS_EINVAL;
        if (e.kind == KVS_SRC_MIX && (e.src1 < 0 || e.src1 >= k->slots)) return KVS_EINVAL;
        *need_kv = true;
    } else if (e.kind == KVS_SRC_LOWRANK) {
        if (e.src0 < 0 || e.src0 >= k->pairs) return KVS_EINVAL;
        *need_lr = true;
    } else {
        return KVS_EINVAL;
    }
    return KVS_OK;
}

// Prefill fills a slot when its owner runs: the first layer (lowest index) of the map that
// reads the slot as a SINGLE source. A two-source target rebuilds its K/V from slots its
// own forward pass has already produced, so each source needs an owner shallower than the
// target ("DepthGraft: Structural Regularization through Hierarchical Cross-Layer KV
// Reconstruction", Abstract: deep layers rebuilt from shallow and middle sources, prefill
// keeping its early completion).
bool prefill_source_ready(const kvshare_ctx* c, int slot, int target) {
    for (int l = 0; l < target; ++l)
        if (c->map[l].kind == KVS_SRC_SINGLE && c->map[l].src0 == slot) return true;
    return false;
}

// The layers of [l0, l1) in the context's decode order.
std::vector<int> ordered_layers(const kvshare_ctx* c, int l0, int l1) {
    std::vector<int> ls;
    ls.reserve(l1 - l0);
    for (int l : c->order)
        if (l >= l0 && l < l1) ls.push_back(l);
    return ls;
}

// Optional statistics outputs of a decode call (all [L]-major, see kvshare_decode_stats).
struct StatsOut {
    float* mass;
    float* score;
    float* entropy;
    float* peak;
};

kvshare_status decode_layers(kvshare_ctx* c, const kvshare_cache* k, const void* q, float* out, float* lse,
                             const int* layers, int n_layers, cudaStream_t st, const StatsOut* stats = nullptr) {
    const kvshare_config& cf = c->cfg;
    const int D = cf.head_dim;
    const int B = k->batch;
    const int T = k->context;
    const int Hq = cf.num_q_heads;
    const int Hkv = cf.num_kv_heads;
    const int g = Hq / Hkv;
    const size_t es = elem_size(cf.dtype);
    if (cudaSetDevice(c->device) != cudaSuccess) return KVS_ECUDA;

    for (int li = 0; li < n_layers; ++li) {
        const int l = layers[li];
        const kvshare_layer& e = c->map[l];
        DecodeArgs a;
        std::memset(&a, 0, sizeof(a));
        a.q = static_cast<const char*>(q) + static_cast<size_t>(l) * B * Hq * D * es;
        a.out = out + static_cast<size_t>(l) * B * Hq * D;
        a.lse = lse ? lse + static_cast<size_t>(l) * B * Hq : nullptr;
        a.k = k->k;
        a.v = k->v;
        a.src0 = e.src0;
        a.src1 = e.src1;
        a.w = c->w_dev + static_cast<size_t>(l) * Hkv;
        a.B = B;
        a.Hq = Hq;
        a.Hkv = Hkv;
        a.T = T;
        a.g = g;
        a.lens = k->lengths;
        // the kept scores feed the per-token statistics (mass, router score); entropy and
        // peak come out of the decode's own merge
        const bool per_token = stats != nullptr && (stats->mass != nullptr || stats->score != nullptr);
        a.sscore = per_token ? c->sscore : nullptr;
        const size_t lbh = static_cast<size_t>(l) * B * Hq;
        a.entropy = stats != nullptr && stats->entropy != nullptr ? stats->entropy + lbh : nullptr;
        a.peak = stats != nullptr && stats->peak != nullptr ? stats->peak + lbh : nullptr;
        a.scale_log2 = c->scale * 1.4426950408889634f;
        a.ws = c->ws;
        a.counters = c->counters;
        a.err = c->err;
        a.wait_limit = c->wait_limit;
        a.stall = c->stall_next;
        a.stall_limit = c->stall_limit;
        c->stall_next = 0;
        // consecutive decode layers overlap launch and prologue with the previous tail
        a.pdl = 1;
        a.kv_early = c->kv_overlap;
        cudaError_t err;
        if (cf.dtype == KVS_F32) {
            if (e.kind == KVS_SRC_LOWRANK) return KVS_EUNSUPPORTED;
            const int tt = decode_f32_tile();
            const int tiles = (T + tt - 1) / tt;
            int s = choose_splits(c, B * Hkv, tiles, 4, g, D);
            if (s > F32_MAX_SPLITS) s = F32_MAX_SPLITS;
            a.tiles_per_split = (tiles + s - 1) / s;
            a.splits = (tiles + a.tiles_per_split - 1) / a.tiles_per_split;
            err = launch_decode_f32(e.kind == KVS_SRC_MIX, D, a, st);
        } else if (e.kind == KVS_SRC_LOWRANK) {
            const int Rb = cf.basis_rank;
            const int tt = decode_lowrank_tile(Rb);
            // occupancy per kernel shape, computed once (racing threads compute the same value)
            static std::atomic<int> occ_lr[2][3];
            std::atomic<int>& occ_slot = occ_lr[D == 128][Rb == 32 ? 0 : (Rb == 64 ? 1 : 2)];
            int o = occ_slot.load(std::memory_order_relaxed);
            if (o == 0) {
                o = decode_lowrank_occupancy(D, Rb);
                occ_slot.store(o, std::memory_order_relaxed);
            }
            const int tiles = (T + tt - 1) / tt;
            int s = choose_splits(c, B * Hkv, tiles, o, g, Rb + 16);   // partials of Rb + 16 values
            a.tiles_per_split = (tiles + s - 1) / s;
            a.splits = (tiles + a.tiles_per_split - 1) / a.tiles_per_split;
            const size_t BHT = static_cast<size_t>(B) * Hkv * T;
            a.pair = e.src0;
            a.Rb = Rb;
            a.Rm = 16;
            a.coef_k = k->coef_k;
            a.coef_v = k->coef_v;
            a.basis_k = static_cast<const uint16_t*>(k->basis_k) + static_cast<size_t>(e.src0) * Hkv * Rb * D;
            a.basis_v = static_cast<const uint16_t*>(k->basis_v) + static_cast<size_t>(e.src0) * Hkv * Rb * D;
            a.u_k = k->u_k + static_cast<size_t>(l) * BHT * 16;
            a.u_v = k->u_v + static_cast<size_t>(l) * BHT * 16;
            a.s_k = k->s_k + static_cast<size_t>(l) * BHT;
            a.s_v = k->s_v + static_cast<size_t>(l) * BHT;
            a.r_k = static_cast<const uint16_t*>(k->r_k) + static_cast<size_t>(l) * Hkv * 16 * D;
            a.r_v = static_cast<const uint16_t*>(k->r_v) + static_cast<size_t>(l) * Hkv * 16 * D;
            a.rank = k->rank + static_cast<size_t>(l) * B * T;
            // coefficient tiles by TMA; the group-packed residual codes by sized bulk copies
            CUtensorMap maps[2];
            const int crows = k->pairs * B * Hkv;
            const int box0 = Rb < 64 ? Rb : 64;
            const CUtensorMapSwizzle sw = Rb == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B;
            if (!get_map(c, k->coef_k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, Rb, T, crows, box0, tt, sw, &maps[0]) ||
                !get_map(c, k->coef_v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, Rb, T, crows, box0, tt, sw, &maps[1]))
                return KVS_ECUDA;
            err = launch_decode_lowrank(D, Rb, a, maps, st);
        } else {
            const bool mix = e.kind == KVS_SRC_MIX;
            const TileShape ts = decode_bf16_shape(D, mix);
            static std::atomic<int> occ[2][2];
            std::atomic<int>& occ_slot = occ[D == 128][mix];
            int o = occ_slot.load(std::memory_order_relaxed);
            if (o == 0) {
                o = decode_bf16_ctas_per_sm(D, mix);
                occ_slot.store(o, std::memory_order_relaxed);
            }
            // balanced grid: the units' token tiles cut into G equal ranges, one CTA each
            const int units = B * Hkv;
            const int n_t = (T + ts.tt - 1) / ts.tt;
            const long long W = static_cast<long long>(units) * n_t;
            // default: a whole number of CTAs per unit, as many as fit in one wave, so no
            // CTA straddles two units (a straddling CTA reloads its queries mid-stream and
            // every unit then pays a merge); ranges that straddle are still handled
            long long G;
            if (c->grid_override > 0) {
                G = c->grid_override;
            } else if (c->splits_override > 0) {
                G = static_cast<long long>(c->splits_override) * units;
            } else {
                const long long per_unit = (static_cast<long long>(c->sms) * o) / units;
                G = static_cast<long long>(units) * (per_unit > 1 ? per_unit : 1);
            }
            if (G < units) G = units;
            if (G > W) G = W;
            const size_t per = static_cast<size_t>(g) * (D + 4);
            while (G > units && (static_cast<size_t>(units) + G) * per > c->ws_floats) --G;
            a.units = units;
            a.n_t = n_t;
            a.splits = static_cast<int>(G);
            CUtensorMap tmK, tmV;
            const int rows = k->slots * B * Hkv;
            if (!get_store_map(c, k->k, D, T, rows, ts.tt, &tmK) || !get_store_map(c, k->v, D, T, rows, ts.tt, &tmV))
                return KVS_ECUDA;
            err = launch_decode_bf16(D, mix, tmK, tmV, a, st);
        }
        if (err != cudaSuccess) return KVS_ECUDA;
        ++c->launches;
        if (per_token) {
            StatsArgs sa;
            std::memset(&sa, 0, sizeof(sa));
            sa.sscore = c->sscore;
            sa.lse = a.lse;
            sa.lens = k->lengths;
            const size_t lbt = static_cast<size_t>(l) * B;
            sa.mass = stats->mass ? stats->mass + lbt * Hkv * T : nullptr;
            sa.score = stats->score ? stats->score + lbt * T : nullptr;
            sa.err = c->err;
            sa.B = B;
            sa.Hq = Hq;
            sa.Hkv = Hkv;
            sa.T = T;
            sa.g = g;
            const int n = launch_router_stats(sa, st);
            if (n < 0) return KVS_ECUDA;
            c->launches += n;
        }
    }
    return KVS_OK;
}

kvshare_status validate_decode(kvshare_ctx* c, const kvshare_cache* k, const void* q, const float* out,
                               const float* lse, int l0, int l1, bool host_io) {
    if (c == nullptr) return KVS_EINVAL;
    if (!c->map_set) return KVS_EINVAL;
    kvshare_status s = validate_cache_common(c, k);
    if (s != KVS_OK) return s;
    if (l0 < 0 || l1 > c->cfg.num_layers || l0 > l1) return KVS_EINVAL;
    if (q == nullptr || out == nullptr) return KVS_EINVAL;
    if (!aligned16(q) || !aligned16(out) || (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3u))) return KVS_EINVAL;
    if (!host_io && (!is_device_ptr(q) || !is_device_ptr(out) || (lse != nullptr && !is_device_ptr(lse))))
        return KVS_EINVAL;
    bool need_kv = false, need_lr = false;
    for (int l = l0; l < l1; ++l) {
        s = check_layer_sources(c, k, l, &need_kv, &need_lr);
        if (s != KVS_OK) return s;
        if (c->map[l].kind == KVS_SRC_LOWRANK && c->cfg.dtype != KVS_BF16) return KVS_EUNSUPPORTED;
    }
    if (k->lengths != nullptr && (!is_device_ptr(k->lengths) || (reinterpret_cast<uintptr_t>(k->lengths) & 3u)))
        return KVS_EINVAL;
    if (need_kv) {
        if (k->slots < 1 || !dev_ok(k->k) || !dev_ok(k->v)) return KVS_EINVAL;
    }
    if (need_lr) {
        if (k->pairs < 1) return KVS_EINVAL;
        const void* ps[] = {k->coef_k, k->coef_v, k->basis_k, k->basis_v, k->u_k, k->u_v,
                            k->s_k, k->s_v, k->r_k, k->r_v, k->rank};
        for (const void* p : ps)
            if (!dev_ok(p)) return KVS_EINVAL;
    }
    return KVS_OK;
}

// One low-rank layer of a prefill: the query projection pre-pass, then the tcgen05 kernel.
// The K/V operand maps end at seqlen, so rows past the sequence arrive as zeros.
kvshare_status prefill_lowrank_layer(kvshare_ctx* ctx, const kvshare_cache* cache, const void* q, void* out,
                                     float* lse, int l, int seqlen, cudaStream_t st) {
    const kvshare_config& cf = ctx->cfg;
    const kvshare_layer& e = ctx->map[l];
    const int D = cf.head_dim, B = cache->batch, Hq = cf.num_q_heads, Hkv = cf.num_kv_heads, T = cache->context;
    const size_t per_layer = static_cast<size_t>(B) * Hq * seqlen;
    const size_t BHT = static_cast<size_t>(B) * Hkv * T;
    PrefillLrArgs a;
    std::memset(&a, 0, sizeof(a));
    a.q = static_cast<const uint16_t*>(q) + static_cast<size_t>(l) * per_layer * D;
    a.qp = ctx->qp;
    a.lse = lse ? lse + static_cast<size_t>(l) * per_layer : nullptr;
    a.basis_k = static_cast<const uint16_t*>(cache->basis_k) + static_cast<size_t>(e.src0) * Hkv * 32 * D;
    a.basis_v = static_cast<const uint16_t*>(cache->basis_v) + static_cast<size_t>(e.src0) * Hkv * 32 * D;
    a.r_k = static_cast<const uint16_t*>(cache->r_k) + static_cast<size_t>(l) * Hkv * 16 * D;
    a.r_v = static_cast<const uint16_t*>(cache->r_v) + static_cast<size_t>(l) * Hkv * 16 * D;
    a.s_k = cache->s_k + static_cast<size_t>(l) * BHT;
    a.s_v = cache->s_v + static_cast<size_t>(l) * BHT;
    a.rank = cache->rank + static_cast<size_t>(l) * B * T;
    a.pair = e.src0;
    a.B = B;
    a.Hq = Hq;
    a.Hkv = Hkv;
    a.S = seqlen;
    a.T = T;
    a.g = Hq / Hkv;
    a.d = D;
    a.scale_log2 = ctx->scale * 1.4426950408889634f;
    a.err = ctx->err;
    a.wait_limit = ctx->wait_limit;
    const int8_t* uk = cache->u_k + static_cast<size_t>(l) * BHT * 16;
    const int8_t* uv = cache->u_v + static_cast<size_t>(l) * BHT * 16;
    void* o = static_cast<uint16_t*>(out) + static_cast<size_t>(l) * per_layer * D;
    const int crows = cache->pairs * B * Hkv;
    CUtensorMap maps[6];
    const int bn = prefill_lowrank_tile();
    if (!get_map(ctx, ctx->qp, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, LR_QW, seqlen, B * Hq, 64, 128,
                 CU_TENSOR_MAP_SWIZZLE_128B, &maps[0]) ||
        !get_map(ctx, o, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, D, seqlen, B * Hq, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B,
                 &maps[1]) ||
        !get_map(ctx, cache->coef_k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, 32, seqlen, crows, 32, bn,
                 CU_TENSOR_MAP_SWIZZLE_NONE, &maps[2], T) ||
        !get_map(ctx, cache->coef_v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, 32, seqlen, crows, 32, bn,
                 CU_TENSOR_MAP_SWIZZLE_NONE, &maps[3], T) ||
        !get_map(ctx, uk, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, 16, seqlen, B * Hkv, 16, bn, CU_TENSOR_MAP_SWIZZLE_NONE,
                 &maps[4], T) ||
        !get_map(ctx, uv, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, 16, seqlen, B * Hkv, 16, bn, CU_TENSOR_MAP_SWIZZLE_NONE,
                 &maps[5], T))
        return KVS_ECUDA;
    if (launch_lr_qproj(a, st) != cudaSuccess) return KVS_ECUDA;
    ++ctx->launches;
    if (launch_prefill_lowrank(D, maps, a, st) != cudaSuccess) return KVS_ECUDA;
    ++ctx->launches;
    return KVS_OK;
}

}  // namespace

extern "C" {

kvshare_status kvshare_create(const kvshare_config* cfg, kvshare_t* out) {
    if (out == nullptr) return KVS_EINVAL;
    *out = nullptr;
    if (cfg == nullptr) return KVS_EINVAL;
    const kvshare_config& c = *cfg;
    if (c.num_layers < 1 || c.num_q_heads < 1 || c.num_kv_heads < 1 || c.max_batch < 1 || c.max_context < 1)
        return KVS_EINVAL;
    if (c.num_q_heads % c.num_kv_heads != 0) return KVS_EINVAL;
    if (c.dtype != KVS_F32 && c.dtype != KVS_BF16) return KVS_EINVAL;
    if (!(c.softmax_scale >= 0.f) || std::isinf(c.softmax_scale)) return KVS_EINVAL;
    if (c.head_dim != 64 && c.head_dim != 128) return KVS_EUNSUPPORTED;
    if (c.num_q_heads / c.num_kv_heads > MAX_GROUP) return KVS_EUNSUPPORTED;
    if (c.basis_rank != 0 && c.basis_rank != 32 && c.basis_rank != c.head_dim) return KVS_EUNSUPPORTED;
    if (c.max_resid_rank != 0 && c.max_resid_rank != 16) return KVS_EUNSUPPORTED;

    kvshare_ctx* ctx = new (std::nothrow) kvshare_ctx();
    if (ctx == nullptr) return KVS_ENOMEM;
    ctx->cfg = c;
    if (ctx->cfg.basis_rank == 0) ctx->cfg.basis_rank = 32;
    if (ctx->cfg.max_resid_rank == 0) ctx->cfg.max_resid_rank = 16;
    ctx->scale = c.softmax_scale > 0.f ? c.softmax_scale : 1.0f / std::sqrt(static_cast<float>(c.head_dim));
    if (cudaGetDevice(&ctx->device) != cudaSuccess) {
        delete ctx;
        return KVS_ECUDA;
    }
    cudaDeviceGetAttribute(&ctx->sms, cudaDevAttrMultiProcessorCount, ctx->device);
    const int g = c.num_q_heads / c.num_kv_heads;
    const size_t units = static_cast<size_t>(c.max_batch) * c.num_kv_heads;
    const int max_tiles = (c.max_context + 15) / 16;
    const int ms = max_tiles < MAX_SPLITS ? max_tiles : MAX_SPLITS;
    // a split's partial per q head: d values (forms a, b) or Rb + 16 coefficient-space
    // values (form c), plus m and l, padded to 16 bytes
    const int part_values = std::max(c.head_dim, ctx->cfg.basis_rank + ctx->cfg.max_resid_rank);
    ctx->ws_floats = units * ms * g * (part_values + 4);
    ctx->map.assign(c.num_layers, kvshare_layer{KVS_SRC_SINGLE, 0, 0});
    ctx->order.resize(c.num_layers);
    for (int l = 0; l < c.num_layers; ++l) ctx->order[l] = l;
    ctx->w_host.assign(static_cast<size_t>(c.num_layers) * c.num_kv_heads, 1.0f);
    if (cudaMalloc(&ctx->ws, ctx->ws_floats * sizeof(float)) != cudaSuccess ||
        cudaMalloc(&ctx->counters, units * sizeof(unsigned)) != cudaSuccess ||
        cudaMalloc(&ctx->err, sizeof(unsigned)) != cudaSuccess ||
        cudaMalloc(&ctx->w_dev, ctx->w_host.size() * sizeof(float)) != cudaSuccess) {
        cudaGetLastError();
        kvshare_destroy(ctx);
        return KVS_ENOMEM;
    }
    if (cudaMemset(ctx->counters, 0, units * sizeof(unsigned)) != cudaSuccess ||
        cudaMemset(ctx->err, 0, sizeof(unsigned)) != cudaSuccess ||
        cudaMemcpy(ctx->w_dev, ctx->w_host.data(), ctx->w_host.size() * sizeof(float), cudaMemcpyHostToDevice) !=
            cudaSuccess) {
        kvshare_destroy(ctx);
        return KVS_ECUDA;
    }
    *out = ctx;
    return KVS_OK;
}

kvshare_status kvshare_destroy(kvshare_t ctx) {
    if (ctx == nullptr) return KVS_OK;
    int prev = 0;
    cudaGetDevice(&prev);
    cudaSetDevice(ctx->device);
    cudaFree(ctx->ws);
    cudaFree(ctx->counters);
    cudaFree(ctx->err);
    cudaFree(ctx->w_dev);
    cudaFree(ctx->sscore);
    cudaFree(ctx->qp);
    cudaFree(ctx->q_stage);
    cudaFree(ctx->out_stage);
    cudaFree(ctx->lse_stage);
    if (ctx->h2d != nullptr) cudaStreamDestroy(ctx->h2d);
    if (ctx->d2h != nullptr) cudaStreamDestroy(ctx->d2h);
    for (cudaEvent_t ev : {ctx->ev_start, ctx->ev_done})
        if (ev != nullptr) cudaEventDestroy(ev);
    for (int c = 0; c < kvshare_ctx::HOST_CHUNKS; ++c) {
        if (ctx->ev_in[c] != nullptr) cudaEventDestroy(ctx->ev_in[c]);
        if (ctx->ev_out[c] != nullptr) cudaEventDestroy(ctx->ev_out[c]);
    }
    cudaSetDevice(prev);
    delete ctx;
    return KVS_OK;
}

kvshare_status kvshare_set_map(kvshare_t ctx, const kvshare_layer* map, const float* w) {
    if (ctx == nullptr || map == nullptr) return KVS_EINVAL;
    const int L = ctx->cfg.num_layers;
    const int Hkv = ctx->cfg.num_kv_heads;
    bool any_mix = false;
    for (int l = 0; l < L; ++l) {
        const kvshare_layer& e = map[l];
        if (e.kind != KVS_SRC_SINGLE && e.kind != KVS_SRC_MIX && e.kind != KVS_SRC_LOWRANK) return KVS_EINVAL;
        if (e.src0 < 0) return KVS_EINVAL;
        if (e.kind == KVS_SRC_MIX) {
            any_mix = true;
            if (e.src1 < 0 || e.src1 == e.src0) return KVS_EINVAL;
        }
        if (e.kind == KVS_SRC_LOWRANK && ctx->cfg.dtype != KVS_BF16) return KVS_EUNSUPPORTED;
    }
    if (any_mix) {
        if (w == nullptr) return KVS_EINVAL;
        for (int l = 0; l < L; ++l) {
            if (map[l].kind != KVS_SRC_MIX) continue;
            for (int j = 0; j < Hkv; ++j) {
                const float x = w[static_cast<size_t>(l) * Hkv + j];
                if (!(x >= 0.f && x <= 1.f)) return KVS_EINVAL;
            }
        }
    }
    for (int l = 0; l < L; ++l) {
        for (int j = 0; j < Hkv; ++j)
            ctx->w_host[static_cast<size_t>(l) * Hkv + j] =
                (map[l].kind == KVS_SRC_MIX) ? w[static_cast<size_t>(l) * Hkv + j] : 1.0f;
    }
    if (cudaSetDevice(ctx->device) != cudaSuccess) return KVS_ECUDA;
    if (cudaMemcpy(ctx->w_dev, ctx->w_host.data(), ctx->w_host.size() * sizeof(float), cudaMemcpyHostToDevice) !=
        cudaSuccess)
        return KVS_ECUDA;
    ctx->map.assign(map, map + L);
    ctx->map_set = true;
    return KVS_OK;
}

kvshare_status kvshare_decode(kvshare_t ctx, const kvshare_cache* cache, const void* q, float* out, float* lse,
                              int l0, int l1, void* stream) {
    kvshare_status s = validate_decode(ctx, cache, q, out, lse, l0, l1, false);
    if (s != KVS_OK) return s;
    const std::vector<int> ls = ordered_layers(ctx, l0, l1);
    return decode_layers(ctx, cache, q, out, lse, ls.data(), static_cast<int>(ls.size()),
                         static_cast<cudaStream_t>(stream));
}

kvshare_status kvshare_decode_stats(kvshare_t ctx, const kvshare_cache* cache, const void* q, float* out, float* lse,
                                    float* mass, float* score, float* entropy, float* peak, int l0, int l1,
                                    void* stream) {
    kvshare_status s = validate_decode(ctx, cache, q, out, lse, l0, l1, false);
    if (s != KVS_OK) return s;
    if (lse == nullptr) return KVS_EINVAL;
    for (const float* p : {mass, score, entropy, peak})
        if (p != nullptr && (!is_device_ptr(p) || (reinterpret_cast<uintptr_t>(p) & 3u))) return KVS_EINVAL;
    const std::vector<int> ls = ordered_layers(ctx, l0, l1);
    if (mass == nullptr && score == nullptr && entropy == nullptr && peak == nullptr)
        return decode_layers(ctx, cache, q, out, lse, ls.data(), static_cast<int>(ls.size()),
                             static_cast<cudaStream_t>(stream));
    if (cudaSetDevice(ctx->device) != cudaSuccess) return KVS_ECUDA;
    if (ctx->sscore == nullptr && (mass != nullptr || score != nullptr)) {
        const kvshare_config& cf = ctx->cfg;
        const size_t n = static_cast<size_t>(cf.max_batch) * cf.num_q_heads * cf.max_context;
        if (cudaMalloc(&ctx->sscore, n * sizeof(float)) != cudaSuccess) {
            cudaGetLastError();
            ctx->sscore = nullptr;
            return KVS_ENOMEM;
        }
    }
    const StatsOut so{mass, score, entropy, peak};
    return decode_layers(ctx, cache, q, out, lse, ls.data(), static_cast<int>(ls.size()),
                         static_cast<cudaStream_t>(stream), &so);
}

kvshare_status kvshare_decode_host(kvshare_t ctx, const kvshare_cache* cache, const void* q_host, float* out_host,
                                   float* lse_host, int l0, int l1, void* stream) {
    kvshare_status s = validate_decode(ctx, cache, q_host, out_host, lse_host, l0, l1, true);
    if (s != KVS_OK) return s;
    const kvshare_config& cf = ctx->cfg;
    const size_t es = elem_size(cf.dtype);
    const size_t per_layer = static_cast<size_t>(cf.max_batch) * cf.num_q_heads * cf.head_dim;
    if (cudaSetDevice(ctx->device) != cudaSuccess) return KVS_ECUDA;
    if (ctx->q_stage == nullptr) {
        if (cudaMalloc(&ctx->q_stage, per_layer * cf.num_layers * es) != cudaSuccess ||
            cudaMalloc(&ctx->out_stage, per_layer * cf.num_layers * sizeof(float)) != cudaSuccess ||
            cudaMalloc(&ctx->lse_stage, static_cast<size_t>(cf.max_batch) * cf.num_q_heads * cf.num_layers *
                                            sizeof(float)) != cudaSuccess) {
            cudaGetLastError();
            return KVS_ENOMEM;
        }
    }
    if (ctx->h2d == nullptr) {
        bool ok = cudaStreamCreateWithFlags(&ctx->h2d, cudaStreamNonBlocking) == cudaSuccess &&
                  cudaStreamCreateWithFlags(&ctx->d2h, cudaStreamNonBlocking) == cudaSuccess &&
                  cudaEventCreateWithFlags(&ctx->ev_start, cudaEventDisableTiming) == cudaSuccess &&
                  cudaEventCreateWithFlags(&ctx->ev_done, cudaEventDisableTiming) == cudaSuccess;
        for (int c = 0; ok && c < kvshare_ctx::HOST_CHUNKS; ++c)
            ok = cudaEventCreateWithFlags(&ctx->ev_in[c], cudaEventDisableTiming) == cudaSuccess &&
                 cudaEventCreateWithFlags(&ctx->ev_out[c], cudaEventDisableTiming) == cudaSuccess;
        if (!ok) {
            cudaGetLastError();
            return KVS_ECUDA;
        }
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const size_t lay = static_cast<size_t>(cache->batch) * cf.num_q_heads * cf.head_dim;   // elements per layer
    const size_t layh = static_cast<size_t>(cache->batch) * cf.num_q_heads;
    const int nl = l1 - l0;
    if (nl == 0) return KVS_OK;
    // q is copied in as up to 8 contiguous chunks of layers on h2d; the layers decode on
    // `stream` in the context's order, each after the chunk holding its q has landed; a
    // chunk's out and lse are copied back on d2h as soon as its last layer has decoded.
    // The copy streams first wait for work already on `stream` (an earlier call may still
    // be using the staging buffers), and `stream` waits for the last copy out, so the call
    // is ordered on `stream` exactly like one that ran everything there. In model order
    // this pipelines the copies of one chunk under the decode of the others.
    const int nch = nl < kvshare_ctx::HOST_CHUNKS ? nl : kvshare_ctx::HOST_CHUNKS;
    auto chunk_begin = [&](int c) { return l0 + static_cast<int>((static_cast<long long>(nl) * c) / nch); };
    auto chunk_of = [&](int l) {
        int c = 0;
        while (c + 1 < nch && chunk_begin(c + 1) <= l) ++c;
        return c;
    };
    cudaError_t e = cudaEventRecord(ctx->ev_start, st);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(ctx->h2d, ctx->ev_start, 0);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(ctx->d2h, ctx->ev_start, 0);
    for (int c = 0; c < nch && e == cudaSuccess; ++c) {
        const size_t a = chunk_begin(c), n = chunk_begin(c + 1) - a;
        e = cudaMemcpyAsync(static_cast<char*>(ctx->q_stage) + a * lay * es,
                            static_cast<const char*>(q_host) + a * lay * es, n * lay * es, cudaMemcpyHostToDevice,
                            ctx->h2d);
        if (e == cudaSuccess) e = cudaEventRecord(ctx->ev_in[c], ctx->h2d);
    }
    if (e != cudaSuccess) return KVS_ECUDA;
    const std::vector<int> ls = ordered_layers(ctx, l0, l1);
    int remaining[kvshare_ctx::HOST_CHUNKS];
    bool waited[kvshare_ctx::HOST_CHUNKS];
    for (int c = 0; c < nch; ++c) {
        remaining[c] = chunk_begin(c + 1) - chunk_begin(c);
        waited[c] = false;
    }
    for (int l : ls) {
        const int c = chunk_of(l);
        if (!waited[c]) {
            if (cudaStreamWaitEvent(st, ctx->ev_in[c], 0) != cudaSuccess) return KVS_ECUDA;
            waited[c] = true;
        }
        s = decode_layers(ctx, cache, ctx->q_stage, ctx->out_stage, lse_host ? ctx->lse_stage : nullptr, &l, 1, st);
        if (s != KVS_OK) return s;
        if (--remaining[c] > 0) continue;
        const size_t a = chunk_begin(c), b = chunk_begin(c + 1);
        e = cudaEventRecord(ctx->ev_out[c], st);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(ctx->d2h, ctx->ev_out[c], 0);
        if (e == cudaSuccess)
            e = cudaMemcpyAsync(out_host + a * lay, ctx->out_stage + a * lay, (b - a) * lay * sizeof(float),
                                cudaMemcpyDeviceToHost, ctx->d2h);
        if (e == cudaSuccess && lse_host != nullptr)
            e = cudaMemcpyAsync(lse_host + a * layh, ctx->lse_stage + a * layh, (b - a) * layh * sizeof(float),
                                cudaMemcpyDeviceToHost, ctx->d2h);
        if (e != cudaSuccess) return KVS_ECUDA;
    }
    e = cudaEventRecord(ctx->ev_done, ctx->d2h);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(st, ctx->ev_done, 0);
    return cuda_status(e);
}

kvshare_status kvshare_prefill(kvshare_t ctx, const kvshare_cache* cache, const void* q, void* out, float* lse,
                               int l0, int l1, int seqlen, void* stream) {
    if (ctx == nullptr || !ctx->map_set) return KVS_EINVAL;
    kvshare_status s = validate_cache_common(ctx, cache);
    if (s != KVS_OK) return s;
    const kvshare_config& cf = ctx->cfg;
    if (l0 < 0 || l1 > cf.num_layers || l0 > l1) return KVS_EINVAL;
    if (seqlen < 1 || seqlen > cache->context) return KVS_EINVAL;
    if (cache->lengths != nullptr) return KVS_EUNSUPPORTED;   // one seqlen for every sequence
    if (!dev_ok(q) || !dev_ok(out) || (lse != nullptr && (!is_device_ptr(lse) || (reinterpret_cast<uintptr_t>(lse) & 3u))))
        return KVS_EINVAL;
    bool need_kv = false, need_lr = false;
    if (cf.dtype != KVS_BF16) return KVS_EUNSUPPORTED;
    for (int l = l0; l < l1; ++l)
        if (ctx->map[l].kind == KVS_SRC_LOWRANK && cf.basis_rank != 32) return KVS_EUNSUPPORTED;
    for (int l = l0; l < l1; ++l) {
        s = check_layer_sources(ctx, cache, l, &need_kv, &need_lr);
        if (s != KVS_OK) return s;
        if (ctx->map[l].kind == KVS_SRC_MIX && !(prefill_source_ready(ctx, ctx->map[l].src0, l) &&
                                                  prefill_source_ready(ctx, ctx->map[l].src1, l)))
            return KVS_EINVAL;
    }
    if (need_kv && (cache->slots < 1 || !dev_ok(cache->k) || !dev_ok(cache->v))) return KVS_EINVAL;
    if (need_lr) {
        const void* ps[] = {cache->coef_k, cache->coef_v, cache->basis_k, cache->basis_v, cache->u_k, cache->u_v,
                            cache->s_k, cache->s_v, cache->r_k, cache->r_v, cache->rank};
        for (const void* p : ps)
            if (!dev_ok(p)) return KVS_EINVAL;
    }
    if (cudaSetDevice(ctx->device) != cudaSuccess) return KVS_ECUDA;
    if (need_lr && ctx->qp == nullptr) {
        const size_t n = static_cast<size_t>(cf.max_batch) * cf.num_q_heads * cf.max_context * LR_QW;
        if (cudaMalloc(&ctx->qp, n * sizeof(uint16_t)) != cudaSuccess) {
            cudaGetLastError();
            ctx->qp = nullptr;
            return KVS_ENOMEM;
        }
    }
    const int D = cf.head_dim, B = cache->batch, Hq = cf.num_q_heads, Hkv = cf.num_kv_heads, T = cache->context;
    const size_t per_layer = static_cast<size_t>(B) * Hq * seqlen;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    for (int l = l0; l < l1; ++l) {
        const kvshare_layer& e = ctx->map[l];
        if (e.kind == KVS_SRC_LOWRANK) {
            s = prefill_lowrank_layer(ctx, cache, q, out, lse, l, seqlen, st);
            if (s != KVS_OK) return s;
            continue;
        }
        const bool mix = e.kind == KVS_SRC_MIX;
        PrefillArgs a;
        std::memset(&a, 0, sizeof(a));
        a.q = static_cast<const uint16_t*>(q) + static_cast<size_t>(l) * per_layer * D;
        a.out = static_cast<uint16_t*>(out) + static_cast<size_t>(l) * per_layer * D;
        a.lse = lse ? lse + static_cast<size_t>(l) * per_layer : nullptr;
        a.src0 = e.src0;
        a.src1 = mix ? e.src1 : e.src0;
        a.mix = mix ? 1 : 0;
        a.w = ctx->w_dev + static_cast<size_t>(l) * Hkv;
        a.B = B;
        a.Hq = Hq;
        a.Hkv = Hkv;
        a.S = seqlen;
        a.T = T;
        a.g = Hq / Hkv;
        a.scale_log2 = ctx->scale * 1.4426950408889634f;
        a.err = ctx->err;
        a.wait_limit = ctx->wait_limit;
        const int bn = prefill_kv_tile(D, mix);
        CUtensorMap tq, tk, tv, to;
        const int rows = cache->slots * B * Hkv;
        if (!get_map(ctx, a.q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, D, seqlen, B * Hq, 64, 128,
                     CU_TENSOR_MAP_SWIZZLE_128B, &tq) ||
            !get_map(ctx, a.out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, D, seqlen, B * Hq, 64, 128,
                     CU_TENSOR_MAP_SWIZZLE_128B, &to) ||
            !get_map(ctx, cache->k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, D, seqlen, rows, 64, bn,
                     CU_TENSOR_MAP_SWIZZLE_128B, &tk, T) ||
            !get_map(ctx, cache->v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, D, seqlen, rows, 64, bn,
                     CU_TENSOR_MAP_SWIZZLE_128B, &tv, T))
            return KVS_ECUDA;
        if (launch_prefill(D, mix, tq, tk, tv, to, a, st) != cudaSuccess) return KVS_ECUDA;
        ++ctx->launches;
    }
    return KVS_OK;
}

kvshare_status kvshare_pack_residual(kvshare_t ctx, const float* score, const float* u_k, const float* u_v,
                                     uint8_t* rank, int8_t* u_k8, int8_t* u_v8, uint16_t* s_k, uint16_t* s_v,
                                     int batch, int context, void* stream) {
    if (ctx == nullptr) return KVS_EINVAL;
    if (batch < 1 || context < 1) return KVS_EINVAL;
    if (ctx->cfg.max_resid_rank != 16) return KVS_EUNSUPPORTED;
    const void* in[] = {score, u_k, u_v};
    for (const void* p : in)
        if (p == nullptr || !is_device_ptr(p)) return KVS_EINVAL;
    if (!aligned16(u_k) || !aligned16(u_v) || (reinterpret_cast<uintptr_t>(score) & 3u)) return KVS_EINVAL;
    const void* outp[] = {rank, u_k8, u_v8, s_k, s_v};
    for (const void* p : outp)
        if (p == nullptr || !is_device_ptr(p)) return KVS_EINVAL;
    if (!aligned16(u_k8) || !aligned16(u_v8) || (reinterpret_cast<uintptr_t>(s_k) & 1u) ||
        (reinterpret_cast<uintptr_t>(s_v) & 1u))
        return KVS_EINVAL;
    if (cudaSetDevice(ctx->device) != cudaSuccess) return KVS_ECUDA;
    PackArgs a;
    a.score = score; a.u_k = u_k; a.u_v = u_v;
    a.rank = rank; a.u_k8 = u_k8; a.u_v8 = u_v8; a.s_k = s_k; a.s_v = s_v;
    a.tokens = static_cast<long long>(ctx->cfg.num_layers) * batch * context;
    a.Hkv = ctx->cfg.num_kv_heads;
    a.T = context;
    a.Rm = 16;
    cudaError_t e = launch_pack_residual(a, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return KVS_ECUDA;
    ++ctx->launches;
    return KVS_OK;
}

kvshare_status kvshare_append_lowrank(kvshare_t ctx, const kvshare_cache* cache, const void* k_new, const void* v_new,
                                      const float* score, const int* pos, void* stream) {
    if (ctx == nullptr || !ctx->map_set) return KVS_EINVAL;
    kvshare_status s = validate_cache_common(ctx, cache);
    if (s != KVS_OK) return s;
    const kvshare_config& cf = ctx->cfg;
    if (cf.dtype != KVS_BF16) return KVS_EUNSUPPORTED;
    if (cache->pairs < 1 || cache->pairs > APPEND_MAX_PAIRS) return cache->pairs < 1 ? KVS_EINVAL : KVS_EUNSUPPORTED;
    AppendArgs a;
    std::memset(&a, 0, sizeof(a));
    for (int i = 0; i < 2 * APPEND_MAX_PAIRS; ++i) a.pair_layers[i] = -1;
    bool any = false;
    for (int l = 0; l < cf.num_layers; ++l) {
        const kvshare_layer& e = ctx->map[l];
        if (e.kind != KVS_SRC_LOWRANK) continue;
        if (e.src0 < 0 || e.src0 >= cache->pairs) return KVS_EINVAL;
        int* pl = &a.pair_layers[2 * e.src0];
        if (pl[0] < 0) {
            pl[0] = pl[1] = l;
        } else if (pl[1] == pl[0]) {
            pl[1] = l;
        } else {
            return KVS_EUNSUPPORTED;   // a basis shared by more than two layers
        }
        any = true;
    }
    if (!any) return KVS_EINVAL;
    const void* ins[] = {k_new, v_new};
    for (const void* p : ins)
        if (!dev_ok(p)) return KVS_EINVAL;
    const void* small[] = {score, pos};
    for (const void* p : small)
        if (p == nullptr || !is_device_ptr(p) || (reinterpret_cast<uintptr_t>(p) & 3u)) return KVS_EINVAL;
    const void* cs[] = {cache->coef_k, cache->coef_v, cache->basis_k, cache->basis_v, cache->u_k, cache->u_v,
                        cache->s_k, cache->s_v, cache->r_k, cache->r_v, cache->rank};
    for (const void* p : cs)
        if (!dev_ok(p)) return KVS_EINVAL;
    if (cudaSetDevice(ctx->device) != cudaSuccess) return KVS_ECUDA;
    a.k_new = static_cast<const uint16_t*>(k_new);
    a.v_new = static_cast<const uint16_t*>(v_new);
    a.score = score;
    a.pos = pos;
    a.basis_k = static_cast<const uint16_t*>(cache->basis_k);
    a.basis_v = static_cast<const uint16_t*>(cache->basis_v);
    a.r_k = static_cast<const uint16_t*>(cache->r_k);
    a.r_v = static_cast<const uint16_t*>(cache->r_v);
    // the cache arrays the decode reads are the ones the append writes
    a.coef_k = static_cast<uint16_t*>(const_cast<void*>(cache->coef_k));
    a.coef_v = static_cast<uint16_t*>(const_cast<void*>(cache->coef_v));
    a.u_k = const_cast<int8_t*>(cache->u_k);
    a.u_v = const_cast<int8_t*>(cache->u_v);
    a.s_k = const_cast<uint16_t*>(cache->s_k);
    a.s_v = const_cast<uint16_t*>(cache->s_v);
    a.rank = const_cast<uint8_t*>(cache->rank);
    a.err = ctx->err;
    a.P = cache->pairs;
    a.B = cache->batch;
    a.Hkv = cf.num_kv_heads;
    a.T = cache->context;
    a.d = cf.head_dim;
    a.Rb = cf.basis_rank;
    if (launch_append_lowrank(a, static_cast<cudaStream_t>(stream)) != cudaSuccess) return KVS_ECUDA;
    ++ctx->launches;
    return KVS_OK;
}

kvshare_status kvshare_sync_status(kvshare_t ctx, void* stream) {
    if (ctx == nullptr) return KVS_EINVAL;
    if (cudaSetDevice(ctx->device) != cudaSuccess) return KVS_ECUDA;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return KVS_ECUDA;
    unsigned word = 0;
    if (cudaMemcpy(&word, ctx->err, sizeof(unsigned), cudaMemcpyDeviceToHost) != cudaSuccess) return KVS_ECUDA;
    if (word != 0) {
        if (cudaMemset(ctx->err, 0, sizeof(unsigned)) != cudaSuccess) return KVS_ECUDA;
        if (word & ERR_TIMEOUT) return KVS_ETIMEOUT;
        if (word & ERR_RANGE) return KVS_EINVAL;
    }
    return KVS_OK;
}

kvshare_status kvshare_set_splits(kvshare_t ctx, int splits) {
    if (ctx == nullptr || splits < 0) return KVS_EINVAL;
    ctx->splits_override = splits;
    return KVS_OK;
}

kvshare_status kvshare_set_kv_overlap(kvshare_t ctx, int on) {
    if (ctx == nullptr) return KVS_EINVAL;
    ctx->kv_overlap = on ? 1 : 0;
    return KVS_OK;
}

kvshare_status kvshare_set_layer_order(kvshare_t ctx, const int* order) {
    if (ctx == nullptr) return KVS_EINVAL;
    const int L = ctx->cfg.num_layers;
    std::vector<int> o(L);
    if (order == nullptr) {
        for (int l = 0; l < L; ++l) o[l] = l;
    } else {
        std::vector<char> seen(L, 0);
        for (int i = 0; i < L; ++i) {
            const int l = order[i];
            if (l < 0 || l >= L || seen[l]) return KVS_EINVAL;
            seen[l] = 1;
            o[i] = l;
        }
    }
    ctx->order.swap(o);
    return KVS_OK;
}

kvshare_status kvshare_debug_set_grid(kvshare_t ctx, int ctas) {
    if (ctx == nullptr || ctas < 0) return KVS_EINVAL;
    ctx->grid_override = ctas;
    return KVS_OK;
}

kvshare_status kvshare_debug_stall_next(kvshare_t ctx, int on) {
    if (ctx == nullptr) return KVS_EINVAL;
    ctx->stall_next = on ? 1 : 0;
    return KVS_OK;
}

uint64_t kvshare_launch_count(kvshare_t ctx) { return ctx ? ctx->launches : 0; }

const char* kvshare_status_string(kvshare_status s) {
    switch (s) {
        case KVS_OK: return "ok";
        case KVS_EINVAL: return "invalid argument";
        case KVS_EUNSUPPORTED: return "unsupported configuration";
        case KVS_ENOMEM: return "out of device memory";
        case KVS_ECUDA: return "CUDA runtime error";
        case KVS_ETIMEOUT: return "device wait timed out";
    }
    return "unknown status";
}

}  // extern "C"

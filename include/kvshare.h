/*
 * kvshare.h - C ABI of attention over a cross-layer shared KV cache (B200, sm_100a).
 *
 * What is computed. For every layer l, batch b and query head h (kv head
 * j = h / g, g = num_q_heads / num_kv_heads, contiguous GQA groups), softmax
 * attention of the query over K~, V~ with scale 1/sqrt(d), where K~, V~ are
 * rebuilt from a shared cache through the layer table:
 *
 *   KVS_SRC_SINGLE   K~ = K[src0]                      - a layer reuses another
 *                    layer's K/V ("Reducing Transformer Key-Value Cache Size with
 *                    Cross-Layer Attention", Methodology: some layers compute
 *                    K/V, the others reuse it; sharing factors CLA2/3/4).
 *   KVS_SRC_MIX      K~ = w[l][j] K[src0] + (1 - w[l][j]) K[src1], same for V -
 *                    a deep layer rebuilt from a stride-aligned shallow/middle
 *                    source pair ("DepthGraft: Structural Regularization through
 *                    Hierarchical Cross-Layer KV Reconstruction", Abstract; the
 *                    page gives no operator, this convex mix is the reading used).
 *   KVS_SRC_LOWRANK  K~_t = sum_{i<Rb} C_K[p][b][j][t][i] B_K[p][j][i][:]
 *                         + s_K[l][b][j][t] sum_{i<r[l][b][t]} U_K[l][b][j][t][i] R_K[l][j][i][:]
 *                    with p = src0, same for V - a layer pair shares a low-rank
 *                    basis and each layer adds its own int8 low-rank residual at a
 *                    per-token rank ("DepthWeave-KV: Smarter KV Cache Compression
 *                    by Sharing Across Layers and Adapting Per Token", Core
 *                    Mechanism and Framework Shift).
 *
 * Decode: the query attends to the cached tokens of its sequence (all `context`
 * of them, or its own length, see kvshare_cache.lengths). Prefill: query row i
 * attends to tokens 0..i (causal, no earlier context).
 *
 * Conventions for every entry point
 *   - Tensors are caller-owned DEVICE pointers (any allocator), dense and
 *     row-major in the layouts given below, 16-byte aligned. The library never
 *     frees them and keeps no reference after the call returns.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     Work is enqueued on it; no call synchronises except kvshare_sync_status.
 *   - Every call validates its arguments on the host first and returns a status
 *     without launching anything if they are invalid. Faults detected on the
 *     device (a bounded wait that ran out) are recorded in a device word and
 *     returned by the next kvshare_sync_status.
 *   - One context per host thread at a time; calls on one context are not
 *     thread-safe. Kernels of one context that overlap on the GPU (the same
 *     context used on two streams at once) share its split workspace and race.
 *   - bf16 and fp16 values travel as their 16-bit patterns (uint16_t or void*).
 */
#ifndef KVSHARE_H
#define KVSHARE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct kvshare_ctx* kvshare_t;

typedef enum {
    KVS_OK = 0,
    KVS_EINVAL = 1,        /* bad argument: null/misaligned pointer, shape, map entry, range */
    KVS_EUNSUPPORTED = 2,  /* valid but not implemented (head_dim, dtype/kind combination)   */
    KVS_ENOMEM = 3,        /* device allocation failed in kvshare_create                      */
    KVS_ECUDA = 4,         /* a CUDA runtime call failed                                      */
    KVS_ETIMEOUT = 5       /* a device-side bounded wait ran out (reported by sync_status)    */
} kvshare_status;

typedef enum { KVS_F32 = 0, KVS_BF16 = 1 } kvshare_dtype;

typedef enum { KVS_SRC_SINGLE = 0, KVS_SRC_MIX = 1, KVS_SRC_LOWRANK = 2 } kvshare_kind;

typedef struct {
    int num_layers;        /* L                                                    */
    int num_q_heads;       /* Hq, a multiple of num_kv_heads, Hq / Hkv <= 16       */
    int num_kv_heads;      /* Hkv                                                  */
    int head_dim;          /* d: 64 or 128                                         */
    kvshare_dtype dtype;   /* storage type of q, k, v (form (c) is bf16 only)      */
    float softmax_scale;   /* 0 selects 1/sqrt(d)                                  */
    int basis_rank;        /* Rb of form (c): 32, or head_dim (full-rank basis)    */
    int max_resid_rank;    /* Rm of form (c): must be 16                           */
    int max_batch;         /* largest batch any call will use                      */
    int max_context;       /* largest context any call will use                    */
} kvshare_config;

typedef struct {
    kvshare_kind kind;
    int src0;              /* store slot (SINGLE, MIX) or basis pair (LOWRANK)     */
    int src1;              /* second store slot (MIX); ignored otherwise           */
} kvshare_layer;

/* The shared cache. Forms (a)/(b) use k, v, slots. Form (c) uses the rest.
 * T below is `context`, the token count of every store.                        */
typedef struct {
    const void* k;         /* [slots][batch][Hkv][T][d]  dtype of the config     */
    const void* v;         /* [slots][batch][Hkv][T][d]                          */
    int slots;
    const void* coef_k;    /* [pairs][batch][Hkv][T][Rb] bf16                    */
    const void* coef_v;
    const void* basis_k;   /* [pairs][Hkv][Rb][d] bf16                           */
    const void* basis_v;
    const int8_t* u_k;     /* [L][batch][Hkv][T x 16] int8 residual codes, group-
                              packed: each (layer, sequence, kv head) row of T x 16
                              bytes holds its tokens in groups of 32 (group g: tokens
                              32g .. 32g+31, the last possibly shorter), group g owning
                              bytes [512 g, 512 g + 16 n_g); within a group the tokens'
                              code slots follow one another in token order, token t's
                              slot k_t = 8 ceil(min(rank_t, 16) / 8) bytes (0, 8 or 16)
                              holding its first min(rank_t, 16) codes, then zeros. The
                              other bytes of a group are unused and never read: readers
                              fetch the first pad16(sum of k) bytes of each group, so a
                              rank-0 token costs no code traffic. kvshare_pack_residual
                              and kvshare_append_lowrank write this layout. */
    const int8_t* u_v;
    const uint16_t* s_k;   /* [L][batch][Hkv][T] fp16 per-token residual scale   */
    const uint16_t* s_v;
    const void* r_k;       /* [L][Hkv][Rm][d] bf16 residual factor               */
    const void* r_v;
    const uint8_t* rank;   /* [L][batch][T] per-token residual rank, <= Rm       */
    int pairs;
    int batch;             /* 1 .. max_batch                                     */
    int context;           /* 1 .. max_context: tokens every store holds (T)      */
    const int* lengths;    /* [batch] int32 DEVICE array or NULL: sequence b's own
                              token count n_b in [0, T]; decode attends to tokens
                              0 .. n_b - 1 only, and a sequence with n_b = 0 gets
                              out 0 and lse -inf. The values are read on the device:
                              one outside [0, T] is clamped and makes the next
                              kvshare_sync_status return KVS_EINVAL. NULL: every
                              sequence has T tokens. Prefill takes NULL only. */
} kvshare_cache;

/* Create a context on the current CUDA device. Allocates the split workspace
 * (sized by max_batch / max_context) and a device status word. `out` receives
 * the handle; on failure it is set to NULL. */
kvshare_status kvshare_create(const kvshare_config* cfg, kvshare_t* out);

/* Free the context and everything it allocated. Safe with NULL. The caller
 * must make sure no work of the context is still running. */
kvshare_status kvshare_destroy(kvshare_t ctx);

/* Install the layer table (HOST pointers; both are copied).
 *   map: [num_layers] entries. SINGLE/MIX sources are store slots, LOWRANK src0
 *        a basis pair; MIX needs src0 != src1. Slot/pair ranges are checked
 *        against the cache at each decode/prefill call.
 *   w:   [num_layers][num_kv_heads] mix weights in [0, 1]; may be NULL when no
 *        entry is MIX. Rows of non-MIX layers are ignored. */
kvshare_status kvshare_set_map(kvshare_t ctx, const kvshare_layer* map, const float* w);

/* One decode step for layers [l0, l1), launched on `stream` in the context's
 * layer order (model order unless kvshare_set_layer_order changed it).
 *   q:   [L][batch][Hq][d] in the config dtype (layer l at offset l*batch*Hq*d)
 *   out: [L][batch][Hq][d] fp32
 *   lse: [L][batch][Hq] fp32 natural-log sum of exp of the scaled scores, or NULL
 * Only rows of layers [l0, l1) are written. Each launch uses programmatic
 * dependent launch: it may be scheduled while the kernel ahead of it on the
 * stream drains, but reads q and writes anything only after that kernel has
 * completed (see kvshare_set_kv_overlap for the one exception). One
 * (batch, kv head) unit may be split over several CTAs whose partials merge in
 * the context's workspace; results agree to fp32 rounding whatever the split. */
kvshare_status kvshare_decode(kvshare_t ctx, const kvshare_cache* cache, const void* q,
                              float* out, float* lse, int l0, int l1, void* stream);

/* kvshare_decode plus the attention statistics the online rank router reads
 * ("DepthWeave-KV: Smarter KV Cache Compression by Sharing Across Layers and
 * Adapting Per Token", Core Mechanism, second component: attention statistics,
 * entropy and peak, read online per token and step). With p_{h,t} the softmax
 * weight of query head h on cached token t (exactly what kvshare_decode attends
 * with), for each layer of [l0, l1):
 *   mass    [L][batch][Hkv][T] fp32: sum of p_{h,t} over the g query heads of kv
 *           head j (sums to g over t; 0 past a sequence's length)
 *   score   [L][batch][T] fp32 router score of token t: x / (1 + x) with
 *           x = (n_b * sum_j mass[j][t]) / Hq, evaluated in fp32 in that order
 *           (sum over j from 0 up, each operation correctly rounded); a token at
 *           the uniform share 1/n_b scores 0.5. kvshare_pack_residual maps it to a
 *           rank: 8 from 7/3 times the uniform share, 16 from 9 times.
 *   entropy [L][batch][Hq] fp32: -sum_t p ln p (nats) per query head
 *   peak    [L][batch][Hq] fp32: max_t p per query head
 * Any of the four may be NULL; lse is required. Entropy and peak come out of the
 * decode kernel's own online softmax and split merge (no extra pass). Mass and
 * score need the layer's final lse: the first call asking for either allocates a
 * score buffer of max_batch x Hq x max_context floats in the context (KVS_ENOMEM if
 * that fails), the decode keeps every valid token's score there, and one statistics
 * kernel per layer follows its decode kernel. Results are the same bits run to run. */
kvshare_status kvshare_decode_stats(kvshare_t ctx, const kvshare_cache* cache, const void* q, float* out,
                                    float* lse, float* mass, float* score, float* entropy, float* peak,
                                    int l0, int l1, void* stream);

/* kvshare_decode with HOST buffers: copies q for layers [l0, l1) from
 * `q_host` into a device staging buffer the context owns, decodes, and copies
 * out/lse of those layers back to `out_host`/`lse_host` (same layouts as
 * kvshare_decode, host memory; pinned memory makes the copies asynchronous).
 * The cache stays on the device. Results are valid after the stream has
 * synchronised. The staging buffers, two copy streams and their events are
 * created on the first call and reused. q is copied in as up to 8 contiguous
 * chunks of layers on one copy stream; the layers decode on `stream` in the
 * context's layer order (kvshare_set_layer_order), each once its chunk has
 * landed; a chunk's out and lse are copied back on the other copy stream once its
 * last layer has decoded (in model order: copies of one chunk under the decode of
 * the others). The copy streams wait for work already on `stream` first, and
 * `stream` waits for the last copy out, so the call is ordered on `stream` like a
 * serial one. */
kvshare_status kvshare_decode_host(kvshare_t ctx, const kvshare_cache* cache, const void* q_host,
                                   float* out_host, float* lse_host, int l0, int l1, void* stream);

/* Causal prefill of `seqlen` tokens for layers [l0, l1) (bf16 only). A MIX
 * layer's K/V operands are mixed from its two source slots inside the kernel and
 * never written to HBM. A LOWRANK layer (basis_rank 32 only, else
 * KVS_EUNSUPPORTED) runs in the absorbed form ("DepthWeave-KV: Token-Adaptive
 * Cross-Layer Residual Factorization for Long-Context KV Cache Compression",
 * Detailed Explanation: basis lookup, dequantisation and attention projection in
 * one pass): a pre-pass projects every query row to [B_K q | R_K q] (bf16, into a
 * buffer of max_batch x Hq x max_context x 64 bf16 the context allocates on first
 * use, KVS_ENOMEM if it cannot), the kernel attends over [C | s U] operands built
 * per tile in shared memory and projects the result once through [B_V; R_V]; the
 * rebuilt K/V never exist. Maps may mix all three kinds.
 * In a forward pass a slot is filled by its owner, the first layer of the map that
 * reads it as a SINGLE source, so a MIX layer's two sources must each be read as
 * SINGLE by some layer shallower than it; otherwise KVS_EINVAL ("DepthGraft:
 * Structural Regularization through Hierarchical Cross-Layer KV Reconstruction",
 * Abstract: deep layers rebuilt from shallow and middle sources). The check covers
 * the whole map, not only [l0, l1).
 *   q:   [L][batch][Hq][seqlen][d] bf16
 *   out: [L][batch][Hq][seqlen][d] bf16
 *   lse: [L][batch][Hq][seqlen] fp32 or NULL
 * K/V rows 0..seqlen-1 of each store are used (seqlen <= context); cache.lengths
 * must be NULL (KVS_EUNSUPPORTED otherwise). */
kvshare_status kvshare_prefill(kvshare_t ctx, const kvshare_cache* cache, const void* q,
                               void* out, float* lse, int l0, int l1, int seqlen, void* stream);

/* Write side of form (c) for all L layers: rank routing and int8 quantisation.
 *   score [L][batch][T] fp32 router score -> rank [L][batch][T]:
 *         0 if score < 0.7f, 8 if score < 0.9f, else 16
 *   u_k, u_v [L][batch][Hkv][T][16] fp32 residual rows ->
 *   u_k8, u_v8 [L][batch][Hkv][T x 16] int8 codes, group-packed (see
 *         kvshare_cache.u_k: token t's codes 0 .. r_t - 1 only), and s_k, s_v
 *         [L][batch][Hkv][T] fp16 scales: amax = max_{i<r}|u_i|,
 *         scale = fp16_rne(min(amax/127f, 65504)),
 *         code_i = clamp(rint(u_i / scale), -127, 127) for i < r;
 *         a zero scale gives zero codes. fp32 IEEE arithmetic, bit-exact.
 * Inputs must be finite. The unused bytes of each code group are not written. */
kvshare_status kvshare_pack_residual(kvshare_t ctx, const float* score, const float* u_k,
                                     const float* u_v, uint8_t* rank, int8_t* u_k8, int8_t* u_v8,
                                     uint16_t* s_k, uint16_t* s_v, int batch, int context,
                                     void* stream);

/* Append one new token to the form-(c) arrays of `cache`, in place (the read-only
 * fields of kvshare_cache are written here: coef_k/v, u_k/v, s_k/v, rank). A layer
 * pair shares a low-rank basis and each layer keeps a light quantised residual
 * ("DepthWeave-KV: Smarter KV Cache Compression by Sharing Across Layers and
 * Adapting Per Token", Core Mechanism, first component and diagram). For every
 * basis pair p of the layer table (its one or two LOWRANK layers la, lb), sequence
 * b and kv head j, at token index t = pos[b], for K and for V:
 *   m = (k_la + k_lb) * 0.5, c = B_p m, coef[p][b][j][t] = bf16_rne(c)
 *   e_a = k_a - B_p^T coef,  u_a = R_a e_a  (16 values) for a = la, lb
 *   rank[a][b][t] = 0 / 8 / 16 for score[a][b] below 0.7f / below 0.9f / above;
 *   codes and scale of u_a at that rank as in kvshare_pack_residual.
 * Every dot product is fp32 from index 0 up with each product and sum correctly
 * rounded (no fused multiply-add), so coefficients and codes are bit-reproducible.
 *   k_new, v_new: [L][batch][Hkv][d] bf16 DEVICE: the token's key and value in
 *                 every layer (rows of non-LOWRANK layers are not read)
 *   score:        [L][batch] fp32 DEVICE router score of the token per layer
 *   pos:          [batch] int32 DEVICE token index to write; an index outside
 *                 [0, context) writes nothing for that sequence and makes the next
 *                 kvshare_sync_status return KVS_EINVAL. The token's codes go after
 *                 those of its code group's earlier tokens (group-packed layout, by
 *                 their stored ranks), so later tokens of the same 32-token group
 *                 must not have been written yet (appends run in token order; the
 *                 last token may be rewritten).
 * The caller then raises the sequences' lengths. A basis pair read by more than two
 * layers, or more than 64 pairs: KVS_EUNSUPPORTED. A decode that follows an append
 * on the same stream must run with kvshare_set_kv_overlap off. */
kvshare_status kvshare_append_lowrank(kvshare_t ctx, const kvshare_cache* cache, const void* k_new,
                                      const void* v_new, const float* score, const int* pos, void* stream);

/* Synchronise `stream`, then read and clear the device status word.
 * Returns KVS_OK, KVS_ETIMEOUT (a bounded device wait ran out), KVS_EINVAL (a
 * per-sequence length outside [0, context] was clamped) or KVS_ECUDA. */
kvshare_status kvshare_sync_status(kvshare_t ctx, void* stream);

/* Split-KV override for decode: 0 = automatic (default), n > 0 = n splits per
 * (batch, kv head), clamped to the number of token tiles and the workspace. */
kvshare_status kvshare_set_splits(kvshare_t ctx, int splits);

/* Overlap of consecutive decode launches (default off). Every decode launch may
 * start (barrier set-up, tensor-map fetch) while the kernel ahead of it on the
 * stream drains, and waits for that kernel before it reads q or writes anything.
 * With `on` != 0 the bf16 decode also requests its first K/V tiles before that
 * wait, and the low-rank decode its bases, residual factors, first coefficient
 * and code tiles and their per-token scales and ranks. Set it only when no kernel that can still be running when kvshare_decode
 * is called writes the cache regions the call reads (for example: the step's
 * cache appends were made before the kernels ahead of the decode, or the layers
 * decoded read sources nothing is appending to); otherwise a tile could be read
 * before it is written. Results are identical either way. */
kvshare_status kvshare_set_kv_overlap(kvshare_t ctx, int on);

/* Order in which kvshare_decode and kvshare_decode_host launch the layers of a
 * call: `order` is a HOST array of num_layers distinct layer indices (a
 * permutation, copied); a call over [l0, l1) runs the layers of that range in the
 * order they appear in it. NULL restores model order 0, 1, ..., L-1. Each layer's
 * attention depends only on its own q and sources, so results do not change; the
 * order decides which shared sources are still in L2 when a layer reads them.
 * KVS_EINVAL if an entry is out of range or repeated. */
kvshare_status kvshare_set_layer_order(kvshare_t ctx, const int* order);


/* Test hook: force the bf16 decode grid to `ctas` CTAs (0 = automatic). The
 * units' token tiles are cut into that many equal ranges, so a CTA may cover
 * the end of one (batch, kv head) unit and the start of the next; the units'
 * partial results merge exactly as with the automatic grid. Values are
 * clamped to [batch * Hkv, total tiles]. */
kvshare_status kvshare_debug_set_grid(kvshare_t ctx, int ctas);

/* Test hook for the bounded waits: when `on` is non-zero, the next decode
 * launch makes one warp wait on a barrier nothing arrives on, with a limit of
 * about 10 ms; the wait gives up, records KVS_ETIMEOUT and the kernel still
 * completes. The hook clears itself after one launch. */
kvshare_status kvshare_debug_stall_next(kvshare_t ctx, int on);

/* Number of kernels this context has launched since it was created. */
uint64_t kvshare_launch_count(kvshare_t ctx);

/* One bf16 decode layer that allocates no device memory. The paper has no
 * counterpart; this entry point exists for callers that cannot call cudaMalloc
 * (code inside a capture or a host framework whose own allocator must own all
 * device memory, or a process whose footprint must not grow after start-up).
 * It needs no context: the split partials, arrival counters and status word
 * live in a fixed 2 MiB device array inside this library, which every GPU that
 * loads the library holds until the process exits.
 *   q:   [batch][Hq][d] bf16        out: [batch][Hq][d] fp32
 *   lse: [batch][Hq] fp32 or NULL   k, v: [slots][batch][Hkv][T][d] bf16 (T = context)
 *   src1 < 0: single source src0; src1 >= 0: convex mix of src0 and src1 with
 *   w: [Hkv] fp32 device weights in [0, 1] (ignored for a single source).
 *   Softmax scale 1/sqrt(d); d is 64 or 128; Hq / Hkv <= 16.
 * Limits: batch * Hkv <= 4096, else KVS_EINVAL; the split count is lowered
 * until the partials fit the array. Every pointer must be device (or managed)
 * memory, checked with cudaPointerGetAttributes: host memory, mapped pinned
 * memory included, gives KVS_EINVAL. The first call on each device looks up
 * the array's device address (cudaGetSymbolAddress) and should come before
 * any stream capture. Every call shares the array and keeps the previous
 * call's contents; the call clears the counters and status word on `stream`
 * first. Calls that overlap on the GPU (two streams, two host threads) race on
 * the array. Device-side wait timeouts are recorded in the array's status word
 * and not reported. */
kvshare_status kvshare_decode_layer_noalloc(const void* q, const void* k, const void* v, const float* w,
                                            float* out, float* lse, int batch, int num_q_heads,
                                            int num_kv_heads, int head_dim, int context, int slots,
                                            int src0, int src1, void* stream);

/* Static text for a status code. */
const char* kvshare_status_string(kvshare_status s);

#ifdef __cplusplus
}
#endif
#endif /* KVSHARE_H */

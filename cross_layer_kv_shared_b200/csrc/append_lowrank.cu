// Append one new token to a low-rank cache: shared coefficients, per-layer residual codes.
//
// A layer pair shares a low-rank channel basis and each layer keeps a light
// residual for what the basis misses ("DepthWeave-KV: Smarter KV Cache Compression
// by Sharing Across Layers and Adapting Per Token", Core Mechanism, first
// component and diagram). For the new token of sequence b at position pos[b], per
// basis pair p (layers la, lb; la == lb for a pair of one layer), kv head j, and
// for K and V alike, with k_la, k_lb the token's vectors in the two layers:
//   m     = (k_la + k_lb) * 0.5                          (the pair's least-squares fit
//   c     = B_p m,  c_stored = bf16_rne(c)                  in an orthonormal basis)
//   e_a   = k_a - B_p^T c_stored                         (what the stored part misses)
//   u_a   = R_a e_a                                       (16 residual coordinates)
//   codes, scale of u_a at the rank the router gives the token in layer a
// Every dot product runs in fp32 from index 0 up, each product and each sum
// correctly rounded (no fused multiply-add), so the bf16 coefficients and the
// integer codes are reproducible bit for bit. One CTA per (pair, sequence, kv head,
// K or V): the two sides' dependent chains run side by side on different SMs. A CTA
// first copies the pair's basis and both layers' residual factors into shared memory
// (one coalesced pass), then walks them there.
#include "kvs_quant.cuh"

namespace kvs {
namespace {

constexpr int NT = 128;
constexpr int LDB = 128 + 2;   // padded bf16 rows: a walk along a row (thread per row) and down a
                               // column (thread per column) both fall on distinct banks

__device__ __forceinline__ float bf(uint16_t v) { return __uint_as_float(static_cast<uint32_t>(v) << 16); }

__global__ void __launch_bounds__(NT) append_lowrank_kernel(const AppendArgs a) {
    const int p = blockIdx.x;
    const int b = blockIdx.y;
    const int j = blockIdx.z >> 1;
    const int side = blockIdx.z & 1;                      // 0: K, 1: V
    const int tid = threadIdx.x;
    const int la = a.pair_layers[2 * p], lb = a.pair_layers[2 * p + 1];
    if (la < 0) return;                                   // a pair no layer reads
    const int nl = lb == la ? 1 : 2;
    const int t = a.pos[b];
    if (t < 0 || t >= a.T) {
        if (tid == 0) atomicOr(a.err, ERR_RANGE);
        return;
    }
    const int D = a.d, RB = a.Rb;
    extern __shared__ uint16_t sfac[];                    // [RB basis rows | nl x 16 factor rows][LDB]
    __shared__ float kk[2][128], m[128], cst[128], e[2][128], us[2][QUANT_RM];
    const size_t BHkv = static_cast<size_t>(a.B) * a.Hkv;
    const size_t bj = static_cast<size_t>(b) * a.Hkv + j;
    const int rows = RB + nl * QUANT_RM;
    {
        const uint16_t* nw = side == 0 ? a.k_new : a.v_new;
        const uint16_t* basis = (side == 0 ? a.basis_k : a.basis_v) + (static_cast<size_t>(p) * a.Hkv + j) * RB * D;
        const uint16_t* Rf = side == 0 ? a.r_k : a.r_v;
        // the pair's basis and both layers' residual factors, in one coalesced pass
        // (loads in groups of eight per thread before any store: one round trip a group)
        constexpr int G = 8;
        for (int i0 = tid; i0 < rows * (D / 8); i0 += G * NT) {
            uint4 v[G];
#pragma unroll
            for (int k = 0; k < G; ++k) {
                const int idx = i0 + k * NT;
                if (idx >= rows * (D / 8)) break;
                const int r = idx / (D / 8), c8 = idx % (D / 8);
                const uint16_t* src;
                if (r < RB) {
                    src = basis + static_cast<size_t>(r) * D;
                } else {
                    const int ai = (r - RB) / QUANT_RM, s = (r - RB) % QUANT_RM;
                    src = Rf + ((static_cast<size_t>(ai == 0 ? la : lb) * a.Hkv + j) * QUANT_RM + s) * D;
                }
                v[k] = *reinterpret_cast<const uint4*>(src + c8 * 8);
            }
#pragma unroll
            for (int k = 0; k < G; ++k) {
                const int idx = i0 + k * NT;
                if (idx >= rows * (D / 8)) break;
                const int r = idx / (D / 8), c8 = idx % (D / 8);
                uint32_t* dst = reinterpret_cast<uint32_t*>(sfac + r * LDB + c8 * 8);
                dst[0] = v[k].x; dst[1] = v[k].y; dst[2] = v[k].z; dst[3] = v[k].w;
            }
        }
        if (tid < D) {
            const float x0 = bf(nw[(la * BHkv + bj) * D + tid]);
            const float x1 = bf(nw[(lb * BHkv + bj) * D + tid]);
            kk[0][tid] = x0;
            kk[1][tid] = x1;
            m[tid] = __fmul_rn(__fadd_rn(x0, x1), 0.5f);
        }
        __syncthreads();
        if (tid < RB) {
            const uint16_t* row = sfac + tid * LDB;
            float c = __fmul_rn(bf(row[0]), m[0]);
            for (int i = 1; i < D; ++i) c = __fadd_rn(c, __fmul_rn(bf(row[i]), m[i]));
            const __nv_bfloat16 cb = __float2bfloat16_rn(c);
            cst[tid] = __bfloat162float(cb);
            uint16_t* coef = side == 0 ? a.coef_k : a.coef_v;
            coef[((static_cast<size_t>(p) * BHkv + bj) * a.T + t) * RB + tid] = __bfloat16_as_ushort(cb);
        }
        __syncthreads();
        if (tid < D) {
            float r = __fmul_rn(cst[0], bf(sfac[tid]));
            for (int i = 1; i < RB; ++i) r = __fadd_rn(r, __fmul_rn(cst[i], bf(sfac[i * LDB + tid])));
            e[0][tid] = __fsub_rn(kk[0][tid], r);
            e[1][tid] = __fsub_rn(kk[1][tid], r);
        }
        __syncthreads();
        if (tid < nl * QUANT_RM) {
            const int ai = tid / QUANT_RM;
            const uint16_t* R = sfac + (RB + tid) * LDB;
            float u = __fmul_rn(bf(R[0]), e[ai][0]);
            for (int i = 1; i < D; ++i) u = __fadd_rn(u, __fmul_rn(bf(R[i]), e[ai][i]));
            us[ai][tid % QUANT_RM] = u;
        }
        __syncthreads();
        if (tid < nl) {
            const int l = tid == 0 ? la : lb;
            const uint8_t r = route_rank(a.score[static_cast<size_t>(l) * a.B + b]);
            float x[QUANT_RM];
#pragma unroll
            for (int i = 0; i < QUANT_RM; ++i) x[i] = us[tid][i];
            uint32_t packed[4];
            uint16_t sc;
            quantize16(x, r, packed, sc);
            const size_t row = (static_cast<size_t>(l) * BHkv + bj) * a.T + t;
            // group-packed codes: after those of the group's earlier tokens
            const int t0 = t - t % CODE_GROUP;
            const uint8_t* rk = a.rank + (static_cast<size_t>(l) * a.B + b) * a.T;
            int o = 0;
            for (int tt = t0; tt < t; ++tt) o += code_len(rk[tt]);
            int8_t* codes = side == 0 ? a.u_k : a.u_v;
            store_codes(codes + (row - (t - t0)) * QUANT_RM + o, packed, code_len(r));
            (side == 0 ? a.s_k : a.s_v)[row] = sc;
            if (side == 0 && j == 0) a.rank[(static_cast<size_t>(l) * a.B + b) * a.T + t] = r;
        }
    }
}

}  // namespace

cudaError_t launch_append_lowrank(const AppendArgs& a, cudaStream_t st) {
    dim3 grid(a.P, a.B, 2 * a.Hkv);
    // at most (128 + 32) rows of LDB bf16 (41.6 KB), with the static arrays under 48 KB
    const size_t smem = static_cast<size_t>(a.Rb + 2 * QUANT_RM) * LDB * sizeof(uint16_t);
    append_lowrank_kernel<<<grid, NT, smem, st>>>(a);
    return cudaGetLastError();
}

}  // namespace kvs

// bwd.cu -- backward pass of the DashAttention forward: dL/dQ, dL/dK, dL/dV for an
// output gradient dO ("DashAttention", §3.3-3.4 and the differentiable hierarchy of
// App. A; the chain rule in the forward's order reversed).
//
// For each row i of head h (KV group r) the forward computes
//   l_j = z_j + b_j,  z_j = <q_i, k_j>/sqrt(d),  P = softmax(l),  o_i = sum_j P_j v_j,
// over the routed chunks' keys (b_j = d_c = (log w_c - mu_i)/sigma) and the local
// window (b_j = 0).  Its gradient, with D_i = <dO_i, o_i>:
//   dl_j = P_j (<dO_i, v_j> - D_i),  dv_j += P_j dO_i,  dk_j += dl_j q_i / sqrt(d),
//   dq_i += sum_j dl_j k_j / sqrt(d),
// and the prior bias of each routed chunk c collects G_c(i) = sum over the group's heads
// and the chunk's keys of dl_j.  Through Prop. 1's d_c = (log w_c - mu)/sigma with mu the
// mean of log w over R_i: d(log w_c) = (G_c - mean_R G)/sigma; w_c = (1/g) sum_h p_c^(h)
// gives dp_c^(h) = dw_c / g; the alpha-entmax of §2 Eq. 2 has the Jacobian
// diag(u) - u u^T / sum u with u = p^(2-alpha) on the head's support, so
// ds_c = u_c (dp_c - <u, dp> / sum u) for the Stage-1 score s_c = gamma <q, kbar_c>/sqrt(d)
// (Eq. 4), which sends gamma ds_c kbar_c / sqrt(d) to q and gamma ds_c q / sqrt(d) to
// kbar_c; Stage 0's mean pooling (Eq. 3 with a zero summary query) hands each key of
// chunk c the share dkbar_c / |C_c|.  Supports are piecewise constant: no gradient.
//
// Kernels here (CUDA cores; the tensor-core Stage-2 kernels are in attn_bwd_tc.cu):
//   bwd_rowdot_kernel     D = <dO, O> per (row, head)
//   bwd_dq_simt_kernel    per query tile: P, dP, dl; dQ (Stage 2) and G per routed chunk
//   refs_mark_kernel,     the work lists transposed: for every key block the (tile,
//   refs_build_kernel     entry) pairs that attend it, tiles ascending (deterministic)
//   bwd_dkdv_simt_kernel  per key block: dK (Stage 2 + pooling share), dV over its pairs
//   bwd_route_kernel      per (row, kv head): the prior / entmax / score chain above, added
//                         to the Stage-2 part of dQ, which it writes in the caller's dtype,
//                         and (atomically) to the chunk summaries' gradient
//   bwd_dq_finish_kernel  dQ to the caller's dtype when no row routes anything
#include <math.h>

#include "dash_common.cuh"
#include "kernels.h"

namespace dash {

namespace {

constexpr float kLog2e = 1.4426950408889634f;

// ---------------------------------------------------------------------------
// D_i = <dO_i, O_i>, one warp per (batch, row, head)
// ---------------------------------------------------------------------------
template <typename T>
__global__ void bwd_rowdot_kernel(TView dO, TView O, Geom G, float *__restrict__ Drow) {
    const int64_t w = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / 32;
    const int lane = threadIdx.x % 32;
    const int64_t n = G.b * G.nq * G.hq;
    if (w >= n) return;
    const int h = (int)(w % G.hq);
    const int64_t i = (w / G.hq) % G.nq, b = w / ((int64_t)G.hq * G.nq);
    const T *a = reinterpret_cast<const T *>(dO.p) + b * dO.s0 + i * dO.s1 + (int64_t)h * dO.s2;
    const T *o = reinterpret_cast<const T *>(O.p) + b * O.s0 + i * O.s1 + (int64_t)h * O.s2;
    float acc = 0.f;
    for (int e = lane; e < G.d; e += 32) acc = fmaf(to_f<T>(a[e]), to_f<T>(o[e]), acc);
    acc = warp_sum(acc);
    if (lane == 0) Drow[w] = acc;
}

// Is chunk c routed (not part of the local window) for row i?
__device__ __forceinline__ bool routable(const Geom &G, int64_t i, int c) { return c < row_nvis(G, i); }

// ---------------------------------------------------------------------------
// Stage 2, query side on CUDA cores: one CTA per (tile, kv head, batch), thread m = tile
// row m = pos * g + head.  Recomputes P from the forward's lse, then dl, dQ and G.
// ---------------------------------------------------------------------------
constexpr int kRows = 128;
constexpr int kSubB = 16;  // keys staged per step

template <typename T>
__global__ void __launch_bounds__(kRows) bwd_dq_simt_kernel(TView Q, TView K, TView V, TView dO, Geom G, ListsView L,
                                                            const float *__restrict__ lse,
                                                            const float *__restrict__ Drow, float *__restrict__ dQacc,
                                                            float *__restrict__ Gd) {
    extern __shared__ __align__(16) float sm[];
    const int d = G.d, g = G.g, dp = d + 1;
    float *Qs = sm;                     // [128][d+1]
    float *dOs = Qs + kRows * dp;       // [128][d+1]
    float *dQs = dOs + kRows * dp;      // [128][d+1]
    float *Ks = dQs + kRows * dp;       // [kSubB][d+1]
    float *Vs = Ks + kSubB * dp;        // [kSubB][d+1]
    float *Gsm = Vs + kSubB * dp;       // [128] per-row G of the current entry

    const int64_t t = blockIdx.x;
    const int r = blockIdx.y;
    const int64_t b = blockIdx.z;
    const int TR = L.tile_rows, M = TR * g, m = threadIdx.x;
    const int pos = m / g, hh = m % g;
    const size_t tile_idx = ((size_t)b * G.hkv + r) * L.n_tiles + t;
    const int64_t i = m < M ? tile_row(L, G, tile_idx, t, pos) : -1;
    const bool valid = i >= 0;
    const int64_t p_i = row_pos(G, i);
    const int h = r * g + hh;
    const size_t row_id = valid ? ((size_t)b * G.nq + i) * G.hq + h : 0;

    const T *qp = reinterpret_cast<const T *>(Q.p) + b * Q.s0 + (valid ? i : 0) * Q.s1 + (int64_t)h * Q.s2;
    const T *gp = reinterpret_cast<const T *>(dO.p) + b * dO.s0 + (valid ? i : 0) * dO.s1 + (int64_t)h * dO.s2;
    for (int e = 0; e < d; ++e) {
        Qs[m * dp + e] = valid ? to_f<T>(qp[e]) : 0.f;
        dOs[m * dp + e] = valid ? to_f<T>(gp[e]) : 0.f;
        dQs[m * dp + e] = 0.f;
    }
    const float sl2 = rsqrtf((float)d) * kLog2e;
    const float L2 = valid ? lse[row_id] * kLog2e : INFINITY;
    const float Dv = valid ? Drow[row_id] : 0.f;
    const T *kbp = reinterpret_cast<const T *>(K.p) + b * K.s0 + (int64_t)r * K.s2;
    const T *vbp = reinterpret_cast<const T *>(V.p) + b * V.s0 + (int64_t)r * V.s2;
    const int count = L.count[tile_idx];
    const int32_t *ids = L.ids + tile_idx * L.cap;
    const float *bias = L.bias + tile_idx * (size_t)L.cap * TR;

    for (int e_idx = 0; e_idx < count; ++e_idx) {
        const int c = ids[e_idx];
        const float bv = (m < M) ? bias[(size_t)e_idx * TR + pos] : -INFINITY;
        const float bl2 = bv * kLog2e;
        const int64_t k0 = (int64_t)c * G.B;
        float gsum = 0.f;
        for (int j0 = 0; j0 < G.B; j0 += kSubB) {
            __syncthreads();
            for (int idx = threadIdx.x; idx < kSubB * d; idx += kRows) {
                const int jj = idx / d, e = idx % d;
                const int64_t key = k0 + j0 + jj;
                const bool in = (j0 + jj < G.B) && key < G.nk;
                Ks[jj * dp + e] = in ? to_f<T>(kbp[key * K.s1 + e]) : 0.f;
                Vs[jj * dp + e] = in ? to_f<T>(vbp[key * V.s1 + e]) : 0.f;
            }
            __syncthreads();
            if (!valid || bv == -INFINITY) continue;
            for (int jj = 0; jj < kSubB; ++jj) {
                const int64_t key = k0 + j0 + jj;
                if (j0 + jj >= G.B || key >= G.nk || (G.causal && key > p_i)) continue;
                float s = 0.f, dpv = 0.f;
                for (int e = 0; e < d; ++e) {
                    s = fmaf(Qs[m * dp + e], Ks[jj * dp + e], s);
                    dpv = fmaf(dOs[m * dp + e], Vs[jj * dp + e], dpv);
                }
                const float P = exp2f(s * sl2 + bl2 - L2);
                const float dl = P * (dpv - Dv);
                gsum += dl;
                for (int e = 0; e < d; ++e) dQs[m * dp + e] = fmaf(dl, Ks[jj * dp + e], dQs[m * dp + e]);
            }
        }
        // G of this chunk for the row's position: the sum over the group's g heads
        // (rows pos * g .. pos * g + g - 1)
        Gsm[m] = gsum;
        __syncthreads();
        if (valid && hh == 0 && bv > -INFINITY && routable(G, i, c)) {
            float gs = 0.f;
            for (int x = 0; x < g; ++x) gs += Gsm[m + x];
            Gd[logw_index(G, b, r, i, c)] = gs;
        }
    }
    if (valid) {
        const float sc = rsqrtf((float)d);
        float *dst = dQacc + row_id * d;
        for (int e = 0; e < d; ++e) dst[e] = dQs[m * dp + e] * sc;
    }
}

// ---------------------------------------------------------------------------
// Transposed work lists.  refs_mark: one thread per (tile, entry) marks the key block
// in a per-block bitmap over tiles and records the entry index.  refs_build: one CTA
// per (kv head, batch) counts each block's tiles, scans, and writes the (tile, entry)
// pairs of every block with tiles ascending.
// ---------------------------------------------------------------------------
__global__ void refs_mark_kernel(Geom G, ListsView L, uint32_t *__restrict__ bitmap, int32_t *__restrict__ E,
                                 int tw) {
    const int64_t t = blockIdx.x;
    const int r = blockIdx.y;
    const int64_t b = blockIdx.z;
    const size_t tile_idx = ((size_t)b * G.hkv + r) * L.n_tiles + t;
    const int count = L.count[tile_idx];
    const size_t bh = (size_t)b * G.hkv + r;
    for (int e = threadIdx.x; e < count; e += blockDim.x) {
        const int c = L.ids[tile_idx * L.cap + e];
        atomicOr(bitmap + (bh * G.n_blk + c) * tw + t / 32, 1u << (t % 32));
        E[(bh * G.n_blk + c) * L.n_tiles + t] = e;
    }
}

__global__ void __launch_bounds__(1024) refs_build_kernel(Geom G, int64_t n_tiles, const uint32_t *__restrict__ bitmap,
                                                          const int32_t *__restrict__ E, int tw,
                                                          int32_t *__restrict__ ref_off, int32_t *__restrict__ ref_cnt,
                                                          int2 *__restrict__ refs) {
    __shared__ int part[1024];
    const int r = blockIdx.x;
    const int64_t b = blockIdx.y;
    const size_t bh = (size_t)b * G.hkv + r;
    const int nb = G.n_blk;
    const int per = (nb + blockDim.x - 1) / blockDim.x;
    const int c0 = threadIdx.x * per, c1 = min(nb, c0 + per);
    int mine = 0;
    for (int c = c0; c < c1; ++c) {
        int n = 0;
        for (int w = 0; w < tw; ++w) n += __popc(bitmap[(bh * nb + c) * tw + w]);
        ref_cnt[bh * nb + c] = n;
        mine += n;
    }
    part[threadIdx.x] = mine;
    __syncthreads();
    // exclusive scan of the per-thread totals (Hillis-Steele in shared memory)
    for (int o = 1; o < (int)blockDim.x; o <<= 1) {
        const int v = threadIdx.x >= (unsigned)o ? part[threadIdx.x - o] : 0;
        __syncthreads();
        part[threadIdx.x] += v;
        __syncthreads();
    }
    int off = part[threadIdx.x] - mine;
    int2 *out = refs + bh * (size_t)n_tiles * nb;
    for (int c = c0; c < c1; ++c) {
        ref_off[bh * nb + c] = off;
        for (int w = 0; w < tw; ++w) {
            uint32_t bits = bitmap[(bh * nb + c) * tw + w];
            while (bits) {
                const int t = w * 32 + __ffs(bits) - 1;
                bits &= bits - 1;
                out[off++] = make_int2(t, E[(bh * nb + c) * n_tiles + t]);
            }
        }
    }
}

// ---------------------------------------------------------------------------
// Stage 2, key side on CUDA cores: one CTA per (key block of KB = min(B, 64) keys, kv
// head, batch); thread (key j, part) with parts = 128 / KB threads per key, each part a
// d / parts slice.  The attending rows stream through shared memory 32 at a time.
// ---------------------------------------------------------------------------
constexpr int kRowChunk = 32;

template <typename T>
__global__ void __launch_bounds__(128) bwd_dkdv_simt_kernel(TView Q, TView K, TView V, TView dO, TView dK, TView dV,
                                                            Geom G, ListsView L, const float *__restrict__ lse,
                                                            const float *__restrict__ Drow,
                                                            const int32_t *__restrict__ ref_off,
                                                            const int32_t *__restrict__ ref_cnt,
                                                            const int2 *__restrict__ refs,
                                                            const float *__restrict__ dKbar) {
    extern __shared__ __align__(16) float sm[];
    const int d = G.d, g = G.g, dp = d + 1;
    const int KB = G.B < 64 ? G.B : 64;
    const int parts = 128 / KB, slice = d / parts;
    float *Ks = sm;                          // [KB][d+1]
    float *Vs = Ks + KB * dp;                // [KB][d+1]
    float *dKs = Vs + KB * dp;               // [KB][d+1]
    float *dVs = dKs + KB * dp;              // [KB][d+1]
    float *Qs = dVs + KB * dp;               // [kRowChunk][d+1]
    float *Gs = Qs + kRowChunk * dp;         // [kRowChunk][d+1] dO rows
    float *rowL = Gs + kRowChunk * dp;       // [kRowChunk] lse (exp2 domain), +inf = no row
    float *rowD = rowL + kRowChunk;          // [kRowChunk]
    float *rowB = rowD + kRowChunk;          // [kRowChunk] bias (exp2 domain)
    long long *rowP = reinterpret_cast<long long *>(rowB + kRowChunk);  // [kRowChunk] key position p_i

    const int kb = blockIdx.x, r = blockIdx.y;
    const int64_t b = blockIdx.z;
    const int c = (int)((int64_t)kb * KB / G.B);           // chunk (list entry id) of this key block
    const int64_t key0 = (int64_t)kb * KB;
    const int j = threadIdx.x / parts, part = threadIdx.x % parts;
    const int e0 = part * slice;
    const int64_t key = key0 + j;
    const T *kbp = reinterpret_cast<const T *>(K.p) + b * K.s0 + (int64_t)r * K.s2;
    const T *vbp = reinterpret_cast<const T *>(V.p) + b * V.s0 + (int64_t)r * V.s2;
    for (int idx = threadIdx.x; idx < KB * d; idx += 128) {
        const int jj = idx / d, e = idx % d;
        const int64_t kk = key0 + jj;
        Ks[jj * dp + e] = kk < G.nk ? to_f<T>(kbp[kk * K.s1 + e]) : 0.f;
        Vs[jj * dp + e] = kk < G.nk ? to_f<T>(vbp[kk * V.s1 + e]) : 0.f;
        dKs[jj * dp + e] = 0.f;
        dVs[jj * dp + e] = 0.f;
    }
    const size_t bh = (size_t)b * G.hkv + r;
    const int nref = ref_cnt[bh * G.n_blk + c];
    const int2 *rl = refs + bh * (size_t)L.n_tiles * G.n_blk + ref_off[bh * G.n_blk + c];
    const float sl2 = rsqrtf((float)d) * kLog2e;
    const int TR = L.tile_rows, M = TR * g;
    for (int q = 0; q < nref; ++q) {
        const int64_t t = rl[q].x;
        const int e = rl[q].y;
        const size_t tile_idx = bh * L.n_tiles + t;
        const float *bias = L.bias + tile_idx * (size_t)L.cap * TR + (size_t)e * TR;
        for (int m0 = 0; m0 < M; m0 += kRowChunk) {
            __syncthreads();
            if (threadIdx.x < kRowChunk) {
                const int m = m0 + threadIdx.x;
                const int64_t i = m < M ? tile_row(L, G, tile_idx, t, m / g) : -1;
                const float bv = i >= 0 ? bias[m / g] : -INFINITY;
                const size_t rid = ((size_t)b * G.nq + (i >= 0 ? i : 0)) * G.hq + r * g + m % g;
                rowL[threadIdx.x] = (i >= 0 && bv > -INFINITY) ? lse[rid] * kLog2e : INFINITY;
                rowD[threadIdx.x] = i >= 0 ? Drow[rid] : 0.f;
                rowB[threadIdx.x] = bv * kLog2e;
                rowP[threadIdx.x] = i >= 0 ? row_pos(G, i) : -1;
            }
            for (int idx = threadIdx.x; idx < kRowChunk * d; idx += 128) {
                const int mm = idx / d, ee = idx % d, m = m0 + mm;
                const int64_t i = m < M ? tile_row(L, G, tile_idx, t, m / g) : -1;
                const int hq = r * g + m % g;
                Qs[mm * dp + ee] = i >= 0 ? to_f<T>(reinterpret_cast<const T *>(Q.p)[b * Q.s0 + i * Q.s1 +
                                                                                     (int64_t)hq * Q.s2 + ee])
                                          : 0.f;
                Gs[mm * dp + ee] = i >= 0 ? to_f<T>(reinterpret_cast<const T *>(dO.p)[b * dO.s0 + i * dO.s1 +
                                                                                       (int64_t)hq * dO.s2 + ee])
                                          : 0.f;
            }
            __syncthreads();
            for (int mm = 0; mm < kRowChunk; ++mm) {
                float s = 0.f, dpv = 0.f;
                for (int x = 0; x < slice; ++x) {
                    s = fmaf(Qs[mm * dp + e0 + x], Ks[j * dp + e0 + x], s);
                    dpv = fmaf(Gs[mm * dp + e0 + x], Vs[j * dp + e0 + x], dpv);
                }
                for (int o = 1; o < parts; o <<= 1) {  // the key's parts are consecutive lanes
                    s += __shfl_xor_sync(0xffffffffu, s, o);
                    dpv += __shfl_xor_sync(0xffffffffu, dpv, o);
                }
                const bool live = rowL[mm] < INFINITY && key < G.nk && (!G.causal || key <= rowP[mm]);
                if (!live) continue;
                const float P = exp2f(s * sl2 + rowB[mm] - rowL[mm]);
                const float dl = P * (dpv - rowD[mm]);
                for (int x = 0; x < slice; ++x) {
                    dVs[j * dp + e0 + x] = fmaf(P, Gs[mm * dp + e0 + x], dVs[j * dp + e0 + x]);
                    dKs[j * dp + e0 + x] = fmaf(dl, Qs[mm * dp + e0 + x], dKs[j * dp + e0 + x]);
                }
            }
        }
    }
    __syncthreads();
    // keys of a routing chunk also receive their share of the summary's gradient
    const float sc = rsqrtf((float)d);
    for (int idx = threadIdx.x; idx < KB * d; idx += 128) {
        const int jj = idx / d, e = idx % d;
        const int64_t kk = key0 + jj;
        if (kk >= G.nk) continue;
        float dk = dKs[jj * dp + e] * sc;
        if (c < G.n_chunks) {
            const int64_t size = min((int64_t)G.B, G.nk - (int64_t)c * G.B);
            dk += dKbar[(((size_t)b * G.n_chunks + c) * G.hkv + r) * d + e] / (float)size;
        }
        reinterpret_cast<T *>(const_cast<void *>(dK.p))[b * dK.s0 + kk * dK.s1 + (int64_t)r * dK.s2 + e] = from_f<T>(dk);
        reinterpret_cast<T *>(const_cast<void *>(dV.p))[b * dV.s0 + kk * dV.s1 + (int64_t)r * dV.s2 + e] =
            from_f<T>(dVs[jj * dp + e]);
    }
}

// ---------------------------------------------------------------------------
// Routing gradient on CUDA cores: one warp per (batch, row, kv head), four warps per CTA.
// The group's g query rows are staged in shared memory.  The routed set R_i (mask bits)
// is walked 32 chunks at a time, one chunk per lane:
//   pass 1  mean G over R_i;
//   pass 2  each lane forms x = xs <q_h, kbar_c> for the g heads of its chunk (q from
//           shared memory, kbar_c from global) and sums u and u dp per head; one warp
//           reduction per head at the end gives <u, dp> / sum u;
//   pass 3  each lane forms ds_h = u dp - u <u, dp> / sum u for its chunk; then the lanes
//           take dimensions and, chunk by chunk, add ds_h kbar_c to dq_h and
//           sum_h ds_h q_h to the chunk summary's gradient (atomically).
// dQ (the Stage-2 part from dQacc plus this part) is written in the caller's dtype.
// ---------------------------------------------------------------------------
constexpr int kRouteWarps = 4;

// The per-chunk arithmetic: for head h's x = xs <q, kbar_c> and threshold th,
// p = (x - th)^(1/(alpha-1)), u = p^(2-alpha) and u dp with dp = d(log w_c) / (g w_c);
// false outside the head's own support (u = 0 there).
__device__ __forceinline__ bool route_terms(float x, float th, float kexp, float uexp, float lw, float dlw, int g,
                                            float &u, float &ud) {
    if (!(x > th)) return false;
    const float lp = kexp * __logf(x - th);        // log p
    u = __expf(uexp * lp);                          // p^(2 - alpha)
    ud = __expf(uexp * lp - lw) * dlw / (float)g;   // u dp
    return true;
}

// chunk id of routed-set element n (ascending) of the row, from its mask words; -1 past the end
__device__ __forceinline__ int nth_routed(const uint32_t *mrow, int wv, int nvis, int n) {
    for (int wd = 0; wd < wv; ++wd) {
        uint32_t bits = mrow[wd];
        if (wd == wv - 1 && (nvis & 31)) bits &= (1u << (nvis & 31)) - 1u;
        const int pc = __popc(bits);
        if (n < pc) {
            for (; n > 0; --n) bits &= bits - 1u;
            return wd * 32 + __ffs(bits) - 1;
        }
        n -= pc;
    }
    return -1;
}

template <typename T, int DL, int GM>  // DL = d / 32 dims per lane, GM >= g heads
__global__ void __launch_bounds__(32 * kRouteWarps) bwd_route_kernel(
    TView Q, const float *__restrict__ kbar, Geom G, float alpha, float gamma, float sigma,
    const float *__restrict__ tau, const uint32_t *__restrict__ mask, const float *__restrict__ logw,
    const float *__restrict__ Gd, const float *__restrict__ dQacc, TView dQ, float *__restrict__ dKbar) {
    constexpr int D = DL * 32;
    __shared__ __align__(16) float qs_all[kRouteWarps][GM][D];
    __shared__ float ds_all[kRouteWarps][32][GM];
    __shared__ int cs_all[kRouteWarps][32];
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int64_t w = (int64_t)blockIdx.x * kRouteWarps + warp;
    if (w >= G.b * G.nq * G.hkv) return;
    float(&qs)[GM][D] = qs_all[warp];
    float(&dsb)[32][GM] = ds_all[warp];
    int *csb = cs_all[warp];
    const int r = (int)(w % G.hkv);
    const int64_t i = (w / G.hkv) % G.nq, b = w / ((int64_t)G.hkv * G.nq);
    const int g = G.g;
    const int nvis = row_nvis(G, i);
    const float sc = gamma * rsqrtf((float)D);
    float dq[GM][DL];
#pragma unroll
    for (int h = 0; h < GM; ++h)
#pragma unroll
        for (int k = 0; k < DL; ++k) dq[h][k] = 0.f;
    auto store = [&]() {
#pragma unroll
        for (int h = 0; h < GM; ++h) {
            if (h >= g) break;
            const float *src = dQacc + (((size_t)b * G.nq + i) * G.hq + r * g + h) * D;
            T *dst = reinterpret_cast<T *>(const_cast<void *>(dQ.p)) + b * dQ.s0 + i * dQ.s1 +
                     (int64_t)(r * g + h) * dQ.s2;
#pragma unroll
            for (int k = 0; k < DL; ++k) dst[DL * lane + k] = from_f<T>(src[DL * lane + k] + sc * dq[h][k]);
        }
    };
    const uint32_t *mrow = mask + (((size_t)b * G.nq + i) * G.hkv + r) * G.words;
    const int wv = nvis > 0 ? (nvis + 31) / 32 : 0;
    // pass 1: |R_i| and mean G
    int nR = 0;
    for (int wd = 0; wd < wv; ++wd) {
        uint32_t bits = mrow[wd];
        if (wd == wv - 1 && (nvis & 31)) bits &= (1u << (nvis & 31)) - 1u;
        nR += __popc(bits);
    }
    if (nR == 0) {  // nothing routed: the Stage-2 part alone
        store();
        return;
    }
    float sG = 0.f;
    for (int n0 = 0; n0 < nR; n0 += 32) {
        const int c = n0 + lane < nR ? nth_routed(mrow, wv, nvis, n0 + lane) : -1;
        if (c >= 0) sG += Gd[logw_index(G, b, r, i, c)];
    }
    const float meanG = warp_sum(sG) / (float)nR;
    // the group's queries into shared memory
#pragma unroll
    for (int h = 0; h < GM; ++h) {
        if (h >= g) break;
        const T *qp = reinterpret_cast<const T *>(Q.p) + b * Q.s0 + i * Q.s1 + (int64_t)(r * g + h) * Q.s2;
#pragma unroll
        for (int k = 0; k < DL; ++k) qs[h][DL * lane + k] = to_f<T>(qp[DL * lane + k]);
    }
    __syncwarp();
    const float inv_sigma = 1.f / sigma;
    const float xs = (alpha - 1.f) * gamma * rsqrtf((float)D);
    const float kexp = 1.f / (alpha - 1.f), uexp = 2.f - alpha;
    float th[GM];
#pragma unroll
    for (int h = 0; h < GM; ++h) th[h] = h < g ? tau[((size_t)b * G.nq + i) * G.hq + r * g + h] : INFINITY;
    const float *kb_base = kbar + ((size_t)b * G.kbar_cap * G.hkv + r) * D;  // chunk c at + c * hkv * D
    // x of every head for the lane's chunk: GM dot products over D from shared q
    auto scores = [&](int c, float (&x)[GM]) {
        const float4 *kp = reinterpret_cast<const float4 *>(kb_base + (size_t)c * G.hkv * D);
#pragma unroll
        for (int h = 0; h < GM; ++h) x[h] = 0.f;
#pragma unroll 4
        for (int e4 = 0; e4 < D / 4; ++e4) {
            const float4 kv = kp[e4];
#pragma unroll
            for (int h = 0; h < GM; ++h) {
                if (h < g) {
                    const float4 qv = *reinterpret_cast<const float4 *>(&qs[h][4 * e4]);
                    x[h] = fmaf(qv.x, kv.x, fmaf(qv.y, kv.y, fmaf(qv.z, kv.z, fmaf(qv.w, kv.w, x[h]))));
                }
            }
        }
#pragma unroll
        for (int h = 0; h < GM; ++h) x[h] *= xs;
    };
    // pass 2: sum u and sum u dp per head
    float su[GM], sud[GM];
#pragma unroll
    for (int h = 0; h < GM; ++h) su[h] = sud[h] = 0.f;
    for (int n0 = 0; n0 < nR; n0 += 32) {
        const int c = n0 + lane < nR ? nth_routed(mrow, wv, nvis, n0 + lane) : -1;
        if (c < 0) continue;
        const size_t li = logw_index(G, b, r, i, c);
        const float dlw = (Gd[li] - meanG) * inv_sigma, lw = logw[li];
        float x[GM];
        scores(c, x);
#pragma unroll
        for (int h = 0; h < GM; ++h) {
            float u, ud;
            if (h < g && route_terms(x[h], th[h], kexp, uexp, lw, dlw, g, u, ud)) {
                su[h] += u;
                sud[h] += ud;
            }
        }
    }
    float rho[GM];
#pragma unroll
    for (int h = 0; h < GM; ++h) {
        const float a = warp_sum(su[h]), bb = warp_sum(sud[h]);
        rho[h] = a > 0.f ? bb / a : 0.f;
    }
    // pass 3: ds per (chunk, head) by the chunk's lane, then lanes over dimensions
    const float sck = gamma * rsqrtf((float)D);
    for (int n0 = 0; n0 < nR; n0 += 32) {
        const int c = n0 + lane < nR ? nth_routed(mrow, wv, nvis, n0 + lane) : -1;
        csb[lane] = c;
        if (c >= 0) {
            const size_t li = logw_index(G, b, r, i, c);
            const float dlw = (Gd[li] - meanG) * inv_sigma, lw = logw[li];
            float x[GM];
            scores(c, x);
#pragma unroll
            for (int h = 0; h < GM; ++h) {
                float u = 0.f, ud = 0.f;
                const bool in = h < g && route_terms(x[h], th[h], kexp, uexp, lw, dlw, g, u, ud);
                dsb[lane][h] = in ? ud - u * rho[h] : 0.f;
            }
        }
        __syncwarp();
        const int nb = min(32, nR - n0);
        // lanes over dimensions: lane l holds dimensions DL*l .. DL*l + DL - 1 (one vector
        // load of kbar_c and one vector atomic into its gradient per chunk)
        for (int j = 0; j < nb; ++j) {
            const int cj = csb[j];
            const float *kp = kb_base + (size_t)cj * G.hkv * D + DL * lane;
            float kv[DL], dkb[DL];
#pragma unroll
            for (int k = 0; k < DL; ++k) {
                kv[k] = kp[k];
                dkb[k] = 0.f;
            }
#pragma unroll
            for (int h = 0; h < GM; ++h) {
                if (h >= g) break;
                const float ds = dsb[j][h];
#pragma unroll
                for (int k = 0; k < DL; ++k) {
                    dq[h][k] = fmaf(ds, kv[k], dq[h][k]);
                    dkb[k] = fmaf(ds, qs[h][DL * lane + k], dkb[k]);
                }
            }
            float *dst = dKbar + (((size_t)b * G.n_chunks + cj) * G.hkv + r) * D + DL * lane;
            if (DL == 4)
                atomicAdd(reinterpret_cast<float4 *>(dst),
                          make_float4(sck * dkb[0], sck * dkb[DL > 1 ? 1 : 0], sck * dkb[DL > 2 ? 2 : 0],
                                      sck * dkb[DL > 3 ? 3 : 0]));
            else
                atomicAdd(reinterpret_cast<float2 *>(dst), make_float2(sck * dkb[0], sck * dkb[DL > 1 ? 1 : 0]));
        }
        __syncwarp();
    }
    store();
}

// Sum over the 32 lanes of each of the 32 values P[v], left in lane v (recursive halving:
// 5 exchange rounds, 31 shuffles).
__device__ __forceinline__ float reduce_scatter32(float (&P)[32], int lane) {
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) {
        const bool up = (lane & m) != 0;
#pragma unroll
        for (int k = 0; k < m; ++k) {
            const float keep = up ? P[k + m] : P[k], send = up ? P[k] : P[k + m];
            P[k] = keep + __shfl_xor_sync(0xffffffffu, send, m);
        }
    }
    return P[0];
}

constexpr int kRouteMaxChunks = 2048;  // routed-list capacity of the batched kernel (per warp)

// The routing chain as bwd_route_kernel computes it, for g <= 4, with the chunk summaries
// read once per batch of 8 routed chunks by the whole warp (lane l holds dimensions
// DL*l .. DL*l + DL - 1 of each: one coalesced row per chunk) instead of one lane per chunk
// streaming its own row.  The scores of the batch (8 chunks x 4 heads) are formed as
// per-lane partial dot products and summed by a reduce-scatter, which leaves the score of
// (chunk slot cs, head hs) in lane 4 cs + hs; the entmax terms are that lane's, and the
// summaries already in registers serve the updates of dQ and of the summaries' gradient.
template <typename T, int DL>
__global__ void __launch_bounds__(32 * kRouteWarps, 4) bwd_route8_kernel(
    TView Q, const float *__restrict__ kbar, Geom G, float alpha, float gamma, float sigma,
    const float *__restrict__ tau, const uint32_t *__restrict__ mask, const float *__restrict__ logw,
    const float *__restrict__ Gd, const float *__restrict__ dQacc, TView dQ, float *__restrict__ dKbar) {
    constexpr int D = DL * 32, GM = 4, NCB = 8;
    __shared__ int rl_all[kRouteWarps][kRouteMaxChunks];
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int64_t w = (int64_t)blockIdx.x * kRouteWarps + warp;
    if (w >= G.b * G.nq * G.hkv) return;
    int *rl = rl_all[warp];
    const int r = (int)(w % G.hkv);
    const int64_t i = (w / G.hkv) % G.nq, b = w / ((int64_t)G.hkv * G.nq);
    const int g = G.g;
    const int nvis = row_nvis(G, i);
    const float sc = gamma * rsqrtf((float)D);
    float dq[GM][DL];
#pragma unroll
    for (int h = 0; h < GM; ++h)
#pragma unroll
        for (int k = 0; k < DL; ++k) dq[h][k] = 0.f;
    auto store = [&]() {
#pragma unroll
        for (int h = 0; h < GM; ++h) {
            if (h >= g) break;
            const float *src = dQacc + (((size_t)b * G.nq + i) * G.hq + r * g + h) * D;
            T *dst = reinterpret_cast<T *>(const_cast<void *>(dQ.p)) + b * dQ.s0 + i * dQ.s1 +
                     (int64_t)(r * g + h) * dQ.s2;
#pragma unroll
            for (int k = 0; k < DL; ++k) dst[DL * lane + k] = from_f<T>(src[DL * lane + k] + sc * dq[h][k]);
        }
    };
    // pass 1: the routed chunks, ascending, into the warp's list (lanes over mask words)
    const uint32_t *mrow = mask + (((size_t)b * G.nq + i) * G.hkv + r) * G.words;
    const int wv = nvis > 0 ? (nvis + 31) / 32 : 0;
    int nR = 0;
    for (int w0 = 0; w0 < wv; w0 += 32) {
        const int wd = w0 + lane;
        uint32_t bits = wd < wv ? mrow[wd] : 0u;
        if (wd == wv - 1 && (nvis & 31)) bits &= (1u << (nvis & 31)) - 1u;
        const int pc = __popc(bits);
        int incl = pc;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        int pos = nR + incl - pc;
        while (bits) {
            rl[pos++] = wd * 32 + __ffs(bits) - 1;
            bits &= bits - 1u;
        }
        nR += __shfl_sync(0xffffffffu, incl, 31);
    }
    __syncwarp();
    if (nR == 0) {  // nothing routed: the Stage-2 part alone
        store();
        return;
    }
    float sG = 0.f;
    for (int n = lane; n < nR; n += 32) sG += Gd[logw_index(G, b, r, i, rl[n])];
    const float meanG = warp_sum(sG) / (float)nR;
    // this lane's dimensions of the group's queries
    float qv[GM][DL];
#pragma unroll
    for (int h = 0; h < GM; ++h) {
        const T *qp = reinterpret_cast<const T *>(Q.p) + b * Q.s0 + i * Q.s1 + (int64_t)(r * g + (h < g ? h : 0)) * Q.s2;
#pragma unroll
        for (int k = 0; k < DL; ++k) qv[h][k] = h < g ? to_f<T>(qp[DL * lane + k]) : 0.f;
    }
    const float inv_sigma = 1.f / sigma;
    const float xs = (alpha - 1.f) * gamma * rsqrtf((float)D);
    const float kexp = 1.f / (alpha - 1.f), uexp = 2.f - alpha;
    const int cs = lane / GM, hs = lane % GM;  // this lane's (chunk slot, head) of a batch
    const float th = hs < g ? tau[((size_t)b * G.nq + i) * G.hq + r * g + hs] : INFINITY;
    const float *kb_base = kbar + ((size_t)b * G.kbar_cap * G.hkv + r) * D + DL * lane;  // chunk c at + c * hkv * D
    // batch n0: chunk ids, their summaries (this lane's dimensions) and the lane's score
    auto batch = [&](int n0, int (&cid)[NCB], float (&kv)[NCB][DL]) -> float {
        float P[32];
#pragma unroll
        for (int k = 0; k < NCB; ++k) {
            cid[k] = n0 + k < nR ? rl[n0 + k] : -1;
            if (cid[k] >= 0) {
                const float *kp = kb_base + (size_t)cid[k] * G.hkv * D;
                if (DL == 4) {
                    const float4 t4 = *reinterpret_cast<const float4 *>(kp);
                    kv[k][0] = t4.x;
                    kv[k][DL > 1 ? 1 : 0] = t4.y;
                    kv[k][DL > 2 ? 2 : 0] = t4.z;
                    kv[k][DL > 3 ? 3 : 0] = t4.w;
                } else {
#pragma unroll
                    for (int j = 0; j < DL; ++j) kv[k][j] = kp[j];
                }
            } else {
#pragma unroll
                for (int j = 0; j < DL; ++j) kv[k][j] = 0.f;
            }
#pragma unroll
            for (int h = 0; h < GM; ++h) {
                float a = 0.f;
#pragma unroll
                for (int j = 0; j < DL; ++j) a = fmaf(qv[h][j], kv[k][j], a);
                P[k * GM + h] = a;
            }
        }
        return reduce_scatter32(P, lane) * xs;
    };
    // pass 2: sum u and sum u dp per head (lane (cs, hs) adds its own pair)
    float su = 0.f, sud = 0.f;
    for (int n0 = 0; n0 < nR; n0 += NCB) {
        int cid[NCB];
        float kv[NCB][DL];
        const float x = batch(n0, cid, kv);
        const int c = n0 + cs < nR ? rl[n0 + cs] : -1;  // this lane's chunk
        if (c >= 0 && hs < g) {
            const size_t li = logw_index(G, b, r, i, c);
            float u, ud;
            if (route_terms(x, th, kexp, uexp, logw[li], (Gd[li] - meanG) * inv_sigma, g, u, ud)) {
                su += u;
                sud += ud;
            }
        }
    }
#pragma unroll
    for (int o = GM; o < 32; o <<= 1) {  // over the chunk slots of the lane's head
        su += __shfl_xor_sync(0xffffffffu, su, o);
        sud += __shfl_xor_sync(0xffffffffu, sud, o);
    }
    const float rho = su > 0.f ? sud / su : 0.f;
    // pass 3: ds per (chunk, head) in its lane, then lanes over dimensions
    const float sck = gamma * rsqrtf((float)D);
    for (int n0 = 0; n0 < nR; n0 += NCB) {
        int cid[NCB];
        float kv[NCB][DL];
        const float x = batch(n0, cid, kv);
        const int c = n0 + cs < nR ? rl[n0 + cs] : -1;  // this lane's chunk
        float ds = 0.f;
        if (c >= 0 && hs < g) {
            const size_t li = logw_index(G, b, r, i, c);
            float u, ud;
            if (route_terms(x, th, kexp, uexp, logw[li], (Gd[li] - meanG) * inv_sigma, g, u, ud)) ds = ud - u * rho;
        }
#pragma unroll
        for (int k = 0; k < NCB; ++k) {
            float dkb[DL];
#pragma unroll
            for (int j = 0; j < DL; ++j) dkb[j] = 0.f;
#pragma unroll
            for (int h = 0; h < GM; ++h) {
                const float dsh = __shfl_sync(0xffffffffu, ds, k * GM + h);
#pragma unroll
                for (int j = 0; j < DL; ++j) {
                    dq[h][j] = fmaf(dsh, kv[k][j], dq[h][j]);
                    dkb[j] = fmaf(dsh, qv[h][j], dkb[j]);
                }
            }
            if (cid[k] >= 0) {
                float *dst = dKbar + (((size_t)b * G.n_chunks + cid[k]) * G.hkv + r) * D + DL * lane;
                if (DL == 4)
                    atomicAdd(reinterpret_cast<float4 *>(dst),
                              make_float4(sck * dkb[0], sck * dkb[DL > 1 ? 1 : 0], sck * dkb[DL > 2 ? 2 : 0],
                                          sck * dkb[DL > 3 ? 3 : 0]));
                else
                    atomicAdd(reinterpret_cast<float2 *>(dst), make_float2(sck * dkb[0], sck * dkb[DL > 1 ? 1 : 0]));
            }
        }
    }
    store();
}

template <typename T>
__global__ void bwd_dq_finish_kernel(const float *__restrict__ dQacc, TView dQ, Geom G) {
    const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t n = G.b * G.nq * G.hq * (int64_t)G.d;
    if (idx >= n) return;
    const int e = (int)(idx % G.d);
    const int64_t row = idx / G.d;
    const int h = (int)(row % G.hq);
    const int64_t i = (row / G.hq) % G.nq, b = row / ((int64_t)G.hq * G.nq);
    reinterpret_cast<T *>(const_cast<void *>(dQ.p))[b * dQ.s0 + i * dQ.s1 + (int64_t)h * dQ.s2 + e] =
        from_f<T>(dQacc[idx]);
}

template <typename T>
cudaError_t launch_bwd_t(const BwdArgs &a, cudaStream_t st) {
    const Geom &G = a.G;
    const ListsView &L = a.L;
    cudaError_t e;
    const int64_t rows = G.b * G.nq * G.hq;
    if (!a.use_tc) {  // the tensor-core path forms D in its tile preparation
        bwd_rowdot_kernel<T><<<(unsigned)((rows * 32 + 255) / 256), 256, 0, st>>>(a.dO, a.O, G, a.Drow);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    // Stage 2, query side: dQ and the prior's G
    if (a.use_tc) {
        if ((e = launch_attn_bwd_tc_dq(a, st)) != cudaSuccess) return e;
    } else {
        const int dp = G.d + 1;
        const size_t smem = (size_t)(3 * kRows + 2 * kSubB) * dp * sizeof(float) + kRows * sizeof(float);
        if ((e = cudaFuncSetAttribute(bwd_dq_simt_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)smem)) != cudaSuccess)
            return e;
        bwd_dq_simt_kernel<T><<<dim3((unsigned)L.n_tiles, (unsigned)G.hkv, (unsigned)G.b), kRows, smem, st>>>(
            a.Q, a.K, a.V, a.dO, G, L, a.lse, a.Drow, a.dQacc, a.Gd);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    // the routing chain (prior, group average, entmax, Stage-1 scores) into dQ and the summaries
    if (G.n_chunks > 0) {
        if ((e = cudaMemsetAsync(a.dKbar, 0, (size_t)G.b * G.n_chunks * G.hkv * G.d * sizeof(float), st)) !=
            cudaSuccess)
            return e;
        const int64_t warps = G.b * G.nq * G.hkv;
        const unsigned blocks = (unsigned)((warps + kRouteWarps - 1) / kRouteWarps);
#define DASH_ROUTE(DL, GM)                                                                                         \
    bwd_route_kernel<T, DL, GM><<<blocks, 32 * kRouteWarps, 0, st>>>(a.Q, a.kbar, G, a.alpha, a.gamma, a.sigma,  \
                                                                     a.tau, a.mask, a.logw, a.Gd, a.dQacc, a.dQ, \
                                                                     a.dKbar)
        if (G.g <= 4 && G.n_chunks <= kRouteMaxChunks) {
            if (G.d == 128)
                bwd_route8_kernel<T, 4><<<blocks, 32 * kRouteWarps, 0, st>>>(a.Q, a.kbar, G, a.alpha, a.gamma, a.sigma,
                                                                            a.tau, a.mask, a.logw, a.Gd, a.dQacc,
                                                                            a.dQ, a.dKbar);
            else
                bwd_route8_kernel<T, 2><<<blocks, 32 * kRouteWarps, 0, st>>>(a.Q, a.kbar, G, a.alpha, a.gamma, a.sigma,
                                                                            a.tau, a.mask, a.logw, a.Gd, a.dQacc,
                                                                            a.dQ, a.dKbar);
        } else if (G.d == 128 && G.g <= 4) DASH_ROUTE(4, 4);
        else if (G.d == 128) DASH_ROUTE(4, 16);
        else if (G.g <= 4) DASH_ROUTE(2, 4);
        else DASH_ROUTE(2, 16);
#undef DASH_ROUTE
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    // transposed lists
    const int tw = (int)((L.n_tiles + 31) / 32);
    if ((e = cudaMemsetAsync(a.bitmap, 0, (size_t)G.b * G.hkv * G.n_blk * tw * sizeof(uint32_t), st)) != cudaSuccess)
        return e;
    refs_mark_kernel<<<dim3((unsigned)L.n_tiles, (unsigned)G.hkv, (unsigned)G.b), 128, 0, st>>>(G, L, a.bitmap,
                                                                                                a.E, tw);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    refs_build_kernel<<<dim3((unsigned)G.hkv, (unsigned)G.b), 1024, 0, st>>>(G, L.n_tiles, a.bitmap, a.E, tw,
                                                                            a.ref_off, a.ref_cnt, a.refs);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    // Stage 2, key side: dK (with the pooling share), dV
    if (a.use_tc) {
        if ((e = launch_attn_bwd_tc_dkdv(a, st)) != cudaSuccess) return e;
    } else {
        const int KB = G.B < 64 ? G.B : 64;
        const int dp = G.d + 1;
        const size_t smem = (size_t)(4 * KB + 2 * kRowChunk) * dp * sizeof(float) + 3 * kRowChunk * sizeof(float) +
                            kRowChunk * sizeof(long long) + 16;
        if ((e = cudaFuncSetAttribute(bwd_dkdv_simt_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)smem)) != cudaSuccess)
            return e;
        const int nkb = (int)((G.nk + KB - 1) / KB);
        bwd_dkdv_simt_kernel<T><<<dim3((unsigned)nkb, (unsigned)G.hkv, (unsigned)G.b), 128, smem, st>>>(
            a.Q, a.K, a.V, a.dO, a.dK, a.dV, G, L, a.lse, a.Drow, a.ref_off, a.ref_cnt, a.refs, a.dKbar);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    if (G.n_chunks == 0) {  // no routing at all: dQ is the Stage-2 part
        const int64_t n = rows * G.d;
        bwd_dq_finish_kernel<T><<<(unsigned)((n + 255) / 256), 256, 0, st>>>(a.dQacc, a.dQ, G);
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_bwd(const BwdArgs &a, dash_dtype_t dt, cudaStream_t st) {
    if (a.G.nq == 0 || a.G.b == 0) return cudaSuccess;
    return dt == DASH_BF16 ? launch_bwd_t<__nv_bfloat16>(a, st) : launch_bwd_t<float>(a, st);
}

}  // namespace dash

// block_select.cu -- Stage 1: entmax chunk routing and Stage-2 work-list compaction.
//
// For query row i, head h of KV group r ("DashAttention" §3.2 Eq. 4; App. G Alg. 2):
//   zbar_c = <q_i^(h), k̄_c^(r)> / sqrt(d)              for the visible chunks c
//   x_c    = (alpha - 1) * gamma * zbar_c
//   tau    : sum_c [x_c - tau]_+^{1/(alpha-1)} = 1      (alpha-entmax threshold, §2 Eq. 2)
//   p_c    = [x_c - tau]_+^{1/(alpha-1)}
// Group prior (§3.2): w_c = (1/g) sum_{h in G_r} p_c^(h); the routed set R is the
// union of the heads' supports.  Bias (§3.4 Prop. 1): mu = mean_{c in R} log w_c,
// d_c = (log w_c - mu) / sigma.
//
// select_rows_kernel: one CTA per (batch, kv head, group of S query rows).
//   (1) logits of the S*g (row, head) pairs against the visible chunk summaries,
//       kept in shared memory (never written to HBM);
//   (2) tau per pair, one warp per pair: shared-memory histogram of x over the
//       bracket [max x - 1, max x) gives a starting point (AdaSplash-2's
//       histogram initialisation), then safeguarded Newton / bisection with
//       warp-shuffle reductions, then an exact closed-form polish on the final
//       support for alpha = 2 (linear) and alpha = 1.5 (quadratic);
//   (3) per row (one warp): membership by comparison x > tau, log w in the log
//       domain (1/(alpha-1) = 4 at alpha = 1.25 underflows fp32 otherwise), mu,
//       d, the bit-packed mask and optionally w.
// compact_kernel: one CTA per (batch, kv head, query tile): union of the tile's
//   routed chunks, its rows' local-window chunks first (the diagonal chunk, and the one
//   before it with the two-block window of App. B.1.1), and the per-row bias table
//   (bias 0 on every routed chunk when the mask is a caller's, without log w).
#include <math.h>

#include "dash_common.cuh"
#include "kernels.h"

namespace dash {

namespace {

constexpr int kSelThreads = 256;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kDirectMaxPairs = 16;  // logits computed straight from L2 when pairs <= this
constexpr int kTileChunks = 32;      // chunk tile of the shared-memory logits path

struct SelParams {
    float alpha, gamma, sigma;
    float kexp;   // 1/(alpha-1)
    int kint;     // 1/(alpha-1) when it is 1, 2 or 4; else 0
    int S;        // rows per CTA
    int ldx;      // row stride of the logits buffer
    int dpad;     // padded row length (floats) of q / k̄ tiles in shared memory
};

__device__ __forceinline__ float relu_pow(float t, const SelParams &P) {
    if (t <= 0.f) return 0.f;
    switch (P.kint) {
        case 1: return t;
        case 2: return t * t;
        case 4: { float u = t * t; return u * u; }
        default: return powf(t, P.kexp);
    }
}
// [t]^{k-1} for t > 0 (derivative helper)
__device__ __forceinline__ float relu_pow_m1(float t, const SelParams &P) {
    if (t <= 0.f) return 0.f;
    switch (P.kint) {
        case 1: return 1.f;
        case 2: return t;
        case 4: return t * t * t;
        default: return powf(t, P.kexp - 1.f);
    }
}

// Solve the entmax threshold of one (row, head) pair over x = (alpha-1) * X[0..n)
// in shared memory; the whole warp calls it.
//   bracket  f(mx - 1) >= 0 (the largest term alone is 1), f(mx - n^{1-alpha}) <= 0
//            (every term is at most 1/n);
//   start    a 32-bin histogram of x over [mx - 1, mx) estimates f at the bin edges
//            (mass at the bin centres): the highest edge still estimated >= 0;
//   iterate  alpha = 2 / 1.5: the exact closed form on the current support
//            {x > tau}, until the support no longer changes; other alpha: Newton.
//            Steps leaving the bracket fall back to bisection.
__device__ float solve_tau(const float *X, int n, const SelParams &P, int *hist) {
    const int lane = threadIdx.x % 32;
    const float am1 = P.alpha - 1.f;
    float mx = -INFINITY;
    for (int c = lane; c < n; c += 32) mx = fmaxf(mx, am1 * X[c]);
    mx = warp_max(mx);
    float lo = mx - 1.f;
    float hi = mx - powf((float)n, 1.f - P.alpha);
    if (n == 1) return lo;

    hist[lane] = 0;
    __syncwarp();
    for (int c = lane; c < n; c += 32) {
        const float y = am1 * X[c] - lo;
        if (y >= 0.f) atomicAdd(&hist[min(31, (int)(y * 32.f))], 1);
    }
    __syncwarp();
    float tau = lo;
    {
        const float edge = (float)lane * (1.f / 32.f);
        float fe = -1.f;
        for (int j = lane; j < 32; ++j) fe += (float)hist[j] * relu_pow(((float)j + 0.5f) * (1.f / 32.f) - edge, P);
        const unsigned okb = __ballot_sync(0xffffffffu, fe >= 0.f);
        const float t0 = lo + (float)(31 - __clz(okb | 1u)) * (1.f / 32.f);
        if (t0 > lo && t0 < hi) tau = t0;
    }
    __syncwarp();

    int prev_cnt = -1;
    for (int it = 0; it < 40; ++it) {
        float f = 0.f, df = 0.f, s1 = 0.f, s2 = 0.f;
        int cnt = 0;
        for (int c = lane; c < n; c += 32) {
            const float xv = am1 * X[c];
            const float t = xv - tau;
            if (t > 0.f) {
                f += relu_pow(t, P);
                df += relu_pow_m1(t, P);
                const float y = xv - mx;
                s1 += y;
                s2 += y * y;
                ++cnt;
            }
        }
        f = warp_sum(f) - 1.f;
        df = -P.kexp * warp_sum(df);
        s1 = warp_sum(s1);
        s2 = warp_sum(s2);
        cnt = warp_sum_i(cnt);
        if (f >= 0.f) lo = tau;
        else hi = tau;
        float nt;
        if ((P.kint == 1 || P.kint == 2) && cnt > 0) {
            // the previous step was the exact closed form on this same support
            // (supports {x > tau} are nested, so equal counts mean equal sets): done
            if (cnt == prev_cnt) break;
            prev_cnt = cnt;
            const float m1 = s1 / (float)cnt;
            if (P.kint == 1) {
                nt = mx + (s1 - 1.f) / (float)cnt;
            } else {
                const float var = fmaxf(s2 / (float)cnt - m1 * m1, 0.f);
                nt = mx + m1 - sqrtf(fmaxf(1.f / (float)cnt - var, 0.f));
            }
            // at the root the closed form can land a rounding error outside the bracket:
            // a step that close is clamped into it, a farther one is replaced by bisection
            const float slack = 4e-7f * fmaxf(1.f, fabsf(tau));
            if (nt >= lo - slack && nt <= hi + slack) {
                nt = fminf(fmaxf(nt, lo), hi);
            } else {
                nt = 0.5f * (lo + hi);  // a bisection step: the next count proves nothing
                prev_cnt = -1;
            }
            if (hi - lo <= slack) {
                tau = nt;
                break;
            }
        } else {
            nt = df < 0.f ? tau - f / df : 0.5f * (lo + hi);
            if (!(nt > lo && nt < hi)) nt = 0.5f * (lo + hi);
            if (fabsf(nt - tau) <= 1e-7f * fmaxf(1.f, fabsf(tau)) || hi - lo <= 1e-7f * fmaxf(1.f, fabsf(tau))) {
                tau = nt;
                break;
            }
        }
        tau = nt;
    }
    return tau;
}

// log w_c of one row and chunk: w_c = (1/g) sum_h [x_c^(h) - tau_h]_+^{1/(alpha-1)}.
// Returns -inf when no head routes the chunk.  The direct power sum is used
// unless it underflows, then the log-sum-exp form of the same sum.
__device__ __forceinline__ float group_logw(const float *X, int ldx, const float *taus, int g, int c,
                                            const SelParams &P, float log_g) {
    const float am1 = P.alpha - 1.f;
    float v = 0.f;
    bool sel = false;
    for (int hh = 0; hh < g; ++hh) {
        const float t = am1 * X[(size_t)hh * ldx + c] - taus[hh];
        if (t > 0.f) {
            sel = true;
            v += relu_pow(t, P);
        }
    }
    if (!sel) return -INFINITY;
    if (v > 0.f) return logf(v) - log_g;
    float mlog = -INFINITY;
    for (int hh = 0; hh < g; ++hh) {
        const float t = am1 * X[(size_t)hh * ldx + c] - taus[hh];
        if (t > 0.f) mlog = fmaxf(mlog, P.kexp * logf(t));
    }
    float acc = 0.f;
    for (int hh = 0; hh < g; ++hh) {
        const float t = am1 * X[(size_t)hh * ldx + c] - taus[hh];
        if (t > 0.f) acc += expf(P.kexp * logf(t) - mlog);
    }
    return mlog + logf(acc) - log_g;
}

// Logits of P pairs against chunks [0, nvis) -> X[p][c] (scaled by gamma/sqrt(d)).
template <typename T>
__device__ void compute_logits(const float *Qs, int npairs, const float *__restrict__ kb, int64_t kb_row_stride,
                               int nvis, int d, const SelParams &P, float scale, float *X, float *Ks) {
    if (npairs <= kDirectMaxPairs) {
        // Direct path: thread per chunk, k̄ rows straight from L2, q broadcast from smem.
        for (int c = threadIdx.x; c < nvis; c += kSelThreads) {
            float acc[kDirectMaxPairs];
#pragma unroll
            for (int p = 0; p < kDirectMaxPairs; ++p) acc[p] = 0.f;
            const float *kr = kb + (int64_t)c * kb_row_stride;
            for (int e = 0; e < d; e += 4) {
                float4 kv = *reinterpret_cast<const float4 *>(kr + e);
#pragma unroll
                for (int p = 0; p < kDirectMaxPairs; ++p) {
                    if (p < npairs) {
                        float4 qv = *reinterpret_cast<const float4 *>(Qs + p * P.dpad + e);
                        acc[p] = fmaf(qv.x, kv.x, fmaf(qv.y, kv.y, fmaf(qv.z, kv.z, fmaf(qv.w, kv.w, acc[p]))));
                    }
                }
            }
#pragma unroll
            for (int p = 0; p < kDirectMaxPairs; ++p)
                if (p < npairs) X[p * P.ldx + c] = acc[p] * scale;
        }
        __syncthreads();
        return;
    }
    // Tiled path: 32 chunk summaries at a time staged in shared memory.
    for (int c0 = 0; c0 < nvis; c0 += kTileChunks) {
        const int nc = min(kTileChunks, nvis - c0);
        for (int idx = threadIdx.x; idx < kTileChunks * (d / 4); idx += kSelThreads) {
            const int cc = idx / (d / 4), e = (idx % (d / 4)) * 4;
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            if (cc < nc) v = *reinterpret_cast<const float4 *>(kb + (int64_t)(c0 + cc) * kb_row_stride + e);
            *reinterpret_cast<float4 *>(Ks + cc * P.dpad + e) = v;
        }
        __syncthreads();
        for (int o = threadIdx.x; o < npairs * kTileChunks; o += kSelThreads) {
            const int p = o / kTileChunks, cc = o % kTileChunks;
            if (cc < nc) {
                const float *qr = Qs + p * P.dpad;
                const float *kr = Ks + cc * P.dpad;
                float acc = 0.f;
                for (int e = 0; e < d; e += 4) {
                    float4 qv = *reinterpret_cast<const float4 *>(qr + e);
                    float4 kv = *reinterpret_cast<const float4 *>(kr + e);
                    acc = fmaf(qv.x, kv.x, fmaf(qv.y, kv.y, fmaf(qv.z, kv.z, fmaf(qv.w, kv.w, acc))));
                }
                X[p * P.ldx + c0 + cc] = acc * scale;
            }
        }
        __syncthreads();
    }
}

template <typename T>
__global__ void __launch_bounds__(kSelThreads) select_rows_kernel(TView Q, const float *__restrict__ kbar, Geom G,
                                                                  SelParams P, SelectOut out) {
    extern __shared__ __align__(16) float smem[];
    const int g = G.g, d = G.d;
    const int r = blockIdx.y;
    const int64_t b = blockIdx.z;
    const int64_t i0 = (int64_t)blockIdx.x * P.S;
    const int nrows = (int)min((int64_t)P.S, G.nq - i0);
    const int npairs = nrows * g;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

    float *Qs = smem;                                   // [S*g][dpad]
    float *Ks = Qs + (size_t)P.S * g * P.dpad;          // [kTileChunks][dpad]
    float *X = Ks + (size_t)kTileChunks * P.dpad;       // [S*g][ldx]
    float *taus = X + (size_t)P.S * g * P.ldx;          // [S*g]
    int *hist = reinterpret_cast<int *>(taus + P.S * g);  // [warps][32]

    // (0) query rows of this group -> fp32 shared memory
    const T *qbase = reinterpret_cast<const T *>(Q.p) + b * Q.s0;
    for (int idx = threadIdx.x; idx < npairs * d; idx += kSelThreads) {
        const int p = idx / d, e = idx % d;
        const int s = p / g, hh = p % g;
        Qs[p * P.dpad + e] = to_f<T>(qbase[(i0 + s) * Q.s1 + (int64_t)(r * g + hh) * Q.s2 + e]);
    }
    __syncthreads();

    // (1) logits against the chunks visible to the last row of the group
    const int nvis_max = row_nvis(G, i0 + nrows - 1);
    const float *kb = kbar + ((size_t)b * G.kbar_cap * G.hkv + r) * d;
    compute_logits<T>(Qs, npairs, kb, (int64_t)G.hkv * d, nvis_max, d, P, P.gamma * rsqrtf((float)d), X, Ks);

    // (2) threshold per (row, head) pair
    for (int p = warp; p < npairs; p += kSelWarps) {
        const int s = p / g, hh = p % g;
        const int n = row_nvis(G, i0 + s);
        float tau = NAN;
        if (n > 0) tau = solve_tau(X + (size_t)p * P.ldx, n, P, hist + warp * 32);
        if (lane == 0) {
            taus[p] = tau;
            if (out.tau) out.tau[((b * G.nq) + i0 + s) * G.hq + r * g + hh] = tau;
        }
    }
    __syncthreads();

    // (3) group prior, routed set, bias and mask; every warp works on each row
    const float log_g = logf((float)g);
    float *red = taus + P.S * g;   // [2 * warps] block reduction scratch (after the histogram)
    red += kSelWarps * 32;
    for (int s = 0; s < nrows; ++s) {
        const int64_t i = i0 + s;
        const int n = row_nvis(G, i);
        const size_t rowoff = ((size_t)(b * G.nq + i) * G.hkv + r);
        const float *Xs = X + (size_t)(s * g) * P.ldx;
        const float *ts = taus + s * g;
        // sweep 1: log w per chunk into the first head's logits row (no longer needed), mu
        float *lw = X + (size_t)(s * g) * P.ldx;
        float lsum = 0.f;
        int cnt = 0;
        // each column is read and then overwritten by the one thread that owns it
        for (int c = threadIdx.x; c < n; c += kSelThreads) {
            const float v = group_logw(Xs, P.ldx, ts, g, c, P, log_g);
            if (v > -INFINITY) {
                lsum += v;
                ++cnt;
            }
            lw[c] = v;
        }
        __syncthreads();
        lsum = warp_sum(lsum);
        cnt = warp_sum_i(cnt);
        if (lane == 0) {
            red[warp] = lsum;
            reinterpret_cast<int *>(red)[kSelWarps + warp] = cnt;
        }
        __syncthreads();
        float tl = 0.f;
        int tc = 0;
        for (int w = 0; w < kSelWarps; ++w) {
            tl += red[w];
            tc += reinterpret_cast<int *>(red)[kSelWarps + w];
        }
        const float mu = tc ? tl / (float)tc : 0.f;
        if (out.mu && threadIdx.x == 0) out.mu[rowoff] = mu;
        // sweep 2: bias, mask bits, optional w (a warp per 32-chunk word)
        for (int wd = warp; wd < G.words; wd += kSelWarps) {
            const int c = wd * 32 + lane;
            const float v = c < n ? lw[c] : -INFINITY;
            const bool sel = v > -INFINITY;
            const unsigned bits = __ballot_sync(0xffffffffu, sel);
            if (lane == 0) out.mask[rowoff * G.words + wd] = bits;
            if (sel && out.logw) out.logw[logw_index(G, b, r, i, c)] = v;
            if (out.w && c < G.n_chunks) out.w[rowoff * G.n_chunks + c] = sel ? expf(v) : 0.f;
        }
        __syncthreads();
    }
}

// One CTA per (batch, kv head, query tile).
__global__ void __launch_bounds__(128) compact_kernel(Geom G0, const uint32_t *__restrict__ mask,
                                                      const float *__restrict__ logw, const float *__restrict__ mu,
                                                      float inv_sigma, ListsView L) {
    extern __shared__ __align__(16) uint32_t csm[];
    Geom G = G0;
    geom_live(G);
    uint32_t *uw = csm;                 // [words] union bits (diagonal range removed)
    int *wofs = reinterpret_cast<int *>(uw + G.words);  // [words + 1] exclusive prefix of popcounts
    const int64_t t = blockIdx.x;
    const int r = blockIdx.y;
    const int64_t b = blockIdx.z;
    const int T = L.tile_rows;
    const int64_t i0 = t * T;
    const int nrows = (int)min((int64_t)T, G.nq - i0);
    const size_t tile_idx = ((size_t)b * G.hkv + r) * L.n_tiles + t;
    if (L.rows)
        for (int s = threadIdx.x; s < T; s += blockDim.x) L.rows[tile_idx * T + s] = s < nrows ? (int)(i0 + s) : -1;

    // diagonal chunk range of the tile's rows (causal)
    int dlo = 0, dhi = -1;
    if (G.causal) {
        dlo = first_local(G, i0);
        dhi = (int)(row_pos(G, i0 + nrows - 1) / G.B);
        if (dhi > G.n_blk - 1) dhi = G.n_blk - 1;
    }
    const int nd = dhi - dlo + 1;

    for (int w = threadIdx.x; w < G.words; w += blockDim.x) {
        uint32_t u = 0;
        for (int s = 0; s < nrows; ++s) u |= mask[((size_t)(b * G.nq + i0 + s) * G.hkv + r) * G.words + w];
        // drop the diagonal range: those chunks are listed first
        for (int c = max(dlo, w * 32); c <= min(dhi, w * 32 + 31); ++c) u &= ~(1u << (c - w * 32));
        uw[w] = u;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int acc = nd > 0 ? nd : 0;
        for (int w = 0; w < G.words; ++w) {
            wofs[w] = acc;
            acc += __popc(uw[w]);
        }
        wofs[G.words] = acc;
        L.count[tile_idx] = acc;
    }
    __syncthreads();
    int32_t *ids = L.ids + tile_idx * L.cap;
    for (int e = threadIdx.x; e < nd; e += blockDim.x) ids[e] = dlo + e;
    for (int w = threadIdx.x; w < G.words; w += blockDim.x) {
        uint32_t u = uw[w];
        int pos = wofs[w];
        while (u) {
            int bit = __ffs(u) - 1;
            u &= u - 1;
            ids[pos++] = w * 32 + bit;
        }
    }
    __syncthreads();
    const int count = wofs[G.words];
    float *bias = L.bias + tile_idx * (size_t)L.cap * T;
    // rows past the query length have no bias entries: Stage 2 never reads them (their
    // scores are masked before the bias is used), so only the tile's nrows rows are filled
    for (int idx = threadIdx.x; idx < count * nrows; idx += blockDim.x) {
        const int e = idx / nrows, s = idx % nrows;
        const int c = ids[e];
        float v = -INFINITY;
        {
            const int64_t i = i0 + s;
            const size_t rowoff = ((size_t)(b * G.nq + i) * G.hkv + r);
            if (G.causal && c >= first_local(G, i) && c <= (int)(row_pos(G, i) / G.B)) {
                v = 0.f;  // local window (diagonal chunk): bias 0, causal mask in Stage 2
            } else if (c < row_nvis(G, i) && ((mask[rowoff * G.words + c / 32] >> (c % 32)) & 1u)) {
                // d_c = (log w_c - mu) / sigma; 0 for a caller's mask (uniform prior over R)
                v = logw ? (logw[logw_index(G, b, r, i, c)] - mu[rowoff]) * inv_sigma : 0.f;
            }
        }
        bias[(size_t)e * T + s] = v;
    }
}

// Regroup + compact: one CTA per (window of kTilesPerWindow tiles, kv head, batch),
// kWarpsPerTile warps per output tile.  The window's query rows are sorted by the size
// of their routed set (stable), consecutive runs of tile_rows rows form the tiles, and
// each tile's list is built as in compact_kernel: the rows' diagonal chunks first
// (ascending), then the union of their routed chunks (ascending), and the per-row bias
// table.  Rows with similar routed sets share a tile, so the union a tile streams
// through Stage 2 is smaller than for consecutive rows.  The window's mask words are
// cached in shared memory with an odd row stride (column reads are bank-conflict free)
// and each tile's list is kept there for the bias fill.
constexpr int kTilesPerWindow = 8;
constexpr int kWarpsPerTile = 4;
constexpr int kRegroupThreads = 32 * kTilesPerWindow * kWarpsPerTile;

struct RegroupSmem {
    int wpow2, W, ws, words, cap;
    size_t key, rowi, mrow, murow, uw, wofs, ids, total;
    __host__ __device__ RegroupSmem(const Geom &G, int tile_rows, int cap_) {
        W = tile_rows * kTilesPerWindow;
        wpow2 = 1;
        while (wpow2 < W) wpow2 *= 2;
        words = G.words;
        ws = G.words | 1;
        cap = cap_;
        key = 0;
        rowi = key + (size_t)wpow2 * 4;
        mrow = rowi + (size_t)W * 4;
        murow = mrow + (size_t)W * ws * 4;
        uw = murow + (size_t)W * 4;
        wofs = uw + (size_t)kTilesPerWindow * words * 4;
        ids = wofs + (size_t)kTilesPerWindow * (words + 1) * 4;
        total = ids + (size_t)kTilesPerWindow * cap * 4;
    }
};

// named barrier over the kWarpsPerTile warps of output tile tt (ids 1..kTilesPerWindow)
__device__ __forceinline__ void tile_sync(int tt) {
    asm volatile("bar.sync %0, %1;" ::"r"(tt + 1), "r"(32 * kWarpsPerTile) : "memory");
}

__global__ void __launch_bounds__(kRegroupThreads) regroup_compact_kernel(Geom G, const uint32_t *__restrict__ mask,
                                                                         const float *__restrict__ logw,
                                                                         const float *__restrict__ mu,
                                                                         float inv_sigma, ListsView L) {
    extern __shared__ __align__(16) uint8_t rsm_raw[];
    const int T = L.tile_rows;
    const RegroupSmem R(G, T, L.cap);
    uint32_t *key = reinterpret_cast<uint32_t *>(rsm_raw + R.key);   // [wpow2] sort keys
    int *rowi = reinterpret_cast<int *>(rsm_raw + R.rowi);           // [W] window slot per sorted position
    uint32_t *mrow = reinterpret_cast<uint32_t *>(rsm_raw + R.mrow);  // [W][ws] mask words per window slot
    float *murow = reinterpret_cast<float *>(rsm_raw + R.murow);     // [W] mu per window slot
    const int64_t win = blockIdx.x;
    const int r = blockIdx.y;
    const int64_t b = blockIdx.z;
    const int64_t i0 = win * R.W;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

    // the window's rows: mask words (cached), mu, and sort keys (popcount, slot)
    for (int j = threadIdx.x; j < R.wpow2; j += kRegroupThreads) {
        const int64_t i = i0 + j;
        uint32_t k = 0xffffffffu;
        if (j < R.W && i < G.nq) {
            const uint32_t *mw = mask + ((size_t)(b * G.nq + i) * G.hkv + r) * G.words;
            int cnt = 0;
            for (int w = 0; w < G.words; ++w) {
                const uint32_t m = mw[w];
                mrow[j * R.ws + w] = m;
                cnt += __popc(m);
            }
            murow[j] = mu ? mu[(size_t)(b * G.nq + i) * G.hkv + r] : 0.f;
            k = ((uint32_t)cnt << 16) | (uint32_t)j;
        } else if (j < R.W) {
            for (int w = 0; w < G.words; ++w) mrow[j * R.ws + w] = 0u;
            murow[j] = 0.f;
        }
        key[j] = k;
    }
    __syncthreads();
    // bitonic sort, ascending
    for (int k2 = 2; k2 <= R.wpow2; k2 <<= 1) {
        for (int jj = k2 >> 1; jj > 0; jj >>= 1) {
            for (int idx = threadIdx.x; idx < R.wpow2; idx += kRegroupThreads) {
                const int ixj = idx ^ jj;
                if (ixj > idx) {
                    const bool asc = (idx & k2) == 0;
                    const uint32_t a = key[idx], c = key[ixj];
                    if ((a > c) == asc) {
                        key[idx] = c;
                        key[ixj] = a;
                    }
                }
            }
            __syncthreads();
        }
    }
    for (int j = threadIdx.x; j < R.W; j += kRegroupThreads) {
        const uint32_t k = key[j];
        rowi[j] = k == 0xffffffffu ? -1 : (int)(k & 0xffffu);
    }
    __syncthreads();

    const int tt = warp / kWarpsPerTile;           // output tile of this warp
    const int tq = threadIdx.x % (32 * kWarpsPerTile);  // thread within the tile's group
    const int64_t tile = win * kTilesPerWindow + tt;
    if (tile >= L.n_tiles) return;  // whole tile groups leave together
    const size_t tile_idx = ((size_t)b * G.hkv + r) * L.n_tiles + tile;
    const int *slot = rowi + tt * T;                // window slot of each tile row (-1 unused)
    for (int j = tq; j < T; j += 32 * kWarpsPerTile)
        L.rows[tile_idx * T + j] = slot[j] >= 0 ? (int)(i0 + slot[j]) : -1;

    // diagonal chunks of the tile's rows, relative to the window's first chunk
    // (local windows: the diagonal chunk and, with local = 2, the one before it)
    const int dbase = G.causal ? first_local(G, i0) : 0;
    uint64_t dmask = 0;
    if (G.causal)
        for (int j = lane; j < T; j += 32)
            if (slot[j] >= 0)
                for (int c = first_local(G, i0 + slot[j]); c <= (int)(row_pos(G, i0 + slot[j]) / G.B); ++c)
                    dmask |= 1ull << (c - dbase);
    dmask = ((uint64_t)__reduce_or_sync(0xffffffffu, (uint32_t)(dmask >> 32)) << 32) |
            __reduce_or_sync(0xffffffffu, (uint32_t)dmask);
    const int nd = __popcll(dmask);

    // union of routed chunks, diagonal ones removed
    uint32_t *uw = reinterpret_cast<uint32_t *>(rsm_raw + R.uw) + tt * R.words;
    int *wofs = reinterpret_cast<int *>(rsm_raw + R.wofs) + tt * (R.words + 1);
    int *ids_s = reinterpret_cast<int *>(rsm_raw + R.ids) + (size_t)tt * R.cap;
    for (int wd = tq; wd < G.words; wd += 32 * kWarpsPerTile) {
        uint32_t acc = 0;
        for (int j = 0; j < T; ++j)
            if (slot[j] >= 0) acc |= mrow[slot[j] * R.ws + wd];
        for (int c = wd * 32; c < wd * 32 + 32; ++c) {
            const int rel = c - dbase;
            if (rel >= 0 && rel < 64 && ((dmask >> rel) & 1ull)) acc &= ~(1u << (c - wd * 32));
        }
        uw[wd] = acc;
    }
    tile_sync(tt);
    if (tq < 32) {
        // exclusive prefix of the words' popcounts (lane l owns words [l*wpl, (l+1)*wpl))
        const int wpl = (G.words + 31) / 32;
        int cnt = 0;
        for (int wd = lane * wpl; wd < min(G.words, (lane + 1) * wpl); ++wd) cnt += __popc(uw[wd]);
        int incl = cnt;
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        int run = nd + incl - cnt;
        for (int wd = lane * wpl; wd < min(G.words, (lane + 1) * wpl); ++wd) {
            wofs[wd] = run;
            run += __popc(uw[wd]);
        }
        if (lane == 31) {
            wofs[G.words] = run;
            L.count[tile_idx] = run;
        }
        if (lane == 0) {
            int e = 0;
            uint64_t dm = dmask;
            while (dm) {
                const int bit = __ffsll((long long)dm) - 1;
                dm &= dm - 1;
                ids_s[e++] = dbase + bit;
            }
        }
    }
    tile_sync(tt);
    for (int wd = tq; wd < G.words; wd += 32 * kWarpsPerTile) {
        uint32_t acc = uw[wd];
        int pos = wofs[wd];
        while (acc) {
            const int bit = __ffs(acc) - 1;
            acc &= acc - 1;
            ids_s[pos++] = wd * 32 + bit;
        }
    }
    tile_sync(tt);
    const int count = wofs[G.words];
    int32_t *ids = L.ids + tile_idx * L.cap;
    for (int e = tq; e < count; e += 32 * kWarpsPerTile) ids[e] = ids_s[e];
    float *bias = L.bias + tile_idx * (size_t)L.cap * T;
#pragma unroll 4
    for (int idx = tq; idx < count * T; idx += 32 * kWarpsPerTile) {
        const int e = idx / T, j = idx % T;
        const int c = ids_s[e];
        const int sl = slot[j];
        float v = -INFINITY;
        if (sl < 0) {
            v = 0.f;  // unused row: never stored
        } else {
            const int64_t i = i0 + sl;
            if (G.causal && c >= first_local(G, i) && c <= (int)(row_pos(G, i) / G.B)) {
                v = 0.f;
            } else if (c < row_nvis(G, i) && ((mrow[sl * R.ws + c / 32] >> (c % 32)) & 1u)) {
                // d_c = (log w_c - mu) / sigma; 0 for a caller's mask (uniform prior over R)
                v = logw ? (logw[logw_index(G, b, r, i, c)] - murow[sl]) * inv_sigma : 0.f;
            }
        }
        bias[(size_t)e * T + j] = v;
    }
}

}  // namespace

static int pick_rows_per_cta(const Geom &G, int dpad, int ldx, size_t *smem_out) {
    int best = 1;
    size_t best_smem = 0;
    for (int S = 1; S <= 32; S *= 2) {
        if (S * G.g > 128 && S > 1) break;
        size_t sm = ((size_t)S * G.g * dpad + (size_t)kTileChunks * dpad + (size_t)S * G.g * ldx + S * G.g) * 4 +
                    kSelWarps * 32 * 4 + 2 * kSelWarps * 4;
        if (sm > 200 * 1024 && S > 1) break;
        best = S;
        best_smem = sm;
        if (S >= G.nq) break;
    }
    *smem_out = best_smem;
    return best;
}

cudaError_t launch_select_rows(const TView &Q, dash_dtype_t dt, const float *kbar, const Geom &G, float alpha,
                               float gamma, float sigma, const SelectOut &o, cudaStream_t st) {
    if (G.nq == 0 || G.b == 0) return cudaSuccess;
    SelParams P;
    P.alpha = alpha;
    P.gamma = gamma;
    P.sigma = sigma;
    P.kexp = 1.f / (alpha - 1.f);
    P.kint = (alpha == 2.f) ? 1 : (alpha == 1.5f) ? 2 : (alpha == 1.25f) ? 4 : 0;
    P.dpad = G.d + 4;
    P.ldx = G.n_chunks > 0 ? G.n_chunks : 1;
    size_t smem = 0;
    P.S = pick_rows_per_cta(G, P.dpad, P.ldx, &smem);
    if (smem > 227 * 1024) return cudaErrorInvalidConfiguration;
    dim3 grid((unsigned)((G.nq + P.S - 1) / P.S), (unsigned)G.hkv, (unsigned)G.b);
    cudaError_t e;
    if (dt == DASH_BF16) {
        e = cudaFuncSetAttribute(select_rows_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem);
        if (e != cudaSuccess) return e;
        select_rows_kernel<__nv_bfloat16><<<grid, kSelThreads, smem, st>>>(Q, kbar, G, P, o);
    } else {
        e = cudaFuncSetAttribute(select_rows_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        select_rows_kernel<float><<<grid, kSelThreads, smem, st>>>(Q, kbar, G, P, o);
    }
    return cudaGetLastError();
}

static size_t regroup_smem(const Geom &G) { return RegroupSmem(G, G.tile_rows, G.n_blk).total; }

bool regroup_supported(const Geom &G) {
    // the tile_rows of a window must fit the sort key's slot field; the local-window chunks
    // a window's rows touch must fit the 64-bit mask; shared memory is bounded
    const int64_t span = ((int64_t)G.tile_rows * kTilesPerWindow + G.B - 1) / G.B + 1 + (G.local - 1);
    return G.tile_rows * kTilesPerWindow <= 65536 && span <= 64 && regroup_smem(G) <= 200 * 1024;
}

cudaError_t launch_regroup_compact(const Geom &G, const uint32_t *mask, const float *logw, const float *mu,
                                   float sigma, const ListsView &L, cudaStream_t st) {
    if (G.nq == 0 || G.b == 0) return cudaSuccess;
    const RegroupSmem R(G, L.tile_rows, L.cap);
    const int64_t nwin = (L.n_tiles + kTilesPerWindow - 1) / kTilesPerWindow;
    const size_t smem = R.total;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(regroup_compact_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess) return e;
    }
    regroup_compact_kernel<<<dim3((unsigned)nwin, (unsigned)G.hkv, (unsigned)G.b), kRegroupThreads, smem, st>>>(
        G, mask, logw, mu, 1.f / sigma, L);
    return cudaGetLastError();
}

cudaError_t launch_compact(const Geom &G, const uint32_t *mask, const float *logw, const float *mu, float sigma,
                           const ListsView &L, cudaStream_t st) {
    if (G.nq == 0 || G.b == 0) return cudaSuccess;
    dim3 grid((unsigned)L.n_tiles, (unsigned)G.hkv, (unsigned)G.b);
    const size_t smem = (size_t)G.words * 4 + (size_t)(G.words + 1) * 4 + 16;
    compact_kernel<<<grid, 128, smem, st>>>(G, mask, logw, mu, 1.f / sigma, L);
    return cudaGetLastError();
}

}  // namespace dash

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
//   routed chunks, its diagonal chunks first, and the per-row bias table.
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

// f(tau) and f'(tau) over x = (alpha-1) * X[0..n) read from shared memory.
__device__ __forceinline__ void residual(const float *X, int n, float am1, float tau, const SelParams &P,
                                         float &f, float &df) {
    float a = 0.f, b = 0.f;
    for (int c = threadIdx.x % 32; c < n; c += 32) {
        float t = am1 * X[c] - tau;
        a += relu_pow(t, P);
        b += relu_pow_m1(t, P);
    }
    f = warp_sum(a) - 1.f;
    df = -P.kexp * warp_sum(b);
}

// Solve the entmax threshold of one (row, head) pair; the whole warp calls it.
__device__ float solve_tau(const float *X, int n, const SelParams &P, int *hist) {
    const int lane = threadIdx.x % 32;
    const float am1 = P.alpha - 1.f;
    float mx = -INFINITY;
    for (int c = lane; c < n; c += 32) mx = fmaxf(mx, am1 * X[c]);
    mx = warp_max(mx);
    // Bracket: f(mx - 1) >= 0 (the largest term alone is 1) and
    //          f(mx - n^{1-alpha}) <= 0 (every term is at most 1/n).
    float lo = mx - 1.f;
    float hi = mx - powf((float)n, 1.f - P.alpha);
    if (n == 1) return lo;

    // Histogram initialisation: 32 bins over [mx - 1, mx); estimate f at each
    // bin's lower edge from the bin counts (mass at bin centres), start from
    // the highest edge whose estimate is still >= 0.
    hist[lane] = 0;
    __syncwarp();
    for (int c = lane; c < n; c += 32) {
        float y = am1 * X[c] - lo;  // in [.., 1]
        if (y >= 0.f) {
            int bin = min(31, (int)(y * 32.f));
            atomicAdd(&hist[bin], 1);
        }
    }
    __syncwarp();
    {
        const float edge = (float)lane * (1.f / 32.f);
        float fe = 0.f;
        for (int j = lane; j < 32; ++j) fe += (float)hist[j] * relu_pow(((float)j + 0.5f) * (1.f / 32.f) - edge, P);
        fe -= 1.f;
        unsigned ok = __ballot_sync(0xffffffffu, fe >= 0.f);
        int jstar = 31 - __clz(ok | 1u);
        float t0 = lo + (float)jstar * (1.f / 32.f);
        if (t0 > lo && t0 < hi) {
            float f, df;
            residual(X, n, am1, t0, P, f, df);
            if (f >= 0.f) lo = t0;
            else hi = t0;
        }
    }
    __syncwarp();

    // Safeguarded Newton: f is decreasing; Newton steps that leave (lo, hi)
    // are replaced by bisection.
    float tau = lo;
    for (int it = 0; it < 60; ++it) {
        float f, df;
        residual(X, n, am1, tau, P, f, df);
        if (f == 0.f) break;
        if (f > 0.f) lo = tau;
        else hi = tau;
        float nt = (df < 0.f) ? tau - f / df : 0.5f * (lo + hi);
        if (!(nt > lo && nt < hi)) nt = 0.5f * (lo + hi);
        if (fabsf(nt - tau) <= 1e-7f * fmaxf(1.f, fabsf(tau)) || hi - lo <= 1e-7f * fmaxf(1.f, fabsf(tau))) {
            tau = nt;
            break;
        }
        tau = nt;
    }

    // Exact polish on the support for alpha = 2 and alpha = 1.5.
    if (P.kint == 1 || P.kint == 2) {
        for (int pass = 0; pass < 4; ++pass) {
            float s1 = 0.f;
            int k = 0;
            for (int c = lane; c < n; c += 32) {
                float x = am1 * X[c];
                if (x > tau) { s1 += x; ++k; }
            }
            s1 = warp_sum(s1);
            k = warp_sum_i(k);
            if (k == 0) break;
            float nt;
            if (P.kint == 1) {
                nt = (s1 - 1.f) / (float)k;
            } else {
                const float m = s1 / (float)k;
                float v = 0.f;
                for (int c = lane; c < n; c += 32) {
                    float x = am1 * X[c];
                    if (x > tau) v += (x - m) * (x - m);
                }
                v = warp_sum(v) / (float)k;
                nt = m - sqrtf(fmaxf(1.f / (float)k - v, 0.f));
            }
            // same support under the new threshold?
            int k2 = 0;
            for (int c = lane; c < n; c += 32) k2 += (am1 * X[c] > nt);
            k2 = warp_sum_i(k2);
            tau = nt;
            if (k2 == k) break;
        }
    }
    return tau;
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
    const float *kb = kbar + ((size_t)b * G.n_chunks * G.hkv + r) * d;
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

    // (3) group prior, routed set, bias and mask, one warp per row
    const float am1 = P.alpha - 1.f;
    const float log_g = logf((float)g);
    for (int s = warp; s < nrows; s += kSelWarps) {
        const int64_t i = i0 + s;
        const int n = row_nvis(G, i);
        const size_t rowoff = ((size_t)(b * G.nq + i) * G.hkv + r);
        float lsum = 0.f;
        int cnt = 0;
        // first sweep: mu
        for (int c = lane; c < n; c += 32) {
            float mlog = -INFINITY;
            for (int hh = 0; hh < g; ++hh) {
                float t = am1 * X[(size_t)(s * g + hh) * P.ldx + c] - taus[s * g + hh];
                if (t > 0.f) mlog = fmaxf(mlog, P.kexp * logf(t));
            }
            if (mlog > -INFINITY) {
                float acc = 0.f;
                for (int hh = 0; hh < g; ++hh) {
                    float t = am1 * X[(size_t)(s * g + hh) * P.ldx + c] - taus[s * g + hh];
                    if (t > 0.f) acc += expf(P.kexp * logf(t) - mlog);
                }
                lsum += mlog + logf(acc) - log_g;
                ++cnt;
            }
        }
        lsum = warp_sum(lsum);
        cnt = warp_sum_i(cnt);
        const float mu = cnt ? lsum / (float)cnt : 0.f;
        // second sweep: bias, mask bits, optional w
        for (int c0 = 0; c0 < G.words * 32; c0 += 32) {
            const int c = c0 + lane;
            bool sel = false;
            float lw = -INFINITY;
            if (c < n) {
                float mlog = -INFINITY;
                for (int hh = 0; hh < g; ++hh) {
                    float t = am1 * X[(size_t)(s * g + hh) * P.ldx + c] - taus[s * g + hh];
                    if (t > 0.f) mlog = fmaxf(mlog, P.kexp * logf(t));
                }
                if (mlog > -INFINITY) {
                    float acc = 0.f;
                    for (int hh = 0; hh < g; ++hh) {
                        float t = am1 * X[(size_t)(s * g + hh) * P.ldx + c] - taus[s * g + hh];
                        if (t > 0.f) acc += expf(P.kexp * logf(t) - mlog);
                    }
                    lw = mlog + logf(acc) - log_g;
                    sel = true;
                }
            }
            const unsigned bits = __ballot_sync(0xffffffffu, sel);
            if (lane == 0) out.mask[rowoff * G.words + c0 / 32] = bits;
            if (sel && out.dvals) out.dvals[rowoff * G.n_chunks + c] = (lw - mu) / P.sigma;
            if (out.w && c < G.n_chunks) out.w[rowoff * G.n_chunks + c] = sel ? expf(lw) : 0.f;
        }
    }
}

// One CTA per (batch, kv head, query tile).
__global__ void __launch_bounds__(128) compact_kernel(Geom G, const uint32_t *__restrict__ mask,
                                                      const float *__restrict__ dvals, ListsView L) {
    extern __shared__ __align__(16) uint32_t csm[];
    uint32_t *uw = csm;                 // [words] union bits (diagonal range removed)
    int *wofs = reinterpret_cast<int *>(uw + G.words);  // [words + 1] exclusive prefix of popcounts
    const int64_t t = blockIdx.x;
    const int r = blockIdx.y;
    const int64_t b = blockIdx.z;
    const int T = L.tile_rows;
    const int64_t i0 = t * T;
    const int nrows = (int)min((int64_t)T, G.nq - i0);
    const size_t tile_idx = ((size_t)b * G.hkv + r) * L.n_tiles + t;

    // diagonal chunk range of the tile's rows (causal)
    int dlo = 0, dhi = -1;
    if (G.causal) {
        dlo = (int)(row_pos(G, i0) / G.B);
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
    for (int idx = threadIdx.x; idx < count * T; idx += blockDim.x) {
        const int e = idx / T, s = idx % T;
        const int c = ids[e];
        float v = -INFINITY;
        if (s >= nrows) {
            v = 0.f;  // padding row: never stored
        } else {
            const int64_t i = i0 + s;
            const size_t rowoff = ((size_t)(b * G.nq + i) * G.hkv + r);
            if (G.causal && c == (int)(row_pos(G, i) / G.B)) {
                v = 0.f;  // diagonal chunk: bias 0, causal mask in Stage 2
            } else if (c < row_nvis(G, i) && ((mask[rowoff * G.words + c / 32] >> (c % 32)) & 1u)) {
                v = dvals[rowoff * G.n_chunks + c];
            }
        }
        bias[(size_t)e * T + s] = v;
    }
}

}  // namespace

static int pick_rows_per_cta(const Geom &G, int dpad, int ldx, size_t *smem_out) {
    int best = 1;
    size_t best_smem = 0;
    for (int S = 1; S <= 32; S *= 2) {
        if (S * G.g > 128 && S > 1) break;
        size_t sm = ((size_t)S * G.g * dpad + (size_t)kTileChunks * dpad + (size_t)S * G.g * ldx + S * G.g) * 4 +
                    kSelWarps * 32 * 4;
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

cudaError_t launch_compact(const Geom &G, const uint32_t *mask, const float *dvals, const ListsView &L,
                           cudaStream_t st) {
    if (G.nq == 0 || G.b == 0) return cudaSuccess;
    dim3 grid((unsigned)L.n_tiles, (unsigned)G.hkv, (unsigned)G.b);
    const size_t smem = (size_t)G.words * 4 + (size_t)(G.words + 1) * 4 + 16;
    compact_kernel<<<grid, 128, smem, st>>>(G, mask, dvals, L);
    return cudaGetLastError();
}

}  // namespace dash

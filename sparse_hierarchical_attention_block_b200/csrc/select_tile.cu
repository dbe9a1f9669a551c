// select_tile.cu -- Stage 1 fused on tensor cores: routing + work-list compaction for
// one Stage-2 query tile per CTA (bf16 inputs, up to 512 routing chunks).
//
// For the 128 (query row, head) pairs of one (batch, kv head, query tile)
// ("DashAttention" §3.2 Eq. 4, App. G Alg. 2):
//   logits   X = gamma/sqrt(d) * Q K̄^T on tcgen05 into tensor memory: Q is bf16,
//            the fp32 chunk summaries are split k̄ = hi + lo into two bf16 operands
//            and both products accumulate in fp32 (relative error ~2^-17, i.e.
//            fp32-class logits); one TMEM lane per pair, one column per chunk;
//   tau      one thread per pair walks its TMEM row: max, a 32-bin shared-memory
//            histogram over [max x - 1, max x) for the starting point (AdaSplash-2's
//            initialisation), then a bracketed iteration: for alpha = 2 and 1.5 the
//            exact closed form on the current support (support shrinks until it is
//            stable), otherwise Newton, bisection as the safeguard;
//   prior    the g heads of a query row sit in g adjacent lanes of one warp:
//            w_c = (1/g) sum_h [x_c - tau_h]_+^{1/(alpha-1)} by shuffles, membership by
//            comparison (ballot), mu = mean log w over the routed chunks,
//            d_c = (log w_c - mu) / sigma (§3.4 Prop. 1);
//   lists    union of the tile's routed chunks (warp OR + shared atomics), the
//            diagonal chunks first, then the routed chunks ascending, and the
//            per-row bias table, written straight into the Stage-2 work lists.
#include <math.h>

#include "dash_common.cuh"
#include "kernels.h"
#include "tma_host.h"

namespace dash {

namespace {

constexpr int kTileThreads = 256;  // two threads per (row, head) pair
constexpr int kChunkTile = 128;  // chunks per logits MMA (N)
constexpr int kMaxTileChunks = 512;
constexpr uint64_t kTileWaitNs = 2000000000ull;

struct TileP {
    float am1;    // alpha - 1
    float kexp;   // 1 / (alpha - 1)
    int kint;     // 1/(alpha-1) when it is 1, 2 or 4, else 0
    float alpha;
    float scale;  // gamma / sqrt(d)
    float sigma;
    int ncols;    // allocated TMEM columns
};

struct TileOut {
    float *tau;
    float *w;
    uint32_t *mask;   // [b][nq][hkv][words]; required when lists are not built here
    float *logw;      // [b][nq][hkv][n_chunks] log w of the routed chunks (lists built later)
    float *mu;        // [b][nq][hkv] mean log w over the routed chunks (lists built later)
};

// [t]_+^{1/(alpha-1)} and [t]_+^{1/(alpha-1) - 1}; KINT is the exponent when it is
// 1, 2 or 4 (alpha = 2, 1.5, 1.25), 0 for a general alpha.
template <int KINT>
__device__ __forceinline__ float rpow(float t, const TileP &P) {
    if (t <= 0.f) return 0.f;
    if (KINT == 1) return t;
    if (KINT == 2) return t * t;
    if (KINT == 4) { const float u = t * t; return u * u; }
    return powf(t, P.kexp);
}
template <int KINT>
__device__ __forceinline__ float rpow_m1(float t, const TileP &P) {
    if (t <= 0.f) return 0.f;
    if (KINT == 1) return 1.f;
    if (KINT == 2) return t;
    if (KINT == 4) return t * t * t;
    return powf(t, P.kexp - 1.f);
}

template <int D>
struct TSmem {
    static constexpr int kRegion = 128 * 128;              // 128 rows x 128 bytes
    static constexpr int kDh = D / 64;
    // MMA phase: Q tile and one chunk tile of k̄ hi / lo operands
    static constexpr int kQ = 0;
    static constexpr int kHi = kQ + kDh * kRegion;
    static constexpr int kLo = kHi + kDh * kRegion;
    static constexpr int kMmaEnd = kLo + kDh * kRegion;
    // solve phase (reuses the MMA region once the logits are in TMEM)
    static constexpr int kHist = 0;                          // [2 halves][32 bins][128 pairs] uint16
    static constexpr int kXch = kHist + 2 * 32 * 128 * 2;     // [2 parity][2 halves][128 pairs][8] float
    static constexpr int kSolveEnd = kXch + 2 * 2 * 128 * 8 * 4;
    static constexpr int kData = kMmaEnd > kSolveEnd ? kMmaEnd : kSolveEnd;
    static constexpr int kUnion = kData;                     // [16] uint32
    static constexpr int kWofs = kUnion + 16 * 4;            // [17] int
    static constexpr int kBars = (kWofs + 17 * 4 + 7) & ~7;  // q_full, mma_done, k_full
    static constexpr int kSlot = kBars + 3 * 8;
    static constexpr int kTotal = kSlot + 16;
};

// k̄ [b][n_chunks][hkv][d] fp32 -> per (b, kv head, tile of 128 chunks) the bf16 pair
// hi = bf16(k̄), lo = bf16(k̄ - hi), each laid out exactly as the logits MMA reads it
// (K-major, 64-column regions of 128 rows x 128 bytes, 128-byte swizzle), so a CTA
// fetches a chunk tile with two bulk copies.  Chunks past n_chunks are zero.
template <int D>
__global__ void __launch_bounds__(256) kbar_split_kernel(const float *__restrict__ kbar, Geom G,
                                                         uint8_t *__restrict__ split) {
    constexpr int kDh = D / 64, kRegion = 128 * 128;
    const int ct = blockIdx.x, r = blockIdx.y;
    const int64_t b = blockIdx.z;
    const int n_ct = gridDim.x;
    uint8_t *dst = split + ((((size_t)b * G.hkv + r) * n_ct + ct) * 2) * (size_t)(kDh * kRegion);
    for (int u = threadIdx.x; u < 128 * (D / 8); u += 256) {
        const int c = u / (D / 8), j = u % (D / 8);
        const int cg = ct * 128 + c;
        float v[8];
        if (cg < G.n_chunks) {
            const float *src = kbar + (((size_t)b * G.n_chunks + cg) * G.hkv + r) * D + j * 8;
            const float4 a = *reinterpret_cast<const float4 *>(src);
            const float4 q = *reinterpret_cast<const float4 *>(src + 4);
            v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = q.x; v[5] = q.y; v[6] = q.z; v[7] = q.w;
        } else {
#pragma unroll
            for (int x = 0; x < 8; ++x) v[x] = 0.f;
        }
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int x = 0; x < 4; ++x) {
            const __nv_bfloat16 h0 = __float2bfloat16_rn(v[2 * x]), h1 = __float2bfloat16_rn(v[2 * x + 1]);
            __nv_bfloat162 hv;
            hv.x = h0;
            hv.y = h1;
            hi[x] = *reinterpret_cast<uint32_t *>(&hv);
            lo[x] = pack_bf16x2(v[2 * x] - __bfloat162float(h0), v[2 * x + 1] - __bfloat162float(h1));
        }
        const int off = (j / 8) * kRegion + c * 128 + (((j % 8) ^ (c & 7)) << 4);
        *reinterpret_cast<uint4 *>(dst + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        *reinterpret_cast<uint4 *>(dst + kDh * kRegion + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
    }
}

// Exchange of per-pass partial sums between the two threads of a pair (warps w and
// w + 4 share TMEM lanes): each writes its NV values, a named barrier over those two
// warps, each reads its partner's.  `parity` alternates the buffer so one barrier per
// pass suffices.
// Named barrier over the two warps (64 threads) that share TMEM lane quadrant `quad`;
// constant ids 1..4 (0 is __syncthreads).
__device__ __forceinline__ void quad_sync(int quad) {
    switch (quad) {
        case 0: asm volatile("bar.sync 1, 64;" ::: "memory"); break;
        case 1: asm volatile("bar.sync 2, 64;" ::: "memory"); break;
        case 2: asm volatile("bar.sync 3, 64;" ::: "memory"); break;
        default: asm volatile("bar.sync 4, 64;" ::: "memory"); break;
    }
}

template <int NV>
__device__ __forceinline__ void pair_exchange(float *xch, int parity, int half, int p, int quad, float (&v)[NV]) {
    float *mine = xch + ((size_t)(parity * 2 + half) * 128 + p) * 8;
    const float *other = xch + ((size_t)(parity * 2 + (half ^ 1)) * 128 + p) * 8;
#pragma unroll
    for (int k = 0; k < NV; ++k) mine[k] = v[k];
    quad_sync(quad);
#pragma unroll
    for (int k = 0; k < NV; ++k) v[k] = other[k];
}

template <int D, int KINT>
__global__ void __launch_bounds__(kTileThreads, 1) select_tile_kernel(const __grid_constant__ CUtensorMap tmQ,
                                                                      const uint8_t *__restrict__ ksplit, Geom G,
                                                                      TileP P, TileOut out, ListsView L) {
    using S = TSmem<D>;
    extern __shared__ uint8_t tsm_raw[];
    uint8_t *sm = tsm_raw + ((1024 - (smem_u32(tsm_raw) & 1023)) & 1023);
    uint64_t *q_full = reinterpret_cast<uint64_t *>(sm + S::kBars);
    uint64_t *mma_done = q_full + 1;
    uint64_t *k_full = q_full + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + S::kSlot);
    uint16_t *hist = reinterpret_cast<uint16_t *>(sm + S::kHist);
    float *xch = reinterpret_cast<float *>(sm + S::kXch);
    uint32_t *uni = reinterpret_cast<uint32_t *>(sm + S::kUnion);
    int *wofs = reinterpret_cast<int *>(sm + S::kWofs);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int quad = warp & 3, half = warp >> 2;  // TMEM lane quadrant; which 32-column blocks
    const int64_t t = (int64_t)L.n_tiles - 1 - blockIdx.x;
    const int r = blockIdx.y;
    const int64_t b = blockIdx.z;
    const int g = G.g, T = L.tile_rows;
    const int p = quad * 32 + lane;  // pair == TMEM lane
    const int pos = p / g, hh = p % g;
    const int64_t i = t * T + pos;
    const bool row_ok = i < G.nq;
    const int nvis = row_ok ? row_nvis(G, i) : 0;
    const int64_t last_row = min(G.nq - 1, t * T + T - 1);
    const int nvis_max = row_nvis(G, last_row);
    const size_t tile_idx = ((size_t)b * G.hkv + r) * L.n_tiles + t;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const bool lead = hh == 0;

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        mbar_init(mma_done, 1);
        mbar_init(k_full, 1);
        fence_mbar_init();
    }
    if (threadIdx.x < 16) uni[threadIdx.x] = 0u;
    if (warp == 0) {
        tmem_alloc(tmem_slot, (uint32_t)P.ncols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // ---------------------------------------------------------------- logits
    const int n_ct = (nvis_max + kChunkTile - 1) / kChunkTile;
    if (n_ct > 0 && threadIdx.x == 0) {
        mbar_arrive_expect_tx(q_full, 128 * D * 2);
        for (int dh = 0; dh < S::kDh; ++dh)
            tma_load_4d(sm + S::kQ + dh * S::kRegion, &tmQ, q_full, dh * 64, r * g, (int)(t * T), (int)b);
    }
    const int n_ct_all = (G.n_chunks + kChunkTile - 1) / kChunkTile;
    const uint8_t *ks = ksplit + (((size_t)b * G.hkv + r) * n_ct_all) * 2 * (size_t)(S::kDh * S::kRegion);
    for (int ct = 0; ct < n_ct; ++ct) {
        if (threadIdx.x == 0) {
            // the chunk tile's hi / lo operands, pre-split and pre-swizzled: two bulk copies
            const uint8_t *src = ks + (size_t)ct * 2 * S::kDh * S::kRegion;
            mbar_arrive_expect_tx(k_full, 2 * S::kDh * S::kRegion);
            bulk_load(sm + S::kHi, src, S::kDh * S::kRegion, k_full);
            bulk_load(sm + S::kLo, src + S::kDh * S::kRegion, S::kDh * S::kRegion, k_full);
            if (ct == 0) mbar_wait_ns(q_full, 0, kTileWaitNs);
            mbar_wait_ns(k_full, ct & 1, kTileWaitNs);
            tc_fence_after();
            constexpr uint32_t id = idesc_bf16_f32(128, kChunkTile, 0, 0);
            const uint32_t qb = smem_u32(sm + S::kQ), hb = smem_u32(sm + S::kHi), lb = smem_u32(sm + S::kLo);
            const uint32_t dcol = tmem + (uint32_t)(ct * kChunkTile);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t qa = qb + (kk / 4) * S::kRegion + (kk % 4) * 32;
                const uint32_t ka = hb + (kk / 4) * S::kRegion + (kk % 4) * 32;
                mma_ss(dcol, smem_desc_sw128(qa, 16, 1024), smem_desc_sw128(ka, 16, 1024), id, kk > 0 ? 1u : 0u);
            }
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t qa = qb + (kk / 4) * S::kRegion + (kk % 4) * 32;
                const uint32_t ka = lb + (kk / 4) * S::kRegion + (kk % 4) * 32;
                mma_ss(dcol, smem_desc_sw128(qa, 16, 1024), smem_desc_sw128(ka, 16, 1024), id, 1u);
            }
            mma_commit(mma_done);
        }
        mbar_wait_ns(mma_done, ct & 1, kTileWaitNs);  // smem tile free, TMEM columns written
        tc_fence_after();
    }
    __syncthreads();  // the MMA staging memory is reused below

    // ---------------------------------------------------------------- tau per pair
    // Thread (quad, half) owns the 32-column blocks blk = half, half + 2, ... of its
    // pair's TMEM row; the loop bound is uniform across each warp (tcgen05.ld is
    // warp-collective) and the two threads of a pair combine partial sums per pass.
    const int nb = (__reduce_max_sync(0xffffffffu, (unsigned)nvis) + 31) / 32;
    const float xs = P.am1 * P.scale;  // x = (alpha - 1) * gamma / sqrt(d) * <q, k̄>
    int parity = 0;
    // pass 0: x = (alpha-1) gamma/sqrt(d) <q, k̄> written back over the logits (later
    // passes read x directly), and its maximum over the visible chunks
    float mx = -INFINITY;
    for (int blk = half; blk < nb; blk += 2) {
        uint32_t u[32];
        tmem_ld32(tmem + lane_off + blk * 32, u);
#pragma unroll
        for (int x = 0; x < 32; ++x) {
            const float xv = xs * __uint_as_float(u[x]);
            if (blk * 32 + x < nvis) mx = fmaxf(mx, xv);
            u[x] = __float_as_uint(xv);
        }
        tmem_st32(tmem + lane_off + blk * 32, u);
    }
    tmem_wait_st();
    {
        float v[1] = {mx};
        pair_exchange<1>(xch, parity, half, p, quad, v);
        parity ^= 1;
        mx = fmaxf(mx, v[0]);
    }
    // bracket: f(mx - 1) >= 0 (the largest term alone is 1), f(mx - n^{1-alpha}) <= 0
    float lo = mx - 1.f;
    float hi = nvis > 0 ? mx - powf((float)nvis, 1.f - P.alpha) : 0.f;
    // histogram initialisation: bins [half][bin][pair] over [mx - 1, mx)
    uint16_t *hmine = hist + (size_t)half * 32 * 128;
#pragma unroll
    for (int j = 0; j < 32; ++j) hmine[j * 128 + p] = 0;
    for (int blk = half; blk < nb; blk += 2) {
        uint32_t u[32];
        tmem_ld32(tmem + lane_off + blk * 32, u);
#pragma unroll
        for (int x = 0; x < 32; ++x) {
            const float y = __uint_as_float(u[x]) - lo;
            if (blk * 32 + x < nvis && y >= 0.f) hmine[min(31, (int)(y * 32.f)) * 128 + p] += 1;
        }
    }
    quad_sync(quad);
    float t0 = lo;
    if (nvis > 1) {
        // estimated f at a bin edge e (every element at its bin centre c_j):
        //   f~(e) = sum_{j >= bin(e)} n_j (c_j - e)^k - 1, decreasing in e;
        // start from the highest edge still estimated >= 0.  For k = 1, 2, 4 the sum is
        // expanded in suffix moments A_m = sum_{j >= bin} n_j c_j^m (one sweep from the top).
        int elo = 0;
        if (KINT == 1 || KINT == 2 || KINT == 4) {
            float A0 = 0.f, A1 = 0.f, A2 = 0.f, A3 = 0.f, A4 = 0.f;
            for (int e = 31; e >= 1; --e) {
                const float n = (float)(hist[e * 128 + p] + hist[32 * 128 + e * 128 + p]);
                const float c = ((float)e + 0.5f) * (1.f / 32.f), c2 = c * c;
                A0 += n;
                A1 += n * c;
                A2 += n * c2;
                if (KINT == 4) {
                    A3 += n * c2 * c;
                    A4 += n * c2 * c2;
                }
                const float x = (float)e * (1.f / 32.f);
                float fe;
                if (KINT == 1) fe = A1 - x * A0;
                else if (KINT == 2) fe = A2 - 2.f * x * A1 + x * x * A0;
                else fe = A4 - 4.f * x * A3 + 6.f * x * x * A2 - 4.f * x * x * x * A1 + x * x * x * x * A0;
                if (fe - 1.f >= 0.f) {
                    elo = e;
                    break;
                }
            }
        } else {
            int ehi = 31;
            while (elo < ehi) {
                const int e = (elo + ehi + 1) / 2;
                const float edge = (float)e * (1.f / 32.f);
                float fe = -1.f;
                for (int j = e; j < 32; ++j)
                    fe += (float)(hist[j * 128 + p] + hist[32 * 128 + j * 128 + p]) *
                          rpow<KINT>(((float)j + 0.5f) * (1.f / 32.f) - edge, P);
                if (fe >= 0.f) elo = e;
                else ehi = e - 1;
            }
        }
        t0 = lo + (float)elo * (1.f / 32.f);
        if (!(t0 < hi)) t0 = lo;
    }
    // bracketed iteration (identical on both threads of the pair: same combined sums)
    float tau = nvis == 1 ? lo : t0;
    bool done = nvis <= 1;
    int prev_cnt = -1;
    for (int it = 0; it < 40; ++it) {
        if (__all_sync(0xffffffffu, done)) break;
        // partial sums over the support {x > tau}: for alpha = 2 / 1.5 only the moments of
        // y = x - mx (f follows from them), otherwise f + 1 and -f'/k as well
        float acc[5] = {0.f, 0.f, 0.f, 0.f, 0.f};  // s1, s2, count, f + 1, -f'/k
        for (int blk = half; blk < nb; blk += 2) {
            uint32_t u[32];
            tmem_ld32(tmem + lane_off + blk * 32, u);
#pragma unroll
            for (int x = 0; x < 32; ++x) {
                const float xv = __uint_as_float(u[x]);
                const float tt = xv - tau;
                if (blk * 32 + x < nvis && tt > 0.f) {
                    const float yv = xv - mx;
                    acc[0] += yv;
                    acc[1] = fmaf(yv, yv, acc[1]);
                    acc[2] += 1.f;
                    if (KINT != 1 && KINT != 2) {
                        acc[3] += rpow<KINT>(tt, P);
                        acc[4] += rpow_m1<KINT>(tt, P);
                    }
                }
            }
        }
        {
            float v[5] = {acc[0], acc[1], acc[2], acc[3], acc[4]};
            pair_exchange<5>(xch, parity, half, p, quad, v);
            parity ^= 1;
            // the same order of additions on both threads of the pair
#pragma unroll
            for (int k = 0; k < 5; ++k) acc[k] = half == 0 ? acc[k] + v[k] : v[k] + acc[k];
        }
        if (done) continue;
        const float s1 = acc[0], s2 = acc[1];
        const int cnt = (int)acc[2];
        const float tr = tau - mx;  // tau in the y = x - mx frame
        float f, df;
        if (KINT == 1) {
            f = s1 - tr * (float)cnt - 1.f;  // sum (y - tr) - 1
            df = -(float)cnt;
        } else if (KINT == 2) {
            f = s2 - 2.f * tr * s1 + tr * tr * (float)cnt - 1.f;  // sum (y - tr)^2 - 1
            df = -2.f * (s1 - tr * (float)cnt);
        } else {
            f = acc[3] - 1.f;
            df = -P.kexp * acc[4];
        }
        if (f >= 0.f) lo = tau;
        else hi = tau;
        float nt;
        if ((KINT == 1 || KINT == 2) && cnt > 0) {
            // the previous step was the exact closed form on this same support
            // (supports {x > tau} are nested, so equal counts mean equal sets): done
            if (cnt == prev_cnt) {
                done = true;
                continue;
            }
            prev_cnt = cnt;
            const float m1 = s1 / (float)cnt;
            if (KINT == 1) {
                nt = mx + (s1 - 1.f) / (float)cnt;
            } else {
                const float var = fmaxf(s2 / (float)cnt - m1 * m1, 0.f);
                nt = mx + m1 - sqrtf(fmaxf(1.f / (float)cnt - var, 0.f));
            }
            if (!(nt >= lo && nt <= hi)) {
                nt = 0.5f * (lo + hi);  // a bisection step: the next count proves nothing
                prev_cnt = -1;
            }
        } else {
            nt = df < 0.f ? tau - f / df : 0.5f * (lo + hi);
            if (!(nt > lo && nt < hi)) nt = 0.5f * (lo + hi);
            if (fabsf(nt - tau) <= 1e-7f * fmaxf(1.f, fabsf(tau)) || hi - lo <= 1e-7f * fmaxf(1.f, fabsf(tau)))
                done = true;
        }
        tau = nt;
    }
    if (nvis == 0) tau = NAN;
    if (half == 0) {
        if (out.tau && row_ok) out.tau[((size_t)b * G.nq + i) * G.hq + r * g + hh] = tau;
        if (L.rows && lead) L.rows[tile_idx * T + pos] = row_ok ? (int)i : -1;
    }

    // ---------------------------------------------------------------- group prior, pass 1: mu, union
    // When this kernel builds the tile's lists itself, log w_c replaces x_c in this lane's
    // TMEM row (-inf where the row does not route c) and pass 2 writes the bias table once
    // mu is known.  Otherwise (rows regrouped across tiles) pass 1 writes log w, the mask
    // and mu, and the regroup kernel forms d = (log w - mu) / sigma.
    const bool lists_mode = L.count != nullptr;
    const size_t rowoff = ((size_t)b * G.nq + i) * G.hkv + r;
    const int gshift = (lane / g) * g;
    const uint32_t gmask = (g == 32) ? 0xffffffffu : ((1u << g) - 1u);
    const float log_g = logf((float)g);
    const float tau_r = nvis > 0 ? tau : INFINITY;  // rows without chunks select nothing
    float lsum = 0.f, lcnt = 0.f;
    for (int blk = half; blk < nb; blk += 2) {
        uint32_t u[32];
        tmem_ld32(tmem + lane_off + blk * 32, u);
        uint32_t word = 0;
#pragma unroll
        for (int x = 0; x < 32; ++x) {
            const float tt = __uint_as_float(u[x]) - tau_r;
            const bool own = (blk * 32 + x < nvis) && tt > 0.f;
            float v = own ? rpow<KINT>(tt, P) : 0.f;
            for (int o = 1; o < g; o <<= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
            const uint32_t bal = __ballot_sync(0xffffffffu, own);
            const bool sel = ((bal >> gshift) & gmask) != 0u;
            float lw = -INFINITY;
            if (sel) {
                // the power sum underflows only for scores within ~1e-10 of tau at alpha = 1.25;
                // keep such a chunk routed with the smallest representable weight
                lw = v > 0.f ? __logf(v) - log_g : -103.28f - log_g;
                lsum += lw;
                lcnt += 1.f;
                word |= 1u << x;
            }
            u[x] = __float_as_uint(lw);
            if (!lists_mode && lead && row_ok && blk * 32 + x < nvis) {
                if (sel) out.logw[rowoff * G.n_chunks + blk * 32 + x] = lw;
                if (out.w) out.w[rowoff * G.n_chunks + blk * 32 + x] = sel ? expf(lw) : 0.f;
            }
        }
        if (lists_mode) tmem_st32(tmem + lane_off + blk * 32, u);
        else if (lead && row_ok) out.mask[rowoff * G.words + blk] = word;
        const uint32_t wu = __reduce_or_sync(0xffffffffu, word);
        if (lane == 0 && wu) atomicOr(&uni[blk], wu);
    }
    if (lists_mode) tmem_wait_st();
    {
        float v[2] = {lsum, lcnt};
        pair_exchange<2>(xch, parity, half, p, quad, v);
        parity ^= 1;
        lsum = half == 0 ? lsum + v[0] : v[0] + lsum;
        lcnt = half == 0 ? lcnt + v[1] : v[1] + lcnt;
    }
    const float mu = lcnt > 0.f ? lsum / lcnt : 0.f;
    if (!lists_mode && lead && row_ok && half == 0) {
        out.mu[rowoff] = mu;
        for (int blk = nb; blk < G.words; ++blk) out.mask[rowoff * G.words + blk] = 0u;
        if (out.w)
            for (int c = nvis; c < G.n_chunks; ++c) out.w[rowoff * G.n_chunks + c] = 0.f;
    }
    __syncthreads();

    // ---------------------------------------------------------------- the tile's list
    int dlo = 0, dhi = -1;
    if (G.causal) {
        dlo = (int)(row_pos(G, t * T) / G.B);
        dhi = (int)(row_pos(G, last_row) / G.B);
        if (dhi > G.n_blk - 1) dhi = G.n_blk - 1;
    }
    const int nd = dhi - dlo + 1;
    const int nwords = (nvis_max + 31) / 32;
    if (threadIdx.x == 0 && lists_mode) {
        int acc = nd;
        for (int w = 0; w < nwords; ++w) {
            uint32_t uw = uni[w];
            for (int c = max(dlo, w * 32); c <= min(dhi, w * 32 + 31); ++c) uw &= ~(1u << (c - w * 32));
            uni[w] = uw;
            wofs[w] = acc;
            acc += __popc(uw);
        }
        wofs[nwords] = acc;
        L.count[tile_idx] = acc;
    }
    __syncthreads();
    const int count = lists_mode ? wofs[nwords] : 0;
    int32_t *ids = lists_mode ? L.ids + tile_idx * L.cap : nullptr;
    float *bias = lists_mode ? L.bias + tile_idx * (size_t)L.cap * T : nullptr;
    for (int e = threadIdx.x; lists_mode && e < nd; e += kTileThreads) ids[e] = dlo + e;
    for (int w = threadIdx.x; lists_mode && w < nwords; w += kTileThreads) {
        uint32_t uw = uni[w];
        int q = wofs[w];
        while (uw) {
            const int bit = __ffs(uw) - 1;
            uw &= uw - 1;
            ids[q++] = w * 32 + bit;
        }
    }
    // default bias: -inf (row does not attend), 0 for padding rows and for each row's own diagonal chunk
    for (int idx = threadIdx.x; lists_mode && idx < count * T; idx += kTileThreads) {
        const int e = idx / T, s = idx % T;
        float v = -INFINITY;
        if (t * T + s >= G.nq) v = 0.f;
        else if (e < nd && dlo + e == (int)(row_pos(G, t * T + s) / G.B)) v = 0.f;
        bias[idx] = v;
    }
    __syncthreads();

    // ---------------------------------------------------------------- pass 2 (lists mode): bias, optional w / mask
    const float inv_sigma = 1.f / P.sigma;
    for (int blk = half; lists_mode && blk < nb; blk += 2) {
        uint32_t u[32];
        tmem_ld32(tmem + lane_off + blk * 32, u);
        uint32_t word = 0;
        const uint32_t uw = uni[blk];
        const int base = wofs[blk];
#pragma unroll
        for (int x = 0; x < 32; ++x) {
            const int c = blk * 32 + x;
            const float lw = __uint_as_float(u[x]);
            const bool sel = lw > -INFINITY;
            if (lead && row_ok && c < nvis) {
                if (sel) word |= 1u << x;
                if ((uw >> x) & 1u) {
                    const int e = base + __popc(uw & ((1u << x) - 1u));
                    bias[(size_t)e * T + pos] = sel ? (lw - mu) * inv_sigma : -INFINITY;
                } else if (c >= dlo && c <= dhi && sel) {
                    bias[(size_t)(c - dlo) * T + pos] = (lw - mu) * inv_sigma;
                }
                if (out.w) out.w[rowoff * G.n_chunks + c] = sel ? expf(lw) : 0.f;
            }
        }
        if (out.mask && lead && row_ok && blk < G.words) out.mask[rowoff * G.words + blk] = word;
    }
    if (lists_mode && lead && row_ok && half == 0) {
        if (out.mask)
            for (int blk = nb; blk < G.words; ++blk) out.mask[rowoff * G.words + blk] = 0u;
        if (out.w)
            for (int c = nvis; c < G.n_chunks; ++c) out.w[rowoff * G.n_chunks + c] = 0.f;
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, (uint32_t)P.ncols);
    }
}

}  // namespace

int take_device_error_select() { return take_device_error_local(); }

bool select_tile_supported(const Geom &G, dash_dtype_t dt) {
    if (dt != DASH_BF16) return false;
    if (G.d != 64 && G.d != 128) return false;
    if (G.g & (G.g - 1)) return false;
    if (G.tile_rows * G.g != 128) return false;
    if (G.n_chunks > kMaxTileChunks) return false;
    return tma_encode_fn() != nullptr;
}

size_t select_tile_workspace(const Geom &G) {
    const size_t n_ct = (G.n_chunks + kChunkTile - 1) / kChunkTile;
    return (size_t)G.b * G.hkv * n_ct * 2 * (G.d / 64) * 128 * 128;
}

cudaError_t launch_select_tile(const TView &Q, const float *kbar, const Geom &G, float alpha, float gamma,
                               float sigma, float *tau, float *w, uint32_t *mask, float *logw, float *mu,
                               const ListsView &L, void *work, cudaStream_t st) {
    if (G.nq == 0 || G.b == 0) return cudaSuccess;
    uint8_t *ksplit = static_cast<uint8_t *>(work);
    const int n_ct = (G.n_chunks + kChunkTile - 1) / kChunkTile;
    if (n_ct > 0) {
        dim3 sg((unsigned)n_ct, (unsigned)G.hkv, (unsigned)G.b);
        if (G.d == 128) kbar_split_kernel<128><<<sg, 256, 0, st>>>(kbar, G, ksplit);
        else kbar_split_kernel<64><<<sg, 256, 0, st>>>(kbar, G, ksplit);
        cudaError_t e0 = cudaGetLastError();
        if (e0 != cudaSuccess) return e0;
    }
    CUtensorMap tmQ;
    if (!make_map_bf16(&tmQ, Q, G.b, G.nq, G.hq, G.d, G.g, G.tile_rows)) return cudaErrorInvalidValue;
    TileP P;
    P.alpha = alpha;
    P.am1 = alpha - 1.f;
    P.kexp = 1.f / (alpha - 1.f);
    P.kint = (alpha == 2.f) ? 1 : (alpha == 1.5f) ? 2 : (alpha == 1.25f) ? 4 : 0;
    P.scale = gamma / sqrtf((float)G.d);
    P.sigma = sigma;
    int nc = ((G.n_chunks + kChunkTile - 1) / kChunkTile) * kChunkTile;
    int ncols = 32;
    while (ncols < nc) ncols *= 2;
    P.ncols = ncols;
    TileOut o{tau, w, mask, logw, mu};
    dim3 grid((unsigned)L.n_tiles, (unsigned)G.hkv, (unsigned)G.b);
    cudaError_t e = cudaErrorNotSupported;
#define DASH_SEL_CASE(DD, KK)                                                                              \
    if (G.d == DD && P.kint == KK) {                                                                       \
        const size_t smem = TSmem<DD>::kTotal + 1024;                                                      \
        e = cudaFuncSetAttribute(select_tile_kernel<DD, KK>, cudaFuncAttributeMaxDynamicSharedMemorySize, \
                                 (int)smem);                                                               \
        if (e != cudaSuccess) return e;                                                                    \
        select_tile_kernel<DD, KK><<<grid, kTileThreads, smem, st>>>(tmQ, ksplit, G, P, o, L);            \
        return cudaGetLastError();                                                                         \
    }
    DASH_SEL_CASE(128, 2)
    DASH_SEL_CASE(128, 1)
    DASH_SEL_CASE(128, 4)
    DASH_SEL_CASE(128, 0)
    DASH_SEL_CASE(64, 2)
    DASH_SEL_CASE(64, 1)
    DASH_SEL_CASE(64, 4)
    DASH_SEL_CASE(64, 0)
#undef DASH_SEL_CASE
    return e;
}

}  // namespace dash

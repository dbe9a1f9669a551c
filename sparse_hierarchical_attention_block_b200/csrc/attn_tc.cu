// attn_tc.cu -- Stage 2 on the 5th-generation tensor cores (tcgen05 + TMEM + TMA), bf16.
//
// Prior-induced sparse softmax in the bias form of "DashAttention" §3.4 Prop. 1
// (App. G Alg. 3): for every row of a query tile
//   o = sum_j exp(z_j + d_j) v_j / sum_t exp(z_t + d_t),   z_j = <q, k_j>/sqrt(d),
// over the keys of the chunks in the tile's work list, d_j the list's per-row
// bias (-inf where the row does not attend the chunk), keys j > p_i masked when
// causal.  Online softmax in the exp2 domain with fp32 statistics.
//
// One CTA per (batch, kv head, query tile of 128/g positions x g heads = 128 rows), the
// heaviest (latest, causal) tiles first within groups of heads whose K and V fit in L2
// together (all heads at 8K, one at a time at 128K), two CTAs resident per SM.  A step
// covers 64 keys (one or more listed chunks, or half of a 128-key chunk); S is
// double-buffered in tensor memory, so the MMA of step j+1 runs during the softmax of
// step j.  Warp roles (192 threads):
//   warp 0     TMA producer: Q tile once; per step the listed K and V blocks (one TMA
//              box per chunk, or half chunk, and 64-column half, 128-byte swizzle) into
//              two-stage rings, and the step's bias rows (bulk copy);
//   warp 1     TMEM allocator (256 columns: S[0], S[1] of 64 columns each, O) and MMA
//              issuer (one thread), order S_0, S_1, PV_0, S_2, PV_1, ...:
//              S_j = Q K_j^T  (SS, M=128 N=64 K=d) into S[j % 2] once PV_{j-2}, the last
//              reader of that buffer, has completed;
//              O  += P_j V_j  (TS: P read from TMEM, V from smem as an MN-major operand);
//   warps 2-5  softmax: thread = TMEM lane = tile row; two passes over S_j in TMEM
//              (row max, then exp2 / sum / bf16 P written over S_j's first 32 columns), bias added and
//              keys masked only on steps that hold a diagonal or partial chunk; after
//              the first step a single pass on the running maximum (scale and row sum
//              on packed f32x2 pairs), redone as two passes only if a row's sum of p
//              exceeds 2^16 (O is rescaled when the maximum grows by more than 16 in
//              the exp2 domain); epilogue O / l -> bf16.
// Every mbarrier wait is bounded (globaltimer); a waiting thread suspends on the
// barrier rather than polling.  On expiry the kernel records a device error, drains
// what it issued, frees TMEM and returns.
#include <math.h>

#include "dash_common.cuh"
#include "kernels.h"
#include "tma_host.h"

namespace dash {

namespace {

constexpr int kThreads = 192;
constexpr int kRows = 128;      // MMA M
constexpr int kStepKeys = 64;   // keys per step = MMA N of S and K of PV
constexpr int kNS = 2;          // K / V stages
constexpr int kNM = 2;          // bias / id stages
constexpr uint32_t kTmemCols = 256;
// The running maximum (exp2 domain) is kept until a step's maximum exceeds it by more
// than this: p <= 2^16, so P (bf16), l and O (fp32) stay far from overflow.
constexpr float kRescaleL2 = 16.f;
constexpr float kRescaleP = 65536.f;  // 2^kRescaleL2
constexpr uint64_t kWaitNs = 2000000000ull;      // 2 s
constexpr uint64_t kWaitNsTest = 20000000ull;    // 20 ms under DASH_FLAG_TEST_TIMEOUT

struct TcParams {
    CUtensorMap tmQ, tmK, tmV;
};


template <int D, int BLK>
struct Smem {
    static constexpr int kRegion = kRows * 128;                 // bytes of one 64-column, 128-row swizzled region (Q)
    static constexpr int kSRegion = kStepKeys * 128;            // one 64-column region of a K or V stage
    static constexpr int kDh = D / 64;                          // regions per operand
    static constexpr int kE = BLK < kStepKeys ? kStepKeys / BLK : 1;   // list entries per step
    static constexpr int kSub = BLK > kStepKeys ? BLK / kStepKeys : 1; // steps per list entry
    static constexpr int kRowsE = BLK < kStepKeys ? BLK : kStepKeys;   // keys of one entry in a step
    static constexpr int kQ = 0;
    static constexpr int kK = kQ + kDh * kRegion;
    static constexpr int kV = kK + kNS * kDh * kSRegion;
    static constexpr int kBias = kV + kNS * kDh * kSRegion;     // [kNM][kE * 128] floats (tile_rows <= 128)
    static constexpr int kIds = kBias + kNM * kE * 128 * 4;     // [kNM][kE] int
    static constexpr int kBars = (kIds + kNM * kE * 4 + 7) & ~7;
    // barriers: q_full, k_full[NS], k_empty[NS], v_full[NS], v_empty[NS], m_full[NM], m_empty[NM],
    //           s_full[2], p_full[2], pv_done[2], fin
    static constexpr int kNumBars = 1 + 4 * kNS + 2 * kNM + 6 + 1;
    static constexpr int kMisc = kBars + kNumBars * 8;          // tmem base, abort flag, p_min
    static constexpr int kTotal = kMisc + 16 + 8;
};

struct Bars {
    uint64_t *q_full, *k_full, *k_empty, *v_full, *v_empty, *m_full, *m_empty, *s_full, *p_full, *pv_done, *fin;
};


// One 64-key step of the single-pass softmax for this thread's row: p = 2^(s * sl2 + cbm)
// from the step's S columns at taddr, packed to bf16 pairs in pk; returns the row's sum of
// p.  kMask applies the per-entry key limits (keys past the list or the row's position).
template <int kE, int kRowsE, bool kMask>
__device__ __forceinline__ float exp_step(uint32_t taddr, float sl2, const float (&cbm)[kE], const int (&lim)[kE],
                                          uint32_t (&pk)[32]) {
    const uint64_t sc2 = f32x2(sl2, sl2);
    uint64_t acc[2] = {f32x2(0.f, 0.f), f32x2(0.f, 0.f)};
#pragma unroll
    for (int qc = 0; qc < 4; ++qc) {
        uint32_t u[16];
        tmem_ld16(taddr + qc * 16, u);
#pragma unroll
        for (int x = 0; x < 8; ++x) {
            const int kc = qc * 16 + 2 * x;  // an entry spans an even number of keys: kc, kc + 1 share it
            const float cb = cbm[kc / kRowsE];
            float v0, v1;
            f32x2_split(fma_f32x2(f32x2(__uint_as_float(u[2 * x]), __uint_as_float(u[2 * x + 1])), sc2, f32x2(cb, cb)),
                        v0, v1);
            if (kMask) {  // select before exp2: S outside the list may be any bit pattern
                v0 = (kc % kRowsE) < lim[kc / kRowsE] ? v0 : -INFINITY;
                v1 = ((kc + 1) % kRowsE) < lim[kc / kRowsE] ? v1 : -INFINITY;
            }
            const float p0 = ex2(v0), p1 = ex2(v1);
            acc[x & 1] = add_f32x2(acc[x & 1], f32x2(p0, p1));
            pk[qc * 8 + x] = pack_bf16x2(p0, p1);
        }
    }
    float a, b;
    f32x2_split(add_f32x2(acc[0], acc[1]), a, b);
    return a + b;
}

template <int D, int BLK>
__global__ void __launch_bounds__(kThreads, 2) attn_tc_kernel(const __grid_constant__ TcParams tp, TView Qv, TView O,
                                                              Geom G, ListsView L, int flags, float *lse, int hg) {
    using S = Smem<D, BLK>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    // one CTA per (tile, batch, kv head), in the order of tile_order: groups of heads whose
    // K and V share L2, the heaviest (latest, causal) tiles of a group first
    const TileOrder to = tile_order(blockIdx.x, L.n_tiles, G.b * G.hkv, hg);
    const int64_t t = to.t;
    const int r = (int)(to.bh % G.hkv);
    const int64_t b = to.bh / G.hkv;
    const int g = G.g, T = L.tile_rows;
    const size_t tile_idx = ((size_t)b * G.hkv + r) * L.n_tiles + t;
    const int count = L.count[tile_idx];
    // the first step's chunk ids, requested before the set-up below (the first K copy waits on them)
    int ids_pre[Smem<D, BLK>::kE];
    if (threadIdx.x == 0) {
#pragma unroll
        for (int e = 0; e < Smem<D, BLK>::kE; ++e) ids_pre[e] = e < L.cap ? L.ids[tile_idx * L.cap + e] : 0;
    }
    const int nsteps = S::kSub > 1 ? count * S::kSub : (count + S::kE - 1) / S::kE;
    const bool test_timeout = (flags & DASH_FLAG_TEST_TIMEOUT) != 0;
    const uint64_t limit_ns = test_timeout ? kWaitNsTest : kWaitNs;

    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + S::kBars);
    Bars B;
    B.q_full = bars;
    B.k_full = B.q_full + 1;
    B.k_empty = B.k_full + kNS;
    B.v_full = B.k_empty + kNS;
    B.v_empty = B.v_full + kNS;
    B.m_full = B.v_empty + kNS;
    B.m_empty = B.m_full + kNM;
    B.s_full = B.m_empty + kNM;
    B.p_full = B.s_full + 2;
    B.pv_done = B.p_full + 2;
    B.fin = B.pv_done + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + S::kMisc);
    volatile int *abort = reinterpret_cast<volatile int *>(sm + S::kMisc + 4);
    long long *p_min_s = reinterpret_cast<long long *>(sm + S::kMisc + 8);
    float *bias_s = reinterpret_cast<float *>(sm + S::kBias);
    int *ids_s = reinterpret_cast<int *>(sm + S::kIds);

    const bool gather_q = L.rows != nullptr;  // rows regrouped: Q rows are gathered by the softmax threads
    if (threadIdx.x == 0) {
        mbar_init(B.q_full, gather_q ? 128 : 1);
        *p_min_s = 0x7fffffffffffffffll;
        for (int s = 0; s < kNS; ++s) {
            mbar_init(B.k_full + s, 1);
            mbar_init(B.k_empty + s, 1);
            mbar_init(B.v_full + s, 1);
            mbar_init(B.v_empty + s, 1);
        }
        for (int s = 0; s < kNM; ++s) {
            mbar_init(B.m_full + s, 1);
            mbar_init(B.m_empty + s, 128);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(B.s_full + s, 1);
            mbar_init(B.p_full + s, 128);
            mbar_init(B.pv_done + s, 1);
        }
        mbar_init(B.fin, 1);
        *abort = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // S_j in columns (j % 2) * 64.., then P_j (bf16) over its first 32; O from column 128
    const uint32_t tO = tmem + 128;

    if (warp == 0) {
        // ------------------------------------------------------------- producer
        if (lane == 0 && !test_timeout && nsteps > 0) {
            tma_prefetch_desc(&tp.tmK);
            tma_prefetch_desc(&tp.tmV);
            if (!gather_q) {
                mbar_arrive_expect_tx(B.q_full, kRows * D * 2);
                for (int dh = 0; dh < S::kDh; ++dh)
                    tma_load_4d(sm + S::kQ + dh * S::kRegion, &tp.tmQ, B.q_full, dh * 64, r * g, (int)(t * T),
                                (int)b);
            }
            const int32_t *ids_g = L.ids + tile_idx * L.cap;
            const float *bias_g = L.bias + tile_idx * (size_t)L.cap * T;
            int issued_m = 0, issued_k = 0, issued_v = 0;  // steps whose copies were issued
            for (int j = 0; j < nsteps; ++j) {
                // the step's entries e0.. (ne of them) and its first key within them
                const int e0 = S::kSub > 1 ? j / S::kSub : j * S::kE;
                const int ne = S::kSub > 1 ? 1 : min(S::kE, count - e0);
                const int koff = S::kSub > 1 ? (j % S::kSub) * kStepKeys : 0;
                const int ms = j % kNM, ks = j % kNS;
                if (!wait_bar(B.m_empty + ms, ((j / kNM) & 1) ^ 1, limit_ns, abort)) break;
                int *ids_st = ids_s + ms * S::kE;
                if (e0 == 0) {
#pragma unroll
                    for (int e = 0; e < S::kE; ++e)
                        if (e < ne) ids_st[e] = ids_pre[e];
                } else {
                    for (int e = 0; e < ne; ++e) ids_st[e] = ids_g[e0 + e];
                }
                mbar_arrive_expect_tx(B.m_full + ms, (uint32_t)(ne * T * 4));
                bulk_load(bias_s + ms * S::kE * 128, bias_g + (size_t)e0 * T, (uint32_t)(ne * T * 4), B.m_full + ms);
                issued_m = j + 1;
                if (!wait_bar(B.k_empty + ks, ((j / kNS) & 1) ^ 1, limit_ns, abort)) break;
                mbar_arrive_expect_tx(B.k_full + ks, (uint32_t)(ne * S::kDh * S::kRowsE * 128));
                for (int e = 0; e < ne; ++e)
                    for (int dh = 0; dh < S::kDh; ++dh)
                        tma_load_4d(sm + S::kK + (ks * S::kDh + dh) * S::kSRegion + e * S::kRowsE * 128, &tp.tmK,
                                    B.k_full + ks, dh * 64, r, ids_st[e] * BLK + koff, (int)b);
                issued_k = j + 1;
                if (!wait_bar(B.v_empty + ks, ((j / kNS) & 1) ^ 1, limit_ns, abort)) break;
                mbar_arrive_expect_tx(B.v_full + ks, (uint32_t)(ne * S::kDh * S::kRowsE * 128));
                for (int e = 0; e < ne; ++e)
                    for (int dh = 0; dh < S::kDh; ++dh)
                        tma_load_4d(sm + S::kV + (ks * S::kDh + dh) * S::kSRegion + e * S::kRowsE * 128, &tp.tmV,
                                    B.v_full + ks, dh * 64, r, ids_st[e] * BLK + koff, (int)b);
                issued_v = j + 1;
            }
            if (*abort) {
                // drain: every copy issued must land before the CTA's smem goes away.  Issued
                // copies always complete, so each drain wait gets the full bound.
                for (int j = max(0, issued_k - kNS); j < issued_k; ++j)
                    wait_bar(B.k_full + j % kNS, (j / kNS) & 1, kWaitNs, abort, false);
                for (int j = max(0, issued_v - kNS); j < issued_v; ++j)
                    wait_bar(B.v_full + j % kNS, (j / kNS) & 1, kWaitNs, abort, false);
                for (int j = max(0, issued_m - kNM); j < issued_m; ++j)
                    wait_bar(B.m_full + j % kNM, (j / kNM) & 1, kWaitNs, abort, false);
                if (!gather_q) wait_bar(B.q_full, 0, kWaitNs, abort, false);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t idS = idesc_bf16_f32(kRows, kStepKeys, 0, 0);
            constexpr uint32_t idPV = idesc_bf16_f32(kRows, D, 0, 1);
            const uint32_t q_base = smem_u32(sm + S::kQ);
            const uint32_t k_base = smem_u32(sm + S::kK);
            const uint32_t v_base = smem_u32(sm + S::kV);
            bool ok = nsteps == 0 || wait_bar(B.q_full, 0, limit_ns, abort);
            // S_j into S[j % 2]: its K stage, and for j >= 2 the completion of PV_{j-2}
            auto issue_s = [&](int j) -> bool {
                const int ks = j % kNS;
                if (j >= 2 && !wait_bar(B.pv_done + (j & 1), ((j - 2) >> 1) & 1, limit_ns, abort)) return false;
                if (!wait_bar(B.k_full + ks, (j / kNS) & 1, limit_ns, abort)) return false;
                tc_fence_after();
                const uint32_t tS = tmem + (uint32_t)((j & 1) * kStepKeys);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t qa = q_base + (kk / 4) * S::kRegion + (kk % 4) * 32;
                    const uint32_t kb = k_base + (ks * S::kDh + kk / 4) * S::kSRegion + (kk % 4) * 32;
                    mma_ss(tS, smem_desc_sw128(qa, 16, 1024), smem_desc_sw128(kb, 16, 1024), idS, kk > 0 ? 1u : 0u);
                }
                mma_commit(B.s_full + (j & 1));
                mma_commit(B.k_empty + ks);
                return true;
            };
            for (int j = 0; ok && j < min(nsteps, 2); ++j) ok = issue_s(j);
            for (int j = 0; ok && j < nsteps; ++j) {
                const int ks = j % kNS;
                const int ne = S::kSub > 1 ? 1 : min(S::kE, count - j * S::kE);
                if (!(ok = wait_bar(B.p_full + (j & 1), (j >> 1) & 1, limit_ns, abort))) break;
                if (!(ok = wait_bar(B.v_full + ks, (j / kNS) & 1, limit_ns, abort))) break;
                tc_fence_after();
                const uint32_t tS = tmem + (uint32_t)((j & 1) * kStepKeys);
                const int nks = ne * S::kRowsE / 16;
                for (int kk = 0; kk < nks; ++kk) {
                    const uint32_t vb = v_base + (ks * S::kDh) * S::kSRegion + kk * 2048;
                    mma_ts(tO, tS + kk * 8, smem_desc_sw128(vb, S::kSRegion, 1024), idPV, (j > 0 || kk > 0) ? 1u : 0u);
                }
                mma_commit(B.v_empty + ks);
                mma_commit(B.pv_done + (j & 1));
                if (j + 2 < nsteps) ok = issue_s(j + 2);
            }
            // every MMA this thread issued has completed before TMEM is freed
            mma_commit(B.fin);
            wait_bar(B.fin, 0, kWaitNs, abort, false);
        }
    } else {
        // ------------------------------------------------------------- softmax warpgroup
        const int quad = warp & 3;
        const int m = quad * 32 + lane;  // TMEM lane == tile row
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        const int pos = m / g;
        const int hh = m % g;
        const int64_t i = tile_row(L, G, tile_idx, t, pos);
        const bool row_ok = i >= 0;
        const int64_t p_row = row_pos(G, i);
        if (gather_q && nsteps > 0) {
            // this thread's Q row into the 128-byte-swizzled K-major layout the MMA reads
            const __nv_bfloat16 *src = reinterpret_cast<const __nv_bfloat16 *>(Qv.p) + b * Qv.s0 +
                                       (row_ok ? i : 0) * Qv.s1 + (int64_t)(r * g + hh) * Qv.s2;
#pragma unroll
            for (int cc = 0; cc < D / 8; ++cc) {
                const uint4 val = row_ok ? *reinterpret_cast<const uint4 *>(src + cc * 8) : make_uint4(0u, 0u, 0u, 0u);
                *reinterpret_cast<uint4 *>(sm + S::kQ + (cc / 8) * S::kRegion + m * 128 + (((cc % 8) ^ (m & 7)) << 4)) =
                    val;
            }
            fence_proxy_async_smem();
            mbar_arrive(B.q_full);
        }
        // keys of a chunk up to the smallest row position are visible to every row of the tile
        if (row_ok) atomicMin(p_min_s, (long long)p_row);
        asm volatile("bar.sync 1, 128;" ::: "memory");
        const int64_t p_min = *p_min_s;
        const float sl2 = rsqrtf((float)D) * 1.4426950408889634f;
        float m_run = -INFINITY, l_run = 0.f;
        bool ok = true;
        // tcgen05.ld / st are warp-collective: every decision that guards one is
        // made uniform across the warp (__any_sync / __all_sync).
        for (int j = 0; j < nsteps; ++j) {
            const int ms = j % kNM;
            const int ne = S::kSub > 1 ? 1 : min(S::kE, count - j * S::kE);
            const int koff = S::kSub > 1 ? (j % S::kSub) * kStepKeys : 0;  // first key of the step in its chunk
            const uint32_t tS = tmem + (uint32_t)((j & 1) * kStepKeys);
            ok = __all_sync(0xffffffffu, wait_bar(B.m_full + ms, (j / kNM) & 1, limit_ns, abort));
            if (!ok) break;
            // per-entry constants of this step: bias (exp2 domain) and, for masking, the
            // number of leading keys of the entry this row may see
            float bl2[S::kE];
            int lim[S::kE];
            bool need_mask = ne < S::kE;
            const int vis_end = (int)((G.causal && row_ok) ? min((int64_t)G.nk, p_row + 1) : G.nk);
#pragma unroll
            for (int e = 0; e < S::kE; ++e) {
                const int id = e < ne ? ids_s[ms * S::kE + e] : 0;
                bl2[e] = e < ne ? bias_s[ms * S::kE * 128 + e * T + pos] * 1.4426950408889634f : -INFINITY;
                lim[e] = e < ne ? max(0, min(S::kRowsE, vis_end - (id * BLK + koff))) : 0;
                // a chunk needs per-key masks if it reaches past the sequence or past the
                // smallest row position of the tile (it is some row's diagonal chunk)
                if (e < ne) {
                    const int64_t last_key = (int64_t)id * BLK + koff + S::kRowsE - 1;
                    need_mask |= last_key >= G.nk || (G.causal && last_key > p_min);
                }
            }
            mbar_arrive(B.m_empty + ms);
            ok = __all_sync(0xffffffffu, wait_bar(B.s_full + (j & 1), (j >> 1) & 1, limit_ns, abort));
            if (!ok) break;
            tc_fence_after();
            // Single pass on the running maximum of the earlier steps: p = 2^(s * scale +
            // bias - m_run) straight from S.  It stands unless a row of the warp sums p
            // above 2^kRescaleL2 (then P is discarded, S is still intact, and the two-pass
            // path below redoes the step with a new maximum).  P is held in
            // registers and written over S only once the step is known to stand.
            bool step_done = false;
            if (j > 0 && __all_sync(0xffffffffu, !row_ok || m_run > -INFINITY)) {
                float cbm[S::kE];
#pragma unroll
                for (int e = 0; e < S::kE; ++e) cbm[e] = row_ok ? bl2[e] - m_run : -INFINITY;
                uint32_t pk[32];
                const float psum = need_mask ? exp_step<S::kE, S::kRowsE, true>(tS + lane_off, sl2, cbm, lim, pk)
                                             : exp_step<S::kE, S::kRowsE, false>(tS + lane_off, sl2, cbm, lim, pk);
                // the step stands while the row's sum of p = 2^(logit - m_run) stays at most
                // 2^kRescaleL2 (then so does every p); a sum that overflowed is not finite
                if (!__any_sync(0xffffffffu, !(psum <= kRescaleP))) {
                    tmem_st32(tS + lane_off, pk);
                    l_run += psum;
                    step_done = true;
                }
            }
            if (!step_done) {
            // pass 1: row maximum of the biased, masked logits (exp2 domain)
            float mq[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
            for (int qc = 0; qc < 2; ++qc) {
                uint32_t u[32];
                tmem_ld32(tS + lane_off + qc * 32, u);
#pragma unroll
                for (int x = 0; x < 32; ++x) {
                    const int kc = qc * 32 + x;
                    const float v = fmaf(__uint_as_float(u[x]), sl2, bl2[kc / S::kRowsE]);
                    mq[x & 3] = fmaxf(mq[x & 3],
                                      (!need_mask || (kc % S::kRowsE) < lim[kc / S::kRowsE]) ? v : -INFINITY);
                }
            }
            float mx = fmaxf(fmaxf(mq[0], mq[1]), fmaxf(mq[2], mq[3]));
            if (!row_ok) mx = -INFINITY;
            // running maximum: kept unless the step's maximum exceeds it by more than kRescaleL2
            float f = 1.f;
            const bool rescale = mx > -INFINITY && m_run > -INFINITY && mx > m_run + kRescaleL2;
            if (mx > -INFINITY) {
                if (m_run == -INFINITY) {
                    m_run = mx;  // nothing accumulated for this row yet: O holds zeros
                } else if (rescale) {
                    f = ex2(m_run - mx);
                    l_run *= f;
                    m_run = mx;
                }
            }
            if (j > 0 && __any_sync(0xffffffffu, rescale)) {
                // O must hold every PV up to step j-1 before it is rescaled
                ok = __all_sync(0xffffffffu, wait_bar(B.pv_done + ((j - 1) & 1), ((j - 1) >> 1) & 1, limit_ns, abort));
                if (!ok) break;
                tc_fence_after();
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t u[32];
                    tmem_ld32(tO + lane_off + c * 32, u);
    #pragma unroll
                    for (int x = 0; x < 32; ++x) u[x] = __float_as_uint(__uint_as_float(u[x]) * f);
                    tmem_st32(tO + lane_off + c * 32, u);
                }
            }
            // pass 2: p = 2^(s * scale + bias - m), row sum, bf16 P over the first 64 columns of S.
            // A dead row (padding, or nothing visible yet) gets p = 0 through its constants.
            const bool live = row_ok && m_run > -INFINITY;
            float cbm[S::kE];
#pragma unroll
            for (int e = 0; e < S::kE; ++e) cbm[e] = live ? bl2[e] - m_run : -INFINITY;
            float pq[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int qc = 0; qc < 2; ++qc) {
                uint32_t u[32];
                tmem_ld32(tS + lane_off + qc * 32, u);
                uint32_t pk[16];
#pragma unroll
                for (int x = 0; x < 16; ++x) {
                    const int kc = qc * 32 + 2 * x;
                    float v0 = fmaf(__uint_as_float(u[2 * x]), sl2, cbm[kc / S::kRowsE]);
                    float v1 = fmaf(__uint_as_float(u[2 * x + 1]), sl2, cbm[(kc + 1) / S::kRowsE]);
                    if (need_mask) {  // select before exp2: S outside the list may be any bit pattern
                        v0 = (kc % S::kRowsE) < lim[kc / S::kRowsE] ? v0 : -INFINITY;
                        v1 = ((kc + 1) % S::kRowsE) < lim[(kc + 1) / S::kRowsE] ? v1 : -INFINITY;
                    }
                    const float p0 = ex2(v0), p1 = ex2(v1);
                    pq[x & 3] += p0 + p1;
                    pk[x] = pack_bf16x2(p0, p1);
                }
                // P of keys 32qc.. over columns 16qc..: S columns below 32(qc+1) are already read
                tmem_st16(tS + lane_off + qc * 16, pk);
            }
            const float psum = (pq[0] + pq[1]) + (pq[2] + pq[3]);
            l_run += psum;
            }  // two-pass path
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(B.p_full + (j & 1));
        }
        // epilogue: O / l -> bf16
        if (ok && !*abort) {
            bool have = true;
            if (nsteps > 0)
                have = __all_sync(0xffffffffu, wait_bar(B.pv_done + ((nsteps - 1) & 1), ((nsteps - 1) >> 1) & 1,
                                                        limit_ns, abort));
            tc_fence_after();
            if (have) {
                __nv_bfloat16 *op = reinterpret_cast<__nv_bfloat16 *>(const_cast<void *>(O.p)) + b * O.s0 +
                                    i * O.s1 + (int64_t)(r * g + hh) * O.s2;
                const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
                if (lse && row_ok)  // natural log of the row's normaliser: (m + log2 l) ln 2
                    lse[((size_t)b * G.nq_lse + i) * G.hq + r * g + hh] =
                        l_run > 0.f ? (m_run + __log2f(l_run)) * 0.6931471805599453f : -INFINITY;
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t u[32];
                    if (nsteps > 0) {  // uniform across the CTA
                        tmem_ld32(tO + lane_off + c * 32, u);
                            } else {
#pragma unroll
                        for (int x = 0; x < 32; ++x) u[x] = 0u;
                    }
                    if (row_ok) {
                        uint32_t pk[16];
#pragma unroll
                        for (int x = 0; x < 16; ++x)
                            pk[x] = pack_bf16x2(__uint_as_float(u[2 * x]) * inv, __uint_as_float(u[2 * x + 1]) * inv);
                        uint4 *dst = reinterpret_cast<uint4 *>(op + c * 32);
#pragma unroll
                        for (int x = 0; x < 4; ++x)
                            dst[x] = make_uint4(pk[4 * x], pk[4 * x + 1], pk[4 * x + 2], pk[4 * x + 3]);
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// ------------------------------------------------------------------ host side

template <int D, int BLK>
cudaError_t launch_t(const TcParams &tp, const TView &Q, const TView &O, const Geom &G, const ListsView &L, int flags,
                     cudaStream_t st, float *lse) {
    using S = Smem<D, BLK>;
    const size_t smem = S::kTotal + 1024;
    cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<D, BLK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    const int64_t ctas = L.n_tiles * G.hkv * G.b;
    if (ctas > 0x7fffffff) return cudaErrorInvalidValue;
    attn_tc_kernel<D, BLK><<<(unsigned)ctas, kThreads, smem, st>>>(tp, Q, O, G, L, flags, lse,
                                                                    heads_per_group(G));
    return cudaGetLastError();
}

}  // namespace

bool attn_tc_supported(const Geom &G, dash_dtype_t dt) {
    if (dt != DASH_BF16) return false;
    if (G.d != 64 && G.d != 128) return false;
    if (G.g & (G.g - 1)) return false;  // tile_rows * g must be exactly 128
    if (G.tile_rows * G.g != kRows) return false;
    if (G.nq > 0x7fffffff || G.nk > 0x7fffffff) return false;
    return tma_encode_fn() != nullptr;
}

cudaError_t launch_attn_tc(const TView &Q, const TView &K, const TView &V, const TView &O, const Geom &G,
                           const ListsView &L, int flags, cudaStream_t st, float *lse) {
    if (G.nq == 0 || G.b == 0) return cudaSuccess;
    TcParams tp;
    if (!make_map_bf16(&tp.tmQ, Q, G.b, G.nq, G.hq, G.d, G.g, G.tile_rows)) return cudaErrorInvalidValue;
    const int box = G.B < kStepKeys ? G.B : kStepKeys;  // rows of one K / V box: a chunk or half of one
    if (!make_map_bf16(&tp.tmK, K, G.b, G.nk, G.hkv, G.d, 1, box)) return cudaErrorInvalidValue;
    if (!make_map_bf16(&tp.tmV, V, G.b, G.nk, G.hkv, G.d, 1, box)) return cudaErrorInvalidValue;
#define DASH_TC_CASE(DD, BB) \
    if (G.d == DD && G.B == BB) return launch_t<DD, BB>(tp, Q, O, G, L, flags, st, lse);
    DASH_TC_CASE(128, 64)
    DASH_TC_CASE(128, 128)
    DASH_TC_CASE(128, 32)
    DASH_TC_CASE(128, 16)
    DASH_TC_CASE(64, 64)
    DASH_TC_CASE(64, 128)
    DASH_TC_CASE(64, 32)
    DASH_TC_CASE(64, 16)
#undef DASH_TC_CASE
    return cudaErrorNotSupported;
}

int take_device_error_tc() { return take_device_error_local(); }

}  // namespace dash

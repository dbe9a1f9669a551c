// attn_bwd_tc.cu -- Stage-2 backward on the 5th-generation tensor cores (tcgen05 + TMEM +
// TMA), bf16, head dim 128, chunks of 64 or 128 keys, g a power of two.
//
// The gradient of the prior-biased softmax attention of "DashAttention" §3.4 Prop. 1
// (the bias form of Eq. 7), per row i of head h with lse_i from the forward:
//   P_ij = exp(z_ij + b_ij - lse_i),  dP_ij = <dO_i, v_j>,  dl_ij = P_ij (dP_ij - D_i),
//   dq_i = sum_j dl_ij k_j / sqrt(d),  dk_j = sum_i dl_ij q_i / sqrt(d),  dv_j = sum_i P_ij dO_i,
// and G_c(i) = sum over the group's heads and chunk c's keys of dl_ij for every routed
// chunk (the prior's gradient, taken on by the routing chain in bwd.cu).
//
// bwd_tc_prep_kernel   copies each tile's Q and dO rows (the lists' row order) into
//                      contiguous bf16 tiles, with lse (exp2 domain) and D = <dO, O> (formed
//                      from the same rows) beside them, so that both kernels below load
//                      whole tiles with TMA.
// bwd_dq_tc_kernel     one CTA per (batch, kv head, query tile), the latest tiles first
//                      within groups of heads whose K and V fit in L2 together.  Warp 0 loads the tile once and K, V per 64-key step
//                      (three-stage rings); warp 1 (one thread) issues
//                        S_j = Q K_j^T and dP_j = dO V_j^T (SS, M = 128, N = 64) into
//                        double-buffered TMEM, then dQ += dl_j K_j (TS: dl from TMEM);
//                      warps 2-5 (thread = TMEM lane = tile row) form P and dl, write dl as
//                      bf16 over S_j and sum G per list entry and position.
// bwd_dkdv_tc_kernel   one CTA per (64-key block, kv head, batch) over the (tile, entry)
//                      pairs that attend the block (the transposed lists, tiles
//                      ascending).  K and V load once; each pair brings its Q and dO tiles
//                      (two-stage ring).  S = Q K^T and dP = dO V^T as above; the compute
//                      warps write P and dl as bf16 into shared memory (row m = the
//                      128-byte swizzled row of tile row m), and the MMA thread accumulates
//                        dV^T += dO^T P  and  dK^T += Q^T dl   (SS, both operands MN-major,
//                        M = d = 128, N = 64 keys, K = 128 tile rows)
//                      in TMEM.  A block's pairs are split among up to 8 CTAs (a block
//                      many tiles attend would otherwise be one long serial chain); each
//                      adds its share to fp32 accumulators, and bwd_kv_finish_kernel
//                      adds the chunk summary's share to dK and writes dK, dV in bf16.
// Every wait is bounded (globaltimer); on expiry a kernel records a device error, drains
// what it issued, frees TMEM and returns.
#include <math.h>

#include <algorithm>

#include "dash_common.cuh"
#include "kernels.h"
#include "tma_host.h"

namespace dash {

namespace {

constexpr int kThreads = 192;
constexpr int kTileRows = 128;
constexpr int kStepKeys = 64;
constexpr int kD = 128;
constexpr int kRegion = kTileRows * 128;  // 128 rows x 128 B: 64 columns of a tile
constexpr int kKRegion = kStepKeys * 128; // 64 keys x 128 B
constexpr uint64_t kWaitNs = 2000000000ull;
constexpr float kLog2e = 1.4426950408889634f;

struct BwdMaps {
    CUtensorMap tmQp, tmdOp, tmK, tmV;
};

constexpr int kPrefetch = 4;  // pairs ahead whose Q and dO tiles the key-side producer prefetches into L2

// Start bringing `bytes` (a multiple of 16) at a 16-byte aligned global address into L2.
__device__ __forceinline__ void l2_prefetch(const void *p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(reinterpret_cast<uint64_t>(p)), "r"(bytes)
                 : "memory");
}

// ------------------------------------------------------------------ prep
__global__ void __launch_bounds__(kTileRows) bwd_tc_prep_kernel(TView Q, TView dO, TView O, Geom G, ListsView L,
                                                               const float *__restrict__ lse, uint4 *__restrict__ Qp,
                                                               uint4 *__restrict__ dOp, float *__restrict__ Lp,
                                                               float *__restrict__ Dp) {
    const int64_t t = blockIdx.x;
    const int r = blockIdx.y;
    const int64_t b = blockIdx.z;
    const int g = G.g;
    const size_t tile_lin = ((size_t)b * G.hkv + r) * L.n_tiles + t;
    // 16 threads per row, each one 16-byte piece: 8 rows (2 KB contiguous each way) per pass;
    // D = <dO, O> of the row from the same pieces (a sum over the row's 16 threads)
    const int piece = threadIdx.x % 16;
    for (int m = threadIdx.x / 16; m < kTileRows; m += kTileRows / 16) {
        const int64_t i = tile_row(L, G, tile_lin, t, m / g);
        const int h = r * g + m % g;
        const size_t row = tile_lin * kTileRows + m;
        const int64_t ii = i >= 0 ? i : 0;
        const uint4 *qs = reinterpret_cast<const uint4 *>(reinterpret_cast<const __nv_bfloat16 *>(Q.p) + b * Q.s0 +
                                                          ii * Q.s1 + (int64_t)h * Q.s2);
        const uint4 *gs = reinterpret_cast<const uint4 *>(reinterpret_cast<const __nv_bfloat16 *>(dO.p) + b * dO.s0 +
                                                          ii * dO.s1 + (int64_t)h * dO.s2);
        const uint4 *os = reinterpret_cast<const uint4 *>(reinterpret_cast<const __nv_bfloat16 *>(O.p) + b * O.s0 +
                                                          ii * O.s1 + (int64_t)h * O.s2);
        const uint4 gv = i >= 0 ? gs[piece] : make_uint4(0u, 0u, 0u, 0u);
        const uint4 ov = i >= 0 ? os[piece] : make_uint4(0u, 0u, 0u, 0u);
        Qp[row * (kD / 8) + piece] = i >= 0 ? qs[piece] : make_uint4(0u, 0u, 0u, 0u);
        dOp[row * (kD / 8) + piece] = gv;
        const __nv_bfloat162 *g2 = reinterpret_cast<const __nv_bfloat162 *>(&gv);
        const __nv_bfloat162 *o2 = reinterpret_cast<const __nv_bfloat162 *>(&ov);
        float dsum = 0.f;
#pragma unroll
        for (int x = 0; x < 4; ++x) {
            const float2 a2 = __bfloat1622float2(g2[x]), c2 = __bfloat1622float2(o2[x]);
            dsum = fmaf(a2.x, c2.x, fmaf(a2.y, c2.y, dsum));
        }
#pragma unroll
        for (int o = 8; o >= 1; o >>= 1) dsum += __shfl_xor_sync(0xffffffffu, dsum, o);
        if (piece == 0) Dp[row] = dsum;
    }
    const int m = threadIdx.x;
    const int64_t i = tile_row(L, G, tile_lin, t, m / g);
    const size_t row = tile_lin * kTileRows + m;
    const size_t rid = ((size_t)b * G.nq + (i >= 0 ? i : 0)) * G.hq + r * g + m % g;
    Lp[row] = i >= 0 ? lse[rid] * kLog2e : INFINITY;
}

// ------------------------------------------------------------------ dQ (query side)
template <int BLK>
struct DqSmem {
    static constexpr int kNS = 3;  // K / V stages (K is held until dQ_j has read it)
    static constexpr int kNM = 2;  // bias stages
    static constexpr int kSub = BLK / kStepKeys;
    static constexpr int kQ = 0;                          // 2 regions
    static constexpr int kdO = kQ + 2 * kRegion;          // 2 regions
    static constexpr int kK = kdO + 2 * kRegion;          // [kNS][2 regions of 64 keys]
    static constexpr int kV = kK + kNS * 2 * kKRegion;
    static constexpr int kBias = kV + kNS * 2 * kKRegion;  // [kNM][128] floats
    static constexpr int kL = kBias + kNM * 128 * 4;       // [128] lse (exp2 domain)
    static constexpr int kDv = kL + 128 * 4;               // [128] D
    static constexpr int kIds = kDv + 128 * 4;             // [kNM] chunk ids
    static constexpr int kBars = (kIds + kNM * 4 + 7) & ~7;
    // q_full, k_full[NS], k_empty[NS], v_full[NS], v_empty[NS], m_full[NM], m_empty[NM],
    // s_full[2], ds_full[2], dq_done[2], fin
    static constexpr int kNumBars = 1 + 4 * kNS + 2 * kNM + 6 + 1;
    static constexpr int kMisc = kBars + kNumBars * 8;
    static constexpr int kTotal = kMisc + 16 + 8;
};

template <int BLK>
__global__ void __launch_bounds__(kThreads, 1) bwd_dq_tc_kernel(const __grid_constant__ BwdMaps mp, Geom G,
                                                                ListsView L, const float *__restrict__ Lp,
                                                                const float *__restrict__ Dp,
                                                                float *__restrict__ dQacc, float *__restrict__ Gd,
                                                                int hg) {
    using S = DqSmem<BLK>;
    constexpr int kNS = S::kNS, kNM = S::kNM, kSub = S::kSub;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    // groups of heads whose K and V share L2, the latest (longest) tiles of a group first
    const TileOrder to = tile_order(blockIdx.x, L.n_tiles, G.b * G.hkv, hg);
    const int64_t t = to.t;
    const int r = (int)(to.bh % G.hkv);
    const int64_t b = to.bh / G.hkv;
    const int g = G.g, T = L.tile_rows;
    const size_t tile_lin = ((size_t)b * G.hkv + r) * L.n_tiles + t;
    const int count = L.count[tile_lin];
    const int nsteps = count * kSub;

    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + S::kBars);
    uint64_t *q_full = bars, *k_full = q_full + 1, *k_empty = k_full + kNS, *v_full = k_empty + kNS,
             *v_empty = v_full + kNS, *m_full = v_empty + kNS, *m_empty = m_full + kNM, *s_full = m_empty + kNM,
             *ds_full = s_full + 2, *dq_done = ds_full + 2, *fin = dq_done + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + S::kMisc);
    volatile int *abort = reinterpret_cast<volatile int *>(sm + S::kMisc + 4);
    long long *p_min_s = reinterpret_cast<long long *>(sm + S::kMisc + 8);
    float *bias_s = reinterpret_cast<float *>(sm + S::kBias);
    int *ids_s = reinterpret_cast<int *>(sm + S::kIds);

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int s = 0; s < kNS; ++s) {
            mbar_init(k_full + s, 1);
            mbar_init(k_empty + s, 1);
            mbar_init(v_full + s, 1);
            mbar_init(v_empty + s, 1);
        }
        for (int s = 0; s < kNM; ++s) {
            mbar_init(m_full + s, 1);
            mbar_init(m_empty + s, 128);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(s_full + s, 1);
            mbar_init(ds_full + s, 128);
            mbar_init(dq_done + s, 1);
        }
        mbar_init(fin, 1);
        *abort = 0;
        *p_min_s = 0x7fffffffffffffffll;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // S_j in columns (j & 1) * 64, dP_j at 128 + (j & 1) * 64, dQ at 256
    const uint32_t tdQ = tmem + 256;

    if (warp == 0) {
        if (lane == 0 && nsteps > 0) {
            tma_prefetch_desc(&mp.tmK);
            tma_prefetch_desc(&mp.tmV);
            mbar_arrive_expect_tx(q_full, 4 * kRegion + 2 * 128 * 4);
            for (int dh = 0; dh < 2; ++dh) {
                tma_load_4d(sm + S::kQ + dh * kRegion, &mp.tmQp, q_full, dh * 64, 0, (int)(tile_lin * kTileRows), 0);
                tma_load_4d(sm + S::kdO + dh * kRegion, &mp.tmdOp, q_full, dh * 64, 0, (int)(tile_lin * kTileRows),
                            0);
            }
            bulk_load(sm + S::kL, Lp + tile_lin * kTileRows, 512, q_full);
            bulk_load(sm + S::kDv, Dp + tile_lin * kTileRows, 512, q_full);
            const int32_t *ids_g = L.ids + tile_lin * L.cap;
            const float *bias_g = L.bias + tile_lin * (size_t)L.cap * T;
            int issued_k = 0, issued_v = 0, issued_m = 0;
            for (int j = 0; j < nsteps; ++j) {
                const int e = j / kSub, koff = (j % kSub) * kStepKeys;
                const int ms = j % kNM, ks = j % kNS;
                if (!wait_bar(m_empty + ms, ((j / kNM) & 1) ^ 1, kWaitNs, abort)) break;
                const int id = ids_g[e];
                ids_s[ms] = id;
                mbar_arrive_expect_tx(m_full + ms, (uint32_t)(T * 4));
                bulk_load(bias_s + ms * 128, bias_g + (size_t)e * T, (uint32_t)(T * 4), m_full + ms);
                issued_m = j + 1;
                if (!wait_bar(k_empty + ks, ((j / kNS) & 1) ^ 1, kWaitNs, abort)) break;
                mbar_arrive_expect_tx(k_full + ks, 2 * kKRegion);
                for (int dh = 0; dh < 2; ++dh)
                    tma_load_4d(sm + S::kK + (ks * 2 + dh) * kKRegion, &mp.tmK, k_full + ks, dh * 64, r,
                                id * BLK + koff, (int)b);
                issued_k = j + 1;
                if (!wait_bar(v_empty + ks, ((j / kNS) & 1) ^ 1, kWaitNs, abort)) break;
                mbar_arrive_expect_tx(v_full + ks, 2 * kKRegion);
                for (int dh = 0; dh < 2; ++dh)
                    tma_load_4d(sm + S::kV + (ks * 2 + dh) * kKRegion, &mp.tmV, v_full + ks, dh * 64, r,
                                id * BLK + koff, (int)b);
                issued_v = j + 1;
            }
            if (*abort) {  // every copy issued lands before the CTA's shared memory goes away
                for (int j = max(0, issued_k - kNS); j < issued_k; ++j)
                    wait_bar(k_full + j % kNS, (j / kNS) & 1, kWaitNs, abort, false);
                for (int j = max(0, issued_v - kNS); j < issued_v; ++j)
                    wait_bar(v_full + j % kNS, (j / kNS) & 1, kWaitNs, abort, false);
                for (int j = max(0, issued_m - kNM); j < issued_m; ++j)
                    wait_bar(m_full + j % kNM, (j / kNM) & 1, kWaitNs, abort, false);
                wait_bar(q_full, 0, kWaitNs, abort, false);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idS = idesc_bf16_f32(kTileRows, kStepKeys, 0, 0);
            constexpr uint32_t idDQ = idesc_bf16_f32(kTileRows, kD, 0, 1);
            const uint32_t q_base = smem_u32(sm + S::kQ), do_base = smem_u32(sm + S::kdO);
            const uint32_t k_base = smem_u32(sm + S::kK), v_base = smem_u32(sm + S::kV);
            bool ok = nsteps == 0 || wait_bar(q_full, 0, kWaitNs, abort);
            auto issue_sdp = [&](int j) -> bool {
                const int ks = j % kNS;
                if (j >= 2 && !wait_bar(dq_done + (j & 1), ((j - 2) >> 1) & 1, kWaitNs, abort)) return false;
                if (!wait_bar(k_full + ks, (j / kNS) & 1, kWaitNs, abort)) return false;
                tc_fence_after();
                const uint32_t tS = tmem + (uint32_t)((j & 1) * kStepKeys);
#pragma unroll
                for (int kk = 0; kk < kD / 16; ++kk) {
                    const uint32_t qa = q_base + (kk / 4) * kRegion + (kk % 4) * 32;
                    const uint32_t kb = k_base + (ks * 2 + kk / 4) * kKRegion + (kk % 4) * 32;
                    mma_ss(tS, smem_desc_sw128(qa, 16, 1024), smem_desc_sw128(kb, 16, 1024), idS, kk > 0 ? 1u : 0u);
                }
                if (!wait_bar(v_full + ks, (j / kNS) & 1, kWaitNs, abort)) return false;
                tc_fence_after();
                const uint32_t tP = tmem + 128 + (uint32_t)((j & 1) * kStepKeys);
#pragma unroll
                for (int kk = 0; kk < kD / 16; ++kk) {
                    const uint32_t da = do_base + (kk / 4) * kRegion + (kk % 4) * 32;
                    const uint32_t vb = v_base + (ks * 2 + kk / 4) * kKRegion + (kk % 4) * 32;
                    mma_ss(tP, smem_desc_sw128(da, 16, 1024), smem_desc_sw128(vb, 16, 1024), idS, kk > 0 ? 1u : 0u);
                }
                mma_commit(s_full + (j & 1));
                mma_commit(v_empty + ks);
                return true;
            };
            for (int j = 0; ok && j < min(nsteps, 2); ++j) ok = issue_sdp(j);
            for (int j = 0; ok && j < nsteps; ++j) {
                const int ks = j % kNS;
                if (!(ok = wait_bar(ds_full + (j & 1), (j >> 1) & 1, kWaitNs, abort))) break;
                tc_fence_after();
                const uint32_t tS = tmem + (uint32_t)((j & 1) * kStepKeys);
#pragma unroll
                for (int kk = 0; kk < kStepKeys / 16; ++kk) {
                    const uint32_t kb = k_base + (ks * 2) * kKRegion + kk * 2048;
                    mma_ts(tdQ, tS + kk * 8, smem_desc_sw128(kb, kKRegion, 1024), idDQ, (j > 0 || kk > 0) ? 1u : 0u);
                }
                mma_commit(k_empty + ks);
                mma_commit(dq_done + (j & 1));
                if (j + 2 < nsteps) ok = issue_sdp(j + 2);
            }
            mma_commit(fin);
            wait_bar(fin, 0, kWaitNs, abort, false);
        }
    } else {
        const int quad = warp & 3;
        const int m = quad * 32 + lane;
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        const int pos = m / g, hh = m % g;
        const int64_t i = tile_row(L, G, tile_lin, t, pos);
        const bool row_ok = i >= 0;
        const int64_t p_row = row_pos(G, i);
        if (row_ok) atomicMin(p_min_s, (long long)p_row);
        asm volatile("bar.sync 1, 128;" ::: "memory");
        const int64_t p_min = *p_min_s;
        const float sl2 = rsqrtf((float)kD) * kLog2e;
        bool ok = nsteps == 0 || __all_sync(0xffffffffu, wait_bar(q_full, 0, kWaitNs, abort));
        const float L2 = reinterpret_cast<const float *>(sm + S::kL)[m];
        const float Dv = reinterpret_cast<const float *>(sm + S::kDv)[m];
        const int vis_end = (int)((G.causal && row_ok) ? min((int64_t)G.nk, p_row + 1) : G.nk);
        float gacc = 0.f;
        for (int j = 0; ok && j < nsteps; ++j) {
            const int ms = j % kNM, koff = (j % kSub) * kStepKeys;
            if (!(ok = __all_sync(0xffffffffu, wait_bar(m_full + ms, (j / kNM) & 1, kWaitNs, abort)))) break;
            const int id = ids_s[ms];
            const float bv = bias_s[ms * 128 + pos];
            const int k0 = id * BLK + koff;
            const int lim = max(0, min(kStepKeys, vis_end - k0));
            const int64_t last_key = (int64_t)k0 + kStepKeys - 1;
            const bool need_mask = last_key >= G.nk || (G.causal && last_key > p_min);
            mbar_arrive(m_empty + ms);
            const float c0 = (row_ok && bv > -INFINITY) ? bv * kLog2e - L2 : -INFINITY;
            if (!(ok = __all_sync(0xffffffffu, wait_bar(s_full + (j & 1), (j >> 1) & 1, kWaitNs, abort)))) break;
            tc_fence_after();
            const uint32_t tS = tmem + (uint32_t)((j & 1) * kStepKeys) + lane_off;
            const uint32_t tP = tmem + 128 + (uint32_t)((j & 1) * kStepKeys) + lane_off;
#pragma unroll
            for (int qc = 0; qc < 2; ++qc) {
                uint32_t su[32], pu[32], pk[16];
                tmem_ld32(tS + qc * 32, su);
                tmem_ld32(tP + qc * 32, pu);
#pragma unroll
                for (int x = 0; x < 16; ++x) {
                    const int kc = qc * 32 + 2 * x;
                    float v0 = fmaf(__uint_as_float(su[2 * x]), sl2, c0);
                    float v1 = fmaf(__uint_as_float(su[2 * x + 1]), sl2, c0);
                    if (need_mask) {  // select before exp2: S past the row's keys may be anything
                        v0 = kc < lim ? v0 : -INFINITY;
                        v1 = kc + 1 < lim ? v1 : -INFINITY;
                    }
                    const float p0 = ex2(v0), p1 = ex2(v1);
                    const float d0 = p0 * (__uint_as_float(pu[2 * x]) - Dv);
                    const float d1 = p1 * (__uint_as_float(pu[2 * x + 1]) - Dv);
                    gacc += d0 + d1;
                    pk[x] = pack_bf16x2(d0, d1);
                }
                // dl of keys 32qc.. over columns 16qc..: S columns below 32(qc+1) are already read
                tmem_st16(tS + qc * 16, pk);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(ds_full + (j & 1));
            if (j % kSub == kSub - 1) {
                // G of this chunk for the row's position: the sum over its g heads (lanes)
                float gs = gacc;
                for (int o = 1; o < g; o <<= 1) gs += __shfl_xor_sync(0xffffffffu, gs, o);
                if (row_ok && hh == 0 && bv > -INFINITY && id < row_nvis(G, i)) Gd[logw_index(G, b, r, i, id)] = gs;
                gacc = 0.f;
            }
        }
        // epilogue: dQ / sqrt(d) into the fp32 accumulator of the row
        if (ok && !*abort) {
            bool have = true;
            if (nsteps > 0)
                have = __all_sync(0xffffffffu, wait_bar(dq_done + ((nsteps - 1) & 1), ((nsteps - 1) >> 1) & 1, kWaitNs,
                                                        abort));
            tc_fence_after();
            if (have) {
                const float sc = rsqrtf((float)kD);
                float4 *dst = reinterpret_cast<float4 *>(dQacc + (((size_t)b * G.nq + (row_ok ? i : 0)) * G.hq +
                                                                  r * g + hh) * kD);
#pragma unroll
                for (int c = 0; c < kD / 32; ++c) {
                    uint32_t u[32];
                    if (nsteps > 0) {
                        tmem_ld32(tdQ + lane_off + c * 32, u);
                    } else {
#pragma unroll
                        for (int x = 0; x < 32; ++x) u[x] = 0u;
                    }
                    if (row_ok) {
#pragma unroll
                        for (int x = 0; x < 8; ++x)
                            dst[c * 8 + x] = make_float4(__uint_as_float(u[4 * x]) * sc, __uint_as_float(u[4 * x + 1]) * sc,
                                                         __uint_as_float(u[4 * x + 2]) * sc,
                                                         __uint_as_float(u[4 * x + 3]) * sc);
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ------------------------------------------------------------------ dK, dV (key side)
struct KvSmem {
    static constexpr int kNQ = 2;                          // Q / dO tile stages
    static constexpr int kQ = 0;                           // [kNQ][2 regions]
    static constexpr int kdO = kQ + kNQ * 2 * kRegion;     // [kNQ][2 regions]
    static constexpr int kK = kdO + kNQ * 2 * kRegion;     // 2 regions of 64 keys
    static constexpr int kV = kK + 2 * kKRegion;
    static constexpr int kP = kV + 2 * kKRegion;           // 128 rows x 128 B (P, bf16)
    static constexpr int kdS = kP + kRegion;               // 128 rows x 128 B (dl, bf16)
    static constexpr int kMeta = kdS + kRegion;            // [kNQ][bias 128 | L 128 | D 128 | rows 128 | tile]
    static constexpr int kMetaStage = 4 * 128 * 4 + 16;
    static constexpr int kBars = kMeta + kNQ * kMetaStage;
    // kv_full, q_full[NQ], q_empty[NQ], s_full[2], p_full, p_empty, fin
    static constexpr int kNumBars = 1 + 2 * kNQ + 2 + 3;
    static constexpr int kMisc = kBars + kNumBars * 8;
    static constexpr int kTotal = kMisc + 16;
};

template <int BLK>
__global__ void __launch_bounds__(kThreads, 1) bwd_dkdv_tc_kernel(const __grid_constant__ BwdMaps mp, Geom G,
                                                                  ListsView L, const float *__restrict__ Lp,
                                                                  const float *__restrict__ Dp,
                                                                  const int32_t *__restrict__ ref_off,
                                                                  const int32_t *__restrict__ ref_cnt,
                                                                  const int2 *__restrict__ refs,
                                                                  float *__restrict__ dKacc, float *__restrict__ dVacc,
                                                                  const __nv_bfloat16 *__restrict__ Qp_g,
                                                                  const __nv_bfloat16 *__restrict__ dOp_g,
                                                                  int nsplit) {
    using S = KvSmem;
    constexpr int kNQ = S::kNQ;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    // CTA (key block kb, split): the block's (tile, entry) pairs split, j, j + nsplit, ...,
    // among nsplit CTAs, so that a block many tiles attend is not one long serial chain
    const int kb = blockIdx.x / nsplit, split = blockIdx.x % nsplit, r = blockIdx.y;
    const int64_t b = blockIdx.z;
    const int g = G.g, T = L.tile_rows;
    const int c = (int)((int64_t)kb * kStepKeys / BLK);   // the list entry (chunk / block id) of these keys
    const int64_t key0 = (int64_t)kb * kStepKeys;
    const size_t bh = (size_t)b * G.hkv + r;
    const int nref_all = ref_cnt[bh * G.n_blk + c];
    const int nref = nref_all > split ? (nref_all - split + nsplit - 1) / nsplit : 0;
    const int2 *rl_all = refs + bh * (size_t)L.n_tiles * G.n_blk + ref_off[bh * G.n_blk + c];
    auto ref_at = [&](int j) -> int2 { return rl_all[split + (int64_t)j * nsplit]; };
    if (nref == 0) return;  // nothing to add (the accumulators start at zero)

    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + S::kBars);
    uint64_t *kv_full = bars, *q_full = kv_full + 1, *q_empty = q_full + kNQ, *s_full = q_empty + kNQ,
             *p_full = s_full + 2, *p_empty = p_full + 1, *fin = p_empty + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + S::kMisc);
    volatile int *abort = reinterpret_cast<volatile int *>(sm + S::kMisc + 4);

    if (threadIdx.x == 0) {
        mbar_init(kv_full, 1);
        for (int s = 0; s < kNQ; ++s) {
            mbar_init(q_full + s, 1);
            mbar_init(q_empty + s, 1);
        }
        mbar_init(s_full, 1);
        mbar_init(s_full + 1, 1);
        mbar_init(p_full, 128);
        mbar_init(p_empty, 1);
        mbar_init(fin, 1);
        *abort = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // S_j at (j & 1) * 64, dP_j at 128 + (j & 1) * 64, dV^T at 256, dK^T at 320 (lane = dimension)
    const uint32_t tdV = tmem + 256, tdK = tmem + 320;

    if (warp == 0) {
        if (lane == 0 && nref > 0) {
            mbar_arrive_expect_tx(kv_full, 4 * kKRegion);
            for (int dh = 0; dh < 2; ++dh) {
                tma_load_4d(sm + S::kK + dh * kKRegion, &mp.tmK, kv_full, dh * 64, r, (int)key0, (int)b);
                tma_load_4d(sm + S::kV + dh * kKRegion, &mp.tmV, kv_full, dh * 64, r, (int)key0, (int)b);
            }
            for (int j = 0; j < min(nref, kPrefetch); ++j) {
                const size_t tl = bh * L.n_tiles + ref_at(j).x;
                l2_prefetch(Qp_g + tl * kTileRows * kD, kTileRows * kD * 2);
                l2_prefetch(dOp_g + tl * kTileRows * kD, kTileRows * kD * 2);
            }
            int issued = 0;
            for (int j = 0; j < nref; ++j) {
                const int st = j % kNQ;
                if (!wait_bar(q_empty + st, ((j / kNQ) & 1) ^ 1, kWaitNs, abort)) break;
                const int2 ref = ref_at(j);
                const int64_t t = ref.x;
                const int e = ref.y;
                const size_t tile_lin = bh * L.n_tiles + t;
                uint8_t *meta = sm + S::kMeta + st * S::kMetaStage;
                // the tile index for the compute warps (published by the arrive below)
                *reinterpret_cast<long long *>(meta + 2048) = (long long)t;
                const uint32_t bytes = 4 * kRegion + (uint32_t)(T * 4) + 1024 + (L.rows ? (uint32_t)(T * 4) : 0u);
                mbar_arrive_expect_tx(q_full + st, bytes);
                for (int dh = 0; dh < 2; ++dh) {
                    tma_load_4d(sm + S::kQ + (st * 2 + dh) * kRegion, &mp.tmQp, q_full + st, dh * 64, 0,
                                (int)(tile_lin * kTileRows), 0);
                    tma_load_4d(sm + S::kdO + (st * 2 + dh) * kRegion, &mp.tmdOp, q_full + st, dh * 64, 0,
                                (int)(tile_lin * kTileRows), 0);
                }
                bulk_load(meta, L.bias + tile_lin * (size_t)L.cap * T + (size_t)e * T, (uint32_t)(T * 4), q_full + st);
                bulk_load(meta + 512, Lp + tile_lin * kTileRows, 512, q_full + st);
                bulk_load(meta + 1024, Dp + tile_lin * kTileRows, 512, q_full + st);
                if (L.rows) bulk_load(meta + 1536, L.rows + tile_lin * T, (uint32_t)(T * 4), q_full + st);
                issued = j + 1;
                // the tiles of the pair kPrefetch ahead start their way into L2 now, so that
                // the two-stage ring finds them there
                if (j + kPrefetch < nref) {
                    const size_t tl = bh * L.n_tiles + ref_at(j + kPrefetch).x;
                    l2_prefetch(Qp_g + tl * kTileRows * kD, kTileRows * kD * 2);
                    l2_prefetch(dOp_g + tl * kTileRows * kD, kTileRows * kD * 2);
                }
            }
            if (*abort) {
                for (int j = max(0, issued - kNQ); j < issued; ++j)
                    wait_bar(q_full + j % kNQ, (j / kNQ) & 1, kWaitNs, abort, false);
                wait_bar(kv_full, 0, kWaitNs, abort, false);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idS = idesc_bf16_f32(kTileRows, kStepKeys, 0, 0);
            constexpr uint32_t idT = idesc_bf16_f32(kD, kStepKeys, 1, 1);
            const uint32_t k_base = smem_u32(sm + S::kK), v_base = smem_u32(sm + S::kV);
            const uint32_t p_base = smem_u32(sm + S::kP), ds_base = smem_u32(sm + S::kdS);
            bool ok = nref == 0 || wait_bar(kv_full, 0, kWaitNs, abort);
            auto issue_sdp = [&](int j) -> bool {
                const int st = j % kNQ;
                if (!wait_bar(q_full + st, (j / kNQ) & 1, kWaitNs, abort)) return false;
                tc_fence_after();
                const uint32_t q_base = smem_u32(sm + S::kQ + st * 2 * kRegion);
                const uint32_t do_base = smem_u32(sm + S::kdO + st * 2 * kRegion);
                const uint32_t tS = tmem + (uint32_t)((j & 1) * kStepKeys);
                const uint32_t tP = tmem + 128 + (uint32_t)((j & 1) * kStepKeys);
#pragma unroll
                for (int kk = 0; kk < kD / 16; ++kk) {
                    const uint32_t off = (kk / 4) * kRegion + (kk % 4) * 32;
                    const uint32_t koff = (kk / 4) * kKRegion + (kk % 4) * 32;
                    mma_ss(tS, smem_desc_sw128(q_base + off, 16, 1024), smem_desc_sw128(k_base + koff, 16, 1024), idS,
                           kk > 0 ? 1u : 0u);
                }
#pragma unroll
                for (int kk = 0; kk < kD / 16; ++kk) {
                    const uint32_t off = (kk / 4) * kRegion + (kk % 4) * 32;
                    const uint32_t koff = (kk / 4) * kKRegion + (kk % 4) * 32;
                    mma_ss(tP, smem_desc_sw128(do_base + off, 16, 1024), smem_desc_sw128(v_base + koff, 16, 1024),
                           idS, kk > 0 ? 1u : 0u);
                }
                mma_commit(s_full + (j & 1));
                return true;
            };
            // dV^T += dO^T P, dK^T += Q^T dl of pair j over the tile's 128 rows (K steps of 16 rows)
            auto issue_pv = [&](int j) {
                const int st = j % kNQ;
                tc_fence_after();
                const uint32_t q_base = smem_u32(sm + S::kQ + st * 2 * kRegion);
                const uint32_t do_base = smem_u32(sm + S::kdO + st * 2 * kRegion);
#pragma unroll
                for (int kk = 0; kk < kTileRows / 16; ++kk) {
                    mma_ss(tdV, smem_desc_sw128(do_base + kk * 2048, kRegion, 1024),
                           smem_desc_sw128(p_base + kk * 2048, kRegion, 1024), idT, (j > 0 || kk > 0) ? 1u : 0u);
                    mma_ss(tdK, smem_desc_sw128(q_base + kk * 2048, kRegion, 1024),
                           smem_desc_sw128(ds_base + kk * 2048, kRegion, 1024), idT, (j > 0 || kk > 0) ? 1u : 0u);
                }
                mma_commit(p_empty);
                mma_commit(q_empty + st);
            };
            for (int j = 0; ok && j < min(nref, 2); ++j) ok = issue_sdp(j);
            // Whichever product is ready goes first: S, dP of pair next_sdp once its Q / dO
            // stage has landed (and pv of pair next_sdp - 2, the last reader of its TMEM
            // buffers' previous contents, has been issued), or dV, dK of pair next_pv once the
            // softmax warps have written its P and dl.  Waiting on the next pair's tiles no
            // longer holds back the products of a pair that is ready.
            int next_sdp = min(nref, 2), next_pv = 0;
            uint64_t t_last = gtimer();
            while (ok && next_pv < nref) {
                if (next_sdp < nref && next_sdp - 2 < next_pv &&
                    mbar_try_wait(q_full + next_sdp % kNQ, (next_sdp / kNQ) & 1)) {
                    ok = issue_sdp(next_sdp++);
                    t_last = gtimer();
                } else if (next_pv < next_sdp && mbar_try_wait(p_full, next_pv & 1)) {
                    issue_pv(next_pv++);
                    t_last = gtimer();
                } else if (gtimer() - t_last > kWaitNs) {
                    report_timeout();
                    *abort = 1;
                    ok = false;
                } else if (*abort) {
                    ok = false;
                } else {
                    __nanosleep(64);
                }
            }
            mma_commit(fin);
            wait_bar(fin, 0, kWaitNs, abort, false);
        }
    } else {
        const int quad = warp & 3;
        const int m = quad * 32 + lane;  // tile row (S / dP lane), and in the epilogue the dimension
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        const int pos = m / g;
        const float sl2 = rsqrtf((float)kD) * kLog2e;
        uint8_t *prow = sm + S::kP + m * 128;
        uint8_t *drow = sm + S::kdS + m * 128;
        bool ok = true;
        for (int j = 0; j < nref; ++j) {
            const int st = j % kNQ;
            if (!(ok = __all_sync(0xffffffffu, wait_bar(q_full + st, (j / kNQ) & 1, kWaitNs, abort)))) break;
            const uint8_t *meta = sm + S::kMeta + st * S::kMetaStage;
            const float bv = reinterpret_cast<const float *>(meta)[pos];
            const float L2 = reinterpret_cast<const float *>(meta + 512)[m];
            const float Dv = reinterpret_cast<const float *>(meta + 1024)[m];
            const int64_t t = *reinterpret_cast<const long long *>(meta + 2048);
            const int64_t i = L.rows ? (int64_t)reinterpret_cast<const int32_t *>(meta + 1536)[pos]
                                     : (t * T + pos < G.nq ? t * T + pos : -1);
            const bool live = i >= 0 && bv > -INFINITY;
            const int64_t vis_end = (G.causal && i >= 0) ? min((int64_t)G.nk, row_pos(G, i) + 1) : G.nk;
            const int lim = (int)max((int64_t)0, min((int64_t)kStepKeys, vis_end - key0));
            const float c0 = live ? bv * kLog2e - L2 : -INFINITY;
            if (!(ok = __all_sync(0xffffffffu, wait_bar(s_full + (j & 1), (j >> 1) & 1, kWaitNs, abort)))) break;
            tc_fence_after();
            const uint32_t tS = tmem + (uint32_t)((j & 1) * kStepKeys) + lane_off;
            const uint32_t tP = tmem + 128 + (uint32_t)((j & 1) * kStepKeys) + lane_off;
            uint32_t pkP[32], pkD[32];
#pragma unroll
            for (int qc = 0; qc < 2; ++qc) {
                uint32_t su[32], pu[32];
                tmem_ld32(tS + qc * 32, su);
                tmem_ld32(tP + qc * 32, pu);
#pragma unroll
                for (int x = 0; x < 16; ++x) {
                    const int kc = qc * 32 + 2 * x;
                    float v0 = fmaf(__uint_as_float(su[2 * x]), sl2, c0);
                    float v1 = fmaf(__uint_as_float(su[2 * x + 1]), sl2, c0);
                    v0 = kc < lim ? v0 : -INFINITY;
                    v1 = kc + 1 < lim ? v1 : -INFINITY;
                    const float p0 = ex2(v0), p1 = ex2(v1);
                    pkP[qc * 16 + x] = pack_bf16x2(p0, p1);
                    pkD[qc * 16 + x] = pack_bf16x2(p0 * (__uint_as_float(pu[2 * x]) - Dv),
                                                   p1 * (__uint_as_float(pu[2 * x + 1]) - Dv));
                }
            }
            tc_fence_before();
            // the previous pair's dV / dK MMAs must be done reading P and dl
            if (j > 0 && !(ok = __all_sync(0xffffffffu, wait_bar(p_empty, (j - 1) & 1, kWaitNs, abort)))) break;
#pragma unroll
            for (int cc = 0; cc < 8; ++cc) {  // 16-byte chunk cc = keys 8cc .. 8cc + 7, 128-byte swizzle
                const int sw = (cc ^ (m & 7)) << 4;
                *reinterpret_cast<uint4 *>(prow + sw) =
                    make_uint4(pkP[4 * cc], pkP[4 * cc + 1], pkP[4 * cc + 2], pkP[4 * cc + 3]);
                *reinterpret_cast<uint4 *>(drow + sw) =
                    make_uint4(pkD[4 * cc], pkD[4 * cc + 1], pkD[4 * cc + 2], pkD[4 * cc + 3]);
            }
            fence_proxy_async_smem();
            mbar_arrive(p_full);
        }
        // epilogue: lane m of dV^T / dK^T holds dimension m of the 64 keys; this CTA's share
        // is added to the fp32 accumulators (consecutive lanes: consecutive addresses)
        if (ok && !*abort) {
            const bool have = __all_sync(0xffffffffu, wait_bar(p_empty, (nref - 1) & 1, kWaitNs, abort));
            tc_fence_after();
            if (have) {
                const float sc = rsqrtf((float)kD);
                float *dka = dKacc + ((size_t)b * G.nk * G.hkv + r) * kD + m;
                float *dva = dVacc + ((size_t)b * G.nk * G.hkv + r) * kD + m;
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    uint32_t dvu[32], dku[32];
                    tmem_ld32(tdV + lane_off + half * 32, dvu);
                    tmem_ld32(tdK + lane_off + half * 32, dku);
#pragma unroll
                    for (int x = 0; x < 32; ++x) {
                        const int64_t key = key0 + half * 32 + x;
                        if (key < G.nk) {
                            atomicAdd(dka + (size_t)key * G.hkv * kD, __uint_as_float(dku[x]) * sc);
                            atomicAdd(dva + (size_t)key * G.hkv * kD, __uint_as_float(dvu[x]));
                        }
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// dK = the Stage-2 part (accumulated over the split CTAs) + the chunk summary's share,
// dV; both in bf16.  One thread per four consecutive dimensions.
__global__ void bwd_kv_finish_kernel(const float4 *__restrict__ dKacc, const float4 *__restrict__ dVacc,
                                     const float *__restrict__ dKbar, Geom G, TView dK, TView dV) {
    const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t n = G.b * G.nk * G.hkv * (int64_t)(kD / 4);
    if (idx >= n) return;
    const int e4 = (int)(idx % (kD / 4));
    const int64_t row = idx / (kD / 4);  // (b, key, kv head)
    const int r = (int)(row % G.hkv);
    const int64_t key = (row / G.hkv) % G.nk, b = row / ((int64_t)G.hkv * G.nk);
    float4 k = dKacc[idx];
    const float4 v = dVacc[idx];
    const int c = (int)(key / G.B);
    if (c < G.n_chunks) {  // keys of a routing chunk share its summary's gradient
        const float inv = 1.f / (float)min((int64_t)G.B, G.nk - (int64_t)c * G.B);
        const float4 kb = reinterpret_cast<const float4 *>(dKbar + (((size_t)b * G.n_chunks + c) * G.hkv + r) * kD)[e4];
        k.x += kb.x * inv;
        k.y += kb.y * inv;
        k.z += kb.z * inv;
        k.w += kb.w * inv;
    }
    __nv_bfloat16 *dkp = reinterpret_cast<__nv_bfloat16 *>(const_cast<void *>(dK.p)) + b * dK.s0 + key * dK.s1 +
                         (int64_t)r * dK.s2 + 4 * e4;
    __nv_bfloat16 *dvp = reinterpret_cast<__nv_bfloat16 *>(const_cast<void *>(dV.p)) + b * dV.s0 + key * dV.s1 +
                         (int64_t)r * dV.s2 + 4 * e4;
    *reinterpret_cast<uint2 *>(dkp) = make_uint2(pack_bf16x2(k.x, k.y), pack_bf16x2(k.z, k.w));
    *reinterpret_cast<uint2 *>(dvp) = make_uint2(pack_bf16x2(v.x, v.y), pack_bf16x2(v.z, v.w));
}

bool make_maps(BwdMaps *mp, const BwdArgs &a) {
    const Geom &G = a.G;
    const int64_t tile_rows_total = G.b * G.hkv * a.L.n_tiles * kTileRows;
    // the tile buffers as [1][rows][1][d] with a box of 128 rows x 64 columns
    const TView qv{a.Qp, tile_rows_total * kD, kD, kD};
    const TView gv{a.dOp, tile_rows_total * kD, kD, kD};
    if (!make_map_bf16(&mp->tmQp, qv, 1, tile_rows_total, 1, kD, 1, kTileRows)) return false;
    if (!make_map_bf16(&mp->tmdOp, gv, 1, tile_rows_total, 1, kD, 1, kTileRows)) return false;
    if (!make_map_bf16(&mp->tmK, a.K, G.b, G.nk, G.hkv, kD, 1, kStepKeys)) return false;
    if (!make_map_bf16(&mp->tmV, a.V, G.b, G.nk, G.hkv, kD, 1, kStepKeys)) return false;
    return true;
}

template <typename F>
cudaError_t set_smem(F *fn, size_t bytes) {
    return cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

}  // namespace

bool attn_bwd_tc_supported(const Geom &G, dash_dtype_t dt) {
    if (dt != DASH_BF16 || G.d != kD) return false;
    if (G.B != 64 && G.B != 128) return false;
    if (G.g & (G.g - 1)) return false;
    if (G.tile_rows * G.g != kTileRows) return false;
    if (G.nq > 0x7fffffff || G.nk > 0x7fffffff) return false;
    if (G.b * G.hkv * (G.n_tiles + 1) * kTileRows > 0x7fffffff) return false;  // TMA row coordinates
    return tma_encode_fn() != nullptr;
}

cudaError_t launch_attn_bwd_tc_dq(const BwdArgs &a, cudaStream_t st) {
    const Geom &G = a.G;
    const ListsView &L = a.L;
    bwd_tc_prep_kernel<<<dim3((unsigned)L.n_tiles, (unsigned)G.hkv, (unsigned)G.b), kTileRows, 0, st>>>(
        a.Q, a.dO, a.O, G, L, a.lse, reinterpret_cast<uint4 *>(a.Qp), reinterpret_cast<uint4 *>(a.dOp), a.Lp, a.Dp);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    BwdMaps mp;
    if (!make_maps(&mp, a)) return cudaErrorInvalidValue;
    const int64_t ctas = L.n_tiles * G.hkv * G.b;
    if (ctas > 0x7fffffff) return cudaErrorInvalidValue;
    if (G.B == 64) {
        const size_t smem = DqSmem<64>::kTotal + 1024;
        if ((e = set_smem(bwd_dq_tc_kernel<64>, smem)) != cudaSuccess) return e;
        bwd_dq_tc_kernel<64><<<(unsigned)ctas, kThreads, smem, st>>>(mp, G, L, a.Lp, a.Dp, a.dQacc, a.Gd,
                                                                     heads_per_group(G));
    } else {
        const size_t smem = DqSmem<128>::kTotal + 1024;
        if ((e = set_smem(bwd_dq_tc_kernel<128>, smem)) != cudaSuccess) return e;
        bwd_dq_tc_kernel<128><<<(unsigned)ctas, kThreads, smem, st>>>(mp, G, L, a.Lp, a.Dp, a.dQacc, a.Gd,
                                                                      heads_per_group(G));
    }
    return cudaGetLastError();
}

cudaError_t launch_attn_bwd_tc_dkdv(const BwdArgs &a, cudaStream_t st) {
    const Geom &G = a.G;
    BwdMaps mp;
    if (!make_maps(&mp, a)) return cudaErrorInvalidValue;
    const int64_t nkb = (G.nk + kStepKeys - 1) / kStepKeys;
    const size_t smem = KvSmem::kTotal + 1024;
    cudaError_t e;
    const size_t acc_bytes = (size_t)G.b * G.nk * G.hkv * kD * sizeof(float);
    if ((e = cudaMemsetAsync(a.dKacc, 0, acc_bytes, st)) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(a.dVacc, 0, acc_bytes, st)) != cudaSuccess) return e;
    // split the pairs of a block among up to 8 CTAs: one per 64 tiles a block may have
    const int nsplit = (int)std::min<int64_t>(8, std::max<int64_t>(1, a.L.n_tiles / 64));
    dim3 grid((unsigned)(nkb * nsplit), (unsigned)G.hkv, (unsigned)G.b);
    if (G.B == 64) {
        if ((e = set_smem(bwd_dkdv_tc_kernel<64>, smem)) != cudaSuccess) return e;
        bwd_dkdv_tc_kernel<64><<<grid, kThreads, smem, st>>>(mp, G, a.L, a.Lp, a.Dp, a.ref_off, a.ref_cnt, a.refs,
                                                             a.dKacc, a.dVacc,
                                                             reinterpret_cast<const __nv_bfloat16 *>(a.Qp),
                                                             reinterpret_cast<const __nv_bfloat16 *>(a.dOp), nsplit);
    } else {
        if ((e = set_smem(bwd_dkdv_tc_kernel<128>, smem)) != cudaSuccess) return e;
        bwd_dkdv_tc_kernel<128><<<grid, kThreads, smem, st>>>(mp, G, a.L, a.Lp, a.Dp, a.ref_off, a.ref_cnt, a.refs,
                                                              a.dKacc, a.dVacc,
                                                              reinterpret_cast<const __nv_bfloat16 *>(a.Qp),
                                                              reinterpret_cast<const __nv_bfloat16 *>(a.dOp), nsplit);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const int64_t n4 = G.b * G.nk * G.hkv * (int64_t)(kD / 4);
    bwd_kv_finish_kernel<<<(unsigned)((n4 + 255) / 256), 256, 0, st>>>(
        reinterpret_cast<const float4 *>(a.dKacc), reinterpret_cast<const float4 *>(a.dVacc), a.dKbar, G, a.dK, a.dV);
    return cudaGetLastError();
}

int take_device_error_bwd() { return take_device_error_local(); }

}  // namespace dash

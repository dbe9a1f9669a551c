// select_tile.cu -- Stage 1 on tensor cores: entmax routing of the (query row, head)
// pairs of blocks of query rows (bf16 inputs, up to 2048 routing chunks).
//
// For the pairs of one (batch, kv head, block of query rows) ("DashAttention" §3.2
// Eq. 4, App. G Alg. 2):
//   logits   X = gamma/sqrt(d) * Q K̄^T on tcgen05 into tensor memory: Q is bf16,
//            the fp32 chunk summaries are split k̄ = hi + lo into two bf16 operands
//            (per call, or kept across decoding steps in a summary cache) and both
//            products accumulate in fp32 (relative error ~2^-17, i.e. fp32-class
//            logits).  TMEM holds 128 lanes x 512 fp32 columns; with LG lane groups
//            a row block routes 128/LG pairs over up to 512*LG chunks, lane group lg
//            holding chunk tiles lg, lg + LG, ... of its pairs in the same columns.
//            The logits MMA of a tile of lane group lg reads Q through a zero-padded
//            A operand whose only non-zero rows are that group's lanes, so
//            accumulating the LG groups' products into one column block writes each
//            group's lanes and adds zero to the others.
//            Above 256 chunks one persistent CTA per SM walks row blocks: tensor
//            memory is a ring of four 128-column blocks, and a producer warp issues
//            the next block's logits MMAs column block by column block as the 16
//            entmax warps release them after their last pass over the current block.
//            Up to 256 chunks a CTA takes one row block, and two CTAs share an SM;
//   tau      the threads of a pair walk its TMEM row in 32-column blocks: max, a
//            32-bin shared-memory histogram over [max x - 1, max x) for the
//            starting point (AdaSplash-2's initialisation), then a bracketed
//            iteration: for alpha = 2 and 1.5 the exact closed form on the current
//            support (until the support is stable), for alpha = 1.25 the first root of
//            the support's quartic (Newton in registers on its power sums), otherwise
//            Newton on the data, with bisection as the safeguard; partial sums are
//            combined in a fixed order so every thread of a pair takes the same
//            decisions;
//   prior    the g heads of a query row sit in g adjacent lanes of one warp; a
//            reduce-scatter over those lanes (the persistent kernel) or a
//            shared-memory transpose (the two-CTA kernel) gives each lane the g heads'
//            sums for 32/g chunks: w_c = (1/g) sum_h [x_c - tau_h]_+^{1/(alpha-1)},
//            membership by comparison, mu = mean log w over the routed chunks
//            (§3.4 Prop. 1); outputs the bit mask, log w of the routed chunks and mu
//            per row, from which the work lists are built (d = (log w - mu)/sigma).
// Both kernels are compiled for a GQA group of 4 as a constant and for any group.
#include <math.h>

#include <algorithm>

#include "dash_common.cuh"
#include "kernels.h"
#include "tma_host.h"

namespace dash {

namespace {

constexpr int kChunkTile = 128;    // chunks per logits MMA (N)
constexpr int kMaxTileChunks = 2048;
constexpr int kXchVals = 7;  // values a pair exchanges at most at once
constexpr uint64_t kTileWaitNs = 2000000000ull;

// Lane groups of a row block: its logits fill at most the 512 tensor-memory columns, so
// LG groups of 128/LG pairs hold 512*LG chunks.
inline int sel_lane_groups(int n_chunks) { return n_chunks <= 512 ? 1 : n_chunks <= 1024 ? 2 : 4; }

struct TileP {
    float am1;    // alpha - 1
    float kexp;   // 1 / (alpha - 1)
    float alpha;
    float scale;  // gamma / sqrt(d)
};

struct TileOut {
    float *tau;       // [b][nq][hq] or null
    float *w;         // [b][nq][hkv][n_chunks] or null
    uint32_t *mask;   // [b][nq][hkv][words] (required)
    float *logw;      // [b][hkv][n_chunks][nq] log w of the routed chunks (logw_index), or null
    float *mu;        // [b][nq][hkv] mean log w over the routed chunks, or null
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

constexpr int kNSB = 2;                 // stages of the chunk-summary operands
constexpr int kAluThreads = 512;        // 16 entmax warps: 4 TMEM lane quadrants x 4 column parts
constexpr int kSelThreads = kAluThreads + 32;  // + one producer warp (copies, logits MMA)
constexpr int kRing = 4;                // tensor memory as a ring of 4 column blocks of 128
constexpr int kBins = 32;               // histogram bins over [max x - 1, max x)

// Smem layout for D and LG lane groups.
template <int D, int LG>
struct TSmem {
    static constexpr int kNP = 128 / LG;              // pairs per row block
    static constexpr int kDh = D / 64;
    // A operand: rows [0, 128-NP) zero, [128-NP, 128) the Q pairs, [128, 256-NP) zero;
    // the MMA of lane group lg starts at row 128 - NP - lg*NP
    static constexpr int kArows = 256 - kNP;
    static constexpr int kAregion = kArows * 128;     // one 64-column region
    static constexpr int kBregion = 128 * 128;
    static constexpr int kA = 0;
    static constexpr int kB = kA + kDh * kAregion;    // [stage][hi, lo][kDh regions]
    static constexpr int kBstage = 2 * kDh * kBregion;
    static constexpr int kHist = kB + kNSB * kBstage;          // [kBins][NP] uint32
    static constexpr int kXch = kHist + kBins * kNP * 4;       // [2 parity][kXchVals][512] float
    static constexpr int kBars = kXch + 2 * kXchVals * 512 * 4;
    // q_full, k_full[kNSB], mma_done[kNSB], tm_full[kRing], colfree[kRing], drained
    static constexpr int kNBars = 1 + 2 * kNSB + 2 * kRing + 1;
    static constexpr int kSlot = kBars + kNBars * 8;           // TMEM base, abort flag
    static constexpr int kTotal = kSlot + 16;
};

// k̄ [b][n_chunks][hkv][d] fp32 -> per (b, kv head, tile of 128 chunks) the bf16 pair
// hi = bf16(k̄), lo = bf16(k̄ - hi), each laid out exactly as the logits MMA reads it
// (K-major, 64-column regions of 128 rows x 128 bytes, 128-byte swizzle), so a CTA
// fetches a chunk tile with two bulk copies.  Chunks past n_chunks are zero.
// With a device-resident length (G.chunks_dev set) the tiles are taken from the first
// tile holding a chunk the cache has not pooled yet, and only tiles with new chunks run.
template <int D>
__global__ void __launch_bounds__(256) kbar_split_kernel(const float *__restrict__ kbar, Geom G0,
                                                         uint8_t *__restrict__ split, int ct0) {
    constexpr int kDh = D / 64, kRegion = 128 * 128;
    Geom G = G0;
    geom_live(G);
    int ct = ct0 + (int)blockIdx.x;
    if (G.chunks_dev) {
        const int done = *G.chunks_dev;
        if (done >= G.n_chunks) return;  // nothing new since the last step
        ct += done / 128;
        if (ct * 128 >= G.n_chunks) return;
    }
    const int r = blockIdx.y;
    const int64_t b = blockIdx.z;
    uint8_t *dst = split + ((((size_t)b * G.hkv + r) * G.ct_cap + ct) * 2) * (size_t)(kDh * kRegion);
    for (int u = threadIdx.x; u < 128 * (D / 8); u += 256) {
        const int c = u / (D / 8), j = u % (D / 8);
        const int cg = ct * 128 + c;
        float v[8];
        if (cg < G.n_chunks) {
            const float *src = kbar + (((size_t)b * G.kbar_cap + cg) * G.hkv + r) * D + j * 8;
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


// Barrier 1 over the 16 entmax warps (the producer warp runs its own loop).
__device__ __forceinline__ void alu_sync() { asm volatile("bar.sync 1, 512;" ::: "memory"); }
__device__ __forceinline__ bool alu_sync_or(bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred ip, op;\n\tsetp.ne.u32 ip, %1, 0;\n\tbar.red.or.pred op, 1, 512, ip;\n\t"
        "selp.u32 %0, 1, 0, op;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v)
        : "memory");
    return r != 0;
}
__device__ __forceinline__ bool alu_sync_and(bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred ip, op;\n\tsetp.ne.u32 ip, %1, 0;\n\tbar.red.and.pred op, 1, 512, ip;\n\t"
        "selp.u32 %0, 1, 0, op;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v)
        : "memory");
    return r != 0;
}

// Sum, max or min of NV values over the 4*LG threads of each pair: every thread writes
// its partials to slot (lg, cp) of its pair, one barrier, every thread reads the pair's
// slots in the same order (so the threads of a pair hold identical results).  Bit k of
// max_bits / min_bits selects max / min for value k (sum otherwise).  `parity`
// alternates the buffer so one barrier per exchange suffices.
template <int NV, int LG>
__device__ __forceinline__ void pair_reduce(float *xch, int parity, int slot, int p, float (&v)[NV], int max_bits,
                                            int min_bits) {
    constexpr int kNP = 128 / LG, kSlots = 4 * LG;
    float *buf = xch + (size_t)parity * kXchVals * 512;
#pragma unroll
    for (int k = 0; k < NV; ++k) buf[k * 512 + slot * kNP + p] = v[k];
    alu_sync();
#pragma unroll
    for (int k = 0; k < NV; ++k) {
        float a = buf[k * 512 + p];
#pragma unroll
        for (int s = 1; s < kSlots; ++s) {
            const float o = buf[k * 512 + s * kNP + p];
            a = ((max_bits >> k) & 1) ? fmaxf(a, o) : ((min_bits >> k) & 1) ? fminf(a, o) : a + o;
        }
        v[k] = a;
    }
}

// One CTA per SM walks row blocks (units) u = blockIdx.x, + gridDim.x, ...: unit u is
// row block t = n_tblk - 1 - u / (b hkv) (the latest, longest rows first) of kv head
// u % hkv and batch (u / hkv) % b.  A block of n_ct chunk tiles fills ncb = ceil(n_ct/LG)
// column blocks of 128 tensor-memory columns, taken in turn from a ring of 4.  The
// producer warp loads the Q rows and chunk-summary tiles of the next block with a visible
// chunk and issues its logits MMAs column block by column block, each as soon as the 16
// entmax warps have finished the group-prior pass over the block that held it, so the
// next block's logits are computed while the current block's last pass runs.
template <int D, int KINT, int LG, int GQ>
__global__ void __launch_bounds__(kSelThreads, 1) select_tile_kernel(const __grid_constant__ CUtensorMap tmQ,
                                                                    const uint8_t *__restrict__ ksplit, Geom G0,
                                                                    TileP P, TileOut out, int64_t n_units,
                                                                    int64_t n_tblk) {
    using S = TSmem<D, LG>;
    constexpr int kNP = S::kNP;
    Geom G = G0;
    geom_live(G);
    extern __shared__ uint8_t tsm_raw[];
    uint8_t *sm = tsm_raw + ((1024 - (smem_u32(tsm_raw) & 1023)) & 1023);
    uint64_t *q_full = reinterpret_cast<uint64_t *>(sm + S::kBars);
    uint64_t *k_full = q_full + 1;            // [kNSB]
    uint64_t *mma_done = k_full + kNSB;       // [kNSB]
    uint64_t *tm_full = mma_done + kNSB;      // [kRing] logits of the m-th block with a visible chunk
    uint64_t *colfree = tm_full + kRing;      // [kRing] the entmax warps are done with a column block
    uint64_t *drained = colfree + kRing;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + S::kSlot);
    volatile int *abort = reinterpret_cast<volatile int *>(sm + S::kSlot + 4);
    uint32_t *hist = reinterpret_cast<uint32_t *>(sm + S::kHist);
    float *xch = reinterpret_cast<float *>(sm + S::kXch);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int g = GQ > 0 ? GQ : G.g;  // the GQA group (a compile-time 4 in the common case)
    const int npos = kNP / g;                 // query positions per row block
    const int64_t nbh = G.b * G.hkv;
    auto unit = [&](int64_t u, int64_t &t, int &r, int64_t &b) {
        t = n_tblk - 1 - u / nbh;
        const int64_t rb = u % nbh;
        r = (int)(rb % G.hkv);
        b = rb / G.hkv;
    };
    auto unit_nct = [&](int64_t t) -> int {
        const int64_t last_row = min(G.nq - 1, t * npos + npos - 1);
        return (row_nvis(G, last_row) + kChunkTile - 1) / kChunkTile;
    };

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int k = 0; k < kNSB; ++k) {
            mbar_init(k_full + k, 1);
            mbar_init(mma_done + k, 1);
        }
        for (int k = 0; k < kRing; ++k) {
            mbar_init(tm_full + k, 1);
            mbar_init(colfree + k, kAluThreads / 32);
        }
        mbar_init(drained, 1);
        *abort = 0;
        fence_mbar_init();
    }
    if (warp == kAluThreads / 32) {
        tmem_alloc(tmem_slot, kRing * 128);
        tmem_relinquish();
    }
    // zero rows of the A operand (generic-proxy stores, made visible to the MMAs)
    constexpr int kZeroRows = S::kArows - kNP;                   // 0 when LG == 1
    constexpr int kZeroUnits = (kZeroRows > 0 ? kZeroRows : 1) * 8;  // 16-byte units per region
    for (int u = threadIdx.x; kZeroRows > 0 && u < S::kDh * kZeroUnits; u += kSelThreads) {
        const int dh = u / kZeroUnits, rem = u % kZeroUnits;
        int row = rem / 8;
        if (row >= 128 - kNP) row += kNP;  // skip the Q rows
        *reinterpret_cast<uint4 *>(sm + S::kA + dh * S::kAregion + row * 128 + (rem % 8) * 16) =
            make_uint4(0u, 0u, 0u, 0u);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem0 = *tmem_slot;

    if (warp == kAluThreads / 32) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            constexpr uint32_t id = idesc_bf16_f32(128, kChunkTile, 0, 0);
            constexpr uint32_t kTileBytes = 2 * S::kDh * S::kBregion;
            int64_t gt = 0;          // tiles of this CTA so far (stage / phase of the B operands)
            int64_t loaded = 0;      // tiles whose copy was issued
            int64_t waited = 0;      // tiles whose copy was waited for
            int nq_issued = 0, nq_waited = 0;
            int m = 0;               // blocks with a visible chunk so far
            int ring = 0;            // next column block of the ring
            uint32_t uses = 0;       // per ring slot (8 bits each): column-block fills so far (mod 252)
            bool ok = true, issued = false;
            for (int64_t un = blockIdx.x; un < n_units; un += gridDim.x) {
                int64_t t, b;
                int r;
                unit(un, t, r, b);
                const int n_ct = unit_nct(t);
                if (n_ct == 0) continue;  // no visible chunk: the entmax warps need no logits
                // the A operand and both B stages are free once the previous block's MMAs are done
                if (gt > 0 && !(ok = wait_bar(mma_done + (gt - 1) % kNSB, ((gt - 1) / kNSB) & 1, kTileWaitNs, abort)))
                    break;
                mbar_arrive_expect_tx(q_full, kNP * D * 2);
                for (int dh = 0; dh < S::kDh; ++dh)
                    tma_load_4d(sm + S::kA + dh * S::kAregion + (128 - kNP) * 128, &tmQ, q_full, dh * 64, r * g,
                                (int)(t * npos), (int)b);
                ++nq_issued;
                const uint8_t *ks =
                    ksplit + (((size_t)b * G.hkv + r) * G.ct_cap) * 2 * (size_t)(S::kDh * S::kBregion);
                auto load_b = [&](int k) {
                    const int st = (int)((gt + k) % kNSB);
                    mbar_arrive_expect_tx(k_full + st, kTileBytes);
                    bulk_load(sm + S::kB + st * S::kBstage, ks + (size_t)k * kTileBytes, kTileBytes, k_full + st);
                    ++loaded;
                };
                for (int k = 0; k < kNSB && k < n_ct; ++k) load_b(k);
                if (!(ok = wait_bar(q_full, (nq_issued - 1) & 1, kTileWaitNs, abort))) break;
                ++nq_waited;
                for (int k = 0; k < n_ct; ++k) {
                    const int64_t gk = gt + k;
                    const int st = (int)(gk % kNSB);
                    const int klg = k % LG;
                    const int rs = (ring + k / LG) % kRing;
                    if (klg == 0) {  // first tile of a column block: the block that held it is done with it
                        uint32_t n_use = (uses >> (8 * rs)) & 0xffu;
                        if (n_use > 0 && !(ok = wait_bar(colfree + rs, (n_use - 1) & 1, kTileWaitNs, abort))) break;
                        if (++n_use >= 254) n_use -= 252;  // only the parity matters once the slot was used
                        uses = (uses & ~(0xffu << (8 * rs))) | (n_use << (8 * rs));
                    }
                    if (!(ok = wait_bar(k_full + st, (gk / kNSB) & 1, kTileWaitNs, abort))) break;
                    ++waited;
                    tc_fence_after();
                    const uint32_t qb = smem_u32(sm + S::kA) + (uint32_t)((128 - kNP - klg * kNP) * 128);
                    const uint32_t hb = smem_u32(sm + S::kB + st * S::kBstage);
                    const uint32_t lb = hb + S::kDh * S::kBregion;
                    const uint32_t dcol = tmem0 + (uint32_t)(rs * 128);
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t qa = qb + (kk / 4) * S::kAregion + (kk % 4) * 32;
                        const uint32_t ka = hb + (kk / 4) * S::kBregion + (kk % 4) * 32;
                        // the first lane group of a column block initialises it (other lanes get 0)
                        mma_ss(dcol, smem_desc_sw128(qa, 16, 1024), smem_desc_sw128(ka, 16, 1024), id,
                               (kk > 0 || klg > 0) ? 1u : 0u);
                    }
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t qa = qb + (kk / 4) * S::kAregion + (kk % 4) * 32;
                        const uint32_t ka = lb + (kk / 4) * S::kBregion + (kk % 4) * 32;
                        mma_ss(dcol, smem_desc_sw128(qa, 16, 1024), smem_desc_sw128(ka, 16, 1024), id, 1u);
                    }
                    mma_commit(mma_done + st);
                    issued = true;
                    // the stage of tile k+1-kNSB takes tile k+1 once that tile's MMA has read it
                    if (k + 1 < n_ct && k + 1 >= kNSB) {
                        const int64_t gp = gk + 1 - kNSB;
                        if (!(ok = wait_bar(mma_done + gp % kNSB, (gp / kNSB) & 1, kTileWaitNs, abort))) break;
                        load_b(k + 1);
                    }
                }
                if (!ok) break;
                mma_commit(tm_full + m % kRing);  // arrives when the block's MMAs have completed
                ++m;
                ring = (ring + (n_ct + LG - 1) / LG) % kRing;
                gt += n_ct;
            }
            // drain: every MMA issued, then every copy issued, has completed
            if (issued) {
                mma_commit(drained);
                wait_bar(drained, 0, kTileWaitNs, abort, false);
            }
            for (int64_t gk = waited; gk < loaded; ++gk)
                wait_bar(k_full + gk % kNSB, (gk / kNSB) & 1, kTileWaitNs, abort, false);
            if (nq_waited < nq_issued) wait_bar(q_full, (nq_issued - 1) & 1, kTileWaitNs, abort, false);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ entmax warps
        const int qd = warp & 3, cp = warp >> 2;  // TMEM lane quadrant; column part
        const int L = qd * 32 + lane;             // TMEM lane
        const int lg = L / kNP, p = L % kNP;      // lane group; pair
        const int slot = lg * 4 + cp;
        const int pos = p / g, hh = p % g;
        const uint32_t lane_off = (uint32_t)(qd * 32) << 16;
        const bool lead = hh == 0;
        const uint32_t tmem = tmem0;
        int m = 0, ring = 0;
        for (int64_t un = blockIdx.x; un < n_units; un += gridDim.x) {
            int64_t t, b;
            int r;
            unit(un, t, r, b);
            const int n_ct = unit_nct(t);
            const int ncb = (n_ct + LG - 1) / LG;   // column blocks of the block
            if (n_ct > 0) {
                const bool got = wait_bar(tm_full + m % kRing, (m / kRing) & 1, kTileWaitNs, abort);
                if (!alu_sync_and(got)) break;  // every entmax warp takes the same decision
                tc_fence_after();
            }
            const int64_t i = t * npos + pos;
            const bool row_ok = i < G.nq;
            const int nvis = row_ok ? row_nvis(G, i) : 0;
            for (int x = threadIdx.x; x < kBins * kNP; x += kAluThreads) hist[x] = 0u;

            // -------------------------------------------------------- tau per pair
            // this thread's column blocks: jb = 0 .. nb-1, tile jb*LG + lg in ring slot
            // (ring + jb) % 4, columns cp*32 .. cp*32 + 31 of it, chunks (jb*LG + lg)*128 +
            // cp*32 + x; the bound is uniform across the warp (128/LG >= 32 lanes per group)
            const int nb = lg < n_ct ? (n_ct - lg + LG - 1) / LG : 0;
            auto ring_slot = [&](int jb) -> int { return (ring + jb) % kRing; };
            auto blk_col = [&](int jb) -> uint32_t { return (uint32_t)(ring_slot(jb) * 128 + cp * 32); };
            auto blk_chunk = [&](int jb) -> int { return (jb * LG + lg) * 128 + cp * 32; };
            const float xs = P.am1 * P.scale;  // x = (alpha - 1) * gamma / sqrt(d) * <q, k̄>
            int parity = 0;
            // pass 0: x written back over the logits (-inf past the row's visible chunks), max
            float mx = -INFINITY;
            for (int jb = 0; jb < nb; ++jb) {
                uint32_t u[32];
                const uint32_t col = blk_col(jb);
                tmem_ld32(tmem + lane_off + col, u);
                const int lim = nvis - blk_chunk(jb);
#pragma unroll
                for (int x = 0; x < 32; ++x) {
                    const float xv = x < lim ? xs * __uint_as_float(u[x]) : -INFINITY;
                    mx = fmaxf(mx, xv);
                    u[x] = __float_as_uint(xv);
                }
                tmem_st32(tmem + lane_off + col, u);
            }
            tmem_wait_st();
            {
                float v[1] = {mx};
                pair_reduce<1, LG>(xch, parity, slot, p, v, 1, 0);
                parity ^= 1;
                mx = v[0];
            }
            // bracket: f(mx - 1) >= 0 (the largest term alone is 1), f(mx - n^{1-alpha}) <= 0
            float lo = mx - 1.f;
            float hi = nvis > 0 ? mx - powf((float)nvis, 1.f - P.alpha) : 0.f;
            // histogram of x over [mx - 1, mx), 32 bins per pair
            for (int jb = 0; jb < nb; ++jb) {
                uint32_t u[32];
                tmem_ld32(tmem + lane_off + blk_col(jb), u);
#pragma unroll
                for (int x = 0; x < 32; ++x) {
                    const float y = __uint_as_float(u[x]) - lo;
                    // bin floor(y kBins) as the low bits of y kBins + 2^23 rounded toward zero
                    // (an FMA instead of a float-to-int conversion)
                    const int bin = min(kBins - 1, __float_as_int(__fmaf_rz(y, (float)kBins, 8388608.f)) & 0xff);
                    if (y >= 0.f) atomicAdd(hist + bin * kNP + p, 1u);
                }
            }
            alu_sync();
            float t0 = lo;
            if (nvis > 1) {
                // estimated f at a bin edge e (every element at its bin centre c_j):
                //   f~(e) = sum_{j >= bin(e)} n_j (c_j - e)^k - 1, decreasing in e;
                // start from the highest edge still estimated >= 0.  For k = 1, 2, 4 the sum is
                // expanded in suffix moments A_m = sum_{j >= bin} n_j c_j^m (one sweep from the top).
                int elo = 0;
                if (KINT == 1 || KINT == 2 || KINT == 4) {
                    float A0 = 0.f, A1 = 0.f, A2 = 0.f, A3 = 0.f, A4 = 0.f;
                    for (int e = kBins - 1; e >= 1; --e) {
                        const float n = (float)hist[e * kNP + p];
                        const float c = ((float)e + 0.5f) * (1.f / kBins), c2 = c * c;
                        A0 += n;
                        A1 += n * c;
                        A2 += n * c2;
                        if (KINT == 4) {
                            A3 += n * c2 * c;
                            A4 += n * c2 * c2;
                        }
                        const float x = (float)e * (1.f / kBins);
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
                    int ehi = kBins - 1;
                    while (elo < ehi) {
                        const int e = (elo + ehi + 1) / 2;
                        const float edge = (float)e * (1.f / kBins);
                        float fe = -1.f;
                        for (int jb = e; jb < kBins; ++jb)
                            fe += (float)hist[jb * kNP + p] * rpow<KINT>(((float)jb + 0.5f) * (1.f / kBins) - edge, P);
                        if (fe >= 0.f) elo = e;
                        else ehi = e - 1;
                    }
                }
                t0 = lo + (float)elo * (1.f / kBins);
                if (!(t0 < hi)) t0 = lo;
            }
            // bracketed iteration (identical on every thread of the pair: same combined sums)
            float tau = nvis == 1 ? lo : t0;
            bool done = nvis <= 1;
            // a closed form on the current support for alpha = 2 and 1.5; for alpha = 1.25 the
            // support's quartic, solved from its power sums by Newton in registers
            constexpr bool kClosed = KINT == 1 || KINT == 2 || KINT == 4;
            constexpr int kNV = KINT == 4 ? 7 : 5;  // combined values per pass
            int prev_cnt = -1;
            for (int it = 0; it < 40; ++it) {
                if (!alu_sync_or(!done)) break;
                // alpha = 2 / 1.5: moments of z = x - tau over the support {x > tau}, its count,
                // the smallest score inside and the largest outside; alpha = 1.25: the same with the
                // first four power sums of z = x - tau (in 0, 1, 5, 6); otherwise f + 1, -f'/k, count
                float acc[kNV];
                acc[0] = acc[1] = acc[2] = 0.f;
                acc[3] = INFINITY;
                acc[4] = -INFINITY;
                if (kNV > 5) acc[kNV - 2] = acc[kNV - 1] = 0.f;
                // a warp whose pairs are all settled skips the pass (the threads of a pair share
                // their decisions, so the pair's other warps skip it too)
                if (!__all_sync(0xffffffffu, done)) {
                    for (int jb = 0; jb < nb; ++jb) {
                        uint32_t u[32];
                        tmem_ld32(tmem + lane_off + blk_col(jb), u);
#pragma unroll
                        for (int x = 0; x < 32; ++x) {
                            const float xv = __uint_as_float(u[x]);
                            const float tt = xv - tau;
                            if (tt > 0.f) {
                                if (KINT == 4) {
                                    const float z2 = tt * tt;
                                    acc[0] += tt;
                                    acc[1] += z2;
                                    acc[kNV - 2] = fmaf(z2, tt, acc[kNV - 2]);
                                    acc[kNV - 1] = fmaf(z2, z2, acc[kNV - 1]);
                                    acc[3] = fminf(acc[3], xv);
                                } else if (kClosed) {
                                    acc[0] += tt;
                                    acc[1] = fmaf(tt, tt, acc[1]);
                                    acc[3] = fminf(acc[3], xv);
                                } else {
                                    acc[0] += rpow<KINT>(tt, P);
                                    acc[1] += rpow_m1<KINT>(tt, P);
                                }
                                acc[2] += 1.f;
                            } else if (kClosed) {
                                acc[4] = fmaxf(acc[4], xv);
                            }
                        }
                    }
                }
                pair_reduce<kNV, LG>(xch, parity, slot, p, acc, 1 << 4, 1 << 3);
                parity ^= 1;
                if (done) continue;
                const int cnt = (int)acc[2];
                float f;
                if (KINT == 1) f = acc[0] - 1.f;                                                      // sum z - 1
                else if (KINT == 2) f = acc[1] - 1.f;                                                 // sum z^2 - 1
                else if (KINT == 4) f = acc[kNV - 1] - 1.f;                                           // sum z^4 - 1
                else f = acc[0] - 1.f;
                if (f >= 0.f) lo = tau;
                else hi = tau;
                float nt;
                if (kClosed && cnt > 0) {
                    // exact threshold if the support were S = {x > tau}; it is the answer when S is
                    // also {x > nt}: every score of S above nt, every other score at most nt
                    const float m1 = acc[0] / (float)cnt;
                    if (KINT == 1) {
                        nt = tau + (acc[0] - 1.f) / (float)cnt;
                    } else if (KINT == 2) {
                        const float var = fmaxf(acc[1] / (float)cnt - m1 * m1, 0.f);
                        nt = tau + m1 - sqrtf(fmaxf(1.f / (float)cnt - var, 0.f));
                    } else {
                        // g(dl) = sum_S (z - dl)^4 - 1 = Z4 - 4 Z3 dl + 6 Z2 dl^2 - 4 Z1 dl^3 + Z0 dl^4 - 1 is
                        // convex and decreasing at dl = 0: Newton from dl = 0 reaches its first root from
                        // the left (after one step back when g(0) < 0)
                        const float Z0 = (float)cnt, Z1 = acc[0], Z2 = acc[1], Z3 = acc[kNV - 2], Z4 = acc[kNV - 1];
                        float dl = 0.f;
                        for (int k = 0; k < 32; ++k) {
                            const float gv = (((Z0 * dl - 4.f * Z1) * dl + 6.f * Z2) * dl - 4.f * Z3) * dl + Z4 - 1.f;
                            const float dg = ((4.f * Z0 * dl - 12.f * Z1) * dl + 12.f * Z2) * dl - 4.f * Z3;
                            if (!(dg < 0.f)) break;
                            const float nd = dl - gv / dg;
                            const bool conv = fabsf(nd - dl) <= 1e-7f * fmaxf(1.f, fabsf(tau));
                            dl = nd;
                            if (conv) break;
                        }
                        nt = tau + dl;
                    }
                    // (or, with rounding ties, when two closed-form steps in a row saw the same
                    // support: supports {x > tau} are nested, so equal counts mean equal sets)
                    if (cnt == prev_cnt) {
                        done = true;
                        continue;
                    }
                    prev_cnt = cnt;
                    // at the root the closed form can land a rounding error outside the bracket:
                    // a step that close is clamped into it, a farther one is replaced by bisection
                    const float slack = 4e-7f * fmaxf(1.f, fabsf(tau));
                    if (nt >= lo - slack && nt <= hi + slack) {
                        nt = fminf(fmaxf(nt, lo), hi);
                        if (acc[3] > nt && acc[4] <= nt) done = true;
                    } else {
                        nt = 0.5f * (lo + hi);  // a bisection step: the next count proves nothing
                        prev_cnt = -1;
                    }
                    if (hi - lo <= slack) done = true;  // the bracket has collapsed onto the root
                } else {
                    const float df = -P.kexp * acc[1];
                    nt = df < 0.f ? tau - f / df : 0.5f * (lo + hi);
                    if (!(nt > lo && nt < hi)) nt = 0.5f * (lo + hi);
                    if (fabsf(nt - tau) <= 1e-7f * fmaxf(1.f, fabsf(tau)) || hi - lo <= 1e-7f * fmaxf(1.f, fabsf(tau)))
                        done = true;
                }
                tau = nt;
            }
            if (nvis == 0) tau = NAN;
            if (slot == 0 && out.tau && row_ok) out.tau[((size_t)b * G.nq + i) * G.hq + r * g + hh] = tau;

            // ---------------------------------------------------------------- group prior
            // The g heads of a query row sit in g adjacent lanes.  Per 32-column block every lane
            // forms [t]_+^{1/(alpha-1)} of its own head (t = x - tau) for the 32 chunks, then a
            // reduce-scatter over the g lanes (log2 g exchange rounds, each halving the values a
            // lane holds) leaves lane hh with the g-head sums of chunks hh, hh + g, ..., from which
            // it forms w_c = sum / g and log w for those chunks alone; membership (some head's
            // t > 0) is a 32-bit word OR-ed over the g lanes.
            const size_t rowoff = ((size_t)b * G.nq + i) * G.hkv + r;
            const float log_g = logf((float)g);
            const int lg2g = 31 - __clz(g);                 // g is a power of two
            const float tau_r = nvis > 0 ? tau : INFINITY;  // rows without chunks select nothing
            const bool writer = lead && row_ok;
            float lsum = 0.f, lcnt = 0.f;
            for (int jb = 0; jb < nb; ++jb) {
                uint32_t u[32];
                tmem_ld32(tmem + lane_off + blk_col(jb), u);
                const int c0 = blk_chunk(jb);
                uint32_t word = 0;  // bit x: this head's t > 0 for chunk c0 + x
#pragma unroll
                for (int x = 0; x < 32; ++x) {  // u[x] becomes V_x = [t]_+^{1/(alpha-1)} (as bits)
                    const float tt = __uint_as_float(u[x]) - tau_r;
                    u[x] = __float_as_uint(rpow<KINT>(tt, P));
                    word |= (tt > 0.f ? 1u : 0u) << x;
                }
                for (int o = 1; o < g; o <<= 1) word |= __shfl_xor_sync(0xffffffffu, word, o);
                // round s: V_k holds chunk k * 2^s + (hh mod 2^s); the lane keeps the chunk whose
                // bit s matches hh's and adds the partner's (lane ^ 2^s) value of that chunk
#pragma unroll
                for (int sr = 0; sr < 5; ++sr) {
                    if ((1 << sr) < g) {
                        const bool hb = (hh >> sr) & 1;
#pragma unroll
                        for (int k = 0; k < (16 >> sr); ++k) {
                            const float a = __uint_as_float(u[2 * k]), c = __uint_as_float(u[2 * k + 1]);
                            const float keep = hb ? c : a, send = hb ? a : c;
                            u[k] = __float_as_uint(keep + __shfl_xor_sync(0xffffffffu, send, 1 << sr));
                        }
                    }
                }
                // V_j = the g heads' sum for chunk c0 + j * g + hh
#pragma unroll
                for (int jj = 0; jj < 32; ++jj) {
                    if (jj < (32 >> lg2g)) {
                        const int x = (jj << lg2g) + hh;
                        const bool sel = (word >> x) & 1u;
                        float lw = -INFINITY;
                        if (sel) {
                            // the power sum underflows only for scores within ~1e-10 of tau at alpha = 1.25;
                            // keep such a chunk routed with the smallest representable weight
                            const float v = __uint_as_float(u[jj]);
                            lw = v > 0.f ? __logf(v) - log_g : -103.28f - log_g;
                            lsum += lw;
                            lcnt += 1.f;
                            if (row_ok && out.logw) out.logw[logw_index(G, b, r, i, c0 + x)] = lw;
                        }
                        if (out.w && row_ok && c0 + x < G.n_chunks) out.w[rowoff * G.n_chunks + c0 + x] = sel ? expf(lw) : 0.f;
                    }
                }
                if (writer && c0 / 32 < G.words) out.mask[rowoff * G.words + c0 / 32] = word;
                // this warp is done with the column block: the producer may fill it again
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(colfree + ring_slot(jb));
            }
            // column blocks of the block that hold no tile of this warp's lane group
            for (int jb = nb; jb < ncb; ++jb)
                if (lane == 0) mbar_arrive(colfree + ring_slot(jb));
            // the row's sums over the chunks its g lanes took (the same totals on every lane)
            for (int o = 1; o < g; o <<= 1) {
                lsum += __shfl_xor_sync(0xffffffffu, lsum, o);
                lcnt += __shfl_xor_sync(0xffffffffu, lcnt, o);
            }
            {
                float v[2] = {lsum, lcnt};
                pair_reduce<2, LG>(xch, parity, slot, p, v, 0, 0);
                parity ^= 1;
                lsum = v[0];
                lcnt = v[1];
            }
            if (writer && slot == 0) {
                if (out.mu) out.mu[rowoff] = lcnt > 0.f ? lsum / lcnt : 0.f;
                // words and chunks past the computed column blocks
                for (int wd = n_ct * 4; wd < G.words; ++wd) out.mask[rowoff * G.words + wd] = 0u;
                if (out.w)
                    for (int c = n_ct * 128; c < G.n_chunks; ++c) out.w[rowoff * G.n_chunks + c] = 0.f;
            }
            if (n_ct > 0) {
                ++m;
                ring = (ring + ncb) % kRing;
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kAluThreads / 32) {
        tc_fence_after();
        tmem_dealloc(tmem0, kRing * 128);
    }
}

template <int D, int KINT, int LG, int GQ>
cudaError_t launch_sel(const CUtensorMap &tmQ, const uint8_t *ksplit, const Geom &G, const TileP &P,
                       const TileOut &o, cudaStream_t st) {
    using S = TSmem<D, LG>;
    static_assert(S::kTotal + 1024 <= 232448, "shared memory of the Stage-1 kernel");
    const size_t smem = S::kTotal + 1024;
    cudaError_t e = cudaFuncSetAttribute(select_tile_kernel<D, KINT, LG, GQ>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int npos = (128 / LG) / G.g;
    const int64_t n_tblk = (G.nq + npos - 1) / npos;
    const int64_t n_units = n_tblk * G.hkv * G.b;
    int dev = 0, sms = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    const int64_t grid = std::min<int64_t>(n_units, sms);
    select_tile_kernel<D, KINT, LG, GQ><<<(unsigned)grid, kSelThreads, smem, st>>>(tmQ, ksplit, G, P, o, n_units, n_tblk);
    return cudaGetLastError();
}

// ----------------------------------------------------------------------------
// Up to two chunk tiles (n_chunks <= 256): one row block per CTA, two CTAs per SM
// (half the threads, one operand stage, at most 256 tensor-memory columns), so that one
// CTA's logits overlap the other's passes.  Same passes as above; the group prior goes
// through a shared-memory transpose.
// ----------------------------------------------------------------------------

// Smem layout for D, LG lane groups, CP column parts (128 * CP threads) and NSB stages
// of the chunk-summary operands.
template <int D, int LG, int CP, int NSB>
struct TSmemPair {
    static constexpr int kNP = 128 / LG;              // pairs per CTA
    static constexpr int kDh = D / 64;
    // A operand: rows [0, 128-NP) zero, [128-NP, 128) the Q pairs, [128, 256-NP) zero;
    // the MMA of lane group lg starts at row 128 - NP - lg*NP
    static constexpr int kArows = 256 - kNP;
    static constexpr int kAregion = kArows * 128;     // one 64-column region
    static constexpr int kBregion = 128 * 128;
    static constexpr int kA = 0;
    static constexpr int kB = kA + kDh * kAregion;    // [stage][hi, lo][kDh regions]
    static constexpr int kBstage = 2 * kDh * kBregion;
    static constexpr int kMmaEnd = kB + NSB * kBstage;
    // solve phase (reuses the MMA region once every logit is in TMEM)
    static constexpr int kHist = 0;                          // [kBins][NP] uint32
    static constexpr int kXch = kHist + kBins * kNP * 4;     // [2 parity][kXchVals][512] float
    static constexpr int kTr = kXch + 2 * kXchVals * 512 * 4;  // [16 warps][32 lanes][33] float transpose
    static constexpr int kSolveEnd = kTr + 4 * CP * 32 * 33 * 4;
    static constexpr int kData = kMmaEnd > kSolveEnd ? kMmaEnd : kSolveEnd;
    static constexpr int kBars = kData;                      // q_full, k_full[2], mma_done[2], all_done
    static constexpr int kSlot = kBars + 6 * 8;
    static constexpr int kTotal = kSlot + 16;
};

// Sum, max or min of NV values over the 4*LG threads of each pair: every thread writes
// its partials to slot (lg, cp) of its pair, one barrier, every thread reads the pair's
// slots in the same order (so the threads of a pair hold identical results).  Bit k of
// max_bits / min_bits selects max / min for value k (sum otherwise).  `parity`
// alternates the buffer so one barrier per exchange suffices.
template <int NV, int LG, int CP>
__device__ __forceinline__ void pair_reduce_cta(float *xch, int parity, int slot, int p, float (&v)[NV], int max_bits,
                                            int min_bits) {
    constexpr int kNP = 128 / LG, kSlots = CP * LG;
    float *buf = xch + (size_t)parity * kXchVals * 512;
#pragma unroll
    for (int k = 0; k < NV; ++k) buf[k * 512 + slot * kNP + p] = v[k];
    __syncthreads();
#pragma unroll
    for (int k = 0; k < NV; ++k) {
        float a = buf[k * 512 + p];
#pragma unroll
        for (int s = 1; s < kSlots; ++s) {
            const float o = buf[k * 512 + s * kNP + p];
            a = ((max_bits >> k) & 1) ? fmaxf(a, o) : ((min_bits >> k) & 1) ? fminf(a, o) : a + o;
        }
        v[k] = a;
    }
}

template <int D, int KINT, int LG, int CP, int NSB, int GQ>
__global__ void __launch_bounds__(128 * CP, 4 / CP) select_tile_pair_kernel(const __grid_constant__ CUtensorMap tmQ,
                                                                      const uint8_t *__restrict__ ksplit, Geom G0,
                                                                      TileP P, TileOut out, uint32_t ncols) {
    using S = TSmemPair<D, LG, CP, NSB>;
    Geom G = G0;
    geom_live(G);
    constexpr int kT = 128 * CP;       // 4 TMEM lane quadrants x CP column parts
    constexpr int kQB = 4 / CP;        // 32-column blocks per chunk tile and thread
    constexpr int kNP = S::kNP;
    extern __shared__ uint8_t tsm_raw[];
    uint8_t *sm = tsm_raw + ((1024 - (smem_u32(tsm_raw) & 1023)) & 1023);
    uint64_t *q_full = reinterpret_cast<uint64_t *>(sm + S::kBars);
    uint64_t *k_full = q_full + 1;      // [2]
    uint64_t *mma_done = q_full + 3;    // [2]
    uint64_t *all_done = q_full + 5;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + S::kSlot);
    uint32_t *hist = reinterpret_cast<uint32_t *>(sm + S::kHist);
    float *xch = reinterpret_cast<float *>(sm + S::kXch);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int qd = warp & 3, cp = warp >> 2;  // TMEM lane quadrant; column part
    const int L = qd * 32 + lane;             // TMEM lane
    const int lg = L / kNP, p = L % kNP;      // lane group; pair
    const int slot = lg * CP + cp;
    const int g = GQ > 0 ? GQ : G.g;  // the GQA group (a compile-time 4 in the common case)
    const int npos = kNP / g;                 // query positions per CTA
    const int64_t t = (int64_t)gridDim.x - 1 - blockIdx.x;  // latest (longest) rows first
    const int r = blockIdx.y;
    const int64_t b = blockIdx.z;
    const int pos = p / g, hh = p % g;
    const int64_t i = t * npos + pos;
    const bool row_ok = i < G.nq;
    const int nvis = row_ok ? row_nvis(G, i) : 0;
    const int64_t last_row = min(G.nq - 1, t * npos + npos - 1);
    const int nvis_max = row_nvis(G, last_row);
    const int n_ct = (nvis_max + kChunkTile - 1) / kChunkTile;
    const uint32_t lane_off = (uint32_t)(qd * 32) << 16;
    const bool lead = hh == 0;

    if (threadIdx.x == 0) {
        for (int k = 0; k < 6; ++k) mbar_init(q_full + k, 1);
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, ncols);
        tmem_relinquish();
    }
    // zero rows of the A operand (generic-proxy stores, made visible to the MMA below)
    constexpr int kZeroRows = S::kArows - kNP;                   // 0 when LG == 1
    constexpr int kZeroUnits = (kZeroRows > 0 ? kZeroRows : 1) * 8;  // 16-byte units per region
    for (int u = threadIdx.x; kZeroRows > 0 && u < S::kDh * kZeroUnits; u += kT) {
        const int dh = u / kZeroUnits, rem = u % kZeroUnits;
        int row = rem / 8;
        if (row >= 128 - kNP) row += kNP;  // skip the Q rows
        *reinterpret_cast<uint4 *>(sm + S::kA + dh * S::kAregion + row * 128 + (rem % 8) * 16) =
            make_uint4(0u, 0u, 0u, 0u);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // ---------------------------------------------------------------- logits
    if (warp == 0) {
        if (lane == 0 && n_ct > 0) {
            mbar_arrive_expect_tx(q_full, kNP * D * 2);
            for (int dh = 0; dh < S::kDh; ++dh)
                tma_load_4d(sm + S::kA + dh * S::kAregion + (128 - kNP) * 128, &tmQ, q_full, dh * 64, r * g,
                            (int)(t * npos), (int)b);
            const uint8_t *ks = ksplit + (((size_t)b * G.hkv + r) * G.ct_cap) * 2 * (size_t)(S::kDh * S::kBregion);
            auto load_b = [&](int k, int s) {
                const uint8_t *src = ks + (size_t)k * 2 * S::kDh * S::kBregion;
                mbar_arrive_expect_tx(k_full + s, 2 * S::kDh * S::kBregion);
                bulk_load(sm + S::kB + s * S::kBstage, src, 2 * S::kDh * S::kBregion, k_full + s);
            };
            load_b(0, 0);
            if (NSB > 1 && n_ct > 1) load_b(1, 1);
            bool ok = mbar_wait_ns(q_full, 0, kTileWaitNs);
            constexpr uint32_t id = idesc_bf16_f32(128, kChunkTile, 0, 0);
            for (int k = 0; ok && k < n_ct; ++k) {
                const int s = k % NSB;
                if (!(ok = mbar_wait_ns(k_full + s, (k / NSB) & 1, kTileWaitNs))) break;
                tc_fence_after();
                const int klg = k % LG;
                const uint32_t qb = smem_u32(sm + S::kA) + (uint32_t)((128 - kNP - klg * kNP) * 128);
                const uint32_t hb = smem_u32(sm + S::kB + s * S::kBstage);
                const uint32_t lb = hb + S::kDh * S::kBregion;
                const uint32_t dcol = tmem + (uint32_t)((k / LG) * kChunkTile);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t qa = qb + (kk / 4) * S::kAregion + (kk % 4) * 32;
                    const uint32_t ka = hb + (kk / 4) * S::kBregion + (kk % 4) * 32;
                    // the first lane group of a column block initialises it (other lanes get 0)
                    mma_ss(dcol, smem_desc_sw128(qa, 16, 1024), smem_desc_sw128(ka, 16, 1024), id,
                           (kk > 0 || klg > 0) ? 1u : 0u);
                }
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t qa = qb + (kk / 4) * S::kAregion + (kk % 4) * 32;
                    const uint32_t ka = lb + (kk / 4) * S::kBregion + (kk % 4) * 32;
                    mma_ss(dcol, smem_desc_sw128(qa, 16, 1024), smem_desc_sw128(ka, 16, 1024), id, 1u);
                }
                mma_commit(mma_done + s);
                // the stage of tile k+1-NSB takes tile k+1 once that tile's MMA has read it
                if (k + 1 < n_ct && k + 1 >= NSB) {
                    const int kp = k + 1 - NSB, sp = kp % NSB;
                    if (!(ok = mbar_wait_ns(mma_done + sp, (kp / NSB) & 1, kTileWaitNs))) break;
                    load_b(k + 1, sp);
                }
            }
            mma_commit(all_done);  // arrives when every MMA issued above has completed
        }
        __syncwarp();
    }
    if (n_ct > 0) mbar_wait_ns(all_done, 0, kTileWaitNs);
    tc_fence_after();
    __syncthreads();  // the MMA staging memory is reused below
    for (int u = threadIdx.x; u < kBins * kNP; u += kT) hist[u] = 0u;

    // ---------------------------------------------------------------- tau per pair
    // this thread's column blocks: jb = 0 .. nb-1, tile j = jb / kQB and block q = cp + CP (jb %
    // kQB) at TMEM columns j*128 + q*32, chunks (j*LG + lg)*128 + q*32 + x; the bound is
    // uniform across the warp
    const int nj = lg < n_ct ? (n_ct - lg + LG - 1) / LG : 0;
    const int nb = nj * kQB;
    auto blk_col = [&](int jb) -> uint32_t { return (uint32_t)((jb / kQB) * 128 + (cp + CP * (jb % kQB)) * 32); };
    auto blk_chunk = [&](int jb) -> int { return ((jb / kQB) * LG + lg) * 128 + (cp + CP * (jb % kQB)) * 32; };
    const float xs = P.am1 * P.scale;  // x = (alpha - 1) * gamma / sqrt(d) * <q, k̄>
    int parity = 0;
    // pass 0: x written back over the logits (-inf past the row's visible chunks), max
    float mx = -INFINITY;
    for (int jb = 0; jb < nb; ++jb) {
        uint32_t u[32];
        const uint32_t col = blk_col(jb);
        tmem_ld32(tmem + lane_off + col, u);
        const int lim = nvis - blk_chunk(jb);
#pragma unroll
        for (int x = 0; x < 32; ++x) {
            const float xv = x < lim ? xs * __uint_as_float(u[x]) : -INFINITY;
            mx = fmaxf(mx, xv);
            u[x] = __float_as_uint(xv);
        }
        tmem_st32(tmem + lane_off + col, u);
    }
    tmem_wait_st();
    {
        float v[1] = {mx};
        pair_reduce_cta<1, LG, CP>(xch, parity, slot, p, v, 1, 0);
        parity ^= 1;
        mx = v[0];
    }
    // bracket: f(mx - 1) >= 0 (the largest term alone is 1), f(mx - n^{1-alpha}) <= 0
    float lo = mx - 1.f;
    float hi = nvis > 0 ? mx - powf((float)nvis, 1.f - P.alpha) : 0.f;
    // histogram of x over [mx - 1, mx), 32 bins per pair
    for (int jb = 0; jb < nb; ++jb) {
        uint32_t u[32];
        tmem_ld32(tmem + lane_off + blk_col(jb), u);
#pragma unroll
        for (int x = 0; x < 32; ++x) {
            const float y = __uint_as_float(u[x]) - lo;
            if (y >= 0.f) atomicAdd(hist + min(kBins - 1, (int)(y * (float)kBins)) * kNP + p, 1u);
        }
    }
    __syncthreads();
    float t0 = lo;
    if (nvis > 1) {
        // estimated f at a bin edge e (every element at its bin centre c_j):
        //   f~(e) = sum_{j >= bin(e)} n_j (c_j - e)^k - 1, decreasing in e;
        // start from the highest edge still estimated >= 0.  For k = 1, 2, 4 the sum is
        // expanded in suffix moments A_m = sum_{j >= bin} n_j c_j^m (one sweep from the top).
        int elo = 0;
        if (KINT == 1 || KINT == 2 || KINT == 4) {
            float A0 = 0.f, A1 = 0.f, A2 = 0.f, A3 = 0.f, A4 = 0.f;
            for (int e = kBins - 1; e >= 1; --e) {
                const float n = (float)hist[e * kNP + p];
                const float c = ((float)e + 0.5f) * (1.f / kBins), c2 = c * c;
                A0 += n;
                A1 += n * c;
                A2 += n * c2;
                if (KINT == 4) {
                    A3 += n * c2 * c;
                    A4 += n * c2 * c2;
                }
                const float x = (float)e * (1.f / kBins);
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
            int ehi = kBins - 1;
            while (elo < ehi) {
                const int e = (elo + ehi + 1) / 2;
                const float edge = (float)e * (1.f / kBins);
                float fe = -1.f;
                for (int jb = e; jb < kBins; ++jb)
                    fe += (float)hist[jb * kNP + p] * rpow<KINT>(((float)jb + 0.5f) * (1.f / kBins) - edge, P);
                if (fe >= 0.f) elo = e;
                else ehi = e - 1;
            }
        }
        t0 = lo + (float)elo * (1.f / kBins);
        if (!(t0 < hi)) t0 = lo;
    }
    // bracketed iteration (identical on every thread of the pair: same combined sums)
    float tau = nvis == 1 ? lo : t0;
    bool done = nvis <= 1;
    // a closed form on the current support for alpha = 2 and 1.5; for alpha = 1.25 the
    // support's quartic, solved from its power sums by Newton in registers
    constexpr bool kClosed = KINT == 1 || KINT == 2 || KINT == 4;
    constexpr int kNV = KINT == 4 ? 7 : 5;  // combined values per pass
    int prev_cnt = -1;
    for (int it = 0; it < 40; ++it) {
        if (!__syncthreads_or(!done)) break;
        // alpha = 2 / 1.5: moments of y = x - mx over the support {x > tau}, its count,
        // the smallest score inside and the largest outside; alpha = 1.25: the same with the
        // first four power sums of z = x - tau (in 0, 1, 5, 6); otherwise f + 1, -f'/k, count
        float acc[kNV];
        acc[0] = acc[1] = acc[2] = 0.f;
        acc[3] = INFINITY;
        acc[4] = -INFINITY;
        if (kNV > 5) acc[kNV - 2] = acc[kNV - 1] = 0.f;
        // a warp whose pairs are all settled skips the pass (the threads of a pair share
        // their decisions, so the pair's other warps skip it too)
        if (!__all_sync(0xffffffffu, done)) {
            for (int jb = 0; jb < nb; ++jb) {
                uint32_t u[32];
                tmem_ld32(tmem + lane_off + blk_col(jb), u);
#pragma unroll
                for (int x = 0; x < 32; ++x) {
                    const float xv = __uint_as_float(u[x]);
                    const float tt = xv - tau;
                    if (tt > 0.f) {
                        if (KINT == 4) {
                            const float z2 = tt * tt;
                            acc[0] += tt;
                            acc[1] += z2;
                            acc[kNV - 2] = fmaf(z2, tt, acc[kNV - 2]);
                            acc[kNV - 1] = fmaf(z2, z2, acc[kNV - 1]);
                            acc[3] = fminf(acc[3], xv);
                        } else if (kClosed) {
                            const float yv = xv - mx;
                            acc[0] += yv;
                            acc[1] = fmaf(yv, yv, acc[1]);
                            acc[3] = fminf(acc[3], xv);
                        } else {
                            acc[0] += rpow<KINT>(tt, P);
                            acc[1] += rpow_m1<KINT>(tt, P);
                        }
                        acc[2] += 1.f;
                    } else if (kClosed) {
                        acc[4] = fmaxf(acc[4], xv);
                    }
                }
            }
        }
        pair_reduce_cta<kNV, LG, CP>(xch, parity, slot, p, acc, 1 << 4, 1 << 3);
        parity ^= 1;
        if (done) continue;
        const int cnt = (int)acc[2];
        const float tr = tau - mx;  // tau in the y = x - mx frame
        float f;
        if (KINT == 1) f = acc[0] - tr * (float)cnt - 1.f;                                    // sum (y - tr) - 1
        else if (KINT == 2) f = acc[1] - 2.f * tr * acc[0] + tr * tr * (float)cnt - 1.f;     // sum (y - tr)^2 - 1
        else if (KINT == 4) f = acc[kNV - 1] - 1.f;                                           // sum z^4 - 1
        else f = acc[0] - 1.f;
        if (f >= 0.f) lo = tau;
        else hi = tau;
        float nt;
        if (kClosed && cnt > 0) {
            // exact threshold if the support were S = {x > tau}; it is the answer when S is
            // also {x > nt}: every score of S above nt, every other score at most nt
            const float m1 = acc[0] / (float)cnt;
            if (KINT == 1) {
                nt = mx + (acc[0] - 1.f) / (float)cnt;
            } else if (KINT == 2) {
                const float var = fmaxf(acc[1] / (float)cnt - m1 * m1, 0.f);
                nt = mx + m1 - sqrtf(fmaxf(1.f / (float)cnt - var, 0.f));
            } else {
                // g(dl) = sum_S (z - dl)^4 - 1 = Z4 - 4 Z3 dl + 6 Z2 dl^2 - 4 Z1 dl^3 + Z0 dl^4 - 1 is
                // convex and decreasing at dl = 0: Newton from dl = 0 reaches its first root from
                // the left (after one step back when g(0) < 0)
                const float Z0 = (float)cnt, Z1 = acc[0], Z2 = acc[1], Z3 = acc[kNV - 2], Z4 = acc[kNV - 1];
                float dl = 0.f;
                for (int k = 0; k < 32; ++k) {
                    const float gv = (((Z0 * dl - 4.f * Z1) * dl + 6.f * Z2) * dl - 4.f * Z3) * dl + Z4 - 1.f;
                    const float dg = ((4.f * Z0 * dl - 12.f * Z1) * dl + 12.f * Z2) * dl - 4.f * Z3;
                    if (!(dg < 0.f)) break;
                    const float nd = dl - gv / dg;
                    const bool conv = fabsf(nd - dl) <= 1e-7f * fmaxf(1.f, fabsf(tau));
                    dl = nd;
                    if (conv) break;
                }
                nt = tau + dl;
            }
            // (or, with rounding ties, when two closed-form steps in a row saw the same
            // support: supports {x > tau} are nested, so equal counts mean equal sets)
            if (cnt == prev_cnt) {
                done = true;
                continue;
            }
            prev_cnt = cnt;
            // at the root the closed form can land a rounding error outside the bracket:
            // a step that close is clamped into it, a farther one is replaced by bisection
            const float slack = 4e-7f * fmaxf(1.f, fabsf(tau));
            if (nt >= lo - slack && nt <= hi + slack) {
                nt = fminf(fmaxf(nt, lo), hi);
                if (acc[3] > nt && acc[4] <= nt) done = true;
            } else {
                nt = 0.5f * (lo + hi);  // a bisection step: the next count proves nothing
                prev_cnt = -1;
            }
            if (hi - lo <= slack) done = true;  // the bracket has collapsed onto the root
        } else {
            const float df = -P.kexp * acc[1];
            nt = df < 0.f ? tau - f / df : 0.5f * (lo + hi);
            if (!(nt > lo && nt < hi)) nt = 0.5f * (lo + hi);
            if (fabsf(nt - tau) <= 1e-7f * fmaxf(1.f, fabsf(tau)) || hi - lo <= 1e-7f * fmaxf(1.f, fabsf(tau)))
                done = true;
        }
        tau = nt;
    }
    if (nvis == 0) tau = NAN;
    if (slot == 0 && out.tau && row_ok) out.tau[((size_t)b * G.nq + i) * G.hq + r * g + hh] = tau;

    // ---------------------------------------------------------------- group prior
    // The g heads of a query row sit in g adjacent lanes.  Per 32-column block every lane
    // puts its t = x - tau into a padded shared-memory row; lane (pos, k) then reads the
    // g heads' t of the chunks x = k, k + g, ... of its row (32 values, bank-conflict free)
    // and forms w_c = (1/g) sum_h [t_h]_+^{1/(alpha-1)}, membership (some t_h > 0) and
    // log w for those chunks alone, so no work is repeated across the group.
    const size_t rowoff = ((size_t)b * G.nq + i) * G.hkv + r;
    const float log_g = logf((float)g);
    const float tau_r = nvis > 0 ? tau : INFINITY;  // rows without chunks select nothing
    const bool writer = lead && row_ok;
    float *tr = reinterpret_cast<float *>(sm + S::kTr) + warp * 32 * 33;
    const int gbase = lane - hh;  // lane of the row's first head
    float lsum = 0.f, lcnt = 0.f;
    for (int jb = 0; jb < nb; ++jb) {
        uint32_t u[32];
        tmem_ld32(tmem + lane_off + blk_col(jb), u);
        const int c0 = blk_chunk(jb);
#pragma unroll
        for (int x = 0; x < 32; ++x) tr[lane * 33 + x] = __uint_as_float(u[x]) - tau_r;
        __syncwarp();
        uint32_t word = 0;  // membership bits of this lane's chunks
#pragma unroll
        for (int x = hh; x < 32; x += g) {
            float v = 0.f;
            bool sel = false;
#pragma unroll
            for (int h = 0; h < g; ++h) {
                const float tt = tr[(gbase + h) * 33 + x];
                if (tt > 0.f) {
                    sel = true;
                    v += rpow<KINT>(tt, P);
                }
            }
            float lw = -INFINITY;
            if (sel) {
                // the power sum underflows only for scores within ~1e-10 of tau at alpha = 1.25;
                // keep such a chunk routed with the smallest representable weight
                lw = v > 0.f ? __logf(v) - log_g : -103.28f - log_g;
                lsum += lw;
                lcnt += 1.f;
                word |= 1u << x;
                if (row_ok && out.logw) out.logw[logw_index(G, b, r, i, c0 + x)] = lw;
            }
            if (out.w && row_ok && c0 + x < G.n_chunks) out.w[rowoff * G.n_chunks + c0 + x] = sel ? expf(lw) : 0.f;
        }
        __syncwarp();  // the transpose rows are rewritten by the next block
        for (int o = 1; o < g; o <<= 1) word |= __shfl_xor_sync(0xffffffffu, word, o);
        if (writer && c0 / 32 < G.words) out.mask[rowoff * G.words + c0 / 32] = word;
    }
    // the row's sums over the chunks its g lanes took (the same totals on every lane)
    for (int o = 1; o < g; o <<= 1) {
        lsum += __shfl_xor_sync(0xffffffffu, lsum, o);
        lcnt += __shfl_xor_sync(0xffffffffu, lcnt, o);
    }
    {
        float v[2] = {lsum, lcnt};
        pair_reduce_cta<2, LG, CP>(xch, parity, slot, p, v, 0, 0);
        parity ^= 1;
        lsum = v[0];
        lcnt = v[1];
    }
    if (writer && slot == 0) {
        if (out.mu) out.mu[rowoff] = lcnt > 0.f ? lsum / lcnt : 0.f;
        // words and chunks past the computed column blocks
        for (int wd = n_ct * 4; wd < G.words; ++wd) out.mask[rowoff * G.words + wd] = 0u;
        if (out.w)
            for (int c = n_ct * 128; c < G.n_chunks; ++c) out.w[rowoff * G.n_chunks + c] = 0.f;
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, ncols);
    }
}

template <int D, int KINT, int LG, int CP, int NSB, int GQ>
cudaError_t launch_sel_pair(const CUtensorMap &tmQ, const uint8_t *ksplit, const Geom &G, const TileP &P,
                       const TileOut &o, cudaStream_t st) {
    using S = TSmemPair<D, LG, CP, NSB>;
    const size_t smem = S::kTotal + 1024;
    cudaError_t e = cudaFuncSetAttribute(select_tile_pair_kernel<D, KINT, LG, CP, NSB, GQ>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int npos = (128 / LG) / G.g;
    const int64_t nblk = (G.nq + npos - 1) / npos;
    if (nblk > 0x7fffffff) return cudaErrorInvalidValue;
    // tensor-memory columns: the chunk tiles of one lane group, 128 each (a power of two)
    const int n_ct_all = (G.n_chunks + kChunkTile - 1) / kChunkTile;
    uint32_t ncols = 32;
    while (ncols < (uint32_t)(((n_ct_all + LG - 1) / LG) * kChunkTile)) ncols *= 2;
    dim3 grid((unsigned)nblk, (unsigned)G.hkv, (unsigned)G.b);
    select_tile_pair_kernel<D, KINT, LG, CP, NSB, GQ><<<grid, 128 * CP, smem, st>>>(tmQ, ksplit, G, P, o, ncols);
    return cudaGetLastError();
}

template <int D, int KINT>
cudaError_t launch_sel_lg(const TView &Q, const uint8_t *ksplit, const Geom &G, const TileP &P, const TileOut &o,
                          cudaStream_t st) {
    // a row block's logits fill at most the 512 tensor-memory columns: LG lane groups of
    // 128/LG pairs hold 512*LG chunks
    const int LG = sel_lane_groups(G.n_chunks);
    const int npos = (128 / LG) / G.g;
    CUtensorMap tmQ;
    if (!make_map_bf16(&tmQ, Q, G.b, G.nq, G.hq, G.d, G.g, npos)) return cudaErrorInvalidValue;
    if (G.n_chunks <= 2 * kChunkTile)
        return G.g == 4 ? launch_sel_pair<D, KINT, 1, 2, 1, 4>(tmQ, ksplit, G, P, o, st)
                        : launch_sel_pair<D, KINT, 1, 2, 1, 0>(tmQ, ksplit, G, P, o, st);
    if (G.g == 4) {
        if (LG == 1) return launch_sel<D, KINT, 1, 4>(tmQ, ksplit, G, P, o, st);
        if (LG == 2) return launch_sel<D, KINT, 2, 4>(tmQ, ksplit, G, P, o, st);
        return launch_sel<D, KINT, 4, 4>(tmQ, ksplit, G, P, o, st);
    }
    if (LG == 1) return launch_sel<D, KINT, 1, 0>(tmQ, ksplit, G, P, o, st);
    if (LG == 2) return launch_sel<D, KINT, 2, 0>(tmQ, ksplit, G, P, o, st);
    return launch_sel<D, KINT, 4, 0>(tmQ, ksplit, G, P, o, st);
}

}  // namespace

int take_device_error_select() { return take_device_error_local(); }

bool select_tile_supported(const Geom &G, dash_dtype_t dt) {
    if (dt != DASH_BF16) return false;
    if (G.d != 64 && G.d != 128) return false;
    if (G.g & (G.g - 1)) return false;
    const int LG = sel_lane_groups(G.n_chunks);
    if (G.g > 128 / LG || G.g > 32) return false;  // the heads of a row share one warp and one row block
    if (G.n_chunks > kMaxTileChunks) return false;
    return tma_encode_fn() != nullptr;
}

size_t select_tile_workspace(const Geom &G) {
    return kbar_split_bytes(G.b, G.hkv, G.d, (G.n_chunks + kChunkTile - 1) / kChunkTile);
}

cudaError_t launch_kbar_split(const float *kbar, const Geom &G, uint8_t *split, int ct0, int ct1, cudaStream_t st) {
    if (ct1 <= ct0 || G.b == 0) return cudaSuccess;
    if (G.chunks_dev) ct1 = min(ct1, G.ct_cap);  // device range: tiles past the capacity never run
    if (ct1 > G.ct_cap) return cudaErrorInvalidValue;
    dim3 sg((unsigned)(ct1 - ct0), (unsigned)G.hkv, (unsigned)G.b);
    if (G.d == 128) kbar_split_kernel<128><<<sg, 256, 0, st>>>(kbar, G, split, ct0);
    else kbar_split_kernel<64><<<sg, 256, 0, st>>>(kbar, G, split, ct0);
    return cudaGetLastError();
}

size_t kbar_split_bytes(int64_t batch, int hkv, int d, int ct_cap) {
    return (size_t)batch * hkv * ct_cap * 2 * (d / 64) * 128 * 128;
}

cudaError_t launch_select_tile(const TView &Q, const float *kbar, const Geom &G, float alpha, float gamma,
                               float *tau, float *w, uint32_t *mask, float *logw, float *mu, void *work,
                               cudaStream_t st, const uint8_t *presplit) {
    if (G.nq == 0 || G.b == 0) return cudaSuccess;
    if (!mask) return cudaErrorInvalidValue;
    const uint8_t *ksplit = presplit;
    if (!presplit) {
        const int n_ct = (G.n_chunks + kChunkTile - 1) / kChunkTile;
        cudaError_t e0 = launch_kbar_split(kbar, G, static_cast<uint8_t *>(work), 0, n_ct, st);
        if (e0 != cudaSuccess) return e0;
        ksplit = static_cast<const uint8_t *>(work);
    }
    TileP P;
    P.alpha = alpha;
    P.am1 = alpha - 1.f;
    P.kexp = 1.f / (alpha - 1.f);
    P.scale = gamma / sqrtf((float)G.d);
    const int kint = (alpha == 2.f) ? 1 : (alpha == 1.5f) ? 2 : (alpha == 1.25f) ? 4 : 0;
    TileOut o{tau, w, mask, logw, mu};
#define DASH_SEL_CASE(DD, KK) \
    if (G.d == DD && kint == KK) return launch_sel_lg<DD, KK>(Q, ksplit, G, P, o, st);
    DASH_SEL_CASE(128, 2)
    DASH_SEL_CASE(128, 1)
    DASH_SEL_CASE(128, 4)
    DASH_SEL_CASE(128, 0)
    DASH_SEL_CASE(64, 2)
    DASH_SEL_CASE(64, 1)
    DASH_SEL_CASE(64, 4)
    DASH_SEL_CASE(64, 0)
#undef DASH_SEL_CASE
    return cudaErrorNotSupported;
}

}  // namespace dash

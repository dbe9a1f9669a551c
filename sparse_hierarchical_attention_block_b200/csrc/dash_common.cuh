// dash_common.cuh -- shared device helpers of the DashAttention sm_100a kernels:
// problem geometry, bounded mbarrier waits, TMA and tcgen05 wrappers (inline PTX).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "dash_attn.h"

namespace dash {

// ---------------------------------------------------------------------------
// Problem geometry (host and device)
// ---------------------------------------------------------------------------
struct Geom {
    int64_t b, nq, nk;
    int hq, hkv, g, d, B;
    int causal;
    int n_chunks;   // routing chunks: floor(nk/B) causal, ceil(nk/B) otherwise
    int n_blk;      // KV blocks ceil(nk/B) (the trailing partial block is only ever diagonal)
    int tile_rows;  // query positions per Stage-2 tile (128 / g)
    int64_t n_tiles;
    int words;      // ceil(n_chunks / 32) mask words per row
    int kbar_cap;   // chunks per batch element in the chunk-summary buffer (its batch stride;
                    // n_chunks, or a persistent cache's capacity)
    int ct_cap;     // 128-chunk tiles per (batch, kv head) in the split-summary buffer
    int local;      // chunks of the causal local window: 1 (the query's own) or 2 (and the one before)
    // Decoding from a preallocated cache: nk above is the capacity, the number of valid keys
    // is read from *nk_dev when a kernel runs (null: nk is the length), and *chunks_dev is
    // the number of chunks a summary cache has pooled (device-side bookkeeping).
    const int64_t *nk_dev;
    const int *chunks_dev;
    // Key position of query row 0 of this launch: nk - nq, plus the first row of a slice when
    // the rows are processed in slices; and the row count of the lse output's layout.
    int64_t pos0;
    int64_t nq_lse;
};

// The geometry a kernel works with: with a device-resident key length, nk is read from
// device memory (clamped to the capacity the buffers were sized for) and the chunk counts
// that follow from it are recomputed; every kernel of a step derives the same values.
__device__ __forceinline__ void geom_live(Geom &G) {
    if (!G.nk_dev) return;
    int64_t nk = *G.nk_dev;
    nk = nk < 0 ? 0 : (nk > G.nk ? G.nk : nk);
    G.pos0 += nk - G.nk;  // the rows sit at the last positions before the live length
    G.nk = nk;
    G.n_chunks = (int)(G.causal ? nk / G.B : (nk + G.B - 1) / G.B);
    G.n_blk = (int)((nk + G.B - 1) / G.B);
    G.words = (G.n_chunks + 31) / 32;
}

// Strided 4-D tensor view passed by value to kernels (element strides).
struct TView {
    const void *p;
    int64_t s0, s1, s2;  // batch, seq, head strides; dim stride is 1
};

struct ListsView {
    int32_t *count;
    int32_t *ids;
    float *bias;
    int32_t *rows;  // query index of each tile row (-1 unused); null = consecutive rows
    int64_t n_tiles;
    int cap;
    int tile_rows;
};

// Query index held by row `pos` of tile `tile_idx` (flattened [b][hkv][tile]) whose
// tile number is t; -1 if the row is unused.
__host__ __device__ inline int64_t tile_row(const ListsView &L, const Geom &G, size_t tile_idx, int64_t t, int pos) {
    if (L.rows) return L.rows[tile_idx * L.tile_rows + pos];
    const int64_t i = t * L.tile_rows + pos;
    return i < G.nq ? i : -1;
}

// Index of log w for (batch b, kv head r, query row i, chunk c) in the chunk-major
// layout [b][hkv][n_chunks][nq]: the rows of a tile that route one chunk sit together.
__host__ __device__ inline size_t logw_index(const Geom &G, int64_t b, int r, int64_t i, int c) {
    return (((size_t)b * G.hkv + r) * G.n_chunks + c) * (size_t)G.nq + i;
}

// Causal geometry of query row i: key position, own chunk, visible chunks.
__host__ __device__ inline int64_t row_pos(const Geom &G, int64_t i) { return i + G.pos0; }
// first chunk of row i's local window (causal): its own chunk, or the one before with local = 2
__host__ __device__ inline int first_local(const Geom &G, int64_t i) {
    const int64_t c = row_pos(G, i) / G.B - (G.local - 1);
    return (int)(c > 0 ? c : 0);
}
// chunks row i routes over: every chunk before its local window (all of them when non-causal)
__host__ __device__ inline int row_nvis(const Geom &G, int64_t i) {
    if (!G.causal) return G.n_chunks;
    const int c = first_local(G, i);
    return c < G.n_chunks ? c : G.n_chunks;
}

// ---------------------------------------------------------------------------
// Order of the query-tile CTAs of a Stage-2 launch.  The (batch, kv head) pairs are
// taken in groups whose K and V fit in about three quarters of the 126 MB L2 together
// (the rest holds the Q rows, biases and lists in flight); within a group
// the CTAs go longest tile (latest, causal) first across the group's pairs, so that
// the long tiles do not gather at the end of the launch, and the groups follow one
// another, so that the CTAs in flight read K and V that stay in L2.
// ---------------------------------------------------------------------------
struct TileOrder {
    int64_t t;   // tile index
    int64_t bh;  // batch * hkv + kv head
};
inline int heads_per_group(const Geom &G) {
    const double per_head = (double)G.nk * G.d * 2.0 * 2.0;  // K and V, bf16
    int hg = 1;
    while (hg * 2 <= G.b * G.hkv && (double)(hg * 2) * per_head <= 96.0 * (1 << 20)) hg *= 2;
    return hg;
}
__host__ __device__ inline TileOrder tile_order(int64_t cta, int64_t n_tiles, int64_t bh_total, int hg) {
    const int64_t per_group = (int64_t)hg * n_tiles;
    const int64_t gi = cta / per_group, local = cta % per_group;
    const int64_t hsz = bh_total - gi * hg < hg ? bh_total - gi * hg : hg;  // the last group may be smaller
    TileOrder o;
    o.t = n_tiles - 1 - local / hsz;
    o.bh = gi * hg + local % hsz;
    return o;
}

// ---------------------------------------------------------------------------
// Device error word: set by a kernel whose bounded wait ran out.  One word per
// translation unit (internal linkage, no device linking needed); the file that
// uses it exports a host function that reads and clears it.
// ---------------------------------------------------------------------------
static __device__ int g_dash_error;
constexpr int kErrTimeout = 1;

__device__ __forceinline__ void report_timeout() { atomicOr(&g_dash_error, kErrTimeout); }

static inline int take_device_error_local() {
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_dash_error, sizeof v) != cudaSuccess) return 0;
    if (v) {
        const int zero = 0;
        cudaMemcpyToSymbol(g_dash_error, &zero, sizeof zero);
    }
    return v;
}

// ---------------------------------------------------------------------------
// Small math helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
__device__ __forceinline__ int warp_sum_i(int v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

template <typename T>
__device__ __forceinline__ float to_f(T x);
template <>
__device__ __forceinline__ float to_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ T from_f(float x);
template <>
__device__ __forceinline__ float from_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

// ---------------------------------------------------------------------------
// mbarrier (shared memory) with bounded waits
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile(
        "{\n\t.reg .b64 st;\n\t"
        "mbarrier.arrive.release.cta.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar))
        : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile(
        "{\n\t.reg .b64 st;\n\t"
        "mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(smem_u32(bar)),
        "r"(bytes)
        : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait for phase `parity` of `bar` to complete, giving up after `limit`
// polls (each try_wait may itself suspend for a short hardware-defined time).
// Returns false (and sets the device error word) when the bound runs out.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, uint32_t limit) {
    for (uint32_t it = 0; it < limit; ++it)
        if (mbar_try_wait(bar, parity)) return true;
    report_timeout();
    return false;
}

__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Wait for phase `parity` of `bar`, giving up after limit_ns of wall time
// (global timer); on expiry the device error word is set and false returned.
__device__ __forceinline__ bool mbar_wait_ns(uint64_t *bar, uint32_t parity, uint64_t limit_ns) {
    uint64_t t0 = 0;
    for (uint32_t it = 0;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 255u) == 0) {
            const uint64_t now = global_ns();
            if (it == 0) t0 = now;
            else if (now - t0 > limit_ns) {
                report_timeout();
                return false;
            }
        }
    }
}

// ---------------------------------------------------------------------------
// Bounded waits of the warp-specialised tensor-core kernels (a CTA-wide abort flag in
// shared memory lets every role give up once one of them has timed out)
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint64_t gtimer() { return global_ns(); }

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// try_wait that lets the hardware suspend the thread for up to hint_ns while the phase
// is incomplete (it resumes as soon as the phase completes), so that waiting warps do not
// take issue slots from the warps that share their scheduler.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t *bar, uint32_t parity, uint32_t hint_ns) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
        : "memory");
    return ok != 0;
}
constexpr uint32_t kSleepNs = 100000;  // longest single suspension of a waiting thread

// Bounded wait.  Gives up after limit_ns (recording a device error and raising
// the CTA's abort flag) or, when honor_abort is set, as soon as another role
// has raised it.  Drain waits (copies or MMAs in flight) pass honor_abort = false.
__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity, uint64_t limit_ns, volatile int *abort,
                                         bool honor_abort = true) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = gtimer();
    for (;;) {
        if (mbar_try_wait_sleep(bar, parity, kSleepNs)) return true;
        if (gtimer() - t0 > limit_ns) {
            report_timeout();
            *abort = 1;
            return false;
        }
        if (honor_abort && *abort) return false;
    }
}

// Packed fp32 pairs (the f32x2 forms of fma / add on sm_100a): one instruction per two values.
__device__ __forceinline__ uint64_t f32x2(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f32x2_split(uint64_t v, float &lo, float &hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t fma_f32x2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t add_f32x2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

// ---------------------------------------------------------------------------
// TMA (tensor maps are built on the host; no multicast anywhere)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap *m) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}
__device__ __forceinline__ void tma_load_4d(void *dst, const CUtensorMap *m, uint64_t *bar, int c0, int c1, int c2,
                                            int c3) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(m)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(smem_u32(bar))
        : "memory");
}
// 1-D bulk copy global -> shared (16-byte aligned addresses, size multiple of 16)
__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// ---------------------------------------------------------------------------
// tcgen05 (5th-generation tensor core, accumulators in tensor memory)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t *dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// D[tmem] (+)= A[smem desc] * B[smem desc]
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// D[tmem] (+)= A[tmem] * B[smem desc]
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// Arrive on `bar` once every tcgen05 operation issued so far by this thread completes.
__device__ __forceinline__ void mma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

// Load 32 consecutive 32-bit columns of this thread's TMEM lane and wait for them.
// tcgen05.ld is asynchronous; the load and its wait sit in one asm statement so the
// compiler cannot read the destination registers before the data has arrived.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]),
          "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]),
          "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
}
// Load 16 consecutive 32-bit columns of this thread's TMEM lane and wait for them.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
}

// Store 32 consecutive 32-bit columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
        "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
        "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}
// Store 16 consecutive 32-bit columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor (tcgen05 format, version 1), 128-byte swizzle.
//   start: smem byte address; lbo/sbo: byte offsets (multiples of 16).
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t start, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((start >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;  // descriptor version for sm_100
    d |= (uint64_t)2 << 61;  // layout: 128-byte swizzle
    return d;
}

// Instruction descriptor for kind::f16 with bf16 A/B and f32 accumulation.
//   a_mn / b_mn: 1 if the operand is MN-major (else K-major).
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, int a_mn, int b_mn) {
    return (1u << 4)                     // D format f32
           | (1u << 7)                   // A format bf16
           | (1u << 10)                  // B format bf16
           | ((uint32_t)a_mn << 15)      // A major
           | ((uint32_t)b_mn << 16)      // B major
           | ((uint32_t)(N >> 3) << 17)  // N / 8
           | ((uint32_t)(M >> 4) << 24); // M / 16
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

}  // namespace dash

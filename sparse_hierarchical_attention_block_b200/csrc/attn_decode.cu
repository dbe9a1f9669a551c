// attn_decode.cu -- Stage 2 for decoding (a few query rows per sequence), split-KV.
//
// Same mathematics as the prefill kernels ("DashAttention" §3.4 Prop. 1, App. G
// Alg. 3): softmax over the routed chunks plus the diagonal chunk with the
// per-row routing bias.  With one query token per sequence a (batch, kv head)
// pair owns only g rows, so the work list is partitioned along KV across CTAs
// (the split-KV variant the paper's §3.5 describes for incremental decoding)
// and a second kernel merges the per-split (max, sum, O) partials.
//
// attn_decode_kernel: one CTA per (split of the list, kv head, batch), 4 warps; a split
//   takes 16 list entries, or 8 or 4 when few (batch, kv head) units would leave SMs idle.
//   thread 0 streams each listed chunk's K and V (TMA boxes, 128-byte swizzle)
//   into a ring of stages; each warp takes 16-key groups of the chunk and runs
//   its own online softmax on the 16-row mma.sync tile (rows = nq*g <= 16):
//   S = Q K^T, bias + mask, P (bf16) V into fp32 registers.  The warps' states
//   are merged in shared memory into the split's partial.  HBM-bound: the tensor
//   work per byte is tiny, the ring keeps ~64 KB per CTA in flight.
// combine_kernel: one CTA per (row, kv head, batch), a thread per column:
//   O = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s.
#include <math.h>

#include "dash_common.cuh"
#include "kernels.h"
#include "tma_host.h"

namespace dash {

namespace {

constexpr int kDecThreads = 128;
constexpr int kDecRows = 16;  // mma.sync M
constexpr int kEntriesPerSplit = 16;  // most list entries one split takes (shared-memory sizing)
constexpr uint64_t kDecWaitNs = 2000000000ull;

struct DecParams {
    CUtensorMap tmK, tmV;
};

__device__ __forceinline__ uint64_t gtimer_d() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ bool wait_full(uint64_t *bar, uint32_t parity) {
    uint64_t t0 = 0;
    for (uint32_t it = 0;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 255u) == 0) {
            const uint64_t now = gtimer_d();
            if (it == 0) t0 = now;
            else if (now - t0 > kDecWaitNs) {
                report_timeout();
                return false;
            }
        }
    }
}

__device__ __forceinline__ float ex2d(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void mma_bf16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Byte address of 16-byte chunk `chunk` (0..7) of row `row` in a 128-byte-swizzled region.
__device__ __forceinline__ uint32_t sw128(uint32_t region, int row, int chunk) {
    return region + row * 128 + ((chunk ^ (row & 7)) << 4);
}

template <int D, int BLK>
struct DecSmem {
    static constexpr int kDh = D / 64;
    static constexpr int kTile = kDh * BLK * 128;            // one operand of one chunk
    static constexpr int kStage = 2 * kTile;                 // K and V
    static constexpr int kNS = kStage >= 65536 ? 2 : (kStage >= 32768 ? 3 : 4);
    static constexpr int kRing = kNS * kStage;
    static constexpr int kMerge = 4 * kDecRows * (D + 2) * 4;  // per-warp states at the end
    static constexpr int kData = kRing > kMerge ? kRing : kMerge;
    static constexpr int kBars = kData;
    static constexpr int kIds = kBars + kNS * 8;                      // [kEntriesPerSplit] chunk ids
    static constexpr int kBias = kIds + kEntriesPerSplit * 4;         // [kEntriesPerSplit][kDecRows] bias (exp2 domain)
    static constexpr int kTotal = kBias + kEntriesPerSplit * kDecRows * 4;
};

template <int D, int BLK>
__global__ void __launch_bounds__(kDecThreads) attn_decode_kernel(const __grid_constant__ DecParams dp, TView Q,
                                                                  Geom G0, ListsView L, float *__restrict__ part,
                                                                  int nsplit, int eps) {
    using S = DecSmem<D, BLK>;
    Geom G = G0;
    geom_live(G);
    extern __shared__ uint8_t dsm_raw[];
    uint8_t *sm = dsm_raw + ((1024 - (smem_u32(dsm_raw) & 1023)) & 1023);
    uint64_t *full = reinterpret_cast<uint64_t *>(sm + S::kBars);

    const int split = blockIdx.x, r = blockIdx.y;
    const int64_t b = blockIdx.z;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int g = G.g, T = L.tile_rows;
    const int M = (int)G.nq * g;  // valid rows (nq * g <= 16)
    const size_t tile_idx = ((size_t)b * G.hkv + r) * L.n_tiles;
    const int count = L.count[tile_idx];
    const int e_begin = split * eps;  // eps <= kEntriesPerSplit entries per split
    if (e_begin >= count) return;  // the combine kernel ignores splits past the list
    const int e_end = min(count, e_begin + eps);
    const int n = e_end - e_begin;
    const int32_t *ids = L.ids + tile_idx * L.cap;
    const float *bias = L.bias + tile_idx * (size_t)L.cap * T;

    int *ids_s = reinterpret_cast<int *>(sm + S::kIds);
    float *bias_s = reinterpret_cast<float *>(sm + S::kBias);
    if (threadIdx.x == 0) {
        for (int s = 0; s < S::kNS; ++s) mbar_init(full + s, 1);
        fence_mbar_init();
    }
    // the split's chunk ids and per-row biases, read once (they would otherwise sit on
    // the critical path of every chunk)
    for (int idx = threadIdx.x; idx < n * kDecRows; idx += kDecThreads) {
        const int e = idx / kDecRows, row = idx % kDecRows;
        if (row == 0) ids_s[e] = ids[e_begin + e];
        bias_s[idx] = row < M ? bias[(size_t)(e_begin + e) * T + row / g] * 1.4426950408889634f : -INFINITY;
    }
    __syncthreads();
    const uint32_t ring = smem_u32(sm);
    auto issue = [&](int e, int st) {
        const int c = ids_s[e];
        uint8_t *kd = sm + st * S::kStage;
        mbar_arrive_expect_tx(full + st, (uint32_t)S::kStage);
        for (int dh = 0; dh < S::kDh; ++dh) {
            tma_load_4d(kd + dh * BLK * 128, &dp.tmK, full + st, dh * 64, r, c * BLK, (int)b);
            tma_load_4d(kd + S::kTile + dh * BLK * 128, &dp.tmV, full + st, dh * 64, r, c * BLK, (int)b);
        }
    };
    int issued = 0;  // entries whose copies thread 0 has issued
    if (threadIdx.x == 0) {
        tma_prefetch_desc(&dp.tmK);
        tma_prefetch_desc(&dp.tmV);
        for (int e = 0; e < min(n, S::kNS); ++e) issue(e, e);
        issued = min(n, S::kNS);
    }

    // Q fragments (A operand, rows >= M are zero)
    const int gr = lane >> 2, tq = lane & 3;
    uint32_t qa[D / 16][4];
    {
        const __nv_bfloat16 *qb = reinterpret_cast<const __nv_bfloat16 *>(Q.p) + b * Q.s0;
        auto qrow = [&](int m) -> const __nv_bfloat16 * {
            return qb + tile_row(L, G, tile_idx, 0, m / g) * Q.s1 + (int64_t)(r * g + m % g) * Q.s2;
        };
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                const int m = gr + (h & 1) * 8;
                const int col = kk * 16 + (h >> 1) * 8 + 2 * tq;
                qa[kk][h] = m < M ? *reinterpret_cast<const uint32_t *>(qrow(m) + col) : 0u;
            }
        }
    }
    const int row0 = gr, row1 = gr + 8;
    const int64_t p0 = row0 < M ? row_pos(G, tile_row(L, G, tile_idx, 0, row0 / g)) : -1;
    const int64_t p1 = row1 < M ? row_pos(G, tile_row(L, G, tile_idx, 0, row1 / g)) : -1;
    const float sl2 = rsqrtf((float)D) * 1.4426950408889634f;

    float o[D / 8][4];
#pragma unroll
    for (int x = 0; x < D / 8; ++x) o[x][0] = o[x][1] = o[x][2] = o[x][3] = 0.f;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    bool ok = true;
    int e_fail = n;

    for (int e = 0; e < n; ++e) {
        const int st = e % S::kNS;
        const int c = ids_s[e];
        const float b0 = bias_s[e * kDecRows + row0];
        const float b1 = bias_s[e * kDecRows + row1];
        ok = __syncthreads_and(wait_full(full + st, (e / S::kNS) & 1)) != 0;
        if (!ok) {
            e_fail = e;
            break;
        }
        const uint32_t kreg = ring + st * S::kStage;
        const uint32_t vreg = kreg + S::kTile;
        for (int kg = warp; kg < BLK / 16; kg += 4) {
            // ---- S = Q K^T for 16 keys
            float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const int mi = lane >> 3;
                const int kr = kg * 16 + (mi >> 1) * 8 + (lane & 7);
                const int dc = 2 * kk + (mi & 1);
                uint32_t r0, r1, r2, r3;
                ldsm_x4(sw128(kreg + (dc >> 3) * BLK * 128, kr, dc & 7), r0, r1, r2, r3);
                mma_bf16(acc[0], qa[kk], r0, r1);
                mma_bf16(acc[1], qa[kk], r2, r3);
            }
            // ---- bias, mask, online softmax (rows row0 and row1 of this thread)
            float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int x = 0; x < 4; ++x) {
                    const int kin = kg * 16 + nt * 8 + 2 * tq + (x & 1);
                    const int64_t key = (int64_t)c * BLK + kin;
                    const bool top = x < 2;
                    const int64_t pr = top ? p0 : p1;
                    const float bb = top ? b0 : b1;
                    const bool vis = pr >= 0 && key < G.nk && !(G.causal && key > pr);
                    const float v = vis ? fmaf(acc[nt][x], sl2, bb) : -INFINITY;
                    acc[nt][x] = v;
                    if (top) mx0 = fmaxf(mx0, v);
                    else mx1 = fmaxf(mx1, v);
                }
            mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
            mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
            mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
            mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
            const float n0 = fmaxf(m0, mx0), n1 = fmaxf(m1, mx1);
            const float c0 = n0 == -INFINITY ? 1.f : ex2d(m0 - n0);
            const float c1 = n1 == -INFINITY ? 1.f : ex2d(m1 - n1);
            m0 = n0;
            m1 = n1;
            float s0 = 0.f, s1 = 0.f;
            uint32_t pa[4];
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                const float q00 = n0 == -INFINITY ? 0.f : ex2d(acc[nt][0] - n0);
                const float q01 = n0 == -INFINITY ? 0.f : ex2d(acc[nt][1] - n0);
                const float q10 = n1 == -INFINITY ? 0.f : ex2d(acc[nt][2] - n1);
                const float q11 = n1 == -INFINITY ? 0.f : ex2d(acc[nt][3] - n1);
                s0 += q00 + q01;
                s1 += q10 + q11;
                pa[nt * 2 + 0] = pack_bf16x2(q00, q01);
                pa[nt * 2 + 1] = pack_bf16x2(q10, q11);
            }
            s0 += __shfl_xor_sync(0xffffffffu, s0, 1);
            s0 += __shfl_xor_sync(0xffffffffu, s0, 2);
            s1 += __shfl_xor_sync(0xffffffffu, s1, 1);
            s1 += __shfl_xor_sync(0xffffffffu, s1, 2);
            l0 = l0 * c0 + s0;
            l1 = l1 * c1 + s1;
            // A fragment of P: (row g, k 0-7), (row g+8, k 0-7), (row g, k 8-15), (row g+8, k 8-15)
            const uint32_t pfrag[4] = {pa[0], pa[1], pa[2], pa[3]};
            // ---- O = O * c + P V
#pragma unroll
            for (int dn = 0; dn < D / 8; dn += 2) {
                const int mi = lane >> 3;
                const int kr = kg * 16 + (mi & 1) * 8 + (lane & 7);
                const int dc = dn + (mi >> 1);
                uint32_t r0, r1, r2, r3;
                ldsm_x4_t(sw128(vreg + (dc >> 3) * BLK * 128, kr, dc & 7), r0, r1, r2, r3);
                o[dn][0] *= c0;
                o[dn][1] *= c0;
                o[dn][2] *= c1;
                o[dn][3] *= c1;
                o[dn + 1][0] *= c0;
                o[dn + 1][1] *= c0;
                o[dn + 1][2] *= c1;
                o[dn + 1][3] *= c1;
                mma_bf16(o[dn], pfrag, r0, r1);
                mma_bf16(o[dn + 1], pfrag, r2, r3);
            }
        }
        __syncthreads();  // every warp is done with stage st
        if (threadIdx.x == 0 && e + S::kNS < n) {
            issue(e + S::kNS, st);
            issued = e + S::kNS + 1;
        }
    }
    if (!ok) {
        // drain the copies still in flight (issued, not consumed) before the CTA exits
        if (threadIdx.x == 0)
            for (int e = e_fail; e < issued; ++e) wait_full(full + e % S::kNS, (e / S::kNS) & 1);
        __syncthreads();
        return;
    }

    // ---- merge the four warps' states (log2 domain) into the split's partial
    float *ms = reinterpret_cast<float *>(sm);          // [4][16] max
    float *ls = ms + 4 * kDecRows;                       // [4][16] sum
    float *os = ls + 4 * kDecRows;                       // [4][16][D] output
    if (tq == 0) {
        ms[warp * kDecRows + row0] = m0;
        ms[warp * kDecRows + row1] = m1;
        ls[warp * kDecRows + row0] = l0;
        ls[warp * kDecRows + row1] = l1;
    }
#pragma unroll
    for (int dn = 0; dn < D / 8; ++dn) {
        const int col = dn * 8 + 2 * tq;
        os[(warp * kDecRows + row0) * D + col] = o[dn][0];
        os[(warp * kDecRows + row0) * D + col + 1] = o[dn][1];
        os[(warp * kDecRows + row1) * D + col] = o[dn][2];
        os[(warp * kDecRows + row1) * D + col + 1] = o[dn][3];
    }
    __syncthreads();
    float *dst = part + (((size_t)b * G.hkv + r) * nsplit + split) * kDecRows * (D + 2);
    for (int idx = threadIdx.x; idx < M * (D + 2); idx += kDecThreads) {
        const int row = idx / (D + 2), col = idx % (D + 2);
        float mm = -INFINITY;
        for (int w = 0; w < 4; ++w) mm = fmaxf(mm, ms[w * kDecRows + row]);
        float acc = 0.f;
        for (int w = 0; w < 4; ++w) {
            const float mw = ms[w * kDecRows + row];
            const float f = mw == -INFINITY ? 0.f : ex2d(mw - mm);
            acc += f * (col == 0 ? 0.f : col == 1 ? ls[w * kDecRows + row] : os[(w * kDecRows + row) * D + col - 2]);
        }
        dst[(size_t)row * (D + 2) + col] = col == 0 ? mm : acc;
    }
}

// One CTA per (row, kv head, batch), one thread per output column: merge the row's
// split partials (max, sum, O) in the log2 domain.
template <int D>
__global__ void __launch_bounds__(D) combine_kernel(TView O, Geom G, ListsView L, const float *__restrict__ part,
                                                    int nsplit, int eps, float *lse) {
    const int row = blockIdx.x, r = blockIdx.y;
    const int64_t b = blockIdx.z;
    const int g = G.g;
    const int col = threadIdx.x;
    const int count = L.count[((size_t)b * G.hkv + r) * L.n_tiles];
    const int ns = min(nsplit, (count + eps - 1) / eps);
    const float *src = part + ((size_t)b * G.hkv + r) * nsplit * kDecRows * (D + 2) + (size_t)row * (D + 2);
    constexpr size_t kStride = (size_t)kDecRows * (D + 2);  // from one split's partial of this row to the next
    float mm = -INFINITY;
#pragma unroll 4
    for (int s = 0; s < ns; ++s) mm = fmaxf(mm, src[s * kStride]);
    float num = 0.f, den = 0.f;
#pragma unroll 4
    for (int s = 0; s < ns; ++s) {
        const float *p = src + s * kStride;
        const float f = p[0] == -INFINITY ? 0.f : ex2d(p[0] - mm);
        den += f * p[1];
        num += f * p[2 + col];
    }
    const int64_t i = tile_row(L, G, ((size_t)b * G.hkv + r) * L.n_tiles, 0, row / g);
    __nv_bfloat16 *op = reinterpret_cast<__nv_bfloat16 *>(const_cast<void *>(O.p)) + b * O.s0 + i * O.s1 +
                        (int64_t)(r * g + row % g) * O.s2;
    op[col] = __float2bfloat16_rn(den > 0.f ? num / den : 0.f);
    if (lse && col == 0)  // natural log of the row's normaliser (log2 domain partials)
        lse[((size_t)b * G.nq_lse + i) * G.hq + r * g + row % g] =
            den > 0.f ? (mm + __log2f(den)) * 0.6931471805599453f : -INFINITY;
}

// List entries per split: 16, or fewer when the (batch, kv head) units are few, so that
// the splits a list may need still give every SM several CTAs (16 per SM for lists
// that route a sixteenth of their chunks).  The SM count is B200's 148 as a constant,
// not the current device's: the split count sizes the partials in the workspace, and a
// fixed count keeps dash_workspace_bytes() independent of the device (on a part with
// fewer SMs the splits stay correct, only their balance changes).
int entries_per_split(const Geom &G) {
    const int64_t units = G.b * (int64_t)G.hkv;
    for (int eps = kEntriesPerSplit; eps > 4; eps /= 2)
        if ((int64_t)((G.n_blk + eps - 1) / eps) * units >= 16 * 148) return eps;
    return 4;
}

int n_splits(const Geom &G) {
    const int eps = entries_per_split(G);
    return (G.n_blk + eps - 1) / eps;
}

template <int D, int BLK>
cudaError_t launch_dec(const DecParams &dp, const TView &Q, const TView &O, const Geom &G, const ListsView &L,
                       float *part, cudaStream_t st, float *lse) {
    using S = DecSmem<D, BLK>;
    const size_t smem = S::kTotal + 1024;
    cudaError_t e = cudaFuncSetAttribute(attn_decode_kernel<D, BLK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    const int ns = n_splits(G), eps = entries_per_split(G);
    attn_decode_kernel<D, BLK><<<dim3((unsigned)ns, (unsigned)G.hkv, (unsigned)G.b), kDecThreads, smem, st>>>(
        dp, Q, G, L, part, ns, eps);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    combine_kernel<D><<<dim3((unsigned)(G.nq * G.g), (unsigned)G.hkv, (unsigned)G.b), D, 0, st>>>(O, G, L, part,
                                                                                                   ns, eps, lse);
    return cudaGetLastError();
}

}  // namespace

bool attn_decode_supported(const Geom &G, dash_dtype_t dt) {
    if (dt != DASH_BF16) return false;
    if (G.d != 64 && G.d != 128) return false;
    if (G.nq * G.g > kDecRows || G.n_tiles != 1) return false;
    return tma_encode_fn() != nullptr;
}

size_t attn_decode_workspace(const Geom &G) {
    return (size_t)G.b * G.hkv * n_splits(G) * kDecRows * (G.d + 2) * sizeof(float);
}

cudaError_t launch_attn_decode(const TView &Q, const TView &K, const TView &V, const TView &O, const Geom &G,
                               const ListsView &L, void *work, cudaStream_t st, float *lse) {
    if (G.nq == 0 || G.b == 0) return cudaSuccess;
    DecParams dp;
    if (!make_map_bf16(&dp.tmK, K, G.b, G.nk, G.hkv, G.d, 1, G.B)) return cudaErrorInvalidValue;
    if (!make_map_bf16(&dp.tmV, V, G.b, G.nk, G.hkv, G.d, 1, G.B)) return cudaErrorInvalidValue;
    float *part = static_cast<float *>(work);
#define DASH_DEC_CASE(DD, BB) \
    if (G.d == DD && G.B == BB) return launch_dec<DD, BB>(dp, Q, O, G, L, part, st, lse);
    DASH_DEC_CASE(128, 64)
    DASH_DEC_CASE(128, 128)
    DASH_DEC_CASE(128, 32)
    DASH_DEC_CASE(128, 16)
    DASH_DEC_CASE(64, 64)
    DASH_DEC_CASE(64, 128)
    DASH_DEC_CASE(64, 32)
    DASH_DEC_CASE(64, 16)
#undef DASH_DEC_CASE
    return cudaErrorNotSupported;
}

int take_device_error_decode() { return take_device_error_local(); }

}  // namespace dash

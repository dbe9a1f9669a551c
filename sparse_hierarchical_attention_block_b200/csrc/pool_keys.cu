// pool_keys.cu -- Stage 0: chunk summaries.
//
// k̄_c^(r) = sum_{t in chunk c} softmax_t(<q̄_c^(r), k_t>/sqrt(d)) k_t
// ("DashAttention" §3.1 Eq. 3 and App. G Alg. 1).  With the summary query at its
// initial value q̄ = 0 the weights are uniform and k̄_c is the plain mean of the
// chunk's keys (pool_keys_kernel); a learned q̄ (pool_keys_q_kernel) weights the
// keys by an online softmax in which the keys also serve as the values.  A
// trailing partial chunk (non-causal routing only) is pooled over its real keys.
//
// HBM-bound: one pass over K with coalesced loads, fp32 accumulation, fp32
// output [b][n_chunks][hkv][d].
#include "dash_common.cuh"
#include "kernels.h"

namespace dash {

// With a device-resident length (G.chunks_dev set), chunk c0 is counted from the first
// chunk the cache has not pooled and chunks that are not complete yet are skipped.
template <typename T>
__global__ void __launch_bounds__(256) pool_keys_kernel(TView K, Geom G0, float *__restrict__ kbar, int c0) {
    constexpr int VEC = 16 / sizeof(T);  // elements per 16-byte load
    Geom G = G0;
    geom_live(G);
    int c = c0 + (int)blockIdx.x;
    if (G.chunks_dev) {
        c += *G.chunks_dev;
        if (c >= G.n_chunks) return;
    }
    const int64_t b = blockIdx.y;
    const int ncol = G.hkv * G.d / VEC;  // 16-byte column groups of one token row
    const int rs = ncol >= 256 ? 1 : 256 / ncol;
    const int64_t t0 = (int64_t)c * G.B;
    int64_t t1 = t0 + G.B;
    if (t1 > G.nk) t1 = G.nk;
    const int cnt = (int)(t1 - t0);

    extern __shared__ float part[];  // [rs][ncol][VEC] when rs > 1
    const T *base = reinterpret_cast<const T *>(K.p) + b * K.s0;

    for (int cg0 = 0; cg0 < ncol; cg0 += 256 / rs) {
        const int cg = cg0 + (int)threadIdx.x % (256 / rs);
        const int sub = (int)threadIdx.x / (256 / rs);
        float acc[VEC];
#pragma unroll
        for (int e = 0; e < VEC; ++e) acc[e] = 0.f;
        if (cg < ncol && sub < rs) {
            const int r = cg * VEC / G.d;
            const int e0 = cg * VEC % G.d;
            const T *p = base + r * K.s2 + e0;
            int t = sub;
#pragma unroll 4
            for (; t < cnt; t += rs) {
                uint4 raw = *reinterpret_cast<const uint4 *>(p + (t0 + t) * K.s1);
                const T *v = reinterpret_cast<const T *>(&raw);
#pragma unroll
                for (int e = 0; e < VEC; ++e) acc[e] += to_f<T>(v[e]);
            }
        }
        if (rs > 1) {
            if (cg < ncol && sub < rs)
#pragma unroll
                for (int e = 0; e < VEC; ++e) part[((size_t)sub * ncol + cg) * VEC + e] = acc[e];
            __syncthreads();
            if (sub == 0 && cg < ncol) {
                for (int s = 1; s < rs; ++s)
#pragma unroll
                    for (int e = 0; e < VEC; ++e) acc[e] += part[((size_t)s * ncol + cg) * VEC + e];
            }
            __syncthreads();
        }
        if (sub == 0 && cg < ncol) {
            const float inv = 1.f / (float)cnt;
            float *o = kbar + (((size_t)b * G.kbar_cap + c) * G.hkv) * G.d + (size_t)cg * VEC;
#pragma unroll
            for (int e = 0; e < VEC; e += 4)
                *reinterpret_cast<float4 *>(o + e) =
                    make_float4(acc[e] * inv, acc[e + 1] * inv, acc[e + 2] * inv, acc[e + 3] * inv);
        }
    }
}

cudaError_t launch_pool_keys(const TView &K, dash_dtype_t dt, const Geom &G, float *kbar, cudaStream_t st, int c0,
                             int c1) {
    if (c1 < 0) c1 = G.n_chunks;
    if (c1 <= c0 || G.b == 0) return cudaSuccess;
    dim3 grid((unsigned)(c1 - c0), (unsigned)G.b);
    const int vec = dt == DASH_BF16 ? 8 : 4;
    const int ncol = G.hkv * G.d / vec;
    const int rs = ncol >= 256 ? 1 : 256 / ncol;
    const size_t smem = rs > 1 ? (size_t)rs * ncol * vec * sizeof(float) : 0;
    if (dt == DASH_BF16)
        pool_keys_kernel<__nv_bfloat16><<<grid, 256, smem, st>>>(K, G, kbar, c0);
    else
        pool_keys_kernel<float><<<grid, 256, smem, st>>>(K, G, kbar, c0);
    return cudaGetLastError();
}

// After a device-range pooling step: the cache has pooled the chunks up to the live
// count, or kMaxNewChunks more than before, whichever is fewer.
__global__ void cache_advance_kernel(Geom G0, int *done, int max_new) {
    Geom G = G0;
    geom_live(G);
    const int d = *done;
    const int n = min(G.n_chunks, d + max_new);
    if (n > d) *done = n;
}

__global__ void set_int_kernel(int *dst, int v) { *dst = v; }

cudaError_t launch_set_int(int *dst, int v, cudaStream_t st) {
    set_int_kernel<<<1, 1, 0, st>>>(dst, v);
    return cudaGetLastError();
}

cudaError_t launch_cache_catch_up(const TView &K, dash_dtype_t dt, const Geom &G, float *kbar, uint8_t *split,
                                  cudaStream_t st) {
    if (!G.nk_dev || !G.chunks_dev || G.b == 0) return cudaErrorInvalidValue;
    cudaError_t e = launch_pool_keys(K, dt, G, kbar, st, 0, kMaxNewChunks);
    if (e != cudaSuccess) return e;
    // the new chunks fall in at most two 128-chunk tiles of the split form
    if ((e = launch_kbar_split(kbar, G, split, 0, kMaxNewChunks / 128 + 2, st)) != cudaSuccess) return e;
    cache_advance_kernel<<<1, 1, 0, st>>>(G, const_cast<int *>(G.chunks_dev), kMaxNewChunks);
    return cudaGetLastError();
}

// The raw bytes of EPL consecutive elements of one row (the row start is 16-byte
// aligned, so each lane's piece is aligned to its own size), and their values.
template <typename T, int EPL> struct Piece;
template <> struct Piece<__nv_bfloat16, 4> {
    using raw_t = uint2;
    static __device__ __forceinline__ void cvt(const raw_t &r, float (&v)[4]) {
        const __nv_bfloat16 *e = reinterpret_cast<const __nv_bfloat16 *>(&r);
#pragma unroll
        for (int x = 0; x < 4; ++x) v[x] = __bfloat162float(e[x]);
    }
};
template <> struct Piece<__nv_bfloat16, 2> {
    using raw_t = uint32_t;
    static __device__ __forceinline__ void cvt(const raw_t &r, float (&v)[2]) {
        const __nv_bfloat16 *e = reinterpret_cast<const __nv_bfloat16 *>(&r);
        v[0] = __bfloat162float(e[0]);
        v[1] = __bfloat162float(e[1]);
    }
};
template <> struct Piece<float, 4> {
    using raw_t = float4;
    static __device__ __forceinline__ void cvt(const raw_t &r, float (&v)[4]) { v[0] = r.x, v[1] = r.y, v[2] = r.z, v[3] = r.w; }
};
template <> struct Piece<float, 2> {
    using raw_t = float2;
    static __device__ __forceinline__ void cvt(const raw_t &r, float (&v)[2]) { v[0] = r.x, v[1] = r.y; }
};

// Learned summary query: one warp per (chunk, kv head), lane l holding elements
// l*EPL .. l*EPL+EPL-1 of q̄ and of the running sum.  Keys are taken kBatch at a
// time (independent dot products, one butterfly reduction each) while the next
// batch's loads are already in flight, then one online softmax update: m running
// maximum (exp2 domain), l running sum of 2^(s - m).
template <typename T, typename TQ, int D>
__global__ void __launch_bounds__(256) pool_keys_q_kernel(TView K, TView QB, Geom G, float *__restrict__ kbar, int c0,
                                                          int c1) {
    constexpr int EPL = D / 32;
    using PK = Piece<T, EPL>;
    using PQ = Piece<TQ, EPL>;
    using raw_t = typename PK::raw_t;
    // keys per batch: 16 registers of raw data per buffer (the converted values of a
    // batch stay live through its reduction as well)
    constexpr int kRegsPerKey = (int)(sizeof(raw_t) / 4);
    constexpr int kBatch = 16 / kRegsPerKey;
    const int warp = (int)threadIdx.x / 32, lane = (int)threadIdx.x % 32;
    const int64_t unit = (int64_t)blockIdx.x * 8 + warp;
    if (unit >= (int64_t)(c1 - c0) * G.hkv) return;  // whole warps only
    const int c = c0 + (int)(unit / G.hkv), r = (int)(unit % G.hkv);
    const int64_t b = blockIdx.y;
    const int64_t t0 = (int64_t)c * G.B;
    const int64_t t1 = t0 + G.B < G.nk ? t0 + G.B : G.nk;
    const T *kp = reinterpret_cast<const T *>(K.p) + b * K.s0 + r * K.s2 + lane * EPL;

    raw_t cur[kBatch], nxt[kBatch] = {};
    auto load_batch = [&](int64_t tb, raw_t (&dst)[kBatch]) {
#pragma unroll
        for (int j = 0; j < kBatch; ++j)
            if (tb + j < t1) dst[j] = *reinterpret_cast<const raw_t *>(kp + (tb + j) * K.s1);
    };
    load_batch(t0, nxt);

    float qv[EPL];
    PQ::cvt(*reinterpret_cast<const typename PQ::raw_t *>(reinterpret_cast<const TQ *>(QB.p) + b * QB.s0 +
                                                           c * QB.s1 + r * QB.s2 + lane * EPL),
            qv);
    const float qscale = rsqrtf((float)D) * 1.4426950408889634f;  // scores in the exp2 domain
#pragma unroll
    for (int x = 0; x < EPL; ++x) qv[x] *= qscale;

    float m = -INFINITY, l = 0.f, acc[EPL];
#pragma unroll
    for (int x = 0; x < EPL; ++x) acc[x] = 0.f;
    for (int64_t tb = t0; tb < t1; tb += kBatch) {
#pragma unroll
        for (int j = 0; j < kBatch; ++j) cur[j] = nxt[j];
        if (tb + kBatch < t1) load_batch(tb + kBatch, nxt);
        float s[kBatch];
#pragma unroll
        for (int j = 0; j < kBatch; ++j) {
            float kv[EPL];
            PK::cvt(cur[j], kv);
            s[j] = 0.f;
#pragma unroll
            for (int x = 0; x < EPL; ++x) s[j] = fmaf(qv[x], kv[x], s[j]);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1)
#pragma unroll
            for (int j = 0; j < kBatch; ++j) s[j] += __shfl_xor_sync(0xffffffffu, s[j], off);
        float mb = -INFINITY;
#pragma unroll
        for (int j = 0; j < kBatch; ++j) {
            if (tb + j >= t1) s[j] = -INFINITY;
            mb = fmaxf(mb, s[j]);
        }
        const float mn = fmaxf(m, mb);
        const float f = exp2f(m - mn);  // 0 on the first batch (m = -inf)
        l *= f;
#pragma unroll
        for (int x = 0; x < EPL; ++x) acc[x] *= f;
#pragma unroll
        for (int j = 0; j < kBatch; ++j) {
            if (tb + j < t1) {
                const float p = exp2f(s[j] - mn);
                float kv[EPL];
                PK::cvt(cur[j], kv);
                l += p;
#pragma unroll
                for (int x = 0; x < EPL; ++x) acc[x] = fmaf(p, kv[x], acc[x]);
            }
        }
        m = mn;
    }
    const float inv = 1.f / l;
    float *o = kbar + (((size_t)b * G.kbar_cap + c) * G.hkv + r) * D + lane * EPL;
    if constexpr (EPL == 4)
        *reinterpret_cast<float4 *>(o) = make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
    else
        *reinterpret_cast<float2 *>(o) = make_float2(acc[0] * inv, acc[1] * inv);
}

template <typename T, typename TQ>
cudaError_t launch_pool_q_t(const TView &K, const TView &QB, const Geom &G, float *kbar, cudaStream_t st, int c0,
                            int c1) {
    const int64_t units = (int64_t)(c1 - c0) * G.hkv;
    dim3 grid((unsigned)((units + 7) / 8), (unsigned)G.b);
    if (G.d == 128)
        pool_keys_q_kernel<T, TQ, 128><<<grid, 256, 0, st>>>(K, QB, G, kbar, c0, c1);
    else
        pool_keys_q_kernel<T, TQ, 64><<<grid, 256, 0, st>>>(K, QB, G, kbar, c0, c1);
    return cudaGetLastError();
}

cudaError_t launch_pool_keys_q(const TView &K, dash_dtype_t dt, const TView &Qbar, dash_dtype_t qdt, const Geom &G,
                               float *kbar, cudaStream_t st, int c0, int c1) {
    if (c1 < 0) c1 = G.n_chunks;
    if (c1 <= c0 || G.b == 0) return cudaSuccess;
    if (G.d != 64 && G.d != 128) return cudaErrorInvalidValue;
    if (dt == DASH_BF16)
        return qdt == DASH_BF16 ? launch_pool_q_t<__nv_bfloat16, __nv_bfloat16>(K, Qbar, G, kbar, st, c0, c1)
                                : launch_pool_q_t<__nv_bfloat16, float>(K, Qbar, G, kbar, st, c0, c1);
    return qdt == DASH_BF16 ? launch_pool_q_t<float, __nv_bfloat16>(K, Qbar, G, kbar, st, c0, c1)
                            : launch_pool_q_t<float, float>(K, Qbar, G, kbar, st, c0, c1);
}

}  // namespace dash

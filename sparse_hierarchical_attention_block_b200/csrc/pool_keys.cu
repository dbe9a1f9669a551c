// pool_keys.cu -- Stage 0: chunk summaries.
//
// k̄_c^(r) = sum_{t in chunk c} softmax_t(<q̄^(r), k_t>/sqrt(d)) k_t with the
// summary query q̄ = 0 (its initial value), i.e. the plain mean of the chunk's
// keys ("DashAttention" §3.1 Eq. 3 and App. G Alg. 1).  A trailing partial chunk
// (non-causal routing only) is the mean of its real keys.
//
// HBM-bound: one pass over K with 16-byte coalesced loads, fp32 accumulation,
// fp32 output [b][n_chunks][hkv][d].
#include "dash_common.cuh"
#include "kernels.h"

namespace dash {

template <typename T>
__global__ void __launch_bounds__(256) pool_keys_kernel(TView K, Geom G, float *__restrict__ kbar) {
    constexpr int VEC = 16 / sizeof(T);  // elements per 16-byte load
    const int c = blockIdx.x;
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
            float *o = kbar + (((size_t)b * G.n_chunks + c) * G.hkv) * G.d + (size_t)cg * VEC;
#pragma unroll
            for (int e = 0; e < VEC; e += 4)
                *reinterpret_cast<float4 *>(o + e) =
                    make_float4(acc[e] * inv, acc[e + 1] * inv, acc[e + 2] * inv, acc[e + 3] * inv);
        }
    }
}

cudaError_t launch_pool_keys(const TView &K, dash_dtype_t dt, const Geom &G, float *kbar, cudaStream_t st) {
    if (G.n_chunks == 0 || G.b == 0) return cudaSuccess;
    dim3 grid((unsigned)G.n_chunks, (unsigned)G.b);
    const int vec = dt == DASH_BF16 ? 8 : 4;
    const int ncol = G.hkv * G.d / vec;
    const int rs = ncol >= 256 ? 1 : 256 / ncol;
    const size_t smem = rs > 1 ? (size_t)rs * ncol * vec * sizeof(float) : 0;
    if (dt == DASH_BF16)
        pool_keys_kernel<__nv_bfloat16><<<grid, 256, smem, st>>>(K, G, kbar);
    else
        pool_keys_kernel<float><<<grid, 256, smem, st>>>(K, G, kbar);
    return cudaGetLastError();
}

}  // namespace dash

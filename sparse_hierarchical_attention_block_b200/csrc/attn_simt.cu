// attn_simt.cu -- Stage 2 on CUDA cores (any dtype, d in {64, 128}, any block size).
//
// Prior-induced sparse softmax in the bias form of "DashAttention" §3.4 Prop. 1:
// for query row i of head h (KV group r),
//   o_i = sum_j exp(z_ij + d_ij) v_j / sum_t exp(z_it + d_it),  z_ij = <q_i, k_j>/sqrt(d)
// over the keys of the chunks in the tile's list; d_ij is the list's per-row bias
// (-inf: not attended) and keys j > p_i are masked when causal (App. G Alg. 3).
// Online (flash) softmax in fp32, exp2 domain.
//
// One CTA per (batch, kv head, query tile); thread m owns row m = pos * g + head.
// This is the fp32 path and the reference for the tensor-core kernel; it is not
// the fast path for bf16.
#include <math.h>

#include "dash_common.cuh"
#include "kernels.h"

namespace dash {

namespace {

constexpr int kSimtRows = 128;
constexpr int kSub = 32;  // keys staged per step

template <typename T>
__global__ void __launch_bounds__(kSimtRows) attn_simt_kernel(TView Q, TView K, TView V, TView O, Geom G,
                                                              ListsView L, float *lse) {
    extern __shared__ __align__(16) float sm[];
    const int d = G.d, g = G.g, dp = d + 1;
    float *Qs = sm;                        // [128][d+1]
    float *Os = Qs + kSimtRows * dp;       // [128][d+1]
    float *Ks = Os + kSimtRows * dp;       // [kSub][d+1]
    float *Vs = Ks + kSub * dp;            // [kSub][d+1]

    const int64_t t = blockIdx.x;
    const int r = blockIdx.y;
    const int64_t b = blockIdx.z;
    const int TR = L.tile_rows;
    const int M = TR * g;
    const int m = threadIdx.x;
    const int pos = m / g, hh = m % g;
    const size_t tile_idx = ((size_t)b * G.hkv + r) * L.n_tiles + t;
    const int64_t i = m < M ? tile_row(L, G, tile_idx, t, pos) : -1;
    const bool valid = i >= 0;
    const int64_t p_i = row_pos(G, i);

    const T *qb = reinterpret_cast<const T *>(Q.p) + b * Q.s0;
    const T *kbp = reinterpret_cast<const T *>(K.p) + b * K.s0 + (int64_t)r * K.s2;
    const T *vbp = reinterpret_cast<const T *>(V.p) + b * V.s0 + (int64_t)r * V.s2;

    for (int e = 0; e < d; ++e) {
        Qs[m * dp + e] = valid ? to_f<T>(qb[i * Q.s1 + (int64_t)(r * g + hh) * Q.s2 + e]) : 0.f;
        Os[m * dp + e] = 0.f;
    }
    const float sl2 = rsqrtf((float)d) * 1.4426950408889634f;  // 1/sqrt(d) * log2(e)
    float mrun = -INFINITY, lrun = 0.f;

    const int count = L.count[tile_idx];
    const int32_t *ids = L.ids + tile_idx * L.cap;
    const float *bias = L.bias + tile_idx * (size_t)L.cap * TR;

    for (int e_idx = 0; e_idx < count; ++e_idx) {
        const int c = ids[e_idx];
        const float bv = (m < M) ? bias[(size_t)e_idx * TR + pos] * 1.4426950408889634f : -INFINITY;
        const int64_t k0 = (int64_t)c * G.B;
        for (int j0 = 0; j0 < G.B; j0 += kSub) {
            __syncthreads();
            for (int idx = threadIdx.x; idx < kSub * d; idx += kSimtRows) {
                const int jj = idx / d, e = idx % d;
                const int64_t key = k0 + j0 + jj;
                const bool in = (j0 + jj < G.B) && key < G.nk;
                Ks[jj * dp + e] = in ? to_f<T>(kbp[key * K.s1 + e]) : 0.f;
                Vs[jj * dp + e] = in ? to_f<T>(vbp[key * V.s1 + e]) : 0.f;
            }
            __syncthreads();
            if (!valid || bv == -INFINITY) continue;
            float s[kSub];
            float smax = -INFINITY;
#pragma unroll
            for (int jj = 0; jj < kSub; ++jj) {
                const int64_t key = k0 + j0 + jj;
                float acc = 0.f;
                for (int e = 0; e < d; ++e) acc = fmaf(Qs[m * dp + e], Ks[jj * dp + e], acc);
                float v = acc * sl2 + bv;
                if (j0 + jj >= G.B || key >= G.nk || (G.causal && key > p_i)) v = -INFINITY;
                s[jj] = v;
                smax = fmaxf(smax, v);
            }
            if (smax == -INFINITY) continue;
            const float mnew = fmaxf(mrun, smax);
            const float corr = exp2f(mrun - mnew);  // 0 when mrun = -inf
            float psum = 0.f;
#pragma unroll
            for (int jj = 0; jj < kSub; ++jj) {
                s[jj] = exp2f(s[jj] - mnew);
                psum += s[jj];
            }
            lrun = lrun * corr + psum;
            mrun = mnew;
            for (int e = 0; e < d; ++e) {
                float acc = Os[m * dp + e] * corr;
#pragma unroll
                for (int jj = 0; jj < kSub; ++jj) acc = fmaf(s[jj], Vs[jj * dp + e], acc);
                Os[m * dp + e] = acc;
            }
        }
    }
    if (valid) {
        T *ob = reinterpret_cast<T *>(const_cast<void *>(O.p)) + b * O.s0 + i * O.s1 + (int64_t)(r * g + hh) * O.s2;
        const float inv = lrun > 0.f ? 1.f / lrun : 0.f;
        for (int e = 0; e < d; ++e) ob[e] = from_f<T>(Os[m * dp + e] * inv);
        if (lse)  // natural log of the row's normaliser: (m + log2 l) ln 2
            lse[((size_t)b * G.nq_lse + i) * G.hq + r * g + hh] =
                lrun > 0.f ? (mrun + log2f(lrun)) * 0.6931471805599453f : -INFINITY;
    }
}

}  // namespace

cudaError_t launch_attn_simt(const TView &Q, const TView &K, const TView &V, const TView &O, dash_dtype_t dt,
                             const Geom &G, const ListsView &L, cudaStream_t st, float *lse) {
    if (G.nq == 0 || G.b == 0) return cudaSuccess;
    const size_t smem = (size_t)(2 * kSimtRows + 2 * kSub) * (G.d + 1) * sizeof(float);
    dim3 grid((unsigned)L.n_tiles, (unsigned)G.hkv, (unsigned)G.b);
    cudaError_t e;
    if (dt == DASH_BF16) {
        e = cudaFuncSetAttribute(attn_simt_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem);
        if (e != cudaSuccess) return e;
        attn_simt_kernel<__nv_bfloat16><<<grid, kSimtRows, smem, st>>>(Q, K, V, O, G, L, lse);
    } else {
        e = cudaFuncSetAttribute(attn_simt_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        attn_simt_kernel<float><<<grid, kSimtRows, smem, st>>>(Q, K, V, O, G, L, lse);
    }
    return cudaGetLastError();
}

}  // namespace dash

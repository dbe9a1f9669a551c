// tma_host.h -- host-side TMA tensor-map construction (driver entry point obtained
// through the runtime, so the library needs no link-time libcuda).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include "dash_common.cuh"

namespace dash {

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn tma_encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// 4-D bf16 map over a [b][seq][heads][d] tensor (dims innermost first), box
// {64, box_h, box_s, 1} (64 columns = one 128-byte swizzle row), 128-byte swizzle,
// out-of-range elements read as zero.
inline bool make_map_bf16(CUtensorMap *m, const TView &v, int64_t b, int64_t seq, int64_t heads, int d, int box_h,
                          int box_s) {
    EncodeTiledFn fn = tma_encode_fn();
    if (!fn) return false;
    cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)heads, (cuuint64_t)seq, (cuuint64_t)b};
    cuuint64_t strides[3] = {(cuuint64_t)v.s2 * 2, (cuuint64_t)v.s1 * 2, (cuuint64_t)v.s0 * 2};
    if (b == 1) strides[2] = (cuuint64_t)seq * v.s1 * 2;  // extent 1: any valid stride
    cuuint32_t box[4] = {64, (cuuint32_t)box_h, (cuuint32_t)box_s, 1};
    cuuint32_t es[4] = {1, 1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(v.p), dims, strides, box, es,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace dash

// attn_bwd_tc.cu -- Stage-2 backward on the 5th-generation tensor cores (placeholder:
// the CUDA-core kernels of bwd.cu serve every shape until these are in place).
#include "dash_common.cuh"
#include "kernels.h"

namespace dash {

bool attn_bwd_tc_supported(const Geom &, dash_dtype_t) { return false; }
cudaError_t launch_attn_bwd_tc_dq(const BwdArgs &, cudaStream_t) { return cudaErrorNotSupported; }
cudaError_t launch_attn_bwd_tc_dkdv(const BwdArgs &, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace dash

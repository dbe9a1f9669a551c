// attn_decode.cu -- Stage 2 split-KV decode (placeholder until the kernel lands).
#include "dash_common.cuh"
#include "kernels.h"

namespace dash {
bool attn_decode_supported(const Geom &, dash_dtype_t) { return false; }
size_t attn_decode_workspace(const Geom &) { return 0; }
cudaError_t launch_attn_decode(const TView &, const TView &, const TView &, const TView &, const Geom &,
                               const ListsView &, void *, cudaStream_t) {
    return cudaErrorNotSupported;
}
int take_device_error_decode() { return take_device_error_local(); }
}  // namespace dash

// noalloc.cu -- dash_attn_fwd_noalloc: the full forward pass on a scratch area
// that lives in the library's own static device memory, so that the call itself
// allocates nothing.
//
// Who needs it: callers that cannot let a library call cudaMalloc/cudaFree.
//   - Serving engines that reserve almost all of HBM up front for their KV-cache
//     pool: a workspace allocation at run time can fail for lack of memory even
//     though the attention itself fits.
//   - Latency-sensitive loops that run several streams at once: cudaFree (and a
//     cudaMalloc that has to grow the heap) synchronises the whole device, which
//     stalls every other stream of the process.
//   - Hosts that route all device memory through their own allocator and do
//     not want a second, library-owned heap beside it.
// Such a caller still passes q, k, v and out (its own memory) and gets the same
// result as dash_attn_fwd_ex; only the intermediates (chunk summaries, routing
// masks, work lists, split-KV partials) go to the static area below.
//
// The area is a file-scope __device__ array of DASH_NOALLOC_SCRATCH_BYTES.  The
// CUDA runtime reserves it on every device that loads this library, for the
// life of the process.  In host code its name only stands for the symbol: the
// device address is looked up with cudaGetSymbolAddress, once per device, on
// the first call made while that device is current (that first call should come
// before any stream capture).  The address stays valid for the life of the device's
// primary context: after cudaDeviceReset the old address must not be used, so this
// entry point is not to be called again in a process that reset a device.  All
// calls share the one area and it keeps the last call's contents; the forward pass
// writes every scratch word it reads before reading it, so nothing has to be
// cleared between calls.  Calls whose execution overlaps on the GPU (two streams,
// or two host threads) race on the area: serialise them.
#include <stdio.h>

#include <mutex>

#include "dash_common.cuh"
#include "kernels.h"

namespace dash {
int report_error(int code, const char *msg);
int fwd_workspace_need(const dash_tensor_t *q, const dash_tensor_t *k, const dash_tensor_t *v,
                       const dash_tensor_t *out, int block_size, float alpha, int causal, int gqa_groups,
                       const dash_opts_t *opts, size_t budget, size_t *need);
}  // namespace dash

namespace {

__device__ __align__(256) unsigned char g_noalloc_scratch[DASH_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 128;
std::mutex g_noalloc_mu;
void *g_noalloc_ptr[kMaxDevices];  // device address of g_noalloc_scratch, per device

// Device address of the static area on the current device (looked up once).
int noalloc_scratch(void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return dash::report_error(DASH_ERR_CUDA, cudaGetErrorString(e));
    if (dev < 0 || dev >= kMaxDevices) return dash::report_error(DASH_ERR_UNSUPPORTED, "device index out of range");
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || !p)
            return dash::report_error(DASH_ERR_CUDA, e != cudaSuccess ? cudaGetErrorString(e)
                                                                       : "cudaGetSymbolAddress returned NULL");
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return DASH_OK;
}

}  // namespace

extern "C" {

DASH_API int dash_attn_fwd_noalloc(const dash_tensor_t *q, const dash_tensor_t *k, const dash_tensor_t *v,
                                   dash_tensor_t *out, int block_size, float alpha, int causal, int gqa_groups,
                                   const dash_opts_t *opts) {
    dash_opts_t o;
    if (opts) {
        o = *opts;
        if (o.workspace)
            return dash::report_error(DASH_ERR_INVALID_ARG,
                                      "dash_attn_fwd_noalloc uses its own static scratch: opts->workspace must be NULL");
    } else {
        dash_opts_init(&o);
    }
    // the exact scratch this call's forward pass takes in the static area (it depends on the
    // options: a summary cache or given summaries need no pooled-key area, prefill no
    // split-KV area; a long prefill runs its query rows in slices that fit the area)
    size_t need = 0;
    int rc = dash::fwd_workspace_need(q, k, v, out, block_size, alpha, causal, gqa_groups, &o,
                                      DASH_NOALLOC_SCRATCH_BYTES, &need);
    if (rc) return rc;
    if (need > (size_t)DASH_NOALLOC_SCRATCH_BYTES) {
        char msg[256];
        snprintf(msg, sizeof msg,
                 "problem needs %zu bytes of scratch; dash_attn_fwd_noalloc holds at most %zu "
                 "(use dash_attn_fwd_ex with a workspace)",
                 need, (size_t)DASH_NOALLOC_SCRATCH_BYTES);
        return dash::report_error(DASH_ERR_WORKSPACE, msg);
    }
    void *scratch = nullptr;
    rc = noalloc_scratch(&scratch);
    if (rc) return rc;
    o.workspace = scratch;
    o.workspace_bytes = DASH_NOALLOC_SCRATCH_BYTES;
    return dash_attn_fwd_ex(q, k, v, out, block_size, alpha, causal, gqa_groups, &o);
}

}  // extern "C"

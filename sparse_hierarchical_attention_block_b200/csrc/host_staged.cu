// host_staged.cu -- dash_attn_fwd_host: the forward pass on host-resident q, k, v and
// out, through device buffers the caller provides, with the host<->device copies
// overlapped with the computation.
//
// The query rows are taken in slices (multiples of 1024 rows), in order.  With a causal
// mask a slice of rows [a, e) depends only on the keys up to its last row's position, so
// slice s can run as soon as that key prefix and its own query rows are on the device:
//   copy stream 1   K and V rows [prev prefix, prefix of s), Q rows [a, e)  -> event in[s]
//   caller stream   wait in[s]; dash_attn_fwd_ex on (Q rows [a, e), K and V prefix)
//                   -> event out[s]
//   copy stream 2   wait out[s]; O rows [a, e) to the host
// and the caller's stream finally waits for the last copy back.  A slice's forward on
// its key prefix gives exactly the rows the whole forward gives (query row i sits at
// key position i + nk - nq either way, and every chunk it may route lies inside the
// prefix), so the output is bit-identical to dash_attn_fwd_ex on the whole tensors.
// Without a causal mask every slice needs all keys: K and V go first, then the query
// slices, and only the copies of Q and O overlap the computation.
//
// The copies are one cudaMemcpy2DAsync per tensor and slice (a slice's rows in every
// batch element: the batch stride is the pitch), from and to page-locked host memory
// for the copies to run asynchronously.  The two copy streams are created once per
// device and live until dash_release.
#include <algorithm>
#include <mutex>
#include <vector>

#include "dash_common.cuh"
#include "kernels.h"

namespace dash {
int report_error(int code, const char *msg);
int fwd_workspace_need(const dash_tensor_t *q, const dash_tensor_t *k, const dash_tensor_t *v,
                       const dash_tensor_t *out, int block_size, float alpha, int causal, int gqa_groups,
                       const dash_opts_t *opts, size_t budget, size_t *need);
}  // namespace dash

namespace {

constexpr int kMaxDevices = 128;
std::mutex g_stage_mu;
cudaStream_t g_h2d[kMaxDevices], g_d2h[kMaxDevices];

int fail(int code, const char *msg) { return dash::report_error(code, msg); }
int cuda_fail(cudaError_t e) { return dash::report_error(DASH_ERR_CUDA, cudaGetErrorString(e)); }

// The two copy streams of the current device (created on first use).
int staging_streams(cudaStream_t *h2d, cudaStream_t *d2h) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e);
    if (dev < 0 || dev >= kMaxDevices) return fail(DASH_ERR_UNSUPPORTED, "device index out of range");
    std::lock_guard<std::mutex> lk(g_stage_mu);
    if (!g_h2d[dev]) {
        if ((e = cudaStreamCreateWithFlags(&g_h2d[dev], cudaStreamNonBlocking)) != cudaSuccess) return cuda_fail(e);
        if ((e = cudaStreamCreateWithFlags(&g_d2h[dev], cudaStreamNonBlocking)) != cudaSuccess) {
            cudaStreamDestroy(g_h2d[dev]);
            g_h2d[dev] = nullptr;
            return cuda_fail(e);
        }
    }
    *h2d = g_h2d[dev];
    *d2h = g_d2h[dev];
    return DASH_OK;
}

size_t elem_bytes(dash_dtype_t dt) { return dt == DASH_BF16 ? 2 : 4; }

// Rows of one batch element contiguous ([seq][heads][dim] packed), any batch stride.
bool packed_rows(const dash_tensor_t *t) {
    return t->stride[3] == 1 && t->stride[2] == t->shape[3] && t->stride[1] == t->shape[2] * t->shape[3] &&
           (t->shape[0] <= 1 || t->stride[0] >= t->shape[1] * t->stride[1]);
}

bool same_shape(const dash_tensor_t *a, const dash_tensor_t *b) {
    if (a->dtype != b->dtype) return false;
    for (int x = 0; x < 4; ++x)
        if (a->shape[x] != b->shape[x]) return false;
    return true;
}

// Rows [r0, r1) of every batch element of src into dst (same shapes).
cudaError_t copy_rows(const dash_tensor_t *dst, const dash_tensor_t *src, int64_t r0, int64_t r1, cudaMemcpyKind kind,
                      cudaStream_t st) {
    if (r1 <= r0 || dst->shape[0] == 0) return cudaSuccess;
    const size_t es = elem_bytes(dst->dtype);
    char *d = static_cast<char *>(dst->data) + r0 * dst->stride[1] * es;
    const char *s = static_cast<const char *>(src->data) + r0 * src->stride[1] * es;
    const size_t width = (size_t)(r1 - r0) * dst->stride[1] * es;
    return cudaMemcpy2DAsync(d, (size_t)dst->stride[0] * es, s, (size_t)src->stride[0] * es, width,
                             (size_t)dst->shape[0], kind, st);
}

// rows [r0, r1) of t as a tensor of its own
dash_tensor_t row_view(const dash_tensor_t *t, int64_t r0, int64_t r1) {
    dash_tensor_t v = *t;
    v.data = static_cast<char *>(t->data) + r0 * t->stride[1] * (int64_t)elem_bytes(t->dtype);
    v.shape[1] = r1 - r0;
    return v;
}

}  // namespace

namespace dash {
// Frees the copy streams of the current device (dash_release).
void release_host_staging() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return;
    std::lock_guard<std::mutex> lk(g_stage_mu);
    if (g_h2d[dev]) {
        cudaStreamSynchronize(g_h2d[dev]);
        cudaStreamSynchronize(g_d2h[dev]);
        cudaStreamDestroy(g_h2d[dev]);
        cudaStreamDestroy(g_d2h[dev]);
        g_h2d[dev] = g_d2h[dev] = nullptr;
    }
}
}  // namespace dash

extern "C" {

DASH_API int dash_attn_fwd_host(const dash_tensor_t *q_host, const dash_tensor_t *k_host,
                                const dash_tensor_t *v_host, dash_tensor_t *out_host, const dash_tensor_t *q_dev,
                                const dash_tensor_t *k_dev, const dash_tensor_t *v_dev, dash_tensor_t *out_dev,
                                int block_size, float alpha, int causal, int gqa_groups, int n_slices,
                                const dash_opts_t *opts) {
    const dash_tensor_t *pairs[4][2] = {{q_host, q_dev}, {k_host, k_dev}, {v_host, v_dev}, {out_host, out_dev}};
    for (auto &pr : pairs) {
        if (!pr[0] || !pr[1]) return fail(DASH_ERR_INVALID_ARG, "a host or device tensor is NULL");
        if (!same_shape(pr[0], pr[1]))
            return fail(DASH_ERR_INVALID_ARG, "a host tensor and its device buffer differ in shape or dtype");
        if (!packed_rows(pr[0]) || !packed_rows(pr[1]))
            return fail(DASH_ERR_UNSUPPORTED, "host-staged forward: every tensor needs packed [seq][heads][dim] rows");
    }
    if (n_slices < 0) return fail(DASH_ERR_INVALID_ARG, "n_slices must be >= 0");
    dash_opts_t o;
    if (opts) o = *opts;
    else dash_opts_init(&o);
    if (o.summary_cache || o.nk_dev || o.kbar || o.qbar || o.lse)
        return fail(DASH_ERR_UNSUPPORTED,
                    "host-staged forward: summary cache, nk_dev, kbar, qbar and lse are not supported");
    const int64_t nq = q_dev->shape[1], nk = k_dev->shape[1];
    // the whole problem validates as the forward validates it, before anything is enqueued
    size_t need = 0;
    int rc = dash::fwd_workspace_need(q_dev, k_dev, v_dev, out_dev, block_size, alpha, causal, gqa_groups, &o,
                                      o.workspace ? o.workspace_bytes : (size_t)1 << 62, &need);
    if (rc) return rc;
    if (q_dev->shape[0] == 0 || nq == 0) return DASH_OK;
    cudaStream_t h2d, d2h;
    if ((rc = staging_streams(&h2d, &d2h))) return rc;
    cudaStream_t cs = static_cast<cudaStream_t>(o.stream);
    // slices of whole multiples of 1024 rows, the quantum of the forward's own row slices
    // (its tiles and row-regrouping windows then fall as they do in one pass); by default
    // up to 16 for long prefills
    const int want = n_slices > 0 ? n_slices : (nq >= 16384 ? 16 : nq >= 2048 ? 4 : 1);
    int64_t step = (nq + want - 1) / want;
    step = std::min<int64_t>(nq, (step + 1023) / 1024 * 1024);
    const int S = (int)((nq + step - 1) / step);
    std::vector<cudaEvent_t> ev(2 * S + 2, nullptr);
    cudaError_t e = cudaSuccess;
    for (auto &x : ev)
        if ((e = cudaEventCreateWithFlags(&x, cudaEventDisableTiming)) != cudaSuccess) break;
    auto cleanup = [&]() {
        for (auto &x : ev)
            if (x) cudaEventDestroy(x);  // released once the work it marks has completed
    };
    if (e != cudaSuccess) {
        cleanup();
        return cuda_fail(e);
    }
    cudaEvent_t ev_start = ev[2 * S], ev_done = ev[2 * S + 1];
    // the copies into the device buffers wait for the caller's earlier work on them
    if ((e = cudaEventRecord(ev_start, cs)) != cudaSuccess || (e = cudaStreamWaitEvent(h2d, ev_start, 0)) != cudaSuccess ||
        (e = cudaStreamWaitEvent(d2h, ev_start, 0)) != cudaSuccess) {
        cleanup();
        return cuda_fail(e);
    }
    int64_t kdone = 0;
    for (int s = 0; s < S && rc == DASH_OK; ++s) {
        const int64_t a = s * step, z = std::min(nq, a + step);
        const int64_t ke = causal ? std::min(nk, z + nk - nq) : nk;  // the keys rows [a, z) can see
        if ((e = copy_rows(k_dev, k_host, kdone, ke, cudaMemcpyHostToDevice, h2d)) != cudaSuccess ||
            (e = copy_rows(v_dev, v_host, kdone, ke, cudaMemcpyHostToDevice, h2d)) != cudaSuccess ||
            (e = copy_rows(q_dev, q_host, a, z, cudaMemcpyHostToDevice, h2d)) != cudaSuccess ||
            (e = cudaEventRecord(ev[2 * s], h2d)) != cudaSuccess || (e = cudaStreamWaitEvent(cs, ev[2 * s], 0)) != cudaSuccess) {
            rc = cuda_fail(e);
            break;
        }
        kdone = std::max(kdone, ke);
        const dash_tensor_t qs = row_view(q_dev, a, z), ks = row_view(k_dev, 0, ke), vs = row_view(v_dev, 0, ke);
        dash_tensor_t os = row_view(out_dev, a, z);
        if ((rc = dash_attn_fwd_ex(&qs, &ks, &vs, &os, block_size, alpha, causal, gqa_groups, &o))) break;
        if ((e = cudaEventRecord(ev[2 * s + 1], cs)) != cudaSuccess ||
            (e = cudaStreamWaitEvent(d2h, ev[2 * s + 1], 0)) != cudaSuccess ||
            (e = copy_rows(out_host, out_dev, a, z, cudaMemcpyDeviceToHost, d2h)) != cudaSuccess) {
            rc = cuda_fail(e);
            break;
        }
    }
    // the caller's stream goes on once the last copy back (and every copy in) has landed
    if ((e = cudaEventRecord(ev_done, d2h)) == cudaSuccess) e = cudaStreamWaitEvent(cs, ev_done, 0);
    if (e == cudaSuccess && (e = cudaEventRecord(ev_done, h2d)) == cudaSuccess) e = cudaStreamWaitEvent(cs, ev_done, 0);
    cleanup();
    if (rc == DASH_OK && e != cudaSuccess) rc = cuda_fail(e);
    return rc;
}

}  // extern "C"

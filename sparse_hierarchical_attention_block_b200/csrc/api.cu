// api.cu -- the C ABI (include/dash_attn.h): argument validation, workspace,
// stage orchestration on the caller's stream.
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <mutex>
#include <string>

#include "dash_common.cuh"
#include "kernels.h"

namespace dash {
int take_device_error_tc();
int take_device_error_decode();
int take_device_error_select();
int take_device_error_bwd();
}  // namespace dash

using namespace dash;

// The persistent chunk-summary cache (dash_summary_cache_t in the C header).
struct dash_summary_cache {
    int64_t b, max_nk;
    int hkv, d, B;
    int cap;       // chunk capacity floor(max_nk / B): the summaries' batch stride
    int ct_cap;    // 128-chunk tiles of the split form per (batch, kv head)
    int64_t done;  // chunks pooled so far (host-side updates)
    int dev;
    float *kbar;     // [b][cap][hkv][d] fp32
    uint8_t *split;  // [b][hkv][ct_cap] bf16 hi + lo operand tiles
    int *done_dev;   // chunks pooled so far, in device memory (device-resident key length)
};

namespace {

thread_local std::string g_last_error;

int fail(int code, const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return code;
}

int cuda_fail(cudaError_t e, const char *what) {
    return fail(DASH_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

size_t esize(dash_dtype_t dt) { return dt == DASH_BF16 ? 2 : 4; }

int check_tensor(const dash_tensor_t *t, const char *name) {
    if (!t) return fail(DASH_ERR_INVALID_ARG, "%s is NULL", name);
    if (t->dtype != DASH_F32 && t->dtype != DASH_BF16) return fail(DASH_ERR_UNSUPPORTED, "%s: unknown dtype", name);
    for (int a = 0; a < 4; ++a)
        if (t->shape[a] < 0) return fail(DASH_ERR_INVALID_ARG, "%s: negative extent", name);
    if (t->stride[3] != 1) return fail(DASH_ERR_UNSUPPORTED, "%s: the last dimension must be contiguous", name);
    int64_t n = t->shape[0] * t->shape[1] * t->shape[2] * t->shape[3];
    if (n > 0 && !t->data) return fail(DASH_ERR_INVALID_ARG, "%s: data is NULL", name);
    if (reinterpret_cast<uintptr_t>(t->data) % 16) return fail(DASH_ERR_ALIGNMENT, "%s: base not 16-byte aligned", name);
    for (int a = 0; a < 3; ++a)
        if ((t->stride[a] * (int64_t)esize(t->dtype)) % 16)
            return fail(DASH_ERR_ALIGNMENT, "%s: stride %d is not a multiple of 16 bytes", name, a);
    return DASH_OK;
}

TView view(const dash_tensor_t *t) { return TView{t->data, t->stride[0], t->stride[1], t->stride[2]}; }

int make_geom(const dash_tensor_t *q, const dash_tensor_t *k, int B, int causal, int gqa, Geom *G) {
    const int64_t b = q->shape[0], nq = q->shape[1], hq = q->shape[2], d = q->shape[3];
    const int64_t nk = k->shape[1], hkv = k->shape[2];
    if (k->shape[0] != b) return fail(DASH_ERR_INVALID_ARG, "q and k batch differ");
    if (k->shape[3] != d) return fail(DASH_ERR_INVALID_ARG, "q and k head dim differ");
    if (hkv <= 0 || hq % hkv) return fail(DASH_ERR_INVALID_ARG, "q heads (%lld) not a multiple of kv heads (%lld)",
                                          (long long)hq, (long long)hkv);
    if (gqa != hq / hkv) return fail(DASH_ERR_INVALID_ARG, "gqa_groups %d != hq/hkv = %lld", gqa,
                                     (long long)(hq / hkv));
    if (gqa < 1 || gqa > 16) return fail(DASH_ERR_UNSUPPORTED, "gqa_groups must be in [1, 16]");
    if (d != 64 && d != 128) return fail(DASH_ERR_UNSUPPORTED, "head dim %lld not in {64, 128}", (long long)d);
    if (B != 16 && B != 32 && B != 64 && B != 128)
        return fail(DASH_ERR_UNSUPPORTED, "block_size %d not in {16, 32, 64, 128}", B);
    if (causal != 0 && causal != 1) return fail(DASH_ERR_INVALID_ARG, "causal must be 0 or 1");
    if (nk <= 0) return fail(DASH_ERR_INVALID_ARG, "empty key sequence");
    if (causal && nq > nk) return fail(DASH_ERR_INVALID_ARG, "causal attention needs nq <= nk");
    if (nk > (int64_t)1 << 30 || nq > (int64_t)1 << 30) return fail(DASH_ERR_UNSUPPORTED, "sequence too long");
    G->b = b;
    G->nq = nq;
    G->nk = nk;
    G->hq = (int)hq;
    G->hkv = (int)hkv;
    G->g = gqa;
    G->d = (int)d;
    G->B = B;
    G->causal = causal;
    G->n_chunks = (int)(causal ? nk / B : (nk + B - 1) / B);
    G->n_blk = (int)((nk + B - 1) / B);
    G->tile_rows = 128 / gqa;
    G->n_tiles = (nq + G->tile_rows - 1) / G->tile_rows;
    G->words = (G->n_chunks + 31) / 32;
    G->kbar_cap = G->n_chunks;
    G->ct_cap = (G->n_chunks + 127) / 128;
    G->local = 1;
    G->nk_dev = nullptr;
    G->chunks_dev = nullptr;
    G->pos0 = nk - nq;
    G->nq_lse = nq;
    return DASH_OK;
}

// The local window the options ask for (App. B.1.1's two blocks with DASH_FLAG_LOCAL2).
int set_local(const dash_opts_t &o, Geom *G) {
    G->local = 1;
    if (o.flags & DASH_FLAG_LOCAL2) {
        if (!G->causal) return fail(DASH_ERR_INVALID_ARG, "DASH_FLAG_LOCAL2 needs causal attention");
        G->local = 2;
    }
    return DASH_OK;
}

dash_opts_t default_opts() {
    dash_opts_t o;
    memset(&o, 0, sizeof o);
    o.sigma = 1e8f;
    o.gamma = 1.0f;
    return o;
}

int check_opts(const dash_opts_t &o) {
    if (!(o.sigma > 0.f) || !isfinite(o.sigma)) return fail(DASH_ERR_INVALID_ARG, "sigma must be > 0");
    if (!(o.gamma > 0.f) || !isfinite(o.gamma)) return fail(DASH_ERR_INVALID_ARG, "gamma must be > 0");
    if (o.workspace && reinterpret_cast<uintptr_t>(o.workspace) % 256)
        return fail(DASH_ERR_ALIGNMENT, "workspace must be 256-byte aligned");
    if (o.lse && reinterpret_cast<uintptr_t>(o.lse) % 4) return fail(DASH_ERR_ALIGNMENT, "lse not 4-byte aligned");
    return DASH_OK;
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

struct WsLayout {
    size_t kbar, mask, logw, mu, count, ids, bias, rows, decode, split, total;
};

WsLayout ws_layout(const Geom &G, bool need_kbar, bool need_lists, bool need_decode) {
    WsLayout L{};
    size_t off = 0;
    auto take = [&](size_t bytes) {
        size_t o = off;
        off += align256(bytes);
        return o;
    };
    L.kbar = need_kbar ? take((size_t)G.b * G.n_chunks * G.hkv * G.d * 4) : 0;
    L.mask = take((size_t)G.b * G.nq * G.hkv * (size_t)G.words * 4);
    L.logw = need_lists ? take((size_t)G.b * G.nq * G.hkv * (size_t)G.n_chunks * 4) : 0;
    L.mu = need_lists ? take((size_t)G.b * G.nq * G.hkv * 4) : 0;
    L.count = need_lists ? take((size_t)G.b * G.hkv * G.n_tiles * 4) : 0;
    L.ids = need_lists ? take((size_t)G.b * G.hkv * G.n_tiles * G.n_blk * 4) : 0;
    L.bias = need_lists ? take((size_t)G.b * G.hkv * G.n_tiles * G.n_blk * G.tile_rows * 4) : 0;
    L.rows = need_lists ? take((size_t)G.b * G.hkv * G.n_tiles * G.tile_rows * 4) : 0;
    L.decode = need_decode ? take(attn_decode_workspace(G)) : 0;
    L.split = select_tile_supported(G, DASH_BF16) ? take(select_tile_workspace(G)) : 0;
    L.total = off;
    return L;
}

// Query rows in slices.  A prefill's Stage-1 state and work lists grow with nq x n_chunks
// (4.3 GB each for the log-w array and the bias table at 128K), so the rows are processed
// in slices of a multiple of 1024 (whole regrouping windows) that fit a workspace budget:
// Stage 1 and Stage 2 run slice after slice on one per-slice workspace (Stage 0 once).
constexpr size_t kSliceBudget = 1000000000;  // the library-managed workspace's budget (1 GB)
constexpr int64_t kSliceQuantum = 1024;

Geom slice_geom(const Geom &G, int64_t row0, int64_t rows) {
    Geom S = G;
    S.nq = rows;
    S.n_tiles = (rows + G.tile_rows - 1) / G.tile_rows;
    S.pos0 = G.pos0 + row0;
    return S;
}

// Rows per slice: every row when the whole layout fits the budget (or the path is
// decoding), else the largest multiple of kSliceQuantum whose layout fits (at least one
// quantum: a budget below that leaves the workspace check to refuse).
int64_t slice_rows(const Geom &G, bool need_kbar, bool dec, size_t budget) {
    if (dec || G.nq <= kSliceQuantum || ws_layout(G, need_kbar, true, dec).total <= budget) return G.nq;
    int64_t lo = 1, hi = (G.nq - 1) / kSliceQuantum;  // candidate slices of lo..hi quanta
    if (ws_layout(slice_geom(G, 0, kSliceQuantum), need_kbar, true, dec).total > budget) return kSliceQuantum;
    while (lo < hi) {
        const int64_t mid = (lo + hi + 1) / 2;
        if (ws_layout(slice_geom(G, 0, mid * kSliceQuantum), need_kbar, true, dec).total <= budget) lo = mid;
        else hi = mid - 1;
    }
    return lo * kSliceQuantum;
}

// Library-managed workspace, one cached allocation per device.
std::mutex g_ws_mu;
struct DevWs {
    void *p = nullptr;
    size_t bytes = 0;
};
DevWs g_ws[128];

int get_workspace(const dash_opts_t &o, size_t need, char **base) {
    if (o.workspace) {
        if (o.workspace_bytes < need)
            return fail(DASH_ERR_WORKSPACE, "workspace too small: %zu < %zu bytes", o.workspace_bytes, need);
        *base = static_cast<char *>(o.workspace);
        return DASH_OK;
    }
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= 128) return fail(DASH_ERR_UNSUPPORTED, "device index out of range");
    std::lock_guard<std::mutex> lk(g_ws_mu);
    DevWs &w = g_ws[dev];
    if (w.bytes < need) {
        if (w.p) {
            // the old buffer may still be in use by queued work
            e = cudaDeviceSynchronize();
            if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
            cudaFree(w.p);
            w.p = nullptr;
            w.bytes = 0;
        }
        size_t want = need + need / 4;
        e = cudaMalloc(&w.p, want);
        if (e != cudaSuccess) return cuda_fail(e, "cudaMalloc(workspace)");
        w.bytes = want;
    }
    *base = static_cast<char *>(w.p);
    return DASH_OK;
}

int check_lists(const dash_lists_t *l, const Geom &G) {
    if (!l->count || !l->ids || !l->bias) return fail(DASH_ERR_INVALID_ARG, "lists: NULL buffer");
    if (l->n_tiles != G.n_tiles || l->cap != G.n_blk || l->tile_rows != G.tile_rows)
        return fail(DASH_ERR_INVALID_ARG, "lists geometry (n_tiles %lld, cap %d, tile_rows %d) does not match the "
                                          "problem (%lld, %d, %d)",
                    (long long)l->n_tiles, l->cap, l->tile_rows, (long long)G.n_tiles, G.n_blk, G.tile_rows);
    return DASH_OK;
}

ListsView lists_view(const dash_lists_t *l) {
    return ListsView{l->count, l->ids, l->bias, l->rows, l->n_tiles, l->cap, l->tile_rows};
}

ListsView ws_lists(const Geom &G, char *ws, const WsLayout &WL, bool with_rows) {
    return ListsView{reinterpret_cast<int32_t *>(ws + WL.count), reinterpret_cast<int32_t *>(ws + WL.ids),
                     reinterpret_cast<float *>(ws + WL.bias),
                     with_rows ? reinterpret_cast<int32_t *>(ws + WL.rows) : nullptr, G.n_tiles, G.n_blk,
                     G.tile_rows};
}

// Stage 1 (after Stage 0): routing of every (row, head) and, when LV is given, the
// Stage-2 work lists.  With regroup (LV->rows required) the rows of each window of
// tiles are regrouped by routed-set size; otherwise tile t holds consecutive rows
// (and LV->rows, if given, is filled accordingly).
int run_stage1(const dash_tensor_t *q, const Geom &G, float alpha, const dash_opts_t &o, const float *kbar,
               float *tau, float *w, uint32_t *mask_out, const ListsView *LV, bool regroup, char *ws,
               const WsLayout &WL, cudaStream_t st, const uint8_t *presplit = nullptr) {
    cudaError_t e;
    const bool tile = select_tile_supported(G, q->dtype);
    regroup = regroup && LV && LV->rows && regroup_supported(G);
    uint32_t *mask = mask_out ? mask_out : reinterpret_cast<uint32_t *>(ws + WL.mask);
    float *logw = reinterpret_cast<float *>(ws + WL.logw);
    float *mu = reinterpret_cast<float *>(ws + WL.mu);
    if (tile) {
        e = launch_select_tile(view(q), kbar, G, alpha, o.gamma, tau, w, mask, LV ? logw : nullptr,
                               LV ? mu : nullptr, ws + WL.split, st, presplit);
        if (e != cudaSuccess) return cuda_fail(e, "select_tile");
    } else {
        SelectOut so{tau, w, mask, LV ? logw : nullptr, LV ? mu : nullptr};
        e = launch_select_rows(view(q), q->dtype, kbar, G, alpha, o.gamma, o.sigma, so, st);
        if (e != cudaSuccess) return cuda_fail(e, "select_rows");
    }
    if (!LV) return DASH_OK;
    e = regroup ? launch_regroup_compact(G, mask, logw, mu, o.sigma, *LV, st)
                : launch_compact(G, mask, logw, mu, o.sigma, *LV, st);
    return e == cudaSuccess ? DASH_OK : cuda_fail(e, "work-list compaction");
}

int run_stage2(const dash_tensor_t *q, const dash_tensor_t *k, const dash_tensor_t *v, dash_tensor_t *out,
               const Geom &G, const ListsView &LV, const dash_opts_t &o, char *decode_ws, cudaStream_t st) {
    cudaError_t e;
    const dash_dtype_t dt = q->dtype;
    const bool simt = (o.flags & DASH_FLAG_FORCE_SIMT) != 0;
    if (!simt && decode_ws && attn_decode_supported(G, dt)) {
        e = launch_attn_decode(view(q), view(k), view(v), view(out), G, LV, decode_ws, st, o.lse);
        if (e != cudaSuccess) return cuda_fail(e, "stage 2 (decode)");
    } else if (!simt && attn_tc_supported(G, dt)) {
        e = launch_attn_tc(view(q), view(k), view(v), view(out), G, LV, o.flags, st, o.lse);
        if (e != cudaSuccess) return cuda_fail(e, "stage 2 (tensor cores)");
    } else {
        e = launch_attn_simt(view(q), view(k), view(v), view(out), dt, G, LV, st, o.lse);
        if (e != cudaSuccess) return cuda_fail(e, "stage 2 (CUDA cores)");
    }
    return DASH_OK;
}

// Summary queries of Stage 0: [1 or b][n_chunks][hkv][d]; shape[0] == 1 broadcasts over the batch.
int check_qbar(const dash_tensor_t *qb, const Geom &G, TView *v) {
    int rc = check_tensor(qb, "qbar");
    if (rc) return rc;
    if ((qb->shape[0] != 1 && qb->shape[0] != G.b) || qb->shape[1] != G.n_chunks || qb->shape[2] != G.hkv ||
        qb->shape[3] != G.d)
        return fail(DASH_ERR_INVALID_ARG,
                    "qbar shape [%lld, %lld, %lld, %lld] does not match [1 or %lld, %d chunks, %d kv heads, %d]",
                    (long long)qb->shape[0], (long long)qb->shape[1], (long long)qb->shape[2],
                    (long long)qb->shape[3], (long long)G.b, G.n_chunks, G.hkv, G.d);
    *v = view(qb);
    if (qb->shape[0] == 1) v->s0 = 0;
    return DASH_OK;
}

// Stage 0 into kbar: mean pooling, or the learned-query softmax pooling when qb is given
// (qb already validated).
int run_stage0(const dash_tensor_t *k, const dash_tensor_t *qb, const TView &qv, const Geom &G, float *kbar,
               cudaStream_t st) {
    cudaError_t e = qb ? launch_pool_keys_q(view(k), k->dtype, qv, qb->dtype, G, kbar, st)
                       : launch_pool_keys(view(k), k->dtype, G, kbar, st);
    return e == cudaSuccess ? DASH_OK : cuda_fail(e, "pool_keys");
}

// A summary cache given in the options must match the problem and hold every complete chunk.
int check_cache(const dash_summary_cache *sc, const Geom &G, const dash_opts_t &o) {
    if (o.kbar || o.qbar) return fail(DASH_ERR_INVALID_ARG, "opts: summary_cache is not used with kbar or qbar");
    if (!G.causal) return fail(DASH_ERR_INVALID_ARG, "summary_cache needs causal routing");
    if (sc->b != G.b || sc->hkv != G.hkv || sc->d != G.d || sc->B != G.B)
        return fail(DASH_ERR_INVALID_ARG, "summary_cache was made for another shape or block size");
    if (!o.nk_dev && sc->done != G.n_chunks)
        return fail(DASH_ERR_INVALID_ARG, "summary_cache holds %lld chunks; the keys have %d complete chunks",
                    (long long)sc->done, G.n_chunks);
    if (o.nk_dev && G.nk > sc->max_nk)
        return fail(DASH_ERR_INVALID_ARG, "k's capacity (%lld keys) exceeds the summary cache's max_nk (%lld)",
                    (long long)G.nk, (long long)sc->max_nk);
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev != sc->dev)
        return fail(DASH_ERR_INVALID_ARG, "summary_cache lives on another device");
    return DASH_OK;
}

// The geometry Stage 1 sees with a summary cache: the cache's strides.
Geom cache_geom(const Geom &G, const dash_summary_cache *sc) {
    Geom G1 = G;
    if (sc) {
        G1.kbar_cap = sc->cap;
        G1.ct_cap = sc->ct_cap;
    }
    return G1;
}

int validate_qkvo(const dash_tensor_t *q, const dash_tensor_t *k, const dash_tensor_t *v,
                  const dash_tensor_t *out) {
    int rc;
    if ((rc = check_tensor(q, "q")) || (rc = check_tensor(k, "k")) || (rc = check_tensor(v, "v")) ||
        (rc = check_tensor(out, "out")))
        return rc;
    if (q->dtype != k->dtype || q->dtype != v->dtype || q->dtype != out->dtype)
        return fail(DASH_ERR_INVALID_ARG, "q, k, v and out must share a dtype");
    for (int a = 0; a < 4; ++a) {
        if (q->shape[a] != out->shape[a]) return fail(DASH_ERR_INVALID_ARG, "q and out shapes differ");
        if (k->shape[a] != v->shape[a]) return fail(DASH_ERR_INVALID_ARG, "k and v shapes differ");
    }
    return DASH_OK;
}

// Everything dash_attn_fwd_ex decides before it launches: validated geometry, where
// Stage 0's summaries come from, whether Stage 2 takes the split-KV decode path, and
// the workspace layout those choices need.
struct FwdPlan {
    Geom G;
    WsLayout WL;  // the layout of one slice of rows (of every row when not sliced)
    TView qv;
    const dash_summary_cache *sc;
    bool need_kbar, dec;
    int64_t slice;  // query rows per slice
};

int plan_fwd(const dash_tensor_t *q, const dash_tensor_t *k, const dash_tensor_t *v, const dash_tensor_t *out,
             int block_size, float alpha, int causal, int gqa_groups, const dash_opts_t &o, FwdPlan *P,
             size_t budget) {
    int rc;
    if ((rc = check_opts(o))) return rc;
    if ((rc = validate_qkvo(q, k, v, out))) return rc;
    if (!(alpha > 1.f) || !isfinite(alpha)) return fail(DASH_ERR_INVALID_ARG, "alpha must be > 1");
    Geom &G = P->G;
    if ((rc = make_geom(q, k, block_size, causal, gqa_groups, &G))) return rc;
    if ((rc = set_local(o, &G))) return rc;
    if (o.kbar && reinterpret_cast<uintptr_t>(o.kbar) % 16) return fail(DASH_ERR_ALIGNMENT, "kbar not aligned");
    P->qv = TView{};
    P->sc = o.summary_cache;
    if (P->sc && (rc = check_cache(P->sc, G, o))) return rc;
    if (o.qbar && o.kbar) return fail(DASH_ERR_INVALID_ARG, "opts: give kbar or qbar, not both");
    if (o.qbar && (rc = check_qbar(o.qbar, G, &P->qv))) return rc;
    P->need_kbar = o.kbar == nullptr && !P->sc;
    P->dec = attn_decode_supported(G, q->dtype) && !(o.flags & DASH_FLAG_FORCE_SIMT);
    if (o.nk_dev) {
        if (!P->sc) return fail(DASH_ERR_INVALID_ARG, "opts->nk_dev needs opts->summary_cache");
        if (reinterpret_cast<uintptr_t>(o.nk_dev) % 8) return fail(DASH_ERR_ALIGNMENT, "nk_dev not 8-byte aligned");
        if (!P->dec || !select_tile_supported(G, q->dtype) || G.local != 1)
            return fail(DASH_ERR_UNSUPPORTED, "opts->nk_dev: decoding only (bf16, nq * gqa_groups <= 16, the "
                                              "tensor-core Stage 1, the one-block local window)");
        G.nk_dev = o.nk_dev;
    }
    P->slice = slice_rows(G, P->need_kbar, P->dec, budget);
    P->WL = (G.b == 0 || G.nq == 0) ? WsLayout{}
                                    : ws_layout(slice_geom(G, 0, P->slice), P->need_kbar, true, P->dec);
    return DASH_OK;
}

// The slicing budget of a call: the caller's workspace when it gives one, else the
// library's default.
size_t slice_budget(const dash_opts_t &o) { return o.workspace ? o.workspace_bytes : kSliceBudget; }

}  // namespace

namespace dash {
// Records msg as this thread's last error (dash_last_error) and returns code;
// for entry points defined in other translation units.
int report_error(int code, const char *msg) { return fail(code, "%s", msg); }

// The workspace bytes dash_attn_fwd_ex would take for these arguments (validated as it
// validates them); *need = 0 for an empty problem.
int fwd_workspace_need(const dash_tensor_t *q, const dash_tensor_t *k, const dash_tensor_t *v,
                       const dash_tensor_t *out, int block_size, float alpha, int causal, int gqa_groups,
                       const dash_opts_t *opts, size_t budget, size_t *need) {
    const dash_opts_t o = opts ? *opts : default_opts();
    FwdPlan P;
    const int rc = plan_fwd(q, k, v, out, block_size, alpha, causal, gqa_groups, o, &P, budget);
    *need = rc ? 0 : P.WL.total;
    return rc;
}
}  // namespace dash

extern "C" {

DASH_API const char *dash_version(void) { return "dash-attn-b200 0.1 (sm_100a)"; }

DASH_API const char *dash_last_error(void) { return g_last_error.c_str(); }

DASH_API int dash_opts_init(dash_opts_t *opts) {
    if (!opts) return fail(DASH_ERR_INVALID_ARG, "opts is NULL");
    *opts = default_opts();
    return DASH_OK;
}

DASH_API int dash_lists_geometry(int64_t batch, int64_t nq, int64_t nk, int hkv, int block_size, int gqa_groups,
                                 int64_t *n_tiles, int32_t *cap, int32_t *tile_rows, size_t *count_bytes,
                                 size_t *ids_bytes, size_t *bias_bytes, size_t *rows_bytes) {
    if (batch < 0 || nq < 0 || nk <= 0 || hkv <= 0 || block_size <= 0 || gqa_groups < 1 || gqa_groups > 16)
        return fail(DASH_ERR_INVALID_ARG, "bad lists geometry arguments");
    const int64_t tr = 128 / gqa_groups;
    const int64_t nt = (nq + tr - 1) / tr;
    const int64_t cp = (nk + block_size - 1) / block_size;
    if (n_tiles) *n_tiles = nt;
    if (cap) *cap = (int32_t)cp;
    if (tile_rows) *tile_rows = (int32_t)tr;
    if (count_bytes) *count_bytes = (size_t)batch * hkv * nt * 4;
    if (ids_bytes) *ids_bytes = (size_t)batch * hkv * nt * cp * 4;
    if (bias_bytes) *bias_bytes = (size_t)batch * hkv * nt * cp * tr * 4;
    if (rows_bytes) *rows_bytes = (size_t)batch * hkv * nt * tr * 4;
    return DASH_OK;
}

DASH_API size_t dash_workspace_bytes(int64_t batch, int64_t nq, int64_t nk, int hq, int hkv, int d, int block_size,
                                     int causal) {
    if (hkv <= 0 || hq % hkv || block_size <= 0 || nk <= 0) return 0;
    Geom G{};
    G.b = batch;
    G.nq = nq;
    G.nk = nk;
    G.hq = hq;
    G.hkv = hkv;
    G.g = hq / hkv;
    G.d = d;
    G.B = block_size;
    G.causal = causal;
    G.n_chunks = (int)(causal ? nk / block_size : (nk + block_size - 1) / block_size);
    G.n_blk = (int)((nk + block_size - 1) / block_size);
    G.tile_rows = 128 / G.g;
    G.n_tiles = (nq + G.tile_rows - 1) / G.tile_rows;
    G.words = (G.n_chunks + 31) / 32;
    G.kbar_cap = G.n_chunks;
    G.ct_cap = (G.n_chunks + 127) / 128;
    G.local = 1;
    G.pos0 = nk - nq;
    G.nq_lse = nq;
    const bool dec = nq * G.g <= 16 && G.n_tiles == 1;  // the decoding path: never sliced
    const int64_t rows = slice_rows(G, true, dec, kSliceBudget);
    return ws_layout(slice_geom(G, 0, rows), true, true, dec).total;
}

DASH_API int dash_pool_keys(const dash_tensor_t *k, int block_size, int causal, float *kbar, void *stream) {
    int rc = check_tensor(k, "k");
    if (rc) return rc;
    if (!kbar) return fail(DASH_ERR_INVALID_ARG, "kbar is NULL");
    if (reinterpret_cast<uintptr_t>(kbar) % 16) return fail(DASH_ERR_ALIGNMENT, "kbar not 16-byte aligned");
    // Stage 0 only needs the key geometry: use k as its own (empty) query
    dash_tensor_t q0 = *k;
    q0.shape[1] = 0;
    Geom G;
    if ((rc = make_geom(&q0, k, block_size, causal, 1, &G))) return rc;
    cudaError_t e = launch_pool_keys(view(k), k->dtype, G, kbar, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "pool_keys");
    return DASH_OK;
}

DASH_API int dash_pool_keys_q(const dash_tensor_t *k, const dash_tensor_t *qbar, int block_size, int causal,
                              float *kbar, void *stream) {
    int rc = check_tensor(k, "k");
    if (rc) return rc;
    if (!kbar) return fail(DASH_ERR_INVALID_ARG, "kbar is NULL");
    if (reinterpret_cast<uintptr_t>(kbar) % 16) return fail(DASH_ERR_ALIGNMENT, "kbar not 16-byte aligned");
    dash_tensor_t q0 = *k;
    q0.shape[1] = 0;
    Geom G;
    if ((rc = make_geom(&q0, k, block_size, causal, 1, &G))) return rc;
    TView qv;
    if ((rc = check_qbar(qbar, G, &qv))) return rc;
    return run_stage0(k, qbar, qv, G, kbar, static_cast<cudaStream_t>(stream));
}

DASH_API int dash_lists_from_mask(const uint32_t *mask, int64_t batch, int64_t nq, int64_t nk, int hkv,
                                  int block_size, int gqa_groups, int causal, int regroup, dash_lists_t *lists,
                                  void *stream) {
    if (!mask || !lists) return fail(DASH_ERR_INVALID_ARG, "mask or lists is NULL");
    if (reinterpret_cast<uintptr_t>(mask) % 16) return fail(DASH_ERR_ALIGNMENT, "mask not 16-byte aligned");
    if (batch < 0 || nq < 0 || hkv <= 0) return fail(DASH_ERR_INVALID_ARG, "bad batch, nq or hkv");
    if (gqa_groups < 1 || gqa_groups > 16) return fail(DASH_ERR_UNSUPPORTED, "gqa_groups must be in [1, 16]");
    // the geometry from shapes alone (head dim does not enter the lists)
    dash_tensor_t q0{}, k0{};
    q0.dtype = k0.dtype = DASH_BF16;
    q0.data = k0.data = const_cast<uint32_t *>(mask);
    q0.shape[0] = k0.shape[0] = batch;
    q0.shape[1] = nq;
    k0.shape[1] = nk;
    q0.shape[2] = (int64_t)hkv * gqa_groups;
    k0.shape[2] = hkv;
    q0.shape[3] = k0.shape[3] = 128;
    Geom G;
    int rc = make_geom(&q0, &k0, block_size, causal, gqa_groups, &G);
    if (rc) return rc;
    if ((rc = check_lists(lists, G))) return rc;
    if (regroup && !lists->rows) return fail(DASH_ERR_INVALID_ARG, "regroup needs lists->rows");
    if (G.b == 0 || G.nq == 0) return DASH_OK;
    const ListsView LV = lists_view(lists);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const bool rg = regroup && G.n_tiles > 1 && regroup_supported(G);
    cudaError_t e = rg ? launch_regroup_compact(G, mask, nullptr, nullptr, 1.f, LV, st)
                       : launch_compact(G, mask, nullptr, nullptr, 1.f, LV, st);
    return e == cudaSuccess ? DASH_OK : cuda_fail(e, "work-list compaction");
}

DASH_API int dash_block_select(const dash_tensor_t *q, const dash_tensor_t *k, int block_size, float alpha,
                               int causal, int gqa_groups, float *tau, float *w, uint32_t *mask,
                               const dash_lists_t *lists, const dash_opts_t *opts) {
    dash_opts_t o = opts ? *opts : default_opts();
    int rc;
    if ((rc = check_opts(o))) return rc;
    if (o.nk_dev) return fail(DASH_ERR_UNSUPPORTED, "opts->nk_dev is for dash_attn_fwd_ex");
    if ((rc = check_tensor(q, "q")) || (rc = check_tensor(k, "k"))) return rc;
    if (q->dtype != k->dtype) return fail(DASH_ERR_INVALID_ARG, "q and k must share a dtype");
    if (!(alpha > 1.f) || !isfinite(alpha)) return fail(DASH_ERR_INVALID_ARG, "alpha must be > 1");
    Geom G;
    if ((rc = make_geom(q, k, block_size, causal, gqa_groups, &G))) return rc;
    if ((rc = set_local(o, &G))) return rc;
    if (lists && (rc = check_lists(lists, G))) return rc;
    for (const void *p : {(const void *)tau, (const void *)w, (const void *)mask})
        if (reinterpret_cast<uintptr_t>(p) % 16) return fail(DASH_ERR_ALIGNMENT, "outputs must be 16-byte aligned");
    TView qv{};
    const dash_summary_cache *sc = o.summary_cache;
    if (sc && (rc = check_cache(sc, G, o))) return rc;
    if (o.qbar && o.kbar) return fail(DASH_ERR_INVALID_ARG, "opts: give kbar or qbar, not both");
    if (o.qbar && (rc = check_qbar(o.qbar, G, &qv))) return rc;
    if (G.b == 0 || G.nq == 0) return DASH_OK;
    const bool need_kbar = o.kbar == nullptr && !sc;
    WsLayout WL = ws_layout(G, need_kbar, true, false);
    char *ws = nullptr;
    if ((rc = get_workspace(o, WL.total, &ws))) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(o.stream);
    const float *kbar = sc ? sc->kbar : o.kbar;
    if (need_kbar) {
        float *kb = reinterpret_cast<float *>(ws + WL.kbar);
        if ((rc = run_stage0(k, o.qbar, qv, G, kb, st))) return rc;
        kbar = kb;
    }
    ListsView LV;
    if (lists) LV = lists_view(lists);
    const bool regroup = lists && lists->rows && !(o.flags & DASH_FLAG_NO_REGROUP) && G.n_tiles > 1;
    return run_stage1(q, cache_geom(G, sc), alpha, o, kbar, tau, w, mask, lists ? &LV : nullptr, regroup, ws, WL,
                      st, sc ? sc->split : nullptr);
}

DASH_API int dash_sparse_attn_fwd(const dash_tensor_t *q, const dash_tensor_t *k, const dash_tensor_t *v,
                                  dash_tensor_t *out, const dash_lists_t *lists, int block_size, int causal,
                                  int gqa_groups, const dash_opts_t *opts) {
    dash_opts_t o = opts ? *opts : default_opts();
    int rc;
    if ((rc = check_opts(o))) return rc;
    if (o.nk_dev) return fail(DASH_ERR_UNSUPPORTED, "opts->nk_dev is for dash_attn_fwd_ex");
    if ((rc = validate_qkvo(q, k, v, out))) return rc;
    if (!lists) return fail(DASH_ERR_INVALID_ARG, "lists is NULL");
    Geom G;
    if ((rc = make_geom(q, k, block_size, causal, gqa_groups, &G))) return rc;
    if ((rc = check_lists(lists, G))) return rc;
    if (G.b == 0 || G.nq == 0) return DASH_OK;
    char *ws = nullptr;
    const size_t dec = attn_decode_supported(G, q->dtype) ? attn_decode_workspace(G) : 0;
    if (dec && (rc = get_workspace(o, dec, &ws))) return rc;
    return run_stage2(q, k, v, out, G, lists_view(lists), o, ws, static_cast<cudaStream_t>(o.stream));
}

DASH_API int dash_attn_fwd_ex(const dash_tensor_t *q, const dash_tensor_t *k, const dash_tensor_t *v,
                              dash_tensor_t *out, int block_size, float alpha, int causal, int gqa_groups,
                              const dash_opts_t *opts) {
    dash_opts_t o = opts ? *opts : default_opts();
    FwdPlan P;
    int rc = plan_fwd(q, k, v, out, block_size, alpha, causal, gqa_groups, o, &P, slice_budget(o));
    if (rc) return rc;
    const Geom &G = P.G;
    if (G.b == 0 || G.nq == 0) return DASH_OK;
    const dash_summary_cache *sc = P.sc;
    const TView qv = P.qv;
    const bool need_kbar = P.need_kbar, dec = P.dec;
    const WsLayout &WL = P.WL;
    char *ws = nullptr;
    if ((rc = get_workspace(o, WL.total, &ws))) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(o.stream);
    if (G.nk_dev) {
        // the cache catches up on the device with the chunks completed since the last step
        Geom Gc = cache_geom(G, sc);
        Gc.chunks_dev = sc->done_dev;
        cudaError_t e = launch_cache_catch_up(view(k), k->dtype, Gc, sc->kbar, sc->split, st);
        if (e != cudaSuccess) return cuda_fail(e, "summary cache catch-up");
    }
    const float *kbar = sc ? sc->kbar : o.kbar;
    if (need_kbar) {
        float *kb = reinterpret_cast<float *>(ws + WL.kbar);
        if ((rc = run_stage0(k, o.qbar, qv, G, kb, st))) return rc;
        kbar = kb;
    }
    // Stage 1 and Stage 2, one slice of query rows after the other (a single slice unless the
    // rows' lists would not fit the budget)
    for (int64_t row0 = 0; row0 < G.nq; row0 += P.slice) {
        const int64_t rows = std::min(P.slice, G.nq - row0);
        const Geom Gs = slice_geom(G, row0, rows);
        dash_tensor_t qs = *q, os = *out;
        qs.data = static_cast<char *>(q->data) + row0 * q->stride[1] * (int64_t)esize(q->dtype);
        os.data = static_cast<char *>(out->data) + row0 * out->stride[1] * (int64_t)esize(out->dtype);
        qs.shape[1] = os.shape[1] = rows;
        dash_opts_t oslice = o;
        if (o.lse) oslice.lse = o.lse + row0 * G.hq;
        const bool regroup = !(o.flags & DASH_FLAG_NO_REGROUP) && Gs.n_tiles > 1;
        const ListsView LV = ws_lists(Gs, ws, WL, regroup);
        if ((rc = run_stage1(&qs, cache_geom(Gs, sc), alpha, o, kbar, nullptr, nullptr, nullptr, &LV, regroup, ws, WL,
                             st, sc ? sc->split : nullptr)))
            return rc;
        if ((rc = run_stage2(&qs, k, v, &os, Gs, LV, oslice, dec ? ws + WL.decode : nullptr, st))) return rc;
    }
    return DASH_OK;
}

DASH_API int dash_attn_fwd(const dash_tensor_t *q, const dash_tensor_t *k, const dash_tensor_t *v,
                           dash_tensor_t *out, int block_size, float alpha, int causal, int gqa_groups) {
    return dash_attn_fwd_ex(q, k, v, out, block_size, alpha, causal, gqa_groups, nullptr);
}

}  // extern "C"

namespace {

struct BwdLayout {
    WsLayout F;  // Stage 0-1 state (recomputed) and the work lists
    size_t tau, drow, gd, dq, dkbar, bitmap, E, ref_off, ref_cnt, refs, qp, dop, lp, dp, dkacc, dvacc, total;
};

BwdLayout bwd_layout(const Geom &G, bool tc) {
    BwdLayout L{};
    L.F = ws_layout(G, true, true, false);
    size_t off = L.F.total;
    auto take = [&](size_t bytes) {
        size_t o = off;
        off += align256(bytes);
        return o;
    };
    const size_t rows = (size_t)G.b * G.nq * G.hq;
    const size_t bhb = (size_t)G.b * G.hkv * G.n_blk;
    const int tw = (int)((G.n_tiles + 31) / 32);
    L.tau = take(rows * 4);
    L.drow = take(rows * 4);
    L.gd = take((size_t)G.b * G.nq * G.hkv * (size_t)G.n_chunks * 4);
    L.dq = take(rows * G.d * 4);
    L.dkbar = take((size_t)G.b * G.n_chunks * G.hkv * G.d * 4);
    L.bitmap = take(bhb * tw * 4);
    L.E = take(bhb * G.n_tiles * 4);
    L.ref_off = take(bhb * 4);
    L.ref_cnt = take(bhb * 4);
    L.refs = take(bhb * G.n_tiles * 8);
    if (tc) {
        const size_t tiles = (size_t)G.b * G.hkv * G.n_tiles;
        L.qp = take(tiles * 128 * G.d * 2);
        L.dop = take(tiles * 128 * G.d * 2);
        L.lp = take(tiles * 128 * 4);
        L.dp = take(tiles * 128 * 4);
        L.dkacc = take((size_t)G.b * G.nk * G.hkv * G.d * 4);
        L.dvacc = take((size_t)G.b * G.nk * G.hkv * G.d * 4);
    }
    L.total = off;
    return L;
}

}  // namespace

extern "C" {

DASH_API size_t dash_bwd_workspace_bytes(int64_t batch, int64_t nq, int64_t nk, int hq, int hkv, int d,
                                         int block_size, int causal) {
    if (hkv <= 0 || hq % hkv || block_size <= 0 || nk <= 0 || batch < 0 || nq < 0) return 0;
    Geom G{};
    G.b = batch;
    G.nq = nq;
    G.nk = nk;
    G.hq = hq;
    G.hkv = hkv;
    G.g = hq / hkv;
    G.d = d;
    G.B = block_size;
    G.causal = causal;
    G.n_chunks = (int)(causal ? nk / block_size : (nk + block_size - 1) / block_size);
    G.n_blk = (int)((nk + block_size - 1) / block_size);
    G.tile_rows = 128 / G.g;
    G.n_tiles = (nq + G.tile_rows - 1) / G.tile_rows;
    G.words = (G.n_chunks + 31) / 32;
    G.kbar_cap = G.n_chunks;
    G.ct_cap = (G.n_chunks + 127) / 128;
    G.local = 1;
    return bwd_layout(G, true).total;
}

DASH_API int dash_attn_bwd(const dash_tensor_t *q, const dash_tensor_t *k, const dash_tensor_t *v,
                           const dash_tensor_t *out, const dash_tensor_t *dout, const float *lse, dash_tensor_t *dq,
                           dash_tensor_t *dk, dash_tensor_t *dv, int block_size, float alpha, int causal,
                           int gqa_groups, const dash_opts_t *opts) {
    dash_opts_t o = opts ? *opts : default_opts();
    int rc;
    if ((rc = check_opts(o))) return rc;
    if ((rc = validate_qkvo(q, k, v, out))) return rc;
    if ((rc = check_tensor(dout, "dout")) || (rc = check_tensor(dq, "dq")) || (rc = check_tensor(dk, "dk")) ||
        (rc = check_tensor(dv, "dv")))
        return rc;
    const dash_tensor_t *grads[4] = {dout, dq, dk, dv};
    for (const dash_tensor_t *t : grads)
        if (t->dtype != q->dtype) return fail(DASH_ERR_INVALID_ARG, "gradients must share the inputs' dtype");
    for (int a = 0; a < 4; ++a) {
        if (dout->shape[a] != q->shape[a] || dq->shape[a] != q->shape[a])
            return fail(DASH_ERR_INVALID_ARG, "dout and dq must have q's shape");
        if (dk->shape[a] != k->shape[a] || dv->shape[a] != k->shape[a])
            return fail(DASH_ERR_INVALID_ARG, "dk and dv must have k's shape");
    }
    if (!lse) return fail(DASH_ERR_INVALID_ARG, "lse is NULL (take it from the forward's opts->lse)");
    if (reinterpret_cast<uintptr_t>(lse) % 4) return fail(DASH_ERR_ALIGNMENT, "lse not 4-byte aligned");
    if (!(alpha > 1.f) || !isfinite(alpha)) return fail(DASH_ERR_INVALID_ARG, "alpha must be > 1");
    if (o.kbar || o.qbar || o.summary_cache || o.nk_dev)
        return fail(DASH_ERR_UNSUPPORTED,
                    "the backward pass pools the keys itself: no kbar, qbar, summary_cache or nk_dev");
    Geom G;
    if ((rc = make_geom(q, k, block_size, causal, gqa_groups, &G))) return rc;
    if ((rc = set_local(o, &G))) return rc;
    if (G.b == 0 || G.nq == 0) {
        // no query rows: every key and value gradient is zero
        cudaStream_t st = static_cast<cudaStream_t>(o.stream);
        dash_tensor_t *kv_grads[2] = {dk, dv};
        for (dash_tensor_t *t : kv_grads) {
            const size_t bytes = (size_t)t->shape[0] * t->shape[1] * t->shape[2] * t->shape[3] * esize(t->dtype);
            const bool dense = t->stride[2] == t->shape[3] && t->stride[1] == t->shape[2] * t->shape[3] &&
                               t->stride[0] == t->shape[1] * t->shape[2] * t->shape[3];
            if (!dense) return fail(DASH_ERR_UNSUPPORTED, "empty query with strided dk/dv");
            cudaError_t e = cudaMemsetAsync(t->data, 0, bytes, st);
            if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync");
        }
        return DASH_OK;
    }
    const bool tc = !(o.flags & DASH_FLAG_FORCE_SIMT) && attn_bwd_tc_supported(G, q->dtype);
    const BwdLayout BL = bwd_layout(G, tc);
    char *ws = nullptr;
    if ((rc = get_workspace(o, BL.total, &ws))) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(o.stream);
    // Stage 0 and Stage 1 again (deterministic: the forward's routing, thresholds and lists)
    const WsLayout &WL = BL.F;
    float *kb = reinterpret_cast<float *>(ws + WL.kbar);
    if ((rc = run_stage0(k, nullptr, TView{}, G, kb, st))) return rc;
    const bool regroup = !(o.flags & DASH_FLAG_NO_REGROUP) && G.n_tiles > 1;
    const ListsView LV = ws_lists(G, ws, WL, regroup);
    float *tau = reinterpret_cast<float *>(ws + BL.tau);
    uint32_t *mask = reinterpret_cast<uint32_t *>(ws + WL.mask);
    if ((rc = run_stage1(q, G, alpha, o, kb, tau, nullptr, mask, &LV, regroup, ws, WL, st))) return rc;
    BwdArgs a;
    a.G = G;
    a.L = LV;
    a.Q = view(q);
    a.K = view(k);
    a.V = view(v);
    a.O = view(out);
    a.dO = view(dout);
    a.dQ = view(dq);
    a.dK = view(dk);
    a.dV = view(dv);
    a.lse = lse;
    a.alpha = alpha;
    a.gamma = o.gamma;
    a.sigma = o.sigma;
    a.kbar = kb;
    a.tau = tau;
    a.mask = mask;
    a.logw = reinterpret_cast<float *>(ws + WL.logw);
    a.Drow = reinterpret_cast<float *>(ws + BL.drow);
    a.Gd = reinterpret_cast<float *>(ws + BL.gd);
    a.dQacc = reinterpret_cast<float *>(ws + BL.dq);
    a.dKbar = reinterpret_cast<float *>(ws + BL.dkbar);
    a.bitmap = reinterpret_cast<uint32_t *>(ws + BL.bitmap);
    a.E = reinterpret_cast<int32_t *>(ws + BL.E);
    a.ref_off = reinterpret_cast<int32_t *>(ws + BL.ref_off);
    a.ref_cnt = reinterpret_cast<int32_t *>(ws + BL.ref_cnt);
    a.refs = reinterpret_cast<int2 *>(ws + BL.refs);
    a.use_tc = tc;
    a.Qp = tc ? reinterpret_cast<uint8_t *>(ws + BL.qp) : nullptr;
    a.dOp = tc ? reinterpret_cast<uint8_t *>(ws + BL.dop) : nullptr;
    a.Lp = tc ? reinterpret_cast<float *>(ws + BL.lp) : nullptr;
    a.Dp = tc ? reinterpret_cast<float *>(ws + BL.dp) : nullptr;
    a.dKacc = tc ? reinterpret_cast<float *>(ws + BL.dkacc) : nullptr;
    a.dVacc = tc ? reinterpret_cast<float *>(ws + BL.dvacc) : nullptr;
    cudaError_t e = launch_attn_bwd(a, q->dtype, st);
    return e == cudaSuccess ? DASH_OK : cuda_fail(e, "backward pass");
}

DASH_API int dash_summary_cache_create(int64_t batch, int64_t max_nk, int hkv, int d, int block_size,
                                       dash_summary_cache_t **cache) {
    if (!cache) return fail(DASH_ERR_INVALID_ARG, "cache is NULL");
    *cache = nullptr;
    if (batch < 1 || hkv < 1 || max_nk < block_size || max_nk > (int64_t)1 << 30)
        return fail(DASH_ERR_INVALID_ARG, "bad batch, hkv or max_nk for a summary cache");
    if (d != 64 && d != 128) return fail(DASH_ERR_UNSUPPORTED, "head dim %d not in {64, 128}", d);
    if (block_size != 16 && block_size != 32 && block_size != 64 && block_size != 128)
        return fail(DASH_ERR_UNSUPPORTED, "block_size %d not in {16, 32, 64, 128}", block_size);
    auto *c = new dash_summary_cache{};
    c->b = batch;
    c->max_nk = max_nk;
    c->hkv = hkv;
    c->d = d;
    c->B = block_size;
    c->cap = (int)(max_nk / block_size);
    c->ct_cap = (c->cap + 127) / 128;
    c->done = 0;
    cudaError_t e = cudaGetDevice(&c->dev);
    if (e == cudaSuccess) e = cudaMalloc(&c->kbar, (size_t)batch * c->cap * hkv * d * sizeof(float));
    if (e == cudaSuccess) {
        const size_t sb = kbar_split_bytes(batch, hkv, d, c->ct_cap);
        e = cudaMalloc(&c->split, sb);
        if (e == cudaSuccess) e = cudaMemset(c->split, 0, sb);
    }
    if (e == cudaSuccess) e = cudaMalloc(&c->done_dev, sizeof(int));
    if (e == cudaSuccess) e = cudaMemset(c->done_dev, 0, sizeof(int));
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    if (e != cudaSuccess) {
        cudaFree(c->kbar);
        cudaFree(c->split);
        cudaFree(c->done_dev);
        delete c;
        return cuda_fail(e, "summary cache allocation");
    }
    *cache = c;
    return DASH_OK;
}

DASH_API int dash_summary_cache_update(dash_summary_cache_t *c, const dash_tensor_t *k, const dash_tensor_t *qbar,
                                       void *stream) {
    if (!c) return fail(DASH_ERR_INVALID_ARG, "cache is NULL");
    int rc = check_tensor(k, "k");
    if (rc) return rc;
    if (k->shape[0] != c->b || k->shape[2] != c->hkv || k->shape[3] != c->d || k->shape[1] > c->max_nk)
        return fail(DASH_ERR_INVALID_ARG, "k [%lld, %lld, %lld, %lld] does not fit the summary cache",
                    (long long)k->shape[0], (long long)k->shape[1], (long long)k->shape[2], (long long)k->shape[3]);
    dash_tensor_t q0 = *k;
    q0.shape[1] = 0;
    Geom G;
    if ((rc = make_geom(&q0, k, c->B, 1, 1, &G))) return rc;
    const int c1 = G.n_chunks;
    if (c1 < c->done)
        return fail(DASH_ERR_INVALID_ARG, "k has %d complete chunks but the cache pooled %lld (reset it first)", c1,
                    (long long)c->done);
    TView qv{};
    if (qbar) {
        Geom Gq = G;
        Gq.n_chunks = c->cap;
        if ((rc = check_qbar(qbar, Gq, &qv))) return rc;
    }
    if (c1 == c->done) return DASH_OK;
    G.kbar_cap = c->cap;
    G.ct_cap = c->ct_cap;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int c0 = (int)c->done;
    cudaError_t e = qbar ? launch_pool_keys_q(view(k), k->dtype, qv, qbar->dtype, G, c->kbar, st, c0, c1)
                         : launch_pool_keys(view(k), k->dtype, G, c->kbar, st, c0, c1);
    if (e != cudaSuccess) return cuda_fail(e, "summary cache pooling");
    // the split tiles the new chunks fall in (chunks past c1 stay zero until they complete)
    e = launch_kbar_split(c->kbar, G, c->split, c0 / 128, (c1 + 127) / 128, st);
    if (e != cudaSuccess) return cuda_fail(e, "summary cache split");
    c->done = c1;
    e = launch_set_int(c->done_dev, c1, st);  // the device-side count follows
    if (e != cudaSuccess) return cuda_fail(e, "summary cache count");
    return DASH_OK;
}

DASH_API int dash_summary_cache_reset(dash_summary_cache_t *c) {
    if (!c) return fail(DASH_ERR_INVALID_ARG, "cache is NULL");
    cudaError_t e = cudaDeviceSynchronize();  // no step in flight still counts on the old chunks
    if (e == cudaSuccess) e = cudaMemset(c->done_dev, 0, sizeof(int));
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_fail(e, "summary cache reset");
    c->done = 0;
    return DASH_OK;
}

DASH_API int64_t dash_summary_cache_chunks(const dash_summary_cache_t *c) { return c ? c->done : -1; }

DASH_API const float *dash_summary_cache_kbar(const dash_summary_cache_t *c) { return c ? c->kbar : nullptr; }

DASH_API int dash_summary_cache_destroy(dash_summary_cache_t *c) {
    if (!c) return DASH_OK;
    cudaError_t e = cudaDeviceSynchronize();
    cudaFree(c->kbar);
    cudaFree(c->split);
    cudaFree(c->done_dev);
    delete c;
    return e == cudaSuccess ? DASH_OK : cuda_fail(e, "cudaDeviceSynchronize");
}

DASH_API int dash_sync_status(void *stream) {
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    int dev_err = take_device_error_tc() | take_device_error_decode() | take_device_error_select() |
                  take_device_error_bwd();
    if (dev_err) return fail(DASH_ERR_DEVICE_TIMEOUT, "a device-side bounded wait ran out");
    return DASH_OK;
}

DASH_API int dash_release(void) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    dash::release_host_staging();
    std::lock_guard<std::mutex> lk(g_ws_mu);
    if (dev >= 0 && dev < 128 && g_ws[dev].p) {
        e = cudaDeviceSynchronize();
        if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
        cudaFree(g_ws[dev].p);
        g_ws[dev] = DevWs{};
    }
    return DASH_OK;
}

}  // extern "C"

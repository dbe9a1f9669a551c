/*
 * dash_attn.h -- C ABI of the B200 (sm_100a) DashAttention forward library.
 *
 * DashAttention is defined in "DashAttention: Differentiable and Adaptive
 * Sparse Hierarchical Attention" (arXiv 2605.18753), cited here as [Dash].
 * The forward pass has three stages:
 *   Stage 0  chunk summaries  k̄_c = mean of the chunk's keys
 *            ([Dash] §3.1 Eq. 3 with the summary query at its zero
 *            initialisation, which the paper notes is exactly mean pooling)
 *   Stage 1  entmax routing: zbar_{i,c} = <q_i, k̄_c>/sqrt(d) over the chunks
 *            visible to row i, w^(h) = alpha-entmax(gamma * zbar) per head,
 *            averaged over the GQA group, support = union of the heads'
 *            supports ([Dash] §3.2 Eq. 4; §2 Eq. 2)
 *   Stage 2  softmax attention over the routed chunks plus the diagonal
 *            chunk, with the routing distribution folded in as the bias
 *            d = (log w - mu)/sigma ([Dash] §3.3 Eq. 7, §3.4 Prop. 1)
 *
 * Conventions shared by every entry point
 *   - Tensors are [batch, seq, heads, dim] with dim contiguous (stride[3] = 1);
 *     other strides are free (elements).  Q and O: [b, nq, hq, d];
 *     K and V: [b, nk, hkv, d].  hq = gqa_groups * hkv.
 *   - All data pointers are DEVICE pointers on the current CUDA device, owned
 *     by the caller; the library never frees caller memory.
 *   - Causal alignment is bottom-right: query row i sits at key position
 *     p_i = i + nk - nq.  Its chunk is c_i = floor(p_i / B).  It routes over the
 *     complete chunks c < min(c_i, floor(nk / B)) and always attends its
 *     diagonal tokens c_i*B .. p_i (bias 0) ([Dash] App. G Algs. 2-3).
 *     Non-causal: every chunk, a trailing partial chunk included, is routed,
 *     and there is no diagonal branch.
 *   - n_chunks (routing chunks) = floor(nk/B) if causal else ceil(nk/B).
 *   - Calls are asynchronous on the given stream; the return value reports
 *     argument validation and launch errors.  Errors found on the device
 *     (a bounded wait that ran out) are reported by dash_sync_status().
 *   - Supported: dtype f32 or bf16 (q, k, v, out all the same), d in {64, 128},
 *     block_size in {16, 32, 64, 128}, alpha > 1, 1 <= gqa_groups <= 16.
 *   - Base pointers must be 16-byte aligned and every stride but the last a
 *     multiple of 16 bytes, otherwise DASH_ERR_ALIGNMENT.
 */
#ifndef DASH_ATTN_H
#define DASH_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define DASH_API __attribute__((visibility("default")))

typedef enum {
    DASH_OK = 0,
    DASH_ERR_INVALID_ARG = -1,    /* bad shape, value or null pointer */
    DASH_ERR_UNSUPPORTED = -2,    /* valid but outside the supported set above */
    DASH_ERR_ALIGNMENT = -3,      /* base pointer or stride not 16-byte aligned */
    DASH_ERR_WORKSPACE = -4,      /* caller workspace too small */
    DASH_ERR_CUDA = -5,           /* a CUDA runtime call failed */
    DASH_ERR_DEVICE_TIMEOUT = -6  /* a device-side bounded wait ran out */
} dash_status_t;

typedef enum { DASH_F32 = 0, DASH_BF16 = 1 } dash_dtype_t;

/* A strided 4-D device tensor [batch, seq, heads, dim]. */
typedef struct {
    void *data;
    dash_dtype_t dtype;
    int64_t shape[4];
    int64_t stride[4]; /* in elements; stride[3] must be 1 */
} dash_tensor_t;

/* Stage-2 work lists.  The query rows of a (batch, kv head) are grouped into
 * tiles of tile_rows rows (x gqa_groups heads = 128 rows of the tensor-core
 * tile).  For each tile the list holds the union of the chunks any of its rows
 * attends (routed chunks and each row's diagonal chunk), and a per-row bias.
 * Layout (all device memory, caller-owned, contiguous):
 *   count [b][hkv][n_tiles]                    int32   entries in the list
 *   ids   [b][hkv][n_tiles][cap]               int32   chunk ids (any order)
 *   bias  [b][hkv][n_tiles][cap][tile_rows]    float32 bias of that chunk for
 *         that tile row: (log w_c - mu)/sigma if the row routed it, 0 if it is the
 *         row's diagonal chunk, -inf if the row does not attend it.
 *   rows  [b][hkv][n_tiles][tile_rows]         int32   query index of each tile
 *         row, -1 for an unused row; rows may come in any order (Stage 1 groups
 *         rows with similar routed sets into the same tile).  NULL means tile t
 *         holds the consecutive rows t*tile_rows .. t*tile_rows + tile_rows - 1.
 * n_tiles = ceil(nq / tile_rows); cap = ceil(nk / block_size); tile_rows =
 * 128 / gqa_groups.  Stage 2 also masks key j > p_i when causal and keys >= nk. */
typedef struct {
    int32_t *count;
    int32_t *ids;
    float *bias;
    int32_t *rows;
    int64_t n_tiles;
    int32_t cap;
    int32_t tile_rows;
} dash_lists_t;

#define DASH_FLAG_FORCE_SIMT 0x1      /* Stage 2 on the CUDA-core path (testing) */
#define DASH_FLAG_NO_REGROUP 0x2      /* keep consecutive query rows in each tile (no regrouping
                                         of rows by routed-set size) */
#define DASH_FLAG_LOCAL2 0x4         /* the two-block local window of [Dash] App. B.1.1: the chunk
                                         before the query's own is attended in full with bias 0
                                         together with the diagonal chunk, and routing covers the
                                         chunks before it (causal only) */
#define DASH_FLAG_TEST_TIMEOUT 0x100  /* testing only: Stage 2 waits on a barrier nothing
                                         arrives at, gives up after a short bound and
                                         reports DASH_ERR_DEVICE_TIMEOUT */

/* Persistent chunk-summary cache for incremental decoding (see dash_summary_cache_create). */
typedef struct dash_summary_cache dash_summary_cache_t;

/* Optional settings.  Fill with dash_opts_init(). */
typedef struct {
    float sigma;            /* prior strength sigma > 0; default 1e8 ([Dash] App. F.5 picks 1e8) */
    float gamma;            /* Stage-1 logit scale gamma > 0 ([Dash] Eq. 4); default 1 */
    void *stream;           /* cudaStream_t; NULL = the legacy default stream */
    void *workspace;        /* device scratch; NULL = library-managed (cached per device) */
    size_t workspace_bytes; /* size of workspace; see dash_workspace_bytes() */
    const float *kbar;      /* optional precomputed chunk summaries [b][n_chunks][hkv][d] fp32
                               contiguous (from dash_pool_keys, e.g. a decode cache) */
    int flags;              /* DASH_FLAG_* */
    const dash_tensor_t *qbar; /* optional learned summary queries of Stage 0, see
                               dash_pool_keys_q; NULL = q̄ = 0 (mean pooling).  Not
                               together with kbar. */
    const dash_summary_cache_t *summary_cache; /* optional: Stage 0 and the summaries'
                               operand form come from this cache, which must hold every
                               complete chunk of k (causal only; not with kbar or qbar) */
    float *lse;             /* optional output of the forward passes (dash_attn_fwd_ex,
                               dash_sparse_attn_fwd): [b][nq][hq] fp32 contiguous, the natural
                               log-sum-exp of each row's Stage-2 logits z + d over the keys it
                               attends (the normaliser of Eq. 7's softmax); the backward pass
                               (dash_attn_bwd) takes it back.  NULL = not written. */
    const int64_t *nk_dev;  /* optional, dash_attn_fwd_ex only: DEVICE pointer to the number of
                               valid keys, read by the kernels when they run, so that one
                               captured launch sequence (a CUDA graph of a decoding step)
                               serves every length.  k and v then describe the preallocated
                               cache (shape[1] = its capacity, at most the summary cache's
                               max_nk); keys at and past *nk_dev are ignored and the new query
                               rows sit at the last positions before it.  Needs opts->
                               summary_cache, which the call itself brings up to date on the
                               device (up to 16 chunks completed since the previous call;
                               more: call dash_summary_cache_update first), and the decoding
                               path: bf16, nq * gqa_groups <= 16, 1 <= *nk_dev <= capacity,
                               *nk_dev >= nq.  NULL = k's shape[1] is the length. */
} dash_opts_t;

/* Fill *opts with the defaults above.  Returns DASH_OK or DASH_ERR_INVALID_ARG (NULL). */
DASH_API int dash_opts_init(dash_opts_t *opts);

/* Full forward pass, Stages 0-2 ([Dash] §3, App. G Algs. 1-3).
 *   q, out [b, nq, hq, d]; k, v [b, nk, hkv, d]; same dtype.
 *   block_size B, alpha > 1, causal 0/1, gqa_groups = hq / hkv.
 * Uses the default options (sigma 1e8, gamma 1, default stream, library
 * workspace).  Returns a dash_status_t. */
DASH_API int dash_attn_fwd(const dash_tensor_t *q, const dash_tensor_t *k, const dash_tensor_t *v,
                           dash_tensor_t *out, int block_size, float alpha, int causal, int gqa_groups);

/* As dash_attn_fwd with explicit options (opts may be NULL for defaults). */
DASH_API int dash_attn_fwd_ex(const dash_tensor_t *q, const dash_tensor_t *k, const dash_tensor_t *v,
                              dash_tensor_t *out, int block_size, float alpha, int causal, int gqa_groups,
                              const dash_opts_t *opts);

/* Stage 0 alone ([Dash] §3.1 Eq. 3, App. G Alg. 1): kbar [b][n_chunks][hkv][d]
 * fp32 contiguous, n_chunks = floor(nk/B) if causal else ceil(nk/B) (a partial
 * chunk is the mean of its real keys).  stream may be NULL. */
DASH_API int dash_pool_keys(const dash_tensor_t *k, int block_size, int causal, float *kbar, void *stream);

/* Stage 0 with a learned summary query ([Dash] §3.1 Eq. 3, App. G Alg. 1):
 *   kbar_c^(r) = sum_{t in chunk c} softmax_t(<qbar_c^(r), k_t> / sqrt(d)) k_t,
 * one online softmax over the chunk's keys, which also serve as the values.
 *   k     [b, nk, hkv, d] f32 or bf16, as for dash_pool_keys.
 *   qbar  [1 or b, n_chunks, hkv, d] f32 or bf16 (independent of k's dtype): the
 *         summary query of every chunk and kv head, with any rotary position
 *         encoding already applied by the caller (the library applies none).  A
 *         stride of 0 broadcasts one query over the chunks (and shape[0] == 1 over
 *         the batch), e.g. a per-head learned query without position encoding.
 *   kbar  [b][n_chunks][hkv][d] fp32 contiguous output; n_chunks as for dash_pool_keys.
 * qbar = 0 gives exactly the mean of dash_pool_keys.  Errors as for dash_pool_keys,
 * plus DASH_ERR_INVALID_ARG when qbar's shape does not match. */
DASH_API int dash_pool_keys_q(const dash_tensor_t *k, const dash_tensor_t *qbar, int block_size, int causal,
                              float *kbar, void *stream);

/* Persistent chunk-summary cache ([Dash] §3.5: a chunk's summary is written once the
 * chunk is complete and reused by every later query position and decoding step).  It
 * holds, in device memory it owns, the fp32 summaries of up to floor(max_nk / block_size)
 * chunks of `batch` sequences and their bf16 hi + lo split (the operand form of the
 * tensor-core Stage 1), so that a decoding step pools and splits nothing.
 * create: allocates on the current device, no chunk pooled.  Errors DASH_ERR_INVALID_ARG
 *   (sizes, NULL cache), DASH_ERR_UNSUPPORTED (d or block size), DASH_ERR_CUDA (allocation). */
DASH_API int dash_summary_cache_create(int64_t batch, int64_t max_nk, int hkv, int d, int block_size,
                                       dash_summary_cache_t **cache);
/* Pools every chunk completed since the last update: k [batch, nk, hkv, d] (f32 or bf16)
 * holds the sequences' first nk <= max_nk keys; chunks [pooled, floor(nk/B)) are pooled
 * (with the learned summary queries qbar [1 or batch, floor(max_nk/B), hkv, d] when not
 * NULL, as in dash_pool_keys_q) and the split tiles they fall in are rebuilt.  The keys of
 * pooled chunks must not change afterwards (reset the cache first).  Asynchronous on
 * stream.  DASH_ERR_INVALID_ARG when k does not match the cache or holds fewer complete
 * chunks than were pooled. */
DASH_API int dash_summary_cache_update(dash_summary_cache_t *cache, const dash_tensor_t *k,
                                       const dash_tensor_t *qbar, void *stream);
/* Forgets every pooled chunk (new sequences); waits for the device first. */
DASH_API int dash_summary_cache_reset(dash_summary_cache_t *cache);
/* Chunks pooled so far by dash_summary_cache_update (catch-up steps of a forward with
 * opts->nk_dev count on the device only); -1 for a NULL cache. */
DASH_API int64_t dash_summary_cache_chunks(const dash_summary_cache_t *cache);
/* The fp32 summaries [batch][floor(max_nk/B)][hkv][d] (device memory the cache owns). */
DASH_API const float *dash_summary_cache_kbar(const dash_summary_cache_t *cache);
/* Waits for the device, then frees the cache.  NULL is a no-op. */
DASH_API int dash_summary_cache_destroy(dash_summary_cache_t *cache);

/* Stage 1 alone ([Dash] §3.2 Eq. 4; App. G Alg. 2).  Every output is optional
 * (NULL to skip):
 *   tau   [b][nq][hq]             fp32 threshold in the (alpha-1)*gamma*zbar domain;
 *                                 NaN for a row with no visible chunk
 *   w     [b][nq][hkv][n_chunks]  fp32 group distribution, 0 outside the support
 *   mask  [b][nq][hkv][ceil(n_chunks/32)] uint32 routed-chunk bits (bit c%32 of
 *                                 word c/32), the bit-packed mask of [Dash] §3.5
 *   lists Stage-2 work lists (see dash_lists_t), built with opts->sigma
 * Returns a dash_status_t. */
DASH_API int dash_block_select(const dash_tensor_t *q, const dash_tensor_t *k, int block_size, float alpha,
                               int causal, int gqa_groups, float *tau, float *w, uint32_t *mask,
                               const dash_lists_t *lists, const dash_opts_t *opts);

/* Backward pass of dash_attn_fwd_ex: the gradients of sum(dout * out) with respect to
 * q, k and v ([Dash] §3.3-3.4 and App. A: the hierarchy is differentiable end to end).
 * Gradients flow through Stage 2 (softmax attention over the routed and local keys),
 * through the prior bias d_c = (log w_c - mu)/sigma into the group distribution w, through
 * each head's alpha-entmax Jacobian into the Stage-1 scores, and through the mean pooling
 * of Stage 0 into the keys; the routed sets themselves are piecewise constant and carry
 * no gradient.  Stage 0 and Stage 1 are recomputed (deterministically: the forward's
 * routing), Stage 2's probabilities are recomputed from lse.
 *   q, k, v, out, block_size, alpha, causal, gqa_groups and opts (sigma, gamma, flags
 *     DASH_FLAG_LOCAL2 / NO_REGROUP / FORCE_SIMT, stream, workspace) exactly as given to
 *     the forward that produced out;
 *   dout [b, nq, hq, d] the output gradient; lse [b][nq][hq] fp32 from the forward's
 *     opts->lse;
 *   dq [b, nq, hq, d], dk, dv [b, nk, hkv, d]: outputs (overwritten), same dtype as q.
 * Reproducibility: dq is identical between runs; dk (whose chunk-summary share, and on
 * the tensor-core path its Stage-2 share, is summed with fp32 atomics) and, on the
 * tensor-core path with 128 or more query tiles per (batch, kv head), dv may differ in
 * their last bits.
 * Not supported with a summary cache, given summaries or learned summary queries
 * (DASH_ERR_UNSUPPORTED).  Workspace: dash_bwd_workspace_bytes().  Errors as for
 * dash_attn_fwd_ex; DASH_ERR_INVALID_ARG when a gradient's shape or dtype does not
 * match or lse is NULL. */
DASH_API int dash_attn_bwd(const dash_tensor_t *q, const dash_tensor_t *k, const dash_tensor_t *v,
                           const dash_tensor_t *out, const dash_tensor_t *dout, const float *lse, dash_tensor_t *dq,
                           dash_tensor_t *dk, dash_tensor_t *dv, int block_size, float alpha, int causal,
                           int gqa_groups, const dash_opts_t *opts);

/* The forward pass of dash_attn_fwd_ex on host-resident q, k, v and out, through device
 * buffers of the same shapes, with the copies overlapped with the computation: the query
 * rows are taken in up to n_slices slices of whole multiples of 1024 rows, in order (0 =
 * automatic: 16 from 16K rows, 4 from 2K, else 1); slice s's rows and the keys they can see (with a causal mask the key prefix up
 * to the slice's last row position, else all keys) are copied in on one internal stream,
 * the slice's forward runs on opts->stream once they have landed, and its output rows are
 * copied out on a second internal stream, so the copies of later slices and the copy back
 * of earlier ones overlap the computation.  The output is bit-identical to
 * dash_attn_fwd_ex(q_dev, k_dev, v_dev, out_dev, ...).
 *   q_host, k_host, v_host, out_host  host memory (page-locked for the copies to be
 *       asynchronous), [batch, seq, heads, dim] with packed rows: stride = {any >= seq *
 *       heads * dim, heads * dim, dim, 1};
 *   q_dev, k_dev, v_dev, out_dev      device buffers, same shapes, dtypes and row packing
 *       (the caller's; their contents on return are the inputs and the output);
 *   block_size, alpha, causal, gqa_groups, opts as for dash_attn_fwd_ex, without
 *       summary_cache, nk_dev, kbar, qbar or lse (DASH_ERR_UNSUPPORTED).
 * Asynchronous: the call returns once everything is enqueued; the host output is complete
 * when opts->stream reaches the point of the call (the stream waits for the last copy back).
 * The inputs must stay unchanged, and the host output untouched, until then.  The device
 * buffers are not written before the stream's earlier work on them is done.  Not for stream
 * capture (the internal streams are outside it).  Errors as for dash_attn_fwd_ex; a copy
 * that fails returns DASH_ERR_CUDA. */
DASH_API int dash_attn_fwd_host(const dash_tensor_t *q_host, const dash_tensor_t *k_host,
                                const dash_tensor_t *v_host, dash_tensor_t *out_host, const dash_tensor_t *q_dev,
                                const dash_tensor_t *k_dev, const dash_tensor_t *v_dev, dash_tensor_t *out_dev,
                                int block_size, float alpha, int causal, int gqa_groups, int n_slices,
                                const dash_opts_t *opts);

/* Device workspace dash_attn_bwd needs for a problem (bytes, an upper bound). */
DASH_API size_t dash_bwd_workspace_bytes(int64_t batch, int64_t nq, int64_t nk, int hq, int hkv, int d,
                                         int block_size, int causal);

/* Stage-2 work lists from a caller's routing mask, e.g. the random block masks of a
 * controlled-sparsity benchmark ([Dash] §5.2 and App. B.2 inject such a mask at Stage 2)
 * or an external router.
 *   mask  [batch][nq][hkv][words] uint32 device memory, words = ceil(n_chunks / 32) with
 *         n_chunks = floor(nk/B) if causal else ceil(nk/B); bit c % 32 of word c / 32 set
 *         = chunk c routed for that (query row, kv head).  Only chunks the row may route
 *         (c < floor(p_i / B) when causal) may be set; other bits make the list longer
 *         without changing the result.
 *   Every routed chunk gets bias 0 (a uniform prior over the routed set: the sigma -> inf
 *   limit of Prop. 1); each row's diagonal chunk is added as in dash_block_select.
 *   regroup 1 groups rows with similar routed sets into tiles (lists->rows required),
 *   0 keeps consecutive rows.
 * lists: caller-owned buffers with the geometry of dash_lists_geometry.  Asynchronous on
 * stream.  Errors: DASH_ERR_INVALID_ARG (NULL or mismatched buffers, bad sizes),
 * DASH_ERR_UNSUPPORTED (gqa_groups outside [1, 16] or a block size outside {16, 32, 64, 128}). */
DASH_API int dash_lists_from_mask(const uint32_t *mask, int64_t batch, int64_t nq, int64_t nk, int hkv,
                                  int block_size, int gqa_groups, int causal, int regroup, dash_lists_t *lists,
                                  void *stream);

/* Stage 2 alone ([Dash] §3.3 Eq. 7 in the bias form of Prop. 1; App. G Alg. 3)
 * on caller-supplied lists (for example from dash_block_select, or a random
 * mask).  Returns a dash_status_t. */
DASH_API int dash_sparse_attn_fwd(const dash_tensor_t *q, const dash_tensor_t *k, const dash_tensor_t *v,
                                  dash_tensor_t *out, const dash_lists_t *lists, int block_size, int causal,
                                  int gqa_groups, const dash_opts_t *opts);

/* Sizes of the lists buffers for a problem: *count_bytes, *ids_bytes,
 * *bias_bytes, *rows_bytes (any may be NULL) and the geometry (*n_tiles, *cap,
 * *tile_rows).  Returns DASH_OK or DASH_ERR_INVALID_ARG. */
DASH_API int dash_lists_geometry(int64_t batch, int64_t nq, int64_t nk, int hkv, int block_size, int gqa_groups,
                                 int64_t *n_tiles, int32_t *cap, int32_t *tile_rows, size_t *count_bytes,
                                 size_t *ids_bytes, size_t *bias_bytes, size_t *rows_bytes);

/* Device workspace dash_attn_fwd_ex takes for a problem with the library-managed
 * workspace (bytes): an upper bound over the options (it counts the pooled-key area even
 * where a summary cache makes it unnecessary).  A prefill whose Stage-1 state and work
 * lists would exceed 1 GB runs its query rows in slices (multiples of 1024 rows) that fit
 * 1 GB, so the figure stays near 1 GB at any length; with a caller workspace the slices
 * are sized to that workspace instead (at least 1024 rows; DASH_ERR_WORKSPACE when even
 * those do not fit). */
DASH_API size_t dash_workspace_bytes(int64_t batch, int64_t nq, int64_t nk, int hq, int hkv, int d,
                                     int block_size, int causal);

/* Thread-local message describing the last error returned on this thread. */
DASH_API const char *dash_last_error(void);

/* Synchronise the stream (NULL = default) and report device-side errors:
 * DASH_ERR_DEVICE_TIMEOUT if a kernel's bounded wait ran out since the last
 * call (the flag is then cleared), DASH_ERR_CUDA on a CUDA error, else DASH_OK. */
DASH_API int dash_sync_status(void *stream);

/* Free the library-managed workspace of the current device. */
DASH_API int dash_release(void);

/* Size of the static scratch area that dash_attn_fwd_noalloc works in (32 MiB,
 * reserved on every device that loads the library, until the process exits). */
#define DASH_NOALLOC_SCRATCH_BYTES (32u << 20)

/* dash_attn_fwd_ex for callers that cannot let the library allocate device
 * memory: serving engines that hand nearly all of HBM to their own KV-cache
 * pool (a run-time cudaMalloc may fail there), multi-stream loops that cannot
 * take the device-wide synchronisation of cudaFree, hosts that route all device
 * memory through their own allocator.  It calls no cudaMalloc, cudaFree or other
 * allocating routine; the intermediates go to a static device array of
 * DASH_NOALLOC_SCRATCH_BYTES inside the library.  The paper has no counterpart
 * to this entry point: it is a deployment variant of dash_attn_fwd_ex.
 *   Arguments and result as dash_attn_fwd_ex; opts may be NULL, and
 *   opts->workspace must be NULL (DASH_ERR_INVALID_ARG otherwise).
 *   A long prefill runs its query rows in slices that fit the area; a problem whose
 *   smallest slice (1024 rows) still needs more scratch than DASH_NOALLOC_SCRATCH_BYTES
 *   is rejected with DASH_ERR_WORKSPACE before anything is launched.
 *   The first call on a device (with that device current) looks up the array's
 *   device address with cudaGetSymbolAddress; make that first call before any
 *   stream capture.  The address is kept for the life of the device's primary
 *   context: do not call this entry point again after a cudaDeviceReset.
 *   All calls share the one array, which keeps the last call's contents (the
 *   forward pass writes every scratch word before reading it).  Calls whose
 *   execution overlaps on the GPU (different streams or host threads) race on
 *   it: serialise them. */
DASH_API int dash_attn_fwd_noalloc(const dash_tensor_t *q, const dash_tensor_t *k, const dash_tensor_t *v,
                                   dash_tensor_t *out, int block_size, float alpha, int causal, int gqa_groups,
                                   const dash_opts_t *opts);

/* Library version string. */
DASH_API const char *dash_version(void);

#ifdef __cplusplus
}
#endif

#endif /* DASH_ATTN_H */

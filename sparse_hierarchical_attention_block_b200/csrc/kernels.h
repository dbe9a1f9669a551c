// kernels.h -- host-side launchers of the DashAttention kernels (internal).
#pragma once

#include "dash_common.cuh"

namespace dash {

// Stage 0 (pool_keys.cu)
// chunks [c0, c1) (c1 < 0: every chunk) into kbar, whose batch stride is G.kbar_cap chunks
cudaError_t launch_pool_keys(const TView &K, dash_dtype_t dt, const Geom &G, float *kbar, cudaStream_t st, int c0 = 0,
                             int c1 = -1);
// learned summary queries: view [b (stride 0 to broadcast)][n_chunks][hkv][d] of dtype qdt
cudaError_t launch_pool_keys_q(const TView &K, dash_dtype_t dt, const TView &Qbar, dash_dtype_t qdt, const Geom &G,
                               float *kbar, cudaStream_t st, int c0 = 0, int c1 = -1);

// Chunks a decoding step may complete since the previous one when the summary cache
// catches up on the device (a device-resident key length).
constexpr int kMaxNewChunks = 16;
// pool the chunks completed since the cache's device count (G.nk_dev, G.chunks_dev set;
// G.kbar_cap / G.ct_cap the cache's), rebuild their split tiles and advance the count
cudaError_t launch_cache_catch_up(const TView &K, dash_dtype_t dt, const Geom &G, float *kbar, uint8_t *split,
                                  cudaStream_t st);
cudaError_t launch_set_int(int *dst, int v, cudaStream_t st);

// Stage 1 (block_select.cu)
struct SelectOut {
    float *tau;        // [b][nq][hq] or null
    float *w;          // [b][nq][hkv][n_chunks] or null
    uint32_t *mask;    // [b][nq][hkv][words] (required)
    float *logw;       // [b][hkv][n_chunks][nq] (logw_index) log w of the routed chunks (when lists are built)
    float *mu;         // [b][nq][hkv] mean log w over the routed chunks (when lists are built)
};
cudaError_t launch_select_rows(const TView &Q, dash_dtype_t dt, const float *kbar, const Geom &G, float alpha,
                               float gamma, float sigma, const SelectOut &o, cudaStream_t st);
bool select_tile_supported(const Geom &G, dash_dtype_t dt);
size_t select_tile_workspace(const Geom &G);
// Routing of every (row, head) pair on tensor cores (up to 2048 chunks): tau, optional
// dense w, the bit mask (required), log w of the routed chunks and mu (optional; both
// are needed to build work lists).  `work` holds select_tile_workspace(G) bytes.
// presplit: the split summaries already built (a persistent cache, G.ct_cap tiles per
// (batch, kv head)); null = split kbar into work first
cudaError_t launch_select_tile(const TView &Q, const float *kbar, const Geom &G, float alpha, float gamma,
                               float *tau, float *w, uint32_t *mask, float *logw, float *mu, void *work,
                               cudaStream_t st, const uint8_t *presplit = nullptr);
// split the summaries of chunk tiles [ct0, ct1) of kbar (batch stride G.kbar_cap chunks) into
// split (G.ct_cap tiles per (batch, kv head)); chunks >= G.n_chunks are written as zero
cudaError_t launch_kbar_split(const float *kbar, const Geom &G, uint8_t *split, int ct0, int ct1, cudaStream_t st);
size_t kbar_split_bytes(int64_t batch, int hkv, int d, int ct_cap);
// Regroup the query rows of each window of tiles by routed-set size and build the
// tiles' work lists (with the row permutation) from the per-row masks and biases.
bool regroup_supported(const Geom &G);
cudaError_t launch_regroup_compact(const Geom &G, const uint32_t *mask, const float *logw, const float *mu,
                                   float sigma, const ListsView &L, cudaStream_t st);
cudaError_t launch_compact(const Geom &G, const uint32_t *mask, const float *logw, const float *mu, float sigma,
                           const ListsView &L, cudaStream_t st);

// Stage 2 (attn_simt.cu, attn_tc.cu, attn_decode.cu)
// lse (optional, [b][nq][hq] fp32): natural log-sum-exp of each row's biased logits
cudaError_t launch_attn_simt(const TView &Q, const TView &K, const TView &V, const TView &O, dash_dtype_t dt,
                             const Geom &G, const ListsView &L, cudaStream_t st, float *lse = nullptr);
bool attn_tc_supported(const Geom &G, dash_dtype_t dt);
cudaError_t launch_attn_tc(const TView &Q, const TView &K, const TView &V, const TView &O, const Geom &G,
                           const ListsView &L, int flags, cudaStream_t st, float *lse = nullptr);
bool attn_decode_supported(const Geom &G, dash_dtype_t dt);
size_t attn_decode_workspace(const Geom &G);
cudaError_t launch_attn_decode(const TView &Q, const TView &K, const TView &V, const TView &O, const Geom &G,
                               const ListsView &L, void *work, cudaStream_t st, float *lse = nullptr);

// Backward pass (bwd.cu, attn_bwd_tc.cu).  Everything the kernels need: the forward's
// inputs and output, the output gradient, the forward's lse, the recomputed Stage 0-1
// state (summaries, thresholds, masks, log w, work lists) and the workspace areas.
struct BwdArgs {
    Geom G;
    ListsView L;
    TView Q, K, V, O, dO, dQ, dK, dV;
    const float *lse;                  // [b][nq][hq] natural log-sum-exp of the forward
    float alpha, gamma, sigma;
    const float *kbar;                 // [b][kbar_cap][hkv][d] fp32 chunk summaries
    const float *tau;                  // [b][nq][hq] Stage-1 thresholds
    const uint32_t *mask;              // [b][nq][hkv][words] routed chunks
    const float *logw;                 // log w of the routed chunks (logw_index layout)
    float *Drow;                       // [b][nq][hq] <dO, O>
    float *Gd;                         // G per (row, routed chunk), logw_index layout
    float *dQacc;                      // [b][nq][hq][d] fp32
    float *dKbar;                      // [b][n_chunks][hkv][d] fp32
    uint32_t *bitmap;                  // [b][hkv][n_blk][ceil(n_tiles/32)] tiles attending each key block
    int32_t *E;                        // [b][hkv][n_blk][n_tiles] entry index of the block in the tile's list
    int32_t *ref_off, *ref_cnt;        // [b][hkv][n_blk] the block's (tile, entry) pairs
    int2 *refs;                        // [b][hkv][n_tiles * n_blk] pairs
    bool use_tc;                       // tensor-core Stage-2 kernels (bf16, d = 128, B in {64, 128})
    uint8_t *Qp, *dOp;                 // tensor-core path: [b][hkv][n_tiles][128][d] bf16 tile rows
    float *dKacc, *dVacc;              // tensor-core path: [b][nk][hkv][d] fp32 accumulators
    float *Lp, *Dp;                    // [b][hkv][n_tiles][128] lse (exp2 domain, +inf = empty) and D
};
cudaError_t launch_attn_bwd(const BwdArgs &a, dash_dtype_t dt, cudaStream_t st);
bool attn_bwd_tc_supported(const Geom &G, dash_dtype_t dt);
cudaError_t launch_attn_bwd_tc_dq(const BwdArgs &a, cudaStream_t st);
cudaError_t launch_attn_bwd_tc_dkdv(const BwdArgs &a, cudaStream_t st);

// The host-staged forward's copy streams of the current device (freed by dash_release).
void release_host_staging();

}  // namespace dash

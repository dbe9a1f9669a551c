"""Helpers shared by the GPU parity tests: run the CUDA path through the C ABI,
run the oracle on the same inputs, and compare with the acceptance rules.

Acceptance (stated for this method's forward pass):
  * Stage-1 supports identical, except chunks whose score x_c = (alpha-1)*gamma*zbar_c
    lies within 1e-3 of some head's oracle threshold (several supports are then
    equally correct);
  * thresholds within TAU_TOL and block probabilities w within 1e-4;
  * outputs within max-abs 2e-2 and mean-abs 2e-3 (bf16), 1e-4 / 1e-5 (fp32).
  Rows whose support differs at an allowed chunk are scored against the
  oracle's Stage 2 evaluated on the GPU's support (the oracle's own Stage 1
  values for every chunk both select, the GPU's w for a chunk only the GPU
  selected); every other row must match the oracle's own forward outright.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
import sparse_hierarchical_attention_block_b200 as dash

SUPPORT_WINDOW = 1e-3
TAU_TOL = 1e-4      # a tenth of the support window: fp32 threshold of O(1) scores
W_TOL = 1e-4
OUT_TOL = {torch.bfloat16: (2e-2, 2e-3), torch.float32: (1e-4, 1e-5)}


def unpack_mask(mask_words: np.ndarray, n_chunks: int) -> np.ndarray:
    """[..., words] uint32 -> [..., n_chunks] bool."""
    w = mask_words.view(np.uint32)
    c = np.arange(n_chunks)
    return ((w[..., c // 32] >> (c % 32).astype(np.uint32)) & 1).astype(bool)


def gpu_stage1(q, k, block_size, alpha, causal, sigma=1e8, gamma=1.0, qbar=None, local=1):
    b, nq, hq, _ = q.shape
    hkv = k.shape[2]
    nch = dash.n_chunks(k.shape[1], block_size, causal)
    words = (nch + 31) // 32
    tau = torch.empty(b, nq, hq, dtype=torch.float32, device=q.device)
    w = torch.empty(b, nq, hkv, nch, dtype=torch.float32, device=q.device) if nch else None
    mask = torch.zeros(b, nq, hkv, max(words, 1), dtype=torch.int32, device=q.device)
    extra = {} if qbar is None else {"qbar": qbar}
    if local == 2:
        extra["flags"] = dash.DASH_FLAG_LOCAL2
    dash.dash_block_select(q, k, block_size, alpha, causal, tau=tau, w=w, mask=mask, sigma=sigma, gamma=gamma,
                           **extra)
    torch.cuda.synchronize()
    return tau, w, mask


def to_np32(t):
    return t.detach().float().cpu().numpy()


def check_forward(q, k, v, out, block_size, alpha, causal, sigma=1e8, gamma=1.0, rows=None, batches=None,
                  label="", qbar=None, local=1):
    """Compare a GPU forward (``out``) and its Stage 1 with the oracle.

    rows: query indices to check (default all); batches: batch indices (default all);
    qbar: the learned Stage-0 summary queries [1 or b, n_chunks, hkv, d] given to both;
    local: chunks of the local window (2: DASH_FLAG_LOCAL2 on the GPU).
    Returns a dict of statistics.
    """
    b, nq, hq, d = q.shape
    nk, hkv = k.shape[1], k.shape[2]
    nch = dash.n_chunks(nk, block_size, causal)
    tau_g, w_g, mask_g = gpu_stage1(q, k, block_size, alpha, causal, sigma, gamma, qbar, local)
    rows = np.arange(nq) if rows is None else np.asarray(rows, dtype=np.int64)
    batches = range(b) if batches is None else batches
    max_tol, mean_tol = OUT_TOL[q.dtype]
    rows_t = torch.from_numpy(rows).to(q.device)
    stats = dict(rows=0, flagged_rows=0, flagged_chunks=0, max_err=0.0, sum_err=0.0, n_el=0, tau_err=0.0,
                 w_err=0.0, routed=0, visible=0)
    for bi in batches:
        Qr = to_np32(q[bi].index_select(0, rows_t))
        K = to_np32(k[bi])
        V = to_np32(v[bi])
        qb = None if qbar is None else to_np32(qbar[bi if qbar.shape[0] > 1 else 0])
        ref = oracle.fwd_rows(Qr, rows, nq, K, V, block_size, alpha, gamma=gamma, sigma=sigma, causal=causal,
                              want=("out", "tau", "w", "routed", "xmt"), qbar=qb, local=local)
        tg = tau_g[bi].index_select(0, rows_t).cpu().numpy()
        wg = (w_g[bi].index_select(0, rows_t).cpu().numpy().astype(np.float64) if nch
              else np.zeros((len(rows), hkv, 0)))
        rg = unpack_mask(mask_g[bi].index_select(0, rows_t).cpu().numpy(), nch)
        og = to_np32(out[bi].index_select(0, rows_t)).astype(np.float64)
        # --- Stage 1 ---
        nan_o, nan_g = np.isnan(ref["tau"]), np.isnan(tg)
        assert (nan_o == nan_g).all(), f"{label}: rows without visible chunks differ"
        if (~nan_o).any():
            te = np.abs(tg[~nan_o] - ref["tau"][~nan_o]).max()
            stats["tau_err"] = max(stats["tau_err"], float(te))
            assert te <= TAU_TOL, f"{label}: tau error {te}"
        ro = ref["routed"].astype(bool)
        near = (np.abs(ref["xmt"]) <= SUPPORT_WINDOW).reshape(len(rows), hkv, hq // hkv, nch).any(axis=2)
        diff = ro != rg
        assert not (diff & ~near).any(), f"{label}: support differs outside the 1e-3 window " \
                                         f"({int((diff & ~near).sum())} chunks)"
        if nch:
            we = np.abs(wg - ref["w"]).max()
            stats["w_err"] = max(stats["w_err"], float(we))
            assert we <= W_TOL, f"{label}: w error {we}"
        stats["routed"] += int(ro.sum())
        vis = (np.minimum(np.maximum((rows + nk - nq) // block_size - (local - 1), 0), nch) if causal
               else np.full(len(rows), nch))
        stats["visible"] += int(vis.sum()) * hkv
        # --- Stage 2 ---
        flagged = diff.any(axis=2)                # [rows, hkv]
        frow = flagged.any(axis=1)
        exp_out = ref["out"].copy()
        if frow.any():
            fr = np.nonzero(frow)[0]
            # the oracle's own w on every chunk both select; the GPU's w only on a chunk
            # that the GPU alone selected (the oracle gave it no mass)
            both = rg[fr] & ro[fr]
            w_in = np.where(both, ref["w"][fr], np.where(rg[fr], np.maximum(wg[fr], 1e-300), 0.0))
            re = oracle.fwd_rows(Qr[fr], rows[fr], nq, K, V, block_size, alpha, gamma=gamma, sigma=sigma,
                                 causal=causal, w_in=w_in, r_in=rg[fr].astype(np.uint8), want=("out",), qbar=qb,
                                 local=local)
            exp_out[fr] = re["out"]
        err = np.abs(og - exp_out)
        stats["rows"] += len(rows)
        stats["flagged_rows"] += int(frow.sum())
        stats["flagged_chunks"] += int(diff.sum())
        stats["max_err"] = max(stats["max_err"], float(err.max()))
        stats["sum_err"] += float(err.sum())
        stats["n_el"] += err.size
    stats["mean_err"] = stats["sum_err"] / max(stats["n_el"], 1)
    stats["sparsity"] = 1.0 - stats["routed"] / max(stats["visible"], 1)
    assert stats["max_err"] <= max_tol, f"{label}: max-abs error {stats['max_err']} > {max_tol}"
    assert stats["mean_err"] <= mean_tol, f"{label}: mean-abs error {stats['mean_err']} > {mean_tol}"
    print(f"[parity] {label}: rows={stats['rows']} max_err={stats['max_err']:.3g} mean_err={stats['mean_err']:.3g} "
          f"tau_err={stats['tau_err']:.3g} w_err={stats['w_err']:.3g} flagged_rows={stats['flagged_rows']} "
          f"sparsity={stats['sparsity']:.3f}")
    return stats


def sample_rows(nq: int, block: int, n: int, seed: int) -> np.ndarray:
    """Stratified rows: the first rows, the last row, chunk starts and ends, random rows."""
    rng = np.random.default_rng(seed)
    fixed = {0, 1, min(block, nq - 1), nq - 1, nq - 2}
    n_ch = nq // block
    for c in rng.choice(np.arange(1, max(n_ch, 2)), size=min(n // 8, max(n_ch - 1, 1)), replace=False):
        fixed.add(int(min(c * block, nq - 1)))
        fixed.add(int(min(c * block - 1, nq - 1)))
    rest = rng.choice(nq, size=max(0, n - len(fixed)), replace=False)
    return np.unique(np.concatenate([np.array(sorted(fixed)), rest]).clip(0, nq - 1)).astype(np.int64)[:n]

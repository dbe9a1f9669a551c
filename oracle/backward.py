"""Backward pass of the DashAttention forward (fp64, plain numpy): gradients of the
outputs with respect to Q, K and V for a given output gradient dO.

TEST INFRASTRUCTURE ONLY, like the rest of this package: nothing on the product path
imports it.  It differentiates exactly the forward that dash_oracle.c computes
("DashAttention: Differentiable and Adaptive Sparse Hierarchical Attention"), taking
the routing decisions (supports, thresholds, the group distribution) from that
forward and applying the chain rule step by step, in the forward's order reversed:

  Stage 2 [Dash §3.3 Eq. 7 in the bias form of §3.4 Prop. 1]: for each head,
      l_j = z_j + b_j,  z_j = <q, k_j>/sqrt(d),  P = softmax(l),  o = sum_j P_j v_j,
      b_j = d_c = (log w_c - mu)/sigma on the tokens of routed chunks, 0 on the diagonal;
      dV_j += P_j dO,  dl_j = P_j (<dO, v_j> - sum_t P_t <dO, v_t>),
      dq += sum_j dl_j k_j / sqrt(d),  dk_j += dl_j q / sqrt(d),
      and the bias collects G_c = sum over the group's heads and the chunk's tokens of dl_j.
  Prior bias [Dash §3.4 Prop. 1; mu = mean of log w over R]:
      d(log w_c) = (G_c - mean_{c' in R} G_c') / sigma on R,  dw_c = d(log w_c) / w_c.
  Group average [Dash §3.2]: w_c = (1/g) sum_h p_c^(h), so dp_c^(h) = dw_c / g.
  alpha-entmax [Dash §2 Eq. 2]: p_c = [(alpha-1) s_c - tau]_+^(1/(alpha-1)) with sum p = 1.
      On the support, dp_c/ds_c = u_c = p_c^(2-alpha) and tau moves to keep the sum, so the
      Jacobian is diag(u) - u u^T / sum(u) (symmetric); ds = u (dp - <u, dp>/sum(u)).
  Stage-1 scores [Dash §3.2 Eq. 4]: s_c = gamma <q, kbar_c>/sqrt(d):
      dq += gamma sum_c ds_c kbar_c / sqrt(d),  dkbar_c += gamma ds_c q / sqrt(d).
  Stage 0 with the summary query at zero [Dash §3.1 Eq. 3]: kbar_c is the mean of the
      chunk's keys, so every key of chunk c receives dkbar_c / |C_c|.  With a learned
      summary query, kbar_c = sum_t a_t k_t with a = softmax_t(<qbar_c, k_t>/sqrt(d)):
      dk_t += a_t dkbar_c + e_t qbar_c / sqrt(d), dqbar_c = sum_t e_t k_t / sqrt(d), where
      e_t = a_t (<dkbar_c, k_t> - sum_u a_u <dkbar_c, k_u>).  As sigma grows the prior's
      gradient, and with it dqbar, falls as 1/sigma: in the limit the summary query gets
      no gradient at all [Dash App. F.5].

The supports (and R) are piecewise constant in the inputs and carry no gradient.
Parity pins (tests/test_oracle_backward.py): central finite differences of the C
forward, the sigma -> infinity limit against torch autograd of masked softmax
attention, and the entmax Jacobian against finite differences of the C entmax.
"""
from __future__ import annotations

import numpy as np

from . import fwd_rows, n_chunks_for


def entmax_vjp(p: np.ndarray, dp: np.ndarray, alpha: float) -> np.ndarray:
    """Vector-Jacobian product of alpha-entmax (gradient with respect to the scores s)."""
    u = np.where(p > 0, np.power(np.maximum(p, 0.0), 2.0 - alpha), 0.0)
    su = u.sum()
    if su == 0.0:
        return np.zeros_like(p)
    return u * (dp - (u @ dp) / su)


def backward(Q, K, V, dO, block_size: int, alpha: float, *, gamma: float = 1.0, sigma: float = 1e8,
             causal: bool = True, local: int = 1, qbar=None, rows=None):
    """Gradients (dQ, dK, dV, and dQbar with a learned summary query) of sum(dO * out)
    for one batch element.

    Q, dO [nq, hq, d]; K, V [nk, hkv, d] (float32 values, as the forward reads them);
    qbar [n_chunks, hkv, d] or None (q̄ = 0).  Returns a dict with out (the forward's
    output) and the gradients in float64.

    rows: optional query indices.  A row's dQ depends on that row alone (its own Stage 2
    and its own routing), so with rows given only those rows are differentiated and the
    result holds dQ of exactly those rows, in the given order (no dK, dV).

    Beside the gradients: G [rows, hkv, n_chunks] the bias gradient of each routed chunk
    (0 elsewhere), Pmass [rows, hq, n_chunks] each head's Stage-2 probability on each routed
    chunk, and the forward's out, w, xmt (x - tau per head) and the summaries kbar."""
    Q = np.ascontiguousarray(Q, dtype=np.float32)
    K = np.ascontiguousarray(K, dtype=np.float32)
    V = np.ascontiguousarray(V, dtype=np.float32)
    dO = np.asarray(dO, dtype=np.float64)
    nq, hq, d = Q.shape
    nk, hkv, _ = K.shape
    g = hq // hkv
    B = block_size
    nch = n_chunks_for(nk, B, causal)
    sel = np.arange(nq, dtype=np.int64) if rows is None else np.asarray(rows, dtype=np.int64)
    if qbar is not None:
        qbar = np.ascontiguousarray(np.broadcast_to(np.asarray(qbar, dtype=np.float32), (nch, hkv, d)))
    ref = fwd_rows(np.ascontiguousarray(Q[sel]), sel, nq, K, V, B, alpha, gamma=gamma, sigma=sigma, causal=causal,
                   want=("out", "w", "routed", "xmt"), local=local, qbar=qbar)
    Qd, Kd, Vd = Q.astype(np.float64), K.astype(np.float64), V.astype(np.float64)
    scale = 1.0 / np.sqrt(d)
    kexp = 1.0 / (alpha - 1.0)

    # chunk summaries and chunk sizes: the mean of the chunk's real keys, or their
    # softmax-weighted sum under the learned summary query (weights A[c] [size, hkv])
    sizes = np.array([min((c + 1) * B, nk) - c * B for c in range(nch)], dtype=np.float64)
    A = []
    for c in range(nch):
        kc = Kd[c * B:c * B + int(sizes[c])]                       # [size, hkv, d]
        if qbar is None:
            A.append(np.full(kc.shape[:2], 1.0 / sizes[c]))
        else:
            sc = np.einsum("thd,hd->th", kc, qbar[c].astype(np.float64)) * scale
            a = np.exp(sc - sc.max(axis=0))
            A.append(a / a.sum(axis=0))
    Kbar = (np.stack([np.einsum("th,thd->hd", A[c], Kd[c * B:c * B + int(sizes[c])]) for c in range(nch)])
            if nch else np.zeros((0, hkv, d)))

    dQ = np.zeros_like(Qd)
    dK = np.zeros_like(Kd)
    dV = np.zeros_like(Vd)
    dKbar = np.zeros_like(Kbar)
    Gall = np.zeros((len(sel), hkv, nch))  # the bias gradient G of every routed chunk
    Pmass = np.zeros((len(sel), hq, nch))  # each head's Stage-2 probability mass on every routed chunk
    for n, i in enumerate(sel):
        if causal:
            p_i = i + nk - nq
            c_i = p_i // B
            first = max(c_i - (local - 1), 0)
            nvis = min(first, nch)
            diag = np.arange(first * B, p_i + 1)
        else:
            nvis = nch
            diag = np.arange(0)
        for r in range(hkv):
            routed = ref["routed"][n, r, :].astype(bool)
            w = ref["w"][n, r, :]
            Rc = np.nonzero(routed)[0]
            mu = np.log(w[Rc]).mean() if len(Rc) else 0.0
            # tokens attended: routed chunks ascending, then the local window
            toks = [np.arange(c * B, c * B + int(sizes[c])) for c in Rc] + [diag]
            toks = np.concatenate(toks) if toks else np.arange(0)
            chunk_of = np.concatenate([np.full(int(sizes[c]), j) for j, c in enumerate(Rc)] +
                                      [np.full(len(diag), -1)]).astype(np.int64)
            bias = np.where(chunk_of >= 0, (np.log(w[Rc[np.maximum(chunk_of, 0)]]) - mu) / sigma
                            if len(Rc) else 0.0, 0.0)
            G = np.zeros(len(Rc))  # d loss / d bias of each routed chunk, summed over the group
            for hh in range(g):
                h = r * g + hh
                q = Qd[i, h]
                kt, vt = Kd[toks, r], Vd[toks, r]
                z = kt @ q * scale
                ell = z + bias
                P = np.exp(ell - ell.max())
                P /= P.sum()
                dv_rows = np.outer(P, dO[i, h])
                np.add.at(dV[:, r], toks, dv_rows)
                dPj = vt @ dO[i, h]
                dl = P * (dPj - P @ dPj)
                dQ[i, h] += (dl @ kt) * scale
                np.add.at(dK[:, r], toks, np.outer(dl, q) * scale)
                routed_tok = chunk_of >= 0
                np.add.at(G, chunk_of[routed_tok], dl[routed_tok])
                if len(Rc):
                    pm = np.zeros(len(Rc))
                    np.add.at(pm, chunk_of[routed_tok], P[routed_tok])
                    Pmass[n, h, Rc] = pm
            if len(Rc) == 0:
                continue
            Gall[n, r, Rc] = G
            # prior bias -> log w -> w -> each head's entmax probabilities
            dlogw = (G - G.mean()) / sigma
            dw = np.zeros(nch)
            dw[Rc] = dlogw / w[Rc]
            for hh in range(g):
                h = r * g + hh
                xmt = ref["xmt"][n, h, :nvis]
                p = np.power(np.maximum(xmt, 0.0), kexp)
                ds = entmax_vjp(p, dw[:nvis] / g, alpha)
                # s_c = gamma <q, kbar_c> / sqrt(d)
                dQ[i, h] += gamma * scale * (ds @ Kbar[:nvis, r])
                dKbar[:nvis, r] += gamma * scale * np.outer(ds, Qd[i, h])
    if rows is not None:
        return {"dQ": dQ[sel], "rows": sel, "G": Gall, "Pmass": Pmass, "w": ref["w"], "xmt": ref["xmt"],
                "kbar": Kbar, "out": ref["out"]}
    # Stage 0: the chunk's keys through the weights A (uniform for the mean)
    dQbar = np.zeros((nch, hkv, d))
    for c in range(nch):
        sl = slice(c * B, c * B + int(sizes[c]))
        kc = Kd[sl]
        if qbar is None:
            dK[sl] += dKbar[c] / sizes[c]
            continue
        a = A[c]                                                   # [size, hkv]
        dK[sl] += a[:, :, None] * dKbar[c][None]
        da = np.einsum("thd,hd->th", kc, dKbar[c])
        e = a * (da - (a * da).sum(axis=0))
        dK[sl] += e[:, :, None] * qbar[c].astype(np.float64)[None] * scale
        dQbar[c] = np.einsum("th,thd->hd", e, kc) * scale
    res = {"out": ref["out"], "dQ": dQ, "dK": dK, "dV": dV, "G": Gall, "Pmass": Pmass, "w": ref["w"],
           "xmt": ref["xmt"], "kbar": Kbar}
    if qbar is not None:
        res["dQbar"] = dQbar
    return res

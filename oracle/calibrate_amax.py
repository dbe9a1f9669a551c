"""Calibrate the planted-block generator's a_max with the oracle.

Writes ``synthetic/amax.json``: for each block size the a_max at which the
oracle's Stage-1 block sparsity at alpha = 1.5 is the target (75 %).  Block
sparsity follows the DashAttention kernel benchmark's definition: the fraction
of visible chunks a (query row, kv head) pair does NOT route to Stage 2; the
diagonal chunk is not counted.

It estimates sparsity on a seeded sample of query rows of the 32K workload
(block 64) and of the 128K workload (block 128), bisecting a_max.  It runs on
the CPU only and calls nothing but ``oracle`` and ``synthetic``.

    python -m oracle.calibrate_amax
"""
from __future__ import annotations

import json
import sys
import time
from pathlib import Path

import numpy as np
import torch

_ROOT = Path(__file__).resolve().parents[1]
if str(_ROOT) not in sys.path:
    sys.path.insert(0, str(_ROOT))

import oracle  # noqa: E402
import synthetic  # noqa: E402

TARGET = 0.75
N_ROWS = 512


def sparsity(parts, w, rows, a_max, alpha=1.5):
    q = synthetic.assemble_q(parts, a_max)[0].to(torch.bfloat16).float().numpy()
    K = parts.k[0].to(torch.bfloat16).float().numpy()
    V = parts.v[0].to(torch.bfloat16).float().numpy()
    res = oracle.fwd_rows(q[rows], rows, w.nq, K, V, w.block, alpha, want=("routed",))
    vis = np.minimum((rows + w.nk - w.nq) // w.block, w.nk // w.block)
    return 1.0 - res["routed"].sum() / (vis.sum() * w.hkv)


def calibrate(w, seed=123):
    t0 = time.time()
    parts = synthetic.draw_parts(w, "cpu")
    rng = np.random.default_rng(seed)
    rows = np.sort(rng.choice(np.arange(w.block, w.nq), N_ROWS, replace=False)).astype(np.int64)
    lo, hi = 1.0, 128.0
    for _ in range(14):
        mid = 0.5 * (lo + hi)
        if sparsity(parts, w, rows, mid) < TARGET:
            lo = mid
        else:
            hi = mid
    a = round(0.5 * (lo + hi), 3)
    s = sparsity(parts, w, rows, a)
    sweep = {str(al): round(float(sparsity(parts, w, rows, a, al)), 4) for al in (1.25, 1.5, 2.0)}
    print(f"{w.name}: a_max={a} sparsity={s:.4f} alpha sweep {sweep} ({time.time() - t0:.0f}s)")
    return {"a_max": a, "sparsity_alpha1.5": round(float(s), 4), "sparsity_by_alpha": sweep,
            "workload": w.name, "rows_sampled": N_ROWS, "target": TARGET}


def main():
    out = {"b64": calibrate(synthetic.WORKLOADS["prefill32k"]),
           "b128": calibrate(synthetic.WORKLOADS["prefill128k"])}
    path = _ROOT / "synthetic" / "amax.json"
    path.write_text(json.dumps(out, indent=1) + "\n")
    print("wrote", path)


if __name__ == "__main__":
    main()

"""Seeded synthetic inputs for DashAttention workloads.

This module generates inputs only: it holds none of the method's arithmetic,
and both the CUDA library's callers and the oracle's callers use it.

The planted-block generator G(seed, frac, shift, a_max), for Q [b, nq, hq, d]
and K, V [b, nk, hkv, d]:
  1. u = a unit vector drawn from N(0, I_d) (shared by every head and batch);
  2. Q, K, V entries iid N(0, 1); the attention scale 1/sqrt(d) is applied by
     the method itself;
  3. per (batch, kv head) a random floor(frac * Tc) of the Tc = floor(nk/B)
     key blocks are planted: every key row in them gets + shift * u;
  4. every query (batch, row, head) gets + a * u with a ~ U(a_max/4, a_max), so
     the block-logit gap varies four-fold across queries and the entmax
     support is query-adaptive;
  5. V is not shifted.
Without planting (the smallest workload) Q, K, V are plain iid N(0, 1).
a_max per workload was calibrated with the oracle to a target block sparsity
(oracle/calibrate_amax.py writes amax.json beside this file).

Random draws: the planted-block choice, u and the per-query a fractions come
from a CPU torch.Generator; the bulk N(0,1) tensors come from a generator on
the requested device (seeded identically), drawn in the order Q, K, V.
"""
from __future__ import annotations

import json
import math
from dataclasses import dataclass, field, replace
from pathlib import Path

import torch

_AMAX_FILE = Path(__file__).resolve().parent / "amax.json"


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    nq: int
    nk: int
    hq: int
    hkv: int
    d: int
    block: int
    alpha: float
    causal: bool
    dtype: str  # "f32" | "bf16"
    seed: int
    planted: bool
    frac: float = 0.25
    shift: float = 2.0
    amax_key: str = ""  # which calibrated a_max this workload uses
    alphas: tuple = field(default_factory=tuple)

    @property
    def g(self) -> int:
        return self.hq // self.hkv

    @property
    def tc(self) -> int:
        return self.nk // self.block

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


# The five workloads (sizes as the benchmark configurations name them).
WORKLOADS = {
    "tiny": Workload("tiny", 1, 1024, 1024, 1, 1, 64, 64, 1.5, True, "f32", 0, False),
    "prefill8k": Workload("prefill8k", 1, 8192, 8192, 32, 8, 128, 64, 1.5, True, "bf16", 1, True,
                          amax_key="b64"),
    "prefill32k": Workload("prefill32k", 1, 32768, 32768, 32, 8, 128, 64, 1.5, True, "bf16", 2, True,
                           amax_key="b64"),
    "decode": Workload("decode", 16, 1, 131072, 32, 8, 128, 64, 1.5, True, "bf16", 3, True,
                       amax_key="b64"),
    "prefill128k": Workload("prefill128k", 1, 131072, 131072, 32, 8, 128, 128, 1.5, True, "bf16", 4, True,
                            amax_key="b128", alphas=(1.25, 1.5, 2.0)),
}


def load_amax() -> dict:
    if _AMAX_FILE.exists():
        return json.loads(_AMAX_FILE.read_text())
    return {}


def amax_for(w: Workload) -> float:
    if not w.planted:
        return 0.0
    tab = load_amax()
    if w.amax_key in tab:
        return float(tab[w.amax_key]["a_max"])
    return 8.0  # uncalibrated default


def _torch_dtype(name: str):
    return {"f32": torch.float32, "bf16": torch.bfloat16}[name]


@dataclass
class Parts:
    """The random parts of one draw; q = q0 + a * u with a = a_max (1/4 + 3/4 xi)."""
    q0: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    u: torch.Tensor       # [d] float32 (on the device)
    xi: torch.Tensor      # [b, nq, hq] float32 in [0, 1) (on the device); a = a_max (1/4 + 3/4 xi)
    planted: torch.Tensor  # [b, hkv, n_planted] int64 block ids (CPU)


def draw_parts(w: Workload, device="cpu") -> Parts:
    """Draw every random part of workload ``w`` (float32, on ``device``)."""
    device = torch.device(device)
    gcpu = torch.Generator(device="cpu").manual_seed(w.seed)
    u = torch.randn(w.d, generator=gcpu, dtype=torch.float32)
    u = u / u.norm()
    tc = w.nk // w.block
    n_pl = int(math.floor(w.frac * tc)) if w.planted else 0
    planted = torch.stack([torch.stack([torch.randperm(tc, generator=gcpu)[:n_pl] for _ in range(w.hkv)])
                           for _ in range(w.batch)]) if n_pl > 0 else torch.zeros(w.batch, w.hkv, 0,
                                                                                   dtype=torch.int64)
    xi = torch.rand(w.batch, w.nq, w.hq, generator=gcpu, dtype=torch.float32)
    gdev = torch.Generator(device=device).manual_seed(w.seed)
    q0 = torch.randn(w.batch, w.nq, w.hq, w.d, generator=gdev, device=device, dtype=torch.float32)
    k = torch.randn(w.batch, w.nk, w.hkv, w.d, generator=gdev, device=device, dtype=torch.float32)
    v = torch.randn(w.batch, w.nk, w.hkv, w.d, generator=gdev, device=device, dtype=torch.float32)
    u_dev = u.to(device)
    if n_pl > 0:
        mask = torch.zeros(w.batch, w.hkv, tc, dtype=torch.float32)
        mask.scatter_(2, planted, 1.0)
        mask = mask.permute(0, 2, 1).contiguous().to(device)          # [b, tc, hkv]
        body = k[:, :tc * w.block].view(w.batch, tc, w.block, w.hkv, w.d)
        body += (w.shift * mask).view(w.batch, tc, 1, w.hkv, 1) * u_dev.view(1, 1, 1, 1, w.d)
    return Parts(q0, k, v, u_dev, xi.to(device), planted)


A_LO_FRAC = 0.25  # a ~ U(A_LO_FRAC * a_max, a_max)


def assemble_q(parts: Parts, a_max: float) -> torch.Tensor:
    """q = q0 + a * u with a = a_max * (A_LO_FRAC + (1 - A_LO_FRAC) * xi) (float32)."""
    if a_max == 0.0:
        return parts.q0.clone()
    a = a_max * (A_LO_FRAC + (1.0 - A_LO_FRAC) * parts.xi)
    return parts.q0 + a.unsqueeze(-1) * parts.u.view(1, 1, 1, -1)


def make_inputs(w: Workload, device="cpu", a_max: float | None = None):
    """Return (q, k, v) of workload ``w`` in its dtype on ``device``."""
    if a_max is None:
        a_max = amax_for(w)
    parts = draw_parts(w, device)
    dt = _torch_dtype(w.dtype)
    q = assemble_q(parts, a_max if w.planted else 0.0).to(dt)
    k = parts.k.to(dt)
    v = parts.v.to(dt)
    return q, k, v


def random_block_mask(batch: int, nq: int, nk: int, hkv: int, block: int, s: float, seed: int,
                      causal: bool = True, device="cpu") -> torch.Tensor:
    """A random routing mask at block sparsity ``s``, the controlled-sparsity input of the
    Stage-2 benchmark (the pages inject such a mask at Stage 2 in place of the router's).

    Each (batch, query row, kv head) routes round((1 - s) * n_i) of the n_i chunks it may
    route, uniformly without replacement: n_i = min(floor(p_i / B), floor(nk / B)) with
    p_i = i + nk - nq when causal, every one of ceil(nk / B) chunks otherwise.  Returns
    the bit-packed words [batch, nq, hkv, ceil(n_chunks / 32)] as int32 (bit c % 32 of
    word c // 32 = chunk c), drawn from a generator on ``device`` seeded with ``seed``."""
    n_chunks = nk // block if causal else -(-nk // block)
    words = max((n_chunks + 31) // 32, 1)
    gen = torch.Generator(device=device).manual_seed(seed)
    if causal:
        p = torch.arange(nq, device=device, dtype=torch.int64) + (nk - nq)
        n_vis = torch.clamp(p // block, max=n_chunks)
    else:
        n_vis = torch.full((nq,), n_chunks, device=device, dtype=torch.int64)
    n_sel = torch.round((1.0 - s) * n_vis.to(torch.float64)).to(torch.int64)       # [nq]
    u = torch.rand(batch, nq, hkv, max(n_chunks, 1), generator=gen, device=device)
    c = torch.arange(max(n_chunks, 1), device=device)
    u = torch.where(c.view(1, 1, 1, -1) < n_vis.view(1, -1, 1, 1), u, torch.full_like(u, 2.0))
    order = torch.argsort(u, dim=-1)                                                  # visible chunks first
    take = (c.view(1, 1, 1, -1) < n_sel.view(1, -1, 1, 1)).expand_as(order)
    bits = torch.zeros(batch, nq, hkv, words * 32, dtype=torch.int64, device=device)
    bits[..., :max(n_chunks, 1)].scatter_(-1, order, take.to(torch.int64))
    packed = (bits.view(batch, nq, hkv, words, 32) << torch.arange(32, device=device)).sum(-1)
    return torch.where(packed >= 2 ** 31, packed - 2 ** 32, packed).to(torch.int32)

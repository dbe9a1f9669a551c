"""Benchmark of the DashAttention forward pass on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload prefill128k|prefill8k|prefill32k|decode]
                    [--impl ours|reference] [--no-cpu-baseline]

One step = one full forward (Stage 0 pooling, Stage 1 routing + work lists,
Stage 2 sparse attention) of the workload on synthetic seeded inputs resident
in HBM.  Prints ONE JSON line (rank 0).

Metric: selected-block Stage-2 FLOPs per second for prefill (TFLOP/s), selected
K/V bytes per second for decode (GB/s) -- the algorithmic work the method must
do, not the dense work it avoids:
  F2 = sum_{b,i,h} 4 d (B |R_i| + (p_i mod B) + 1)     (routed chunks + diagonal keys)
  Y  = sum_{b,r} (B |R^(r)| + diagonal keys) d * 2 tensors * 2 bytes
Timing: CUDA events on the launching stream, L2 flushed (a 256 MiB write)
before every timed step, outside the event pair; warm-up steps untimed.
Multi-GPU (torchrun): every rank runs an independent replica of the workload
(the method's (batch, kv-head) units share nothing: no collective); value is
the work of all ranks over the max-over-ranks time ("scaling": "weak").

    python bench.py --mask-sweep [--sweep-n 16384,32768,65536,98304] [--sweep-s 0.75,0.875,0.9375]
                    [--sweep-phase prefill,decode]

Controlled-sparsity sweep of Stage 2 (the pages' kernel benchmark: Hq 32, Hkv 2, d 128,
chunk 64, prefill at batch 1, decoding at batch 24): a random routing mask at block
sparsity s stands in for the router's, Stage 2 alone is timed on the work lists built
from it, and torch's dense SDPA on the same inputs is timed beside it for context.  One
JSON line per (phase, N, s); 1 GPU.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time
from pathlib import Path

ROOT = Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

import torch  # noqa: E402

import synthetic  # noqa: E402

METRIC = "DashAttention fwd ms & TFLOP/s (prefill) / GB/s (decode), % of B200 roofline"
L2_FLUSH_BYTES = 256 << 20

# DRAM bytes (read + write) per launch of the dominant kernel, each from one full-size ncu
# capture (dram__bytes_read.sum + dram__bytes_write.sum, one pass) of the current kernel:
# the Stage-2 tensor-core kernel at 128K and 8K, the split-KV decode kernel at batch 16.  A
# workload without a capture of the current kernel reports null.
TRAFFIC_BYTES = {
    ("prefill128k", 1): 3.2890e9,
    ("prefill8k", 1): 1.4396e8,
    ("decode", 16): 1.6258e9,
}


def load_peaks():
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        d = json.loads(p.read_text())
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *a):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in getattr(self, "lines", []):
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------
# work accounting (bench-side, from the routing mask the library exports)
# ---------------------------------------------------------------------------

def routed_counts(dash, q, k, w, alpha, sigma, flags=0):
    """|R_i^(r)| per (b, i, r) from dash_block_select's bit-packed mask."""
    nch = dash.n_chunks(w.nk, w.block, True)
    words = max((nch + 31) // 32, 1)
    mask = torch.zeros(w.batch, w.nq, w.hkv, words, dtype=torch.int32, device=q.device)
    dash.dash_block_select(q, k, w.block, alpha, True, mask=mask, sigma=sigma, flags=flags)
    m = mask.to(torch.int64) & 0xFFFFFFFF
    cnt = torch.zeros(w.batch, w.nq, w.hkv, dtype=torch.int64, device=q.device)
    for bit in range(32):
        cnt += (m >> bit).bitwise_and(1).sum(-1)
    return cnt


def work_of(w, cnt, lists, local=1):
    """Selected FLOPs F2, selected K/V bytes Y, sparsity, and the tile-union FLOPs the kernel
    executes.  local: chunks of the local window (2: the chunk before the query's own as well)."""
    i = torch.arange(w.nq, device=cnt.device, dtype=torch.int64)
    p = i + w.nk - w.nq
    first = torch.clamp(p // w.block - (local - 1), min=0)            # first chunk of the local window
    diag = (p - first * w.block + 1).view(1, -1, 1)                  # keys of the local window
    keys = w.block * cnt + diag                                      # [b, nq, hkv]
    f2 = float((4 * w.d * keys.sum()).item()) * w.g                  # every head of the group
    y = float((keys.sum() * w.d * 2 * 2).item())                     # K and V, bf16, per kv head
    vis = torch.clamp(first, max=w.nk // w.block).view(1, -1, 1).expand_as(cnt)
    sparsity = 1.0 - float(cnt.sum().item()) / max(float(vis.sum().item()), 1.0)
    exec_f = None
    if lists is not None:
        exec_f = float((lists.count.to(torch.int64).sum() * w.block * 128 * 4 * w.d).item())
    return f2, y, sparsity, exec_f


def count_launches(fn, fallback):
    """Library kernels one call of fn launches, counted by the CUDA profiler on an extra,
    untimed call (long prefills run in several row slices, so the count depends on the
    size); `fallback` (the per-slice count) if the profiler is unavailable."""
    try:
        from torch.profiler import ProfilerActivity, profile
        torch.cuda.synchronize()
        with profile(activities=[ProfilerActivity.CUDA]) as prof:
            fn()
            torch.cuda.synchronize()
        n = sum(1 for e in prof.events() if e.device_type == torch.autograd.DeviceType.CUDA
                and "dash::" in e.name and "kernel" in e.name)
        return (n, "counted") if n > 0 else (fallback, "per-slice count (profiler saw no kernel)")
    except Exception as exc:  # noqa: BLE001
        return fallback, f"per-slice count (profiler unavailable: {type(exc).__name__})"


def max_over_ranks(values, world, device):
    """Element-wise maximum of per-rank timings (every rank takes this collective step)."""
    t = torch.tensor(values, dtype=torch.float64, device=device)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return t.tolist()


def job_throughput(work_per_rank, world, ms):
    """Whole-job throughput: the work of every rank over the max-over-ranks step time (per second)."""
    return work_per_rank * world / (ms * 1e-3)


# ---------------------------------------------------------------------------
# our implementation
# ---------------------------------------------------------------------------

def run_ours(args, rank, world, device):
    import sparse_hierarchical_attention_block_b200 as dash

    dash.load_library()
    w = synthetic.WORKLOADS[args.workload]
    if args.batch:
        w = w.with_(batch=args.batch)
    if args.seq and w.nq > 1:
        w = w.with_(nq=args.seq, nk=args.seq, name=f"{w.name}@{args.seq}")
    alpha = args.alpha or w.alpha
    sigma = args.sigma
    decode = w.nq == 1  # one new query token per sequence
    torch.manual_seed(0)
    q, k, v = synthetic.make_inputs(w, device)
    out = torch.empty_like(q)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream()

    cache = None
    local = 2 if args.local2 else 1
    opts = dict(sigma=sigma)
    if local == 2:
        opts["flags"] = dash.DASH_FLAG_LOCAL2
    if decode:
        # the chunk-summary cache persists across decode steps: every complete chunk is
        # pooled (and put in the tensor-core operand form) once, outside the step
        cache = dash.SummaryCache(w.batch, w.nk, w.hkv, w.d, w.block).update(k)
        opts["summary_cache"] = cache

    def step():
        dash.dash_attn_fwd(q, k, v, out, w.block, alpha, True, w.g, **opts)

    lists = dash.make_lists(q, k, w.block, w.g)
    dash.dash_block_select(q, k, w.block, alpha, True, lists=lists, **opts)
    cnt = routed_counts(dash, q, k, w, alpha, sigma, opts.get("flags", 0))
    f2, y, sparsity, exec_f = work_of(w, cnt, lists, local)
    torch.cuda.synchronize()

    for _ in range(args.warmup):
        step()
    rc = dash.dash_sync_status()
    if rc != 0:
        raise RuntimeError(f"warm-up failed with status {rc}")

    def timed(fn, n):
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
        for a, b in ev:
            flush.fill_(1.0)  # evict L2 (outside the timed pair)
            a.record(stream)
            fn()
            b.record(stream)
        torch.cuda.synchronize()
        return [a.elapsed_time(b) for a, b in ev]

    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    smi_id = vis.split(",")[torch.cuda.current_device()] if vis else str(torch.cuda.current_device())
    with ClockSampler(smi_id) as cs:
        times = timed(step, args.steps)
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
    rc = dash.dash_sync_status()
    if rc != 0:
        raise RuntimeError(f"timed steps failed with status {rc}")
    ms = sum(times) / len(times)

    # dominant kernel alone (Stage 2 on the same lists), and Stages 0-1 alone
    n_k = max(3, args.steps)
    t_stage2 = timed(lambda: dash.dash_sparse_attn_fwd(q, k, v, out, lists, w.block, True, w.g, **opts), n_k)
    t_stage01 = timed(lambda: dash.dash_block_select(q, k, w.block, alpha, True, lists=lists, **opts), n_k)
    ms2 = sum(t_stage2) / len(t_stage2)
    ms01 = sum(t_stage01) / len(t_stage01)

    # end to end through the public API with host buffers (pinned), copies inside the timed region.
    # Prefill: the step's inputs are q, k and v.  Decode: the KV cache (and its chunk summaries)
    # persist on the device across steps; a step brings the new token's q, k and v rows.
    if decode:
        qh = q.cpu().pin_memory()
        kh = k[:, -1:].cpu().pin_memory()
        vh = v[:, -1:].cpu().pin_memory()
        k_dst, v_dst = k[:, -1:], v[:, -1:]
    else:
        qh, kh, vh = q.cpu().pin_memory(), k.cpu().pin_memory(), v.cpu().pin_memory()
        k_dst, v_dst = k, v
    oh = torch.empty(out.shape, dtype=out.dtype).pin_memory()

    def e2e_step():
        if not decode:
            # prefill: the host-staged entry point copies row slices in and out on its own
            # streams while the earlier slices compute (output bit-identical to step())
            dash.dash_attn_fwd_host(qh, kh, vh, oh, q, k, v, out, w.block, alpha, True, w.g, **opts)
            return
        q.copy_(qh, non_blocking=True)
        k_dst.copy_(kh, non_blocking=True)
        v_dst.copy_(vh, non_blocking=True)
        if cache is not None:
            cache.update(k)  # pools a chunk only when the new token completes one
        step()
        oh.copy_(out, non_blocking=True)

    e2e_times = timed(e2e_step, max(2, min(args.steps, 5)))
    ms_e2e = sum(e2e_times) / len(e2e_times)
    h2d = sum(t.numel() * t.element_size() for t in (qh, kh, vh))
    d2h = oh.numel() * oh.element_size()

    launches_per_step, launches_src = count_launches(step, 4 if decode else 5)
    ms, ms2, ms01, ms_e2e = max_over_ranks([ms, ms2, ms01, ms_e2e], world, device)

    peaks = load_peaks()
    if decode:
        unit, work = "GB/s", y
        per = lambda msx: job_throughput(work, world, msx) / 1e9  # noqa: E731
        achieved = work / (ms2 * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": round(achieved / peaks["hbm_gbs"], 4), "traffic": TRAFFIC_BYTES.get((w.name, w.batch)),
                "kernel": "attn_decode (+ combine)", "peak_source": peaks["source"] + " hbm_gbs"}
    else:
        unit, work = "TFLOP/s", f2
        per = lambda msx: job_throughput(work, world, msx) / 1e12  # noqa: E731
        achieved = work / (ms2 * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": round(achieved, 2), "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": round(achieved / peaks["bf16_tflops"], 4), "traffic": TRAFFIC_BYTES.get((w.name, w.batch)),
                "kernel": "attn_tc (Stage 2)", "peak_source": peaks["source"] + " bf16_tflops (burst)",
                # the same kernel against the power-capped sustained GEMM rate (for launches of tens
                # of ms, where sw_power_cap holds the clock below its maximum)
                "peak_sustained": peaks["bf16_tflops_sustained"],
                "frac_sustained": round(achieved / peaks["bf16_tflops_sustained"], 4)}
    res = {
        "metric": METRIC,
        "value": round(per(ms), 3),
        "unit": unit,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded planted-block generator)",
        "config": {"workload": w.name, "batch": w.batch, "nq": w.nq, "nk": w.nk, "hq": w.hq, "hkv": w.hkv,
                   "d": w.d, "block": w.block, "alpha": alpha, "sigma": sigma, "gamma": 1.0, "causal": True,
                   "a_max": synthetic.amax_for(w), "sparsity": round(sparsity, 4),
                   "local_window_chunks": local,
                   "l2": "flushed (256 MiB write) before every timed step", "parallelism": f"replicas x{world}"},
        "stages_ms": {"total": round(ms, 4), "stage0_1_select": round(ms01, 4), "stage2": round(ms2, 4)},
        "work": {"selected_flops": f2, "selected_kv_bytes": y,
                 "executed_tile_flops": exec_f, "union_waste": (round(exec_f / f2, 3) if exec_f else None)},
        "roofline": roof,
        "e2e": {"value": round(per(ms_e2e), 3), "unit": unit, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "path": ("dash_attn_fwd_host: query-row slices, copies in and out on two streams beside the compute"
                         if not decode else "new token's q, k, v in; summary cache update; forward; output out"),
                "ms_per_step": round(ms_e2e, 4)},
        # per step, per row slice: prefill pool_keys, kbar_split (once), select_tile,
        # regroup_compact, attn_tc; decode (summaries and their operand form cached)
        # select_tile, compact, attn_decode, combine
        "gpu_launches": args.steps * launches_per_step,
        "gpu_launches_source": launches_src,
        "clocks": cs.summary(),
    }
    return res, (q, k, v, w, alpha, sigma)


# ---------------------------------------------------------------------------
# backward pass (dash_attn_bwd)
# ---------------------------------------------------------------------------

def run_backward(args, device):
    """Times dash_attn_bwd on the workload: one step = the whole backward (Stage 0-1
    recomputed, the Stage-2 gradient on the query and key sides, the routing chain).
    Algorithmic work: the five products of every (row, attended key) pair
    (S, dP, dV, dK, dQ: 2 d FLOPs each) = 2.5 x the forward's selected F2."""
    import sparse_hierarchical_attention_block_b200 as dash

    dash.load_library()
    w = synthetic.WORKLOADS[args.workload]
    if args.batch:
        w = w.with_(batch=args.batch)
    if args.seq and w.nq > 1:
        w = w.with_(nq=args.seq, nk=args.seq, name=f"{w.name}@{args.seq}")
    alpha = args.alpha or w.alpha
    sigma = args.sigma
    q, k, v = synthetic.make_inputs(w, device)
    gen = torch.Generator(device=device).manual_seed(1234)
    dout = torch.randn(q.shape, generator=gen, device=device).to(q.dtype)
    out = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=device)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream()
    flags = dash.DASH_FLAG_FORCE_SIMT if args.simt else 0
    dash.dash_attn_fwd(q, k, v, out, w.block, alpha, True, w.g, sigma=sigma, lse=lse, flags=flags)
    lists = dash.make_lists(q, k, w.block, w.g)
    dash.dash_block_select(q, k, w.block, alpha, True, lists=lists, sigma=sigma)
    cnt = routed_counts(dash, q, k, w, alpha, sigma)
    f2, y, sparsity, exec_f = work_of(w, cnt, lists)
    f_bwd = 2.5 * f2

    def step():
        dash.dash_attn_bwd(q, k, v, out, dout, lse, dq, dk, dv, w.block, alpha, True, w.g, sigma=sigma, flags=flags)

    for _ in range(args.warmup):
        step()
    if dash.dash_sync_status() != 0:
        raise RuntimeError("backward warm-up failed")
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    smi_id = vis.split(",")[torch.cuda.current_device()] if vis else str(torch.cuda.current_device())
    with ClockSampler(smi_id) as cs:
        for a, b in ev:
            flush.fill_(1.0)
            a.record(stream)
            step()
            b.record(stream)
        torch.cuda.synchronize()
    if dash.dash_sync_status() != 0:
        raise RuntimeError("backward failed")
    ms = sum(a.elapsed_time(b) for a, b in ev) / len(ev)
    peaks = load_peaks()
    ach = f_bwd / (ms * 1e-3) / 1e12
    return {
        "mode": "backward", "metric": "DashAttention bwd TFLOP/s on the selected pairs (5 products)",
        "value": round(ach, 3), "unit": "TFLOP/s", "ms_per_step": round(ms, 4), "steps": args.steps,
        "warmup": args.warmup, "dtype": "bf16", "data": "synthetic (seeded planted-block generator)",
        "path": "cuda cores" if args.simt else "tensor cores",
        "config": {"workload": w.name, "batch": w.batch, "nq": w.nq, "nk": w.nk, "hq": w.hq, "hkv": w.hkv,
                   "d": w.d, "block": w.block, "alpha": alpha, "sigma": sigma, "sparsity": round(sparsity, 4),
                   "l2": "flushed (256 MiB write) before every timed step"},
        "work": {"selected_bwd_flops": f_bwd, "forward_selected_flops": f2,
                 "union_waste": (round(exec_f / f2, 3) if exec_f else None)},
        "roofline": {"bound": "tensor", "achieved": round(ach, 2), "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": round(ach / peaks["bf16_tflops"], 4), "traffic": None,
                     "peak_sustained": peaks["bf16_tflops_sustained"],
                     "frac_sustained": round(ach / peaks["bf16_tflops_sustained"], 4),
                     "kernel": "whole dash_attn_bwd call (Stage 0-1 recompute included)",
                     "peak_source": peaks["source"] + " bf16_tflops (burst)"},
        "clocks": cs.summary(),
    }


# ---------------------------------------------------------------------------
# controlled-sparsity sweep of Stage 2 (random routing masks)
# ---------------------------------------------------------------------------

def mask_counts(mask):
    """|R| per (b, i, r) from bit-packed int32 mask words."""
    m = mask.to(torch.int64) & 0xFFFFFFFF
    cnt = torch.zeros(mask.shape[:3], dtype=torch.int64, device=mask.device)
    for bit in range(32):
        cnt += (m >> bit).bitwise_and(1).sum(-1)
    return cnt


def run_mask_sweep(args, device):
    import torch.nn.functional as F

    import sparse_hierarchical_attention_block_b200 as dash

    dash.load_library()
    peaks = load_peaks()
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream()

    def timed(fn, n):
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
        for a, b in ev:
            flush.fill_(1.0)
            a.record(stream)
            fn()
            b.record(stream)
        torch.cuda.synchronize()
        return statistics.median(a.elapsed_time(b) for a, b in ev)

    hq, hkv, d, block = 32, 2, 128, 64
    g = hq // hkv
    for phase in args.sweep_phase.split(","):
        for n in (int(x) for x in args.sweep_n.split(",")):
            b, nq = (1, n) if phase == "prefill" else (24, 1)
            w = synthetic.Workload(f"mask-sweep-{phase}-{n}", b, nq, n, hq, hkv, d, block, 1.5, True, "bf16", 21,
                                   False)
            q, k, v = synthetic.make_inputs(w, device)
            out = torch.empty_like(q)
            qt, kt, vt = (x.transpose(1, 2).contiguous() for x in (q, k, v))

            def dense():
                F.scaled_dot_product_attention(qt, kt, vt, is_causal=phase == "prefill", enable_gqa=True)

            for _ in range(args.warmup):
                dense()
            ms_dense = timed(dense, max(3, min(args.steps, 5)))
            del qt, kt, vt
            for sp in (float(x) for x in args.sweep_s.split(",")):
                mask = synthetic.random_block_mask(b, nq, n, hkv, block, sp, seed=31, device=device)
                lists = dash.lists_from_mask(mask, n, hkv, block, g, causal=True, regroup=True)
                f2, y, sparsity, exec_f = work_of(w, mask_counts(mask), lists)
                del mask

                def stage2():
                    dash.dash_sparse_attn_fwd(q, k, v, out, lists, block, True, g)

                for _ in range(args.warmup):
                    stage2()
                if dash.dash_sync_status() != 0:
                    raise RuntimeError("stage 2 failed")
                ms2 = timed(stage2, args.steps)
                if phase == "prefill":
                    ach, unit, peak = f2 / (ms2 * 1e-3) / 1e12, "TFLOP/s", peaks["bf16_tflops"]
                else:
                    ach, unit, peak = y / (ms2 * 1e-3) / 1e9, "GB/s", peaks["hbm_gbs"]
                print(json.dumps({
                    "mode": "random-mask Stage 2 sweep", "phase": phase, "n": n, "batch": b,
                    "target_sparsity": sp, "sparsity": round(sparsity, 4), "hq": hq, "hkv": hkv, "d": d,
                    "block": block, "stage2_ms": round(ms2, 4), "value": round(ach, 2), "unit": unit,
                    "roofline_frac": round(ach / peak, 4), "peak_source": peaks["source"],
                    "union_waste": (round(exec_f / f2, 3) if (exec_f and phase == "prefill") else None),
                    "dense_sdpa_ms": round(ms_dense, 4), "speedup_vs_dense": round(ms_dense / ms2, 3),
                    "steps": args.steps, "warmup": args.warmup,
                    "l2": "flushed (256 MiB write) before every timed call"}), flush=True)
                del lists
            del q, k, v, out
            torch.cuda.empty_cache()


# ---------------------------------------------------------------------------
# the oracle on the host cores (CPU baseline / reference arm)
# ---------------------------------------------------------------------------

def oracle_sample(w, alpha, sigma, q, k, v, budget_s=15.0, threads=0, batch_rows=0, max_rows=None, seed=0):
    """Time the fp64 oracle on a bounded row sample of the workload: batches of random query
    rows (all heads, batch element 0) until budget_s of oracle time is spent.  threads 0 =
    every host core.  Returns (rows, seconds, flops, bytes, threads used)."""
    import numpy as np

    import oracle

    cores = threads or (os.cpu_count() or 1)
    oracle.set_threads(cores)
    rng = np.random.default_rng(seed)
    # about one second of oracle work per batch: rows cost ~ their visible keys x heads
    per = batch_rows or max(1, min(256, int(cores * 2e9 / max(w.hq * w.nk * w.d * 4, 1))))
    done = []
    el = 0.0
    b = 0
    K = V = None
    while True:
        # decoding (a few rows per sequence): every row of one sequence per round, sequence
        # after sequence; prefill: random rows of the first sequence
        if K is None or w.nq <= 16:
            K = k[b].float().cpu().numpy()
            V = v[b].float().cpu().numpy()
        rows = (np.arange(w.nq) if w.nq <= 16 else
                np.sort(rng.choice(np.arange(w.nq), min(w.nq, per), replace=False)))
        Qr = q[b, torch.from_numpy(rows).to(q.device)].float().cpu().numpy()
        t0 = time.perf_counter()
        res = oracle.fwd_rows(Qr, rows, w.nq, K, V, w.block, alpha, sigma=sigma, want=("out", "routed"))
        el += time.perf_counter() - t0
        done.append((rows, res["routed"]))
        if w.nq <= 16:
            b += 1
        if el > budget_s or (max_rows and sum(len(r) for r, _ in done) >= max_rows) or b >= w.batch:
            break
    f2 = 0.0
    y = 0.0
    nrows = 0
    for rws, routed in done:
        p = rws + w.nk - w.nq
        keys = w.block * routed.sum(-1) + (p % w.block + 1)[:, None]  # [rows, hkv]
        f2 += float(4 * w.d * keys.sum()) * w.g
        y += float(keys.sum() * w.d * 4)
        nrows += len(rws)
    return nrows, el, f2, y, cores


def run_reference(args, device):
    w = synthetic.WORKLOADS[args.workload]
    if args.batch:
        w = w.with_(batch=args.batch)
    if args.seq and w.nq > 1:
        w = w.with_(nq=args.seq, nk=args.seq, name=f"{w.name}@{args.seq}")
    alpha = args.alpha or w.alpha
    q, k, v = synthetic.make_inputs(w, device)
    decode = w.nq == 1
    per_step = []
    flops = byts = 0.0
    rows = 0
    cores = os.cpu_count() or 1
    for s in range(args.warmup + args.steps):
        n, el, f2, y, cores = oracle_sample(w, alpha, args.sigma, q, k, v, budget_s=args.ref_budget, seed=s)
        if s >= args.warmup:
            per_step.append(el)
            flops += f2
            byts += y
            rows += n
    secs = sum(per_step)
    unit = "GB/s" if decode else "TFLOP/s"
    value = (byts / secs / 1e9) if decode else (flops / secs / 1e12)
    sample = (f"{rows} query rows x all heads ({'the new rows of successive sequences' if w.nq <= 16 else 'batch 0'}) "
              f"over {args.steps} steps (fp64 oracle, dense masked Stage 2)")
    return {
        "metric": METRIC, "impl": "reference", "value": value, "unit": unit, "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * secs / max(args.steps, 1), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded planted-block generator)",
        "config": {"workload": w.name, "batch": w.batch, "nq": w.nq, "nk": w.nk, "hq": w.hq, "hkv": w.hkv, "d": w.d,
                   "block": w.block, "alpha": alpha, "sigma": args.sigma},
        "cpu_baseline": {"value": value, "unit": unit, "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="prefill128k", choices=sorted(synthetic.WORKLOADS))
    ap.add_argument("--batch", type=int, default=0, help="override the workload's batch (smaller profiling cases)")
    ap.add_argument("--seq", type=int, default=0,
                    help="override a prefill workload's sequence length (nq = nk; smaller profiling cases)")
    ap.add_argument("--alpha", type=float, default=None)
    ap.add_argument("--sigma", type=float, default=1e8)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ref-budget", type=float, default=5.0, help="seconds of oracle work per reference step")
    ap.add_argument("--local2", action="store_true",
                    help="two-block local window (the chunk before the query's own attended in full)")
    ap.add_argument("--mask-sweep", action="store_true", help="controlled-sparsity sweep of Stage 2 (1 GPU)")
    ap.add_argument("--backward", action="store_true", help="time the backward pass dash_attn_bwd (1 GPU)")
    ap.add_argument("--simt", action="store_true", help="with --backward: the CUDA-core Stage-2 kernels")
    ap.add_argument("--sweep-n", default="16384,32768,65536,98304")
    ap.add_argument("--sweep-s", default="0.75,0.875,0.9375")
    ap.add_argument("--sweep-phase", default="prefill,decode")
    args = ap.parse_args()

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.warmup < 3:
        args.warmup = 3

    if args.backward:
        if rank == 0:
            torch.cuda.set_device(local)
            print(json.dumps(run_backward(args, torch.device("cuda", local))))
        return 0

    if args.mask_sweep:
        if rank == 0:
            torch.cuda.set_device(local)
            run_mask_sweep(args, torch.device("cuda", local))
        return 0

    if args.impl == "reference":
        if rank != 0:
            return 0
        device = "cuda" if torch.cuda.is_available() else "cpu"
        print(json.dumps(run_reference(args, device)))
        return 0

    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=device)
    try:
        res, (q, k, v, w, alpha, sigma) = run_ours(args, rank, world, device)
        if rank == 0:
            if not args.no_cpu_baseline and world == 1:
                decode = res["unit"] == "GB/s"
                n, el, f2, y, cores = oracle_sample(w, alpha, sigma, q, k, v, budget_s=15.0)
                val = (y / el / 1e9) if decode else (f2 / el / 1e12)
                # the same oracle on one thread, on a smaller sample
                n1, el1, f21, y1, _ = oracle_sample(w, alpha, sigma, q, k, v, budget_s=6.0, threads=1, seed=1)
                val1 = (y1 / el1 / 1e9) if decode else (f21 / el1 / 1e12)
                what = (f"the new rows of {n // max(w.nq, 1)} of the {w.batch} sequences" if w.nq <= 16 else
                        f"{n} random query rows of batch 0")
                res["cpu_baseline"] = {"value": val, "unit": res["unit"], "cores": cores, "kind": "oracle",
                                       "sample": f"{what} x all heads, {el:.1f} s "
                                                 f"(fp64 oracle, dense masked Stage 2)",
                                       "single_thread": {"value": val1, "unit": res["unit"], "cores": 1,
                                                         "sample": f"{n1} random query rows x all heads, "
                                                                   f"{el1:.1f} s"}}
            print(json.dumps(res))
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())

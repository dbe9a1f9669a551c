"""dash_attn_fwd_noalloc: the forward pass on the library's static scratch area.

Host-side checks (no GPU): the entry point is exported, rejects a problem
larger than its scratch area with DASH_ERR_WORKSPACE and refuses a caller
workspace, before any CUDA call.  GPU check: consecutive calls through the C
ABI (a prefill, a split-KV decode, a decode with a chunk-summary cache and an
8K-token prefill whose rows run in slices, in turn, so each call finds another's
leftovers in the shared area) agree with dash_attn_fwd within the tolerance of
the parity tests (the cached decode and the sliced prefill bit for bit), and the
calls after the first change the device's free memory by nothing.

Kept in a file of its own, collected last, so it runs both alone in a fresh
process and after every other test."""
import ctypes
import re

import pytest
import torch

import sparse_hierarchical_attention_block_b200 as dash
import synthetic
from sparse_hierarchical_attention_block_b200 import _Opts, _Tensor, build

MAX_ABS, MEAN_ABS = 2e-2, 2e-3  # the bf16 output tolerance of the parity tests
FAKE = 1 << 20  # never dereferenced: the checks fail first


@pytest.fixture(scope="module")
def lib():
    build.build()
    return dash.load_library()


def _t(dtype, shape):
    t = _Tensor()
    t.data = FAKE
    t.dtype = dtype
    stride = [shape[1] * shape[2] * shape[3], shape[2] * shape[3], shape[3], 1]
    for a in range(4):
        t.shape[a] = shape[a]
        t.stride[a] = stride[a]
    return t


def test_noalloc_exported(lib):
    assert hasattr(lib, "dash_attn_fwd_noalloc")
    assert "dash_attn_fwd_noalloc" in dash.EXPORTS


def test_noalloc_rejects_oversize(lib):
    # 128K-token prefill with 1024 chunks of 128: even 1024 query rows take ~70 MiB of lists
    q = _t(dash.DASH_BF16, [1, 131072, 32, 128])
    k = _t(dash.DASH_BF16, [1, 131072, 8, 128])
    bound = dash.dash_workspace_bytes(1, 131072, 131072, 32, 8, 128, 128, True)
    rc = lib.dash_attn_fwd_noalloc(ctypes.byref(q), ctypes.byref(k), ctypes.byref(k), ctypes.byref(q), 128, 1.5,
                                   1, 4, None)
    assert rc == dash.DASH_ERR_WORKSPACE
    msg = lib.dash_last_error().decode()
    # the message states the exact need of this call (its smallest slice of query rows, no
    # split-KV area for a prefill), which dash_workspace_bytes bounds from above
    need = int(re.search(r"needs (\d+) bytes", msg).group(1))
    assert dash.DASH_NOALLOC_SCRATCH_BYTES < need <= bound
    assert str(dash.DASH_NOALLOC_SCRATCH_BYTES) in msg and "dash_attn_fwd_ex" in msg


def test_noalloc_validates_before_sizing(lib):
    # a bad argument is reported as such, not as a size problem
    q = _t(dash.DASH_BF16, [1, 256, 8, 128])
    k = _t(dash.DASH_BF16, [1, 256, 2, 128])
    rc = lib.dash_attn_fwd_noalloc(ctypes.byref(q), ctypes.byref(k), ctypes.byref(k), ctypes.byref(q), 64, 0.5, 1,
                                   4, None)
    assert rc == dash.DASH_ERR_INVALID_ARG and "alpha" in lib.dash_last_error().decode()


def test_noalloc_rejects_caller_workspace(lib):
    q = _t(dash.DASH_BF16, [1, 256, 8, 128])
    k = _t(dash.DASH_BF16, [1, 256, 2, 128])
    o = _Opts()
    lib.dash_opts_init(ctypes.byref(o))
    o.workspace = FAKE
    o.workspace_bytes = 1 << 20
    rc = lib.dash_attn_fwd_noalloc(ctypes.byref(q), ctypes.byref(k), ctypes.byref(k), ctypes.byref(q), 64, 1.5, 1,
                                   4, ctypes.byref(o))
    assert rc == dash.DASH_ERR_INVALID_ARG
    assert "workspace" in lib.dash_last_error().decode()


# b, nq, nk, hq, hkv, d, B, alpha, causal, sigma, cached
PROBLEMS = [
    (1, 1000, 1000, 8, 2, 128, 64, 1.5, True, 1.0, False),  # prefill, ragged tail, regrouped tiles
    (2, 1, 3000, 8, 2, 128, 64, 1.5, True, 1e8, False),  # decode, split-KV partials in the scratch
    # decoding with a persistent chunk-summary cache (the serving case): Stage 0 and the
    # summaries' operand form come from the cache's own memory, not the scratch area
    (2, 1, 5000, 8, 2, 128, 64, 1.5, True, 1.0, True),
    # an 8K-token prefill at 32 heads: its lists need ~70 MiB, so the rows run in slices
    # that fit the area
    (1, 8192, 8192, 32, 8, 128, 64, 1.5, True, 1.0, False),
]


def _inputs(p, seed):
    b, nq, nk, hq, hkv, d, B, alpha, causal = p[:9]
    w = synthetic.Workload("noalloc", b, nq, nk, hq, hkv, d, B, alpha, causal, "bf16", seed, True, amax_key="b64")
    return synthetic.make_inputs(w, "cuda")


@pytest.mark.gpu
def test_noalloc_matches_fwd_on_consecutive_calls(lib):
    if not torch.cuda.is_available():
        pytest.fail("the gpu tests need a CUDA device")
    data = []
    for i, p in enumerate(PROBLEMS):
        b, nq, nk, hq, hkv, d, B, alpha, causal, sigma, cached = p
        q, k, v = _inputs(p, 40 + i)
        opts = {"sigma": sigma}
        if cached:
            opts["summary_cache"] = dash.SummaryCache(b, nk, hkv, d, B).update(k)
        ref = torch.empty_like(q)
        dash.dash_attn_fwd(q, k, v, ref, B, alpha, causal, hq // hkv, **opts)
        assert dash.dash_sync_status() == 0
        data.append((p, q, k, v, ref, opts))
    order = [0, 1, 2, 3, 0, 1, 2, 3]  # each call after the first finds another problem's contents in the scratch
    outs = [torch.full_like(data[j][1], float("nan")) for j in order]
    torch.cuda.synchronize()
    free = []
    for j, out in zip(order, outs):  # no torch allocation between the calls
        p, q, k, v, ref, opts = data[j]
        b, nq, nk, hq, hkv, d, B, alpha, causal = p[:9]
        dash.dash_attn_fwd_noalloc(q, k, v, out, B, alpha, causal, hq // hkv, **opts)
        assert dash.dash_sync_status() == 0, dash.load_library().dash_last_error()
        free.append(torch.cuda.mem_get_info()[0])
    # the first call may load the library's device module (which holds the area);
    # the calls after it allocate nothing
    assert free[1:] == free[:1] * (len(free) - 1), free
    for n, (j, out) in enumerate(zip(order, outs)):
        ref = data[j][4]
        if data[j][0][10] or data[j][0][1] == 8192:  # the same kernels on the same lists: bit for bit
            assert torch.equal(out, ref)
        err = (out.float() - ref.float()).abs()
        print(f"[noalloc] call {n} problem {j}: max_abs={err.max().item():.3g} mean_abs={err.mean().item():.3g}")
        assert torch.isfinite(out.float()).all()
        assert err.max().item() <= MAX_ABS and err.mean().item() <= MEAN_ABS

"""The C-ABI library on the CPU: it builds, loads, exports every entry point
that include/dash_attn.h declares, and its host-side validation rejects bad
arguments before touching a GPU."""
import ctypes
import re
from pathlib import Path

import pytest

import sparse_hierarchical_attention_block_b200 as dash
from sparse_hierarchical_attention_block_b200 import _Opts, _Tensor, build

ROOT = Path(__file__).resolve().parents[1]


@pytest.fixture(scope="module")
def lib():
    build.build()
    return dash.load_library()


def _declared_symbols():
    text = (ROOT / "include" / "dash_attn.h").read_text()
    return sorted(set(re.findall(r"DASH_API\s+[\w\s\*]+?\b(dash_\w+)\s*\(", text)))


def test_exports_every_declared_symbol(lib):
    declared = _declared_symbols()
    assert len(declared) >= 12
    for name in declared:
        assert hasattr(lib, name), name
    assert set(declared) == set(dash.EXPORTS)
    assert b"sm_100a" in lib.dash_version()


def test_library_is_sm100a_only():
    """The shared object carries sm_100a device code (and is self-contained)."""
    data = (ROOT / "sparse_hierarchical_attention_block_b200" / "libdash_attn.so").read_bytes()
    assert b"sm_100a" in data


def test_lists_geometry(lib):
    nt, cap, tr = dash.lists_geometry(2, 1000, 1000, 4, 64, 4)
    assert (tr, nt, cap) == (32, -(-1000 // 32), -(-1000 // 64))
    nt, cap, tr = dash.lists_geometry(1, 1, 131072, 8, 64, 4)
    assert (nt, cap, tr) == (1, 2048, 32)
    cb, ib, bb, rb = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    rc = lib.dash_lists_geometry(2, 1000, 1000, 4, 64, 4, None, None, None, ctypes.byref(cb), ctypes.byref(ib),
                                 ctypes.byref(bb), ctypes.byref(rb))
    assert rc == 0
    assert cb.value == 2 * 4 * 32 * 4 and ib.value == 2 * 4 * 32 * 16 * 4 and bb.value == ib.value * 32
    assert rb.value == 2 * 4 * 32 * 32 * 4
    assert dash.dash_workspace_bytes(1, 8192, 8192, 32, 8, 128, 64) > 0


def _t(data, dtype, shape, stride=None):
    t = _Tensor()
    t.data = data
    t.dtype = dtype
    if stride is None:
        stride = [shape[1] * shape[2] * shape[3], shape[2] * shape[3], shape[3], 1]
    for a in range(4):
        t.shape[a] = shape[a]
        t.stride[a] = stride[a]
    return t


FAKE = 1 << 20  # never dereferenced: validation fails first


@pytest.mark.parametrize("case,code", [
    ("dtype_mix", dash.DASH_ERR_INVALID_ARG),
    ("shape_mismatch", dash.DASH_ERR_INVALID_ARG),
    ("gqa_wrong", dash.DASH_ERR_INVALID_ARG),
    ("head_dim", dash.DASH_ERR_UNSUPPORTED),
    ("block", dash.DASH_ERR_UNSUPPORTED),
    ("alpha", dash.DASH_ERR_INVALID_ARG),
    ("misaligned", dash.DASH_ERR_ALIGNMENT),
    ("stride", dash.DASH_ERR_ALIGNMENT),
    ("causal_long_q", dash.DASH_ERR_INVALID_ARG),
    ("null", dash.DASH_ERR_INVALID_ARG),
    ("sigma", dash.DASH_ERR_INVALID_ARG),
    ("qbar_shape", dash.DASH_ERR_INVALID_ARG),
    ("qbar_with_kbar", dash.DASH_ERR_INVALID_ARG),
    ("local2_noncausal", dash.DASH_ERR_INVALID_ARG),
])
def test_validation_rejects(lib, case, code):
    B, alpha, gqa, causal = 64, 1.5, 4, 1
    q = _t(FAKE, dash.DASH_BF16, [1, 256, 8, 128])
    k = _t(FAKE, dash.DASH_BF16, [1, 256, 2, 128])
    v = _t(FAKE, dash.DASH_BF16, [1, 256, 2, 128])
    o = _t(FAKE, dash.DASH_BF16, [1, 256, 8, 128])
    opts = _Opts()
    lib.dash_opts_init(ctypes.byref(opts))
    if case == "dtype_mix":
        v.dtype = dash.DASH_F32
    elif case == "shape_mismatch":
        o.shape[2] = 4
    elif case == "gqa_wrong":
        gqa = 2
    elif case == "head_dim":
        for t in (q, k, v, o):
            t.shape[3] = 96
    elif case == "block":
        B = 48
    elif case == "alpha":
        alpha = 1.0
    elif case == "misaligned":
        q.data = FAKE + 2
    elif case == "stride":
        k.stride[1] = 2 * 128 + 4
    elif case == "causal_long_q":
        q.shape[1] = o.shape[1] = 300
    elif case == "null":
        q.data = None
    elif case == "sigma":
        opts.sigma = 0.0
    elif case == "qbar_shape":  # 4 chunks of 64 keys, not 5
        qb = _t(FAKE, dash.DASH_F32, [1, 5, 2, 128])
        opts.qbar = ctypes.pointer(qb)
    elif case == "local2_noncausal":
        causal = 0
        opts.flags = dash.DASH_FLAG_LOCAL2
    elif case == "qbar_with_kbar":
        qb = _t(FAKE, dash.DASH_F32, [1, 4, 2, 128])
        opts.qbar = ctypes.pointer(qb)
        opts.kbar = FAKE
    rc = lib.dash_attn_fwd_ex(ctypes.byref(q), ctypes.byref(k), ctypes.byref(v), ctypes.byref(o), B, alpha, causal,
                              gqa, ctypes.byref(opts))
    assert rc == code, lib.dash_last_error()
    assert lib.dash_last_error()


def test_opts_defaults(lib):
    o = _Opts()
    assert lib.dash_opts_init(ctypes.byref(o)) == 0
    assert o.sigma == pytest.approx(1e8) and o.gamma == 1.0 and o.flags == 0 and not o.workspace
    assert not o.qbar and not o.kbar
    assert lib.dash_opts_init(None) == dash.DASH_ERR_INVALID_ARG


def test_summary_cache_arguments(lib):
    """Host-side checks of the summary-cache entry points (no device memory is touched)."""
    h = ctypes.c_void_p()
    assert lib.dash_summary_cache_create(1, 10, 1, 128, 64, ctypes.byref(h)) == dash.DASH_ERR_INVALID_ARG
    assert lib.dash_summary_cache_create(1, 4096, 1, 96, 64, ctypes.byref(h)) == dash.DASH_ERR_UNSUPPORTED
    assert lib.dash_summary_cache_create(1, 4096, 1, 128, 48, ctypes.byref(h)) == dash.DASH_ERR_UNSUPPORTED
    assert lib.dash_summary_cache_create(0, 4096, 1, 128, 64, ctypes.byref(h)) == dash.DASH_ERR_INVALID_ARG
    assert lib.dash_summary_cache_create(1, 4096, 1, 128, 64, None) == dash.DASH_ERR_INVALID_ARG
    assert lib.dash_summary_cache_chunks(None) == -1
    assert lib.dash_summary_cache_kbar(None) is None
    assert lib.dash_summary_cache_destroy(None) == 0
    assert lib.dash_summary_cache_reset(None) == dash.DASH_ERR_INVALID_ARG
    k = _t(FAKE, dash.DASH_BF16, [1, 256, 2, 128])
    assert lib.dash_summary_cache_update(None, ctypes.byref(k), None, None) == dash.DASH_ERR_INVALID_ARG


def test_lists_from_mask_arguments(lib):
    """dash_lists_from_mask rejects bad arguments on the host."""
    nt, cap, tr = dash.lists_geometry(1, 256, 256, 2, 64, 4)
    good = dash._Lists()
    good.count = good.ids = good.bias = good.rows = FAKE
    good.n_tiles, good.cap, good.tile_rows = nt, cap, tr
    call = lambda mask, lists, **kw: lib.dash_lists_from_mask(  # noqa: E731
        mask, kw.get("b", 1), kw.get("nq", 256), kw.get("nk", 256), kw.get("hkv", 2), kw.get("B", 64),
        kw.get("g", 4), 1, kw.get("regroup", 0), ctypes.byref(lists) if lists is not None else None, None)
    assert call(None, good) == dash.DASH_ERR_INVALID_ARG
    assert call(FAKE, None) == dash.DASH_ERR_INVALID_ARG
    assert call(FAKE + 4, good) == dash.DASH_ERR_ALIGNMENT
    assert call(FAKE, good, g=32) == dash.DASH_ERR_UNSUPPORTED
    assert call(FAKE, good, B=48) == dash.DASH_ERR_UNSUPPORTED
    assert call(FAKE, good, nq=512) == dash.DASH_ERR_INVALID_ARG   # lists made for 256 rows
    no_rows = dash._Lists()
    no_rows.count = no_rows.ids = no_rows.bias = FAKE
    no_rows.rows = None
    no_rows.n_tiles, no_rows.cap, no_rows.tile_rows = nt, cap, tr
    assert call(FAKE, no_rows, regroup=1) == dash.DASH_ERR_INVALID_ARG
    assert lib.dash_last_error()


def test_pool_keys_q_arguments(lib):
    """dash_pool_keys_q checks the summary queries' shape against the chunks (every call
    here is invalid, so nothing reaches the device)."""
    k = _t(FAKE, dash.DASH_BF16, [2, 1000, 2, 128])  # 1000 // 64 = 15 chunks
    kbar = FAKE
    for shape in ([3, 15, 2, 128],    # batch neither 1 nor 2
                  [1, 16, 2, 128],    # one chunk too many
                  [1, 15, 1, 128],    # kv heads
                  [1, 15, 2, 64]):    # head dim
        qb = _t(FAKE, dash.DASH_F32, shape)
        rc = lib.dash_pool_keys_q(ctypes.byref(k), ctypes.byref(qb), 64, 1, kbar, None)
        assert rc == dash.DASH_ERR_INVALID_ARG, (shape, lib.dash_last_error())
    qb = _t(FAKE, dash.DASH_F32, [1, 15, 2, 128])
    assert lib.dash_pool_keys_q(ctypes.byref(k), None, 64, 1, kbar, None) == dash.DASH_ERR_INVALID_ARG
    assert lib.dash_pool_keys_q(ctypes.byref(k), ctypes.byref(qb), 64, 1, None, None) == dash.DASH_ERR_INVALID_ARG


def test_host_staged_arguments(lib):
    """dash_attn_fwd_host checks its host / device pairs and options on the host (every call
    here is invalid, so no copy is enqueued and no device memory is touched)."""
    shapes = {"q": [1, 256, 8, 128], "k": [1, 256, 2, 128], "v": [1, 256, 2, 128], "o": [1, 256, 8, 128]}
    host = {n: _t(FAKE, dash.DASH_BF16, s) for n, s in shapes.items()}
    dev = {n: _t(FAKE, dash.DASH_BF16, s) for n, s in shapes.items()}
    opts = _Opts()
    lib.dash_opts_init(ctypes.byref(opts))

    def call(h=host, d=dev, o=opts, n_slices=0, B=64, alpha=1.5):
        return lib.dash_attn_fwd_host(*[ctypes.byref(h[n]) for n in "qkvo"], *[ctypes.byref(d[n]) for n in "qkvo"],
                                      B, alpha, 1, 4, n_slices, ctypes.byref(o))

    bad = dict(dev)
    bad["o"] = _t(FAKE, dash.DASH_BF16, [1, 128, 8, 128])  # not the host output's shape
    assert call(d=bad) == dash.DASH_ERR_INVALID_ARG
    bad = dict(host)
    bad["k"] = _t(FAKE, dash.DASH_F32, shapes["k"])  # another dtype than its device buffer
    assert call(h=bad) == dash.DASH_ERR_INVALID_ARG
    bad = dict(host)
    bad["q"] = _t(FAKE, dash.DASH_BF16, shapes["q"], stride=[256 * 8 * 128, 8 * 128 + 64, 128, 1])  # rows not packed
    assert call(h=bad) == dash.DASH_ERR_UNSUPPORTED
    assert call(n_slices=-1) == dash.DASH_ERR_INVALID_ARG
    with_lse = _Opts()
    lib.dash_opts_init(ctypes.byref(with_lse))
    with_lse.lse = FAKE
    assert call(o=with_lse) == dash.DASH_ERR_UNSUPPORTED
    assert call(B=48) == dash.DASH_ERR_UNSUPPORTED  # the forward's own validation, before any copy
    assert call(alpha=1.0) == dash.DASH_ERR_INVALID_ARG
    assert lib.dash_last_error()


def test_workspace_stays_within_the_slicing_budget(lib):
    """Long prefills run in row slices whose work lists fit about 1 GB of library workspace
    (host-side arithmetic only): 128K keys at batch 1 and 2, block 128 and 64."""
    for b, B in ((1, 128), (2, 128), (1, 64)):
        need = dash.dash_workspace_bytes(b, 131072, 131072, 32, 8, 128, B)
        assert 0 < need <= 10 ** 9, (b, B, need)
    # a short prefill takes the single-slice layout, which is smaller still
    assert dash.dash_workspace_bytes(1, 8192, 8192, 32, 8, 128, 64) < dash.dash_workspace_bytes(1, 131072, 131072,
                                                                                                 32, 8, 128, 128)


def test_backward_arguments(lib):
    """dash_attn_bwd rejects a missing lse and gradients of the wrong shape or dtype on the
    host (every call here is invalid, so nothing reaches the device)."""
    shp = {"q": [1, 256, 8, 128], "k": [1, 256, 2, 128]}
    t = {n: _t(FAKE, dash.DASH_BF16, shp["q" if n in ("q", "o", "do", "dq") else "k"])
         for n in ("q", "k", "v", "o", "do", "dq", "dk", "dv")}
    opts = _Opts()
    lib.dash_opts_init(ctypes.byref(opts))

    def call(lse=FAKE, **kw):
        a = dict(t)
        a.update(kw)
        return lib.dash_attn_bwd(ctypes.byref(a["q"]), ctypes.byref(a["k"]), ctypes.byref(a["v"]),
                                 ctypes.byref(a["o"]), ctypes.byref(a["do"]), lse, ctypes.byref(a["dq"]),
                                 ctypes.byref(a["dk"]), ctypes.byref(a["dv"]), 64, 1.5, 1, 4, ctypes.byref(opts))

    assert call(lse=None) == dash.DASH_ERR_INVALID_ARG
    assert call(dq=_t(FAKE, dash.DASH_BF16, [1, 128, 8, 128])) == dash.DASH_ERR_INVALID_ARG
    assert call(do=_t(FAKE, dash.DASH_BF16, [1, 256, 4, 128])) == dash.DASH_ERR_INVALID_ARG
    assert call(dk=_t(FAKE, dash.DASH_F32, shp["k"])) == dash.DASH_ERR_INVALID_ARG
    assert lib.dash_last_error()
    # the backward keeps the forward's Stage 0-1 state plus its own (transposed lists, tiles)
    assert dash.dash_bwd_workspace_bytes(1, 8192, 8192, 32, 8, 128, 64) > dash.dash_workspace_bytes(
        1, 8192, 8192, 32, 8, 128, 64)

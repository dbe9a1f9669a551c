"""B200-native DashAttention forward (sm_100a CUDA kernels behind a C ABI).

Thin ctypes binding of ``libdash_attn.so`` (declared in ``include/dash_attn.h``):
argument marshalling only, every stage runs in the library's kernels.  Tensors
are torch CUDA tensors laid out [batch, seq, heads, dim] (dim contiguous);
torch provides device memory and the current stream.  There is no CPU path: if
the library is missing or no GPU is present the calls raise.

Functions mirror the C entry points:
  dash_attn_fwd(q, k, v, out, block_size, alpha, causal, gqa_groups, **opts)
  dash_block_select(q, k, block_size, alpha, causal, gqa_groups, tau=, w=, mask=, lists=, **opts)
  dash_sparse_attn_fwd(q, k, v, out, lists, block_size, causal, gqa_groups, **opts)
  dash_pool_keys(k, block_size, causal, kbar, qbar=None)
  make_lists(...), dash_sync_status(), dash_release()
opts: sigma, gamma, kbar (fp32 tensor), qbar (Stage-0 summary queries), workspace (uint8
tensor), flags, stream.
"""
from __future__ import annotations

import ctypes
from pathlib import Path

import torch

_PKG = Path(__file__).resolve().parent
LIB_PATH = _PKG / "libdash_attn.so"

DASH_OK = 0
DASH_ERR_INVALID_ARG = -1
DASH_ERR_UNSUPPORTED = -2
DASH_ERR_ALIGNMENT = -3
DASH_ERR_WORKSPACE = -4
DASH_ERR_CUDA = -5
DASH_ERR_DEVICE_TIMEOUT = -6

DASH_F32 = 0
DASH_BF16 = 1

DASH_FLAG_FORCE_SIMT = 0x1
DASH_FLAG_NO_REGROUP = 0x2
DASH_FLAG_LOCAL2 = 0x4  # the two-block local window (the query's chunk and the one before)
DASH_FLAG_TEST_TIMEOUT = 0x100


class DashError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"dash error {code}: {msg}")
        self.code = code


class _Tensor(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("dtype", ctypes.c_int), ("shape", ctypes.c_int64 * 4),
                ("stride", ctypes.c_int64 * 4)]


class _Lists(ctypes.Structure):
    _fields_ = [("count", ctypes.c_void_p), ("ids", ctypes.c_void_p), ("bias", ctypes.c_void_p),
                ("rows", ctypes.c_void_p), ("n_tiles", ctypes.c_int64), ("cap", ctypes.c_int32),
                ("tile_rows", ctypes.c_int32)]


class _Opts(ctypes.Structure):
    _fields_ = [("sigma", ctypes.c_float), ("gamma", ctypes.c_float), ("stream", ctypes.c_void_p),
                ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
                ("kbar", ctypes.c_void_p), ("flags", ctypes.c_int),
                ("qbar", ctypes.POINTER(_Tensor)), ("summary_cache", ctypes.c_void_p), ("lse", ctypes.c_void_p),
                ("nk_dev", ctypes.c_void_p)]


_lib = None

# every entry point include/dash_attn.h declares
EXPORTS = ("dash_opts_init", "dash_attn_fwd", "dash_attn_fwd_ex", "dash_pool_keys", "dash_block_select",
           "dash_sparse_attn_fwd", "dash_lists_geometry", "dash_workspace_bytes", "dash_last_error",
           "dash_sync_status", "dash_release", "dash_version", "dash_attn_fwd_noalloc", "dash_pool_keys_q",
           "dash_lists_from_mask", "dash_summary_cache_create", "dash_summary_cache_update",
           "dash_summary_cache_reset", "dash_summary_cache_chunks", "dash_summary_cache_kbar",
           "dash_summary_cache_destroy", "dash_attn_bwd", "dash_bwd_workspace_bytes", "dash_attn_fwd_host")

# size of the library's static scratch area used by dash_attn_fwd_noalloc
DASH_NOALLOC_SCRATCH_BYTES = 32 << 20


def load_library():
    """Load libdash_attn.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not LIB_PATH.exists():
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m sparse_hierarchical_attention_block_b200.build`")
    lib = ctypes.CDLL(str(LIB_PATH))
    P, i32, i64, f32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
    T = ctypes.POINTER(_Tensor)
    lib.dash_opts_init.argtypes = [ctypes.POINTER(_Opts)]
    lib.dash_attn_fwd.argtypes = [T, T, T, T, i32, f32, i32, i32]
    lib.dash_attn_fwd_ex.argtypes = [T, T, T, T, i32, f32, i32, i32, ctypes.POINTER(_Opts)]
    lib.dash_attn_fwd_noalloc.argtypes = [T, T, T, T, i32, f32, i32, i32, ctypes.POINTER(_Opts)]
    lib.dash_attn_fwd_host.argtypes = [T, T, T, T, T, T, T, T, i32, f32, i32, i32, i32, ctypes.POINTER(_Opts)]
    lib.dash_pool_keys.argtypes = [T, i32, i32, P, P]
    lib.dash_pool_keys_q.argtypes = [T, T, i32, i32, P, P]
    lib.dash_lists_from_mask.argtypes = [P, i64, i64, i64, i32, i32, i32, i32, i32, ctypes.POINTER(_Lists), P]
    lib.dash_summary_cache_create.argtypes = [i64, i64, i32, i32, i32, ctypes.POINTER(ctypes.c_void_p)]
    lib.dash_summary_cache_update.argtypes = [P, T, T, P]
    lib.dash_summary_cache_reset.argtypes = [P]
    lib.dash_summary_cache_chunks.argtypes = [P]
    lib.dash_summary_cache_chunks.restype = i64
    lib.dash_summary_cache_kbar.argtypes = [P]
    lib.dash_summary_cache_kbar.restype = P
    lib.dash_summary_cache_destroy.argtypes = [P]
    lib.dash_block_select.argtypes = [T, T, i32, f32, i32, i32, P, P, P, ctypes.POINTER(_Lists),
                                      ctypes.POINTER(_Opts)]
    lib.dash_sparse_attn_fwd.argtypes = [T, T, T, T, ctypes.POINTER(_Lists), i32, i32, i32, ctypes.POINTER(_Opts)]
    lib.dash_lists_geometry.argtypes = [i64, i64, i64, i32, i32, i32, ctypes.POINTER(i64), ctypes.POINTER(ctypes.c_int32),
                                        ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(sz), ctypes.POINTER(sz),
                                        ctypes.POINTER(sz), ctypes.POINTER(sz)]
    lib.dash_workspace_bytes.argtypes = [i64, i64, i64, i32, i32, i32, i32, i32]
    lib.dash_workspace_bytes.restype = sz
    lib.dash_attn_bwd.argtypes = [T, T, T, T, T, P, T, T, T, i32, f32, i32, i32, ctypes.POINTER(_Opts)]
    lib.dash_bwd_workspace_bytes.argtypes = [i64, i64, i64, i32, i32, i32, i32, i32]
    lib.dash_bwd_workspace_bytes.restype = sz
    lib.dash_last_error.restype = ctypes.c_char_p
    lib.dash_sync_status.argtypes = [P]
    lib.dash_version.restype = ctypes.c_char_p
    _lib = lib
    return lib


def _check(rc: int):
    if rc != DASH_OK:
        raise DashError(rc, load_library().dash_last_error().decode())


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return DASH_BF16
    if t.dtype == torch.float32:
        return DASH_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _desc(t: torch.Tensor, host: bool = False) -> _Tensor:
    if t.dim() != 4:
        raise ValueError("tensors are [batch, seq, heads, dim]")
    if host:
        if t.is_cuda:
            raise ValueError("host tensors must be CPU tensors (page-locked for asynchronous copies)")
    elif not t.is_cuda:
        raise ValueError("tensors must be CUDA tensors (the library has no CPU path)")
    d = _Tensor()
    d.data = t.data_ptr()
    d.dtype = _dtype_code(t)
    for a in range(4):
        d.shape[a] = t.shape[a]
        d.stride[a] = t.stride(a)
    return d


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _opts(sigma=1e8, gamma=1.0, kbar=None, workspace=None, flags=0, stream=None, qbar=None,
          summary_cache=None, lse=None, nk_dev=None) -> _Opts:
    o = _Opts()
    load_library().dash_opts_init(ctypes.byref(o))
    o.sigma = float(sigma)
    o.gamma = float(gamma)
    if stream is None:
        stream = torch.cuda.current_stream()
    o.stream = stream.cuda_stream if hasattr(stream, "cuda_stream") else stream
    if workspace is not None:
        o.workspace = workspace.data_ptr()
        o.workspace_bytes = workspace.numel() * workspace.element_size()
    if kbar is not None:
        if kbar.dtype != torch.float32 or not kbar.is_contiguous():
            raise ValueError("kbar must be a contiguous float32 tensor")
        o.kbar = kbar.data_ptr()
    if qbar is not None:
        qd = _desc(qbar)
        o._qbar_desc = qd  # kept alive with the options
        o.qbar = ctypes.pointer(qd)
    if summary_cache is not None:
        o.summary_cache = summary_cache.handle
    if nk_dev is not None:
        if nk_dev.dtype != torch.int64 or not nk_dev.is_cuda:
            raise ValueError("nk_dev must be an int64 tensor on the device (one element)")
        o.nk_dev = nk_dev.data_ptr()
    if lse is not None:
        if lse.dtype != torch.float32 or not lse.is_contiguous():
            raise ValueError("lse must be a contiguous float32 tensor [b, nq, hq]")
        o.lse = lse.data_ptr()
    o.flags = int(flags)
    return o


class SummaryCache:
    """Persistent chunk-summary cache for incremental decoding (dash_summary_cache_*):
    the fp32 summaries of every completed chunk and their split operand form, kept on
    the device across decoding steps.  update(k) pools the chunks completed since the
    last update; pass the cache to a forward as ``summary_cache=``."""

    def __init__(self, batch, max_nk, hkv, d, block_size):
        self._lib = load_library()
        h = ctypes.c_void_p()
        _check(self._lib.dash_summary_cache_create(int(batch), int(max_nk), int(hkv), int(d), int(block_size),
                                                   ctypes.byref(h)))
        self.handle = h.value
        self.batch, self.max_nk, self.hkv, self.d, self.block_size = batch, max_nk, hkv, d, block_size

    def update(self, k, qbar=None, stream=None):
        kd = _desc(k)
        qd = ctypes.byref(_desc(qbar)) if qbar is not None else None
        s = torch.cuda.current_stream() if stream is None else stream
        _check(self._lib.dash_summary_cache_update(self.handle, ctypes.byref(kd), qd, ctypes.c_void_p(s.cuda_stream)))
        return self

    def reset(self):
        _check(self._lib.dash_summary_cache_reset(self.handle))

    @property
    def chunks(self) -> int:
        return int(self._lib.dash_summary_cache_chunks(self.handle))

    def kbar(self) -> torch.Tensor:
        """A copy of the cached summaries [batch, max_nk // block_size, hkv, d] (fp32)."""
        shape = (self.batch, self.max_nk // self.block_size, self.hkv, self.d)
        ptr = self._lib.dash_summary_cache_kbar(self.handle)

        class _View:  # the cache's own buffer, read through the CUDA array interface
            __cuda_array_interface__ = {"shape": shape, "typestr": "<f4", "data": (ptr, False), "version": 3,
                                        "strides": None}

        return torch.as_tensor(_View(), device="cuda").clone()

    def close(self):
        if self.handle:
            _check(self._lib.dash_summary_cache_destroy(self.handle))
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def n_chunks(nk: int, block_size: int, causal: bool) -> int:
    return nk // block_size if causal else -(-nk // block_size)


def lists_geometry(batch, nq, nk, hkv, block_size, gqa_groups):
    """(n_tiles, cap, tile_rows) of the Stage-2 work lists."""
    nt, cap, tr = ctypes.c_int64(), ctypes.c_int32(), ctypes.c_int32()
    _check(load_library().dash_lists_geometry(batch, nq, nk, hkv, block_size, gqa_groups, ctypes.byref(nt),
                                              ctypes.byref(cap), ctypes.byref(tr), None, None, None, None))
    return nt.value, cap.value, tr.value


class Lists:
    """Device buffers of the Stage-2 work lists (see dash_lists_t).

    with_rows: allocate the row-permutation buffer, so that Stage 1 may regroup
    rows across tiles; without it every tile holds consecutive query rows."""

    def __init__(self, batch, nq, nk, hkv, block_size, gqa_groups, device="cuda", with_rows=True):
        self.n_tiles, self.cap, self.tile_rows = lists_geometry(batch, nq, nk, hkv, block_size, gqa_groups)
        self.count = torch.zeros(batch, hkv, self.n_tiles, dtype=torch.int32, device=device)
        self.ids = torch.zeros(batch, hkv, self.n_tiles, self.cap, dtype=torch.int32, device=device)
        self.bias = torch.zeros(batch, hkv, self.n_tiles, self.cap, self.tile_rows, dtype=torch.float32,
                                device=device)
        self.rows = (torch.full((batch, hkv, self.n_tiles, self.tile_rows), -1, dtype=torch.int32, device=device)
                     if with_rows else None)

    def c(self) -> _Lists:
        l = _Lists()
        l.count, l.ids, l.bias = self.count.data_ptr(), self.ids.data_ptr(), self.bias.data_ptr()
        l.rows = self.rows.data_ptr() if self.rows is not None else None
        l.n_tiles, l.cap, l.tile_rows = self.n_tiles, self.cap, self.tile_rows
        return l


def make_lists(q, k, block_size, gqa_groups, with_rows=True) -> Lists:
    return Lists(q.shape[0], q.shape[1], k.shape[1], k.shape[2], block_size, gqa_groups, device=q.device,
                 with_rows=with_rows)


def lists_from_mask(mask, nk, hkv, block_size, gqa_groups, causal=True, regroup=False, stream=None) -> Lists:
    """Stage-2 work lists from a routing mask [b, nq, hkv, words] int32 (bit-packed chunks,
    dash_lists_from_mask): routed chunks get bias 0, each row's diagonal chunk is added."""
    if not mask.is_cuda or mask.dtype != torch.int32 or not mask.is_contiguous():
        raise ValueError("mask must be a contiguous int32 CUDA tensor")
    b, nq = mask.shape[0], mask.shape[1]
    lists = Lists(b, nq, nk, hkv, block_size, gqa_groups, device=mask.device, with_rows=True)
    s = torch.cuda.current_stream() if stream is None else stream
    lc = lists.c()
    _check(load_library().dash_lists_from_mask(ctypes.c_void_p(mask.data_ptr()), b, nq, nk, hkv, int(block_size),
                                               int(gqa_groups), int(bool(causal)), int(bool(regroup)),
                                               ctypes.byref(lc), ctypes.c_void_p(s.cuda_stream)))
    return lists


def dash_attn_fwd(q, k, v, out, block_size, alpha, causal=True, gqa_groups=None, **opts):
    """Full forward (Stages 0-2) into ``out``; returns ``out``."""
    lib = load_library()
    g = gqa_groups if gqa_groups is not None else q.shape[2] // k.shape[2]
    qd, kd, vd, od = _desc(q), _desc(k), _desc(v), _desc(out)
    if opts:
        o = _opts(**opts)
        _check(lib.dash_attn_fwd_ex(ctypes.byref(qd), ctypes.byref(kd), ctypes.byref(vd), ctypes.byref(od),
                                    int(block_size), float(alpha), int(bool(causal)), int(g), ctypes.byref(o)))
    else:
        _check(lib.dash_attn_fwd(ctypes.byref(qd), ctypes.byref(kd), ctypes.byref(vd), ctypes.byref(od),
                                 int(block_size), float(alpha), int(bool(causal)), int(g)))
    return out


def dash_attn_fwd_noalloc(q, k, v, out, block_size, alpha, causal=True, gqa_groups=None, **opts):
    """Full forward into ``out`` without any device allocation by the library:
    the intermediates go to its static scratch area of DASH_NOALLOC_SCRATCH_BYTES
    (problems that need more raise DashError with DASH_ERR_WORKSPACE).  Calls
    share that area: do not let two of them run concurrently on the GPU.
    ``opts`` as for dash_attn_fwd, except ``workspace``."""
    lib = load_library()
    g = gqa_groups if gqa_groups is not None else q.shape[2] // k.shape[2]
    qd, kd, vd, od = _desc(q), _desc(k), _desc(v), _desc(out)
    o = _opts(**opts)
    _check(lib.dash_attn_fwd_noalloc(ctypes.byref(qd), ctypes.byref(kd), ctypes.byref(vd), ctypes.byref(od),
                                     int(block_size), float(alpha), int(bool(causal)), int(g), ctypes.byref(o)))
    return out


def dash_attn_fwd_host(q_host, k_host, v_host, out_host, q_dev, k_dev, v_dev, out_dev, block_size, alpha,
                       causal=True, gqa_groups=None, n_slices=0, **opts):
    """Full forward of host tensors (pinned CPU memory) into ``out_host`` through the device
    buffers ``*_dev`` (same shapes and dtypes), query rows in ``n_slices`` slices whose
    copies in and out overlap the computation (0 = automatic).  Asynchronous on ``stream``
    (default: the current stream): ``out_host`` is complete once that stream has reached
    this point.  Returns ``out_host``."""
    lib = load_library()
    g = gqa_groups if gqa_groups is not None else q_dev.shape[2] // k_dev.shape[2]
    ds = [_desc(t, host=True) for t in (q_host, k_host, v_host, out_host)] + [_desc(t) for t in (q_dev, k_dev, v_dev, out_dev)]
    o = _opts(**opts)
    _check(lib.dash_attn_fwd_host(*[ctypes.byref(d) for d in ds], int(block_size), float(alpha), int(bool(causal)),
                                  int(g), int(n_slices), ctypes.byref(o)))
    return out_host


def dash_attn_bwd(q, k, v, out, dout, lse, dq, dk, dv, block_size, alpha, causal=True, gqa_groups=None, **opts):
    """Backward pass: writes dq, dk, dv (the gradients of sum(dout * out)) for the forward
    that produced ``out`` and ``lse`` (pass ``lse=`` to dash_attn_fwd) with the same
    ``block_size``, ``alpha``, ``causal`` and options (sigma, gamma, flags)."""
    lib = load_library()
    g = gqa_groups if gqa_groups is not None else q.shape[2] // k.shape[2]
    if lse.dtype != torch.float32 or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous float32 tensor [b, nq, hq]")
    ds = [_desc(t) for t in (q, k, v, out, dout, dq, dk, dv)]
    o = _opts(**opts)
    _check(lib.dash_attn_bwd(ctypes.byref(ds[0]), ctypes.byref(ds[1]), ctypes.byref(ds[2]), ctypes.byref(ds[3]),
                             ctypes.byref(ds[4]), ctypes.c_void_p(lse.data_ptr()), ctypes.byref(ds[5]),
                             ctypes.byref(ds[6]), ctypes.byref(ds[7]), int(block_size), float(alpha),
                             int(bool(causal)), int(g), ctypes.byref(o)))
    return dq, dk, dv


def dash_bwd_workspace_bytes(batch, nq, nk, hq, hkv, d, block_size, causal=True) -> int:
    return int(load_library().dash_bwd_workspace_bytes(int(batch), int(nq), int(nk), int(hq), int(hkv), int(d),
                                                       int(block_size), int(bool(causal))))


def dash_pool_keys(k, block_size, causal, kbar, stream=None, qbar=None):
    """Stage 0 into ``kbar`` [b, n_chunks, hkv, d] fp32: the chunk means, or with
    ``qbar`` [1 or b, n_chunks, hkv, d] (a broadcast view is fine) the learned-query
    softmax pooling of dash_pool_keys_q."""
    lib = load_library()
    kd = _desc(k)
    s = torch.cuda.current_stream() if stream is None else stream
    if qbar is None:
        _check(lib.dash_pool_keys(ctypes.byref(kd), int(block_size), int(bool(causal)), _ptr(kbar),
                                  ctypes.c_void_p(s.cuda_stream)))
    else:
        qd = _desc(qbar)
        _check(lib.dash_pool_keys_q(ctypes.byref(kd), ctypes.byref(qd), int(block_size), int(bool(causal)),
                                    _ptr(kbar), ctypes.c_void_p(s.cuda_stream)))
    return kbar


def dash_block_select(q, k, block_size, alpha, causal=True, gqa_groups=None, tau=None, w=None, mask=None,
                      lists: Lists | None = None, **opts):
    lib = load_library()
    g = gqa_groups if gqa_groups is not None else q.shape[2] // k.shape[2]
    qd, kd = _desc(q), _desc(k)
    o = _opts(**opts)
    lc = lists.c() if lists is not None else None
    _check(lib.dash_block_select(ctypes.byref(qd), ctypes.byref(kd), int(block_size), float(alpha),
                                 int(bool(causal)), int(g), _ptr(tau), _ptr(w), _ptr(mask),
                                 ctypes.byref(lc) if lc is not None else None, ctypes.byref(o)))


def dash_sparse_attn_fwd(q, k, v, out, lists: Lists, block_size, causal=True, gqa_groups=None, **opts):
    lib = load_library()
    g = gqa_groups if gqa_groups is not None else q.shape[2] // k.shape[2]
    qd, kd, vd, od = _desc(q), _desc(k), _desc(v), _desc(out)
    o = _opts(**opts)
    lc = lists.c()
    _check(lib.dash_sparse_attn_fwd(ctypes.byref(qd), ctypes.byref(kd), ctypes.byref(vd), ctypes.byref(od),
                                    ctypes.byref(lc), int(block_size), int(bool(causal)), int(g), ctypes.byref(o)))
    return out


def dash_workspace_bytes(batch, nq, nk, hq, hkv, d, block_size, causal=True) -> int:
    return int(load_library().dash_workspace_bytes(batch, nq, nk, hq, hkv, d, block_size, int(bool(causal))))


def dash_sync_status(stream=None) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return int(load_library().dash_sync_status(ctypes.c_void_p(s.cuda_stream)))


def dash_release() -> None:
    _check(load_library().dash_release())


def version() -> str:
    return load_library().dash_version().decode()

"""Incremental decoding with the persistent chunk-summary cache (dash_summary_cache_*),
and a decoding step captured in a CUDA graph."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import sparse_hierarchical_attention_block_b200 as dash
import synthetic
from parity import check_forward

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.fail("the gpu tests need a CUDA device")
    dash.load_library()
    oracle.set_threads(oracle.max_threads())
    yield
    dash.dash_release()


def _kv(b, n, hkv, d, seed, dtype=torch.bfloat16):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(b, n, hkv, d, generator=g).to(dtype).cuda(),
            torch.randn(b, n, hkv, d, generator=g).to(dtype).cuda())


@pytest.mark.parametrize("learned", [False, True])
def test_incremental_pooling_equals_one_shot(learned):
    b, max_nk, hkv, d, B = 2, 1100, 2, 128, 64
    k, _ = _kv(b, max_nk, hkv, d, seed=1)
    qbar = None
    if learned:
        qbar = torch.randn(1, max_nk // B, hkv, d, generator=torch.Generator().manual_seed(2)).cuda()
    cache = dash.SummaryCache(b, max_nk, hkv, d, B)
    for nk in (300, 300, 700, 1100):
        cache.update(k[:, :nk], qbar=qbar)
        assert cache.chunks == nk // B
    full = torch.empty(b, max_nk // B, hkv, d, dtype=torch.float32, device="cuda")
    dash.dash_pool_keys(k, B, True, full, qbar=qbar)
    torch.cuda.synchronize()
    assert torch.equal(cache.kbar(), full)
    cache.close()


def test_decode_steps_with_cache_equal_full_forward():
    """Steps of one new token each, across a chunk boundary: the forward with the cache
    (Stage 0 and the split summaries reused) is bit-identical to the forward that pools
    and splits everything itself; one step is also checked against the oracle."""
    b, hq, hkv, d, B, max_nk = 2, 32, 8, 128, 64, 4200
    k, v = _kv(b, max_nk, hkv, d, seed=3)
    cache = dash.SummaryCache(b, max_nk, hkv, d, B)
    gen = torch.Generator().manual_seed(4)
    for nk in range(4093, 4099):
        q = (3 * torch.randn(b, 1, hq, d, generator=gen)).to(torch.bfloat16).cuda()
        cache.update(k[:, :nk])
        a = torch.empty_like(q)
        c = torch.empty_like(q)
        dash.dash_attn_fwd(q, k[:, :nk], v[:, :nk], a, B, 1.5, True, hq // hkv, summary_cache=cache)
        dash.dash_attn_fwd(q, k[:, :nk], v[:, :nk], c, B, 1.5, True, hq // hkv, sigma=1e8)
        assert dash.dash_sync_status() == 0
        assert torch.equal(a, c), nk
    check_forward(q, k[:, :nk], v[:, :nk], a, B, 1.5, True, label="decode with summary cache")
    cache.close()


def test_prefill_with_cache_equals_full_forward():
    w = synthetic.Workload("cache-prefill", 1, 1000, 1000, 8, 2, 128, 64, 1.5, True, "bf16", 9, True,
                           amax_key="b64")
    q, k, v = synthetic.make_inputs(w, "cuda")
    cache = dash.SummaryCache(1, 1024, 2, 128, 64).update(k)
    a, c = torch.empty_like(q), torch.empty_like(q)
    dash.dash_attn_fwd(q, k, v, a, 64, 1.5, True, 4, summary_cache=cache)
    dash.dash_attn_fwd(q, k, v, c, 64, 1.5, True, 4, sigma=1e8)
    assert dash.dash_sync_status() == 0
    assert torch.equal(a, c)
    cache.close()


def test_cache_misuse_is_rejected():
    b, hq, hkv, d, B = 1, 8, 2, 64, 64
    k, v = _kv(b, 1024, hkv, d, seed=5)
    q = torch.randn(b, 1, hq, d, device="cuda").to(torch.bfloat16)
    out = torch.empty_like(q)
    cache = dash.SummaryCache(b, 1024, hkv, d, B).update(k[:, :600])
    with pytest.raises(dash.DashError):  # two chunks completed since the update
        dash.dash_attn_fwd(q, k[:, :729], v[:, :729], out, B, 1.5, True, 4, summary_cache=cache)
    with pytest.raises(dash.DashError):  # the keys shrank below what was pooled
        cache.update(k[:, :400])
    with pytest.raises(dash.DashError):  # another head dim
        dash.SummaryCache(b, 1024, hkv, 128, B).update(k)
    cache.reset()
    assert cache.chunks == 0
    cache.update(k[:, :729])
    dash.dash_attn_fwd(q, k[:, :729], v[:, :729], out, B, 1.5, True, 4, summary_cache=cache)
    assert dash.dash_sync_status() == 0
    cache.close()


def test_decode_step_replays_from_a_cuda_graph():
    """A decoding step (cached summaries, caller workspace) captured once and replayed:
    the replay writes the same output as the direct call."""
    b, hq, hkv, d, B, nk = 4, 32, 8, 128, 64, 8192
    k, v = _kv(b, nk, hkv, d, seed=6)
    q = (3 * torch.randn(b, 1, hq, d, generator=torch.Generator().manual_seed(7))).to(torch.bfloat16).cuda()
    cache = dash.SummaryCache(b, nk, hkv, d, B).update(k)
    ws = torch.empty(dash.dash_workspace_bytes(b, 1, nk, hq, hkv, d, B), dtype=torch.uint8, device="cuda")
    direct = torch.empty_like(q)
    dash.dash_attn_fwd(q, k, v, direct, B, 1.5, True, hq // hkv, summary_cache=cache, workspace=ws)
    torch.cuda.synchronize()
    out = torch.zeros_like(q)
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph, stream=side):
            dash.dash_attn_fwd(q, k, v, out, B, 1.5, True, hq // hkv, summary_cache=cache, workspace=ws,
                               stream=side)
    torch.cuda.current_stream().wait_stream(side)
    for _ in range(3):
        out.zero_()
        graph.replay()
        torch.cuda.synchronize()
        assert torch.equal(out, direct)
    del graph
    cache.close()


def test_one_graph_serves_growing_lengths():
    """Decoding from a preallocated KV cache with a device-resident length (opts nk_dev):
    one captured step is replayed while the sequences grow one token per step across
    chunk boundaries (the call itself pools each completed chunk on the device).  Every
    replay equals, bit for bit, the plain forward on the keys written so far."""
    b, hq, hkv, d, B, cap = 2, 16, 4, 128, 64, 2048
    k, v = _kv(b, cap, hkv, d, seed=11)
    nk0 = 1000
    cache = dash.SummaryCache(b, cap, hkv, d, B).update(k[:, :nk0])
    nk_dev = torch.tensor([nk0], dtype=torch.int64, device="cuda")
    gen = torch.Generator().manual_seed(12)
    q = torch.empty(b, 1, hq, d, dtype=torch.bfloat16, device="cuda")
    q.copy_((3 * torch.randn(b, 1, hq, d, generator=gen)).to(torch.bfloat16))
    out = torch.empty_like(q)
    ws = torch.empty(dash.dash_workspace_bytes(b, 1, cap, hq, hkv, d, B), dtype=torch.uint8, device="cuda")
    opts = dict(summary_cache=cache, workspace=ws, nk_dev=nk_dev)
    dash.dash_attn_fwd(q, k, v, out, B, 1.5, True, hq // hkv, **opts)  # warm-up outside the capture
    assert dash.dash_sync_status() == 0
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph, stream=side):
            dash.dash_attn_fwd(q, k, v, out, B, 1.5, True, hq // hkv, stream=side, **opts)
    torch.cuda.current_stream().wait_stream(side)
    ref = torch.empty_like(q)
    # one token per step, then jumps of at most 16 chunks (what one call catches up on)
    for nk in list(range(nk0 + 1, nk0 + 90)) + [1600, 1601, 1664, 2048]:
        nk_dev.fill_(nk)
        q.copy_((3 * torch.randn(b, 1, hq, d, generator=gen)).to(torch.bfloat16))
        graph.replay()
        torch.cuda.synchronize()
        dash.dash_attn_fwd(q, k[:, :nk], v[:, :nk], ref, B, 1.5, True, hq // hkv)
        assert dash.dash_sync_status() == 0
        assert torch.equal(out, ref), nk
    del graph
    cache.close()


def test_device_length_misuse_is_rejected():
    b, hq, hkv, d, B = 1, 8, 2, 128, 64
    k, v = _kv(b, 1024, hkv, d, seed=13)
    q = torch.randn(b, 1, hq, d, device="cuda").to(torch.bfloat16)
    out = torch.empty_like(q)
    nk_dev = torch.tensor([700], dtype=torch.int64, device="cuda")
    with pytest.raises(dash.DashError):  # a device length needs a summary cache
        dash.dash_attn_fwd(q, k, v, out, B, 1.5, True, 4, nk_dev=nk_dev)
    small = dash.SummaryCache(b, 512, hkv, d, B)
    with pytest.raises(dash.DashError):  # the keys' capacity exceeds the cache's
        dash.dash_attn_fwd(q, k, v, out, B, 1.5, True, 4, nk_dev=nk_dev, summary_cache=small)
    small.close()
    cache = dash.SummaryCache(b, 1024, hkv, d, B)
    with pytest.raises(dash.DashError):  # prefill rows: not the decoding path
        qq = torch.randn(b, 64, hq, d, device="cuda").to(torch.bfloat16)
        dash.dash_attn_fwd(qq, k, v, torch.empty_like(qq), B, 1.5, True, 4, nk_dev=nk_dev, summary_cache=cache)
    cache.close()

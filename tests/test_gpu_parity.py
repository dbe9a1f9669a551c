"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the
same seeded inputs.  Small cases run every row; the large workloads run every
row where the oracle finishes in seconds (8K prefill, decode) and stratified
row samples otherwise (32K, 128K)."""
import numpy as np
import pytest
import torch

import oracle
import sparse_hierarchical_attention_block_b200 as dash
import synthetic
from parity import check_forward, sample_rows, to_np32

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.fail("the gpu tests need a CUDA device")
    dash.load_library()
    oracle.set_threads(oracle.max_threads())
    yield
    dash.dash_release()


def _run(q, k, v, block, alpha, causal, **opts):
    out = torch.empty_like(q)
    dash.dash_attn_fwd(q, k, v, out, block, alpha, causal, q.shape[2] // k.shape[2], **opts)
    assert dash.dash_sync_status() == 0
    return out


def _planted(b, nq, nk, hq, hkv, d, block, dtype, seed, causal=True, planted=True):
    w = synthetic.Workload("case", b, nq, nk, hq, hkv, d, block, 1.5, causal, dtype, seed, planted,
                           amax_key="b64")
    q, k, v = synthetic.make_inputs(w, "cuda")
    return q, k, v


@pytest.mark.parametrize("sigma", [1e8, 1.0])
def test_tiny_full(sigma):
    w = synthetic.WORKLOADS["tiny"]
    q, k, v = synthetic.make_inputs(w, "cuda")
    out = _run(q, k, v, w.block, w.alpha, True, sigma=sigma)
    check_forward(q, k, v, out, w.block, w.alpha, True, sigma=sigma, label=f"tiny sigma={sigma:g}")


@pytest.mark.parametrize("sigma", [1e8, 1.0])
def test_tiny_planted_full(sigma):
    """The Tiny shape (fp32, 1 head, 16 chunks) with planted blocks, so that its
    routing is sparse and the fp32 CUDA-core path routes and masks chunks."""
    w = synthetic.WORKLOADS["tiny"].with_(planted=True, amax_key="b64", seed=9)
    q, k, v = synthetic.make_inputs(w, "cuda")
    out = _run(q, k, v, w.block, w.alpha, True, sigma=sigma)
    st = check_forward(q, k, v, out, w.block, w.alpha, True, sigma=sigma, label=f"tiny-planted sigma={sigma:g}")
    assert st["sparsity"] > 0.3


CASES = [
    # b, nq, nk, hq, hkv, d, B, dtype, alpha, causal, sigma
    (2, 512, 512, 8, 2, 128, 64, "bf16", 1.5, True, 1.0),
    (1, 512, 512, 8, 2, 128, 64, "bf16", 1.25, True, 1.0),
    (1, 512, 512, 8, 2, 128, 64, "bf16", 2.0, True, 1e8),
    (1, 1000, 1000, 8, 2, 128, 64, "bf16", 1.5, True, 1.0),      # ragged: nk % B != 0
    (1, 130, 1000, 8, 2, 128, 64, "bf16", 1.5, True, 1.0),       # nq < nk, bottom-right alignment
    (1, 700, 700, 4, 4, 64, 32, "bf16", 1.5, True, 3.0),         # hq == hkv, d = 64
    (1, 600, 600, 16, 2, 128, 16, "bf16", 1.5, True, 1.0),       # g = 8, B = 16
    (1, 1024, 1024, 8, 2, 128, 128, "bf16", 1.5, True, 1.0),     # B = 128
    (1, 300, 1000, 4, 2, 64, 64, "bf16", 1.5, False, 1.0),       # non-causal, partial chunk routed
    (1, 777, 777, 2, 1, 64, 64, "f32", 1.5, True, 1.0),          # fp32, g = 2
    (1, 40, 40, 4, 2, 64, 64, "bf16", 1.5, True, 1.0),           # no visible chunk at all
]


@pytest.mark.parametrize("case", CASES, ids=[f"c{i}" for i in range(len(CASES))])
def test_small_cases(case):
    b, nq, nk, hq, hkv, d, B, dt, alpha, causal, sigma = case
    q, k, v = _planted(b, nq, nk, hq, hkv, d, B, dt, seed=100 + nq, causal=causal)
    out = _run(q, k, v, B, alpha, causal, sigma=sigma)
    check_forward(q, k, v, out, B, alpha, causal, sigma=sigma, label=f"case {case}")


@pytest.mark.parametrize("case", CASES[:3] + CASES[9:10], ids=["c0", "c1", "c2", "c9"])
def test_simt_path_matches_oracle(case):
    """The CUDA-core Stage 2 (forced) also meets the bar."""
    b, nq, nk, hq, hkv, d, B, dt, alpha, causal, sigma = case
    q, k, v = _planted(b, nq, nk, hq, hkv, d, B, dt, seed=100 + nq, causal=causal)
    out = _run(q, k, v, B, alpha, causal, sigma=sigma, flags=dash.DASH_FLAG_FORCE_SIMT)
    check_forward(q, k, v, out, B, alpha, causal, sigma=sigma, label=f"simt {case}")


_DT = {"bf16": torch.bfloat16, "f32": torch.float32}


@pytest.mark.parametrize("kdt,qdt,d,B,causal,bcast", [
    ("bf16", "f32", 128, 64, False, False),   # trailing partial chunk pooled over its real keys
    ("f32", "bf16", 64, 16, True, True),      # one query per head, broadcast over batch and chunks
    ("bf16", "bf16", 128, 128, True, False),
])
def test_pool_keys_q_matches_oracle(kdt, qdt, d, B, causal, bcast):
    """Stage 0 with a learned summary query (Eq. 3) against the oracle's pooling."""
    gen = torch.Generator().manual_seed(41 + d + B)
    b, nk, hkv = 2, 1000, 2
    nch = dash.n_chunks(nk, B, causal)
    k = torch.randn(b, nk, hkv, d, generator=gen).to(_DT[kdt]).cuda()
    if bcast:
        qbar = (2 * torch.randn(1, 1, hkv, d, generator=gen)).to(_DT[qdt]).cuda().expand(1, nch, hkv, d)
    else:
        qbar = (2 * torch.randn(b, nch, hkv, d, generator=gen)).to(_DT[qdt]).cuda()
    kbar = torch.empty(b, nch, hkv, d, dtype=torch.float32, device="cuda")
    dash.dash_pool_keys(k, B, causal, kbar, qbar=qbar)
    assert dash.dash_sync_status() == 0
    for bi in range(b):
        ref = oracle.pool_q(to_np32(k[bi]), to_np32(qbar[bi if qbar.shape[0] > 1 else 0]), B, n_chunks=nch)
        err = np.abs(to_np32(kbar[bi]).astype(np.float64) - ref).max()
        assert err <= 5e-5, f"learned pooling error {err}"


@pytest.mark.parametrize("case", [CASES[0], CASES[3], CASES[5]], ids=["c0", "c3", "c5"])
def test_learned_summary_forward(case):
    """The full forward with learned summary queries against the oracle's forward with the same q̄."""
    b, nq, nk, hq, hkv, d, B, dt, alpha, causal, sigma = case
    q, k, v = _planted(b, nq, nk, hq, hkv, d, B, dt, seed=300 + nq, causal=causal)
    gen = torch.Generator().manual_seed(7 + nq)
    nch = dash.n_chunks(nk, B, causal)
    qbar = (0.5 * torch.randn(b, nch, hkv, d, generator=gen)).to(q.dtype).cuda()
    out = _run(q, k, v, B, alpha, causal, sigma=sigma, qbar=qbar)
    check_forward(q, k, v, out, B, alpha, causal, sigma=sigma, label=f"learned q̄ {case}", qbar=qbar)


def test_learned_summary_arguments_are_checked():
    q, k, v = _planted(1, 256, 256, 4, 2, 64, 64, "bf16", seed=5)
    out = torch.empty_like(q)
    nch = dash.n_chunks(256, 64, True)
    with pytest.raises(dash.DashError):  # wrong number of chunks
        dash.dash_attn_fwd(q, k, v, out, 64, 1.5, True, 2, qbar=torch.zeros(1, nch + 1, 2, 64, device="cuda"))
    kb = torch.zeros(1, nch, 2, 64, device="cuda")
    with pytest.raises(dash.DashError):  # summaries given twice
        dash.dash_attn_fwd(q, k, v, out, 64, 1.5, True, 2, kbar=kb, qbar=torch.zeros(1, nch, 2, 64, device="cuda"))


@pytest.mark.parametrize("b,nq,nk,hq,hkv,B,s,regroup", [
    (1, 1024, 1024, 32, 2, 64, 0.75, False),    # the controlled-sparsity benchmark's heads (g = 16)
    (1, 1024, 1024, 32, 2, 64, 0.9375, True),
    (2, 700, 1000, 8, 2, 64, 0.5, True),        # ragged, nq < nk
    (4, 1, 4096, 32, 8, 64, 0.875, False),      # decode (split-KV path)
])
def test_random_mask_stage2(b, nq, nk, hq, hkv, B, s, regroup):
    """Stage 2 on work lists built from a random routing mask (dash_lists_from_mask) against
    the oracle's Stage 2 given the same routed sets and a uniform prior (bias 0)."""
    q, k, v = _planted(b, nq, nk, hq, hkv, 128, B, "bf16", seed=500 + nq, planted=False)
    g = hq // hkv
    mask = synthetic.random_block_mask(b, nq, nk, hkv, B, s, seed=17, device="cuda")
    lists = dash.lists_from_mask(mask, nk, hkv, B, g, causal=True, regroup=regroup)
    out = torch.empty_like(q)
    dash.dash_sparse_attn_fwd(q, k, v, out, lists, B, True, g)
    assert dash.dash_sync_status() == 0
    nch = dash.n_chunks(nk, B, True)
    bits = ((mask.to(torch.int64) & 0xFFFFFFFF).unsqueeze(-1) >> torch.arange(32, device="cuda")) & 1
    routed = bits.flatten(-2)[..., :nch].to(torch.uint8).cpu().numpy()
    max_tol, mean_tol = 2e-2, 2e-3
    rows = np.arange(nq)
    for bi in range(b):
        r_in = routed[bi]
        ref = oracle.fwd_rows(to_np32(q[bi]), rows, nq, to_np32(k[bi]), to_np32(v[bi]), B, 1.5,
                              w_in=r_in.astype(np.float64), r_in=r_in, want=("out",))
        err = np.abs(to_np32(out[bi]).astype(np.float64) - ref["out"])
        assert err.max() <= max_tol and err.mean() <= mean_tol, (err.max(), err.mean())


@pytest.mark.parametrize("dt,causal", [("bf16", True), ("bf16", False), ("f32", True)])
def test_uniform_all_chunk_prior_is_dense_attention(dt, causal):
    """Stage 2 alone on lists that route every visible chunk with bias 0 equals
    dense softmax attention (the paper's KL-to-uniform statement, Eq. 5)."""
    b, nq, nk, hq, hkv, d, B = 1, 300, 520, 8, 2, 128, 64
    q, k, v = _planted(b, nq, nk, hq, hkv, d, B, dt, seed=7, causal=causal, planted=False)
    g = hq // hkv
    L = dash.make_lists(q, k, B, g, with_rows=False)
    nblk = -(-nk // B)
    for t in range(L.n_tiles):
        i0 = t * L.tile_rows
        last = min(i0 + L.tile_rows, nq) - 1
        hi = min((last + nk - nq) // B, nblk - 1) if causal else nblk - 1
        L.count[:, :, t] = hi + 1
        L.ids[:, :, t, :hi + 1] = torch.arange(hi + 1, dtype=torch.int32, device="cuda")
    L.bias.zero_()
    out = torch.empty_like(q)
    dash.dash_sparse_attn_fwd(q, k, v, out, L, B, causal, g)
    assert dash.dash_sync_status() == 0
    ref = oracle.dense_attention(to_np32(q[0]), to_np32(k[0]), to_np32(v[0]), causal=causal)
    err = np.abs(to_np32(out[0]) - ref)
    tol = (2e-2, 2e-3) if dt == "bf16" else (1e-4, 1e-5)
    assert err.max() <= tol[0] and err.mean() <= tol[1], (err.max(), err.mean())


DECODE_CASES = [
    # b, nq, nk, hq, hkv, d, B, alpha, sigma
    (3, 1, 1000, 8, 2, 128, 64, 1.5, 1.0),     # ragged cache length
    (2, 2, 3000, 8, 2, 128, 64, 1.5, 1e8),     # two new tokens per sequence
    (2, 1, 2048, 16, 1, 128, 128, 2.0, 1.0),   # g = 16 fills the 16-row tile, B = 128
    (2, 1, 1500, 4, 2, 64, 16, 1.25, 1.0),     # d = 64, B = 16
    (1, 1, 50, 4, 1, 128, 64, 1.5, 1.0),       # cache shorter than one chunk
]


@pytest.mark.parametrize("case", DECODE_CASES, ids=[f"d{i}" for i in range(len(DECODE_CASES))])
def test_decode_cases(case):
    b, nq, nk, hq, hkv, d, B, alpha, sigma = case
    q, k, v = _planted(b, nq, nk, hq, hkv, d, B, "bf16", seed=200 + nk)
    out = _run(q, k, v, B, alpha, True, sigma=sigma)
    check_forward(q, k, v, out, B, alpha, True, sigma=sigma, label=f"decode case {case}")


@pytest.mark.parametrize("case", [CASES[0], CASES[3], CASES[6], CASES[7]], ids=["c0", "c3", "c6", "c7"])
def test_two_block_local_window(case):
    """App. B.1.1's local window (DASH_FLAG_LOCAL2): the chunk before the query's own is
    attended in full with bias 0 and not routed; against the oracle with the same window."""
    b, nq, nk, hq, hkv, d, B, dt, alpha, causal, sigma = case
    q, k, v = _planted(b, nq, nk, hq, hkv, d, B, dt, seed=700 + nq, causal=causal)
    out = _run(q, k, v, B, alpha, causal, sigma=sigma, flags=dash.DASH_FLAG_LOCAL2)
    check_forward(q, k, v, out, B, alpha, causal, sigma=sigma, label=f"local2 {case}", local=2)


@pytest.mark.parametrize("case", DECODE_CASES[:2], ids=["d0", "d1"])
def test_two_block_local_window_decode(case):
    b, nq, nk, hq, hkv, d, B, alpha, sigma = case
    q, k, v = _planted(b, nq, nk, hq, hkv, d, B, "bf16", seed=800 + nk)
    out = _run(q, k, v, B, alpha, True, sigma=sigma, flags=dash.DASH_FLAG_LOCAL2)
    check_forward(q, k, v, out, B, alpha, True, sigma=sigma, label=f"local2 decode {case}", local=2)


def test_two_block_local_window_prefill8k_sampled():
    w = synthetic.WORKLOADS["prefill8k"]
    q, k, v = synthetic.make_inputs(w, "cuda")
    out = _run(q, k, v, w.block, w.alpha, True, sigma=1.0, flags=dash.DASH_FLAG_LOCAL2)
    check_forward(q, k, v, out, w.block, w.alpha, True, sigma=1.0, rows=sample_rows(w.nq, w.block, 512, 3),
                  label="local2 prefill8k", local=2)


def test_decode_with_cached_summaries():
    """A chunk-summary cache from dash_pool_keys (kept across decode steps) gives the same result."""
    b, nq, nk, hq, hkv, d, B = 2, 1, 4096, 8, 2, 128, 64
    q, k, v = _planted(b, nq, nk, hq, hkv, d, B, "bf16", seed=77)
    kbar = torch.empty(b, nk // B, hkv, d, dtype=torch.float32, device="cuda")
    dash.dash_pool_keys(k, B, True, kbar)
    a = _run(q, k, v, B, 1.5, True, sigma=1.0)
    c = _run(q, k, v, B, 1.5, True, sigma=1.0, kbar=kbar)
    assert torch.equal(a, c)


@pytest.mark.parametrize("case", [CASES[0], CASES[3], CASES[5], CASES[9]], ids=["c0", "c3", "c5", "c9"])
def test_consecutive_tiles_match_oracle(case):
    """Without regrouping rows by routed-set size (every tile holds consecutive rows)."""
    b, nq, nk, hq, hkv, d, B, dt, alpha, causal, sigma = case
    q, k, v = _planted(b, nq, nk, hq, hkv, d, B, dt, seed=100 + nq, causal=causal)
    out = _run(q, k, v, B, alpha, causal, sigma=sigma, flags=dash.DASH_FLAG_NO_REGROUP)
    check_forward(q, k, v, out, B, alpha, causal, sigma=sigma, label=f"consecutive {case}")


def test_regrouped_rows_are_a_permutation():
    """Regrouping permutes the query rows within windows of 8 tiles: every row appears
    once, tiles are filled before padding, and a tile's rows come from its window."""
    b, nq, nk, hq, hkv, d, B = 2, 1000, 1000, 8, 2, 128, 64
    q, k, v = _planted(b, nq, nk, hq, hkv, d, B, "bf16", seed=3)
    L = dash.make_lists(q, k, B, hq // hkv)
    dash.dash_block_select(q, k, B, 1.5, True, lists=L, sigma=1.0)
    torch.cuda.synchronize()
    rows = L.rows.cpu().numpy()          # [b, hkv, n_tiles, T]
    T, nt = L.tile_rows, L.n_tiles
    for bi in range(b):
        for r in range(hkv):
            flat = rows[bi, r].reshape(-1)
            valid = np.sort(flat[flat >= 0])
            assert np.array_equal(valid, np.arange(nq))
            for t in range(nt):
                tile = rows[bi, r, t]
                w0 = (t // 8) * 8 * T
                assert ((tile < 0) | ((tile >= w0) & (tile < w0 + 8 * T))).all()
    counts = L.count.cpu().numpy()
    assert (counts >= 1).all() and (counts <= L.cap).all()


def test_regrouping_shrinks_the_union():
    """On the planted workload, regrouped tiles stream fewer chunk entries than consecutive ones."""
    w = synthetic.WORKLOADS["prefill8k"]
    q, k, v = synthetic.make_inputs(w, "cuda")
    La = dash.make_lists(q, k, w.block, w.g)
    Lb = dash.make_lists(q, k, w.block, w.g, with_rows=False)
    dash.dash_block_select(q, k, w.block, w.alpha, True, lists=La)
    dash.dash_block_select(q, k, w.block, w.alpha, True, lists=Lb)
    torch.cuda.synchronize()
    ea, eb = int(La.count.sum()), int(Lb.count.sum())
    print(f"[regroup] list entries regrouped {ea} vs consecutive {eb} ({ea / eb:.3f})")
    assert ea < 0.85 * eb


def test_deterministic():
    q, k, v = _planted(1, 512, 512, 8, 2, 128, 64, "bf16", seed=5)
    a = _run(q, k, v, 64, 1.5, True, sigma=1.0)
    b = _run(q, k, v, 64, 1.5, True, sigma=1.0)
    assert torch.equal(a, b)


def test_prefill8k_full():
    w = synthetic.WORKLOADS["prefill8k"]
    q, k, v = synthetic.make_inputs(w, "cuda")
    for sigma in (1e8, 1.0):
        out = _run(q, k, v, w.block, w.alpha, True, sigma=sigma)
        check_forward(q, k, v, out, w.block, w.alpha, True, sigma=sigma, label=f"prefill8k sigma={sigma:g}")


def test_prefill32k_sampled():
    w = synthetic.WORKLOADS["prefill32k"]
    q, k, v = synthetic.make_inputs(w, "cuda")
    rows = sample_rows(w.nq, w.block, 1024, seed=32)
    for sigma in (1e8, 1.0):
        out = _run(q, k, v, w.block, w.alpha, True, sigma=sigma)
        st = check_forward(q, k, v, out, w.block, w.alpha, True, sigma=sigma, rows=rows,
                           label=f"prefill32k sigma={sigma:g}")
    assert 0.6 < st["sparsity"] < 0.9


def test_decode_full():
    w = synthetic.WORKLOADS["decode"]
    q, k, v = synthetic.make_inputs(w, "cuda")
    for sigma in (1e8, 1.0):
        out = _run(q, k, v, w.block, w.alpha, True, sigma=sigma)
        check_forward(q, k, v, out, w.block, w.alpha, True, sigma=sigma, label=f"decode sigma={sigma:g}")


@pytest.mark.parametrize("alpha,sigma", [(1.25, 1.0), (1.5, 1.0), (1.5, 1e8), (2.0, 1.0), (2.0, 1e8)])
def test_prefill128k_sampled(alpha, sigma):
    w = synthetic.WORKLOADS["prefill128k"]
    q, k, v = synthetic.make_inputs(w, "cuda")
    rows = sample_rows(w.nq, w.block, 512, seed=128)
    out = _run(q, k, v, w.block, alpha, True, sigma=sigma)
    check_forward(q, k, v, out, w.block, alpha, True, sigma=sigma, rows=rows,
                  label=f"prefill128k alpha={alpha} sigma={sigma:g}")


# Shapes that take the persistent Stage-1 kernel (more than 256 routing chunks) outside the
# benchmark configurations: GQA groups other than 4 (its general code), d = 64, one, two and
# four lane groups, every alpha with a closed form, nq < nk and a non-causal case.
PERSISTENT_CASES = [
    (1, 5000, 5000, 16, 2, 128, 16, 1.5, True, 1.0),   # g = 8, 312 chunks: one lane group
    (1, 6000, 6000, 4, 2, 64, 16, 1.5, True, 1e8),     # g = 2, d = 64
    (1, 10000, 10000, 8, 2, 128, 16, 2.0, True, 1.0),  # g = 4, 625 chunks: two lane groups
    (1, 3000, 20000, 8, 8, 64, 16, 1.25, True, 1.0),   # g = 1, nq < nk, 1250 chunks: four lane groups
    (1, 2000, 9000, 8, 2, 128, 32, 1.5, False, 1.0),   # non-causal, 282 chunks
]


@pytest.mark.parametrize("case", PERSISTENT_CASES, ids=[f"p{i}" for i in range(len(PERSISTENT_CASES))])
def test_persistent_stage1_shapes(case):
    b, nq, nk, hq, hkv, d, B, alpha, causal, sigma = case
    q, k, v = _planted(b, nq, nk, hq, hkv, d, B, "bf16", seed=nq + hq, causal=causal)
    rows = sample_rows(nq, B, 192, seed=nk)
    out = _run(q, k, v, B, alpha, causal, sigma=sigma)
    check_forward(q, k, v, out, B, alpha, causal, sigma=sigma, rows=rows, label=f"persistent {case}")


def test_row_slices_equal_one_pass():
    """A caller workspace too small for every row's lists makes the forward run its query
    rows in slices; the output (and lse) equals the single-pass forward bit for bit."""
    w = synthetic.WORKLOADS["prefill8k"]
    q, k, v = synthetic.make_inputs(w, "cuda")
    a, c = torch.empty_like(q), torch.empty_like(q)
    la = torch.empty(q.shape[:3], dtype=torch.float32, device="cuda")
    lc = torch.empty_like(la)
    dash.dash_attn_fwd(q, k, v, a, w.block, w.alpha, True, w.g, sigma=1.0, lse=la)
    full = dash.dash_workspace_bytes(1, w.nq, w.nk, w.hq, w.hkv, w.d, w.block)
    ws = torch.empty(full // 3, dtype=torch.uint8, device="cuda")  # room for about a third of the rows
    dash.dash_attn_fwd(q, k, v, c, w.block, w.alpha, True, w.g, sigma=1.0, lse=lc, workspace=ws)
    assert dash.dash_sync_status() == 0
    assert torch.equal(a, c) and torch.equal(la, lc)


def test_prefill128k_batch2_sampled():
    """128K keys at batch 2: the library workspace stays within its 1 GB budget (rows in
    slices) and the second sequence matches the oracle on sampled rows."""
    w = synthetic.WORKLOADS["prefill128k"].with_(batch=2)
    assert dash.dash_workspace_bytes(2, w.nq, w.nk, w.hq, w.hkv, w.d, w.block) <= 10 ** 9
    q, k, v = synthetic.make_inputs(w, "cuda")
    out = _run(q, k, v, w.block, w.alpha, True, sigma=1.0)
    rows = sample_rows(w.nq, w.block, 256, seed=129)
    check_forward(q, k, v, out, w.block, w.alpha, True, sigma=1.0, rows=rows, batches=[1],
                  label="prefill128k batch 2 (second sequence)")

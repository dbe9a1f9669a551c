"""GPU parity of the backward pass (dash_attn_bwd through the C ABI) against the fp64
oracle of oracle/backward.py on the same seeded inputs, plus the forward's lse output.

Small problems are differentiated in full (every element of dQ, dK, dV); the 8K
workload is checked on sampled rows of dQ (a row's dQ depends on that row alone) and,
for dK and dV, by identities that hold at any size:
  * sum over keys of dV = sum over the group's rows and heads of dO (rows of P sum to 1);
  * sum over keys of dK = 0 (each row of dl sums to zero, each row of the entmax
    Jacobian sums to zero, and mean pooling spreads a summary's gradient over its keys).

Tolerance (bf16): the gradients are returned in bf16 (relative rounding 2^-9) and the
tensor-core path rounds P and dl to bf16 before their products; max-abs error <= 2e-2 of
the largest reference magnitude, mean-abs error <= 1e-2 of the mean magnitude.  fp32
inputs (CUDA-core path in fp32): 1e-4 and 1e-5 of the same scales."""
import numpy as np
import pytest
import torch

import oracle
import sparse_hierarchical_attention_block_b200 as dash
import synthetic
from oracle.backward import backward as oracle_backward
from parity import sample_rows, to_np32

pytestmark = pytest.mark.gpu

TOL = {torch.bfloat16: (2e-2, 1e-2), torch.float32: (1e-4, 1e-5)}


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.fail("the gpu tests need a CUDA device")
    dash.load_library()
    oracle.set_threads(oracle.max_threads())
    yield
    dash.dash_release()


def _inputs(b, nq, nk, hq, hkv, d, B, dt, seed, causal=True):
    w = synthetic.Workload("bwd", b, nq, nk, hq, hkv, d, B, 1.5, causal, dt, seed, True, amax_key="b64")
    q, k, v = synthetic.make_inputs(w, "cuda")
    gen = torch.Generator(device="cuda").manual_seed(seed + 1000)
    dout = torch.randn(q.shape, generator=gen, device="cuda").to(q.dtype)
    return q, k, v, dout


def _fwd_bwd(q, k, v, dout, B, alpha, causal, **opts):
    g = q.shape[2] // k.shape[2]
    out = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device)
    dash.dash_attn_fwd(q, k, v, out, B, alpha, causal, g, lse=lse, **opts)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    dash.dash_attn_bwd(q, k, v, out, dout, lse, dq, dk, dv, B, alpha, causal, g, **opts)
    assert dash.dash_sync_status() == 0
    return out, lse, dq, dk, dv


def _close(name, got, ref, dtype, label):
    tmax, tmean = TOL[dtype]
    got = got.astype(np.float64)
    err = np.abs(got - ref)
    scale_max = max(np.abs(ref).max(), 1e-30)
    scale_mean = max(np.abs(ref).mean(), 1e-30)
    print(f"[bwd] {label} {name}: max_err={err.max():.3g} (ref max {scale_max:.3g}) "
          f"mean_err={err.mean():.3g} (ref mean {scale_mean:.3g})")
    assert err.max() <= tmax * scale_max, f"{label} {name}: max-abs error {err.max()} > {tmax} x {scale_max}"
    assert err.mean() <= tmean * scale_mean, f"{label} {name}: mean-abs error {err.mean()} > {tmean} x {scale_mean}"


CASES = [
    # b, nq, nk, hq, hkv, d, B, dtype, alpha, causal, sigma, flags
    (1, 256, 256, 4, 2, 128, 64, "bf16", 1.5, True, 1.0, 0),
    (2, 300, 300, 8, 2, 128, 64, "bf16", 1.5, True, 3.0, 0),          # ragged tail, two batch elements
    (1, 256, 256, 4, 1, 128, 64, "bf16", 2.0, True, 1.0, 0),           # sparsemax, g = 4
    (1, 200, 256, 4, 2, 64, 16, "bf16", 1.25, True, 1.0, 0),           # nq < nk, B = 16, d = 64
    (1, 150, 300, 4, 2, 64, 64, "bf16", 1.5, False, 1.0, 0),           # non-causal, partial chunk routed
    (1, 300, 300, 4, 2, 128, 64, "bf16", 1.5, True, 1.0, "local2"),    # two-block local window
    (1, 512, 512, 8, 2, 128, 128, "bf16", 1.5, True, 1.0, 0),          # B = 128
    (1, 200, 200, 6, 2, 64, 32, "bf16", 1.5, True, 1.0, 0),            # g = 3 (CUDA-core path)
    (1, 256, 256, 4, 2, 128, 64, "bf16", 1.5, True, 1e8, 0),           # the default sigma
    (1, 256, 256, 2, 1, 64, 64, "f32", 1.5, True, 1.0, 0),             # fp32
]


@pytest.mark.parametrize("case", CASES, ids=[f"b{i}" for i in range(len(CASES))])
def test_backward_matches_oracle(case):
    b, nq, nk, hq, hkv, d, B, dt, alpha, causal, sigma, flags = case
    q, k, v, dout = _inputs(b, nq, nk, hq, hkv, d, B, dt, seed=900 + nq + d, causal=causal)
    opts = {"sigma": sigma}
    local = 1
    if flags == "local2":
        opts["flags"] = dash.DASH_FLAG_LOCAL2
        local = 2
    out, lse, dq, dk, dv = _fwd_bwd(q, k, v, dout, B, alpha, causal, **opts)
    for bi in range(b):
        ref = oracle_backward(to_np32(q[bi]), to_np32(k[bi]), to_np32(v[bi]), to_np32(dout[bi]).astype(np.float64),
                              B, alpha, sigma=sigma, causal=causal, local=local)
        label = f"case {case} batch {bi}"
        _close("dQ", to_np32(dq[bi]), ref["dQ"], q.dtype, label)
        _close("dK", to_np32(dk[bi]), ref["dK"], q.dtype, label)
        _close("dV", to_np32(dv[bi]), ref["dV"], q.dtype, label)


@pytest.mark.parametrize("case", [CASES[0], CASES[6]], ids=["b0", "b6"])
def test_backward_simt_path_matches_oracle(case):
    """The CUDA-core Stage-2 backward (forced) meets the same bar."""
    b, nq, nk, hq, hkv, d, B, dt, alpha, causal, sigma, _ = case
    q, k, v, dout = _inputs(b, nq, nk, hq, hkv, d, B, dt, seed=900 + nq + d, causal=causal)
    out, lse, dq, dk, dv = _fwd_bwd(q, k, v, dout, B, alpha, causal, sigma=sigma, flags=dash.DASH_FLAG_FORCE_SIMT)
    ref = oracle_backward(to_np32(q[0]), to_np32(k[0]), to_np32(v[0]), to_np32(dout[0]).astype(np.float64), B,
                          alpha, sigma=sigma, causal=causal)
    for name, got in (("dQ", dq), ("dK", dk), ("dV", dv)):
        _close(name, to_np32(got[0]), ref[name], q.dtype, f"simt {case}")


def test_forward_lse_is_dense_logsumexp():
    """lse of Stage 2 on lists that route every visible chunk with bias 0 is the log-sum-exp
    of dense causal attention's logits, computed here in fp64."""
    b, nq, nk, hq, hkv, d, B = 1, 300, 520, 8, 2, 128, 64
    w = synthetic.Workload("lse", b, nq, nk, hq, hkv, d, B, 1.5, True, "bf16", 7, False)
    q, k, v = synthetic.make_inputs(w, "cuda")
    g = hq // hkv
    L = dash.make_lists(q, k, B, g, with_rows=False)
    nblk = -(-nk // B)
    for t in range(L.n_tiles):
        last = min(t * L.tile_rows + L.tile_rows, nq) - 1
        hi = min((last + nk - nq) // B, nblk - 1)
        L.count[:, :, t] = hi + 1
        L.ids[:, :, t, :hi + 1] = torch.arange(hi + 1, dtype=torch.int32, device="cuda")
    L.bias.zero_()
    out = torch.empty_like(q)
    lse = torch.empty(b, nq, hq, dtype=torch.float32, device="cuda")
    dash.dash_sparse_attn_fwd(q, k, v, out, L, B, True, g, lse=lse)
    assert dash.dash_sync_status() == 0
    Q = q[0].double().cpu().numpy()
    K = k[0].double().cpu().numpy()
    z = np.einsum("ihd,jhd->hij", Q, np.repeat(K, g, axis=1)) / np.sqrt(d)
    pos = np.arange(nq)[:, None] + nk - nq
    z = np.where(np.arange(nk)[None, :] <= pos, z, -np.inf)
    zmax = z.max(-1, keepdims=True)
    ref = (zmax[..., 0] + np.log(np.exp(z - zmax).sum(-1))).T  # [nq, hq]
    err = np.abs(lse[0].cpu().numpy() - ref).max()
    assert err <= 1e-3, err


def test_backward_prefill8k_sampled_and_identities():
    w = synthetic.WORKLOADS["prefill8k"]
    q, k, v = synthetic.make_inputs(w, "cuda")
    gen = torch.Generator(device="cuda").manual_seed(88)
    dout = torch.randn(q.shape, generator=gen, device="cuda").to(q.dtype)
    sigma = 1.0
    out, lse, dq, dk, dv = _fwd_bwd(q, k, v, dout, w.block, w.alpha, True, sigma=sigma)
    # identities over every key
    g = w.g
    sum_dv = dv[0].double().sum(0)                                          # [hkv, d]
    sum_do = dout[0].double().view(w.nq, w.hkv, g, w.d).sum((0, 2))        # [hkv, d]
    e_dv = (sum_dv - sum_do).abs().max().item()
    assert e_dv <= 2e-2 * sum_do.abs().max().item() + 0.5, e_dv
    sum_dk = dk[0].double().sum(0).abs().max().item()
    assert sum_dk <= 2e-2 * dk[0].double().abs().sum(0).max().item() / 8 + 0.5, sum_dk
    # sampled rows of dQ against the oracle
    rows = sample_rows(w.nq, w.block, 48, seed=81)
    ref = oracle_backward(to_np32(q[0]), to_np32(k[0]), to_np32(v[0]), to_np32(dout[0]).astype(np.float64),
                          w.block, w.alpha, sigma=sigma, rows=rows)
    got = to_np32(dq[0].index_select(0, torch.from_numpy(rows).cuda()))
    _close("dQ (sampled rows)", got, ref["dQ"], q.dtype, "prefill8k")


def test_backward_deterministic():
    """dQ and dV are bit-for-bit reproducible; dK takes the summaries' gradient through
    fp32 atomic sums, so it may differ in the last bit between runs."""
    q, k, v, dout = _inputs(1, 512, 512, 8, 2, 128, 64, "bf16", seed=5)
    a = _fwd_bwd(q, k, v, dout, 64, 1.5, True, sigma=1.0)
    b = _fwd_bwd(q, k, v, dout, 64, 1.5, True, sigma=1.0)
    assert torch.equal(a[2], b[2]) and torch.equal(a[4], b[4])
    assert torch.allclose(a[3].float(), b[3].float(), rtol=1e-2, atol=1e-3)

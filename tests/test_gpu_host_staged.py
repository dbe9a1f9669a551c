"""The host-staged forward (dash_attn_fwd_host): host inputs and output, query rows in
slices whose copies overlap the computation.  Its output must be bit-identical to the
forward on the device tensors, for any slice count, with and without a causal mask."""
import pytest
import torch

import sparse_hierarchical_attention_block_b200 as dash
import synthetic

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.fail("the gpu tests need a CUDA device")
    dash.load_library()
    yield
    dash.dash_release()


def _inputs(b, nq, nk, hq, hkv, d, seed):
    w = synthetic.Workload("staged", b, nq, nk, hq, hkv, d, 64, 1.5, True, "bf16", seed, True, amax_key="b64")
    return synthetic.make_inputs(w, "cpu")


def _staged(q, k, v, block, alpha, causal, n_slices, **opts):
    qh, kh, vh = (t.pin_memory() for t in (q, k, v))
    oh = torch.full(q.shape, float("nan"), dtype=q.dtype).pin_memory()
    qd, kd, vd = (torch.empty_like(t, device="cuda") for t in (q, k, v))
    od = torch.empty_like(qd)
    dash.dash_attn_fwd_host(qh, kh, vh, oh, qd, kd, vd, od, block, alpha, causal, n_slices=n_slices, **opts)
    torch.cuda.current_stream().synchronize()
    assert dash.dash_sync_status() == 0
    return oh


@pytest.mark.parametrize("b,nq,nk,causal", [(2, 3000, 3000, True), (1, 1000, 2500, True), (1, 700, 1500, False)])
@pytest.mark.parametrize("n_slices", [1, 3, 0])
def test_host_staged_equals_device_forward(b, nq, nk, causal, n_slices):
    q, k, v = _inputs(b, nq, nk, 8, 2, 128, seed=21)
    ref = torch.empty(q.shape, dtype=q.dtype, device="cuda")
    dash.dash_attn_fwd(q.cuda(), k.cuda(), v.cuda(), ref, 64, 1.5, causal, 4, sigma=1.0)
    out = _staged(q, k, v, 64, 1.5, causal, n_slices, sigma=1.0)
    assert torch.equal(out, ref.cpu())


def test_host_staged_misuse_is_rejected():
    q, k, v = _inputs(1, 512, 512, 8, 2, 64, seed=22)
    qh, kh, vh = (t.pin_memory() for t in (q, k, v))
    oh = torch.empty(q.shape, dtype=q.dtype).pin_memory()
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    od = torch.empty_like(qd)
    with pytest.raises(dash.DashError):  # a device buffer of another shape
        dash.dash_attn_fwd_host(qh, kh, vh, oh, qd[:, :256], kd, vd, od[:, :256], 64, 1.5, True)
    with pytest.raises(dash.DashError):  # lse is not produced by this entry point
        dash.dash_attn_fwd_host(qh, kh, vh, oh, qd, kd, vd, od, 64, 1.5, True,
                                lse=torch.empty(1, 512, 8, device="cuda"))
    with pytest.raises(ValueError):  # host tensors on the host, device buffers on the device
        dash.dash_attn_fwd_host(qd, kh, vh, oh, qd, kd, vd, od, 64, 1.5, True)

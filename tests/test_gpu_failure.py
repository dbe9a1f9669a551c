"""Failure detection on the GPU without a fault: a bounded device-side wait that
runs out is reported as DASH_ERR_DEVICE_TIMEOUT by dash_sync_status, and the
context stays usable.

Under DASH_FLAG_TEST_TIMEOUT the tensor-core Stage 2 issues no copy and no MMA:
its MMA thread waits on a barrier that nothing arrives at, gives up after
20 ms, the other roles see the CTA's abort flag, TMEM is freed and the kernel
returns.  Nothing traps, faults or hangs."""
import pytest
import torch

import sparse_hierarchical_attention_block_b200 as dash
import synthetic

pytestmark = pytest.mark.gpu


def test_device_timeout_is_reported_and_recoverable():
    w = synthetic.Workload("t", 1, 256, 256, 8, 2, 128, 64, 1.5, True, "bf16", 9, True, amax_key="b64")
    q, k, v = synthetic.make_inputs(w, "cuda")
    out = torch.zeros_like(q)
    dash.dash_attn_fwd(q, k, v, out, 64, 1.5, True, 4, flags=dash.DASH_FLAG_TEST_TIMEOUT)
    assert dash.dash_sync_status() == dash.DASH_ERR_DEVICE_TIMEOUT
    # the flag is cleared and the next call runs normally
    assert dash.dash_sync_status() == dash.DASH_OK
    ref = torch.empty_like(q)
    dash.dash_attn_fwd(q, k, v, ref, 64, 1.5, True, 4, flags=dash.DASH_FLAG_FORCE_SIMT)
    dash.dash_attn_fwd(q, k, v, out, 64, 1.5, True, 4)
    assert dash.dash_sync_status() == dash.DASH_OK
    assert (out.float() - ref.float()).abs().max().item() < 2e-2


def test_errors_surface_as_exceptions():
    w = synthetic.Workload("t", 1, 128, 128, 4, 2, 64, 64, 1.5, True, "bf16", 9, False)
    q, k, v = synthetic.make_inputs(w, "cuda")
    out = torch.empty_like(q)
    with pytest.raises(dash.DashError) as e:
        dash.dash_attn_fwd(q, k, v, out, 48, 1.5, True, 2)
    assert e.value.code == dash.DASH_ERR_UNSUPPORTED
    with pytest.raises(dash.DashError):
        dash.dash_attn_fwd(q, k, v, out, 64, 0.5, True, 2)

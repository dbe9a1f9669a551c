"""The random routing masks of the controlled-sparsity Stage-2 benchmark (host logic)."""
import pytest
import torch

import synthetic


def _unpack(m, n_chunks):
    bits = ((m.to(torch.int64) & 0xFFFFFFFF).unsqueeze(-1) >> torch.arange(32)) & 1
    return bits.flatten(-2)[..., :n_chunks].bool()


@pytest.mark.parametrize("nq,nk,B,s,causal", [(300, 1000, 64, 0.75, True), (1, 4096, 64, 0.875, True),
                                              (128, 2048, 32, 0.9375, True), (50, 1000, 64, 0.5, False)])
def test_exact_count_of_routable_chunks(nq, nk, B, s, causal):
    n_chunks = nk // B if causal else -(-nk // B)
    m = synthetic.random_block_mask(2, nq, nk, 3, B, s, seed=4, causal=causal)
    assert m.shape == (2, nq, 3, max((n_chunks + 31) // 32, 1)) and m.dtype == torch.int32
    bits = _unpack(m, n_chunks)
    if causal:
        n_vis = torch.clamp((torch.arange(nq) + nk - nq) // B, max=n_chunks)
    else:
        n_vis = torch.full((nq,), n_chunks)
    want = torch.round((1 - s) * n_vis.double()).long()
    assert torch.equal(bits.sum(-1), want.view(1, -1, 1).expand(2, nq, 3))
    c = torch.arange(n_chunks)
    assert not (bits & (c.view(1, 1, 1, -1) >= n_vis.view(1, -1, 1, 1))).any()
    # padding bits past the last chunk stay clear
    full = ((m.to(torch.int64) & 0xFFFFFFFF).unsqueeze(-1) >> torch.arange(32)) & 1
    assert not full.flatten(-2)[..., n_chunks:].any()


def test_seeded_and_spread():
    a = synthetic.random_block_mask(1, 512, 8192, 2, 64, 0.75, seed=1)
    assert torch.equal(a, synthetic.random_block_mask(1, 512, 8192, 2, 64, 0.75, seed=1))
    assert not torch.equal(a, synthetic.random_block_mask(1, 512, 8192, 2, 64, 0.75, seed=2))
    bits = _unpack(a, 128)
    # every routable chunk of the last rows is chosen about (1 - s) of the time
    freq = bits[0, -64:, :, :120].float().mean(dim=(0, 1))
    assert freq.min() > 0.05 and freq.max() < 0.5


def test_extremes():
    n_chunks = 1000 // 64
    full = _unpack(synthetic.random_block_mask(1, 1000, 1000, 1, 64, 0.0, seed=0), n_chunks)
    n_vis = torch.clamp(torch.arange(1000) // 64, max=n_chunks)
    assert torch.equal(full.sum(-1)[0, :, 0], n_vis)
    none = synthetic.random_block_mask(1, 1000, 1000, 1, 64, 1.0, seed=0)
    assert not none.any()

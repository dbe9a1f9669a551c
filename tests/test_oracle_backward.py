"""Pins of the oracle's backward pass (oracle/backward.py) against what the mathematics
fixes: central finite differences of the C forward oracle, the sigma -> infinity limit
(plain masked softmax attention, differentiated by torch autograd), and the alpha-entmax
Jacobian against finite differences of the C entmax."""
import numpy as np
import pytest
import torch

import oracle
from oracle.backward import backward, entmax_vjp

STEP = 2.0 ** -14  # exact in float32 on the 2^-6 input grid below


def _grid_case(seed, nq, nk, hq, hkv, d, qscale=2.0):
    """Inputs on a 2^-6 grid (so +- STEP stays exact in float32), with every chunk score
    at least 1e-3 away from every threshold (no support changes under the steps)."""
    for s in range(seed, seed + 200):
        rng = np.random.default_rng(s)
        Q = (rng.integers(-128, 128, size=(nq, hq, d)) / 64 * qscale).astype(np.float32)
        K = (rng.integers(-128, 128, size=(nk, hkv, d)) / 64).astype(np.float32)
        V = (rng.integers(-128, 128, size=(nk, hkv, d)) / 64).astype(np.float32)
        dO = rng.normal(size=(nq, hq, d))
        yield Q, K, V, dO


def _safe(Q, K, V, B, alpha, causal, local):
    x = oracle.fwd(Q, K, V, B, alpha, causal=causal, want=("xmt",), local=local)["xmt"]
    return np.nanmin(np.abs(x)) > 1e-3 if np.isfinite(x).any() else True


def _fd(Q, K, V, dO, B, alpha, sigma, causal, local):
    def loss(q, k, v):
        out = oracle.fwd(q, k, v, B, alpha, sigma=sigma, causal=causal, want=("out",), local=local)["out"]
        return float((out * dO).sum())

    grads = {}
    for name, X in (("dQ", Q), ("dK", K), ("dV", V)):
        G = np.zeros(X.shape)
        for idx in np.ndindex(X.shape):
            args = {"dQ": Q, "dK": K, "dV": V}
            Xp, Xm = X.copy(), X.copy()
            Xp[idx] += STEP
            Xm[idx] -= STEP
            args[name] = Xp
            lp = loss(args["dQ"], args["dK"], args["dV"])
            args[name] = Xm
            lm = loss(args["dQ"], args["dK"], args["dV"])
            G[idx] = (lp - lm) / (2 * STEP)
        grads[name] = G
    return grads


@pytest.mark.parametrize("alpha,sigma,hq,hkv,causal,local", [
    (1.5, 1.0, 2, 1, True, 1),
    (2.0, 3.0, 4, 2, True, 1),     # sparsemax, a group of two heads per kv head
    (1.25, 1.0, 2, 1, True, 1),
    (1.5, 1.0, 2, 1, False, 1),    # non-causal: every chunk routable, the partial one too
    (1.5, 1.0, 2, 1, True, 2),     # the two-block local window
])
def test_backward_matches_finite_differences(alpha, sigma, hq, hkv, causal, local):
    nq, nk, d, B = (36, 44, 4, 8) if not causal else (40, 40, 4, 8)
    for Q, K, V, dO in _grid_case(11, nq, nk, hq, hkv, d):
        if _safe(Q, K, V, B, alpha, causal, local):
            break
    else:
        pytest.fail("no input without near-threshold chunks")
    got = backward(Q, K, V, dO, B, alpha, sigma=sigma, causal=causal, local=local)
    fd = _fd(Q, K, V, dO, B, alpha, sigma, causal, local)
    for name in ("dQ", "dK", "dV"):
        err = np.abs(got[name] - fd[name]).max()
        assert err <= 1e-6 * max(1.0, np.abs(fd[name]).max()), (name, err)
    # the routing path (through the prior) is exercised: it moves the gradient at this sigma
    plain = backward(Q, K, V, dO, B, alpha, sigma=1e12, causal=causal, local=local)
    assert np.abs(plain["dQ"] - got["dQ"]).max() > 1e-3


def test_sigma_to_infinity_is_masked_attention_gradient():
    """With sigma -> infinity the prior bias is constant: the gradient is that of softmax
    attention restricted to the routed tokens and the local window (torch autograd, fp64)."""
    nq, nk, hq, hkv, d, B = 48, 48, 4, 2, 8, 8
    Q, K, V, dO = next(_grid_case(3, nq, nk, hq, hkv, d))
    got = backward(Q, K, V, dO, B, 1.5, sigma=1e12)
    routed = oracle.fwd(Q, K, V, B, 1.5, want=("routed",))["routed"].astype(bool)  # [nq, hkv, nch]
    mask = np.zeros((nq, hkv, nk), dtype=bool)
    for i in range(nq):
        c_i = i // B
        mask[i, :, c_i * B:i + 1] = True
        for r in range(hkv):
            for c in np.nonzero(routed[i, r])[0]:
                mask[i, r, c * B:(c + 1) * B] = True
    q = torch.tensor(Q, dtype=torch.float64, requires_grad=True)
    k = torch.tensor(K, dtype=torch.float64, requires_grad=True)
    v = torch.tensor(V, dtype=torch.float64, requires_grad=True)
    g = hq // hkv
    kk, vv = k.repeat_interleave(g, 1), v.repeat_interleave(g, 1)                 # [nk, hq, d]
    logits = torch.einsum("ihd,jhd->hij", q, kk) / np.sqrt(d)
    m = torch.tensor(mask).repeat_interleave(g, 1).permute(1, 0, 2)                # [hq, nq, nk]
    out = torch.einsum("hij,jhd->ihd", torch.softmax(logits.masked_fill(~m, float("-inf")), -1), vv)
    (out * torch.tensor(dO)).sum().backward()
    for name, t in (("dQ", q), ("dK", k), ("dV", v)):
        assert np.abs(got[name] - t.grad.numpy()).max() < 1e-9, name


@pytest.mark.parametrize("alpha", [1.25, 1.5, 2.0])
def test_entmax_jacobian(alpha):
    """entmax_vjp is the transpose of the Jacobian of the C entmax (central differences);
    for sparsemax it is the projection dp - mean over the support."""
    rng = np.random.default_rng(int(alpha * 100))
    s = rng.normal(size=12) * 2
    p = oracle.entmax_sort(s, alpha)[0]
    h = 1e-6
    J = np.zeros((12, 12))
    for c in range(12):
        e = np.zeros(12)
        e[c] = h
        J[:, c] = (oracle.entmax_sort(s + e, alpha)[0] - oracle.entmax_sort(s - e, alpha)[0]) / (2 * h)
    for _ in range(3):
        v = rng.normal(size=12)
        np.testing.assert_allclose(entmax_vjp(p, v, alpha), J.T @ v, atol=1e-7)
    np.testing.assert_allclose(J, J.T, atol=1e-7)
    if alpha == 2.0:
        v = rng.normal(size=12)
        S = p > 0
        want = np.where(S, v - v[S].mean(), 0.0)
        np.testing.assert_allclose(entmax_vjp(p, v, alpha), want, atol=1e-12)


BACKWARD_MUTATIONS = [
    ("group average not divided by g", "ds = entmax_vjp(p, dw[:nvis] / g, alpha)", "ds = entmax_vjp(p, dw[:nvis], alpha)"),
    ("prior bias gradient not centred by mu", "dlogw = (G - G.mean()) / sigma", "dlogw = G / sigma"),
    ("entmax Jacobian without the threshold's move", "return u * (dp - (u @ dp) / su)", "return u * dp"),
    ("pooling gradient not divided by the chunk size", "dK[sl] += dKbar[c] / sizes[c]", "dK[sl] += dKbar[c]"),
]


def test_backward_pins_catch_planted_mistakes():
    """Each planted mistake in a copy of the backward disagrees with the finite differences."""
    import types
    from pathlib import Path

    src = (Path(oracle.__file__).parent / "backward.py").read_text()
    alpha, sigma, hq, hkv, B = 2.0, 3.0, 4, 2, 8
    for Q, K, V, dO in _grid_case(11, 40, 40, hq, hkv, 4):
        if _safe(Q, K, V, B, alpha, True, 1):
            break
    fd = _fd(Q, K, V, dO, B, alpha, sigma, True, 1)
    for name, orig, mut in BACKWARD_MUTATIONS:
        assert src.count(orig) == 1, name
        mod = types.ModuleType("oracle.mutated_backward")
        mod.__package__ = "oracle"
        exec(compile(src.replace(orig, mut), "mutated_backward", "exec"), mod.__dict__)
        got = mod.backward(Q, K, V, dO, B, alpha, sigma=sigma)
        worst = max(np.abs(got[n] - fd[n]).max() / max(1.0, np.abs(fd[n]).max()) for n in ("dQ", "dK", "dV"))
        assert worst > 1e-4, "the pins miss: " + name


def _fd_qbar(Q, K, V, dO, Qb, B, alpha, sigma):
    def loss(qb, k):
        out = oracle.fwd(Q, k, V, B, alpha, sigma=sigma, want=("out",), qbar=qb)["out"]
        return float((out * dO).sum())

    grads = {}
    for name, X in (("dQbar", Qb), ("dK", K)):
        G = np.zeros(X.shape)
        for idx in np.ndindex(X.shape):
            Xp, Xm = X.copy(), X.copy()
            Xp[idx] += STEP
            Xm[idx] -= STEP
            if name == "dQbar":
                G[idx] = (loss(Xp, K) - loss(Xm, K)) / (2 * STEP)
            else:
                G[idx] = (loss(Qb, Xp) - loss(Qb, Xm)) / (2 * STEP)
        grads[name] = G
    return grads


def test_learned_summary_gradients():
    """With a learned summary query the keys also reach Stage 1 through the pooling softmax,
    and the query itself gets a gradient (finite differences); that gradient falls as
    1/sigma (the summary query becomes untrainable as the prior weakens, App. F.5)."""
    alpha, sigma, B, nq, nk, hq, hkv, d = 1.5, 1.0, 8, 40, 40, 2, 1, 4
    for Q, K, V, dO in _grid_case(21, nq, nk, hq, hkv, d):
        Qb = (np.random.default_rng(int(Q[0, 0, 0] * 64) + 300).integers(-96, 96, size=(nk // B, hkv, d)) / 64
              ).astype(np.float32)
        x = oracle.fwd(Q, K, V, B, alpha, want=("xmt",), qbar=Qb)["xmt"]
        if np.nanmin(np.abs(x)) > 1e-3:
            break
    got = backward(Q, K, V, dO, B, alpha, sigma=sigma, qbar=Qb)
    fd = _fd_qbar(Q, K, V, dO, Qb, B, alpha, sigma)
    for name in ("dQbar", "dK"):
        err = np.abs(got[name] - fd[name]).max()
        assert err <= 1e-6 * max(1.0, np.abs(fd[name]).max()), (name, err)
    assert np.abs(got["dQbar"]).max() > 1e-3
    a = backward(Q, K, V, dO, B, alpha, sigma=1e5, qbar=Qb)["dQbar"]
    b = backward(Q, K, V, dO, B, alpha, sigma=1e6, qbar=Qb)["dQbar"]
    np.testing.assert_allclose(a, 10 * b, rtol=1e-3, atol=1e-12)


def test_learned_pooling_backward_pin_catches_a_planted_mistake():
    import types
    from pathlib import Path

    src = (Path(oracle.__file__).parent / "backward.py").read_text()
    orig, mut = "e = a * (da - (a * da).sum(axis=0))", "e = a * da"
    assert src.count(orig) == 1
    mod = types.ModuleType("oracle.mutated_backward")
    mod.__package__ = "oracle"
    exec(compile(src.replace(orig, mut), "mutated_backward", "exec"), mod.__dict__)
    alpha, B, nq, nk, hq, hkv, d = 1.5, 8, 40, 40, 2, 1, 4
    Q, K, V, dO = next(_grid_case(21, nq, nk, hq, hkv, d))
    Qb = (np.random.default_rng(5).integers(-96, 96, size=(nk // B, hkv, d)) / 64).astype(np.float32)
    fd = _fd_qbar(Q, K, V, dO, Qb, B, alpha, 1.0)
    got = mod.backward(Q, K, V, dO, B, alpha, sigma=1.0, qbar=Qb)
    assert np.abs(got["dQbar"] - fd["dQbar"]).max() > 1e-4

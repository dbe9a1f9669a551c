"""Pins of the fp64 oracle against what the DashAttention paper and the
mathematics fix (CPU only).

Each test checks the oracle against something other than itself: hand-derived
closed forms, an independent solver (a QP for the simplex projection, brute
force over supports, a library softmax / scaled_dot_product_attention),
invariants, limits, or the identity of the paper's Proposition 1 between two
independently coded routes.  The mutation test (test_oracle_mutations.py)
shows that plausible mistakes planted in the oracle fail at least one of
these.
"""
import itertools
import json
from pathlib import Path

import numpy as np
import pytest
import scipy.optimize
import torch

import oracle

GOLDEN = Path(__file__).resolve().parent / "golden"


# ---------------------------------------------------------------- entmax ----

def test_entmax_closed_form_fixtures():
    """Hand-derived cases of Eq. 2 / Eq. 13 (tests/golden/entmax_closed_form.json)."""
    cases = json.loads((GOLDEN / "entmax_closed_form.json").read_text())["cases"]
    for c in cases:
        p, tau, _ = oracle.entmax_sort(c["s"], c["alpha"])
        np.testing.assert_allclose(p, c["p"], rtol=0, atol=1e-13, err_msg=c["derivation"])
        assert abs(tau - c["tau"]) < 1e-13, c["derivation"]
        pb, taub = oracle.entmax_bisect(c["s"], c["alpha"], 200)
        np.testing.assert_allclose(pb, c["p"], rtol=0, atol=1e-12, err_msg=c["derivation"])


def _simplex_projection_qp(z):
    """argmin ||p - z||^2 over the simplex, by a generic constrained solver."""
    n = z.size
    res = scipy.optimize.minimize(lambda p: 0.5 * np.sum((p - z) ** 2), np.full(n, 1.0 / n),
                                  jac=lambda p: p - z, method="SLSQP",
                                  bounds=[(0.0, None)] * n,
                                  constraints=[{"type": "eq", "fun": lambda p: p.sum() - 1.0,
                                                "jac": lambda p: np.ones_like(p)}],
                                  options={"ftol": 1e-15, "maxiter": 500})
    return res.x


@pytest.mark.parametrize("n", [5, 12, 40])
def test_alpha2_is_sparsemax_projection(n):
    """alpha = 2 is the Euclidean projection onto the simplex (App. A, Special Cases)."""
    rng = np.random.default_rng(n)
    for _ in range(5):
        z = rng.normal(size=n) * rng.uniform(0.2, 3.0)
        p, _, _ = oracle.entmax_sort(z, 2.0)
        q = _simplex_projection_qp(z)
        np.testing.assert_allclose(p, q, atol=2e-7)


def test_alpha_to_one_approaches_softmax():
    """alpha -> 1+ recovers softmax (Sec. 2; App. A), error shrinking with alpha - 1."""
    rng = np.random.default_rng(1)
    s = rng.normal(size=30) * 2.0
    ref = np.exp(s - s.max())
    ref /= ref.sum()
    errs = []
    for a in (1.1, 1.01, 1.001):
        p, _, _ = oracle.entmax_sort(s, a)
        errs.append(np.abs(p - ref).max())
    assert errs[0] > errs[1] > errs[2]
    assert errs[2] < 5e-3
    # roughly linear in alpha - 1
    assert errs[1] / errs[2] > 5


@pytest.mark.parametrize("alpha", [1.25, 1.5, 2.0, 3.0])
def test_entmax_invariants(alpha):
    """Output on the simplex; shift invariance; permutation equivariance (Eq. 2)."""
    rng = np.random.default_rng(int(alpha * 100))
    for n in (1, 2, 7, 64, 513):
        s = rng.normal(size=n) * 1.5
        p, tau, ks = oracle.entmax_sort(s, alpha)
        assert (p >= 0).all()
        assert abs(p.sum() - 1.0) < 1e-12
        assert ks == int((p > 0).sum())
        c = 0.731
        p2, tau2, _ = oracle.entmax_sort(s + c, alpha)
        np.testing.assert_allclose(p2, p, atol=1e-12)
        assert abs(tau2 - (tau + (alpha - 1) * c)) < 1e-12
        perm = rng.permutation(n)
        p3, _, _ = oracle.entmax_sort(s[perm], alpha)
        np.testing.assert_allclose(p3, p[perm], atol=1e-13)


def _brute_force_entmax(s, alpha):
    """Enumerate every support S; keep the one whose threshold is self-consistent."""
    x = (alpha - 1.0) * np.asarray(s, dtype=np.float64)
    k = 1.0 / (alpha - 1.0)
    n = x.size
    found = []
    for m in range(1, n + 1):
        for S in itertools.combinations(range(n), m):
            xs = x[list(S)]
            lo = xs.min()
            f = lambda t: np.sum((xs - t) ** k) - 1.0  # noqa: E731
            if f(lo) >= 0:       # the root must lie strictly below min over S
                continue
            a = lo - 1.0
            while f(a) < 0:
                a -= 1.0
            tau = scipy.optimize.brentq(f, a, lo, xtol=1e-16, rtol=1e-15, maxiter=500)
            rest = np.delete(x, list(S))
            if rest.size == 0 or rest.max() <= tau:
                found.append((S, tau))
    assert len(found) == 1, found
    S, tau = found[0]
    p = np.zeros(n)
    p[list(S)] = (x[list(S)] - tau) ** k
    return p, tau


@pytest.mark.parametrize("alpha", [1.25, 1.5, 2.0, 2.5])
def test_sort_bisect_bruteforce_agree(alpha):
    """Sort-based exact tau == bisection == brute force over supports (n <= 10)."""
    rng = np.random.default_rng(7)
    for n in (1, 2, 3, 6, 10):
        for _ in range(3):
            s = rng.normal(size=n) * rng.uniform(0.3, 4.0)
            p_bf, tau_bf = _brute_force_entmax(s, alpha)
            p, tau, _ = oracle.entmax_sort(s, alpha)
            pb, taub = oracle.entmax_bisect(s, alpha, 200)
            assert abs(tau - tau_bf) < 1e-12
            np.testing.assert_allclose(p, p_bf, atol=1e-12)
            assert abs(taub - tau_bf) < 1e-12
            np.testing.assert_allclose(pb, p_bf, atol=1e-12)


@pytest.mark.parametrize("alpha", [1.25, 1.5, 2.0])
def test_variational_optimality(alpha):
    """entmax(z) maximises p.z + H_alpha(p) over the simplex (App. A Eqs. 11-12)."""
    rng = np.random.default_rng(3)

    def objective(p, z):
        return p @ z + np.sum(p - p ** alpha, axis=-1) / (alpha * (alpha - 1.0))

    for n in (4, 16):
        z = rng.normal(size=n) * 2.0
        p, _, _ = oracle.entmax_sort(z, alpha)
        best = objective(p, z)
        cand = rng.dirichlet(np.full(n, 0.5), size=10000)
        assert best >= objective(cand, z).max() - 1e-12
        # small feasible perturbations do not improve it either
        for _ in range(200):
            e = rng.normal(size=n) * 1e-3
            e -= e.mean()
            q = np.clip(p + e, 0, None)
            q /= q.sum()
            assert best >= objective(q, z) - 1e-13


# ---------------------------------------------------------------- pooling ---

def test_pool_mean_closed_form():
    """q̄ = 0 makes Eq. 3 the chunk mean (Sec. 3.1); arithmetic rows give (first + last)/2."""
    nk, hkv, d, B = 200, 2, 3, 64
    t = np.arange(nk, dtype=np.float64)
    K = np.empty((nk, hkv, d), dtype=np.float32)
    for r in range(hkv):
        for e in range(d):
            K[:, r, e] = (r + 1) * t + e
    out = oracle.pool(K, B, n_chunks=-(-nk // B))
    for c in range(out.shape[0]):
        t0, t1 = c * B, min((c + 1) * B, nk) - 1
        for r in range(hkv):
            for e in range(d):
                assert out[c, r, e] == (r + 1) * (t0 + t1) / 2.0 + e


def test_pool_q_zero_query_is_the_mean():
    """A zero summary query gives uniform weights (Sec. 3.1): the pinned chunk mean."""
    rng = np.random.default_rng(5)
    K = rng.normal(size=(200, 3, 16)).astype(np.float32)
    nch = -(-200 // 64)
    assert np.abs(oracle.pool_q(K, np.zeros((nch, 3, 16)), 64, n_chunks=nch) -
                  oracle.pool(K, 64, n_chunks=nch)).max() < 1e-15


def test_pool_q_two_keys_is_a_logistic_mix():
    """For a chunk of two keys Eq. 3 reduces to s(D) k1 + (1 - s(D)) k2 with the logistic
    s and D = <q, k1 - k2>/sqrt(d); every (chunk, head) has its own query."""
    from scipy.special import expit
    rng = np.random.default_rng(6)
    nk, hkv, d = 12, 3, 8
    K = rng.normal(size=(nk, hkv, d)).astype(np.float32)
    Qb = rng.normal(size=(nk // 2, hkv, d)).astype(np.float32)
    out = oracle.pool_q(K, Qb, 2)
    for c in range(nk // 2):
        for r in range(hkv):
            k1, k2 = K[2 * c, r].astype(np.float64), K[2 * c + 1, r].astype(np.float64)
            a = expit(float(Qb[c, r].astype(np.float64) @ (k1 - k2)) / np.sqrt(d))
            assert np.abs(out[c, r] - (a * k1 + (1 - a) * k2)).max() < 1e-14


def test_pool_q_large_query_selects_the_best_key():
    """Scaling q̄ to infinity turns the softmax weights into the indicator of the key
    with the largest <q̄, k_t> (distinct projections): the summary is that key."""
    rng = np.random.default_rng(7)
    nk, hkv, d, B = 96, 2, 16, 32
    K = rng.normal(size=(nk, hkv, d)).astype(np.float32)
    u = rng.normal(size=(nk // B, hkv, d))
    out = oracle.pool_q(K, (1e6 * u).astype(np.float32), B)
    for c in range(nk // B):
        for r in range(hkv):
            u32 = (1e6 * u[c, r]).astype(np.float32).astype(np.float64)
            best = int(np.argmax(K[c * B:(c + 1) * B, r].astype(np.float64) @ u32))
            assert np.array_equal(out[c, r], K[c * B + best, r].astype(np.float64))


def test_pool_q_invariants():
    """Identical keys pool to that key; permuting a chunk's keys changes nothing; adding
    one vector to every key shifts the summary by that vector (the weights are
    unchanged: every score moves by the same amount)."""
    rng = np.random.default_rng(8)
    nk, hkv, d, B = 64, 2, 8, 16
    K = (rng.integers(-64, 64, size=(nk, hkv, d)) / 16.0).astype(np.float32)
    Qb = rng.normal(size=(nk // B, hkv, d)).astype(np.float32)
    base = oracle.pool_q(K, Qb, B)
    same = np.repeat(K[::B], B, axis=0)
    assert np.array_equal(oracle.pool_q(same, Qb, B), K[::B].astype(np.float64))
    perm = np.concatenate([c * B + rng.permutation(B) for c in range(nk // B)])
    assert np.abs(oracle.pool_q(K[perm], Qb, B) - base).max() < 1e-14
    shift = (rng.integers(-8, 8, size=(hkv, d)) / 4.0).astype(np.float32)
    assert np.abs(oracle.pool_q(K + shift, Qb, B) - (base + shift)).max() < 1e-13


def test_fwd_uses_the_learned_summaries():
    """Stage 1 sees only the summaries: with q̄ so large that each chunk's summary is its
    best-matching key, routing equals mean-pooled routing over keys where every chunk
    is filled with that key; a zero q̄ reproduces the default forward exactly."""
    rng = np.random.default_rng(9)
    nq = nk = 256
    hq, hkv, d, B = 4, 2, 16, 32
    Q = rng.normal(size=(nq, hq, d)).astype(np.float32) * 3
    K = rng.normal(size=(nk, hkv, d)).astype(np.float32)
    V = rng.normal(size=(nk, hkv, d)).astype(np.float32)
    u = (1e6 * rng.normal(size=(nk // B, hkv, d))).astype(np.float32)
    best = oracle.pool_q(K, u, B).astype(np.float32)
    K_best = np.repeat(best, B, axis=0)
    a = oracle.fwd(Q, K, V, B, 1.5, sigma=1.0, qbar=u)
    b = oracle.fwd(Q, K_best, V, B, 1.5, sigma=1.0)
    assert np.array_equal(a["routed"], b["routed"])
    assert np.abs(a["w"] - b["w"]).max() < 1e-12
    assert np.allclose(a["tau"], b["tau"], atol=1e-12, equal_nan=True)
    z = oracle.fwd(Q, K, V, B, 1.5, sigma=1.0, qbar=np.zeros((nk // B, hkv, d)))
    ref = oracle.fwd(Q, K, V, B, 1.5, sigma=1.0)
    for key in ("out", "w", "routed"):
        assert np.array_equal(z[key], ref[key])


# ------------------------------------------------------------ full forward --

def _case(seed, nq, nk, hq, hkv, d, B, planted=True):
    rng = np.random.default_rng(seed)
    u = rng.normal(size=d)
    u /= np.linalg.norm(u)
    Q = rng.normal(size=(nq, hq, d))
    K = rng.normal(size=(nk, hkv, d))
    V = rng.normal(size=(nk, hkv, d))
    if planted:
        tc = nk // B
        for r in range(hkv):
            for c in rng.choice(tc, max(1, tc // 4), replace=False):
                K[c * B:(c + 1) * B, r] += 2.0 * u
        Q += rng.uniform(2.0, 8.0, size=(nq, hq, 1)) * u
    return Q.astype(np.float32), K.astype(np.float32), V.astype(np.float32)


@pytest.mark.parametrize("sigma", [1.0, 3.0, 1e8])
@pytest.mark.parametrize("shape", [(96, 96, 4, 2, 16, 16), (70, 100, 2, 1, 8, 16), (128, 128, 3, 3, 8, 32)])
def test_prop1_bias_form_equals_prior_form(sigma, shape):
    """Prop. 1: Eq. 7 with g from Eqs. 8-10 equals softmax(z + d) V (two independent routes)."""
    nq, nk, hq, hkv, d, B = shape
    Q, K, V = _case(11, nq, nk, hq, hkv, d, B)
    for alpha in (1.5, 1.25):
        a = oracle.fwd(Q, K, V, B, alpha, sigma=sigma, route=0, want=("out", "routed"))
        b = oracle.fwd(Q, K, V, B, alpha, sigma=sigma, route=1, want=("out",))
        assert a["routed"].any()
        np.testing.assert_allclose(b["out"], a["out"], rtol=0, atol=1e-12)


def test_sigma_to_infinity_lambda():
    """sigma -> inf gives lambda -> |R|/(|R| + |D|) (Sec. 3.4)."""
    nq, nk, hq, hkv, d, B = 80, 80, 2, 1, 8, 16
    Q, K, V = _case(5, nq, nk, hq, hkv, d, B)
    res = oracle.fwd(Q, K, V, B, 1.5, sigma=1e12, route=1, want=("lambda", "routed"))
    for i in range(nq):
        nR = res["routed"][i, 0].sum() * B
        nD = i % B + 1
        exp = nR / (nR + nD)
        np.testing.assert_allclose(res["lambda"][i], exp, atol=1e-9)


@pytest.mark.parametrize("causal", [True, False])
def test_uniform_all_chunk_prior_is_dense_attention(causal):
    """Every chunk routed with a uniform prior (d = 0) reduces Stage 2 to dense
    softmax attention (Eq. 5 with g uniform); reference: torch SDPA in fp64."""
    nq, nk, hq, hkv, d, B = 60, 100, 4, 2, 16, 16
    Q, K, V = _case(3, nq, nk, hq, hkv, d, B, planted=False)
    nch = oracle.n_chunks_for(nk, B, causal)
    rows = np.arange(nq)
    r_in = np.zeros((nq, hkv, nch), dtype=np.uint8)
    w_in = np.zeros((nq, hkv, nch))
    for i in range(nq):
        nvis = min((i + nk - nq) // B, nch) if causal else nch
        r_in[i, :, :nvis] = 1
        w_in[i, :, :nvis] = 1.0 / max(nvis, 1)
    res = oracle.fwd_rows(Q, rows, nq, K, V, B, 1.5, causal=causal, w_in=w_in, r_in=r_in, want=("out",))
    q = torch.from_numpy(Q).double().permute(1, 0, 2)
    k = torch.from_numpy(K).double().permute(1, 0, 2).repeat_interleave(hq // hkv, 0)
    v = torch.from_numpy(V).double().permute(1, 0, 2).repeat_interleave(hq // hkv, 0)
    mask = None
    if causal:
        ii = torch.arange(nq).view(-1, 1) + (nk - nq)
        jj = torch.arange(nk).view(1, -1)
        mask = jj <= ii
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=mask).permute(1, 0, 2)
    np.testing.assert_allclose(res["out"], ref.numpy(), atol=1e-12)
    dense = oracle.dense_attention(Q, K, V, causal=causal)
    np.testing.assert_allclose(dense, ref.numpy(), atol=1e-12)


def test_two_block_window_with_all_chunks_is_dense_attention():
    """App. B.1.1's local window (the query's chunk and the one before it): with every chunk
    before the window routed under a uniform prior, Stage 2 covers exactly the keys j <= p_i
    once each, so it is dense causal attention; rows in the first two chunks route nothing
    and no row ever routes the chunk just before its own."""
    nq, nk, hq, hkv, d, B = 70, 100, 4, 2, 16, 16
    Q, K, V = _case(4, nq, nk, hq, hkv, d, B, planted=False)
    nch = oracle.n_chunks_for(nk, B, True)
    rows = np.arange(nq)
    r_in = np.zeros((nq, hkv, nch), dtype=np.uint8)
    for i in range(nq):
        r_in[i, :, :max(0, min((i + nk - nq) // B - 1, nch))] = 1
    res = oracle.fwd_rows(Q, rows, nq, K, V, B, 1.5, causal=True, w_in=r_in.astype(np.float64), r_in=r_in,
                          want=("out",), local=2)
    np.testing.assert_allclose(res["out"], oracle.dense_attention(Q, K, V, causal=True), atol=1e-12)
    own = oracle.fwd_rows(Q, rows, nq, K, V, B, 1.5, causal=True, want=("out", "tau", "routed"), local=2)
    c_i = (rows + nk - nq) // B
    assert np.isnan(own["tau"][c_i <= 1]).all() and not np.isnan(own["tau"][c_i >= 2]).any()
    for i in range(nq):
        assert not own["routed"][i, :, max(c_i[i] - 1, 0):].any()


def test_group_prior_properties():
    """w sums to 1, its support is the union of the heads' supports, g = 1 gives w = p (Sec. 3.2)."""
    nq, nk, hq, hkv, d, B = 64, 128, 4, 1, 16, 16
    Q, K, V = _case(9, nq, nk, hq, hkv, d, B)
    res = oracle.fwd(Q, K, V, B, 1.5, want=("w", "routed", "xmt", "tau"))
    w, routed, xmt = res["w"], res["routed"], res["xmt"]
    for i in range(nq):
        nvis = (i + nk - nq) // B
        if nvis == 0:
            assert not routed[i].any()
            continue
        assert abs(w[i, 0].sum() - 1.0) < 1e-12
        union = (xmt[i, :, :nvis] > 0).any(axis=0)
        assert (routed[i, 0, :nvis] == union).all()
        assert ((w[i, 0, :nvis] > 0) == union).all()
    # g = 1: the group distribution is the head's own entmax of gamma<q,kbar>/sqrt(d)
    Kbar = oracle.pool(K, B)
    res1 = oracle.fwd(Q[:, :1], K, V, B, 1.5, gamma=0.7, want=("w",))
    for i in (20, 63):
        nvis = (i + nk - nq) // B
        s = 0.7 * (Kbar[:nvis, 0] @ Q[i, 0].astype(np.float64)) / np.sqrt(d)
        p, _, _ = oracle.entmax_sort(s, 1.5)
        np.testing.assert_allclose(res1["w"][i, 0, :nvis], p, atol=1e-14)


def test_first_chunk_rows_attend_diagonal_only():
    """Rows in chunk 0 have no visible chunk: R is empty and Stage 2 is causal softmax on D."""
    nq, nk, hq, hkv, d, B = 32, 32, 2, 1, 8, 32
    Q, K, V = _case(2, nq, nk, hq, hkv, d, B, planted=False)
    res = oracle.fwd(Q, K, V, B, 1.5, want=("out", "tau"))
    assert np.isnan(res["tau"]).all()
    dense = oracle.dense_attention(Q, K, V, causal=True)
    np.testing.assert_allclose(res["out"], dense, atol=1e-13)


@pytest.mark.parametrize("gamma", [0.5, 1.0])
def test_stage1_scores_closed_form(gamma):
    """Eq. 4 end to end: with q = (sqrt(d)/gamma) e_1 and chunk means whose first
    coordinate is s_c, the routed distribution of a single head is entmax(s);
    at alpha = 2 that is the simplex projection of s (independent QP)."""
    d, B, nc = 4, 4, 9
    rng = np.random.default_rng(4)
    s = rng.normal(size=nc) * 0.6
    nk = B * (nc + 1)
    K = rng.normal(size=(nk, 1, d))
    for c in range(nc):
        eps = rng.normal(size=B)
        eps -= eps.mean()
        K[c * B:(c + 1) * B, 0, 0] = s[c] + eps
    V = rng.normal(size=(nk, 1, d))
    q = np.zeros((1, 1, d))
    q[0, 0, 0] = np.sqrt(d) / gamma
    rows = np.array([nk - 1])
    res = oracle.fwd_rows(q.astype(np.float32), rows, nk, K.astype(np.float32), V.astype(np.float32), B,
                          2.0, gamma=gamma, want=("w", "routed"))
    # the float32 rounding of the inputs moves s by < 1e-6
    s32 = K.astype(np.float32).astype(np.float64)[:nc * B, 0, 0].reshape(nc, B).mean(1)
    np.testing.assert_allclose(res["w"][0, 0, :nc], _simplex_projection_qp(s32), atol=2e-7)
    assert res["w"][0, 0, nc:].sum() == 0.0

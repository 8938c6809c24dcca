"""Pins of the oracle's backward (oracle/backward.py) against things other than
itself (CPU only).

- its masked-attention forward, rebuilt from the trace, equals the pinned C
  oracle's outputs (so the live-state partition it reads from the trace is
  the one the forward used);
- central differences of the C oracle's forward (fp64 inputs, trace checked
  unchanged at +-eps) equal its gradients, element by element;
- one token: the closed form;
- tau > 2 (every token joins, one state): plain causal linear attention,
  differentiated by torch's fp64 autograd;
- a hand-written live-state list;
- planted mistakes (the means term dropped, the state weight taken as 1, the
  softmax gradient uncentred, phi' dropped, the mask's owner off by one
  state) each fail the central-difference comparison.
"""
import numpy as np
import pytest

from dynamic_state_memory_b200 import synth
from oracle import backward as BW
from oracle import oracle as O


def stream(seed, T, d, n_centres=3, mean_len=6.0):
    st = synth.HeadStream(seed, 0, 0, T=T, d=d, n_centres=n_centres,
                          lengths=("geometric", mean_len), sigma=0.05)
    return (st.q.astype(np.float64), st.k.astype(np.float64), st.v.astype(np.float64))


def oracle_fwd(q, k, v, C, tau):
    orc = O.Oracle(1, q.shape[1], v.shape[1], C)
    r = orc.run(k[None], q[None], v[None], tau=tau, dtype="f64")
    return r["out"][0], r["boundary"][0], r["merges"][0], r["margins"][0]


def test_live_starts_by_hand():
    # boundaries at 0, 2, 3, 5; at token 5 the sealed pair (0, 1) merges
    b = [1, 0, 1, 1, 0, 1, 0]
    got = BW.live_starts(b, [(5, 0)])
    assert got == [[0], [0], [0, 2], [0, 2, 3], [0, 2, 3], [0, 3, 5], [0, 3, 5]]
    with pytest.raises(ValueError):
        BW.live_starts(b, [(4, 0)])       # not on a boundary


@pytest.mark.parametrize("seed,C", [(3, 2), (7, 3), (5, 4), (6, 16)])
def test_masked_forward_equals_oracle(seed, C):
    q, k, v = stream(seed, 90, 8)
    o, b, merges, _ = oracle_fwd(q, k, v, C, 0.5)
    if C < 16:
        assert merges, "the case must merge"
    o2 = BW.forward_head(q, k, v, b, merges)
    assert np.abs(o2 - o).max() <= 1e-12 * max(1.0, np.abs(o).max())


def _loss(q, k, v, dO, C, tau, ref_trace):
    o, b, merges, _ = oracle_fwd(q, k, v, C, tau)
    assert np.array_equal(b, ref_trace[0]) and merges == ref_trace[1], "decision moved"
    return float(np.sum(o * dO))


@pytest.mark.parametrize("seed,C", [(11, 2), (12, 3), (13, 5)])
def test_central_differences_of_the_oracle_forward(seed, C):
    T, d, tau, eps = 48, 6, 0.5, 1e-6
    q, k, v = stream(seed, T, d)
    o, b, merges, margins = oracle_fwd(q, k, v, C, tau)
    assert merges, "the case must merge"
    # decisions far from their thresholds compared with eps
    assert margins[0] > 1e-4 and margins[1] > 1e-4, margins
    dO = np.random.default_rng(seed).standard_normal(o.shape)
    gq, gk, gv = BW.backward_head(q, k, v, dO, b, merges)
    rng = np.random.default_rng(seed + 100)
    for name, x, g in (("q", q, gq), ("k", k, gk), ("v", v, gv)):
        scale = np.abs(g).max()
        for _ in range(40):
            t, c = int(rng.integers(T)), int(rng.integers(d))
            xp, xm = x.copy(), x.copy()
            xp[t, c] += eps
            xm[t, c] -= eps
            args = {"q": q, "k": k, "v": v}
            lp = _loss(**{**args, name: xp}, dO=dO, C=C, tau=tau, ref_trace=(b, merges))
            lm = _loss(**{**args, name: xm}, dO=dO, C=C, tau=tau, ref_trace=(b, merges))
            fd = (lp - lm) / (2 * eps)
            assert abs(fd - g[t, c]) <= 1e-6 * scale, (name, t, c, fd, g[t, c])


def test_one_token_closed_form():
    rng = np.random.default_rng(1)
    q, k, v, dO = (rng.standard_normal((1, 5)) for _ in range(4))
    gq, gk, gv = BW.backward_head(q, k, v, dO, [1], [])
    fq, fk = BW.phi(q[0]), BW.phi(k[0])
    # o = (phi(q) . phi(k)) v, one state (lambda = 1)
    np.testing.assert_allclose(gv[0], np.dot(fq, fk) * dO[0], rtol=1e-14)
    np.testing.assert_allclose(gq[0], np.dot(dO[0], v[0]) * fk * BW.dphi(q[0]), rtol=1e-14)
    np.testing.assert_allclose(gk[0], np.dot(dO[0], v[0]) * fq * BW.dphi(k[0]), rtol=1e-14)


def test_one_state_is_causal_linear_attention():
    torch = pytest.importorskip("torch")
    q, k, v = stream(21, 40, 6)
    o, b, merges, _ = oracle_fwd(q, k, v, 4, 2.5)   # r <= 2 < tau: every token joins
    assert b.sum() == 1 and not merges
    dO = np.random.default_rng(2).standard_normal(o.shape)
    tq, tk, tv = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (q, k, v))
    f = lambda x: torch.where(x > 0, x + 1.0, torch.exp(torch.clamp(x, max=0.0)))
    A = torch.tril(f(tq) @ f(tk).T)
    (A @ tv * torch.tensor(dO)).sum().backward()
    gq, gk, gv = BW.backward_head(q, k, v, dO, b, merges)
    for g, t in ((gq, tq), (gk, tk), (gv, tv)):
        np.testing.assert_allclose(g, t.grad.numpy(), rtol=1e-11, atol=1e-11)


MUTANTS = {
    "no_means_term": ("c = dA * Lam + (da * rs / n)[owner]", "c = dA * Lam"),
    "state_weight_one": ("c = dA * Lam + (da * rs / n)[owner]", "c = dA + (da * rs / n)[owner]"),
    "softmax_uncentred": ("da = lam * (dlam - np.dot(lam, dlam))", "da = lam * dlam"),
    "no_dphi": ("return dfq * dphi(q), dfk * dphi(k), dv", "return dfq, dfk, dv"),
    "owner_shifted": ("Lam = lam[owner]", "Lam = lam[np.minimum(owner + 1, len(lam) - 1)]"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistakes_fail_the_difference_check(name):
    import inspect
    src = inspect.getsource(BW)
    old, new = MUTANTS[name]
    assert src.count(old) == 1
    ns = {}
    exec(compile(src.replace(old, new), "mutant", "exec"), ns)
    T, d, C, tau, eps = 48, 6, 3, 0.5, 1e-6
    q, k, v = stream(12, T, d)
    o, b, merges, _ = oracle_fwd(q, k, v, C, tau)
    dO = np.random.default_rng(12).standard_normal(o.shape)
    grads = dict(zip("qkv", ns["backward_head"](q, k, v, dO, b, merges)))
    rng = np.random.default_rng(5)
    worst = 0.0
    for name_x in "qkv":
        x = {"q": q, "k": k, "v": v}[name_x]
        g = grads[name_x]
        for _ in range(15):
            t, c = int(rng.integers(T)), int(rng.integers(d))
            xp, xm = x.copy(), x.copy()
            xp[t, c] += eps
            xm[t, c] -= eps
            args = {"q": q, "k": k, "v": v}
            lp = _loss(**{**args, name_x: xp}, dO=dO, C=C, tau=tau, ref_trace=(b, merges))
            lm = _loss(**{**args, name_x: xm}, dO=dO, C=C, tau=tau, ref_trace=(b, merges))
            worst = max(worst, abs((lp - lm) / (2 * eps) - g[t, c]) / max(np.abs(g).max(), 1e-30))
    assert worst > 1e-6, (name, worst)

"""Pins of the oracle's information policy (CPU only).

The policy is the pages' own decision and merge rule (Dynamic Linear
Attention | Chlience Paper Archive, section 5.1: score of the per-token state
against the open state after RMSNorm, a boundary at or above tau; section 5.2:
capacity merge of the adjacent pair of least information density).  Each
check is independent of the oracle's elementwise arithmetic:
- a hand-derived trace at d = 1 (tests/golden/info_hand_trace.json), where
  the score is a sign-change detector, and an exact-tie case;
- closed forms of the score (a positive multiple of the open state scores 0,
  a negative one 2, an orthogonal one sqrt 2);
- a brute-force re-simulation computing the score in Gram form from token
  ranges, with every output rebuilt from explicit outer products;
- invariants (score sums, counts, states) and the special cases of one state
  (causal linear attention) and all singletons.
"""
import json
import os

import numpy as np
import pytest

from dynamic_state_memory_b200 import synth
from oracle import oracle as O
from tests import bruteforce as bf

HERE = os.path.dirname(os.path.abspath(__file__))


def info_case(seed, T, d, n_centres=3, mean_len=6.0, sigma=0.05):
    st = synth.HeadStream(seed, 0, 0, T=T, d=d, n_centres=n_centres,
                          lengths=("geometric", mean_len), sigma=sigma, value_regimes=True)
    return (st.q.astype(np.float64), st.k.astype(np.float64), st.v.astype(np.float64))


def run_info(q, k, v, C, tau, lib=None, want_out=True):
    T, d = k.shape
    orc = O.Oracle(1, d, v.shape[1], C, "info", lib=lib)
    res = orc.run(k[None], None if q is None else q[None], v[None], tau=tau, dtype="f64",
                  nthreads=1, want_out=want_out)
    return res, orc


def check_info_hand_trace(lib=None):
    g = json.load(open(os.path.join(HERE, "golden", "info_hand_trace.json")))
    v = np.array(g["v"], dtype=np.float64)[:, None]
    k = np.zeros_like(v)
    q = np.zeros_like(v)
    res, orc = run_info(q, k, v, g["C"], g["tau"], lib=lib)
    assert res["boundary"][0].tolist() == g["boundary"]
    assert [list(m) for m in res["merges"][0]] == g["merges"]
    assert res["live"][0].tolist() == g["live"]
    assert np.allclose(res["out"][0, :, 0], g["out"], rtol=0, atol=1e-12)
    flips = np.array(g["boundary"], dtype=bool)
    flips[0] = False
    assert np.allclose(res["score"][0][flips], g["flip_score_approx"], atol=1e-5)
    assert np.all(res["score"][0][~flips] < 1e-5)
    st = orc.state(0)
    assert st["ts"].tolist() == g["final_ts"]
    assert st["n"].tolist() == g["final_n"]
    assert np.allclose(st["info"], g["final_info_approx"], atol=1e-5)
    # exact ties: zero values score 0 everywhere
    T = g["zero_T"]
    z = np.zeros((T, 1))
    res, _ = run_info(z, z, z, g["zero_C"], g["zero_tau"], lib=lib)
    assert res["boundary"][0].all()
    assert [list(m) for m in res["merges"][0]] == g["zero_merges"]


def test_info_hand_trace():
    check_info_hand_trace()


def check_info_score_closed_forms(lib=None):
    rng = np.random.default_rng(5)
    d = 4
    k0 = rng.standard_normal(d)
    v0 = rng.standard_normal(d)
    w = rng.standard_normal(d)
    w_perp = w - (w @ v0) / (v0 @ v0) * v0       # orthogonal to v0
    cases = [(2.5 * v0, 0.0), (-0.7 * v0, 2.0), (w_perp, np.sqrt(2.0))]
    for v1, want in cases:
        k = np.stack([k0, k0])
        v = np.stack([v0, v1])
        res, _ = run_info(np.zeros_like(k), k, v, 4, 10.0, lib=lib)
        assert abs(res["score"][0, 1] - want) < 1e-5, (want, res["score"][0, 1])


def test_info_score_closed_forms():
    check_info_score_closed_forms()


INFO_GRID = [(seed, C, tau) for seed in range(16) for C in (2, 3, 5) for tau in (0.3, 0.5, 1.0)]


def check_info_against_bruteforce(seed, C, tau, lib=None):
    T, d = 48, 6
    q, k, v = info_case(seed, T, d)
    res, _ = run_info(q, k, v, C, tau, lib=lib)
    bnd, mer, score = bf.info_simulate(k, v, C, tau)
    # every score agrees with the Gram form; decisions are compared only when
    # no score lies within rounding of tau
    assert np.allclose(res["score"][0], score, rtol=0, atol=1e-6)
    assert np.min(np.abs(score[1:] - tau)) > 1e-6
    assert res["boundary"][0].tolist() == bnd.tolist()
    assert [tuple(m) for m in res["merges"][0]] == mer
    ranges = bf.replay(bnd, mer, C)
    assert res["live"][0].tolist() == [len(r) for r in ranges]
    assert max(len(r) for r in ranges) <= C
    o = bf.outputs(q, k, v, ranges)
    scale = np.abs(o).max()
    assert np.allclose(res["out"][0], o, rtol=0, atol=1e-11 * scale)


@pytest.mark.parametrize("seed,C,tau", INFO_GRID)
def test_info_against_bruteforce(seed, C, tau):
    check_info_against_bruteforce(seed, C, tau)


def test_info_inputs_have_both_decisions():
    # the value-regime inputs give boundaries and joins at every tau of the grid
    for tau in (0.3, 0.5, 1.0):
        nb = 0
        for seed in range(16):
            q, k, v = info_case(seed, 48, 6)
            b, mer, _ = bf.info_simulate(k, v, 3, tau)
            nb += int(b.sum())
        assert 16 < nb < 16 * 47


def check_info_invariants(lib=None):
    T, d, C = 80, 5, 4
    q, k, v = info_case(21, T, d)
    res, orc = run_info(q, k, v, C, 0.5, lib=lib)
    st = orc.state(0)
    assert st["m"] <= C
    assert st["n"].sum() == T
    assert (np.diff(st["ts"]) > 0).all()
    assert np.isclose(st["info"].sum(), res["score"][0].sum(), rtol=1e-12, atol=0)
    U = bf.phi(k)
    assert np.allclose(st["S"].sum(axis=0), v.T @ U, rtol=1e-12, atol=1e-12)
    assert np.allclose(st["z"].sum(axis=0), U.sum(axis=0), rtol=1e-12, atol=1e-12)


def test_info_invariants():
    check_info_invariants()


def check_info_single_state(lib=None):
    # the score is at most 2 (two unit-RMS matrices), so tau = 3 never opens
    # a second state: causal linear attention
    T, d = 40, 5
    q, k, v = info_case(7, T, d)
    res, _ = run_info(q, k, v, 4, 3.0, lib=lib)
    assert res["boundary"][0].sum() == 1
    assert (res["score"][0] <= 2.0 + 1e-12).all()
    P, U = bf.phi(q), bf.phi(k)
    assert np.allclose(res["out"][0], np.tril(P @ U.T) @ v, rtol=1e-12, atol=1e-10)


def test_info_single_state():
    check_info_single_state()


def check_info_all_singletons(lib=None):
    # tau <= 0: every score is >= tau, so every token opens a state
    T, d = 30, 4
    q, k, v = info_case(3, T, d)
    res, _ = run_info(q, k, v, T + 1, 0.0, lib=lib)
    assert res["boundary"][0].all()
    assert res["merge_count"][0] == 0
    P, U = bf.phi(q), bf.phi(k)
    G = P @ U.T
    o = np.zeros((T, d))
    for t in range(T):
        a = G[t, :t + 1] / np.sqrt(d)
        w = np.exp(a - a.max())
        w /= w.sum()
        o[t] = (w * G[t, :t + 1]) @ v[:t + 1]
    assert np.allclose(res["out"][0], o, rtol=1e-12, atol=1e-10)


def test_info_all_singletons():
    check_info_all_singletons()


def test_info_split_calls_equal_one_call():
    T, d, C = 60, 5, 3
    q, k, v = info_case(4, T, d)
    one, _ = run_info(q, k, v, C, 0.5)
    orc = O.Oracle(1, d, d, C, "info")
    parts = []
    for a, b in ((0, 17), (17, 18), (18, 60)):
        parts.append(orc.run(k[None, a:b], q[None, a:b], v[None, a:b], tau=0.5, dtype="f64",
                             nthreads=1))
    assert np.concatenate([p["boundary"][0] for p in parts]).tolist() == one["boundary"][0].tolist()
    assert np.array_equal(np.concatenate([p["out"][0] for p in parts]), one["out"][0])
    assert np.array_equal(np.concatenate([p["score"][0] for p in parts]), one["score"][0])


def test_info_trace_only_mode_matches():
    # without outputs the oracle still needs v (the score reads the states)
    T, d = 50, 4
    q, k, v = info_case(9, T, d)
    full, _ = run_info(q, k, v, 3, 0.5)
    tr, _ = run_info(None, k, v, 3, 0.5, want_out=False)
    assert tr["out"] is None
    assert tr["boundary"].tolist() == full["boundary"].tolist()
    assert tr["merges"] == full["merges"]


def _f(x):
    return float("inf") if x == "inf" else float(x)


def check_info_margins_hand(lib=None):
    """min |I_t - tau|, the least relative gap between the best and the
    second-best pair density over the merges and the count of exact ties,
    derived by hand for the golden trace (tests/golden/info_hand_trace.json)."""
    g = json.load(open(os.path.join(HERE, "golden", "info_hand_trace.json")))
    v = np.array(g["v"], dtype=np.float64)[:, None]
    z = np.zeros_like(v)
    res, _ = run_info(z, z, v, g["C"], g["tau"], lib=lib)
    got = res["margins"][0]
    want = g["margins_approx"]
    assert abs(got[0] - want[0]) < 1e-5 and abs(got[1] - want[1]) < 1e-5 and got[2] == want[2], got
    T = g["zero_T"]
    z = np.zeros((T, 1))
    res, _ = run_info(z, z, z, g["zero_C"], g["zero_tau"], lib=lib)
    got = res["margins"][0]
    want = [_f(x) for x in g["zero_margins"]]
    assert got[0] == want[0] and got[1] == want[1] and got[2] == want[2], got


def test_info_margins_hand():
    check_info_margins_hand()


def check_info_forced_mode(seed, C, tau, lib=None):
    """The information policy with merges taken from a list: its own list
    reproduces the run (excess 0); the first merge forced onto another pair
    gives brute-force outputs over the implied ranges and the relative excess
    of that pair's density, recomputed from the ranges' score sums (Gram-form
    scores), over the least one."""
    T, d = 48, 6
    q, k, v = info_case(seed, T, d)
    res, _ = run_info(q, k, v, C, tau, lib=lib)
    merges = res["merges"][0]

    def forced(lst):
        orc = O.Oracle(1, d, d, C, "info", lib=lib)
        return orc.run(k[None], q[None], v[None], tau=tau, dtype="f64", nthreads=1,
                       force_merges=[lst])

    same = forced(merges)
    assert np.array_equal(same["out"], res["out"]) and same["excess"][0] == 0.0
    if not merges or C < 3:
        return
    t0, i0 = merges[0]
    alt = (t0, (i0 + 1) % (C - 1))
    lst = forced([alt])["merges"][0]
    got = forced(lst)
    assert got["merges"][0] == lst and lst[0] == alt
    bnd, _, score = bf.info_simulate(k, v, C, tau)
    assert res["boundary"][0].tolist() == bnd.tolist()
    o = bf.outputs(q, k, v, bf.replay(bnd, lst, C))
    assert np.allclose(got["out"][0], o, rtol=0, atol=1e-11 * np.abs(o).max())
    sealed = bf.replay(bnd[:t0], [], C)[t0 - 1]
    dens = np.array([(score[a0:b1 + 1].sum()) / (b1 - a0 + 1)
                     for (a0, _), (_, b1) in zip(sealed[:-1], sealed[1:])])
    best = dens.min()
    want = (dens[alt[1]] - best) / best if best > 0 else (0.0 if dens[alt[1]] == 0 else np.inf)
    assert abs(got["excess"][0] - want) <= 1e-6 * max(1.0, want), (got["excess"][0], want)


@pytest.mark.parametrize("seed,C", [(s, C) for s in range(8) for C in (3, 5)])
def test_info_forced_mode(seed, C):
    check_info_forced_mode(seed, C, 0.5)


def all_info_pins(lib):
    check_info_hand_trace(lib)
    check_info_margins_hand(lib)
    for seed in range(3):
        check_info_forced_mode(seed, 3, 0.5, lib)
    check_info_score_closed_forms(lib)
    for seed in range(6):
        for C in (2, 3, 5):
            for tau in (0.3, 0.5, 1.0):
                check_info_against_bruteforce(seed, C, tau, lib)
    check_info_invariants(lib)
    check_info_single_state(lib)
    check_info_all_singletons(lib)


def test_value_regimes_leave_other_inputs_unchanged():
    # the value-regime draws come after all others: q and k are those of the
    # plain recipe, and v follows each token's regime (one value centre per
    # key centre), within the noise
    kw = dict(T=200, d=16, n_centres=5, lengths=("geometric", 12.0), sigma=0.05)
    plain = synth.HeadStream(77, 0, 1, **kw)
    vr = synth.HeadStream(77, 0, 1, value_regimes=True, **kw)
    assert np.array_equal(plain.q, vr.q) and np.array_equal(plain.k, vr.k)
    assert not np.array_equal(plain.v, vr.v)
    # each v is nearest to its regime's value centre, whose key centre is
    # nearest to k
    kc = np.argmax(vr.k @ plain.centres.T, axis=1)
    vc = np.argmax(vr.v @ vr.vcentres.T, axis=1)
    assert (kc == vc).mean() > 0.95
    # and the workloads without the option draw what they drew before
    wl = dict(synth.WORKLOADS["tiny_f32"], T=64)
    a = synth.make_prefill(wl)
    b = synth.make_prefill(dict(wl, value_regimes=False))
    assert all(np.array_equal(x, y) for x, y in zip(a, b))

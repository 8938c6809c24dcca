"""Pins of the fp64 oracle against things other than itself (CPU only).

- a hand-derived decision trace (tests/golden/hand_trace.json);
- boundaries recomputed from numpy scores;
- every output recomputed from explicit per-token outer products over the
  state ranges the trace implies;
- every merge checked, over all adjacent pairs, against the scatter increase
  of Corollary 1 (Dynamic Linear Attention | Chlience Paper Archive), which
  equals the Ward loss n_a n_b/(n_a+n_b)|mu_a-mu_b|^2;
- invariants (m <= C, sum of states = all outer products, sum of n = t);
- special cases with textbook closed forms (one state: causal linear
  attention, section 1 of the same page; all singletons: per-token softmax);
- split calls equal one call; Fenwick buckets against the lowbit formula.
"""
import json
import os

import numpy as np
import pytest

from dynamic_state_memory_b200 import synth
from oracle import oracle as O
from tests import bruteforce as bf

HERE = os.path.dirname(os.path.abspath(__file__))


def small_case(seed, T, d, n_centres=3, mean_len=6.0, sigma=0.05):
    st = synth.HeadStream(seed, 0, 0, T=T, d=d, n_centres=n_centres,
                          lengths=("geometric", mean_len), sigma=sigma)
    return (st.q.astype(np.float64), st.k.astype(np.float64), st.v.astype(np.float64))


def run_one(q, k, v, C, tau, policy="dla", lib=None):
    T, d = k.shape
    orc = O.Oracle(1, d, v.shape[1], C, policy, lib=lib)
    res = orc.run(k[None], q[None], v[None], tau=tau, dtype="f64", nthreads=1)
    return res, orc


GRID = [(seed, C, tau) for seed in range(24) for C in (2, 3, 5) for tau in (0.3, 0.5, 1.0)]


def test_hand_trace():
    check_hand_trace()


def check_hand_trace(lib=None):
    g = json.load(open(os.path.join(HERE, "golden", "hand_trace.json")))
    for keys, bnd, mer, tau in (("keys", "boundary", "merges", "tau"),
                                ("keys2", "boundary2", "merges2", "tau"),
                                ("keys3", "boundary3", "merges3", "tau3")):
        k = np.array(g[keys], dtype=np.float64)
        q = np.ones_like(k)
        v = np.ones_like(k)
        res, _ = run_one(q, k, v, g["C"], g[tau], lib=lib)
        assert res["boundary"][0].tolist() == g[bnd]
        assert [list(m) for m in res["merges"][0]] == g[mer]


@pytest.mark.parametrize("seed,C,tau", GRID)
def test_against_bruteforce(seed, C, tau):
    check_against_bruteforce(seed, C, tau)


def check_against_bruteforce(seed, C, tau, lib=None):
    T, d = 48, 6
    q, k, v = small_case(seed, T, d)
    res, orc = run_one(q, k, v, C, tau, lib=lib)
    b = res["boundary"][0]
    merges = res["merges"][0]
    # boundaries from numpy scores (decision margins are far from rounding)
    r = bf.scores(k)
    join = np.zeros(T, dtype=bool)
    join[1:] = (r[1:] < tau) & (r[:-1] < tau)
    assert (b == (~join).astype(np.uint8)).all()
    ranges = bf.replay(b, merges, C)
    # capacity invariant and live counts
    for t in range(T):
        assert len(ranges[t]) <= C
        assert res["live"][0, t] == len(ranges[t])
    # every merge is the leftmost minimum of the scatter increase
    sealed = []
    open_ = None
    mi = 0
    for t in range(T):
        if b[t]:
            if open_ is not None:
                sealed.append(tuple(open_))
            if mi < len(merges) and merges[mi][0] == t:
                costs = bf.merge_costs_sse(k, sealed)
                i = merges[mi][1]
                tol = 1e-9 * max(1.0, float(np.abs(costs).max()))
                assert costs[i] <= costs.min() + tol
                assert (costs[:i] > costs[i] - tol).all()
                sealed[i:i + 2] = [(sealed[i][0], sealed[i + 1][1])]
                mi += 1
            open_ = [t, t]
        else:
            open_[1] = t
    # outputs from scratch
    o_ref = bf.outputs(q, k, v, ranges)
    err = np.abs(res["out"][0] - o_ref).max() / np.abs(o_ref).max()
    assert err < 1e-12
    # final state: sum of states, counts, timestamps
    st = orc.state(0)
    U = bf.phi(k)
    assert np.allclose(st["S"].sum(axis=0), v.T @ U, rtol=1e-12, atol=1e-12)
    assert st["n"].sum() == T
    assert (np.diff(st["ts"]) > 0).all()
    assert [int(x) for x in st["ts"]] == [a for (a, _) in ranges[-1]]


def test_single_state_is_causal_linear_attention():
    check_single_state()


def check_single_state(lib=None):
    # tau > 2: r <= 2 always, so after t = 0 every token joins the one state.
    T, d = 40, 5
    q, k, v = small_case(7, T, d)
    res, _ = run_one(q, k, v, 4, 2.5, lib=lib)
    assert res["boundary"][0].sum() == 1
    P, U = bf.phi(q), bf.phi(k)
    A = np.tril(P @ U.T)                # causal masked quadratic form
    assert np.allclose(res["out"][0], A @ v, rtol=1e-12, atol=1e-10)


def test_all_singletons_closed_form():
    check_all_singletons()


def check_all_singletons(lib=None):
    # tau <= 0 and C >= T: every token is its own state and nothing merges.
    T, d = 30, 4
    q, k, v = small_case(3, T, d)
    res, _ = run_one(q, k, v, T + 1, 0.0, lib=lib)
    assert res["boundary"][0].all()
    assert res["merge_count"][0] == 0
    P, U = bf.phi(q), bf.phi(k)
    G = P @ U.T
    o = np.zeros((T, d))
    for t in range(T):
        w = np.exp(G[t, :t + 1] / np.sqrt(d) - (G[t, :t + 1] / np.sqrt(d)).max())
        w /= w.sum()
        o[t] = (w * G[t, :t + 1]) @ v[:t + 1]
    assert np.allclose(res["out"][0], o, rtol=1e-12, atol=1e-10)


def test_no_merge_below_capacity():
    T, d = 64, 6
    q, k, v = small_case(11, T, d)
    res, _ = run_one(q, k, v, 10_000, 0.5)
    assert res["merge_count"][0] == 0
    assert res["live"][0, -1] == res["boundary"][0].sum()


@pytest.mark.parametrize("policy", ["dla", "fenwick"])
def test_split_calls_equal_one_call(policy):
    T, d, C = 60, 5, 3
    q, k, v = small_case(5, T, d)
    one, _ = run_one(q, k, v, C, 0.5, policy)
    orc = O.Oracle(1, d, d, C, policy)
    outs, bnds, mers = [], [], []
    for a, b in ((0, 17), (17, 18), (18, 60)):
        r = orc.run(k[None, a:b], q[None, a:b], v[None, a:b], tau=0.5, dtype="f64")
        outs.append(r["out"][0])
        bnds.append(r["boundary"][0])
        mers += r["merges"][0]
    assert np.array_equal(np.concatenate(outs), one["out"][0])
    assert np.array_equal(np.concatenate(bnds), one["boundary"][0])
    assert mers == one["merges"][0]


def test_fenwick_buckets():
    check_fenwick()


def check_fenwick(lib=None):
    T, d = 45, 4
    q, k, v = small_case(9, T, d)
    res, orc = run_one(q, k, v, 0, 0.5, "fenwick", lib=lib)
    ranges = bf.replay(res["boundary"][0], res["merges"][0], policy="fenwick")
    for t in range(T):
        assert ranges[t] == bf.fenwick_ranges(t)
        assert len(ranges[t]) == bin(t).count("1") + 1
        assert sum(b - a + 1 for a, b in ranges[t]) == t + 1
    o_ref = bf.outputs(q, k, v, ranges)
    assert np.abs(res["out"][0] - o_ref).max() < 1e-12 * np.abs(o_ref).max()


def test_bf16_and_f32_inputs_widen_exactly():
    T, d = 20, 4
    q, k, v = small_case(2, T, d)
    qb, kb, vb = (synth.to_bf16_bits(x.astype(np.float32)) for x in (q, k, v))
    o1 = O.Oracle(1, d, d, 3).run(kb[None], qb[None], vb[None], tau=0.5, dtype="bf16")
    wq, wk, wv = (synth.widen(x, "bf16") for x in (qb, kb, vb))
    o2 = O.Oracle(1, d, d, 3).run(wk[None], wq[None], wv[None], tau=0.5, dtype="f64")
    assert np.array_equal(o1["out"], o2["out"])


def test_synth_recipe():
    wl = synth.WORKLOADS["tiny_f32"]
    st = synth.HeadStream(1, 0, 0, **dict(wl, T=20000))
    assert np.allclose(np.linalg.norm(st.centres, axis=1), 1.0, atol=1e-6)
    # keys: centre + N(0, 0.05^2): residual std close to 0.05
    x = np.asarray([0.5, -1.25, 3.0, 1e-3], dtype=np.float32)
    assert np.array_equal(synth.bf16_bits_to_f32(synth.to_bf16_bits(x)),
                          np.asarray([0.5, -1.25, 3.0, 1.0234375 * 2.0 ** -10], dtype=np.float32))
    # and agrees with torch's float32 -> bfloat16 conversion on random values
    import torch
    r = np.random.default_rng(0).standard_normal(100000).astype(np.float32)
    tb = torch.from_numpy(r).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(synth.to_bf16_bits(r), tb)
    # round-to-nearest-even on a tie: 1 + 2^-8 is halfway between bf16 neighbours
    tie = np.asarray([1.0 + 2.0 ** -8], dtype=np.float32)
    assert synth.bf16_bits_to_f32(synth.to_bf16_bits(tie))[0] == 1.0
    lens = synth._draw_lengths(np.random.default_rng(0), ("geometric", 48.0), 200000)
    assert abs(lens.mean() - 48.0) < 1.5 and lens.min() >= 1
    ln = synth._draw_lengths(np.random.default_rng(0), ("lognormal", 64.0, 1.5), 2_000_000)
    assert abs(np.median(ln) - 64) <= 4


@pytest.mark.parametrize("policy", ["dla", "fenwick"])
def test_masked_readout_equals_full_readout(policy):
    """The masked readout (used for sampled outputs at full workload sizes)
    updates states at every token: its rows equal the full run's at the marked
    tokens and are zero elsewhere."""
    T, d = 200, 6
    q, k, v = small_case(3, T, d)
    full = O.Oracle(1, d, d, 4, policy).run(k[None], q[None], v[None], tau=0.5, dtype="f64")
    mask = np.zeros(T, dtype=np.uint8)
    mask[[0, 1, 63, 64, 127, 150, 199]] = 1
    part = O.Oracle(1, d, d, 4, policy).run(k[None], q[None], v[None], tau=0.5, dtype="f64",
                                            out_mask=mask)
    sel = mask.astype(bool)
    assert np.array_equal(part["out"][0, sel], full["out"][0, sel])
    assert not part["out"][0, ~sel].any()
    assert np.array_equal(part["boundary"], full["boundary"])
    assert part["merges"] == full["merges"]


# ---- the margins diagnostic and the forced-merge mode -----------------------

def _f(x):
    return float("inf") if x == "inf" else float(x)


def check_margins_hand(lib=None):
    """min |r_t - tau|, the least relative gap between the best and the
    second-best Ward loss over the merges and the count of exact ties, derived
    by hand for the golden keys (tests/golden/hand_trace.json)."""
    g = json.load(open(os.path.join(HERE, "golden", "hand_trace.json")))
    for keys, tau, want in (("keys", "tau", "margins"), ("keys2", "tau", "margins2"),
                            ("keys3", "tau3", "margins3"), ("keys4", "tau4", "margins4")):
        k = np.array(g[keys], dtype=np.float64)
        res, _ = run_one(np.ones_like(k), k, np.ones_like(k), g["C"], g[tau], lib=lib)
        got = res["margins"][0]
        exp = [_f(x) for x in g[want]]
        assert abs(got[0] - exp[0]) < 1e-12, (keys, got)
        assert (got[1] == exp[1]) if exp[1] == float("inf") else abs(got[1] - exp[1]) < 1e-12, (keys, got)
        assert got[2] == exp[2], (keys, got)


def test_margins_hand():
    check_margins_hand()


def check_forced_mode(seed, C, tau, lib=None):
    """Merges taken from a given list instead of the argmin.

    - The oracle's own merge list reproduces its run bit for bit, excess 0.
    - Forcing the first merge onto another pair (the later merges are then the
      argmin choices of that path) gives the outputs of brute force over the
      ranges the list implies, and an excess equal to the relative excess of
      the forced pair's scatter increase (Corollary 1) over the least one,
      recomputed from the token ranges.
    - A list whose token is not a capacity merge reports an infinite excess.
    """
    T, d = 48, 6
    q, k, v = small_case(seed, T, d)
    res, _ = run_one(q, k, v, C, tau, lib=lib)
    merges = res["merges"][0]
    b = res["boundary"][0]

    def forced(lst, want_out=True):
        orc = O.Oracle(1, d, d, C, lib=lib)
        return orc.run(k[None], q[None] if want_out else None, v[None] if want_out else None,
                       tau=tau, dtype="f64", nthreads=1, want_out=want_out,
                       force_merges=[lst])

    same = forced(merges)
    assert np.array_equal(same["out"], res["out"]) and same["merges"] == res["merges"]
    assert same["excess"][0] == 0.0
    if not merges:
        return
    t0, i0 = merges[0]
    assert forced([(t0 + 1, i0)] + merges[1:], want_out=False)["excess"][0] == np.inf
    # an entry left over, or one missing, is a mismatch too
    assert forced(merges + [(T + 5, 0)], want_out=False)["excess"][0] == np.inf
    assert forced(merges[:-1], want_out=False)["excess"][0] == np.inf
    if C < 3:
        return
    alt = (t0, (i0 + 1) % (C - 1))
    lst = forced([alt], want_out=False)["merges"][0]  # alt, then the argmin path
    assert lst[0] == alt
    got = forced(lst)
    assert got["merges"][0] == lst
    ranges = bf.replay(b, lst, C)
    o = bf.outputs(q, k, v, ranges)
    assert np.allclose(got["out"][0], o, rtol=0, atol=1e-11 * np.abs(o).max())
    # the sealed states just before the first merge: every state present at t0 - 1
    sealed = bf.replay(b[:t0], [], C)[t0 - 1]
    cost = bf.merge_costs_sse(k, sealed)
    best = cost.min()
    want = (cost[alt[1]] - best) / best if best > 0 else (0.0 if cost[alt[1]] == 0 else np.inf)
    assert abs(got["excess"][0] - want) <= 1e-9 * max(1.0, want), (got["excess"][0], want)


@pytest.mark.parametrize("seed,C,tau", [(s, C, tau) for s in range(8) for C in (2, 3, 5)
                                        for tau in (0.3, 0.5)])
def test_forced_mode(seed, C, tau):
    check_forced_mode(seed, C, tau)


# ---- DLA(I): no capacity bound ------------------------------------------------

def check_unbounded(seed, tau, lib=None):
    """The unbounded policy (the ablation row "Mamba-2 + DLA(I)"): boundaries
    from numpy scores, no merge ever, one state per segment, every output
    rebuilt from explicit outer products over the segments' token ranges."""
    T, d = 96, 6
    q, k, v = small_case(seed, T, d, mean_len=3.0)
    orc = O.Oracle(1, d, d, 2, "unbounded", lib=lib)
    res = orc.run(k[None], q[None], v[None], tau=tau, dtype="f64", nthreads=1)
    b = res["boundary"][0]
    r = bf.scores(k)
    join = np.zeros(T, dtype=bool)
    join[1:] = (r[1:] < tau) & (r[:-1] < tau)
    assert (b == (~join).astype(np.uint8)).all()
    assert res["merges"][0] == []
    ranges = bf.replay(b, [], policy="unbounded")
    assert res["live"][0].tolist() == [len(x) for x in ranges]
    assert res["live"][0].tolist() == np.cumsum(b).tolist()
    o = bf.outputs(q, k, v, ranges)
    assert np.allclose(res["out"][0], o, rtol=0, atol=1e-11 * np.abs(o).max())
    st = orc.state(0)
    assert st["m"] == int(b.sum()) and st["n"].sum() == T
    assert st["ts"].tolist() == np.flatnonzero(b).tolist()


@pytest.mark.parametrize("seed,tau", [(s, tau) for s in range(12) for tau in (0.3, 0.5, 1.0)])
def test_unbounded(seed, tau):
    check_unbounded(seed, tau)


def test_unbounded_split_calls_equal_one_call():
    T, d = 120, 5
    q, k, v = small_case(3, T, d, mean_len=2.0)
    one = O.Oracle(1, d, d, 2, "unbounded")
    full = one.run(k[None], q[None], v[None], tau=0.5, dtype="f64", nthreads=1)
    two = O.Oracle(1, d, d, 2, "unbounded")
    a = two.run(k[None, :50], q[None, :50], v[None, :50], tau=0.5, dtype="f64", nthreads=1)
    b = two.run(k[None, 50:], q[None, 50:], v[None, 50:], tau=0.5, dtype="f64", nthreads=1)
    assert np.array_equal(np.concatenate([a["out"][0], b["out"][0]]), full["out"][0])
    assert np.array_equal(np.concatenate([a["boundary"][0], b["boundary"][0]]), full["boundary"][0])
    assert full["live"][0].max() > 40  # far past any small capacity

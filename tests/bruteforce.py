"""Brute-force numpy checks used to pin the oracle (test helper, CPU only).

Nothing here is incremental: every state is rebuilt from explicit per-token
outer products over its token range, so a slip in the oracle's running sums,
merge bookkeeping or ordering shows up as a mismatch.
"""
from __future__ import annotations

import numpy as np


def phi(x):
    """elu(x) + 1."""
    x = np.asarray(x, dtype=np.float64)
    return np.where(x > 0, x + 1.0, np.exp(np.minimum(x, 0.0)))


def replay(boundary, merges, C=None, policy="dla"):
    """State token ranges [(first, last)] present at each token, in time order.

    ``merges`` is the trace's list of (t, i): at token t the sealed pair
    (i, i+1) (0-based, time order) is merged.  For DLA it asserts that a merge
    happens exactly when a boundary leaves C sealed states.
    """
    T = len(boundary)
    sealed = []
    open_ = None
    mi = 0
    out = []
    for t in range(T):
        if boundary[t]:
            if open_ is not None:
                sealed.append(tuple(open_))
            n_here = 0
            while mi < len(merges) and merges[mi][0] == t:
                i = merges[mi][1]
                assert 0 <= i < len(sealed) - 1, (t, i, len(sealed))
                if policy == "dla":
                    assert len(sealed) == C, (t, len(sealed), C)
                sealed[i:i + 2] = [(sealed[i][0], sealed[i + 1][1])]
                mi += 1
                n_here += 1
            if policy == "dla":
                assert n_here <= 1
                assert len(sealed) <= C - 1, (t, len(sealed))
            open_ = [t, t]
        else:
            assert open_ is not None
            assert not (mi < len(merges) and merges[mi][0] == t)
            open_[1] = t
        out.append(sealed + [tuple(open_)])
    assert mi == len(merges), "merge recorded at a token that is not a boundary"
    return out


def outputs(q, k, v, ranges):
    """o_t = sum_i softmax_i(phi(q_t).mu_i/sqrt(d)) S_i phi(q_t), S_i from scratch."""
    T, d = k.shape
    U = phi(k)
    P = phi(q)
    o = np.zeros((T, v.shape[1]))
    for t in range(T):
        logits = []
        reads = []
        for (a, b) in ranges[t]:
            Ur = U[a:b + 1]
            S = v[a:b + 1].T @ Ur           # sum_s v_s phi(k_s)^T
            mu = Ur.mean(axis=0)
            logits.append(P[t] @ mu / np.sqrt(d))
            reads.append(S @ P[t])
        logits = np.array(logits)
        w = np.exp(logits - logits.max())
        w /= w.sum()
        o[t] = (w[:, None] * np.array(reads)).sum(axis=0)
    return o


def scatter(U):
    if len(U) == 0:
        return 0.0
    return float(((U - U.mean(axis=0)) ** 2).sum())


def merge_costs_sse(k, sealed):
    """Scatter increase of merging each adjacent sealed pair (Corollary 1 form)."""
    U = phi(k)
    costs = []
    for j in range(len(sealed) - 1):
        A = U[sealed[j][0]:sealed[j][1] + 1]
        B = U[sealed[j + 1][0]:sealed[j + 1][1] + 1]
        costs.append(scatter(np.vstack([A, B])) - scatter(A) - scatter(B))
    return np.array(costs)


def scores(k):
    """r_t = 1 - cos(k_t, k_{t-1}), r_0 = 0, zero norm -> r = 1 (numpy dot order)."""
    T = k.shape[0]
    r = np.zeros(T)
    for t in range(1, T):
        na = np.linalg.norm(k[t])
        nb = np.linalg.norm(k[t - 1])
        r[t] = 1.0 if na == 0 or nb == 0 else 1.0 - float(k[t] @ k[t - 1]) / (na * nb)
    return r


def fenwick_ranges(t):
    """Buckets read by token t: Fenwick blocks of [0, t-1] (one per set bit of t,
    oldest first) and the singleton {t}."""
    out = []
    start = 0
    for b in reversed(range(t.bit_length())):
        if t >> b & 1:
            out.append((start, start + (1 << b) - 1))
            start += 1 << b
    out.append((t, t))
    return out


# ---- information policy (the pages' own decision and merge criteria) --------

INFO_EPS = 1e-6


def info_score_gram(U, V, t, a):
    """Information score of token t against the open state over tokens [a, t-1].

    Written from Gram sums instead of the d_v x d_k matrices: with
    s_t = v_t u_t^T and S = sum_s v_s u_s^T,
    <s_t, S> = sum_s (v_t.v_s)(u_t.u_s), |S|^2 = sum_{s,s'} (v_s.v_s')(u_s.u_s'),
    |s_t|^2 = |v_t|^2 |u_t|^2; N(X) = X / sqrt(|X|^2 / (d_k d_v) + eps), and
    |N(s) - N(S)|^2 = |s|^2/a + |S|^2/b - 2 <s,S>/sqrt(ab) with a, b the two
    RMS denominators squared.
    """
    D2 = U.shape[1] * V.shape[1]
    Ur, Vr = U[a:t], V[a:t]
    x = float(((Vr @ V[t]) * (Ur @ U[t])).sum())
    SS = float(((Vr @ Vr.T) * (Ur @ Ur.T)).sum())
    ss = float(V[t] @ V[t]) * float(U[t] @ U[t])
    ra = ss / D2 + INFO_EPS
    rb = SS / D2 + INFO_EPS
    num2 = ss / ra + SS / rb - 2.0 * x / np.sqrt(ra * rb)
    return float(np.sqrt(max(num2, 0.0)) / (np.sqrt(SS / rb) + INFO_EPS))


def info_simulate(k, v, C, tau):
    """The information policy's decisions from scratch, on token ranges.

    A token with no open state opens one (score 0); otherwise it joins the
    open state when its score is below tau.  Each state is a range with the sum
    of its tokens' scores; at capacity the adjacent sealed pair of least
    (sum_i + sum_{i+1}) / (tokens in both ranges) merges, first minimum on ties.
    Returns (boundary [T], merges [(t, i)], score [T]).
    """
    T = k.shape[0]
    U = phi(k)
    V = np.asarray(v, dtype=np.float64)
    score = np.zeros(T)
    boundary = np.zeros(T, dtype=np.uint8)
    merges = []
    sealed = []  # [first, last, score sum]
    open_ = None
    for t in range(T):
        if open_ is None:
            it, join = 0.0, False
        else:
            it = info_score_gram(U, V, t, open_[0])
            join = it < tau
        score[t] = it
        if not join:
            boundary[t] = 1
            if open_ is not None:
                sealed.append(open_)
            if len(sealed) == C:
                dens = [(sealed[i][2] + sealed[i + 1][2]) / (sealed[i + 1][1] - sealed[i][0] + 1)
                        for i in range(C - 1)]
                i = int(np.argmin(dens))
                sealed[i:i + 2] = [[sealed[i][0], sealed[i + 1][1], sealed[i][2] + sealed[i + 1][2]]]
                merges.append((t, i))
            open_ = [t, t, 0.0]
        open_[1] = t
        open_[2] += it
    return boundary, merges, score

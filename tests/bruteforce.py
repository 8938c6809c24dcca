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

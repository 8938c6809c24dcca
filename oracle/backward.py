"""Gradient of the DLA forward with its decision trace held fixed (test infrastructure).

Only tests/, the package's smoke check and bench.py's CPU baseline use this
module; the CUDA path never imports it.

What it computes (Dynamic Linear Attention | Chlience Paper Archive, section
5.1 for the states, 5.2 for the merges, 5.3 for the readout; section 5.1's
closing note says training uses a soft gate and inference hard segmentation,
and gives no gate form).  Boundaries and merges are piecewise constant in the
keys, so wherever the forward is differentiable its gradient is the one with
the trace held fixed.  With the trace fixed, every token s <= t belongs to
exactly one live state at time t (states are contiguous token ranges), and
the readout of section 5.3 is a masked attention:

    o_t = sum_{s <= t} Lambda[t, s] (phi(q_t) . phi(k_s)) v_s
    Lambda[t, s] = lambda_{t, i(s, t)},  i(s, t) = the live state holding s
    lambda_{t, .] = softmax_i(phi(q_t) . mu_i / sqrt(d_k)),
    mu_i = mean of phi(k_s) over the state's tokens at time t.

Given dO = dL/do, with P[t, s] = phi(q_t) . phi(k_s) and dA[t, s] = dO_t . v_s:

    dlambda_{t, i} = sum_{s in state i} dA[t, s] P[t, s]
    da_{t, i}      = lambda_{t, i} (dlambda_{t, i} - sum_j lambda_{t, j} dlambda_{t, j})
    c[t, s]        = dA[t, s] Lambda[t, s] + da_{t, i(s, t)} / (sqrt(d_k) n_{i(s, t)})
    dphi(q_t)      = sum_s c[t, s] phi(k_s)        (the attention term and the means term)
    dphi(k_s)      = sum_t c[t, s] phi(q_t)
    dv_s           = sum_t Lambda[t, s] P[t, s] dO_t
    dq = dphi(q) * phi'(q),  dk = dphi(k) * phi'(k),  phi'(x) = 1 (x > 0), e^x (x <= 0).

The score's dependence on k only moves the decisions, so it contributes
nothing.  The forward starts from an empty cache.  Everything is fp64 and
written per token, in the order above.
"""
from __future__ import annotations

import numpy as np


def phi(x):
    """elu(x) + 1: x + 1 for x > 0, e^x otherwise."""
    x = np.asarray(x, dtype=np.float64)
    return np.where(x > 0, x + 1.0, np.exp(np.minimum(x, 0.0)))


def dphi(x):
    """Derivative of phi: 1 for x > 0, e^x otherwise."""
    x = np.asarray(x, dtype=np.float64)
    return np.where(x > 0, 1.0, np.exp(np.minimum(x, 0.0)))


def live_starts(boundary, merges):
    """First token of every live state just after token t's decision (the
    states token t's readout sees), in time order, for t = 0 .. T-1.

    boundary: [T] flags of one stream (token 0 of an empty cache is one).
    merges:   (t, i) pairs of that stream in time order: at the boundary t the
              sealed pair (i, i + 1) merged, so state i + 1's start goes away.
    """
    T = len(boundary)
    starts = []
    out = []
    mp = 0
    for t in range(T):
        if boundary[t]:
            if mp < len(merges) and merges[mp][0] == t:
                i = merges[mp][1]
                if not 0 <= i < len(starts) - 1:
                    raise ValueError(f"merge index {i} at token {t} with {len(starts)} sealed states")
                del starts[i + 1]
                mp += 1
            starts.append(t)
        if not starts:
            raise ValueError("token 0 must open a state")
        out.append(list(starts))
    if mp != len(merges):
        raise ValueError("a merge does not fall on a boundary")
    return out


def backward_head(q, k, v, dO, boundary, merges):
    """dq, dk, dv [T, d] of one stream (inputs widened to fp64 by the caller)."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    dO = np.asarray(dO, dtype=np.float64)
    T, dk_ = k.shape
    fq, fk = phi(q), phi(k)
    dfq = np.zeros_like(fq)
    dfk = np.zeros_like(fk)
    dv = np.zeros_like(v)
    rs = 1.0 / np.sqrt(dk_)
    for t, st in enumerate(live_starts(boundary, merges)):
        ends = st[1:] + [t + 1]
        n = np.array([e - s for s, e in zip(st, ends)], dtype=np.float64)
        mu = np.stack([fk[s:e].mean(axis=0) for s, e in zip(st, ends)])
        a = mu @ fq[t] * rs
        lam = np.exp(a - a.max())
        lam /= lam.sum()
        P = fk[:t + 1] @ fq[t]
        dA = v[:t + 1] @ dO[t]
        owner = np.empty(t + 1, dtype=np.int64)
        for i, (s, e) in enumerate(zip(st, ends)):
            owner[s:e] = i
        Lam = lam[owner]
        dlam = np.array([np.dot(dA[s:e], P[s:e]) for s, e in zip(st, ends)])
        da = lam * (dlam - np.dot(lam, dlam))
        c = dA * Lam + (da * rs / n)[owner]
        dfq[t] = c @ fk[:t + 1]
        dfk[:t + 1] += np.outer(c, fq[t])
        dv[:t + 1] += np.outer(Lam * P, dO[t])
    return dfq * dphi(q), dfk * dphi(k), dv


def forward_head(q, k, v, boundary, merges):
    """The same masked form's output [T, d] (the oracle's forward computes it
    from the states; tests compare the two)."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    T, dk_ = k.shape
    fq, fk = phi(q), phi(k)
    o = np.zeros_like(v)
    for t, st in enumerate(live_starts(boundary, merges)):
        ends = st[1:] + [t + 1]
        mu = np.stack([fk[s:e].mean(axis=0) for s, e in zip(st, ends)])
        a = mu @ fq[t] / np.sqrt(dk_)
        lam = np.exp(a - a.max())
        lam /= lam.sum()
        owner = np.empty(t + 1, dtype=np.int64)
        for i, (s, e) in enumerate(zip(st, ends)):
            owner[s:e] = i
        o[t] = (lam[owner] * (fk[:t + 1] @ fq[t])) @ v[:t + 1]
    return o


def backward(q, k, v, dO, boundary, merges):
    """dq, dk, dv [B, H, T, d] for fp64 [B, H, T, d] inputs, the trace's
    boundary flags [B, H, T] and merges (one list of (t, i) per stream, in
    (b, h) order)."""
    B, H, T, d = k.shape
    out = [np.zeros((B, H, T, d)) for _ in range(3)]
    for b in range(B):
        for h in range(H):
            g = backward_head(q[b, h], k[b, h], v[b, h], dO[b, h], boundary[b, h],
                              merges[b * H + h])
            for j in range(3):
                out[j][b, h] = g[j]
    return tuple(out)

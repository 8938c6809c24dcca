"""Seeded synthetic inputs for the DLA hot path (regime-switching keys).

This module is shared by the CUDA path's tests/bench and by the CPU oracle's
callers.  It holds none of the method's arithmetic: it only draws q, k, v.

Recipe (per (batch, head) stream, numpy ``default_rng([seed, b, h])``, all
draws in float32, in this order):

1. ``n_centres`` regime centres ~ N(0, I_d), each normalised to unit length.
2. Regime lengths, drawn in batches until they cover T tokens:
   geometric on {1, 2, ...} with p = 1/mean, or
   lognormal ``max(1, round(exp(N(ln median, sigma_log^2))))``.
3. The first regime's centre is uniform over all centres; each later regime
   draws its centre uniformly from the centres other than the current one.
4. Keys: ``k_t = centre(t) + sigma * N(0, I_d)`` (no re-normalisation).
5. Queries ``q ~ N(0, I)``, then values ``v ~ N(0, I)``.
6. Only with ``value_regimes`` (inputs for the information-score policy, whose
   score compares the token's rank-1 state v phi(k)^T with the open state, so
   values must follow the regimes too): ``n_centres`` value centres ~ N(0, I_d),
   unit-normalised, then ``v_t = value_centre(t) + sigma * N(0, I_d)``,
   replacing the draw of step 5.  These draws come after all others, so the
   other inputs are the same with or without the option.

Decode continuation (the decode-step workload): after the prefill tokens, each
step switches to another centre with probability ``switch_p`` and draws fresh
q, v ~ N(0, I); keys follow step 4.

bf16 tensors are the float32 draws rounded to nearest-even (as raw uint16
bits), so the oracle widens exactly the values the GPU reads.
"""
from __future__ import annotations

import numpy as np

# The five workloads of the DLA hot path (sizes as stated for the method's
# benchmark): tiny fp32 check, bf16 prefill at T=8192, long-context bf16
# prefill at T=131072, a decode step over 256 sequences, and the fixed
# Fenwick-bucket policy compared with DLA at C=16.
WORKLOADS = {
    "tiny_f32": dict(B=1, H=2, T=512, d=32, C=16, tau=0.5, dtype="f32",
                     n_centres=8, lengths=("geometric", 48.0), sigma=0.05,
                     seed=1001),
    "prefill_t8192": dict(B=4, H=16, T=8192, d=128, C=64, tau=0.5,
                          dtype="bf16", n_centres=64,
                          lengths=("geometric", 96.0), sigma=0.05, seed=1002),
    "prefill_t131072": dict(B=1, H=16, T=131072, d=128, C=128, tau=0.5,
                            dtype="bf16", n_centres=64,
                            lengths=("lognormal", 64.0, 1.5), sigma=0.05,
                            seed=1003),
    "decode_n256": dict(B=256, H=16, T=4096, d=128, C=64, tau=0.5,
                        dtype="bf16", n_centres=64,
                        lengths=("geometric", 96.0), sigma=0.05,
                        steps=1024, switch_p=1.0 / 48.0, seed=1004),
    "fixed_t32768": dict(B=2, H=16, T=32768, d=128, C=16, tau=0.5,
                         dtype="bf16", n_centres=64,
                         lengths=("geometric", 96.0), sigma=0.05, seed=1005),
    # DLA(I), no capacity bound, on the T=8192 prefill's sizes with shorter
    # regimes (mean 32): about 460 states per stream by the end (230 live on
    # average), in a cache of 1024 slots
    "unbounded_t8192": dict(B=4, H=16, T=8192, d=128, C=1024, tau=0.5,
                            dtype="bf16", n_centres=64,
                            lengths=("geometric", 32.0), sigma=0.05, seed=1007),
    # the gradient at a forward's decisions (dla_prefill_backward, quadratic
    # in T): the T=8192 prefill's distribution on 16 streams of 2048 tokens
    "backward_t2048": dict(B=1, H=16, T=2048, d=128, C=64, tau=0.5, dtype="bf16",
                           n_centres=64, lengths=("geometric", 96.0), sigma=0.05, seed=1008),
    # the information policy on the T=8192 prefill's sizes; values follow the
    # regimes (recipe step 6) and tau sits between the within-regime score
    # (about 0.6 at d = 128) and the score of a regime switch (about 1.4)
    "info_t8192": dict(B=4, H=16, T=8192, d=128, C=64, tau=1.0,
                       dtype="bf16", n_centres=64,
                       lengths=("geometric", 96.0), sigma=0.05, seed=1006,
                       value_regimes=True),
}


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (nearest-even); returns the uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = u + (np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1)))
    return (r >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bfloat16 bits to float32."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32)
            << np.uint32(16)).view(np.float32)


def _draw_lengths(rng, lengths, total):
    kind = lengths[0]
    out = []
    covered = 0
    while covered < total:
        if kind == "geometric":
            batch = rng.geometric(1.0 / lengths[1], size=256).astype(np.int64)
        elif kind == "lognormal":
            batch = np.rint(rng.lognormal(np.log(lengths[1]), lengths[2],
                                          size=256)).astype(np.int64)
            batch = np.maximum(batch, 1)
        else:
            raise ValueError(f"unknown length law {kind!r}")
        out.append(batch)
        covered += int(batch.sum())
    return np.concatenate(out)


def _centre_sequence(rng, n_regimes, n_centres, first=None):
    seq = np.empty(n_regimes, dtype=np.int64)
    cur = int(rng.integers(n_centres)) if first is None else int(first)
    draws = rng.integers(n_centres - 1, size=n_regimes)
    for i in range(n_regimes):
        if i > 0:
            nxt = int(draws[i])
            cur = nxt + 1 if nxt >= cur else nxt
        seq[i] = cur
    return seq


class HeadStream:
    """One (batch, head) stream: prefill tokens, then optional decode steps."""

    def __init__(self, stream_seed, b, h, *, T, d, n_centres, lengths, sigma,
                 value_regimes=False, **_):
        self.rng = np.random.default_rng([int(stream_seed), int(b), int(h)])
        self.d = d
        self.sigma = np.float32(sigma)
        c = self.rng.standard_normal((n_centres, d), dtype=np.float32)
        c /= np.linalg.norm(c, axis=1, keepdims=True).astype(np.float32)
        self.centres = c.astype(np.float32)
        lens = _draw_lengths(self.rng, lengths, T)
        cseq = _centre_sequence(self.rng, len(lens), n_centres)
        tok_centre = np.repeat(cseq, lens)[:T]
        self.cur = int(tok_centre[-1]) if T > 0 else int(cseq[0])
        noise = self.rng.standard_normal((T, d), dtype=np.float32)
        self.k = self.centres[tok_centre] + self.sigma * noise
        self.q = self.rng.standard_normal((T, d), dtype=np.float32)
        self.v = self.rng.standard_normal((T, d), dtype=np.float32)
        self.vcentres = None
        if value_regimes:
            vc = self.rng.standard_normal((n_centres, d), dtype=np.float32)
            vc /= np.linalg.norm(vc, axis=1, keepdims=True).astype(np.float32)
            self.vcentres = vc.astype(np.float32)
            vnoise = self.rng.standard_normal((T, d), dtype=np.float32)
            self.v = self.vcentres[tok_centre] + self.sigma * vnoise

    def decode_steps(self, steps, switch_p):
        """Keys continue the last regime and switch w.p. switch_p per step."""
        n_centres = self.centres.shape[0]
        sw = self.rng.random(steps) < switch_p
        draws = self.rng.integers(n_centres - 1, size=steps)
        idx = np.empty(steps, dtype=np.int64)
        cur = self.cur
        for s in range(steps):
            if sw[s]:
                nxt = int(draws[s])
                cur = nxt + 1 if nxt >= cur else nxt
            idx[s] = cur
        self.cur = cur
        noise = self.rng.standard_normal((steps, self.d), dtype=np.float32)
        k = self.centres[idx] + self.sigma * noise
        q = self.rng.standard_normal((steps, self.d), dtype=np.float32)
        v = self.rng.standard_normal((steps, self.d), dtype=np.float32)
        if self.vcentres is not None:
            vnoise = self.rng.standard_normal((steps, self.d), dtype=np.float32)
            v = self.vcentres[idx] + self.sigma * vnoise
        return q, k, v


def _cast(x, dtype):
    if dtype == "f32":
        return np.ascontiguousarray(x, dtype=np.float32)
    if dtype == "bf16":
        return to_bf16_bits(x)
    raise ValueError(dtype)


def make_prefill(wl: dict, *, B=None, H=None, T=None, heads=None, seed=None):
    """q, k, v of shape [B, H, T, d] in the workload's dtype.

    ``dtype == 'bf16'`` returns uint16 bit arrays.  ``heads`` (list of (b, h))
    restricts generation to those streams (others are left zero) so a caller
    can draw a sample of a large workload without drawing all of it.
    """
    B = wl["B"] if B is None else B
    H = wl["H"] if H is None else H
    T = wl["T"] if T is None else T
    seed = wl["seed"] if seed is None else seed
    d = wl["d"]
    npdt = np.float32 if wl["dtype"] == "f32" else np.uint16
    q = np.zeros((B, H, T, d), dtype=npdt)
    k = np.zeros_like(q)
    v = np.zeros_like(q)
    todo = heads if heads is not None else [(b, h) for b in range(B) for h in range(H)]
    params = dict(wl, T=T)
    for (b, h) in todo:
        st = HeadStream(seed, b, h, **params)
        q[b, h] = _cast(st.q, wl["dtype"])
        k[b, h] = _cast(st.k, wl["dtype"])
        v[b, h] = _cast(st.v, wl["dtype"])
    return q, k, v


def make_decode(wl: dict, *, N=None, H=None, T=None, steps=None, heads=None,
                seed=None):
    """Prefill q, k, v [N, H, T, d] and per-step q, k, v [steps, N, H, d]."""
    N = wl["B"] if N is None else N
    H = wl["H"] if H is None else H
    T = wl["T"] if T is None else T
    steps = wl["steps"] if steps is None else steps
    seed = wl["seed"] if seed is None else seed
    d = wl["d"]
    npdt = np.float32 if wl["dtype"] == "f32" else np.uint16
    pq = np.zeros((N, H, T, d), dtype=npdt)
    pk = np.zeros_like(pq)
    pv = np.zeros_like(pq)
    sq = np.zeros((steps, N, H, d), dtype=npdt)
    sk = np.zeros_like(sq)
    sv = np.zeros_like(sq)
    todo = heads if heads is not None else [(n, h) for n in range(N) for h in range(H)]
    params = dict(wl, T=T)
    for (n, h) in todo:
        st = HeadStream(seed, n, h, **params)
        pq[n, h] = _cast(st.q, wl["dtype"])
        pk[n, h] = _cast(st.k, wl["dtype"])
        pv[n, h] = _cast(st.v, wl["dtype"])
        q, k, v = st.decode_steps(steps, wl["switch_p"])
        sq[:, n, h] = _cast(q, wl["dtype"])
        sk[:, n, h] = _cast(k, wl["dtype"])
        sv[:, n, h] = _cast(v, wl["dtype"])
    return (pq, pk, pv), (sq, sk, sv)


def widen(x: np.ndarray, dtype: str) -> np.ndarray:
    """Exact float64 copy of an f32 array or of bf16 bits."""
    if dtype == "bf16":
        return bf16_bits_to_f32(x).astype(np.float64)
    return np.asarray(x, dtype=np.float32).astype(np.float64)

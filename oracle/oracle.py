"""ctypes front end of the fp64 CPU oracle (``dla_oracle.c``).

TEST INFRASTRUCTURE ONLY: imported by tests/, by ``__graft_entry__.smoke()``
and by bench.py's cpu_baseline / reference legs.  It never imports the CUDA
package and the CUDA package never imports it.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dla_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

DTYPES = {"f32": 0, "bf16": 1, "f64": 2}
POLICIES = {"dla": 0, "fenwick": 1, "info": 2, "unbounded": 3}


def build(force: bool = False) -> str:
    """Compile the oracle (plain C, -O2, no FP contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
               "-pthread", "-o", _LIB + ".tmp", _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


_lib = None


def load_library(path: str):
    """Load an oracle shared object and declare its C signatures."""
    lib = ctypes.CDLL(path)
    P = ctypes.c_void_p
    lib.dla_oracle_new.restype = P
    lib.dla_oracle_new.argtypes = [ctypes.c_int] * 6
    lib.dla_oracle_free.argtypes = [P]
    lib.dla_oracle_run.restype = ctypes.c_int
    lib.dla_oracle_run.argtypes = [P, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                   ctypes.c_double, ctypes.c_int, P, P, P, P, P, P, P,
                                   P, ctypes.c_int, P, P, ctypes.c_int]
    lib.dla_oracle_run_masked.restype = ctypes.c_int
    lib.dla_oracle_run_masked.argtypes = [P, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                          ctypes.c_double, ctypes.c_int, P, P, P, P, P, P, P,
                                          P, P, ctypes.c_int, P, P, ctypes.c_int]
    lib.dla_oracle_run_scored.restype = ctypes.c_int
    lib.dla_oracle_run_scored.argtypes = [P, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                          ctypes.c_double, ctypes.c_int, P, P, P, P, P, P, P,
                                          P, P, ctypes.c_int, P, P, P, ctypes.c_int]
    lib.dla_oracle_run_forced.restype = ctypes.c_int
    lib.dla_oracle_run_forced.argtypes = [P, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                          ctypes.c_double, ctypes.c_int, P, P, P, P, P, P, P,
                                          P, P, ctypes.c_int, P, P, P, P, P, P, ctypes.c_int,
                                          P, ctypes.c_int]
    lib.dla_oracle_state.restype = ctypes.c_int
    lib.dla_oracle_state.argtypes = [P, ctypes.c_int, ctypes.c_int, P, P, P, P, P, P]
    lib.dla_oracle_state_info.restype = ctypes.c_int
    lib.dla_oracle_state_info.argtypes = [P, ctypes.c_int, ctypes.c_int, P, P, P, P, P, P, P]
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = load_library(build())
    return _lib


def cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


class Oracle:
    """Per-head oracle state that persists across calls (prefill, then steps)."""

    def __init__(self, nheads: int, d_k: int, d_v: int, C: int, policy: str = "dla",
                 want_S: bool = True, lib=None):
        self.lib = _load() if lib is None else lib
        self.nheads, self.d_k, self.d_v, self.C = nheads, d_k, d_v, C
        self.want_S = want_S or policy == "info"
        self.policy = policy
        self.h = self.lib.dla_oracle_new(nheads, d_k, d_v, C, POLICIES[policy], int(self.want_S))

    def __del__(self):
        if getattr(self, "h", None):
            self.lib.dla_oracle_free(self.h)
            self.h = None

    def run(self, k, q=None, v=None, *, tau: float, dtype: str, head_lo: int = 0,
            want_out: bool = True, cap: int | None = None, nthreads: int | None = None,
            out_mask=None, force_merges=None):
        """Run T tokens for heads [head_lo, head_lo + k.shape[0]).

        k, q, v: arrays [nrun, T, d] (float32, float64 or bf16 uint16 bits).
        ``out_mask`` ([T] bool) limits the readout to the marked tokens (rows
        elsewhere stay zero); states are updated at every token regardless.
        Returns dict with out [nrun, T, d_v] (fp64 or None), boundary
        [nrun, T] u8, merges as lists of (t, i) per head, live [nrun, T],
        score [nrun, T] (each token's decision score: r_t, or I_t for the
        information policy) and margins [nrun, 3] (min |score - tau|, min
        relative gap of the merge criterion, exact ties).  The information
        policy needs v even without outputs.

        ``force_merges`` (one list of (t, i) per run head) makes every
        capacity merge take the listed pair instead of the argmin; the result
        then has ``excess`` [nrun]: the largest relative excess of a forced
        pair's merge criterion over the minimum at its merge (0 when every
        forced pair was a minimum, inf when the list does not match the
        capacity merges the decisions call for).
        """
        k = np.ascontiguousarray(k)
        nrun, T = k.shape[0], k.shape[1]
        if want_out:
            q = np.ascontiguousarray(q)
            v = np.ascontiguousarray(v)
        else:
            q = None
            v = np.ascontiguousarray(v) if self.policy == "info" else None
        out = np.zeros((nrun, T, self.d_v), dtype=np.float64) if want_out else None
        boundary = np.zeros((nrun, T), dtype=np.uint8)
        cap = (T + 1) if cap is None else cap
        mt = np.zeros((nrun, max(cap, 1)), dtype=np.int32)
        mi = np.zeros_like(mt)
        mc = np.zeros(nrun, dtype=np.int32)
        live = np.zeros((nrun, T), dtype=np.int32)
        margins = np.zeros((nrun, 3), dtype=np.float64)
        margins[:, 0] = np.inf
        margins[:, 1] = np.inf
        score = np.zeros((nrun, T), dtype=np.float64)
        nthreads = cores() if nthreads is None else nthreads
        if out_mask is not None:
            out_mask = np.ascontiguousarray(out_mask, dtype=np.uint8)
            if out_mask.shape != (T,):
                raise ValueError("out_mask must have shape [T]")
        ft = fi = fc = excess = None
        fcap = 0
        if force_merges is not None:
            if len(force_merges) != nrun:
                raise ValueError("force_merges needs one list per run head")
            fcap = max(1, max(len(m) for m in force_merges))
            ft = np.zeros((nrun, fcap), dtype=np.int32)
            fi = np.zeros((nrun, fcap), dtype=np.int32)
            fc = np.array([len(m) for m in force_merges], dtype=np.int32)
            for r, m in enumerate(force_merges):
                for j, (t_, i_) in enumerate(m):
                    ft[r, j], fi[r, j] = t_, i_
            excess = np.zeros(nrun, dtype=np.float64)
        rc = self.lib.dla_oracle_run_forced(self.h, head_lo, head_lo + nrun, T, float(tau),
                                            DTYPES[dtype], _ptr(q), _ptr(k), _ptr(v), _ptr(out),
                                            _ptr(out_mask), _ptr(boundary), _ptr(mt), _ptr(mi),
                                            _ptr(mc), cap, _ptr(live), _ptr(margins),
                                            _ptr(score), _ptr(ft), _ptr(fi), _ptr(fc), fcap,
                                            _ptr(excess), nthreads)
        if rc != 0:
            raise RuntimeError(f"dla_oracle_run failed with code {rc}")
        merges = [list(zip(mt[r, :min(mc[r], cap)].tolist(), mi[r, :min(mc[r], cap)].tolist()))
                  for r in range(nrun)]
        return dict(out=out, boundary=boundary, merges=merges, merge_count=mc, live=live,
                    margins=margins, score=score, excess=excess)

    def state(self, head: int):
        """Live states of a head in time order: S, z, n, ts, info (score sums),
        prev_r, t."""
        maxm = 64 if self.policy == "fenwick" else self.C
        if self.policy == "unbounded":
            maxm = self.lib.dla_oracle_state_info(self.h, head, 0, None, None, None, None, None,
                                                  None, None)
        S = np.zeros((maxm, self.d_v, self.d_k)) if self.want_S else None
        z = np.zeros((maxm, self.d_k))
        n = np.zeros(maxm, dtype=np.int64)
        ts = np.zeros(maxm, dtype=np.int64)
        info = np.zeros(maxm)
        pr = np.zeros(1)
        t = np.zeros(1, dtype=np.int64)
        m = self.lib.dla_oracle_state_info(self.h, head, maxm, _ptr(S), _ptr(z), _ptr(n),
                                           _ptr(ts), _ptr(info), _ptr(pr), _ptr(t))
        return dict(S=None if S is None else S[:m], z=z[:m], n=n[:m], ts=ts[:m], info=info[:m],
                    prev_r=float(pr[0]), t=int(t[0]), m=m)


def prefill(q, k, v, *, C: int, tau: float, dtype: str, policy: str = "dla",
            want_out: bool = True, nthreads: int | None = None):
    """One-shot oracle over [B, H, T, d] inputs; returns outputs shaped [B, H, ...]."""
    B, H, T, d = k.shape
    d_v = v.shape[-1] if v is not None else d
    orc = Oracle(B * H, d, d_v, C, policy, want_S=want_out)
    res = orc.run(k.reshape(B * H, T, d),
                  None if q is None or not want_out else q.reshape(B * H, T, d),
                  None if v is None else v.reshape(B * H, T, d_v),
                  tau=tau, dtype=dtype, want_out=want_out, nthreads=nthreads)
    if res["out"] is not None:
        res["out"] = res["out"].reshape(B, H, T, d_v)
    res["boundary"] = res["boundary"].reshape(B, H, T)
    res["live"] = res["live"].reshape(B, H, T)
    res["score"] = res["score"].reshape(B, H, T)
    res["oracle"] = orc
    return res

"""Helpers for GPU parity tests: host inputs -> device tensors, oracle runs."""
from __future__ import annotations

import numpy as np
import torch

from dynamic_state_memory_b200 import synth
from oracle import oracle as O

TOL = {"f32": 1e-4, "bf16": 2e-2}


def to_device(x: np.ndarray, dtype: str, device="cuda"):
    if dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).to(device)
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(device)


def from_device(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        return synth.bf16_bits_to_f32(t.view(torch.int16).cpu().numpy().view(np.uint16)).astype(np.float64)
    return t.float().cpu().numpy().astype(np.float64)


def case(B, H, T, d, dtype="f32", seed=7, n_centres=6, mean_len=20.0, lengths=None, sigma=0.05):
    wl = dict(B=B, H=H, T=T, d=d, dtype=dtype, n_centres=n_centres,
              lengths=lengths or ("geometric", mean_len), sigma=sigma, seed=seed)
    return synth.make_prefill(wl)


def oracle_run(q, k, v, C, tau, dtype, policy="dla", want_out=True):
    return O.prefill(q, k, v, C=C, tau=tau, dtype=dtype, policy=policy, want_out=want_out)


def rel_err(o_gpu: np.ndarray, o_ref: np.ndarray) -> float:
    return float(np.abs(o_gpu - o_ref).max() / max(np.abs(o_ref).max(), 1e-30))


def _gen_prefill_head(args):
    wl, b, h = args
    st = synth.HeadStream(wl["seed"], b, h, **wl)
    cast = synth.to_bf16_bits if wl["dtype"] == "bf16" else (lambda x: np.ascontiguousarray(x, np.float32))
    return b, h, cast(st.q), cast(st.k), cast(st.v)


def _gen_decode_head(args):
    wl, b, h = args
    st = synth.HeadStream(wl["seed"], b, h, **wl)
    cast = synth.to_bf16_bits if wl["dtype"] == "bf16" else (lambda x: np.ascontiguousarray(x, np.float32))
    pre = (cast(st.q), cast(st.k), cast(st.v))
    q, k, v = st.decode_steps(wl["steps"], wl["switch_p"])
    return b, h, pre, (cast(q), cast(k), cast(v))


def _pool_map(fn, jobs):
    """Map over a spawn-started process pool (safe after CUDA has been used)."""
    import multiprocessing as mp
    import os
    from concurrent.futures import ProcessPoolExecutor
    workers = max(1, min(len(jobs), len(os.sched_getaffinity(0))))
    if workers == 1:
        return list(map(fn, jobs))
    with ProcessPoolExecutor(workers, mp_context=mp.get_context("spawn")) as ex:
        return list(ex.map(fn, jobs, chunksize=max(1, len(jobs) // (4 * workers))))


def gen_prefill_parallel(wl: dict):
    """The workload's q, k, v [B, H, T, d] (same values as synth.make_prefill)."""
    B, H, T, d = wl["B"], wl["H"], wl["T"], wl["d"]
    npdt = np.uint16 if wl["dtype"] == "bf16" else np.float32
    q = np.empty((B, H, T, d), dtype=npdt)
    k = np.empty_like(q)
    v = np.empty_like(q)
    for b, h, qq, kk, vv in _pool_map(_gen_prefill_head, [(wl, b, h) for b in range(B) for h in range(H)]):
        q[b, h], k[b, h], v[b, h] = qq, kk, vv
    return q, k, v


def gen_decode_parallel(wl: dict, steps: int):
    """Prefill q, k, v [N, H, T, d] and step q, k, v [steps, N, H, d] (as synth.make_decode)."""
    wl = dict(wl, steps=steps)
    N, H, T, d = wl["B"], wl["H"], wl["T"], wl["d"]
    npdt = np.uint16 if wl["dtype"] == "bf16" else np.float32
    pre = [np.empty((N, H, T, d), dtype=npdt) for _ in range(3)]
    stp = [np.empty((steps, N, H, d), dtype=npdt) for _ in range(3)]
    for b, h, p, s in _pool_map(_gen_decode_head, [(wl, n, h) for n in range(N) for h in range(H)]):
        for i in range(3):
            pre[i][b, h] = p[i]
            stp[i][:, b, h] = s[i]
    return tuple(pre), tuple(stp)

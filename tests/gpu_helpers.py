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

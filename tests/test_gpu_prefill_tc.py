"""GPU parity of the tensor-core prefill path (bf16 inputs, d = 128).

Trace bit-exact, outputs within 2e-2 of max|o| against the fp64 oracle, on
small shapes that cover ragged tails, several windows, capacity 2..128 and
degenerate tiles (every token a boundary, every token a merge).
"""
import numpy as np
import pytest

from tests.gpu_helpers import TOL, case, from_device, oracle_run, rel_err, to_device

pytestmark = pytest.mark.gpu


def gpu_prefill(q, k, v, C, tau, window=0):
    import torch
    from dynamic_state_memory_b200 import dla
    B, H, T, d = k.shape
    cache = dla.Cache(B, H, C, d)
    o, tr = dla.prefill(to_device(q, "bf16"), to_device(k, "bf16"), to_device(v, "bf16"), cache,
                        tau, window=window)
    torch.cuda.synchronize()
    return from_device(o), tr


def check(q, k, v, C, tau, window=0):
    B, H, T, d = k.shape
    ref = oracle_run(q, k, v, C, tau, "bf16")
    o, tr = gpu_prefill(q, k, v, C, tau, window)
    assert np.array_equal(tr.boundary.cpu().numpy().reshape(B, H, T), ref["boundary"])
    assert tr.merges() == ref["merges"]
    err = rel_err(o, ref["out"])
    assert err <= TOL["bf16"], err
    return err


@pytest.mark.parametrize("T", [1, 100, 128, 129, 300, 700])
def test_ragged_lengths(gpu, T):
    q, k, v = case(1, 2, T, 128, "bf16", seed=T, mean_len=30.0)
    check(q, k, v, 8, 0.5)


@pytest.mark.parametrize("C", [2, 4, 16, 64, 128])
def test_capacities(gpu, C):
    q, k, v = case(1, 2, 900, 128, "bf16", seed=C, mean_len=6.0)
    check(q, k, v, C, 0.5)


@pytest.mark.parametrize("window", [128, 256, 384])
def test_windows(gpu, window):
    q, k, v = case(2, 2, 777, 128, "bf16", seed=window, mean_len=12.0)
    check(q, k, v, 6, 0.5, window)


@pytest.mark.parametrize("C", [3, 128])
def test_every_token_a_boundary(gpu, C):
    # tau = 0: 128 pieces per tile, a merge at every token once C states exist
    q, k, v = case(1, 2, 400, 128, "bf16", seed=11)
    check(q, k, v, C, 0.0)


def test_single_state(gpu):
    q, k, v = case(1, 2, 500, 128, "bf16", seed=12)
    check(q, k, v, 4, 2.5)


def test_many_heads_regime_switching(gpu):
    q, k, v = case(3, 5, 1100, 128, "bf16", seed=13, n_centres=16, mean_len=40.0)
    check(q, k, v, 16, 0.5)

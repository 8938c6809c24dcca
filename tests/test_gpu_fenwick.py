"""GPU parity of dla_fixed_policy_prefill (Fenwick buckets) against the
oracle's fixed policy: outputs within the dtype's tolerance of max|o|."""
import numpy as np
import pytest

from tests.gpu_helpers import TOL, case, from_device, oracle_run, rel_err, to_device

pytestmark = pytest.mark.gpu


def run(q, k, v, dtype):
    import torch
    from dynamic_state_memory_b200 import dla
    o = dla.fixed_policy_prefill(to_device(q, dtype), to_device(k, dtype), to_device(v, dtype))
    torch.cuda.synchronize()
    return from_device(o)


@pytest.mark.parametrize("T", [1, 100, 128, 129, 300, 1000, 2100])
def test_fenwick_bf16_d128(gpu, T):
    q, k, v = case(1, 2, T, 128, "bf16", seed=T + 1)
    ref = oracle_run(q, k, v, 2, 0.5, "bf16", policy="fenwick")
    assert rel_err(run(q, k, v, "bf16"), ref["out"]) <= TOL["bf16"]


@pytest.mark.parametrize("d,dtype", [(32, "f32"), (64, "f32"), (64, "bf16")])
def test_fenwick_simt(gpu, d, dtype):
    q, k, v = case(2, 2, 777, d, dtype, seed=d)
    ref = oracle_run(q, k, v, 2, 0.5, dtype, policy="fenwick")
    assert rel_err(run(q, k, v, dtype), ref["out"]) <= TOL[dtype]


def test_fenwick_more_tiles_than_sms(gpu):
    """160 streams x 8 tiles: the atom loop's CTAs each walk about nine tiles
    whose atom counts (the popcounts of the tile indices) run 0, 1, 1, 2, ...
    so a CTA often meets a tile with no atom or one between busier ones."""
    q, k, v = case(4, 40, 1024, 128, "bf16", seed=5)
    ref = oracle_run(q, k, v, 2, 0.5, "bf16", policy="fenwick")
    assert rel_err(run(q, k, v, "bf16"), ref["out"]) <= TOL["bf16"]


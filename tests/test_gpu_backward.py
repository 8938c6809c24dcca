"""GPU parity of dla_prefill_backward with the oracle's gradient
(oracle/backward.py): the gradient of the forward with its decision trace
held fixed.  The forward runs on the GPU (dla_prefill from empty caches); its
trace must equal the C oracle's bit for bit, and the oracle's gradient is
taken at the oracle's own trace.  dq, dk, dv are compared element by element
within 1e-4 of max|grad| (fp32 arithmetic on both input dtypes: bf16 inputs
widen exactly on both sides).
"""
import numpy as np
import pytest

from oracle import backward as BW
from oracle import oracle as O
from tests.gpu_helpers import case, from_device, to_device
from dynamic_state_memory_b200 import synth

pytestmark = pytest.mark.gpu

TOL = 1e-4


def run_case(B, H, T, d, C, dtype, seed, tau=0.5, mean_len=12.0):
    import torch
    from dynamic_state_memory_b200 import dla
    q, k, v = case(B, H, T, d, dtype, seed=seed, mean_len=mean_len)
    rng = np.random.default_rng(seed + 1)
    dO = rng.standard_normal((B, H, T, d)).astype(np.float32)
    if dtype == "bf16":
        dO = synth.to_bf16_bits(dO)
    qd, kd, vd, dod = (to_device(x, dtype) for x in (q, k, v, dO))
    cache = dla.Cache(B, H, C, d)
    _, tr = dla.prefill(qd, kd, vd, cache, tau)
    dq, dk, dv = dla.prefill_backward(qd, kd, vd, dod, tr, C)
    torch.cuda.synchronize()
    # the oracle's own decisions, then its gradient at them
    ref = O.prefill(q, k, v, C=C, tau=tau, dtype=dtype, want_out=False)
    assert np.array_equal(tr.boundary.cpu().numpy().reshape(B, H, T), ref["boundary"])
    assert tr.merges() == ref["merges"]
    w = lambda x: synth.widen(x, dtype)
    gq, gk, gv = BW.backward(w(q), w(k), w(v), w(dO), ref["boundary"], ref["merges"])
    for name, got, want in (("dq", dq, gq), ("dk", dk, gk), ("dv", dv, gv)):
        got = got.cpu().numpy().astype(np.float64)
        err = np.abs(got - want).max() / max(np.abs(want).max(), 1e-30)
        assert err <= TOL, (name, err)
    return ref


@pytest.mark.parametrize("B,H,T,d,C,dtype", [
    (1, 2, 1, 32, 2, "f32"),
    (1, 2, 100, 32, 4, "f32"),
    (2, 2, 300, 64, 4, "f32"),
    (1, 3, 129, 128, 2, "bf16"),
    (2, 2, 700, 128, 16, "bf16"),
    (1, 2, 400, 128, 64, "bf16"),
])
def test_backward_matches_oracle(gpu, B, H, T, d, C, dtype):
    ref = run_case(B, H, T, d, C, dtype, seed=T + C)
    if T > 1 and C < 64:
        assert any(ref["merges"]), "the case should merge"


def test_backward_every_token_a_boundary(gpu):
    # tau = 0: no score is below it, every token opens a state and (C = 3)
    # nearly every token merges
    run_case(1, 2, 200, 64, 3, "f32", seed=5, tau=0.0)


def test_backward_longer_streams(gpu):
    run_case(1, 4, 2048, 128, 64, "bf16", seed=9, mean_len=96.0)


def test_backward_rejects_a_trace_off_its_boundaries(gpu):
    import torch
    from dynamic_state_memory_b200 import dla
    B, H, T, d, C = 1, 2, 300, 64, 3
    q, k, v = case(B, H, T, d, "f32", seed=3)
    qd, kd, vd = (to_device(x, "f32") for x in (q, k, v))
    cache = dla.Cache(B, H, C, d)
    _, tr = dla.prefill(qd, kd, vd, cache, 0.5)
    b = tr.boundary.cpu().numpy()
    n = int(tr.merge_count[0].item())
    assert n > 0
    off = int(np.flatnonzero(b[0] == 0)[-1])      # a token that opened no state
    tr.merge_t[0, n - 1] = off
    with pytest.raises(dla.DlaError) as e:
        dla.prefill_backward(qd, kd, vd, qd, tr, C)
    assert e.value.code == 1  # DLA_ERR_INVALID_ARG, from the device

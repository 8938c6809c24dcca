"""GPU parity of dla_decode_step: prefill T1 tokens, then T2 single-token
steps, against the oracle run over the same T1 + T2 tokens (trace bit-exact,
outputs within tolerance), and decode-only sequences from an empty cache."""
import numpy as np
import pytest

from tests.gpu_helpers import TOL, case, from_device, oracle_run, rel_err, to_device

pytestmark = pytest.mark.gpu


def run(q, k, v, C, tau, dtype, T1):
    import torch
    from dynamic_state_memory_b200 import dla
    B, H, T, d = k.shape
    cache = dla.Cache(B, H, C, d)
    outs, bnd, mrg = [], [], []
    if T1 > 0:
        o, tr = dla.prefill(to_device(q[:, :, :T1], dtype), to_device(k[:, :, :T1], dtype),
                            to_device(v[:, :, :T1], dtype), cache, tau)
        outs.append(from_device(o))
        bnd.append(tr.boundary.cpu().numpy().reshape(B, H, T1))
        merges = tr.merges()
    else:
        merges = [[] for _ in range(B * H)]
    dec = dla.Decoder(cache)
    for t in range(T1, T):
        o = dec.step(to_device(np.ascontiguousarray(q[:, :, t]), dtype),
                     to_device(np.ascontiguousarray(k[:, :, t]), dtype),
                     to_device(np.ascontiguousarray(v[:, :, t]), dtype), tau)
        torch.cuda.synchronize()
        dla.check_device_status(dec.status, "decode")
        outs.append(from_device(o)[:, :, None])
        bnd.append(dec.boundary.cpu().numpy().reshape(B, H, 1))
        mi = dec.merge_i.cpu().numpy()
        for u in range(B * H):
            if mi[u] >= 0:
                merges[u].append((t, int(mi[u])))
    return np.concatenate(outs, axis=2), np.concatenate(bnd, axis=2), merges


@pytest.mark.parametrize("d,dtype", [(32, "f32"), (64, "bf16"), (128, "bf16"), (128, "f32")])
@pytest.mark.parametrize("T1", [0, 37, 130])
def test_prefill_then_decode(gpu, d, dtype, T1):
    q, k, v = case(2, 2, T1 + 60, d, dtype, seed=d + T1, mean_len=10.0)
    ref = oracle_run(q, k, v, 4, 0.5, dtype)
    o, bnd, merges = run(q, k, v, 4, 0.5, dtype, T1)
    assert np.array_equal(bnd, ref["boundary"])
    assert merges == ref["merges"]
    assert rel_err(o, ref["out"]) <= TOL[dtype]


def test_decode_singletons_every_step_merges(gpu):
    q, k, v = case(1, 3, 50, 128, "f32", seed=1)
    ref = oracle_run(q, k, v, 3, 0.0, "f32")
    o, bnd, merges = run(q, k, v, 3, 0.0, "f32", 5)
    assert bnd.all()
    assert merges == ref["merges"]
    assert rel_err(o, ref["out"]) <= TOL["f32"]

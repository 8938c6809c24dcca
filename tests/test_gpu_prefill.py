"""GPU parity of dla_prefill against the CPU oracle (same seeded inputs).

The decision trace (boundary flags, merge tokens and pair indices) must be
bit-identical; outputs must match within 1e-4 (fp32) or 2e-2 (bf16) of
max|o|.
"""
import numpy as np
import pytest

from dynamic_state_memory_b200 import synth
from tests.gpu_helpers import TOL, case, from_device, oracle_run, rel_err, to_device

pytestmark = pytest.mark.gpu


def run_gpu(q, k, v, C, tau, dtype, window=0, cache=None, d=None):
    import torch
    from dynamic_state_memory_b200 import dla
    B, H, T, dd = k.shape
    if cache is None:
        cache = dla.Cache(B, H, C, dd)
    o, tr = dla.prefill(to_device(q, dtype), to_device(k, dtype), to_device(v, dtype), cache, tau,
                        window=window)
    torch.cuda.synchronize()
    return from_device(o), tr, cache


def check(q, k, v, C, tau, dtype, window=0):
    B, H, T, d = k.shape
    ref = oracle_run(q, k, v, C, tau, dtype)
    o, tr, cache = run_gpu(q, k, v, C, tau, dtype, window)
    bnd = tr.boundary.cpu().numpy().reshape(B, H, T)
    assert np.array_equal(bnd, ref["boundary"]), "boundary flags differ"
    assert tr.merges() == ref["merges"], "merge trace differs"
    err = rel_err(o, ref["out"])
    assert err <= TOL[dtype], f"max error {err:.3e} > {TOL[dtype]}"
    return ref, cache, err


@pytest.mark.parametrize("d", [32, 64, 128])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_small_ragged(gpu, d, dtype):
    q, k, v = case(1, 2, 300, d, dtype, seed=d)
    check(q, k, v, 4, 0.5, dtype)


@pytest.mark.parametrize("window", [64, 128, 192])
def test_windows_do_not_change_results(gpu, window):
    q, k, v = case(2, 2, 500, 32, "f32", seed=3)
    check(q, k, v, 5, 0.5, "f32", window=window)


@pytest.mark.parametrize("C", [2, 3, 16])
@pytest.mark.parametrize("tau", [0.3, 0.5, 1.0])
def test_capacity_and_threshold_grid(gpu, C, tau):
    q, k, v = case(1, 3, 257, 32, "f32", seed=C * 10 + int(tau * 10), mean_len=8.0)
    check(q, k, v, C, tau, "f32")


def test_tiny_f32_workload(gpu):
    wl = synth.WORKLOADS["tiny_f32"]
    q, k, v = synth.make_prefill(wl)
    ref, _, err = check(q, k, v, wl["C"], wl["tau"], "f32")
    assert ref["merge_count"].sum() > 0


def test_all_singletons(gpu):
    # tau = 0: every token opens a state; C < T forces a merge at every token.
    q, k, v = case(1, 2, 200, 32, "f32", seed=5)
    check(q, k, v, 8, 0.0, "f32")


def test_single_state(gpu):
    q, k, v = case(1, 2, 333, 64, "f32", seed=6)
    check(q, k, v, 4, 2.5, "f32")


def test_split_calls_equal_one_call(gpu):
    import torch
    from dynamic_state_memory_b200 import dla
    q, k, v = case(1, 2, 400, 32, "f32", seed=9)
    o_one, tr_one, _ = run_gpu(q, k, v, 4, 0.5, "f32")
    cache = dla.Cache(1, 2, 4, 32)
    outs, bnds = [], []
    for a, b in ((0, 150), (150, 151), (151, 400)):
        o, tr = dla.prefill(to_device(q[:, :, a:b], "f32"), to_device(k[:, :, a:b], "f32"),
                            to_device(v[:, :, a:b], "f32"), cache, 0.5)
        outs.append(from_device(o))
        bnds.append(tr.boundary.cpu().numpy())
    o_split = np.concatenate(outs, axis=2)
    assert np.array_equal(np.concatenate(bnds, axis=1), tr_one.boundary.cpu().numpy())
    assert np.abs(o_split - o_one).max() <= 1e-5 * np.abs(o_one).max()


def test_cache_matches_oracle_state(gpu):
    import torch
    q, k, v = case(1, 2, 350, 32, "f32", seed=12)
    ref, cache, _ = check(q, k, v, 6, 0.5, "f32")
    orc = ref["oracle"]
    vw = cache.views()
    for h in range(2):
        st = orc.state(h)
        m = int(vw["m"][0, h])
        assert m == st["m"]
        order = vw["order"][0, h, :m].cpu().numpy()
        assert vw["ts"][0, h].cpu().numpy()[order].tolist() == st["ts"].tolist()
        assert vw["n"][0, h].cpu().numpy()[order].tolist() == st["n"].tolist()
        S = vw["S"][0, h].cpu().numpy()[order].astype(np.float64)
        assert np.abs(S - st["S"]).max() <= 1e-4 * np.abs(st["S"]).max()
        z = vw["z"][0, h].cpu().numpy()[order]
        assert np.allclose(z, st["z"], rtol=1e-12)
        assert int(vw["t"][0, h]) == 350

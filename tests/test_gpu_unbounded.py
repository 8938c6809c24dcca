"""GPU parity of DLA(I), the unbounded policy (dla_unbounded_prefill).

The ablation row "Mamba-2 + DLA(I)" of the Dynamic Linear Attention |
Chlience Paper Archive page: the dynamic decisions with no capacity merge, so
every segment stays a state and the readout's softmax runs over all of them.
Boundaries must equal the oracle's bit for bit and no merge may occur;
outputs within 1e-4 (fp32) or 2e-2 (bf16) of max|o|.  Short regimes give
hundreds of states per stream, past the 128 atoms one chunk of the
tensor-core prologue and atom loop holds.
"""
import numpy as np
import pytest

from dynamic_state_memory_b200 import synth
from oracle import oracle as O
from tests.gpu_helpers import TOL, case, from_device, gen_prefill_parallel, rel_err, to_device

pytestmark = pytest.mark.gpu


def run(q, k, v, C, tau, dtype, window=0, split=None):
    import torch
    from dynamic_state_memory_b200 import dla
    B, H, T, d = k.shape
    cache = dla.Cache(B, H, C, d)
    parts = [(0, T)] if split is None else [(0, split), (split, T)]
    outs, bnds = [], []
    for a, b in parts:
        o, tr = dla.unbounded_prefill(*(to_device(np.ascontiguousarray(x[:, :, a:b]), dtype)
                                        for x in (q, k, v)), cache, tau, window=window)
        assert tr.merge_count.cpu().sum() == 0
        outs.append(from_device(o))
        bnds.append(tr.boundary.cpu().numpy().reshape(B, H, b - a))
    torch.cuda.synchronize()
    return np.concatenate(outs, axis=2), np.concatenate(bnds, axis=2), cache


def oracle(q, k, v, tau, dtype):
    return O.prefill(q, k, v, C=2, tau=tau, dtype=dtype, policy="unbounded")


@pytest.mark.parametrize("d,dtype", [(128, "bf16"), (32, "f32"), (64, "bf16")])
@pytest.mark.parametrize("T", [1, 37, 300, 700])
def test_small(gpu, d, dtype, T):
    q, k, v = case(2, 2, T, d, dtype, seed=T + d, mean_len=3.0)
    ref = oracle(q, k, v, 0.5, dtype)
    C = 448 if dtype == "f32" or d != 128 else 1024
    o, bnd, _ = run(q, k, v, C, 0.5, dtype)
    assert np.array_equal(bnd, ref["boundary"])
    assert ref["live"].max() <= C
    assert rel_err(o, ref["out"]) <= TOL[dtype]


def test_hundreds_of_states_per_tile(gpu):
    """Every token its own state (tau = 0): m0 reaches the 700 states of the
    sequence, several 128-atom chunks per tile."""
    q, k, v = case(1, 2, 700, 128, "bf16", seed=5, mean_len=40.0)
    ref = oracle(q, k, v, 0.0, "bf16")
    assert ref["live"].max() == 700
    o, bnd, _ = run(q, k, v, 1024, 0.0, "bf16")
    assert bnd.all()
    assert rel_err(o, ref["out"]) <= TOL["bf16"]


@pytest.mark.parametrize("window,split", [(256, None), (0, 333), (128, 200)])
def test_windows_and_split_calls(gpu, window, split):
    q, k, v = case(1, 3, 600, 128, "bf16", seed=17, mean_len=4.0)
    ref = oracle(q, k, v, 0.5, "bf16")
    o, bnd, _ = run(q, k, v, 512, 0.5, "bf16", window=window, split=split)
    assert np.array_equal(bnd, ref["boundary"])
    assert rel_err(o, ref["out"]) <= TOL["bf16"]


def test_cache_matches_oracle_states(gpu):
    B, H, T, d = 1, 2, 260, 32
    q, k, v = case(B, H, T, d, "f32", seed=23, mean_len=5.0)
    res = oracle(q, k, v, 0.5, "f32")
    _, _, cache = run(q, k, v, 128, 0.5, "f32")
    vw = cache.views()
    for h in range(H):
        st = res["oracle"].state(h)
        m = int(vw["m"][0, h])
        assert m == st["m"] and int(vw["t"][0, h]) == T
        order = vw["order"][0, h, :m].cpu().numpy()
        assert vw["n"][0, h].cpu().numpy()[order].tolist() == st["n"].tolist()
        assert vw["ts"][0, h].cpu().numpy()[order].tolist() == st["ts"].tolist()
        S = vw["S"][0, h].cpu().numpy().astype(np.float64)[order]
        assert np.abs(S - st["S"]).max() <= 1e-4 * np.abs(st["S"]).max()
        z = vw["z"][0, h].cpu().numpy()[order]
        assert np.abs(z - st["z"]).max() <= 1e-9 * np.abs(st["z"]).max()


def test_capacity_exceeded_is_reported(gpu):
    import torch
    from dynamic_state_memory_b200 import dla
    q, k, v = case(1, 2, 200, 32, "f32", seed=29, mean_len=3.0)
    cache = dla.Cache(1, 2, 8, 32)
    with pytest.raises(dla.DlaError) as ei:
        dla.unbounded_prefill(*(to_device(x, "f32") for x in (q, k, v)), cache, 0.5)
    assert ei.value.code == 8  # DLA_ERR_CAPACITY
    torch.cuda.synchronize()


def test_other_policies_caches_are_refused(gpu):
    from dynamic_state_memory_b200 import dla
    q, k, v = (to_device(x, "f32") for x in case(1, 2, 60, 32, "f32", seed=31, mean_len=5.0))
    c1 = dla.Cache(1, 2, 64, 32)
    dla.unbounded_prefill(q, k, v, c1, 0.5)
    with pytest.raises(dla.DlaError) as ei:       # capacity-bounded prefill on a DLA(I) cache
        dla.prefill(q, k, v, c1, 0.5)
    assert ei.value.code == 2
    c2 = dla.Cache(1, 2, 64, 32)
    dla.prefill(q, k, v, c2, 0.5)
    with pytest.raises(dla.DlaError) as ei:       # DLA(I) does not continue another policy
        dla.unbounded_prefill(q, k, v, c2, 0.5)
    assert ei.value.code == 2


def test_unbounded_full_size(gpu):
    """unbounded_t8192 (every stream, the benchmark's launch configuration):
    every stream's boundaries bit for bit, no merge, hundreds of states per
    stream; two streams' outputs at sampled tokens."""
    import torch
    from dynamic_state_memory_b200 import dla
    from tests.test_gpu_fullsize import sample_mask
    wl = synth.WORKLOADS["unbounded_t8192"]
    q, k, v = gen_prefill_parallel(wl)
    B, H, T, d = k.shape
    cache = dla.Cache(B, H, wl["C"], d)
    o, tr = dla.unbounded_prefill(to_device(q, "bf16"), to_device(k, "bf16"), to_device(v, "bf16"),
                                  cache, wl["tau"])
    torch.cuda.synchronize()
    o = from_device(o)
    orc = O.Oracle(B * H, d, d, 2, "unbounded", want_S=False)
    res = orc.run(k.reshape(B * H, T, d), tau=wl["tau"], dtype="bf16", want_out=False)
    assert np.array_equal(tr.boundary.cpu().numpy().reshape(B * H, T), res["boundary"])
    assert int(tr.merge_count.cpu().sum()) == 0
    live = res["live"][:, -1]
    assert live.min() >= 200 and live.max() <= wl["C"], (live.min(), live.max())
    mask = sample_mask(T, wl["seed"])
    for (b, h) in [(0, 0), (3, 15)]:
        ro = O.Oracle(1, d, d, 2, "unbounded")
        ref = ro.run(k[b, h][None], q[b, h][None], v[b, h][None], tau=wl["tau"], dtype="bf16",
                     out_mask=mask)["out"][0][mask.astype(bool)]
        got = o[b, h][mask.astype(bool)]
        err = float(np.abs(got - ref).max() / max(np.abs(ref).max(), 1e-30))
        assert err <= TOL["bf16"], (b, h, err)

"""GPU parity of the information policy (dla_info_policy_prefill).

The pages' own decision and merge rule (Dynamic Linear Attention | Chlience
Paper Archive, section 5.1 and section 5.2): boundaries and merges must equal
the fp64 oracle's wherever no score lies within the kernel's rounding of tau
and no two pair densities within rounding of each other (the oracle reports
both margins and each case asserts them); outputs within 1e-4 (fp32) or 2e-2
(bf16) of max|o|.  Inputs draw values from per-regime centres, so the state
score sees the regime switches.
"""
import numpy as np
import pytest

from dynamic_state_memory_b200 import synth
from tests.gpu_helpers import TOL, from_device, rel_err, to_device

pytestmark = pytest.mark.gpu

# the kernel's scores agree with the oracle's to ~1e-7 near I = 0 and far
# better elsewhere; a case is compared decision by decision when its margins
# exceed these
SCORE_MARGIN = 1e-6
DENSITY_GAP = 1e-6


def tau_for(d):
    # value noise adds up over d: within a regime the score is about 0.2
    # (d = 32) to 0.6 (d = 128), across a regime switch about 1.4
    return 1.0 if d == 128 else 0.5


def info_case(B, H, T, d, dtype, seed, mean_len=20.0, n_centres=6):
    wl = dict(B=B, H=H, T=T, d=d, dtype=dtype, n_centres=n_centres,
              lengths=("geometric", mean_len), sigma=0.05, seed=seed, value_regimes=True)
    return synth.make_prefill(wl)


def check(q, k, v, C, tau, dtype, window=0):
    import torch
    from dynamic_state_memory_b200 import dla
    from oracle import oracle as O
    B, H, T, d = k.shape
    ref = O.prefill(q, k, v, C=C, tau=tau, dtype=dtype, policy="info")
    mg = ref["margins"]
    assert mg[:, 0].min() > SCORE_MARGIN, mg
    assert mg[:, 2].max() == 0 and mg[:, 1].min() > DENSITY_GAP, mg
    cache = dla.Cache(B, H, C, d)
    o, tr = dla.info_prefill(to_device(q, dtype), to_device(k, dtype), to_device(v, dtype), cache,
                             tau, window=window)
    torch.cuda.synchronize()
    assert np.array_equal(tr.boundary.cpu().numpy().reshape(B, H, T), ref["boundary"])
    assert tr.merges() == ref["merges"]
    err = rel_err(from_device(o), ref["out"])
    assert err <= TOL[dtype], err
    return ref, cache


@pytest.mark.parametrize("d,dtype", [(32, "f32"), (64, "f32"), (64, "bf16"), (128, "bf16"),
                                     (128, "f32")])
@pytest.mark.parametrize("T", [1, 37, 130, 300])
def test_small_ragged(gpu, d, dtype, T):
    q, k, v = info_case(1, 2, T, d, dtype, seed=T + d)
    check(q, k, v, 4, tau_for(d), dtype)


@pytest.mark.parametrize("C", [2, 3, 16])
@pytest.mark.parametrize("tau", [0.8, 1.0, 1.2])
def test_capacity_and_threshold_grid(gpu, C, tau):
    q, k, v = info_case(1, 2, 400, 128, "bf16", seed=10 * C + int(10 * tau), mean_len=10.0)
    check(q, k, v, C, tau, "bf16")


@pytest.mark.parametrize("window", [128, 256])
def test_windows_carry_the_open_state(gpu, window):
    q, k, v = info_case(2, 2, 700, 128, "bf16", seed=window, mean_len=25.0)
    check(q, k, v, 6, 1.0, "bf16", window)


def test_states_match_oracle(gpu):
    # the cache after the call: counts, first tokens and time order of the
    # oracle's states
    from oracle import oracle as O
    q, k, v = info_case(1, 2, 500, 64, "f32", seed=3, mean_len=15.0)
    ref, cache = check(q, k, v, 5, 0.5, "f32")
    orc = ref["oracle"]
    vw = cache.views()
    for h in range(2):
        st = orc.state(h)
        m = int(vw["m"][0, h])
        order = vw["order"][0, h, :m].cpu().numpy()
        assert m == st["m"]
        assert vw["n"][0, h].cpu().numpy()[order].tolist() == st["n"].tolist()
        assert vw["ts"][0, h].cpu().numpy()[order].tolist() == st["ts"].tolist()


def test_every_token_a_boundary(gpu):
    # tau = 0: every score is >= 0, so every token opens a state and merges
    # run at every token once C states exist
    q, k, v = info_case(1, 2, 300, 128, "bf16", seed=5)
    from oracle import oracle as O
    ref = O.prefill(q, k, v, C=3, tau=0.0, dtype="bf16", policy="info")
    assert ref["boundary"].all()
    check(q, k, v, 3, 0.0, "bf16")


def test_nonempty_cache_is_refused(gpu):
    import torch
    from dynamic_state_memory_b200 import dla
    q, k, v = (to_device(x, "f32") for x in info_case(1, 1, 40, 32, "f32", seed=1))
    cache = dla.Cache(1, 1, 4, 32)
    dla.prefill(q, k, v, cache, 0.5)  # the dynamic policy leaves t = 40
    with pytest.raises(dla.DlaError) as ei:
        dla.info_prefill(q, k, v, cache, 0.5)
    assert ei.value.code == 2


def test_info_cache_is_refused_by_the_cosine_policy(gpu):
    """After the information policy, the cache's pair entries are densities
    and prev_r an information score: dla_prefill and both decode steps report
    DLA_ERR_UNSUPPORTED on it until dla_cache_init resets it."""
    import torch
    from dynamic_state_memory_b200 import dla
    q, k, v = (to_device(x, "f32") for x in info_case(1, 2, 40, 32, "f32", seed=3))
    cache = dla.Cache(1, 2, 4, 32)
    dla.info_prefill(q, k, v, cache, 0.5)
    assert float(cache.views()["pair_loss"][0, 0, 3]) == -1.0
    with pytest.raises(dla.DlaError) as ei:
        dla.prefill(q, k, v, cache, 0.5)
    assert ei.value.code == 2
    cache2 = dla.Cache(1, 2, 4, 32)
    dla.info_prefill(q, k, v, cache2, 0.5)
    dec = dla.Decoder(cache2)
    dec.step(q[:, :, 0].contiguous(), k[:, :, 0].contiguous(), v[:, :, 0].contiguous(), 0.5)
    torch.cuda.synchronize()
    assert int(dec.status.item()) == 2
    cache3 = dla.Cache(1, 2, 4, 32)
    dla.info_prefill(q, k, v, cache3, 0.5)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    o = torch.empty(1, 2, 32, device="cuda")
    dla.dla_decode_step_static(cache3.c, 0.5, dla.DLA_F32, q[:, :, 0].contiguous(),
                               k[:, :, 0].contiguous(), v[:, :, 0].contiguous(), o, None, None, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 2
    # a reset cache is the cosine policy's again
    dla.dla_cache_init(cache.c, 1, 2, 4, 32, 32, cache.base)
    dla.prefill(q, k, v, cache, 0.5)

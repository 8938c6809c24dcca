"""dla_trace_stats: the device summary of a prefill's decision trace against
the oracle's per-token live counts (states read by each token) and its
boundaries and merges, for fresh caches, a continued cache, ragged lengths
and DLA(I)."""
import numpy as np
import pytest

from oracle import oracle as O
from tests.gpu_helpers import case, to_device

pytestmark = pytest.mark.gpu


def expect(live, boundary, merges, tile=128):
    T = live.shape[-1]
    rows = sum(min(tile, T - c * tile) * int(live[c * tile - 1]) for c in range(1, (T + tile - 1) // tile))
    return dict(boundaries=int(boundary.sum()), merges=len(merges), live_sum=int(live.sum()),
                live_max=int(live.max()) if T else 0, atom_rows=rows)


def check(stats, res, u, tile=128, live_slice=slice(None)):
    live = res["live"].reshape(-1, res["live"].shape[-1])[u][live_slice]
    bnd = res["boundary"].reshape(-1, res["boundary"].shape[-1])[u][live_slice]
    want = expect(live, bnd, res["merges"][u], tile)
    got = dict(boundaries=int(stats.boundaries[u]), merges=int(stats.merges[u]),
               live_sum=int(stats.live_sum[u]), live_max=int(stats.live_max[u]),
               atom_rows=int(stats.atom_rows[u]))
    assert got == want, (u, got, want)


@pytest.mark.parametrize("d,dtype,T,C", [(128, "bf16", 700, 8), (32, "f32", 4200, 16), (32, "f32", 9000, 4)])
def test_stats_fresh(gpu, d, dtype, T, C):
    from dynamic_state_memory_b200 import dla
    q, k, v = case(2, 2, T, d, dtype, seed=T, mean_len=12.0)
    ref = O.prefill(q, k, v, C=C, tau=0.5, dtype=dtype, want_out=False)
    cache = dla.Cache(2, 2, C, d)
    o, tr = dla.prefill(*(to_device(x, dtype) for x in (q, k, v)), cache, 0.5)
    st = dla.Stats(4)
    assert int(st.reduce(tr, T).item()) == 0
    for u in range(4):
        check(st, ref, u)


def test_stats_continued_cache(gpu):
    """A second prefill on a cache: m_before and t_before saved before it."""
    import torch
    from dynamic_state_memory_b200 import dla
    T1, T2, d, C = 300, 500, 32, 6
    q, k, v = case(1, 3, T1 + T2, d, "f32", seed=3, mean_len=8.0)
    ref = O.prefill(q, k, v, C=C, tau=0.5, dtype="f32", want_out=False)
    cache = dla.Cache(1, 3, C, d)
    dla.prefill(*(to_device(np.ascontiguousarray(x[:, :, :T1]), "f32") for x in (q, k, v)), cache, 0.5)
    vw = cache.views()
    m0, t0 = vw["m"].reshape(-1).clone(), vw["t"].reshape(-1).clone()
    o, tr = dla.prefill(*(to_device(np.ascontiguousarray(x[:, :, T1:]), "f32") for x in (q, k, v)),
                        cache, 0.5)
    st = dla.Stats(3)
    st.reduce(tr, T2, m0, t0)
    torch.cuda.synchronize()
    for u in range(3):
        live = ref["live"].reshape(3, -1)[u][T1:]
        bnd = ref["boundary"].reshape(3, -1)[u][T1:]
        mer = [m for m in ref["merges"][u] if m[0] >= T1]
        want = expect(live, bnd, mer)
        assert int(st.live_sum[u]) == want["live_sum"] and int(st.merges[u]) == want["merges"]
        assert int(st.boundaries[u]) == want["boundaries"] and int(st.atom_rows[u]) == want["atom_rows"]


def test_stats_unbounded_and_overflow(gpu):
    import torch
    from dynamic_state_memory_b200 import dla
    q, k, v = case(1, 2, 600, 128, "bf16", seed=9, mean_len=4.0)
    ref = O.prefill(q, k, v, C=2, tau=0.5, dtype="bf16", policy="unbounded", want_out=False)
    cache = dla.Cache(1, 2, 512, 128)
    o, tr = dla.unbounded_prefill(*(to_device(x, "bf16") for x in (q, k, v)), cache, 0.5)
    st = dla.Stats(2)
    st.reduce(tr, 600)
    torch.cuda.synchronize()
    for u in range(2):
        check(st, ref, u)
    # a trace that lost merges reports it
    q, k, v = case(1, 2, 300, 32, "f32", seed=11, mean_len=4.0)
    cache = dla.Cache(1, 2, 4, 32)
    o, tr = dla.prefill(*(to_device(x, "f32") for x in (q, k, v)), cache, 0.5, cap=2, sync=False)
    torch.cuda.synchronize()
    assert int(dla.Stats(2).reduce(tr, 300).item()) == 4  # DLA_ERR_TRACE_OVERFLOW

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


@pytest.mark.parametrize("window", [0, 256])
def test_cuda_graph_capture_and_replay(gpu, window):
    """A prefill (cache reset + call) captured in a CUDA graph and replayed
    gives the eager call's outputs and trace bit for bit: the library's fork
    onto its auxiliary streams and the join go through events on the caller's
    stream, which stream capture follows."""
    import torch
    from dynamic_state_memory_b200 import dla
    q, k, v = case(2, 2, 700, 128, "bf16", seed=77, mean_len=14.0)
    B, H, T, d = k.shape
    C, tau = 8, 0.5
    tq, tk, tv = (to_device(x, "bf16") for x in (q, k, v))
    cache = dla.Cache(B, H, C, d)
    cfg = dla.make_config(B, H, T, d, C, tau, dla.DLA_BF16, window, None)
    ws = torch.empty(dla.dla_workspace_bytes(cfg), dtype=torch.uint8, device="cuda")
    tr = dla.Trace(B * H, T, T + 1, "cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    o = torch.empty_like(tq)

    def call(stream):
        dla.dla_cache_init(cache.c, B, H, C, d, d, cache.base, stream)
        dla.dla_prefill(cfg, tq, tk, tv, o, cache.c, tr.c, ws, st, stream)

    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        call(s)
    torch.cuda.synchronize()
    o_eager = o.clone()
    b_eager = tr.boundary.clone()
    m_eager = tr.merges()
    o.zero_()
    tr.boundary.zero_()

    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        call(s)
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    dla.check_device_status(st, "graph replay")
    assert torch.equal(o, o_eager)
    assert torch.equal(tr.boundary, b_eager)
    assert tr.merges() == m_eager
    ref = oracle_run(q, k, v, C, tau, "bf16")
    assert tr.merges() == ref["merges"]
    assert rel_err(from_device(o), ref["out"]) <= TOL["bf16"]


@pytest.mark.parametrize("mean_len", [3.0, 40.0])
def test_more_tiles_than_sms(gpu, mean_len):
    """160 streams x 5 tiles: the atom loop's CTAs each walk several tiles,
    many of them with no atom or one (the first tile of every stream)."""
    q, k, v = case(4, 40, 640, 128, "bf16", seed=int(mean_len) + 90, mean_len=mean_len)
    check(q, k, v, 4, 0.5)


"""GPU parity of ragged batches: dla_prefill_varlen and dla_decode_step_masked.

Requests of different lengths in one prefill call (sequence b uses the first
lens[b] rows), and decode steps that only some sequences take (continuous
batching).  Each stream must equal the oracle run on its own tokens alone:
boundaries and merges bit for bit, outputs within 1e-4 (fp32) or 2e-2 (bf16)
of max|o|; rows past a sequence's length, and inactive sequences' rows and
caches, are left untouched.
"""
import numpy as np
import pytest

from dynamic_state_memory_b200 import synth
from oracle import oracle as O
from tests.gpu_helpers import TOL, case, from_device, rel_err, to_device

pytestmark = pytest.mark.gpu

POLICY = {"dla": 0, "unbounded": 3, "info": 2}


def oracle_ragged(q, k, v, lens, C, tau, dtype, policy="dla", orc=None):
    """Each stream run alone on its first lens[b] tokens (continuing `orc`,
    one oracle per stream, when given)."""
    B, H, T, d = k.shape
    out = np.zeros((B, H, T, d))
    bnd = np.zeros((B, H, T), dtype=np.uint8)
    merges = [[] for _ in range(B * H)]
    orcs = orc if orc is not None else [O.Oracle(1, d, d, C, policy) for _ in range(B * H)]
    for b in range(B):
        L = int(lens[b])
        for h in range(H):
            if L == 0:
                continue
            r = orcs[b * H + h].run(k[b, h, :L][None], q[b, h, :L][None], v[b, h, :L][None],
                                    tau=tau, dtype=dtype)
            out[b, h, :L] = r["out"][0]
            bnd[b, h, :L] = r["boundary"][0]
            merges[b * H + h] = r["merges"][0]
    return out, bnd, merges, orcs


def gpu_ragged(q, k, v, lens, cache, tau, dtype, policy, window=0, sentinel=3.0):
    import torch
    from dynamic_state_memory_b200 import dla
    qd, kd, vd = (to_device(x, dtype) for x in (q, k, v))
    o = torch.full_like(qd, sentinel)
    ld = torch.tensor(lens, dtype=torch.int32, device="cuda")
    o, tr = dla.prefill_varlen(qd, kd, vd, ld, cache, tau, policy=POLICY[policy], window=window, o=o)
    return from_device(o), tr


def check(q, k, v, lens, C, tau, dtype, policy, window=0):
    from dynamic_state_memory_b200 import dla
    B, H, T, d = k.shape
    ref_o, ref_b, ref_m, _ = oracle_ragged(q, k, v, lens, C, tau, dtype, policy)
    cache = dla.Cache(B, H, C, d)
    o, tr = gpu_ragged(q, k, v, lens, cache, tau, dtype, policy, window)
    bnd = tr.boundary.cpu().numpy().reshape(B, H, T)
    for b in range(B):
        L = int(lens[b])
        assert np.array_equal(bnd[b, :, :L], ref_b[b, :, :L]), b
        assert not bnd[b, :, L:].any(), b
        assert np.all(o[b, :, L:] == 3.0), b          # rows past the length untouched
    assert tr.merges() == ref_m
    mask = np.zeros((B, H, T), dtype=bool)
    for b in range(B):
        mask[b, :, :int(lens[b])] = True
    assert rel_err(o[mask], ref_o[mask]) <= TOL[dtype]
    t = cache.views()["t"].cpu().numpy()
    assert (t == np.array(lens)[:, None]).all()


LENS = [0, 1, 37, 128, 129, 300]


@pytest.mark.parametrize("d,dtype", [(128, "bf16"), (32, "f32")])
@pytest.mark.parametrize("window", [0, 128])
def test_ragged_dynamic(gpu, d, dtype, window):
    q, k, v = case(len(LENS), 2, 300, d, dtype, seed=41 + d, mean_len=10.0)
    check(q, k, v, LENS, 8, 0.5, dtype, "dla", window)


def test_ragged_unbounded(gpu):
    q, k, v = case(len(LENS), 2, 300, 128, "bf16", seed=43, mean_len=3.0)
    check(q, k, v, LENS, 512, 0.5, "bf16", "unbounded", 128)


def test_ragged_info(gpu):
    wl = dict(B=len(LENS), H=2, T=300, d=32, dtype="f32", n_centres=6,
              lengths=("geometric", 20.0), sigma=0.05, seed=47, value_regimes=True)
    q, k, v = synth.make_prefill(wl)
    check(q, k, v, LENS, 4, 0.5, "f32", "info", 128)


def test_ragged_calls_continue_each_stream(gpu):
    """Two ragged calls on one cache equal each stream's oracle run over its
    concatenated tokens."""
    from dynamic_state_memory_b200 import dla
    B, H, d, C, tau = 4, 2, 128, 6, 0.5
    l1, l2 = [0, 50, 130, 200], [70, 0, 129, 56]
    Tt = max(a + b for a, b in zip(l1, l2))
    q, k, v = case(B, H, Tt, d, "bf16", seed=53, mean_len=8.0)
    ref_o, ref_b, ref_m, orcs = oracle_ragged(q, k, v, [a + b for a, b in zip(l1, l2)], C, tau,
                                              "bf16")
    cache = dla.Cache(B, H, C, d)

    def part(x, off, ln, T):
        y = np.zeros((B, H, T, d), dtype=x.dtype)
        for b in range(B):
            y[b, :, :ln[b]] = x[b, :, off[b]:off[b] + ln[b]]
        return y

    o1, _ = gpu_ragged(*(part(x, [0] * B, l1, max(l1)) for x in (q, k, v)), l1, cache, tau,
                       "bf16", "dla")
    o2, _ = gpu_ragged(*(part(x, l1, l2, max(l2)) for x in (q, k, v)), l2, cache, tau, "bf16",
                       "dla")
    got, want = [], []
    for b in range(B):
        got += [o1[b, :, :l1[b]], o2[b, :, :l2[b]]]
        want += [ref_o[b, :, :l1[b]], ref_o[b, :, l1[b]:l1[b] + l2[b]]]
    got = np.concatenate([g.reshape(-1, d) for g in got])
    want = np.concatenate([w.reshape(-1, d) for w in want])
    assert rel_err(got, want) <= TOL["bf16"]
    vw = cache.views()
    for b in range(B):
        for h in range(H):
            st = orcs[b * H + h].state(0)
            assert int(vw["m"][b, h]) == st["m"] and int(vw["t"][b, h]) == l1[b] + l2[b]


def test_masked_decode_steps(gpu):
    """Decode steps that only some sequences take: active streams equal their
    oracle stepped only when active; inactive ones keep cache and rows."""
    import torch
    from dynamic_state_memory_b200 import dla
    N, H, d, C, tau, T0, steps = 6, 2, 128, 5, 0.5, 80, 24
    q, k, v = case(N, H, T0 + steps, d, "bf16", seed=59, mean_len=6.0)
    cache = dla.Cache(N, H, C, d)
    dla.prefill(*(to_device(np.ascontiguousarray(x[:, :, :T0]), "bf16") for x in (q, k, v)), cache,
                tau)
    orcs = [O.Oracle(1, d, d, C) for _ in range(N * H)]
    for u in range(N * H):
        b, h = divmod(u, H)
        orcs[u].run(k[b, h, :T0][None], q[b, h, :T0][None], v[b, h, :T0][None], tau=tau,
                    dtype="bf16", out_mask=np.zeros(T0, dtype=np.uint8))
    dec = dla.Decoder(cache)
    rng = np.random.default_rng(7)
    pos = np.full(N, T0)        # each sequence's next token
    o = torch.full((N, H, d), 5.0, dtype=torch.bfloat16, device="cuda")
    got, want = [], []
    for s in range(steps):
        act = (rng.random(N) < 0.6).astype(np.uint8)
        act[s % N] = 1
        qs, ks, vs = (np.stack([x[n, :, pos[n]] for n in range(N)]) for x in (q, k, v))
        before = {kk: t.clone() for kk, t in cache.views().items()}
        o_prev = o.clone()
        dec.step_masked(torch.from_numpy(act).cuda(), *(to_device(x, "bf16") for x in (qs, ks, vs)),
                        tau, o)
        torch.cuda.synchronize()
        dla.check_device_status(dec.status, "masked decode")
        after = cache.views()
        for n in range(N):
            if not act[n]:
                assert torch.equal(o[n], o_prev[n])
                for kk, t in before.items():
                    assert torch.equal(after[kk][n], t[n]), (s, n, kk)
                continue
            for h in range(H):
                u = n * H + h
                r = orcs[u].run(ks[n, h][None, None], qs[n, h][None, None], vs[n, h][None, None],
                                tau=tau, dtype="bf16")
                assert int(dec.boundary[u]) == int(r["boundary"][0, 0])
                want_i = r["merges"][0][0][1] if r["merges"][0] else -1
                assert int(dec.merge_i[u]) == want_i
                got.append(from_device(o[n, h]))
                want.append(r["out"][0, 0])
            pos[n] += 1
    assert rel_err(np.stack(got), np.stack(want)) <= TOL["bf16"]


def test_ragged_more_tiles_than_sms(gpu):
    """40 sequences of 0 to 1000 tokens x 8 heads (over 148 tiles in all, with
    empty and partial ones): the atom loop skips every tile past a length."""
    rng = np.random.default_rng(5)
    lens = [0, 1000, 129, 1] + [int(x) for x in rng.integers(0, 1001, size=36)]
    q, k, v = case(len(lens), 8, 1000, 128, "bf16", seed=57, mean_len=12.0)
    check(q, k, v, lens, 8, 0.5, "bf16", "dla")


"""dla_decode_step_static: the decode step for callers that cannot allocate
device memory (fixed memory budgets, plug-ins inside another engine's pool).

It must give the same results as dla_decode_step on the same cache state, on
two calls in a row (its scratch array keeps the previous call's contents), and
refuse caches whose scratch need exceeds the static array.
"""
import ctypes

import numpy as np
import pytest

from tests.gpu_helpers import case, from_device, to_device

pytestmark = pytest.mark.gpu


def _twin_caches(q, k, v, C, tau):
    import torch
    from dynamic_state_memory_b200 import dla
    B, H, T, d = k.shape
    caches = []
    for _ in range(2):
        c = dla.Cache(B, H, C, d)
        dla.prefill(to_device(q, "bf16"), to_device(k, "bf16"), to_device(v, "bf16"), c, tau)
        caches.append(c)
    torch.cuda.synchronize()
    return caches


def test_static_scratch_matches_workspace_variant(gpu):
    import torch
    from dynamic_state_memory_b200 import dla
    B, H, d, C, tau = 2, 3, 128, 4, 0.5
    q, k, v = case(B, H, 52, d, "bf16", seed=77, mean_len=5.0)
    ca, cb = _twin_caches(q[:, :, :50], k[:, :, :50], v[:, :, :50], C, tau)
    dec = dla.Decoder(ca)
    U = B * H
    bnd_b = torch.zeros(U, dtype=torch.uint8, device="cuda")
    mi_b = torch.zeros(U, dtype=torch.int32, device="cuda")
    st_b = torch.zeros(1, dtype=torch.int32, device="cuda")
    for t in (50, 51):  # two calls in a row
        qs, ks, vs = (to_device(np.ascontiguousarray(x[:, :, t]), "bf16") for x in (q, k, v))
        o_a = dec.step(qs, ks, vs, tau)
        o_b = torch.empty_like(o_a)
        dla.dla_decode_step_static(cb.c, tau, dla.DLA_BF16, qs, ks, vs, o_b, bnd_b, mi_b, st_b)
        torch.cuda.synchronize()
        dla.check_device_status(dec.status, "dla_decode_step")
        dla.check_device_status(st_b, "dla_decode_step_static")
        ra, rb = from_device(o_a), from_device(o_b)
        assert np.abs(ra - rb).max() <= 2e-2 * np.abs(ra).max()
        assert torch.equal(dec.boundary, bnd_b)
        assert torch.equal(dec.merge_i, mi_b)
    va, vb = ca.views(), cb.views()
    assert torch.equal(va["m"], vb["m"]) and torch.equal(va["order"], vb["order"])


def test_static_scratch_rejects_oversized_cache(gpu):
    import torch
    from dynamic_state_memory_b200 import dla
    dummy = torch.zeros(256, dtype=torch.uint8, device="cuda")
    c = dla.dla_cache()
    c.N, c.H, c.C, c.d_k, c.d_v = 4096, 16, 64, 128, 128   # needs > 8 MiB of scratch
    for name in ("S", "z", "n", "ts", "pair_loss", "order", "m", "prev_k", "prev_r", "t"):
        setattr(c, name, dummy.data_ptr())
    assert dla.dla_decode_workspace_bytes(4096, 16, 64, 128, 128) > (8 << 20)
    code = dla._lib.dla_decode_step_static(ctypes.byref(c), 0.5, dla.DLA_BF16, ctypes.c_void_p(1),
                                           ctypes.c_void_p(1), ctypes.c_void_p(1),
                                           ctypes.c_void_p(1), None, None, None, None)
    assert code == 5  # DLA_ERR_WORKSPACE

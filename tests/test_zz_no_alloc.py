"""dla_decode_step_static: the decode step for callers that cannot allocate
device memory (fixed memory budgets, plug-ins inside another engine's pool).

It must give the same results as dla_decode_step on the same cache state, on
two calls in a row (its scratch array keeps the previous call's contents):
the same kernels run on the same inputs, so outputs, decisions and the
updated caches are compared bit for bit.  Its refusal of caches whose scratch
need exceeds the static array is tested without a device
(tests/test_static_reject.py, which runs the _REJECT snippet below).
"""
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
    for t in (50, 51):  # two calls in a row: the array keeps the first call's contents
        qs, ks, vs = (to_device(np.ascontiguousarray(x[:, :, t]), "bf16") for x in (q, k, v))
        o_a = dec.step(qs, ks, vs, tau)
        o_b = torch.empty_like(o_a)
        dla.dla_decode_step_static(cb.c, tau, dla.DLA_BF16, qs, ks, vs, o_b, bnd_b, mi_b, st_b)
        torch.cuda.synchronize()
        dla.check_device_status(dec.status, "dla_decode_step")
        dla.check_device_status(st_b, "dla_decode_step_static")
        # the same kernels on the same cache state: identical to the bit
        assert torch.equal(o_a, o_b), t
        assert torch.equal(dec.boundary, bnd_b)
        assert torch.equal(dec.merge_i, mi_b)
    va, vb = ca.views(), cb.views()
    for name in ("m", "order", "n", "ts", "z", "t", "prev_r", "prev_k"):
        assert torch.equal(va[name], vb[name]), name
    # the live states' fp32 slots (free slots hold stale values on both sides)
    m = va["m"].cpu()
    order = va["order"].cpu()
    for b in range(B):
        for h in range(H):
            for p in range(int(m[b, h])):
                sl = int(order[b, h, p])
                assert torch.equal(va["S"][b, h, sl], vb["S"][b, h, sl]), (b, h, sl)


_REJECT = r"""
import ctypes, sys
sys.path.insert(0, sys.argv[1])
from dynamic_state_memory_b200 import dla
c = dla.dla_cache()
c.N, c.H, c.C, c.d_k, c.d_v = 4096, 16, 64, 128, 128   # needs more than 8 MiB of scratch
for name in ("S", "z", "n", "ts", "pair_loss", "order", "m", "prev_k", "prev_r", "t"):
    setattr(c, name, 256)   # never dereferenced: the size check returns first
assert dla.dla_decode_workspace_bytes(4096, 16, 64, 128, 128) > (8 << 20)
code = dla._lib.dla_decode_step_static(ctypes.byref(c), 0.5, dla.DLA_BF16, ctypes.c_void_p(256),
                                       ctypes.c_void_p(256), ctypes.c_void_p(256),
                                       ctypes.c_void_p(256), None, None, None, None)
print(code)
"""

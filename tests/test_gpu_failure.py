"""Failure paths of the device side, exercised without faulting a GPU.

- Trace overflow: a prefill whose trace holds fewer merges than the call
  makes must report DLA_ERR_TRACE_OVERFLOW, count every merge, record the
  first `cap` of them, and still produce the oracle's boundaries and outputs
  (the trace is a report; the decisions do not depend on it).
- Bounded waits: the mbarrier wait of the tensor-core kernels (tc_ptx.cuh),
  run by a probe kernel on a barrier nothing arrives on (no copy or MMA is
  issued), must give up after its poll limit, raise the abort flag, make a
  later wait return at once and report DLA_ERR_TIMEOUT; the GPU stays usable.
"""
import ctypes

import numpy as np
import pytest

from tests.gpu_helpers import TOL, case, from_device, oracle_run, rel_err, to_device

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("d,dtype", [(128, "bf16"), (32, "f32")])
def test_trace_overflow(gpu, d, dtype):
    import torch
    from dynamic_state_memory_b200 import dla
    B, H, T, C, tau = 1, 2, 300, 4, 0.5
    q, k, v = case(B, H, T, d, dtype, seed=91, mean_len=4.0)
    ref = oracle_run(q, k, v, C, tau, dtype)
    counts = [len(m) for m in ref["merges"]]
    cap = 3
    assert min(counts) > cap
    cache = dla.Cache(B, H, C, d)
    code = dla.DLA_BF16 if dtype == "bf16" else dla.DLA_F32
    cfg = dla.make_config(B, H, T, d, C, tau, code)
    ws = torch.empty(dla.dla_workspace_bytes(cfg), dtype=torch.uint8, device="cuda")
    tr = dla.Trace(B * H, T, cap)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    qd, kd, vd = (to_device(x, dtype) for x in (q, k, v))
    o = torch.empty_like(qd)
    dla.dla_prefill(cfg, qd, kd, vd, o, cache.c, tr.c, ws, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 4  # DLA_ERR_TRACE_OVERFLOW
    assert tr.merge_count.cpu().tolist() == counts
    assert tr.merges() == [m[:cap] for m in ref["merges"]]
    assert np.array_equal(tr.boundary.cpu().numpy().reshape(B, H, T), ref["boundary"])
    assert rel_err(from_device(o), ref["out"]) <= TOL[dtype]


def _probe():
    from tests import probe_build
    lib = ctypes.CDLL(probe_build.build())
    lib.dla_probe_bounded_wait.restype = ctypes.c_int
    lib.dla_probe_bounded_wait.argtypes = [ctypes.c_int, ctypes.c_uint, ctypes.c_void_p,
                                           ctypes.c_void_p, ctypes.c_void_p]
    return lib


def test_bounded_wait_times_out_and_reports(gpu):
    import torch
    lib = _probe()
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.full((4,), -1, dtype=torch.int32, device="cuda")
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert lib.dla_probe_bounded_wait(0, 1 << 12, ctypes.c_void_p(st.data_ptr()),
                                      ctypes.c_void_p(out.data_ptr()), s) == 0
    torch.cuda.synchronize()
    first, flag, second, cycles = out.cpu().tolist()
    assert first == 0 and flag == 1 and second == 0
    assert cycles < 100_000   # the second wait gave up at once (its limit alone is far longer)
    assert int(st.item()) == 7  # DLA_ERR_TIMEOUT
    # the context is still usable, and a barrier that completes is waited for
    st.zero_()
    out.fill_(-1)
    assert lib.dla_probe_bounded_wait(1, 1 << 12, ctypes.c_void_p(st.data_ptr()),
                                      ctypes.c_void_p(out.data_ptr()), s) == 0
    torch.cuda.synchronize()
    first, flag, second, _ = out.cpu().tolist()
    assert first == 1 and flag == 0 and second == 1
    assert int(st.item()) == 0
    assert float(torch.ones(4, device="cuda").sum()) == 4.0

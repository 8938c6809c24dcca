"""Thin ctypes binding of libdla.so (argument marshalling only).

Every step of the DLA path runs in the library's CUDA kernels; PyTorch only
provides device memory and streams.  Importing this module fails loudly when
the library is missing: there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdla.so")

DLA_OK = 0
DLA_F32, DLA_BF16 = 0, 1
DLA_POLICY_DYNAMIC, DLA_POLICY_FENWICK, DLA_POLICY_INFO, DLA_POLICY_UNBOUNDED = 0, 1, 2, 3
DLA_MAX_SLOTS = 1024
STATUS_NAMES = {0: "DLA_OK", 1: "DLA_ERR_INVALID_ARG", 2: "DLA_ERR_UNSUPPORTED", 3: "DLA_ERR_CUDA",
                4: "DLA_ERR_TRACE_OVERFLOW", 5: "DLA_ERR_WORKSPACE", 6: "DLA_ERR_INVARIANT",
                7: "DLA_ERR_TIMEOUT", 8: "DLA_ERR_CAPACITY"}

c_i32, c_f32, c_vp, c_size = ctypes.c_int32, ctypes.c_float, ctypes.c_void_p, ctypes.c_size_t


class dla_profile(ctypes.Structure):
    _fields_ = [("begin", ctypes.POINTER(c_vp)), ("end", ctypes.POINTER(c_vp)),
                ("kind", ctypes.POINTER(c_i32)), ("cap", c_i32), ("count", c_i32)]


class dla_config(ctypes.Structure):
    _fields_ = [("B", c_i32), ("H", c_i32), ("T", c_i32), ("d_k", c_i32), ("d_v", c_i32),
                ("C", c_i32), ("tau", c_f32), ("in_dtype", c_i32), ("window", c_i32),
                ("profile", ctypes.POINTER(dla_profile))]


class dla_cache(ctypes.Structure):
    _fields_ = [("N", c_i32), ("H", c_i32), ("C", c_i32), ("d_k", c_i32), ("d_v", c_i32),
                ("S", c_vp), ("z", c_vp), ("n", c_vp), ("ts", c_vp), ("pair_loss", c_vp),
                ("order", c_vp), ("m", c_vp), ("prev_k", c_vp), ("prev_r", c_vp), ("t", c_vp)]


class dla_trace(ctypes.Structure):
    _fields_ = [("boundary", c_vp), ("merge_t", c_vp), ("merge_i", c_vp),
                ("merge_count", c_vp), ("cap", c_i32)]


class dla_stats(ctypes.Structure):
    _fields_ = [("boundaries", c_vp), ("merges", c_vp), ("live_sum", c_vp), ("live_max", c_vp),
                ("atom_rows", c_vp)]


class DlaError(RuntimeError):
    def __init__(self, code, where=""):
        self.code = code
        super().__init__(f"{where}: {STATUS_NAMES.get(code, code)} ({status_string(code)})")


if not os.path.exists(LIB_PATH):
    raise ImportError(f"libdla.so not built at {LIB_PATH}; run dynamic_state_memory_b200/build.py")

_lib = ctypes.CDLL(LIB_PATH)
_P = ctypes.POINTER
_lib.dla_status_string.restype = ctypes.c_char_p
_lib.dla_status_string.argtypes = [c_i32]
_lib.dla_cache_bytes.restype = c_size
_lib.dla_cache_bytes.argtypes = [c_i32] * 5
_lib.dla_cache_init.restype = c_i32
_lib.dla_cache_init.argtypes = [_P(dla_cache), c_i32, c_i32, c_i32, c_i32, c_i32, c_vp, c_size, c_vp]
_lib.dla_workspace_bytes.restype = c_size
_lib.dla_workspace_bytes.argtypes = [_P(dla_config), c_i32]
_lib.dla_prefill.restype = c_i32
_lib.dla_prefill.argtypes = [_P(dla_config), c_vp, c_vp, c_vp, c_vp, _P(dla_cache), _P(dla_trace),
                             c_vp, c_size, c_vp, c_vp]
_lib.dla_info_policy_prefill.restype = c_i32
_lib.dla_info_policy_prefill.argtypes = [_P(dla_config), c_vp, c_vp, c_vp, c_vp, _P(dla_cache),
                                         _P(dla_trace), c_vp, c_size, c_vp, c_vp]
_lib.dla_unbounded_prefill.restype = c_i32
_lib.dla_unbounded_prefill.argtypes = [_P(dla_config), c_vp, c_vp, c_vp, c_vp, _P(dla_cache),
                                       _P(dla_trace), c_vp, c_size, c_vp, c_vp]
_lib.dla_prefill_varlen.restype = c_i32
_lib.dla_prefill_varlen.argtypes = [_P(dla_config), c_i32, c_vp, c_vp, c_vp, c_vp, c_vp,
                                    _P(dla_cache), _P(dla_trace), c_vp, c_size, c_vp, c_vp]
_lib.dla_decode_step_masked.restype = c_i32
_lib.dla_decode_step_masked.argtypes = [_P(dla_cache), c_f32, c_i32, c_vp, c_vp, c_vp, c_vp, c_vp,
                                        c_vp, c_vp, c_vp, c_size, c_vp, c_vp]
_lib.dla_trace_stats.restype = c_i32
_lib.dla_trace_stats.argtypes = [_P(dla_trace), c_i32, c_i32, c_vp, c_vp, c_i32, _P(dla_stats),
                                 c_vp, c_vp]
_lib.dla_decode_workspace_bytes.restype = c_size
_lib.dla_decode_workspace_bytes.argtypes = [c_i32] * 5
_lib.dla_decode_step.restype = c_i32
_lib.dla_decode_step.argtypes = [_P(dla_cache), c_f32, c_i32, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp,
                                 c_vp, c_size, c_vp, c_vp, _P(dla_profile)]
_lib.dla_decode_step_static.restype = c_i32
_lib.dla_decode_step_static.argtypes = [_P(dla_cache), c_f32, c_i32, c_vp, c_vp, c_vp, c_vp, c_vp,
                                        c_vp, c_vp, c_vp]
_lib.dla_fixed_policy_prefill.restype = c_i32
_lib.dla_fixed_policy_prefill.argtypes = [_P(dla_config), c_vp, c_vp, c_vp, c_vp, c_vp, c_size,
                                          c_vp, c_vp]
_lib.dla_backward_workspace_bytes.restype = c_size
_lib.dla_backward_workspace_bytes.argtypes = [_P(dla_config)]
_lib.dla_prefill_backward.restype = c_i32
_lib.dla_prefill_backward.argtypes = [_P(dla_config), c_vp, c_vp, c_vp, c_vp, _P(dla_trace), c_vp,
                                      c_vp, c_vp, c_vp, c_size, c_vp, c_vp]

EXPORTS = ["dla_status_string", "dla_cache_bytes", "dla_cache_init", "dla_workspace_bytes",
           "dla_prefill", "dla_decode_workspace_bytes", "dla_decode_step",
           "dla_decode_step_static", "dla_fixed_policy_prefill", "dla_info_policy_prefill",
           "dla_unbounded_prefill", "dla_prefill_varlen", "dla_decode_step_masked",
           "dla_trace_stats", "dla_backward_workspace_bytes", "dla_prefill_backward"]


def status_string(code: int) -> str:
    return _lib.dla_status_string(int(code)).decode()


def _check(code, where):
    if code != DLA_OK:
        raise DlaError(code, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return DLA_F32
    if t.dtype == torch.bfloat16:
        return DLA_BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


# ---- raw C entry points (same names, argument marshalling only) -----------

def dla_cache_bytes(N, H, C, d_k, d_v) -> int:
    return int(_lib.dla_cache_bytes(N, H, C, d_k, d_v))


def dla_cache_init(cache: dla_cache, N, H, C, d_k, d_v, base: torch.Tensor, stream=None):
    _check(_lib.dla_cache_init(ctypes.byref(cache), N, H, C, d_k, d_v, _ptr(base),
                               base.numel() * base.element_size(), _stream(stream)),
           "dla_cache_init")


def dla_workspace_bytes(cfg: dla_config, policy=DLA_POLICY_DYNAMIC) -> int:
    return int(_lib.dla_workspace_bytes(ctypes.byref(cfg), policy))


def dla_prefill(cfg, q, k, v, o, cache, trace, ws, dev_status, stream=None):
    tr = ctypes.byref(trace) if trace is not None else None
    _check(_lib.dla_prefill(ctypes.byref(cfg), _ptr(q), _ptr(k), _ptr(v), _ptr(o),
                            ctypes.byref(cache), tr, _ptr(ws),
                            0 if ws is None else ws.numel(), _ptr(dev_status), _stream(stream)),
           "dla_prefill")


def dla_info_policy_prefill(cfg, q, k, v, o, cache, trace, ws, dev_status, stream=None):
    tr = ctypes.byref(trace) if trace is not None else None
    _check(_lib.dla_info_policy_prefill(ctypes.byref(cfg), _ptr(q), _ptr(k), _ptr(v), _ptr(o),
                                        ctypes.byref(cache), tr, _ptr(ws),
                                        0 if ws is None else ws.numel(), _ptr(dev_status),
                                        _stream(stream)),
           "dla_info_policy_prefill")


def dla_backward_workspace_bytes(cfg: dla_config) -> int:
    return int(_lib.dla_backward_workspace_bytes(ctypes.byref(cfg)))


def dla_prefill_backward(cfg, q, k, v, d_o, trace, dq, dk, dv, ws, dev_status, stream=None):
    _check(_lib.dla_prefill_backward(ctypes.byref(cfg), _ptr(q), _ptr(k), _ptr(v), _ptr(d_o),
                                     ctypes.byref(trace), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(ws),
                                     0 if ws is None else ws.numel(), _ptr(dev_status),
                                     _stream(stream)),
           "dla_prefill_backward")


def dla_unbounded_prefill(cfg, q, k, v, o, cache, trace, ws, dev_status, stream=None):
    tr = ctypes.byref(trace) if trace is not None else None
    _check(_lib.dla_unbounded_prefill(ctypes.byref(cfg), _ptr(q), _ptr(k), _ptr(v), _ptr(o),
                                      ctypes.byref(cache), tr, _ptr(ws),
                                      0 if ws is None else ws.numel(), _ptr(dev_status),
                                      _stream(stream)),
           "dla_unbounded_prefill")


def dla_prefill_varlen(cfg, policy, lens, q, k, v, o, cache, trace, ws, dev_status, stream=None):
    tr = ctypes.byref(trace) if trace is not None else None
    _check(_lib.dla_prefill_varlen(ctypes.byref(cfg), int(policy), _ptr(lens), _ptr(q), _ptr(k),
                                   _ptr(v), _ptr(o), ctypes.byref(cache), tr, _ptr(ws),
                                   0 if ws is None else ws.numel(), _ptr(dev_status),
                                   _stream(stream)),
           "dla_prefill_varlen")


def dla_decode_step_masked(cache, tau, in_dtype, active, q, k, v, o, boundary, merge_i, ws,
                           dev_status, stream=None):
    _check(_lib.dla_decode_step_masked(ctypes.byref(cache), float(tau), int(in_dtype),
                                       _ptr(active), _ptr(q), _ptr(k), _ptr(v), _ptr(o),
                                       _ptr(boundary), _ptr(merge_i), _ptr(ws),
                                       0 if ws is None else ws.numel(), _ptr(dev_status),
                                       _stream(stream)),
           "dla_decode_step_masked")


def dla_trace_stats(trace, heads, T, m_before, t_before, tile, out, dev_status, stream=None):
    _check(_lib.dla_trace_stats(ctypes.byref(trace), int(heads), int(T), _ptr(m_before),
                                _ptr(t_before), int(tile), ctypes.byref(out), _ptr(dev_status),
                                _stream(stream)),
           "dla_trace_stats")


def dla_decode_workspace_bytes(N, H, C, d_k, d_v) -> int:
    return int(_lib.dla_decode_workspace_bytes(N, H, C, d_k, d_v))


def dla_decode_step(cache, tau, in_dtype, q, k, v, o, boundary, merge_i, ws, dev_status,
                    stream=None, profile=None):
    _check(_lib.dla_decode_step(ctypes.byref(cache), float(tau), int(in_dtype), _ptr(q), _ptr(k),
                                _ptr(v), _ptr(o), _ptr(boundary), _ptr(merge_i), _ptr(ws),
                                0 if ws is None else ws.numel(), _ptr(dev_status),
                                _stream(stream),
                                None if profile is None else ctypes.byref(profile)),
           "dla_decode_step")


def dla_decode_step_static(cache, tau, in_dtype, q, k, v, o, boundary, merge_i, dev_status,
                           stream=None):
    _check(_lib.dla_decode_step_static(ctypes.byref(cache), float(tau), int(in_dtype), _ptr(q),
                                       _ptr(k), _ptr(v), _ptr(o), _ptr(boundary), _ptr(merge_i),
                                       _ptr(dev_status), _stream(stream)),
           "dla_decode_step_static")


def dla_fixed_policy_prefill(cfg, q, k, v, o, ws, dev_status, stream=None):
    _check(_lib.dla_fixed_policy_prefill(ctypes.byref(cfg), _ptr(q), _ptr(k), _ptr(v), _ptr(o),
                                         _ptr(ws), 0 if ws is None else ws.numel(),
                                         _ptr(dev_status), _stream(stream)),
           "dla_fixed_policy_prefill")


# ---- convenience layer ------------------------------------------------------

class Cache:
    """A DLA state cache in one torch uint8 buffer (256-byte aligned)."""

    def __init__(self, N, H, C, d, device="cuda", stream=None):
        self.N, self.H, self.C, self.d = N, H, C, d
        nbytes = dla_cache_bytes(N, H, C, d, d)
        if nbytes == 0:
            raise DlaError(1, "dla_cache_bytes")
        self.buf = torch.empty(nbytes + 256, dtype=torch.uint8, device=device)
        off = (-self.buf.data_ptr()) % 256
        self.base = self.buf[off:off + nbytes]
        self.c = dla_cache()
        dla_cache_init(self.c, N, H, C, d, d, self.base, stream)

    def _view(self, name, dtype, shape):
        off = getattr(self.c, name) - self.base.data_ptr()
        n = 1
        for s in shape:
            n *= s
        nb = n * torch.empty((), dtype=dtype).element_size()
        return self.base[off:off + nb].view(dtype).view(*shape)

    def sub(self, n0: int, n1: int) -> dla_cache:
        """dla_cache struct over sequences [n0, n1) of this cache (same memory)."""
        H, C, d = self.H, self.C, self.d
        per_u = {"S": C * d * d * 4, "z": C * d * 8, "n": C * 8, "ts": C * 8, "pair_loss": C * 8,
                 "order": C * 4, "m": 4, "prev_k": d * 4, "prev_r": 8, "t": 8}
        c = dla_cache()
        c.N, c.H, c.C, c.d_k, c.d_v = n1 - n0, H, C, d, d
        for name, sz in per_u.items():
            setattr(c, name, getattr(self.c, name) + n0 * H * sz)
        return c

    def views(self):
        N, H, C, d = self.N, self.H, self.C, self.d
        return dict(S=self._view("S", torch.float32, (N, H, C, d, d)),
                    z=self._view("z", torch.float64, (N, H, C, d)),
                    n=self._view("n", torch.int64, (N, H, C)),
                    ts=self._view("ts", torch.int64, (N, H, C)),
                    pair_loss=self._view("pair_loss", torch.float64, (N, H, C)),
                    order=self._view("order", torch.int32, (N, H, C)),
                    m=self._view("m", torch.int32, (N, H)),
                    prev_k=self._view("prev_k", torch.float32, (N, H, d)),
                    prev_r=self._view("prev_r", torch.float64, (N, H)),
                    t=self._view("t", torch.int64, (N, H)))


def make_config(B, H, T, d, C, tau, dtype_code, window=0, profile=None) -> dla_config:
    cfg = dla_config(B, H, T, d, d, C, float(tau), dtype_code, window)
    if profile is not None:
        cfg.profile = ctypes.pointer(profile)
    return cfg


class Profiler:
    """Caller-owned CUDA events the library records around each launch."""

    KINDS = ["score", "segscan", "segsum", "engine", "materialize", "readout",
             "decode_decide", "decode_stream", "build", "readout_pre", "phi", "info_score"]

    def __init__(self, cap=4096):
        self.events = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                       for _ in range(cap)]
        for b, e in self.events:      # force creation of the underlying cudaEvent_t
            b.record()
            e.record()
        torch.cuda.synchronize()
        self._b = (c_vp * cap)(*[b.cuda_event for b, _ in self.events])
        self._e = (c_vp * cap)(*[e.cuda_event for _, e in self.events])
        self._k = (c_i32 * cap)()
        self.p = dla_profile(ctypes.cast(self._b, ctypes.POINTER(c_vp)),
                             ctypes.cast(self._e, ctypes.POINTER(c_vp)),
                             ctypes.cast(self._k, ctypes.POINTER(c_i32)), cap, 0)

    def reset(self):
        self.p.count = 0

    def times_ms(self):
        """{kind: [ms per recorded launch]} (call after synchronising)."""
        out = {}
        for i in range(min(self.p.count, self.p.cap)):
            b, e = self.events[i]
            out.setdefault(self.KINDS[self._k[i]], []).append(b.elapsed_time(e))
        return out


class Stats:
    """Device summary of a trace (dla_trace_stats): boundaries, merges,
    live_sum, live_max and atom_rows per stream."""

    def __init__(self, heads, device="cuda"):
        self.boundaries = torch.zeros(heads, dtype=torch.int32, device=device)
        self.merges = torch.zeros(heads, dtype=torch.int32, device=device)
        self.live_sum = torch.zeros(heads, dtype=torch.int64, device=device)
        self.live_max = torch.zeros(heads, dtype=torch.int32, device=device)
        self.atom_rows = torch.zeros(heads, dtype=torch.int64, device=device)
        self.c = dla_stats(self.boundaries.data_ptr(), self.merges.data_ptr(),
                           self.live_sum.data_ptr(), self.live_max.data_ptr(),
                           self.atom_rows.data_ptr())

    def reduce(self, trace, T, m_before=None, t_before=None, tile=128, stream=None):
        st = torch.zeros(1, dtype=torch.int32, device=self.boundaries.device)
        dla_trace_stats(trace.c, self.boundaries.numel(), T, m_before, t_before, tile, self.c, st,
                        stream)
        return st


class Trace:
    def __init__(self, heads, T, cap, device="cuda"):
        self.boundary = torch.zeros(heads, max(T, 1), dtype=torch.uint8, device=device)
        self.merge_t = torch.zeros(heads, max(cap, 1), dtype=torch.int32, device=device)
        self.merge_i = torch.zeros_like(self.merge_t)
        self.merge_count = torch.zeros(heads, dtype=torch.int32, device=device)
        self.c = dla_trace(self.boundary.data_ptr(), self.merge_t.data_ptr(),
                           self.merge_i.data_ptr(), self.merge_count.data_ptr(), cap)

    def merges(self):
        mc = self.merge_count.cpu().tolist()
        mt = self.merge_t.cpu()
        mi = self.merge_i.cpu()
        cap = self.c.cap
        return [list(zip(mt[h, :min(c, cap)].tolist(), mi[h, :min(c, cap)].tolist()))
                for h, c in enumerate(mc)]


def check_device_status(dev_status: torch.Tensor, where: str):
    code = int(dev_status.item())
    if code != DLA_OK:
        raise DlaError(code, where + " (device)")


def prefill(q, k, v, cache: Cache, tau: float, *, trace: bool = True, cap=None, window=0,
            stream=None, sync=True, profile=None):
    """o = DLA prefill of q, k, v [B, H, T, d] (fp32 or bf16 CUDA tensors)."""
    B, H, T, d = k.shape
    for t in (q, k, v):
        if not t.is_cuda or not t.is_contiguous() or t.shape != k.shape or t.dtype != k.dtype:
            raise ValueError("q, k, v must be contiguous CUDA tensors of one shape and dtype")
    cfg = make_config(B, H, T, d, cache.C, tau, _dtype_code(k), window, profile)
    ws = torch.empty(max(dla_workspace_bytes(cfg), 1), dtype=torch.uint8, device=k.device)
    o = torch.empty_like(q)
    tr = Trace(B * H, T, T + 1 if cap is None else cap, k.device) if trace else None
    st = torch.zeros(1, dtype=torch.int32, device=k.device)
    dla_prefill(cfg, q, k, v, o, cache.c, None if tr is None else tr.c, ws, st, stream)
    if sync:
        torch.cuda.synchronize()
        check_device_status(st, "dla_prefill")
    return o, tr


def info_prefill(q, k, v, cache: Cache, tau: float, *, trace: bool = True, cap=None, window=0,
                 stream=None, sync=True, profile=None):
    """o = prefill under the information policy (state score, density merges)
    of q, k, v [B, H, T, d]; `cache` must be freshly initialised."""
    B, H, T, d = k.shape
    for t in (q, k, v):
        if not t.is_cuda or not t.is_contiguous() or t.shape != k.shape or t.dtype != k.dtype:
            raise ValueError("q, k, v must be contiguous CUDA tensors of one shape and dtype")
    cfg = make_config(B, H, T, d, cache.C, tau, _dtype_code(k), window, profile)
    ws = torch.empty(max(dla_workspace_bytes(cfg, DLA_POLICY_INFO), 1), dtype=torch.uint8,
                     device=k.device)
    o = torch.empty_like(q)
    tr = Trace(B * H, T, T + 1 if cap is None else cap, k.device) if trace else None
    st = torch.zeros(1, dtype=torch.int32, device=k.device)
    dla_info_policy_prefill(cfg, q, k, v, o, cache.c, None if tr is None else tr.c, ws, st, stream)
    if sync:
        torch.cuda.synchronize()
        check_device_status(st, "dla_info_policy_prefill")
    return o, tr


def unbounded_prefill(q, k, v, cache: Cache, tau: float, *, trace: bool = True, cap=None,
                      window=0, stream=None, sync=True, profile=None):
    """o = DLA(I) prefill (no capacity bound; cache.C is the slot storage) of
    q, k, v [B, H, T, d]."""
    B, H, T, d = k.shape
    for t in (q, k, v):
        if not t.is_cuda or not t.is_contiguous() or t.shape != k.shape or t.dtype != k.dtype:
            raise ValueError("q, k, v must be contiguous CUDA tensors of one shape and dtype")
    cfg = make_config(B, H, T, d, cache.C, tau, _dtype_code(k), window, profile)
    ws = torch.empty(max(dla_workspace_bytes(cfg, DLA_POLICY_UNBOUNDED), 1), dtype=torch.uint8,
                     device=k.device)
    o = torch.empty_like(q)
    tr = Trace(B * H, T, 1 if cap is None else cap, k.device) if trace else None
    st = torch.zeros(1, dtype=torch.int32, device=k.device)
    dla_unbounded_prefill(cfg, q, k, v, o, cache.c, None if tr is None else tr.c, ws, st, stream)
    if sync:
        torch.cuda.synchronize()
        check_device_status(st, "dla_unbounded_prefill")
    return o, tr


def prefill_backward(q, k, v, d_o, trace: Trace, C: int, *, stream=None, sync=True):
    """dq, dk, dv (fp32, [B, H, T, d]) of a dla_prefill of q, k, v [B, H, T, d]
    from empty caches of capacity C, at the decisions its `trace` recorded;
    d_o = dL/do in the inputs' dtype."""
    B, H, T, d = k.shape
    for t in (q, k, v, d_o):
        if not t.is_cuda or not t.is_contiguous() or t.shape != k.shape or t.dtype != k.dtype:
            raise ValueError("q, k, v, d_o must be contiguous CUDA tensors of one shape and dtype")
    cfg = make_config(B, H, T, d, C, 0.0, _dtype_code(k), 0, None)
    need = dla_backward_workspace_bytes(cfg)
    if need == 0:
        raise DlaError(2, "dla_prefill_backward (shape)")  # DLA_ERR_UNSUPPORTED
    ws = torch.empty(need, dtype=torch.uint8, device=k.device)
    dq, dk, dv = (torch.empty(B, H, T, d, dtype=torch.float32, device=k.device) for _ in range(3))
    st = torch.zeros(1, dtype=torch.int32, device=k.device)
    dla_prefill_backward(cfg, q, k, v, d_o, trace.c, dq, dk, dv, ws, st, stream)
    if sync:
        torch.cuda.synchronize()
        check_device_status(st, "dla_prefill_backward")
    return dq, dk, dv


def prefill_varlen(q, k, v, lens, cache: Cache, tau: float, *, policy=DLA_POLICY_DYNAMIC,
                   trace: bool = True, window=0, stream=None, sync=True, o=None):
    """Ragged prefill: sequence b uses the first lens[b] of its T rows of
    q, k, v [B, H, T, d]; lens is a CUDA int32 tensor [B].  Rows past a
    sequence's length of o (and of the trace's boundaries) are left as given."""
    B, H, T, d = k.shape
    for t in (q, k, v):
        if not t.is_cuda or not t.is_contiguous() or t.shape != k.shape or t.dtype != k.dtype:
            raise ValueError("q, k, v must be contiguous CUDA tensors of one shape and dtype")
    if lens.dtype != torch.int32 or not lens.is_cuda or lens.shape != (B,):
        raise ValueError("lens must be a CUDA int32 tensor [B]")
    cfg = make_config(B, H, T, d, cache.C, tau, _dtype_code(k), window)
    ws = torch.empty(max(dla_workspace_bytes(cfg, policy), 1), dtype=torch.uint8, device=k.device)
    o = torch.zeros_like(q) if o is None else o
    tr = Trace(B * H, T, T + 1, k.device) if trace else None
    st = torch.zeros(1, dtype=torch.int32, device=k.device)
    dla_prefill_varlen(cfg, policy, lens, q, k, v, o, cache.c, None if tr is None else tr.c, ws,
                       st, stream)
    if sync:
        torch.cuda.synchronize()
        check_device_status(st, "dla_prefill_varlen")
    return o, tr


class Decoder:
    """Reusable buffers for dla_decode_step on one cache."""

    def __init__(self, cache: Cache, device="cuda"):
        self.cache = cache
        U = cache.N * cache.H
        nb = dla_decode_workspace_bytes(cache.N, cache.H, cache.C, cache.d, cache.d)
        if nb == 0:
            raise DlaError(2, "dla_decode_workspace_bytes")
        self.ws = torch.empty(nb, dtype=torch.uint8, device=device)
        self.boundary = torch.zeros(U, dtype=torch.uint8, device=device)
        self.merge_i = torch.zeros(U, dtype=torch.int32, device=device)
        self.status = torch.zeros(1, dtype=torch.int32, device=device)

    def step(self, q, k, v, tau, o=None, stream=None, profile=None):
        """One token for every stream: q, k, v [N, H, d] -> o [N, H, d]."""
        if o is None:
            o = torch.empty_like(q)
        dla_decode_step(self.cache.c, tau, _dtype_code(k), q, k, v, o, self.boundary,
                        self.merge_i, self.ws, self.status, stream, profile)
        return o

    def step_masked(self, active, q, k, v, tau, o, stream=None):
        """One token for the sequences with active[n] != 0 (CUDA uint8 [N]);
        the others' caches and rows of o, boundary and merge_i are untouched."""
        dla_decode_step_masked(self.cache.c, tau, _dtype_code(k), active, q, k, v, o,
                               self.boundary, self.merge_i, self.ws, self.status, stream)
        return o


def fixed_policy_prefill(q, k, v, *, window=0, stream=None, sync=True, profile=None):
    """o = fixed Fenwick-bucket policy over q, k, v [B, H, T, d] (streams start at t = 0)."""
    B, H, T, d = k.shape
    cfg = make_config(B, H, T, d, 2, 0.0, _dtype_code(k), window, profile)
    ws = torch.empty(max(dla_workspace_bytes(cfg, DLA_POLICY_FENWICK), 1), dtype=torch.uint8,
                     device=k.device)
    o = torch.empty_like(q)
    st = torch.zeros(1, dtype=torch.int32, device=k.device)
    dla_fixed_policy_prefill(cfg, q, k, v, o, ws, st, stream)
    if sync:
        torch.cuda.synchronize()
        check_device_status(st, "dla_fixed_policy_prefill")
    return o

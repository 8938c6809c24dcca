"""libdla.so loads and exports every entry point include/dla.h declares (CPU).

Only argument checks that return before any CUDA call are exercised here.
"""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dla.h")


def declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(dla_[a-z_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    from dynamic_state_memory_b200 import build
    build.build()
    return ctypes.CDLL(build.LIB)


def test_every_declared_symbol_is_exported(lib):
    names = declared()
    assert "dla_prefill" in names and "dla_decode_step" in names
    for n in names:
        assert hasattr(lib, n), f"{n} declared in dla.h but not exported"


def test_binding_covers_header():
    from dynamic_state_memory_b200 import dla
    assert sorted(dla.EXPORTS) == declared()


def test_size_queries_and_argument_errors():
    from dynamic_state_memory_b200 import dla
    assert dla.dla_cache_bytes(0, 1, 4, 32, 32) == 0
    assert dla.dla_cache_bytes(1, 1, 4, 32, 32) > 4 * 32 * 32 * 4
    bad = dla.make_config(1, 1, 16, 48, 4, 0.5, dla.DLA_F32)      # d = 48 unsupported
    assert dla.dla_workspace_bytes(bad) == 0
    bad_c = dla.make_config(1, 1, 16, 32, 1, 0.5, dla.DLA_F32)    # C < 2
    assert dla.dla_workspace_bytes(bad_c) == 0
    good = dla.make_config(1, 1, 16, 32, 4, 0.5, dla.DLA_F32)
    assert dla.dla_workspace_bytes(good) > 0
    assert dla.dla_workspace_bytes(good, dla.DLA_POLICY_FENWICK) > 0
    # the information policy carries its fp64 open states across windows
    assert dla.dla_workspace_bytes(good, dla.DLA_POLICY_INFO) > dla.dla_workspace_bytes(good)
    assert dla.dla_workspace_bytes(good, 7) == 0
    lib = dla._lib
    cache = dla.dla_cache()
    # null config / null cache -> invalid argument, synchronously
    assert lib.dla_prefill(None, None, None, None, None, ctypes.byref(cache), None, None, 0,
                           None, None) == 1
    assert lib.dla_prefill(ctypes.byref(good), None, None, None, None, None, None, None, 0,
                           None, None) == 1
    # shape mismatch between config and cache
    cache.N, cache.H, cache.C, cache.d_k, cache.d_v = 2, 1, 4, 32, 32
    assert lib.dla_prefill(ctypes.byref(good), None, None, None, None, ctypes.byref(cache), None,
                           None, 0, None, None) == 1
    assert lib.dla_cache_init(ctypes.byref(cache), 1, 1, 4, 32, 32, None, 0, None) == 1
    # the information policy's entry point checks the same way
    assert lib.dla_info_policy_prefill(None, None, None, None, None, ctypes.byref(cache), None,
                                       None, 0, None, None) == 1
    assert lib.dla_info_policy_prefill(ctypes.byref(good), None, None, None, None,
                                       ctypes.byref(cache), None, None, 0, None, None) == 1
    assert lib.dla_info_policy_prefill(ctypes.byref(bad_c), None, None, None, None,
                                       ctypes.byref(cache), None, None, 0, None, None) == 2
    # the backward's limits and its argument checks (returned before any launch)
    assert dla.dla_backward_workspace_bytes(good) > 0
    assert dla.dla_backward_workspace_bytes(dla.make_config(1, 1, 4097, 32, 4, 0.5, dla.DLA_F32)) == 0
    assert dla.dla_backward_workspace_bytes(dla.make_config(1, 1, 16, 32, 129, 0.5, dla.DLA_F32)) == 0
    assert dla.dla_backward_workspace_bytes(bad) == 0
    assert lib.dla_prefill_backward(ctypes.byref(bad), None, None, None, None, None, None, None,
                                    None, None, 0, None, None) == 2
    assert lib.dla_prefill_backward(ctypes.byref(good), None, None, None, None, None, None, None,
                                    None, None, 0, None, None) == 1
    for code in range(8):
        assert dla.status_string(code)

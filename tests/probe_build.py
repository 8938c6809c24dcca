"""Build the test-only CUDA probes under tests/csrc (sm_100a, in-tree)."""
from __future__ import annotations

import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "csrc", "wait_probe.cu")
LIB = os.path.join(HERE, "libwait_probe.so")
DEPS = [SRC] + [os.path.join(HERE, "..", "dynamic_state_memory_b200", "csrc", f)
                for f in ("tc_ptx.cuh", "dla_internal.cuh")]


def build(force: bool = False) -> str:
    if force or not os.path.exists(LIB) or any(os.path.getmtime(p) > os.path.getmtime(LIB)
                                               for p in DEPS):
        nvcc = os.environ.get("NVCC", "nvcc")
        cmd = [nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O2", "-lineinfo",
               "-std=c++17", "-Xcompiler", "-fPIC", "-shared", "-o", LIB + ".tmp", SRC]
        subprocess.run(cmd, check=True)
        os.replace(LIB + ".tmp", LIB)
    return LIB

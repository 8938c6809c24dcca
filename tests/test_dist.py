"""Multi-process host logic of bench.py on CPU: two ranks over gloo.

Streams are independent, so N GPUs run N replicas (weak scaling): the data
path has no collective. What does run across ranks is the timing plumbing
and the per-rank inputs:
- the barrier;
- the max-over-ranks reduction of the step time;
- a per-rank seed offset, so replicas work on different synthetic data;
- rank 0 alone printing the reference arm's line.
"""
import json
import os
import socket
import subprocess
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

TINY = dict(B=1, H=2, T=64, d=32, C=4, tau=0.5, dtype="f32", n_centres=4,
            lengths=("geometric", 16.0), sigma=0.05, seed=5)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    bench.barrier(world)
    slowest = bench.reduce_max(1.5 + rank, world, "cpu")
    q, k, v = bench.make_inputs(TINY, rank)
    digest = torch.tensor([float(np.abs(k).sum() + np.abs(q).sum())], dtype=torch.float64)
    every = [torch.zeros(1, dtype=torch.float64) for _ in range(world)]
    dist.all_gather(every, digest)
    again = bench.make_inputs(TINY, rank)[1]
    out.put((rank, slowest, [float(x) for x in every], bool(np.array_equal(k, again))))
    bench.barrier(world)
    dist.destroy_process_group()


def test_two_ranks_barrier_max_and_seeds():
    import multiprocessing as mp
    ctx = mp.get_context("spawn")
    port = _free_port()
    out = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    try:
        res = sorted(out.get(timeout=180) for _ in range(2))
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert [p.exitcode for p in procs] == [0, 0]
    for rank, slowest, every, deterministic in res:
        assert slowest == 2.5            # the max over ranks, on every rank
        assert every[0] != every[1]      # each replica draws its own inputs
        assert deterministic             # and the same ones on every call
    assert res[0][2] == res[1][2]


@pytest.mark.parametrize("rank", [0, 1])
def test_reference_arm_prints_on_rank0_only(rank):
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank),
               MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "tiny_f32", "--steps", "1", "--warmup", "3",
                        "--ref-tokens", "32", "--gpus", "2"],
                       env=env, capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    if rank == 0:
        assert len(lines) == 1
        line = json.loads(lines[0])
        assert line["impl"] == "reference" and line["value"] > 0
        assert line["e2e"]["h2d_bytes_per_step"] == 0
    else:
        assert lines == []


def test_reference_arm_decode_half():
    """On the headline workload the reference arm also times the metric's
    decode half: a 16-stream sample of decode_n256, extrapolated to its 4096
    streams (value and description agree)."""
    env = dict(os.environ)
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        env.pop(k, None)
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "prefill_t8192", "--steps", "1", "--warmup", "3",
                        "--ref-tokens", "32"],
                       env=env, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    dec = json.loads(lines[0])["decode"]
    assert dec["unit"] == "steps/s" and dec["value"] > 0
    assert abs(dec["ms_per_step"] - 1e3 / dec["value"]) <= 1e-3 * dec["ms_per_step"] + 1e-3
    assert "16 streams" in dec["cpu_baseline"]["sample"]
    assert "extrapolated to 4096 streams" in dec["cpu_baseline"]["sample"]


def test_gpus_flag_must_match_world_size():
    """Under an outer launcher, --gpus N must equal WORLD_SIZE (no silent
    single replica)."""
    env = dict(os.environ, RANK="0", WORLD_SIZE="2", LOCAL_RANK="0",
               MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "tiny_f32", "--steps", "1", "--gpus", "1"],
                       env=env, capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 2 and "WORLD_SIZE=2" in r.stderr


def test_gpus_flag_relaunches_under_torchrun():
    """--gpus 2 without WORLD_SIZE relaunches itself as two ranks (torchrun
    on 127.0.0.1); rank 0 alone prints the line."""
    env = {k: v for k, v in os.environ.items()
           if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT")}
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "tiny_f32", "--steps", "1", "--warmup", "3",
                        "--ref-tokens", "32", "--gpus", "2"],
                       env=env, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [json.loads(l) for l in r.stdout.splitlines() if l.strip().startswith("{")]
    assert len(lines) == 1 and lines[0]["impl"] == "reference"


def test_tensor_peak_follows_the_clock_record():
    """Burst peak when the timed region stayed at the max SM clock with no
    power cap, sustained otherwise."""
    sys.path.insert(0, ROOT)
    import bench
    peaks = {"bf16_tflops": 1656.2, "bf16_tflops_sustained": 1371.4}
    at_max = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": []}
    assert bench.tensor_peak(peaks, "measured", at_max)[0] == 1656.2
    capped = dict(at_max, reasons=["sw_power_cap"])
    assert bench.tensor_peak(peaks, "measured", capped)[0] == 1371.4
    slow = dict(at_max, sm_mhz=1400.0)
    assert bench.tensor_peak(peaks, "measured", slow)[0] == 1371.4
    assert bench.tensor_peak(peaks, "measured", None)[0] == 1371.4

#!/usr/bin/env python
"""Throughput of the DLA hot path on B200, one JSON line on rank 0.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one pass of the whole hot path over one batch of synthetic input:
  prefill workloads: dla_cache_init + dla_prefill of B x H x T tokens
  decode workload:   one dla_decode_step of N x H streams (cache pre-filled)
The default run times prefill_t8192 (the line's value) and nests the metric's
decode half (decode_n256, "decode") and the long-context and fixed-policy
configurations ("configs") in the same line; --only times the named workload
alone.
Timing: CUDA events on the launching stream around exactly K steps after W
warm-up steps, barrier + synchronize on both sides, max over ranks.  Inputs
are larger than L2 (126 MB) so no flush is needed between steps.
The kernel-level roofline uses events the library records around each of
its launches in the timed region (dla_profile).
--gpus N runs N independent replicas (weak scaling), one process per GPU: under
an outer torchrun, or relaunched under one when WORLD_SIZE is not set.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

METRIC = "DLA prefill Mtok/s and decode steps/s at C=64,d=128; % of roofline"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                  "sm_max_mhz": 1965.0}
SMS = 148
FP32_LANES_PER_SM = 128
FP64_LANES_PER_SM = 64


def policy_of(workload):
    """The decision policy a workload runs: the fixed Fenwick buckets, the
    information policy or the dynamic (cosine score, Ward merge) one."""
    if workload.startswith("fixed"):
        return "fenwick"
    if workload.startswith("info"):
        return "info"
    if workload.startswith("unbounded"):
        return "unbounded"
    return "dla"


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(PEAKS_FALLBACK), "fallback"


def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), \
        int(os.environ.get("LOCAL_RANK", 0))


class ClockSampler:
    """SM clock and throttle reasons sampled during the timed region.

    A background thread reads NVML (read-only queries) every 10 ms, plus one
    sample at start and one at stop, so even a short timed region has several
    samples; without NVML it falls back to ``nvidia-smi -lms 50``.
    """
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    PERIOD_S = 0.010

    def __init__(self, gpu_index):
        self.idx = gpu_index
        self.proc = None
        self.path = None
        self.thread = None
        self.rows = []

    def _nvml_sample(self):
        import pynvml as nv
        sm = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
        try:
            rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        except AttributeError:  # older bindings
            rs = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
        self.rows.append(dict(sm=float(sm), smax=float(self.smax),
                              hw=bool(rs & 0x8), hwt=bool(rs & 0x40), swt=bool(rs & 0x20),
                              pcap=bool(rs & 0x4)))

    def start(self):
        self.rows = []
        try:
            import threading
            import pynvml as nv
            nv.nvmlInit()
            self.h = None
            try:  # the physical GPU behind cuda:idx (CUDA_VISIBLE_DEVICES may remap)
                import torch
                uuid = str(torch.cuda.get_device_properties(self.idx).uuid)
                self.h = nv.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
            except Exception:
                self.h = None
            if self.h is None:
                self.h = nv.nvmlDeviceGetHandleByIndex(self.idx)
            self.smax = nv.nvmlDeviceGetMaxClockInfo(self.h, nv.NVML_CLOCK_SM)
            self.stop_evt = threading.Event()
            self._nvml_sample()

            def loop():
                while not self.stop_evt.wait(self.PERIOD_S):
                    try:
                        self._nvml_sample()
                    except Exception:
                        return
            self.thread = threading.Thread(target=loop, daemon=True)
            self.thread.start()
            return
        except Exception:
            self.thread = None
        try:
            import tempfile
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=self.fh, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        rows = self.rows
        if self.thread is not None:
            self.stop_evt.set()
            self.thread.join(timeout=2)
            try:
                self._nvml_sample()
            except Exception:
                pass
            rows = self.rows
        elif self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.fh.close()
            for line in open(self.path):
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    rows.append(dict(sm=float(parts[1]), smax=float(parts[2]),
                                     hw=parts[5].lower().startswith("active"),
                                     hwt=parts[6].lower().startswith("active"),
                                     swt=parts[7].lower().startswith("active"),
                                     pcap=parts[8].lower().startswith("active")))
                except ValueError:
                    continue
            os.unlink(self.path)
        else:
            return None
        if not rows:
            return None
        smax = max(r["smax"] for r in rows)
        load = [r["sm"] for r in rows if r["sm"] > 0.3 * smax] or [r["sm"] for r in rows]
        reasons = set()
        for r in rows:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                              ("swt", "sw_thermal_slowdown"), ("pcap", "sw_power_cap")):
                if r[key]:
                    reasons.add(name)
        return {"sm_mhz": statistics.median(load), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(rows), "source": "nvml" if self.thread is not None else "nvidia-smi"}


# ------------------------------------------------------------ ncu traffic ----

# kernel slot -> (ncu summary under profiles/, source files the kernel is built from)
TRAFFIC_SOURCES = {
    ("readout", "tc"): ("readout_tc", ["readout_tc.cu", "tc_ptx.cuh", "dla_internal.cuh"]),
    ("decode_stream", "-"): ("decode_stream", ["decode.cu", "dla_internal.cuh"]),
    ("info_score", "tc"): ("info_score", ["info.cu", "dla_internal.cuh"]),
}


def source_sha256(files):
    import hashlib
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "dynamic_state_memory_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def ncu_traffic(kernel, path, workload):
    """DRAM bytes per launch (read + write) from the committed ncu summary of
    this kernel and workload, or None when there is none or the kernel's
    source has changed since it was captured."""
    key = TRAFFIC_SOURCES.get((kernel, path))
    if key is None:
        return None
    name, files = key
    fn = os.path.join(ROOT, "profiles", f"{name}_{workload}.md")
    if not os.path.exists(fn):
        return None
    fields = {}
    for line in open(fn):
        line = line.strip()
        if ":" in line and line.split(":", 1)[0] in ("source_sha256", "dram_bytes_per_launch",
                                                    "units_per_launch_scale"):
            k, v = line.split(":", 1)
            fields[k] = v.strip()
    if fields.get("source_sha256") != source_sha256(files):
        return None
    try:
        return float(fields["dram_bytes_per_launch"]) * float(fields.get("units_per_launch_scale", 1))
    except (KeyError, ValueError):
        return None


# ---------------------------------------------------------------- inputs ----

def _gen_head(args):
    from dynamic_state_memory_b200 import synth
    wl, b, h = args
    st = synth.HeadStream(wl["seed"], b, h, **wl)
    cast = synth.to_bf16_bits if wl["dtype"] == "bf16" else (lambda x: x)
    return b, h, cast(st.q), cast(st.k), cast(st.v)


def make_inputs(wl, rank=0):
    """Host q, k, v [B, H, T, d] of a workload (rank offsets the seed)."""
    from concurrent.futures import ProcessPoolExecutor
    import multiprocessing as mp
    wl = dict(wl, seed=wl["seed"] + 7919 * rank)
    B, H, T, d = wl["B"], wl["H"], wl["T"], wl["d"]
    npdt = np.uint16 if wl["dtype"] == "bf16" else np.float32
    q = np.empty((B, H, T, d), dtype=npdt)
    k = np.empty_like(q)
    v = np.empty_like(q)
    jobs = [(wl, b, h) for b in range(B) for h in range(H)]
    workers = min(len(jobs), max(1, len(os.sched_getaffinity(0))))
    if B * H * T * d < 4_000_000 or workers == 1:
        res = map(_gen_head, jobs)
        for b, h, qq, kk, vv in res:
            q[b, h], k[b, h], v[b, h] = qq, kk, vv
    else:
        with ProcessPoolExecutor(workers, mp_context=mp.get_context("spawn")) as ex:
            for b, h, qq, kk, vv in ex.map(_gen_head, jobs, chunksize=4):
                q[b, h], k[b, h], v[b, h] = qq, kk, vv
    return q, k, v


def to_torch(x, dtype, device):
    import torch
    if dtype == "bf16":
        return torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(device)
    return torch.from_numpy(x).to(device)


# ------------------------------------------------------------ roofline peaks ----

def tensor_peak(peaks, peaks_kind, clocks):
    """The bf16 tensor peak a kernel of this run is held to.

    The measured burst figure (a GEMM timed alone at full clock) when the
    timed region's SM clock stayed at its maximum with no power cap; the
    sustained figure (seconds under the power cap) otherwise."""
    burst = peaks.get("bf16_tflops", PEAKS_FALLBACK["bf16_tflops"])
    sust = peaks.get("bf16_tflops_sustained", PEAKS_FALLBACK["bf16_tflops_sustained"])
    if clocks is None:
        return sust, f"bf16 dense, {peaks_kind} sustained (no clock record)"
    mhz, mx = clocks.get("sm_mhz", 0.0), clocks.get("sm_max_mhz", 0.0)
    capped = "sw_power_cap" in clocks.get("reasons", [])
    if mx and mhz >= 0.98 * mx and not capped:
        return burst, (f"bf16 dense, {peaks_kind} burst: the timed region ran at a median "
                       f"{mhz:.0f} MHz (max {mx:.0f}) with no power cap")
    return sust, (f"bf16 dense, {peaks_kind} sustained: the timed region ran at a median "
                  f"{mhz:.0f} MHz (max {mx:.0f}){', power cap active' if capped else ''}")


# ------------------------------------------------------------ prefill arm ----

def prefill_flops(trace_live_sum, heads_tokens, d):
    """Readout FLOPs: sum_t 2 m_t d^2 + 2 m_t d; plus the state build 2 d^2/token."""
    readout = 2.0 * trace_live_sum * d * d + 2.0 * trace_live_sum * d
    build = 2.0 * heads_tokens * d * d
    return readout, build


def atom_flops(m0_rows_sum, d):
    """FLOPs of the tensor-core readout's atom loop: each row of a 128-token
    tile takes one d x d product per state present before the tile (atom)."""
    return 2.0 * m0_rows_sum * d * d


def _time_steps(step, steps, warmup, stream, world, dev):
    import torch
    for _ in range(warmup):
        step()
    torch.cuda.synchronize(dev)
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    return reduce_max(e0.elapsed_time(e1), world, dev) / steps


def bench_prefill(args, wl, rank, world, local_rank, e2e=True):
    import torch
    from dynamic_state_memory_b200 import dla
    dev = torch.device(f"cuda:{local_rank}")
    torch.cuda.set_device(dev)
    peaks, peaks_kind = load_peaks()
    q_h, k_h, v_h = make_inputs(wl, rank)
    B, H, T, d, C = wl["B"], wl["H"], wl["T"], wl["d"], wl["C"]
    dt = wl["dtype"]
    q, k, v = (to_torch(x, dt, dev) for x in (q_h, k_h, v_h))
    cache = dla.Cache(B, H, C, d, device=dev)
    prof = dla.Profiler(cap=4096)
    dcode = dla.DLA_BF16 if dt == "bf16" else dla.DLA_F32
    cfg = dla.make_config(B, H, T, d, C, wl["tau"], dcode, args.window, prof.p)
    pol = policy_of(args.workload)
    info = pol == "info"
    policy_code = {"info": dla.DLA_POLICY_INFO, "unbounded": dla.DLA_POLICY_UNBOUNDED}.get(
        pol, dla.DLA_POLICY_DYNAMIC)
    run = {"info": dla.dla_info_policy_prefill, "unbounded": dla.dla_unbounded_prefill}.get(
        pol, dla.dla_prefill)
    ws = torch.empty(dla.dla_workspace_bytes(cfg, policy_code), dtype=torch.uint8, device=dev)
    o = torch.empty_like(q)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)

    # one traced run (untimed) whose trace the library reduces on the device
    # (dla_trace_stats) to the live-state counts of the FLOP model
    tr = dla.Trace(B * H, T, T + 1, dev)
    dla.dla_cache_init(cache.c, B, H, C, d, d, cache.base, stream)
    run(cfg, q, k, v, o, cache.c, tr.c, ws, st, stream)
    stats = dla.Stats(B * H, dev)
    sst = stats.reduce(tr, T, tile=128, stream=stream)
    torch.cuda.synchronize(dev)
    dla.check_device_status(st, "dla_prefill")
    dla.check_device_status(sst, "dla_trace_stats")
    del tr
    live_sum = int(stats.live_sum.sum())
    m0_rows = int(stats.atom_rows.sum())
    trace_stats = {"boundaries_per_stream": round(float(stats.boundaries.float().mean()), 2),
                   "merges_per_stream": round(float(stats.merges.float().mean()), 2),
                   "live_max": int(stats.live_max.max())}
    readout_flops, build_flops = prefill_flops(live_sum, B * H * T, d)
    loop_flops = atom_flops(m0_rows, d)

    def step(qq=q, kk=k, vv=v, oo=o):
        dla.dla_cache_init(cache.c, B, H, C, d, d, cache.base, stream)
        run(cfg, qq, kk, vv, oo, cache.c, None, ws, st, stream)

    fixed = args.workload.startswith("fixed")
    if fixed:
        # the fixed Fenwick policy is the timed path; DLA at C is reported beside it
        dla_ms = _time_steps(step, args.steps, args.warmup, stream, world, dev)
        dla_live = live_sum
        fcfg = dla.make_config(B, H, T, d, C, wl["tau"], dcode, 0, prof.p)
        fws = torch.empty(dla.dla_workspace_bytes(fcfg, dla.DLA_POLICY_FENWICK), dtype=torch.uint8,
                          device=dev)
        del ws
        live_sum = int(sum(bin(t).count("1") + 1 for t in range(T))) * B * H
        readout_flops, build_flops = prefill_flops(live_sum, B * H * T, d)
        # Fenwick atoms of tile c: the tree blocks of [0, 128 c), one per set bit of c
        loop_flops = atom_flops(sum(min(128, T - c * 128) * bin(c).count("1")
                                    for c in range((T + 127) // 128)) * B * H, d)

        def step(qq=q, kk=k, vv=v, oo=o):
            dla.dla_fixed_policy_prefill(fcfg, qq, kk, vv, oo, fws, st, stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    prof.reset()
    clk = ClockSampler(local_rank)
    if rank == 0:
        clk.start()
    barrier(world)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier(world)
    clocks = clk.stop() if rank == 0 else None
    dla.check_device_status(st, "dla_prefill")
    ms = e0.elapsed_time(e1)
    ms_max = reduce_max(ms, world, dev)
    launches = prof.p.count
    kt = prof.times_ms()

    in_bytes = sum(x.nbytes for x in (q_h, k_h, v_h))
    e2e_ms = None
    if e2e:
        e2e_ms, out_bytes = _prefill_e2e(args, q_h, k_h, v_h, q, k, v, o, dt, step, stream, st,
                                         world, dev)

    if rank != 0:
        return None
    ms_step = ms_max / args.steps
    tokens = B * T * world
    value = tokens / (ms_step * 1e-3) / 1e6
    # CUDA-event time of each kernel on its own stream. Kernels on concurrent
    # streams overlap, so a low-priority kernel's event time includes the time
    # it waits for SMs: these are not the serialised shares of an ncu launch
    # list. The roofline is the readout's (the contraction), the largest
    # kernel of that serialised list on every prefill workload here.
    # Under the information policy the sequential fp64 score dominates the
    # step and carries the roofline instead.
    tot = {kname: sum(v_) for kname, v_ in kt.items()}
    if info:
        dom = "info_score"
    else:
        dom = "readout" if "readout" in kt else max(tot, key=tot.get)
    per_launch_ms = statistics.mean(kt[dom])
    n_launch = len(kt[dom])
    steps_recorded = args.steps
    step_flops = readout_flops + build_flops
    step_frac = None
    if dom == "readout":
        # the tensor-core readout's timed kernel is its atom loop (the prologue,
        # "readout_pre", runs beside the materializer); the SIMT readout is one
        # kernel doing all of the readout's work
        work = readout_flops if args.path == "simt" else loop_flops
        flops_per_launch = work / (n_launch / steps_recorded)
        if args.path == "simt":
            bound, unit = "alu", "TFLOP/s"
            peak = SMS * FP32_LANES_PER_SM * 2 * peaks.get("sm_max_mhz", 1965.0) * 1e6 / 1e12
            peak_note = "fp32 FMA: 148 SMs x 128 lanes x 2 FLOP x max SM clock (derived)"
        else:
            bound, unit = "tensor", "TFLOP/s"
            peak, peak_note = tensor_peak(peaks, peaks_kind, clocks)
        achieved = flops_per_launch / (per_launch_ms * 1e-3) / 1e12
        # the whole step: every algorithmic FLOP of the readout and the state
        # build over the step time, against the same peak
        step_frac = round(step_flops / (ms_step * 1e-3) / 1e12 / peak, 4)
    elif dom == "info_score":
        # per token: x_t = v_t^T S u_t (2 d^2 FLOP) and the state update
        # S += v_t u_t^T (2 d^2 FLOP), fp64; one CTA (one SM) per head
        flops_per_launch = 4.0 * d * d * B * H * T / (n_launch / steps_recorded)
        bound, unit = "alu", "TFLOP/s"
        peak = SMS * FP64_LANES_PER_SM * 2 * peaks.get("sm_max_mhz", 1965.0) * 1e6 / 1e12
        peak_note = ("fp64 FMA: 148 SMs x 64 lanes x 2 FLOP x max SM clock (derived); the "
                     "kernel runs one SM per head, %d of 148" % min(B * H, SMS))
        achieved = flops_per_launch / (per_launch_ms * 1e-3) / 1e12
    else:
        bound, unit, peak, peak_note = "hbm", "GB/s", peaks.get("hbm_gbs", 6540.8), peaks_kind
        achieved = float("nan")
    traffic = None if args.B else ncu_traffic(dom, "simt" if args.path == "simt" else "tc",
                                              args.workload)
    roof = {"kernel": dom, "bound": bound,
            "achieved": round(achieved, 3), "peak": peak,
            "unit": unit, "frac": round(achieved / peak, 4), "traffic": traffic,
            "peak_source": peak_note, "launch_ms": round(per_launch_ms, 4),
            "launches": n_launch,
            "step_flops": step_flops, "step_frac": step_frac,
            "step_frac_note": "flops_per_step / ms_per_step / peak (readout + state build)"
                              if step_frac is not None else None,
            "event_share": {kk: round(vv / sum(tot.values()), 4) for kk, vv in tot.items()},
            "event_share_note": "CUDA-event time per kernel on its own stream; concurrent "
                                "streams overlap, so these are not serialised shares"}
    cpu = None if args.no_cpu_baseline or world > 1 else cpu_baseline_prefill(
        wl, q_h, k_h, v_h, policy=policy_of(args.workload), target_s=args.cpu_seconds)
    extra = {}
    if info and "readout" in kt:
        # the readout is the dynamic policy's; its atom loop's rate beside
        rl_ms = statistics.mean(kt["readout"])
        ra = loop_flops / (len(kt["readout"]) / steps_recorded) / (rl_ms * 1e-3) / 1e12
        rp, rnote = tensor_peak(peaks, peaks_kind, clocks)
        extra["readout_atom_loop"] = {"achieved": round(ra, 3), "peak": rp, "unit": "TFLOP/s",
                                      "frac": round(ra / rp, 4), "launch_ms": round(rl_ms, 4),
                                      "peak_source": rnote}
    if fixed:
        extra = {"dla_same_inputs": {
            "C": C, "value": round(tokens / (dla_ms * 1e-3) / 1e6, 4), "unit": "Mtok/s",
            "ms_per_step": round(dla_ms, 4), "mean_live_states": round(dla_live / (B * H * T), 2)}}
    return {
        **({"policy": pol} if pol != "dla" else {}), **extra,
        "metric": METRIC, "value": round(value, 4), "unit": "Mtok/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32" if args.path == "simt" else "bf16", "data": "synthetic",
        "config": {"workload": args.workload, "B": B, "H": H, "T": T, "d": d, "C": C,
                   "tau": wl["tau"], "input_dtype": dt, "path": args.path,
                   "l2": "inputs larger than L2 (q+k+v %d MiB), no flush" % (in_bytes >> 20),
                   "flops_per_step": step_flops,
                   "mean_live_states": round(live_sum / (B * H * T), 2),
                   "trace_stats": trace_stats},
        "roofline": roof, "cpu_baseline": cpu,
        "e2e": None if e2e_ms is None else {
            "value": round(tokens / (e2e_ms * 1e-3) / 1e6, 4), "unit": "Mtok/s",
            "h2d_bytes_per_step": in_bytes, "d2h_bytes_per_step": out_bytes},
        "gpu_launches": launches, "clocks": clocks,
    }


def _prefill_e2e(args, q_h, k_h, v_h, q, k, v, o, dt, step, stream, st, world, dev):
    """End to end through the public API with host buffers: every step copies
    its q, k, v in from pinned host memory and its o back out.  Two device
    buffer sets and two copy streams let step i+1's upload and step i's
    download run while step i computes, as a stream of requests would.
    Returns (ms per step, max over ranks; output bytes per step)."""
    import torch
    from dynamic_state_memory_b200 import dla
    pin = [torch.from_numpy(x.view(np.int16) if dt == "bf16" else x).pin_memory()
           for x in (q_h, k_h, v_h)]
    o_host = torch.empty(o.shape, dtype=torch.int16 if dt == "bf16" else torch.float32).pin_memory()
    sets = [(q, k, v, o), tuple(torch.empty_like(x) for x in (q, k, v, o))]
    up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in sets]    # inputs of the set uploaded
    ev_used = [torch.cuda.Event() for _ in sets]  # its step has read the inputs, written o
    ev_out = [torch.cuda.Event() for _ in sets]   # its o downloaded

    def e2e_run(n):
        up.wait_stream(stream)
        for i in range(n):
            j = i % 2
            qq, kk, vv, oo = sets[j]
            up.wait_event(ev_used[j])
            with torch.cuda.stream(up):
                for hsrc, ddst in zip(pin, (qq, kk, vv)):
                    ddst.view(hsrc.dtype).copy_(hsrc, non_blocking=True)
                ev_in[j].record(up)
            stream.wait_event(ev_in[j])
            stream.wait_event(ev_out[j])
            step(qq, kk, vv, oo)
            ev_used[j].record(stream)
            down.wait_event(ev_used[j])
            with torch.cuda.stream(down):
                o_host.copy_(oo.view(o_host.dtype), non_blocking=True)
                ev_out[j].record(down)
        stream.wait_stream(down)

    e2e_run(max(2, args.warmup // 2))
    torch.cuda.synchronize(dev)
    barrier(world)
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    e2e_steps = max(2, args.steps)
    e2e_run(e2e_steps)
    f1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = reduce_max(f0.elapsed_time(f1) / e2e_steps, world, dev)
    dla.check_device_status(st, "dla_prefill")
    # the pipelined output is the device-timed step's output, bit for bit
    if not torch.equal(o_host, o.view(o_host.dtype).cpu()):
        raise RuntimeError("end-to-end output differs from the device-timed output")
    return e2e_ms, o_host.numel() * o_host.element_size()


def oracle_heads(wl, cores):
    """The streams the oracle runs as its bounded sample of a prefill
    workload: the first min(B*H, cores) streams, full length."""
    return min(wl["B"] * wl["H"], cores)


def cpu_baseline_prefill(wl, q, k, v, target_s=15.0, policy="dla"):
    """The oracle as it stands on a bounded sample of the same workload: the
    first streams (one per host core), full per-token work, from the first
    256 tokens up until one run takes a quarter of the target or covers the
    whole sequence (each longer prefix sized from the last run's time, at
    most x4)."""
    from oracle import oracle as O
    cores = O.cores()
    B, H, T, d = wl["B"], wl["H"], wl["T"], wl["d"]
    heads = oracle_heads(wl, cores)
    Ts = min(T, 256)
    t_used = 0.0
    while True:
        qs = q.reshape(B * H, T, d)[:heads, :Ts]
        ks = k.reshape(B * H, T, d)[:heads, :Ts]
        vs = v.reshape(B * H, T, d)[:heads, :Ts]
        orc = O.Oracle(heads, d, d, wl["C"], policy)
        t0 = time.perf_counter()
        orc.run(ks, qs, vs, tau=wl["tau"], dtype=wl["dtype"], nthreads=cores)
        t_used = time.perf_counter() - t0
        if t_used > target_s / 4 or Ts >= T:
            break
        # a longer prefix costs more than in proportion (more live states),
        # so aim at half the remaining factor
        grow = min(4.0, 0.5 * (target_s / 4) / max(t_used, 1e-3) + 1.0)
        Ts = min(T, max(Ts + 256, int(Ts * grow) // 256 * 256))
    head_tokens_s = heads * Ts / t_used
    return {"value": round(head_tokens_s / H / 1e6, 6), "unit": "Mtok/s", "cores": cores,
            "kind": "oracle",
            "sample": f"{policy} policy, {heads} heads x first {Ts} tokens of the workload, "
                      f"full per-token work; "
                      f"Mtok/s = head-tokens/s / H ({t_used:.1f} s)"}


# ----------------------------------------------------------- backward arm ----

def backward_flops(T, d, heads):
    """The masked form's products per stream: every (t, s <= t) pair takes
    phi(q_t).phi(k_s), dO_t.v_s and dphi(q_t)'s term in the row pass, and the
    two dot products again plus dv_s's and dphi(k_s)'s terms in the column
    pass: 7 d T (T + 1) FLOP (2 per multiply-add)."""
    return 7.0 * d * T * (T + 1) * heads


def bench_backward(args, wl, rank, world, local_rank):
    """dla_prefill_backward at the decisions of one traced dla_prefill
    (untimed): each step is one call (its three kernels) over the batch."""
    import torch
    from dynamic_state_memory_b200 import dla
    dev = torch.device(f"cuda:{local_rank}")
    torch.cuda.set_device(dev)
    peaks, peaks_kind = load_peaks()
    B, H, T, d, C = wl["B"], wl["H"], wl["T"], wl["d"], wl["C"]
    dt = wl["dtype"]
    q_h, k_h, v_h = make_inputs(wl, rank)
    do32 = np.random.default_rng([wl["seed"], 7, rank]).standard_normal(q_h.shape).astype(np.float32)
    from dynamic_state_memory_b200 import synth
    do_h = synth.to_bf16_bits(do32) if dt == "bf16" else do32
    q, k, v, d_o = (to_torch(x, dt, dev) for x in (q_h, k_h, v_h, do_h))
    cache = dla.Cache(B, H, C, d, device=dev)
    _, tr = dla.prefill(q, k, v, cache, wl["tau"])
    dcode = dla.DLA_BF16 if dt == "bf16" else dla.DLA_F32
    cfg = dla.make_config(B, H, T, d, C, wl["tau"], dcode)
    ws = torch.empty(dla.dla_backward_workspace_bytes(cfg), dtype=torch.uint8, device=dev)
    dq, dk, dv = (torch.empty(B, H, T, d, dtype=torch.float32, device=dev) for _ in range(3))
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        dla.dla_prefill_backward(cfg, q, k, v, d_o, tr.c, dq, dk, dv, ws, st, stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    clk = ClockSampler(local_rank)
    if rank == 0:
        clk.start()
    barrier(world)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier(world)
    clocks = clk.stop() if rank == 0 else None
    dla.check_device_status(st, "dla_prefill_backward")
    ms_step = reduce_max(e0.elapsed_time(e1), world, dev) / args.steps
    if rank != 0:
        return None
    flops = backward_flops(T, d, B * H)
    achieved = flops / (ms_step * 1e-3) / 1e12
    peak = SMS * FP32_LANES_PER_SM * 2 * peaks.get("sm_max_mhz", 1965.0) * 1e6 / 1e12
    cpu = None if args.no_cpu_baseline or world > 1 else cpu_baseline_backward(
        wl, q_h, k_h, v_h, do_h, target_s=min(args.cpu_seconds, 8.0))
    return {
        "metric": METRIC, "value": round(B * T * world / (ms_step * 1e-3) / 1e6, 4),
        "unit": "Mtok/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms_step, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": args.workload, "B": B, "H": H, "T": T, "d": d, "C": C,
                   "tau": wl["tau"], "input_dtype": dt, "path": "simt",
                   "l2": "q, k, v, dO %d MiB; the kernels re-read them from L2" %
                         (4 * q_h.nbytes >> 20),
                   "flops_per_step": flops},
        "roofline": {"kernel": "backward (3 kernels)", "bound": "alu",
                     "achieved": round(achieved, 3), "peak": round(peak, 1), "unit": "TFLOP/s",
                     "frac": round(achieved / peak, 4), "traffic": None,
                     "peak_source": "fp32 FMA: 148 SMs x 128 lanes x 2 FLOP x max SM clock "
                                    "(derived)"},
        "cpu_baseline": cpu, "e2e": None, "gpu_launches": 3 * args.steps, "clocks": clocks,
    }


def cpu_baseline_backward(wl, q, k, v, d_o, target_s=8.0):
    """The oracle's gradient (oracle/backward.py, BLAS held to one thread) on
    the first streams of the workload, full length, until target_s of work;
    the C oracle's forward gives each stream's trace (untimed)."""
    from threadpoolctl import threadpool_limits
    from dynamic_state_memory_b200 import synth
    from oracle import backward as BW
    from oracle import oracle as O
    B, H, T, d = wl["B"], wl["H"], wl["T"], wl["d"]
    w = lambda x: synth.widen(x, wl["dtype"])
    used, heads = 0.0, 0
    with threadpool_limits(1):
        while heads < B * H and used < target_s:
            b, h = divmod(heads, H)
            ref = O.prefill(q[b:b + 1, h:h + 1], k[b:b + 1, h:h + 1], v[b:b + 1, h:h + 1],
                            C=wl["C"], tau=wl["tau"], dtype=wl["dtype"], want_out=False)
            t0 = time.perf_counter()
            BW.backward_head(w(q[b, h]), w(k[b, h]), w(v[b, h]), w(d_o[b, h]),
                             ref["boundary"][0, 0], ref["merges"][0])
            used += time.perf_counter() - t0
            heads += 1
    return {"value": round(heads * T / used / H / 1e6, 6), "unit": "Mtok/s", "cores": 1,
            "kind": "oracle",
            "sample": f"oracle gradient, {heads} streams x {T} tokens, one thread; "
                      f"Mtok/s = stream-tokens/s / H ({used:.1f} s)"}


# ------------------------------------------------------------- decode arm ----

def _gen_decode_head(args):
    from dynamic_state_memory_b200 import synth
    wl, n, h, steps = args
    st = synth.HeadStream(wl["seed"], n, h, **wl)
    q, k, v = st.decode_steps(steps, wl["switch_p"])
    c = synth.to_bf16_bits
    return n, h, c(st.q), c(st.k), c(st.v), c(q), c(k), c(v)


def make_decode_inputs(wl, steps, rank=0):
    from concurrent.futures import ProcessPoolExecutor
    import multiprocessing as mp
    wl = dict(wl, seed=wl["seed"] + 7919 * rank)
    N, H, T, d = wl["B"], wl["H"], wl["T"], wl["d"]
    pre = [np.empty((N, H, T, d), dtype=np.uint16) for _ in range(3)]
    stp = [np.empty((steps, N, H, d), dtype=np.uint16) for _ in range(3)]
    jobs = [(wl, n, h, steps) for n in range(N) for h in range(H)]
    workers = min(len(jobs), max(1, len(os.sched_getaffinity(0))))
    with ProcessPoolExecutor(workers, mp_context=mp.get_context("spawn")) as ex:
        for n, h, pq, pk, pv, sq, sk, sv in ex.map(_gen_decode_head, jobs, chunksize=16):
            pre[0][n, h], pre[1][n, h], pre[2][n, h] = pq, pk, pv
            stp[0][:, n, h], stp[1][:, n, h], stp[2][:, n, h] = sq, sk, sv
    return pre, stp


def bench_decode(args, wl, rank, world, local_rank):
    import torch
    from dynamic_state_memory_b200 import dla
    dev = torch.device(f"cuda:{local_rank}")
    torch.cuda.set_device(dev)
    peaks, peaks_kind = load_peaks()
    N, H, T, d, C, tau = wl["B"], wl["H"], wl["T"], wl["d"], wl["C"], wl["tau"]
    nsteps = args.warmup + args.steps
    pre_h, stp_h = make_decode_inputs(wl, nsteps, rank)
    cache = dla.Cache(N, H, C, d, device=dev)
    stream = torch.cuda.current_stream(dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    # pre-fill every stream's cache with a T-token prefill, in sequence chunks
    chunk = 8
    cfg = dla.make_config(chunk, H, T, d, C, tau, dla.DLA_BF16, 1024)
    ws = torch.empty(dla.dla_workspace_bytes(cfg), dtype=torch.uint8, device=dev)
    for n0 in range(0, N, chunk):
        qq, kk, vv = (to_torch(np.ascontiguousarray(x[n0:n0 + chunk]), "bf16", dev) for x in pre_h)
        o = torch.empty_like(qq)
        dla.dla_prefill(cfg, qq, kk, vv, o, cache.sub(n0, n0 + chunk), None, ws, st, stream)
    torch.cuda.synchronize(dev)
    dla.check_device_status(st, "prefill of the decode cache")
    del ws, o, qq, kk, vv
    sq, sk, sv = (to_torch(x, "bf16", dev) for x in stp_h)
    dec = dla.Decoder(cache, dev)
    prof = dla.Profiler(cap=4 * nsteps + 16)
    o = torch.empty(N, H, d, dtype=torch.bfloat16, device=dev)
    for i in range(args.warmup):
        dec.step(sq[i], sk[i], sv[i], tau, o, stream)
    torch.cuda.synchronize(dev)
    m_before = int(cache.views()["m"].sum())
    prof.reset()
    clk = ClockSampler(local_rank)
    if rank == 0:
        clk.start()
    barrier(world)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(args.warmup, nsteps):
        dec.step(sq[i], sk[i], sv[i], tau, o, stream, prof.p)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier(world)
    clocks = clk.stop() if rank == 0 else None
    dla.check_device_status(dec.status, "dla_decode_step")
    m_after = int(cache.views()["m"].sum())
    ms = reduce_max(e0.elapsed_time(e1), world, dev)
    kt = prof.times_ms()
    launches = prof.p.count
    # End to end: each step's q, k, v come in from pinned host memory and its o
    # goes back. Steps depend on one another through the cache, so only the
    # copies overlap: step i+1's upload and step i's download run on copy
    # streams while step i computes (two device buffer sets).
    hq, hk, hv = (torch.from_numpy(x.view(np.int16)).pin_memory() for x in stp_h)
    dsets = [tuple(torch.empty(N, H, d, dtype=torch.int16, device=dev) for _ in range(4))
             for _ in range(2)]
    ho = torch.empty(N, H, d, dtype=torch.int16).pin_memory()
    up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in dsets]
    ev_used = [torch.cuda.Event() for _ in dsets]
    ev_out = [torch.cuda.Event() for _ in dsets]
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    f0.record(stream)
    up.wait_stream(stream)
    e2e_steps = min(args.steps, 8)
    for i in range(e2e_steps):
        j, b = args.warmup + i, i % 2
        dq, dk_, dv, do = dsets[b]
        up.wait_event(ev_used[b])
        with torch.cuda.stream(up):
            dq.copy_(hq[j], non_blocking=True)
            dk_.copy_(hk[j], non_blocking=True)
            dv.copy_(hv[j], non_blocking=True)
            ev_in[b].record(up)
        stream.wait_event(ev_in[b])
        stream.wait_event(ev_out[b])
        dec.step(dq.view(torch.bfloat16), dk_.view(torch.bfloat16), dv.view(torch.bfloat16), tau,
                 do.view(torch.bfloat16), stream)
        ev_used[b].record(stream)
        down.wait_event(ev_used[b])
        with torch.cuda.stream(down):
            ho.copy_(do, non_blocking=True)
            ev_out[b].record(down)
    stream.wait_stream(down)
    f1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = reduce_max(f0.elapsed_time(f1) / e2e_steps, world, dev)
    dla.check_device_status(dec.status, "dla_decode_step")
    del cache, dec, sq, sk, sv, dsets
    if rank != 0:
        return None
    ms_step = ms / args.steps
    value = world * 1000.0 / ms_step
    tot = {kk: sum(vv) for kk, vv in kt.items()}
    stream_ms = statistics.mean(kt["decode_stream"])
    live = 0.5 * (m_before + m_after)
    state_bytes = live * d * d * 4
    achieved = state_bytes / (stream_ms * 1e-3) / 1e9
    peak = peaks.get("hbm_gbs", 6540.8)
    step_bytes_frac = state_bytes / (ms_step * 1e-3) / 1e9 / peak
    roof = {"kernel": "decode_stream", "bound": "hbm", "achieved": round(achieved, 1), "peak": peak,
            "unit": "GB/s", "frac": round(achieved / peak, 4),
            "traffic": None if args.B else ncu_traffic("decode_stream", "-", "decode_n256"),
            "peak_source": f"{peaks_kind} copy bandwidth",
            "algorithmic_bytes_per_launch": state_bytes, "launch_ms": round(stream_ms, 4),
            "launches": len(kt["decode_stream"]),
            "step_frac": round(step_bytes_frac, 4),
            "step_frac_note": "state bytes per step / ms_per_step / peak (decision kernel included)",
            "kernel_share": {kk: round(vv / sum(tot.values()), 4) for kk, vv in tot.items()}}
    cpu = None if args.no_cpu_baseline or world > 1 else cpu_baseline_decode(wl, pre_h, stp_h)
    return {
        "metric": METRIC, "value": round(value, 3), "unit": "steps/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic",
        "config": {"workload": "decode_n256", "N": N, "H": H, "prefill_T": T, "d": d, "C": C,
                   "tau": tau, "input_dtype": "bf16", "state_dtype": "f32",
                   "mean_live_states": round(live / (N * H), 2),
                   "l2": "state cache %d GiB >> L2, no flush" % ((N * H * C * d * d * 4) >> 30)},
        "roofline": roof, "cpu_baseline": cpu,
        "e2e": {"value": round(world * 1000.0 / e2e_ms, 3), "unit": "steps/s",
                "h2d_bytes_per_step": 3 * N * H * d * 2, "d2h_bytes_per_step": N * H * d * 2},
        "gpu_launches": launches, "clocks": clocks,
    }


def oracle_decode(wl, pre, stp, steps, cores, streams=16, prefill_tokens=4096, total=None):
    """Oracle decode on a bounded sample: `streams` streams pre-filled with
    their workload tokens (untimed; states updated at every token, no
    readout), then `steps` timed single-token steps with full per-token work.
    Returns (seconds per step for the sample, sample description); the
    description names `total` streams (default: all of `wl`'s) as the
    extrapolation target."""
    from oracle import oracle as O
    N, H, d = wl["B"], wl["H"], wl["d"]
    U = min(streams, N * H)
    Tp = min(prefill_tokens, wl["T"])
    k = pre[1].reshape(N * H, -1, d)[:U, :Tp]
    q = pre[0].reshape(N * H, -1, d)[:U, :Tp]
    v = pre[2].reshape(N * H, -1, d)[:U, :Tp]
    orc = O.Oracle(U, d, d, wl["C"])
    orc.run(k, q, v, tau=wl["tau"], dtype="bf16", nthreads=cores,
            out_mask=np.zeros(Tp, dtype=np.uint8))
    sk = stp[1].reshape(stp[1].shape[0], N * H, d)
    sq = stp[0].reshape(stp[0].shape[0], N * H, d)
    sv = stp[2].reshape(stp[2].shape[0], N * H, d)
    n = min(steps, sk.shape[0])
    t0 = time.perf_counter()
    for i in range(n):
        orc.run(np.ascontiguousarray(sk[i, :U, None]), np.ascontiguousarray(sq[i, :U, None]),
                np.ascontiguousarray(sv[i, :U, None]), tau=wl["tau"], dtype="bf16",
                nthreads=cores)
    dt = (time.perf_counter() - t0) / n
    total = N * H if total is None else total
    return dt, U, (f"{U} streams pre-filled with {Tp} tokens (untimed), {n} timed steps; "
                   f"steps/s extrapolated to {total} streams")


def cpu_baseline_decode(wl, pre, stp, steps=8):
    """Oracle decode steps/s, extrapolated from its sample to every stream."""
    from oracle import oracle as O
    cores = O.cores()
    dt, U, sample = oracle_decode(wl, pre, stp, steps, cores)
    N, H = wl["B"], wl["H"]
    return {"value": round(1.0 / (dt * (N * H) / U), 6), "unit": "steps/s", "cores": cores,
            "kind": "oracle", "sample": sample}


# ------------------------------------------------------------ reference arm ----

def bench_reference(args, wl):
    """The oracle as it stands, on the same bounded sample as our arm's
    cpu_baseline: the first min(B*H, cores) streams at full length (or the
    first --ref-tokens tokens), full per-token work, every step."""
    from oracle import oracle as O
    from dynamic_state_memory_b200 import synth
    cores = O.cores()
    B, H, T, d = wl["B"], wl["H"], wl["T"], wl["d"]
    heads = oracle_heads(wl, cores)
    Ts = T if args.ref_tokens <= 0 else min(T, args.ref_tokens)
    pol = policy_of(args.workload)
    q, k, v = (np.empty((heads, Ts, d), dtype=np.uint16 if wl["dtype"] == "bf16" else np.float32)
               for _ in range(3))
    cast = synth.to_bf16_bits if wl["dtype"] == "bf16" else (lambda x: np.ascontiguousarray(x, np.float32))
    for i in range(heads):
        stv = synth.HeadStream(wl["seed"], i // H, i % H, **wl)
        q[i], k[i], v[i] = cast(stv.q[:Ts]), cast(stv.k[:Ts]), cast(stv.v[:Ts])
    times = []
    for i in range(args.warmup + args.steps):
        orc = O.Oracle(heads, d, d, wl["C"], pol)
        t0 = time.perf_counter()
        orc.run(k, q, v, tau=wl["tau"], dtype=wl["dtype"], nthreads=cores)
        dt = time.perf_counter() - t0
        if i >= args.warmup:
            times.append(dt)
    mean = sum(times) / len(times)
    val = heads * Ts / mean / H / 1e6
    sample = (f"{pol} policy, {heads} heads x first {Ts} tokens of the workload per step, full "
              f"per-token work (the sample of the GPU arm's cpu_baseline); Mtok/s = "
              f"head-tokens/s / H")
    line = {"impl": "reference", "metric": METRIC, "value": round(val, 6), "unit": "Mtok/s",
            "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(mean * 1e3, 3), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": args.workload, "B": B, "H": H, "T": T, "d": d,
                       "C": wl["C"], "tau": wl["tau"]},
            "cpu_baseline": {"value": round(val, 6), "unit": "Mtok/s", "cores": cores,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(val, 6), "unit": "Mtok/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    if args.workload == "prefill_t8192" and not args.only:
        # the decode half of the metric, on the decode workload's sample
        dwl = dict(synth.WORKLOADS["decode_n256"])
        U = 16
        pre = [np.empty((1, U, dwl["T"], d), dtype=np.uint16) for _ in range(3)]
        nst = min(args.steps, 8)
        stp = [np.empty((nst, 1, U, d), dtype=np.uint16) for _ in range(3)]
        for i in range(U):
            stv = synth.HeadStream(dwl["seed"], i // dwl["H"], i % dwl["H"], **dwl)
            sq_, sk_, sv_ = stv.decode_steps(nst, dwl["switch_p"])
            for j, (p_, s_) in enumerate(((stv.q, sq_), (stv.k, sk_), (stv.v, sv_))):
                pre[j][0, i] = synth.to_bf16_bits(p_)
                stp[j][:, 0, i] = synth.to_bf16_bits(s_)
        dt, Us, dsample = oracle_decode(dict(dwl, B=1, H=U), pre, stp, nst, cores, streams=U,
                                        total=dwl["B"] * dwl["H"])
        dval = 1.0 / (dt * (dwl["B"] * dwl["H"]) / Us)
        line["decode"] = {"value": round(dval, 6), "unit": "steps/s",
                          "ms_per_step": round(1e3 / dval, 3),
                          "config": {"workload": "decode_n256"},
                          "cpu_baseline": {"value": round(dval, 6), "unit": "steps/s",
                                           "cores": cores, "kind": "oracle",
                                           "sample": dsample}}
    return line


# ------------------------------------------------------------------ plumbing ----

def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def reduce_max(x, world, dev):
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def _free_port():
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def relaunch(n):
    """Run this command as n ranks under torchrun (one process per GPU) and
    return its exit status: `--gpus N` without an outer launcher."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr", "127.0.0.1", f"--master-port={_free_port()}",
           os.path.abspath(__file__), *sys.argv[1:]]
    return subprocess.run(cmd, timeout=3 * 3600).returncode


def sub_args(args, workload, steps=None, warmup=None):
    """A copy of the command's arguments for another workload."""
    from dynamic_state_memory_b200 import synth
    a = argparse.Namespace(**vars(args))
    a.workload = workload
    a.steps = args.steps if steps is None else steps
    a.warmup = args.warmup if warmup is None else warmup
    wl = synth.WORKLOADS[workload]
    a.path = "tc" if (wl["dtype"] == "bf16" and wl["d"] == 128) else "simt"
    a.B = 0
    a.window = 0
    return a


def guarded(fn, *a, **kw):
    """A secondary measurement: its failure is reported in the line, it does
    not lose the headline."""
    try:
        return fn(*a, **kw)
    except Exception as exc:  # noqa: BLE001
        return {"error": f"{type(exc).__name__}: {exc}"[:300]}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="prefill_t8192")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--window", type=int, default=0)
    ap.add_argument("--path", default="auto", help="reported path; auto = tc for bf16 d=128")
    ap.add_argument("--ref-tokens", type=int, default=0,
                    help="reference arm: tokens per stream (0 = the whole sequence)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="target CPU time of the oracle's cpu_baseline sample")
    ap.add_argument("--only", action="store_true",
                    help="the named workload alone (no decode or other configurations nested)")
    ap.add_argument("--B", type=int, default=0, help="override the batch (profiling runs)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        sys.exit(relaunch(args.gpus))
    from dynamic_state_memory_b200 import synth
    wl = dict(synth.WORKLOADS[args.workload])
    if args.B:
        wl["B"] = args.B
    if args.path == "auto":
        args.path = "tc" if (wl["dtype"] == "bf16" and wl["d"] == 128) else "simt"
    rank, world, local_rank = dist_env()
    if world != args.gpus:
        print(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={world}", file=sys.stderr)
        sys.exit(2)
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(bench_reference(args, wl)), flush=True)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600))
    if args.workload.startswith("decode"):
        res = bench_decode(args, wl, rank, world, local_rank)
    elif args.workload.startswith("backward"):
        res = bench_backward(args, wl, rank, world, local_rank)
    else:
        res = bench_prefill(args, wl, rank, world, local_rank)
        if args.workload == "prefill_t8192" and not args.only:
            # the metric's other half and the other configurations, nested in
            # the same line (every rank runs them: they hold barriers)
            import torch
            torch.cuda.empty_cache()
            dec = guarded(bench_decode, sub_args(args, "decode_n256"),
                          dict(synth.WORKLOADS["decode_n256"]), rank, world, local_rank)
            torch.cuda.empty_cache()
            others = {}
            for name in ("prefill_t131072", "fixed_t32768", "unbounded_t8192"):
                a = sub_args(args, name, steps=min(args.steps, 10), warmup=3)
                a.cpu_seconds = min(args.cpu_seconds, 8.0)
                others[name] = guarded(bench_prefill, a, dict(synth.WORKLOADS[name]), rank, world,
                                       local_rank, e2e=False)
                torch.cuda.empty_cache()
            a = sub_args(args, "backward_t2048", steps=min(args.steps, 10), warmup=3)
            a.cpu_seconds = min(args.cpu_seconds, 8.0)
            others["backward_t2048"] = guarded(bench_backward, a,
                                               dict(synth.WORKLOADS["backward_t2048"]), rank,
                                               world, local_rank)
            torch.cuda.empty_cache()
            if rank == 0:
                res["decode"] = dec
                res["configs"] = others
    if rank == 0:
        print(json.dumps(res), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()

"""Benchmark of the fused exact-attention forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

Metric: attention forward TFLOP/s = 4*B*Hq*Nq*Nkv*d / t, halved for causal,
also given as a fraction of the measured dense bf16 tensor peak. One step is
one attn_fwd call over the whole workload (inputs resident in HBM). Prints ONE
JSON line (rank 0). Under torchrun each rank runs its own independent batch of
the workload (weak scaling; no data-path collective), the timed region is
bracketed by barriers and the time is the max over ranks.

``--impl reference`` times the fp64 CPU oracle on the host cores over a
bounded sample of the same workload (the only other use of ``oracle/`` here,
besides the ``cpu_baseline`` leg of the default run).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from synthetic import (VARLEN_WORKLOADS, WORKLOADS, Workload, bf16_bits, make_dout, make_qkv,  # noqa: E402
                       make_varlen, make_varlen_dout)

HEADLINE = "outlier_8k_causal"
EXTRA_BF16 = ["tiny_256_d64", "causal_2k_d128", "outlier_8k_full", "gqa_32k_d128", "gqa_32k_d64",
              "d256_8k_causal", "kvcache_128k_q128", "kvcache_128k_q128_splitkv"]
# short workloads also timed as CUDA-graph replays (launch path off the device clock)
GRAPH_TIMED = {"tiny_256_d64", "causal_2k_d128"}
METRIC = "attn fwd TFLOP/s (4·B·H·N²·d, causal halved), % of B200 dense BF16 peak"
L2_BYTES = 126 * 2 ** 20
KERNEL_SOURCES = ["exact_attention_134_b200/csrc/attn_fwd_sm100.cu",
                  "exact_attention_134_b200/csrc/sm100_ptx.cuh"]


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {"bf16": d["bf16_tflops"], "bf16_sustained": d.get("bf16_tflops_sustained"),
                "hbm": d["hbm_gbs"], "source": "measured"}
    return {"bf16": 1590.0, "bf16_sustained": 1400.0, "hbm": 6650.0, "source": "fallback"}


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def _traffic_from_profile(workload: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current kernel source; else None."""
    path = os.path.join(ROOT, "profiles", "attn_fwd_bf16_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    if d.get("kernel_source_hash") != kernel_source_hash():
        return None
    per = d.get("per_workload", {}).get(workload)
    return None if per is None else per.get("dram_bytes_per_launch")


class NvmlClockSampler:
    """SM clock and throttle reasons read through NVML (read-only queries) by a
    thread polling about every millisecond, so even a timed region of a few
    milliseconds is sampled. The GPU is found by the CUDA device's PCI bus id."""

    def __init__(self, device_index: int):
        import pynvml
        import torch
        self.nv = pynvml
        pynvml.nvmlInit()
        prop = torch.cuda.get_device_properties(device_index)
        bus = f"{prop.pci_domain_id:08x}:{prop.pci_bus_id:02x}:{prop.pci_device_id:02x}.0"
        self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM))
        self.samples = []
        self.stop_event = threading.Event()

    def start(self):
        self.thread = threading.Thread(target=self._poll, daemon=True)
        self.thread.start()

    def _poll(self):
        nv = self.nv
        while True:
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                reasons = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((float(mhz), int(reasons)))
            except Exception:  # a failed read is skipped, not fatal
                pass
            if self.stop_event.wait(0.001):
                return

    def stop(self):
        self.stop_event.set()
        self.thread.join(timeout=5)
        nv = self.nv
        bits = {"hw_slowdown": nv.nvmlClocksEventReasonHwSlowdown,
                "hw_thermal_slowdown": nv.nvmlClocksEventReasonHwThermalSlowdown,
                "sw_thermal_slowdown": nv.nvmlClocksEventReasonSwThermalSlowdown,
                "sw_power_cap": nv.nvmlClocksEventReasonSwPowerCap}
        try:
            nv.nvmlShutdown()
        except Exception:
            pass
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["no samples"], "source": "nvml"}
        reasons = sorted(n for n, b in bits.items() if any(r & b for _, r in self.samples))
        return {"sm_mhz": statistics.median(m for m, _ in self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(self.samples), "source": "nvml"}


def clock_sampler(device_index: int):
    """NVML sampler when NVML answers for this device, else nvidia-smi."""
    try:
        return NvmlClockSampler(device_index)
    except Exception:
        return ClockSampler(device_index)


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200", "-i", str(self.dev)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (FileNotFoundError, OSError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=5)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for n, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax),
                "reasons": sorted(reasons), "samples": len(sm)}


def _dist_setup():
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def _barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def _max_over_ranks(x: float, world: int) -> float:
    """Timing only (not on the data path): the slowest rank's time."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    on_gpu = dist.get_backend() == "nccl"
    t = torch.tensor([x], dtype=torch.float64, device="cuda" if on_gpu else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_tflops(flops_per_rank: float, world: int, max_ms: float) -> float:
    """Whole-job throughput: all ranks' work over the slowest rank's time."""
    return world * flops_per_rank / (max_ms * 1e-3) / 1e12


def workload_config(w: Workload, l2_mode: str) -> dict:
    """The JSON line's `config`: the same dict for both arms of a workload."""
    return {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "Nq": w.Nq, "Nkv": w.Nkv, "d": w.d,
            "causal": w.causal, "scale": "1/sqrt(d)", "l2": l2_mode,
            "per_rank": "independent batch (seed + 1000*rank)"}


def l2_mode_of(w: Workload) -> str:
    """Inputs larger than L2, or an L2 flush between steps (as bench_workload)."""
    in_bytes = 2 * (2 * w.B * w.Hq * w.Nq * w.d + 2 * w.B * w.Hkv * w.Nkv * w.d) + 4 * w.B * w.Hq * w.Nq
    return "inputs_larger_than_l2" if in_bytes >= 2 * L2_BYTES else "l2_flushed_between_steps"


def rank_workload(w: Workload, rank: int) -> Workload:
    """Each rank owns an independent batch of the workload (its own seed)."""
    if rank == 0:
        return w
    return Workload(**{**w.__dict__, "seed": w.seed + 1000 * rank})


# --------------------------------------------------------------------------- ours
def time_device(fn, steps: int, warmup: int, flush=None):
    """CUDA-event time of each call on the current stream (ms list)."""
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    times = []
    for _ in range(steps):
        if flush is not None:
            flush()
        s = torch.cuda.Event(enable_timing=True)
        e = torch.cuda.Event(enable_timing=True)
        s.record()
        fn()
        e.record()
        e.synchronize()
        times.append(s.elapsed_time(e))
    return times


def time_graph_replays(step, steps: int, flush):
    """The same step captured once in a CUDA graph and replayed: the device
    time without the host-side launch path (argument checks, tensor-map
    encoding, the launch itself) between the two events."""
    import torch
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    # relaxed: the library sets a kernel attribute (not a stream operation) per call
    with torch.cuda.graph(g, capture_error_mode="relaxed"):
        step()
    times = time_device(g.replay, steps, 3, flush)
    del g
    return times


def bench_workload(w: Workload, steps: int, warmup: int, world: int, rank: int, lib_mod,
                   graph: bool = False, qk_format: str = "int8"):
    import torch
    wr = rank_workload(w, rank)
    q, k, v = make_qkv(wr.B, wr.Hq, wr.Hkv, wr.Nq, wr.Nkv, wr.d, wr.seed, wr.dist)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    o = torch.empty_like(qd)
    lse = torch.empty((wr.B, wr.Hq, wr.Nq), dtype=torch.float32, device="cuda")
    in_bytes = 2 * (q.numel() + k.numel() + v.numel()) + 2 * o.numel() + 4 * lse.numel()
    flush = None
    l2_mode = l2_mode_of(w)
    if l2_mode != "inputs_larger_than_l2":
        scratch = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device="cuda")
        flush = lambda: scratch.zero_()  # noqa: E731

    if w.path == "q8":
        ws = torch.empty(lib_mod.q8_workspace_size(wr.B, wr.Hq, wr.Hkv, wr.Nq, wr.Nkv, wr.d),
                         dtype=torch.uint8, device="cuda")

        def step():
            lib_mod.attn_fwd_q8(qd, kd, vd, causal=w.causal, workspace=ws, out=o, lse=lse,
                                qk_format=qk_format)
    elif w.path == "splitkv":
        need = int(lib_mod.lib().attn_fwd_splitkv_workspace_size(wr.B, wr.Hq, wr.Hkv, wr.Nq, wr.Nkv,
                                                                   wr.d, 0))
        ws = torch.empty(max(need, 16), dtype=torch.uint8, device="cuda")

        def step():
            lib_mod.attn_fwd_splitkv(qd, kd, vd, causal=w.causal, workspace=ws, out=o, lse=lse)
    else:
        def step():
            lib_mod.attn_fwd(qd, kd, vd, causal=w.causal, out=o, lse=lse)

    for _ in range(max(warmup, 3)):
        step()
    torch.cuda.synchronize()
    _barrier(world)
    torch.cuda.synchronize()
    times = time_device(step, steps, 0, flush)
    torch.cuda.synchronize()
    _barrier(world)
    st, where = lib_mod.get_status()
    if st != 0:
        raise RuntimeError(f"device status {st} at {where:#x}")
    total_ms = _max_over_ranks(sum(times), world)
    res = {"total_ms": total_ms, "times": times, "l2": l2_mode, "inputs": (q, k, v),
           "flops": w.flops}
    if graph:
        # every rank takes part in both reductions, whatever happened locally
        err, local_ms = None, 0.0
        try:
            gt = time_graph_replays(step, steps, flush)
            st, where = lib_mod.get_status()
            if st != 0:
                raise RuntimeError(f"device status {st} at {where:#x}")
            local_ms = sum(gt)
        except Exception as e:  # noqa: BLE001 - reported in the JSON line, eager time stands
            err = f"{type(e).__name__}: {e}"[:200]
        any_err = _max_over_ranks(1.0 if err else 0.0, world)
        graph_ms = _max_over_ranks(local_ms, world)
        if any_err == 0.0:
            res["graph_total_ms"] = graph_ms
        else:
            res["graph_error"] = err or "graph timing failed on another rank"
    return res


def bench_q8(w: Workload, steps: int, warmup: int, world: int, rank: int, lib_mod,
             qk_format: str = "int8"):
    """8-bit path (INT8 Q K^T after smoothing, or with qk_format="fp8" FP8 Q K^T
    with block scales): time of the whole call (3 prepass launches + main
    kernel) and of the prepass alone; the main kernel's share is the difference."""
    import torch
    wr = rank_workload(w, rank)
    q, k, v = make_qkv(wr.B, wr.Hq, wr.Hkv, wr.Nq, wr.Nkv, wr.d, wr.seed, wr.dist)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    o = torch.empty_like(qd)
    lse = torch.empty((wr.B, wr.Hq, wr.Nq), dtype=torch.float32, device="cuda")
    ws = torch.empty(lib_mod.q8_workspace_size(wr.B, wr.Hq, wr.Hkv, wr.Nq, wr.Nkv, wr.d),
                     dtype=torch.uint8, device="cuda")

    def full():
        lib_mod.attn_fwd_q8(qd, kd, vd, causal=w.causal, workspace=ws, out=o, lse=lse,
                            qk_format=qk_format)

    def pre():
        lib_mod.q8_prepass(qd, kd, vd, ws, qk_format=qk_format)

    _barrier(world)
    t_full = time_device(full, steps, max(warmup, 3))
    t_pre = time_device(pre, steps, 3)
    _barrier(world)
    st, where = lib_mod.get_status()
    if st != 0:
        raise RuntimeError(f"device status {st} at {where:#x}")
    full_ms = _max_over_ranks(statistics.mean(t_full), world)
    pre_ms = _max_over_ranks(statistics.mean(t_pre), world)
    return full_ms, pre_ms


def bench_varlen(name: str, steps: int, warmup: int, world: int, lib_mod):
    """Packed variable-length prefill (inputs larger than L2)."""
    import torch
    w = VARLEN_WORKLOADS[name]
    q, k, v, cu = make_varlen(w)
    qd, kd, vd, cud = q.cuda(), k.cuda(), v.cuda(), cu.cuda()
    o = torch.empty_like(qd)
    lse = torch.empty((w.Hq, q.shape[0]), dtype=torch.float32, device="cuda")
    max_len = max(w.lengths())

    def step():
        lib_mod.attn_fwd_varlen(qd, kd, vd, cud, cud, max_len, causal=w.causal, out=o, lse=lse)

    _barrier(world)
    times = time_device(step, steps, max(warmup, 3))
    _barrier(world)
    st, where = lib_mod.get_status()
    if st != 0:
        raise RuntimeError(f"device status {st} at {where:#x}")
    ms = _max_over_ranks(statistics.mean(times), world)
    return {"tflops": round(world * w.flops / (ms * 1e-3) / 1e12, 1), "ms_per_step": round(ms, 4),
            "sequences": w.num_seqs, "total_tokens": int(q.shape[0]),
            "lengths": f"log-uniform in [{w.min_len}, {w.max_len}], seed {w.seed}",
            "l2": "inputs_larger_than_l2"}


BWD_WORKLOADS = ["outlier_8k_causal", "outlier_8k_full", "gqa_32k_d128"]


def bench_bwd(w: Workload, steps: int, warmup: int, world: int, rank: int, lib_mod, peak: float):
    """Backward (attn_bwd: preprocess, main and dQ-conversion kernels) after
    one forward that provides O and LSE; inputs larger than L2. FLOPs counted
    as 2.5 x the forward's (five N x N x d products instead of two)."""
    import torch
    wr = rank_workload(w, rank)
    q, k, v = make_qkv(wr.B, wr.Hq, wr.Hkv, wr.Nq, wr.Nkv, wr.d, wr.seed, wr.dist)
    do = make_dout(wr.B, wr.Hq, wr.Nq, wr.d, wr.seed)
    qd, kd, vd, dod = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    o, lse = lib_mod.attn_fwd(qd, kd, vd, causal=w.causal)
    ws = torch.empty(lib_mod.bwd_workspace_size(wr.B, wr.Hq, wr.Hkv, wr.Nq, wr.Nkv, wr.d),
                     dtype=torch.uint8, device="cuda")
    dq, dk, dv = torch.empty_like(qd), torch.empty_like(kd), torch.empty_like(vd)

    def step():
        lib_mod.attn_bwd(qd, kd, vd, o, lse, dod, causal=w.causal, workspace=ws, dq=dq, dk=dk, dv=dv)

    _barrier(world)
    times = time_device(step, steps, max(warmup, 3))
    _barrier(world)
    st, where = lib_mod.get_status()
    if st != 0:
        raise RuntimeError(f"device status {st} at {where:#x}")
    ms = _max_over_ranks(statistics.mean(times), world)
    tf = world * 2.5 * w.flops / (ms * 1e-3) / 1e12
    return {"tflops": round(tf, 1), "ms_per_step": round(ms, 4),
            "frac_of_bf16_peak": round(tf / world / peak, 4),
            "flops": "2.5 x forward (five N x N x d products)", "launches_per_step": 3,
            "l2": "inputs_larger_than_l2"}


def bench_varlen_bwd(name: str, steps: int, warmup: int, world: int, lib_mod, peak: float):
    """Backward of the packed variable-length workload (after one forward)."""
    import torch
    w = VARLEN_WORKLOADS[name]
    q, k, v, cu = make_varlen(w)
    do = make_varlen_dout(w)
    qd, kd, vd, dod, cud = q.cuda(), k.cuda(), v.cuda(), do.cuda(), cu.cuda()
    max_len = max(w.lengths())
    o, lse = lib_mod.attn_fwd_varlen(qd, kd, vd, cud, cud, max_len, causal=w.causal)
    need = lib_mod.lib().attn_bwd_varlen_workspace_size(w.num_seqs, w.Hq, max_len, w.d)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    dq, dk, dv = torch.empty_like(qd), torch.empty_like(kd), torch.empty_like(vd)

    def step():
        lib_mod.attn_bwd_varlen(qd, kd, vd, o, lse, dod, cud, cud, max_len, max_len, causal=w.causal,
                                workspace=ws, dq=dq, dk=dk, dv=dv)

    _barrier(world)
    times = time_device(step, steps, max(warmup, 3))
    _barrier(world)
    st, where = lib_mod.get_status()
    if st != 0:
        raise RuntimeError(f"device status {st} at {where:#x}")
    ms = _max_over_ranks(statistics.mean(times), world)
    tf = world * 2.5 * w.flops / (ms * 1e-3) / 1e12
    return {"tflops": round(tf, 1), "ms_per_step": round(ms, 4), "frac_of_bf16_peak": round(tf / world / peak, 4),
            "flops": "2.5 x forward (five N x N x d products)", "sequences": w.num_seqs,
            "total_tokens": int(q.shape[0]), "l2": "inputs_larger_than_l2"}


def bench_e2e(w: Workload, steps: int, warmup: int, world: int, rank: int, lib_mod):
    """Same metric through the host-buffer entry point: every step copies the
    step's inputs from pinned host memory and reads O and LSE back."""
    import torch
    wr = rank_workload(w, rank)
    q, k, v = make_qkv(wr.B, wr.Hq, wr.Hkv, wr.Nq, wr.Nkv, wr.d, wr.seed, wr.dist)
    qh, kh, vh = q.pin_memory(), k.pin_memory(), v.pin_memory()
    oh = torch.empty_like(qh).pin_memory()
    lh = torch.empty((wr.B, wr.Hq, wr.Nq), dtype=torch.float32).pin_memory()
    buf = torch.empty(lib_mod.host_buffer_size(wr.B, wr.Hq, wr.Hkv, wr.Nq, wr.Nkv, wr.d),
                      dtype=torch.uint8, device="cuda")

    def step():
        lib_mod.attn_fwd_host(qh, kh, vh, causal=w.causal, dev_buf=buf, out=oh, lse=lh)

    for _ in range(max(warmup, 3)):
        step()
    torch.cuda.synchronize()
    _barrier(world)
    times = time_device(step, steps, 0)
    _barrier(world)
    total_ms = _max_over_ranks(sum(times), world)
    h2d = 2 * (q.numel() + k.numel() + v.numel())
    d2h = 2 * q.numel() + 4 * lh.numel()
    return total_ms, h2d, d2h


def cpu_baseline(w: Workload, q, k, v, budget_s: float = 12.0):
    """The fp64 oracle, as it stands, on the host cores over a bounded sample:
    whole (batch, head) pairs in order until ~budget_s of CPU work."""
    import oracle
    cores = len(os.sched_getaffinity(0))
    qb, kb, vb = bf16_bits(q), bf16_bits(k), bf16_bits(v)
    g = w.Hq // w.Hkv
    done, flops, t0 = 0, 0.0, time.perf_counter()
    per_head = w.flops / (w.B * w.Hq)
    for b in range(w.B):
        for h in range(w.Hq):
            hk = h // g
            oracle.attention_fp64(qb[b:b + 1, h:h + 1], kb[b:b + 1, hk:hk + 1], vb[b:b + 1, hk:hk + 1],
                                  w.causal, w.scale)
            done += 1
            flops += per_head
            if time.perf_counter() - t0 > budget_s:
                break
        else:
            continue
        break
    dt = time.perf_counter() - t0
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "sample": f"{done} of {w.B * w.Hq} (batch, head) pairs, all {w.Nq} query rows, "
                      f"fp64 numpy, {dt:.1f} s"}


def run_ours(args):
    import torch
    import exact_attention_134_b200 as attn
    world, rank, local = _dist_setup()
    peaks = _peaks()
    w = WORKLOADS[args.workload]
    clocks = clock_sampler(local)
    attn.lib()
    # warm the kernel and sample clocks only over the timed region
    res = None
    clocks.start()
    res = bench_workload(w, args.steps, args.warmup, world, rank, attn, qk_format=args.qk_format)
    clk = clocks.stop()
    ms = res["total_ms"] / args.steps
    value = aggregate_tflops(w.flops, world, ms)
    per_launch_tflops = w.flops / (statistics.mean(res["times"]) * 1e-3) / 1e12
    e2e = None
    if not args.kernel_only and w.path == "bf16":
        e2e_steps = max(2, args.steps // 2)
        e2e_ms, h2d, d2h = bench_e2e(w, e2e_steps, 1, world, rank, attn)
        e2e = {"value": round(world * w.flops / (e2e_ms / e2e_steps * 1e-3) / 1e12, 2),
               "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}
    extras = {}
    if not args.no_extra and not args.kernel_only:
        for name in EXTRA_BF16:
            if name == args.workload:
                continue
            wx = WORKLOADS[name]
            r = bench_workload(wx, max(3, args.steps // 2), 3, world, rank, attn,
                               graph=name in GRAPH_TIMED)
            msx = r["total_ms"] / max(3, args.steps // 2)
            tf = world * wx.flops / (msx * 1e-3) / 1e12
            gbs = world * wx.min_hbm_bytes / (msx * 1e-3) / 1e9
            extras[name] = {"tflops": round(tf, 1), "ms_per_step": round(msx, 4),
                            "us_per_step": round(msx * 1e3, 2),
                            "frac_of_bf16_peak": round(tf / world / peaks["bf16"], 4),
                            "hbm_gbs_algorithmic": round(gbs, 1),
                            "frac_of_hbm_peak": round(gbs / world / peaks["hbm"], 4),
                            "l2": r["l2"]}
            if "graph_total_ms" in r:
                msg = r["graph_total_ms"] / max(3, args.steps // 2)
                extras[name]["graph_replay"] = {
                    "us_per_step": round(msg * 1e3, 2),
                    "tflops": round(world * wx.flops / (msg * 1e-3) / 1e12, 1)}
            elif "graph_error" in r:
                extras[name]["graph_replay"] = {"error": r["graph_error"]}
            del r
            torch.cuda.empty_cache()
        extras["varlen_prefill_mixed"] = bench_varlen("varlen_prefill_mixed", max(3, args.steps // 2),
                                                      3, world, attn)
        torch.cuda.empty_cache()
        for name in BWD_WORKLOADS:
            extras["backward_" + name] = bench_bwd(WORKLOADS[name], max(3, args.steps // 2), 3, world,
                                                   rank, attn, peaks["bf16"])
            torch.cuda.empty_cache()
        extras["backward_varlen_prefill_mixed"] = bench_varlen_bwd("varlen_prefill_mixed",
                                                                   max(3, args.steps // 2), 3, world,
                                                                   attn, peaks["bf16"])
        torch.cuda.empty_cache()
        wq = WORKLOADS["q8_8k_outlier"]
        fp8_peak = 2.0 * peaks["bf16"]
        # the same workload through both 8-bit variants: INT8 Q K^T after K
        # smoothing, and FP8 e4m3 Q K^T with block scales (no smoothing)
        for line, fmt in (("q8_8k_outlier", "int8"), ("fp8qk_8k_outlier", "fp8")):
            full_ms, pre_ms = bench_q8(wq, max(3, args.steps // 2), 3, world, rank, attn, qk_format=fmt)
            extras[line] = {
                "qk_format": fmt,
                "tflops": round(world * wq.flops / (full_ms * 1e-3) / 1e12, 1),
                "ms_per_step": round(full_ms, 4), "prepass_ms": round(pre_ms, 4),
                "main_ms": round(full_ms - pre_ms, 4),
                "main_tflops": round(world * wq.flops / ((full_ms - pre_ms) * 1e-3) / 1e12, 1),
                "frac_of_fp8_peak_main": round(wq.flops / ((full_ms - pre_ms) * 1e-3) / 1e12 / fp8_peak, 4),
                "fp8_peak": f"{fp8_peak:.0f} TFLOP/s = 2 x measured bf16 (nominal fp8/bf16 ratio)",
                "l2": "inputs_larger_than_l2"}
            torch.cuda.empty_cache()
    out = None
    if rank == 0:
        cpu = None
        if world == 1 and not args.kernel_only:
            cpu = cpu_baseline(w, *res["inputs"], budget_s=args.cpu_budget)
        traffic = _traffic_from_profile(args.workload)
        out = {
            "metric": METRIC,
            "value": round(value, 2),
            "unit": "TFLOP/s",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": max(args.warmup, 3),
            "ms_per_step": round(ms, 4),
            "ms_min": round(min(res["times"]), 4),
            "ms_median": round(statistics.median(res["times"]), 4),
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "bf16" if w.path != "q8" else
                     f"{'int8' if args.qk_format == 'int8' else 'e4m3'} QK^T + e4m3 PV (fp32 accumulation)",
            "data": "synthetic (seeded torch CPU randn -> bf16; outlier-K offsets per head/channel)",
            "config": ({**workload_config(w, res["l2"]), "qk_format": args.qk_format} if w.path == "q8"
                       else workload_config(w, res["l2"])),
            "frac_of_bf16_peak": round(value / world / peaks["bf16"], 4),
            "roofline": {"bound": "tensor", "achieved": round(per_launch_tflops, 2),
                         "peak": peaks["bf16"] * (2 if w.path == "q8" else 1), "unit": "TFLOP/s",
                         "frac": round(per_launch_tflops / (peaks["bf16"] * (2 if w.path == "q8" else 1)), 4),
                         "traffic": traffic,
                         "peak_source": (f"{peaks['source']} bf16 burst (cuBLAS)" if w.path != "q8" else
                                         f"2 x {peaks['source']} bf16 burst (nominal fp8/bf16 ratio)"),
                         "kernel": "attn_fwd_bf16_kernel" if w.path != "q8" else
                                   "attn_fwd_q8 (3 prepass kernels + main kernel)",
                         "algorithmic_min_bytes": w.min_hbm_bytes},
            "e2e": e2e,
            # per call: 1 kernel; the 8-bit path 3 prepass kernels + main; split keys partial + merge
            "gpu_launches": args.steps * (4 if w.path == "q8" else
                                          (2 if w.path == "splitkv" and attn.splitkv_num_splits(
                                              w.B, w.Hq, w.Hkv, w.Nq, w.Nkv, w.d) > 1 else 1)),
            "clocks": clk,
            "cpu_baseline": cpu,
            "other_workloads": extras,
        }
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if out is not None:
        print(json.dumps(out), flush=True)


def kv_shard_inputs(w: Workload, world: int, rank: int):
    """This rank's inputs for the key-sharded run: every query row and the
    contiguous key range kv_shard.shard_bounds gives it (CPU bf16 tensors),
    plus the full key count."""
    from exact_attention_134_b200.kv_shard import shard_bounds
    q, k, v = make_qkv(w.B, w.Hq, w.Hkv, w.Nq, w.Nkv, w.d, w.seed, w.dist)
    lo, hi = shard_bounds(w.Nkv, world, rank)
    return q, k[:, :, lo:hi].contiguous(), v[:, :, lo:hi].contiguous(), w.Nkv


def run_kv_shard(args):
    """Key-sharded forward of one long-context workload over the ranks (strong
    scaling: the total work is fixed). Each step runs attn_fwd_partial on the
    rank's key range (split over CTAs and merged on the device when the range's
    grid alone would leave SMs idle), one NCCL all-gather of the packed fp32
    partials and the merge (kv_shard.attention_kv_sharded); time = max over
    ranks of the CUDA-event time. One JSON line from rank 0."""
    import datetime
    import torch
    import torch.distributed as dist
    import exact_attention_134_b200 as attn
    from exact_attention_134_b200.kv_shard import attention_kv_sharded
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    else:  # one rank: a process group of one, so that the same code path runs
        dist.init_process_group("nccl", store=dist.HashStore(), world_size=1, rank=0)
    peaks = _peaks()
    w = WORKLOADS[args.workload]
    attn.lib()
    q, ks, vs, n_keys = kv_shard_inputs(w, world, rank)
    qd, kd, vd = q.cuda(), ks.cuda(), vs.cuda()

    def step():
        return attention_kv_sharded(qd, kd, vd, n_keys, causal=w.causal)

    clocks = clock_sampler(local)
    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    times = time_device(step, args.steps, 0)
    clk = clocks.stop()
    torch.cuda.synchronize()
    dist.barrier()
    st, where = attn.get_status()
    err = 1.0 if st != 0 else 0.0
    t = torch.tensor([sum(times), err], dtype=torch.float64, device="cuda")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    total_ms, any_err = float(t[0]), float(t[1])
    ms = total_ms / args.steps
    value = w.flops / (ms * 1e-3) / 1e12
    exchange = world * attn.partial_packed_floats(w.B, w.Hq, w.Nq, w.d) * 4  # fp32 O and LSE, packed
    # partial (+ the range's own merge when it is split) + the final merge
    local_splits = attn.splitkv_num_splits(w.B, w.Hq, w.Hkv, w.Nq, ks.shape[2], w.d)
    launches_per_step = 3 if local_splits > 1 else 2
    if rank == 0:
        out = {"metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world,
               "steps": args.steps, "warmup": max(args.warmup, 3), "ms_per_step": round(ms, 4),
               "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
               "data": "synthetic (seeded torch CPU randn -> bf16)",
               "config": {**workload_config(w, "inputs_larger_than_l2"),
                          "per_rank": "contiguous key range (kv_shard.shard_bounds), all query rows",
                          "shard": "kv"},
               "frac_of_bf16_peak": round(value / world / peaks["bf16"], 4),
               "exchange_bytes_per_rank": exchange,
               "collectives_per_step": "1 NCCL all-gather (fp32 O and LSE partials, packed)",
               "local_key_ranges": local_splits,
               "gpu_launches": launches_per_step * args.steps,
               "clocks": clk, "device_status_error": bool(any_err)}
        print(json.dumps(out), flush=True)
    dist.barrier()
    dist.destroy_process_group()


def run_bwd_only(args):
    """Only the backward of one workload (for timing and profiling it alone):
    one JSON line with its device-timed TFLOP/s."""
    import exact_attention_134_b200 as attn
    world, rank, _ = _dist_setup()
    peaks = _peaks()
    w = WORKLOADS[args.workload]
    attn.lib()
    r = bench_bwd(w, args.steps, args.warmup, world, rank, attn, peaks["bf16"])
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps({"metric": "attention backward throughput (dQ, dK, dV)", "value": r["tflops"],
                          "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
                          "warmup": max(args.warmup, 3), "ms_per_step": r["ms_per_step"],
                          "higher_is_better": True, "scaling": "weak", "dtype": "bf16",
                          "data": "synthetic", "config": {"workload": w.name, "direction": "bwd",
                                                          "l2": r["l2"], "flops": r["flops"]},
                          "frac_of_bf16_peak": r["frac_of_bf16_peak"]}), flush=True)


def run_reference(args):
    """The oracle, as it stands, on the host cores: each step is a bounded
    sample of the workload (whole (batch, head) pairs, all query rows), timed
    by wall clock; `ms_per_step` is that measured time and `value` the sample's
    FLOPs over it. Under torchrun only rank 0 runs."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    w = WORKLOADS[args.workload]
    q, k, v = make_qkv(w.B, w.Hq, w.Hkv, w.Nq, w.Nkv, w.d, w.seed, w.dist)
    # per step about 120 s / (steps + warmup) of CPU work, 1..8 s
    budget = max(1.0, min(8.0, 120.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        cpu_baseline(w, q, k, v, budget_s=budget)
    vals, secs, samples = [], [], []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        r = cpu_baseline(w, q, k, v, budget_s=budget)
        secs.append(time.perf_counter() - t0)
        vals.append(r["value"])
        samples.append(r["sample"])
    value = statistics.mean(vals)
    ms = statistics.mean(secs) * 1e3
    sample = (f"each step: whole (batch, head) pairs of the workload in order, all {w.Nq} query rows, "
              f"until {budget:.1f} s of CPU work; last step: {samples[-1]}")
    out = {"impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s",
           "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 3),
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
           "data": "synthetic (seeded torch CPU randn -> bf16; outlier-K offsets per head/channel)",
           "config": workload_config(w, l2_mode_of(w)),
           "sample": sample,
           "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s",
                            "cores": len(os.sched_getaffinity(0)), "kind": "oracle", "sample": sample},
           "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=HEADLINE, choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-extra", action="store_true", help="skip the other bf16 workloads")
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    ap.add_argument("--kernel-only", action="store_true",
                    help="only the device-timed leg (for profiling runs): no e2e, CPU or extra legs")
    ap.add_argument("--direction", default="fwd", choices=["fwd", "bwd"],
                    help="bwd: time only the backward of --workload (one JSON line)")
    ap.add_argument("--qk-format", default="int8", choices=["int8", "fp8"],
                    help="8-bit workloads: INT8 Q K^T after K smoothing, or FP8 e4m3 Q K^T with block scales")
    ap.add_argument("--shard", default="batch", choices=["batch", "kv"],
                    help="kv: split the keys of --workload over the ranks (key-sharded forward, "
                         "partial -> NCCL all-gather -> merge; default workload kvcache_128k_q128)")
    args = ap.parse_args()
    if args.shard == "kv" and args.workload == HEADLINE:
        args.workload = "kvcache_128k_q128"
    if args.impl == "reference":
        run_reference(args)
    elif args.shard == "kv":
        run_kv_shard(args)
    elif args.direction == "bwd":
        run_bwd_only(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()

"""Benchmark of the DAMP-style decode step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]

A step is one decode step (dequantize, gated delta rule, readout,
requantize in place) over every (slot, head) of the workload, i.e. one
launch of the decode kernel.  The default workload is the 512-slot x 48-head
GDN batch at d = 128 with 27 FP16 rows per head (9.885 bits/value, bf16 q/k/v):
the batch >= 256, d = 128 point the throughput target is stated for.  Lines
for the 256-slot x 32-head GDN batch and the 128-slot x 32-head KDA batch are
printed beside it (`sub_lines`, same keys).  Consecutive steps rotate over
enough pools and input sets to touch at least 4x L2 (every step reads cold
state and pays for earlier write-backs); each step is timed with CUDA events
on the launching stream and the durations are summed.

Printed: one JSON line (rank 0).  `value` is head-steps/s over all ranks;
`roofline` is the decode kernel's algorithmic bytes per launch over its mean
event-timed duration against the measured HBM copy peak; `e2e` times the same
steps through the public API from pinned host buffers (inputs H2D, out D2H);
`cpu_baseline` times the oracle on a bounded sample of units on one host
core.  Multi-GPU: one process per GPU, each rank steps its own pool (slots
sharded across ranks, no collective on the data path), time = max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "head-steps/s and achieved HBM GB/s (% of B200 roofline) per decode step"
FALLBACK_HBM_GBS = 6650.0
KERNEL_SOURCES = ["damp_decode_unit.cu", "damp_device.cuh", "damp_internal.h"]   # the profiled kernel
PROFILE_DIR = os.path.join(ROOT, "profiles")


# ---------------------------------------------------------------- accounting

def unit_bytes(w: W.Workload, fmt: str) -> int:
    """Algorithmic bytes of one (slot, head) step: state read + write, q, k, v,
    alpha, beta, out (block padding excluded)."""
    import quantized_linear_attention_damp_b200 as D
    block, _ = D.damp_layout(D.FORMATS[fmt], w.d, w.d, w.hp if fmt == "mixed" else 0)
    elt = 2 if w.in_dtype == "bf16" else 4
    alpha = 4 * w.d if w.gate == W.GATE_KDA else 4
    return 2 * block + 3 * w.d * elt + alpha + 4 + 4 * w.d


def describe(w: W.Workload, fmt: str) -> str:
    return (f"{w.name}: {w.n} slots x {w.H} heads, d_k=d_v={w.d}, {fmt} state"
            + (f" ({w.hp} FP16 rows/head)" if fmt == "mixed" else "")
            + f", {w.gate.upper()}, {w.in_dtype} q/k/v")


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "quantized_linear_attention_damp_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def profiled_traffic(w: W.Workload, fmt: str, units: int):
    """DRAM bytes per launch from the committed ncu summary of this workload
    and format (profiles/decode_unit_<workload>_<fmt>.txt), scaled to this
    launch's units; None if absent or taken on different kernel sources."""
    try:
        kv = {}
        for line in open(os.path.join(PROFILE_DIR, f"decode_unit_{w.name}_{fmt}.txt")):
            if ":" in line:
                k, v = line.split(":", 1)
                kv[k.strip()] = v.strip()
        if kv.get("kernel_source_sha256_16") != kernel_source_hash():
            return None
        per_unit = float(kv["dram_bytes_per_unit"])
        return int(per_unit * units)
    except Exception:
        return None


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML in a thread."""

    REASONS = {  # NVML clocks-event reason bits
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
        0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
        0x100: "display_clock_setting",
    }

    def __init__(self, device_index: int, period_s: float = 0.002):
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self._stop = threading.Event()
        self.period = period_s
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

    def _sample(self):
        nv = self.nv
        self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
        try:
            bits = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        except Exception:
            bits = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
        for b, name in self.REASONS.items():
            if bits & b and name != "gpu_idle":
                self.reasons.add(name)

    def _run(self):
        while not self._stop.is_set():
            self._sample()
            time.sleep(self.period)

    def __enter__(self):
        if self.nv:
            self._sample()
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.nv:
            self._stop.set()
            self.t.join()
            self._sample()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["nvml unavailable"]}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ---------------------------------------------------------------- ranks

def rank_workload(name: str, rank: int) -> W.Workload:
    """The workload a rank steps: the same shape on every rank, its own slots
    (a data-parallel shard of a larger serving pool: independent seed)."""
    return W.WORKLOADS[name].with_(seed=rank)


def max_over_ranks(seconds: float, world: int, device=None) -> float:
    """Device time of a step sequence as the max over ranks (every rank calls)."""
    if world <= 1:
        return seconds
    import torch
    import torch.distributed as dist
    t = torch.tensor([seconds], dtype=torch.float64,
                     device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------- native arm

class Bench:
    """One workload on one GPU.

    L2 handling: the steps rotate over enough pools (and input sets) that the
    data a step touches is at least 4x the L2 size, so every timed step reads
    its state from HBM and pays for the write-back of earlier steps, as a
    serving pool much larger than L2 does.  No step is flushed or skipped.
    """

    def __init__(self, w: W.Workload, fmt: str, device, n_inputs: int | None = None,
                 fp16_map=None):
        import torch

        import quantized_linear_attention_damp_b200 as D
        self.torch, self.D = torch, D
        self.w, self.fmt, self.dev = w, fmt, device
        self.hs = W.head_structure(w.with_(fmt=fmt))
        hp = self.hs.hp_row_idx if fmt == "mixed" else None
        l2 = torch.cuda.get_device_properties(device).L2_cache_size
        if fp16_map is not None:
            state_bytes = D.damp_pool_bytes_map(w.n_slots, w.H, w.d, w.d, fp16_map)
        else:
            _, stride = D.damp_layout(D.FORMATS[fmt], w.d, w.d, w.hp if fmt == "mixed" else 0)
            state_bytes = w.n_slots * w.H * stride
        self.n_pools = max(1, -(-4 * l2 // state_bytes))
        S0 = torch.from_numpy(W.initial_state(w, range(w.n_slots))).to(device)
        ident = torch.arange(w.n_slots, dtype=torch.int32, device=device)
        self.pools = []
        for _ in range(self.n_pools):
            p = D.DampPool(fmt, w.n_slots, w.H, w.d, hp, device=device, fp16_map=fp16_map)
            p.pack(ident, S0)
            self.pools.append(p)
        del S0
        x0 = self._host_inputs(W.step_inputs(w, 0, self.hs))
        in_bytes = sum(v.numel() * v.element_size() for v in x0.values())
        if n_inputs is None:
            n_inputs = max(4, -(-2 * l2 // in_bytes))
        self.host = [x0] + [self._host_inputs(W.step_inputs(w, s, self.hs))
                            for s in range(1, n_inputs)]
        self.dev_in = [{k: v.to(device) for k, v in h.items()} for h in self.host]
        self.out = torch.empty((w.n, w.H, w.d), dtype=torch.float32, device=device)
        self.touched_bytes = self.n_pools * state_bytes
        torch.cuda.synchronize(device)

    def _host_inputs(self, x):
        torch = self.torch
        if self.w.in_dtype == "bf16":
            cv = lambda b: torch.from_numpy(b.view(np.int16)).view(torch.bfloat16)
            q, k, v = cv(x.q_bits), cv(x.k_bits), cv(x.v_bits)
        else:
            q, k, v = (torch.from_numpy(a) for a in (x.q, x.k, x.v))
        d = dict(slot_idx=torch.from_numpy(x.slot_idx), q=q, k=k, v=v,
                 alpha=torch.from_numpy(x.alpha), beta=torch.from_numpy(x.beta))
        return {k: t.contiguous().pin_memory() for k, t in d.items()}

    def step(self, i: int):
        a = self.dev_in[i % len(self.dev_in)]
        self.pools[i % self.n_pools].step(a["slot_idx"], a["q"], a["k"], a["v"], a["alpha"],
                                          a["beta"], self.out)

    def timed(self, steps: int, warmup: int, sampler=None) -> float:
        """Seconds of device time over `steps` consecutive steps: one event pair
        around all of them, so consecutive launches overlap as they do in use
        (programmatic dependent launch).  A second pass with events around each
        step gives the per-step distribution (`step_ms`)."""
        torch = self.torch
        for i in range(warmup):
            self.step(i)
        torch.cuda.synchronize(self.dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(steps)]
        ctx = sampler if sampler is not None else _Null()
        with ctx:
            # keep the device busy while the host enqueues the timed steps, so
            # that the events time the kernels and not the host's launch rate
            torch.cuda._sleep(min(steps, 4000) * 200_000)
            e0.record()
            for i in range(steps):
                self.step(warmup + i)
            e1.record()
            torch.cuda.synchronize(self.dev)
            torch.cuda._sleep(min(steps, 4000) * 200_000)
            for i in range(steps):
                ev[i][0].record()
                self.step(warmup + steps + i)
                ev[i][1].record()
            torch.cuda.synchronize(self.dev)
        self.step_ms = sorted(a.elapsed_time(b) for a, b in ev)
        return e0.elapsed_time(e1) / 1e3

    def timed_e2e(self, steps: int) -> tuple[float, int, int]:
        """Same steps through the public API from pinned host memory: each step
        copies its inputs H2D, runs, and copies `out` D2H (device-timed, one
        event pair around all steps).  As a serving loop would, the copies run
        on their own streams, double-buffered, so that step i's kernel overlaps
        the input copy of step i+1 and the output copy of step i-1."""
        torch = self.torch
        dev_in = [{k: torch.empty_like(v, device=self.dev) for k, v in self.host[0].items()}
                  for _ in range(2)]
        outs = [torch.empty_like(self.out) for _ in range(2)]
        out_host = [torch.empty(self.out.shape, dtype=torch.float32).pin_memory() for _ in range(2)]
        h2d = sum(v.numel() * v.element_size() for v in self.host[0].values())
        d2h = out_host[0].numel() * 4
        comp = torch.cuda.current_stream(self.dev)
        s_in, s_out = torch.cuda.Stream(self.dev), torch.cuda.Stream(self.dev)
        ev = lambda: torch.cuda.Event()
        copied = [ev() for _ in range(steps)]    # inputs of step i on the device
        ran = [ev() for _ in range(steps)]       # kernel of step i done
        read = [ev() for _ in range(steps)]      # out of step i on the host
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(self.dev)
        e0.record(comp)
        s_in.wait_event(e0)
        s_out.wait_event(e0)
        for i in range(steps):
            src, buf, o = self.host[i % len(self.host)], dev_in[i % 2], outs[i % 2]
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(ran[i - 2])          # buffer free again
                for k_, v_ in src.items():
                    buf[k_].copy_(v_, non_blocking=True)
                copied[i].record(s_in)
            comp.wait_event(copied[i])
            if i >= 2:
                comp.wait_event(read[i - 2])             # out buffer read back
            self.pools[i % self.n_pools].step(buf["slot_idx"], buf["q"], buf["k"], buf["v"],
                                              buf["alpha"], buf["beta"], o, stream=comp)
            ran[i].record(comp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ran[i])
                out_host[i % 2].copy_(o, non_blocking=True)
                read[i].record(s_out)
        comp.wait_stream(s_in)
        comp.wait_stream(s_out)
        e1.record(comp)
        torch.cuda.synchronize(self.dev)
        return e0.elapsed_time(e1) / 1e3, h2d, d2h

    def close(self):
        for p in self.pools:
            p.close()


class _Null:
    def __enter__(self):
        return self

    def __exit__(self, *a):
        pass


def cpu_baseline(w: W.Workload, fmt: str, seconds: float, max_units: int = 10 ** 9):
    """Oracle head-steps/s on one host core over a bounded sample of units."""
    import oracle as O
    hs = W.head_structure(w.with_(fmt=fmt))
    ofmt = {"fp32": O.FMT_FP32, "fp8": O.FMT_FP8}.get(fmt, O.FMT_QUANT)
    x = W.step_inputs(w, 0, hs)
    slots = list(x.slot_idx[: min(w.n, 8)])
    S0 = W.initial_state(w, slots)
    st = O.pack(ofmt, hs.is_fp16[None], S0)
    gate = O.GATE_VECTOR if w.gate == W.GATE_KDA else O.GATE_SCALAR
    done, t0 = 0, time.perf_counter()
    while done < max_units:
        b, h = (done // w.H) % len(slots), done % w.H
        O.step_unit(st[b, h], gate, hs.is_fp16[h], x.q[b, h], x.k[b, h], x.v[b, h],
                    x.alpha[b, h], x.beta[b, h])
        done += 1
        if time.perf_counter() - t0 >= seconds:
            break
    el = time.perf_counter() - t0
    return done / el, done, el


def cpu_baseline_threads(w: W.Workload, fmt: str, seconds: float, threads: int):
    """Oracle head-steps/s with `threads` host threads, each stepping its own
    units (the same bounded sample per thread as cpu_baseline)."""
    from concurrent.futures import ThreadPoolExecutor
    with ThreadPoolExecutor(threads) as ex:
        res = list(ex.map(lambda _: cpu_baseline(w, fmt, seconds), range(threads)))
    n = sum(r[1] for r in res)
    el = max(r[2] for r in res)
    return n / el, n, el


def config_of(w: W.Workload, fmt: str, world: int, l2: str, timing: str) -> dict:
    """The workload description shared by both arms (same keys)."""
    return {"workload": describe(w, fmt), "units_per_step_per_gpu": w.n * w.H,
            "algorithmic_bytes_per_unit": unit_bytes(w, fmt), "l2": l2, "timing": timing,
            "parallelism": f"dp{world} (slots sharded, no collective)"}


def measure(w: W.Workload, fmt: str, dev, steps: int, warmup: int, world: int = 1,
            local_rank: int = 0, cpu_seconds: float = 0.0, e2e: bool = True) -> dict:
    """One workload's line: device-timed steps (max over ranks), roofline of
    the decode kernel, clocks during the timed region, the same steps end to
    end through the public API, and the oracle on the host cores."""
    import torch
    import torch.distributed as dist
    b = Bench(w, fmt, device=dev)
    units = w.n * w.H
    ub = unit_bytes(w, fmt)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    sampler = ClockSampler(local_rank)
    secs = max_over_ranks(b.timed(steps, warmup, sampler), world, dev)
    if world > 1:
        dist.barrier()
    e2e_secs, h2d, d2h = b.timed_e2e(steps) if e2e else (float("nan"), 0, 0)
    e2e_secs = max_over_ranks(e2e_secs, world, dev)
    b.close()
    per_launch = secs / steps
    gbs = ub * units / per_launch / 1e9
    peak, src = measured_peak()
    line = {
        "value": units * world * steps / secs, "unit": "head-steps/s",
        "ms_per_step": per_launch * 1e3,
        "config": config_of(w, fmt, world,
                            l2=f"steps rotate over {b.n_pools} pools "
                               f"({b.touched_bytes / 1e6:.0f} MB) and their inputs, >= 4x L2: "
                               "inputs larger than L2",
                            timing="one CUDA event pair around the K consecutive steps on the "
                                   "launch stream (launches overlap by programmatic dependent "
                                   "launch); step_us: a second pass with events around each step"),
        "hbm_gbs": gbs,
        "roofline": {"bound": "hbm", "achieved": gbs, "peak": peak, "unit": "GB/s",
                     "frac": gbs / peak, "peak_source": src,
                     "frac_of_8tbs_nominal": gbs / 8000.0,
                     "traffic": profiled_traffic(w, fmt, units)},
        "step_us": {"median": b.step_ms[len(b.step_ms) // 2] * 1e3, "min": b.step_ms[0] * 1e3,
                    "mean": sum(b.step_ms) / len(b.step_ms) * 1e3},
        "gpu_launches": steps,
        "clocks": sampler.summary(),
        "e2e": ({"value": units * world * steps / e2e_secs, "unit": "head-steps/s",
                 "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h} if e2e else None),
    }
    if world == 1 and cpu_seconds > 0:
        v, n, el = cpu_baseline(w, fmt, cpu_seconds)
        line["cpu_baseline"] = {"value": v, "unit": "head-steps/s", "cores": 1, "kind": "oracle",
                                "sample": f"{n} (slot, head) units of {w.name} ({fmt}), "
                                          f"one step each, single thread, {el:.1f} s"}
    return line


# sub-lines printed beside the headline: the other d = 128 target points
SUB_LINES = [("gdn_256x32", "mixed"), ("kda", "mixed")]


def run_native(args, rank, world, local_rank):
    import torch
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = rank_workload(args.workload, rank)
    fmt = args.fmt
    head = measure(w, fmt, dev, args.steps, args.warmup, world, local_rank,
                   args.cpu_seconds if world == 1 else 0.0, e2e=not args.no_e2e)
    subs = []
    if not args.no_sub_lines:
        for name, sfmt in SUB_LINES:
            if name == args.workload and sfmt == fmt:
                continue
            sl = measure(rank_workload(name, rank), sfmt, dev, args.steps, args.warmup, world,
                         local_rank, min(args.cpu_seconds, 3.0) if world == 1 else 0.0,
                         e2e=not args.no_e2e)
            sl["metric"] = METRIC
            subs.append(sl)
    if rank != 0:
        return
    line = {"metric": METRIC, "value": head["value"], "unit": "head-steps/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": head["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic"}
    line.update({k: v for k, v in head.items() if k not in ("value", "unit", "ms_per_step")})
    if world == 1 and args.cpu_seconds > 0:
        t = os.cpu_count() or 1
        v, n, el = cpu_baseline_threads(w, fmt, args.cpu_seconds, t)
        line["cpu_baseline_all_cores"] = {
            "value": v, "unit": "head-steps/s", "cores": t, "kind": "oracle",
            "sample": f"{n} (slot, head) units of {w.name} ({fmt}), one step each, "
                      f"{t} threads over units (the oracle's C calls release the GIL), {el:.1f} s"}
    if subs:
        line["sub_lines"] = subs
    if world == 1 and not args.no_variants:
        line["variants"] = variants(args, dev)
    if world == 1 and not args.no_variants:
        line["state_error_vs_fp32"] = quality(dev)
    if world == 1 and not args.no_serving:
        line["serving_pool"] = serving(args, dev)
    print(json.dumps(line), flush=True)


def variants(args, dev):
    """Context: the same kernel on the other workloads and state formats."""
    res = []
    steps = max(20, min(args.steps, 200))
    for name, fmt in [("hiconc_gdn", "int8"), ("hiconc_gdn", "fp8"), ("hiconc_gdn", "fp32"),
                      ("gdn_batch", "mixed"), ("gdn_batch", "int8"), ("gdn_batch", "fp32"),
                      ("d64_gdn", "mixed"), ("d256_gdn", "mixed")]:
        w = W.WORKLOADS[name]
        b = Bench(w, fmt, device=dev)
        secs = b.timed(steps, 3)
        each = sum(b.step_ms) / len(b.step_ms) * 1e3
        b.close()
        units = w.n * w.H
        ub = unit_bytes(w, fmt)
        gbs = ub * units * steps / secs / 1e9
        peak, _ = measured_peak()
        res.append({"workload": describe(w, fmt), "head_steps_per_s": units * steps / secs,
                    "us_per_step": secs / steps * 1e6, "us_per_step_timed_alone": each,
                    "hbm_gbs": gbs, "frac": gbs / peak, "bytes_per_unit": ub})
    # pack / unpack at pool scale (prefill hand-off and restore): 512 x 48 units
    import torch

    import quantized_linear_attention_damp_b200 as D
    w = W.WORKLOADS["hiconc_gdn"]
    b = Bench(w, "mixed", device=dev, n_inputs=1)
    units = w.n_slots * w.H
    S = torch.empty((w.n_slots, w.H, w.d, w.d), dtype=torch.float32, device=dev)
    ident = torch.arange(w.n_slots, dtype=torch.int32, device=dev)
    for name_, fn in (("unpack", lambda p: p.unpack(ident, S)), ("pack", lambda p: p.pack(ident, S))):
        for i in range(3):
            fn(b.pools[i % b.n_pools])
        torch.cuda.synchronize(dev)
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(10)]
        for i in range(10):
            ev[i][0].record()
            fn(b.pools[i % b.n_pools])
            ev[i][1].record()
        torch.cuda.synchronize(dev)
        secs = sum(a_.elapsed_time(b_) for a_, b_ in ev) / 1e3
        # FP32 state (d*d*4) one way, the block's algorithmic bytes the other
        ub = 4 * w.d * w.d + D.damp_layout(D.DAMP_FMT_MIXED, w.d, w.d, w.hp)[0]
        gbs = ub * units * 10 / secs / 1e9
        res.append({"workload": f"{name_}: {w.n_slots} slots x {w.H} heads, d={w.d}, mixed "
                                f"({w.hp} FP16 rows/head) <-> FP32 states",
                    "head_steps_per_s": units * 10 / secs, "us_per_step": secs / 10 * 1e6,
                    "hbm_gbs": gbs, "frac": gbs / measured_peak()[0], "bytes_per_unit": ub})
    b.close()
    del S
    # calibrated FP16 rows under one budget for all heads (counts differ per head)
    w = W.WORKLOADS["gdn_256x32"]
    acc = calibrate(w, dev)
    is16, hp, _ = D.damp_calib_select_budget(w.H, w.d, w.hp * w.H, acc)
    fmap = is16.cpu().numpy()
    b = Bench(w, "mixed", device=dev, fp16_map=fmap)
    secs = b.timed(steps, 3)
    blk = [b.pools[0].heads[h][0] for h in range(w.H)]
    b.close()
    elt = 2 if w.in_dtype == "bf16" else 4
    ub = 2 * float(np.mean(blk)) + 3 * w.d * elt + 4 + 4 + 4 * w.d
    units = w.n * w.H
    gbs = ub * units * steps / secs / 1e9
    res.append({"workload": describe(w, "mixed").replace(
                    f"({w.hp} FP16 rows/head)",
                    f"(calibrated, {w.hp * w.H} FP16 rows over {w.H} heads, "
                    f"{int(hp.min())}..{int(hp.max())} per head)"),
                "head_steps_per_s": units * steps / secs, "us_per_step": secs / steps * 1e6,
                "hbm_gbs": gbs, "frac": gbs / measured_peak()[0], "bytes_per_unit": ub})
    return res


def calibrate(w: W.Workload, dev, steps: int = 8):
    """GPU calibration of the FP16-row choice on workload ``w``: the FP32
    recurrence runs ``steps`` steps from the workload's initial state and
    every step's states are recorded (damp_calib_accumulate)."""
    import torch

    import quantized_linear_attention_damp_b200 as D
    hs = W.head_structure(w.with_(fmt="fp32"))
    p = D.DampPool("fp32", w.n_slots, w.H, w.d, device=dev)
    p.pack(torch.arange(w.n_slots, dtype=torch.int32, device=dev),
           torch.from_numpy(W.initial_state(w, range(w.n_slots))).to(dev))
    acc = D.calib_acc(w.H, w.d, device=dev)
    out = torch.empty((w.n, w.H, w.d), dtype=torch.float32, device=dev)
    for s in range(steps):
        x = W.step_inputs(w.with_(name=w.name + "_calib"), s, hs)
        cv = lambda bits: torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(dev)
        t = dict(slot_idx=torch.from_numpy(x.slot_idx).to(dev), q=cv(x.q_bits), k=cv(x.k_bits),
                 v=cv(x.v_bits), alpha=torch.from_numpy(x.alpha).to(dev),
                 beta=torch.from_numpy(x.beta).to(dev))
        p.step(t["slot_idx"], t["q"], t["k"], t["v"], t["alpha"], t["beta"], out)
        D.damp_calib_accumulate(p.handle, t["slot_idx"], t["alpha"], acc)
    p.close()
    return acc


def quality(dev, steps: int = 64):
    """Context: state error of each format after ``steps`` decode steps, as
    the relative Frobenius distance of the dequantized state from the FP32
    recurrence fed the same inputs (64 slots x 32 heads GDN and 128 x 32 KDA,
    d = 128).  Maps: the configurations' FP16 rows, and the calibrated rows
    (per head, and under one budget for all heads)."""
    import torch

    import quantized_linear_attention_damp_b200 as D
    res = {}
    for name in ("gdn_batch", "kda"):
        w = W.WORKLOADS[name]
        hs = W.head_structure(w)
        acc = calibrate(w, dev)
        cal_idx, _ = D.damp_calib_select(w.H, w.d, w.hp, acc)
        is16_b, hp_b, _ = D.damp_calib_select_budget(w.H, w.d, w.hp * w.H, acc)
        cal_map = np.zeros((w.H, w.d), np.uint8)
        np.put_along_axis(cal_map, cal_idx.cpu().numpy().astype(np.int64), 1, axis=1)
        pools = {"fp32": D.DampPool("fp32", w.n_slots, w.H, w.d, device=dev),
                 "int8": D.DampPool("int8", w.n_slots, w.H, w.d, device=dev),
                 "fp8": D.DampPool("fp8", w.n_slots, w.H, w.d, device=dev),
                 "mixed_config_rows": D.DampPool("mixed", w.n_slots, w.H, w.d, hs.hp_row_idx,
                                                 device=dev),
                 "mixed_calibrated": D.DampPool("mixed", w.n_slots, w.H, w.d,
                                                fp16_map=cal_map, device=dev),
                 "mixed_calibrated_budget": D.DampPool("mixed", w.n_slots, w.H, w.d,
                                                       fp16_map=is16_b.cpu().numpy(), device=dev)}
        ident = torch.arange(w.n_slots, dtype=torch.int32, device=dev)
        S0 = torch.from_numpy(W.initial_state(w, range(w.n_slots))).to(dev)
        for p in pools.values():
            p.pack(ident, S0)
        out = torch.empty((w.n, w.H, w.d), dtype=torch.float32, device=dev)
        cv = lambda bits: torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(dev)
        for s in range(steps):
            x = W.step_inputs(w, s, hs)
            t = [torch.from_numpy(x.slot_idx).to(dev), cv(x.q_bits), cv(x.k_bits), cv(x.v_bits),
                 torch.from_numpy(x.alpha).to(dev), torch.from_numpy(x.beta).to(dev)]
            for p in pools.values():
                p.step(*t, out)
        ref = torch.empty((w.n_slots, w.H, w.d, w.d), dtype=torch.float32, device=dev)
        pools["fp32"].unpack(ident, ref)
        cur = torch.empty_like(ref)
        line = {"steps": steps, "fp16_rows_per_head_budget": w.hp,
                "budget_rows_per_head_min_max": [int(hp_b.min()), int(hp_b.max())]}
        for k, p in pools.items():
            if k == "fp32":
                continue
            p.unpack(ident, cur)
            line[k] = float(torch.linalg.vector_norm((cur - ref).double()) /
                            torch.linalg.vector_norm(ref.double()))
        for p in pools.values():
            p.close()
        res[name] = line
    return res


def serving(args, dev, steps: int = 16, warmup: int = 3):
    """Context: the serving-shaped pool.  36 layer pools of 4096 slots x 32
    heads (mixed format, d = 128; layers 3, 7, ... use KDA decay), one decode
    step per layer per token on the same random 1024-slot subset.  Timed as
    plain launches and as one CUDA graph replay per token.  Each layer's
    q/k/v/alpha/beta are drawn once and reused; the slot subset changes every
    step.  Needs about 97 GB of device memory; skipped (with the reason) if
    that is not free."""
    from concurrent.futures import ThreadPoolExecutor

    import torch

    import quantized_linear_attention_damp_b200 as D
    from quantized_linear_attention_damp_b200.graph import DecodeGraph
    L, nt = W.SERVING_LAYERS, W.SERVING_TEMPLATES
    ws = [W.serving_layer(l) for l in range(L)]
    pool_bytes = D.damp_pool_bytes(D.DAMP_FMT_MIXED, ws[0].n_slots, ws[0].H, ws[0].d, ws[0].d,
                                   ws[0].hp)
    free, _ = torch.cuda.mem_get_info(dev)
    if free < L * pool_bytes + (8 << 30):
        return {"skipped": f"needs {L * pool_bytes / 1e9:.1f} GB of pools, "
                           f"{free / 1e9:.1f} GB free"}

    def host(l):
        hs = W.head_structure(ws[l])
        return hs, W.serving_templates(ws[l]), W.serving_step_inputs(ws[l], 0, hs)

    with ThreadPoolExecutor(min(16, os.cpu_count() or 1)) as ex:
        gen = list(ex.map(host, range(L)))
    pools, calls = [], []
    slot_static = torch.empty(ws[0].n, dtype=torch.int32, device=dev)
    for w, (hs, T, x) in zip(ws, gen):
        p = D.DampPool("mixed", w.n_slots, w.H, w.d, hs.hp_row_idx, device=dev)
        p.pack(torch.arange(nt, dtype=torch.int32, device=dev), torch.from_numpy(T).to(dev))
        b = p.blocks()
        g = w.n_slots // nt
        b.view(g, nt, w.H, -1)[1:].copy_(b[:nt].unsqueeze(0).expand(g - 1, -1, -1, -1))
        cv = lambda bits: torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(dev)
        a = dict(slot_idx=slot_static, q=cv(x.q_bits), k=cv(x.k_bits), v=cv(x.v_bits),
                 alpha=torch.from_numpy(x.alpha).to(dev), beta=torch.from_numpy(x.beta).to(dev),
                 out=torch.empty((w.n, w.H, w.d), dtype=torch.float32, device=dev))
        pools.append(p)
        calls.append((p, a))
    del gen
    n_total = warmup + steps
    slot_tab = torch.from_numpy(np.stack([W.serving_slot_idx(s) for s in range(2 * n_total)]))
    slot_tab = slot_tab.to(dev)
    graph = DecodeGraph(calls, device=dev)
    torch.cuda.synchronize(dev)

    def run(i, use_graph):
        slot_static.copy_(slot_tab[i])
        if use_graph:
            graph.replay()
        else:
            for p, a in calls:
                p.step(a["slot_idx"], a["q"], a["k"], a["v"], a["alpha"], a["beta"], a["out"])

    res = {"workload": f"serving pool: {L} layers x {ws[0].n_slots} slots x {ws[0].H} heads, "
                       f"d_k=d_v={ws[0].d}, mixed state ({ws[0].hp} FP16 rows/head), "
                       f"{ws[0].n} random slots per step, every 4th layer KDA, bf16 q/k/v",
           "pool_bytes": L * pool_bytes}
    step_bytes = sum(unit_bytes(w, "mixed") * w.n * w.H for w in ws)
    units = sum(w.n * w.H for w in ws)
    peak, _ = measured_peak()
    for mode, use_graph in (("plain", False), ("graph", True)):
        base = 0 if mode == "plain" else n_total
        for i in range(warmup):
            run(base + i, use_graph)
        torch.cuda.synchronize(dev)
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(steps)]
        for i in range(steps):
            ev[i][0].record()
            run(base + warmup + i, use_graph)
            ev[i][1].record()
        torch.cuda.synchronize(dev)
        secs = sum(a_.elapsed_time(b_) for a_, b_ in ev) / 1e3
        gbs = step_bytes * steps / secs / 1e9
        res[mode] = {"ms_per_step": secs / steps * 1e3, "head_steps_per_s": units * steps / secs,
                     "hbm_gbs": gbs, "frac": gbs / peak, "launches_per_step": L}
    res["algorithmic_bytes_per_step"] = step_bytes
    errs = [p.get_error() for p in pools]
    res["error_flags"] = int(np.bitwise_or.reduce(errs))
    graph.reset()
    for p in pools:
        p.close()
    del calls, pools
    torch.cuda.empty_cache()
    return res


# ---------------------------------------------------------------- reference arm

def run_reference(args, rank, world):
    """The oracle (plain CPU C) timed as it stands on the host cores, on the
    same workload, metric and unit: each step is a bounded sample of units."""
    if rank != 0:
        return
    w = W.WORKLOADS[args.workload]
    fmt = args.fmt
    budget = 60.0
    t_unit = cpu_baseline(w, fmt, 0.5)[2] / max(1, cpu_baseline(w, fmt, 0.5)[1])
    per_step = int(max(1, min(w.n * w.H, budget / (args.steps + args.warmup) / t_unit)))
    for _ in range(args.warmup):
        cpu_baseline(w, fmt, 1e9, per_step)
    total_u, total_t = 0, 0.0
    for _ in range(args.steps):
        _, n, el = cpu_baseline(w, fmt, 1e9, per_step)
        total_u += n
        total_t += el
    value = total_u / total_t
    line = {
        "metric": METRIC, "value": value, "unit": "head-steps/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": total_t / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "impl": "reference",
        "config": config_of(w, fmt, world,
                            l2="host CPU run of the oracle: no GPU cache involved",
                            timing="host wall clock (time.perf_counter) around the oracle's "
                                   f"unit steps; each step a sample of {per_step} of the "
                                   f"{w.n * w.H} (slot, head) units"),
        "cpu_baseline": {"value": value, "unit": "head-steps/s", "cores": 1, "kind": "oracle",
                         "sample": f"{per_step} units per step x {args.steps} steps, "
                                   "single thread"},
        "e2e": {"value": value, "unit": "head-steps/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--workload", default="hiconc_gdn", choices=list(W.WORKLOADS))
    ap.add_argument("--fmt", default="mixed", choices=["mixed", "int8", "fp8", "fp32"])
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-variants", action="store_true")
    ap.add_argument("--no-serving", action="store_true",
                    help="skip the 36-layer serving-pool context run (about 97 GB)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-sub-lines", action="store_true",
                    help="skip the 256x32 GDN and 128x32 KDA lines printed beside the headline")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        run_native(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()

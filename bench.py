"""Benchmark of the DAMP-style decode step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]

A step is one decode step (dequantize, gated delta rule, readout,
requantize in place) over every (slot, head) of the workload, i.e. one
launch of the decode kernel.  The default workload is the 64-slot x 32-head
GDN batch at d = 128 with 27 FP16 rows per head (9.885 bits/value).  Its state
(41.5 MB) fits in L2, so consecutive steps rotate over several pools and input
sets totalling at least 4x L2 (every step reads cold state and pays for
earlier write-backs); each step is timed with CUDA events on the launching
stream and the durations are summed.

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
KERNEL_SOURCES = ["damp_decode.cu", "damp_decode_pair.cu", "damp_device.cuh", "damp_internal.h"]
PROFILE = os.path.join(ROOT, "profiles", "decode_step_hiconc_gdn_mixed.txt")


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


def profiled_traffic(units: int):
    """DRAM bytes per launch from the committed ncu summary, scaled to this
    launch's units; None if absent or taken on different kernel sources."""
    try:
        kv = {}
        for line in open(PROFILE):
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

    def __init__(self, w: W.Workload, fmt: str, device, n_inputs: int | None = None):
        import torch

        import quantized_linear_attention_damp_b200 as D
        self.torch, self.D = torch, D
        self.w, self.fmt, self.dev = w, fmt, device
        self.hs = W.head_structure(w.with_(fmt=fmt))
        hp = self.hs.hp_row_idx if fmt == "mixed" else None
        l2 = torch.cuda.get_device_properties(device).L2_cache_size
        _, stride = D.damp_layout(D.FORMATS[fmt], w.d, w.d, w.hp if fmt == "mixed" else 0)
        state_bytes = w.n_slots * w.H * stride
        self.n_pools = max(1, -(-4 * l2 // state_bytes))
        S0 = torch.from_numpy(W.initial_state(w, range(w.n_slots))).to(device)
        ident = torch.arange(w.n_slots, dtype=torch.int32, device=device)
        self.pools = []
        for _ in range(self.n_pools):
            p = D.DampPool(fmt, w.n_slots, w.H, w.d, hp, device=device)
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
        """Seconds of device time over `steps` consecutive steps."""
        torch = self.torch
        for i in range(warmup):
            self.step(i)
        torch.cuda.synchronize(self.dev)
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(steps)]
        ctx = sampler if sampler is not None else _Null()
        with ctx:
            for i in range(steps):
                ev[i][0].record()
                self.step(warmup + i)
                ev[i][1].record()
            torch.cuda.synchronize(self.dev)
        return sum(a.elapsed_time(b) for a, b in ev) / 1e3

    def timed_e2e(self, steps: int) -> tuple[float, int, int]:
        """Same steps through the public API from pinned host memory: each step
        copies its inputs H2D, runs, and copies out D2H (device-timed)."""
        torch = self.torch
        dev_in = {k: torch.empty_like(v, device=self.dev) for k, v in self.host[0].items()}
        out_host = torch.empty(self.out.shape, dtype=torch.float32).pin_memory()
        h2d = sum(v.numel() * v.element_size() for v in self.host[0].values())
        d2h = out_host.numel() * 4
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(steps)]
        torch.cuda.synchronize(self.dev)
        for i in range(steps):
            src = self.host[i % len(self.host)]
            ev[i][0].record()
            for k_, v_ in src.items():
                dev_in[k_].copy_(v_, non_blocking=True)
            self.pools[i % self.n_pools].step(dev_in["slot_idx"], dev_in["q"], dev_in["k"],
                                              dev_in["v"], dev_in["alpha"], dev_in["beta"],
                                              self.out)
            out_host.copy_(self.out, non_blocking=True)
            ev[i][1].record()
        torch.cuda.synchronize(self.dev)
        return sum(a.elapsed_time(b) for a, b in ev) / 1e3, h2d, d2h

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
    ofmt = O.FMT_FP32 if fmt == "fp32" else O.FMT_QUANT
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


def run_native(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = rank_workload(args.workload, rank)
    fmt = args.fmt
    b = Bench(w, fmt, device=dev)
    units = w.n * w.H
    ub = unit_bytes(w, fmt)

    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    sampler = ClockSampler(local_rank)
    secs = max_over_ranks(b.timed(args.steps, args.warmup, sampler), world, dev)
    if world > 1:
        dist.barrier()
    e2e_secs, h2d, d2h = (b.timed_e2e(args.steps) if not args.no_e2e else (float("nan"), 0, 0))
    e2e_secs = max_over_ranks(e2e_secs, world, dev)
    b.close()

    if rank != 0:
        return
    per_launch = secs / args.steps
    value = units * world * args.steps / secs
    gbs = ub * units / per_launch / 1e9
    peak, src = measured_peak()
    line = {
        "metric": METRIC, "value": value, "unit": "head-steps/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": per_launch * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic",
        "config": {"workload": describe(w, fmt), "units_per_step_per_gpu": units,
                   "algorithmic_bytes_per_unit": ub,
                   "l2": f"steps rotate over {b.n_pools} pools ({b.touched_bytes / 1e6:.0f} MB) "
                         "and their inputs, >= 4x L2: inputs larger than L2",
                   "timing": "CUDA events around each step on the launch stream, summed",
                   "parallelism": f"dp{world} (slots sharded, no collective)"},
        "hbm_gbs": gbs,
        "roofline": {"bound": "hbm", "achieved": gbs, "peak": peak, "unit": "GB/s",
                     "frac": gbs / peak, "peak_source": src,
                     "frac_of_8tbs_nominal": gbs / 8000.0,
                     "traffic": profiled_traffic(units)},
        "gpu_launches": args.steps,
        "clocks": sampler.summary(),
        "e2e": ({"value": units * world * args.steps / e2e_secs, "unit": "head-steps/s",
                 "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}
                if not args.no_e2e else None),
    }
    if world == 1 and args.cpu_seconds > 0:
        v, n, el = cpu_baseline(w, fmt, args.cpu_seconds)
        line["cpu_baseline"] = {"value": v, "unit": "head-steps/s", "cores": 1, "kind": "oracle",
                                "sample": f"{n} (slot, head) units of {w.name} ({fmt}), "
                                          f"one step each, single thread, {el:.1f} s"}
    if world == 1 and not args.no_variants:
        line["variants"] = variants(args, dev)
    print(json.dumps(line), flush=True)


def variants(args, dev):
    """Context: the same kernel on the other workloads and state formats."""
    res = []
    steps = max(20, min(args.steps, 200))
    for name, fmt in [("gdn_256x32", "mixed"), ("kda", "mixed"), ("hiconc_gdn", "mixed"),
                      ("hiconc_gdn", "int8"), ("hiconc_gdn", "fp32"), ("gdn_batch", "int8"),
                      ("gdn_batch", "fp32")]:
        w = W.WORKLOADS[name]
        b = Bench(w, fmt, device=dev)
        secs = b.timed(steps, 3)
        b.close()
        units = w.n * w.H
        ub = unit_bytes(w, fmt)
        gbs = ub * units * steps / secs / 1e9
        peak, _ = measured_peak()
        res.append({"workload": describe(w, fmt), "head_steps_per_s": units * steps / secs,
                    "us_per_step": secs / steps * 1e6, "hbm_gbs": gbs, "frac": gbs / peak,
                    "bytes_per_unit": ub})
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
        "config": {"workload": describe(w, fmt),
                   "sample": f"{per_step} (slot, head) units per step of the {w.n * w.H}"},
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
    ap.add_argument("--workload", default="gdn_batch", choices=list(W.WORKLOADS))
    ap.add_argument("--fmt", default="mixed", choices=["mixed", "int8", "fp32"])
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-variants", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
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

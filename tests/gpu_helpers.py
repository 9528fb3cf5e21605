"""Helpers for GPU-vs-oracle parity tests (test code: may use the oracle).

Both sides start from the same seeded FP32 initial state and consume the same
seeded step inputs; each side packs and steps its own state.  Nothing the GPU
produces is ever fed to the oracle.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle as O
import quantized_linear_attention_damp_b200 as D
import workloads as W

# tolerances fixed by the benchmark spec for this path
RTOL_OUT = 1e-4
ATOL_OUT = 1e-5


def oracle_fmt(fmt: str) -> int:
    return {"fp32": O.FMT_FP32, "fp8": O.FMT_FP8}.get(fmt, O.FMT_QUANT)


def gate_of(w: W.Workload) -> int:
    return O.GATE_VECTOR if w.gate == W.GATE_KDA else O.GATE_SCALAR


def torch_inputs(w: W.Workload, x: W.StepInputs, device="cuda") -> dict:
    if w.in_dtype == "bf16":
        cv = lambda bits: torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16)
        q, k, v = cv(x.q_bits), cv(x.k_bits), cv(x.v_bits)
    else:
        q, k, v = (torch.from_numpy(a) for a in (x.q, x.k, x.v))
    return dict(slot_idx=torch.from_numpy(x.slot_idx).to(device),
                q=q.to(device), k=k.to(device), v=v.to(device),
                alpha=torch.from_numpy(x.alpha).to(device),
                beta=torch.from_numpy(x.beta).to(device))


class Pair:
    """A GPU pool and an oracle pool built from the same workload."""

    def __init__(self, w: W.Workload, fmt: str | None = None, oracle_slots=None,
                 fp16_map=None, S0=None):
        self.w = w
        self.fmt = fmt or w.fmt
        self.hs = W.head_structure(w.with_(fmt=self.fmt))
        if fp16_map is not None:           # per-head FP16-row counts may differ
            self.is_fp16 = np.ascontiguousarray(fp16_map, np.uint8)
            self.gpu = D.DampPool("mixed", w.n_slots, w.H, w.d, fp16_map=self.is_fp16,
                                  d_v=w.d_v)
        else:
            self.is_fp16 = self.hs.is_fp16
            hp_idx = self.hs.hp_row_idx if self.fmt == "mixed" else None
            self.gpu = D.DampPool(self.fmt, w.n_slots, w.H, w.d, hp_idx, d_v=w.d_v)
        if S0 is None:
            S0 = W.initial_state(w, range(w.n_slots))
        S0 = np.ascontiguousarray(S0, np.float32)
        self.gpu.pack(torch.arange(w.n_slots, dtype=torch.int32, device="cuda"),
                      torch.from_numpy(S0).cuda())
        # oracle: all slots, or only the sampled ones (dict slot -> index)
        self.oracle_slots = list(range(w.n_slots)) if oracle_slots is None else list(oracle_slots)
        self.slot_pos = {s: i for i, s in enumerate(self.oracle_slots)}
        self.ora = O.pack(oracle_fmt(self.fmt), self.is_fp16[None],
                          S0[self.oracle_slots])
        self.diverged = set()

    # ---------------------------------------------------------------- steps
    def gpu_step(self, x: W.StepInputs) -> np.ndarray:
        t = torch_inputs(self.w, x)
        out = torch.empty((self.w.n, self.w.H, self.w.d_v), dtype=torch.float32, device="cuda")
        self.gpu.step(t["slot_idx"], t["q"], t["k"], t["v"], t["alpha"], t["beta"], out)
        torch.cuda.synchronize()
        return out.cpu().numpy()

    def oracle_step(self, x: W.StepInputs) -> dict:
        """Step the oracle's slots; returns {(b, h): o}."""
        res = {}
        gate = gate_of(self.w)
        for b, slot in enumerate(x.slot_idx):
            pos = self.slot_pos.get(int(slot))
            if pos is None:
                continue
            for h in range(self.w.H):
                st = self.ora[pos, h]
                res[(b, h)] = O.step_unit(st, gate, self.is_fp16[h], x.q[b, h], x.k[b, h],
                                          x.v[b, h], x.alpha[b, h], x.beta[b, h])
        return res

    def oracle_step_full(self, x: W.StepInputs) -> np.ndarray:
        assert len(self.oracle_slots) == self.w.n_slots
        return O.decode_step(self.ora, gate_of(self.w), self.is_fp16, x.slot_idx, x.q, x.k,
                             x.v, x.alpha, x.beta)

    # ---------------------------------------------------------------- checks
    def check_out(self, out_gpu: np.ndarray, out_ora) -> float:
        if isinstance(out_ora, dict):
            keys = list(out_ora)
            g = np.stack([out_gpu[b, h] for b, h in keys])
            o = np.stack([out_ora[k] for k in keys])
        else:
            g, o = out_gpu, out_ora
        err = np.abs(g.astype(np.float64) - o)
        bad = err > ATOL_OUT + RTOL_OUT * np.abs(o)
        assert not bad.any(), (
            f"out mismatch: {int(bad.sum())} entries, max err {err.max():.3g}")
        return float(err.max())

    def check_state(self) -> dict:
        """Compare the GPU state of the oracle's slots with the oracle state.

        Bit-exact expected (both sides take each rounding in the same
        precision and order); the stated tolerances are asserted: FP16 rows
        and scales within 1 ulp; INT8 codes +-1 on at most 0.1 % of entries.
        """
        lg = self.gpu.read_logical(self.oracle_slots)
        rep = {}
        if self.fmt == "fp32":
            g, o = lg["f32"], self.ora.f32
            err = np.abs(g.astype(np.float64) - o)
            assert not (err > ATOL_OUT + RTOL_OUT * np.abs(o)).any()
            rep["exact"] = bool(np.array_equal(g.view(np.uint32), o.view(np.uint32)))
            return rep
        dh = np.abs(lg["half"].astype(np.int64) - self.ora.half.astype(np.int64))
        ds = np.abs(lg["scale"].view(np.int32).astype(np.int64)
                    - self.ora.scale.view(np.int32).astype(np.int64))
        dc = np.abs(lg["code"].astype(np.int64) - self.ora.code.astype(np.int64))
        assert dh.max(initial=0) <= 1, "FP16 rows differ by more than 1 ulp"
        assert ds.max(initial=0) <= 1, "scales differ by more than 1 ulp"
        assert dc.max(initial=0) <= 1, "INT8 codes differ by more than 1"
        n_int8 = int((1 - self.is_fp16).sum()) * self.w.d_v * len(self.oracle_slots)
        assert dc.sum() <= max(1, 0.001 * n_int8), "more than 0.1 % of codes differ"
        rep.update(half_diff=int((dh > 0).sum()), scale_diff=int((ds > 0).sum()),
                   code_diff=int((dc > 0).sum()),
                   exact=bool(dh.max(initial=0) == 0 and ds.max(initial=0) == 0
                              and dc.max(initial=0) == 0))
        return rep

    def close(self):
        self.gpu.close()

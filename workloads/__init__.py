"""Seeded synthetic workloads for the DAMP-style decode step.

This module only draws random inputs.  It holds none of the method's
arithmetic (no dequantization, decay, delta rule, readout or requantization),
so both the CUDA path and the oracle may take their inputs from it.

Input recipe (the pages' workloads are real models on reasoning benchmarks;
none of their weights, prompts or activations exist here, so every tensor is
synthetic, with the shapes and structure the pages describe):

* q, k ~ N(0, 1), L2-normalised per (slot, head) in float32, then rounded to
  bf16 (round to nearest even) when the workload runs bf16 inputs; v ~ N(0, 1)
  rounded likewise.  beta = sigmoid(N(0, 1)).
* Decay: alpha = exp(-softplus(z) * a) with fresh z ~ N(0, 1) per step, where
  a = 1 / h and h is log-uniform on [1, 4096] steps: one h per head (GDN) or
  per (head, key channel) (KDA), so median half-lives span 1 to 4096 steps
  (the DAMP abstracts' decay-based persistence; STEPQuant Fig. 1b / B1 show
  half-lives of that spread).  The tiny GDN case instead holds one alpha per
  head, fixed over steps, uniform on [0.9, 0.999].
* Initial state: N(0, 0.1) per entry, times a per-(head, row) multiplier
  lognormal(0, 1) and x8 on 4 per-head columns (outliers concentrated in a few
  key channels and value dimensions, shared across slots: the DAMP v2
  abstract; STEPQuant Fig. 2b / B2).  The tiny case has 2 seeded rows x10 and
  no column outliers.
* Frozen FP16-row map (the calibration output the decode step consumes):
  GDN heads take the hp rows of largest expected energy (row multiplier; the
  tiny case ranks by the realised RMS of its one slot); KDA heads take the hp
  key channels of slowest decay (smallest a).  Ties go to the lower index.
* slot_idx: a seeded permutation of the slots per step (a random subset for
  the serving-shaped pool).

Every array is drawn from ``numpy.random.default_rng`` seeded with
``(seed, workload tag, tensor tag, index)``, so a unit's inputs can be
regenerated alone (the oracle checks sampled units of full-size workloads).
"""
from __future__ import annotations

import zlib
from dataclasses import dataclass, replace

import numpy as np

GATE_GDN = "gdn"
GATE_KDA = "kda"


@dataclass(frozen=True)
class Workload:
    name: str
    n: int            # batch entries per step
    n_slots: int      # slots in the pool
    H: int
    d: int            # d_k (and d_v, unless dv is set)
    hp: int           # FP16 rows per head (0 = uniform INT8)
    steps: int
    gate: str         # "gdn" | "kda"
    in_dtype: str     # "bf16" | "f32"
    fmt: str = "mixed"  # "mixed" | "int8" | "fp8" | "fp32"
    tiny: bool = False
    seed: int = 0
    dv: int = 0         # d_v when it differs from d (= d_k); 0: d_v = d

    @property
    def units(self) -> int:
        return self.n * self.H

    @property
    def d_v(self) -> int:
        return self.dv or self.d

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    # 1 slot x 2 heads, d=16, 64 steps, 4 FP16 rows/head, fp32 inputs
    "tiny_gdn": Workload("tiny_gdn", n=1, n_slots=1, H=2, d=16, hp=4, steps=64,
                         gate=GATE_GDN, in_dtype="f32", tiny=True),
    # 64 slots x 32 heads, d=128, 256 steps, 27 FP16 rows/head (~9.9 bits/value)
    "gdn_batch": Workload("gdn_batch", n=64, n_slots=64, H=32, d=128, hp=27, steps=256,
                          gate=GATE_GDN, in_dtype="bf16"),
    # 128 slots x 32 heads, KDA per-channel decay, 128 steps
    "kda": Workload("kda", n=128, n_slots=128, H=32, d=128, hp=27, steps=128,
                    gate=GATE_KDA, in_dtype="bf16"),
    # 512 slots x 48 heads, 32 steps (mixed; the fp32 and int8 variants via with_)
    "hiconc_gdn": Workload("hiconc_gdn", n=512, n_slots=512, H=48, d=128, hp=27, steps=32,
                           gate=GATE_GDN, in_dtype="bf16"),
    # 256 slots x 32 heads: the batch >= 256, 32-head, d=128 point
    "gdn_256x32": Workload("gdn_256x32", n=256, n_slots=256, H=32, d=128, hp=27, steps=32,
                           gate=GATE_GDN, in_dtype="bf16"),
    # other state sizes (context for the other kernels): d=64 (square thread-tile kernel) and
    # d=256 (any-shape kernel), FP16 rows ~21 % of the key rows as at d=128
    "d64_gdn": Workload("d64_gdn", n=1024, n_slots=1024, H=32, d=64, hp=13, steps=32,
                        gate=GATE_GDN, in_dtype="bf16"),
    "d256_gdn": Workload("d256_gdn", n=256, n_slots=256, H=8, d=256, hp=54, steps=32,
                         gate=GATE_GDN, in_dtype="bf16"),
}


def _tag(s: str) -> int:
    return zlib.crc32(s.encode())


def rng(w: Workload, tensor: str, *index: int) -> np.random.Generator:
    return np.random.default_rng([w.seed, _tag(w.name), _tag(tensor), *index])


def bf16_round(x: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """Round float32 to bf16 (nearest even): (bits uint16, exact float32 value)."""
    x = np.ascontiguousarray(x, np.float32)
    b = x.view(np.uint32).astype(np.uint64)
    b = (b + 0x7FFF + ((b >> 16) & 1)) >> 16
    bits = b.astype(np.uint16)
    val = (bits.astype(np.uint32) << 16).view(np.float32)
    return bits, val


@dataclass
class HeadStructure:
    row_mult: np.ndarray   # [H][d] float64
    col_mult: np.ndarray   # [H][d] float64
    decay_a: np.ndarray    # GDN [H], KDA [H][d]; tiny: unused
    tiny_alpha: np.ndarray | None  # tiny: [H] fixed alpha
    hp_row_idx: np.ndarray  # [H][hp] uint16, increasing
    is_fp16: np.ndarray     # [H][d] uint8


def head_structure(w: Workload) -> HeadStructure:
    H, d = w.H, w.d
    g = rng(w, "heads")
    if w.tiny:
        row_mult = np.ones((H, d))
        col_mult = np.ones((H, w.d_v))
        for h in range(H):
            rows = g.permutation(d)[:2]
            row_mult[h, rows] = 10.0
        tiny_alpha = g.uniform(0.9, 0.999, size=H)
        decay_a = np.zeros(H)
    else:
        row_mult = g.lognormal(0.0, 1.0, size=(H, d))
        col_mult = np.ones((H, w.d_v))
        for h in range(H):
            col_mult[h, g.permutation(w.d_v)[:4]] = 8.0
        tiny_alpha = None
        shape = (H, d) if w.gate == GATE_KDA else (H,)
        half_life = np.exp(g.uniform(np.log(1.0), np.log(4096.0), size=shape))
        decay_a = 1.0 / half_life
    hp_idx = np.zeros((H, w.hp), np.uint16)
    for h in range(H):
        if w.hp == 0:
            continue
        if w.gate == GATE_KDA:
            key = decay_a[h]                 # slowest decay first
            order = np.lexsort((np.arange(d), key))
        elif w.tiny:
            S0 = initial_state(w, [0], _structure=(row_mult, col_mult))[0, h]
            rms = np.sqrt(np.mean(S0.astype(np.float64) ** 2, axis=1))
            order = np.lexsort((np.arange(d), -rms))
        else:
            order = np.lexsort((np.arange(d), -row_mult[h]))
        hp_idx[h] = np.sort(order[: w.hp])
    is_fp16 = np.zeros((H, d), np.uint8)
    for h in range(H):
        is_fp16[h, hp_idx[h]] = 1
    if w.fmt in ("int8", "fp8"):
        hp_idx = np.zeros((H, 0), np.uint16)
        is_fp16[:] = 0
    return HeadStructure(row_mult, col_mult, decay_a, tiny_alpha, hp_idx, is_fp16)


def initial_state(w: Workload, slots, _structure=None) -> np.ndarray:
    """FP32 initial states [len(slots)][H][d][d_v] of the given pool slots."""
    if _structure is None:
        hs = head_structure(w)
        row_mult, col_mult = hs.row_mult, hs.col_mult
    else:
        row_mult, col_mult = _structure
    out = np.empty((len(slots), w.H, w.d, w.d_v), np.float32)
    for i, s in enumerate(slots):
        z = rng(w, "state", int(s)).standard_normal((w.H, w.d, w.d_v))
        out[i] = (0.1 * z * row_mult[:, :, None] * col_mult[:, None, :]).astype(np.float32)
    return out


@dataclass
class StepInputs:
    slot_idx: np.ndarray        # int32 [n]
    q: np.ndarray               # float32 [n][H][d] (exact values the kernel sees)
    k: np.ndarray
    v: np.ndarray
    q_bits: np.ndarray | None   # uint16 bf16 bits when in_dtype == "bf16"
    k_bits: np.ndarray | None
    v_bits: np.ndarray | None
    alpha: np.ndarray           # float32 [n][H] (GDN) or [n][H][d] (KDA)
    beta: np.ndarray            # float32 [n][H]


def step_inputs(w: Workload, step: int, hs: HeadStructure | None = None) -> StepInputs:
    hs = hs if hs is not None else head_structure(w)
    n, H, d = w.n, w.H, w.d
    g = rng(w, "step", step)
    if w.n == w.n_slots:
        slot_idx = g.permutation(w.n_slots).astype(np.int32)
    else:
        slot_idx = g.permutation(w.n_slots)[:n].astype(np.int32)
    q = g.standard_normal((n, H, d))
    k = g.standard_normal((n, H, d))
    v = g.standard_normal((n, H, w.d_v))
    q = (q / np.linalg.norm(q, axis=-1, keepdims=True)).astype(np.float32)
    k = (k / np.linalg.norm(k, axis=-1, keepdims=True)).astype(np.float32)
    v = v.astype(np.float32)
    beta = (1.0 / (1.0 + np.exp(-g.standard_normal((n, H))))).astype(np.float32)
    if w.tiny:
        alpha = np.broadcast_to(hs.tiny_alpha[None, :], (n, H)).astype(np.float32)
    elif w.gate == GATE_KDA:
        z = g.standard_normal((n, H, d))
        alpha = np.exp(-np.logaddexp(0.0, z) * hs.decay_a[None]).astype(np.float32)
    else:
        z = g.standard_normal((n, H))
        alpha = np.exp(-np.logaddexp(0.0, z) * hs.decay_a[None]).astype(np.float32)
    qb = kb = vb = None
    if w.in_dtype == "bf16":
        qb, q = bf16_round(q)
        kb, k = bf16_round(k)
        vb, v = bf16_round(v)
    return StepInputs(slot_idx, q, k, v, qb, kb, vb, np.ascontiguousarray(alpha),
                      np.ascontiguousarray(beta))


# ----------------------------------------------------------------------------
# Serving-shaped slot pool: 36 GDN-family layers x 32 heads, d = 128, a pool of
# 4096 slots per layer, and per step a random subset of 1024 slots (the same
# requests in every layer).  Every fourth layer (index 3 mod 4) is a KDA layer
# with per-key-channel decay.  To keep set-up tractable on the host, the
# initial state of slot s is the state drawn for template slot s mod 64 of
# that layer (64 templates per layer, each drawn as in initial_state).
# ----------------------------------------------------------------------------

SERVING_LAYERS = 36
SERVING_TEMPLATES = 64


def serving_layer(layer: int, seed: int = 0) -> Workload:
    gate = GATE_KDA if layer % 4 == 3 else GATE_GDN
    return Workload(f"serving_pool_l{layer}", n=1024, n_slots=4096, H=32, d=128, hp=27,
                    steps=16, gate=gate, in_dtype="bf16", seed=seed)


def serving_slot_idx(step: int, seed: int = 0, n: int = 1024, n_slots: int = 4096) -> np.ndarray:
    """The step's batch: a random subset of n pool slots, shared by all layers."""
    g = np.random.default_rng([seed, _tag("serving_pool"), _tag("slots"), step])
    return g.permutation(n_slots)[:n].astype(np.int32)


def serving_templates(w: Workload) -> np.ndarray:
    """Template states [SERVING_TEMPLATES][H][d][d]; slot s starts as template s % 64."""
    return initial_state(w, range(SERVING_TEMPLATES))


def serving_step_inputs(w: Workload, step: int, hs: HeadStructure | None = None) -> StepInputs:
    x = step_inputs(w, step, hs)
    x.slot_idx = serving_slot_idx(step, w.seed, w.n, w.n_slots)
    return x

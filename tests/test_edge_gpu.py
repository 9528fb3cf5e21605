"""GPU parity on the method's edge cases (through the C ABI, against the oracle).

Each case plants, in one small pool, the rows where the quantizer's special
rules or IEEE corner cases decide the stored bytes, and checks that the CUDA
step stores exactly what the oracle stores:

* a zero byte row (absmax 0: scale 0, codes 0) that the step keeps at zero
  (its k entry is 0);
* a byte row so small that 127/a overflows FP32 (stored as scale 0, codes 0),
  before and after the step;
* a byte row whose scale is an FP32 subnormal (absmax ~1e-36), whose
  dequantized values, decayed values and X are FP32 subnormals: the packed
  FP32 arithmetic must keep subnormals (no flush to zero) on the GPU;
* FP16 rows holding FP16 subnormals;
* an FP16 row driven past 65504 (X rounds to +-inf in binary16, IEEE
  overflow), next to values that round to 65504;
* a byte row whose pre-rounding values x*inv land exactly on .5 (INT8: absmax
  127 so inv = 1 and X = integer + 0.5; FP8: X on the midpoint of two E4M3
  values with inv = 1), where ties go to even.

Passages: Table C2 steps 1 and 6 of "STEPQuant ..." (reconstruct, requantize);
the readings the oracle states for zero rows, overflowing inverses, FP16
overflow and subnormals (no flush to zero on either side).
"""
import numpy as np
import pytest

import oracle as O
import workloads as W
from tests.gpu_helpers import Pair

pytestmark = pytest.mark.gpu

TIE, ZERO, TINY, SUB, BIG, F16SUB = 0, 1, 2, 4, 3, 5   # planted key rows
N_SLOTS, H = 3, 4


def e4m3_values():
    """Positive finite E4M3 values in increasing order (from the oracle's decoder)."""
    v = O.f32_from_e4m3(np.arange(0x01, 0x7F, dtype=np.uint8))
    return np.unique(v[np.isfinite(v)])


def fp16_map(d, seed):
    """FP16 rows of every head: BIG and F16SUB plus others, never the planted
    byte rows."""
    g = np.random.default_rng(seed)
    n = 4 if d == 16 else 27
    m = np.zeros((H, d), np.uint8)
    rest = [i for i in range(d) if i not in (TIE, ZERO, TINY, SUB, BIG, F16SUB)]
    for h in range(H):
        m[h, [BIG, F16SUB]] = 1
        m[h, g.permutation(rest)[: n - 2]] = 1
    return m


def edge_case(d, fmt, gate, in_dtype, overflow, seed=0):
    """(workload, initial states [N_SLOTS][H][d][d], per-step inputs)."""
    g = np.random.default_rng(seed)
    w = W.Workload(f"edge_d{d}_{fmt}_{gate}_{in_dtype}", n=N_SLOTS, n_slots=N_SLOTS, H=H, d=d,
                   hp=0, steps=1, gate=gate, in_dtype=in_dtype, fmt=fmt)
    S0 = (g.standard_normal((N_SLOTS, H, d, d)) * np.exp(g.standard_normal((N_SLOTS, H, d, 1)))
          ).astype(np.float32)
    e4 = e4m3_values()
    for s in range(N_SLOTS):
        # head 0, row TIE: X = integer + 0.5 (INT8) or an E4M3 midpoint (FP8)
        if fmt == "fp8":
            idx = g.integers(0, len(e4) - 2, d)
            row = e4[idx] * np.where(g.random(d) < 0.5, -1.0, 1.0)
            row[0] = 448.0
        else:
            row = g.integers(-127, 127, d).astype(np.float64)
            row[0] = 127.0
        S0[s, 0, TIE] = row
        # head 1: zero row, row too small for 127/a, subnormal-scale row, FP16 subnormals
        S0[s, 1, ZERO] = 0.0
        S0[s, 1, TINY] = g.standard_normal(d) * 1e-38
        # absmax where the scale a/Q is an FP32 subnormal and Q/a is finite:
        # Q = 127 needs a in (3.7e-37, 1.5e-36), Q = 448 (FP8) a in (1.3e-36, 5.3e-36)
        amax_sub = 3e-36 if fmt == "fp8" else 1e-36
        sub = g.standard_normal(d) * 0.3 * amax_sub
        sub[0] = amax_sub
        sub[1:4] = [1e-40, -3e-41, 7e-45]
        S0[s, 1, SUB] = sub
        S0[s, 1, F16SUB] = g.standard_normal(d) * 3e-6
        # head 2, row BIG: FP16 values near the top of the binary16 range
        if overflow:
            big = g.uniform(-3e4, 3e4, d)
            big[:8] = [60000.0, -60000.0, 65000.0, 30000.0, 1024.0, 2048.0, 4096.0, -4096.0]
            S0[s, 2, BIG] = big
    steps = []
    n_steps = 1 if overflow else 3
    for t in range(n_steps):
        slot_idx = np.int32(np.roll(np.arange(N_SLOTS), t + 1))
        q = g.standard_normal((N_SLOTS, H, d))
        k = g.standard_normal((N_SLOTS, H, d))
        v = g.standard_normal((N_SLOTS, H, d))
        alpha = (g.uniform(0.5, 1.0, (N_SLOTS, H, d)) if gate == W.GATE_KDA
                 else g.uniform(0.5, 1.0, (N_SLOTS, H)))
        beta = g.uniform(0.1, 1.0, (N_SLOTS, H))
        for b, slot in enumerate(slot_idx):
            # head 0: k = e_TIE, alpha = 1, beta = 1/2: X_TIE = (S_TIE + v) / 2
            k[b, 0] = 0.0
            k[b, 0, TIE] = 1.0
            alpha[b, 0] = 1.0
            beta[b, 0] = 0.5
            cur = S0[slot, 0, TIE].astype(np.float64) if t == 0 else None
            if cur is not None:
                if fmt == "fp8":
                    # the next E4M3 value away from zero: X on the midpoint
                    mag = np.abs(cur)
                    nxt = e4[np.minimum(np.searchsorted(e4, mag) + 1, len(e4) - 1)]
                    v[b, 0] = np.sign(cur) * nxt
                else:
                    v[b, 0] = cur + 1.0      # X = cur + 0.5
                v[b, 0, 0] = cur[0]          # absmax stays exactly 127 / 448
            # head 1: no delta update of the planted rows; a tiny one of TINY
            kk = k[b, 1]
            kk[[ZERO, SUB, F16SUB]] = 0.0
            kk[TINY] = 0.0
            kk /= np.linalg.norm(kk)
            kk[TINY] = 2e-37
            if overflow:
                # head 2: k = e_BIG, alpha = beta = 1: X_BIG = v exactly
                k[b, 2] = 0.0
                k[b, 2, BIG] = 1.0
                alpha[b, 2] = 1.0
                beta[b, 2] = 1.0
                tops = [70144.0, -70144.0, 65536.0, 65280.0]
                if in_dtype == "f32":
                    tops += [65504.0, 65519.99, 65520.0, -65520.0]
                v[b, 2] = g.uniform(-3e4, 3e4, d)
                v[b, 2, : len(tops)] = tops[:d]
            for h in ((3,) if overflow else (2, 3)):
                k[b, h] /= np.linalg.norm(k[b, h])
            q[b] /= np.linalg.norm(q[b], axis=-1, keepdims=True)
        q, k, v = (a.astype(np.float32) for a in (q, k, v))
        qb = kb = vb = None
        if in_dtype == "bf16":
            qb, q = W.bf16_round(q)
            kb, k2 = W.bf16_round(k)
            vb, v2 = W.bf16_round(v)
            # the planted values are bf16 numbers: rounding must not move them
            assert np.array_equal(k2[:, 0], k[:, 0])
            if t == 0:
                assert np.array_equal(v2[:, 0], v[:, 0])
            if overflow:
                assert np.array_equal(v2[:, 2, :4], v[:, 2, :4])
            k, v = k2, v2
        steps.append(W.StepInputs(slot_idx, q, k, v, qb, kb, vb,
                                  np.ascontiguousarray(alpha, np.float32),
                                  np.ascontiguousarray(beta, np.float32)))
    return w, S0, steps


CASES = [(16, fmt, gate, "f32") for fmt in ("mixed", "int8", "fp8")
         for gate in (W.GATE_GDN, W.GATE_KDA)]
CASES += [(128, fmt, gate, "bf16") for fmt in ("mixed", "int8", "fp8")
          for gate in (W.GATE_GDN, W.GATE_KDA)]
CASES += [(128, "mixed", W.GATE_GDN, "f32")]


@pytest.mark.parametrize("overflow", [True, False], ids=["fp16_overflow", "three_steps"])
@pytest.mark.parametrize("d,fmt,gate,in_dtype", CASES)
def test_edge_rows_bit_exact(d, fmt, gate, in_dtype, overflow):
    w, S0, steps = edge_case(d, fmt, gate, in_dtype, overflow, seed=d + len(fmt))
    fmap = fp16_map(d, 3) if fmt == "mixed" else None
    p = Pair(w, fmt, fp16_map=fmap, S0=S0)
    try:
        rep = p.check_state()
        assert rep["exact"], rep                          # pack parity on the planted rows
        lg = p.gpu.read_logical()
        if fmt != "fp32":
            # the planted rows were stored by the special rules
            assert not lg["code"][:, 1, ZERO].any() and not lg["scale"][:, 1, ZERO].any()
            assert not lg["code"][:, 1, TINY].any() and not lg["scale"][:, 1, TINY].any()
            s_sub = lg["scale"][:, 1, SUB]
            assert np.all((s_sub > 0) & (s_sub < np.finfo(np.float32).tiny))   # FP32 subnormal
        for x in steps:
            out_g = p.gpu_step(x)
            out_o = p.oracle_step_full(x)
            p.check_out(out_g, out_o)
            rep = p.check_state()
            assert rep["exact"], rep
        lg = p.gpu.read_logical()
        assert not lg["code"][:, 1, ZERO].any() and not lg["scale"][:, 1, ZERO].any()
        if fmt == "mixed":
            h16 = lg["half"][:, 1, F16SUB] & 0x7FFF
            assert np.any((h16 > 0) & (h16 < 0x0400))          # FP16 subnormals kept
            if overflow:
                big = lg["half"][:, 2, BIG]
                assert np.all(big[:, 0] == 0x7C00) and np.all(big[:, 1] == 0xFC00)
                assert np.all(big[:, 2] == 0x7C00)             # 65536 -> +inf
                if in_dtype == "f32":
                    assert np.all(big[:, 4] == 0x7BFF) and np.all(big[:, 5] == 0x7BFF)
                    assert np.all(big[:, 6] == 0x7C00) and np.all(big[:, 7] == 0xFC00)
        if overflow and fmt != "fp32":
            # the tie row: absmax exactly 127 (448), codes at ties to even
            sc = lg["scale"][:, 0, TIE]
            assert np.all(sc == np.float32(1.0))
            if fmt != "fp8":
                X = (S0[:, 0, TIE].astype(np.float64) + steps[0].v[:, 0].astype(np.float64)) / 2
                slot_of = {int(s): b for b, s in enumerate(steps[0].slot_idx)}
                for s in range(N_SLOTS):
                    Xs = (S0[s, 0, TIE].astype(np.float64)
                          + steps[0].v[slot_of[s], 0].astype(np.float64)) / 2
                    ties = np.abs(Xs - np.floor(Xs) - 0.5) == 0
                    assert ties.sum() > d // 2
                    want = np.round(Xs)          # numpy: half to even
                    assert np.array_equal(lg["code"][s, 0, TIE].astype(np.float64), want)
        assert p.gpu.get_error() == 0
    finally:
        p.close()

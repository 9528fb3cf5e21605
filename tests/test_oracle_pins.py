"""Pins of the oracle to facts other than itself (CPU only).

Each test ties one part of the oracle to something it does not compute by
itself: numpy's IEEE binary16 conversion, exact rational arithmetic, hand
values fixed by the definition of pairwise summation, an FP64 brute force of
the gated delta rule in matrix form, and invariants the mathematics fixes.
A plausible slip in the oracle (a dropped term, a wrong sign or index, a
transposed operand, a wrong scale or rounding rule, a readout taken after
requantization) fails at least one of them.
"""
import math
from fractions import Fraction

import numpy as np
import pytest

import oracle as O
import workloads as W
from tests import bruteforce as BF

RNG = np.random.default_rng(1234)


# ---------------------------------------------------------------- binary16

def test_f16_from_f32_matches_numpy_on_edges_and_random():
    # every binary16 value, the midpoints between neighbours (ties), and the
    # points just beside each midpoint
    h = np.arange(0, 0x7C00, dtype=np.uint16)            # +0 .. max finite
    vals = h.view(np.float16).astype(np.float64)
    mids = (vals[:-1] + vals[1:]) / 2.0                  # exact in float32? not always
    f32_mids = mids.astype(np.float32)
    nudges = np.concatenate([np.nextafter(f32_mids, np.float32(np.inf)),
                             np.nextafter(f32_mids, np.float32(0))])
    x = np.concatenate([vals.astype(np.float32), f32_mids, nudges,
                        np.float32([65504, 65519.996, 65520, 65536, 1e30, 6e-8, 3e-8, 2.9e-8,
                                    5.960464477539063e-08, 2.980232238769531e-08, 1e-45,
                                    np.inf])])
    x = np.concatenate([x, -x])
    x = np.concatenate([x, RNG.standard_normal(200000).astype(np.float32)
                        * np.float32(10.0) ** RNG.integers(-9, 6, 200000).astype(np.float32)])
    ours = O.f16_from_f32(x)
    ref = x.astype(np.float16).view(np.uint16)
    bad = np.nonzero(ours != ref)[0]
    assert bad.size == 0, (x[bad[:5]], ours[bad[:5]], ref[bad[:5]])


def test_f32_from_f16_all_bit_patterns():
    h = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = O.f32_from_f16(h)
    ref = h.view(np.float16).astype(np.float32)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan].view(np.uint32), ref[~nan].view(np.uint32))


# ---------------------------------------------------------------- INT8 rows

def _exact_codes(x):
    """Codes by exact rational arithmetic: nearest integer (ties to even) to
    x * fl32(127 / absmax), clamped to [-127, 127]."""
    x = np.asarray(x, np.float32)
    a = np.max(np.abs(x))
    with np.errstate(divide="ignore", over="ignore"):
        inv = np.float32(127.0) / a
    if a == 0 or not np.isfinite(inv):
        return np.zeros(x.shape, np.int8), np.float32(0.0)
    out = []
    for xv in x:
        t = Fraction(float(xv)) * Fraction(float(inv))
        fl = math.floor(t)
        r = t - fl
        c = fl + (1 if r > Fraction(1, 2) else 0 if r < Fraction(1, 2) else (fl & 1))
        out.append(max(-127, min(127, c)))
    return np.array(out, np.int8), np.float32(a / np.float32(127.0))


@pytest.mark.parametrize("seed", range(6))
def test_quantize_row_matches_exact_rational(seed):
    g = np.random.default_rng(seed)
    n = [16, 32, 64, 128, 128, 256][seed]
    x = (g.standard_normal(n) * 10.0 ** g.uniform(-6, 3)).astype(np.float32)
    code, scale = O.quantize_row(x)
    ref_code, ref_scale = _exact_codes(x)
    assert np.array_equal(code, ref_code)
    assert scale.view(np.uint32) == ref_scale.view(np.uint32)
    assert np.max(np.abs(code.astype(int))) == 127


def test_quantize_row_ties_go_to_even():
    # absmax 127 makes inv exactly 1, so x itself is the pre-rounding value
    x = np.float32([127.0, 2.5, 3.5, -2.5, -3.5, 0.5, -0.5, 1.5, 126.5, -126.5, 0.49999997])
    code, scale = O.quantize_row(x)
    assert list(code) == [127, 2, 4, -2, -4, 0, 0, 2, 126, -126, 0]
    assert scale == np.float32(1.0)


def test_quantize_row_zero_and_underflowing_rows():
    code, scale = O.quantize_row(np.zeros(16, np.float32))
    assert scale == 0 and not code.any()
    # 127 / 1e-38 overflows float32: stored as zero
    x = np.full(16, 1e-38, np.float32)
    code, scale = O.quantize_row(x)
    assert scale == 0 and not code.any()
    # just above the overflow threshold: quantized normally
    x = np.full(16, 1e-36, np.float32)
    code, scale = O.quantize_row(x)
    assert scale > 0 and np.all(code == 127)


def test_quantize_row_prerounding_is_the_exact_product():
    x = RNG.standard_normal(64).astype(np.float32)
    t = O.quantize_row_prerounding(x)
    inv = np.float32(127.0) / np.max(np.abs(x))
    assert np.array_equal(t, x.astype(np.float64) * np.float64(inv))


# ---------------------------------------------------------------- pairwise sum

def test_pairwise_sum_order_fixed_by_definition():
    f = np.float32
    # halves first: (1e8 + 1) + (-1e8 + 1) = 1e8 + -1e8 = 0 in float32,
    # whereas left-to-right gives 1
    assert O.pairwise_sum(f([1e8, 1, -1e8, 1])) == 0.0
    # adjacent pairs, not strided ones: (1e8 - 1e8) + (1 + 1) = 2,
    # whereas pairing i with i + n/2 gives 0
    assert O.pairwise_sum(f([1e8, -1e8, 1, 1])) == 2.0
    # eight terms: ((a+b)+(c+d)) + ((e+f)+(g+h))
    assert O.pairwise_sum(f([1e8, 1, 1, 1, -1e8, 1, 1, 1])) == 0.0


@pytest.mark.parametrize("n", [16, 32, 64, 128, 256])
def test_pairwise_sum_within_error_bound(n):
    x = (RNG.standard_normal(n) * np.exp(RNG.standard_normal(n) * 3)).astype(np.float32)
    exact = math.fsum(float(v) for v in x)
    u = 2.0 ** -24
    k = math.ceil(math.log2(n))
    bound = (k * u / (1 - k * u)) * float(np.sum(np.abs(x.astype(np.float64))))
    assert abs(float(O.pairwise_sum(x)) - exact) <= bound


# ---------------------------------------------------------------- FP32 state vs FP64

def _random_case(g, dk, dv, kda):
    S = (g.standard_normal((dk, dv)) * np.exp(g.standard_normal((dk, 1)))).astype(np.float32)
    q = g.standard_normal(dk)
    k = g.standard_normal(dk)
    q = (q / np.linalg.norm(q)).astype(np.float32)
    k = (k / np.linalg.norm(k)).astype(np.float32)
    v = g.standard_normal(dv).astype(np.float32)
    alpha = g.uniform(0.5, 1.0, dk if kda else 1).astype(np.float32)
    beta = np.float32(g.uniform(0.1, 1.0))
    return S, q, k, v, alpha, beta


@pytest.mark.parametrize("kda", [False, True])
@pytest.mark.parametrize("dk,dv", [(16, 16), (16, 32), (32, 16), (128, 128)])
def test_fp32_step_matches_fp64_bruteforce(kda, dk, dv):
    g = np.random.default_rng(dk * 7 + dv + kda)
    S, q, k, v, alpha, beta = _random_case(g, dk, dv, kda)
    st = O.pack(O.FMT_FP32, np.zeros(dk), S)
    gate = O.GATE_VECTOR if kda else O.GATE_SCALAR
    o = O.step_unit(st, gate, np.zeros(dk), q, k, v, alpha, beta)
    Sn, on = BF.step(S, q, k, v, alpha, beta)
    scale = np.max(np.abs(Sn))
    assert np.max(np.abs(st.f32 - Sn)) <= 1e-5 * scale
    assert np.max(np.abs(o - on)) <= 1e-5 * max(1.0, np.max(np.abs(on)))


def test_fp32_trajectory_tiny_gdn_matches_fp64():
    w = W.WORKLOADS["tiny_gdn"]
    hs = W.head_structure(w)
    S0 = W.initial_state(w, [0])
    pool = O.pack(O.FMT_FP32, np.zeros((w.H, w.d)), S0)
    ref = S0[0].astype(np.float64)
    for s in range(w.steps):
        x = W.step_inputs(w, s, hs)
        o = O.decode_step(pool, O.GATE_SCALAR, np.zeros((w.H, w.d)), x.slot_idx,
                          x.q, x.k, x.v, x.alpha, x.beta)
        for h in range(w.H):
            ref[h], on = BF.step(ref[h], x.q[0, h], x.k[0, h], x.v[0, h], x.alpha[0, h],
                                 x.beta[0, h])
            assert np.max(np.abs(o[0, h] - on)) <= 1e-5 * max(1.0, np.max(np.abs(on)))
    err = np.linalg.norm(pool.f32[0] - ref) / np.linalg.norm(ref)
    assert err < 1e-5


def test_delta_rule_write_invariant():
    # unit k, beta = 1, alpha = 1: the new state maps k to v exactly: k^T X = v^T
    g = np.random.default_rng(7)
    for dk, dv in [(16, 16), (128, 128), (32, 64)]:
        S, q, k, v, _, _ = _random_case(g, dk, dv, False)
        k = (k.astype(np.float64) / np.linalg.norm(k.astype(np.float64))).astype(np.float32)
        st = O.pack(O.FMT_FP32, np.zeros(dk), S)
        _, X = O.step_unit(st, O.GATE_SCALAR, np.zeros(dk), q, k, v, np.float32([1.0]), 1.0,
                           want_x=True)
        kx = k.astype(np.float64) @ X.astype(np.float64)
        assert np.max(np.abs(kx - v)) <= 1e-5 * max(1.0, np.max(np.abs(S)))


# ---------------------------------------------------------------- mixed format

def _mixed_case(seed, dk=128, hp=27, kda=False):
    g = np.random.default_rng(seed)
    S, q, k, v, alpha, beta = _random_case(g, dk, dk, kda)
    flags = np.zeros(dk, np.uint8)
    flags[g.permutation(dk)[:hp]] = 1
    return S, q, k, v, alpha, beta, flags


@pytest.mark.parametrize("kda", [False, True])
@pytest.mark.parametrize("hp", [0, 27, 128])
def test_mixed_step_against_fp64_from_dequantized_state(kda, hp):
    """Readout from X before requantization; new state = X within one
    quantization step (half a code times the row scale, or half an FP16 ulp)."""
    S, q, k, v, alpha, beta, flags = _mixed_case(11 + hp + kda, hp=hp, kda=kda)
    st = O.pack(O.FMT_QUANT, flags, S)
    Shat = O.unpack(st, flags)
    gate = O.GATE_VECTOR if kda else O.GATE_SCALAR
    o = O.step_unit(st, gate, flags, q, k, v, alpha, beta)
    Xbf, obf = BF.step(Shat, q, k, v, alpha, beta)
    # readout: FP32 X read out, within FP32 rounding of the FP64 value
    assert np.max(np.abs(o - obf)) <= 1e-5 * max(1.0, np.max(np.abs(obf)))
    # reading out the requantized state instead would be visibly different
    Snew = O.unpack(st, flags).astype(np.float64)
    if hp < 128:
        assert np.max(np.abs(Snew.T @ q - obf)) > 10 * np.max(np.abs(o - obf))
    # state: every entry within half a quantum (+ FP32 rounding of X)
    amax = np.max(np.abs(Xbf), axis=1)
    for i in range(128):
        if flags[i]:
            ulp = np.spacing(np.abs(Xbf[i]).astype(np.float16)).astype(np.float64)
            tol = 0.5 * ulp + 1e-6 * amax[i]
        else:
            tol = 0.5 * st.scale[i] + 1e-6 * amax[i]
        assert np.all(np.abs(Snew[i] - Xbf[i]) <= tol), i


@pytest.mark.parametrize("hp", [0, 27])
def test_identity_step_leaves_codes_unchanged(hp):
    # alpha = 1, beta = 0: X = S^, and requantizing a dequantized state is idempotent
    S, q, k, v, _, _, flags = _mixed_case(21 + hp, hp=hp)
    st = O.pack(O.FMT_QUANT, flags, S)
    before = st.copy()
    for _ in range(3):
        O.step_unit(st, O.GATE_SCALAR, flags, q, k, v, np.float32([1.0]), 0.0)
    assert np.array_equal(st.code, before.code)
    assert np.array_equal(st.half, before.half)
    d = np.abs(st.scale.view(np.int32).astype(np.int64) - before.scale.view(np.int32))
    assert d.max() <= 1


def test_pure_decay_leaves_int8_codes_unchanged():
    # beta = 0, alpha < 1 scales each row; the per-row scale absorbs it
    S, q, k, v, _, _, flags = _mixed_case(31, hp=0)
    st = O.pack(O.FMT_QUANT, flags, S)
    before = st.copy()
    O.step_unit(st, O.GATE_SCALAR, flags, q, k, v, np.float32([0.75]), 0.0)
    assert np.array_equal(st.code, before.code)
    assert np.allclose(st.scale, before.scale * np.float32(0.75), rtol=4e-7, atol=0)


def test_gdn_equals_kda_with_constant_vector():
    S, q, k, v, _, beta, flags = _mixed_case(41)
    a = np.float32(0.93)
    s1 = O.pack(O.FMT_QUANT, flags, S)
    s2 = s1.copy()
    o1 = O.step_unit(s1, O.GATE_SCALAR, flags, q, k, v, np.float32([a]), beta)
    o2 = O.step_unit(s2, O.GATE_VECTOR, flags, q, k, v, np.full(128, a, np.float32), beta)
    assert np.array_equal(o1, o2)
    for f in ("scale", "half", "code"):
        assert np.array_equal(getattr(s1, f), getattr(s2, f))


def test_pack_unpack_pack_round_trip():
    S, _, _, _, _, _, flags = _mixed_case(51)
    p1 = O.pack(O.FMT_QUANT, flags, S)
    p2 = O.pack(O.FMT_QUANT, flags, O.unpack(p1, flags))
    assert np.array_equal(p1.code, p2.code)
    assert np.array_equal(p1.half, p2.half)
    d = np.abs(p1.scale.view(np.int32).astype(np.int64) - p2.scale.view(np.int32))
    assert d.max() <= 1


def test_all_fp16_pool_tracks_fp64_rounded_each_step():
    """hp = d_k: from the same pre-state, one oracle step equals the FP64 step
    rounded to binary16 within one FP16 ulp per entry (tiny workload, 64 steps)."""
    w = W.WORKLOADS["tiny_gdn"].with_(hp=16)
    hs = W.head_structure(w)
    assert hs.is_fp16.all()
    pool = O.pack(O.FMT_QUANT, hs.is_fp16, W.initial_state(w, [0]))
    for s in range(w.steps):
        x = W.step_inputs(w, s, hs)
        pre = O.unpack(pool, hs.is_fp16[None])[0]
        o = O.decode_step(pool, O.GATE_SCALAR, hs.is_fp16, x.slot_idx, x.q, x.k, x.v,
                          x.alpha, x.beta)
        post = O.f32_from_f16(pool.half[0])
        for h in range(w.H):
            Xbf, obf = BF.step(pre[h], x.q[0, h], x.k[0, h], x.v[0, h], x.alpha[0, h],
                               x.beta[0, h])
            ref = BF.round_f16(Xbf).astype(np.float64)
            ulp = np.spacing(np.abs(ref).astype(np.float16)).astype(np.float64)
            assert np.all(np.abs(post[h] - ref) <= ulp), (s, h)
            assert np.max(np.abs(o[0, h] - obf)) <= 1e-5 * max(1.0, np.max(np.abs(obf)))


def test_int8_codes_match_exact_quantization_of_fp64_step():
    """hp = 0: codes of one step equal the exact quantization of the FP64 X,
    except +-1 where the FP64 value lies within FP32 noise of a .5 boundary."""
    S, q, k, v, alpha, beta, flags = _mixed_case(61, hp=0, kda=True)
    st = O.pack(O.FMT_QUANT, flags, S)
    Shat = O.unpack(st, flags)
    O.step_unit(st, O.GATE_VECTOR, flags, q, k, v, alpha, beta)
    Xbf, _ = BF.step(Shat, q, k, v, alpha, beta)
    n_near = 0
    for i in range(128):
        a = np.max(np.abs(Xbf[i]))
        t = Xbf[i] * (127.0 / a)
        ref = np.clip(np.round(t), -127, 127)       # numpy rounds half to even
        diff = st.code[i].astype(np.float64) - ref
        near = np.abs(np.abs(t - np.floor(t)) - 0.5) < 2e-4
        assert np.all(np.abs(diff) <= 1)
        assert np.all(near[diff != 0])
        n_near += int(near.sum())
        assert abs(float(st.scale[i]) - a / 127.0) <= 1e-5 * a / 127.0
    assert n_near < 20


def test_padding_and_range_of_slot_index():
    w = W.WORKLOADS["tiny_gdn"]
    hs = W.head_structure(w)
    pool = O.pack(O.FMT_QUANT, hs.is_fp16, W.initial_state(w, [0]))
    before = pool.copy()
    x = W.step_inputs(w, 0, hs)
    o = O.decode_step(pool, O.GATE_SCALAR, hs.is_fp16, np.int32([-1]), x.q, x.k, x.v,
                      x.alpha, x.beta)
    assert not o.any()
    assert np.array_equal(pool.code, before.code) and np.array_equal(pool.half, before.half)
    with pytest.raises(ValueError):
        O.decode_step(pool, O.GATE_SCALAR, hs.is_fp16, np.int32([1]), x.q, x.k, x.v,
                      x.alpha, x.beta)


def test_update_is_one_rounding_of_the_exact_value():
    """With k = e_0 and alpha = 1, u_j = S_0j exactly, delta_j = fl(v_j - S_0j)
    and b_0 = fl(beta); row 0 of X must be the exact b_0*delta_j + S_0j rounded
    once to FP32 (exact rational arithmetic), and the other rows stay S."""
    g = np.random.default_rng(71)
    dk, dv = 16, 256
    hits = 0
    for trial in range(8):
        S = (g.standard_normal((dk, dv))).astype(np.float32)
        v = (S[0] * np.float32(1.0 + g.uniform(-0.5, 0.5)) + g.standard_normal(dv)
             .astype(np.float32)).astype(np.float32)
        k = np.zeros(dk, np.float32)
        k[0] = 1.0
        beta = np.float32(g.uniform(0.2, 0.9))
        st = O.pack(O.FMT_FP32, np.zeros(dk), S)
        _, X = O.step_unit(st, O.GATE_SCALAR, np.zeros(dk), np.ones(dk, np.float32), k, v,
                           np.float32([1.0]), beta, want_x=True)
        assert np.array_equal(X[1:], S[1:])
        delta = (v - S[0]).astype(np.float32)               # one float32 subtraction
        for j in range(dv):
            exact = Fraction(float(beta)) * Fraction(float(delta[j])) + Fraction(float(S[0, j]))
            ref = np.float32(float(exact))                  # double then float32
            # skip the (vanishingly rare) double-rounding tie case
            lo, hi = np.nextafter(ref, np.float32(-np.inf)), np.nextafter(ref, np.float32(np.inf))
            if abs(Fraction(float(ref)) - exact) > min(abs(Fraction(float(lo)) - exact),
                                                       abs(Fraction(float(hi)) - exact)):
                continue
            assert X[0, j] == ref, (trial, j)
            two_step = np.float32(np.float32(beta * delta[j]) + S[0, j])
            hits += int(two_step != ref)
    assert hits > 0   # the case does separate one rounding from two


# ---------------------------------------------------------------- batch slot gather

def _gather_case(seed, dk, dv, kda):
    """A pool of 6 slots x 2 heads and a batch of 4 entries whose slot
    indices are permuted, with one padding entry: entry b steps slot
    slot_idx[b], which differs from b for every stepped entry."""
    g = np.random.default_rng(seed)
    n_slots, H = 6, 2
    S = (g.standard_normal((n_slots, H, dk, dv))
         * np.exp(g.standard_normal((n_slots, H, dk, 1)))).astype(np.float32)
    slot_idx = np.int32([4, -1, 0, 5])
    n = slot_idx.size
    q = g.standard_normal((n, H, dk))
    k = g.standard_normal((n, H, dk))
    q = (q / np.linalg.norm(q, axis=-1, keepdims=True)).astype(np.float32)
    k = (k / np.linalg.norm(k, axis=-1, keepdims=True)).astype(np.float32)
    v = g.standard_normal((n, H, dv)).astype(np.float32)
    alpha = g.uniform(0.5, 1.0, (n, H, dk) if kda else (n, H)).astype(np.float32)
    beta = g.uniform(0.1, 1.0, (n, H)).astype(np.float32)
    return S, slot_idx, q, k, v, alpha, beta


@pytest.mark.parametrize("kda", [False, True])
@pytest.mark.parametrize("dk,dv", [(16, 16), (16, 32)])
def test_batch_step_gathers_each_entry_slot(kda, dk, dv):
    """Entry b reads and writes pool slot slot_idx[b] with entry b's inputs:
    each stepped slot and each readout o[b] equal the FP64 brute force of the
    matrix form applied to that slot's own pre-state and entry b's inputs;
    the padding entry reads out zeros and slots nobody stepped keep their
    bytes.  (Swapping the entry and slot indices anywhere in the batch step
    fails here: every stepped slot differs from its entry.)"""
    S, slot_idx, q, k, v, alpha, beta = _gather_case(91 + dk + dv + kda, dk, dv, kda)
    n_slots, H = S.shape[:2]
    gate = O.GATE_VECTOR if kda else O.GATE_SCALAR
    pool = O.pack(O.FMT_FP32, np.zeros((H, dk)), S)
    o = O.decode_step(pool, gate, np.zeros((H, dk), np.uint8), slot_idx, q, k, v, alpha, beta)
    stepped = set()
    for b, slot in enumerate(slot_idx):
        if slot < 0:
            assert not o[b].any()
            continue
        stepped.add(int(slot))
        for h in range(H):
            Sn, on = BF.step(S[slot, h], q[b, h], k[b, h], v[b, h], alpha[b, h], beta[b, h])
            assert np.max(np.abs(pool.f32[slot, h] - Sn)) <= 1e-5 * np.max(np.abs(Sn)), (b, h)
            assert np.max(np.abs(o[b, h] - on)) <= 1e-5 * max(1.0, np.max(np.abs(on))), (b, h)
    for slot in range(n_slots):
        if slot not in stepped:
            assert np.array_equal(pool.f32[slot].view(np.uint32), S[slot].view(np.uint32))


def test_batch_step_gather_quantized_matches_unit_steps():
    """Mixed format: the batch step equals unit steps taken on the slot that
    each entry names, bit for bit (the unit step is pinned on its own above)."""
    S, slot_idx, q, k, v, alpha, beta = _gather_case(97, 32, 32, False)
    n_slots, H, dk, dv = S.shape
    g = np.random.default_rng(98)
    flags = np.zeros((H, dk), np.uint8)
    for h in range(H):
        flags[h, g.permutation(dk)[:7]] = 1
    pool = O.pack(O.FMT_QUANT, flags[None], S)
    ref = pool.copy()
    o = O.decode_step(pool, O.GATE_SCALAR, flags, slot_idx, q, k, v, alpha, beta)
    for b, slot in enumerate(slot_idx):
        if slot < 0:
            continue
        for h in range(H):
            ou = O.step_unit(ref[slot, h], O.GATE_SCALAR, flags[h], q[b, h], k[b, h], v[b, h],
                             alpha[b, h], beta[b, h])
            assert np.array_equal(o[b, h], ou)
    for f in ("scale", "half", "code"):
        assert np.array_equal(getattr(pool, f), getattr(ref, f))
    assert not np.array_equal(pool.code[4], O.pack(O.FMT_QUANT, flags[None], S).code[4])

"""Pins of the oracle's FP8 (E4M3) comparison format.

The E4M3 encoding is fixed by the OCP 8-bit floating point specification
(sign, 4 exponent bits with bias 7, 3 mantissa bits, subnormals, no
infinities, S.1111.111 = NaN, largest finite 448).  Checked: values of named
codes, an exhaustive nearest-value brute force against a table built here from
the bit-field definition, and the per-row scaling.
"""
import numpy as np
import pytest

import oracle as O


def spec_value(c: int) -> float:
    """E4M3 value from the bit fields (independent restatement for the pins)."""
    s, e, m = c >> 7, (c >> 3) & 15, c & 7
    if e == 15 and m == 7:
        return float("nan")
    v = m * 2.0 ** -9 if e == 0 else (8 + m) * 2.0 ** (e - 10)
    return -v if s else v


FINITE = [c for c in range(256) if not np.isnan(spec_value(c))]


def test_named_codes():
    named = {0x00: 0.0, 0x38: 1.0, 0x40: 2.0, 0xB8: -1.0, 0x7E: 448.0, 0xFE: -448.0,
             0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6, 0x30: 0.5, 0x3C: 1.5,
             0x77: 240.0}
    for c, v in named.items():
        assert O.f32_from_e4m3(np.array([c], np.uint8))[0] == v, hex(c)
        assert O.e4m3_from_f32(np.array([v], np.float32))[0] == c, v
    assert np.isnan(O.f32_from_e4m3(np.array([0x7F, 0xFF], np.uint8))).all()


def test_decoder_matches_the_bit_field_definition():
    codes = np.arange(256, dtype=np.uint8)
    got = O.f32_from_e4m3(codes)
    want = np.array([spec_value(c) for c in range(256)], np.float32)
    same = (got == want) | (np.isnan(got) & np.isnan(want))
    assert same.all()


def test_every_finite_code_round_trips():
    codes = np.array(FINITE, np.uint8)
    back = O.e4m3_from_f32(O.f32_from_e4m3(codes))
    # +0 and -0 both encode back to their own sign
    assert np.array_equal(back, codes)


def test_nearest_value_bruteforce():
    """Random FP32 inputs (all binades from below the subnormals to past 448)
    encode to the nearest finite E4M3 value; exact midpoints go to the code
    with an even mantissa; magnitudes beyond 448 saturate."""
    g = np.random.default_rng(0)
    x = (g.choice([-1, 1], 4000) * 2.0 ** g.uniform(-12, 9.5, 4000)).astype(np.float32)
    # plus every exact midpoint between neighbouring positive finite values
    pos = sorted({spec_value(c) for c in FINITE if spec_value(c) >= 0})
    mids = np.array([(a + b) / 2 for a, b in zip(pos, pos[1:])], np.float32)
    x = np.concatenate([x, mids, -mids, np.float32([448.1, 470, 1e6, -500])])
    vals = np.array([spec_value(c) for c in FINITE])
    got = O.e4m3_from_f32(x)
    for xi, ci in zip(x.astype(np.float64), got):
        if abs(xi) > 448:
            assert spec_value(int(ci)) == np.sign(xi) * 448
            continue
        d = np.abs(vals - xi)
        best = d.min()
        cands = [FINITE[i] for i in np.flatnonzero(d == best)
                 if np.signbit(vals[i]) == np.signbit(xi) or vals[i] != 0]
        if len(cands) > 1:            # tie: even mantissa
            cands = [c for c in cands if (c & 1) == 0]
        assert int(ci) in cands, (xi, hex(ci), [hex(c) for c in cands])


def test_row_scaling():
    code, s = O.quantize_row_fp8(np.array([448, 1, -3.5, 0.0078125], np.float32))
    assert s == np.float32(1.0)
    assert code.tolist() == [0x7E, 0x38, 0xC6, 0x04]     # 448, 1, -3.5, 2^-7 (subnormal)
    code, s = O.quantize_row_fp8(np.zeros(5, np.float32))
    assert s == 0 and not code.any()
    # absmax maps to 448 whatever its size; scale = fl(a/448)
    g = np.random.default_rng(1)
    for _ in range(20):
        x = (g.standard_normal(32) * 10.0 ** g.uniform(-5, 5)).astype(np.float32)
        code, s = O.quantize_row_fp8(x)
        a = np.max(np.abs(x))
        assert s == np.float32(a) / np.float32(448)
        assert O.f32_from_e4m3(code[np.argmax(np.abs(x))])[()] in (448.0, -448.0)


@pytest.mark.parametrize("seed", range(3))
def test_fp8_state_error_is_within_half_a_quantum(seed):
    """Round trip of a state: each entry is within half an E4M3 quantum (of
    the scaled value's binade) times the scale, plus the FP32 roundings."""
    g = np.random.default_rng(seed)
    S = (g.standard_normal((4, 16)) * g.lognormal(0, 1, (4, 1))).astype(np.float32)
    st = O.pack(O.FMT_FP8, np.zeros(4, np.uint8), S)
    R = O.unpack(st, np.zeros(4, np.uint8))
    for i in range(4):
        s = np.float64(st.scale[i])
        y = np.abs(S[i].astype(np.float64)) / s
        quantum = np.where(y < 2.0 ** -6, 2.0 ** -9, 2.0 ** (np.floor(np.log2(np.maximum(y, 2.0 ** -6))) - 3))
        err = np.abs(R[i].astype(np.float64) - S[i])
        assert (err <= (quantum / 2) * s * (1 + 1e-6) + 4 * np.spacing(np.abs(S[i]))).all()


def test_identity_step_keeps_fp8_codes():
    """alpha = 1, beta = 0: the step requantizes the dequantized state, which
    reproduces every E4M3 code (scales within 1 ulp)."""
    g = np.random.default_rng(7)
    dk = dv = 16
    S = (g.standard_normal((dk, dv)) * g.lognormal(0, 1, (dk, 1))).astype(np.float32)
    flags = np.zeros(dk, np.uint8)
    st = O.pack(O.FMT_FP8, flags, S)
    before = st.copy()
    q, k, v = (g.standard_normal(dk).astype(np.float32) for _ in range(3))
    O.step_unit(st, O.GATE_SCALAR, flags, q, k, v, np.float32(1.0), np.float32(0.0))
    assert np.array_equal(st.code, before.code)
    assert np.abs(st.scale.view(np.int32).astype(np.int64)
                  - before.scale.view(np.int32).astype(np.int64)).max() <= 1
    assert not st.half.any()

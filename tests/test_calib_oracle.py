"""Pins of the calibration oracle (offline selection of the FP16 key rows).

Each check rests on something other than the oracle itself: closed forms of
the INT8 quantizer's error on rows chosen so every code is known, an exact
rational brute force on random tiny rows, the geometric-series persistence for
a constant decay, and the configurations' own hand rules for the special cases
where the calibration must reduce to them (uniform error energy in a KDA head:
the slowest-decay channels; a scalar GDN decay: the error-energy ranking).
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle as O
import workloads as W


def test_row_error_closed_forms():
    # absmax 127: scale 1, inverse 1; 0.5 -> 0, 1.5 -> 2, -2.5 -> -2 (ties to even)
    assert O.row_quant_error(np.array([127, 0.5, 1.5, -2.5], np.float32)) == 0.75
    # absmax 254: scale 2, inverse 0.5; 3 -> 1.5 -> 2 -> 4, 5 -> 2.5 -> 2 -> 4, 7 -> 3.5 -> 4 -> 8
    assert O.row_quant_error(np.array([254, 3, 5, 7], np.float32)) == 3.0
    # rows on the grid have no error; the zero row has none either
    assert O.row_quant_error(np.array([127, -3, 0, 64, -127], np.float32)) == 0.0
    assert O.row_quant_error(np.zeros(16, np.float32)) == 0.0
    # a single nonzero entry is always exact (code +-127, scale a/127)
    s = np.float32(0.3) / np.float32(127)
    dq = np.float32(-127) * s
    assert O.row_quant_error(np.array([0, 0, -0.3, 0], np.float32)) == \
        float((np.float64(np.float32(-0.3)) - np.float64(dq)) ** 2)


def _exact_error(x: np.ndarray) -> Fraction:
    """Brute force: codes from the exact product x * fl32(127/a), ties to even
    (Python's round on a Fraction), dequantized in FP32, error in rationals."""
    a = np.max(np.abs(x))
    if a == 0:
        return Fraction(0)
    inv = np.float32(127) / np.float32(a)
    s = np.float32(a) / np.float32(127)
    tot = Fraction(0)
    for xj in x:
        c = round(Fraction(float(xj)) * Fraction(float(inv)))
        c = max(-127, min(127, c))
        dq = np.float32(np.float32(c) * s)
        tot += (Fraction(float(xj)) - Fraction(float(dq))) ** 2
    return tot


@pytest.mark.parametrize("seed", range(6))
def test_row_error_matches_exact_bruteforce(seed):
    g = np.random.default_rng(seed)
    n = int(g.integers(1, 40))
    x = (g.standard_normal(n) * 10.0 ** g.uniform(-6, 3)).astype(np.float32)
    exact = _exact_error(x)
    got = O.row_quant_error(x)
    assert abs(Fraction(got) - exact) <= Fraction(1, 10 ** 12) * max(exact, Fraction(1, 10 ** 300))


def test_accumulate_counts_retention_and_geometric_persistence():
    """Constant GDN decay: retention/count = alpha^2 exactly, and the score is
    the mean error energy times the geometric sum 1/(1 - alpha^2)."""
    g = np.random.default_rng(3)
    H, dk, dv, n_slots = 2, 8, 8, 5
    acc = O.calib_acc(H, dk)
    alpha = np.float32(0.9)
    per_step = []
    for t in range(3):
        pool = g.standard_normal((n_slots, H, dk, dv)).astype(np.float32)
        slots = np.array([4, -1, 0], np.int32)            # one padding entry
        O.calib_accumulate(acc, O.GATE_SCALAR, pool, slots, np.full((3, H), alpha, np.float32))
        e = np.zeros((H, dk))
        for s in (4, 0):
            for h in range(H):
                for i in range(dk):
                    e[h, i] += O.row_quant_error(pool[s, h, i])
        per_step.append(e)
    energy = acc[:H * dk].reshape(H, dk)
    retention = acc[H * dk:2 * H * dk].reshape(H, dk)
    count = acc[2 * H * dk:]
    assert np.array_equal(count, [6.0, 6.0])
    a2 = float(np.float64(alpha) ** 2)
    assert np.allclose(retention, 6 * a2, rtol=0, atol=1e-15)
    assert np.allclose(energy, sum(per_step), rtol=1e-15, atol=0)
    score = O.calib_scores(acc, H, dk)
    assert np.allclose(score, energy / 6 / (1 - a2), rtol=1e-14, atol=0)


def test_retention_follows_each_batch_entry_and_channel():
    """KDA: the decay of batch entry b, head h, channel i is credited to row i
    of head h only when entry b is not padding."""
    g = np.random.default_rng(4)
    H, dk, n = 2, 4, 3
    alpha = g.uniform(0.1, 1.0, (n, H, dk)).astype(np.float32)
    acc = O.calib_acc(H, dk)
    O.calib_accumulate(acc, O.GATE_VECTOR, np.zeros((3, H, dk, dk), np.float32),
                       np.array([2, -1, 0], np.int32), alpha)
    a64 = alpha.astype(np.float64)
    assert np.array_equal(acc[H * dk:2 * H * dk].reshape(H, dk), a64[0] ** 2 + a64[2] ** 2)
    assert not acc[:H * dk].any()


def test_accumulate_rejects_out_of_range_slots():
    acc = O.calib_acc(1, 4)
    pool = np.ones((2, 1, 4, 4), np.float32)
    with pytest.raises(ValueError):
        O.calib_accumulate(acc, O.GATE_SCALAR, pool, np.array([2], np.int32),
                           np.ones((1, 1), np.float32))


def test_never_decaying_row_gets_the_floor_not_infinity():
    acc = O.calib_acc(1, 2)
    pool = np.array([[[[127, 0.5], [1, 1]]]], np.float32)
    O.calib_accumulate(acc, O.GATE_VECTOR, pool, np.array([0], np.int32),
                       np.array([[[1.0, 0.5]]], np.float32))
    score = O.calib_scores(acc, 1, 2)
    assert score[0, 0] == 0.25 * 2.0 ** 30
    assert score[0, 1] == 0.0


def test_select_ties_go_to_the_lower_row():
    score = np.array([[1.0, 3.0, 3.0, 2.0, 3.0]])
    assert O.calib_select(score, 2).tolist() == [[1, 2]]
    assert O.calib_select(score, 4).tolist() == [[1, 2, 3, 4]]
    assert O.calib_select(score, 0).shape == (1, 0)
    assert O.calib_select(np.zeros((2, 4)), 1).tolist() == [[0], [0]]


def test_kda_with_uniform_error_energy_selects_the_slowest_decay_channels():
    """Every row of every state identical -> equal error energy per row; with
    each channel decaying at its median rate 2^(-a_c) (softplus(0) = ln 2) the
    score orders rows by decay, and the selection is the KDA configuration's
    rule (the channels with the longest half-life)."""
    w = W.WORKLOADS["kda"].with_(n=4, n_slots=4, H=3, d=32, hp=6)
    hs = W.head_structure(w)
    g = np.random.default_rng(0)
    acc = O.calib_acc(w.H, w.d)
    alpha = np.broadcast_to(np.exp2(-hs.decay_a).astype(np.float32), (w.n, w.H, w.d)).copy()
    for t in range(4):
        row = g.standard_normal(w.d).astype(np.float32)
        pool = np.broadcast_to(row, (w.n_slots, w.H, w.d, w.d)).copy()
        O.calib_accumulate(acc, O.GATE_VECTOR, pool, g.permutation(w.n).astype(np.int32), alpha)
    sel = O.calib_select(O.calib_scores(acc, w.H, w.d), w.hp)
    assert np.array_equal(sel, np.sort(hs.hp_row_idx, axis=1))


def test_gdn_selection_is_the_error_energy_ranking():
    """Scalar decay: persistence is the same for every row of a head, so the
    rows with planted large quantization error are the ones selected."""
    H, dk, dv = 2, 16, 16
    g = np.random.default_rng(1)
    acc = O.calib_acc(H, dk)
    planted = [[3, 9, 12], [0, 7, 15]]
    for t in range(3):
        # rows on the INT8 grid (no error) except the planted ones
        pool = np.zeros((1, H, dk, dv), np.float32)
        pool[..., 0] = 127
        pool[..., 1:] = g.integers(-127, 128, (1, H, dk, dv - 1))
        for h in range(H):
            for r, i in enumerate(planted[h]):
                pool[0, h, i, 1:] += 0.25 + 0.1 * r          # off-grid: error grows with r
        O.calib_accumulate(acc, O.GATE_SCALAR, pool, np.array([0], np.int32),
                           g.uniform(0.5, 0.99, (1, H)).astype(np.float32))
    sel = O.calib_select(O.calib_scores(acc, H, dk), 3)
    assert sel.tolist() == [sorted(p) for p in planted]
    # with hp = 2 the two largest planted errors win
    assert O.calib_select(O.calib_scores(acc, H, dk), 2).tolist() == \
        [sorted(p[1:]) for p in planted]


def test_budget_selection():
    score = np.array([[5.0, 1.0, 4.0, 0.0],
                      [6.0, 5.0, 0.5, 2.0],
                      [0.1, 0.2, 0.3, 0.4]])
    is16, hp = O.calib_select_budget(score, 4)
    assert hp.tolist() == [2, 2, 0]
    assert is16.tolist() == [[1, 0, 1, 0], [1, 1, 0, 0], [0, 0, 0, 0]]
    # equal scores: lower head first, then lower row
    is16, hp = O.calib_select_budget(np.ones((2, 3)), 4)
    assert is16.tolist() == [[1, 1, 1], [1, 0, 0]] and hp.tolist() == [3, 1]
    is16, hp = O.calib_select_budget(score, 0)
    assert not is16.any() and not hp.any()
    is16, hp = O.calib_select_budget(score, 12)
    assert is16.all() and hp.tolist() == [4, 4, 4]

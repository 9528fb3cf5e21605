"""GPU calibration against the calibration oracle.

Both sides run the same seeded FP32 recurrence (the FP32-format decode step,
bit-exact against the oracle elsewhere) and accumulate records after every
step.  Counts and retention sums are bit-exact (the same additions in the same
order); error energies agree to 1e-12 relative (the per-row sum order
differs); the selections are identical unless two scores tie to within 1e-9
relative, where either choice is correct.
"""
import numpy as np
import pytest
import torch

import oracle as O
import quantized_linear_attention_damp_b200 as D
import workloads as W
from tests.gpu_helpers import gate_of, torch_inputs

pytestmark = pytest.mark.gpu

CASES = {
    "kda_d128": W.WORKLOADS["kda"].with_(name="calib_kda", n=6, n_slots=9, H=4, steps=5),
    "gdn_d64": W.WORKLOADS["gdn_batch"].with_(name="calib_gdn", n=7, n_slots=7, H=3, d=64,
                                               hp=12, steps=6),
    "gdn_d16": W.WORKLOADS["tiny_gdn"].with_(name="calib_tiny", n=3, n_slots=4, H=2, steps=8),
    "kda_d32": W.WORKLOADS["kda"].with_(name="calib_kda32", n=5, n_slots=5, H=3, d=32, hp=6,
                                        steps=4, in_dtype="f32"),
}


def run_calibration(w):
    hs = W.head_structure(w.with_(fmt="fp32"))
    gpu = D.DampPool("fp32", w.n_slots, w.H, w.d)
    S0 = W.initial_state(w, range(w.n_slots))
    gpu.pack(torch.arange(w.n_slots, dtype=torch.int32, device="cuda"),
             torch.from_numpy(S0).cuda())
    ora = O.pack(O.FMT_FP32, np.zeros(w.d, np.uint8)[None], S0)
    acc_g = D.calib_acc(w.H, w.d)
    acc_o = O.calib_acc(w.H, w.d)
    is16 = np.zeros((w.H, w.d), np.uint8)
    out = torch.empty((w.n, w.H, w.d), dtype=torch.float32, device="cuda")
    for s in range(w.steps):
        x = W.step_inputs(w, s, hs)
        if s == 1:
            x.slot_idx[-1] = -1                     # padding entries are skipped
        t = torch_inputs(w, x)
        gpu.step(t["slot_idx"], t["q"], t["k"], t["v"], t["alpha"], t["beta"], out)
        D.damp_calib_accumulate(gpu.handle, t["slot_idx"], t["alpha"], acc_g)
        O.decode_step(ora, gate_of(w), is16, x.slot_idx, x.q, x.k, x.v, x.alpha, x.beta)
        O.calib_accumulate(acc_o, gate_of(w), ora.f32, x.slot_idx, x.alpha)
    torch.cuda.synchronize()
    assert gpu.get_error() == 0
    gpu.close()
    return acc_g, acc_o


def check_selection(sel_g, sel_o, score_o):
    for h in range(sel_g.shape[0]):
        a, b = set(sel_g[h].tolist()), set(sel_o[h].tolist())
        for i, j in zip(sorted(a - b), sorted(b - a)):
            assert abs(score_o[h, i] - score_o[h, j]) <= 1e-9 * abs(score_o[h, j]), (h, i, j)


@pytest.mark.parametrize("name", list(CASES))
def test_calibration_matches_oracle(name):
    w = CASES[name]
    acc_g, acc_o = run_calibration(w)
    g = acc_g.cpu().numpy()
    HD = w.H * w.d
    assert np.array_equal(g[2 * HD:], acc_o[2 * HD:])                       # counts
    assert np.array_equal(g[HD:2 * HD], acc_o[HD:2 * HD])                   # retention
    assert np.allclose(g[:HD], acc_o[:HD], rtol=1e-12, atol=0)             # energy
    assert acc_o[2 * HD:].tolist() == [float(w.n * w.steps - 1)] * w.H

    score_o = O.calib_scores(acc_o, w.H, w.d)
    sel_g, score_g = D.damp_calib_select(w.H, w.d, w.hp, acc_g)
    assert np.allclose(score_g.cpu().numpy(), score_o, rtol=1e-12, atol=0)
    sel_o = O.calib_select(score_o, w.hp)
    sel_g = sel_g.cpu().numpy().astype(np.uint16)
    assert (np.diff(sel_g.astype(np.int64), axis=1) > 0).all()
    check_selection(sel_g, sel_o, score_o)

    budget = w.hp * w.H
    is16_g, hp_g, _ = D.damp_calib_select_budget(w.H, w.d, budget, acc_g)
    is16_o, hp_o = O.calib_select_budget(score_o, budget)
    is16_g, hp_g = is16_g.cpu().numpy(), hp_g.cpu().numpy()
    assert is16_g.sum() == budget and np.array_equal(hp_g, is16_g.sum(axis=1))
    diff = np.argwhere(is16_g != is16_o)
    if len(diff):
        vals = score_o[tuple(diff.T)]
        assert np.ptp(vals) <= 1e-9 * np.abs(vals).max()


def test_calibrated_map_drives_a_mixed_pool():
    """The GPU's selection is a valid FP16-row map for damp_pool_create."""
    w = CASES["kda_d128"]
    acc_g, _ = run_calibration(w)
    sel, _ = D.damp_calib_select(w.H, w.d, w.hp, acc_g)
    pool = D.DampPool("mixed", w.n_slots, w.H, w.d, sel.cpu().numpy().astype(np.uint16))
    assert pool.hp == w.hp
    pool.close()


def test_out_of_range_slot_is_flagged_and_skipped():
    w = CASES["gdn_d16"]
    gpu = D.DampPool("fp32", w.n_slots, w.H, w.d)
    acc = D.calib_acc(w.H, w.d)
    slots = torch.tensor([0, w.n_slots + 2, -1, 1], dtype=torch.int32, device="cuda")
    alpha = torch.full((4, w.H), 0.5, dtype=torch.float32, device="cuda")
    D.damp_calib_accumulate(gpu.handle, slots, alpha, acc)
    torch.cuda.synchronize()
    a = acc.cpu().numpy()
    HD = w.H * w.d
    assert a[2 * HD:].tolist() == [2.0] * w.H
    assert np.all(a[HD:2 * HD] == 0.5)
    assert gpu.get_error(clear=True) == D.DAMP_EFLAG_SLOT_RANGE
    gpu.close()

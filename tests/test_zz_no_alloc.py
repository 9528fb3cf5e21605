"""The allocation-free budget selection (damp_calib_select_budget_static).

Some callers cannot allocate device memory when they pick the FP16 rows: a
serving process that has already handed every free byte of HBM to its state
pools, or a C host without an allocator that only holds the buffers it was
given.  For them the library keeps the ranking's scores in one static device
array instead of a caller buffer.  These tests call that entry point through
the C ABI and check that its selection equals the one of the entry point that
takes a score buffer, on two calls in a row of different sizes (the array
keeps the previous call's scores, which must not leak into the next), and
that a size beyond the array is refused before anything is enqueued.

This file is named to be collected last, so that a run stopping at the first
failure has run every other test first.
"""
import numpy as np
import pytest
import torch

import quantized_linear_attention_damp_b200 as D

pytestmark = pytest.mark.gpu


def _accumulator(H, d, seed, count=8.0):
    """A calibration accumulator (energy [H][d], retention [H][d], count [H])
    with scores over six decades, repeated values (ties) and rows that never
    decay (retention == count, the score's floor)."""
    g = np.random.default_rng(seed)
    energy = g.gamma(2.0, 1.0, (H, d)) * 10.0 ** g.uniform(-3, 3, (H, 1)) * count
    retention = g.uniform(0.0, 0.999, (H, d)) * count
    energy[0, :6] = energy[0, 6]
    retention[0, :6] = retention[0, 6]
    retention[1, :3] = count
    acc = np.concatenate([energy.ravel(), retention.ravel(), np.full(H, count)])
    return torch.from_numpy(acc).cuda()


@pytest.mark.parametrize("shapes", [((48, 128, 1296, 11), (32, 128, 864, 12)),
                                    ((16, 64, 200, 13), (128, 128, 3456, 14))])
def test_static_scratch_selection_matches_caller_buffer_selection(shapes):
    for H, d, budget, seed in shapes:      # two calls in a row
        acc = _accumulator(H, d, seed)
        is16_ref, hp_ref, _ = D.damp_calib_select_budget(H, d, budget, acc)
        is16 = torch.full((H, d), 7, dtype=torch.uint8, device="cuda")
        hp = torch.full((H,), -1, dtype=torch.int32, device="cuda")
        D.damp_calib_select_budget_static(H, d, budget, acc, is16, hp)
        torch.cuda.synchronize()
        assert torch.equal(is16, is16_ref)
        assert torch.equal(hp, hp_ref)
        assert int(is16.sum()) == budget


def test_static_scratch_refuses_sizes_beyond_the_array():
    H, d = D.DAMP_SELECT_BUDGET_STATIC_MAX // 128 + 1, 128
    acc = torch.zeros(D.damp_calib_bytes(H, d) // 8, dtype=torch.float64, device="cuda")
    is16 = torch.full((H, d), 7, dtype=torch.uint8, device="cuda")
    hp = torch.full((H,), -1, dtype=torch.int32, device="cuda")
    with pytest.raises(D.DampError) as ei:
        D.damp_calib_select_budget_static(H, d, 10, acc, is16, hp)
    assert ei.value.status == D.DAMP_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert bool((is16 == 7).all()) and bool((hp == -1).all())

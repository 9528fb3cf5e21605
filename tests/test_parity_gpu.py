"""GPU parity: the CUDA decode step (through the C ABI) against the oracle.

Every test drives libdamp through its Python binding (C-ABI marshalling
only) and the oracle from the same seeded inputs; each side keeps its own
state.  States are expected bit-exact (each rounding is taken in the same
precision and order on both sides); the asserted bar is the stated one:
readouts within 1e-4 relative / 1e-5 absolute, FP16 rows and scales within
1 ulp, INT8 codes within +-1 on at most 0.1 % of entries (FP8 E4M3 codes,
a comparison format with no stated bar, are held to the same).
"""
import numpy as np
import pytest
import torch

import oracle as O
import quantized_linear_attention_damp_b200 as D
import workloads as W
from tests.gpu_helpers import Pair, torch_inputs

pytestmark = pytest.mark.gpu

SMALL = {
    # d=16, 1 slot x 2 heads, GDN, fp32 inputs, 4 FP16 rows/head (the tiny workload)
    "tiny_gdn": W.WORKLOADS["tiny_gdn"],
    # d=16 KDA, batch a strict subset of the pool (padding-free gather), 6 units:
    # not a multiple of the 8 units a d=16 work item holds (ragged item)
    "tiny_kda": W.Workload("tiny_kda", n=3, n_slots=4, H=2, d=16, hp=4, steps=8,
                           gate=W.GATE_KDA, in_dtype="f32"),
    "d32_gdn_bf16": W.Workload("d32_gdn_bf16", n=5, n_slots=6, H=3, d=32, hp=5, steps=4,
                               gate=W.GATE_GDN, in_dtype="bf16"),
    "d64_kda_bf16": W.Workload("d64_kda_bf16", n=7, n_slots=7, H=3, d=64, hp=13, steps=4,
                               gate=W.GATE_KDA, in_dtype="bf16"),
    # d=128 with a ragged tail: 37 x 5 = 185 units over ~296 resident CTAs
    "d128_ragged": W.Workload("d128_ragged", n=37, n_slots=40, H=5, d=128, hp=27, steps=3,
                              gate=W.GATE_GDN, in_dtype="bf16"),
    "d128_kda_f32": W.Workload("d128_kda_f32", n=9, n_slots=9, H=4, d=128, hp=27, steps=3,
                               gate=W.GATE_KDA, in_dtype="f32"),
    # the other two (gate, input type) pairs of the d = 128 kernel, so that every
    # instantiation (row formats x gate x input type) runs
    "d128_kda_bf16": W.Workload("d128_kda_bf16", n=11, n_slots=12, H=3, d=128, hp=27, steps=3,
                                gate=W.GATE_KDA, in_dtype="bf16"),
    "d128_gdn_f32": W.Workload("d128_gdn_f32", n=10, n_slots=10, H=3, d=128, hp=27, steps=3,
                               gate=W.GATE_GDN, in_dtype="f32"),
}


def run_full(w, fmt, steps, fp16_map=None):
    p = Pair(w, fmt, fp16_map=fp16_map)
    try:
        rep = p.check_state()
        assert rep["exact"], rep            # pack parity
        for s in range(steps):
            x = W.step_inputs(w, s, p.hs)
            out_g = p.gpu_step(x)
            out_o = p.oracle_step_full(x)
            p.check_out(out_g, out_o)
            rep = p.check_state()
            assert rep["exact"], (s, rep)
        assert p.gpu.get_error() == 0
    finally:
        p.close()


def test_tiny_gdn_full_trajectory():
    """The tiny GDN workload: all 64 steps, whole state compared every step."""
    w = W.WORKLOADS["tiny_gdn"]
    run_full(w, "mixed", w.steps)


@pytest.mark.parametrize("name", list(SMALL))
@pytest.mark.parametrize("fmt", ["mixed", "int8", "fp8", "fp32"])
def test_small_shapes_all_formats(name, fmt):
    w = SMALL[name]
    run_full(w, fmt, min(w.steps, 8))


@pytest.mark.parametrize("hp", [0, 1, 16])
def test_tiny_extreme_fp16_row_counts(hp):
    """No FP16 row, one FP16 row, every row FP16 (block without scales)."""
    w = W.WORKLOADS["tiny_gdn"].with_(hp=hp, name=f"tiny_hp{hp}")
    run_full(w, "mixed", 8)


def test_all_fp16_rows_d128():
    w = W.Workload("d128_allfp16", n=6, n_slots=6, H=2, d=128, hp=128, steps=3,
                   gate=W.GATE_KDA, in_dtype="bf16")
    run_full(w, "mixed", 3)


def random_map(H, d, counts, seed):
    g = np.random.default_rng(seed)
    m = np.zeros((H, d), np.uint8)
    for h, c in enumerate(counts):
        m[h, g.permutation(d)[:c]] = 1
    return m


@pytest.mark.parametrize("name", ["tiny_kda", "d32_gdn_bf16", "d64_kda_bf16", "d128_ragged",
                                  "d128_kda_f32"])
def test_per_head_fp16_row_counts(name):
    """Heads with different FP16-row counts (incl. none and all rows) in one
    pool: per-head block layouts, per-head offsets inside a slot."""
    w = SMALL[name]
    base = [0, w.d, w.d // 3, 1, w.d - 1]
    counts = [base[h % len(base)] for h in range(w.H)]
    run_full(w, "mixed", min(w.steps, 4), fp16_map=random_map(w.H, w.d, counts, w.H * w.d))


def test_per_head_fp16_row_counts_unit_kernel():
    """d = 128 with every head's block small enough for the d = 128 kernel's
    stages (no all-FP16 head)."""
    w = SMALL["d128_ragged"].with_(name="d128_varhp", H=6)
    counts = [0, 27, 60, 1, 100, 27]
    run_full(w, "mixed", 3, fp16_map=random_map(w.H, w.d, counts, 77))


@pytest.mark.parametrize("name,steps", [("gdn_batch", 3), ("kda", 2)])
def test_full_size_whole_state(name, steps):
    """The 64x32 GDN and 128x32 KDA workloads at full size, every unit compared."""
    run_full(W.WORKLOADS[name], "mixed", steps)


@pytest.mark.parametrize("fmt", ["mixed", "int8", "fp8", "fp32"])
def test_high_concurrency_sampled_units(fmt):
    """512 slots x 48 heads at full size (the launch the benchmark times);
    sampled slots followed by the oracle over 4 steps."""
    w = W.WORKLOADS["hiconc_gdn"]
    slots = np.random.default_rng(5).choice(w.n_slots, 6, replace=False)
    p = Pair(w, fmt, oracle_slots=slots)
    try:
        assert p.check_state()["exact"]
        for s in range(4):
            x = W.step_inputs(w, s, p.hs)
            out_g = p.gpu_step(x)
            out_o = p.oracle_step(x)
            p.check_out(out_g, out_o)
            assert p.check_state()["exact"], s
        assert p.gpu.get_error() == 0
    finally:
        p.close()


def test_long_trajectory_sampled_units():
    """All 256 steps of the 64x32 GDN workload; 4 slots followed by the oracle."""
    w = W.WORKLOADS["gdn_batch"]
    p = Pair(w, "mixed", oracle_slots=[3, 17, 40, 63])
    try:
        for s in range(w.steps):
            x = W.step_inputs(w, s, p.hs)
            out_g = p.gpu_step(x)
            p.check_out(out_g, p.oracle_step(x))
            if s % 32 == 31:
                assert p.check_state()["exact"], s
        assert p.check_state()["exact"]
    finally:
        p.close()


def test_padding_and_out_of_range_slots():
    w = SMALL["d128_ragged"]
    p = Pair(w, "mixed")
    try:
        x = W.step_inputs(w, 0, p.hs)
        before = p.gpu.blocks().clone()
        x.slot_idx[:] = -1
        x.slot_idx[2] = 5
        x.slot_idx[4] = w.n_slots + 3         # out of range: flagged, skipped
        out_g = p.gpu_step(x)
        assert not out_g[[0, 1, 3] + list(range(5, w.n))].any()
        assert not out_g[4].any()
        assert p.gpu.get_error(clear=True) == D.DAMP_EFLAG_SLOT_RANGE
        assert p.gpu.get_error() == 0
        after = p.gpu.blocks()
        changed = (after != before).any(dim=-1)
        assert changed[5].all() and changed.sum() == w.H
        x.slot_idx[4] = -1
        out_o = p.oracle_step_full(x)
        p.check_out(out_g, out_o)
        assert p.check_state()["exact"]
    finally:
        p.close()


def test_identity_step_keeps_codes_on_gpu():
    """alpha = 1, beta = 0 at full size: requantizing the dequantized state
    leaves every code and FP16 value unchanged (scales within 1 ulp)."""
    w = W.WORKLOADS["gdn_batch"]
    p = Pair(w, "mixed", oracle_slots=[0])
    try:
        before = p.gpu.read_logical()
        x = W.step_inputs(w, 0, p.hs)
        x.alpha[:] = 1.0
        x.beta[:] = 0.0
        p.gpu_step(x)
        after = p.gpu.read_logical()
        assert np.array_equal(before["code"], after["code"])
        assert np.array_equal(before["half"], after["half"])
        ds = np.abs(before["scale"].view(np.int32).astype(np.int64)
                    - after["scale"].view(np.int32))
        assert ds.max() <= 1
    finally:
        p.close()


def test_delta_rule_write_invariant_on_gpu():
    """FP32 state, unit k (normalised in FP32 inputs), beta = alpha = 1: the
    step writes v along k, so k^T X = v^T to 1e-5 (relative to the state's
    size) for every unit of the batch."""
    w = W.Workload("inv_fp32", n=6, n_slots=8, H=4, d=128, hp=0, steps=1, gate=W.GATE_GDN,
                   in_dtype="f32")
    p = Pair(w, "fp32", oracle_slots=[0])
    try:
        x = W.step_inputs(w, 0, p.hs)
        k64 = x.k.astype(np.float64)
        x.k = (k64 / np.linalg.norm(k64, axis=-1, keepdims=True)).astype(np.float32)
        x.alpha[:] = 1.0
        x.beta[:] = 1.0
        S0 = p.gpu.read_logical()["f32"]
        p.gpu_step(x)
        X = p.gpu.read_logical()["f32"].astype(np.float64)
        for b, slot in enumerate(x.slot_idx):
            for h in range(w.H):
                kx = x.k[b, h].astype(np.float64) @ X[slot, h]
                bound = 1e-5 * max(1.0, float(np.abs(S0[slot, h]).max()))
                assert np.abs(kx - x.v[b, h]).max() <= bound, (b, h)
    finally:
        p.close()


def test_unpack_matches_oracle_reconstruction():
    w = SMALL["d64_kda_bf16"]
    p = Pair(w, "mixed")
    try:
        x = W.step_inputs(w, 0, p.hs)
        p.gpu_step(x)
        p.oracle_step_full(x)
        out = torch.empty((w.n_slots, w.H, w.d, w.d), dtype=torch.float32, device="cuda")
        p.gpu.unpack(torch.arange(w.n_slots, dtype=torch.int32, device="cuda"), out)
        ref = O.unpack(p.ora, p.is_fp16[None])
        assert np.array_equal(out.cpu().numpy().view(np.uint32), ref.view(np.uint32))
    finally:
        p.close()


def test_empty_batch_is_a_noop():
    w = SMALL["tiny_kda"]
    p = Pair(w, "mixed")
    try:
        before = p.gpu.blocks().clone()
        e = torch.empty(0, dtype=torch.int32, device="cuda")
        z = torch.empty((0, w.H, w.d), dtype=torch.float32, device="cuda")
        a = torch.empty((0, w.H, w.d), dtype=torch.float32, device="cuda")
        b = torch.empty((0, w.H), dtype=torch.float32, device="cuda")
        p.gpu.step(e, z, z, z, a, b, z)
        torch.cuda.synchronize()
        assert torch.equal(before, p.gpu.blocks())
    finally:
        p.close()


def test_argument_errors_enqueue_nothing():
    w = SMALL["tiny_kda"]
    p = Pair(w, "mixed")
    try:
        x = torch_inputs(w, W.step_inputs(w, 0, p.hs))
        out = torch.empty((w.n, w.H, w.d), dtype=torch.float32, device="cuda")
        before = p.gpu.blocks().clone()
        mis = torch.empty(w.n * w.H * w.d + 1, dtype=torch.float32, device="cuda")[1:]
        mis = mis.view(w.n, w.H, w.d)
        with pytest.raises(D.DampError) as ei:
            p.gpu.step(x["slot_idx"], mis, x["k"], x["v"], x["alpha"], x["beta"], out)
        assert ei.value.status == D.DAMP_ERR_MISALIGNED
        torch.cuda.synchronize()
        assert torch.equal(before, p.gpu.blocks())
    finally:
        p.close()


# ---------------------------------------------------------------- every shape

SHAPES = [(48, 48), (96, 96), (256, 256), (64, 128), (128, 64), (48, 80), (256, 32), (32, 256),
          (112, 144)]


@pytest.mark.parametrize("dk,dv", SHAPES)
@pytest.mark.parametrize("fmt", ["mixed", "int8", "fp8", "fp32"])
def test_every_shape_all_formats(dk, dv, fmt):
    """d_k x d_v states outside the square fast shapes (one CTA per unit):
    whole state bit-exact and readout within tolerance at every step, GDN and
    KDA, bf16 and fp32 inputs, a ragged batch (not every slot stepped)."""
    i = SHAPES.index((dk, dv))
    w = W.Workload(f"shape_{dk}x{dv}", n=5, n_slots=6, H=3, d=dk, dv=dv, hp=max(1, dk // 5),
                   steps=3, gate=W.GATE_KDA if i % 2 else W.GATE_GDN,
                   in_dtype="f32" if i % 3 == 2 else "bf16")
    run_full(w, fmt, 3)


@pytest.mark.parametrize("dk,dv", [(48, 80), (256, 256)])
def test_every_shape_per_head_fp16_row_counts(dk, dv):
    w = W.Workload(f"shape_map_{dk}x{dv}", n=4, n_slots=5, H=5, d=dk, dv=dv, hp=0, steps=2,
                   gate=W.GATE_GDN, in_dtype="bf16")
    counts = [0, dk, dk // 3, 1, dk - 1]
    run_full(w, "mixed", 2, fp16_map=random_map(w.H, dk, counts, dk + dv))


def test_every_shape_unpack_and_read_raw():
    """Unpack of a non-square pool equals the oracle's reconstruction, and
    damp_pool_read_raw returns each block's logical form."""
    w = W.Workload("shape_unpack", n=4, n_slots=4, H=2, d=96, dv=160, hp=20, steps=1,
                   gate=W.GATE_GDN, in_dtype="bf16")
    p = Pair(w, "mixed")
    try:
        x = W.step_inputs(w, 0, p.hs)
        p.gpu_step(x)
        p.oracle_step_full(x)
        out = torch.empty((w.n_slots, w.H, w.d, w.d_v), dtype=torch.float32, device="cuda")
        p.gpu.unpack(torch.arange(w.n_slots, dtype=torch.int32, device="cuda"), out)
        ref = O.unpack(p.ora, p.is_fp16[None])
        assert np.array_equal(out.cpu().numpy().view(np.uint32), ref.view(np.uint32))
        for s in range(w.n_slots):
            for h in range(w.H):
                lg = D.damp_pool_read_raw(p.gpu.handle, s, h)
                assert np.array_equal(lg["code"], p.ora.code[s, h])
                assert np.array_equal(lg["half"], p.ora.half[s, h])
                assert np.array_equal(lg["scale"].view(np.uint32), p.ora.scale[s, h].view(np.uint32))
    finally:
        p.close()


@pytest.mark.parametrize("gate", [W.GATE_GDN, W.GATE_KDA])
def test_sharded_pools_match_one_pool(gate):
    """The data-parallel split a multi-GPU run uses, on one GPU: two pools
    holding alternate slots of a workload, each stepped with its own entries
    of the batch, give bit for bit the out rows and the states of one pool
    holding every slot (units are independent; no exchange is needed)."""
    w = W.Workload(f"shard_{gate}", n=8, n_slots=8, H=4, d=128, hp=27, steps=3, gate=gate,
                   in_dtype="bf16")
    hs = W.head_structure(w)
    S0 = torch.from_numpy(W.initial_state(w, range(w.n_slots))).cuda()
    whole = D.DampPool("mixed", w.n_slots, w.H, w.d, hs.hp_row_idx)
    whole.pack(torch.arange(w.n_slots, dtype=torch.int32, device="cuda"), S0)
    owned = [list(range(r, w.n_slots, 2)) for r in range(2)]
    shards = []
    for mine in owned:
        p = D.DampPool("mixed", len(mine), w.H, w.d, hs.hp_row_idx)
        p.pack(torch.arange(len(mine), dtype=torch.int32, device="cuda"),
               S0[torch.tensor(mine, device="cuda")].contiguous())
        shards.append(p)
    try:
        for s in range(w.steps):
            x = W.step_inputs(w, s, hs)
            t = torch_inputs(w, x)
            out = torch.empty((w.n, w.H, w.d), dtype=torch.float32, device="cuda")
            whole.step(t["slot_idx"], t["q"], t["k"], t["v"], t["alpha"], t["beta"], out)
            out_sh = torch.full_like(out, float("nan"))
            for mine, p in zip(owned, shards):
                sel = [b for b in range(w.n) if int(x.slot_idx[b]) in mine]
                ib = torch.tensor(sel, device="cuda")
                local = torch.tensor([mine.index(int(x.slot_idx[b])) for b in sel],
                                     dtype=torch.int32, device="cuda")
                o = torch.empty((len(sel), w.H, w.d), dtype=torch.float32, device="cuda")
                p.step(local, t["q"][ib].contiguous(), t["k"][ib].contiguous(),
                       t["v"][ib].contiguous(), t["alpha"][ib].contiguous(),
                       t["beta"][ib].contiguous(), o)
                out_sh[ib] = o
            torch.cuda.synchronize()
            assert torch.equal(out, out_sh), s
        # the states, compared in their logical form (a block's 16-byte padding
        # is never written and holds whatever each buffer held)
        for mine, p in zip(owned, shards):
            lw, ls = whole.read_logical(mine), p.read_logical()
            for f in ("scale", "half", "code"):
                assert np.array_equal(lw[f], ls[f]), f
    finally:
        whole.close()
        for p in shards:
            p.close()


@pytest.mark.parametrize("fmt", ["mixed", "int8"])
def test_back_to_back_steps_same_pool(fmt):
    """Consecutive steps on one pool launched with no host synchronisation in
    between (each launch a programmatic dependent of the previous one, which
    reads the blocks the previous one writes): after all of them, the state and
    every step's readout equal the oracle's, bit for bit and within tolerance.
    The batches repeat slots from step to step, so each step depends on the
    last one's write-back."""
    w = W.Workload("b2b_d128", n=40, n_slots=44, H=4, d=128, hp=27, steps=6,
                   gate=W.GATE_GDN, in_dtype="bf16")
    p = Pair(w, fmt)
    try:
        xs = [W.step_inputs(w, s, p.hs) for s in range(w.steps)]
        ts = [torch_inputs(w, x) for x in xs]
        outs = [torch.empty((w.n, w.H, w.d_v), dtype=torch.float32, device="cuda")
                for _ in range(w.steps)]
        torch.cuda.synchronize()
        for t, o in zip(ts, outs):
            p.gpu.step(t["slot_idx"], t["q"], t["k"], t["v"], t["alpha"], t["beta"], o)
        torch.cuda.synchronize()
        for x, o in zip(xs, outs):
            p.check_out(o.cpu().numpy(), p.oracle_step_full(x))
        rep = p.check_state()
        assert rep["exact"], rep
        assert p.gpu.get_error() == 0
    finally:
        p.close()

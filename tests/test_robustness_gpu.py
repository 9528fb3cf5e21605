"""GPU robustness checks: canary bytes around the pool buffer and the output,
and checkpoint / resume of a pool (raw bytes, and unpack -> pack)."""
import io

import numpy as np
import pytest
import torch

import quantized_linear_attention_damp_b200 as D
import workloads as W
from tests.gpu_helpers import torch_inputs

pytestmark = pytest.mark.gpu

CANARY = 0xA5


def _step(pool_handle, w, x, out):
    t = torch_inputs(w, x)
    D.damp_decode_step(pool_handle, t["slot_idx"], t["q"], t["k"], t["v"], t["alpha"],
                       t["beta"], out)


@pytest.mark.parametrize("fmt,gate", [("mixed", W.GATE_GDN), ("mixed", W.GATE_KDA),
                                      ("fp8", W.GATE_GDN), ("fp32", W.GATE_GDN)])
def test_canaries_around_pool_and_output(fmt, gate):
    """Nothing is written past the end of the pool buffer or of `out`."""
    w = W.Workload("canary", n=9, n_slots=11, H=3, d=128, hp=27, steps=3, gate=gate,
                   in_dtype="bf16")
    hs = W.head_structure(w.with_(fmt=fmt))
    f = D.FORMATS[fmt]
    hp = w.hp if fmt == "mixed" else 0
    nbytes = D.damp_pool_bytes(f, w.n_slots, w.H, w.d, w.d, hp)
    big = torch.full((nbytes + 4096,), CANARY, dtype=torch.uint8, device="cuda")
    h = D.damp_pool_create(f, w.n_slots, w.H, w.d, w.d, hp,
                           hs.hp_row_idx if fmt == "mixed" else None, big[:nbytes])
    try:
        S0 = torch.from_numpy(W.initial_state(w, range(w.n_slots))).cuda()
        D.damp_pool_pack(h, torch.arange(w.n_slots, dtype=torch.int32, device="cuda"), S0)
        n_out = w.n * w.H * w.d
        out_big = torch.full((n_out + 1024,), -7.5, dtype=torch.float32, device="cuda")
        out = out_big[:n_out].view(w.n, w.H, w.d)
        for s in range(w.steps):
            _step(h, w, W.step_inputs(w, s, hs), out)
        back = torch.empty_like(S0)
        D.damp_pool_unpack(h, torch.arange(w.n_slots, dtype=torch.int32, device="cuda"), back)
        torch.cuda.synchronize()
        assert bool((big[nbytes:] == CANARY).all())
        assert bool((out_big[n_out:] == -7.5).all())
        assert torch.isfinite(back).all()
        assert D.damp_pool_get_error(h, device=big.device) == 0
    finally:
        D.damp_pool_destroy(h)


def test_checkpoint_and_resume():
    """A pool saved as raw bytes (torch.save of its buffer) and restored into a
    new descriptor continues bit for bit; a pool rebuilt by unpack -> pack holds
    the same logical state."""
    w = W.WORKLOADS["kda"].with_(name="ckpt", n=16, n_slots=20, H=4, steps=6)
    hs = W.head_structure(w)
    a = D.DampPool("mixed", w.n_slots, w.H, w.d, hs.hp_row_idx)
    ident = torch.arange(w.n_slots, dtype=torch.int32, device="cuda")
    a.pack(ident, torch.from_numpy(W.initial_state(w, range(w.n_slots))).cuda())
    out_a = torch.empty((w.n, w.H, w.d), dtype=torch.float32, device="cuda")
    out_b = torch.empty_like(out_a)
    for s in range(3):
        _step(a.handle, w, W.step_inputs(w, s, hs), out_a)
    torch.cuda.synchronize()
    blob = io.BytesIO()
    torch.save(a.buf.cpu(), blob)
    blob.seek(0)
    b = D.DampPool("mixed", w.n_slots, w.H, w.d, hs.hp_row_idx)
    b.buf.copy_(torch.load(blob).cuda())
    for s in range(3, w.steps):
        x = W.step_inputs(w, s, hs)
        _step(a.handle, w, x, out_a)
        _step(b.handle, w, x, out_b)
        torch.cuda.synchronize()
        assert torch.equal(out_a, out_b)
    assert torch.equal(a.slots(), b.slots())
    # resume through the FP32 form: unpack -> pack reproduces the logical state
    S = torch.empty((w.n_slots, w.H, w.d, w.d), dtype=torch.float32, device="cuda")
    a.unpack(ident, S)
    c = D.DampPool("mixed", w.n_slots, w.H, w.d, hs.hp_row_idx)
    c.pack(ident, S)
    la, lc = a.read_logical(), c.read_logical()
    assert np.array_equal(la["code"], lc["code"]) and np.array_equal(la["half"], lc["half"])
    ds = np.abs(la["scale"].view(np.int32).astype(np.int64) - lc["scale"].view(np.int32))
    assert ds.max() <= 1
    for p in (a, b, c):
        p.close()


# ---------------------------------------------------------------- failure paths

def _small(d, gate=W.GATE_GDN, in_dtype=None):
    return W.Workload(f"fail_d{d}_{gate}", n=6, n_slots=8, H=3, d=d, hp=d // 5, steps=2,
                      gate=gate, in_dtype=in_dtype or ("f32" if d == 16 else "bf16"))


@pytest.mark.parametrize("d,fmt", [(16, "mixed"), (128, "mixed"), (128, "fp8"), (128, "fp32")])
def test_bounded_wait_runs_out_and_the_kernel_returns(d, fmt):
    """A pipeline wait that runs out, made on purpose: with
    DAMP_HOOK_HOLD_FIRST_ITEM every CTA leaves its first item unloaded, and the
    wait for it is bounded at 5 ms.  The kernel sets DAMP_EFLAG_TIMEOUT, waits
    (bounded) for its other copies in flight and returns: the stream drains,
    no block is written, and the next normal steps on the same pool match the
    oracle bit for bit (the context stays usable)."""
    import time

    from tests.gpu_helpers import Pair
    w = _small(d)
    p = Pair(w, fmt)
    try:
        x = W.step_inputs(w, 0, p.hs)
        before = p.gpu.slots().clone()
        D.damp_set_test_hooks(5_000_000, D.DAMP_HOOK_HOLD_FIRST_ITEM)
        try:
            t0 = time.time()
            p.gpu_step(x)                      # synchronises
            elapsed = time.time() - t0
        finally:
            D.damp_set_test_hooks(0, 0)
        assert elapsed < 5.0
        assert p.gpu.get_error(clear=True) == D.DAMP_EFLAG_TIMEOUT
        assert p.gpu.get_error() == 0
        assert torch.equal(before, p.gpu.slots())
        for s in range(2):
            x = W.step_inputs(w, s, p.hs)
            p.check_out(p.gpu_step(x), p.oracle_step_full(x))
            assert p.check_state()["exact"], s
        assert p.gpu.get_error() == 0
    finally:
        p.close()


def _plant(x, name, b, h, j, value):
    """Set one input element (its float value and, for bf16 inputs, its bits)."""
    arr = getattr(x, name)
    if name in ("alpha", "beta"):
        arr[(b, h) if arr.ndim == 2 else (b, h, j)] = value
        return
    arr[b, h, j] = value
    bits = getattr(x, name + "_bits")
    if bits is not None:
        bits[b, h, j] = np.float32(value).view(np.uint32) >> 16


@pytest.mark.parametrize("d,fmt,gate", [(16, "mixed", W.GATE_GDN), (16, "int8", W.GATE_KDA),
                                        (128, "mixed", W.GATE_GDN), (128, "mixed", W.GATE_KDA),
                                        (128, "fp8", W.GATE_GDN), (128, "fp32", W.GATE_KDA)])
def test_nonfinite_inputs_are_skipped_and_flagged(d, fmt, gate):
    """damp_decode_step_validated: units whose q, k, v, alpha or beta hold a
    NaN or an infinity are skipped (out row zero, block untouched) and flagged
    with DAMP_EFLAG_NONFINITE; every other unit is stepped exactly as the
    oracle steps it.  The plain step on clean inputs sets no flag."""
    from tests.gpu_helpers import Pair
    w = _small(d, gate)
    p = Pair(w, fmt)
    try:
        x = W.step_inputs(w, 0, p.hs)
        bad = {(1, 0): ("q", 3, np.nan), (2, 1): ("v", d - 1, np.inf), (0, 2): ("beta", 0, np.nan),
               (3, 0): ("alpha", 5, np.inf), (4, 1): ("k", 0, -np.inf)}
        for (b, h), (name, j, val) in bad.items():
            _plant(x, name, b, h, j, val)
        t = torch_inputs(w, x)
        out = torch.full((w.n, w.H, w.d), 3.0, dtype=torch.float32, device="cuda")
        p.gpu.step(t["slot_idx"], t["q"], t["k"], t["v"], t["alpha"], t["beta"], out,
                   check_inputs=True)
        out_g = out.cpu().numpy()
        # the oracle steps the clean units only
        res = {}
        gate_o = 1 if gate == W.GATE_KDA else 0
        for b, slot in enumerate(x.slot_idx):
            for h in range(w.H):
                if (b, h) in bad:
                    assert not out_g[b, h].any()
                    continue
                st = p.ora[int(slot), h]
                import oracle as O
                res[(b, h)] = O.step_unit(st, gate_o, p.is_fp16[h], x.q[b, h], x.k[b, h],
                                          x.v[b, h], x.alpha[b, h], x.beta[b, h])
        p.check_out(out_g, res)
        assert p.check_state()["exact"]
        assert p.gpu.get_error(clear=True) == D.DAMP_EFLAG_NONFINITE
        x2 = W.step_inputs(w, 1, p.hs)
        p.check_out(p.gpu_step(x2), p.oracle_step_full(x2))
        assert p.check_state()["exact"]
        assert p.gpu.get_error() == 0
    finally:
        p.close()

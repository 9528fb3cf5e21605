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

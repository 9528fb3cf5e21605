"""Serving-shaped slot pool on the GPU: 4096-slot mixed pools, 32 heads, d = 128,
a random 1024-slot subset per step, a GDN layer and a KDA layer stepped by one
captured CUDA graph.

Checks: the graph replay and plain launches give bit-identical pools and
outputs; slots followed by the oracle (picked among those updated in both
steps, in one step only, and in neither) match it bit for bit; slots outside
the subset are left untouched.
"""
import numpy as np
import pytest
import torch

import oracle as O
import quantized_linear_attention_damp_b200 as D
import workloads as W
from quantized_linear_attention_damp_b200.graph import DecodeGraph
from tests.gpu_helpers import ATOL_OUT, RTOL_OUT, gate_of, torch_inputs

pytestmark = pytest.mark.gpu

LAYERS = (2, 3)          # layer 3 is a KDA layer (index 3 mod 4), layer 2 a GDN layer
STEPS = 2


def build_layer(layer: int):
    w = W.serving_layer(layer)
    hs = W.head_structure(w)
    pool = D.DampPool("mixed", w.n_slots, w.H, w.d, hs.hp_row_idx)
    T = W.serving_templates(w)
    nt = W.SERVING_TEMPLATES
    pool.pack(torch.arange(nt, dtype=torch.int32, device="cuda"), torch.from_numpy(T).cuda())
    b = pool.blocks()
    groups = w.n_slots // nt
    b.view(groups, nt, w.H, -1)[1:].copy_(b[:nt].unsqueeze(0).expand(groups - 1, -1, -1, -1))
    pool.templates = b[:nt].clone()
    return w, hs, pool, T


def static_args(w: W.Workload):
    dt = torch.bfloat16
    shape = (w.n, w.H, w.d)
    a_shape = shape if w.gate == W.GATE_KDA else (w.n, w.H)
    return dict(slot_idx=torch.empty(w.n, dtype=torch.int32, device="cuda"),
                q=torch.empty(shape, dtype=dt, device="cuda"),
                k=torch.empty(shape, dtype=dt, device="cuda"),
                v=torch.empty(shape, dtype=dt, device="cuda"),
                alpha=torch.empty(a_shape, dtype=torch.float32, device="cuda"),
                beta=torch.empty((w.n, w.H), dtype=torch.float32, device="cuda"),
                out=torch.empty(shape, dtype=torch.float32, device="cuda"))


def logical(pool, slots):
    raw = pool.blocks()[torch.as_tensor(slots, device="cuda")].cpu().numpy()
    res = {"half": [], "scale": [], "code": []}
    for i in range(len(slots)):
        per = [D.damp_block_to_logical(pool.handle, h, raw[i, h], pool.fmt, pool.d)
               for h in range(pool.H)]
        for key in res:
            res[key].append(np.stack([p[key] for p in per]))
    return {k: np.stack(v) for k, v in res.items()}


def test_serving_pool_graph_matches_plain_and_oracle():
    free, _ = torch.cuda.mem_get_info()
    need = 2 * len(LAYERS) * D.damp_pool_bytes(D.DAMP_FMT_MIXED, 4096, 32, 128, 128, 27)
    if free < need + (4 << 30):
        pytest.skip("not enough device memory for two copies of the test pools")

    layers = [build_layer(l) for l in LAYERS]
    plain = []
    for w, hs, pool, _ in layers:
        twin = D.DampPool("mixed", w.n_slots, w.H, w.d, hs.hp_row_idx)
        twin.buf.copy_(pool.buf)
        plain.append(twin)
    args = [static_args(w) for w, *_ in layers]
    graph = DecodeGraph([(pool, a) for (_, _, pool, _), a in zip(layers, args)])
    torch.cuda.synchronize()

    # slots followed by the oracle
    s0 = set(W.serving_slot_idx(0).tolist())
    s1 = set(W.serving_slot_idx(1).tolist())
    g = np.random.default_rng(11)
    pick = lambda pool_: sorted(g.choice(sorted(pool_), 3, replace=False).tolist())
    every = set(range(4096))
    follow = pick(s0 & s1) + pick(s0 - s1) + pick(s1 - s0) + pick(every - s0 - s1)
    ora = []
    for w, hs, _, T in layers:
        ora.append(O.pack(O.FMT_QUANT, hs.is_fp16[None],
                          T[[s % W.SERVING_TEMPLATES for s in follow]]))
    pos = {s: i for i, s in enumerate(follow)}

    for step in range(STEPS):
        xs = [W.serving_step_inputs(w, step, hs) for w, hs, _, _ in layers]
        outs_plain = []
        for (w, hs, pool, _), x, a, twin in zip(layers, xs, args, plain):
            t = torch_inputs(w, x)
            for key in t:
                a[key].copy_(t[key])
            out = torch.empty_like(a["out"])
            twin.step(t["slot_idx"], t["q"], t["k"], t["v"], t["alpha"], t["beta"], out)
            outs_plain.append(out)
        graph.replay()
        torch.cuda.synchronize()
        for (w, hs, pool, _), x, a, twin, o_plain, st in zip(layers, xs, args, plain,
                                                             outs_plain, ora):
            assert torch.equal(a["out"], o_plain)
            assert torch.equal(pool.buf, twin.buf)
            out = a["out"].cpu().numpy()
            gate = gate_of(w)
            for b, slot in enumerate(x.slot_idx):
                i = pos.get(int(slot))
                if i is None:
                    continue
                for h in range(w.H):
                    o = O.step_unit(st[i, h], gate, hs.is_fp16[h], x.q[b, h], x.k[b, h],
                                    x.v[b, h], x.alpha[b, h], x.beta[b, h])
                    err = np.abs(out[b, h].astype(np.float64) - o)
                    assert (err <= ATOL_OUT + RTOL_OUT * np.abs(o)).all(), (step, slot, h)

    for (w, hs, pool, T), st in zip(layers, ora):
        lg = logical(pool, follow)
        assert np.array_equal(lg["half"], st.half)
        assert np.array_equal(lg["scale"].view(np.uint32), st.scale.view(np.uint32))
        assert np.array_equal(lg["code"], st.code)
        # slots in neither subset still hold their template's block
        untouched = [s for s in follow if s not in s0 and s not in s1]
        blocks = pool.blocks()
        for s in untouched:
            assert torch.equal(blocks[s], pool.templates[s % W.SERVING_TEMPLATES])
        assert pool.get_error() == 0
    graph.reset()
    for _, _, pool, _ in layers:
        pool.close()
    for twin in plain:
        twin.close()

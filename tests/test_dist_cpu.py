"""Multi-rank host logic on CPU (gloo, world size 2).

The decode step has no exchange: units are independent, so ranks step
disjoint shards of slots and only the timing is reduced (max over ranks).
These tests run two gloo ranks that each step their shard with the oracle
and check that the gathered result equals the unsharded run, and that the
timing reduction bench.py uses returns the max.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle as O
import workloads as W

WORLD = 2


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, port, result_q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=WORLD)
    try:
        import bench
        w = W.Workload("shard", n=4, n_slots=4, H=2, d=16, hp=4, steps=3,
                       gate=W.GATE_KDA, in_dtype="f32")
        hs = W.head_structure(w)
        S0 = W.initial_state(w, range(w.n_slots))
        # rank r owns slots {r, r + WORLD, ...}
        mine = list(range(rank, w.n_slots, WORLD))
        pool = O.pack(O.FMT_QUANT, hs.is_fp16[None], S0[mine])
        outs = []
        for s in range(w.steps):
            x = W.step_inputs(w, s, hs)
            sel = [b for b in range(w.n) if int(x.slot_idx[b]) in mine]
            local_idx = np.array([mine.index(int(x.slot_idx[b])) for b in sel], np.int32)
            o = O.decode_step(pool, O.GATE_VECTOR, hs.is_fp16, local_idx, x.q[sel], x.k[sel],
                              x.v[sel], x.alpha[sel], x.beta[sel])
            full = np.zeros((w.n, w.H, w.d))
            full[sel] = o
            outs.append(torch.from_numpy(full))
        out = torch.stack(outs)
        dist.all_reduce(out)          # disjoint shards: the sum is the concatenation
        # the rank's shard in libdamp's own block layout (host-only descriptor):
        # raw slot bytes encoded from the rank's logical state, gathered by slot
        import quantized_linear_attention_damp_b200 as D
        hd = D.damp_pool_create(D.DAMP_FMT_MIXED, len(mine), w.H, w.d, w.d, w.hp, hs.hp_row_idx,
                                None)
        try:
            _, stride = D.damp_layout(D.DAMP_FMT_MIXED, w.d, w.d, w.hp)
            raw = torch.zeros((w.n_slots, w.H, stride), dtype=torch.int32)
            for i, slot in enumerate(mine):
                for h in range(w.H):
                    blk = D.damp_block_from_logical(hd, h, stride, scale=pool.scale[i, h],
                                                    half=pool.half[i, h], code=pool.code[i, h])
                    raw[slot, h] = torch.from_numpy(blk.astype(np.int32))
        finally:
            D.damp_pool_destroy(hd)
        dist.all_reduce(raw)
        state = torch.zeros((w.n_slots, w.H, w.d, w.d), dtype=torch.int32)
        state[mine] = torch.from_numpy(pool.code.astype(np.int32))
        dist.all_reduce(state)
        t = bench.max_over_ranks(0.5 + rank, WORLD)
        if rank == 0:
            result_q.put((out.numpy(), state.numpy(), t, raw.numpy()))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_match_unsharded_oracle():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, port, q)) for r in range(WORLD)]
    for p in procs:
        p.start()
    out, codes, t, raw = q.get(timeout=240)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # unsharded reference on one process
    w = W.Workload("shard", n=4, n_slots=4, H=2, d=16, hp=4, steps=3,
                   gate=W.GATE_KDA, in_dtype="f32")
    hs = W.head_structure(w)
    pool = O.pack(O.FMT_QUANT, hs.is_fp16[None], W.initial_state(w, range(w.n_slots)))
    for s in range(w.steps):
        x = W.step_inputs(w, s, hs)
        o = O.decode_step(pool, O.GATE_VECTOR, hs.is_fp16, x.slot_idx, x.q, x.k, x.v,
                          x.alpha, x.beta)
        assert np.array_equal(out[s], o)
    assert np.array_equal(codes, pool.code.astype(np.int32))
    assert t == pytest.approx(1.5)
    # the gathered raw shards are the unsharded pool's blocks, byte for byte
    import quantized_linear_attention_damp_b200 as D
    hd = D.damp_pool_create(D.DAMP_FMT_MIXED, w.n_slots, w.H, w.d, w.d, w.hp, hs.hp_row_idx, None)
    try:
        _, stride = D.damp_layout(D.DAMP_FMT_MIXED, w.d, w.d, w.hp)
        for slot in range(w.n_slots):
            for h in range(w.H):
                blk = D.damp_block_from_logical(hd, h, stride, scale=pool.scale[slot, h],
                                                half=pool.half[slot, h], code=pool.code[slot, h])
                assert np.array_equal(raw[slot, h].astype(np.uint8), blk)
    finally:
        D.damp_pool_destroy(hd)


def test_rank_workloads_differ_only_in_seed():
    import bench
    a, b = bench.rank_workload("gdn_batch", 0), bench.rank_workload("gdn_batch", 1)
    assert (a.n, a.H, a.d, a.hp) == (b.n, b.H, b.d, b.hp) and a.seed != b.seed
    assert not np.array_equal(W.initial_state(a, [0]), W.initial_state(b, [0]))

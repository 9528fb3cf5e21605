"""CPU checks of the C ABI: exported symbols, layout, host-side validation and
block conversions.  No kernel is launched (no GPU needed)."""
import ctypes
import os
import re

import numpy as np
import pytest

import quantized_linear_attention_damp_b200 as D
from tests.conftest import ROOT

HEADER = os.path.join(ROOT, "include", "damp.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(damp_[a-z_]+)\s*\(", src)))


def test_library_exports_every_declared_function():
    names = declared_functions()
    assert len(names) >= 12
    lib = ctypes.CDLL(D.LIB_PATH)
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing


def test_binding_has_the_same_names():
    for n in declared_functions():
        assert callable(getattr(D, n)), n


def _golden():
    vals = {}
    for line in open(os.path.join(ROOT, "tests", "golden", "format_accounting.txt")):
        line = line.split("#")[0].split()
        if len(line) == 2:
            vals[line[0]] = float(line[1])
    return vals


def test_format_accounting_matches_published_figures():
    """27 FP16 rows + 101 INT8 rows + 101 FP32 scales at d = 128 give 9.885
    bits/value (printed as 9.9) and 69.11 % less than FP32 (printed 69.1 %)."""
    g = _golden()
    d = int(g["d_k"])
    block, stride = D.damp_layout(D.DAMP_FMT_MIXED, d, d, 27)
    assert block == 20244 and stride == 20256
    bits = block * 8 / (d * d)
    assert round(bits, 1) == g["bits_per_value"]
    assert round(100 * (1 - bits / 32), 1) == g["storage_reduction_percent"]
    # 27 is the only FP16-row count that prints both figures
    hits = []
    for hp in range(0, d + 1):
        b = D.damp_layout(D.DAMP_FMT_MIXED, d, d, hp)[0] * 8 / (d * d)
        if round(b, 1) == g["bits_per_value"] and \
                round(100 * (1 - b / 32), 1) == g["storage_reduction_percent"]:
            hits.append(hp)
    assert hits == [27]
    # FP16 scales would not reproduce the figures (they give 9.8 bits)
    b16 = (27 * d * 16 + 101 * d * 8 + 101 * 16) / (d * d)
    assert round(b16, 1) != g["bits_per_value"]


def test_layouts_of_other_formats():
    assert D.damp_layout(D.DAMP_FMT_FP32, 128, 128, 0) == (65536, 65536)
    assert D.damp_layout(D.DAMP_FMT_INT8_ROW, 128, 128, 0) == (16896, 16896)
    assert D.damp_layout(D.DAMP_FMT_FP8_ROW, 128, 128, 0) == (16896, 16896)
    assert D.damp_layout(D.DAMP_FMT_MIXED, 128, 128, 0) == (16896, 16896)
    assert D.damp_layout(D.DAMP_FMT_MIXED, 128, 128, 128) == (32768, 32768)
    assert D.damp_layout(D.DAMP_FMT_MIXED, 16, 16, 4) == (368, 368)
    for d in (16, 32, 64, 128):
        for hp in range(d + 1):
            b, s = D.damp_layout(D.DAMP_FMT_MIXED, d, d, hp)
            assert s % 16 == 0 and b <= s < b + 16 + 16


def test_pool_bytes():
    n = D.damp_pool_bytes(D.DAMP_FMT_MIXED, 64, 32, 128, 128, 27)
    # status word; per head a 32-byte FP16-row mask, a 4*d_k-byte row
    # directory and a 16-byte block-table entry; rounded up to 256 bytes
    hdr = 256 * ((16 + 32 * 32 + 32 * 512 + 32 * 16 + 255) // 256)
    assert n == hdr + 64 * 32 * 20256
    n = D.damp_pool_bytes(D.DAMP_FMT_MIXED, 3, 5, 256, 48, 9)
    hdr = 256 * ((16 + 5 * 32 + 5 * 1024 + 5 * 16 + 255) // 256)
    r = 256 - 9
    stride = 16 * ((16 * ((4 * r + 15) // 16) + 2 * 9 * 48 + r * 48 + 15) // 16)
    assert n == hdr + 3 * 5 * stride


@pytest.mark.parametrize("args,status", [
    ((4, 128, 128, 0), D.DAMP_ERR_INVALID_ARGUMENT),         # bad format
    ((D.DAMP_FMT_FP8_ROW, 128, 128, 2), D.DAMP_ERR_INVALID_ARGUMENT),
    ((D.DAMP_FMT_MIXED, 128, 128, 129), D.DAMP_ERR_INVALID_ARGUMENT),
    ((D.DAMP_FMT_MIXED, 128, 128, -1), D.DAMP_ERR_INVALID_ARGUMENT),
    ((D.DAMP_FMT_INT8_ROW, 128, 128, 3), D.DAMP_ERR_INVALID_ARGUMENT),
    ((D.DAMP_FMT_FP32, 128, 128, 1), D.DAMP_ERR_INVALID_ARGUMENT),
    ((D.DAMP_FMT_MIXED, 128, 120, 0), D.DAMP_ERR_UNSUPPORTED),    # d_v not a multiple of 16
    ((D.DAMP_FMT_MIXED, 8, 8, 0), D.DAMP_ERR_UNSUPPORTED),
    ((D.DAMP_FMT_MIXED, 272, 272, 0), D.DAMP_ERR_UNSUPPORTED),
    ((D.DAMP_FMT_FP32, 128, 264, 0), D.DAMP_ERR_UNSUPPORTED),
    ((D.DAMP_FMT_INT8_ROW, 0, 128, 0), D.DAMP_ERR_UNSUPPORTED),
])
def test_layout_rejects_bad_shapes(args, status):
    with pytest.raises(D.DampError) as ei:
        D.damp_layout(*args)
    assert ei.value.status == status


def test_layout_accepts_every_supported_shape():
    """d_k, d_v in {16, 32, ..., 256}, square or not: block sizes from the
    format's definition (FP32: 4 d_k d_v; quantized: 4r + 2 hp d_v + r d_v
    with r = d_k - hp), strides padded to 16 bytes."""
    for d_k in range(16, 257, 16):
        for d_v in range(16, 257, 16):
            assert D.damp_layout(D.DAMP_FMT_FP32, d_k, d_v, 0)[0] == 4 * d_k * d_v
            for hp in (0, d_k // 3, d_k):
                b, s = D.damp_layout(D.DAMP_FMT_MIXED, d_k, d_v, hp)
                r = d_k - hp
                assert b == 4 * r + 2 * hp * d_v + r * d_v
                assert s % 16 == 0 and b <= s < b + 32
            assert D.damp_layout(D.DAMP_FMT_FP8_ROW, d_k, d_v, 0)[0] == 4 * d_k + d_k * d_v


def test_status_strings():
    for s in (0, -1, -2, -3, -4, -5, -6, -99):
        assert isinstance(D.damp_status_string(s), str) and D.damp_status_string(s)


def test_create_validates_the_fp16_row_map():
    ok = np.array([[0, 5, 9], [1, 2, 3]])
    h = D.damp_pool_create(D.DAMP_FMT_MIXED, 4, 2, 16, 16, 3, ok, None)
    D.damp_pool_destroy(h)
    for bad in (np.array([[0, 5, 5], [1, 2, 3]]), np.array([[0, 5, 16], [1, 2, 3]])):
        with pytest.raises(D.DampError) as ei:
            D.damp_pool_create(D.DAMP_FMT_MIXED, 4, 2, 16, 16, 3, bad, None)
        assert ei.value.status == D.DAMP_ERR_INVALID_ARGUMENT
    with pytest.raises(D.DampError):
        D.damp_pool_create(D.DAMP_FMT_MIXED, 0, 2, 16, 16, 0, None, None)


def test_create_checks_buffer_before_touching_the_device():
    lib = ctypes.CDLL(D.LIB_PATH)
    lib.damp_pool_create.argtypes = [ctypes.c_int] * 6 + [ctypes.c_void_p, ctypes.c_void_p,
                                                          ctypes.c_size_t,
                                                          ctypes.POINTER(ctypes.c_void_p)]
    out = ctypes.c_void_p()
    need = D.damp_pool_bytes(D.DAMP_FMT_INT8_ROW, 2, 2, 16, 16, 0)
    rc = lib.damp_pool_create(D.DAMP_FMT_INT8_ROW, 2, 2, 16, 16, 0, None, 0x10000, need - 1,
                              ctypes.byref(out))
    assert rc == D.DAMP_ERR_BUFFER_TOO_SMALL and not out.value
    rc = lib.damp_pool_create(D.DAMP_FMT_INT8_ROW, 2, 2, 16, 16, 0, None, 0x10008, need,
                              ctypes.byref(out))
    assert rc == D.DAMP_ERR_MISALIGNED and not out.value


def test_host_only_descriptor_rejects_device_calls():
    h = D.damp_pool_create(D.DAMP_FMT_INT8_ROW, 2, 2, 16, 16, 0, None, None)
    try:
        lib = D._lib
        assert lib.damp_decode_step(h, 1, 16, 0, 16, 16, 16, 0, 16, 16, 16, None) == \
            D.DAMP_ERR_INVALID_ARGUMENT
        assert lib.damp_pool_pack(h, 1, 16, 16, None) == D.DAMP_ERR_INVALID_ARGUMENT
        assert lib.damp_decode_step(None, 1, 16, 0, 16, 16, 16, 0, 16, 16, 16, None) == \
            D.DAMP_ERR_INVALID_ARGUMENT
    finally:
        D.damp_pool_destroy(h)


@pytest.mark.parametrize("d,dv,hp", [(16, 16, 4), (64, 64, 0), (128, 128, 27), (128, 128, 128),
                                     (48, 80, 7), (256, 32, 100), (32, 256, 32)])
def test_block_logical_round_trip(d, dv, hp):
    g = np.random.default_rng(d + dv + hp)
    H = 3
    idx = np.stack([np.sort(g.permutation(d)[:hp]) for _ in range(H)])
    h = D.damp_pool_create(D.DAMP_FMT_MIXED, 2, H, d, dv, hp, idx if hp else None, None)
    try:
        _, stride = D.damp_layout(D.DAMP_FMT_MIXED, d, dv, hp)
        for head in range(H):
            is16 = np.zeros(d, bool)
            is16[idx[head]] = True
            scale = np.where(is16, 0, g.uniform(0.1, 2, d)).astype(np.float32)
            half = np.where(is16[:, None], g.integers(0, 0x7C00, (d, dv)), 0).astype(np.uint16)
            code = np.where(is16[:, None], 0, g.integers(-127, 128, (d, dv))).astype(np.int8)
            raw = D.damp_block_from_logical(h, head, stride, scale=scale, half=half, code=code)
            assert raw.size == stride
            back = D.damp_block_to_logical(h, head, raw, D.DAMP_FMT_MIXED, d, dv)
            assert np.array_equal(back["scale"], scale)
            assert np.array_equal(back["half"], half)
            assert np.array_equal(back["code"], code)
            # byte order: scales of INT8 rows first, then FP16 rows, then INT8 rows;
            # an FP16 row is two planes: values 4g, 4g+1 of each column group g,
            # then values 4g+2, 4g+3
            r = d - hp
            assert np.array_equal(raw[:4 * r].view(np.float32), scale[~is16])
            f16_off = (4 * r + 15) // 16 * 16
            groups = half[is16].reshape(hp, dv // 4, 4)
            planes = np.concatenate([groups[:, :, 0:2].reshape(hp, dv // 2),
                                     groups[:, :, 2:4].reshape(hp, dv // 2)], axis=1)
            assert np.array_equal(raw[f16_off:f16_off + 2 * hp * dv].view(np.uint16),
                                  planes.reshape(-1))
            assert np.array_equal(raw[f16_off + 2 * hp * dv:f16_off + 2 * hp * dv + r * dv]
                                  .view(np.int8), code[~is16].reshape(-1))
    finally:
        D.damp_pool_destroy(h)


def test_per_head_map_layout():
    """Heads with different FP16-row counts: each head's block has the layout
    of its own count, the slot is their concatenation, and a map with one
    count everywhere is the fixed-count pool."""
    d, H = 64, 4
    g = np.random.default_rng(2)
    counts = [0, 5, 64, 17]
    m = np.zeros((H, d), np.uint8)
    for h, c in enumerate(counts):
        m[h, g.permutation(d)[:c]] = 1
    h = D.damp_pool_create_map(3, H, d, d, m, None)
    try:
        off = 0
        for head, c in enumerate(counts):
            b, st, o = D.damp_pool_head_layout(h, head)
            assert (b, st) == D.damp_layout(D.DAMP_FMT_MIXED, d, d, c) and o == off
            off += st
        hdr = D.damp_pool_block_offset(h, 0, 0)
        assert D.damp_pool_block_offset(h, 2, 3) == hdr + 2 * off + D.damp_pool_head_layout(h, 3)[2]
        assert D.damp_pool_bytes_map(3, H, d, d, m) == hdr + 3 * off
        # logical round trip through the per-head layout
        for head, c in enumerate(counts):
            st = D.damp_pool_head_layout(h, head)[1]
            is16 = m[head].astype(bool)
            scale = np.where(is16, 0, g.uniform(0.1, 2, d)).astype(np.float32)
            half = np.where(is16[:, None], g.integers(0, 0x7C00, (d, d)), 0).astype(np.uint16)
            code = np.where(is16[:, None], 0, g.integers(-127, 128, (d, d))).astype(np.int8)
            raw = D.damp_block_from_logical(h, head, st, scale=scale, half=half, code=code)
            back = D.damp_block_to_logical(h, head, raw, D.DAMP_FMT_MIXED, d)
            assert np.array_equal(back["half"], half) and np.array_equal(back["code"], code)
            assert np.array_equal(back["scale"], scale)
    finally:
        D.damp_pool_destroy(h)
    same = np.zeros((H, d), np.uint8)
    same[:, :7] = 1
    assert D.damp_pool_bytes_map(5, H, d, d, same) == \
        D.damp_pool_bytes(D.DAMP_FMT_MIXED, 5, H, d, d, 7)
    with pytest.raises(D.DampError):
        bad = same.copy()
        bad[0, 0] = 2
        D.damp_pool_bytes_map(5, H, d, d, bad)


def test_validate_slots():
    D.damp_validate_slots(np.array([3, -1, 0, 5, -1], np.int32), 6)
    D.damp_validate_slots(np.zeros(0, np.int32), 1)
    for bad, pos in ((np.array([1, 2, 1], np.int32), 2), (np.array([0, 6], np.int32), 1)):
        with pytest.raises(D.DampError) as ei:
            D.damp_validate_slots(bad, 6)
        assert ei.value.status == D.DAMP_ERR_INVALID_ARGUMENT and f"entry {pos}" in str(ei.value)


# ---------------------------------------------------------------- binding checks

def _host_pool(fmt=D.DAMP_FMT_MIXED, n_slots=4, H=2, d=16, hp=4):
    """A host-only descriptor (no device buffer): enough for the binding's
    argument checks, which all run before anything would be enqueued."""
    idx = np.tile(np.arange(hp, dtype=np.uint16), (H, 1)) if hp else None
    return D.damp_pool_create(fmt, n_slots, H, d, d, hp, idx, None)


def _step_tensors(n=3, H=2, d=16, kda=False, dtype=None):
    import torch
    dtype = dtype or torch.float32
    return dict(slot_idx=torch.arange(n, dtype=torch.int32),
                q=torch.zeros((n, H, d), dtype=dtype), k=torch.zeros((n, H, d), dtype=dtype),
                v=torch.zeros((n, H, d), dtype=dtype),
                alpha=torch.zeros((n, H, d) if kda else (n, H)), beta=torch.zeros((n, H)),
                out=torch.zeros((n, H, d)))


@pytest.mark.parametrize("bad", ["q", "k", "v", "beta", "out", "alpha"])
def test_binding_rejects_wrong_shapes_before_launch(bad):
    """The C ABI cannot see tensor sizes: the binding checks every tensor of a
    step against (n, H, d_k, d_v) of the pool and raises before any call."""
    import torch
    h = _host_pool()
    try:
        t = _step_tensors()
        t[bad] = torch.zeros((3, 2, 15)) if bad != "beta" else torch.zeros((3, 3))
        with pytest.raises(ValueError, match=bad):
            D.damp_decode_step(h, **t)
        t = _step_tensors()
        t["slot_idx"] = torch.arange(4, dtype=torch.int32)        # n = 4 vs tensors of 3
        with pytest.raises(ValueError):
            D.damp_decode_step(h, **t)
    finally:
        D.damp_pool_destroy(h)


def test_binding_gate_from_alpha_shape_and_device_checks():
    import torch
    h = _host_pool()
    try:
        # correct shapes (GDN and KDA) pass the shape checks and stop at the
        # device check: these tensors are on the CPU
        for kda in (False, True):
            with pytest.raises(ValueError, match="CUDA"):
                D.damp_decode_step(h, **_step_tensors(kda=kda))
        t = _step_tensors()
        t["alpha"] = torch.zeros((3, 2, 1))
        with pytest.raises(ValueError, match="alpha"):
            D.damp_decode_step(h, **t)
        with pytest.raises(ValueError, match="state"):
            D.damp_pool_pack(h, torch.arange(3, dtype=torch.int32), torch.zeros((3, 2, 16, 8)))
        with pytest.raises(ValueError, match="unknown pool"):
            D.damp_decode_step(12345, **_step_tensors())
    finally:
        D.damp_pool_destroy(h)

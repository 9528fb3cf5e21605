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
    # status word; per head a 16-byte FP16-row mask, a 512-byte row directory
    # followed by its 16-byte row-group order, and a 16-byte block-table entry
    hdr = 256 * ((16 + 32 * 16 + 32 * (512 + 16) + 32 * 16 + 255) // 256)
    assert n == hdr + 64 * 32 * 20256


@pytest.mark.parametrize("args,status", [
    ((4, 128, 128, 0), D.DAMP_ERR_INVALID_ARGUMENT),         # bad format
    ((D.DAMP_FMT_FP8_ROW, 128, 128, 2), D.DAMP_ERR_INVALID_ARGUMENT),
    ((D.DAMP_FMT_MIXED, 128, 128, 129), D.DAMP_ERR_INVALID_ARGUMENT),
    ((D.DAMP_FMT_MIXED, 128, 128, -1), D.DAMP_ERR_INVALID_ARGUMENT),
    ((D.DAMP_FMT_INT8_ROW, 128, 128, 3), D.DAMP_ERR_INVALID_ARGUMENT),
    ((D.DAMP_FMT_FP32, 128, 128, 1), D.DAMP_ERR_INVALID_ARGUMENT),
    ((D.DAMP_FMT_MIXED, 128, 64, 0), D.DAMP_ERR_UNSUPPORTED),
    ((D.DAMP_FMT_MIXED, 48, 48, 0), D.DAMP_ERR_UNSUPPORTED),
    ((D.DAMP_FMT_MIXED, 256, 256, 0), D.DAMP_ERR_UNSUPPORTED),
])
def test_layout_rejects_bad_shapes(args, status):
    with pytest.raises(D.DampError) as ei:
        D.damp_layout(*args)
    assert ei.value.status == status


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


@pytest.mark.parametrize("d,hp", [(16, 4), (64, 0), (128, 27), (128, 128)])
def test_block_logical_round_trip(d, hp):
    g = np.random.default_rng(d + hp)
    H = 3
    idx = np.stack([np.sort(g.permutation(d)[:hp]) for _ in range(H)])
    h = D.damp_pool_create(D.DAMP_FMT_MIXED, 2, H, d, d, hp, idx if hp else None, None)
    try:
        _, stride = D.damp_layout(D.DAMP_FMT_MIXED, d, d, hp)
        for head in range(H):
            is16 = np.zeros(d, bool)
            is16[idx[head]] = True
            scale = np.where(is16, 0, g.uniform(0.1, 2, d)).astype(np.float32)
            half = np.where(is16[:, None], g.integers(0, 0x7C00, (d, d)), 0).astype(np.uint16)
            code = np.where(is16[:, None], 0, g.integers(-127, 128, (d, d))).astype(np.int8)
            raw = D.damp_block_from_logical(h, head, stride, scale=scale, half=half, code=code)
            assert raw.size == stride
            back = D.damp_block_to_logical(h, head, raw, D.DAMP_FMT_MIXED, d)
            assert np.array_equal(back["scale"], scale)
            assert np.array_equal(back["half"], half)
            assert np.array_equal(back["code"], code)
            # byte order: scales of INT8 rows first, then FP16 rows, then INT8 rows
            r = d - hp
            assert np.array_equal(raw[:4 * r].view(np.float32), scale[~is16])
            f16_off = (4 * r + 15) // 16 * 16
            assert np.array_equal(raw[f16_off:f16_off + 2 * hp * d].view(np.uint16),
                                  half[is16].reshape(-1))
            assert np.array_equal(raw[f16_off + 2 * hp * d:f16_off + 2 * hp * d + r * d]
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


def _group_masks(is16_row):
    return [int(sum(int(is16_row[8 * g + i]) << i for i in range(8))) for g in range(16)]


def _pair_cost(m, order):
    return sum(bin(m[order[2 * k]] ^ m[order[2 * k + 1]]).count("1") for k in range(8))


def _min_pair_cost(m):
    """Minimum over all perfect matchings of the 16 groups, by recursion over
    the lowest unmatched group (memoised on the set of matched groups)."""
    import functools

    @functools.lru_cache(None)
    def f(left):
        if not left:
            return 0
        i, rest = left[0], left[1:]
        return min(bin(m[i] ^ m[j]).count("1") + f(rest[:t] + rest[t + 1:])
                   for t, j in enumerate(rest))
    return f(tuple(range(16)))


def test_row_group_order_is_a_minimum_cost_pairing():
    """The d = 128 decode step's row-group order: a permutation of the 16
    groups whose warp pairs differ in format at the fewest row positions."""
    g = np.random.default_rng(7)
    H, d = 6, 128
    m = np.zeros((H, d), np.uint8)
    for head, c in enumerate([0, 1, 27, 40, 64, 128]):
        m[head, g.choice(d, c, replace=False)] = 1
    h = D.damp_pool_create_map(3, H, d, d, m, None)
    try:
        for head in range(H):
            order = D.damp_pool_row_groups(h, head)
            assert sorted(order) == list(range(16))
            gm = _group_masks(m[head])
            assert _pair_cost(gm, order) == _min_pair_cost(gm)
            lows = [min(order[2 * k], order[2 * k + 1]) for k in range(8)]
            assert lows == sorted(lows) and all(order[2 * k] < order[2 * k + 1] for k in range(8))
        # no FP16 row, or every row FP16: nothing to pair, groups in order
        assert D.damp_pool_row_groups(h, 0) == list(range(16))
        assert D.damp_pool_row_groups(h, 5) == list(range(16))
        with pytest.raises(D.DampError):
            D.damp_pool_row_groups(h, H)
    finally:
        D.damp_pool_destroy(h)


def test_row_group_order_worked_example():
    """Groups 0 and 2 hold FP16 rows at the same 8 positions, all others none:
    0 pairs with 2 at no cost, then 1 with its lowest free partner 3, and the
    rest in order."""
    row = np.zeros(128, np.uint8)
    row[0:8] = 1
    row[16:24] = 1
    h = D.damp_pool_create_map(1, 1, 128, 128, row[None, :], None)
    try:
        assert D.damp_pool_row_groups(h, 0) == [0, 2, 1, 3] + list(range(4, 16))
    finally:
        D.damp_pool_destroy(h)

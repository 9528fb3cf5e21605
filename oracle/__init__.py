"""Python wrapper of the C oracle -- TEST INFRASTRUCTURE ONLY.

The oracle is a plain, slow CPU statement of the DAMP-style decode step (see
``damp_oracle.c`` for the passages it follows and the readings it takes where
the pages are silent).  Only ``tests/``, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may import this package.  It shares no code with
the CUDA library and never imports it.

Logical state of a quantized (slot, head) state, rows in key-channel order:
``scale`` float32 [..., d_k], ``half`` uint16 [..., d_k, d_v] (binary16 bits of
FP16 rows), ``code`` int8 [..., d_k, d_v] (codes of INT8 rows); unused entries
are zero.  The FP8 comparison format uses ``scale`` and ``code`` (E4M3 bit
patterns, viewed as int8) for every row.  An FP32 state is ``f32`` float32 [..., d_k, d_v].
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import numpy as np

from . import build as _build

FMT_FP32 = 0
FMT_QUANT = 1
FMT_FP8 = 2
GATE_SCALAR = 0
GATE_VECTOR = 1

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        _lib = ctypes.CDLL(path)
        P = ctypes.c_void_p
        I = ctypes.c_int
        _lib.oracle_f16_from_f32.restype = ctypes.c_uint16
        _lib.oracle_f16_from_f32.argtypes = [ctypes.c_float]
        _lib.oracle_f32_from_f16.restype = ctypes.c_float
        _lib.oracle_f32_from_f16.argtypes = [ctypes.c_uint16]
        _lib.oracle_f16_from_f32_array.argtypes = [P, P, ctypes.c_long]
        _lib.oracle_f32_from_f16_array.argtypes = [P, P, ctypes.c_long]
        _lib.oracle_quantize_row.argtypes = [P, I, P, P]
        _lib.oracle_quantize_row_fp8.argtypes = [P, I, P, P]
        _lib.oracle_e4m3_from_f32_array.argtypes = [P, P, ctypes.c_long]
        _lib.oracle_f32_from_e4m3_array.argtypes = [P, P, ctypes.c_long]
        _lib.oracle_quantize_row_prerounding.argtypes = [P, I, P]
        _lib.oracle_pairwise_sum.restype = ctypes.c_float
        _lib.oracle_pairwise_sum.argtypes = [P, I]
        _lib.oracle_pack_unit.argtypes = [I, I, I, P, P, P, P, P, P]
        _lib.oracle_unpack_unit.argtypes = [I, I, I, P, P, P, P, P, P]
        _lib.oracle_step_unit.argtypes = [I, I, I, I, P, P, P, P, P, P, P, P, P,
                                          ctypes.c_float, P, P]
        _lib.oracle_decode_step.argtypes = [I, I, I, I, I, I, I, P, P, P, P, P, P,
                                            P, P, P, P, P, P]
        _lib.oracle_row_quant_error.restype = ctypes.c_double
        _lib.oracle_row_quant_error.argtypes = [P, I]
        _lib.oracle_calib_accumulate.argtypes = [I, I, I, I, I, I, P, P, P, P]
        _lib.oracle_calib_scores.argtypes = [I, I, P, P]
        _lib.oracle_calib_select.argtypes = [I, I, I, P, P]
        _lib.oracle_calib_select_budget.argtypes = [I, I, I, P, P, P]
        for f in ("oracle_pack_unit", "oracle_unpack_unit", "oracle_step_unit",
                  "oracle_decode_step", "oracle_calib_accumulate", "oracle_calib_scores",
                  "oracle_calib_select", "oracle_calib_select_budget"):
            getattr(_lib, f).restype = I
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# --------------------------------------------------------------------------
# element and row primitives
# --------------------------------------------------------------------------

def f16_from_f32(x) -> np.ndarray:
    x = _c(x, np.float32)
    out = np.empty(x.shape, np.uint16)
    lib().oracle_f16_from_f32_array(_p(x), _p(out), x.size)
    return out


def f32_from_f16(h) -> np.ndarray:
    h = _c(h, np.uint16)
    out = np.empty(h.shape, np.float32)
    lib().oracle_f32_from_f16_array(_p(h), _p(out), h.size)
    return out


def quantize_row(x):
    """(codes int8[n], scale float32) of one INT8 row."""
    x = _c(x, np.float32)
    code = np.empty(x.shape, np.int8)
    scale = np.zeros(1, np.float32)
    lib().oracle_quantize_row(_p(x), x.size, _p(code), _p(scale))
    return code, scale[0]


def e4m3_from_f32(x) -> np.ndarray:
    """E4M3 codes (uint8 bit patterns), nearest-even with saturation at 448."""
    x = _c(x, np.float32)
    out = np.empty(x.shape, np.uint8)
    lib().oracle_e4m3_from_f32_array(_p(x), _p(out), x.size)
    return out


def f32_from_e4m3(c) -> np.ndarray:
    c = _c(c, np.uint8)
    out = np.empty(c.shape, np.float32)
    lib().oracle_f32_from_e4m3_array(_p(c), _p(out), c.size)
    return out


def quantize_row_fp8(x):
    """(E4M3 codes uint8[n], scale float32) of one FP8 row."""
    x = _c(x, np.float32)
    code = np.empty(x.shape, np.uint8)
    scale = np.zeros(1, np.float32)
    lib().oracle_quantize_row_fp8(_p(x), x.size, _p(code), _p(scale))
    return code, scale[0]


def quantize_row_prerounding(x) -> np.ndarray:
    x = _c(x, np.float32)
    t = np.empty(x.shape, np.float64)
    lib().oracle_quantize_row_prerounding(_p(x), x.size, _p(t))
    return t


def pairwise_sum(x) -> np.float32:
    x = _c(x, np.float32)
    return np.float32(lib().oracle_pairwise_sum(_p(x), x.size))


# --------------------------------------------------------------------------
# states
# --------------------------------------------------------------------------

@dataclass
class State:
    """Logical state of one or many (slot, head) units; leading dims free."""
    fmt: int
    scale: np.ndarray | None = None
    half: np.ndarray | None = None
    code: np.ndarray | None = None
    f32: np.ndarray | None = None

    def copy(self) -> "State":
        c = lambda a: None if a is None else a.copy()
        return State(self.fmt, c(self.scale), c(self.half), c(self.code), c(self.f32))

    def __getitem__(self, idx) -> "State":
        g = lambda a: None if a is None else a[idx]
        return State(self.fmt, g(self.scale), g(self.half), g(self.code), g(self.f32))


def empty_state(fmt: int, lead: tuple, dk: int, dv: int) -> State:
    if fmt == FMT_FP32:
        return State(fmt, f32=np.zeros(lead + (dk, dv), np.float32))
    return State(fmt, scale=np.zeros(lead + (dk,), np.float32),
                 half=np.zeros(lead + (dk, dv), np.uint16),
                 code=np.zeros(lead + (dk, dv), np.int8))


def pack(fmt: int, is_fp16, S) -> State:
    """Compress FP32 states S [..., d_k, d_v]; is_fp16 [d_k] or [..., d_k]."""
    S = _c(S, np.float32)
    dk, dv = S.shape[-2:]
    lead = S.shape[:-2]
    st = empty_state(fmt, lead, dk, dv)
    flags = np.broadcast_to(np.asarray(is_fp16, np.uint8), lead + (dk,)).copy()
    for idx in np.ndindex(*lead) if lead else [()]:
        u = st[idx] if lead else st
        rc = lib().oracle_pack_unit(fmt, dk, dv, _p(flags[idx]), _p(S[idx]),
                                    _p(u.scale), _p(u.half), _p(u.code), _p(u.f32))
        assert rc == 0, rc
    return st


def unpack(st: State, is_fp16) -> np.ndarray:
    arr = st.f32 if st.fmt == FMT_FP32 else st.half
    dk, dv = arr.shape[-2:]
    lead = arr.shape[:-2]
    out = np.empty(lead + (dk, dv), np.float32)
    flags = np.broadcast_to(np.asarray(is_fp16, np.uint8), lead + (dk,)).copy()
    for idx in np.ndindex(*lead) if lead else [()]:
        u = st[idx] if lead else st
        rc = lib().oracle_unpack_unit(st.fmt, dk, dv, _p(flags[idx]), _p(u.scale),
                                      _p(u.half), _p(u.code), _p(u.f32), _p(out[idx]))
        assert rc == 0, rc
    return out


def step_unit(st: State, gate: int, is_fp16, q, k, v, alpha, beta, want_x=False):
    """One decode step of ONE unit, in place on ``st`` (arrays without lead dims).

    Returns o (float64 [d_v]) or (o, X) when want_x.
    """
    arr = st.f32 if st.fmt == FMT_FP32 else st.half
    dk, dv = arr.shape
    q = _c(q, np.float32)
    k = _c(k, np.float32)
    v = _c(v, np.float32)
    alpha = _c(np.atleast_1d(alpha), np.float32)
    flags = _c(is_fp16, np.uint8)
    o = np.empty(dv, np.float64)
    X = np.empty((dk, dv), np.float32) if want_x else None
    rc = lib().oracle_step_unit(st.fmt, gate, dk, dv, _p(flags), _p(st.scale), _p(st.half),
                                _p(st.code), _p(st.f32), _p(q), _p(k), _p(v), _p(alpha),
                                float(beta), _p(o), _p(X))
    assert rc == 0, rc
    return (o, X) if want_x else o


def decode_step(pool: State, gate: int, is_fp16, slot_idx, q, k, v, alpha, beta):
    """One decode step over a batch, in place on ``pool`` ([n_slots][H] lead dims).

    is_fp16 [H][d_k]; slot_idx int32 [n]; q,k [n][H][d_k]; v [n][H][d_v];
    alpha [n][H] (GDN) or [n][H][d_k] (KDA); beta [n][H].  Returns o float64
    [n][H][d_v].  Raises ValueError on a slot index >= n_slots.
    """
    arr = pool.f32 if pool.fmt == FMT_FP32 else pool.half
    n_slots, H, dk, dv = arr.shape
    slot_idx = _c(slot_idx, np.int32)
    n = slot_idx.shape[0]
    flags = _c(is_fp16, np.uint8)
    assert flags.shape == (H, dk)
    q = _c(q, np.float32)
    k = _c(k, np.float32)
    v = _c(v, np.float32)
    alpha = _c(alpha, np.float32)
    beta = _c(beta, np.float32)
    o = np.zeros((n, H, dv), np.float64)
    rc = lib().oracle_decode_step(pool.fmt, gate, n, H, dk, dv, n_slots, _p(flags),
                                  _p(slot_idx), _p(pool.scale), _p(pool.half), _p(pool.code),
                                  _p(pool.f32), _p(q), _p(k), _p(v), _p(alpha), _p(beta), _p(o))
    if rc == -2:
        raise ValueError("slot index out of range")
    assert rc == 0, rc
    return o


# --------------------------------------------------------------------------
# offline calibration (calib_oracle.c)
# --------------------------------------------------------------------------

def row_quant_error(x) -> float:
    """Squared error of the INT8 row quantizer on one row (double)."""
    x = _c(x, np.float32)
    return float(lib().oracle_row_quant_error(_p(x), x.size))


def calib_acc(H: int, dk: int) -> np.ndarray:
    """Zeroed accumulator: energy [H][d_k], retention [H][d_k], count [H]."""
    return np.zeros(2 * H * dk + H, np.float64)


def calib_accumulate(acc: np.ndarray, gate: int, f32_pool, slot_idx, alpha) -> None:
    """Add one step's records (FP32 states after the step) to ``acc``."""
    f32_pool = _c(f32_pool, np.float32)
    n_slots, H, dk, dv = f32_pool.shape
    slot_idx = _c(slot_idx, np.int32)
    alpha = _c(alpha, np.float32)
    assert acc.dtype == np.float64 and acc.size == 2 * H * dk + H
    rc = lib().oracle_calib_accumulate(gate, slot_idx.size, H, dk, dv, n_slots, _p(f32_pool),
                                       _p(slot_idx), _p(alpha), _p(acc))
    if rc == -2:
        raise ValueError("slot index out of range")
    assert rc == 0, rc


def calib_scores(acc: np.ndarray, H: int, dk: int) -> np.ndarray:
    score = np.empty((H, dk), np.float64)
    rc = lib().oracle_calib_scores(H, dk, _p(_c(acc, np.float64)), _p(score))
    assert rc == 0, rc
    return score


def calib_select(score, hp: int) -> np.ndarray:
    """hp_row_idx uint16 [H][hp], ascending per head."""
    score = _c(score, np.float64)
    H, dk = score.shape
    out = np.zeros((H, hp), np.uint16)
    rc = lib().oracle_calib_select(H, dk, hp, _p(score), _p(out))
    assert rc == 0, rc
    return out


def calib_select_budget(score, budget: int):
    """(is_fp16 uint8 [H][d_k], hp int32 [H]) for a total of ``budget`` FP16 rows."""
    score = _c(score, np.float64)
    H, dk = score.shape
    is16 = np.zeros((H, dk), np.uint8)
    hp = np.zeros(H, np.int32)
    rc = lib().oracle_calib_select_budget(H, dk, budget, _p(score), _p(is16), _p(hp))
    assert rc == 0, rc
    return is16, hp

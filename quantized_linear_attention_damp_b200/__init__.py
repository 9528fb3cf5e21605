"""Python binding of libdamp, the B200 decode step of DAMP-style mixed-precision
recurrent states (Gated DeltaNet / Kimi Delta Attention).

Every function here has the name of the C entry point it marshals arguments
for (declared in include/damp.h); all work happens in libdamp's CUDA kernels.
PyTorch supplies device memory and streams only.  Importing this module
fails if libdamp.so has not been built: there is no fallback path.

Tensor arguments must be contiguous CUDA tensors of the documented dtype;
``stream`` defaults to the current PyTorch stream of the tensors' device.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdamp.so")

DAMP_OK = 0
DAMP_ERR_INVALID_ARGUMENT = -1
DAMP_ERR_UNSUPPORTED = -2
DAMP_ERR_MISALIGNED = -3
DAMP_ERR_BUFFER_TOO_SMALL = -4
DAMP_ERR_CUDA = -5
DAMP_ERR_TIMEOUT = -6

DAMP_EFLAG_SLOT_RANGE = 1
DAMP_EFLAG_TIMEOUT = 2
DAMP_EFLAG_NONFINITE = 4
DAMP_HOOK_HOLD_FIRST_ITEM = 1

DAMP_FMT_FP32 = 0
DAMP_FMT_INT8_ROW = 1
DAMP_FMT_MIXED = 2
DAMP_FMT_FP8_ROW = 3
DAMP_GATE_SCALAR = 0
DAMP_GATE_VECTOR = 1
DAMP_DTYPE_BF16 = 0
DAMP_DTYPE_F32 = 1

FORMATS = {"fp32": DAMP_FMT_FP32, "int8": DAMP_FMT_INT8_ROW, "mixed": DAMP_FMT_MIXED,
           "fp8": DAMP_FMT_FP8_ROW}


class DampError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {damp_status_string(status)} ({status})")
        self.status = status


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing; build it with "
            "`python quantized_linear_attention_damp_b200/build.py`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    sig = {
        "damp_status_string": (ctypes.c_char_p, [I]),
        "damp_layout": (I, [I, I, I, I, ctypes.POINTER(S), ctypes.POINTER(S)]),
        "damp_pool_bytes": (I, [I, I, I, I, I, I, ctypes.POINTER(S)]),
        "damp_pool_create": (I, [I, I, I, I, I, I, P, P, S, ctypes.POINTER(P)]),
        "damp_pool_destroy": (I, [P]),
        "damp_pool_block_offset": (I, [P, I, I, ctypes.POINTER(S)]),
        "damp_pool_pack": (I, [P, I, P, P, P]),
        "damp_pool_unpack": (I, [P, I, P, P, P]),
        "damp_decode_step": (I, [P, I, P, I, P, P, P, I, P, P, P, P]),
        "damp_decode_step_validated": (I, [P, I, P, I, P, P, P, I, P, P, P, P]),
        "damp_set_test_hooks": (I, [ctypes.c_uint64, ctypes.c_uint32]),
        "damp_pool_get_error": (I, [P, ctypes.POINTER(ctypes.c_uint32), I, P]),
        "damp_block_to_logical": (I, [P, I, P, P, P, P, P]),
        "damp_block_from_logical": (I, [P, I, P, P, P, P, P]),
        "damp_pool_bytes_map": (I, [I, I, I, I, P, ctypes.POINTER(S)]),
        "damp_pool_create_map": (I, [I, I, I, I, P, P, S, ctypes.POINTER(P)]),
        "damp_pool_head_layout": (I, [P, I, ctypes.POINTER(S), ctypes.POINTER(S),
                                      ctypes.POINTER(S)]),
        "damp_pool_read_raw": (I, [P, I, I, P]),
        "damp_validate_slots": (I, [P, I, I, ctypes.POINTER(I)]),
        "damp_calib_bytes": (S, [I, I]),
        "damp_calib_accumulate": (I, [P, I, P, I, P, P, P]),
        "damp_calib_select": (I, [I, I, I, P, P, P, P]),
        "damp_calib_select_budget": (I, [I, I, I, P, P, P, P, P]),
        "damp_calib_select_budget_static": (I, [I, I, I, P, P, P, P]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    return lib


_lib = _load()


def _check(status: int, where: str):
    if status != DAMP_OK:
        raise DampError(status, where)


# (format, n_slots, H, d_k, d_v) of every pool descriptor made through this
# module: the C ABI cannot see tensor sizes, so the binding checks them
# against the pool before anything is enqueued.
_POOLS: dict[int, tuple[int, int, int, int, int]] = {}


def _pool_shape(pool: int):
    try:
        return _POOLS[int(pool)]
    except (KeyError, TypeError):
        raise ValueError("unknown pool handle: create pools through this module") from None


def _shape(t, name: str, shape: tuple):
    if not isinstance(t, torch.Tensor):
        raise ValueError(f"{name} must be a torch tensor")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _same_device(stream, *tensors):
    dev = tensors[0].device
    for t in tensors[1:]:
        if t.device != dev:
            raise ValueError(f"tensors on different devices: {dev} and {t.device}")
    if isinstance(stream, torch.cuda.Stream) and stream.device != dev:
        raise ValueError(f"stream on {stream.device}, tensors on {dev}")


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, torch.Tensor):
        if not t.is_contiguous():
            raise ValueError("tensor arguments must be contiguous")
        return t.data_ptr()
    if isinstance(t, np.ndarray):
        if not t.flags["C_CONTIGUOUS"]:
            raise ValueError("array arguments must be C-contiguous")
        return t.ctypes.data
    raise TypeError(f"unsupported argument type {type(t)}")


def _cuda(t: torch.Tensor, dtype, name: str):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    return t


def _stream(stream, device) -> int | None:
    if stream is None:
        return torch.cuda.current_stream(device).cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


# ---------------------------------------------------------------- host-side calls

def damp_status_string(status: int) -> str:
    return _lib.damp_status_string(int(status)).decode()


def damp_layout(format: int, d_k: int, d_v: int, hp_rows: int) -> tuple[int, int]:
    """(block_bytes, block_stride) of one (slot, head) block."""
    b, s = ctypes.c_size_t(), ctypes.c_size_t()
    _check(_lib.damp_layout(format, d_k, d_v, hp_rows, ctypes.byref(b), ctypes.byref(s)),
           "damp_layout")
    return b.value, s.value


def damp_pool_bytes(format: int, n_slots: int, H: int, d_k: int, d_v: int, hp_rows: int) -> int:
    b = ctypes.c_size_t()
    _check(_lib.damp_pool_bytes(format, n_slots, H, d_k, d_v, hp_rows, ctypes.byref(b)),
           "damp_pool_bytes")
    return b.value


def damp_pool_create(format: int, n_slots: int, H: int, d_k: int, d_v: int, hp_rows: int,
                     hp_row_idx, dev_buf: torch.Tensor | None) -> int:
    """Descriptor handle.  hp_row_idx: [H][hp_rows] integer array (host) or None.
    dev_buf: CUDA uint8 tensor of >= damp_pool_bytes(...) bytes, or None for a
    host-only descriptor (layout queries and block conversions only)."""
    idx = None
    if hp_row_idx is not None and hp_rows > 0:
        idx = np.ascontiguousarray(np.asarray(hp_row_idx).reshape(H, hp_rows), np.uint16)
    buf_ptr, nbytes = None, 0
    if dev_buf is not None:
        _cuda(dev_buf, torch.uint8, "dev_buf")
        buf_ptr, nbytes = _ptr(dev_buf), dev_buf.numel()
    h = ctypes.c_void_p()
    _check(_lib.damp_pool_create(format, n_slots, H, d_k, d_v, hp_rows, _ptr(idx), buf_ptr,
                                 nbytes, ctypes.byref(h)), "damp_pool_create")
    _POOLS[h.value] = (int(format), n_slots, H, d_k, d_v)
    return h.value


def damp_pool_bytes_map(n_slots: int, H: int, d_k: int, d_v: int, is_fp16) -> int:
    m = np.ascontiguousarray(is_fp16, np.uint8)
    if m.shape != (H, d_k):
        raise ValueError("is_fp16 must be [H][d_k]")
    out = ctypes.c_size_t()
    _check(_lib.damp_pool_bytes_map(n_slots, H, d_k, d_v, _ptr(m), ctypes.byref(out)),
           "damp_pool_bytes_map")
    return out.value


def damp_pool_create_map(n_slots: int, H: int, d_k: int, d_v: int, is_fp16, buf) -> int:
    """Mixed pool with a per-head FP16-row map (counts may differ per head)."""
    m = np.ascontiguousarray(is_fp16, np.uint8)
    if m.shape != (H, d_k):
        raise ValueError("is_fp16 must be [H][d_k]")
    h = ctypes.c_void_p()
    ptr, nbytes = None, 0
    if buf is not None:
        _cuda(buf, torch.uint8, "dev_buf")
        ptr, nbytes = _ptr(buf), buf.numel()
    _check(_lib.damp_pool_create_map(n_slots, H, d_k, d_v, _ptr(m), ptr, nbytes,
                                     ctypes.byref(h)), "damp_pool_create_map")
    _POOLS[h.value] = (DAMP_FMT_MIXED, n_slots, H, d_k, d_v)
    return h.value


def damp_pool_head_layout(pool: int, h: int) -> tuple[int, int, int]:
    """(block_bytes, block_stride, offset_in_slot) of head h."""
    b, s, o = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    _check(_lib.damp_pool_head_layout(pool, h, ctypes.byref(b), ctypes.byref(s),
                                      ctypes.byref(o)), "damp_pool_head_layout")
    return b.value, s.value, o.value


def damp_pool_destroy(pool: int) -> None:
    _check(_lib.damp_pool_destroy(pool), "damp_pool_destroy")
    _POOLS.pop(pool, None)


def damp_pool_block_offset(pool: int, slot: int, h: int) -> int:
    o = ctypes.c_size_t()
    _check(_lib.damp_pool_block_offset(pool, slot, h, ctypes.byref(o)), "damp_pool_block_offset")
    return o.value


def damp_block_to_logical(pool: int, h: int, block, fmt: int, d_k: int,
                          d_v: int | None = None) -> dict:
    """Logical per-row form of one raw block (host bytes)."""
    d_v = d_k if d_v is None else d_v
    block = np.ascontiguousarray(np.frombuffer(bytes(block), np.uint8))
    if fmt == DAMP_FMT_FP32:
        f32 = np.empty((d_k, d_v), np.float32)
        _check(_lib.damp_block_to_logical(pool, h, _ptr(block), None, None, None, _ptr(f32)),
               "damp_block_to_logical")
        return {"f32": f32}
    scale = np.empty(d_k, np.float32)
    half = np.empty((d_k, d_v), np.uint16)
    code = np.empty((d_k, d_v), np.int8)
    _check(_lib.damp_block_to_logical(pool, h, _ptr(block), _ptr(scale), _ptr(half), _ptr(code),
                                      None), "damp_block_to_logical")
    return {"scale": scale, "half": half, "code": code}


def damp_pool_read_raw(pool: int, slot: int, h: int) -> dict:
    """Block (slot, h) in its logical form, read from the device (host arrays:
    f32 [d_k][d_v], or scale [d_k], half [d_k][d_v], code [d_k][d_v])."""
    fmt, _, _, d_k, d_v = _pool_shape(pool)
    if fmt == DAMP_FMT_FP32:
        out = np.empty(4 * d_k * d_v, np.uint8)
    else:
        out = np.empty(4 * d_k + 3 * d_k * d_v, np.uint8)
    _check(_lib.damp_pool_read_raw(pool, slot, h, _ptr(out)), "damp_pool_read_raw")
    if fmt == DAMP_FMT_FP32:
        return {"f32": out.view(np.float32).reshape(d_k, d_v)}
    ne = d_k * d_v
    return {"scale": out[:4 * d_k].view(np.float32).copy(),
            "half": out[4 * d_k:4 * d_k + 2 * ne].view(np.uint16).reshape(d_k, d_v).copy(),
            "code": out[4 * d_k + 2 * ne:].view(np.int8).reshape(d_k, d_v).copy()}


def damp_block_from_logical(pool: int, h: int, stride: int, scale=None, half=None, code=None,
                            f32=None) -> np.ndarray:
    out = np.zeros(stride, np.uint8)
    c = lambda a, t: None if a is None else np.ascontiguousarray(a, t)
    scale, half, code, f32 = (c(scale, np.float32), c(half, np.uint16), c(code, np.int8),
                              c(f32, np.float32))
    _check(_lib.damp_block_from_logical(pool, h, _ptr(scale), _ptr(half), _ptr(code), _ptr(f32),
                                        _ptr(out)), "damp_block_from_logical")
    return out


# ---------------------------------------------------------------- device calls

def _codec_args(pool, slot_idx, state, stream, where):
    _, _, H, d_k, d_v = _pool_shape(pool)
    if not isinstance(slot_idx, torch.Tensor) or slot_idx.dim() != 1:
        raise ValueError(f"{where}: slot_idx must be a 1-D tensor")
    _shape(state, "state", (slot_idx.numel(), H, d_k, d_v))
    _cuda(slot_idx, torch.int32, "slot_idx")
    _cuda(state, torch.float32, "state")
    _same_device(stream, slot_idx, state)


def damp_pool_pack(pool: int, slot_idx: torch.Tensor, state: torch.Tensor, stream=None) -> None:
    """Compress FP32 states [n][H][d_k][d_v] into the slots slot_idx [n]."""
    _codec_args(pool, slot_idx, state, stream, "damp_pool_pack")
    _check(_lib.damp_pool_pack(pool, slot_idx.numel(), _ptr(slot_idx), _ptr(state),
                               _stream(stream, state.device)), "damp_pool_pack")


def damp_pool_unpack(pool: int, slot_idx: torch.Tensor, state: torch.Tensor, stream=None) -> None:
    """Reconstruct FP32 states [n][H][d_k][d_v] of the slots slot_idx [n]."""
    _codec_args(pool, slot_idx, state, stream, "damp_pool_unpack")
    _check(_lib.damp_pool_unpack(pool, slot_idx.numel(), _ptr(slot_idx), _ptr(state),
                                 _stream(stream, state.device)), "damp_pool_unpack")


def _step_args(pool, slot_idx, q, k, v, alpha, beta, out, stream):
    """Check every tensor against the pool's (H, d_k, d_v) and the batch size
    n = slot_idx.numel() before anything is enqueued; returns (dtype, gate)."""
    _, _, H, d_k, d_v = _pool_shape(pool)
    if not isinstance(slot_idx, torch.Tensor) or slot_idx.dim() != 1:
        raise ValueError("slot_idx must be a 1-D tensor")
    n = slot_idx.numel()
    _shape(q, "q", (n, H, d_k))
    _shape(k, "k", (n, H, d_k))
    _shape(v, "v", (n, H, d_v))
    _shape(beta, "beta", (n, H))
    _shape(out, "out", (n, H, d_v))
    if tuple(alpha.shape) == (n, H, d_k) and alpha.dim() == 3:
        gate = DAMP_GATE_VECTOR
    elif tuple(alpha.shape) == (n, H):
        gate = DAMP_GATE_SCALAR
    else:
        raise ValueError(f"alpha must have shape {(n, H)} (GDN) or {(n, H, d_k)} (KDA), "
                         f"got {tuple(alpha.shape)}")
    _cuda(slot_idx, torch.int32, "slot_idx")
    _cuda(q, None, "q")
    if q.dtype == torch.bfloat16:
        dt = DAMP_DTYPE_BF16
    elif q.dtype == torch.float32:
        dt = DAMP_DTYPE_F32
    else:
        raise ValueError("q, k, v must be bfloat16 or float32")
    _cuda(k, q.dtype, "k")
    _cuda(v, q.dtype, "v")
    _cuda(alpha, torch.float32, "alpha")
    _cuda(beta, torch.float32, "beta")
    _cuda(out, torch.float32, "out")
    _same_device(stream, slot_idx, q, k, v, alpha, beta, out)
    return dt, gate


def damp_decode_step(pool: int, slot_idx: torch.Tensor, q: torch.Tensor, k: torch.Tensor,
                     v: torch.Tensor, alpha: torch.Tensor, beta: torch.Tensor, out: torch.Tensor,
                     stream=None) -> None:
    """One decode step.  q, k [n][H][d_k] and v [n][H][d_v] in bf16 or fp32;
    alpha fp32 [n][H] (GDN) or [n][H][d_k] (KDA); beta fp32 [n][H]; out fp32
    [n][H][d_v]; n = slot_idx.numel()."""
    dt, gate = _step_args(pool, slot_idx, q, k, v, alpha, beta, out, stream)
    _check(_lib.damp_decode_step(pool, slot_idx.numel(), _ptr(slot_idx), dt, _ptr(q), _ptr(k),
                                 _ptr(v), gate, _ptr(alpha), _ptr(beta), _ptr(out),
                                 _stream(stream, q.device)), "damp_decode_step")


def damp_decode_step_validated(pool: int, slot_idx: torch.Tensor, q: torch.Tensor,
                               k: torch.Tensor, v: torch.Tensor, alpha: torch.Tensor,
                               beta: torch.Tensor, out: torch.Tensor, stream=None) -> None:
    """damp_decode_step that skips (and flags with DAMP_EFLAG_NONFINITE) every
    unit whose inputs hold a NaN or an infinity."""
    dt, gate = _step_args(pool, slot_idx, q, k, v, alpha, beta, out, stream)
    _check(_lib.damp_decode_step_validated(pool, slot_idx.numel(), _ptr(slot_idx), dt, _ptr(q),
                                           _ptr(k), _ptr(v), gate, _ptr(alpha), _ptr(beta),
                                           _ptr(out), _stream(stream, q.device)),
           "damp_decode_step_validated")


def damp_set_test_hooks(wait_limit_ns: int = 0, hooks: int = 0) -> None:
    """Test hooks of the failure path (process-wide): the bound of the decode
    step's internal waits (0 = default, 2 s) and DAMP_HOOK_HOLD_FIRST_ITEM."""
    _check(_lib.damp_set_test_hooks(int(wait_limit_ns), int(hooks)), "damp_set_test_hooks")


def damp_validate_slots(slot_idx, n_slots: int) -> None:
    """Host check of a batch's slot indices (distinct, below n_slots; negative
    entries are padding).  Raises DampError naming the first bad entry."""
    if isinstance(slot_idx, torch.Tensor):
        slot_idx = slot_idx.detach().cpu().numpy()
    s = np.ascontiguousarray(slot_idx, np.int32)
    bad = ctypes.c_int(-1)
    rc = _lib.damp_validate_slots(_ptr(s), s.size, n_slots, ctypes.byref(bad))
    if rc != DAMP_OK:
        raise DampError(rc, f"damp_validate_slots (entry {bad.value})")


def damp_pool_get_error(pool: int, clear: bool = False, stream=None, device=None) -> int:
    f = ctypes.c_uint32()
    _check(_lib.damp_pool_get_error(pool, ctypes.byref(f), int(bool(clear)),
                                    _stream(stream, device)), "damp_pool_get_error")
    return f.value


# ---------------------------------------------------------------- calibration

def damp_calib_bytes(H: int, d_k: int) -> int:
    return int(_lib.damp_calib_bytes(H, d_k))


def calib_acc(H: int, d_k: int, device="cuda") -> torch.Tensor:
    """Zeroed calibration accumulator (float64): energy [H][d_k], retention
    [H][d_k], count [H]."""
    return torch.zeros(damp_calib_bytes(H, d_k) // 8, dtype=torch.float64, device=device)


def damp_calib_accumulate(pool: int, slot_idx: torch.Tensor, alpha: torch.Tensor,
                          acc: torch.Tensor, stream=None) -> None:
    """Add one step's records of an FP32 pool (states after the step)."""
    fmt, _, H, d_k, _ = _pool_shape(pool)
    if fmt != DAMP_FMT_FP32:
        raise ValueError("damp_calib_accumulate records an FP32 pool")
    if not isinstance(slot_idx, torch.Tensor) or slot_idx.dim() != 1:
        raise ValueError("slot_idx must be a 1-D tensor")
    n = slot_idx.numel()
    if tuple(alpha.shape) == (n, H, d_k) and alpha.dim() == 3:
        gate = DAMP_GATE_VECTOR
    elif tuple(alpha.shape) == (n, H):
        gate = DAMP_GATE_SCALAR
    else:
        raise ValueError(f"alpha must have shape {(n, H)} or {(n, H, d_k)}")
    _shape(acc, "acc", (damp_calib_bytes(H, d_k) // 8,))
    _cuda(slot_idx, torch.int32, "slot_idx")
    _cuda(alpha, torch.float32, "alpha")
    _cuda(acc, torch.float64, "acc")
    _same_device(stream, slot_idx, alpha, acc)
    _check(_lib.damp_calib_accumulate(pool, slot_idx.numel(), _ptr(slot_idx), gate, _ptr(alpha),
                                      _ptr(acc), _stream(stream, acc.device)),
           "damp_calib_accumulate")


def damp_calib_select(H: int, d_k: int, hp_rows: int, acc: torch.Tensor, score=None,
                      hp_row_idx=None, stream=None):
    """Per-head selection; returns (hp_row_idx [H][hp_rows], score float64
    [H][d_k]).  Row indices are int16 (every index is below d_k <= 128)."""
    _cuda(acc, torch.float64, "acc")
    if score is None:
        score = torch.empty((H, d_k), dtype=torch.float64, device=acc.device)
    if hp_row_idx is None:
        hp_row_idx = torch.empty((H, hp_rows), dtype=torch.int16, device=acc.device)
    _cuda(score, torch.float64, "score")
    _cuda(hp_row_idx, torch.int16, "hp_row_idx")
    _check(_lib.damp_calib_select(H, d_k, hp_rows, _ptr(acc), _ptr(score), _ptr(hp_row_idx),
                                  _stream(stream, acc.device)), "damp_calib_select")
    return hp_row_idx, score


def damp_calib_select_budget(H: int, d_k: int, budget: int, acc: torch.Tensor, stream=None):
    """Selection under a budget shared by all heads; returns (is_fp16 uint8
    [H][d_k], hp_per_head int32 [H], score float64 [H][d_k])."""
    _cuda(acc, torch.float64, "acc")
    score = torch.empty((H, d_k), dtype=torch.float64, device=acc.device)
    is16 = torch.empty((H, d_k), dtype=torch.uint8, device=acc.device)
    hp = torch.empty(H, dtype=torch.int32, device=acc.device)
    _check(_lib.damp_calib_select_budget(H, d_k, budget, _ptr(acc), _ptr(score), _ptr(is16),
                                         _ptr(hp), _stream(stream, acc.device)),
           "damp_calib_select_budget")
    return is16, hp, score


DAMP_SELECT_BUDGET_STATIC_MAX = 16384


def damp_calib_select_budget_static(H: int, d_k: int, budget: int, acc: torch.Tensor,
                                    is_fp16: torch.Tensor, hp_per_head: torch.Tensor,
                                    stream=None) -> None:
    """Budget selection that allocates nothing: for callers that cannot
    allocate device memory at selection time (every free byte already handed
    to the state pools, or a host with no allocator that only holds buffers
    it was given).  The caller passes the outputs, is_fp16 uint8 [H][d_k] and
    hp_per_head int32 [H]; the scores go to the library's static device array
    (H * d_k <= DAMP_SELECT_BUDGET_STATIC_MAX).  Calls that overlap on the GPU
    share that array and race: keep them on one stream."""
    _cuda(acc, torch.float64, "acc")
    _cuda(is_fp16, torch.uint8, "is_fp16")
    _cuda(hp_per_head, torch.int32, "hp_per_head")
    if is_fp16.numel() != H * d_k or hp_per_head.numel() != H:
        raise ValueError("is_fp16 must hold H*d_k bytes and hp_per_head H entries")
    _check(_lib.damp_calib_select_budget_static(H, d_k, budget, _ptr(acc), _ptr(is_fp16),
                                                _ptr(hp_per_head), _stream(stream, acc.device)),
           "damp_calib_select_budget_static")


# ---------------------------------------------------------------- convenience

class DampPool:
    """A pool buffer (allocated by PyTorch) bound to a libdamp descriptor.

    ``hp_row_idx`` [H][hp] gives every head the same FP16-row count;
    ``fp16_map`` [H][d] (0/1, mixed format only) lets the count differ per
    head."""

    def __init__(self, fmt, n_slots: int, H: int, d: int, hp_row_idx=None,
                 device="cuda", fp16_map=None, d_v: int | None = None):
        self.fmt = FORMATS[fmt] if isinstance(fmt, str) else int(fmt)
        d_v = d if d_v is None else d_v
        self.n_slots, self.H, self.d, self.d_k, self.d_v = n_slots, H, d, d, d_v
        if fp16_map is not None:
            if self.fmt != DAMP_FMT_MIXED:
                raise ValueError("an FP16-row map needs the mixed format")
            fp16_map = np.ascontiguousarray(fp16_map, np.uint8).reshape(H, d)
            self.nbytes = damp_pool_bytes_map(n_slots, H, d, d_v, fp16_map)
            self.buf = torch.empty(self.nbytes, dtype=torch.uint8, device=device)
            self.handle = damp_pool_create_map(n_slots, H, d, d_v, fp16_map, self.buf)
            counts = fp16_map.sum(axis=1)
            self.hp = int(counts[0]) if (counts == counts[0]).all() else -1
        else:
            hp_row_idx = None if hp_row_idx is None else np.asarray(hp_row_idx).reshape(H, -1)
            self.hp = 0 if hp_row_idx is None else hp_row_idx.shape[1]
            self.nbytes = damp_pool_bytes(self.fmt, n_slots, H, d, d_v, self.hp)
            self.buf = torch.empty(self.nbytes, dtype=torch.uint8, device=device)
            self.handle = damp_pool_create(self.fmt, n_slots, H, d, d_v, self.hp, hp_row_idx,
                                           self.buf)
        self.header_bytes = damp_pool_block_offset(self.handle, 0, 0)
        self.heads = [damp_pool_head_layout(self.handle, h) for h in range(H)]
        self.slot_stride = sum(st for _, st, _ in self.heads)
        strides = {st for _, st, _ in self.heads}
        self.block_stride = max(strides)
        self.block_bytes = max(b for b, _, _ in self.heads)
        self.uniform = len(strides) == 1

    def close(self):
        if getattr(self, "handle", None):
            damp_pool_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def slots(self) -> torch.Tensor:
        """View of the slot area: uint8 [n_slots][slot_stride]."""
        return self.buf[self.header_bytes:].view(self.n_slots, self.slot_stride)

    def blocks(self) -> torch.Tensor:
        """View of the blocks: uint8 [n_slots][H][block_stride] (every head the
        same block size)."""
        if not self.uniform:
            raise ValueError("heads differ in block size; use slots() / block()")
        return self.slots().view(self.n_slots, self.H, self.block_stride)

    def block(self, slot: int, h: int) -> torch.Tensor:
        """View of block (slot, h): uint8 [head block stride]."""
        _, st, off = self.heads[h]
        return self.slots()[slot, off:off + st]

    def pack(self, slot_idx, state, stream=None):
        damp_pool_pack(self.handle, slot_idx, state, stream)

    def unpack(self, slot_idx, state, stream=None):
        damp_pool_unpack(self.handle, slot_idx, state, stream)

    def step(self, slot_idx, q, k, v, alpha, beta, out, stream=None, validate=False,
             check_inputs=False):
        """One decode step; ``validate`` first checks the slot indices on the
        host (a device-to-host copy: for debugging, not the serving path);
        ``check_inputs`` skips and flags units with non-finite inputs on the
        device (damp_decode_step_validated)."""
        if validate:
            damp_validate_slots(slot_idx, self.n_slots)
        f = damp_decode_step_validated if check_inputs else damp_decode_step
        f(self.handle, slot_idx, q, k, v, alpha, beta, out, stream)

    def get_error(self, clear=False, stream=None) -> int:
        return damp_pool_get_error(self.handle, clear, stream, self.buf.device)

    def read_logical(self, slots=None) -> dict:
        """Logical form of blocks [len(slots)][H] (host numpy)."""
        slots = list(range(self.n_slots)) if slots is None else [int(x) for x in slots]
        raw = self.slots()[torch.as_tensor(slots, device=self.buf.device)].cpu().numpy()
        out = None
        for i in range(len(slots)):
            for h in range(self.H):
                _, st, off = self.heads[h]
                lg = damp_block_to_logical(self.handle, h, raw[i, off:off + st], self.fmt,
                                           self.d_k, self.d_v)
                if out is None:
                    out = {k: np.empty((len(slots), self.H) + v.shape, v.dtype)
                           for k, v in lg.items()}
                for k_, v_ in lg.items():
                    out[k_][i, h] = v_
        return out

    def write_logical(self, slot: int, logical: dict):
        """Write the logical form [H][...] of one slot into the pool (host -> device)."""
        raw = np.concatenate([damp_block_from_logical(self.handle, h, self.heads[h][1],
                                                      **{k: v[h] for k, v in logical.items()})
                              for h in range(self.H)])
        self.slots()[slot].copy_(torch.from_numpy(raw))

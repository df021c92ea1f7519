"""Python binding of libstq.so (include/stq.h): argument marshalling only.

Every function keeps the C name and forwards to the CUDA library; torch is
used for device memory (``data_ptr()``) and streams (``cuda_stream``).  There
is no fallback: if libstq.so is missing or fails to load, every call raises.
"""
from __future__ import annotations

import ctypes as C
import os

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libstq.so")

STQ_GDN, STQ_KDA = 0, 1
STQ_SCALE_F16 = 1  # desc flag: per-row scales stored as IEEE binary16
STQ_FIT_COLUMNS = 2  # desc flag: per-page column factors refitted at every quantisation
STQ_ALLOC_DP, STQ_ALLOC_LAGRANGE = 0, 1  # bit allocation methods
STATUS = {0: "STQ_OK", 1: "STQ_ERR_ARG", 2: "STQ_ERR_OOM", 3: "STQ_ERR_CUDA", 4: "STQ_ERR_INDEX",
          5: "STQ_ERR_NONFINITE", 6: "STQ_ERR_UNSUPPORTED", 7: "STQ_ERR_TIMEOUT"}
STQ_OK, STQ_ERR_ARG, STQ_ERR_OOM, STQ_ERR_CUDA, STQ_ERR_INDEX, STQ_ERR_NONFINITE, \
    STQ_ERR_UNSUPPORTED, STQ_ERR_TIMEOUT = range(8)

# every symbol include/stq.h declares
EXPORTS = ("stq_pool_create", "stq_pool_destroy", "stq_pool_bytes", "stq_desc_bytes",
           "stq_page_layout", "stq_quantize_state", "stq_dequantize_state", "stq_decode_step",
           "stq_decode_readout", "stq_decode_writeback", "stq_decode_step_split", "stq_pool_join",
           "stq_decode_step_static", "stq_decode_step_host", "stq_host_block_layout",
           "stq_decode_step_host_block", "stq_lifetime_weight", "stq_allocate_bits",
           "stq_export_slot", "stq_import_slot", "stq_pool_check", "stq_launch_count",
           "stq_status_str", "stq_last_error")


class StqError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS.get(status, status)}: {msg}")
        self.status = status


class _Desc(C.Structure):
    _fields_ = [("kind", C.c_int32), ("num_requests", C.c_int32), ("num_slots", C.c_int32),
                ("num_heads", C.c_int32), ("d_k", C.c_int32), ("d_v", C.c_int32),
                ("unit_bits", C.c_void_p), ("row_factor", C.c_void_p), ("col_factor", C.c_void_p),
                ("flags", C.c_uint32), ("row_weight", C.c_void_p)]


_lib = None


def load():
    """Load libstq.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m quantized_linear_attention_decode_b200.build`")
    L = C.CDLL(LIB_PATH)
    P, I32, SZ = C.c_void_p, C.c_int32, C.c_size_t
    sig = {
        "stq_pool_create": [P, P],
        "stq_pool_destroy": [P],
        "stq_pool_bytes": [P, P, P],
        "stq_desc_bytes": [P, P, P],
        "stq_page_layout": [P, I32, P, P],
        "stq_quantize_state": [P, P, P, I32, P, P],
        "stq_dequantize_state": [P, P, P, I32, P, P],
        "stq_decode_step": [P, P, P, I32, P, P, P, P, P, P, P],
        "stq_decode_step_host": [P, P, P, I32, P, P, P, P, P, P, P],
        "stq_host_block_layout": [P, I32, P, P],
        "stq_decode_step_host_block": [P, I32, P, SZ, P, P],
        "stq_decode_readout": [P, P, P, I32, P, P, P, P, P, P, P, P],
        "stq_decode_writeback": [P, P, P, I32, P, P, P, P],
        "stq_decode_step_split": [P, P, P, I32, P, P, P, P, P, P, P, P, P],
        "stq_pool_join": [P, P],
        "stq_decode_step_static": [P, P, P, I32, P, P, P, P, P, P, P],
        "stq_lifetime_weight": [I32, P, I32, P],
        "stq_allocate_bits": [I32, P, I32, P, P, P, C.c_double, I32, I32, C.c_uint8, P, P],
        "stq_export_slot": [P, I32, I32, P, SZ],
        "stq_import_slot": [P, I32, I32, P, SZ],
        "stq_pool_check": [P, P],
    }
    for name, args in sig.items():
        f = getattr(L, name)
        f.argtypes = args
        f.restype = C.c_int
    L.stq_launch_count.argtypes = []
    L.stq_launch_count.restype = C.c_uint64
    L.stq_status_str.argtypes = [C.c_int]
    L.stq_status_str.restype = C.c_char_p
    L.stq_last_error.argtypes = []
    L.stq_last_error.restype = C.c_char_p
    _lib = L
    return L


def _check(st: int) -> None:
    if st != STQ_OK:
        raise StqError(st, load().stq_last_error().decode())


def _stream(stream) -> C.c_void_p:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, int):
        return C.c_void_p(stream)
    return C.c_void_p(stream.cuda_stream)


def _dev(t, dtype, shape=None, name="tensor"):
    import torch
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be on a CUDA device")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    return C.c_void_p(t.data_ptr())


def _desc(kind, R, S, H, unit_bits, row_factor, col_factor, keep, flags=0, row_weight=None):
    ub = np.ascontiguousarray(unit_bits, np.uint8)
    rf = None if row_factor is None else np.ascontiguousarray(row_factor, np.float32)
    cf = None if col_factor is None else np.ascontiguousarray(col_factor, np.float32)
    rw = None if row_weight is None else np.ascontiguousarray(row_weight, np.float32)
    keep.extend([ub, rf, cf, rw])
    ptr = lambda a: None if a is None else a.ctypes.data  # noqa: E731
    return _Desc(int(kind), int(R), int(S), int(H), 128, 128, ptr(ub), ptr(rf), ptr(cf), int(flags), ptr(rw))


class Pool:
    """Owner of one stq_pool handle (destroyed with the object)."""

    def __init__(self, handle, kind, R, S, H, unit_bits, flags=0):
        self.handle = handle
        self.kind, self.R, self.S, self.H = kind, R, S, H
        self.unit_bits = np.asarray(unit_bits, np.uint8).copy()
        self.flags = int(flags)

    def __del__(self):
        self.close()

    def close(self):
        h = getattr(self, "handle", None)
        self.handle = None
        if h and _lib is not None:
            try:
                _lib.stq_pool_destroy(h)
            except Exception:  # noqa: BLE001  (interpreter shutdown)
                pass

    @property
    def row_bits(self) -> np.ndarray:
        if self.kind == STQ_GDN:
            return np.repeat(self.unit_bits.reshape(-1, 1), 128, axis=1)
        return self.unit_bits.reshape(self.H, 128)

    @property
    def slot_bytes(self) -> int:
        return stq_pool_bytes(self)[1]


def stq_pool_create(kind, num_requests, num_slots, num_heads, unit_bits, row_factor=None,
                    col_factor=None, flags=0, row_weight=None) -> Pool:
    keep = []
    d = _desc(kind, num_requests, num_slots, num_heads, unit_bits, row_factor, col_factor, keep, flags,
              row_weight)
    h = C.c_void_p()
    _check(load().stq_pool_create(C.byref(d), C.byref(h)))
    return Pool(h, kind, num_requests, num_slots, num_heads, unit_bits, flags)


def stq_pool_destroy(pool: Pool) -> None:
    pool.close()


def stq_pool_bytes(pool: Pool):
    a, b = C.c_size_t(), C.c_size_t()
    _check(load().stq_pool_bytes(pool.handle, C.byref(a), C.byref(b)))
    return a.value, b.value


def stq_desc_bytes(kind, num_requests, num_slots, num_heads, unit_bits, row_factor=None,
                   col_factor=None, flags=0, row_weight=None):
    keep = []
    d = _desc(kind, num_requests, num_slots, num_heads, unit_bits, row_factor, col_factor, keep, flags,
              row_weight)
    a, b = C.c_size_t(), C.c_size_t()
    _check(load().stq_desc_bytes(C.byref(d), C.byref(a), C.byref(b)))
    return a.value, b.value


def stq_page_layout(pool: Pool, head: int):
    a, b = C.c_size_t(), C.c_size_t()
    _check(load().stq_page_layout(pool.handle, int(head), C.byref(a), C.byref(b)))
    return a.value, b.value


def _idx(pool, req_idx, slot_idx):
    import torch
    n = int(req_idx.numel())
    return (n, _dev(req_idx, torch.int32, (n,), "req_idx"), _dev(slot_idx, torch.int32, (n,), "slot_idx"))


def stq_quantize_state(pool: Pool, req_idx, slot_idx, state, stream=None) -> None:
    import torch
    n, r, s = _idx(pool, req_idx, slot_idx)
    st = _dev(state, torch.float32, (n, pool.H, 128, 128), "state")
    _check(load().stq_quantize_state(pool.handle, r, s, n, st, _stream(stream)))


def stq_dequantize_state(pool: Pool, req_idx, slot_idx, state_out, stream=None) -> None:
    import torch
    n, r, s = _idx(pool, req_idx, slot_idx)
    st = _dev(state_out, torch.float32, (n, pool.H, 128, 128), "state_out")
    _check(load().stq_dequantize_state(pool.handle, r, s, n, st, _stream(stream)))


def stq_decode_step(pool: Pool, req_idx, slot_idx, q, k, v, beta, gate, y, stream=None) -> None:
    import torch
    n, r, s = _idx(pool, req_idx, slot_idx)
    f = torch.float32
    vec = (n, pool.H, 128)
    gshape = (n, pool.H) if pool.kind == STQ_GDN else vec
    _check(load().stq_decode_step(
        pool.handle, r, s, n, _dev(q, f, vec, "q"), _dev(k, f, vec, "k"), _dev(v, f, vec, "v"),
        _dev(beta, f, (n, pool.H), "beta"), _dev(gate, f, gshape, "gate"), _dev(y, f, vec, "y"),
        _stream(stream)))


def _host(t, dtype, shape, name):
    import torch
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch tensor")
    if t.device.type != "cpu":
        raise ValueError(f"{name} must be in host memory (pinned for overlapped copies)")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    return C.c_void_p(t.data_ptr())


def stq_decode_step_host(pool: Pool, req_idx, slot_idx, q, k, v, beta, gate, y, stream=None) -> None:
    """stq_decode_step with host (CPU) tensors: the library copies the inputs in,
    decodes and copies y out, ordered on `stream`; y is valid once `stream` is
    synchronized.  Keep every tensor referenced (and the inputs unchanged)
    until then: torch may hand a freed pinned block out again before the
    library's copy from it has run."""
    import torch
    n = int(req_idx.numel())
    f = torch.float32
    vec, gshape = _vecs(pool, n)
    _check(load().stq_decode_step_host(
        pool.handle, _host(req_idx, torch.int32, (n,), "req_idx"), _host(slot_idx, torch.int32, (n,), "slot_idx"),
        n, _host(q, f, vec, "q"), _host(k, f, vec, "k"), _host(v, f, vec, "v"),
        _host(beta, f, (n, pool.H), "beta"), _host(gate, f, gshape, "gate"), _host(y, f, vec, "y"),
        _stream(stream)))


def stq_host_block_layout(pool: Pool, n: int):
    """(offsets of req_idx, slot_idx, q, k, v, beta, gate; block bytes) of the
    one-block host layout for n entries."""
    offs = (C.c_size_t * 7)()
    nb = C.c_size_t()
    _check(load().stq_host_block_layout(pool.handle, int(n), offs, C.byref(nb)))
    return [int(o) for o in offs], nb.value


def stq_decode_step_host_block(pool: Pool, n: int, block, y, stream=None) -> None:
    """stq_decode_step_host with every input in one host block (a uint8 CPU
    tensor laid out by stq_host_block_layout): one copy in; a pinned y is written by the
    kernels directly, any other y is copied back."""
    import torch
    if not isinstance(block, torch.Tensor) or block.device.type != "cpu" or block.dtype != torch.uint8 \
            or not block.is_contiguous():
        raise TypeError("block must be a contiguous uint8 CPU tensor")
    vec, _ = _vecs(pool, n)
    _check(load().stq_decode_step_host_block(pool.handle, int(n), C.c_void_p(block.data_ptr()), block.numel(),
                                             _host(y, torch.float32, vec, "y"), _stream(stream)))


def _vecs(pool, n):
    vec = (n, pool.H, 128)
    return vec, ((n, pool.H) if pool.kind == STQ_GDN else vec)


def stq_decode_readout(pool: Pool, req_idx, slot_idx, q, k, v, beta, gate, y, u_tilde, stream=None) -> None:
    import torch
    n, r, s = _idx(pool, req_idx, slot_idx)
    f = torch.float32
    vec, gshape = _vecs(pool, n)
    _check(load().stq_decode_readout(
        pool.handle, r, s, n, _dev(q, f, vec, "q"), _dev(k, f, vec, "k"), _dev(v, f, vec, "v"),
        _dev(beta, f, (n, pool.H), "beta"), _dev(gate, f, gshape, "gate"), _dev(y, f, vec, "y"),
        _dev(u_tilde, f, vec, "u_tilde"), _stream(stream)))


def stq_decode_writeback(pool: Pool, req_idx, slot_idx, k, gate, u_tilde, stream=None) -> None:
    import torch
    n, r, s = _idx(pool, req_idx, slot_idx)
    f = torch.float32
    vec, gshape = _vecs(pool, n)
    _check(load().stq_decode_writeback(
        pool.handle, r, s, n, _dev(k, f, vec, "k"), _dev(gate, f, gshape, "gate"),
        _dev(u_tilde, f, vec, "u_tilde"), _stream(stream)))


def stq_decode_step_split(pool: Pool, req_idx, slot_idx, q, k, v, beta, gate, y, u_tilde, stream=None,
                          side_stream=None) -> None:
    import torch
    n, r, s = _idx(pool, req_idx, slot_idx)
    f = torch.float32
    vec, gshape = _vecs(pool, n)
    _check(load().stq_decode_step_split(
        pool.handle, r, s, n, _dev(q, f, vec, "q"), _dev(k, f, vec, "k"), _dev(v, f, vec, "v"),
        _dev(beta, f, (n, pool.H), "beta"), _dev(gate, f, gshape, "gate"), _dev(y, f, vec, "y"),
        _dev(u_tilde, f, vec, "u_tilde"), _stream(stream), _stream(side_stream)))


def stq_decode_step_static(pool: Pool, req_idx, slot_idx, q, k, v, beta, gate, y, stream=None) -> None:
    """stq_decode_step without any device allocation: u~ lives in the
    library's built-in 4 MiB array (at most 8192 (entry, head) tiles per call;
    calls that overlap on the GPU must be serialized by the caller)."""
    import torch
    n, r, s = _idx(pool, req_idx, slot_idx)
    f = torch.float32
    vec, gshape = _vecs(pool, n)
    _check(load().stq_decode_step_static(
        pool.handle, r, s, n, _dev(q, f, vec, "q"), _dev(k, f, vec, "k"), _dev(v, f, vec, "v"),
        _dev(beta, f, (n, pool.H), "beta"), _dev(gate, f, gshape, "gate"), _dev(y, f, vec, "y"),
        _stream(stream)))


def stq_lifetime_weight(log_retention, horizon: int) -> np.ndarray:
    """L_u = sum_{j < horizon} exp(2 j l_u) for each unit's mean log retention."""
    ell = np.ascontiguousarray(log_retention, np.float64).reshape(-1)
    out = np.empty_like(ell)
    _check(load().stq_lifetime_weight(len(ell), ell.ctypes.data, int(horizon), out.ctypes.data))
    return out


def stq_allocate_bits(unit_values, choices, distortion, weight, mean_bits: float, method: int = STQ_ALLOC_DP,
                      num_pivots: int = 0, pivot_bits: int = 16):
    """Per-unit widths minimising sum L_u d_u(b_u) under the mean-bits budget
    (then the num_pivots riskiest units at pivot_bits); returns (bits, objective)."""
    n = np.ascontiguousarray(unit_values, np.float64).reshape(-1)
    ch = np.ascontiguousarray(choices, np.uint8).reshape(-1)
    d = np.ascontiguousarray(distortion, np.float64).reshape(len(n), len(ch))
    w = np.ascontiguousarray(weight, np.float64).reshape(len(n))
    bits = np.zeros(len(n), np.uint8)
    obj = C.c_double()
    _check(load().stq_allocate_bits(len(n), n.ctypes.data, len(ch), ch.ctypes.data, d.ctypes.data, w.ctypes.data,
                                    float(mean_bits), int(method), int(num_pivots), int(pivot_bits),
                                    bits.ctypes.data, C.byref(obj)))
    return bits, obj.value


def stq_pool_join(pool: Pool, stream=None) -> None:
    _check(load().stq_pool_join(pool.handle, _stream(stream)))


def stq_export_slot(pool: Pool, req: int, slot: int) -> np.ndarray:
    nb = pool.slot_bytes
    out = np.empty(nb, np.uint8)
    _check(load().stq_export_slot(pool.handle, int(req), int(slot), out.ctypes.data, nb))
    return out


def stq_import_slot(pool: Pool, req: int, slot: int, data) -> None:
    data = np.ascontiguousarray(data, np.uint8)
    _check(load().stq_import_slot(pool.handle, int(req), int(slot), data.ctypes.data, data.nbytes))


def stq_pool_check(pool: Pool, stream=None, raise_on_error: bool = True) -> int:
    st = load().stq_pool_check(pool.handle, _stream(stream))
    if raise_on_error:
        _check(st)
    return st


def stq_launch_count() -> int:
    return int(load().stq_launch_count())


def stq_status_str(status: int) -> str:
    return load().stq_status_str(int(status)).decode()


def stq_last_error() -> str:
    return load().stq_last_error().decode()

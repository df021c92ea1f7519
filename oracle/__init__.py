"""CPU oracle for the quantized gated delta-rule decode step (ctypes wrapper).

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  It shares no code
with the CUDA library: the arithmetic lives in ``stq_oracle.c`` (plain C,
fp64 continuous part, fp32 quantisation decision), compiled here with gcc.

Every function follows the page "STEPQuant: When and Where Errors Matter in
Delta-Rule Recurrent State Quantization" (see the header of stq_oracle.c for
the section-by-section citations and the readings taken where it is silent).
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "stq_oracle.c")
_LIB = os.path.join(_HERE, "libstq_oracle.so")
CFLAGS = ["-O2", "-fno-tree-vectorize", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
          "-fPIC", "-shared", "-Wall", "-Wextra"]

OK, NONFINITE, BADARG = 0, 1, 2
_lib = None


def build(force: bool = False) -> str:
    """Compile stq_oracle.c into libstq_oracle.so (if missing or stale)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, _SRC])
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    if _lib is None:
        build()
        L = C.CDLL(_LIB)
        P = C.c_void_p
        L.orc_page_bytes.restype = C.c_size_t
        L.orc_page_bytes.argtypes = [C.c_int, C.c_int, P]
        L.orc_page_bytes_fmt.restype = C.c_size_t
        L.orc_page_bytes_fmt.argtypes = [C.c_int, C.c_int, P, C.c_int]
        L.orc_half_to_double.restype = C.c_double
        L.orc_half_to_double.argtypes = [C.c_uint16]
        L.orc_double_to_half.restype = C.c_uint16
        L.orc_double_to_half.argtypes = [C.c_double]
        L.orc_quantize_unit_fmt.argtypes = [C.c_int, C.c_int, P, P, P, C.c_int, P, P, P]
        L.orc_dequantize_unit_fmt.argtypes = [C.c_int, C.c_int, P, P, P, C.c_int, P, P]
        L.orc_step_unit_fmt.argtypes = [C.c_int, C.c_int, P, P, P, C.c_int, P, P, P, P, P,
                                        C.c_float, P, P, P]
        L.orc_quantize_unit_w.argtypes = [C.c_int, C.c_int, P, P, P, P, C.c_int, P, P, P]
        L.orc_step_unit_w.argtypes = [C.c_int, C.c_int, P, P, P, P, C.c_int, P, P, P, P, P,
                                      C.c_float, P, P, P]
        L.orc_get_code.restype = C.c_int32
        L.orc_get_code.argtypes = [P, C.c_int, C.c_int, C.c_int]
        L.orc_put_code.restype = None
        L.orc_put_code.argtypes = [P, C.c_int, C.c_int, C.c_int, C.c_int32]
        L.orc_quantize_unit.argtypes = [C.c_int, C.c_int, P, P, P, P, P, P]
        L.orc_dequantize_unit.argtypes = [C.c_int, C.c_int, P, P, P, P, P]
        L.orc_step_unit.argtypes = [C.c_int, C.c_int, P, P, P, P, P, P, P, P, C.c_float, P, P, P]
        L.orc_step_unit_f64.argtypes = [C.c_int, C.c_int, P, P, P, P, C.c_float, P, P]
        L.orc_step_many.argtypes = [C.c_int, C.c_int, C.c_int, P, P, P, P, P, P, P, P, P, P, P,
                                    P, P, P, C.c_int]
        L.orc_default_threads.restype = C.c_int
        _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _u8(a):
    return np.ascontiguousarray(a, dtype=np.uint8)


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


def _f64(a):
    return np.ascontiguousarray(a, dtype=np.float64)


# scale formats: fp32 scales (0), IEEE binary16 scales (1); flag FMT_PIVOT (4):
# 16-bit rows are FP16 pivots among quantized rows (scale slot 1, binary16
# mu = X / (r c)).  Without the flag, units whose rows are all 16 or all 32
# bits wide are raw (binary16 / binary32 values, no scales).
FMT_F32, FMT_F16, FMT_PIVOT, FMT_FITC = 0, 1, 4, 8


def is_raw(bits, fmt: int = FMT_F32) -> bool:
    return not (fmt & FMT_PIVOT) and int(np.asarray(bits).reshape(-1)[0]) in (16, 32)


def page_bytes(bits, dv: int | None = None, fmt: int = FMT_F32) -> int:
    bits = _u8(bits)
    dv = len(bits) if dv is None else dv
    return int(lib().orc_page_bytes_fmt(len(bits), dv, _p(bits), int(fmt)))


def row_offsets(bits, dv: int | None = None, fmt: int = FMT_F32) -> np.ndarray:
    """Byte offset of every packed row inside a page (scales come first)."""
    bits = np.asarray(bits, dtype=np.int64)
    dv = len(bits) if dv is None else dv
    sizes = dv * bits // 8
    sb = 0 if is_raw(bits, fmt) else (2 if fmt & FMT_F16 else 4)
    cf = 4 * dv if fmt & FMT_FITC else 0  # the page's own column factors
    return sb * len(bits) + cf + np.concatenate([[0], np.cumsum(sizes)[:-1]])


def half_to_double(h: int) -> float:
    """The value of the binary16 bit pattern h (the oracle's own decoder)."""
    return float(lib().orc_half_to_double(int(h)))


def double_to_half(x: float) -> int:
    """x rounded once to binary16, ties to even (the oracle's own encoder)."""
    return int(lib().orc_double_to_half(float(x)))


def get_code(row: np.ndarray, b: int, j: int, dv: int = 128) -> int:
    """Code j of a packed row of dv codes of b bits."""
    row = _u8(row)
    return int(lib().orc_get_code(_p(row), b, dv, j))


def put_code(row: np.ndarray, b: int, j: int, z: int, dv: int = 128) -> None:
    assert row.dtype == np.uint8 and row.flags.c_contiguous
    lib().orc_put_code(_p(row), b, dv, j, int(z))


def quantize_unit(bits, r, c, S, *, with_quot: bool = False, fmt: int = FMT_F32, w=None):
    """fp32 state [dk, dv] -> packed page (uint8).  Optionally the fp32
    quotients mu / s the codes were rounded from.  w: row weights of the
    column fit (FMT_FITC; None for 1)."""
    bits, r, c, S = _u8(bits), _f32(r), _f32(c), _f32(S)
    w = None if w is None else _f32(w)
    dk, dv = S.shape
    page = np.zeros(page_bytes(bits, dv, fmt), np.uint8)
    quot = np.zeros((dk, dv), np.float32) if with_quot else None
    st = lib().orc_quantize_unit_w(dk, dv, _p(bits), _p(r), _p(c), _p(w), int(fmt), _p(S), _p(page),
                                   _p(quot))
    if st == BADARG:
        raise ValueError("bad bit widths")
    return (page, quot, st) if with_quot else page


def dequantize_unit(bits, r, c, page, dv: int | None = None, fmt: int = FMT_F32) -> np.ndarray:
    bits, r, c, page = _u8(bits), _f32(r), _f32(c), _u8(page)
    dk = len(bits)
    dv = dk if dv is None else dv
    S = np.zeros((dk, dv), np.float32)
    st = lib().orc_dequantize_unit_fmt(dk, dv, _p(bits), _p(r), _p(c), int(fmt), _p(page), _p(S))
    if st == BADARG:
        raise ValueError("bad bit widths")
    return S


def step_unit(bits, r, c, page_in, q, k, v, beta, g, dv: int | None = None, fmt: int = FMT_F32, w=None):
    """One quantized decode step of one unit.

    Returns (page_out uint8, y float64 [dv], quot float32 [dk, dv], status).
    For a raw unit quot holds fl32(X), the value before its rounding on store."""
    bits, r, c, page_in = _u8(bits), _f32(r), _f32(c), _u8(page_in)
    q, k, v, g = _f32(q), _f32(k), _f32(v), _f32(g)
    w = None if w is None else _f32(w)
    dk = len(bits)
    dv = len(v) if dv is None else dv
    if g.size == 1:
        g = np.full(dk, g.reshape(()), np.float32)
    page_out = np.zeros(page_bytes(bits, dv, fmt), np.uint8)
    y = np.zeros(dv, np.float64)
    quot = np.zeros((dk, dv), np.float32)
    st = lib().orc_step_unit_w(dk, dv, _p(bits), _p(r), _p(c), _p(w), int(fmt), _p(page_in),
                               _p(page_out), _p(q), _p(k), _p(v), float(beta), _p(g), _p(y),
                               _p(quot))
    if st == BADARG:
        raise ValueError("bad bit widths")
    return page_out, y, quot, st


def step_unit_f64(S, q, k, v, beta, g):
    """Unquantized recurrence in fp64.  Returns (S_new float64, y float64)."""
    S = np.array(S, dtype=np.float64, order="C", copy=True)
    q, k, v, g = _f32(q), _f32(k), _f32(v), _f32(g)
    dk, dv = S.shape
    if g.size == 1:
        g = np.full(dk, g.reshape(()), np.float32)
    y = np.zeros(dv, np.float64)
    lib().orc_step_unit_f64(dk, dv, _p(S), _p(q), _p(k), _p(v), float(beta), _p(g), _p(y))
    return S, y


def step_many(head, bits_table, r_table, c_table, pages_in, off_in, off_out, out_size,
              q, k, v, beta, g, nthreads: int = 0):
    """Many units (OpenMP over units).  Tables are per head: bits [H, dk],
    r [H, dk], c [H, dv].  Returns (pages_out uint8, y float64 [n, dv], bad)."""
    head = np.ascontiguousarray(head, np.int32)
    bits_table, r_table, c_table = _u8(bits_table), _f32(r_table), _f32(c_table)
    pages_in = _u8(pages_in)
    off_in = np.ascontiguousarray(off_in, np.int64)
    off_out = np.ascontiguousarray(off_out, np.int64)
    q, k, v, beta, g = _f32(q), _f32(k), _f32(v), _f32(beta), _f32(g)
    n = len(head)
    dk = bits_table.shape[1]
    dv = c_table.shape[1]
    pages_out = np.zeros(out_size, np.uint8)
    y = np.zeros((n, dv), np.float64)
    bad = lib().orc_step_many(n, dk, dv, _p(head), _p(bits_table), _p(r_table), _p(c_table),
                              _p(pages_in), _p(off_in), _p(pages_out), _p(off_out), _p(q), _p(k),
                              _p(v), _p(beta), _p(g), _p(y), int(nthreads))
    return pages_out, y, int(bad)


def default_threads() -> int:
    return int(lib().orc_default_threads())


def near_tie(quot: np.ndarray, rel: float = 1e-4) -> np.ndarray:
    """Elements whose quotient lies within rel * |x| of a half-integer."""
    x = np.asarray(quot, np.float64)
    frac = np.abs(x - np.floor(x) - 0.5)
    return frac <= rel * np.maximum(np.abs(x), 1.0)


# ---------------------------------------------------------------- bit allocation (pure Python, tiny cases)


def lifetime_weight_sum(ell: float, horizon: int) -> float:
    """L_u = sum_{j=0}^{H-1} exp(2 j l_u), term by term ("core innovation",
    first point: an error's square decays by exp(2 l_u) per step)."""
    import math
    return math.fsum(math.exp(2.0 * j * ell) for j in range(horizon))


def allocate_brute_force(unit_values, choices, distortion, weight, mean_bits, max_cost=None):
    """Every assignment of widths to units (tiny instances only): the minimum
    of sum_u L_u d_u(b_u) subject to sum_u n_u b_u <= mean_bits sum_u n_u
    (Eq. 8), or <= max_cost when given.  Returns (objective, widths) of the
    cheapest minimiser, or (inf, None) if nothing fits."""
    import itertools
    n = [float(x) for x in unit_values]
    budget = mean_bits * sum(n) if max_cost is None else max_cost
    best, best_cost, arg = float("inf"), float("inf"), None
    for pick in itertools.product(range(len(choices)), repeat=len(n)):
        cost = sum(n[u] * choices[k] for u, k in enumerate(pick))
        if cost > budget * (1 + 1e-12):
            continue
        f = sum(weight[u] * distortion[u][k] for u, k in enumerate(pick))
        if f < best or (f == best and cost < best_cost):
            best, best_cost, arg = f, cost, [choices[k] for k in pick]
    return best, arg


"""Seeded synthetic inputs for the quantized gated delta-rule decode step.

This module only draws numbers: it holds none of the method's arithmetic
(no quantizer, no recurrence, no packing).  Both the CUDA path and the CPU
oracle are fed from it, so that the two see identical inputs.

Generator: SplitMix64 (Steele, Lea and Flood, "Fast splittable pseudorandom
number generators", OOPSLA 2014), used counter-based.  Every tensor of every
step has its own 64-bit key, folded from (seed, workload id, tensor tag,
step) with the SplitMix64 finaliser; element n of the tensor is the
finaliser applied to ``key + (n + 1) * GOLDEN``.  Uniforms take the top 53
bits; normals use Box-Muller on consecutive pairs of uniforms.  Everything is
computed in float64 and rounded to float32 at the end, so any subset of
steps can be regenerated independently.

Workload shapes follow the serving setting of "STEPQuant: When and Where
Errors Matter in Delta-Rule Recurrent State Quantization" (background
section "linear attention and recurrent state": d_k = d_v = 128; section
"SGLang state pool": five state slots per request; structured result table:
batch 512 serving).  The outlier structure of the configuration-2 initial
state follows the same page's figure captions (seven to eight key rows and
value columns above 5x the axis median; 10.3x / 19.4x max-to-median RMS in
the motivation section).
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_MASK = (1 << 64) - 1

D = 128  # d_k = d_v on every workload here

# tensor tags (part of each tensor's key)
TAG_BITS, TAG_R, TAG_C, TAG_S0, TAG_S0_ROWS, TAG_S0_COLS = 1, 2, 3, 4, 5, 6
TAG_Q, TAG_K, TAG_V, TAG_BETA, TAG_GATE, TAG_SLOT = 11, 12, 13, 14, 15, 16


def _fin_int(z: int) -> int:
    z &= _MASK
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _MASK
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _MASK
    return z ^ (z >> 31)


def _fin(z: np.ndarray) -> np.ndarray:
    with np.errstate(over="ignore"):
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def stream_key(seed: int, *tags: int) -> int:
    """Fold (seed, tags...) into one 64-bit key."""
    k = _fin_int(seed * 0x9E3779B97F4A7C15 + 0x632BE59BD9B4E019)
    for t in tags:
        k = _fin_int(k ^ _fin_int((t + 1) * 0x9E3779B97F4A7C15))
    return k


def raw_u64(key: int, n: int, offset: int = 0) -> np.ndarray:
    idx = np.arange(offset + 1, offset + n + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return _fin(np.uint64(key) + idx * GOLDEN)


def uniform(key: int, n: int, offset: int = 0) -> np.ndarray:
    """n float64 uniforms in [0, 1)."""
    return (raw_u64(key, n, offset) >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)


def normal(key: int, n: int) -> np.ndarray:
    """n float64 standard normals (Box-Muller on uniform pairs)."""
    u = uniform(key, 2 * n)
    u1, u2 = u[0::2], u[1::2]
    return np.sqrt(-2.0 * np.log1p(-u1)) * np.cos(2.0 * math.pi * u2)


def permutation(key: int, n: int) -> np.ndarray:
    """Seeded permutation of range(n) (argsort of uniform keys)."""
    return np.argsort(uniform(key, n), kind="stable")


def log_uniform(key: int, n: int, lo: float, hi: float) -> np.ndarray:
    return np.exp(math.log(lo) + (math.log(hi) - math.log(lo)) * uniform(key, n))


def l2_normalise(x: np.ndarray) -> np.ndarray:
    """Normalise the last axis to unit L2 norm (float64 in, float64 out)."""
    n = np.sqrt(np.sum(x * x, axis=-1, keepdims=True))
    return x / np.where(n > 0, n, 1.0)


# ---------------------------------------------------------------------------
# workloads
# ---------------------------------------------------------------------------

GDN, KDA = 0, 1


@dataclasses.dataclass
class Workload:
    """One synthetic decode workload (all host numpy arrays)."""

    name: str
    wid: int                 # workload id, part of every key
    kind: int                # GDN or KDA
    R: int                   # requests in each decode call
    S: int                   # slots per request
    H: int                   # heads
    T: int                   # sequential decode steps
    unit_bits: np.ndarray    # uint8: GDN [H], KDA [H*128]
    row_factor: np.ndarray   # float32 [H*128]
    col_factor: np.ndarray   # float32 [H*128]
    slot_of_request: np.ndarray  # int32 [R]
    alpha_range: tuple = (0.90, 0.999)
    decay_range: tuple = (0.8, 0.9995)
    init: str = "zero"       # "zero" | "outlier"
    seed: int = 0

    @property
    def units(self) -> int:
        return self.R * self.H

    def row_bits(self) -> np.ndarray:
        """uint8 [H, 128]: the bit width of every key row of every head."""
        if self.kind == GDN:
            return np.repeat(self.unit_bits.reshape(self.H, 1), D, axis=1).astype(np.uint8)
        return self.unit_bits.reshape(self.H, D).astype(np.uint8)

    def initial_state(self, requests: np.ndarray | None = None) -> np.ndarray | None:
        """float32 [n, H, 128, 128] initial state of the given requests, or
        None when the workload starts from the zero state."""
        if self.init == "zero":
            return None
        reqs = np.arange(self.R) if requests is None else np.asarray(requests)
        out = np.empty((len(reqs), self.H, D, D), dtype=np.float32)
        for a, rq in enumerate(reqs):
            for h in range(self.H):
                u = int(rq) * self.H + h
                s = normal(stream_key(self.seed, self.wid, TAG_S0, u), D * D).reshape(D, D)
                rows = permutation(stream_key(self.seed, self.wid, TAG_S0_ROWS, u), D)[:8]
                cols = permutation(stream_key(self.seed, self.wid, TAG_S0_COLS, u), D)[:8]
                s[rows, :] *= 10.0
                s[:, cols] *= 20.0
                out[a, h] = s.astype(np.float32)
        return out

    def step_inputs(self, t: int, requests: np.ndarray | None = None) -> dict:
        """Inputs of decode step t for the given requests (default: all).

        q, k, v: float32 [n, H, 128]; beta: float32 [n, H];
        gate: float32 [n, H] (GDN alpha) or [n, H, 128] (KDA diagonal)."""
        reqs = np.arange(self.R) if requests is None else np.asarray(requests)
        n = len(reqs)
        key = lambda tag: stream_key(self.seed, self.wid, tag, t)
        full = self.R * self.H * D

        def per_elem(tag, fn):
            a = fn(key(tag), full).reshape(self.R, self.H, D)
            return a[reqs]

        q = l2_normalise(per_elem(TAG_Q, normal)).astype(np.float32)
        k = l2_normalise(per_elem(TAG_K, normal)).astype(np.float32)
        v = per_elem(TAG_V, normal).astype(np.float32)
        beta = uniform(key(TAG_BETA), self.R * self.H).reshape(self.R, self.H)[reqs]
        if self.kind == GDN:
            lo, hi = self.alpha_range
            g = lo + (hi - lo) * uniform(key(TAG_GATE), self.R * self.H).reshape(self.R, self.H)[reqs]
        else:
            lo, hi = self.decay_range
            g = lo + (hi - lo) * per_elem(TAG_GATE, uniform)
        return dict(q=q, k=k, v=v, beta=beta.astype(np.float32), gate=g.astype(np.float32))


def _shuffled_bits(key: int, counts: dict) -> np.ndarray:
    vals = np.concatenate([np.full(n, b, dtype=np.uint8) for b, n in counts.items()])
    return vals[permutation(key, len(vals))]


def _ones() -> np.ndarray:
    return np.ones(D, dtype=np.float32)


def make_workload(config: int, seed: int = 0, *, R: int | None = None, H: int | None = None,
                  T: int | None = None, bits: int | None = None) -> Workload:
    """The five synthetic workloads of the decode benchmark.

    1: GDN, uniform INT8, 4 requests x 4 heads, 64 steps, r = c = 1, zero start.
    2: GDN, per-head 4/6/8 bits (25/50/25 %, mean 6), 64 x 32 heads, 256 steps,
       r, c ~ logU(0.25, 4), outlier initial state.
    3: KDA, per-row 4/6/8 bits (32/64/32 rows per head), 128 x 32 heads,
       128 steps, per-row decay U(0.8, 0.9995), r = c = 1, zero start.
    4: serving pool, one token: R requests (default 64) x 5 slots x 768 heads
       (48 layers x 16 heads), mixed 6-bit GDN as in 2, active slot seeded.
    5: long-generation drift: 32 x 32 heads, GDN at ``bits`` (default 6),
       alpha ~ U(0.95, 0.9999).
    """
    if config == 1:
        R, H, T = R or 4, H or 4, T or 64
        return Workload("gdn_int8_4x4", 1, GDN, R, 1, H, T,
                        np.full(H, bits or 8, dtype=np.uint8),
                        np.ones(H * D, np.float32), np.ones(H * D, np.float32),
                        np.zeros(R, np.int32), seed=seed)
    if config in (2, 4):
        if config == 2:
            R, H, T, S, wid, name = R or 64, H or 32, T or 256, 1, 2, "gdn_mixed6_64x32"
        else:
            R, H, T, S, wid, name = R or 64, H or 768, T or 1, 5, 4, "gdn_mixed6_pool"
        assert H % 4 == 0
        ub = _shuffled_bits(stream_key(seed, wid, TAG_BITS), {4: H // 4, 6: H // 2, 8: H // 4})
        r = log_uniform(stream_key(seed, wid, TAG_R), H * D, 0.25, 4.0).astype(np.float32)
        c = log_uniform(stream_key(seed, wid, TAG_C), H * D, 0.25, 4.0).astype(np.float32)
        if config == 2:
            slots = np.zeros(R, np.int32)
        else:
            slots = np.floor(uniform(stream_key(seed, wid, TAG_SLOT), R) * S).astype(np.int32)
        return Workload(name if config == 2 else f"{name}_R{R}", wid, GDN, R, S, H, T, ub, r, c,
                        slots, init="outlier" if config == 2 else "zero", seed=seed)
    if config == 3:
        R, H, T = R or 128, H or 32, T or 128
        ub = np.concatenate([
            _shuffled_bits(stream_key(seed, 3, TAG_BITS, h), {4: 32, 6: 64, 8: 32}) for h in range(H)])
        return Workload("kda_mixed6_128x32", 3, KDA, R, 1, H, T, ub,
                        np.ones(H * D, np.float32), np.ones(H * D, np.float32),
                        np.zeros(R, np.int32), seed=seed)
    if config == 5:
        R, H, T = R or 32, H or 32, T or 8192
        b = bits or 6
        return Workload(f"drift_gdn_int{b}", 5, GDN, R, 1, H, T, np.full(H, b, np.uint8),
                        np.ones(H * D, np.float32), np.ones(H * D, np.float32),
                        np.zeros(R, np.int32), alpha_range=(0.95, 0.9999), seed=seed)
    raise ValueError(f"unknown workload {config}")


def algorithmic_bytes_per_head_step(kind: int, row_bits_sum: int, scale_bytes: int = 4) -> int:
    """HBM bytes one (request, head) decode step must move: packed codes read
    and written, 128 row scales of `scale_bytes` bytes read and written (4:
    fp32, 2: binary16, 0: a raw fp16 / fp32 state), q, k, v read, y written,
    beta and the gate read."""
    codes = 2 * 16 * row_bits_sum
    scales = 2 * D * scale_bytes
    io = 3 * D * 4 + D * 4 + 4
    gate = 4 if kind == GDN else D * 4
    return codes + scales + io + gate

"""Test helpers: read packed pages and compare a GPU step with the oracle.

A vectorised reader of the documented page format (128 fp32 scales, then
rows of 128 b-bit two's complement codes, little-endian bit order, 6-bit
codes in groups of eight split into a word and a half, page padded to 128
bytes).  It belongs to neither implementation; the CPU tests
check it against the oracle's bit-by-bit packer.
"""
from __future__ import annotations

import numpy as np

D = 128


PIVOT = 4  # format flag: 16-bit rows are FP16 pivots among quantized rows
FITC = 8   # format flag: the page carries its own fp32 column factors after the scales


def _scale_bytes(row_bits, fmt) -> int:
    if not (fmt & PIVOT) and int(np.asarray(row_bits).reshape(-1)[0]) in (16, 32):
        return 0  # raw page
    return 2 if fmt & 1 else 4


def page_bytes(row_bits, fmt: int = 0) -> int:
    n = _scale_bytes(row_bits, fmt) * D + (4 * D if fmt & FITC else 0) + 16 * int(np.sum(np.asarray(row_bits, np.int64)))
    return (n + 127) // 128 * 128


def row_offsets(row_bits, fmt: int = 0) -> np.ndarray:
    rb = np.asarray(row_bits, np.int64)
    base = _scale_bytes(row_bits, fmt) * D + (4 * D if fmt & FITC else 0)
    return base + np.concatenate([[0], np.cumsum(16 * rb)[:-1]])


def head_offsets(pool_row_bits, fmt: int = 0) -> np.ndarray:
    sizes = [page_bytes(pool_row_bits[h], fmt) for h in range(len(pool_row_bits))]
    return np.concatenate([[0], np.cumsum(sizes)[:-1]]).astype(np.int64)


def raw_values(page: np.ndarray, row_bits) -> np.ndarray:
    """The [128, 128] state of a raw page (binary16 or fp32 rows), as float64."""
    b = int(np.asarray(row_bits).reshape(-1)[0])
    dt = np.float16 if b == 16 else np.float32
    return np.asarray(page, np.uint8)[: D * D * b // 8].view(dt).reshape(D, D).astype(np.float64)


def decode_page(page: np.ndarray, row_bits, fmt: int = 0) -> tuple[np.ndarray, np.ndarray]:
    """(scales float32 [128], codes int32 [128, 128]) of one page."""
    page = np.asarray(page, np.uint8)
    if fmt & 1:
        scales = page[: 2 * D].view(np.float16).astype(np.float32)
    else:
        scales = page[: 4 * D].view(np.float32).copy()
    codes = np.zeros((D, D), np.int32)
    offs = row_offsets(row_bits, fmt)
    for b in (4, 6, 8):
        rows = np.nonzero(np.asarray(row_bits) == b)[0]
        if len(rows) == 0:
            continue
        nb = 16 * b
        raw = np.stack([page[offs[i]: offs[i] + nb] for i in rows])
        if b == 6:  # group g: word bytes [4g, 4g+4) then half bytes [64+2g, 66+2g), contiguous again
            n = len(rows)
            raw = np.concatenate([raw[:, :64].reshape(n, 16, 4), raw[:, 64:].reshape(n, 16, 2)],
                                 axis=2).reshape(n, nb)
        bits = np.unpackbits(raw, axis=1, bitorder="little").reshape(len(rows), D, b).astype(np.int64)
        u = (bits << np.arange(b)).sum(axis=2)
        codes[rows] = np.where(u >= (1 << (b - 1)), u - (1 << b), u)
    return scales, codes


def col_factors(page: np.ndarray, row_bits, fmt: int = FITC) -> np.ndarray:
    """The page's own column factors (fp32 [128]) of a fitted page."""
    o = _scale_bytes(row_bits, fmt) * D
    return np.asarray(page, np.uint8)[o: o + 4 * D].view(np.float32).copy()


def pivot_values(page: np.ndarray, row_bits, fmt: int = PIVOT) -> np.ndarray:
    """[128, 128] binary16 values of the pivot (16-bit) rows as float64; NaN elsewhere."""
    page = np.asarray(page, np.uint8)
    out = np.full((D, D), np.nan)
    offs = row_offsets(row_bits, fmt)
    for i in np.nonzero(np.asarray(row_bits) == 16)[0]:
        out[i] = page[offs[i]: offs[i] + 2 * D].view(np.float16).astype(np.float64)
    return out


def split_slot(slot: np.ndarray, pool_row_bits, fmt: int = 0) -> list[np.ndarray]:
    offs = head_offsets(pool_row_bits, fmt)
    return [slot[offs[h]: offs[h] + page_bytes(pool_row_bits[h], fmt)] for h in range(len(pool_row_bits))]


class Compare:
    """Accumulates the parity of GPU steps against oracle steps.

    Tolerances (fp32): y and scales within max relative error 1e-5 per
    (request, head); codes bit-exact except for +-1 at near rounding ties
    (the oracle's quotient within 1e-4 relative of a half-integer), whose
    count must stay at or below 1e-4 of all codes compared.

    Binary16 scales must be bit-exact, except a row whose fp32 scale a / q_b
    lies within 1e-5 relative of a binary16 rounding midpoint: the GPU's a
    differs from the oracle's by an ulp or two, so it may round to the
    neighbour; that row's codes are then checked against the GPU's scale.

    Raw pages: fp32 values within 1e-5 of the unit's largest; binary16
    values bit-exact except where the GPU's value is the binary16 rounding of
    a value within 4e-6 x max|X| of the unit from X (near a rounding
    midpoint, or in the subnormal range where the spacing is absolute).  The
    GPU evaluates X (or a pivot row's mu) in fp32, a few ulps off the exact
    value, and rounds that to binary16, whose rounding midpoints are 2^-10 |X|
    apart: a value flips with probability of order 2^-12 max|X| / |X|.
    Measured over every GPU test: 483 of 6.4 M binary16 values (7.6e-5), at
    most 1.4e-4 in one test; the count is bounded by 3e-4 of the values.
    Binary16 scale flips: 5 in 626 K rows (8e-6), at most 2 of 4,800 rows in
    one test; bounded by max(3, 1e-3 x rows)."""

    def __init__(self, rtol: float = 1e-5, tie_rel: float = 1e-4, max_tie_frac: float = 1e-4,
                 scale_flip_rel: float = 1e-5, raw_tie_rel: float = 4e-6, max_raw_tie_frac: float = 3e-4,
                 max_scale_flip_frac: float = 1e-3):
        self.rtol, self.tie_rel, self.max_tie_frac = rtol, tie_rel, max_tie_frac
        self.scale_flip_rel = scale_flip_rel
        self.raw_tie_rel, self.max_raw_tie_frac = raw_tie_rel, max_raw_tie_frac
        self.max_scale_flip_frac = max_scale_flip_frac
        self.codes = 0
        self.values = 0
        self.ties = []
        self.flips = []
        self.raw_ties = 0
        self.raw_flips = []  # (where, row, column, gpu value, oracle value, oracle's fp32 value)
        self.worst_y = 0.0
        self.worst_s = 0.0
        self.worst_x = 0.0
        self.worst_c = 0.0
        self.tied_columns = 0
        self.flip_pages = 0

    def y(self, y_gpu, y_ref, where=""):
        y_gpu = np.asarray(y_gpu, np.float64)
        y_ref = np.asarray(y_ref, np.float64)
        den = max(np.abs(y_ref).max(), 1e-30)
        err = np.abs(y_gpu - y_ref).max() / den
        self.worst_y = max(self.worst_y, err)
        assert err <= self.rtol, f"y rel err {err:.3g} {where}"

    def page(self, page_gpu, page_ref, quot, row_bits, where="", fmt=0):
        sg, zg = decode_page(page_gpu, row_bits, fmt)
        sr, zr = decode_page(page_ref, row_bits, fmt)
        piv = np.asarray(row_bits) == 16
        if piv.any():
            self._pivots(page_gpu, page_ref, quot, row_bits, piv, where, fmt)
            assert np.all(sg[piv] == 1) and np.all(sr[piv] == 1), f"pivot scale slot not 1 {where}"
        self.codes += int((~piv).sum()) * D
        qref = np.asarray(quot, np.float64).copy()
        zref = zr.copy()
        flipped = False
        if fmt & 1:
            # binary16 scales: a row whose s = a / q_b lies next to a rounding midpoint of
            # binary16 may round to the other neighbour on the GPU (its a differs by an ulp
            # or two); then its codes follow the GPU's scale
            for i in np.nonzero(sg != sr)[0]:
                h16 = np.array([sr[i], sg[i]], np.float16).view(np.uint16).astype(np.int64)
                qb = (1 << (int(row_bits[i]) - 1)) - 1
                mu = qref[i] * float(sr[i])
                s = np.abs(mu).max() / qb
                mid = (float(sr[i]) + float(sg[i])) / 2
                assert abs(h16[0] - h16[1]) == 1 and abs(s - mid) <= self.scale_flip_rel * s, (
                    f"scale mismatch row {i} {where}: gpu {sg[i]} ref {sr[i]} (s = {s})")
                qref[i] = mu / float(sg[i])
                zref[i] = np.clip(np.rint(qref[i]), -qb, qb)
                self.flips.append((where, int(i), float(sr[i]), float(sg[i])))
                flipped = True
        diff = zg != zref
        if fmt & FITC:
            # fitted factors: fp32 sums on the GPU, fp64 in the oracle; a column that holds a
            # near-tie code is refitted from a different code and is logged, not compared
            cg_, cr_ = col_factors(page_gpu, row_bits, fmt), col_factors(page_ref, row_bits, fmt)
            tied = diff.any(axis=0)
            if flipped:
                # a row's binary16 scale took the other neighbour: every column was refitted
                # with that scale, so this page's factors are logged, not compared
                tied[:] = True
                self.flip_pages += 1
            rel = np.abs(cg_.astype(np.float64) - cr_) / np.maximum(np.abs(cr_), 1e-30)
            self.worst_c = max(self.worst_c, float(rel[~tied].max()) if (~tied).any() else 0.0)
            self.tied_columns += int(tied.sum())
            assert np.all(rel[~tied] <= self.rtol), f"column factor rel err {rel[~tied].max():.3g} {where}"
        if diff.any():
            ii, jj = np.nonzero(diff)
            x = qref[ii, jj]
            frac = np.abs(x - np.floor(x) - 0.5)
            near = frac <= self.tie_rel * np.maximum(np.abs(x), 1.0)
            one = np.abs(zg[ii, jj] - zref[ii, jj]) == 1
            bad = ~(near & one)
            assert not bad.any(), (
                f"{int(bad.sum())} code mismatches that are not near-ties {where}: rows {ii[bad][:5]}, "
                f"cols {jj[bad][:5]}, gpu {zg[ii, jj][bad][:5]}, ref {zref[ii, jj][bad][:5]}, quot {x[bad][:5]}")
            for a, b in zip(ii, jj):
                self.ties.append((where, int(a), int(b), float(qref[a, b]), int(zg[a, b]), int(zref[a, b])))
        if fmt & 1:
            return  # every scale is equal or an accepted flip
        den = np.maximum(np.abs(sr.astype(np.float64)), 1e-38)
        rel = np.abs(sg.astype(np.float64) - sr) / den
        rel[(sr == 0) & (sg == 0)] = 0.0
        self.worst_s = max(self.worst_s, float(rel.max()))
        assert rel.max() <= self.rtol, f"scale rel err {rel.max():.3g} {where}"

    def _pivots(self, page_gpu, page_ref, quot, row_bits, piv, where, fmt):
        """FP16 pivot rows: binary16 values of mu = X / (r c), equal except where the
        GPU's value rounds a value within raw_tie_rel x max|mu| (over the unit's pivot
        rows) of the oracle's fl32(mu), passed in quot."""
        xg, xr = pivot_values(page_gpu, row_bits, fmt)[piv], pivot_values(page_ref, row_bits, fmt)[piv]
        self.values += xg.size
        diff = xg != xr
        if diff.any():
            M = np.asarray(quot, np.float64)[piv]
            x = M[diff]
            half_ulp = np.abs(np.spacing(xg[diff].astype(np.float16)).astype(np.float64)) / 2
            near = np.abs(xg[diff] - x) <= self.raw_tie_rel * np.abs(M).max() + half_ulp
            assert near.all(), (f"{int((~near).sum())} pivot mismatches beyond the fp32 error window {where}: "
                                f"gpu {xg[diff][~near][:5]} ref {xr[diff][~near][:5]} mu {x[~near][:5]}")
            self.raw_ties += int(diff.sum())
            rows = np.nonzero(piv)[0]
            for (a, b) in zip(*np.nonzero(diff)):
                self.raw_flips.append((where, int(rows[a]), int(b), float(xg[a, b]), float(xr[a, b]), float(M[a, b])))

    def raw(self, page_gpu, page_ref, quot, row_bits, where=""):
        """A raw page: fp32 values within rtol of the unit's largest; binary16
        values equal except where the GPU's value rounds a value within
        raw_tie_rel x max|X| of X (the oracle's fl32(X), passed as quot)."""
        xg, xr = raw_values(page_gpu, row_bits), raw_values(page_ref, row_bits)
        self.values += xg.size
        if int(np.asarray(row_bits).reshape(-1)[0]) == 32:
            err = np.abs(xg - xr).max() / max(np.abs(xr).max(), 1e-30)
            self.worst_x = max(self.worst_x, float(err))
            assert err <= self.rtol, f"state rel err {err:.3g} {where}"
            return
        diff = xg != xr
        if diff.any():
            ii, jj = np.nonzero(diff)
            X = np.asarray(quot, np.float64)
            x = X[ii, jj]
            # the GPU's value must be the binary16 rounding of a value within the window of X
            half_ulp = np.abs(np.spacing(xg[ii, jj].astype(np.float16)).astype(np.float64)) / 2
            near = np.abs(xg[ii, jj] - x) <= self.raw_tie_rel * np.abs(X).max() + half_ulp
            bad = ~near
            assert not bad.any(), (f"{int(bad.sum())} binary16 mismatches beyond the fp32 error window {where}: "
                                   f"gpu {xg[ii, jj][bad][:5]} ref {xr[ii, jj][bad][:5]} X {x[bad][:5]}")
            self.raw_ties += len(ii)
            for a, b in zip(ii, jj):
                self.raw_flips.append((where, int(a), int(b), float(xg[a, b]), float(xr[a, b]), float(X[a, b])))

    def finish(self):
        frac = len(self.ties) / max(self.codes, 1)
        for t in self.ties[:20]:
            print("near-tie:", t)
        for f in self.flips[:10]:
            print("binary16 scale flip:", f)
        for f in self.raw_flips[:20]:
            print("binary16 value flip (where, row, col, gpu, oracle, oracle fp32):", f)
        print(f"codes compared {self.codes}, near-ties {len(self.ties)} ({frac:.2e}), "
              f"scale flips {len(self.flips)}, raw values {self.values}, raw ties {self.raw_ties}, "
              f"worst y rel {self.worst_y:.2e}, worst scale rel {self.worst_s:.2e}, "
              f"worst raw rel {self.worst_x:.2e}, worst column factor rel {self.worst_c:.2e} "
              f"({self.tied_columns} columns with a near-tie not compared; factors of {self.flip_pages} pages "
              f"with a scale flip not compared)")
        assert frac <= self.max_tie_frac, f"tie fraction {frac:.3g} above {self.max_tie_frac}"
        rows = self.codes // 128
        assert len(self.flips) <= max(3, self.max_scale_flip_frac * rows), f"{len(self.flips)} scale flips in {rows} rows"
        rfrac = self.raw_ties / max(self.values, 1)
        assert rfrac <= self.max_raw_tie_frac, f"raw tie fraction {rfrac:.3g} above {self.max_raw_tie_frac}"

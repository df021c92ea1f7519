"""Test helpers: read packed pages and compare a GPU step with the oracle.

A vectorised reader of the documented page format (128 fp32 scales, then
rows of 128 b-bit two's complement codes, little-endian bit order, page
padded to 128 bytes).  It belongs to neither implementation; the CPU tests
check it against the oracle's bit-by-bit packer.
"""
from __future__ import annotations

import numpy as np

D = 128


def page_bytes(row_bits) -> int:
    n = 4 * D + 16 * int(np.sum(np.asarray(row_bits, np.int64)))
    return (n + 127) // 128 * 128


def row_offsets(row_bits) -> np.ndarray:
    rb = np.asarray(row_bits, np.int64)
    return 4 * D + np.concatenate([[0], np.cumsum(16 * rb)[:-1]])


def head_offsets(pool_row_bits) -> np.ndarray:
    sizes = [page_bytes(pool_row_bits[h]) for h in range(len(pool_row_bits))]
    return np.concatenate([[0], np.cumsum(sizes)[:-1]]).astype(np.int64)


def decode_page(page: np.ndarray, row_bits) -> tuple[np.ndarray, np.ndarray]:
    """(scales float32 [128], codes int32 [128, 128]) of one page."""
    page = np.asarray(page, np.uint8)
    scales = page[: 4 * D].view(np.float32).copy()
    codes = np.zeros((D, D), np.int32)
    offs = row_offsets(row_bits)
    for b in (4, 6, 8):
        rows = np.nonzero(np.asarray(row_bits) == b)[0]
        if len(rows) == 0:
            continue
        nb = 16 * b
        raw = np.stack([page[offs[i]: offs[i] + nb] for i in rows])
        bits = np.unpackbits(raw, axis=1, bitorder="little").reshape(len(rows), D, b).astype(np.int64)
        u = (bits << np.arange(b)).sum(axis=2)
        codes[rows] = np.where(u >= (1 << (b - 1)), u - (1 << b), u)
    return scales, codes


def split_slot(slot: np.ndarray, pool_row_bits) -> list[np.ndarray]:
    offs = head_offsets(pool_row_bits)
    return [slot[offs[h]: offs[h] + page_bytes(pool_row_bits[h])] for h in range(len(pool_row_bits))]


class Compare:
    """Accumulates the parity of GPU steps against oracle steps.

    Tolerances (fp32): y and scales within max relative error 1e-5 per
    (request, head); codes bit-exact except for +-1 at near rounding ties
    (the oracle's quotient within 1e-4 relative of a half-integer), whose
    count must stay at or below 1e-4 of all codes compared."""

    def __init__(self, rtol: float = 1e-5, tie_rel: float = 1e-4, max_tie_frac: float = 1e-4):
        self.rtol, self.tie_rel, self.max_tie_frac = rtol, tie_rel, max_tie_frac
        self.codes = 0
        self.ties = []
        self.worst_y = 0.0
        self.worst_s = 0.0

    def y(self, y_gpu, y_ref, where=""):
        y_gpu = np.asarray(y_gpu, np.float64)
        y_ref = np.asarray(y_ref, np.float64)
        den = max(np.abs(y_ref).max(), 1e-30)
        err = np.abs(y_gpu - y_ref).max() / den
        self.worst_y = max(self.worst_y, err)
        assert err <= self.rtol, f"y rel err {err:.3g} {where}"

    def page(self, page_gpu, page_ref, quot, row_bits, where=""):
        sg, zg = decode_page(page_gpu, row_bits)
        sr, zr = decode_page(page_ref, row_bits)
        self.codes += zg.size
        diff = zg != zr
        if diff.any():
            ii, jj = np.nonzero(diff)
            x = quot[ii, jj].astype(np.float64)
            frac = np.abs(x - np.floor(x) - 0.5)
            near = frac <= self.tie_rel * np.maximum(np.abs(x), 1.0)
            one = np.abs(zg[ii, jj] - zr[ii, jj]) == 1
            bad = ~(near & one)
            assert not bad.any(), (
                f"{int(bad.sum())} code mismatches that are not near-ties {where}: rows {ii[bad][:5]}, "
                f"cols {jj[bad][:5]}, gpu {zg[ii, jj][bad][:5]}, ref {zr[ii, jj][bad][:5]}, quot {x[bad][:5]}")
            for a, b in zip(ii, jj):
                self.ties.append((where, int(a), int(b), float(quot[a, b]), int(zg[a, b]), int(zr[a, b])))
        den = np.maximum(np.abs(sr.astype(np.float64)), 1e-38)
        rel = np.abs(sg.astype(np.float64) - sr) / den
        rel[(sr == 0) & (sg == 0)] = 0.0
        self.worst_s = max(self.worst_s, float(rel.max()))
        assert rel.max() <= self.rtol, f"scale rel err {rel.max():.3g} {where}"

    def finish(self):
        frac = len(self.ties) / max(self.codes, 1)
        for t in self.ties[:20]:
            print("near-tie:", t)
        print(f"codes compared {self.codes}, near-ties {len(self.ties)} ({frac:.2e}), "
              f"worst y rel {self.worst_y:.2e}, worst scale rel {self.worst_s:.2e}")
        assert frac <= self.max_tie_frac, f"tie fraction {frac:.3g} above {self.max_tie_frac}"

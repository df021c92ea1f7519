"""Pins of the oracle's online column fit ("core method": c_j minimises
sum_{i,j} w_i^2 (X_ij - r_i c_j z_ij)^2; "method steps", steps 4-5, its
closed form): the page carries its own column factors, refitted at every
quantisation from the codes just taken.  Each pin checks the oracle against
something other than itself: the normal equations of the least-squares
problem on an independently computed X, the weighted error before and after,
exact reconstruction of a state built from chosen codes and factors."""
import numpy as np
import pytest

import oracle as orc

FIT = orc.FMT_FITC
D = 8


def _unit(n, rng):
    x = rng.standard_normal(n)
    return (x / np.linalg.norm(x)).astype(np.float32)


def _read(page, bits, dv, fmt):
    """(scales, column factors, codes) of a page, read with numpy."""
    sb = 2 if fmt & orc.FMT_F16 else 4
    dk = len(bits)
    s = (page[: 2 * dk].view(np.float16) if sb == 2 else page[: 4 * dk].view(np.float32)).astype(np.float64)
    c = page[sb * dk: sb * dk + 4 * dv].view(np.float32).astype(np.float64)
    offs = orc.row_offsets(bits, dv, fmt)
    z = np.zeros((dk, dv), np.int64)
    for i, b in enumerate(bits):
        row = page[offs[i]: offs[i] + dv * int(b) // 8]
        z[i] = [orc.get_code(row, int(b), j, dv=dv) for j in range(dv)]
    return s, c, z


def _read_np(page, bits, dv, fmt):
    """_read for pages with FP16 pivot rows: their codes are reported as 0."""
    sb = 2 if fmt & orc.FMT_F16 else 4
    dk = len(bits)
    s = (page[: 2 * dk].view(np.float16) if sb == 2 else page[: 4 * dk].view(np.float32)).astype(np.float64)
    c = page[sb * dk: sb * dk + 4 * dv].view(np.float32).astype(np.float64)
    offs = orc.row_offsets(bits, dv, fmt)
    z = np.zeros((dk, dv), np.int64)
    for i, b in enumerate(bits):
        if b == 16:
            continue
        row = page[offs[i]: offs[i] + dv * int(b) // 8]
        z[i] = [orc.get_code(row, int(b), j, dv=dv) for j in range(dv)]
    return s, c, z


def _explicit(S, q, k, v, beta, g):
    """S_t = (I - beta k k^T) D S + beta k v^T with explicit matrices, fp64."""
    k = k.astype(np.float64)
    A = (np.eye(len(k)) - beta * np.outer(k, k)) @ np.diag(g.astype(np.float64))
    X = A @ S + beta * np.outer(k, v.astype(np.float64))
    return X, X.T @ q.astype(np.float64)


def _case(seed, fmt=FIT):
    rng = np.random.default_rng(seed)
    bits = rng.choice(np.array([4, 6, 8], np.uint8), D)
    r = np.exp(rng.uniform(-1, 1, D)).astype(np.float32)
    c = np.exp(rng.uniform(-1, 1, D)).astype(np.float32)
    w = np.exp(rng.uniform(-1, 1, D)).astype(np.float32)
    S0 = (rng.standard_normal((D, D)) * np.exp(rng.uniform(-1, 1, (1, D)))).astype(np.float32)
    page = orc.quantize_unit(bits, r, c, S0, fmt=fmt, w=w)
    return rng, bits, r, c, w, page


@pytest.mark.parametrize("seed", range(12))
def test_fitted_factors_solve_the_normal_equations(seed):
    """After a step, every column's factor zeroes sum_i w_i^2 v_ij (X_ij - c_j v_ij)
    (up to its rounding to fp32), with X the explicit recurrence on the old
    reconstruction and v_ij = s_i r_i z_ij read from the new page."""
    fmt = FIT | (orc.FMT_F16 if seed % 2 else 0)
    rng, bits, r, c, w, page = _case(seed, fmt)
    S_hat = orc.dequantize_unit(bits, r, c, page, D, fmt).astype(np.float64)
    q, k = _unit(D, rng), _unit(D, rng)
    v = rng.standard_normal(D).astype(np.float32)
    g = rng.uniform(0.8, 1.0, D).astype(np.float32)
    out, y, _, st = orc.step_unit(bits, r, c, page, q, k, v, np.float32(0.6), g, D, fmt, w=w)
    assert st == orc.OK
    # the reconstruction uses the page's factors, not the table's
    s_old, c_old, z_old = _read(page, bits, D, fmt)
    S64 = s_old[:, None] * r[:, None].astype(np.float64) * c_old[None, :] * z_old
    np.testing.assert_array_equal(S_hat, S64.astype(np.float32))
    X, y_ref = _explicit(S64, q, k, v, float(np.float32(0.6)), g)
    np.testing.assert_allclose(y, y_ref, rtol=1e-9, atol=1e-12)
    s, cn, z = _read(out, bits, D, fmt)
    V = s[:, None] * r[:, None].astype(np.float64) * z
    W2 = (w.astype(np.float64) ** 2)[:, None]
    resid = (W2 * V * (X - cn[None, :] * V)).sum(0)
    scale = (W2 * V * V).sum(0) * np.abs(cn)
    assert np.all(np.abs(resid) <= 2e-7 * scale + 1e-300), (resid, scale)


@pytest.mark.parametrize("seed", range(8))
def test_fit_never_raises_the_weighted_error(seed):
    """For the codes just taken, the refitted factors' weighted error is at most the old factors'."""
    rng, bits, r, c, w, page = _case(100 + seed)
    s_old, c_old, z_old = _read(page, bits, D, FIT)
    S64 = s_old[:, None] * r[:, None].astype(np.float64) * c_old[None, :] * z_old
    q, k = _unit(D, rng), _unit(D, rng)
    v = rng.standard_normal(D).astype(np.float32)
    g = rng.uniform(0.8, 1.0, D).astype(np.float32)
    out, _, _, st = orc.step_unit(bits, r, c, page, q, k, v, np.float32(0.9), g, D, FIT, w=w)
    X, _ = _explicit(S64, q, k, v, float(np.float32(0.9)), g)
    s, cn, z = _read(out, bits, D, FIT)
    V = s[:, None] * r[:, None].astype(np.float64) * z
    W2 = (w.astype(np.float64) ** 2)[:, None]
    err = lambda cc: float((W2 * (X - cc[None, :] * V) ** 2).sum())  # noqa: E731
    assert err(cn) <= err(c_old) * (1 + 1e-12)


def test_state_built_from_codes_is_refitted_exactly():
    """X = s_i r_i c_j z_ij with chosen integer codes (the largest code of every row at
    q_b so the absmax scale is s_i) quantizes to the same codes and refits c exactly."""
    rng = np.random.default_rng(7)
    bits = np.array([8, 6, 4, 8, 6, 4, 8, 6], np.uint8)
    qb = (1 << (bits.astype(np.int64) - 1)) - 1
    z = np.stack([rng.integers(-qb[i], qb[i] + 1, D) for i in range(D)])
    z[np.arange(D), rng.integers(0, D, D)] = qb
    s = 2.0 ** rng.integers(-3, 3, D)
    r = (2.0 ** rng.integers(-2, 2, D)).astype(np.float32)
    c = (2.0 ** rng.integers(-2, 2, D)).astype(np.float32)
    S = (s[:, None] * r[:, None] * c[None, :] * z).astype(np.float32)
    w = np.exp(rng.uniform(-1, 1, D)).astype(np.float32)
    page = orc.quantize_unit(bits, r, c, S, fmt=FIT, w=w)
    s2, c2, z2 = _read(page, bits, D, FIT)
    np.testing.assert_array_equal(z2, z)
    np.testing.assert_array_equal(c2, c)
    np.testing.assert_array_equal(orc.dequantize_unit(bits, r, c, page, D, FIT), S)


def test_zero_column_keeps_its_factor_and_weights_steer_the_fit():
    rng = np.random.default_rng(8)
    bits = np.full(D, 8, np.uint8)
    r = np.ones(D, np.float32)
    c = np.exp(rng.uniform(-1, 1, D)).astype(np.float32)
    S = rng.standard_normal((D, D)).astype(np.float32)
    S[:, 3] = 0.0
    w = np.full(D, 1e-4, np.float32)
    w[5] = 1.0
    page = orc.quantize_unit(bits, r, c, S, fmt=FIT, w=w)
    s, cn, z = _read(page, bits, D, FIT)
    assert cn[3] == c[3]
    # the heavy row dominates: c_j is close to X_5j / (s_5 z_5j)
    j = [t for t in range(D) if t != 3 and z[5, t] != 0]
    np.testing.assert_allclose(cn[j], S[5, j] / (s[5] * z[5, j]), rtol=1e-3)


def test_fit_page_layout_and_flag_rules():
    bits = np.array([6] * D, np.uint8)
    assert orc.page_bytes(bits, D, FIT) == (4 * D + 4 * D + D * D * 6 // 8 + 127) // 128 * 128
    offs, offs0 = orc.row_offsets(bits, D, FIT), orc.row_offsets(bits, D)
    np.testing.assert_array_equal(offs - offs0, 4 * D)
    # FP16 pivot rows in a fitted page: 2 bytes per value after the scales and factors
    pbits = np.array([16] + [6] * (D - 1), np.uint8)
    assert orc.page_bytes(pbits, D, FIT | orc.FMT_PIVOT) == (4 * D + 4 * D + 2 * D + (D - 1) * D * 6 // 8
                                                             + 127) // 128 * 128
    np.testing.assert_array_equal(np.diff(orc.row_offsets(pbits, D, FIT | orc.FMT_PIVOT))[:1], [2 * D])


# ---------------------------------------------------------------- pivot rows in a fitted page
#
# "core innovation": the column factors are fitted per head "across non-pivot rows"; pivot
# rows are read in FP16 directly.  Reading: in a fitted page a pivot row holds
# mu_ij = X_ij / r_i in binary16 (its value must not move when the factors are refitted) and
# the fit's sums skip it.

PF = FIT | orc.FMT_PIVOT


def _pivot_values(page, bits, dv, fmt):
    offs = orc.row_offsets(bits, dv, fmt)
    return {i: page[offs[i]: offs[i] + 2 * dv].view(np.float16).astype(np.float64)
            for i in np.nonzero(bits == 16)[0]}


def _codes_case(seed):
    """Non-pivot rows built from chosen codes and power-of-two factors (each row's
    largest code at q_b), pivot rows 1, 4 and 6 holding arbitrary large values."""
    rng = np.random.default_rng(seed)
    bits = np.array([8, 16, 6, 4, 16, 8, 16, 6], np.uint8)
    piv = bits == 16
    qb = np.where(piv, 1, (1 << (bits.astype(np.int64) - 1)) - 1)
    z = np.stack([rng.integers(-qb[i], qb[i] + 1, D) for i in range(D)])
    z[np.arange(D), rng.integers(0, D, D)] = qb
    s = 2.0 ** rng.integers(-3, 3, D)
    r = (2.0 ** rng.integers(-2, 2, D)).astype(np.float32)
    c = (2.0 ** rng.integers(-2, 2, D)).astype(np.float32)
    S = (s[:, None] * r[:, None] * c[None, :] * z).astype(np.float32)
    S[piv] = (rng.standard_normal((int(piv.sum()), D)) * 50).astype(np.float32)
    w = np.exp(rng.uniform(-1, 1, D)).astype(np.float32)
    return rng, bits, piv, z, r, c, S, w


@pytest.mark.parametrize("seed", range(4))
def test_pivot_rows_are_left_out_of_the_fit(seed):
    """The non-pivot rows refit c exactly whatever the pivot rows hold (large
    values that would pull any fit that included them); pivot rows store
    numpy's binary16 of fl32(S / r) and reconstruct as r times that value,
    without c; non-pivot rows reconstruct S exactly."""
    rng, bits, piv, z, r, c, S, w = _codes_case(20 + seed)
    page = orc.quantize_unit(bits, r, c, S, fmt=PF, w=w)
    s2, c2, z2 = _read_np(page, bits, D, PF)
    np.testing.assert_array_equal(c2, c)
    np.testing.assert_array_equal(z2[~piv], z[~piv])
    np.testing.assert_array_equal(s2[piv], 1.0)
    pv = _pivot_values(page, bits, D, PF)
    for i, vals in pv.items():
        want = (S[i] / r[i]).astype(np.float32).astype(np.float16).astype(np.float64)
        np.testing.assert_array_equal(vals, want)
    Sh = orc.dequantize_unit(bits, r, c, page, D, PF)
    np.testing.assert_array_equal(Sh[~piv], S[~piv])
    for i, vals in pv.items():
        np.testing.assert_array_equal(Sh[i], (r[i] * vals).astype(np.float32))
    # other pivot content: the same factors, the same non-pivot bytes
    S2 = S.copy()
    S2[piv] = (rng.standard_normal((int(piv.sum()), D)) * 1e3).astype(np.float32)
    page2 = orc.quantize_unit(bits, r, c, S2, fmt=PF, w=w)
    offs = orc.row_offsets(bits, D, PF)
    for i in np.nonzero(~piv)[0]:
        n = D * int(bits[i]) // 8
        np.testing.assert_array_equal(page2[offs[i]: offs[i] + n], page[offs[i]: offs[i] + n])
    np.testing.assert_array_equal(_read_np(page2, bits, D, PF)[1], c)


@pytest.mark.parametrize("seed", range(6))
def test_pivot_fit_step_matches_explicit_form(seed):
    """One step of a fitted page with pivot rows: the readout is the explicit
    recurrence's on the old reconstruction (non-pivot rows s r c_page z, pivot
    rows r mu); the new pivot rows hold binary16 of fl32(X / r); the new factors
    solve the normal equations over the non-pivot rows."""
    rng, bits, piv, z, r, c, S, w = _codes_case(40 + seed)
    fmt = PF | (orc.FMT_F16 if seed % 2 else 0)
    page = orc.quantize_unit(bits, r, c, S, fmt=fmt, w=w)
    s_old, c_old, z_old = _read_np(page, bits, D, fmt)
    S64 = s_old[:, None] * r[:, None].astype(np.float64) * c_old[None, :] * z_old
    for i, vals in _pivot_values(page, bits, D, fmt).items():
        S64[i] = float(r[i]) * vals
    q, k = _unit(D, rng), _unit(D, rng)
    v = rng.standard_normal(D).astype(np.float32)
    g = rng.uniform(0.8, 1.0, D).astype(np.float32)
    beta = np.float32(0.7)
    out, y, _, st = orc.step_unit(bits, r, c, page, q, k, v, beta, g, D, fmt, w=w)
    assert st == orc.OK
    X, y_ref = _explicit(S64, q, k, v, float(beta), g)
    np.testing.assert_allclose(y, y_ref, rtol=1e-9, atol=1e-12)
    for i, vals in _pivot_values(out, bits, D, fmt).items():
        want = (X[i] / float(r[i])).astype(np.float32).astype(np.float16).astype(np.float64)
        np.testing.assert_array_equal(vals, want)
    s, cn, zn = _read_np(out, bits, D, fmt)
    V = (s[:, None] * r[:, None].astype(np.float64) * zn)[~piv]
    W2 = (w.astype(np.float64) ** 2)[~piv, None]
    resid = (W2 * V * (X[~piv] - cn[None, :] * V)).sum(0)
    scale = (W2 * V * V).sum(0) * np.abs(cn)
    assert np.all(np.abs(resid) <= 2e-7 * scale + 1e-300), (resid, scale)

"""Pins of the oracle's storage formats: binary16 scales and raw units.

The page stores per-row scales in FP16 ("method steps", step 6, and the
kernel-efficiency paragraph) and keeps a few "pivot" units in FP16 without
quantisation ("core method"); the fp32 control state is the unquantized
recurrence the page's state-update timings compare against.  Each pin checks
the oracle against something other than itself: numpy's IEEE binary16
conversion, the explicit-matrix form of the gated delta rule, or an exact
identity of the quantiser.
"""
import numpy as np
import pytest

import oracle as orc

RNG = lambda s: np.random.default_rng(s)  # noqa: E731  (test-local inputs only)
D = 8  # tiny heads keep the pure-Python readers fast


def _explicit_step(S, q, k, v, beta, g):
    """S_t = (I - beta k k^T) D S + beta k v^T, y = S_t^T q, explicit matrices, fp64."""
    k = k.astype(np.float64)
    dk = len(k)
    A = (np.eye(dk) - beta * np.outer(k, k)) @ np.diag(np.broadcast_to(g, (dk,)).astype(np.float64))
    X = A @ S + beta * np.outer(k, v.astype(np.float64))
    return X, X.T @ q.astype(np.float64)


def _unit(n, rng):
    x = rng.standard_normal(n)
    return (x / np.linalg.norm(x)).astype(np.float32)


def _codes(page, bits, dv, fmt):
    offs = orc.row_offsets(bits, dv, fmt)
    z = np.zeros((len(bits), dv), np.int64)
    for i, b in enumerate(bits):
        row = page[offs[i]: offs[i] + dv * int(b) // 8]
        for j in range(dv):
            z[i, j] = orc.get_code(row, int(b), j, dv=dv)
    return z


def _raw_values(page, bits, dv):
    b = int(bits[0])
    dt = np.float16 if b == 16 else np.float32
    return page[: len(bits) * dv * b // 8].view(dt).reshape(len(bits), dv).astype(np.float64)


# ---------------------------------------------------------------- binary16


def test_half_decoder_exhaustive_against_numpy():
    pats = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    ref = pats.view(np.float16).astype(np.float64)
    got = np.array([orc.half_to_double(int(h)) for h in pats])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


def test_half_encoder_against_numpy_including_exact_ties():
    rng = RNG(1)
    finite = np.arange(0, 0x7C00, dtype=np.uint16).view(np.float16).astype(np.float64)
    # exact midpoints between neighbouring binary16 values (ties to even), both signs
    mids = (finite[:-1] + finite[1:]) / 2
    xs = np.concatenate([
        mids, -mids,
        rng.uniform(-70000, 70000, 20000),
        rng.standard_normal(20000) * 1e-5,                 # subnormal range
        np.exp(rng.uniform(np.log(1e-9), np.log(7e4), 20000)),
        [0.0, -0.0, 65504.0, 65519.999, 65520.0, 1e30, -1e30, 2.0 ** -25, 2.0 ** -24 * 1.5],
    ])
    with np.errstate(over="ignore"):
        ref = xs.astype(np.float16).view(np.uint16)
    got = np.array([orc.double_to_half(float(x)) for x in xs], np.uint16)
    bad = np.nonzero(got != ref)[0]
    assert len(bad) == 0, (xs[bad][:5], got[bad][:5], ref[bad][:5])


# ---------------------------------------------------------------- binary16 scales


@pytest.mark.parametrize("b", [4, 6, 8])
def test_f16_scale_grid(b):
    """s16 = half(a / q_b), and every code is round(mu / s16) clipped: the
    row's argmax gets +-q_b and no code leaves [-q_b, q_b]."""
    rng = RNG(b)
    qb = (1 << (b - 1)) - 1
    bits = np.full(D, b, np.uint8)
    r = np.exp(rng.uniform(-1, 1, D)).astype(np.float32)
    c = np.exp(rng.uniform(-1, 1, D)).astype(np.float32)
    S = (rng.standard_normal((D, D)) * np.exp(rng.uniform(-3, 3, (D, 1)))).astype(np.float32)
    S[3] = 0.0
    page, quot, st = orc.quantize_unit(bits, r, c, S, with_quot=True, fmt=orc.FMT_F16)
    assert st == orc.OK
    assert len(page) == orc.page_bytes(bits, D, orc.FMT_F16) == 128  # 2 D + D^2 b / 8, padded
    s16 = page[: 2 * D].view(np.float16)
    mu = (S.astype(np.float64) / (r[:, None].astype(np.float64) * c[None, :])).astype(np.float32)
    a = np.abs(mu).max(axis=1)
    assert np.array_equal(s16.view(np.uint16), (a / np.float32(qb)).astype(np.float16).view(np.uint16))
    z = _codes(page, bits, D, orc.FMT_F16)
    assert np.all(np.abs(z) <= qb)
    for i in range(D):
        if a[i] == 0:
            assert s16[i] == 0 and np.all(z[i] == 0)
            continue
        jm = np.argmax(np.abs(mu[i]))
        assert z[i, jm] == np.sign(mu[i, jm]) * qb
        ref = np.clip(np.rint(mu[i] / np.float32(s16[i])), -qb, qb)
        assert np.array_equal(z[i], ref)


def test_f16_scale_requant_idempotent():
    """beta = 0, gate = 1: X is the reconstruction s16 r c z itself, so the
    step reproduces codes and binary16 scales bit for bit (s16 q_b / q_b = s16
    exactly, and the row's argmax code is +-q_b)."""
    rng = RNG(7)
    for b in (4, 6, 8):
        bits = np.full(D, b, np.uint8)
        r = np.exp(rng.uniform(-1, 1, D)).astype(np.float32)
        c = np.exp(rng.uniform(-1, 1, D)).astype(np.float32)
        S = rng.standard_normal((D, D)).astype(np.float32)
        page = orc.quantize_unit(bits, r, c, S, fmt=orc.FMT_F16)
        q, k, v = _unit(D, rng), _unit(D, rng), rng.standard_normal(D).astype(np.float32)
        out, _, _, st = orc.step_unit(bits, r, c, page, q, k, v, 0.0, np.float32(1.0), fmt=orc.FMT_F16)
        assert st == orc.OK
        assert out.tobytes() == page.tobytes()


def test_f16_scale_overflow_is_reported():
    bits = np.full(D, 8, np.uint8)
    S = np.zeros((D, D), np.float32)
    S[2, 5] = 127.0 * 70000.0  # a / q_b = 70000 > 65504
    page, _, st = orc.quantize_unit(bits, np.ones(D), np.ones(D), S, with_quot=True, fmt=orc.FMT_F16)
    assert st == orc.NONFINITE
    s16 = page[: 2 * D].view(np.float16)
    assert np.isinf(s16[2]) and np.all(_codes(page, bits, D, orc.FMT_F16)[2] == 0)


# ---------------------------------------------------------------- raw units


@pytest.mark.parametrize("b", [16, 32])
@pytest.mark.parametrize("kind", ["gdn", "kda"])
def test_raw_step_is_the_rounded_explicit_recurrence(b, kind):
    rng = RNG(b + (kind == "kda"))
    bits = np.full(D, b, np.uint8)
    dt = np.float16 if b == 16 else np.float32
    S0 = (rng.standard_normal((D, D)) * 3).astype(dt)
    page = orc.quantize_unit(bits, np.ones(D), np.ones(D), S0.astype(np.float32))
    assert len(page) == 128 * ((D * D * b // 8 + 127) // 128)
    assert np.array_equal(_raw_values(page, bits, D), S0.astype(np.float64))
    q, k, v = _unit(D, rng), _unit(D, rng), rng.standard_normal(D).astype(np.float32)
    beta = np.float32(rng.uniform(0, 1))
    g = rng.uniform(0.8, 1.0, D).astype(np.float32) if kind == "kda" else np.float32(0.93)
    r = np.exp(rng.uniform(-1, 1, D)).astype(np.float32)  # ignored by raw units
    out, y, quot, st = orc.step_unit(bits, r, r, page, q, k, v, beta, g)
    assert st == orc.OK
    X, y_ref = _explicit_step(S0.astype(np.float64), q, k, v, float(beta), g)
    np.testing.assert_allclose(y, y_ref, rtol=1e-12, atol=1e-12 * np.abs(y_ref).max())
    got = _raw_values(out, bits, D)
    want = X.astype(dt).astype(np.float64)
    # identical except where X lies within fp64 noise of a rounding midpoint
    diff = got != want
    if diff.any():
        ulp = np.abs(np.spacing(X.astype(dt)).astype(np.float64))
        assert np.all(np.abs(got - want)[diff] <= ulp[diff])
        assert diff.sum() <= 1
    np.testing.assert_allclose(quot, X.astype(np.float32), rtol=1e-6)
    back = orc.dequantize_unit(bits, r, r, out)
    assert np.array_equal(back.astype(np.float64), got)


def test_raw_retrieval_identity():
    """beta = 1, q = k unit-norm: y = v exactly in exact arithmetic ("gated delta rule")."""
    rng = RNG(3)
    bits = np.full(D, 32, np.uint8)
    S0 = rng.standard_normal((D, D)).astype(np.float32)
    page = orc.quantize_unit(bits, np.ones(D), np.ones(D), S0)
    k = _unit(D, rng)
    v = rng.standard_normal(D).astype(np.float32)
    _, y, _, _ = orc.step_unit(bits, np.ones(D), np.ones(D), page, k, k, v, 1.0, np.float32(0.9))
    np.testing.assert_allclose(y, v, rtol=0, atol=1e-6 * np.abs(v).max())


def test_raw_units_must_be_uniform():
    bits = np.full(D, 16, np.uint8)
    bits[3] = 8
    with pytest.raises(ValueError):
        orc.quantize_unit(bits, np.ones(D), np.ones(D), np.zeros((D, D), np.float32))


# ---------------------------------------------------------------- FP16 pivot rows among quantized rows


PIV = orc.FMT_PIVOT


def _pivot_values(page, bits, dv, fmt):
    offs = orc.row_offsets(bits, dv, fmt)
    out = np.full((len(bits), dv), np.nan)
    for i, b in enumerate(bits):
        if b == 16:
            out[i] = page[offs[i]: offs[i] + 2 * dv].view(np.float16).astype(np.float64)
    return out


@pytest.mark.parametrize("fmt", [PIV, PIV | orc.FMT_F16])
def test_pivot_rows_round_trip_exactly_and_leave_other_rows_alone(fmt):
    """Values representable in binary16 come back exactly from pivot rows (scale slot 1);
    the quantized rows are byte-identical to the same rows quantized without pivots."""
    rng = RNG(40)
    bits = np.array([6, 16, 8, 4, 16, 6, 8, 16], np.uint8)
    S = rng.standard_normal((D, D)).astype(np.float16).astype(np.float32)
    ones = np.ones(D, np.float32)
    page = orc.quantize_unit(bits, ones, ones, S, fmt=fmt)
    assert len(page) == orc.page_bytes(bits, D, fmt)
    back = orc.dequantize_unit(bits, ones, ones, page, D, fmt)
    piv = bits == 16
    np.testing.assert_array_equal(back[piv], S[piv])
    sc = page[: 2 * D].view(np.float16).astype(np.float32) if fmt & orc.FMT_F16 else page[: 4 * D].view(np.float32)
    np.testing.assert_array_equal(sc[piv], 1.0)
    alt = bits.copy()
    alt[piv] = 8
    ref = orc.quantize_unit(alt, ones, ones, S, fmt=fmt & orc.FMT_F16)
    offs, offs_alt = orc.row_offsets(bits, D, fmt), orc.row_offsets(alt, D, fmt & orc.FMT_F16)
    for i in np.nonzero(~piv)[0]:
        n = D * int(bits[i]) // 8
        assert page[offs[i]: offs[i] + n].tobytes() == ref[offs_alt[i]: offs_alt[i] + n].tobytes()
    np.testing.assert_array_equal(sc[~piv], (ref[: 2 * D].view(np.float16).astype(np.float32)
                                            if fmt & orc.FMT_F16 else ref[: 4 * D].view(np.float32))[~piv])


def test_pivot_rows_hold_the_binary16_state_over_the_factors():
    """With r, c != 1 a pivot row stores half(fl32(X / (r c))): the rank-one first step
    from zero, X = beta k v^T, checked element by element with numpy's binary16."""
    rng = RNG(41)
    bits = np.array([16, 6, 16, 8, 16, 4, 6, 16], np.uint8)
    r = np.exp(rng.uniform(-1, 1, D)).astype(np.float32)
    c = np.exp(rng.uniform(-1, 1, D)).astype(np.float32)
    page0 = orc.quantize_unit(bits, r, c, np.zeros((D, D), np.float32), fmt=PIV)
    k, q = _unit(D, rng), _unit(D, rng)
    v = rng.standard_normal(D).astype(np.float32)
    beta = np.float32(0.7)
    out, y, quot, st = orc.step_unit(bits, r, c, page0, q, k, v, beta, np.full(D, 0.9, np.float32), D, PIV)
    assert st == orc.OK
    X = float(beta) * np.outer(k.astype(np.float64), v.astype(np.float64))
    mu = (X / np.outer(r.astype(np.float64), c.astype(np.float64))).astype(np.float32)
    got = _pivot_values(out, bits, D, PIV)
    piv = bits == 16
    np.testing.assert_array_equal(got[piv], mu[piv].astype(np.float16).astype(np.float64))
    np.testing.assert_allclose(y, X.T @ q.astype(np.float64), rtol=1e-12, atol=1e-15)


def test_pivot_unit_equals_raw16_unit_when_factors_are_one():
    """A head made only of pivot rows (r = c = 1) takes the raw binary16 unit's step:
    same readout, same stored values."""
    rng = RNG(42)
    bits = np.full(D, 16, np.uint8)
    ones = np.ones(D, np.float32)
    S = rng.standard_normal((D, D)).astype(np.float32)
    p_piv = orc.quantize_unit(bits, ones, ones, S, fmt=PIV)
    p_raw = orc.quantize_unit(bits, ones, ones, S)
    for t in range(4):
        q, k = _unit(D, rng), _unit(D, rng)
        v = rng.standard_normal(D).astype(np.float32)
        g = rng.uniform(0.8, 1.0, D).astype(np.float32)
        p_piv, y1, _, s1 = orc.step_unit(bits, ones, ones, p_piv, q, k, v, np.float32(0.6), g, D, PIV)
        p_raw, y2, _, s2 = orc.step_unit(bits, ones, ones, p_raw, q, k, v, np.float32(0.6), g, D)
        assert s1 == s2 == orc.OK
        np.testing.assert_array_equal(y1, y2)
        np.testing.assert_array_equal(_pivot_values(p_piv, bits, D, PIV), _raw_values(p_raw, bits, D))


def test_pivot_step_is_the_rounded_explicit_recurrence():
    """Mixed unit: the pivot rows of the next page are the explicit recurrence (fp64, on
    the reconstructed state) over r c, rounded to fp32 then binary16; the readout is
    the explicit readout."""
    rng = RNG(43)
    bits = np.array([6, 16, 8, 16, 4, 6, 16, 8], np.uint8)
    r = np.exp(rng.uniform(-0.5, 0.5, D)).astype(np.float32)
    c = np.exp(rng.uniform(-0.5, 0.5, D)).astype(np.float32)
    page = orc.quantize_unit(bits, r, c, rng.standard_normal((D, D)).astype(np.float32), fmt=PIV)
    q, k = _unit(D, rng), _unit(D, rng)
    v = rng.standard_normal(D).astype(np.float32)
    g = rng.uniform(0.8, 1.0, D).astype(np.float32)
    S_hat = orc.dequantize_unit(bits, r, c, page, D, PIV).astype(np.float64)
    # the reconstruction itself, recomputed from the stored values
    Sv = _pivot_values(page, bits, D, PIV)
    piv = bits == 16
    np.testing.assert_array_equal(S_hat[piv], (np.outer(r.astype(np.float64), c.astype(np.float64)) * Sv)[piv].astype(np.float32))
    exact = np.outer(r.astype(np.float64), c.astype(np.float64)) * np.where(np.isnan(Sv), 0, Sv)
    exact[~piv] = S_hat[~piv]
    out, y, _, st = orc.step_unit(bits, r, c, page, q, k, v, np.float32(0.8), g, D, PIV)
    X, y_ref = _explicit_step(exact, q, k, v, 0.8, g)
    np.testing.assert_allclose(y, y_ref, rtol=1e-6, atol=1e-6 * np.abs(y_ref).max())
    mu = (X / np.outer(r.astype(np.float64), c.astype(np.float64))).astype(np.float32).astype(np.float16)
    got = _pivot_values(out, bits, D, PIV)
    # the explicit form and the oracle's delta form agree to fp64 rounding; both then round
    # to binary16, which can differ by one step only next to a rounding midpoint
    d = np.abs(got[piv] - mu[piv].astype(np.float64))
    spacing = np.abs(np.spacing(mu[piv])).astype(np.float64)
    assert np.all(d <= spacing)
    assert np.count_nonzero(d) <= 1


def test_pivot_rows_need_the_flag_and_reject_32():
    ones = np.ones(D, np.float32)
    S = np.zeros((D, D), np.float32)
    with pytest.raises(ValueError):
        orc.quantize_unit(np.array([6, 16, 6, 6, 6, 6, 6, 6], np.uint8), ones, ones, S)
    with pytest.raises(ValueError):
        orc.quantize_unit(np.array([6, 32, 6, 6, 6, 6, 6, 6], np.uint8), ones, ones, S, fmt=PIV)

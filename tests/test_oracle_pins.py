"""Pins of the CPU oracle against facts the STEPQuant page and mathematics fix.

Nothing here compares the oracle with itself: each test checks it against a
hand-worked example, a closed form, an invariant of the recurrence, the
explicit-matrix form of the gated delta rule (a different formula from the
delta form the oracle evaluates), or brute force on tiny heads.

Page: "STEPQuant: When and Where Errors Matter in Delta-Rule Recurrent State
Quantization"; sections cited by name.
"""
import os

import numpy as np
import pytest

import oracle as orc
from quantized_linear_attention_decode_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
RNG = lambda s: np.random.default_rng(s)  # noqa: E731  (test-local inputs only)


def _codes(page, bits, dv):
    """All codes of a page, read with the oracle's unpacker (itself pinned
    by the pack tests below)."""
    offs = orc.row_offsets(bits, dv)
    z = np.zeros((len(bits), dv), np.int64)
    for i, b in enumerate(bits):
        row = page[offs[i]: offs[i] + dv * int(b) // 8]
        for j in range(dv):
            z[i, j] = orc.get_code(row, int(b), j, dv=dv)
    return z


def _scales(page, dk):
    return page[: 4 * dk].view(np.float32).copy()


def _reconstruct64(page, bits, r, c, dv):
    z = _codes(page, bits, dv)
    s = _scales(page, len(bits)).astype(np.float64)
    return s[:, None] * r.astype(np.float64)[:, None] * c.astype(np.float64)[None, :] * z


def _explicit_step(S, q, k, v, beta, g):
    """[gated delta rule]: S_t = (I - beta k k^T) D S + beta k v^T, y = S_t^T q,
    with explicit dk x dk matrices, in fp64."""
    k = k.astype(np.float64)
    dk = len(k)
    A = (np.eye(dk) - beta * np.outer(k, k)) @ np.diag(np.broadcast_to(g, (dk,)).astype(np.float64))
    X = A @ S + beta * np.outer(k, v.astype(np.float64))
    return X, X.T @ q.astype(np.float64)


def _unit(n, rng):
    x = rng.standard_normal(n)
    return (x / np.linalg.norm(x)).astype(np.float32)


# ---------------------------------------------------------------- packing


def test_pack_golden_rows():
    for line in open(os.path.join(GOLDEN, "pack_rows.txt")):
        if not line.strip() or line.startswith("#"):
            continue
        parts = line.split()
        b = int(parts[0])
        codes = [int(x) for x in parts[1].split(",")]
        want = bytes(int(h, 16) for h in parts[2:])
        row = np.zeros(len(want), np.uint8)
        n = len(codes)
        for j, z in enumerate(codes):
            orc.put_code(row, b, j, z, dv=n)
        assert row.tobytes() == want, (b, codes, row.tobytes().hex())
        assert [orc.get_code(row, b, j, dv=n) for j in range(n)] == codes


@pytest.mark.parametrize("b", [4, 6, 8])
def test_pack_roundtrip_every_code_every_position(b):
    dv = 128
    nb = dv * b // 8
    rng = RNG(b)
    lo, hi = -(1 << (b - 1)), (1 << (b - 1)) - 1
    for j in range(dv):
        base = rng.integers(lo, hi + 1, size=dv)
        row = np.zeros(nb, np.uint8)
        for jj in range(dv):
            orc.put_code(row, b, jj, int(base[jj]))
        for z in range(lo, hi + 1):
            orc.put_code(row, b, j, z)
            assert orc.get_code(row, b, j) == z
            # neighbours untouched
            if j > 0:
                assert orc.get_code(row, b, j - 1) == base[j - 1]
            if j + 1 < dv:
                assert orc.get_code(row, b, j + 1) == base[j + 1]


def test_page_layout_sizes():
    # scales (4 dk bytes) + rows of dv*b/8 bytes, padded to 128
    for b in (4, 6, 8):
        assert orc.page_bytes(np.full(128, b, np.uint8)) == 512 + 2048 * b
    bits = np.array([4] * 32 + [6] * 64 + [8] * 32, np.uint8)
    assert orc.page_bytes(bits) == 512 + 16 * (32 * 4 + 64 * 6 + 32 * 8)
    assert orc.page_bytes(np.array([4, 4, 4, 4], np.uint8), 4) == 128


# ---------------------------------------------------------------- worked example


def _read_fixture(name):
    d = {}
    for line in open(os.path.join(GOLDEN, name)):
        if not line.strip() or line.startswith("#"):
            continue
        key, val = line.split(None, 1)
        d[key] = val.strip()
    return d


def test_worked_step_d4():
    fx = _read_fixture("worked_step_d4.txt")
    vec = lambda key: np.array([float(x) for x in fx[key].split(",")])  # noqa: E731
    dk, dv = int(fx["dk"]), int(fx["dv"])
    bits = np.array([int(x) for x in fx["bits"].split(",")], np.uint8)
    ones = np.ones(dk, np.float32)
    page0 = orc.quantize_unit(bits, ones, ones, np.zeros((dk, dv), np.float32))
    assert not page0.any()
    page1, y, quot, st = orc.step_unit(bits, ones, ones, page0, vec("q"), vec("k"), vec("v"),
                                       float(fx["beta"]), vec("gate"))
    assert st == orc.OK
    assert len(page1) == int(fx["page_bytes"])
    np.testing.assert_array_equal(y, vec("y"))
    np.testing.assert_array_equal(_scales(page1, dk), vec("scales").astype(np.float32))
    z = _codes(page1, bits, dv)
    for i in range(dk):
        np.testing.assert_array_equal(z[i], vec(f"codes_row{i}"))
    row0 = bytes(int(h, 16) for h in fx["row0_bytes"].split())
    assert page1[4 * dk: 4 * dk + 2].tobytes() == row0


# ---------------------------------------------------------------- recurrence


@pytest.mark.parametrize("kind", ["gdn", "kda"])
def test_unquantized_step_matches_explicit_matrix_form(kind):
    rng = RNG(1)
    for d in (2, 4, 8):
        S = rng.standard_normal((d, d))
        for _ in range(5):
            q, k = _unit(d, rng), _unit(d, rng)
            v = rng.standard_normal(d).astype(np.float32)
            beta = np.float32(rng.uniform())
            g = (np.full(d, rng.uniform(0.5, 1.0)) if kind == "gdn"
                 else rng.uniform(0.5, 1.0, d)).astype(np.float32)
            S_new, y = orc.step_unit_f64(S, q, k, v, beta, g)
            X, y_ref = _explicit_step(S, q, k, v, float(beta), g)
            np.testing.assert_allclose(S_new, X, rtol=0, atol=1e-12 * np.abs(X).max())
            np.testing.assert_allclose(y, y_ref, rtol=0, atol=1e-12 * np.abs(y_ref).max())
            S = S_new


def test_retrieval_identity_unquantized():
    """beta = 1, |k| = 1: S_t^T k = v (the delta rule writes v at key k)."""
    rng = RNG(2)
    d = 16
    S = rng.standard_normal((d, d))
    for _ in range(10):
        k = _unit(d, rng)
        v = rng.standard_normal(d).astype(np.float32)
        g = np.full(d, 0.97, np.float32)
        S, _ = orc.step_unit_f64(S, k, k, v, 1.0, g)
        kk = float(np.dot(k.astype(np.float64), k.astype(np.float64)))
        slack = abs(kk - 1.0) * 10 * (np.abs(S).max() + 1)
        np.testing.assert_allclose(S.T @ k.astype(np.float64), v, rtol=0, atol=1e-12 + slack)


@pytest.mark.parametrize("bits", [4, 6, 8])
def test_retrieval_identity_quantized_readout(bits):
    """Readout before requantisation ([method steps], step 3): with beta = 1,
    q = k, |k| = 1, y = X^T k = v even though the state is quantized."""
    rng = RNG(3)
    d = 32
    b = np.full(d, bits, np.uint8)
    r = np.exp(rng.uniform(-1, 1, d)).astype(np.float32)
    c = np.exp(rng.uniform(-1, 1, d)).astype(np.float32)
    page = orc.quantize_unit(b, r, c, rng.standard_normal((d, d)).astype(np.float32))
    for _ in range(6):
        k = _unit(d, rng)
        v = rng.standard_normal(d).astype(np.float32)
        page, y, _, st = orc.step_unit(b, r, c, page, k, k, v, 1.0, np.full(d, 0.95, np.float32))
        assert st == orc.OK
        np.testing.assert_allclose(y, v, rtol=0, atol=2e-6 * np.abs(v).max())


@pytest.mark.parametrize("kind", ["gdn", "kda"])
def test_quantized_step_continuous_part_matches_explicit_form(kind):
    """The pre-quantisation state X and readout y of the oracle's step equal
    the explicit-matrix recurrence applied to the reconstructed state."""
    rng = RNG(4)
    for d, bits in ((4, 4), (8, 6), (8, 8)):
        # 6-bit rows pack codes in groups of eight, so they need dv % 8 == 0
        widths = [4, 6, 8] if d % 8 == 0 else [4, 8]
        b = np.full(d, bits, np.uint8) if kind == "gdn" else rng.choice(widths, d).astype(np.uint8)
        r = np.exp(rng.uniform(-1.4, 1.4, d)).astype(np.float32)
        c = np.exp(rng.uniform(-1.4, 1.4, d)).astype(np.float32)
        page = orc.quantize_unit(b, r, c, rng.standard_normal((d, d)).astype(np.float32))
        for _ in range(4):
            q, k = _unit(d, rng), _unit(d, rng)
            v = rng.standard_normal(d).astype(np.float32)
            beta = np.float32(rng.uniform())
            g = (np.full(d, rng.uniform(0.8, 1.0)) if kind == "gdn" else rng.uniform(0.8, 1.0, d)
                 ).astype(np.float32)
            Shat = _reconstruct64(page, b, r, c, d)
            X, y_ref = _explicit_step(Shat, q, k, v, float(beta), g)
            page_new, y, quot, st = orc.step_unit(b, r, c, page, q, k, v, beta, g)
            assert st == orc.OK
            np.testing.assert_allclose(y, y_ref, rtol=0, atol=1e-12 * max(np.abs(y_ref).max(), 1))
            # quantizer bound [PTQ]: |Q(x) - x| <= s/2 in the (r, c)-scaled grid
            s_new = _scales(page_new, d).astype(np.float64)
            rc = r.astype(np.float64)[:, None] * c.astype(np.float64)[None, :]
            err = np.abs(_reconstruct64(page_new, b, r, c, d) - X)
            bound = 0.5 * s_new[:, None] * rc * (1 + 1e-5) + 1e-6 * np.abs(X)
            assert (err <= bound).all()
            page = page_new


# ---------------------------------------------------------------- quantizer


def test_absmax_grid():
    """s_i = a_i / q_b with a_i the row absmax of X/(r c); the argmax element
    gets code +-q_b; every |z| <= q_b ([PTQ], [smoothing] absmax)."""
    rng = RNG(5)
    d = 128
    for bits in (4, 6, 8):
        qb = (1 << (bits - 1)) - 1
        b = np.full(d, bits, np.uint8)
        r = np.exp(rng.uniform(-1.4, 1.4, d)).astype(np.float32)
        c = np.exp(rng.uniform(-1.4, 1.4, d)).astype(np.float32)
        S = (rng.standard_normal((d, d)) * np.exp(rng.uniform(-3, 3, (d, 1)))).astype(np.float32)
        S[7] = 0.0  # an all-zero row
        page = orc.quantize_unit(b, r, c, S)
        z = _codes(page, b, d)
        s = _scales(page, d)
        mu = (S.astype(np.float64) / (r.astype(np.float64)[:, None] * c.astype(np.float64)[None, :])
              ).astype(np.float32)
        a = np.abs(mu).max(axis=1)
        np.testing.assert_array_equal(s, a / np.float32(qb))
        assert np.abs(z).max() <= qb
        for i in range(d):
            if a[i] == 0:
                assert s[i] == 0 and not z[i].any()
            else:
                jmax = int(np.argmax(np.abs(mu[i])))
                assert abs(z[i, jmax]) == qb and np.sign(z[i, jmax]) == np.sign(mu[i, jmax])


def test_requant_idempotent_and_power_of_two_gate():
    """beta = 0, alpha = 1: X = S^ and requantisation reproduces the codes;
    with alpha = 2^-m the codes stay and the scales scale exactly by 2^-m."""
    rng = RNG(6)
    d = 128
    for bits in (4, 6, 8):
        b = np.full(d, bits, np.uint8)
        r = np.exp(rng.uniform(-1.4, 1.4, d)).astype(np.float32)
        c = np.exp(rng.uniform(-1.4, 1.4, d)).astype(np.float32)
        page = orc.quantize_unit(b, r, c, rng.standard_normal((d, d)).astype(np.float32))
        z0, s0 = _codes(page, b, d), _scales(page, d)
        zero = np.zeros(d, np.float32)
        q = _unit(d, rng)
        p1, _, _, _ = orc.step_unit(b, r, c, page, q, _unit(d, rng), zero, 0.0, np.ones(d, np.float32))
        np.testing.assert_array_equal(_codes(p1, b, d), z0)
        np.testing.assert_allclose(_scales(p1, d), s0, rtol=2.5e-7, atol=0)
        for m in (1, 3):
            p2, _, _, _ = orc.step_unit(b, r, c, p1, q, _unit(d, rng), zero, 0.0,
                                        np.full(d, 2.0 ** -m, np.float32))
            np.testing.assert_array_equal(_codes(p2, b, d), z0)
            np.testing.assert_array_equal(_scales(p2, d), _scales(p1, d) * np.float32(2.0 ** -m))


def test_rank_one_first_step():
    """S_0 = 0, r = c = 1: X = beta k v^T, so row i's codes are
    sign(k_i) round(q_b v_j / |v|_inf) and y = beta (k.q) v."""
    rng = RNG(7)
    d = 128
    for bits in (4, 6, 8):
        qb = (1 << (bits - 1)) - 1
        b = np.full(d, bits, np.uint8)
        ones = np.ones(d, np.float32)
        page0 = orc.quantize_unit(b, ones, ones, np.zeros((d, d), np.float32))
        q, k = _unit(d, rng), _unit(d, rng)
        v = rng.standard_normal(d).astype(np.float32)
        beta = np.float32(0.625)
        page1, y, _, _ = orc.step_unit(b, ones, ones, page0, q, k, v, beta, np.full(d, 0.9, np.float32))
        np.testing.assert_allclose(y, float(beta) * float(np.dot(k.astype(np.float64), q)) * v.astype(np.float64),
                                   rtol=1e-12, atol=1e-15)
        x = qb * v.astype(np.float64) / np.abs(v).max()
        tie = np.abs(np.abs(x - np.floor(x)) - 0.5) < 1e-4
        want = np.sign(k.astype(np.float64))[:, None] * np.rint(x)[None, :]
        z = _codes(page1, b, d)
        mask = (k != 0)[:, None] & ~tie[None, :]
        np.testing.assert_array_equal(z[mask], want[mask])


# ---------------------------------------------------------------- error propagation


@pytest.mark.parametrize("bits", [4, 8])
def test_prop1_error_bound(bits):
    """Prop. 1 of the page (motivation / core-method sections): the state
    error E_t = S^_t - S_t obeys E_t = A_t E_{t-1} + eps_t with |A_t|_2 <= 1
    when |k| = 1 and beta, alpha in [0, 1], so |E_t|_F <= sum |eps_tau|_F;
    every eps_ij lies within the quantizer's half step."""
    rng = RNG(8)
    d = 32
    b = np.full(d, bits, np.uint8)
    r = np.exp(rng.uniform(-1, 1, d)).astype(np.float32)
    c = np.exp(rng.uniform(-1, 1, d)).astype(np.float32)
    S0 = rng.standard_normal((d, d)).astype(np.float32)
    page = orc.quantize_unit(b, r, c, S0)
    S = _reconstruct64(page, b, r, c, d)  # exact recurrence starts from the same state
    total = 0.0
    for t in range(60):
        q, k = _unit(d, rng), _unit(d, rng)
        v = rng.standard_normal(d).astype(np.float32)
        beta = np.float32(rng.uniform())
        g = np.full(d, rng.uniform(0.9, 1.0), np.float32)
        X, _ = _explicit_step(_reconstruct64(page, b, r, c, d), q, k, v, float(beta), g)
        page, _, _, _ = orc.step_unit(b, r, c, page, q, k, v, beta, g)
        Shat = _reconstruct64(page, b, r, c, d)
        eps = Shat - X
        s = _scales(page, d).astype(np.float64)
        rc = r.astype(np.float64)[:, None] * c.astype(np.float64)[None, :]
        assert (np.abs(eps) <= 0.5 * s[:, None] * rc * (1 + 1e-5) + 1e-6 * np.abs(X)).all()
        total += np.linalg.norm(eps)
        S, _ = orc.step_unit_f64(S, q, k, v, beta, g)
        assert np.linalg.norm(Shat - S) <= total * (1 + 1e-5) + 1e-9


# ---------------------------------------------------------------- accounting


def test_pool_accounting_matches_printed_numbers():
    """Pool = concurrency x slots x per-request state (section "SGLang state
    pool"); the printed serving numbers (results section, batch 512, 5 slots,
    Qwen 2304 GDN heads, Kimi 81920 KDA key rows) follow from it."""
    gib = 2.0 ** 30
    fp32_qwen = 512 * 5 * 2304 * 128 * 128 * 4
    assert fp32_qwen == 360 * 2 ** 30
    # state at 6.3611 bit/value (reproducibility section) shrinks total 419.73 GiB to ~131.18
    saved = fp32_qwen / gib * (1 - 6.3611 / 32)
    assert abs((419.73 - saved) - 131.18) < 0.2
    assert round(32 / 6.3611, 2) == 5.03 and round(32 / 4.6209, 2) == 6.93 and round(32 / 6.30, 2) == 5.08
    fp32_kimi = 512 * 5 * (81920 // 128) * 128 * 128 * 4
    assert fp32_kimi == 100 * 2 ** 30
    assert abs((149.70 - fp32_kimi / gib * (1 - 6.30 / 32)) - 69.36) < 0.1
    # the FP32 pool passes ~54 GB of BF16 weights near 70 concurrent requests
    per_req = 5 * 2304 * 128 * 128 * 4
    assert 68 <= 27e9 * 2 / per_req <= 73


def test_synth_is_deterministic_and_shaped():
    wl = synth.make_workload(2, seed=0, R=3, H=4, T=2)
    a, b = wl.step_inputs(1), wl.step_inputs(1)
    for key in a:
        np.testing.assert_array_equal(a[key], b[key])
    assert a["q"].shape == (3, 4, 128) and a["gate"].shape == (3, 4)
    np.testing.assert_allclose(np.linalg.norm(a["k"].astype(np.float64), axis=-1), 1.0, atol=1e-6)
    sub = wl.step_inputs(1, requests=np.array([2]))
    np.testing.assert_array_equal(sub["v"][0], a["v"][2])
    assert sorted(np.bincount(wl.unit_bits)[[4, 6, 8]]) == [1, 1, 2]
    wk = synth.make_workload(3, R=2, H=2, T=1)
    rb = wk.row_bits()
    assert rb.shape == (2, 128) and all(sorted(np.bincount(rb[h])[[4, 6, 8]]) == [32, 32, 64] for h in range(2))


def test_six_bit_rows_need_whole_groups():
    """6-bit codes are stored in groups of eight: a unit whose rows hold a
    number of codes that is not a multiple of 8 has no 6-bit layout."""
    S = np.ones((8, 4), np.float32)
    ones = np.ones(8, np.float32)
    with pytest.raises(ValueError):
        orc.quantize_unit(np.full(8, 6, np.uint8), ones, np.ones(4, np.float32), S)
    orc.quantize_unit(np.full(8, 8, np.uint8), ones, np.ones(4, np.float32), S)


# ---------------------------------------------------------------- the multi-unit driver


@pytest.mark.parametrize("nthreads", [1, 4])
def test_step_many_matches_unit_by_unit(nthreads):
    """The OpenMP driver that the CPU baseline times advances each unit
    exactly as a single-unit step does: per-head tables picked by head index,
    pages read and written at the given (shuffled, distinct) offsets, per-unit
    vectors and per-row gates.  Heads mix GDN-like uniform widths with
    KDA-like per-row widths, so a wrong head index, table stride or page offset
    changes some unit's page or readout."""
    rng = RNG(11)
    H, n = 5, 12
    bits = np.stack([np.full(128, 8, np.uint8), np.full(128, 4, np.uint8), np.full(128, 6, np.uint8),
                     rng.permutation(np.repeat(np.array([4, 6, 8], np.uint8), [32, 64, 32])),
                     rng.permutation(np.repeat(np.array([4, 8], np.uint8), [64, 64]))])
    r = np.exp(rng.uniform(-1, 1, (H, 128))).astype(np.float32)
    c = np.exp(rng.uniform(-1, 1, (H, 128))).astype(np.float32)
    head = rng.integers(0, H, n).astype(np.int32)
    head[:H] = np.arange(H)  # every head at least once
    sizes = np.array([orc.page_bytes(bits[h]) for h in head])
    # input pages packed in unit order; output pages in a shuffled order with gaps
    off_in = np.concatenate([[0], np.cumsum(sizes)[:-1]]).astype(np.int64)
    order = rng.permutation(n)
    off_out = np.zeros(n, np.int64)
    o = 64
    for u in order:
        off_out[u] = o
        o += sizes[u] + 128
    pages_in = np.zeros(int(sizes.sum()), np.uint8)
    for u in range(n):
        S = rng.standard_normal((128, 128)).astype(np.float32)
        pages_in[off_in[u]: off_in[u] + sizes[u]] = orc.quantize_unit(bits[head[u]], r[head[u]], c[head[u]], S)
    q = np.stack([_unit(128, rng) for _ in range(n)])
    k = np.stack([_unit(128, rng) for _ in range(n)])
    v = rng.standard_normal((n, 128)).astype(np.float32)
    beta = rng.uniform(0, 1, n).astype(np.float32)
    g = rng.uniform(0.8, 1.0, (n, 128)).astype(np.float32)
    out, y, bad = orc.step_many(head, bits, r, c, pages_in, off_in, off_out, o, q, k, v, beta, g, nthreads)
    assert bad == 0
    covered = np.zeros(o, bool)
    for u in range(n):
        h = head[u]
        ref, yref, _, st = orc.step_unit(bits[h], r[h], c[h], pages_in[off_in[u]: off_in[u] + sizes[u]],
                                         q[u], k[u], v[u], beta[u], g[u])
        assert st == orc.OK
        np.testing.assert_array_equal(out[off_out[u]: off_out[u] + sizes[u]], ref, err_msg=f"unit {u} page")
        np.testing.assert_array_equal(y[u], yref, err_msg=f"unit {u} readout")
        covered[off_out[u]: off_out[u] + sizes[u]] = True
    assert not out[~covered].any(), "bytes written outside the units' output pages"

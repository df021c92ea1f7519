"""GPU parity of the online column fit ("core method" dual-axis fit;
"method steps", steps 4-5): every page carries its own column factors,
refitted from the codes each step by the weighted least-squares closed form
with the frozen row weights.  Teacher-forced against the oracle like the
main parity tests (tolerances in tests/pages.py); the factors' own
tolerance is the same max relative error 1e-5."""
import dataclasses

import numpy as np
import pytest

import oracle as orc
from pages import FITC, PIVOT, Compare, col_factors, split_slot
from quantized_linear_attention_decode_b200 import stq, synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _cuda(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _weights(wl, seed):
    rng = np.random.default_rng(seed)
    return np.exp(rng.uniform(np.log(0.5), np.log(2.0), wl.H * 128)).astype(np.float32)


def _pool(wl, w, f16=False):
    flags = stq.STQ_FIT_COLUMNS | (stq.STQ_SCALE_F16 if f16 else 0)
    pool = stq.stq_pool_create(wl.kind, wl.R, wl.S, wl.H, wl.unit_bits, wl.row_factor, wl.col_factor,
                               flags=flags, row_weight=w)
    req = _cuda(np.arange(wl.R, dtype=np.int32))
    slot = _cuda(wl.slot_of_request.astype(np.int32))
    S0 = wl.initial_state()
    if S0 is not None:
        stq.stq_quantize_state(pool, req, slot, _cuda(S0))
        stq.stq_pool_check(pool)
    return pool, req, slot


def _kda_allocated_pivots(R, H, seed):
    """KDA with per-row widths from the lifetime-aware allocator (6-bit budget over
    {4, 6, 8} per head, Lagrangian) and its 8 riskiest rows per head kept as FP16
    pivots, outlier start: the page's KDA setting (pivot rows, column fit)."""
    wl = synth.make_workload(3, R=R, H=H)
    rng = np.random.default_rng(seed)
    ub = []
    for h in range(H):
        d = np.exp(rng.uniform(-2, 2, 128))[:, None] * 4.0 ** (-np.arange(3)[None, :])
        lw = stq.stq_lifetime_weight(np.log(rng.uniform(0.8, 0.9995, 128)), 8192)
        bits, _ = stq.stq_allocate_bits(np.full(128, 128.0), [4, 6, 8], d, lw, 6.0,
                                        method=stq.STQ_ALLOC_LAGRANGE, num_pivots=8, pivot_bits=16)
        assert int(np.count_nonzero(bits == 16)) == 8
        ub.append(bits)
    return dataclasses.replace(wl, unit_bits=np.concatenate(ub), init="outlier")


@pytest.mark.parametrize("config, f16", [(2, False), (3, False), (2, True), ("kda_pivots", False),
                                         ("kda_pivots", True)])
def test_fit_quantize_dequantize(config, f16):
    """Scales and codes bit-exact; the fitted factors (fp64 sums in another order)
    within 1e-7; the dequantized state uses the page's factors (pivot rows: none)."""
    if config == "kda_pivots":
        wl = _kda_allocated_pivots(2, 8, 5)
    else:
        wl = dataclasses.replace(synth.make_workload(config, R=2, H=8), init="outlier")
    w = _weights(wl, 3 if config == "kda_pivots" else config)
    fmt = FITC | (1 if f16 else 0) | (PIVOT if config == "kda_pivots" else 0)
    pool, req, slot = _pool(wl, w, f16)
    rb = wl.row_bits()
    r, c, W = wl.row_factor.reshape(wl.H, 128), wl.col_factor.reshape(wl.H, 128), w.reshape(wl.H, 128)
    S0 = wl.initial_state()
    back = torch.empty((wl.R, wl.H, 128, 128), dtype=torch.float32, device="cuda")
    stq.stq_dequantize_state(pool, req, slot, back)
    stq.stq_pool_check(pool)
    back = back.cpu().numpy()
    sb = (256 if f16 else 512)
    for a in range(wl.R):
        pages = split_slot(stq.stq_export_slot(pool, a, 0), rb, fmt)
        for h in range(wl.H):
            ref = orc.quantize_unit(rb[h], r[h], c[h], S0[a, h], fmt=fmt, w=W[h])
            assert pages[h][:sb].tobytes() == ref[:sb].tobytes(), (a, h)
            assert pages[h][sb + 512:].tobytes() == ref[sb + 512:].tobytes(), (a, h)
            np.testing.assert_allclose(col_factors(pages[h], rb[h], fmt), col_factors(ref, rb[h], fmt), rtol=1e-7)
            np.testing.assert_allclose(back[a, h], orc.dequantize_unit(rb[h], r[h], c[h], pages[h], fmt=fmt),
                                       rtol=0, atol=0)
    pool.close()


def _teacher_forced(wl, w, steps, f16=False, split=False):
    fmt = FITC | (1 if f16 else 0) | (PIVOT if np.any(wl.unit_bits == 16) else 0)
    pool, req, slot = _pool(wl, w, f16)
    rb = wl.row_bits()
    r, c, W = wl.row_factor.reshape(wl.H, 128), wl.col_factor.reshape(wl.H, 128), w.reshape(wl.H, 128)
    cmp = Compare()
    side = torch.cuda.Stream()
    for t in range(steps):
        before = [split_slot(stq.stq_export_slot(pool, a, int(wl.slot_of_request[a])), rb, fmt)
                  for a in range(wl.R)]
        inp = wl.step_inputs(t)
        x = [_cuda(inp[key]) for key in ("q", "k", "v", "beta", "gate")]
        y = torch.empty((wl.R, wl.H, 128), dtype=torch.float32, device="cuda")
        if split:
            stq.stq_decode_step_split(pool, req, slot, *x, y, torch.empty_like(y), side_stream=side)
        else:
            stq.stq_decode_step(pool, req, slot, *x, y)
        stq.stq_pool_check(pool)
        y = y.cpu().numpy()
        for a in range(wl.R):
            after = split_slot(stq.stq_export_slot(pool, a, int(wl.slot_of_request[a])), rb, fmt)
            for h in range(wl.H):
                g = inp["gate"][a, h]
                g = np.full(128, g, np.float32) if np.ndim(g) == 0 else g
                page_ref, y_ref, quot, st = orc.step_unit(rb[h], r[h], c[h], before[a][h], inp["q"][a, h],
                                                          inp["k"][a, h], inp["v"][a, h], inp["beta"][a, h],
                                                          g, fmt=fmt, w=W[h])
                assert st == orc.OK
                where = f"(t={t}, req={a}, head={h})"
                cmp.y(y[a, h], y_ref, where)
                cmp.page(after[h], page_ref, quot, rb[h], where, fmt=fmt)
    cmp.finish()
    pool.close()
    return cmp


def test_fit_gdn_mixed():
    """GDN mixed 4/6/8-bit heads, r, c ~ logU(0.25, 4), outlier start, row weights, 10 steps."""
    wl = dataclasses.replace(synth.make_workload(2, R=3, H=8), init="outlier")
    _teacher_forced(wl, _weights(wl, 1), steps=10)


def test_fit_kda():
    wl = dataclasses.replace(synth.make_workload(3, R=3, H=4), init="outlier")
    _teacher_forced(wl, _weights(wl, 2), steps=8)


def test_fit_gdn_f16_scales_split():
    """Binary16 scales with fitted factors, through the split step."""
    wl = dataclasses.replace(synth.make_workload(2, R=2, H=8), init="outlier")
    _teacher_forced(wl, _weights(wl, 3), steps=6, f16=True, split=True)


def test_fit_split_bit_identical_to_fused():
    wl = dataclasses.replace(synth.make_workload(2, R=4, H=8), init="outlier")
    w = _weights(wl, 4)
    (a, req, slot), (b, _, _) = _pool(wl, w), _pool(wl, w)
    side = torch.cuda.Stream()
    for t in range(5):
        inp = wl.step_inputs(t)
        x = [_cuda(inp[key]) for key in ("q", "k", "v", "beta", "gate")]
        y0 = torch.empty((wl.R, wl.H, 128), dtype=torch.float32, device="cuda")
        y1 = torch.empty_like(y0)
        stq.stq_decode_step(a, req, slot, *x, y0)
        stq.stq_decode_step_split(b, req, slot, *x, y1, torch.empty_like(y0), side_stream=side)
        stq.stq_pool_check(a)
        stq.stq_pool_check(b)
        assert torch.equal(y0, y1)
        for r in range(wl.R):
            assert stq.stq_export_slot(a, r, 0).tobytes() == stq.stq_export_slot(b, r, 0).tobytes()
    a.close()
    b.close()


def test_fit_kda_f16_scales_split():
    """KDA rows (warps of one width take the width-specialised passes) with binary16
    scales and fitted factors, through the split step's readout and write-back."""
    wl = dataclasses.replace(synth.make_workload(3, R=2, H=4), init="outlier")
    _teacher_forced(wl, _weights(wl, 5), steps=6, f16=True, split=True)


def test_fit_zero_start_pages_carry_initial_factors():
    """A fitted pool that was never quantized holds zero states whose pages carry
    the pool's col_factor; decoding from there matches the oracle (KDA, binary16 scales)."""
    wl = synth.make_workload(3, R=2, H=4)
    assert wl.initial_state() is None
    wl = dataclasses.replace(wl, col_factor=synth.log_uniform(synth.stream_key(0, 3, 99), wl.H * 128, 0.5, 2.0)
                             .astype(np.float32))
    w = _weights(wl, 6)
    pool, _, _ = _pool(wl, w, True)
    rb = wl.row_bits()
    fmt = FITC | 1
    c = wl.col_factor.reshape(wl.H, 128)
    for a in range(wl.R):
        for h, page in enumerate(split_slot(stq.stq_export_slot(pool, a, 0), rb, fmt)):
            np.testing.assert_array_equal(col_factors(page, rb[h], fmt), c[h])
            assert not page[:256].any() and not page[256 + 512:].any()
    pool.close()
    _teacher_forced(wl, w, steps=4, f16=True)


def test_fit_with_pivot_rows_kda_allocated():
    """The page's KDA configuration: allocator-chosen per-row widths, 8 FP16 pivot
    rows per head, column factors fitted over the non-pivot rows; 8 steps."""
    wl = _kda_allocated_pivots(3, 4, 11)
    cmp = _teacher_forced(wl, _weights(wl, 6), steps=8)
    assert cmp.values == 8 * 3 * 4 * 8 * 128


def test_fit_with_pivot_rows_split_and_f16():
    """Pivot rows with the fit through the split step, binary16 scales."""
    wl = _kda_allocated_pivots(2, 4, 12)
    _teacher_forced(wl, _weights(wl, 7), steps=5, f16=True, split=True)

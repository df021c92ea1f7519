"""GPU parity of FP16 pivot units among quantized ones ("method steps",
step 1: pivot units are read in FP16 directly; the page keeps 32 of 2304 GDN
heads and 512 of 81920 KDA key rows as pivots).  A pivot row keeps a scale
slot of 1 and stores mu = X / (r c) in binary16.  Teacher-forced like the
main parity tests (tolerances in tests/pages.py)."""
import dataclasses

import numpy as np
import pytest

import oracle as orc
from pages import PIVOT, Compare, split_slot
from quantized_linear_attention_decode_b200 import stq, synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _cuda(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _with_pivots(wl, seed=0, heads=(1, 5), rows_per_head=8):
    ub = wl.unit_bits.copy()
    if wl.kind == synth.GDN:
        ub[list(heads)] = 16
    else:
        rng = np.random.default_rng(seed)
        for h in range(wl.H):
            ub[h * 128 + rng.choice(128, rows_per_head, replace=False)] = 16
    return dataclasses.replace(wl, unit_bits=ub, init="outlier")


def _pool(wl, f16):
    pool = stq.stq_pool_create(wl.kind, wl.R, wl.S, wl.H, wl.unit_bits, wl.row_factor, wl.col_factor,
                               flags=stq.STQ_SCALE_F16 if f16 else 0)
    req = _cuda(np.arange(wl.R, dtype=np.int32))
    slot = _cuda(wl.slot_of_request.astype(np.int32))
    stq.stq_quantize_state(pool, req, slot, _cuda(wl.initial_state()))
    stq.stq_pool_check(pool)
    return pool, req, slot


@pytest.mark.parametrize("config, f16", [(2, False), (3, False), (2, True), (3, True)])
def test_pivot_quantize_dequantize_bit_exact(config, f16):
    wl = _with_pivots(synth.make_workload(config, R=2, H=8))
    fmt = (1 if f16 else 0) | PIVOT
    pool, req, slot = _pool(wl, f16)
    rb = wl.row_bits()
    r, c = wl.row_factor.reshape(wl.H, 128), wl.col_factor.reshape(wl.H, 128)
    S0 = wl.initial_state()
    back = torch.empty((wl.R, wl.H, 128, 128), dtype=torch.float32, device="cuda")
    stq.stq_dequantize_state(pool, req, slot, back)
    stq.stq_pool_check(pool)
    back = back.cpu().numpy()
    for a in range(wl.R):
        pages = split_slot(stq.stq_export_slot(pool, a, 0), rb, fmt)
        for h in range(wl.H):
            ref = orc.quantize_unit(rb[h], r[h], c[h], S0[a, h], fmt=fmt)
            assert pages[h].tobytes() == ref.tobytes(), (a, h)
            np.testing.assert_array_equal(back[a, h], orc.dequantize_unit(rb[h], r[h], c[h], ref, fmt=fmt))
    pool.close()


def _teacher_forced(wl, steps, f16=False, split=False, units=None, check_steps=None):
    """`steps` decode steps on all requests; `units` ((request, head) pairs, default
    all) checked against the oracle at `check_steps` (default all)."""
    fmt = (1 if f16 else 0) | PIVOT
    pool, req, slot = _pool(wl, f16)
    rb = wl.row_bits()
    r, c = wl.row_factor.reshape(wl.H, 128), wl.col_factor.reshape(wl.H, 128)
    units = [(a, h) for a in range(wl.R) for h in range(wl.H)] if units is None else units
    reqs = sorted({a for a, _ in units})
    cmp = Compare()
    side = torch.cuda.Stream()
    for t in range(steps):
        check = check_steps is None or t in check_steps
        before = {a: split_slot(stq.stq_export_slot(pool, a, int(wl.slot_of_request[a])), rb, fmt)
                  for a in (reqs if check else [])}
        inp = wl.step_inputs(t)
        x = [_cuda(inp[key]) for key in ("q", "k", "v", "beta", "gate")]
        y = torch.empty((wl.R, wl.H, 128), dtype=torch.float32, device="cuda")
        if split:
            u = torch.empty_like(y)
            stq.stq_decode_step_split(pool, req, slot, *x, y, u, side_stream=side)
        else:
            stq.stq_decode_step(pool, req, slot, *x, y)
        stq.stq_pool_check(pool)
        if not check:
            continue
        y = y.cpu().numpy()
        after = {a: split_slot(stq.stq_export_slot(pool, a, int(wl.slot_of_request[a])), rb, fmt) for a in reqs}
        for a, h in units:
            g = inp["gate"][a, h]
            g = np.full(128, g, np.float32) if np.ndim(g) == 0 else g
            page_ref, y_ref, quot, st = orc.step_unit(rb[h], r[h], c[h], before[a][h], inp["q"][a, h],
                                                      inp["k"][a, h], inp["v"][a, h], inp["beta"][a, h],
                                                      g, fmt=fmt)
            assert st == orc.OK
            where = f"(t={t}, req={a}, head={h})"
            cmp.y(y[a, h], y_ref, where)
            cmp.page(after[a][h], page_ref, quot, rb[h], where, fmt=fmt)
    cmp.finish()
    pool.close()
    return cmp


def test_pivot_heads_gdn_mixed():
    """GDN, mixed 4/6/8-bit heads with two FP16 pivot heads, r, c ~ logU(0.25, 4)."""
    cmp = _teacher_forced(_with_pivots(synth.make_workload(2, R=3, H=8)), steps=10)
    assert cmp.values == 10 * 3 * 2 * 128 * 128


def test_pivot_rows_kda():
    """KDA, per-row 4/6/8 bits with 8 FP16 pivot rows per head."""
    cmp = _teacher_forced(_with_pivots(synth.make_workload(3, R=3, H=4), seed=3), steps=10)
    assert cmp.values == 10 * 3 * 4 * 8 * 128


def test_pivot_rows_kda_f16_scales_factors():
    """KDA pivot rows with binary16 scales and row / column factors not 1."""
    wl = _with_pivots(synth.make_workload(3, R=2, H=4), seed=4)
    rng = np.random.default_rng(9)
    wl = dataclasses.replace(wl, row_factor=np.exp(rng.uniform(-1, 1, 4 * 128)).astype(np.float32),
                             col_factor=np.exp(rng.uniform(-1, 1, 4 * 128)).astype(np.float32))
    _teacher_forced(wl, steps=8, f16=True)


def test_pivot_split_step():
    """The split step (readout, then write-back on a side stream) with pivot heads."""
    _teacher_forced(_with_pivots(synth.make_workload(2, R=3, H=8), heads=(0, 7)), steps=6, split=True)


def test_allocated_widths_with_pivots_run():
    """Widths from the lifetime-aware allocator (6-bit budget over {4, 6, 8}, two FP16
    pivot heads) make a pool whose decode matches the oracle."""
    wl = synth.make_workload(2, R=2, H=16)
    rng = np.random.default_rng(17)
    d = np.exp(rng.uniform(-2, 2, wl.H))[:, None] * 4.0 ** (-np.arange(3)[None, :])
    w = stq.stq_lifetime_weight(np.log(rng.uniform(0.9, 0.999, wl.H)), 8192)
    bits, _ = stq.stq_allocate_bits(np.full(wl.H, 16384.0), [4, 6, 8], d, w, 6.0, num_pivots=2, pivot_bits=16)
    assert int(np.count_nonzero(bits == 16)) == 2
    _teacher_forced(dataclasses.replace(wl, unit_bits=bits, init="outlier"), steps=4)


def test_allocated_widths_with_pivot_rows_full_size_sampled():
    """The page's KDA setting at the benchmark's size: 128 requests x 32 heads, per-row
    widths from the allocator with 8 FP16 pivot rows per head (every tile on the
    per-row path), three tokens; sampled units checked against the oracle."""
    from test_gpu_fit import _kda_allocated_pivots
    wl = _kda_allocated_pivots(128, 32, 21)
    rng = np.random.default_rng(21)
    units = [(int(a), int(h)) for a, h in zip(rng.integers(0, wl.R, 12), rng.integers(0, wl.H, 12))]
    units += [(wl.R - 1, wl.H - 1), (0, 0)]
    cmp = _teacher_forced(wl, steps=3, units=units, check_steps={0, 2})
    assert cmp.values == 2 * len(units) * 8 * 128  # the pivot rows' binary16 values

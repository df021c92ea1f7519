"""GPU parity of the storage formats: binary16 scales and raw pools.

Binary16 per-row scales are the page's own storage ("method steps", step 6);
raw pools hold the state as binary16 (the page's FP16 pivot storage, applied
to a whole pool) or fp32 (the unquantized control of the page's state-update
timings).  Every step is teacher-forced like the main parity tests: the
oracle advances the GPU's own previous page and the GPU's next page and
readout must agree with it (tolerances in tests/pages.py).
"""
import dataclasses

import numpy as np
import pytest

import oracle as orc
from pages import Compare, split_slot
from quantized_linear_attention_decode_b200 import stq, synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _cuda(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _with_bits(wl, b):
    n = wl.H if wl.kind == synth.GDN else wl.H * 128
    return dataclasses.replace(wl, unit_bits=np.full(n, b, np.uint8))


def _run(wl, steps, fmt=0, init="outlier"):
    """Teacher-forced steps of every unit; returns the Compare record."""
    wl = dataclasses.replace(wl, init=init)
    pool = stq.stq_pool_create(wl.kind, wl.R, wl.S, wl.H, wl.unit_bits, wl.row_factor, wl.col_factor,
                               flags=stq.STQ_SCALE_F16 if fmt == 1 else 0)
    req = _cuda(np.arange(wl.R, dtype=np.int32))
    slot = _cuda(wl.slot_of_request.astype(np.int32))
    rb = wl.row_bits()
    raw = int(rb[0, 0]) in (16, 32)
    r, c = wl.row_factor.reshape(wl.H, 128), wl.col_factor.reshape(wl.H, 128)
    S0 = wl.initial_state()
    if S0 is not None:
        stq.stq_quantize_state(pool, req, slot, _cuda(S0))
        stq.stq_pool_check(pool)
    cmp = Compare()
    for t in range(steps):
        before = [split_slot(stq.stq_export_slot(pool, a, int(wl.slot_of_request[a])), rb, fmt)
                  for a in range(wl.R)]
        inp = wl.step_inputs(t)
        y = torch.empty((wl.R, wl.H, 128), dtype=torch.float32, device="cuda")
        stq.stq_decode_step(pool, req, slot, _cuda(inp["q"]), _cuda(inp["k"]), _cuda(inp["v"]),
                            _cuda(inp["beta"]), _cuda(inp["gate"]), y)
        stq.stq_pool_check(pool)
        y = y.cpu().numpy()
        for a in range(wl.R):
            after = split_slot(stq.stq_export_slot(pool, a, int(wl.slot_of_request[a])), rb, fmt)
            for h in range(wl.H):
                g = inp["gate"][a, h]
                g = np.full(128, g, np.float32) if np.ndim(g) == 0 else g
                page_ref, y_ref, quot, st = orc.step_unit(rb[h], r[h], c[h], before[a][h], inp["q"][a, h],
                                                          inp["k"][a, h], inp["v"][a, h], inp["beta"][a, h],
                                                          g, fmt=fmt)
                assert st == orc.OK
                where = f"(t={t}, req={a}, head={h})"
                cmp.y(y[a, h], y_ref, where)
                if raw:
                    cmp.raw(after[h], page_ref, quot, rb[h], where)
                else:
                    cmp.page(after[h], page_ref, quot, rb[h], where, fmt=fmt)
    cmp.finish()
    pool.close()
    return cmp


# ---------------------------------------------------------------- binary16 scales


@pytest.mark.parametrize("config", [1, 2, 3])
def test_f16_scales_quantize_dequantize_bit_exact(config):
    wl = dataclasses.replace(synth.make_workload(config, R=2, H=8), init="outlier")
    pool = stq.stq_pool_create(wl.kind, wl.R, wl.S, wl.H, wl.unit_bits, wl.row_factor, wl.col_factor,
                               flags=stq.STQ_SCALE_F16)
    req = _cuda(np.arange(wl.R, dtype=np.int32))
    slot = _cuda(wl.slot_of_request.astype(np.int32))
    S0 = wl.initial_state()
    stq.stq_quantize_state(pool, req, slot, _cuda(S0))
    stq.stq_pool_check(pool)
    back = torch.empty((wl.R, wl.H, 128, 128), dtype=torch.float32, device="cuda")
    stq.stq_dequantize_state(pool, req, slot, back)
    stq.stq_pool_check(pool)
    back = back.cpu().numpy()
    rb = wl.row_bits()
    r, c = wl.row_factor.reshape(wl.H, 128), wl.col_factor.reshape(wl.H, 128)
    for a in range(wl.R):
        pages = split_slot(stq.stq_export_slot(pool, a, int(wl.slot_of_request[a])), rb, 1)
        for h in range(wl.H):
            ref = orc.quantize_unit(rb[h], r[h], c[h], S0[a, h], fmt=orc.FMT_F16)
            assert pages[h].tobytes() == ref.tobytes(), (a, h)
            np.testing.assert_array_equal(back[a, h], orc.dequantize_unit(rb[h], r[h], c[h], ref, fmt=orc.FMT_F16))
    pool.close()


def test_f16_scales_decode_gdn_int8():
    _run(synth.make_workload(1, R=2, H=4), steps=24, fmt=1, init="zero")


def test_f16_scales_decode_gdn_mixed_outliers():
    _run(synth.make_workload(2, R=2, H=8), steps=8, fmt=1)


def test_f16_scales_decode_kda_mixed():
    _run(synth.make_workload(3, R=2, H=4), steps=12, fmt=1, init="zero")


# ---------------------------------------------------------------- raw pools


@pytest.mark.parametrize("b", [16, 32])
@pytest.mark.parametrize("config", [2, 3])
def test_raw_pool_quantize_dequantize(b, config):
    wl = dataclasses.replace(_with_bits(synth.make_workload(config, R=2, H=4), b), init="outlier")
    pool = stq.stq_pool_create(wl.kind, wl.R, wl.S, wl.H, wl.unit_bits, wl.row_factor, wl.col_factor)
    assert stq.stq_pool_bytes(pool)[1] == wl.H * 128 * 128 * b // 8
    req = _cuda(np.arange(wl.R, dtype=np.int32))
    slot = _cuda(wl.slot_of_request.astype(np.int32))
    S0 = wl.initial_state()
    stq.stq_quantize_state(pool, req, slot, _cuda(S0))
    stq.stq_pool_check(pool)
    back = torch.empty((wl.R, wl.H, 128, 128), dtype=torch.float32, device="cuda")
    stq.stq_dequantize_state(pool, req, slot, back)
    stq.stq_pool_check(pool)
    rb = wl.row_bits()
    dt = np.float16 if b == 16 else np.float32
    np.testing.assert_array_equal(back.cpu().numpy(), S0.astype(dt).astype(np.float32))
    for a in range(wl.R):
        pages = split_slot(stq.stq_export_slot(pool, a, 0), rb)
        for h in range(wl.H):
            ref = orc.quantize_unit(rb[h], np.ones(128), np.ones(128), S0[a, h])
            assert pages[h].tobytes() == ref.tobytes()
    pool.close()


@pytest.mark.parametrize("b", [16, 32])
def test_raw_pool_decode_gdn(b):
    _run(_with_bits(synth.make_workload(2, R=2, H=4), b), steps=8)


@pytest.mark.parametrize("b", [16, 32])
def test_raw_pool_decode_kda(b):
    _run(_with_bits(synth.make_workload(3, R=2, H=4), b), steps=8)


def test_raw_fp32_retrieval_identity_on_gpu():
    """beta = 1, q = k unit-norm: y = v ("gated delta rule" read back after its own write)."""
    wl = dataclasses.replace(_with_bits(synth.make_workload(2, R=2, H=4), 32), init="outlier")
    pool = stq.stq_pool_create(wl.kind, wl.R, wl.S, wl.H, wl.unit_bits)
    req = _cuda(np.arange(wl.R, dtype=np.int32))
    slot = _cuda(np.zeros(wl.R, np.int32))
    stq.stq_quantize_state(pool, req, slot, _cuda(wl.initial_state()))
    inp = wl.step_inputs(0)
    y = torch.empty((wl.R, wl.H, 128), dtype=torch.float32, device="cuda")
    stq.stq_decode_step(pool, req, slot, _cuda(inp["k"]), _cuda(inp["k"]), _cuda(inp["v"]),
                        _cuda(np.ones_like(inp["beta"])), _cuda(inp["gate"]), y)
    stq.stq_pool_check(pool)
    v = inp["v"]
    np.testing.assert_allclose(y.cpu().numpy(), v, rtol=0, atol=2e-5 * np.abs(v).max())
    pool.close()

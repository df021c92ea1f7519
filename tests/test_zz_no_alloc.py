"""GPU: stq_decode_step_static, the decode step for callers that cannot
allocate device memory while they run (its scratch is a fixed array built
into the library), against the ordinary stq_decode_step on the same inputs.

The static step runs the split step's two kernels (readout, then write-back)
on one stream; both do the fused kernel's arithmetic, so y and the pages
must equal stq_decode_step's byte for byte.

Kept in a file of its own that pytest collects last; it passes run alone in
a fresh process as well as after the other tests."""
import numpy as np
import pytest

from quantized_linear_attention_decode_b200 import stq, synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

KEYS = ("q", "k", "v", "beta", "gate")


def _cuda(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _workload(case):
    """(workload, unit_bits, flags) of each pool kind the static step serves."""
    if case == "gdn":
        wl = synth.make_workload(2, R=6, H=8)
        return wl, wl.unit_bits, 0
    if case == "kda":
        wl = synth.make_workload(3, R=6, H=8)
        return wl, wl.unit_bits, 0
    if case == "gdn_pivot_heads":  # FP16 pivot heads run their own kernel inside the static step
        wl = synth.make_workload(2, R=6, H=8)
        ub = wl.unit_bits.copy()
        ub[[1, 6]] = 16
        return wl, ub, 0
    if case == "kda_pivot_rows":
        wl = synth.make_workload(3, R=6, H=8)
        ub = wl.unit_bits.reshape(wl.H, 128).copy()
        for h in range(wl.H):
            ub[h, np.nonzero(ub[h] == 4)[0][:4]] = 16  # four 4-bit rows become pivots (page stays in a stage)
        return wl, ub.reshape(-1), 0
    if case == "gdn_fit":
        wl = synth.make_workload(2, R=6, H=8)
        return wl, wl.unit_bits, stq.STQ_FIT_COLUMNS
    if case == "gdn_f16_scales":
        wl = synth.make_workload(2, R=6, H=8)
        return wl, wl.unit_bits, stq.STQ_SCALE_F16
    raise ValueError(case)


def _pool(wl, unit_bits, flags):
    pool = stq.stq_pool_create(wl.kind, wl.R, wl.S, wl.H, unit_bits, wl.row_factor, wl.col_factor, flags=flags)
    req = _cuda(np.arange(wl.R, dtype=np.int32))
    slot = _cuda(wl.slot_of_request.astype(np.int32))
    S0 = wl.initial_state()
    if S0 is not None:
        stq.stq_quantize_state(pool, req, slot, _cuda(S0))
    stq.stq_pool_check(pool)
    return pool, req, slot


def _same(wl, ref, got, y_ref, y_got):
    np.testing.assert_array_equal(y_got.cpu().numpy(), y_ref.cpu().numpy())
    for a in range(wl.R):
        s = int(wl.slot_of_request[a])
        assert np.array_equal(stq.stq_export_slot(ref, a, s), stq.stq_export_slot(got, a, s)), a


@pytest.mark.parametrize("case", ["gdn", "kda", "gdn_pivot_heads", "kda_pivot_rows", "gdn_fit",
                                  "gdn_f16_scales"])
def test_static_scratch_decode_matches_decode_step_twice(case):
    """Two calls in a row through the C ABI: y and the pages (codes, scales,
    pivot values, fitted column factors) equal stq_decode_step's on a twin
    pool byte for byte."""
    wl, ub, flags = _workload(case)
    ref, req, slot = _pool(wl, ub, flags)
    got, _, _ = _pool(wl, ub, flags)
    for t in range(2):
        inp = wl.step_inputs(t)
        x = [_cuda(inp[key]) for key in KEYS]
        y_ref = torch.empty((wl.R, wl.H, 128), dtype=torch.float32, device="cuda")
        y_got = torch.full_like(y_ref, float("nan"))
        stq.stq_decode_step(ref, req, slot, *x, y_ref)
        stq.stq_decode_step_static(got, req, slot, *x, y_got)
        stq.stq_pool_check(ref)
        stq.stq_pool_check(got)
        _same(wl, ref, got, y_ref, y_got)
    ref.close()
    got.close()


def test_static_scratch_decode_after_pending_split_write_back():
    """A split step leaves its write-back pending on a side stream; the static
    step called right after (on the main stream) must wait for it: two
    tokens, split then static, equal two fused steps byte for byte."""
    wl, ub, flags = _workload("gdn")
    ref, req, slot = _pool(wl, ub, flags)
    got, _, _ = _pool(wl, ub, flags)
    main, side = torch.cuda.current_stream(), torch.cuda.Stream()
    x0 = [_cuda(wl.step_inputs(0)[key]) for key in KEYS]
    x1 = [_cuda(wl.step_inputs(1)[key]) for key in KEYS]
    y_ref = torch.empty((wl.R, wl.H, 128), dtype=torch.float32, device="cuda")
    y_got = torch.full_like(y_ref, float("nan"))
    u = torch.empty_like(y_ref)
    stq.stq_decode_step(ref, req, slot, *x0, y_ref)
    stq.stq_decode_step(ref, req, slot, *x1, y_ref)
    side.wait_stream(main)
    stq.stq_decode_step_split(got, req, slot, *x0, y_got, u, main, side)
    stq.stq_decode_step_static(got, req, slot, *x1, y_got, main)
    stq.stq_pool_check(ref)
    stq.stq_pool_check(got)
    _same(wl, ref, got, y_ref, y_got)
    ref.close()
    got.close()


def test_static_scratch_decode_rejects_oversize_call():
    """More than 8192 (entry, head) tiles in one call: STQ_ERR_ARG, nothing run."""
    H, n = 128, 65
    pool = stq.stq_pool_create(stq.STQ_GDN, n, 1, H, np.full(H, 4, np.uint8))
    idx = _cuda(np.arange(n, dtype=np.int32))
    zero = torch.zeros(n, dtype=torch.int32, device="cuda")
    vec = torch.zeros((n, H, 128), dtype=torch.float32, device="cuda")
    sc = torch.ones((n, H), dtype=torch.float32, device="cuda")
    launches = stq.stq_launch_count()
    with pytest.raises(stq.StqError) as e:
        stq.stq_decode_step_static(pool, idx, zero, vec, vec, vec, sc, sc, vec.clone())
    assert e.value.status == stq.STQ_ERR_ARG
    assert "8192" in stq.stq_last_error()
    assert stq.stq_launch_count() == launches
    pool.close()

"""GPU: stq_decode_step_static, the decode step for callers that cannot
allocate device memory while they run (its scratch is a fixed array built
into the library), against the ordinary stq_decode_step on the same inputs.

Kept in a file of its own that pytest collects last; it passes run alone in
a fresh process as well as after the other tests."""
import numpy as np
import pytest

from pages import decode_page, split_slot
from quantized_linear_attention_decode_b200 import stq, synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

Y_TOL = 1e-5     # max relative error of y per (request, head), as in the parity tests
TIE_RATE = 1e-4  # at most this share of codes may differ, by one step (rounding ties)


def _cuda(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _pool(wl):
    pool = stq.stq_pool_create(wl.kind, wl.R, wl.S, wl.H, wl.unit_bits, wl.row_factor, wl.col_factor)
    req = _cuda(np.arange(wl.R, dtype=np.int32))
    slot = _cuda(wl.slot_of_request.astype(np.int32))
    S0 = wl.initial_state()
    if S0 is not None:
        stq.stq_quantize_state(pool, req, slot, _cuda(S0))
    stq.stq_pool_check(pool)
    return pool, req, slot


def _agree(wl, ref, got, y_ref, y_got):
    y_ref, y_got = y_ref.cpu().numpy(), y_got.cpu().numpy()
    for a in range(wl.R):
        for h in range(wl.H):
            err = np.abs(y_got[a, h] - y_ref[a, h]).max() / max(np.abs(y_ref[a, h]).max(), 1e-30)
            assert err <= Y_TOL, (a, h, err)
    rb = wl.row_bits()
    codes = diff = 0
    for a in range(wl.R):
        s = int(wl.slot_of_request[a])
        for h, (p0, p1) in enumerate(zip(split_slot(stq.stq_export_slot(ref, a, s), rb),
                                         split_slot(stq.stq_export_slot(got, a, s), rb))):
            s0, z0 = decode_page(p0, rb[h])
            s1, z1 = decode_page(p1, rb[h])
            np.testing.assert_allclose(s1, s0, rtol=Y_TOL, atol=0)
            d = np.abs(z1.astype(np.int64) - z0)
            assert d.max() <= 1
            codes += z0.size
            diff += int(np.count_nonzero(d))
    assert diff <= TIE_RATE * codes, (diff, codes)


@pytest.mark.parametrize("config", [2, 3])
def test_static_scratch_decode_matches_decode_step_twice(config):
    """Two calls in a row through the C ABI: y, scales and codes agree with
    stq_decode_step on a twin pool within the parity tolerances."""
    wl = synth.make_workload(config, R=6, H=8)
    ref, req, slot = _pool(wl)
    got, _, _ = _pool(wl)
    for t in range(2):
        inp = wl.step_inputs(t)
        x = [_cuda(inp[key]) for key in ("q", "k", "v", "beta", "gate")]
        y_ref = torch.empty((wl.R, wl.H, 128), dtype=torch.float32, device="cuda")
        y_got = torch.full_like(y_ref, float("nan"))
        stq.stq_decode_step(ref, req, slot, *x, y_ref)
        stq.stq_decode_step_static(got, req, slot, *x, y_got)
        stq.stq_pool_check(ref)
        stq.stq_pool_check(got)
        _agree(wl, ref, got, y_ref, y_got)
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

"""GPU: the decode kernel's bounded waits end in an error status.

Every mbarrier wait of the fused decode kernel gives up after a limit, sets
the pool's timeout bit, waits (bounded) for the copies it still has in
flight and returns, so that the context stays usable.  STQ_FAULT=timeout
makes one wait run out on purpose: the limit drops to 2 ms and the first
stage of CTA 0 expects 16 bytes that no copy delivers (every copy lands; no
fault, trap or hang is involved).  The other CTAs finish their tiles."""
import time

import numpy as np
import pytest

from quantized_linear_attention_decode_b200 import stq, synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

KEYS = ("q", "k", "v", "beta", "gate")


def _pool(wl):
    pool = stq.stq_pool_create(wl.kind, wl.R, wl.S, wl.H, wl.unit_bits, wl.row_factor, wl.col_factor)
    req = torch.arange(wl.R, dtype=torch.int32, device="cuda")
    slot = torch.zeros(wl.R, dtype=torch.int32, device="cuda")
    S0 = wl.initial_state()
    if S0 is not None:
        stq.stq_quantize_state(pool, req, slot, torch.from_numpy(S0).cuda())
    stq.stq_pool_check(pool)
    return pool, req, slot


def _status(pool):
    return stq.stq_pool_check(pool, raise_on_error=False)


@pytest.mark.parametrize("config", [2, 3])
def test_wait_runs_out_to_timeout_status(config, monkeypatch):
    """8 requests x 8 heads: 64 tiles, one per CTA, so CTA 0 holds tile 0
    alone.  The stalled call reports STQ_ERR_TIMEOUT within far less than the
    default 1 s limit; every other tile equals the twin pool's; the same pool
    and a fresh one then decode normally."""
    wl = synth.make_workload(config, R=8, H=8)
    bad, req, slot = _pool(wl)
    ref, _, _ = _pool(wl)
    x = [torch.from_numpy(wl.step_inputs(0)[k]).cuda() for k in KEYS]
    y_bad = torch.zeros((wl.R, wl.H, 128), device="cuda")
    y_ref = torch.zeros_like(y_bad)
    stq.stq_decode_step(ref, req, slot, *x, y_ref)
    assert _status(ref) == stq.STQ_OK
    monkeypatch.setenv("STQ_FAULT", "timeout")
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    stq.stq_decode_step(bad, req, slot, *x, y_bad)
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    monkeypatch.delenv("STQ_FAULT")
    assert _status(bad) == stq.STQ_ERR_TIMEOUT
    assert "timed out" in stq.stq_last_error()
    assert dt < 0.5, f"the stalled launch took {dt:.3f} s"
    # tiles 1.. (other CTAs) are complete; tile 0 = (request 0, head 0) is not
    yb, yr = y_bad.cpu().numpy().reshape(-1, 128), y_ref.cpu().numpy().reshape(-1, 128)
    np.testing.assert_array_equal(yb[1:], yr[1:])
    sb, sr = stq.stq_export_slot(bad, 0, 0), stq.stq_export_slot(ref, 0, 0)
    off, nb = stq.stq_page_layout(bad, 0)
    assert np.array_equal(sb[off + nb:], sr[off + nb:])  # request 0's other heads
    for a in range(1, wl.R):
        assert np.array_equal(stq.stq_export_slot(bad, a, 0), stq.stq_export_slot(ref, a, 0))
    # the context is usable: the same pool decodes again without error, and a
    # fresh pool's step equals its twin's
    stq.stq_decode_step(bad, req, slot, *x, y_bad)
    assert _status(bad) == stq.STQ_OK
    fresh, _, _ = _pool(wl)
    twin, _, _ = _pool(wl)
    y1, y2 = torch.empty_like(y_bad), torch.empty_like(y_bad)
    stq.stq_decode_step(fresh, req, slot, *x, y1)
    stq.stq_decode_step(twin, req, slot, *x, y2)
    assert _status(fresh) == stq.STQ_OK and _status(twin) == stq.STQ_OK
    assert torch.equal(y1, y2)
    for p in (bad, ref, fresh, twin):
        p.close()

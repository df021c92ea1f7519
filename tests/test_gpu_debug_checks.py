"""GPU: the debug check for a (request, slot) pair named twice in one call
(STQ_DEBUG_CHECKS=1 when the pool is created).  The pages are written in
place by one CTA per tile, so such a call has undefined results; with the
check on, stq_pool_check reports it as STQ_ERR_INDEX."""
import numpy as np
import pytest

from quantized_linear_attention_decode_b200 import stq

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

R, S, H = 4, 2, 4


def _pool(monkeypatch, on):
    if on:
        monkeypatch.setenv("STQ_DEBUG_CHECKS", "1")
    else:
        monkeypatch.delenv("STQ_DEBUG_CHECKS", raising=False)
    return stq.stq_pool_create(stq.STQ_GDN, R, S, H, np.full(H, 6, np.uint8))


def _inputs(n, seed=0):
    g = torch.Generator().manual_seed(seed)
    k = torch.nn.functional.normalize(torch.randn(n, H, 128, generator=g), dim=-1)
    q = torch.nn.functional.normalize(torch.randn(n, H, 128, generator=g), dim=-1)
    v = torch.randn(n, H, 128, generator=g)
    beta = torch.rand(n, H, generator=g)
    alpha = torch.full((n, H), 0.95)
    return [t.contiguous().cuda() for t in (q, k, v, beta, alpha)]


def _idx(req, slot):
    return (torch.tensor(req, dtype=torch.int32, device="cuda"),
            torch.tensor(slot, dtype=torch.int32, device="cuda"))


def _status(pool):
    try:
        stq.stq_pool_check(pool)
        return stq.STQ_OK
    except stq.StqError as e:
        return e.status


def test_duplicate_pair_reported_by_decode_and_quantize(monkeypatch):
    pool = _pool(monkeypatch, True)
    req, slot = _idx([0, 1, 1], [0, 0, 0])  # (1, 0) twice
    y = torch.empty((3, H, 128), device="cuda")
    stq.stq_decode_step(pool, req, slot, *_inputs(3), y)
    assert _status(pool) == stq.STQ_ERR_INDEX
    assert "twice" in stq.stq_last_error()
    state = torch.zeros((3, H, 128, 128), device="cuda")
    stq.stq_quantize_state(pool, req, slot, state)
    assert _status(pool) == stq.STQ_ERR_INDEX
    pool.close()


def test_distinct_pairs_pass_and_every_call_starts_clean(monkeypatch):
    pool = _pool(monkeypatch, True)
    # the same request in two slots, and the same slot of two requests: all distinct
    req, slot = _idx([1, 1, 0, 3], [0, 1, 1, 1])
    y = torch.empty((4, H, 128), device="cuda")
    for t in range(3):  # the bitmap is cleared before every call
        stq.stq_decode_step(pool, req, slot, *_inputs(4, t), y)
        assert _status(pool) == stq.STQ_OK
    pool.close()


def test_duplicate_in_write_back_and_host_step(monkeypatch):
    pool = _pool(monkeypatch, True)
    req, slot = _idx([2, 2], [1, 1])
    q, k, v, beta, alpha = _inputs(2)
    u = torch.zeros((2, H, 128), device="cuda")
    stq.stq_decode_writeback(pool, req, slot, k, alpha, u)
    assert _status(pool) == stq.STQ_ERR_INDEX
    y = torch.empty((2, H, 128)).pin_memory()
    xh = [req.cpu(), slot.cpu()] + [t.cpu().pin_memory() for t in (q, k, v, beta, alpha)]
    stq.stq_decode_step_host(pool, *xh, y)
    assert _status(pool) == stq.STQ_ERR_INDEX
    pool.close()


def test_without_debug_checks_no_check_runs(monkeypatch):
    pool = _pool(monkeypatch, False)
    req, slot = _idx([0, 0], [1, 1])
    y = torch.empty((2, H, 128), device="cuda")
    launches = stq.stq_launch_count()
    stq.stq_decode_step(pool, req, slot, *_inputs(2), y)
    assert _status(pool) == stq.STQ_OK  # undefined results, not reported
    assert stq.stq_launch_count() == launches + 1  # the decode alone
    pool.close()

"""GPU: stq_decode_step_host, the decode step with host-memory buffers
(inputs copied into the pool's staging buffer, y copied out), against
stq_decode_step on a twin pool.  It runs the same kernels on the same
inputs, so y and the pages must agree bit for bit."""
import numpy as np
import pytest

from quantized_linear_attention_decode_b200 import stq, synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

KEYS = ("q", "k", "v", "beta", "gate")


def _cuda(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _host(a, pinned):
    t = torch.from_numpy(np.ascontiguousarray(a))
    return t.pin_memory() if pinned else t.clone()


def _pool(wl, unit_bits=None, flags=0):
    ub = wl.unit_bits if unit_bits is None else unit_bits
    pool = stq.stq_pool_create(wl.kind, wl.R, wl.S, wl.H, ub, wl.row_factor, wl.col_factor, flags=flags)
    req = _cuda(np.arange(wl.R, dtype=np.int32))
    slot = _cuda(wl.slot_of_request.astype(np.int32))
    S0 = wl.initial_state()
    if S0 is not None:
        stq.stq_quantize_state(pool, req, slot, _cuda(S0))
    stq.stq_pool_check(pool)
    return pool


def _slots(pool, wl):
    return [stq.stq_export_slot(pool, a, int(wl.slot_of_request[a])) for a in range(wl.R)]


def _run_twins(wl, steps, *, pinned=True, entries=None, unit_bits=None, stream=None, flags=0):
    """Advance twin pools `steps` tokens, one through device buffers and one
    through host buffers; return both pools' y and slots."""
    ref, got = _pool(wl, unit_bits, flags), _pool(wl, unit_bits, flags)
    for t in range(steps):
        sel = np.arange(wl.R) if entries is None else np.asarray(entries[t])
        n = len(sel)
        inp = wl.step_inputs(t)
        req = sel.astype(np.int32)
        slot = wl.slot_of_request[sel].astype(np.int32)
        x = {key: np.ascontiguousarray(inp[key][sel]) for key in KEYS}
        y_ref = torch.empty((n, wl.H, 128), dtype=torch.float32, device="cuda")
        stq.stq_decode_step(ref, _cuda(req), _cuda(slot), *[_cuda(x[key]) for key in KEYS], y_ref)
        y_got = _host(np.full((n, wl.H, 128), np.nan, np.float32), pinned)
        xh = [_host(req, pinned), _host(slot, pinned)] + [_host(x[key], pinned) for key in KEYS]
        stq.stq_decode_step_host(got, *xh, y_got, stream)
        if stream is None:
            torch.cuda.current_stream().synchronize()
        else:
            stream.synchronize()
        stq.stq_pool_check(ref)
        stq.stq_pool_check(got)
        np.testing.assert_array_equal(y_got.numpy(), y_ref.cpu().numpy())
    a, b = _slots(ref, wl), _slots(got, wl)
    ref.close()
    got.close()
    return a, b


def _same_slots(a, b):
    for r, (s0, s1) in enumerate(zip(a, b)):
        assert np.array_equal(s0, s1), r


def test_host_decode_gdn_pinned():
    """4096 tiles (128 requests x 32 heads), two tokens, pinned host memory."""
    wl = synth.make_workload(2, R=128)
    _same_slots(*_run_twins(wl, 2))


def test_host_decode_kda_side_stream():
    """KDA (a per-row gate), 100 requests x 32 heads, ordered on a non-default stream."""
    wl = synth.make_workload(3, R=100)
    _same_slots(*_run_twins(wl, 2, stream=torch.cuda.Stream()))


def test_host_decode_pageable_memory_and_staging_growth():
    """Pageable host memory; a 3-entry call, then one over all 24 entries
    (the staging buffer grows), then a ragged 7-entry call."""
    wl = synth.make_workload(2, R=24, H=8)
    entries = [[5, 0, 17], list(range(24)), [23, 1, 2, 9, 4, 11, 6]]
    _same_slots(*_run_twins(wl, 3, pinned=False, entries=entries))


def test_host_decode_raw_pool():
    """A raw fp32 pool goes through the raw kernel the same way."""
    wl = synth.make_workload(2, R=6, H=8)
    _same_slots(*_run_twins(wl, 2, unit_bits=np.full(wl.H, 32, np.uint8)))


def test_host_decode_empty_call_is_a_no_op():
    wl = synth.make_workload(2, R=2, H=4)
    pool = _pool(wl)
    before = _slots(pool, wl)
    e32 = torch.empty(0, dtype=torch.int32)
    ev = torch.empty((0, wl.H, 128), dtype=torch.float32)
    es = torch.empty((0, wl.H), dtype=torch.float32)
    launches = stq.stq_launch_count()
    stq.stq_decode_step_host(pool, e32, e32, ev, ev, ev, es, es, ev.clone())
    assert stq.stq_launch_count() == launches
    _same_slots(before, _slots(pool, wl))
    pool.close()


def test_host_decode_gdn_with_pivot_heads():
    """Two GDN heads kept as FP16 pivots: their own kernel runs in every chunk."""
    wl = synth.make_workload(2, R=24, H=8)
    ub = wl.unit_bits.copy()
    ub[[1, 6]] = 16
    _same_slots(*_run_twins(wl, 2, unit_bits=ub))


def test_host_decode_alternating_streams():
    """Steps issued on two streams in turn share the staging buffer: each waits
    for the previous one, so every step sees its own inputs."""
    wl = synth.make_workload(2, R=16, H=8)
    ref, got = _pool(wl), _pool(wl)
    req = np.arange(wl.R, dtype=np.int32)
    slot = wl.slot_of_request.astype(np.int32)
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    ys = []
    for t in range(4):
        x = wl.step_inputs(t)
        y_ref = torch.empty((wl.R, wl.H, 128), dtype=torch.float32, device="cuda")
        stq.stq_decode_step(ref, _cuda(req), _cuda(slot), *[_cuda(x[key]) for key in KEYS], y_ref)
        y_got = _host(np.full((wl.R, wl.H, 128), np.nan, np.float32), True)
        # the host inputs stay referenced until the streams are synchronized: a freed
        # pinned block could be handed out again before its copy has run
        xh = [_host(req, True), _host(slot, True)] + [_host(x[key], True) for key in KEYS]
        stq.stq_decode_step_host(got, *xh, y_got, streams[t % 2])
        ys.append((y_ref, y_got, xh))
    torch.cuda.synchronize()
    stq.stq_pool_check(ref)
    stq.stq_pool_check(got)
    for y_ref, y_got, _ in ys:
        np.testing.assert_array_equal(y_got.numpy(), y_ref.cpu().numpy())
    _same_slots(_slots(ref, wl), _slots(got, wl))
    ref.close()
    got.close()


@pytest.mark.parametrize("config, flags", [(3, stq.STQ_SCALE_F16), (2, stq.STQ_FIT_COLUMNS),
                                           (3, stq.STQ_FIT_COLUMNS | stq.STQ_SCALE_F16)])
def test_host_decode_scale_and_fit_formats(config, flags):
    """Binary16 scales and fitted column factors go through the host-buffer step unchanged."""
    wl = synth.make_workload(config, R=12, H=8)
    _same_slots(*_run_twins(wl, 3, flags=flags))


def _block(pool, n, req, slot, x, pinned=True):
    """The one-block host layout of stq_host_block_layout, filled."""
    offs, nbytes = stq.stq_host_block_layout(pool, n)
    blk = torch.zeros(nbytes, dtype=torch.uint8)
    if pinned:
        blk = blk.pin_memory()
    raw = blk.numpy()
    for o, a in zip(offs, [req, slot] + [x[key] for key in KEYS]):
        b = np.ascontiguousarray(a).view(np.uint8).reshape(-1)
        raw[o: o + b.size] = b
    return blk


@pytest.mark.parametrize("config, pinned", [(2, True), (3, True), (2, False)])
def test_host_block_decode_matches_device_step(config, pinned):
    """The single-copy host block: GDN (per-head gate) and KDA (per-row gate)
    layouts, a subset of requests, three tokens, page-locked and pageable host
    memory; y and pages bit for bit."""
    wl = synth.make_workload(config, R=24)
    ref, got = _pool(wl), _pool(wl)
    offs, nbytes = stq.stq_host_block_layout(got, 0)
    assert nbytes == 0 or all(o % 256 == 0 for o in offs)
    for t in range(3):
        sel = np.arange(t, wl.R, 2)
        n = len(sel)
        inp = wl.step_inputs(t)
        req = sel.astype(np.int32)
        slot = wl.slot_of_request[sel].astype(np.int32)
        x = {key: np.ascontiguousarray(inp[key][sel]) for key in KEYS}
        y_ref = torch.empty((n, wl.H, 128), dtype=torch.float32, device="cuda")
        stq.stq_decode_step(ref, _cuda(req), _cuda(slot), *[_cuda(x[key]) for key in KEYS], y_ref)
        blk = _block(got, n, req, slot, x, pinned)
        offs, nbytes = stq.stq_host_block_layout(got, n)
        assert offs == sorted(offs) and all(o % 256 == 0 for o in offs) and blk.numel() == nbytes
        y_got = torch.full((n, wl.H, 128), float("nan"))
        y_got = y_got.pin_memory() if pinned else y_got
        stq.stq_decode_step_host_block(got, n, blk, y_got)
        torch.cuda.current_stream().synchronize()
        stq.stq_pool_check(ref)
        stq.stq_pool_check(got)
        np.testing.assert_array_equal(y_got.numpy(), y_ref.cpu().numpy())
    _same_slots(_slots(ref, wl), _slots(got, wl))
    # a block of the wrong size is refused before anything is queued
    with pytest.raises(stq.StqError) as e:
        stq.stq_decode_step_host_block(got, 1, torch.zeros(16, dtype=torch.uint8),
                                       torch.empty((1, wl.H, 128)))
    assert e.value.status == stq.STQ_ERR_ARG
    ref.close()
    got.close()


@pytest.mark.parametrize("config", [2, 3])
def test_host_block_writes_a_pinned_y_in_place_at_an_offset(config):
    """A page-locked y that starts inside a larger page-locked buffer (an interior
    pointer, 128 bytes in): the kernels write exactly its n x H x 128 values across
    the bus and leave the bytes around it alone; the values equal those of the
    same step with a pageable y (staged and copied back) bit for bit."""
    wl = synth.make_workload(config, R=12)
    ref, got = _pool(wl), _pool(wl)
    n = wl.R
    inp = wl.step_inputs(0)
    req = np.arange(n, dtype=np.int32)
    slot = wl.slot_of_request.astype(np.int32)
    x = {key: np.ascontiguousarray(inp[key]) for key in KEYS}
    m = n * wl.H * 128
    y_ref = torch.full((n, wl.H, 128), float("nan"))  # pageable
    stq.stq_decode_step_host_block(ref, n, _block(ref, n, req, slot, x), y_ref)
    big = torch.full((m + 96,), -7.0).pin_memory()
    y_got = big[32:32 + m].view(n, wl.H, 128)
    stq.stq_decode_step_host_block(got, n, _block(got, n, req, slot, x), y_got)
    torch.cuda.current_stream().synchronize()
    stq.stq_pool_check(ref)
    stq.stq_pool_check(got)
    np.testing.assert_array_equal(y_got.numpy(), y_ref.numpy())
    assert bool((big[:32] == -7.0).all()) and bool((big[32 + m:] == -7.0).all())
    _same_slots(_slots(ref, wl), _slots(got, wl))
    ref.close()
    got.close()

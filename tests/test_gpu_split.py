"""GPU: the decode step split into a readout and a write-back on a second
stream ("method steps", steps 3-7): parity with the oracle, bit-identity with
the fused step, ordering through the pool, and a per-layer serving loop
captured in a CUDA graph."""
import numpy as np
import pytest

from test_gpu_parity import _cuda, _init, _pool, _simple_pool, _teacher_forced, _unit_vecs, side_stream
from quantized_linear_attention_decode_b200 import stq, synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _inputs(wl, t):
    inp = wl.step_inputs(t)
    return [_cuda(inp[key]) for key in ("q", "k", "v", "beta", "gate")]


def _pages(pool, wl):
    return [stq.stq_export_slot(pool, a, int(wl.slot_of_request[a])) for a in range(wl.R)]


def test_split_teacher_forced_config2():
    """Split step against the oracle: mixed 4/6/8-bit GDN, 4 x 8 heads, 12 steps."""
    _teacher_forced(synth.make_workload(2, R=4, H=8), steps=12, split=True)


def test_split_teacher_forced_config3_kda():
    _teacher_forced(synth.make_workload(3, R=3, H=4), steps=8, split=True)


def _ragged_kda(R, H, seed=23):
    """KDA with row widths drawn independently: pass warps mix widths, so the
    pool runs every tile on the per-row path."""
    rng = np.random.default_rng(seed)
    wl = synth.make_workload(3, R=R, H=H)
    wl.unit_bits = rng.choice(np.array([4, 6, 8], np.uint8), size=H * 128)
    wl.init = "outlier"
    return wl


def test_split_teacher_forced_kda_per_row_widths():
    """Split step against the oracle on a KDA pool whose rows take the per-row path."""
    _teacher_forced(_ragged_kda(3, 4), steps=8, split=True)


@pytest.mark.parametrize("config, flags", [(2, 0), (3, 0), (2, stq.STQ_SCALE_F16), ("kda_rows", 0)])
def test_split_bit_identical_to_fused(config, flags):
    """Same inputs, two pools: the split step's y, codes and scales equal the
    fused step's bit for bit, every step (also on the per-row path)."""
    wl = _ragged_kda(5, 8) if config == "kda_rows" else synth.make_workload(config, R=5, H=8)
    pools = [stq.stq_pool_create(wl.kind, wl.R, wl.S, wl.H, wl.unit_bits, wl.row_factor, wl.col_factor,
                                 flags=flags) for _ in range(2)]
    req, slot = _init(wl, pools[0])
    _init(wl, pools[1])
    u = torch.empty((wl.R, wl.H, 128), dtype=torch.float32, device="cuda")
    for t in range(10):
        x = _inputs(wl, t)
        y0 = torch.empty((wl.R, wl.H, 128), dtype=torch.float32, device="cuda")
        y1 = torch.empty_like(y0)
        stq.stq_decode_step(pools[0], req, slot, *x, y0)
        stq.stq_decode_step_split(pools[1], req, slot, *x, y1, u, side_stream=side_stream())
        stq.stq_pool_check(pools[0])
        stq.stq_pool_check(pools[1])
        assert torch.equal(y0, y1), t
        for a, (p0, p1) in enumerate(zip(_pages(pools[0], wl), _pages(pools[1], wl))):
            assert p0.tobytes() == p1.tobytes(), (t, a)
    for p in pools:
        p.close()


def test_readout_leaves_pages_and_writeback_completes_the_step():
    """The readout only reads the pages; the write-back given its u~ then
    produces the fused step's pages (both on one stream)."""
    pool, req, slot, H, rng = _simple_pool(bits=(4, 6, 8, 6, 8), R=3)
    ref, _, _, _, _ = _simple_pool(bits=(4, 6, 8, 6, 8), R=3)
    before = [stq.stq_export_slot(pool, a, 0) for a in range(3)]
    q, k = _unit_vecs(rng, (3, H, 128)), _unit_vecs(rng, (3, H, 128))
    v = rng.standard_normal((3, H, 128)).astype(np.float32)
    beta = rng.uniform(0, 1, (3, H)).astype(np.float32)
    gate = rng.uniform(0.9, 1.0, (3, H)).astype(np.float32)
    x = [_cuda(a) for a in (q, k, v, beta, gate)]
    y = torch.empty((3, H, 128), dtype=torch.float32, device="cuda")
    u = torch.empty_like(y)
    stq.stq_decode_readout(pool, req, slot, *x, y, u)
    stq.stq_pool_check(pool)
    for a in range(3):
        assert stq.stq_export_slot(pool, a, 0).tobytes() == before[a].tobytes()
    stq.stq_decode_writeback(pool, req, slot, x[1], x[4], u)
    y_ref = torch.empty_like(y)
    stq.stq_decode_step(ref, req, slot, *x, y_ref)
    stq.stq_pool_check(pool)
    stq.stq_pool_check(ref)
    assert torch.equal(y, y_ref)
    for a in range(3):
        assert stq.stq_export_slot(pool, a, 0).tobytes() == stq.stq_export_slot(ref, a, 0).tobytes()
    pool.close()
    ref.close()


def test_split_pending_writeback_is_ordered():
    """Back-to-back split steps with no explicit synchronisation: each
    readout waits for the previous write-back (the pool's pending event), and
    export waits for the last one; results equal the fused sequence."""
    wl = synth.make_workload(2, R=4, H=8)
    a, b = _pool(wl), _pool(wl)
    req, slot = _init(wl, a)
    _init(wl, b)
    u = torch.empty((wl.R, wl.H, 128), dtype=torch.float32, device="cuda")
    ys = []
    for t in range(6):
        x = _inputs(wl, t)
        y0 = torch.empty((wl.R, wl.H, 128), dtype=torch.float32, device="cuda")
        y1 = torch.empty_like(y0)
        stq.stq_decode_step(a, req, slot, *x, y0)
        stq.stq_decode_step_split(b, req, slot, *x, y1, u, side_stream=side_stream())
        ys.append((y0, y1))
    for p0, p1 in zip(_pages(a, wl), _pages(b, wl)):
        assert p0.tobytes() == p1.tobytes()
    torch.cuda.synchronize()
    for y0, y1 in ys:
        assert torch.equal(y0, y1)
    stq.stq_pool_check(a)
    stq.stq_pool_check(b)
    a.close()
    b.close()


def test_split_rejects_raw_pool():
    pool = stq.stq_pool_create(stq.STQ_GDN, 1, 1, 2, np.full(2, 16, np.uint8))
    req = _cuda(np.zeros(1, np.int32))
    e = torch.zeros((1, 2, 128), dtype=torch.float32, device="cuda")
    g = torch.ones((1, 2), dtype=torch.float32, device="cuda")
    with pytest.raises(stq.StqError) as err:
        stq.stq_decode_readout(pool, req, req, e, e, e, g, g, e.clone(), e.clone())
    assert err.value.status == stq.STQ_ERR_UNSUPPORTED
    pool.close()


def test_layer_loop_graph_split_matches_fused():
    """A 3-layer serving loop (one pool per layer) captured in a CUDA graph:
    per layer the readout on the capturing stream and the write-back on a
    side stream, joined at the end; replayed twice, it equals the fused
    step run eagerly layer by layer."""
    layers = 3
    wls = [synth.make_workload(4, R=6, H=16, seed=l) for l in range(layers)]
    pools = [_pool(w) for w in wls]
    refs = [_pool(w) for w in wls]
    idx = []
    for w, p, r in zip(wls, pools, refs):
        idx.append(_init(w, p))
        _init(w, r)
    xs = [_inputs(w, 0) for w in wls]
    ys = [torch.empty((w.R, w.H, 128), dtype=torch.float32, device="cuda") for w in wls]
    us = [torch.empty_like(y) for y in ys]
    main, side = torch.cuda.Stream(), torch.cuda.Stream()
    # one eager split step on a spare pool first (per-kernel set-up happens outside the capture)
    spare = _pool(wls[0])
    stq.stq_decode_step_split(spare, *idx[0], *xs[0], ys[0], us[0], side_stream=side)
    stq.stq_pool_check(spare)
    spare.close()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(main):
        side.wait_stream(main)
        g.capture_begin()
        for l in range(layers):
            stq.stq_decode_step_split(pools[l], *idx[l], *xs[l], ys[l], us[l], stream=main, side_stream=side)
        for p in pools:
            stq.stq_pool_join(p, main)
        g.capture_end()
    for rep in range(2):
        with torch.cuda.stream(main):
            g.replay()
        main.synchronize()
        for l in range(layers):
            y_ref = torch.empty_like(ys[l])
            stq.stq_decode_step(refs[l], *idx[l], *xs[l], y_ref)
            stq.stq_pool_check(refs[l])
            assert torch.equal(ys[l], y_ref), (rep, l)
            for p0, p1 in zip(_pages(pools[l], wls[l]), _pages(refs[l], wls[l])):
                assert p0.tobytes() == p1.tobytes(), (rep, l)
    for p in pools + refs:
        stq.stq_pool_check(p)
        p.close()


def test_split_full_size_sampled():
    """The benchmark workload shape (64 x 32 mixed GDN), split, sampled units
    against the oracle."""
    wl = synth.make_workload(2)
    rng = np.random.default_rng(21)
    units = [(int(a), int(h)) for a, h in zip(rng.integers(0, wl.R, 10), rng.integers(0, wl.H, 10))]
    units += [(wl.R - 1, wl.H - 1)]
    _teacher_forced(wl, steps=3, units=units, split=True)

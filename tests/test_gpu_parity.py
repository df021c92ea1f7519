"""GPU parity: the CUDA path through the C ABI against the CPU oracle.

Every decode step is compared teacher-forced: the oracle advances the
GPU's own page from the previous step (exported raw), and the GPU's next
page and readout must agree with it (codes bit-exact except logged +-1
near-ties, y and scales within max relative error 1e-5).  Quantize and
dequantize are bit-exact.
"""
import numpy as np
import pytest

import oracle as orc
from pages import Compare, decode_page, split_slot
from quantized_linear_attention_decode_b200 import stq, synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _cuda(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.to(dtype)
    return t.cuda()


def _pool(wl):
    return stq.stq_pool_create(wl.kind, wl.R, wl.S, wl.H, wl.unit_bits, wl.row_factor, wl.col_factor)


def _init(wl, pool):
    req = _cuda(np.arange(wl.R, dtype=np.int32))
    slot = _cuda(wl.slot_of_request.astype(np.int32))
    S0 = wl.initial_state()
    if S0 is not None:
        stq.stq_quantize_state(pool, req, slot, _cuda(S0))
        stq.stq_pool_check(pool)
    return req, slot


_side = None


def side_stream():
    global _side
    if _side is None:
        _side = torch.cuda.Stream()
    return _side


def _step(wl, pool, req, slot, t, requests=None, split=False):
    """One decode token: the fused step, or (split=True) the readout on the
    current stream and the write-back on a side stream."""
    inp = wl.step_inputs(t, requests)
    n = len(inp["beta"])
    y = torch.empty((n, wl.H, 128), dtype=torch.float32, device="cuda")
    x = [_cuda(inp[key]) for key in ("q", "k", "v", "beta", "gate")]
    if split:
        u = torch.empty((n, wl.H, 128), dtype=torch.float32, device="cuda")
        stq.stq_decode_step_split(pool, req, slot, *x, y, u, side_stream=side_stream())
    else:
        stq.stq_decode_step(pool, req, slot, *x, y)
    stq.stq_pool_check(pool)
    return inp, y.cpu().numpy()


def _oracle_unit(wl, rb, page, inp, a, h):
    g = inp["gate"][a, h]
    g = np.full(128, g, np.float32) if np.ndim(g) == 0 else g
    return orc.step_unit(rb[h], wl.row_factor.reshape(wl.H, 128)[h], wl.col_factor.reshape(wl.H, 128)[h],
                         page, inp["q"][a, h], inp["k"][a, h], inp["v"][a, h], inp["beta"][a, h], g)


def _teacher_forced(wl, steps, units=None, check_steps=None, split=False):
    """Runs `steps` decode steps on all requests; checks `units` ((request,
    head) pairs, default all) at `check_steps` (default all)."""
    pool = _pool(wl)
    req, slot = _init(wl, pool)
    rb = wl.row_bits()
    units = [(a, h) for a in range(wl.R) for h in range(wl.H)] if units is None else units
    reqs_checked = sorted({a for a, _ in units})
    cmp = Compare()
    for t in range(steps):
        check = check_steps is None or t in check_steps
        before = {a: split_slot(stq.stq_export_slot(pool, a, int(wl.slot_of_request[a])), rb)
                  for a in reqs_checked} if check else None
        inp, y = _step(wl, pool, req, slot, t, split=split)
        if not check:
            continue
        for a in reqs_checked:
            after = split_slot(stq.stq_export_slot(pool, a, int(wl.slot_of_request[a])), rb)
            for aa, h in units:
                if aa != a:
                    continue
                page_ref, y_ref, quot, st = _oracle_unit(wl, rb, before[a][h], inp, a, h)
                assert st == orc.OK
                where = f"(t={t}, req={a}, head={h})"
                cmp.y(y[a, h], y_ref, where)
                cmp.page(after[h], page_ref, quot, rb[h], where)
    cmp.finish()
    pool.close()
    return cmp


def _free_running(wl, steps):
    """Both sides advance their own chains from the same quantized start (the GPU's
    quantizer is bit-exact with the oracle's).  A unit is compared at every step
    until its first logged near-tie: after one, the two chains may differ by an
    LSB that the following steps carry forward.  Returns the comparison record
    and the number of unit-steps compared."""
    pool = _pool(wl)
    req, slot = _init(wl, pool)
    rb = wl.row_bits()
    own = {}
    for a in range(wl.R):
        for h, page in enumerate(split_slot(stq.stq_export_slot(pool, a, int(wl.slot_of_request[a])), rb)):
            own[(a, h)] = page.copy()
    live = set(own)
    cmp = Compare()
    compared = 0
    for t in range(steps):
        inp, y = _step(wl, pool, req, slot, t)
        for a in range(wl.R):
            after = split_slot(stq.stq_export_slot(pool, a, int(wl.slot_of_request[a])), rb)
            for h in range(wl.H):
                page_ref, y_ref, quot, st = _oracle_unit(wl, rb, own[(a, h)], inp, a, h)
                assert st == orc.OK
                own[(a, h)] = page_ref
                if (a, h) not in live:
                    continue
                where = f"(free-running t={t}, req={a}, head={h})"
                ties = len(cmp.ties)
                cmp.y(y[a, h], y_ref, where)
                cmp.page(after[h], page_ref, quot, rb[h], where)
                compared += 1
                if len(cmp.ties) > ties:
                    live.discard((a, h))
    cmp.finish()
    pool.close()
    return cmp, compared


@pytest.mark.parametrize("config, R, H, steps", [(2, 2, 8, 12), (3, 2, 4, 12)])
def test_decode_free_running(config, R, H, steps):
    """GDN mixed with outlier start, and KDA from zero: no teacher forcing."""
    wl = synth.make_workload(config, R=R, H=H)
    cmp, compared = _free_running(wl, steps)
    assert compared >= R * H * steps // 2, (compared, len(cmp.ties))


# ---------------------------------------------------------------- quantize / dequantize


@pytest.mark.parametrize("config", [1, 2, 3])
def test_quantize_dequantize_bit_exact(config):
    wl = synth.make_workload(config, R=3, H=8)
    wl.init = "outlier"  # a dense state with outlier rows and columns on every workload
    pool = _pool(wl)
    req, slot = _init(wl, pool)
    rb = wl.row_bits()
    S0 = wl.initial_state()
    r, c = wl.row_factor.reshape(wl.H, 128), wl.col_factor.reshape(wl.H, 128)
    back = torch.empty((wl.R, wl.H, 128, 128), dtype=torch.float32, device="cuda")
    stq.stq_dequantize_state(pool, req, slot, back)
    stq.stq_pool_check(pool)
    back = back.cpu().numpy()
    for a in range(wl.R):
        pages = split_slot(stq.stq_export_slot(pool, a, 0), rb)
        for h in range(wl.H):
            ref = orc.quantize_unit(rb[h], r[h], c[h], S0[a, h])
            assert pages[h].tobytes() == ref.tobytes(), (a, h)
            np.testing.assert_array_equal(back[a, h], orc.dequantize_unit(rb[h], r[h], c[h], ref))
    pool.close()


# ---------------------------------------------------------------- teacher-forced decode


def test_decode_config1_gdn_int8_full():
    """4 requests x 4 heads, INT8, 64 steps, every unit every step."""
    _teacher_forced(synth.make_workload(1), steps=64)


def test_decode_config2_gdn_mixed_small():
    """Mixed 4/6/8-bit heads, r, c ~ logU(0.25, 4), outlier start; 4 x 8 heads, 24 steps."""
    _teacher_forced(synth.make_workload(2, R=4, H=8), steps=24)


def test_decode_config3_kda_small():
    """KDA, per-row 4/6/8 bits and per-row decay; 4 x 4 heads, 24 steps."""
    _teacher_forced(synth.make_workload(3, R=4, H=4), steps=24)


def test_decode_ragged_kda_random_rows():
    """Odd request and head counts; row widths drawn independently (not
    balanced per head); slots other than 0; factors not 1."""
    rng = np.random.default_rng(11)
    wl = synth.make_workload(3, R=5, H=3)
    wl.unit_bits = rng.choice(np.array([4, 6, 8], np.uint8), size=3 * 128)
    wl.row_factor = np.exp(rng.uniform(-1, 1, 3 * 128)).astype(np.float32)
    wl.col_factor = np.exp(rng.uniform(-1, 1, 3 * 128)).astype(np.float32)
    wl.S = 3
    wl.slot_of_request = np.array([2, 0, 1, 2, 1], np.int32)
    wl.init = "outlier"
    _teacher_forced(wl, steps=12)


@pytest.mark.parametrize("config", [2, 3])
def test_decode_full_size_sampled(config):
    """Full workload shape (64 x 32 GDN mixed / 128 x 32 KDA), the launch the
    benchmark times; sampled units checked against the oracle."""
    wl = synth.make_workload(config)
    rng = np.random.default_rng(config)
    units = [(int(a), int(h)) for a, h in zip(rng.integers(0, wl.R, 12), rng.integers(0, wl.H, 12))]
    units += [(wl.R - 1, wl.H - 1), (0, 0)]
    _teacher_forced(wl, steps=6, units=units, check_steps={0, 1, 5})


def test_decode_serving_pool_max_size_sampled():
    """Serving pool: 256 requests x 5 slots x 768 heads (12 GB packed), one token."""
    wl = synth.make_workload(4, R=256)
    rng = np.random.default_rng(4)
    units = [(int(a), int(h)) for a, h in zip(rng.integers(0, wl.R, 10), rng.integers(0, wl.H, 10))]
    units += [(wl.R - 1, wl.H - 1)]
    _teacher_forced(wl, steps=2, units=units)


# ---------------------------------------------------------------- special cases


def _simple_pool(bits=(4, 6, 8, 6), R=2, S=1, kind=stq.STQ_GDN, seed=0):
    rng = np.random.default_rng(seed)
    H = len(bits) if kind == stq.STQ_GDN else 2
    ub = np.array(bits, np.uint8) if kind == stq.STQ_GDN else rng.choice(np.array([4, 6, 8], np.uint8), H * 128)
    r = np.exp(rng.uniform(-1, 1, H * 128)).astype(np.float32)
    c = np.exp(rng.uniform(-1, 1, H * 128)).astype(np.float32)
    pool = stq.stq_pool_create(kind, R, S, H, ub, r, c)
    S0 = rng.standard_normal((R, H, 128, 128)).astype(np.float32)
    req = _cuda(np.arange(R, dtype=np.int32))
    slot = _cuda(np.zeros(R, np.int32))
    stq.stq_quantize_state(pool, req, slot, _cuda(S0))
    stq.stq_pool_check(pool)
    return pool, req, slot, H, rng


def _unit_vecs(rng, shape):
    x = rng.standard_normal(shape)
    return (x / np.linalg.norm(x, axis=-1, keepdims=True)).astype(np.float32)


def _decode(pool, req, slot, q, k, v, beta, gate):
    n, H = beta.shape
    y = torch.empty((n, H, 128), dtype=torch.float32, device="cuda")
    stq.stq_decode_step(pool, req, slot, _cuda(q), _cuda(k), _cuda(v), _cuda(beta), _cuda(gate), y)
    return y


def test_retrieval_identity_gpu():
    """beta = 1, q = k, |k| = 1: y = v (readout before requantisation)."""
    pool, req, slot, H, rng = _simple_pool()
    for _ in range(3):
        k = _unit_vecs(rng, (2, H, 128))
        v = rng.standard_normal((2, H, 128)).astype(np.float32)
        y = _decode(pool, req, slot, k, k, v, np.ones((2, H), np.float32),
                    np.full((2, H), 0.95, np.float32))
        stq.stq_pool_check(pool)
        np.testing.assert_allclose(y.cpu().numpy(), v, rtol=0, atol=2e-5 * np.abs(v).max())


@pytest.mark.parametrize("kind", [stq.STQ_GDN, stq.STQ_KDA])
def test_idempotent_requant_gpu(kind):
    """beta = 0, gate = 1: codes unchanged bit for bit, scales within 1e-6."""
    pool, req, slot, H, rng = _simple_pool(kind=kind)
    before = [stq.stq_export_slot(pool, a, 0) for a in range(2)]
    gate = np.ones((2, H), np.float32) if kind == stq.STQ_GDN else np.ones((2, H, 128), np.float32)
    _decode(pool, req, slot, _unit_vecs(rng, (2, H, 128)), _unit_vecs(rng, (2, H, 128)),
            rng.standard_normal((2, H, 128)).astype(np.float32), np.zeros((2, H), np.float32), gate)
    stq.stq_pool_check(pool)
    rb = pool.row_bits
    for a in range(2):
        after = stq.stq_export_slot(pool, a, 0)
        for h, (p0, p1) in enumerate(zip(split_slot(before[a], rb), split_slot(after, rb))):
            s0, z0 = decode_page(p0, rb[h])
            s1, z1 = decode_page(p1, rb[h])
            np.testing.assert_array_equal(z1, z0)
            np.testing.assert_allclose(s1, s0, rtol=1e-6)


def test_empty_call_is_noop():
    pool, req, slot, H, rng = _simple_pool()
    e = torch.empty(0, dtype=torch.float32, device="cuda")
    n0 = stq.stq_launch_count()
    empty_i = torch.empty(0, dtype=torch.int32, device="cuda")
    stq.stq_decode_step(pool, empty_i, empty_i, e.view(0, H, 128), e.view(0, H, 128), e.view(0, H, 128),
                        e.view(0, H), e.view(0, H), e.view(0, H, 128))
    assert stq.stq_launch_count() == n0
    stq.stq_pool_check(pool)


def test_index_error_reported_and_tile_skipped():
    pool, req, slot, H, rng = _simple_pool()
    before = stq.stq_export_slot(pool, 1, 0)
    bad_req = _cuda(np.array([0, 7], np.int32))
    _decode(pool, bad_req, slot, _unit_vecs(rng, (2, H, 128)), _unit_vecs(rng, (2, H, 128)),
            rng.standard_normal((2, H, 128)).astype(np.float32), np.ones((2, H), np.float32),
            np.ones((2, H), np.float32))
    assert stq.stq_pool_check(pool, raise_on_error=False) == stq.STQ_ERR_INDEX
    assert stq.stq_pool_check(pool, raise_on_error=False) == stq.STQ_OK  # cleared
    assert stq.stq_export_slot(pool, 1, 0).tobytes() == before.tobytes()


def test_nonfinite_input_reported():
    pool, req, slot, H, rng = _simple_pool()
    v = rng.standard_normal((2, H, 128)).astype(np.float32)
    v[1, 2, 5] = np.nan
    _decode(pool, req, slot, _unit_vecs(rng, (2, H, 128)), _unit_vecs(rng, (2, H, 128)), v,
            np.ones((2, H), np.float32), np.ones((2, H), np.float32))
    assert stq.stq_pool_check(pool, raise_on_error=False) == stq.STQ_ERR_NONFINITE


def test_other_slots_untouched():
    rng = np.random.default_rng(3)
    H = 2
    pool = stq.stq_pool_create(stq.STQ_GDN, 2, 3, H, np.array([6, 8], np.uint8))
    req = _cuda(np.array([0, 1], np.int32))
    for s in range(3):
        stq.stq_quantize_state(pool, req, _cuda(np.full(2, s, np.int32)),
                               _cuda(rng.standard_normal((2, H, 128, 128)).astype(np.float32)))
    snap = {(a, s): stq.stq_export_slot(pool, a, s) for a in range(2) for s in range(3)}
    slot = _cuda(np.array([1, 2], np.int32))
    _decode(pool, req, slot, _unit_vecs(rng, (2, H, 128)), _unit_vecs(rng, (2, H, 128)),
            rng.standard_normal((2, H, 128)).astype(np.float32), np.ones((2, H), np.float32),
            np.full((2, H), 0.9, np.float32))
    stq.stq_pool_check(pool)
    for (a, s), data in snap.items():
        same = stq.stq_export_slot(pool, a, s).tobytes() == data.tobytes()
        assert same == ((a, s) not in ((0, 1), (1, 2))), (a, s)


def test_zero_key_keeps_zero_state():
    """From S = 0 with k = 0: X = 0, so the state stays zero and y = 0."""
    H = 3
    pool = stq.stq_pool_create(stq.STQ_GDN, 1, 1, H, np.array([4, 6, 8], np.uint8))
    req = _cuda(np.zeros(1, np.int32))
    rng = np.random.default_rng(5)
    y = _decode(pool, req, req, _unit_vecs(rng, (1, H, 128)), np.zeros((1, H, 128), np.float32),
                rng.standard_normal((1, H, 128)).astype(np.float32), np.ones((1, H), np.float32),
                np.ones((1, H), np.float32))
    stq.stq_pool_check(pool)
    assert not y.cpu().numpy().any()
    assert not stq.stq_export_slot(pool, 0, 0).any()

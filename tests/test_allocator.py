"""Lifetime-aware bit allocation (library host code) against the pages'
definitions: the lifetime weight as a sum and as a geometric series, the
exact optimum by enumeration on tiny instances, the budget, the Lagrangian
sufficiency property, and pivot selection by remaining risk."""
import math

import numpy as np
import pytest

import oracle as orc
from quantized_linear_attention_decode_b200 import stq

WIDTHS = [2, 4, 6, 8]  # the page's candidate widths


def _instance(rng, U, C=4):
    n = rng.choice([1, 2, 3, 4], U).astype(np.float64)
    # distortion falls with width (about 4x per bit pair), with per-unit scale and noise
    base = np.exp(rng.uniform(-2, 2, U))[:, None]
    d = base * 4.0 ** (-np.arange(C)[None, :]) * rng.uniform(0.7, 1.3, (U, C))
    d = np.minimum.accumulate(d, axis=1)
    w = stq.stq_lifetime_weight(-rng.exponential(0.05, U), 64)
    return n, d, w


@pytest.mark.parametrize("horizon", [1, 2, 7, 100, 4096])
def test_lifetime_weight_is_the_sum(horizon):
    rng = np.random.default_rng(horizon)
    ell = np.concatenate([[0.0, -1e-9, -2.0], -rng.exponential(0.1, 20)])
    got = stq.stq_lifetime_weight(ell, horizon)
    for e, g in zip(ell, got):
        want = orc.lifetime_weight_sum(float(e), horizon)
        assert abs(g - want) <= 1e-12 * want, (e, g, want)


def test_lifetime_weight_geometric_series_long_horizon():
    """For horizons past the explicit sum: (1 - e^{2 H l}) / (1 - e^{2 l}), and H at l = 0."""
    H = 8192
    for ell in (-1e-5, -1e-3, -0.05, -0.7):
        got = stq.stq_lifetime_weight([ell], H)[0]
        closed = (1 - math.exp(2 * H * ell)) / (1 - math.exp(2 * ell))
        assert abs(got - closed) <= 1e-11 * closed
        assert abs(got - orc.lifetime_weight_sum(ell, H)) <= 1e-10 * got
    assert stq.stq_lifetime_weight([0.0], H)[0] == H


@pytest.mark.parametrize("seed", range(60))
def test_dynamic_programme_is_optimal(seed):
    rng = np.random.default_rng(seed)
    U = int(rng.integers(1, 7))
    n, d, w = _instance(rng, U)
    mean = float(rng.choice([2.0, 3.0, 4.5, 5.0, 6.0, 7.5, 8.0]))
    bits, obj = stq.stq_allocate_bits(n, WIDTHS, d, w, mean, stq.STQ_ALLOC_DP)
    want, _ = orc.allocate_brute_force(n, WIDTHS, d.tolist(), w.tolist(), mean)
    assert abs(obj - want) <= 1e-12 * max(want, 1e-300)
    assert float(np.dot(n, bits)) <= mean * n.sum() + 1e-9
    k = [WIDTHS.index(b) for b in bits]
    assert abs(sum(w[u] * d[u, k[u]] for u in range(U)) - obj) <= 1e-12 * max(obj, 1e-300)


@pytest.mark.parametrize("seed", range(60))
def test_lagrangian_is_optimal_for_the_bits_it_uses(seed):
    """A per-unit minimiser of L d + lambda n b is the best assignment among
    all that cost no more than it does; it also respects the budget."""
    rng = np.random.default_rng(100 + seed)
    U = int(rng.integers(1, 7))
    n, d, w = _instance(rng, U)
    mean = float(rng.choice([2.5, 4.0, 5.0, 6.0, 7.0]))
    bits, obj = stq.stq_allocate_bits(n, WIDTHS, d, w, mean, stq.STQ_ALLOC_LAGRANGE)
    used = float(np.dot(n, bits))
    assert used <= mean * n.sum() + 1e-9
    want, _ = orc.allocate_brute_force(n, WIDTHS, d.tolist(), w.tolist(), mean, max_cost=used)
    assert abs(obj - want) <= 1e-12 * max(want, 1e-300)
    dp, dp_obj = stq.stq_allocate_bits(n, WIDTHS, d, w, mean, stq.STQ_ALLOC_DP)
    assert dp_obj <= obj * (1 + 1e-12)


def test_longer_lifetime_gets_no_fewer_bits():
    """Two units alike but for retention: the longer-lived one never gets fewer bits."""
    d = np.array([[1.0, 0.25, 0.06, 0.015]] * 2)
    n = np.array([16384.0, 16384.0])
    for short, long_ in [(-0.5, -0.01), (-0.1, -0.001), (-0.05, 0.0)]:
        w = stq.stq_lifetime_weight([short, long_], 2048)
        for mean in (3.0, 4.0, 5.0, 6.0, 7.0):
            bits, _ = stq.stq_allocate_bits(n, WIDTHS, d, w, mean)
            assert bits[1] >= bits[0], (short, long_, mean, bits)


def test_pivots_take_the_largest_remaining_risk():
    rng = np.random.default_rng(7)
    U = 40
    n, d, w = _instance(rng, U)
    bits, obj = stq.stq_allocate_bits(n, WIDTHS, d, w, 4.0)
    piv, obj2 = stq.stq_allocate_bits(n, WIDTHS, d, w, 4.0, num_pivots=5, pivot_bits=16)
    assert obj == obj2
    risk = np.array([w[u] * d[u, WIDTHS.index(bits[u])] for u in range(U)])
    top = set(np.argsort(-risk, kind="stable")[:5].tolist())
    assert {u for u in range(U) if piv[u] == 16} == top
    assert all(piv[u] == bits[u] for u in range(U) if u not in top)


def test_serving_scale_budgets_hold():
    """2304 GDN heads (exact programme) and 81920 KDA rows (Lagrangian) at a 6-bit budget over {4, 6, 8}."""
    rng = np.random.default_rng(3)
    for U, nv, method in [(2304, 16384.0, stq.STQ_ALLOC_DP), (81920, 128.0, stq.STQ_ALLOC_LAGRANGE)]:
        n = np.full(U, nv)
        d = np.exp(rng.uniform(-3, 3, U))[:, None] * 4.0 ** (-np.arange(3)[None, :])
        w = stq.stq_lifetime_weight(np.log(rng.uniform(0.9, 0.9999, U)), 8192)
        bits, obj = stq.stq_allocate_bits(n, [4, 6, 8], d, w, 6.0, method)
        assert float(np.dot(n, bits)) <= 6.0 * n.sum()
        assert set(np.unique(bits)) <= {4, 6, 8}
        assert float(np.dot(n, bits)) >= 5.99 * n.sum()  # the budget is essentially spent


def test_allocation_builds_a_pool_description():
    """Widths from the allocator make a valid GDN pool whose codes stay within the budget."""
    rng = np.random.default_rng(11)
    H = 32
    d = np.exp(rng.uniform(-2, 2, H))[:, None] * 4.0 ** (-np.arange(3)[None, :])
    w = stq.stq_lifetime_weight(np.log(rng.uniform(0.90, 0.999, H)), 8192)
    bits, _ = stq.stq_allocate_bits(np.full(H, 16384.0), [4, 6, 8], d, w, 6.0)
    _, slot = stq.stq_desc_bytes(stq.STQ_GDN, 1, 1, H, bits)
    assert slot == sum(512 + 2048 * int(b) for b in bits)
    assert slot <= H * (512 + 2048 * 6)


@pytest.mark.parametrize("kw", [
    dict(choices=[4, 4, 8]), dict(choices=[6, 4]), dict(mean=1.0), dict(method=5),
    dict(pivots=9), dict(weight=[-1.0] * 8), dict(dist=np.nan),
])
def test_allocator_rejects_bad_input(kw):
    n = np.full(8, 128.0)
    ch = kw.get("choices", [4, 6, 8])
    d = np.ones((8, len(ch)))
    if "dist" in kw:
        d[3, 1] = kw["dist"]
    w = np.array(kw.get("weight", [1.0] * 8))
    with pytest.raises(stq.StqError) as e:
        stq.stq_allocate_bits(n, ch, d, w, kw.get("mean", 6.0), kw.get("method", 0), kw.get("pivots", 0))
    assert e.value.status == stq.STQ_ERR_ARG
    with pytest.raises(stq.StqError):
        stq.stq_lifetime_weight([0.1], 10)

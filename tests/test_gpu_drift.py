"""GPU: long-generation drift against Proposition 1 of the page ("research
motivation" / "core method": E_t = A_t E_{t-1} + eps_t with ||A_t||_2 <= 1,
so ||E_t||_F <= sum_{tau <= t} ||eps_tau||_F).  The quantized state is run
next to the unquantized fp32 recurrence (a raw fp32 pool) on the same
inputs; each step's rounding error is at most half a quantisation step per
element, |eps_ij| <= s_i r_i c_j / 2, read from the new page's scales."""
import dataclasses

import numpy as np
import pytest

from pages import decode_page, split_slot
from quantized_linear_attention_decode_b200 import stq, synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("case", ["gdn_int4", "gdn_int6", "kda_mixed6"])
def test_state_error_within_proposition_1_bound(case):
    if case.startswith("gdn"):
        wl = synth.make_workload(5, R=2, H=4, T=256, bits=int(case[-1]))
    else:
        wl = dataclasses.replace(synth.make_workload(3, R=2, H=4), decay_range=(0.95, 0.9999))
    n_units = wl.H if wl.kind == synth.GDN else wl.H * 128
    pq = stq.stq_pool_create(wl.kind, wl.R, wl.S, wl.H, wl.unit_bits, wl.row_factor, wl.col_factor)
    pf = stq.stq_pool_create(wl.kind, wl.R, wl.S, wl.H, np.full(n_units, 32, np.uint8))
    req = torch.arange(wl.R, dtype=torch.int32, device="cuda")
    slot = torch.zeros(wl.R, dtype=torch.int32, device="cuda")
    rb = wl.row_bits()
    r, c = wl.row_factor.reshape(wl.H, 128), wl.col_factor.reshape(wl.H, 128)
    bound = np.zeros((wl.R, wl.H))
    Sq = torch.empty((wl.R, wl.H, 128, 128), dtype=torch.float32, device="cuda")
    Sf = torch.empty_like(Sq)
    worst = 0.0
    for t in range(256):
        inp = wl.step_inputs(t)
        x = [torch.from_numpy(inp[key]).cuda() for key in ("q", "k", "v", "beta", "gate")]
        y = torch.empty((wl.R, wl.H, 128), dtype=torch.float32, device="cuda")
        stq.stq_decode_step(pq, req, slot, *x, y)
        stq.stq_decode_step(pf, req, slot, *x, y)
        for a in range(wl.R):
            for h, page in enumerate(split_slot(stq.stq_export_slot(pq, a, 0), rb)):
                s, _ = decode_page(page, rb[h])
                step = s.astype(np.float64)[:, None] * r[h][:, None] * c[h][None, :]
                bound[a, h] += 0.5 * np.sqrt((step ** 2).sum())
        if (t + 1) % 32 == 0:
            stq.stq_dequantize_state(pq, req, slot, Sq)
            stq.stq_dequantize_state(pf, req, slot, Sf)
            E = torch.linalg.vector_norm((Sq - Sf).double(), dim=(2, 3)).cpu().numpy()
            S = torch.linalg.vector_norm(Sf.double(), dim=(2, 3)).cpu().numpy()
            # the fp32 control carries its own rounding: a few ulps of the state per step
            slack = 1e-6 * (t + 1) * S
            assert np.all(E <= bound + slack), (t, E.max(), bound.min())
            worst = max(worst, float((E / bound).max()))
    stq.stq_pool_check(pq)
    stq.stq_pool_check(pf)
    print(f"{case}: worst ||E_t|| / sum ||eps|| bound = {worst:.3f}")
    assert worst > 0.0
    pq.close()
    pf.close()


@pytest.mark.parametrize("bits", [4, 8])
def test_drift_anchored_to_oracle_fp64_recurrence(bits):
    """The drift workload's shape (alpha ~ U(0.95, 0.9999)), 2 requests x 4
    heads, 1024 steps, with the oracle's fp64 unquantized recurrence advanced
    alongside on the same inputs (the explicit-matrix pins fix that
    recurrence).  Every 128 steps:
      - the GPU's fp32 control (raw fp32 pool) stays within fp32 rounding of
        the fp64 state: at most a few ulps per step, accumulated without
        growth since ||A_t||_2 <= 1, so ||S_f32 - S||_F <= 4 * 2^-24 t ||S||_F;
      - the quantized state's error against the fp64 state stays under
        Proposition 1's bound sum_tau ||eps_tau||_F, plus the same fp32 slack."""
    import oracle as orc
    wl = synth.make_workload(5, R=2, H=4, T=1024, bits=bits)
    pq = stq.stq_pool_create(wl.kind, wl.R, wl.S, wl.H, wl.unit_bits, wl.row_factor, wl.col_factor)
    pf = stq.stq_pool_create(wl.kind, wl.R, wl.S, wl.H, np.full(wl.H, 32, np.uint8))
    req = torch.arange(wl.R, dtype=torch.int32, device="cuda")
    slot = torch.zeros(wl.R, dtype=torch.int32, device="cuda")
    rb = wl.row_bits()
    S64 = np.zeros((wl.R, wl.H, 128, 128))
    bound = np.zeros((wl.R, wl.H))
    Sq = torch.empty((wl.R, wl.H, 128, 128), dtype=torch.float32, device="cuda")
    Sf = torch.empty_like(Sq)
    worst_ctl, worst_q = 0.0, 0.0
    for t in range(1024):
        inp = wl.step_inputs(t)
        x = [torch.from_numpy(inp[key]).cuda() for key in ("q", "k", "v", "beta", "gate")]
        y = torch.empty((wl.R, wl.H, 128), dtype=torch.float32, device="cuda")
        stq.stq_decode_step(pq, req, slot, *x, y)
        stq.stq_decode_step(pf, req, slot, *x, y)
        for a in range(wl.R):
            for h in range(wl.H):
                S64[a, h], _ = orc.step_unit_f64(S64[a, h], inp["q"][a, h], inp["k"][a, h], inp["v"][a, h],
                                                 inp["beta"][a, h], inp["gate"][a, h])
            for h, page in enumerate(split_slot(stq.stq_export_slot(pq, a, 0), rb)):
                s, _ = decode_page(page, rb[h])
                bound[a, h] += 0.5 * np.sqrt((s.astype(np.float64) ** 2).sum() * 128)  # r = c = 1
        if (t + 1) % 128 == 0:
            stq.stq_dequantize_state(pq, req, slot, Sq)
            stq.stq_dequantize_state(pf, req, slot, Sf)
            ref = np.sqrt((S64 ** 2).sum(axis=(2, 3)))
            e_ctl = np.sqrt(((Sf.double().cpu().numpy() - S64) ** 2).sum(axis=(2, 3)))
            e_q = np.sqrt(((Sq.double().cpu().numpy() - S64) ** 2).sum(axis=(2, 3)))
            slack = 4 * 2.0 ** -24 * (t + 1) * ref
            assert np.all(e_ctl <= slack), (t, float((e_ctl / ref).max()))
            assert np.all(e_q <= bound + slack), (t, float((e_q / bound).max()))
            worst_ctl = max(worst_ctl, float((e_ctl / ref).max()))
            worst_q = max(worst_q, float((e_q / bound).max()))
    stq.stq_pool_check(pq)
    stq.stq_pool_check(pf)
    print(f"INT{bits}: fp32 control vs fp64 oracle, worst relative error {worst_ctl:.2e}; "
          f"quantized error / Prop. 1 bound, worst {worst_q:.3f}")
    pq.close()
    pf.close()

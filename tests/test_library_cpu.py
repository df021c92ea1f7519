"""Host-side checks of libstq.so that need no GPU: it loads, exports every
symbol include/stq.h declares, validates arguments, reproduces the pool
accounting, and injects faults on the host."""
import ctypes as C
import os
import re

import numpy as np
import pytest

import oracle as orc
from pages import decode_page, page_bytes, row_offsets
from quantized_linear_attention_decode_b200 import stq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "stq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(stq_[a-z_]+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    L = stq.load()
    names = _declared()
    assert "stq_decode_step" in names and len(names) >= 14
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(stq.EXPORTS)


def test_status_strings():
    for code, name in stq.STATUS.items():
        assert stq.stq_status_str(code) == name


def test_desc_bytes_reproduces_pool_formula():
    """pool = requests x slots x per-slot state ("SGLang state pool"); a
    page is 512 B of fp32 scales + 16 b bytes per row, padded to 128 B."""
    rng = np.random.default_rng(0)
    bits = rng.choice(np.array([4, 6, 8], np.uint8), 48)
    packed, slot = stq.stq_desc_bytes(stq.STQ_GDN, 7, 5, 48, bits)
    assert slot == sum(512 + 2048 * int(b) for b in bits)
    assert packed == 7 * 5 * slot
    kbits = rng.choice(np.array([4, 6, 8], np.uint8), 3 * 128)
    packed, slot = stq.stq_desc_bytes(stq.STQ_KDA, 2, 1, 3, kbits)
    assert slot == sum(page_bytes(kbits[h * 128:(h + 1) * 128]) for h in range(3))
    # the page's serving setting: batch 512, 5 slots, 2304 GDN heads of 128 x 128
    packed, _ = stq.stq_desc_bytes(stq.STQ_GDN, 512, 5, 2304, np.full(2304, 6, np.uint8))
    fp32 = 512 * 5 * 2304 * 128 * 128 * 4
    assert fp32 == 360 * 2 ** 30
    bits_per_value = packed * 8 / (512 * 5 * 2304 * 128 * 128)
    assert bits_per_value == 6.25  # 6-bit codes + one fp32 scale per 128 values
    assert abs(fp32 / packed - 32 / 6.25) < 1e-12


@pytest.mark.parametrize("bad", [
    dict(unit_bits=np.array([6, 5], np.uint8)),
    dict(kind=3),
    dict(R=0),
    dict(row_factor=np.array([1.0] * 255 + [0.0], np.float32)),
    dict(col_factor=np.array([1.0] * 255 + [np.nan], np.float32)),
])
def test_desc_validation(bad):
    args = dict(kind=stq.STQ_GDN, R=1, S=1, H=2, unit_bits=np.array([6, 8], np.uint8),
                row_factor=None, col_factor=None)
    args.update(bad)
    with pytest.raises(stq.StqError) as e:
        stq.stq_desc_bytes(args["kind"], args["R"], args["S"], args["H"], args["unit_bits"],
                           args["row_factor"], args["col_factor"])
    assert e.value.status == stq.STQ_ERR_ARG


def test_desc_bytes_formats():
    """Binary16 scales save 256 B per page; raw pools are 128 x 128 values of
    2 or 4 bytes with no scales (the page's fp16 storage and fp32 control)."""
    bits = np.array([4, 6, 8, 6], np.uint8)
    _, f32 = stq.stq_desc_bytes(stq.STQ_GDN, 1, 1, 4, bits)
    _, f16 = stq.stq_desc_bytes(stq.STQ_GDN, 1, 1, 4, bits, flags=stq.STQ_SCALE_F16)
    assert f32 - f16 == 4 * 256
    assert f16 == sum(256 + 2048 * int(b) for b in bits)
    for b in (16, 32):
        _, slot = stq.stq_desc_bytes(stq.STQ_GDN, 1, 1, 4, np.full(4, b, np.uint8))
        assert slot == 4 * 128 * 128 * b // 8
        _, slot = stq.stq_desc_bytes(stq.STQ_KDA, 1, 1, 2, np.full(256, b, np.uint8))
        assert slot == 2 * 128 * 128 * b // 8
    # the page's compression ratios follow 32 / bits (raw 16: exactly 2x)
    _, s32 = stq.stq_desc_bytes(stq.STQ_GDN, 1, 1, 4, np.full(4, 32, np.uint8))
    _, s16 = stq.stq_desc_bytes(stq.STQ_GDN, 1, 1, 4, np.full(4, 16, np.uint8))
    assert s32 == 2 * s16


def test_desc_bytes_fitted_columns():
    """Fitted column factors add 128 fp32 values to every page; row weights must be > 0."""
    bits = np.array([4, 6, 8, 6], np.uint8)
    _, plain = stq.stq_desc_bytes(stq.STQ_GDN, 1, 1, 4, bits)
    _, fit = stq.stq_desc_bytes(stq.STQ_GDN, 1, 1, 4, bits, flags=stq.STQ_FIT_COLUMNS)
    assert fit - plain == 4 * 512
    w = np.ones(4 * 128, np.float32)
    w[7] = 0.0
    with pytest.raises(stq.StqError) as e:
        stq.stq_desc_bytes(stq.STQ_GDN, 1, 1, 4, bits, flags=stq.STQ_FIT_COLUMNS, row_weight=w)
    assert e.value.status == stq.STQ_ERR_ARG


def test_desc_bytes_pivot_pool():
    """16-bit units among quantized ones are FP16 pivots: every page keeps its scale
    section, a pivot head holds 128 rows of 256 B."""
    for flags, sb in ((0, 512), (stq.STQ_SCALE_F16, 256)):
        bits = np.array([16, 6, 8, 16], np.uint8)
        _, slot = stq.stq_desc_bytes(stq.STQ_GDN, 1, 1, 4, bits, flags=flags)
        assert slot == sum(sb + 2048 * int(b) for b in bits)
        kb = np.tile(np.array([16] + [6] * 127, np.uint8), 2)
        _, slot = stq.stq_desc_bytes(stq.STQ_KDA, 1, 1, 2, kb, flags=flags)
        assert slot == 2 * ((sb + 256 + 127 * 96 + 127) // 128 * 128)


@pytest.mark.parametrize("ub, flags, status", [
    ([32, 16, 32, 32], 0, "STQ_ERR_UNSUPPORTED"),  # two raw widths
    ([32, 8, 32, 32], 0, "STQ_ERR_UNSUPPORTED"),   # fp32 units among quantized ones
    ([16, 16, 16, 16], 1, "STQ_ERR_ARG"),          # a raw pool has no scales
    ([6, 6, 6, 6], 4, "STQ_ERR_ARG"),              # unknown flag
    ([16, 16, 16, 16], 2, "STQ_ERR_ARG"),          # a raw pool has no scales or factors
    ([6, 12, 6, 6], 0, "STQ_ERR_ARG"),
])
def test_desc_format_validation(ub, flags, status):
    with pytest.raises(stq.StqError) as e:
        stq.stq_desc_bytes(stq.STQ_GDN, 1, 1, 4, np.array(ub, np.uint8), flags=flags)
    assert stq.STATUS[e.value.status] == status


def test_fitted_pool_with_pivots_layout():
    """FP16 pivot units in a fitted pool: each page keeps its scales, its 128 fp32
    column factors, and 256 bytes per pivot row (GDN: a whole pivot head)."""
    bits = np.array([16, 6, 8, 6], np.uint8)
    _, slot = stq.stq_desc_bytes(stq.STQ_GDN, 1, 1, 4, bits, flags=stq.STQ_FIT_COLUMNS)
    page = lambda b: (512 + 512 + 16 * 128 * b + 127) // 128 * 128  # noqa: E731
    assert slot == sum(page(int(b)) for b in bits)
    kb = np.tile(np.array([16] * 8 + [4] * 120, np.uint8), 2)
    _, kslot = stq.stq_desc_bytes(stq.STQ_KDA, 1, 1, 2, kb, flags=stq.STQ_FIT_COLUMNS | stq.STQ_SCALE_F16)
    assert kslot == 2 * ((256 + 512 + 8 * 256 + 120 * 64 + 127) // 128 * 128)


def test_unsupported_head_dim():
    L = stq.load()
    ub = np.array([6], np.uint8)
    d = stq._Desc(0, 1, 1, 1, 64, 64, ub.ctypes.data, None, None, 0, None)
    a, b = C.c_size_t(), C.c_size_t()
    assert L.stq_desc_bytes(C.byref(d), C.byref(a), C.byref(b)) == stq.STQ_ERR_UNSUPPORTED


def test_null_arguments_rejected_before_any_cuda_call():
    L = stq.load()
    assert L.stq_pool_create(None, None) == stq.STQ_ERR_ARG
    assert L.stq_decode_step(None, None, None, 0, None, None, None, None, None, None, None) == stq.STQ_ERR_ARG
    assert L.stq_decode_step_host(None, None, None, 0, None, None, None, None, None, None, None) == stq.STQ_ERR_ARG
    assert L.stq_decode_readout(None, None, None, 0, None, None, None, None, None, None, None,
                                None) == stq.STQ_ERR_ARG
    assert L.stq_decode_writeback(None, None, None, 0, None, None, None, None) == stq.STQ_ERR_ARG
    assert L.stq_decode_step_split(None, None, None, 0, None, None, None, None, None, None, None, None,
                                   None) == stq.STQ_ERR_ARG
    assert L.stq_pool_join(None, None) == stq.STQ_ERR_ARG
    assert L.stq_pool_check(None, None) == stq.STQ_ERR_ARG
    assert L.stq_export_slot(None, 0, 0, None, 0) == stq.STQ_ERR_ARG


def test_fault_injection_alloc(monkeypatch):
    monkeypatch.setenv("STQ_FAULT", "alloc")
    with pytest.raises(stq.StqError) as e:
        stq.stq_pool_create(stq.STQ_GDN, 1, 1, 1, np.array([8], np.uint8))
    assert e.value.status == stq.STQ_ERR_OOM
    assert "injected" in stq.stq_last_error()


def test_page_reader_agrees_with_oracle_packer():
    """The tests' vectorised page reader and the oracle's bit-by-bit packer
    read the same bytes the same way."""
    rng = np.random.default_rng(9)
    bits = rng.choice(np.array([4, 6, 8], np.uint8), 128)
    page = np.zeros(page_bytes(bits), np.uint8)
    assert len(page) == orc.page_bytes(bits)
    np.testing.assert_array_equal(row_offsets(bits), orc.row_offsets(bits))
    want = np.zeros((128, 128), np.int32)
    offs = row_offsets(bits)
    for i, b in enumerate(bits):
        q = (1 << (int(b) - 1)) - 1
        want[i] = rng.integers(-q, q + 1, 128)
        row = np.zeros(16 * int(b), np.uint8)
        for j in range(128):
            orc.put_code(row, int(b), j, int(want[i, j]))
        page[offs[i]: offs[i] + len(row)] = row
    page[:512] = np.arange(128, dtype=np.float32).view(np.uint8)
    s, z = decode_page(page, bits)
    np.testing.assert_array_equal(z, want)
    np.testing.assert_array_equal(s, np.arange(128, dtype=np.float32))


def test_compare_checks_binary16_pages():
    """The parity checker accepts identical binary16-scale pages and rejects
    a planted code change that is not a rounding tie (planted in an
    oracle-made page, on the CPU)."""
    import oracle as orc
    from pages import Compare
    rng = np.random.default_rng(5)
    bits = np.full(128, 6, np.uint8)
    S = rng.standard_normal((128, 128)).astype(np.float32)
    page, quot, _ = orc.quantize_unit(bits, np.ones(128), np.ones(128), S, with_quot=True, fmt=orc.FMT_F16)
    cmp = Compare()
    cmp.page(page, page, quot, bits, fmt=1)
    bad = page.copy()
    bad[256] ^= 0x3  # code 0 of row 0 changes by more than one step
    with pytest.raises(AssertionError):
        Compare().page(bad, page, quot, bits, fmt=1)


C_PROGRAM = r"""
#include <math.h>
#include <stdio.h>
#include <string.h>
#include "stq.h"

int main(void)
{
    /* pool accounting without a device: 2 requests x 1 slot x 3 GDN heads at 6 bits */
    const uint8_t bits[3] = {6, 6, 6};
    stq_pool_desc d;
    memset(&d, 0, sizeof d);
    d.kind = STQ_GDN;
    d.num_requests = 2;
    d.num_slots = 1;
    d.num_heads = 3;
    d.d_k = 128;
    d.d_v = 128;
    d.unit_bits = bits;
    size_t packed = 0, slot = 0;
    if (stq_desc_bytes(&d, &packed, &slot) != STQ_OK) return 1;
    if (slot != 3u * (512u + 2048u * 6u) || packed != 2u * slot) return 2;
    /* a bad description is refused with a message, an unsupported head size with its own status */
    d.num_requests = 0;
    if (stq_desc_bytes(&d, &packed, &slot) != STQ_ERR_ARG || strlen(stq_last_error()) == 0) return 3;
    d.num_requests = 2;
    d.d_k = 64;
    if (stq_desc_bytes(&d, &packed, &slot) != STQ_ERR_UNSUPPORTED) return 6;
    /* L_u for l_u = log(1/2) over 4 steps: 1 + 1/4 + 1/16 + 1/64 */
    const double l = log(0.5);
    double w = 0.0;
    if (stq_lifetime_weight(1, &l, 4, &w) != STQ_OK || fabs(w - 1.328125) > 1e-15) return 4;
    if (stq_launch_count() != 0) return 5;
    printf("%s\n", stq_status_str(STQ_OK));
    return 0;
}
"""


def test_header_is_plain_c_and_the_library_links_from_c(tmp_path):
    """include/stq.h compiles as strict C99 and a C program links against
    libstq.so and calls its host-side entry points (no device needed)."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    stq.load()
    libdir = os.path.dirname(stq.LIB_PATH)
    src = tmp_path / "t.c"
    src.write_text(C_PROGRAM)
    exe = tmp_path / "t"
    r = subprocess.run([gcc, "-std=c99", "-pedantic", "-Wall", "-Wextra", "-Werror",
                        "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe),
                        "-L", libdir, "-lstq", "-lm", "-Wl,-rpath," + libdir],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0 and r.stdout.strip() == "STQ_OK", (r.returncode, r.stdout, r.stderr)

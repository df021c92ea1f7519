"""Host-side accounting of the benchmark (CPU): the algorithmic bytes each
head-step must move, per launch, and the use of the recorded ncu traffic.

The per-head-step figures are worked out by hand from the step's data flow:
codes read and written (2 x 16 sum_i b_i bytes), 128 fp32 scales read and
written (2 x 512), q, k, v read and y written (4 x 512), beta read (4), and
the gate read (4 bytes of alpha for GDN, 512 bytes of d for KDA)."""
import json
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from quantized_linear_attention_decode_b200 import synth  # noqa: E402


def test_bytes_per_head_step():
    f = synth.algorithmic_bytes_per_head_step
    assert f(synth.GDN, 128 * 4) == 8192 * 2 + 1024 + 2048 + 4 + 4 == 19464
    assert f(synth.GDN, 128 * 6) == 12288 * 2 + 1024 + 2048 + 4 + 4 == 27656
    assert f(synth.GDN, 128 * 8) == 16384 * 2 + 1024 + 2048 + 4 + 4 == 35848
    # KDA head of 32 rows at 4, 64 at 6, 32 at 8 bits: 768 bits per column, as a 6-bit head
    assert f(synth.KDA, 32 * 4 + 64 * 6 + 32 * 8) == 12288 * 2 + 1024 + 2048 + 4 + 512 == 28164
    # binary16 scales: 2 x 256 bytes; raw states (no scales): a binary16 state is 128 x 128 x 16 bits,
    # an fp32 state 128 x 128 x 32 bits, read and written
    assert f(synth.GDN, 128 * 6, scale_bytes=2) == 12288 * 2 + 512 + 2048 + 4 + 4 == 27144
    assert f(synth.GDN, 128 * 16, scale_bytes=0) == 32768 * 2 + 2048 + 4 + 4 == 67592
    assert f(synth.GDN, 128 * 32, scale_bytes=0) == 65536 * 2 + 2048 + 4 + 4 == 133128


def test_bytes_per_launch_of_the_bench_workload():
    """64 requests x 32 heads, heads 25 / 50 / 25 % at 4 / 6 / 8 bits (mean 6), plus the
    r and c tables (1 KiB per head) read once per launch."""
    wl = synth.make_workload(2)
    rb = wl.row_bits()
    widths = rb[:, 0]
    assert (rb == widths[:, None]).all()
    assert sorted(np.unique(widths, return_counts=True)[1].tolist()) == [8, 8, 16]
    per_request = 8 * 19464 + 16 * 27656 + 8 * 35848
    total, mean_bits = bench.workload_info(wl)
    assert total == 64 * per_request + 32 * 1024 == 56672256
    assert mean_bits == 6.0


def test_recorded_traffic_only_for_the_current_kernel(tmp_path, monkeypatch):
    rec = {"config2": {"kernel_sha": "abc", "dram_bytes_per_launch": 123}}
    path = tmp_path / "traffic.json"
    path.write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(path))
    monkeypatch.setattr(bench, "kernel_sha", lambda: "abc")
    assert bench.recorded_traffic(2) == 123
    assert bench.recorded_traffic(3) is None
    monkeypatch.setattr(bench, "kernel_sha", lambda: "changed")
    assert bench.recorded_traffic(2) is None


def test_committed_traffic_record_covers_the_algorithmic_reads():
    """While the committed record belongs to the kernel source as it stands (else the
    bench reports no traffic and this is skipped), its DRAM reads cover at least the
    algorithmic reads of a launch."""
    d = json.load(open(bench.TRAFFIC_FILE))
    if d["config2"]["kernel_sha"] != bench.kernel_sha():
        pytest.skip("the traffic record predates the current kernel source")
    wl = synth.make_workload(2)
    reads = sum(synth.algorithmic_bytes_per_head_step(wl.kind, int(b.sum())) for b in wl.row_bits())
    reads = wl.R * (reads - sum(16 * int(b.sum()) + 512 + 512 for b in wl.row_bits()))  # minus writes
    assert d["config2"]["dram_read"] >= 0.99 * reads

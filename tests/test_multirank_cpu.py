"""The multi-process (N > 1) paths of bench.py, on CPU with the gloo backend.

The decode step shards with no data-path collective: every rank advances
its own requests, and only the timing is combined (max over ranks).
"""
import os
import subprocess
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from quantized_linear_attention_decode_b200 import synth  # noqa: E402


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r, w = bench.rank_world(None)
        slowest = bench.max_over_ranks(float(10 + rank), dist, "cpu")
        wl = synth.make_workload(2, seed=bench.shard_seed(0, r), R=2, H=4, T=1)
        v0 = wl.step_inputs(0)["v"]
        q.put((r, w, slowest, float(v0.sum())))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_max_and_independent_shards():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + os.getpid() % 1000
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [o[0] for o in out] == [0, 1] and all(o[1] == 2 for o in out)
    assert all(o[2] == 11.0 for o in out)          # every rank sees the slowest rank's time
    assert out[0][3] != out[1][3]                   # shards draw different requests


def test_reference_arm_non_zero_rank_exits_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "2", "--warmup", "1"], env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""


@pytest.mark.parametrize("rank", [0, 1])
def test_shard_seeds_distinct(rank):
    assert bench.shard_seed(0, rank) == (0 if rank == 0 else 1000003)
    a = synth.make_workload(2, seed=bench.shard_seed(0, 0), R=1, H=4, T=1).step_inputs(0)["k"]
    b = synth.make_workload(2, seed=bench.shard_seed(0, 1), R=1, H=4, T=1).step_inputs(0)["k"]
    assert not np.array_equal(a, b)

#!/usr/bin/env python
"""Benchmark: quantized gated delta-rule decode on B200.

One step = one decode token over the whole batch of the workload (every
(request, head) unit: unpack, dequantise, decay, retrieve, delta write,
readout, requantise, repack), i.e. one launch of the fused decode kernel.

Default workload: GDN with per-head 4/6/8-bit states averaging 6 bits,
64 requests x 32 heads, d_k = d_v = 128, r, c ~ logU(0.25, 4), outlier
initial state, inputs of a 256-token sequence (cycled when more steps are
timed).  The L2 cache is flushed (a 384 MiB buffer is written) before every
timed step, outside the timed interval, so each step reads its pages from
HBM as it would in a 48-layer model.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Multi-GPU: one process per GPU (torchrun); every rank advances its own
shard of requests (no data-path collective, weak scaling); the timed
duration is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from quantized_linear_attention_decode_b200 import synth  # noqa: E402

METRIC = "quantized-state decode head-steps/s and achieved HBM GB/s vs B200 peak"
UNIT = "head-steps/s"
L2_FLUSH_BYTES = 384 << 20
DECODE_KERNEL = "decode_kernel"
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "decode_traffic.json")
KERNEL_SRC = os.path.join(ROOT, "quantized_linear_attention_decode_b200", "csrc", "stq_decode.cu")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=8)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--kda-allocated", action="store_true",
                    help="config 3 with per-row widths from the allocator and 8 FP16 pivot rows per head "
                         "(no CPU baseline, no recorded traffic)")
    ap.add_argument("--config", type=int, default=2, choices=[2, 3, 4],
                    help="2: GDN mixed 64 x 32 (default); 3: KDA 128 x 32; 4: serving pool (see --requests)")
    ap.add_argument("--requests", type=int, default=None, help="requests of the workload (default: its own)")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--tokens", type=int, default=256, help="distinct input tokens (cycled)")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="oracle sample budget")
    ap.add_argument("--no-sweep", action="store_true", help="skip the serving-pool sweep")
    ap.add_argument("--no-layer-loop", action="store_true", help="skip the 48-layer graph comparison")
    ap.add_argument("--no-drift", action="store_true", help="skip the long-generation drift record")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=200)
    return ap.parse_args()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def kernel_sha() -> str:
    """Hash of the decode kernel's code: its source with comments and white
    space removed, so that a comment edit keeps the recorded counters."""
    import re
    src = open(KERNEL_SRC).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    src = re.sub(r"//[^\n]*", "", src)
    src = re.sub(r"\s+", "", src)
    return hashlib.sha256(src.encode()).hexdigest()[:16]


def recorded_traffic(config: int, requests=None):
    """DRAM bytes (read + write) per launch from the committed ncu summary, if
    the kernel source is unchanged since it was taken and the record is of
    this workload's size; else None."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    d = json.load(open(TRAFFIC_FILE))
    e = d.get(f"config{config}")
    if not e or e.get("kernel_sha") != kernel_sha():
        return None
    if "requests" in e and requests is not None and e["requests"] != requests:
        return None
    return e.get("dram_bytes_per_launch")


def workload_info(wl, unit_bits=None, scale_bytes: int = 4):
    """(algorithmic HBM bytes of one launch over the whole workload, mean
    bits per state value); `unit_bits` replaces the workload's widths (a raw
    fp16 / fp32 pool, scale_bytes 0)."""
    ub = wl.unit_bits if unit_bits is None else np.asarray(unit_bits)
    rb = (np.repeat(ub.reshape(wl.H, 1), 128, axis=1) if wl.kind == synth.GDN else ub.reshape(wl.H, 128))
    rb = rb.astype(np.int64)
    per_head = [synth.algorithmic_bytes_per_head_step(wl.kind, int(rb[h].sum()), scale_bytes) for h in range(wl.H)]
    tables = wl.H * (2 * 128 * 4) if scale_bytes else 0  # r and c read once per head per launch
    bytes_per_launch = wl.R * sum(per_head) + tables
    return bytes_per_launch, float(rb.mean())


# ---------------------------------------------------------------------- ranks


def rank_world(args):
    """(rank, world size) from the torchrun environment; 1 process otherwise."""
    return int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1"))


def shard_seed(base_seed: int, rank: int) -> int:
    """Each rank advances its own shard of requests, drawn from its own seed."""
    return base_seed + 1000003 * rank


def max_over_ranks(x: float, dist=None, device: str = "cpu") -> float:
    """The slowest rank's value (every rank calls this once per quantity)."""
    if dist is None:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------------- clocks


class ClockSampler:
    """Samples SM clock, power and throttle reasons with NVML while running."""

    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4,
        "hw_slowdown": 0x8, "sync_boost": 0x10, "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80, "display_clock_setting": 0x100,
    }

    def __init__(self, index: int, period: float = 0.01):
        self.period = period
        self.samples = []
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # noqa: BLE001
            self.err = str(e)
        self._stop = threading.Event()

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                reasons = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                util = nv.nvmlDeviceGetUtilizationRates(self.h).gpu
                self.samples.append((mhz, reasons, util))
            except Exception:  # noqa: BLE001
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self.ok:
            self.t.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "error": self.err}
        busy = [s for s in self.samples if s[2] > 0] or self.samples
        seen = 0
        for s in busy:
            seen |= s[1]
        names = [n for n, bit in self.REASONS.items() if seen & bit and n != "gpu_idle"]
        return {"sm_mhz": statistics.median([s[0] for s in busy]) if busy else None,
                "sm_max_mhz": self.max_mhz, "reasons": names, "samples": len(busy)}


# ---------------------------------------------------------------------- oracle (CPU baseline)


class OracleRunner:
    """The CPU oracle as it stands (OpenMP over units), set up on the first
    `requests` requests of the workload (pages quantized by the oracle)."""

    def __init__(self, config: int, seed: int, requests: int = 8):
        import oracle as orc
        self.orc = orc
        wl = self.wl = synth.make_workload(config, seed=seed)
        self.R = R = min(wl.R, requests)
        self.rb = rb = wl.row_bits()
        self.r, self.c = wl.row_factor.reshape(wl.H, 128), wl.col_factor.reshape(wl.H, 128)
        S0 = wl.initial_state(np.arange(R))
        sizes = [orc.page_bytes(rb[h]) for h in range(wl.H)]
        head_off = np.concatenate([[0], np.cumsum(sizes)[:-1]])
        slot = int(sum(sizes))
        self.pages = np.zeros(R * slot, np.uint8)
        for a in range(R):
            for h in range(wl.H):
                st = S0[a, h] if S0 is not None else np.zeros((128, 128), np.float32)
                o = a * slot + head_off[h]
                self.pages[o: o + sizes[h]] = orc.quantize_unit(rb[h], self.r[h], self.c[h], st)
        self.head = np.tile(np.arange(wl.H, dtype=np.int32), R)
        self.offs = (np.repeat(np.arange(R), wl.H) * slot + np.tile(head_off, R)).astype(np.int64)
        self.threads = orc.default_threads()
        self.inputs = {}

    def _inp(self, t):
        if t not in self.inputs:
            wl, R = self.wl, self.R
            inp = wl.step_inputs(t, np.arange(R))
            g = inp["gate"]
            g = np.repeat(g.reshape(R * wl.H, 1), 128, axis=1) if g.ndim == 2 else g.reshape(R * wl.H, 128)
            self.inputs = {t: (inp["q"].reshape(-1, 128), inp["k"].reshape(-1, 128),
                               inp["v"].reshape(-1, 128), inp["beta"].reshape(-1), np.ascontiguousarray(g))}
        return self.inputs[t]

    def step(self, t: int, units: int) -> float:
        """Advances the first `units` units by token t; returns seconds."""
        q, k, v, beta, g = self._inp(t)
        u = min(units, len(self.head))
        t0 = time.perf_counter()
        out, _, _ = self.orc.step_many(self.head[:u], self.rb, self.r, self.c, self.pages,
                                       self.offs[:u], self.offs[:u], len(self.pages), q[:u], k[:u],
                                       v[:u], beta[:u], g[:u], self.threads)
        dt = time.perf_counter() - t0
        self.pages = out if u == len(self.head) else self._merge(out, u)
        return dt

    def _merge(self, out, u):
        pages = self.pages.copy()
        for n in range(u):
            h = self.head[n]
            o = self.offs[n]
            nb = self.orc.page_bytes(self.rb[h])
            pages[o: o + nb] = out[o: o + nb]
        return pages


def oracle_baseline(config: int, seed: int, seconds: float):
    """Times the oracle on a bounded sample: consecutive tokens over all units
    of its first requests until the time budget is spent."""
    run = OracleRunner(config, seed)
    units = len(run.head)
    done, total, t = 0, 0.0, 0
    while total < seconds:
        total += run.step(t, units)
        done += units
        t += 1
    sample = (f"{t} consecutive tokens x {run.R} requests x {run.wl.H} heads of {run.wl.name} "
              f"({done} head-steps, {total:.1f} s of oracle time)")
    threads = run.threads
    # the same oracle on one core, for a quarter of the budget
    run.threads = 1
    done1, total1 = 0, 0.0
    while total1 < seconds / 4:
        total1 += run.step(t, units)
        done1 += units
        t += 1
    return done / total, threads, sample, done1 / total1


def run_reference(args, rank: int, world: int):
    if rank != 0:
        return
    run = OracleRunner(args.config, args.seed)
    wl = run.wl
    nsteps = args.warmup + args.steps
    per_step_s = min(1.0, max(0.02, 150.0 / max(nsteps, 1)))
    # size each step's sample of units to the per-step budget
    dt = run.step(0, 8)
    units = int(max(1, min(len(run.head), 8 * per_step_s / max(dt, 1e-6))))
    done, total = 0, 0.0
    for i in range(nsteps):
        s = run.step(1 + i, units)
        if i >= args.warmup:
            total += s
            done += units
    value = done / total
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * wl.R * wl.H / value, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64+f32", "data": "synthetic",
        "config": {"workload": wl.name, "requests": wl.R, "heads": wl.H, "d_k": 128, "d_v": 128},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": run.threads, "kind": "oracle",
                         "sample": f"{units} units of {wl.name} per step, {args.steps} timed steps "
                                   f"({done} head-steps, {total:.1f} s)"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------- GPU arm


def run_ours(args, rank: int, world: int):
    import torch
    from quantized_linear_attention_decode_b200 import stq

    dev = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(dev)
    dist = None
    # under torchrun (LOCAL_WORLD_SIZE set) the process group is used even by a single rank,
    # so that a one-GPU launch runs the same collective path as the scaling runs
    if world > 1 or "LOCAL_WORLD_SIZE" in os.environ:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", dev))
    wl = synth.make_workload(args.config, seed=shard_seed(args.seed, rank), R=args.requests)
    if args.kda_allocated:
        if args.config != 3:
            raise SystemExit("--kda-allocated needs --config 3")
        import dataclasses
        wl = dataclasses.replace(wl, unit_bits=kda_allocated_bits(stq, wl.H, 0),
                                 name=wl.name.replace("mixed6", "allocated_pivots"))
    pool = stq.stq_pool_create(wl.kind, wl.R, wl.S, wl.H, wl.unit_bits, wl.row_factor, wl.col_factor)
    req = torch.arange(wl.R, dtype=torch.int32, device="cuda")
    slot = torch.from_numpy(wl.slot_of_request.astype(np.int32)).cuda()
    S0 = wl.initial_state()
    if S0 is not None:
        stq.stq_quantize_state(pool, req, slot, torch.from_numpy(S0).cuda())
        stq.stq_pool_check(pool)
        del S0
    ntok = max(1, args.tokens)
    toks = []
    for t in range(ntok):
        inp = wl.step_inputs(t)
        toks.append({k: torch.from_numpy(v).cuda() for k, v in inp.items()})
    y = torch.empty((wl.R, wl.H, 128), dtype=torch.float32, device="cuda")
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()

    def step(t):
        x = toks[t % ntok]
        stq.stq_decode_step(pool, req, slot, x["q"], x["k"], x["v"], x["beta"], x["gate"], y, stream)

    for t in range(args.warmup):
        flush.zero_()
        step(t)
    stq.stq_pool_check(pool, stream)

    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    n0 = stq.stq_launch_count()
    sampler = ClockSampler(dev)
    with sampler, torch.cuda.nvtx.range("bench: timed decode steps"):
        for i in range(args.steps):
            flush.zero_()
            starts[i].record(stream)
            step(args.warmup + i)
            ends[i].record(stream)
        torch.cuda.synchronize()
    launches = stq.stq_launch_count() - n0
    if dist:
        dist.barrier()
    stq.stq_pool_check(pool, stream)
    times = [s.elapsed_time(e) for s, e in zip(starts, ends)]  # ms
    total_ms = max_over_ranks(float(sum(times)), dist, "cuda")
    units = wl.R * wl.H
    value = world * units * args.steps / (total_ms * 1e-3)
    ms_per_step = total_ms / args.steps

    bytes_per_launch, mean_bits = workload_info(wl)
    kernel_s = statistics.mean(times) * 1e-3
    peak, peak_kind = peaks()
    achieved = bytes_per_launch / kernel_s / 1e9
    traffic = None if args.kda_allocated else recorded_traffic(args.config, wl.R)

    # ---- end to end through the public API: one pinned host block of inputs in,
    # y out, through stq_decode_step_host_block (its input copy and the decode,
    # whose kernels write the pinned y across the bus, are in the timed interval)
    e2e = None
    if args.e2e_steps > 0:
        n = wl.R
        offs, nbytes = stq.stq_host_block_layout(pool, n)
        blocks = []
        for t in range(min(ntok, 16)):
            blk = torch.zeros(nbytes, dtype=torch.uint8).pin_memory()
            raw = blk.numpy()
            parts = [req.cpu().numpy(), slot.cpu().numpy()] + [toks[t][k].cpu().numpy()
                                                               for k in ("q", "k", "v", "beta", "gate")]
            for o, a in zip(offs, parts):
                b = np.ascontiguousarray(a).view(np.uint8).reshape(-1)
                raw[o: o + b.size] = b
            blocks.append(blk)
        y_host = torch.empty(y.shape, dtype=y.dtype).pin_memory()
        h2d = nbytes
        d2h = y.numel() * y.element_size()

        def host_step(i):
            stq.stq_decode_step_host_block(pool, n, blocks[i % len(blocks)], y_host, stream)

        for i in range(args.warmup):
            host_step(i)
        e_s = [torch.cuda.Event(enable_timing=True) for _ in range(args.e2e_steps)]
        e_e = [torch.cuda.Event(enable_timing=True) for _ in range(args.e2e_steps)]
        if dist:
            dist.barrier()
        torch.cuda.synchronize()
        for i in range(args.e2e_steps):
            flush.zero_()
            e_s[i].record(stream)
            host_step(i)
            e_e[i].record(stream)
        torch.cuda.synchronize()
        e_ms = max_over_ranks(float(sum(s.elapsed_time(e) for s, e in zip(e_s, e_e))), dist, "cuda")
        stq.stq_pool_check(pool, stream)
        # the box's pinned copy rates for the same byte counts (plain copies, no decode)
        h2d_s, d2h_s = copy_rates(torch, blocks[0], y_host, stream)
        step_s = e_ms * 1e-3 / args.e2e_steps
        e2e = {"value": world * units * args.e2e_steps / (e_ms * 1e-3), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "api": "stq_decode_step_host_block (one pinned host block copied in; "
                      "the kernels write the pinned y across the bus)",
               "ms_per_step": step_s * 1e3,
               "pinned_h2d_gbs": h2d / h2d_s / 1e9, "pinned_d2h_gbs": d2h / d2h_s / 1e9,
               "h2d_plus_kernel_ms": (h2d_s + kernel_s) * 1e3,
               "copies_plus_kernel_ms": (h2d_s + d2h_s + kernel_s) * 1e3}

    sweep = None
    if rank == 0 and world == 1 and not args.no_sweep:
        with torch.cuda.nvtx.range("bench: pool sweep"):
            sweep = pool_sweep(stq, flush, stream, peak)
    kda = None
    if rank == 0 and world == 1 and not args.no_sweep:
        with torch.cuda.nvtx.range("bench: KDA variants"):
            kda = kda_variants(stq, flush, stream, peak)
    gpiv = None
    if rank == 0 and world == 1 and not args.no_sweep:
        with torch.cuda.nvtx.range("bench: GDN pivot heads"):
            gpiv = gdn_pivot_heads(stq, flush, stream, peak)
    loop = None
    if rank == 0 and world == 1 and not args.no_layer_loop:
        with torch.cuda.nvtx.range("bench: layer loop"):
            loop = layer_loop(stq, flush)
    drift_log = None
    if rank == 0 and world == 1 and not args.no_drift:
        with torch.cuda.nvtx.range("bench: drift"):
            drift_log = drift(stq)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not args.kda_allocated:
        v, threads, sample, v1 = oracle_baseline(args.config, args.seed, args.cpu_seconds)
        cpu = {"value": v, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": sample,
               "value_1core": v1}

    pool.close()
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": wl.name, "kind": "GDN" if wl.kind == synth.GDN else "KDA",
                   "requests_per_gpu": wl.R, "heads": wl.H, "d_k": 128, "d_v": 128,
                   "mean_bits": mean_bits, "slots": wl.S, "tokens_cycled": ntok,
                   "l2": "flushed before every timed step (384 MiB write, outside the timed interval)",
                   "parallelism": f"dp{world} (independent request shards)"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": traffic, "peak_kind": peak_kind,
                     "algorithmic_bytes_per_launch": bytes_per_launch, "kernel": DECODE_KERNEL,
                     "kernel_us": kernel_s * 1e6},
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": launches,
        "clocks": sampler.summary(),
        # the supplementary records, rounded, the steady-state serving-pool sweep last
        "drift": compact(drift_log),
        "layer_loop": compact(loop),
        "kda_variants": compact(kda),
        "gdn_pivot_heads": compact(gpiv),
        "pool_sweep": compact(sweep),
    }
    print(json.dumps(line), flush=True)


def compact(obj, digits: int = 4):
    """obj with every float rounded to `digits` significant digits (short JSON)."""
    if isinstance(obj, float):
        return float(f"{obj:.{digits}g}")
    if isinstance(obj, dict):
        return {k: compact(v, digits) for k, v in obj.items()}
    if isinstance(obj, list):
        return [compact(v, digits) for v in obj]
    return obj


def copy_rates(torch, host_in, host_out, stream, reps: int = 20):
    """Median seconds of one pinned host-to-device copy of `host_in` and one
    device-to-host copy into `host_out` (plain copies on `stream`)."""
    dev_in = torch.empty(host_in.shape, dtype=host_in.dtype, device="cuda")
    dev_out = torch.empty(host_out.shape, dtype=host_out.dtype, device="cuda")
    out = []
    for src, dst in ((host_in, dev_in), (dev_out, host_out)):
        ts = []
        for i in range(reps + 3):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            dst.copy_(src, non_blocking=True)
            b.record(stream)
            if i >= 3:
                ts.append((a, b))
        torch.cuda.synchronize()
        out.append(statistics.median(a.elapsed_time(b) for a, b in ts) * 1e-3)
    return out[0], out[1]


def pool_sweep(stq, flush, stream, peak, reps: int = 20):
    """Serving-pool sweep: R requests x 5 slots x 768 heads (48 layers x 16
    heads), one token per launch over all heads; median kernel time over
    `reps` launches with the L2 flushed before each.  Each R runs the mixed
    6-bit GDN pool, and the same shape with an unquantized fp32 state (the
    page's FP32 control) and a binary16 state; fp32_over_quant is the
    state-update speedup of the quantized pool over the fp32 one."""
    import torch
    out = []
    for R in (16, 32, 64, 128, 256):
        wl = synth.make_workload(4, R=R)
        req = torch.arange(wl.R, dtype=torch.int32, device="cuda")
        slot = torch.from_numpy(wl.slot_of_request.astype(np.int32)).cuda()
        x = {k: torch.from_numpy(v).cuda() for k, v in wl.step_inputs(0).items()}
        y = torch.empty((wl.R, wl.H, 128), dtype=torch.float32, device="cuda")
        row = {"requests": R, "heads": wl.H}
        for tag, bits, sb in (("quant", wl.unit_bits, 4), ("fp32", np.full(wl.H, 32, np.uint8), 0),
                              ("fp16", np.full(wl.H, 16, np.uint8), 0)):
            if tag == "quant":
                pool = stq.stq_pool_create(wl.kind, wl.R, wl.S, wl.H, bits, wl.row_factor, wl.col_factor)
            else:
                pool = stq.stq_pool_create(wl.kind, wl.R, wl.S, wl.H, bits)
            ts = []
            for i in range(reps + 3):
                flush.zero_()
                s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                s.record(stream)
                stq.stq_decode_step(pool, req, slot, x["q"], x["k"], x["v"], x["beta"], x["gate"], y, stream)
                e.record(stream)
                if i >= 3:
                    ts.append((s, e))
            torch.cuda.synchronize()
            stq.stq_pool_check(pool, stream)
            med = statistics.median(s.elapsed_time(e) for s, e in ts) * 1e-3
            nbytes, _ = workload_info(wl, bits, sb)
            packed, _ = stq.stq_pool_bytes(pool)
            pool.close()
            torch.cuda.empty_cache()
            if tag == "quant":
                row.update({"pool_gb": packed / 1e9, "touched_gb": nbytes / 1e9, "kernel_us": med * 1e6,
                            "head_steps_per_s": wl.R * wl.H / med, "gbs": nbytes / med / 1e9,
                            "frac": nbytes / med / 1e9 / peak})
            else:
                row.update({f"{tag}_pool_gb": packed / 1e9, f"{tag}_kernel_us": med * 1e6,
                            f"{tag}_frac": nbytes / med / 1e9 / peak})
        row["fp32_over_quant"] = row["fp32_kernel_us"] / row["kernel_us"]
        out.append(row)
        del x, y
        torch.cuda.empty_cache()
    return out


def kda_allocated_bits(stq, H: int, seed: int, pivots: int = 8):
    """Per-row widths of H KDA heads from the lifetime-aware allocator: a 6-bit budget
    over {4, 6, 8} per head (Lagrangian) on synthetic calibration statistics (row
    distortion d_u(b) ~ logU(e^-2, e^2) 4^-k, mean log retention of U(0.8, 0.9995) decays,
    horizon 8192), then the head's `pivots` riskiest rows kept as FP16 pivots."""
    out = []
    for h in range(H):
        d0 = synth.log_uniform(synth.stream_key(seed, 90, 1, h), 128, np.exp(-2.0), np.exp(2.0))
        dist = d0[:, None] * 4.0 ** (-np.arange(3)[None, :])
        keep = 0.8 + (0.9995 - 0.8) * synth.uniform(synth.stream_key(seed, 90, 2, h), 128)
        w = stq.stq_lifetime_weight(np.log(keep), 8192)
        bits, _ = stq.stq_allocate_bits(np.full(128, 128.0), [4, 6, 8], dist, w, 6.0,
                                        method=stq.STQ_ALLOC_LAGRANGE, num_pivots=pivots, pivot_bits=16)
        out.append(bits)
    return np.concatenate(out)


def kda_variants(stq, flush, stream, peak, reps: int = 20):
    """KDA 128 requests x 32 heads, one token per launch (median over `reps`
    launches, L2 flushed before each, from the zero state after 3 warm-up steps):
    the workload's 32/64/32 rows per head at 4/6/8 bits; widths from the
    lifetime-aware allocator with 8 FP16 pivot rows per head; and those widths
    with column factors refitted every step (the page's KDA setting: pivot
    rows, fit over the non-pivot rows)."""
    import dataclasses
    import torch
    wl = synth.make_workload(3)
    alloc = kda_allocated_bits(stq, wl.H, 0)
    rw = synth.log_uniform(synth.stream_key(0, 90, 3), wl.H * 128, 0.5, 2.0).astype(np.float32)
    req = torch.arange(wl.R, dtype=torch.int32, device="cuda")
    slot = torch.zeros(wl.R, dtype=torch.int32, device="cuda")
    x = {k: torch.from_numpy(v).cuda() for k, v in wl.step_inputs(0).items()}
    y = torch.empty((wl.R, wl.H, 128), dtype=torch.float32, device="cuda")
    out = {"requests": wl.R, "heads": wl.H, "mean_bits_allocated": float(alloc.astype(np.float64).mean())}
    for tag, bits, flags in (("rows_32_64_32", wl.unit_bits, 0), ("allocated_pivots", alloc, 0),
                             ("allocated_pivots_fit", alloc, stq.STQ_FIT_COLUMNS)):
        pool = stq.stq_pool_create(wl.kind, wl.R, wl.S, wl.H, bits, wl.row_factor, wl.col_factor,
                                   flags=flags, row_weight=rw if flags else None)
        ts = []
        for i in range(reps + 3):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            stq.stq_decode_step(pool, req, slot, x["q"], x["k"], x["v"], x["beta"], x["gate"], y, stream)
            b.record(stream)
            if i >= 3:
                ts.append((a, b))
        torch.cuda.synchronize()
        stq.stq_pool_check(pool, stream)
        med = statistics.median(a.elapsed_time(b) for a, b in ts) * 1e-3
        nbytes, _ = workload_info(dataclasses.replace(wl, unit_bits=np.asarray(bits)))
        if flags:
            nbytes += wl.R * wl.H * 2 * 512  # the page's own column factors, read and written
        out[tag] = {"kernel_us": med * 1e6, "head_steps_per_s": wl.R * wl.H / med,
                    "gbs": nbytes / med / 1e9, "frac": nbytes / med / 1e9 / peak}
        pool.close()
    torch.cuda.empty_cache()
    return out


def gdn_pivot_heads(stq, flush, stream, peak, R: int = 64, pivots: int = 11, reps: int = 20):
    """The serving pool (R requests x 5 slots x 768 heads, mixed 6-bit GDN) with
    `pivots` heads held in FP16 (the page keeps 32 of 2304 GDN heads so: 11 of 768),
    one token per step over all heads (the fused kernel, then the pivot heads'
    kernel); median over `reps` steps with the L2 flushed before each, against the
    same pool without pivot heads."""
    import dataclasses
    import torch
    wl = synth.make_workload(4, R=R)
    piv = wl.unit_bits.copy()
    piv[np.linspace(0, wl.H - 1, pivots).astype(int)] = 16
    req = torch.arange(wl.R, dtype=torch.int32, device="cuda")
    slot = torch.from_numpy(wl.slot_of_request.astype(np.int32)).cuda()
    x = {k: torch.from_numpy(v).cuda() for k, v in wl.step_inputs(0).items()}
    y = torch.empty((wl.R, wl.H, 128), dtype=torch.float32, device="cuda")
    out = {"requests": R, "slots": wl.S, "heads": wl.H, "pivot_heads": pivots}
    for tag, bits in (("without", wl.unit_bits), ("with", piv)):
        w = dataclasses.replace(wl, unit_bits=bits)
        pool = stq.stq_pool_create(w.kind, w.R, w.S, w.H, bits, w.row_factor, w.col_factor)
        S0 = w.initial_state()
        if S0 is not None:
            stq.stq_quantize_state(pool, req, slot, torch.from_numpy(S0).cuda())
            del S0
        ts = []
        for i in range(reps + 3):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            stq.stq_decode_step(pool, req, slot, x["q"], x["k"], x["v"], x["beta"], x["gate"], y, stream)
            b.record(stream)
            if i >= 3:
                ts.append((a, b))
        torch.cuda.synchronize()
        stq.stq_pool_check(pool, stream)
        med = statistics.median(a.elapsed_time(b) for a, b in ts) * 1e-3
        nbytes, _ = workload_info(w)
        out[tag] = {"step_us": med * 1e6, "head_steps_per_s": R * wl.H / med, "gbs": nbytes / med / 1e9,
                    "frac": nbytes / med / 1e9 / peak}
        pool.close()
        torch.cuda.empty_cache()
    return out


def layer_loop(stq, flush, layers: int = 48, R: int = 64, reps: int = 20):
    """Per-layer serving loop: one pool per layer (R requests x 5 slots x 16
    heads, mixed 6-bit GDN), one token through all layers, each variant
    captured in one CUDA graph and replayed with the L2 flushed before each
    replay.  fused: one decode launch per layer.  split: per layer the readout
    on the main stream and the write-back on a side stream, joined at the end.
    readout_only: the main-stream half alone (pages unchanged), the path that
    gates the next layer when the write-backs overlap other work.
    The *_gemm variants add, after each layer's decode (fused) or readout
    (split) on the main stream, a stand-in for the rest of the layer: a bf16
    projection [R, 5120] x [5120, 5120] with its own weights per layer (read
    from HBM, as decode-time projections are); gemm_only is that work alone.
    split_gemm below fused_gemm means the side-stream write-backs are hidden
    behind it."""
    import torch
    wls = [synth.make_workload(4, R=R, H=16, seed=l) for l in range(layers)]
    pools, idx, xs, ys, us = [], [], [], [], []
    for w in wls:
        p = stq.stq_pool_create(w.kind, w.R, w.S, w.H, w.unit_bits, w.row_factor, w.col_factor)
        pools.append(p)
        idx.append((torch.arange(w.R, dtype=torch.int32, device="cuda"),
                    torch.from_numpy(w.slot_of_request.astype(np.int32)).cuda()))
        inp = w.step_inputs(0)
        xs.append([torch.from_numpy(inp[k]).cuda() for k in ("q", "k", "v", "beta", "gate")])
        ys.append(torch.empty((w.R, w.H, 128), dtype=torch.float32, device="cuda"))
        us.append(torch.empty((w.R, w.H, 128), dtype=torch.float32, device="cuda"))
    main, side = torch.cuda.Stream(), torch.cuda.Stream()
    hidden = 5120
    act = torch.randn((R, hidden), dtype=torch.bfloat16, device="cuda")
    weights = [torch.randn((hidden, hidden), dtype=torch.bfloat16, device="cuda") * 0.01 for _ in range(layers)]
    proj = torch.empty((R, hidden), dtype=torch.bfloat16, device="cuda")

    def body(kind):
        for l in range(layers):
            if kind.startswith("fused"):
                stq.stq_decode_step(pools[l], *idx[l], *xs[l], ys[l], main)
            elif kind.startswith("split"):
                stq.stq_decode_step_split(pools[l], *idx[l], *xs[l], ys[l], us[l], main, side)
            elif kind == "readout_only":
                stq.stq_decode_readout(pools[l], *idx[l], *xs[l], ys[l], us[l], main)
            if "gemm" in kind:
                torch.mm(act, weights[l], out=proj)
        if kind.startswith("split"):
            for p in pools:
                stq.stq_pool_join(p, main)

    out = {"layers": layers, "heads_per_layer": 16, "requests": R, "slots": 5,
           "gemm": f"bf16 [{R}, {hidden}] x [{hidden}, {hidden}] per layer"}
    for kind in ("fused", "split", "readout_only", "gemm_only", "fused_gemm", "split_gemm"):
        torch.cuda.synchronize()
        with torch.cuda.stream(main):
            body(kind)  # eager warm-up (sets the kernels' shared-memory attributes)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(main):
            side.wait_stream(main)
            g.capture_begin()
            body(kind)
            g.capture_end()
        ts = []
        for i in range(reps + 3):
            with torch.cuda.stream(main):
                flush.zero_()
                s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                s.record(main)
                g.replay()
                e.record(main)
            if i >= 3:
                ts.append((s, e))
        torch.cuda.synchronize()
        med = statistics.median(s.elapsed_time(e) for s, e in ts) * 1e-3
        out[f"{kind}_graph_us"] = med * 1e6
        out[f"{kind}_head_steps_per_s"] = layers * R * 16 / med
        del g
    out["split_gemm_over_fused_gemm"] = out["split_gemm_graph_us"] / out["fused_gemm_graph_us"]
    for p in pools:
        stq.stq_pool_check(p)
        p.close()
    del weights
    torch.cuda.empty_cache()
    return out


def drift(stq, steps: int = 8192, every: int = 512, tokens: int = 256):
    """Long-generation drift: 32 requests x 32 heads, alpha ~ U(0.95, 0.9999),
    GDN at INT4 / INT6 / INT8 and KDA at 6-bit mixed widths (decay per row in
    the same range), each advanced `steps` tokens next to the unquantized fp32
    recurrence (a raw fp32 pool) on the same inputs.  Every `every` steps the
    relative state error ||S^ - S||_F / ||S||_F and readout error
    ||y^ - y|| / ||y|| per (request, head) are taken; the record keeps, per
    case, the mean and max of the last checkpoint, the largest mean and max
    over all checkpoints, and (KDA) the last checkpoint's mean state error
    over the rows of each width.  The inputs of `tokens` distinct steps are
    cycled (a periodic input after the first `tokens` steps)."""
    import dataclasses
    import torch
    cases = [(f"gdn_int{b}", synth.make_workload(5, bits=b)) for b in (4, 6, 8)]
    kda = synth.make_workload(3, R=32, H=32)
    cases.append(("kda_mixed6", dataclasses.replace(kda, decay_range=(0.95, 0.9999), name="drift_kda_mixed6")))
    out = {"steps": steps, "every": every, "tokens_cycled": tokens, "requests": 32, "heads": 32, "cases": {}}
    for name, wl in cases:
        n_units = wl.H if wl.kind == synth.GDN else wl.H * 128
        ctl = dataclasses.replace(wl, unit_bits=np.full(n_units, 32, np.uint8))
        pq = stq.stq_pool_create(wl.kind, wl.R, wl.S, wl.H, wl.unit_bits, wl.row_factor, wl.col_factor)
        pf = stq.stq_pool_create(ctl.kind, ctl.R, ctl.S, ctl.H, ctl.unit_bits)
        req = torch.arange(wl.R, dtype=torch.int32, device="cuda")
        slot = torch.zeros(wl.R, dtype=torch.int32, device="cuda")
        xs = []
        for t in range(tokens):
            inp = wl.step_inputs(t)
            xs.append([torch.from_numpy(inp[k]).cuda() for k in ("q", "k", "v", "beta", "gate")])
        yq = torch.empty((wl.R, wl.H, 128), dtype=torch.float32, device="cuda")
        yf = torch.empty_like(yq)
        Sq = torch.empty((wl.R, wl.H, 128, 128), dtype=torch.float32, device="cuda")
        Sf = torch.empty_like(Sq)
        width = torch.from_numpy(wl.row_bits().astype(np.int64)).cuda()  # [H, 128]
        es_mean, es_max, ey_mean, ey_max = [], [], [], []
        by_width = {}
        for t in range(steps):
            x = xs[t % tokens]
            stq.stq_decode_step(pq, req, slot, *x, yq)
            stq.stq_decode_step(pf, req, slot, *x, yf)
            if (t + 1) % every == 0:
                stq.stq_dequantize_state(pq, req, slot, Sq)
                stq.stq_dequantize_state(pf, req, slot, Sf)
                es = (torch.linalg.vector_norm(Sq - Sf, dim=(2, 3)) /
                      torch.linalg.vector_norm(Sf, dim=(2, 3)).clamp_min(1e-30))
                ey = torch.linalg.vector_norm(yq - yf, dim=2) / torch.linalg.vector_norm(yf, dim=2).clamp_min(1e-30)
                es_mean.append(float(es.mean()))
                es_max.append(float(es.max()))
                ey_mean.append(float(ey.mean()))
                ey_max.append(float(ey.max()))
                if wl.kind == synth.KDA and t + 1 == steps:
                    d2 = ((Sq - Sf) ** 2).sum(dim=3)  # [R, H, 128] per row
                    f2 = (Sf ** 2).sum(dim=3)
                    for b in (4, 6, 8):
                        m = (width == b).unsqueeze(0)
                        num = (d2 * m).sum(dim=2).sqrt()
                        den = (f2 * m).sum(dim=2).sqrt().clamp_min(1e-30)
                        by_width[str(b)] = float((num / den).mean())
        stq.stq_pool_check(pq)
        stq.stq_pool_check(pf)
        rec = {"state_rel_err_mean": es_mean[-1], "state_rel_err_max": es_max[-1],
               "y_rel_err_mean": ey_mean[-1], "y_rel_err_max": ey_max[-1],
               "state_rel_err_mean_peak": max(es_mean), "state_rel_err_max_peak": max(es_max),
               "y_rel_err_max_peak": max(ey_max), "checkpoints": len(es_mean)}
        if by_width:
            rec["state_rel_err_mean_by_row_width"] = by_width
        out["cases"][name] = rec
        pq.close()
        pf.close()
        del xs, Sq, Sf
        torch.cuda.empty_cache()
    return out


def main():
    args = parse()
    rank, world = rank_world(args)
    if args.impl == "reference":
        run_reference(args, rank, world)
    else:
        run_ours(args, rank, world)


if __name__ == "__main__":
    main()

#!/usr/bin/env python
"""Throughput of the fused attention forward on B200.

One step = one call of the fused forward (the whole hot path) over one batch of
synthetic input of the headline workload: B=4, H=16, N=8192, d=128, causal,
scale 1/sqrt(d), bf16 inputs drawn from N(0,1) (seed 2).  The metric is forward
TFLOP/s with FLOPs = 4*B*H*N^2*d / 2 (causal), inputs resident in HBM.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...      # the fp64 CPU oracle, timed

With N > 1 (``--gpus N`` starts N ranks through torch.distributed.run unless
it already runs under it) the heads are split over the ranks: by default each
rank runs one batch block of an N-times larger problem (block r seeded with
seed + 1000*r; weak scaling), with ``--scaling strong`` the workload's own heads
are split into contiguous ranges.  Heads are independent, so there is no
data-path collective; ``--gather`` also times an NCCL all-gather of O and LSE.
Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from exact_attention_127_b200 import inputs as _inputs  # noqa: E402

METRIC = "attention fwd TFLOP/s and % of B200 dense BF16 peak (causal N=8192 d=128)"
UNIT = "TFLOP/s"
DATASHEET_BF16_TFLOPS = 2250.0
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
KERNEL_NAME = "attn_fwd_sm100_kernel"
SRC = os.path.join(ROOT, "exact_attention_127_b200", "csrc", "attn_fwd_sm100.cu")
DECODE_SRC = os.path.join(ROOT, "exact_attention_127_b200", "csrc", "attn_decode.cuh")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "attn_fwd_traffic.json")
L2_BYTES = 126 * 1024 * 1024


# ---------------------------------------------------------------------------
# Host-side helpers (unit-tested on CPU)
# ---------------------------------------------------------------------------
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    return rank, local, world


def rank_seed(seed: int, rank: int) -> int:
    """Each rank draws its own independent batch of the same shape."""
    return int(seed) + 1000 * int(rank)


def aggregate_value(flops_per_rank: float, world: int, ms_max: float) -> float:
    """Whole-job TFLOP/s: all ranks' useful FLOPs over the slowest rank's time."""
    return flops_per_rank * world / (ms_max * 1e-3) / 1e12


def reduce_max(values, device):
    """Element-wise max over ranks of a few timings (identity on one rank)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(x) for x in values]
    t = torch.tensor([float(x) for x in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK), "fallback"


def source_digest() -> str:
    """sha256 of the forward kernel's device code: the part of the source file
    before its host-side section (device helpers, the schedule, the kernel).
    DRAM traffic depends on that code only; host-side changes (argument checks,
    the host-buffer entry point) do not invalidate a capture."""
    with open(SRC, "rb") as f:
        text = f.read()
    cut = text.find(b"/* Host side: validation, tensor maps, launch")
    return hashlib.sha256(text[:cut] if cut >= 0 else text).hexdigest()


def decode_source_digest() -> str:
    """sha256 of the decode kernels' source file."""
    with open(DECODE_SRC, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()


def load_traffic(workload: str, section: str | None = None):
    """DRAM bytes per launch from a committed ncu capture, or None when the
    capture is missing, for another workload, or taken on older kernel source.
    section=None reads the forward kernel's record; "decode" reads the decode
    stream kernel's, which carries the digest of its own source file."""
    try:
        with open(TRAFFIC_FILE) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    if section is not None:
        rec = rec.get(section, {})
        digest = decode_source_digest()
    else:
        digest = source_digest()
    if rec.get("kernel_source_sha256") != digest:
        return None
    per = rec.get("per_launch_dram_bytes", {})
    val = per.get(workload)
    return float(val) if val is not None else None


REASON_BITS = {
    0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
    0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
    0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
    0x100: "display_clock_setting",
}


def decode_reasons(mask: int):
    return [name for bit, name in sorted(REASON_BITS.items()) if mask & bit]


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""

    def __init__(self, device_index: int, period_s: float = 0.01):
        self.samples = []
        self.max_mhz = None
        self._stop = threading.Event()
        self._period = period_s
        self._thread = None
        self._ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._ok = True
        except Exception as e:  # noqa: BLE001
            self.error = repr(e)

    def _sample(self):
        nv = self._nv
        sm = nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM)
        try:
            reasons = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
        except AttributeError:
            reasons = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self._h)
        self.samples.append((time.time(), sm, int(reasons)))

    def _run(self):
        while not self._stop.is_set():
            try:
                self._sample()
            except Exception:  # noqa: BLE001
                pass
            self._stop.wait(self._period)

    def start(self):
        if self._ok:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()

    def stop(self):
        if self._thread:
            self._stop.set()
            self._thread.join()
            try:
                self._sample()
            except Exception:  # noqa: BLE001
                pass

    def summary(self):
        if not self._ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [],
                    "samples": 0, "note": getattr(self, "error", "no samples")}
        mhz = [s[1] for s in self.samples]
        mask = 0
        for s in self.samples:
            mask |= s[2]
        reasons = [r for r in decode_reasons(mask) if r != "gpu_idle"]
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": self.max_mhz,
                "sm_mhz_min": min(mhz), "reasons": reasons, "samples": len(mhz)}


# ---------------------------------------------------------------------------
# CPU baseline: the fp64 oracle as it stands, on a bounded sample
# ---------------------------------------------------------------------------
def oracle_sample_flops(w, rows, n_heads):
    """Useful FLOPs of the sampled rows: 4*d per allowed key per row."""
    keys = sum((int(r) + 1) if w.causal else w.N for r in rows)
    return 4.0 * w.d * keys * n_heads


def time_oracle(w, q, k, v, target_s: float, max_heads: int = 16):
    """Time the oracle on sampled query rows of the first few heads, growing the
    row sample until one evaluation takes about target_s seconds (bounded by
    N rows per head).  Returns a dict (value in the bench's unit)."""
    import oracle
    nthreads = oracle.default_threads()
    heads = list(range(min(max_heads, w.B * w.H)))
    count = 4
    while True:
        rows = _inputs.sample_rows(w.N, count, w.seed)
        t0 = time.perf_counter()
        oracle.attention_rows(q, k, v, w.causal, w.scale, rows=rows, heads=heads,
                              nthreads=nthreads)
        dt = time.perf_counter() - t0
        if dt >= 0.5 * target_s or count >= w.N:
            break
        grow = max(2.0, min(16.0, target_s / max(dt, 1e-3)))
        count = min(w.N, int(count * grow))
    flops = oracle_sample_flops(w, rows, len(heads))
    return {"value": flops / dt / 1e12, "unit": UNIT, "cores": nthreads, "kind": "oracle",
            "seconds": dt, "rows": rows, "heads": heads,
            "sample": f"{len(rows)} query rows (boundary rows + seeded uniform draws) x "
                      f"{len(heads)} heads of {w.name}; FLOPs = 4*d*(allowed keys) per row; "
                      f"includes widening the heads' bf16 inputs to fp64"}


# ---------------------------------------------------------------------------
# Arms
# ---------------------------------------------------------------------------
def run_reference(args, w):
    """The oracle as it stands, timed on the host cores: every step evaluates a
    fixed sample of query rows, sized so the whole run ends within minutes."""
    rank, _, world = dist_env()
    if rank != 0:
        return 0
    import oracle
    q, k, v = _inputs.workload_inputs(w)
    per_step = min(args.ref_step_seconds, args.ref_budget_seconds / (args.steps + args.warmup))
    probe = time_oracle(w, q, k, v, target_s=per_step, max_heads=4)   # sizes the sample
    rows, heads, nthreads = probe.pop("rows"), probe.pop("heads"), probe["cores"]
    flops = oracle_sample_flops(w, rows, len(heads))
    for _ in range(max(0, args.warmup - 1)):
        oracle.attention_rows(q, k, v, w.causal, w.scale, rows=rows, heads=heads,
                              nthreads=nthreads)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle.attention_rows(q, k, v, w.causal, w.scale, rows=rows, heads=heads,
                              nthreads=nthreads)
        times.append(time.perf_counter() - t0)
    ms = 1e3 * sum(times) / len(times)
    value = flops / (ms * 1e-3) / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(w, world),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": nthreads, "kind": "oracle",
                         "sample": probe["sample"] + " per step"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def config_of(w, world, scaling="weak"):
    BH = w.B * w.H
    if world > 1 and scaling == "weak":
        per_rank = (f"global problem [{world * w.B}, {w.H}, {w.N}, {w.d}]: rank r runs heads "
                    f"[r*{BH}, (r+1)*{BH}) (batch block r, seed + 1000*r)")
    elif world > 1:
        per_rank = (f"global problem [{w.B}, {w.H}, {w.N}, {w.d}] (seed {w.seed}): rank r runs a "
                    f"contiguous range of about {BH / world:.1f} of its {BH} heads")
    else:
        per_rank = "all heads on one GPU"
    return {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d, "causal": w.causal,
            "scale": w.scale, "seed": w.seed, "inputs": "bf16; " + (
                "Q,K ~ N(0,16), V ~ U(-1,1)" if w.v_dist == "uniform" else "Q,K,V ~ N(0,1)"),
            "per_rank": per_rank,
            "parallelism": f"heads split over {world} GPUs" if world > 1 else "single GPU",
            "l2": ("inputs larger than L2 (q,k,v %.0f MB per step)" % (
                3 * 2 * w.B * w.H * w.N * w.d / 1e6))
            if 3 * 2 * w.B * w.H * w.N * w.d > L2_BYTES else "L2 flushed between steps"}


def rank_inputs(w, world, rank, scaling):
    """This rank's q, k, v head slices ([count, N, d] CPU bf16) and the global
    head count.  weak: the global problem is `world` batch blocks of the
    workload, block r seeded with seed + 1000*r, and rank r owns block r.
    strong: the global problem is the workload itself, split by head_range."""
    from exact_attention_127_b200 import shard
    if scaling == "weak" or world == 1:
        q, k, v = _inputs.make_qkv(w.B, w.H, w.N, w.d, rank_seed(w.seed, rank), w.qk_std,
                                   w.v_dist)
        flat = [t.reshape(w.B * w.H, w.N, w.d) for t in (q, k, v)]
        return flat, w.B * w.H * world
    q, k, v = _inputs.workload_inputs(w)
    return [shard.head_slice(t, world, rank).clone() for t in (q, k, v)], w.B * w.H


def run_cuda(args, w):
    import torch
    import torch.distributed as dist

    import exact_attention_127_b200 as attn
    from exact_attention_127_b200 import shard

    rank, local, world = dist_env()
    if world > 1 and torch.cuda.device_count() < world:
        raise SystemExit(f"{world} ranks need {world} visible GPUs; "
                         f"found {torch.cuda.device_count()}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    attn.load_library()

    (q, k, v), n_heads = rank_inputs(w, world, rank, args.scaling)
    count = q.shape[0]
    qd, kd, vd = (t.to(dev) for t in (q, k, v))
    o = torch.empty_like(qd)
    lse = torch.empty((count, w.N), dtype=torch.float32, device=dev)
    stream = torch.cuda.Stream(dev)
    flush = None
    big_enough = 3 * qd.numel() * 2 > L2_BYTES
    if not big_enough:
        flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)

    def fwd():
        if count:
            shard.attn_fwd_heads(qd, kd, vd, causal=w.causal, scale=w.scale, out=o, lse=lse,
                                 stream=stream)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            if flush is not None:
                flush.fill_(1.0)   # evict L2 between iterations
            fwd()
    stream.synchronize()
    if attn.device_status(reset=True, stream=stream) != 0:
        raise RuntimeError("kernel reported a device-side error during warm-up")

    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    sampler = ClockSampler(local)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    sampler.start()
    with torch.cuda.stream(stream):
        for i in range(args.steps):
            if flush is not None:
                flush.fill_(1.0)   # outside the events: a step is the forward call alone
            starts[i].record(stream)
            fwd()
            ends[i].record(stream)
    stream.synchronize()
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    sampler.stop()
    launches = args.steps if count else 0
    kernel_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    ms_kernel = sum(kernel_ms) / len(kernel_ms)
    if flush is None:
        ms_step = starts[0].elapsed_time(ends[-1]) / args.steps   # back-to-back steps
    else:
        ms_step = ms_kernel          # L2 flushed between steps: the steps' own time
    status = attn.device_status(reset=True, stream=stream)
    if status != 0:
        raise RuntimeError(f"kernel reported device status {status}")

    # ---- latency of one call (host call + launch + kernel), for launch-bound shapes
    lat_us = None
    if w.flops() < 1e9 and count:
        host = []
        for _ in range(args.latency_calls):
            t0 = time.perf_counter()
            fwd()
            stream.synchronize()
            host.append((time.perf_counter() - t0) * 1e6)
        lat_us = {"call_median_us": statistics.median(host),
                  "kernel_median_us": 1e3 * statistics.median(kernel_ms),
                  "calls": args.latency_calls,
                  "what": "host wall time of attn_fwd + stream synchronize, one call at a time"}
        # the same call captured once in a CUDA graph and replayed: the host work of
        # a call (checks, tensor maps, launch) is paid at capture only
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            shard.attn_fwd_heads(qd, kd, vd, causal=w.causal, scale=w.scale, out=o, lse=lse)
        cap = torch.cuda.current_stream()
        for _ in range(3):
            graph.replay()
        cap.synchronize()
        replay = []
        for _ in range(args.latency_calls):
            t0 = time.perf_counter()
            graph.replay()
            cap.synchronize()
            replay.append((time.perf_counter() - t0) * 1e6)
        lat_us["graph_replay_median_us"] = statistics.median(replay)
        lat_us["graph_what"] = "host wall time of CUDAGraph.replay() + synchronize of one captured attn_fwd"
        del graph

    # ---- optional gather of every rank's O and LSE onto all ranks (NCCL all-gather)
    gather = None
    if args.gather and world > 1:
        for _ in range(2):
            shard.gather_heads(o, lse, n_heads)
        torch.cuda.synchronize(dev)
        dist.barrier()
        g0 = torch.cuda.Event(enable_timing=True)
        g1 = torch.cuda.Event(enable_timing=True)
        g0.record()
        for _ in range(args.steps):
            o_all, lse_all = shard.gather_heads(o, lse, n_heads)
        g1.record()
        torch.cuda.synchronize(dev)
        (g_ms,) = reduce_max([g0.elapsed_time(g1) / args.steps], dev)
        nbytes = n_heads * w.N * (w.d * 2 + 4)
        gather = {"ms_per_step": g_ms, "bytes_gathered": nbytes,
                  "what": "NCCL all-gather of every rank's O and LSE slices, timed after the "
                          "forward steps; not part of value"}

    # ---- end to end: host (pinned) buffers through the C ABI host entry point
    e2e_ms, h2d, d2h = None, 0, 0
    if count:
        qp, kp, vp = (t.reshape(1, count, w.N, w.d).pin_memory() for t in (q, k, v))
        op = torch.empty(qp.shape, dtype=torch.bfloat16).pin_memory()
        lp = torch.empty((1, count, w.N), dtype=torch.float32).pin_memory()
        ws = torch.empty(attn.host_workspace_bytes(1, count, w.N, w.d), dtype=torch.uint8,
                         device=dev)
        e2e_steps = max(1, min(args.steps, args.e2e_steps))
        for _ in range(min(2, args.warmup)):
            attn.attn_fwd_host(qp, kp, vp, w.causal, w.scale, out=op, lse=lp, workspace=ws,
                               device=dev, stream=stream, synchronize=True)
        if world > 1:
            dist.barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(e2e_steps):
            attn.attn_fwd_host(qp, kp, vp, w.causal, w.scale, out=op, lse=lp, workspace=ws,
                               device=dev, stream=stream, synchronize=False)
        e1.record(stream)
        stream.synchronize()
        e2e_ms = e0.elapsed_time(e1) / e2e_steps
        h2d = 3 * qp.numel() * 2
        d2h = op.numel() * 2 + lp.numel() * 4
        if attn.device_status(reset=True, stream=stream) != 0:
            raise RuntimeError("kernel reported a device-side error in the e2e leg")
    elif world > 1:
        dist.barrier()
    if e2e_ms is None:
        e2e_ms = 0.0

    ms_max, kern_max, e2e_max = reduce_max([ms_step, ms_kernel, e2e_ms], dev)

    # useful FLOPs of every rank's heads (a head of the workload: flops / (B*H))
    flops_per_head = w.flops() / (w.B * w.H)
    total_flops = flops_per_head * n_heads
    value = total_flops / (ms_max * 1e-3) / 1e12
    line = None
    if rank == 0:
        peaks, peak_src = load_peaks()
        rank_flops = flops_per_head * count
        achieved = rank_flops / (kern_max * 1e-3) / 1e12
        traffic = load_traffic(w.name) if world == 1 else None
        clocks = sampler.summary()
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max,
            "higher_is_better": True, "scaling": args.scaling if world > 1 else "weak",
            "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic", "config": config_of(w, world, args.scaling),
            "roofline": {
                "bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "frac": achieved / peaks["bf16_tflops"],
                "traffic": traffic,
                "peak_source": f"{peak_src} bf16 dense matmul, burst (MEASURED_PEAKS.json)"
                if peak_src == "measured" else "fallback 1.59 PFLOP/s",
                "frac_of_sustained": achieved / peaks["bf16_tflops_sustained"],
                "frac_of_datasheet_2250": achieved / DATASHEET_BF16_TFLOPS,
                "kernel": KERNEL_NAME, "kernel_ms": kern_max,
                "algorithmic_flops_per_launch": rank_flops,
                "compulsory_bytes_per_launch": w.compulsory_bytes() * count // (w.B * w.H),
            },
            "e2e": {"value": total_flops / (e2e_max * 1e-3) / 1e12 if e2e_max else None,
                    "unit": UNIT, "ms_per_step": e2e_max,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "path": "attn_fwd_host (pinned host buffers; above 32 MB the copies in, kernels and copies out of up to 8 chunks of heads overlap on helper streams)"},
            "gpu_launches": launches,
            "clocks": clocks,
        }
        rank_bytes = w.compulsory_bytes() * count // (w.B * w.H)
        gbs = rank_bytes / (kern_max * 1e-3) / 1e9
        line["hbm"] = {"achieved_gbs": gbs, "peak_gbs": peaks["hbm_gbs"],
                       "frac": gbs / peaks["hbm_gbs"],
                       "what": "compulsory bytes (q, k, v read, o, lse written once) per launch "
                               "over the launch time"
                               + ("; L2 flushed before each launch" if flush is not None else
                                  "; inputs larger than L2")}
        if lat_us is not None:
            line["latency"] = lat_us
        if gather is not None:
            line["gather"] = gather
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        if world == 1 and not args.no_cpu_baseline:
            qf, kf, vf = (t.reshape(w.B, w.H, w.N, w.d) for t in (q, k, v))
            cpu = time_oracle(w, qf, kf, vf, target_s=args.cpu_seconds)
            cpu.pop("rows")
            cpu.pop("heads")
            line["cpu_baseline"] = cpu
        print(json.dumps(line), flush=True)
    return 0


DECODE_METRIC = "split-K/V decode attention GB/s (K/V cache bytes read / time)"


BWD_METRIC = "attention bwd TFLOP/s (2.5 x forward FLOPs: five GEMMs)"


def run_backward(args, w):
    """One step = one attn_bwd call (D/LSE preparation, the fused backward
    kernel, dQ conversion) on a forward workload; tensor-core bound."""
    import torch

    import exact_attention_127_b200 as attn

    rank, local, world = dist_env()
    if world > 1:
        raise SystemExit("--pass bwd runs on one GPU")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    attn.load_library()
    q, k, v = (t.to(dev) for t in _inputs.workload_inputs(w))
    dout = _inputs.make_qkv(w.B, w.H, w.N, w.d, w.seed + 100)[0].to(dev)
    o, lse = attn.attn_fwd(q, k, v, causal=w.causal, scale=w.scale)
    ws = torch.empty(attn.bwd_workspace_bytes(w.B, w.H, w.N, w.d), dtype=torch.uint8, device=dev)
    stream = torch.cuda.Stream(dev)
    torch.cuda.synchronize(dev)
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            attn.attn_bwd(q, k, v, o, lse, dout, w.causal, w.scale, workspace=ws, stream=stream)
    stream.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local)
    sampler.start()
    e0.record(stream)
    with torch.cuda.stream(stream):
        for _ in range(args.steps):
            attn.attn_bwd(q, k, v, o, lse, dout, w.causal, w.scale, workspace=ws, stream=stream)
    e1.record(stream)
    stream.synchronize()
    sampler.stop()
    if attn.device_status(reset=True, stream=stream) != 0:
        raise RuntimeError("device-side error in the backward pass")
    ms = e0.elapsed_time(e1) / args.steps
    flops = 2.5 * w.flops()
    peaks, peak_src = load_peaks()
    tf = flops / (ms * 1e-3) / 1e12
    line = {
        "metric": BWD_METRIC, "value": tf, "unit": UNIT, "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": config_of(w, 1),
        "roofline": {"bound": "tensor", "achieved": tf, "peak": peaks["bf16_tflops"],
                     "unit": "TFLOP/s", "frac": tf / peaks["bf16_tflops"], "traffic": None,
                     "peak_source": f"{peak_src} bf16 dense matmul, burst (MEASURED_PEAKS.json)",
                     "kernel": "bwd_pre_kernel + bwd_main_kernel + bwd_post_kernel",
                     "algorithmic_flops_per_launch": flops},
        "e2e": None, "gpu_launches": 3 * args.steps, "clocks": sampler.summary(),
    }
    print(json.dumps(line), flush=True)
    return 0


FP8_METRIC = "attention fwd TFLOP/s, e4m3 inputs (fp32 accumulate, e4m3 P)"
FP8_OVER_BF16 = 2.0   # nominal dense e4m3 : bf16 tensor rate (4.5 : 2.25 PFLOP/s)


def run_fp8(args, w):
    """One step = one attn_fwd_fp8 call (V transposed into the workspace, then
    the fused kernel on e4m3 operands) on a forward workload (d = 64 or 128)."""
    import torch

    import exact_attention_127_b200 as attn

    rank, local, world = dist_env()
    if world > 1:
        raise SystemExit("--dtype e4m3 runs on one GPU")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    attn.load_library()
    q8, k8, v8 = (t.to(dev) for t in _inputs.make_qkv_e4m3(w.B, w.H, w.N, w.d, seed=w.seed))
    o = torch.empty(q8.shape, dtype=torch.bfloat16, device=dev)
    lse = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device=dev)
    ws = torch.empty(attn.fp8_workspace_bytes(w.B, w.H, w.N, w.d), dtype=torch.uint8, device=dev)
    stream = torch.cuda.Stream(dev)
    torch.cuda.synchronize(dev)

    def step():
        attn.attn_fwd_fp8(q8, k8, v8, causal=w.causal, scale=w.scale, out=o, lse=lse,
                          workspace=ws, stream=stream)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            step()
    stream.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local)
    sampler.start()
    e0.record(stream)
    with torch.cuda.stream(stream):
        for _ in range(args.steps):
            step()
    e1.record(stream)
    stream.synchronize()
    sampler.stop()
    if attn.device_status(reset=True, stream=stream) != 0:
        raise RuntimeError("device-side error in the e4m3 forward")
    ms = e0.elapsed_time(e1) / args.steps
    flops = w.flops()
    peaks, peak_src = load_peaks()
    peak = FP8_OVER_BF16 * peaks["bf16_tflops"]
    tf = flops / (ms * 1e-3) / 1e12
    cfg = config_of(w, 1)
    cfg["inputs"] = "e4m3 (make_qkv's N(0,1) draws rounded to nearest), descales 1"
    line = {
        "metric": FP8_METRIC, "value": tf, "unit": UNIT, "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "e4m3", "data": "synthetic", "config": cfg,
        "roofline": {"bound": "tensor", "achieved": tf, "peak": peak, "unit": "TFLOP/s",
                     "frac": tf / peak, "traffic": None,
                     "peak_source": f"{peak_src} bf16 dense matmul, burst (MEASURED_PEAKS.json), "
                                    f"x {FP8_OVER_BF16:g} (nominal e4m3 : bf16 dense rate)",
                     "frac_of_bf16_peak": tf / peaks["bf16_tflops"],
                     "kernel": f"fp8_transpose_v_kernel + attn_fwd_sm100_kernel<{w.d}, causal, e4m3>",
                     "algorithmic_flops_per_launch": flops},
        "e2e": None, "gpu_launches": 2 * args.steps, "clocks": sampler.summary(),
    }
    print(json.dumps(line), flush=True)
    return 0


def run_standard(args, w):
    """The unfused three-kernel path on a forward workload (context for the
    fused kernel): same metric (useful TFLOP/s); its roofline is HBM, since the
    N x N matrices cross device memory four times."""
    import torch

    import exact_attention_127_b200 as attn

    rank, local, world = dist_env()
    if world > 1:
        raise SystemExit("--path standard runs on one GPU")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    attn.load_library()
    q, k, v = (t.to(dev) for t in _inputs.workload_inputs(w))
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device=dev)
    ws = torch.empty(attn.standard_workspace_bytes(w.B, w.H, w.N, w.d), dtype=torch.uint8,
                     device=dev)
    stream = torch.cuda.Stream(dev)
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            attn.attn_standard(q, k, v, w.causal, w.scale, out=o, lse=lse, workspace=ws,
                               stream=stream)
    stream.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local)
    sampler.start()
    e0.record(stream)
    with torch.cuda.stream(stream):
        for _ in range(args.steps):
            attn.attn_standard(q, k, v, w.causal, w.scale, out=o, lse=lse, workspace=ws,
                               stream=stream)
    e1.record(stream)
    stream.synchronize()
    sampler.stop()
    if attn.device_status(reset=True, stream=stream) != 0:
        raise RuntimeError("device-side error in the standard path")
    ms = e0.elapsed_time(e1) / args.steps
    Np = (w.N + 127) // 128 * 128
    nn_bytes = w.B * w.H * Np * Np * (4 + 4 + 2 + 2)    # S written+read (fp32), P written+read
    nbytes = nn_bytes + w.compulsory_bytes()
    peaks, peak_src = load_peaks()
    gbs = nbytes / (ms * 1e-3) / 1e9
    line = {
        "metric": METRIC, "value": w.flops() / (ms * 1e-3) / 1e12, "unit": UNIT, "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "path": "standard: S = scale*QK^T (fp32) -> HBM, softmax -> P (bf16) in place, O = PV",
        "config": config_of(w, 1),
        "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": gbs / peaks["hbm_gbs"], "traffic": None,
                     "algorithmic_bytes_per_launch": nbytes,
                     "peak_source": f"{peak_src} HBM copy (MEASURED_PEAKS.json)",
                     "kernel": "std_qk_kernel + std_softmax_kernel + std_pv_kernel"},
        "e2e": None, "gpu_launches": 3 * args.steps, "clocks": sampler.summary(),
    }
    print(json.dumps(line), flush=True)
    return 0


def run_decode(args, w):
    """One step = one attn_decode call (stream kernel + combine kernel) over a
    batch of one query row per head against N cached keys; HBM-bound."""
    import torch
    import torch.distributed as dist

    import exact_attention_127_b200 as attn

    rank, local, world = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    attn.load_library()
    q, k, v = _inputs.make_decode_qkv(w.B, w.H, w.N, w.d, rank_seed(w.seed, rank))
    qd, kd, vd = (t.to(dev) for t in (q, k, v))
    o = torch.empty_like(qd)
    lse = torch.empty((w.B, w.H), dtype=torch.float32, device=dev)
    ws = torch.empty(attn.decode_workspace_bytes(w.B, w.H, w.N, w.d), dtype=torch.uint8, device=dev)
    stream = torch.cuda.Stream(dev)
    flush = None
    if 2 * kd.numel() * 2 <= L2_BYTES:
        flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            attn.attn_decode(qd, kd, vd, scale=w.scale, out=o, lse=lse, workspace=ws, stream=stream)
    stream.synchronize()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    sampler = ClockSampler(local)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    sampler.start()
    with torch.cuda.stream(stream):
        for i in range(args.steps):
            if flush is not None:
                flush.fill_(1.0)
            starts[i].record(stream)
            attn.attn_decode(qd, kd, vd, scale=w.scale, out=o, lse=lse, workspace=ws, stream=stream)
            ends[i].record(stream)
    stream.synchronize()
    if world > 1:
        dist.barrier()
    sampler.stop()
    if attn.device_status(reset=True, stream=stream) != 0:
        raise RuntimeError("device-side error in the decode kernels")
    step_ms = sum(s.elapsed_time(e) for s, e in zip(starts, ends)) / args.steps
    (ms_max,) = reduce_max([step_ms], dev)
    nbytes = w.compulsory_bytes()
    value = nbytes * world / (ms_max * 1e-3) / 1e9
    line = None
    if rank == 0:
        peaks, peak_src = load_peaks()
        line = {
            "metric": DECODE_METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d,
                       "queries_per_head": 1, "scale": w.scale, "seed": w.seed,
                       "parallelism": f"dp{world}" if world > 1 else "single GPU",
                       "l2": "K/V cache larger than L2" if flush is None else "L2 flushed"},
            "roofline": {"bound": "hbm", "achieved": value / world, "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": value / world / peaks["hbm_gbs"],
                         "traffic": load_traffic(w.name, "decode"),
                         "traffic_kernel": "decode_stream_kernel",
                         "peak_source": f"{peak_src} HBM copy (MEASURED_PEAKS.json)",
                         "kernel": "decode_stream_kernel + decode_combine_kernel (one call)",
                         "compulsory_bytes_per_launch": nbytes},
            "e2e": None, "gpu_launches": 2 * args.steps, "clocks": sampler.summary(),
        }
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        if world == 1 and not args.no_cpu_baseline:
            import oracle
            heads = list(range(min(16, w.B * w.H)))
            t0 = time.perf_counter()
            oracle.attention_qk(q.reshape(w.B * w.H, 1, 1, w.d)[heads],
                                k.reshape(w.B * w.H, 1, w.N, w.d)[heads],
                                v.reshape(w.B * w.H, 1, w.N, w.d)[heads], w.scale)
            dt = time.perf_counter() - t0
            cpu_bytes = nbytes * len(heads) / (w.B * w.H)
            line["cpu_baseline"] = {"value": cpu_bytes / dt / 1e9, "unit": "GB/s",
                                    "cores": oracle.default_threads(), "kind": "oracle",
                                    "sample": f"{len(heads)} heads of {w.name}"}
        print(json.dumps(line), flush=True)
    return 0


def free_port() -> int:
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def relaunch(argv, n: int, limit_s: float = 3600.0) -> int:
    """`--gpus N` without a launcher: start N ranks of this script through
    torch.distributed.run on 127.0.0.1 and return their exit status.  The
    ranks' own process-group timeout ends a stuck collective; limit_s bounds
    the whole run as a last resort (the process group is killed)."""
    import signal
    import subprocess
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           f"--nproc-per-node={n}", "--master-addr", "127.0.0.1",
           "--master-port", str(free_port()), os.path.abspath(__file__), *argv]
    proc = subprocess.Popen(cmd, start_new_session=True)
    try:
        return proc.wait(timeout=limit_s)
    except subprocess.TimeoutExpired:
        os.killpg(proc.pid, signal.SIGKILL)
        proc.wait()
        sys.stderr.write(f"bench: {n} ranks did not finish within {limit_s:.0f} s\n")
        return 1


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=_inputs.HEADLINE,
                    choices=_inputs.WORKLOAD_ORDER + sorted(_inputs.DECODE_WORKLOADS))
    ap.add_argument("--impl", default="cuda", choices=["cuda", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--ref-step-seconds", type=float, default=2.0)
    ap.add_argument("--ref-budget-seconds", type=float, default=150.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--dtype", default="bf16", choices=["bf16", "e4m3"],
                    help="forward operand type: bf16 (default) or e4m3 (attn_fwd_fp8)")
    ap.add_argument("--pass", dest="pass_", default="fwd", choices=["fwd", "bwd"],
                    help="forward (default) or the backward pass of the workload")
    ap.add_argument("--path", default="fused", choices=["fused", "standard"],
                    help="fused kernel (default) or the unfused three-kernel path for comparison")
    ap.add_argument("--batch", type=int, default=None,
                    help="override B of the workload (smaller cases for profiler captures)")
    ap.add_argument("--scaling", default="weak", choices=["weak", "strong"],
                    help="N > 1: weak = each rank runs one batch block of an N-times larger "
                         "problem (default); strong = the workload's heads split over the ranks")
    ap.add_argument("--gather", action="store_true",
                    help="N > 1: also time an NCCL all-gather of every rank's O and LSE")
    ap.add_argument("--latency-calls", type=int, default=200,
                    help="calls timed one at a time for the latency line of small workloads")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.steps < 1:
        ap.error("--steps must be >= 1")
    if args.workload in _inputs.DECODE_WORKLOADS:
        if args.impl == "reference":
            print(json.dumps({"impl": "reference", "unavailable": "the decode mode has no "
                              "reference arm; the oracle is timed in its cpu_baseline"}))
            return 0
        return run_decode(args, _inputs.DECODE_WORKLOADS[args.workload])
    w = _inputs.WORKLOADS[args.workload]
    if args.batch is not None:
        import dataclasses
        w = dataclasses.replace(w, B=args.batch, name=f"{w.name}@B{args.batch}")
    _, _, world = dist_env()
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        return relaunch(argv if argv is not None else sys.argv[1:], args.gpus)
    if world != args.gpus:
        sys.stderr.write(f"note: --gpus {args.gpus} but WORLD_SIZE={world}; using WORLD_SIZE\n")
    if args.impl == "reference":
        return run_reference(args, w)
    if args.pass_ == "bwd":
        return run_backward(args, w)
    if args.dtype == "e4m3":
        return run_fp8(args, w)
    if args.path == "standard":
        return run_standard(args, w)
    return run_cuda(args, w)


if __name__ == "__main__":
    sys.exit(main())

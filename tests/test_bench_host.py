"""Host logic of bench.py, on CPU: FLOP and byte counts, the whole-job
aggregation, clock-reason decoding, the stale-profile guard, and the N>1 paths
with world_size-2 gloo process groups."""
import json
import math
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from exact_attention_127_b200 import inputs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_headline_flops_and_bytes():
    w = inputs.WORKLOADS[inputs.HEADLINE]
    assert (w.B, w.H, w.N, w.d, w.causal) == (4, 16, 8192, 128, True)
    assert w.flops() == 4 * 4 * 16 * 8192 ** 2 * 128 / 2      # 1.0995e12
    assert math.isclose(w.flops(), 1.0995e12, rel_tol=1e-4)
    assert w.compulsory_bytes() == 8 * 4 * 16 * 8192 * 128 + 4 * 4 * 16 * 8192
    assert inputs.WORKLOADS["b32h32_n512_d64"].flops() == 4 * 32 * 32 * 512 ** 2 * 64


def test_aggregate_value_is_whole_job():
    # two ranks each doing 1e12 FLOPs, slowest 1 ms -> 2000 TFLOP/s
    assert bench.aggregate_value(1e12, 2, 1.0) == pytest.approx(2000.0)
    assert bench.aggregate_value(1e12, 1, 2.0) == pytest.approx(500.0)


def test_rank_seeds_are_distinct():
    seeds = {bench.rank_seed(2, r) for r in range(8)}
    assert len(seeds) == 8 and bench.rank_seed(2, 0) == 2


def test_decode_reasons():
    assert bench.decode_reasons(0x4 | 0x40) == ["sw_power_cap", "hw_thermal_slowdown"]
    assert bench.decode_reasons(0) == []


def test_traffic_ignored_when_kernel_changed(tmp_path, monkeypatch):
    rec = {"kernel_source_sha256": "0" * 64, "per_launch_dram_bytes": {inputs.HEADLINE: 1.0}}
    p = tmp_path / "t.json"
    p.write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(p))
    assert bench.load_traffic(inputs.HEADLINE) is None
    rec["kernel_source_sha256"] = bench.source_digest()
    p.write_text(json.dumps(rec))
    assert bench.load_traffic(inputs.HEADLINE) == 1.0
    assert bench.load_traffic("other") is None


def test_decode_traffic_keyed_by_its_own_source(tmp_path, monkeypatch):
    rec = {"kernel_source_sha256": bench.source_digest(), "per_launch_dram_bytes": {},
           "decode": {"kernel_source_sha256": "0" * 64,
                      "per_launch_dram_bytes": {"decode_b16h16_n8192_d128": 2.0}}}
    p = tmp_path / "t.json"
    p.write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(p))
    assert bench.load_traffic("decode_b16h16_n8192_d128", "decode") is None
    rec["decode"]["kernel_source_sha256"] = bench.decode_source_digest()
    p.write_text(json.dumps(rec))
    assert bench.load_traffic("decode_b16h16_n8192_d128", "decode") == 2.0
    assert bench.load_traffic("decode_b16h16_n8192_d128") is None   # not in the forward record


def test_oracle_sample_flops_counts_allowed_keys():
    w = inputs.WORKLOADS[inputs.HEADLINE]
    assert bench.oracle_sample_flops(w, [0, 9], 2) == 4 * 128 * (1 + 10) * 2
    w2 = inputs.WORKLOADS["b32h32_n512_d64"]
    assert bench.oracle_sample_flops(w2, [0, 9], 1) == 4 * 64 * 512 * 2


def test_sample_rows_include_boundaries():
    rows = inputs.sample_rows(8192, 256, 2)
    assert len(rows) == 256 and len(set(rows.tolist())) == 256
    for r in (0, 1, 127, 128, 129, 8192 - 129, 8192 - 128, 8191):
        assert r in rows
    assert inputs.sample_rows(100, 256, 0).tolist() == list(range(100))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _reduce_worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        vals = bench.reduce_max([1.0 + rank, 10.0 - rank, 3.0], torch.device("cpu"))
        out[rank] = vals
    finally:
        dist.destroy_process_group()


def test_reduce_max_over_two_gloo_ranks():
    port = _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_reduce_worker, args=(2, port, out), nprocs=2, join=True)
        assert out[0] == out[1] == [2.0, 10.0, 3.0]


def test_reduce_max_single_process_is_identity():
    assert bench.reduce_max([1.5, 2.5], torch.device("cpu")) == [1.5, 2.5]


def test_reference_arm_under_two_ranks_prints_one_line():
    """Under torchrun with 2 ranks only rank 0 runs the oracle and prints."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
           "--workload", "tiny_n128_d64", "--steps", "2", "--warmup", "3",
           "--ref-step-seconds", "0.05"]
    res = subprocess.run(cmd, capture_output=True, text=True, timeout=240, cwd=ROOT)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [l for l in res.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["n_gpus"] == 2 and rec["value"] > 0
    assert rec["e2e"]["h2d_bytes_per_step"] == 0 and rec["cpu_baseline"]["kind"] == "oracle"

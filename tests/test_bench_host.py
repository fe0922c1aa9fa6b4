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


# ---------------------------------------------------------------------------
# One problem split over ranks by heads (exact_attention_127_b200.shard)
# ---------------------------------------------------------------------------
from exact_attention_127_b200 import shard  # noqa: E402


@pytest.mark.parametrize("n_heads", [0, 1, 5, 16, 64, 1024, 1031])
@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
def test_head_range_partitions(n_heads, world):
    ranges = [shard.head_range(n_heads, world, r) for r in range(world)]
    assert ranges[0][0] == 0 and ranges[-1][1] == n_heads
    for (a, b), (c, _) in zip(ranges, ranges[1:]):
        assert b == c                                    # contiguous, in rank order
    sizes = [b - a for a, b in ranges]
    assert max(sizes) - min(sizes) <= 1 and sorted(sizes, reverse=True) == sizes


def test_head_range_rejects_bad_arguments():
    for args in ((4, 0, 0), (4, 2, 2), (4, 2, -1), (-1, 2, 0)):
        with pytest.raises(ValueError):
            shard.head_range(*args)


def test_strong_split_slices_concatenate_to_the_problem():
    w = inputs.WORKLOADS["tiny_n128_d64"]
    w = type(w)(**{**w.__dict__, "B": 2, "H": 3})
    full = [t.reshape(6, w.N, w.d) for t in inputs.workload_inputs(w)]
    for world in (1, 2, 4):
        parts = [bench.rank_inputs(w, world, r, "strong") for r in range(world)]
        assert all(n == 6 for _, n in parts)
        for i in range(3):
            cat = torch.cat([p[0][i] for p in parts])
            assert torch.equal(cat.view(torch.int16), full[i].view(torch.int16))


def test_weak_split_gives_each_rank_its_own_block():
    w = inputs.WORKLOADS["tiny_n128_d64"]
    (q0, _, _), n0 = bench.rank_inputs(w, 2, 0, "weak")
    (q1, _, _), n1 = bench.rank_inputs(w, 2, 1, "weak")
    assert n0 == n1 == 2 * w.B * w.H
    ref = inputs.make_qkv(w.B, w.H, w.N, w.d, bench.rank_seed(w.seed, 1))[0]
    assert torch.equal(q1.view(torch.int16), ref.reshape(q1.shape).view(torch.int16))
    assert not torch.equal(q0, q1)


def _gather_worker(rank, world, port, out):
    """Each rank computes its heads' O and LSE with the fp64 oracle (the CPU
    stand-in for the kernel), rounds them like the kernel's outputs, and
    gathers; every rank must end with the one-rank layout."""
    import oracle
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        B, H, N, d = 1, 5, 40, 8
        q, k, v = inputs.make_qkv(B, H, N, d, seed=9)
        qs, ks, vs = (shard.head_slice(t, world, rank) for t in (q, k, v))
        c = qs.shape[0]
        if c:
            O, L = oracle.attention(qs.view(1, c, N, d), ks.view(1, c, N, d),
                                    vs.view(1, c, N, d), True, 0.3)
            o_loc = torch.from_numpy(O).reshape(c, N, d).to(torch.bfloat16)
            l_loc = torch.from_numpy(L).reshape(c, N).to(torch.float32)
        else:
            o_loc = torch.empty((0, N, d), dtype=torch.bfloat16)
            l_loc = torch.empty((0, N), dtype=torch.float32)
        o_all, l_all = shard.gather_heads(o_loc, l_loc, B * H)
        O1, L1 = oracle.attention(q, k, v, True, 0.3)
        o_ref = torch.from_numpy(O1).reshape(B * H, N, d).to(torch.bfloat16)
        l_ref = torch.from_numpy(L1).reshape(B * H, N).to(torch.float32)
        out[rank] = (torch.equal(o_all.view(torch.int16), o_ref.view(torch.int16)) and
                     torch.equal(l_all.view(torch.int32), l_ref.view(torch.int32)) and
                     o_all.dtype == torch.bfloat16)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_gather_heads_matches_one_rank_layout(world):
    """Heads split 3/2 (world 2) or 2/2/1 (world 3): the gathered O and LSE equal
    the one-rank result byte for byte on every rank."""
    port = _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_gather_worker, args=(world, port, out), nprocs=world, join=True)
        assert [out[r] for r in range(world)] == [True] * world


def test_bench_gpus_2_starts_its_own_ranks():
    """`bench.py --gpus 2` run plainly (no launcher) starts two ranks itself."""
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
           "--workload", "tiny_n128_d64", "--steps", "2", "--warmup", "3",
           "--ref-step-seconds", "0.05"]
    env = {k: v for k, v in os.environ.items()
           if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT")}
    res = subprocess.run(cmd, capture_output=True, text=True, timeout=240, cwd=ROOT, env=env)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [l for l in res.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    assert json.loads(lines[0])["n_gpus"] == 2

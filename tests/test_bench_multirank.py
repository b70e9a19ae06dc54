"""Host logic of bench.py's multi-rank path, on CPU with two gloo ranks.

Each rank scores its own session (weak scaling, no collective on the data
path); the only collectives are the timing reductions: the job's keys are
summed over ranks and divided by the slowest rank's step time.
"""

import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w, r, lr = bench.dist_setup()
        assert (w, r, lr) == (world, rank, rank)
        # rank r processed (r+1) * 1e9 keys in (r+1) * 10 ms
        keys = (rank + 1) * 1e9
        ms = (rank + 1) * 10.0
        value, t = bench.job_throughput(keys, ms, world)
        mx = bench.reduce_max(float(rank) * 3.0, world)
        sm = bench.reduce_sum(1.5, world)
        bench.barrier(world)
        results[rank] = (value, t, mx, sm)
    finally:
        dist.destroy_process_group()


def test_two_rank_reductions():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        results = m.dict()
        procs = [ctx.Process(target=_worker, args=(r, world, port, results)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        res = dict(results)
    total_keys = 1e9 + 2e9
    slowest_ms = 20.0
    for r in range(world):
        value, t, mx, sm = res[r]
        assert t == slowest_ms
        assert value == pytest.approx(total_keys / (slowest_ms * 1e-3) / 1e9)
        assert mx == 3.0
        assert sm == 3.0


def test_single_rank_is_identity():
    value, t = bench.job_throughput(4e9, 8.0, 1)
    assert t == 8.0
    assert value == pytest.approx(4e9 / 8e-3 / 1e9)
    assert bench.reduce_max(2.5, 1) == 2.5
    assert bench.reduce_sum(2.5, 1) == 2.5


def test_union_plane_bytes():
    # two KV heads, GQA 2, d=3: the union takes the per-channel max over each group
    alloc = [[4, 0, 1], [2, 3, 1], [0, 0, 0], [1, 4, 2]]
    # head 0 union: 4+3+1 = 8 planes, head 1: 1+4+2 = 7 planes; 10 words per plane
    assert bench.union_plane_bytes(alloc, 320, 2, 10) == (8 + 7) * 10 * 4


def test_reference_arm_other_ranks_exit_silently():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "0", "--config", "tiny_4k"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def test_reference_arm_line():
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "2", "--warmup", "1", "--config", "tiny_4k"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    out = json.loads(lines[0])
    assert out["impl"] == "reference"
    assert out["higher_is_better"] is True and out["value"] > 0
    assert out["cpu_baseline"]["kind"] == "oracle"
    assert out["cpu_baseline"]["value"] == out["value"]
    assert out["e2e"] == {"value": out["value"], "unit": out["unit"], "h2d_bytes_per_step": 0,
                          "d2h_bytes_per_step": 0}
    assert out["config"]["workload"].startswith("tiny_4k")


def test_reference_arm_uniform_allocation():
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0", "--config", "tiny_4k", "--uniform",
                        "--budget", "136"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    out = json.loads([ln for ln in r.stdout.splitlines() if ln.strip()][-1])
    assert "uniform allocation" in out["config"]["workload"]
    assert out["config"]["budget_bits"] == 136


def test_reference_arm_token_groups():
    """The reference arm times the grouped oracle when --token-group is given."""
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0", "--config", "tiny_4k",
                        "--token-group", "65536"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    out = json.loads([ln for ln in r.stdout.splitlines() if ln.strip()][-1])
    assert "65536-key token group" in out["config"]["workload"]
    assert out["value"] > 0


def test_profile_traffic_needs_matching_workload():
    src = "bit_plane_kv_scan_b200/csrc/scan_tc.cu"
    assert bench.profiled_traffic("decode_1m_b92_uniform", src) is None
    assert bench.profiled_traffic("decode_1m_b136", src) is None  # another budget, other bytes
    assert bench.profiled_traffic("no_such_workload", src) is None
    t = bench.profiled_traffic("decode_1m_b92", src)
    assert t is None or t > 155_000_000  # at least the algorithmic union bytes when current
    t = bench.profiled_traffic("decode_1m_b92", "bit_plane_kv_scan_b200/csrc/scan.cu")
    assert t is None or t > 155_000_000

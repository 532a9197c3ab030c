"""The benchmark's multi-rank host logic on CPU: two gloo ranks (one process
each, as torchrun starts them) take the max of their device times, draw
different token batches and report the whole-job throughput; the reference
arm runs on rank 0 only. No GPU is needed."""
import os
import socket
import subprocess
import sys

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import datetime
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        local_ms = 10.0 + 5.0 * rank  # the second rank is slower
        ms = bench.max_over_ranks(local_ms, dist, "cpu", world)
        out[rank] = (ms, bench.job_throughput(world, bench.M_TOK, ms / 100), bench.rank_seed(0, rank))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time():
    world = 2
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
        res = dict(out)
    assert res[0][0] == res[1][0] == 15.0  # both ranks see the max
    assert res[0][1] == res[1][1] == world * bench.M_TOK / (0.15 * 1e-3)
    assert res[0][2] != res[1][2]  # each rank its own batch


def test_single_rank_needs_no_collective():
    assert bench.max_over_ranks(3.5, None, "cpu", 1) == 3.5
    assert bench.job_throughput(1, 4096, 0.1) == 4096 / 1e-4


def test_reference_arm_runs_on_rank_zero_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "0"],
                       env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def test_reference_arm_line_matches_the_metis_config():
    """The reference arm prints one line on rank 0 with the metis arm's
    config, metric, unit and direction (the oracle on a bounded sample)."""
    import json
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0", "--ref-budget", "0.5"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    assert line["config"] == bench.bench_config(1)
    assert line["metric"] == bench.METRIC and line["unit"] == "tok/s" and line["higher_is_better"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"


def test_gemm_traffic_needs_counters_of_the_current_source(tmp_path, monkeypatch):
    """roofline.traffic comes from the committed ncu counters only while the
    kernel sources hash to the value recorded with them."""
    import json
    p = tmp_path / "c.json"
    monkeypatch.setattr(bench, "GEMM_COUNTERS", str(p))
    p.write_text(json.dumps({"kernel_sources_sha256_16": bench.gemm_source_sha(),
                             "dram_bytes_read": 100, "dram_bytes_write": 23}))
    assert bench.gemm_traffic_from_profile() == 123.0
    p.write_text(json.dumps({"kernel_sources_sha256_16": "0" * 16,
                             "dram_bytes_read": 100, "dram_bytes_write": 23}))
    assert bench.gemm_traffic_from_profile() is None

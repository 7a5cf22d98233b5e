"""Multi-rank host logic of bench.py on CPU with the gloo backend (2 ranks):
the step time is the max over ranks and the job throughput counts every
rank's bytes; the reference arm runs on rank 0 only."""
import os
import socket
import subprocess
import sys
from datetime import timedelta

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        t = bench.max_over_ranks(10.0 + 5.0 * rank, torch.device("cpu"))
        q.put((rank, t, bench.dist_env()))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_with_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [g[1] for g in got] == [15.0, 15.0]          # both ranks see the slowest time
    assert [g[2] for g in got] == [(0, 2, 0), (1, 2, 1)]


def test_job_throughput_counts_all_ranks():
    sys.path.insert(0, ROOT)
    import bench
    one = bench.job_throughput(302_000_000, 10, 1.0, 1)
    assert one == pytest.approx(302_000_000 * 10 / 1e-3 / 1e9)
    assert bench.job_throughput(302_000_000, 10, 1.0, 8) == pytest.approx(8 * one)
    assert bench.job_throughput(302_000_000, 10, 2.0, 8) == pytest.approx(4 * one)


def test_reference_arm_runs_on_rank_zero_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1",
                        "--warmup", "0"], cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_reference_arm_prints_one_json_line():
    import json
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "decode_4k",
                        "--steps", "2", "--warmup", "0"], cwd=ROOT, env=env, capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "GB/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["e2e"]["h2d_bytes_per_step"] == 0
    assert d["steps"] == 2 and d["higher_is_better"] is True


def test_zero_copy_needs_a_mapped_buffer():
    # without a device (or for memory that is not pinned and mapped) the end-to-end
    # loop keeps the explicit copies
    import torch
    sys.path.insert(0, ROOT)
    import bench
    assert bench.host_mapped(torch.zeros(16, dtype=torch.uint8)) is False


def test_stage_tensors_packs_views_at_256_byte_boundaries():
    import torch
    sys.path.insert(0, ROOT)
    import bench
    ts = [torch.arange(5, dtype=torch.int64), torch.ones((3, 7), dtype=torch.bfloat16),
          torch.arange(3, dtype=torch.int32)]
    buf, views = bench.stage_tensors(ts, "cpu")
    assert [v.data_ptr() - buf.data_ptr() for v in views] == [0, 256, 512]
    for t, v in zip(ts, views):
        assert torch.equal(t, v)

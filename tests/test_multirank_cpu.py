"""The multi-rank plumbing of the benchmark on CPU: two gloo ranks on this host.  The
decode shards by request with no data-path collective, so what runs across ranks is the
timing: a barrier, the maximum of the ranks' times, whole-job throughput, and the
reference arm, which rank 0 alone runs and prints."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import bench
    torch.distributed.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                                         world_size=world)
    try:
        bench.barrier(world)
        slowest = bench.max_over_ranks(10.0 + 5.0 * rank, world)
        bench.barrier(world)
        q.put((rank, slowest, bench.aggregate_rate(1e9, world, slowest)))
    finally:
        torch.distributed.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_slowest_time():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(world))
    assert [g[1] for g in got] == [15.0, 15.0]                # max over ranks, on every rank
    # 1 GB per rank per step, two ranks, 15 ms: 2 GB / 15 ms
    assert all(abs(g[2] - 2e9 / 15e-3 / 1e9) < 1e-9 for g in got)


def test_single_rank_passes_times_through():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.25, 1) == 3.25
    assert bench.aggregate_rate(3e9, 1, 1.5) == pytest.approx(2000.0)


def test_reference_arm_prints_on_rank_zero_only():
    """Under two ranks the reference arm (the oracle, host cores) runs on rank 0 alone; the
    other rank exits 0 at once without output."""
    outs = []
    for rank in (0, 1):
        env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank))
        r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                            "--gpus", "2", "--steps", "1", "--warmup", "1"],
                           capture_output=True, text=True, env=env, cwd=ROOT, timeout=600)
        assert r.returncode == 0, r.stderr[-2000:]
        outs.append(r.stdout.strip())
    assert outs[1] == ""
    line = json.loads(outs[0].splitlines()[-1])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0

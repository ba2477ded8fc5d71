"""The multi-process (replica) path of the benchmark on CPU: two gloo ranks
exercise the cross-rank reduction the benchmark uses (slowest rank's time)
and the whole-job throughput (the units all ranks processed over that time).
No GPU is involved."""
import datetime
import multiprocessing as mp
import os
import socket

import pytest


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, times, q):
    import torch
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world,
                                         timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        ms = bench.max_over_ranks(torch, times[rank], torch.device("cpu"))
        q.put((rank, ms, bench.job_rate(world, 1.5e9, ms, 1e9)))
    finally:
        torch.distributed.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_replicas_report_slowest_rank_and_whole_job_rate(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    times = [2.0, 5.0, 3.0][:world]
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, times, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    alive = [p for p in procs if p.is_alive()]
    for p in alive:
        p.kill()
    assert not alive and all(p.exitcode == 0 for p in procs)
    out = sorted(q.get(timeout=5) for _ in range(world))
    for rank, ms, rate in out:
        assert ms == 5.0                                   # every rank sees the slowest time
        assert rate == pytest.approx(world * 1.5 / 5e-3)   # world x 1.5 GB over 5 ms, in GB/s


def test_job_rate_single_rank():
    import bench
    assert bench.job_rate(1, 2e12, 10.0, 1e12) == pytest.approx(200.0)


def test_cpu_baseline_reports_rate_and_measured_cores():
    """The CPU-baseline leg on the smallest workload with a tiny budget: both legs
    present, rates positive, `cores` measured (at least 1, at most the host's)."""
    import bench
    wl = dict(bench.WORKLOADS["decode-single-2048"])
    out = bench.cpu_baseline(wl, 0.05, True)
    assert out["kind"] == "oracle" and out["unit"] == "GB/s"
    assert out["single_thread"]["blas_threads"] == 1 and out["single_thread"]["value"] > 0
    assert out["value"] == out["all_cores"]["value"] > 0
    assert 1.0 <= out["cores"] <= (os.cpu_count() or 1) + 0.5
    short = bench.cpu_baseline(wl, 0.05, True, legs=("all_cores",))
    assert "single_thread" not in short and short["value"] > 0


def test_reference_arm_prints_one_line_from_rank_zero():
    """`bench.py --impl reference` under a 2-rank launch: rank 0 times the oracle
    and prints the one JSON line, the other rank exits 0 without work."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), "bench.py", "--impl", "reference",
           "--gpus", "2", "--steps", "2", "--warmup", "1"]
    out = subprocess.run(cmd, cwd=root, capture_output=True, text=True, timeout=240)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [json.loads(l) for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    line = lines[0]
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["steps"] == 2 and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"] == {"value": line["value"], "unit": line["unit"], "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}

"""Multi-rank host logic of the benchmark, on CPU with the gloo backend (world size 2):
the max-over-ranks timing reduction, the barrier, per-rank batches and the whole-job
rate. The data path itself has no collective: each rank encodes its own points."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

import bench
import workloads


def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        assert bench.dist_env() == (rank, world, rank)
        bench.barrier()
        ms = [12.5, 40.0][rank]
        mx = bench.max_over_ranks(ms)
        rate = bench.whole_job_rate(1 << 20, world, mx * 1e-3)
        w = workloads.WORKLOADS["tiny_L4F2T10"]
        x = workloads.make_inputs(w, seed=bench.rank_seed(rank), n_points=64).x
        gathered = [torch.zeros(64, 3) for _ in range(world)]
        dist.all_gather(gathered, torch.from_numpy(x))
        distinct = not torch.equal(gathered[0], gathered[1])
        q.put((rank, mx, rate, distinct))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_rank_timing_reduction():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(100)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(q.get(timeout=5) for _ in range(2))
    for rank, mx, rate, distinct in res:
        assert mx == 40.0                                   # slowest rank decides
        assert rate == pytest.approx(2 * (1 << 20) / 0.040)  # all ranks' points / max time
        assert distinct                                      # each rank has its own batch


def test_single_process_helpers():
    assert bench.max_over_ranks(3.5) == 3.5
    bench.barrier()
    assert bench.rank_seed(0) != bench.rank_seed(1)
    w = workloads.WORKLOADS["rays_L16F2T19"]
    assert bench.algorithmic_bytes_per_point(w, "fwd") == 1164
    assert bench.algorithmic_bytes_per_point(w, "bwd") == 1164
    assert bench.algorithmic_bytes_per_point(workloads.WORKLOADS["half_L16F2T19"], "fwdbwd") == 1816
    assert bench.algorithmic_bytes_per_point(workloads.WORKLOADS["large_L16F4T22"], "fwdbwd") == 4632


def test_cpu_oracle_timers():
    # the bench's CPU legs run the oracle as it stands on a bounded sample
    w = workloads.WORKLOADS["tiny_L4F2T10"]
    base = bench.cpu_baseline(w, 512, budget_s=0.05)
    assert base["kind"] == "oracle" and base["value"] > 0 and base["cores"] >= 1
    rows = bench.cpu_next_rows(w, 512, budget_s=0.05)
    assert rows["backward_input"]["value"] > 0
    assert rows["adam_step"]["value"] > 0 and rows["adam_step"]["unit"] == "elements/s"
    assert "mlp_forward" not in rows   # L*F = 8 has no MLP


@pytest.mark.timeout(180)
def test_gpus_flag_starts_that_many_ranks():
    """``bench.py --gpus 2`` without a launcher starts two ranks itself (torch.distributed.run
    on 127.0.0.1); with the CPU stub step in place of the GPU work they rendezvous over gloo
    and rank 0 alone prints one line that reports both ranks."""
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK", "MASTER_PORT")}
    r = subprocess.run([sys.executable, "bench.py", "--gpus", "2", "--steps", "4", "--warmup", "3", "--stub-step"],
                       cwd=root, env=env, capture_output=True, text=True, timeout=170)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    line = json.loads(lines[0])
    assert line["impl"] == "stub" and line["n_gpus"] == 2 and line["steps"] == 4
    # rank 1 sleeps twice as long per step: the slowest rank sets the time
    assert line["ms_per_step"] >= 4.0
    assert line["value"] == pytest.approx(2 * (1 << 20) / (line["ms_per_step"] * 1e-3), rel=1e-2)


def test_loop_repeats():
    assert bench.loop_repeats(20, 0.7e-3, 1.0) == 72      # 20 steps x 0.7 ms -> 72 loops >= 1 s
    assert bench.loop_repeats(20, 0.1, 1.0) == 1
    assert bench.loop_repeats(20, 0.7e-3, 0.0) == 1

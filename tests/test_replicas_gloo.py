"""Host-side logic of the multi-GPU path, run as two gloo ranks on the CPU.

The sampler has no exchange step, so N GPUs run N independent replicas: the only
collectives are a barrier and a max over ranks of each rank's device time, and the job's
throughput is every rank's frames over the slowest rank's time. These tests run the same
helpers bench.py uses (rank environment, max over ranks, whole-job throughput) in two
spawned processes, and check bench.py's reference arm under torch.distributed.run: rank 0
alone prints its line and the other rank exits 0 without work."""
import datetime
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _replica(index, world, port, times, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(index), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(index))
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist

    import bench

    w, r, lr = bench.rank_env()
    dist.init_process_group("gloo", rank=r, world_size=w, timeout=datetime.timedelta(seconds=60))
    try:
        dist.barrier()
        ms = bench.max_over_ranks(times[r], w, torch.device("cpu"))
        fps = bench.job_frames_per_s(5, w, ms)
        dist.barrier()
        with open(os.path.join(out_dir, f"rank{r}.json"), "w") as f:
            json.dump({"world": w, "rank": r, "local_rank": lr, "ms": ms, "fps": fps}, f)
    finally:
        dist.destroy_process_group()


def test_two_replicas_report_the_slowest_rank_time_and_all_frames(tmp_path):
    import torch.multiprocessing as mp

    times = [120.0, 150.5]   # rank 1 is the slower replica
    mp.start_processes(_replica, args=(2, _free_port(), times, str(tmp_path)), nprocs=2, join=True,
                       start_method="spawn")
    for r in range(2):
        d = json.load(open(tmp_path / f"rank{r}.json"))
        assert (d["world"], d["rank"], d["local_rank"]) == (2, r, r)
        assert d["ms"] == 150.5                                  # every rank sees the max
        assert d["fps"] == pytest.approx(24 * 5 * 2 / 0.1505)   # both ranks' frames over it


def test_single_process_environment_defaults():
    sys.path.insert(0, ROOT)
    import bench

    env = {k: os.environ.pop(k) for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK") if k in os.environ}
    try:
        assert bench.rank_env() == (1, 0, 0)
        import torch
        assert bench.max_over_ranks(3.5, 1, torch.device("cpu")) == 3.5   # no collective alone
    finally:
        os.environ.update(env)


def test_reference_arm_under_torchrun_prints_once_from_rank_zero():
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2", "--master-addr",
           "127.0.0.1", "--master-port", str(_free_port()), os.path.join(ROOT, "bench.py"), "--impl", "reference",
           "--gpus", "2", "--steps", "1", "--warmup", "0"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [json.loads(x) for x in r.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1
    line = lines[0]
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
    # a step is one block: the timed work is steps x ms_per_step, and the slice figure is
    # stated apart as the extrapolation it is
    ex = line["slice_extrapolation"]
    assert line["steps"] == 1 and ex["blocks_per_slice"] == 120
    assert abs(ex["ms_per_slice"] - 120 * line["ms_per_step"]) < 1e-6 * ex["ms_per_slice"]
    assert abs(line["value"] - 24 / (ex["ms_per_slice"] / 1000.0)) < 1e-9 * line["value"]


def _replica_that_dies(index, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(index), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(index))
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist

    import bench

    w, r, _ = bench.rank_env()
    dist.init_process_group("gloo", rank=r, world_size=w, timeout=datetime.timedelta(seconds=5))
    dist.barrier()
    if r == 1:
        os._exit(0)   # this rank is gone before the timing collective, without a goodbye
    try:
        bench.max_over_ranks(1.0, w, torch.device("cpu"))
        outcome = "returned"
    except Exception as e:  # the collective must end with an error, not wait for ever
        outcome = "error " + type(e).__name__
    with open(os.path.join(out_dir, "rank0.txt"), "w") as f:
        f.write(outcome)
    os._exit(0)


def test_a_rank_that_dies_turns_the_next_collective_into_an_error(tmp_path):
    import time

    import torch.multiprocessing as mp

    t0 = time.time()
    ctx = mp.start_processes(_replica_that_dies, args=(2, _free_port(), str(tmp_path)), nprocs=2, join=False,
                             start_method="spawn")
    try:
        for p in ctx.processes:
            p.join(timeout=120)
        assert all(not p.is_alive() for p in ctx.processes)
    finally:
        for p in ctx.processes:  # only the two processes this test started
            if p.is_alive():
                p.kill()
    assert time.time() - t0 < 120
    assert (tmp_path / "rank0.txt").read_text().startswith("error")

"""Multi-rank host logic of bench.py on CPU: two gloo ranks on 127.0.0.1.

The decode path shards by sequence with no data-path collective; the only
cross-rank steps are the barrier around the timed region and the max over
ranks of the measured times, and each rank draws its own batch.  These run
here with the gloo backend exactly as they run with NCCL on GPUs.
"""

import datetime
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        # rank r measured (1 + r, 5 - r, 2) ms: the slowest rank sets each entry
        vals = bench.reduce_max_over_ranks([1.0 + rank, 5.0 - rank, 2.0], world, "cpu")
        dist.barrier()
        q.put((rank, vals, bench.rank_seed(rank)))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_gloo_ranks_take_the_max_and_draw_distinct_batches():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = {}
    try:
        for _ in range(world):
            rank, vals, seed = q.get(timeout=90)
            got[rank] = (vals, seed)
    finally:
        for p in procs:
            p.join(timeout=30)
            if p.is_alive():
                p.kill()
    assert sorted(got) == [0, 1]
    for rank in range(world):
        assert got[rank][0] == [2.0, 5.0, 2.0]
    assert got[0][1] != got[1][1]
    assert all(p.exitcode == 0 for p in procs)


def test_whole_job_throughput_counts_every_rank():
    one = bench.whole_job_gbs(604e6, 1, 0.25)
    assert one == pytest.approx(604e6 / 0.25e-3 / 1e9)
    assert bench.whole_job_gbs(604e6, 4, 0.25) == pytest.approx(4 * one)
    # a slower max-over-ranks time lowers the whole-job number
    assert bench.whole_job_gbs(604e6, 4, 0.5) == pytest.approx(2 * one)


def test_single_rank_reduce_is_identity():
    assert bench.reduce_max_over_ranks([3.0, 1.5], 1, "cpu") == [3.0, 1.5]


def test_reference_arm_on_nonzero_rank_does_no_work(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")

    class A:
        workload = "v2_b64_ctx8k"
        steps = 1
        warmup = 0

    bench.run_reference(A())
    assert capsys.readouterr().out == ""


@pytest.mark.timeout(180)
def test_gpus_flag_starts_one_rank_per_gpu():
    """`python bench.py --gpus 2` started as a plain process starts the two
    ranks itself (torch.distributed.run on 127.0.0.1); each joins the process
    group (gloo here, without a GPU) and rank 0 reports both."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = {k: v for k, v in os.environ.items()
           if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT")}
    env["CUDA_VISIBLE_DEVICES"] = ""
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--gpus", "2", "--launch-check"],
                       capture_output=True, text=True, timeout=170, env=env, cwd=root)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [json.loads(l) for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    assert lines[0]["world"] == 2 and lines[0]["ranks"] == [0, 1]


def test_rank_launch_command_matches_the_driver_form():
    cmd = bench.rank_launch_command(4, ["--gpus", "4", "--steps", "3"], 29500)
    assert cmd[1:4] == ["-m", "torch.distributed.run", "--nnodes=1"]
    assert "--nproc-per-node=4" in cmd and cmd[cmd.index("--master-addr") + 1] == "127.0.0.1"
    assert cmd[-4:] == ["--gpus", "4", "--steps", "3"]

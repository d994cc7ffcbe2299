"""The multi-rank plumbing of bench.py, on the CPU with two gloo ranks.

The VSA path itself needs no exchange between GPUs (every (batch, head) is
independent), so the only cross-rank steps are the barrier around the timed
region, the max over ranks of the measured time and the whole-job throughput.
"""

import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    from video_dit_block_vsa_b200 import dist as vdist
    info = vdist.init("gloo", timeout_s=60)
    vdist.barrier(info)
    slowest = vdist.max_over_ranks(10.0 + 5.0 * rank, info)
    value = vdist.job_throughput(2.0e12, 4, slowest, info.world)
    out.put((rank, info.world, slowest, value))
    vdist.shutdown(info)


def test_two_gloo_ranks_share_the_slowest_time():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    results = sorted(out.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    for rank, w, slowest, value in results:
        assert w == world
        assert slowest == 15.0  # the slowest rank's time
        assert value == pytest.approx(world * 2.0e12 * 4 / 15.0e-3)


def test_single_rank_needs_no_process_group(monkeypatch):
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    sys.path.insert(0, ROOT)
    from video_dit_block_vsa_b200 import dist as vdist
    info = vdist.init("gloo")
    assert (info.rank, info.world) == (0, 1)
    assert vdist.max_over_ranks(3.5, info) == 3.5
    assert vdist.job_throughput(1.0, 2, 1000.0, 1) == 2.0


def test_reference_arm_runs_on_rank_zero_only(monkeypatch):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    sys.path.insert(0, ROOT)
    import bench
    from video_dit_block_vsa_b200 import workloads as wl

    class Args:
        steps, warmup, gpus = 1, 1, 2

    # rank 1 returns at once without drawing inputs or timing anything
    assert bench.run_reference(Args, wl.WORKLOADS["wan14b_720p_21x45x80_k180"]) == 0

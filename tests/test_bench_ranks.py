"""The multi-rank plumbing of bench.py (weak scaling: one independent problem
per rank) on the CPU: two gloo ranks, each with its own timing; the barrier
returns, the maximum over ranks is the slowest rank's time, the whole-job
value counts the pairs of both ranks over that maximum, and the reference arm
leaves every rank but 0 idle."""

import os
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _rank_main(rank: int, world: int, port: int, out):
    sys.path.insert(0, ROOT)
    import bench

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ranks = bench.Ranks(dist, world, rank, torch.device("cpu"))
        ranks.barrier()
        local_ms = 2.0 + 3.0 * rank  # rank 1 is the slow one
        slowest = ranks.max_over_ranks(local_ms)
        value = ranks.job_value(1000, slowest)
        out.put((rank, slowest, value))
        ranks.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time():
    world = 2
    port = 29500 + (os.getpid() % 2000)
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, slowest, value in res:
        assert slowest == pytest.approx(5.0)
        # both ranks' 1000 pairs over the slowest rank's 5 ms
        assert value == pytest.approx(2 * 1000 / 5e-3)


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench

    ranks = bench.Ranks(None, 1, 0, torch.device("cpu"))
    ranks.barrier()
    assert ranks.max_over_ranks(3.5) == 3.5
    assert ranks.job_value(500, 2.0) == pytest.approx(500 / 2e-3)


def test_reference_arm_idle_on_other_ranks(monkeypatch, capsys):
    sys.path.insert(0, ROOT)
    import bench
    import synth

    monkeypatch.setenv("RANK", "1")

    class A:
        steps = 1
        warmup = 0
        gpus = 2

    assert bench.run_reference(A, synth.shape("tiny")) == 0
    assert capsys.readouterr().out == ""


def test_launch_count_follows_the_plan():
    # bench.py counts launches from the library's own plan query: one key
    # chunk gives a score and a bucket-sort finishing launch per query block,
    # no row sort whatever k; several chunks give score + merge per block and
    # the row sort above k = 512; FP8 adds the two quantiser launches; rows
    # finished in the fused kernel take one launch (and the sort above 512)
    sys.path.insert(0, ROOT)
    import bench
    import synth

    class A:
        key_chunk = 0
        row_finish = 0
        key_tile = 0
        strip_slots = 0
        fp8 = False

    assert bench.kernel_launches_per_step(synth.shape("v4flash_s16k"), A) == 2
    assert bench.kernel_launches_per_step(synth.shape("tiny"), A) == 2
    # top-2048 lists at S = 65,536 need three query blocks of the 512 MiB
    # budget, at S = 262,144 eleven
    assert bench.kernel_launches_per_step(synth.shape("large_s64k"), A) == 6
    assert bench.kernel_launches_per_step(synth.shape("long_s256k"), A) == 22
    assert bench.library_plan(synth.shape("long_s256k"), A)["query_blocks"] == 11
    A.fp8 = True
    assert bench.kernel_launches_per_step(synth.shape("v4flash_s16k"), A) == 4
    A.fp8 = False
    # eight chunks of 1024 keys at S = 32,768: 8 x 4 x 704 x 8 B of lists per
    # query tile gives three query blocks for top-512; top-1024's longer lists
    # give six, and the merge leaves rows of more than 512 keys to the row sort
    A.key_chunk = 1024
    assert bench.kernel_launches_per_step(synth.shape("sweep_s32k", topk=512), A) == 6
    assert bench.kernel_launches_per_step(synth.shape("sweep_s32k", topk=1024), A) == 13
    A.key_chunk = 0
    A.row_finish = 1
    assert bench.kernel_launches_per_step(synth.shape("v4flash_s16k"), A) == 1
    assert bench.kernel_launches_per_step(synth.shape("large_s64k"), A) == 2

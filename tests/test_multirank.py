"""Host logic of the multi-GPU bench path, run as two gloo ranks on the CPU.

The decode shards by sequence with no exchange step: every rank decodes its own batch and the
only collectives are the timing reductions. These tests check that logic without a GPU:
the max over ranks of the timed region, the whole-job throughput, that replicas draw
different sequences, and that the reference arm prints from rank 0 only.
"""
import contextlib
import io
import os
import socket

import numpy as np
import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import mla_inputs as mi


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime

    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        r, wsz, local = bench.dist_env()
        assert (r, wsz, local) == (rank, world, rank)
        # per-rank times: rank 1 is the slow one for the first value, rank 0 for the second
        mine = [10.0 + 5.0 * rank, 7.0 - 3.0 * rank, float(rank)]
        got = bench.max_over_ranks(mine, world)
        # the reference arm: ranks other than 0 return without work or output
        buf = io.StringIO()
        with contextlib.redirect_stdout(buf):
            rc = bench.run_reference(None, mi.WORKLOADS["dsv2"]) if rank != 0 else 0
        out.put((rank, got, rc, buf.getvalue()))
    finally:
        dist.destroy_process_group()


def test_two_ranks_reduce_to_the_slowest_and_only_rank0_reports():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, rc, printed in results:
        assert got == [15.0, 7.0, 1.0], (rank, got)
        assert rc == 0
        if rank != 0:
            assert printed == ""


def test_aggregate_rate_counts_every_rank_over_the_slowest_time():
    # 64 tokens per rank per step, 2 ranks, 100 steps in 50 ms on the slowest rank
    assert bench.aggregate_rate(64, 2, 100, 50.0) == pytest.approx(64 * 2 * 100 / 0.05)
    # weak scaling: at equal time, twice the ranks give twice the throughput
    assert bench.aggregate_rate(64, 4, 100, 50.0) == pytest.approx(
        2 * bench.aggregate_rate(64, 2, 100, 50.0))


def test_replicas_decode_different_sequences():
    w = mi.WORKLOADS["small_bf16"]
    seeds = [bench.rank_seed(r) for r in range(4)]
    assert len(set(seeds)) == 4
    draws = [mi.sequence_draw(w, 0, 16, s).ckv_raw for s in seeds]
    for i in range(4):
        for j in range(i + 1, 4):
            assert not np.array_equal(draws[i], draws[j])

"""bench.py's multi-rank plumbing on CPU: two gloo ranks over 127.0.0.1 (no GPU).

A multi-GPU run is independent replicas; its only collectives are the barrier around each
timed region and the max over ranks of the measured time, and the reference arm runs on
rank 0 alone. These are the host-side pieces a two-GPU run depends on.
"""

import os
import socket

import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        barrier, max_over_ranks = bench.rank_tools(world, "cpu")
        barrier()
        got = max_over_ranks(1.5 + rank)       # each rank's time; the job's is the largest
        barrier()

        class Args:
            ref_seconds, warmup, steps, seqlen = 1.0, 1, 1, 32768
        ref = bench.reference_main(Args, rank, world) if rank != 0 else "skipped"
        out.put((rank, got, ref))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_time_is_max_and_reference_runs_on_rank0_only():
    ctx = mp.get_context("spawn")
    out = ctx.SimpleQueue()
    port = _free_port()
    mp.start_processes(_rank, args=(2, port, out), nprocs=2, join=True, start_method="spawn")
    res = sorted(out.get() for _ in range(2))
    assert [r[1] for r in res] == [2.5, 2.5]
    assert res[1][2] is None          # rank 1 does no reference work


def test_single_rank_tools_are_identity():
    barrier, max_over_ranks = bench.rank_tools(1, "cpu")
    barrier()
    assert max_over_ranks(3.25) == 3.25

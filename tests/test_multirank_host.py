"""The multi-GPU benchmark path on the host: every rank draws its own batch, the job time is
the max over ranks, and the whole-job throughput counts every rank's bytes.  Two gloo ranks on
the CPU (no GPU, no NCCL)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = [0.25, 0.40][rank]          # rank 1 is the slow one
        slowest = bench.max_over_ranks(local_ms, dist, "cpu")
        value = bench.whole_job_gbps(world, 1.2e9, slowest)
        out[rank] = (slowest, value, bench.rank_seed_offset(rank))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_and_count_every_rank():
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
    assert out[0][0] == out[1][0] == pytest.approx(0.40)
    # 2 ranks x 1.2 GB per step in 0.40 ms (the slowest rank) = 6000 GB/s
    assert out[0][1] == out[1][1] == pytest.approx(6000.0)
    assert out[0][2] != out[1][2]            # independent batches


def test_single_process_needs_no_process_group():
    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.whole_job_gbps(1, 1e9, 1.0) == pytest.approx(1000.0)


def test_rank_batches_differ():
    from ragged_paged_attention_forward_b200 import workloads as wl
    a = wl.ragged_batch([40, 50], [1, 1], 4, 2, 16, 16, seed=1002 + bench.rank_seed_offset(0))
    b = wl.ragged_batch([40, 50], [1, 1], 4, 2, 16, 16, seed=1002 + bench.rank_seed_offset(1))
    assert not torch.equal(a.q, b.q)

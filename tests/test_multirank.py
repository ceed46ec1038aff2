"""Host logic of the N>1 benchmark path on CPU: two gloo ranks.

Heads are independent, so ranks share no data; the only cross-rank step is
the max over ranks of the measured time.  Checked here without a GPU.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mx = bench.max_over_ranks(1.5 + rank, "cpu")
        from exact_tiled_attention_45_b200.inputs import make_qkv
        q, _, _ = make_qkv(1, 1, 8, 64, seed=bench.shard_seed(rank))
        gathered = [torch.zeros_like(q.float()) for _ in range(world)]
        dist.all_gather(gathered, q.float())
        out[rank] = (mx, bool(torch.equal(gathered[0], gathered[1])))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_time_and_draw_distinct_shards():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, join=True, start_method="spawn")
    assert out[0][0] == out[1][0] == 2.5
    assert out[0][1] is False  # the shards differ


def test_aggregate_is_total_flops_over_slowest_rank():
    assert bench.aggregate_tflops(1e12, 4, 2.0) == pytest.approx(2000.0)
    assert bench.max_over_ranks(3.25, "cpu") == 3.25

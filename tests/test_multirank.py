"""The N > 1 host logic of bench.py on CPU: two gloo ranks, each with its own
seeded layer, reduce their timings to the maximum (no data-path collective)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        from video_vae_decode_b200 import synth
        seed = bench.rank_seed(synth.WORKLOADS["single_96_64x64"].seed, rank)
        layer = synth.draw_custom(synth.LayerShape(32, 32, 4, 4), seed=seed)
        got = bench.max_over_ranks([10.0 * (rank + 1), 5.0 - rank], "cpu")
        out[rank] = (got, float(layer.x.float().sum()))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reduce_to_max_and_draw_distinct_layers():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, start_method="spawn")
    assert out[0][0] == [20.0, 5.0] and out[1][0] == [20.0, 5.0]
    assert out[0][1] != out[1][1]


def test_single_process_max_is_identity():
    import bench
    assert bench.max_over_ranks([1.5, 2.5], "cpu") == [1.5, 2.5]
    assert bench.rank_seed(4, 3) == 7

"""Host logic of the multi-GPU benchmark path, run as 2 gloo ranks on CPU:
the max-over-ranks step time and the per-rank token shards (weak scaling with
no data-path collective)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    import synth
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w, r, local = bench.dist_env()
        assert (w, r, local) == (world, rank, rank)
        step_ms = 1.0 + rank * 0.25  # rank 1 is the slow one
        mx = bench.max_over_ranks(step_ms, world, torch.device("cpu"))
        seed = bench.rank_activation_seed(rank, synth.MLP_UP.seed)
        x = synth.activations_with_outlier_channels(8, 64, seed=seed)
        seeds = [None] * world
        dist.all_gather_object(seeds, (seed, float(x.float().sum())))
        out[rank] = (mx, seeds)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_time_and_distinct_shards():
    world, port = 2, _free_port()
    manager = mp.get_context("spawn").Manager()
    out = manager.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
    for rank in range(world):
        mx, seeds = out[rank]
        assert mx == pytest.approx(1.25)  # the max, seen identically by every rank
        assert seeds[0][0] != seeds[1][0] and seeds[0][1] != seeds[1][1]


def test_single_rank_max_is_identity():
    import bench
    assert bench.max_over_ranks(3.5, 1, torch.device("cpu")) == 3.5

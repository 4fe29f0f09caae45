"""Host logic of the multi-GPU bench on CPU: every rank runs an independent replica, the job's
time is the max over ranks (gloo here, NCCL on GPUs) and the throughput counts all ranks'
units.  No data-path collective exists to test: the path does not exchange data."""
import os

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    d = bench.init_dist(world, "gloo")
    assert bench.dist_env() == (rank, rank, world)
    local_seconds = 1.0 + rank                     # rank 1 is the slow one
    m = bench.reduce_max(local_seconds, d, torch.device("cpu"))
    out[rank] = (m, bench.aggregate(10.0, world, m))
    d.barrier()
    d.destroy_process_group()


def test_two_rank_max_and_aggregate():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, 29517, out), nprocs=world, join=True)
    assert out[0] == out[1] == (2.0, 10.0)        # 2 ranks x 10 units / 2.0 s


def test_single_rank_is_identity():
    assert bench.reduce_max(3.5, None, torch.device("cpu")) == 3.5
    assert bench.aggregate(7.0, 1, 2.0) == 3.5


def test_arg_defaults_fit_the_contract():
    a = bench.parse_args([])
    assert a.gpus == 1 and a.warmup >= 3 and a.steps >= 1 and a.impl == "ours"

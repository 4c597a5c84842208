"""Multi-rank host logic of bench.py on CPU (gloo, world size 2): the max-over-ranks timing reduction
and the per-rank workload replicas (weak scaling, no data-path collective)."""
import os
import socket

import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        m = bench.reduce_max(10.0 + 5.0 * rank, world)
        w = bench.rank_workload("tiny", rank)
        out[rank] = (m, w.seed, tuple(w.ctx_lens), w.num_q_heads)
    finally:
        dist.destroy_process_group()


def test_reduce_max_and_rank_replicas_gloo():
    world, port = 2, _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn")
        res = dict(out)
    assert res[0][0] == res[1][0] == 15.0               # every rank sees the slowest rank's time
    assert res[0][1] != res[1][1]                       # independent replicas: different seeds
    assert res[0][2:] == res[1][2:]                     # same shapes on every rank (weak scaling)

"""Replica runs on N > 1 ranks: every rank times its own replica and the
reported step time is the maximum over ranks.  Checked here with two gloo
ranks on CPU (the GPU runs use NCCL through the same helpers)."""
import os
import socket

import torch
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import datetime
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world,
                                         timeout=datetime.timedelta(seconds=60))
    import bench
    out[rank] = bench.dist_max(1.0 + 0.5 * rank)     # this rank's step time (ms)
    bench.barrier()
    torch.distributed.destroy_process_group()


def test_step_time_is_the_max_over_ranks():
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(2, _free_port(), out), nprocs=2, join=True)
        assert dict(out) == {0: 1.5, 1: 1.5}


def test_single_process_is_unchanged():
    import bench
    assert bench.dist_max(2.25) == 2.25

"""The N>1 host path on CPU: two gloo ranks, independent seeds, max-over-ranks timing, aggregate rate."""
import os
import socket

import pytest
import torch.multiprocessing as mp

from block_sparse_long_idx_b200 import replicas


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    replicas.init("gloo", timeout_s=60)
    r, w, _ = replicas.rank_info()
    times = [1.0 + r, 10.0 - r]  # rank-dependent "device times"
    mx = replicas.max_over_ranks(times)
    out[r] = (replicas.replica_seed(7, r), mx, replicas.aggregate_rate(100.0, w, mx[0]))
    import torch.distributed as dist

    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_gloo_max_and_rate():
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
    seeds = {out[r][0] for r in range(world)}
    assert seeds == {7, 1007}
    for r in range(world):
        assert out[r][1] == [2.0, 10.0]            # max over ranks, element-wise
        assert out[r][2] == pytest.approx(100.0)   # 2 ranks x 100 units / 2.0 s


def test_single_process_identity():
    assert replicas.max_over_ranks([3.0, 4.0]) == [3.0, 4.0]
    assert replicas.aggregate_rate(10.0, 1, 2.0) == 5.0

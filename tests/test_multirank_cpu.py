"""The multi-rank side of bench.py on CPU ranks (gloo, world size 2).

Every rank indexes its own batch of the same shape (weak scaling, no
collective on the data path); the only collectives are the barrier and the
max over ranks of the step time, which every rank must see identically.
"""
import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime

    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        local_ms = [0.25, 0.75][rank]
        m = bench.reduce_max(local_ms, dist, torch.device("cpu"))
        dist.barrier()
        out[rank] = m
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo():
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    assert out[0] == out[1] == 0.75


def test_ranks_get_distinct_batches_of_one_shape():
    import bench
    from workloads import make_decode

    a = bench.rank_batch(0)
    # rank 1's batch is drawn from its own seed; compare on a small slice of the draw order
    b = make_decode("r1", 2 + 1000 * 1, T=2, L=64, H=4, h=2, B=8, k=4, n_planted=0)
    c = make_decode("r0", 2, T=2, L=64, H=4, h=2, B=8, k=4, n_planted=0)
    assert not torch.equal(b.keys, c.keys)
    assert a.T == 32 and a.L == 32768 and a.H == 64 and a.h == 8 and a.k == 2048
    assert bench.reduce_max(1.5, None, torch.device("cpu")) == 1.5


def test_selection_agreement_and_planted_recall():
    import numpy as np

    import bench
    a = np.array([[1, 2, 3, -1], [5, 6, 7, 8]])
    b = np.array([[2, 3, 4, -1], [5, 6, 7, 8]])
    iou, rec = bench.selection_agreement(a, b)
    assert abs(iou - (0.5 + 1.0) / 2) < 1e-12          # {2,3} of {1,2,3,4}; identical rows
    assert abs(rec - (2 / 3 + 1.0) / 2) < 1e-12        # 2 of b's 3 valid ids; all 4
    assert bench.planted_recall(a, np.array([[3, 9], [8, 5]])) == 3 / 4
    assert bench.planted_recall(a, np.zeros((2, 0), dtype=np.int64)) is None

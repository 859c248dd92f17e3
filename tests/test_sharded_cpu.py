"""The key-sharded indexer's algebra and exchanges on the CPU.

* shard bounds cover [0, L) with whole blocks;
* on the fp64 oracle, per-shard head importances (each shard's own block means
  and prefix lengths) add up to the unsharded importance, the heads picked from
  the sum are the unsharded heads, and the top-k of the union of the per-shard
  top-k lists (as (score, global id) pairs in shard order) is the unsharded
  top-k -- decode and causal prefill, 2 and 3 shards;
* the two exchanges (TorchShardComm over gloo, world size 2): the sum
  all-reduce and the gather whose rows the merge reads in shard order.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from sparse_attention_token_misa_b200.sharded import TorchShardComm, candidate_rows, shard_bounds
from gpu_helpers import to_ora
from workloads import make_decode, make_prefill


@pytest.mark.parametrize("L,B,world", [(1000, 64, 3), (4096, 128, 2), (129, 128, 2), (4096, 128, 32)])
def test_shard_bounds(L, B, world):
    b = shard_bounds(L, B, world)
    assert len(b) == world and b[0][0] == 0 and b[-1][1] == L
    for (s0, s1), (n0, _) in zip(b[:-1], b[1:]):
        assert s1 == n0 and s0 % B == 0 and s1 % B == 0 and s1 > s0
    with pytest.raises(ValueError):
        shard_bounds(L, B, (L + B - 1) // B + 1)


def sharded_oracle(o, B, q_block, h, k, bounds):
    """The sharded step written with the oracle's own functions."""
    T, H, _ = o["q"].shape
    parts, locals_ = [], []
    for s0, s1 in bounds:
        keys_r = o["keys"][:, s0:s1]
        means_r = np.stack([oracle.block_means(keys_r[b], B) for b in range(keys_r.shape[0])])
        p_r = np.clip(o["prefix_len"] - s0, 0, s1 - s0)
        _, imp_r = oracle.route_heads(o["q"], o["w"], means_r, o["seq_of"], p_r, s1 - s0, B, q_block, h)
        parts.append(imp_r)
        locals_.append((keys_r, p_r, s0))
    imp = np.sum(parts, axis=0)
    heads = np.stack([oracle.topk_ascending(imp[g], h) for g in range(imp.shape[0])])
    per_query = np.stack([heads[t // q_block] for t in range(T)])
    cs, ci = [], []
    for keys_r, p_r, s0 in locals_:
        S_r = oracle.index_scores(o["q"], o["w"], keys_r, o["seq_of"], p_r, per_query)
        loc = oracle.topk_rows(S_r, k)
        cs.append(np.where(loc >= 0, np.take_along_axis(S_r, np.maximum(loc, 0), axis=1), -np.inf))
        ci.append(np.where(loc >= 0, loc + s0, -1))
    all_s, all_i = np.concatenate(cs, axis=1), np.concatenate(ci, axis=1)
    return imp, heads, oracle.topk_rows(all_s, k, id_map=all_i)


@pytest.mark.parametrize("mode,world", [("decode", 2), ("decode", 3), ("prefill", 2), ("prefill", 3)])
def test_sharded_decomposition_oracle(mode, world):
    if mode == "decode":
        wl = make_decode("sh", 61 + world, T=5, L=1000, H=16, h=4, B=64, k=40, n_planted=2)
    else:
        wl = make_prefill("sh", 62 + world, T=8, L=900, H=16, h=4, B=64, k=40, q_block=4, n_regions=1,
                          region_len=128, first_pos=500)
    o = to_ora(wl)
    full = oracle.misa_indexer(o["q"], o["w"], o["keys"], o["seq_of"], o["prefix_len"], wl.B, wl.q_block, wl.h,
                               wl.k)
    imp, heads, idx = sharded_oracle(o, wl.B, wl.q_block, wl.h, wl.k, shard_bounds(wl.L, wl.B, world))
    assert np.allclose(imp, full["importance"], rtol=1e-12, atol=1e-12)
    assert np.array_equal(heads, full["heads"])
    assert np.array_equal(idx, full["idx"])


def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _comm_worker(rank, world, port, out):
    import datetime

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        comm = TorchShardComm()
        T, k = 3, 5
        imp = torch.full((2, 4), float(rank + 1))
        comm.all_reduce_sum_(imp)
        scores = torch.arange(T * k, dtype=torch.float32).view(T, k) + 100 * rank
        ids = torch.arange(T * k, dtype=torch.int32).view(T, k) + 1000 * rank
        rows_s = candidate_rows(comm.all_gather(scores))
        rows_i = candidate_rows(comm.all_gather(ids))
        out[rank] = (imp.tolist(), rows_s.tolist(), rows_i.tolist())
    finally:
        dist.destroy_process_group()


def test_shard_comm_gloo():
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_comm_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    assert out[0] == out[1]
    imp, rows_s, rows_i = out[0]
    assert imp == [[3.0] * 4] * 2
    T, k = 3, 5
    for t in range(T):
        # row t: rank 0's k candidates, then rank 1's
        assert rows_s[t] == [float(t * k + i) for i in range(k)] + [float(100 + t * k + i) for i in range(k)]
        assert rows_i[t] == [t * k + i for i in range(k)] + [1000 + t * k + i for i in range(k)]


def test_sharded_run_orchestration(monkeypatch):
    """ShardedMisaIndexer.run on the CPU with the library calls stubbed: the
    means tuple reaches the router as (means, hi, lo), the importances are
    all-reduced before the heads are picked, both candidate arrays are gathered
    and the merge reads the gathered rows."""
    import sparse_attention_token_misa_b200.sharded as sh

    log = []

    class Nat:
        OP_ROUTE_HEADS = 1

        def workspace_bytes(self, *a):
            return 256

        def alloc_workspace(self, n, device=None):
            return torch.zeros(max(n, 256), dtype=torch.uint8)

        def shard_prefix(self, prefix_len, s0, Ls, out=None, stream=None):
            log.append(("shard_prefix", s0, Ls))
            out.copy_((prefix_len - s0).clamp(0, Ls))

        def route_heads(self, q, w, means, seq_of, prefix_len, L, B, q_block, h, heads=None, importance=None,
                        workspace=None, stream=None, means_hi=None, means_lo=None):
            log.append(("route", means is not None, means_hi is not None, means_lo is not None, L))
            importance.fill_(1.0)

        def topk(self, scores, k, n=None, row_valid=None, id_map=None, idx=None, workspace=None, stream=None):
            log.append(("topk", k, n, id_map is not None, float(scores[0, 0])))
            idx.copy_(torch.arange(k, dtype=torch.int32).expand_as(idx))

        def index_score(self, *a, **kw):
            log.append(("score",))

        def gather_candidates(self, scores, idx, n, s0, out_scores=None, out_ids=None, stream=None):
            log.append(("gather", s0))
            out_scores.fill_(float(s0))
            out_ids.copy_(idx + s0)

    class Comm:
        world = 2

        def all_reduce_sum_(self, t):
            log.append(("all_reduce", tuple(t.shape)))
            t.mul_(2)                               # two ranks' equal partials
            return t

        def all_gather(self, t):
            log.append(("all_gather", tuple(t.shape)))
            return torch.stack([t, t + 1])

    monkeypatch.setattr(sh, "nat", Nat())
    T, H, h, L, B, k = 3, 8, 4, 1000, 128, 8
    ix = sh.ShardedMisaIndexer(T, H, h, L, B, k, 512, 1000, world=2, device="cpu")
    q, w = torch.zeros(T, H, 128), torch.zeros(T, H)
    keys, means = torch.zeros(1, 488, 128), (torch.zeros(1, 4, 128), torch.zeros(1, 4, 128), torch.zeros(1, 4, 128))
    so, pl = torch.zeros(T, dtype=torch.int32), torch.full((T,), 1000, dtype=torch.int32)
    idx = ix.run(q, w, keys, means, so, pl, Comm())
    names = [e[0] for e in log]
    assert names == ["shard_prefix", "route", "all_reduce", "topk", "score", "topk", "gather", "all_gather",
                     "all_gather", "topk"]
    assert log[0] == ("shard_prefix", 512, 488)
    assert log[1] == ("route", True, True, True, 488)          # the split means reached the router
    assert log[3][1:3] == (h, H) and log[3][4] == 2.0          # heads picked from the all-reduced sum
    assert log[-1][1:4] == (k, 2 * k, True)                    # merge over W * k candidates with the id map
    assert float(ix.all_scores[0, 0]) == 512.0 and float(ix.all_scores[0, k]) == 513.0   # rank 0's, then rank 1's
    assert idx.shape == (T, k)

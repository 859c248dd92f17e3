"""The key-sharded indexer on one GPU: the W ranks of a group run one after the
other in this process (each on its own copy of its key shard and that shard's
block statistics) and the test does the two exchanges itself -- the sum of the
partial importances in rank order, the stack of the candidate lists.  Kernels
that wait on one another never run, so nothing here needs two GPUs.

Checked: every rank merges to the same indices; the heads against the oracle's
importances (selection rule); the indices against the oracle's scores of the
heads the GPU routed; and, when the heads agree with the unsharded GPU indexer,
the indices equal its indices exactly (a key's score does not depend on the
shard it sits in, and the merge keeps the tie rule).
"""
import numpy as np
import pytest
import torch

import oracle
import sparse_attention_token_misa_b200 as misa
from gpu_helpers import np_i, to_gpu, to_ora
from parity import check_selection
from workloads import make_decode, make_prefill

pytestmark = pytest.mark.gpu


def run_sharded(wl, g, world, split=True):
    bounds = misa.shard_bounds(wl.L, wl.B, world)
    ranks = []
    for s0, s1 in bounds:
        ix = misa.ShardedMisaIndexer(wl.T, wl.H, wl.h, wl.L, wl.B, wl.k, s0, s1, world, q_block=wl.q_block)
        keys_r = g["keys"][:, s0:s1].contiguous()
        ranks.append((ix, keys_r, misa.block_stats(keys_r, wl.B, split=split)))
    imps = []
    for ix, keys_r, means_r in ranks:
        m = dict(zip(("means", "means_hi", "means_lo"), means_r)) if split else dict(means=means_r)
        imps.append(ix.route_partial(g["q"], g["w"], m["means"], g["seq_of"], g["prefix_len"],
                                     means_hi=m.get("means_hi"), means_lo=m.get("means_lo")).clone())
    total = imps[0].clone()
    for x in imps[1:]:
        total += x                                   # the all-reduce, in rank order
    cands = []
    for ix, keys_r, _ in ranks:
        ix.importance_buf.copy_(total)
        ix.select_heads()
        cs, ci = ix.local_candidates(g["q"], g["w"], keys_r, g["seq_of"])
        cands.append((cs.clone(), ci.clone()))
    gs = torch.stack([c[0] for c in cands])          # the all-gather
    gi = torch.stack([c[1] for c in cands])
    outs = [ix.merge(gs, gi).clone() for ix, _, _ in ranks]
    torch.cuda.synchronize()
    for ix, _, _ in ranks:
        assert misa.error_query(ix.ws) == 0 and misa.error_query(ix.ws_route) == 0
    for o_ in outs[1:]:
        assert torch.equal(o_, outs[0])
    return ranks[0][0], outs[0], total


@pytest.mark.parametrize("mode,world", [("decode", 2), ("decode", 3), ("prefill", 2), ("decode", 5)])
def test_sharded_matches_oracle_and_unsharded(mode, world):
    if mode == "decode":
        wl = make_decode("gsh", 81 + world, T=6, L=5000, H=64, h=8, B=128, k=256, n_planted=3)
    else:
        wl = make_prefill("gsh", 82 + world, T=128, L=6000, H=64, h=8, B=128, k=256, q_block=64, n_regions=1,
                          region_len=512)
    g, o = to_gpu(wl), to_ora(wl)
    ix0, idx, imp = run_sharded(wl, g, world)
    heads = np_i(ix0.heads)
    r = oracle.misa_indexer(o["q"], o["w"], o["keys"], o["seq_of"], o["prefix_len"], wl.B, wl.q_block, wl.h, wl.k)
    for gi in range(heads.shape[0]):
        check_selection(heads[gi], r["importance"][gi], wl.h, what=f"heads g{gi}")
    # the indices against the oracle's scores with the heads the GPU routed
    per_query = np.stack([heads[t // wl.q_block] for t in range(wl.T)])
    S_o = oracle.index_scores(o["q"], o["w"], o["keys"], o["seq_of"], o["prefix_len"], per_query)
    idx_g = np_i(idx)
    for t in range(wl.T):
        check_selection(idx_g[t], S_o[t], wl.k, what=f"sharded t{t}")
    # against the unsharded GPU indexer
    means = misa.block_stats(g["keys"], wl.B, split=True)
    ux = misa.MisaIndexer(wl.T, wl.H, wl.h, wl.L, wl.B, wl.k, wl.q_block)
    ux.run(g["q"], g["w"], g["keys"], means, g["seq_of"], g["prefix_len"])
    torch.cuda.synchronize()
    same_heads = torch.equal(ux.heads, ix0.heads)
    if same_heads:
        assert torch.equal(ux.idx, idx)
    assert np.allclose(imp.cpu().numpy(), ux.importance.cpu().numpy(), rtol=1e-4, atol=1e-3)

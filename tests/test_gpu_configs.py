"""End-to-end parity on the five workloads at full size, in the launch
configuration the benchmark uses (the preallocated indexers of the package).

The CUDA path runs on the whole batch; the fp64 oracle runs on every query
where it finishes in seconds and on a seeded sample of queries (whole routing
blocks, first and last included) otherwise.  Upstream choices (routed heads,
coarse candidates, HISA blocks) are checked with the selection rule; where the
GPU's choice legitimately differs from the oracle's inside the tolerance band
the downstream comparison of that query is skipped and counted (the stage tests
cover the downstream kernels on the oracle's own choices).
"""
import numpy as np
import pytest
import torch

import oracle
import sparse_attention_token_misa_b200 as misa
from gpu_helpers import np_f, np_i, to_gpu, to_ora
from parity import check_bit_exact_topk, check_scores, check_selection
from workloads import make_workload

pytestmark = pytest.mark.gpu

MAX_DIVERGENT_FRAC = 0.05


def _sub(o, ts, seqs):
    """Oracle arrays restricted to queries ts (their caches `seqs` already cut)."""
    return dict(q=o["q"][ts], w=o["w"][ts], keys=o["keys"], seq_of=o["seq_of"][ts], prefix_len=o["prefix_len"][ts])


def _run_misa(wl, g, dense=False):
    means = misa.block_stats(g["keys"], wl.B)
    if dense:
        ix = misa.DenseIndexer(wl.T, wl.H, wl.L, wl.k)
        ix.run(g["q"], g["w"], g["keys"], g["seq_of"], g["prefix_len"])
    else:
        ix = misa.MisaIndexer(wl.T, wl.H, wl.h, wl.L, wl.B, wl.k, wl.q_block)
        ix.run(g["q"], g["w"], g["keys"], means, g["seq_of"], g["prefix_len"])
    torch.cuda.synchronize()
    return ix, means


def _check_misa(wl, ix, ts, o_sub, dense=False):
    """ts: sampled query ids (whole routing blocks)."""
    idx_g = np_i(ix.idx[ts])
    S_g = ix.scores[ts].cpu().numpy()
    check_bit_exact_topk(idx_g, S_g, wl.k, what="idx vs CPU sort of GPU scores")
    if dense:
        idx_o, S_o = oracle.dense_indexer(o_sub["q"], o_sub["w"], o_sub["keys"], o_sub["seq_of"],
                                          o_sub["prefix_len"], wl.k)
        check_scores(S_g.astype(np.float64), S_o, wl.k)
        for i in range(len(ts)):
            check_selection(idx_g[i], S_o[i], wl.k, what=f"dense t{ts[i]}")
        return 0
    r = oracle.misa_indexer(o_sub["q"], o_sub["w"], o_sub["keys"], o_sub["seq_of"], o_sub["prefix_len"], wl.B,
                            wl.q_block, wl.h, wl.k)
    groups = sorted({t // wl.q_block for t in ts})
    heads_g = np_i(ix.heads[groups])
    divergent = 0
    for gi, g in enumerate(groups):
        check_selection(heads_g[gi], r["importance"][gi], wl.h, what=f"heads g{g}")
        same = np.array_equal(heads_g[gi], r["heads"][gi])
        rows = [i for i, t in enumerate(ts) if t // wl.q_block == g]
        if not same:
            divergent += len(rows)
            continue
        check_scores(S_g[rows].astype(np.float64), r["scores"][rows], wl.k)
        for i in rows:
            check_selection(idx_g[i], r["scores"][i], wl.k, what=f"misa t{ts[i]}")
    assert divergent <= MAX_DIVERGENT_FRAC * len(ts), divergent
    return divergent


def test_tiny_decode_all_indexers():
    wl = make_workload("tiny_decode_L4096")
    g, o = to_gpu(wl), to_ora(wl)
    ts = list(range(wl.T))
    ix, means = _run_misa(wl, g)
    _check_misa(wl, ix, ts, o)
    dx, _ = _run_misa(wl, g, dense=True)
    _check_misa(wl, dx, ts, o, dense=True)
    # MISA-dagger and HISA on the same batch
    dg = misa.MisaDaggerIndexer(wl.T, wl.H, wl.h, wl.L, wl.B, 1024, wl.k)
    dg.run(g["q"], g["w"], g["keys"], means, g["seq_of"], g["prefix_len"], want_scores=True)
    hx = misa.HisaIndexer(wl.T, wl.H, wl.L, wl.B, 8, wl.k)
    hx.run(g["q"], g["w"], g["keys"], means, g["seq_of"], g["prefix_len"])
    torch.cuda.synchronize()
    _check_dagger(wl, dg, ts, o, kp=1024)
    _check_hisa(wl, hx, ts, o, B=wl.B, m=8)


def test_dsv32_decode_misa_and_dense():
    wl = make_workload("dsv32_decode_L32768")
    g, o = to_gpu(wl), to_ora(wl)
    ts = list(range(wl.T))
    ix, _ = _run_misa(wl, g)
    _check_misa(wl, ix, ts, o)
    dx, _ = _run_misa(wl, g, dense=True)
    sample = [0, 13, 31]
    o_s = to_ora(wl, seqs=sample)
    _check_misa(wl, dx, sample, _sub(o_s, sample, sample), dense=True)


def test_prefill_128k_sampled_blocks():
    wl = make_workload("prefill_L131072")
    g = to_gpu(wl)
    ix, _ = _run_misa(wl, g)
    G = wl.T // wl.q_block
    rng = np.random.default_rng(31)
    blocks = sorted({0, G - 1, *rng.choice(np.arange(1, G - 1), size=2, replace=False).tolist()})
    ts = [t for b in blocks for t in range(b * wl.q_block, (b + 1) * wl.q_block)]
    o = to_ora(wl)
    o_sub = _sub(o, ts, None)
    # the oracle's q_block grouping over the concatenated sample matches the sampled blocks
    _check_misa(wl, _Sliced(ix, ts, blocks, wl.q_block), list(range(len(ts))), o_sub)


class _Sliced:
    """View of an indexer's outputs restricted to sampled whole routing blocks,
    renumbered 0.. so that the oracle's grouping of the sample lines up."""

    def __init__(self, ix, ts, blocks, q_block):
        self.idx = ix.idx[ts]
        self.scores = ix.scores[ts]
        self.heads = ix.heads[blocks]


def _check_dagger(wl, dg, ts, o_sub, kp):
    idx_g = np_i(dg.idx[ts])
    cand_g = np_i(dg.coarse.idx[ts])
    cs_g = dg.cand_scores[ts].cpu().numpy()
    check_bit_exact_topk(idx_g, cs_g, wl.k, ids=cand_g, what="dagger idx vs CPU sort")
    check_bit_exact_topk(cand_g, dg.coarse.scores[ts].cpu().numpy(), kp, what="dagger coarse vs CPU sort")
    r = oracle.misa_dagger_indexer(o_sub["q"], o_sub["w"], o_sub["keys"], o_sub["seq_of"], o_sub["prefix_len"],
                                   wl.B, wl.q_block, wl.h, kp, wl.k)
    heads_g = np_i(dg.coarse.heads[ts])
    divergent = 0
    for i in range(len(ts)):
        check_selection(heads_g[i], r["importance"][i], wl.h, what=f"dagger heads t{ts[i]}")
        if not np.array_equal(heads_g[i], r["heads"][i]):
            divergent += 1
            continue
        check_selection(cand_g[i], r["coarse_scores"][i], kp, what=f"dagger coarse t{ts[i]}")
        if not np.array_equal(cand_g[i], r["cand"][i]):
            divergent += 1
            continue
        check_scores(cs_g[i:i + 1].astype(np.float64), r["cand_scores"][i:i + 1], wl.k)
        check_selection(idx_g[i], r["cand_scores"][i], wl.k, what=f"dagger t{ts[i]}", ids=r["cand"][i])
    assert divergent <= MAX_DIVERGENT_FRAC * len(ts), divergent


def _check_hisa(wl, hx, ts, o_sub, B, m):
    idx_g = np_i(hx.idx[ts])
    cand_g = np_i(hx.cand[ts])
    S_g = hx.scores[ts].cpu().numpy()
    check_bit_exact_topk(idx_g, S_g, wl.k, ids=cand_g, what="hisa idx vs CPU sort")
    r = oracle.hisa_indexer(o_sub["q"], o_sub["w"], o_sub["keys"], o_sub["seq_of"], o_sub["prefix_len"], B, m, wl.k)
    blocks_g = np_i(hx.blocks[ts])
    divergent = 0
    for i in range(len(ts)):
        check_selection(blocks_g[i], r["block_scores"][i], m, what=f"hisa blocks t{ts[i]}")
        if not np.array_equal(blocks_g[i], r["blocks"][i]):
            divergent += 1
            continue
        assert np.array_equal(cand_g[i], r["cand"][i])
        check_scores(S_g[i:i + 1].astype(np.float64), r["cand_scores"][i:i + 1], wl.k)
        check_selection(idx_g[i], r["cand_scores"][i], wl.k, what=f"hisa t{ts[i]}", ids=r["cand"][i])
    assert divergent <= MAX_DIVERGENT_FRAC * len(ts), divergent


@pytest.mark.parametrize("fused", [False, True])
def test_glm5_dagger_sampled(fused):
    """fused: the coarse stage through misa_index_decode."""
    wl = make_workload("glm5_dagger_decode_L65536")
    g = to_gpu(wl)
    means = misa.block_stats(g["keys"], wl.B, split=True)
    dg = misa.MisaDaggerIndexer(wl.T, wl.H, wl.h, wl.L, wl.B, wl.kp, wl.k, fused=fused)
    dg.run(g["q"], g["w"], g["keys"], means, g["seq_of"], g["prefix_len"], want_scores=True)
    torch.cuda.synchronize()
    sample = [0, 9, 22, 40, 63]
    o = to_ora(wl, seqs=sample)
    _check_dagger(wl, dg, sample, _sub(o, sample, sample), kp=wl.kp)


@pytest.mark.parametrize("B,m", [(128, 64), (64, 128)])
def test_hisa_decode_sampled(B, m):
    wl = make_workload("hisa_decode_L131072")
    g = to_gpu(wl)
    means = misa.block_stats(g["keys"], B)
    hx = misa.HisaIndexer(wl.T, wl.H, wl.L, B, m, wl.k)
    hx.run(g["q"], g["w"], g["keys"], means, g["seq_of"], g["prefix_len"])
    torch.cuda.synchronize()
    sample = [0, 7, 15]
    o = to_ora(wl, seqs=sample)
    _check_hisa(wl, hx, sample, _sub(o, sample, sample), B=B, m=m)


def test_prefill_128k_dagger_sampled_blocks():
    """MISA-dagger on the causal 128K prefill (coarse top-8192 of the routed
    scores per query, all-head rerank of the candidates, top-2048): the first
    and the last routing block against the oracle."""
    wl = make_workload("prefill_L131072")
    kp = 8192
    g = to_gpu(wl)
    means = misa.block_stats(g["keys"], wl.B)
    dg = misa.MisaDaggerIndexer(wl.T, wl.H, wl.h, wl.L, wl.B, kp, wl.k, wl.q_block)
    dg.run(g["q"], g["w"], g["keys"], means, g["seq_of"], g["prefix_len"], want_scores=True)
    torch.cuda.synchronize()
    G = wl.T // wl.q_block
    blocks = [0, G - 1]
    ts = [t for b in blocks for t in range(b * wl.q_block, (b + 1) * wl.q_block)]
    o_sub = _sub(to_ora(wl), ts, None)
    idx_g = np_i(dg.idx[ts])
    cand_g = np_i(dg.coarse.idx[ts])
    cs_g = dg.cand_scores[ts].cpu().numpy()
    check_bit_exact_topk(idx_g, cs_g, wl.k, ids=cand_g, what="dagger idx vs CPU sort")
    check_bit_exact_topk(cand_g, dg.coarse.scores[ts].cpu().numpy(), kp, what="dagger coarse vs CPU sort")
    r = oracle.misa_dagger_indexer(o_sub["q"], o_sub["w"], o_sub["keys"], o_sub["seq_of"], o_sub["prefix_len"],
                                   wl.B, wl.q_block, wl.h, kp, wl.k)
    heads_g = np_i(dg.coarse.heads[blocks])
    divergent = 0
    for gi in range(len(blocks)):
        check_selection(heads_g[gi], r["importance"][gi], wl.h, what=f"dagger heads block {blocks[gi]}")
        rows = range(gi * wl.q_block, (gi + 1) * wl.q_block)
        if not np.array_equal(heads_g[gi], r["heads"][gi]):
            divergent += len(rows)
            continue
        for i in rows:
            check_selection(cand_g[i], r["coarse_scores"][i], kp, what=f"dagger coarse t{ts[i]}")
            if not np.array_equal(cand_g[i], r["cand"][i]):
                divergent += 1
                continue
            check_scores(cs_g[i:i + 1].astype(np.float64), r["cand_scores"][i:i + 1], wl.k)
            check_selection(idx_g[i], r["cand_scores"][i], wl.k, what=f"dagger t{ts[i]}", ids=r["cand"][i])
    assert divergent <= MAX_DIVERGENT_FRAC * len(ts), divergent


def test_prefill_128k_hisa_sampled():
    """HISA on the causal 128K prefill (B = 128, m = 64): every query keeps the
    block its prefix cuts; sampled queries against the oracle."""
    wl = make_workload("prefill_L131072")
    B, m = 128, 64
    g = to_gpu(wl)
    means = misa.block_stats(g["keys"], B)
    hx = misa.HisaIndexer(wl.T, wl.H, wl.L, B, m, wl.k)
    hx.run(g["q"], g["w"], g["keys"], means, g["seq_of"], g["prefix_len"])
    torch.cuda.synchronize()
    ts = [0, 1, 127, 1000, 2047, 4094, 4095]
    o_sub = _sub(to_ora(wl), ts, None)
    _check_hisa(wl, hx, ts, o_sub, B=B, m=m)
    # the cut block is among the chosen ones wherever the prefix ends inside a block
    blocks_g = np_i(hx.blocks[ts])
    for i, t in enumerate(ts):
        p = int(wl.prefix_len[t])
        if p % B:
            assert p // B in blocks_g[i], (t, p)

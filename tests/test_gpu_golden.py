"""The hand-worked 2-head / 8-token case through the CUDA library.

tests/golden/hand_case_2head_8token.json holds values derived by hand from the
definitions (dense scores, block means, router importances and head choice,
MISA-1 scores and top-k, MISA-dagger candidates and top-k, HISA block scores,
block choice and top-k, and a partial last block with B = 3).  Here the same
inputs, zero-padded from d = 2 to d = 128 (which leaves every dot product
unchanged), go through misa_block_stats, misa_route_heads, misa_index_score,
misa_topk, misa_hier_rerank and hisa_block_filter, and every result is compared
with the stored value: exactly where the value is exact in fp32 (which covers
the dense tie between tokens 0 and 6 at score 1.0, settled toward token 0, and
HISA missing token 5), within fp32 rounding where a mean divides by 3.
"""
import json
import os

import numpy as np
import pytest
import torch

import sparse_attention_token_misa_b200 as misa

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_case_2head_8token.json")


def _load():
    with open(GOLDEN) as f:
        g = json.load(f)
    q2 = np.asarray(g["q"], dtype=np.float32)        # [1, 2, 2]
    w = np.asarray(g["w"], dtype=np.float32)         # [1, 2]
    k2 = np.asarray(g["keys"], dtype=np.float32)     # [1, 8, 2]
    q = np.zeros((1, 2, 128), np.float32)
    q[..., :2] = q2
    keys = np.zeros((1, 8, 128), np.float32)
    keys[..., :2] = k2
    dev = torch.device("cuda", 0)
    t = dict(q=torch.from_numpy(q).to(torch.bfloat16).to(dev), w=torch.from_numpy(w).to(dev),
             keys=torch.from_numpy(keys).to(torch.bfloat16).to(dev),
             seq_of=torch.zeros(1, dtype=torch.int32, device=dev),
             prefix_len=torch.full((1,), 8, dtype=torch.int32, device=dev))
    return g, t


def _list(x):
    return x.cpu().numpy().reshape(-1).tolist()


def test_golden_dense_scores_and_topk():
    g, t = _load()
    S = misa.index_score(t["q"], t["w"], t["keys"], t["seq_of"], t["prefix_len"])
    torch.cuda.synchronize()
    assert _list(S) == g["dense_scores"]
    assert _list(misa.topk(S, 3)) == g["dense_top3"]      # 1.0 tie: token 0 wins over token 6
    assert _list(misa.topk(S, 4)) == g["dense_top4"]


@pytest.mark.parametrize("split", [False, True])
def test_golden_block_means_router_and_misa(split):
    g, t = _load()
    B = g["B"]
    means = misa.block_stats(t["keys"], B, split=split)
    m32 = means[0] if split else means
    torch.cuda.synchronize()
    assert np.array_equal(m32[0, :, :2].cpu().numpy(), np.asarray(g["block_means"], np.float32))
    assert torch.count_nonzero(m32[0, :, 2:]) == 0
    kw = dict(means=means[0], means_hi=means[1], means_lo=means[2]) if split else dict(means=means)
    heads, imp = misa.route_heads(t["q"], t["w"], seq_of=t["seq_of"], prefix_len=t["prefix_len"], L=8, B=B,
                                  q_block=1, h=1, **kw)
    torch.cuda.synchronize()
    assert _list(imp) == g["router_importance"]
    assert _list(heads) == g["router_heads_h1"]
    S1 = misa.index_score(t["q"], t["w"], t["keys"], t["seq_of"], t["prefix_len"], heads=heads, h=1)
    assert _list(S1) == g["misa1_scores"]
    cand = misa.topk(S1, 4)
    assert _list(cand) == g["misa1_top4"] == g["dagger_h1_kp4_cand"]
    idx, cs = misa.hier_rerank(t["q"], t["w"], t["keys"], t["seq_of"], t["prefix_len"], cand, 3, want_scores=True)
    torch.cuda.synchronize()
    assert _list(idx) == g["dagger_h1_kp4_top3"]
    assert _list(cs) == [g["dense_scores"][i] for i in g["dagger_h1_kp4_cand"]]


def test_golden_causal_router():
    """prefix 6 with B = 4: only block 0 is wholly visible."""
    g, t = _load()
    means = misa.block_stats(t["keys"], g["B"])
    pl = torch.full((1,), 6, dtype=torch.int32, device=t["q"].device)
    heads, imp = misa.route_heads(t["q"], t["w"], means, t["seq_of"], pl, L=8, B=g["B"], q_block=1, h=1)
    torch.cuda.synchronize()
    assert _list(imp) == g["causal_prefix6_importance"]
    assert _list(heads) == g["causal_prefix6_heads_h1"]


def test_golden_hisa():
    g, t = _load()
    B = g["B"]
    means = misa.block_stats(t["keys"], B)
    blocks, cand, bs = misa.hisa_block_filter(t["q"], t["w"], means, t["seq_of"], t["prefix_len"], L=8, B=B, m=1,
                                              want_scores=True)
    torch.cuda.synchronize()
    assert _list(bs) == g["hisa_block_scores"]
    assert _list(blocks) == g["hisa_m1_blocks"]
    assert _list(cand) == [0, 1, 2, 3]
    S = misa.index_score(t["q"], t["w"], t["keys"], t["seq_of"], t["prefix_len"], cand=cand)
    idx = misa.topk(S, 3, id_map=cand)
    torch.cuda.synchronize()
    assert _list(idx) == g["hisa_m1_top3"]     # token 5 (the dense maximum) lies in the dropped block


def test_golden_hisa_partial_last_block():
    g, t = _load()
    p = g["partial_block_B3"]
    means = misa.block_stats(t["keys"], 3)
    torch.cuda.synchronize()
    ref = np.asarray(p["block_means"])
    got = means[0, :, :2].cpu().numpy().astype(np.float64)
    assert np.allclose(got, ref, rtol=2 ** -21, atol=0)      # fp32 division by 3 (or 2)
    blocks, cand, bs = misa.hisa_block_filter(t["q"], t["w"], means, t["seq_of"], t["prefix_len"], L=8, B=3, m=2,
                                              want_scores=True)
    torch.cuda.synchronize()
    # the router multiplies the fp32 means split into two bf16 halves (about 16 significant bits)
    assert np.allclose(bs.cpu().numpy().reshape(-1), p["hisa_block_scores"], rtol=2 ** -14, atol=0)
    assert _list(blocks) == p["hisa_m2_blocks"]
    assert _list(cand) == p["hisa_m2_cand"]
    # score rows padded to a multiple of 4 entries (the top-k reads 16-byte aligned rows)
    S = torch.empty((1, 8), dtype=torch.float32, device=cand.device)
    misa.index_score(t["q"], t["w"], t["keys"], t["seq_of"], t["prefix_len"], cand=cand, scores=S)
    assert _list(misa.topk(S, 3, n=6, id_map=cand)) == p["hisa_m2_top3"]
    assert _list(misa.topk(S, 4, n=6, id_map=cand)) == p["hisa_m2_top4"]

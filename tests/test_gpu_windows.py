"""Block statistics over overlapping windows and max pooling, on the GPU,
against the fp64 oracle.

HISA explainer (zhichai.net), section 七 (局限与未来方向, 潜在改进): overlapping
blocks and max pooling instead of mean pooling, as ways around what a block
mean loses.  Window j covers keys [j*S, min(j*S + B, L)), M = 1 + ceil(max(L -
B, 0) / S); the statistic is the mean or the coordinate-wise maximum.  Covered
here: the statistics themselves (the maximum bit for bit), their maintenance on
key append (bit-identical to a full recompute), the router and the HISA block
filter over windows (visibility, cut windows, candidate lists without repeats),
HISA end to end, and the full-size HISA decode with both statistics.
"""
import numpy as np
import pytest
import torch

import oracle
import sparse_attention_token_misa_b200 as misa
from gpu_helpers import assert_no_device_error, dev, f64, np_f, np_i, to_gpu, to_ora
from parity import check_bit_exact_topk, check_scores, check_selection
from workloads import make_decode, make_prefill, make_workload

pytestmark = pytest.mark.gpu

MAX_DIVERGENT_FRAC = 0.05


# ------------------------------------------------------------------ the statistics
@pytest.mark.parametrize("nseq,L,B,S", [(2, 1000, 128, 64), (1, 4096, 128, 32), (3, 777, 64, 64), (1, 300, 100, 30),
                                        (2, 129, 128, 1), (1, 5, 8, 3), (1, 4100, 256, 128)])
@pytest.mark.parametrize("pool", ["mean", "max"])
def test_window_stats(nseq, L, B, S, pool):
    wl = make_decode("ws", 51 + L + S, T=nseq, L=L, H=2, h=1, B=B, k=1, n_planted=0)
    keys = dev(wl.keys)
    st, hi, lo = misa.block_stats(keys, B, stride=S, pool=pool, split=True)
    torch.cuda.synchronize()
    M = oracle.num_windows(L, B, S)
    assert st.shape == (nseq, M, 128) and misa.num_windows(L, B, S) == M
    k64 = f64(wl.keys)
    for b in range(nseq):
        ref = oracle.window_stats(k64[b], B, S, pool)
        got = np_f(st[b])
        if pool == "max":
            assert np.array_equal(got, ref), b                  # a max of bf16 values is exact
            assert torch.equal(hi[b], st[b].to(torch.bfloat16))  # ... and its split is (max, 0)
            assert torch.count_nonzero(lo[b].float()) == 0
        else:
            for j in range(M):
                win = k64[b, j * S:min(j * S + B, L)]
                allow = 2e-5 * np.abs(win).mean(axis=0) + 1e-12
                assert np.all(np.abs(got[j] - ref[j]) <= allow), (b, j)
            # the split: hi = bf16(stat), lo = bf16(stat - hi)
            assert torch.equal(hi[b], st[b].to(torch.bfloat16))
            assert torch.equal(lo[b], (st[b] - hi[b].float()).to(torch.bfloat16))


@pytest.mark.parametrize("B,S,pool", [(128, 64, "mean"), (128, 32, "max"), (64, 64, "max"), (100, 30, "mean"),
                                      (16, 5, "max")])
def test_append_windows_bit_identical_to_recompute(B, S, pool):
    """Keys appended in steps of 1, 7, 300, 1, 130 and 2 rows: after each step
    the maintained statistics (and their bf16 split) equal, bit for bit, the
    statistics computed from scratch over the longer caches."""
    nseq, L_cap = 3, 1200
    wl = make_decode("wa", 61 + B + S, T=nseq, L=L_cap, H=2, h=1, B=B, k=1, n_planted=0)
    full = dev(wl.keys)
    cache = torch.zeros_like(full)
    M_cap = misa.num_windows(L_cap, B, S)
    st = torch.zeros((nseq, M_cap, 128), dtype=torch.float32, device=full.device)
    hi = torch.zeros((nseq, M_cap, 128), dtype=torch.bfloat16, device=full.device)
    lo = torch.zeros_like(hi)
    lens = torch.tensor([0, 5, 17], dtype=torch.int32, device=full.device)
    for b in range(nseq):               # caches start with a few rows already in place
        n0 = int(lens[b])
        cache[b, :n0] = full[b, :n0]
    l0 = lens.clone()
    ref0 = [misa.block_stats(cache[b:b + 1, :int(l0[b])], B, stride=S, pool=pool, split=True)
            if int(l0[b]) else None for b in range(nseq)]
    for b in range(nseq):
        if ref0[b] is not None:
            M0 = ref0[b][0].shape[1]
            st[b, :M0], hi[b, :M0], lo[b, :M0] = ref0[b][0][0], ref0[b][1][0], ref0[b][2][0]
    ws = misa.alloc_workspace(256)
    for n_new in (1, 7, 300, 1, 130, 2):
        new = torch.stack([full[b, int(lens[b]):int(lens[b]) + n_new] for b in range(nseq)])
        misa.append_keys(cache, lens, new.contiguous(), B, st, workspace=ws, means_hi=hi, means_lo=lo, stride=S,
                         pool=pool)
        lens += n_new
        torch.cuda.synchronize()
        assert_no_device_error(ws)
        for b in range(nseq):
            n = int(lens[b])
            assert torch.equal(cache[b, :n], full[b, :n])
            r, rh, rl = misa.block_stats(full[b:b + 1, :n], B, stride=S, pool=pool, split=True)
            M = r.shape[1]
            assert torch.equal(st[b, :M], r[0]), (n_new, b)
            assert torch.equal(hi[b, :M], rh[0]) and torch.equal(lo[b, :M], rl[0]), (n_new, b)


# ------------------------------------------------------------------ router over windows
@pytest.mark.parametrize("T,L,H,h,B,S,q_block,pool", [
    (4, 5000, 64, 8, 128, 64, 1, "mean"),
    (4, 5000, 64, 8, 128, 64, 1, "max"),
    (130, 3000, 32, 6, 64, 32, 64, "mean"),      # causal prefill: windows cut by the routing prefix are excluded
    (70, 2000, 64, 8, 128, 48, 16, "max"),
])
def test_route_heads_windows(T, L, H, h, B, S, q_block, pool):
    if q_block == 1:
        wl = make_decode("rw", 71 + T, T=T, L=L, H=H, h=h, B=B, k=16, n_planted=2)
    else:
        wl = make_prefill("rw", 71 + T, T=T, L=L, H=H, h=h, B=B, k=16, q_block=q_block, n_regions=1, region_len=256)
    g, o = to_gpu(wl), to_ora(wl)
    st_o = np.stack([oracle.window_stats(o["keys"][b], B, S, pool) for b in range(o["keys"].shape[0])])
    heads_o, imp_o = oracle.route_heads(o["q"], o["w"], st_o, o["seq_of"], o["prefix_len"], L, B, q_block, h, S)
    st = misa.block_stats(g["keys"], B, stride=S, pool=pool, split=True)
    ws = misa.alloc_workspace(misa.workspace_bytes(1, T, H, L, S))
    heads, imp = misa.route_heads(g["q"], g["w"], seq_of=g["seq_of"], prefix_len=g["prefix_len"], L=L, B=B,
                                  q_block=q_block, h=h, workspace=ws, stride=S, means=st[0], means_hi=st[1],
                                  means_lo=st[2])
    torch.cuda.synchronize()
    assert_no_device_error(ws)
    check_scores(np_f(imp), imp_o, h, what="importance")
    heads_g = np_i(heads)
    for gi in range(heads_o.shape[0]):
        check_selection(heads_g[gi], imp_o[gi], h, what=f"heads g{gi}")
    check_bit_exact_topk(heads_g, imp.cpu().numpy(), h, what="heads vs CPU sort of GPU importance")


# ------------------------------------------------------------------ HISA block filter over windows
def _expected_cand(blocks_row, limit, B, S):
    """Candidate list of a row given its chosen windows (integer work)."""
    m = blocks_row.shape[0]
    exp = np.full(m * B, -1)
    prev_end = -1
    for i, j in enumerate(blocks_row):
        if j < 0:
            continue
        ids = np.arange(j * S, j * S + B)
        ids[(ids >= limit) | (ids < prev_end)] = -1
        exp[i * B:(i + 1) * B] = ids
        prev_end = j * S + B
    return exp


@pytest.mark.parametrize("T,L,B,S,m,pool", [(4, 5000, 128, 64, 8, "mean"), (4, 5000, 128, 64, 8, "max"),
                                            (3, 1000, 64, 16, 40, "mean"), (2, 777, 100, 30, 5, "max"),
                                            (3, 4096, 128, 128, 12, "max")])
def test_hisa_block_filter_windows(T, L, B, S, m, pool):
    wl = make_decode("hw", 81 + L + S, T=T, L=L, H=64, h=64, B=B, k=16, n_planted=3, mode="hisa", m=m)
    wl.prefix_len[-1] = max(1, L // 2 + 3)           # a causal query whose prefix cuts windows
    g, o = to_gpu(wl), to_ora(wl)
    st_o = np.stack([oracle.window_stats(o["keys"][b], B, S, pool) for b in range(o["keys"].shape[0])])
    blocks_o, cand_o, bs_o = oracle.hisa_block_filter(o["q"], o["w"], st_o, o["seq_of"], o["prefix_len"], L, B, m, S)
    st = misa.block_stats(g["keys"], B, stride=S, pool=pool)
    blocks, cand, bs = misa.hisa_block_filter(g["q"], g["w"], st, g["seq_of"], g["prefix_len"], L, B, m,
                                              want_scores=True, stride=S)
    torch.cuda.synchronize()
    check_scores(np_f(bs), bs_o, m, what="window scores")
    blocks_g, cand_g = np_i(blocks), np_i(cand)
    for t in range(T):
        check_selection(blocks_g[t], bs_o[t], m, what=f"windows t{t}")
        limit = min(int(o["prefix_len"][t]), L)
        assert np.array_equal(cand_g[t], _expected_cand(blocks_g[t], limit, B, S)), t
        ids = cand_g[t][cand_g[t] >= 0]
        assert np.all(np.diff(ids) > 0), t                  # listed once, ascending
    check_bit_exact_topk(blocks_g, bs.cpu().numpy(), m, what="windows vs CPU sort of GPU window scores")


@pytest.mark.parametrize("B,S,m,pool", [(128, 64, 16, "mean"), (128, 128, 8, "max"), (64, 32, 30, "max")])
def test_hisa_indexer_windows(B, S, m, pool):
    wl = make_decode("hi", 91 + S, T=6, L=9000, H=64, h=64, B=B, k=300, n_planted=4, mode="hisa", m=m)
    wl.prefix_len[2] = 5000
    g, o = to_gpu(wl), to_ora(wl)
    st = misa.block_stats(g["keys"], B, stride=S, pool=pool, split=True)
    hx = misa.HisaIndexer(wl.T, wl.H, wl.L, B, m, wl.k, stride=S)
    hx.run(g["q"], g["w"], g["keys"], st, g["seq_of"], g["prefix_len"])
    torch.cuda.synchronize()
    assert_no_device_error(hx.ws_filter)
    _check_hisa(wl, hx, list(range(wl.T)), o, B, S, m, pool)


def _check_hisa(wl, hx, ts, o, B, S, m, pool):
    idx_g, cand_g = np_i(hx.idx[ts]), np_i(hx.cand[ts])
    S_g = hx.scores[ts].cpu().numpy()
    check_bit_exact_topk(idx_g, S_g, wl.k, ids=cand_g, what="hisa idx vs CPU sort")
    r = oracle.hisa_indexer(o["q"][ts], o["w"][ts], o["keys"], o["seq_of"][ts], o["prefix_len"][ts], B, m, wl.k,
                            S=S, pool=pool)
    blocks_g = np_i(hx.blocks[ts])
    divergent = 0
    for i in range(len(ts)):
        check_selection(blocks_g[i], r["block_scores"][i], m, what=f"hisa windows t{ts[i]}")
        if not np.array_equal(blocks_g[i], r["blocks"][i]):
            divergent += 1
            continue
        assert np.array_equal(cand_g[i], r["cand"][i])
        check_scores(S_g[i:i + 1].astype(np.float64), r["cand_scores"][i:i + 1], wl.k)
        check_selection(idx_g[i], r["cand_scores"][i], wl.k, what=f"hisa t{ts[i]}", ids=r["cand"][i])
    assert divergent <= MAX_DIVERGENT_FRAC * len(ts), divergent


@pytest.mark.parametrize("B,S,m,pool", [(128, 128, 64, "max"), (128, 64, 64, "mean")])
def test_hisa_decode_windows_full_size_sampled(B, S, m, pool):
    """The HISA decode workload (16 queries over 128K keys, k = 2048) with
    max-pooled blocks and with half-overlapping mean-pooled windows: sampled
    queries against the oracle."""
    wl = make_workload("hisa_decode_L131072")
    g = to_gpu(wl)
    st = misa.block_stats(g["keys"], B, stride=S, pool=pool, split=True)
    hx = misa.HisaIndexer(wl.T, wl.H, wl.L, B, m, wl.k, stride=S)
    hx.run(g["q"], g["w"], g["keys"], st, g["seq_of"], g["prefix_len"])
    torch.cuda.synchronize()
    sample = [0, 8, 15]
    o = to_ora(wl, seqs=sample)
    o = dict(q=o["q"][sample], w=o["w"][sample], keys=o["keys"], seq_of=o["seq_of"][sample],
             prefix_len=o["prefix_len"][sample])
    # the oracle arrays are already cut to the sampled queries: index them 0..2
    idx_g, cand_g = np_i(hx.idx[sample]), np_i(hx.cand[sample])
    S_g = hx.scores[sample].cpu().numpy()
    check_bit_exact_topk(idx_g, S_g, wl.k, ids=cand_g, what="hisa idx vs CPU sort")
    r = oracle.hisa_indexer(o["q"], o["w"], o["keys"], o["seq_of"], o["prefix_len"], B, m, wl.k, S=S, pool=pool)
    blocks_g = np_i(hx.blocks[sample])
    divergent = 0
    for i in range(len(sample)):
        check_selection(blocks_g[i], r["block_scores"][i], m, what=f"windows q{sample[i]}")
        if not np.array_equal(blocks_g[i], r["blocks"][i]):
            divergent += 1
            continue
        assert np.array_equal(cand_g[i], r["cand"][i])
        check_scores(S_g[i:i + 1].astype(np.float64), r["cand_scores"][i:i + 1], wl.k)
        check_selection(idx_g[i], r["cand_scores"][i], wl.k, what=f"hisa q{sample[i]}", ids=r["cand"][i])
    assert divergent <= MAX_DIVERGENT_FRAC * len(sample), divergent

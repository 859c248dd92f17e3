"""misa_index_decode (router + routed scoring in one kernel, the top-k behind it) on the GPU.

The fused step must compute what misa_route_heads, misa_index_score and
misa_topk compute one after the other (MISA page, gist.science, "Methodology:
MISA"): heads against the oracle's importances under the selection rule and
bit-exactly against a CPU sort of the kernel's own importances; scores equal,
bit for bit, those of misa_index_score run with the kernel's heads, and within
the score tolerance of the oracle on those heads; indices bit-exactly the
top-k of the kernel's own scores (CPU sort, ties to the lower position) and
within the tolerance band of the oracle's.  Rows with massive exact ties check
that the top-k, started while the scoring kernel still runs, reads the whole
rows the scoring kernel wrote.
"""
import numpy as np
import pytest
import torch

import oracle
import sparse_attention_token_misa_b200 as misa
from gpu_helpers import assert_no_device_error, dev, np_f, np_i, to_gpu, to_ora
from parity import check_bit_exact_topk, check_scores, check_selection
from workloads import make_decode, make_workload

pytestmark = pytest.mark.gpu


def _fused(g, wl, ws=None):
    means = misa.block_stats(g["keys"], wl.B, split=True)
    if ws is None:
        ws = misa.alloc_workspace(misa.workspace_bytes(misa._native.OP_INDEX_DECODE, wl.T, wl.H, wl.L, wl.B, wl.k))
    heads, imp, S, idx = misa.index_decode(g["q"], g["w"], g["keys"], means[1], means[2], g["seq_of"],
                                           g["prefix_len"], wl.B, wl.h, wl.k, workspace=ws)
    torch.cuda.synchronize()
    assert_no_device_error(ws)
    return means, heads, imp, S, idx


def _check(wl, g, means, heads, imp, S, idx, o=None, check_oracle=True):
    L, k, h = wl.L, wl.k, wl.h
    S_l = S[:, :L]
    # scores: bit for bit those of the scoring call with the same heads
    ref = misa.index_score(g["q"], g["w"], g["keys"], g["seq_of"], g["prefix_len"], heads=heads, h=h)
    torch.cuda.synchronize()
    assert torch.equal(S_l, ref), "fused scores differ from misa_index_score on the fused heads"
    # heads: the exact top-h of the kernel's own importances
    check_bit_exact_topk(np_i(heads), imp.cpu().numpy(), h, what="heads vs CPU sort of GPU importance")
    # indices: the exact top-k of the kernel's own scores
    check_bit_exact_topk(np_i(idx), S_l.cpu().numpy(), k, what="idx vs CPU sort of GPU scores")
    if not check_oracle:
        return
    o = o or to_ora(wl)
    means_o = np.stack([oracle.block_means(o["keys"][b], wl.B) for b in range(o["keys"].shape[0])])
    heads_o, imp_o = oracle.route_heads(o["q"], o["w"], means_o, o["seq_of"], o["prefix_len"], L, wl.B, 1, h)
    check_scores(np_f(imp), imp_o, h, what="importance")
    heads_g = np_i(heads)
    for t in range(wl.T):
        check_selection(heads_g[t], imp_o[t], h, what=f"heads t{t}")
    # scores and indices against the oracle on the kernel's heads
    S_o = oracle.index_scores(o["q"], o["w"], o["keys"], o["seq_of"], o["prefix_len"], heads_g)
    check_scores(S_l.cpu().numpy().astype(np.float64), S_o, k)
    idx_g = np_i(idx)
    for t in range(wl.T):
        check_selection(idx_g[t], S_o[t], k, what=f"idx t{t}")


@pytest.mark.parametrize("T,L,H,h,B,k,shared,ragged", [
    (4, 5000, 64, 8, 128, 256, False, False),
    (3, 32768, 64, 8, 128, 2048, False, False),
    (5, 9000, 32, 8, 128, 700, False, True),      # prefixes shorter than L, not multiples of B
    (6, 4097, 16, 4, 64, 100, True, True),        # one shared cache; 16 router columns
    (2, 65536, 48, 16, 128, 8192, False, False),  # 48 heads padded to 64 columns; h = 16; k' = 8192
    (3, 1000, 64, 8, 128, 2000, False, False),    # k above the row length: -1 padding
    (3, 1000, 64, 1, 128, 100, False, False),     # one routed head
    (3, 300, 64, 8, 100, 1, False, True),         # k = 1; rows shorter than one tile
    (40, 2048, 64, 8, 128, 64, False, False),     # several queries per CTA
])
def test_fused_decode_parity(T, L, H, h, B, k, shared, ragged):
    wl = make_decode("fd", 1000 + T + L, T=T, L=L, H=H, h=h, B=B, k=k, n_planted=min(4, L // 8),
                     shared_cache=shared)
    if ragged:
        rng = np.random.default_rng(T)
        wl.prefix_len[:] = torch.from_numpy(rng.integers(max(1, L // 3), L + 1, size=T).astype(np.int32))
        wl.prefix_len[0] = L
    g = to_gpu(wl)
    means, heads, imp, S, idx = _fused(g, wl)
    _check(wl, g, means, heads, imp, S, idx)


@pytest.mark.parametrize("distinct", [16, 4, 1])
def test_fused_decode_massive_ties(distinct):
    """Keys repeat `distinct` rows over the cache, so every score value occurs
    L / distinct times (2048, 8192, or all 32768 entries equal); the top-k must
    still be the lowest positions among the ties."""
    T, L, H, h, B, k = 3, 32768, 64, 8, 128, 2048
    wl = make_decode("ft", 77 + distinct, T=T, L=L, H=H, h=h, B=B, k=k, n_planted=0)
    base = wl.keys[:, :distinct].clone()
    reps = L // distinct
    wl.keys[:] = base.repeat(1, reps, 1)
    g = to_gpu(wl)
    means, heads, imp, S, idx = _fused(g, wl)
    _check(wl, g, means, heads, imp, S, idx, check_oracle=False)


def test_fused_decode_zero_weights_and_garbage_workspace():
    """A query with all head weights zero scores every token 0 (all importances
    0: the first h heads; top-k: the first k positions); the workspace may hold
    anything on entry."""
    T, L, H, h, B, k = 4, 20000, 64, 8, 128, 1500
    wl = make_decode("fz", 91, T=T, L=L, H=H, h=h, B=B, k=k, n_planted=2)
    wl.w[1] = 0.0
    g = to_gpu(wl)
    ws = misa.alloc_workspace(misa.workspace_bytes(misa._native.OP_INDEX_DECODE, T, H, L, B, k))
    ws.fill_(0xFF)
    misa.error_reset(ws)
    for _ in range(2):
        means, heads, imp, S, idx = _fused(g, wl, ws)
        _check(wl, g, means, heads, imp, S, idx)
        assert np_i(heads)[1].tolist() == list(range(h))
        assert np_i(idx)[1].tolist() == list(range(k))


def test_fused_decode_matches_three_calls_full_size():
    """The bench workload (32 x 32768 keys, 8 of 64 heads, k = 2048): the fused
    step and the three separate calls agree (heads equal unless two
    importances tie within the tolerance; indices equal where the heads are);
    sampled queries against the oracle."""
    wl = make_workload("dsv32_decode_L32768")
    g = to_gpu(wl)
    means, heads, imp, S, idx = _fused(g, wl)
    ix = misa.MisaIndexer(wl.T, wl.H, wl.h, wl.L, wl.B, wl.k)
    ix.run(g["q"], g["w"], g["keys"], means, g["seq_of"], g["prefix_len"])
    torch.cuda.synchronize()
    same_heads = (heads == ix.heads).all(dim=1)
    assert int(same_heads.sum()) >= wl.T - 1
    assert torch.equal(idx[same_heads], ix.idx[same_heads])
    scale = float(ix.importance.abs().max())
    assert torch.allclose(imp, ix.importance, rtol=1e-4, atol=1e-5 * scale)   # two fp32 summation orders
    _check(wl, g, means, heads, imp, S, idx, check_oracle=False)
    sample = [0, 13, 31]
    o = to_ora(wl, seqs=sample)
    o = dict(q=o["q"][sample], w=o["w"][sample], keys=o["keys"], seq_of=o["seq_of"][sample],
             prefix_len=o["prefix_len"][sample])
    means_o = np.stack([oracle.block_means(o["keys"][b], wl.B) for b in range(len(sample))])
    _, imp_o = oracle.route_heads(o["q"], o["w"], means_o, o["seq_of"], o["prefix_len"], wl.L, wl.B, 1, wl.h)
    check_scores(np_f(imp[sample]), imp_o, wl.h, what="importance")
    heads_g = np_i(heads[sample])
    S_o = oracle.index_scores(o["q"], o["w"], o["keys"], o["seq_of"], o["prefix_len"], heads_g)
    check_scores(S[sample, :wl.L].cpu().numpy().astype(np.float64), S_o, wl.k)
    for i, t in enumerate(sample):
        check_selection(heads_g[i], imp_o[i], wl.h, what=f"heads t{t}")
        check_selection(np_i(idx[t]), S_o[i], wl.k, what=f"idx t{t}")


def test_fused_decode_scores_only():
    """idx = NULL: the call ends with heads, importances and scores (the same
    as the full call's) and writes no indices."""
    wl = make_decode("fs", 321, T=5, L=7000, H=64, h=8, B=128, k=300, n_planted=3)
    g = to_gpu(wl)
    means = misa.block_stats(g["keys"], wl.B, split=True)
    ws = misa.alloc_workspace(misa.workspace_bytes(misa._native.OP_INDEX_DECODE, wl.T, wl.H, wl.L, wl.B, wl.k))
    heads, imp, S, idx = misa.index_decode(g["q"], g["w"], g["keys"], means[1], means[2], g["seq_of"],
                                           g["prefix_len"], wl.B, wl.h, wl.k, workspace=ws)
    h2, imp2, S2, idx2 = misa.index_decode(g["q"], g["w"], g["keys"], means[1], means[2], g["seq_of"],
                                           g["prefix_len"], wl.B, wl.h, wl.k, workspace=ws, select=False)
    torch.cuda.synchronize()
    assert_no_device_error(ws)
    assert idx2 is None
    assert torch.equal(heads, h2) and torch.equal(imp, imp2)
    assert torch.equal(S[:, :wl.L], S2[:, :wl.L])

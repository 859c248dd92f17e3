"""The bf16 hi / lo split of the block means (written by misa_block_stats and
misa_append_keys, read by misa_route_heads and hisa_block_filter).

* block_stats writes hi = bf16(m) and lo = bf16(m - hi) of the fp32 mean m it
  writes beside them (round to nearest even, as torch converts);
* the router and the block filter fed the split give bit for bit what they give
  when they split the fp32 means themselves, in every launch mode (clusters
  per decision, persistent CTAs, several queries per MMA row group);
* append_keys keeps the split of the touched blocks current.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import sparse_attention_token_misa_b200 as misa
from gpu_helpers import assert_no_device_error, dev, np_f, np_i, to_gpu, to_ora
from parity import check_selection
from workloads import make_decode, make_prefill

pytestmark = pytest.mark.gpu


def _check_split(means, hi, lo):
    assert hi.dtype == torch.bfloat16 and lo.dtype == torch.bfloat16
    assert torch.equal(hi, means.to(torch.bfloat16))
    assert torch.equal(lo, (means - hi.float()).to(torch.bfloat16))
    # together about 16 significant bits: |m - hi - lo| <= 2^-16 |m| (+ subnormal slack)
    rest = (means.double() - hi.double() - lo.double()).abs()
    assert torch.all(rest <= means.double().abs() * 2.0 ** -16 + 1e-30)


@pytest.mark.parametrize("nseq,L,B", [(1, 4096, 128), (3, 1000, 128), (2, 777, 64), (1, 5, 1), (2, 129, 128)])
def test_block_stats_split(nseq, L, B):
    wl = make_decode("bss", 21 + L, T=nseq, L=L, H=2, h=1, B=B, k=1, n_planted=0)
    keys = dev(wl.keys)
    plain = misa.block_stats(keys, B)
    means, hi, lo = misa.block_stats(keys, B, split=True)
    torch.cuda.synchronize()
    assert torch.equal(means, plain)          # the fp32 output does not change
    _check_split(means, hi, lo)


def _route_both(wl, L, B, q_block, h):
    g = to_gpu(wl)
    T, H, _ = wl.q.shape
    means, hi, lo = misa.block_stats(g["keys"], B, split=True)
    ws = misa.alloc_workspace(misa.workspace_bytes(1, T, H, L, B))
    h1, i1 = misa.route_heads(g["q"], g["w"], means, g["seq_of"], g["prefix_len"], L, B, q_block, h, workspace=ws)
    h1, i1 = h1.clone(), i1.clone()
    h2, i2 = misa.route_heads(g["q"], g["w"], None, g["seq_of"], g["prefix_len"], L, B, q_block, h, workspace=ws,
                              means_hi=hi, means_lo=lo)
    torch.cuda.synchronize()
    assert_no_device_error(ws)
    return means, (h1, i1), (h2, i2)


@pytest.mark.parametrize("T,L,H,h,B,q_block,mode", [
    (16, 4096, 64, 8, 128, 1, "decode"),       # one cluster per decision
    (300, 3000, 64, 8, 128, 1, "decode"),      # more decisions than one wave of clusters: persistent CTAs
    (130, 2000, 64, 8, 128, 64, "prefill"),    # shared cache, two queries per MMA row group
    (9, 100, 64, 64, 16, 4, "prefill"),
    (3, 777, 128, 5, 50, 2, "decode"),
])
def test_route_heads_split_is_bit_identical(T, L, H, h, B, q_block, mode):
    if mode == "decode":
        wl = make_decode("rts", 700 + T, T=T, L=L, H=H, h=h, B=B, k=16, n_planted=2)
    else:
        wl = make_prefill("rts", 700 + T, T=T, L=L, H=H, h=h, B=B, k=16, q_block=q_block, n_regions=1,
                          region_len=min(256, L // 2))
    means, (h1, i1), (h2, i2) = _route_both(wl, L, B, q_block, h)
    assert torch.equal(h1, h2)
    assert torch.equal(i1.view(torch.int32), i2.view(torch.int32))
    if T <= 16:
        # and the split path's heads are the oracle's
        o = to_ora(wl)
        m64 = np.stack([oracle.block_means(o["keys"][b], B) for b in range(o["keys"].shape[0])])
        _, imp_ora = oracle.route_heads(o["q"], o["w"], m64, o["seq_of"], o["prefix_len"], L, B, q_block, h)
        hg = np_i(h2)
        for gi in range(hg.shape[0]):
            check_selection(hg[gi], imp_ora[gi], h, what=f"heads g{gi}")


@pytest.mark.parametrize("T,L,H,B,m,shared", [(4, 5000, 64, 128, 8, False), (9, 3000, 32, 128, 6, True),
                                              (5, 2000, 64, 100, 4, True)])
def test_hisa_block_filter_split_is_bit_identical(T, L, H, B, m, shared):
    if shared:
        wl = make_prefill("hfs", 800 + L, T=T, L=L, H=H, h=H, B=B, k=16, q_block=1, n_regions=0, region_len=1,
                          first_pos=L // 3)
    else:
        wl = make_decode("hfs", 800 + L, T=T, L=L, H=H, h=H, B=B, k=16, n_planted=3, mode="hisa", m=m)
        wl.prefix_len[-1] = max(1, L // 2)
    g = to_gpu(wl)
    means, hi, lo = misa.block_stats(g["keys"], B, split=True)
    b1, c1, s1 = misa.hisa_block_filter(g["q"], g["w"], means, g["seq_of"], g["prefix_len"], L, B, m,
                                        want_scores=True)
    b1, c1, s1 = b1.clone(), c1.clone(), s1.clone()
    b2, c2, s2 = misa.hisa_block_filter(g["q"], g["w"], None, g["seq_of"], g["prefix_len"], L, B, m,
                                        want_scores=True, means_hi=hi, means_lo=lo)
    torch.cuda.synchronize()
    assert torch.equal(s1.view(torch.int32), s2.view(torch.int32))
    assert torch.equal(b1, b2) and torch.equal(c1, c2)


@pytest.mark.parametrize("B,n_new,lens", [(128, 1, [0, 127, 128, 1023]), (64, 200, [0, 64, 300, 824])])
def test_append_keys_keeps_split_current(B, n_new, lens):
    rng = np.random.default_rng(1300 + B)
    nseq, L_cap = len(lens), 1024
    M_cap = (L_cap + B - 1) // B
    cache = torch.from_numpy(rng.standard_normal((nseq, L_cap, 128), dtype=np.float32) / np.float32(np.sqrt(128)))
    new = torch.from_numpy(rng.standard_normal((nseq, n_new, 128), dtype=np.float32) / np.float32(np.sqrt(128)))
    keys = cache.to(torch.bfloat16).cuda()
    sentinel = 7.0
    means = torch.full((nseq, M_cap, 128), sentinel, dtype=torch.float32, device="cuda")
    hi = torch.full((nseq, M_cap, 128), sentinel, dtype=torch.bfloat16, device="cuda")
    lo = torch.full_like(hi, sentinel)
    lens_t = torch.tensor(lens, dtype=torch.int32, device="cuda")
    ws = misa.alloc_workspace(256)
    misa.append_keys(keys, lens_t, new.to(torch.bfloat16).cuda(), B, means, workspace=ws, means_hi=hi, means_lo=lo)
    torch.cuda.synchronize()
    assert misa.error_query(ws) == 0
    for b, l0 in enumerate(lens):
        l1 = l0 + n_new
        fm, fh, fl = misa.block_stats(keys[b:b + 1, :l1], B, split=True)
        touched = set(range(l0 // B, (l1 - 1) // B + 1))
        for j in range(M_cap):
            if j in touched:
                assert torch.equal(means[b, j], fm[0, j]) and torch.equal(hi[b, j], fh[0, j]), (b, j)
                assert torch.equal(lo[b, j], fl[0, j]), (b, j)
            else:
                assert bool(torch.all(hi[b, j] == sentinel)) and bool(torch.all(lo[b, j] == sentinel)), (b, j)


def test_indexer_with_split_means_matches_fp32():
    """The MISA indexer fed the (means, hi, lo) tuple selects the same tokens."""
    from sparse_attention_token_misa_b200.indexer import MisaIndexer
    T, L, H, h, B, k = 8, 5000, 64, 8, 128, 256
    wl = make_decode("ixs", 31, T=T, L=L, H=H, h=h, B=B, k=k, n_planted=3)
    g = to_gpu(wl)
    split = misa.block_stats(g["keys"], B, split=True)
    ix = MisaIndexer(T, H, h, L, B, k)
    a = ix.run(g["q"], g["w"], g["keys"], split[0], g["seq_of"], g["prefix_len"]).clone()
    b = ix.run(g["q"], g["w"], g["keys"], split, g["seq_of"], g["prefix_len"]).clone()
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    assert np_f(ix.importance).shape == (T, H)

"""misa_index_score_blocks (the HISA page, section 三, Stage 2: the token
indexer over the tokens of the chosen blocks) on the GPU.

Reading the chosen blocks' keys as whole tiles must give, bit for bit, what
misa_index_score gives on the candidate list cand[t][i*B + r] = blocks[t][i]*B
+ r (-1 past the prefix or for an empty block slot), which the other tests pin
to the oracle: the same epilogue (ReLU, head weights, heads summed in order)
over the same keys.  Covers blocks of 64 and 128 keys, blocks the prefix cuts,
empty slots anywhere in the list, a shared cache, a last tile past the list,
and an out-of-range block id (error bit, -inf)."""
import numpy as np
import pytest
import torch

import sparse_attention_token_misa_b200 as misa
from gpu_helpers import assert_no_device_error, to_gpu
from workloads import make_decode, make_workload

pytestmark = pytest.mark.gpu


def _cand_of(blocks, B, plen, L):
    T, m = blocks.shape
    r = torch.arange(B, device=blocks.device, dtype=torch.int64)
    ids = blocks.to(torch.int64).unsqueeze(-1) * B + r
    lim = torch.clamp(plen.to(torch.int64), 0, L).view(T, 1, 1)
    ok = (blocks.unsqueeze(-1) >= 0) & (ids < lim)
    return torch.where(ok, ids, torch.full_like(ids, -1)).view(T, m * B).to(torch.int32)


def _both(g, blocks, B, L):
    ws = misa.alloc_workspace(256)
    S_b = misa.index_score_blocks(g["q"], g["w"], g["keys"], g["seq_of"], g["prefix_len"], blocks, B, workspace=ws)
    cand = _cand_of(blocks, B, g["prefix_len"], L)
    S_c = misa.index_score(g["q"], g["w"], g["keys"], g["seq_of"], g["prefix_len"], cand=cand)
    torch.cuda.synchronize()
    return S_b, S_c, ws


@pytest.mark.parametrize("B,m", [(128, 64), (64, 128)])
def test_blocks_equal_candidate_gather_on_the_filter_output(B, m):
    wl = make_workload("hisa_decode_L131072")
    g = to_gpu(wl)
    means = misa.block_stats(g["keys"], B, split=True)
    blocks, cand, _ = misa.hisa_block_filter(g["q"], g["w"], means[0], g["seq_of"], g["prefix_len"], wl.L, B, m,
                                             means_hi=means[1], means_lo=means[2])
    S_b, S_c, ws = _both(g, blocks, B, wl.L)
    assert_no_device_error(ws)
    assert torch.equal(_cand_of(blocks, B, g["prefix_len"], wl.L), cand)   # the filter's list is the same
    assert torch.equal(S_b, S_c)


@pytest.mark.parametrize("B", [64, 128])
@pytest.mark.parametrize("shared", [False, True])
def test_blocks_cut_empty_and_ragged(B, shared):
    T, L, H = 5, 5000, 64
    wl = make_decode("sb", 17 + B, T=T, L=L, H=H, h=8, B=B, k=100, n_planted=2, shared_cache=shared)
    rng = np.random.default_rng(B)
    wl.prefix_len[:] = torch.from_numpy(rng.integers(1, L + 1, size=T).astype(np.int32))
    wl.prefix_len[0] = L
    g = to_gpu(wl)
    nb = (L + B - 1) // B
    m = 7
    blk = np.full((T, m), -1, dtype=np.int32)
    for t in range(T):
        vis = (int(wl.prefix_len[t]) + B - 1) // B
        ids = np.sort(rng.choice(nb, size=min(m, nb), replace=False))
        blk[t, :len(ids)] = ids
        blk[t, rng.integers(0, m)] = -1                       # an empty slot anywhere
        blk[t, 0] = vis - 1                                   # the block the prefix cuts (or the last)
    blk[1, :] = -1                                            # a query with no block at all
    blocks = torch.from_numpy(blk).cuda()
    S_b, S_c, ws = _both(g, blocks, B, L)
    assert_no_device_error(ws)
    assert torch.equal(S_b, S_c)
    assert torch.isinf(S_b[1]).all() and (S_b[1] < 0).all()


def test_blocks_out_of_range_id_is_reported():
    T, L, H, B = 2, 1000, 64, 128
    wl = make_decode("sbe", 5, T=T, L=L, H=H, h=8, B=B, k=10, n_planted=1)
    g = to_gpu(wl)
    blocks = torch.tensor([[0, 1, 99], [2, -1, 3]], dtype=torch.int32, device="cuda")   # 99 >= ceil(1000 / 128)
    ws = misa.alloc_workspace(256)
    S = misa.index_score_blocks(g["q"], g["w"], g["keys"], g["seq_of"], g["prefix_len"], blocks, B, workspace=ws)
    torch.cuda.synchronize()
    assert misa.error_query(ws) & misa._native.DEVERR_BAD_INDEX
    assert torch.isinf(S[0, 2 * B:]).all() and (S[0, 2 * B:] < 0).all()
    assert torch.isfinite(S[0, :2 * B]).all()

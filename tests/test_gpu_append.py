"""misa_append_keys on the GPU: new keys land in the cache, the blocks they
touch get the oracle's block means (and bit for bit misa_block_stats' on the
longer cache), every other block and row is left alone."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import sparse_attention_token_misa_b200 as misa
from gpu_helpers import f64, np_f

pytestmark = pytest.mark.gpu


def _bf16_keys(rng, shape):
    return torch.from_numpy((rng.standard_normal(shape, dtype=np.float32) / np.float32(np.sqrt(128)))).to(
        torch.bfloat16)


@pytest.mark.parametrize("B,n_new,lens", [
    (128, 1, [0, 1, 127, 128, 500, 1023]),     # decode: one key per sequence, block edges
    (128, 3, [0, 126, 127, 255, 700, 1021]),   # a few keys crossing a block edge
    (64, 200, [0, 1, 64, 300, 500, 824]),      # a long append spanning several blocks
    (7, 5, [0, 6, 7, 13, 99, 1019]),           # odd block size
])
def test_append_keys(B, n_new, lens):
    rng = np.random.default_rng(900 + B + n_new)
    nseq, L_cap = len(lens), 1024
    M_cap = (L_cap + B - 1) // B
    cache = _bf16_keys(rng, (nseq, L_cap, 128))
    new = _bf16_keys(rng, (nseq, n_new, 128))
    sentinel = np.float32(12345.0)
    keys = cache.cuda()
    means = torch.full((nseq, M_cap, 128), float(sentinel), dtype=torch.float32, device="cuda")
    lens_t = torch.tensor(lens, dtype=torch.int32, device="cuda")
    ws = misa.alloc_workspace(256)
    misa.append_keys(keys, lens_t, new.cuda(), B, means, workspace=ws)
    torch.cuda.synchronize()
    assert misa.error_query(ws) == 0
    got_keys = keys.cpu()
    got_means = np_f(means)
    for b, l0 in enumerate(lens):
        l1 = l0 + n_new
        expect = cache[b].clone()
        expect[l0:l1] = new[b]
        assert torch.equal(got_keys[b], expect), b           # exact copy, nothing else written
        k64 = f64(expect[:l1])
        ref = oracle.block_means(k64, B)
        touched = range(l0 // B, (l1 - 1) // B + 1)
        for j in range(M_cap):
            if j in touched:
                blk = k64[j * B:min((j + 1) * B, l1)]
                allow = 2e-5 * np.abs(blk).mean(axis=0) + 1e-12
                assert np.all(np.abs(got_means[b, j] - ref[j]) <= allow), (b, j)
            else:
                assert np.all(got_means[b, j] == sentinel), (b, j)  # untouched
        # the same blocks as a full recompute over the longer cache, bit for bit
        full = np_f(misa.block_stats(keys[b:b + 1, :l1], B))[0]
        for j in touched:
            assert np.array_equal(got_means[b, j], full[j]), (b, j)


def test_append_keys_bad_length_is_recorded():
    rng = np.random.default_rng(7)
    nseq, L_cap, B, n_new = 3, 256, 128, 4
    cache = _bf16_keys(rng, (nseq, L_cap, 128))
    keys = cache.cuda()
    means = torch.zeros((nseq, 2, 128), dtype=torch.float32, device="cuda")
    lens_t = torch.tensor([10, 254, -1], dtype=torch.int32, device="cuda")   # 254 + 4 > 256; -1 < 0
    ws = misa.alloc_workspace(256)
    misa.append_keys(keys, lens_t, _bf16_keys(rng, (nseq, n_new, 128)).cuda(), B, means, workspace=ws)
    torch.cuda.synchronize()
    assert misa.error_query(ws) & 8                      # MISA_DEVERR_BAD_LEN
    got = keys.cpu()
    assert torch.equal(got[1], cache[1]) and torch.equal(got[2], cache[2])   # skipped, untouched
    assert not torch.equal(got[0], cache[0])                                  # the valid one was appended

"""misa_sparse_mla (attention over the selected tokens) against the fp64 oracle.

Tolerance, from the arithmetic: scores are fp32 from bf16 inputs (relative error
far below 1e-5), each weight p is rounded to bf16 before the value product
(relative 2^-9, so the normalised weights move by at most about 2^-8 of
themselves) and the output is rounded to bf16 (2^-9 of |out|).  With
A = sum_i p_i |v_i| / sum_i p_i (the oracle's abs-weighted value scale) the
error is at most (2^-8 + 2^-9) A; the tests allow 8e-3 A + 1e-6.  The
log-sum-exp carries the bf16 rounding of the weights in its sum: 3e-3.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import sparse_attention_token_misa_b200 as misa
from workloads import make_mla, mla_cache_rows

pytestmark = pytest.mark.gpu

DV = 512


def _f64(x):
    return x.to(torch.float64).numpy()


def _run(batch, idx=None, want_lse=True):
    idx = batch.idx if idx is None else idx
    T, Hq, _ = batch.q.shape
    ws = misa.alloc_workspace(misa.workspace_bytes(misa._native.OP_SPARSE_MLA, T, Hq, 0, 0, idx.shape[1]))
    out, lse = misa.sparse_mla(batch.q.cuda(), batch.kv.cuda(), batch.seq_of.cuda(), idx.cuda(), batch.scale,
                               want_lse=want_lse, workspace=ws)
    torch.cuda.synchronize()
    return out.float().cpu().numpy(), (lse.cpu().numpy() if lse is not None else None), misa.error_query(ws)


def _check(out, lse, ref_out, ref_lse, A, what=""):
    err = np.abs(out - ref_out)
    bound = 8e-3 * A + 1e-6
    bad = err > bound
    assert not bad.any(), f"{what}: {bad.sum()} outputs off, worst excess {(err - bound).max():.3g}"
    if lse is not None:
        fin = np.isfinite(ref_lse)
        assert np.array_equal(np.isneginf(lse), ~fin), what
        assert np.all(np.abs(lse[fin] - ref_lse[fin]) <= 3e-3 + 1e-6 * np.abs(ref_lse[fin])), what


@pytest.mark.parametrize("T,Hq,L,nseq,k,n_pad,scale_mult,shared", [
    (3, 128, 3000, 3, 700, 50, 1.0, False),     # three chunks, ragged, padded tail
    (2, 16, 1000, 1, 100, 0, 1.0, True),        # one chunk, few heads, one shared cache
    (4, 64, 5000, 2, 1300, 300, 4.0, False),    # peaked weights; a chunk of padding only
    (2, 128, 600, 2, 256, 0, 0.0, False),       # zero scale: the plain mean of the values
    (2, 128, 100000, 2, 2048, 0, 1.0, False),   # ids beyond 65535, eight chunks
    (1, 128, 300, 1, 17, 0, 1.0, False),        # k not a multiple of 16
])
def test_sparse_mla_parity(T, Hq, L, nseq, k, n_pad, scale_mult, shared):
    b = make_mla(40 + T + k, T, Hq, L, nseq, k, n_pad=n_pad, shared_cache=shared)
    b.scale = b.scale * scale_mult
    out, lse, err = _run(b)
    assert err == 0
    q64, kv64, so, idx = _f64(b.q), _f64(b.kv), b.seq_of.numpy(), b.idx.numpy()
    ref_out, ref_lse = oracle.sparse_attention(q64, kv64, so, idx, b.scale, DV)
    A = oracle.sparse_attention_abs_weights(q64, kv64, so, idx, b.scale, DV)
    _check(out, lse, ref_out, ref_lse, A, what=f"T{T} Hq{Hq} k{k}")


def test_sparse_mla_empty_query_and_empty_chunk():
    b = make_mla(77, 3, 128, 2000, 3, 768)
    idx = b.idx.clone()
    idx[0] = -1                      # no valid slot: zeros, lse -inf
    idx[1, 256:512] = -1             # its second chunk is empty
    out, lse, err = _run(b, idx)
    assert err == 0
    assert np.all(out[0] == 0.0) and np.all(np.isneginf(lse[0]))
    q64, kv64, so = _f64(b.q), _f64(b.kv), b.seq_of.numpy()
    ref_out, ref_lse = oracle.sparse_attention(q64, kv64, so, idx.numpy(), b.scale, DV)
    A = oracle.sparse_attention_abs_weights(q64, kv64, so, idx.numpy(), b.scale, DV)
    _check(out, lse, ref_out, ref_lse, A)


def test_sparse_mla_single_slot_is_exact():
    # one listed token: weight 1, the output is that row's value part exactly
    b = make_mla(78, 4, 128, 500, 2, 300)
    idx = torch.full_like(b.idx, -1)
    idx[:, 123] = torch.tensor([5, 17, 499, 0], dtype=torch.int32)
    out, _, err = _run(b, idx, want_lse=False)
    assert err == 0
    for t in range(4):
        row = b.kv[int(b.seq_of[t]), int(idx[t, 123]), :DV].float().numpy()
        assert np.array_equal(out[t], np.broadcast_to(row, out[t].shape)), t


def test_sparse_mla_bad_index_is_recorded():
    b = make_mla(79, 2, 128, 800, 2, 300)
    idx = b.idx.clone()
    idx[0, 3] = 800          # == L
    idx[1, 7] = -5
    out, lse, err = _run(b, idx)
    assert err & misa._native.DEVERR_BAD_INDEX
    clean = idx.numpy().copy()
    clean[0, 3] = -1
    clean[1, 7] = -1
    q64, kv64, so = _f64(b.q), _f64(b.kv), b.seq_of.numpy()
    ref_out, ref_lse = oracle.sparse_attention(q64, kv64, so, clean, b.scale, DV)
    A = oracle.sparse_attention_abs_weights(q64, kv64, so, clean, b.scale, DV)
    _check(out, lse, ref_out, ref_lse, A)


def test_sparse_mla_full_size_sampled():
    """The decode shape the bench times (32 sequences x L = 32768, 128 heads,
    k = 2048), sampled queries against the oracle; every output finite and
    inside the range of its values."""
    T, Hq, L, k = 32, 128, 32768, 2048
    b = make_mla(2, T, Hq, L, T, k)
    out, lse, err = _run(b)
    assert err == 0
    assert np.all(np.isfinite(out)) and np.all(np.isfinite(lse))
    for t in (0, 13, 31):
        s = int(b.seq_of[t])
        rows = mla_cache_rows(b.seed, s, L)
        assert torch.equal(rows, b.kv[s])
        kv64 = rows.to(torch.float64).numpy()[None]
        q64 = _f64(b.q[t:t + 1])
        idx = b.idx[t:t + 1].numpy()
        ref_out, ref_lse = oracle.sparse_attention(q64, kv64, np.zeros(1, np.int64), idx, b.scale, DV)
        A = oracle.sparse_attention_abs_weights(q64, kv64, np.zeros(1, np.int64), idx, b.scale, DV)
        _check(out[t:t + 1], lse[t:t + 1], ref_out, ref_lse, A, what=f"t{t}")

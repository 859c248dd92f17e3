"""Pins that tie the fp64 sparse-attention oracle to something other than
itself.  Every check takes the oracle module (or a deliberately broken copy of
it, see test_oracle_attention.py) and raises if it disagrees.

Kinds of pin:
* the hand-worked case in tests/golden/hand_case_sparse_attention.json;
* closed forms: one listed slot gives that row's value; equal scores give the
  plain mean of the values; a zero scale gives the plain mean; a very large
  scale with well separated scores gives the value of the best row;
* a library routine: torch's scaled_dot_product_attention (CPU, float64) over
  the whole cache with a boolean mask of the listed tokens, and scipy's
  logsumexp for the log-sum-exp;
* invariants: the order of the slots and where the empty slots sit do not
  matter; a shift of every key along coordinates outside the value part that
  moves all scores of a head by the same amount changes nothing.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_case_sparse_attention.json")


def _rand_case(seed, T=3, Hq=4, L=40, d_qk=12, d_v=8, k=9, nseq=2):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((T, Hq, d_qk))
    kv = rng.standard_normal((nseq, L, d_qk))
    seq_of = rng.integers(0, nseq, size=T)
    idx = np.stack([rng.choice(L, size=k, replace=False) for _ in range(T)]).astype(np.int64)
    idx[:, -2:] = -1   # padding
    return q, kv, seq_of, idx, d_v


def check_attn_hand_case(orc):
    with open(GOLDEN, encoding="utf-8") as f:
        g = json.load(f)
    rows = np.asarray(g["rows"], dtype=np.float64)[None]
    qh = np.array([[0.0, math.log(3.0), 0.0], [0.0, 0.0, math.log(2.0)]])
    q = np.stack([qh, qh, qh])
    idx = np.asarray(g["idx"])
    out, lse = orc.sparse_attention(q, rows, np.zeros(3, dtype=np.int64), idx, g["scale"], g["d_v"])
    assert np.allclose(out, np.asarray(g["out"]), rtol=0, atol=1e-12), out
    assert np.allclose(lse[0], [math.log(5.0), math.log(4.0)], atol=1e-12)
    assert np.all(np.isneginf(lse[1]))
    assert np.allclose(lse[2], [0.0, math.log(2.0)], atol=1e-12)


def check_attn_single_slot(orc):
    q, kv, seq_of, idx, d_v = _rand_case(1)
    idx[:] = -1
    idx[:, 3] = [5, 17, 39]
    out, lse = orc.sparse_attention(q, kv, seq_of, idx, 0.7, d_v)
    for t in range(q.shape[0]):
        row = kv[seq_of[t], idx[t, 3]]
        assert np.array_equal(out[t], np.broadcast_to(row[:d_v], out[t].shape))
        assert np.allclose(lse[t], 0.7 * (q[t] @ row), atol=1e-12)


def check_attn_equal_scores_is_mean(orc):
    q, kv, seq_of, idx, d_v = _rand_case(2)
    # queries blind to the value part; every row shares one non-value part
    q[:, :, :d_v] = 0.0
    kv[:, :, d_v:] = kv[0, 0, d_v:]
    out, _ = orc.sparse_attention(q, kv, seq_of, idx, 1.3, d_v)
    for t in range(q.shape[0]):
        ids = idx[t][idx[t] >= 0]
        mean = kv[seq_of[t], ids, :d_v].mean(axis=0)
        assert np.allclose(out[t], mean[None], atol=1e-12)


def check_attn_zero_scale_is_mean(orc):
    q, kv, seq_of, idx, d_v = _rand_case(3)
    out, lse = orc.sparse_attention(q, kv, seq_of, idx, 0.0, d_v)
    for t in range(q.shape[0]):
        ids = idx[t][idx[t] >= 0]
        assert np.allclose(out[t], kv[seq_of[t], ids, :d_v].mean(axis=0)[None], atol=1e-12)
        assert np.allclose(lse[t], math.log(ids.size), atol=1e-12)


def check_attn_large_scale_is_argmax(orc):
    q, kv, seq_of, idx, d_v = _rand_case(4)
    out, _ = orc.sparse_attention(q, kv, seq_of, idx, 1e4, d_v)
    for t in range(q.shape[0]):
        ids = idx[t][idx[t] >= 0]
        s = q[t] @ kv[seq_of[t], ids].T
        best = ids[np.argmax(s, axis=1)]
        gap = np.sort(s, axis=1)[:, -1] - np.sort(s, axis=1)[:, -2]
        assert gap.min() > 1e-2   # the seeded case is well separated
        assert np.allclose(out[t], kv[seq_of[t], best, :d_v], atol=1e-9)


def check_attn_matches_torch_sdpa(orc):
    import torch

    q, kv, seq_of, idx, d_v = _rand_case(5, T=4, Hq=3, L=50, d_qk=16, d_v=10, k=12)
    scale = 0.37
    out, _ = orc.sparse_attention(q, kv, seq_of, idx, scale, d_v)
    L = kv.shape[1]
    for t in range(q.shape[0]):
        mask = np.zeros(L, dtype=bool)
        mask[idx[t][idx[t] >= 0]] = True
        K = torch.from_numpy(kv[seq_of[t]])[None, None]          # [1, 1, L, d_qk]
        V = K[..., :d_v]
        Q = torch.from_numpy(q[t])[None, :, None]                 # [1, Hq, 1, d_qk]
        ref = torch.nn.functional.scaled_dot_product_attention(
            Q, K.expand(1, q.shape[1], L, -1), V.expand(1, q.shape[1], L, -1),
            attn_mask=torch.from_numpy(mask)[None, None, None], scale=scale)
        assert np.allclose(out[t], ref[0, :, 0].numpy(), atol=1e-12), t


def check_attn_lse_library(orc):
    from scipy.special import logsumexp

    q, kv, seq_of, idx, d_v = _rand_case(6)
    _, lse = orc.sparse_attention(q, kv, seq_of, idx, 0.9, d_v)
    for t in range(q.shape[0]):
        ids = idx[t][idx[t] >= 0]
        s = 0.9 * (q[t] @ kv[seq_of[t], ids].T)
        assert np.allclose(lse[t], logsumexp(s, axis=1), atol=1e-12)


def check_attn_slot_order_invariant(orc):
    q, kv, seq_of, idx, d_v = _rand_case(7)
    out, lse = orc.sparse_attention(q, kv, seq_of, idx, 0.5, d_v)
    rng = np.random.default_rng(70)
    perm = np.stack([rng.permutation(idx.shape[1]) for _ in range(idx.shape[0])])
    idx2 = np.take_along_axis(idx, perm, axis=1)
    out2, lse2 = orc.sparse_attention(q, kv, seq_of, idx2, 0.5, d_v)
    assert np.allclose(out, out2, atol=1e-12) and np.allclose(lse, lse2, atol=1e-12)


def check_attn_nonvalue_shift_invariant(orc):
    q, kv, seq_of, idx, d_v = _rand_case(8)
    out, _ = orc.sparse_attention(q, kv, seq_of, idx, 0.8, d_v)
    kv2 = kv.copy()
    kv2[:, :, d_v:] += np.random.default_rng(80).standard_normal(kv.shape[2] - d_v)  # same shift for every row
    out2, _ = orc.sparse_attention(q, kv2, seq_of, idx, 0.8, d_v)
    assert np.allclose(out, out2, atol=1e-10)


def check_attn_empty_query(orc):
    q, kv, seq_of, idx, d_v = _rand_case(9)
    idx[1] = -1
    out, lse = orc.sparse_attention(q, kv, seq_of, idx, 1.0, d_v)
    assert np.all(out[1] == 0.0) and np.all(np.isneginf(lse[1]))
    assert np.all(np.isfinite(out[0])) and np.all(np.isfinite(lse[0]))


def check_attn_abs_weights(orc):
    # the error-scale helper is the attention of |v| under the same weights
    q, kv, seq_of, idx, d_v = _rand_case(10)
    a = orc.sparse_attention_abs_weights(q, kv, seq_of, idx, 0.6, d_v)
    kv_abs = kv.copy()
    kv_abs[:, :, :d_v] = np.abs(kv[:, :, :d_v])
    q2 = q.copy()
    out, _ = orc.sparse_attention(q2, kv_abs, seq_of, idx, 0.6, d_v)
    # equal only where the scores do not involve the value part: compare on a
    # query blind to it
    q3 = q.copy()
    q3[:, :, :d_v] = 0.0
    a3 = orc.sparse_attention_abs_weights(q3, kv, seq_of, idx, 0.6, d_v)
    out3, _ = orc.sparse_attention(q3, kv_abs, seq_of, idx, 0.6, d_v)
    assert np.allclose(a3, out3, atol=1e-12)
    assert np.all(a >= 0.0) and np.all(a + 1e-12 >= np.abs(orc.sparse_attention(q, kv, seq_of, idx, 0.6, d_v)[0]))
    assert out.shape == a.shape


ATTN_CHECKS = [
    check_attn_hand_case, check_attn_single_slot, check_attn_equal_scores_is_mean, check_attn_zero_scale_is_mean,
    check_attn_large_scale_is_argmax, check_attn_matches_torch_sdpa, check_attn_lse_library,
    check_attn_slot_order_invariant, check_attn_nonvalue_shift_invariant, check_attn_empty_query,
    check_attn_abs_weights,
]

"""Plain fp64 CPU oracle for the sparse attention that consumes the indexer's
token indices.

TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
benchmark's CPU-baseline leg may import it; the library never does.

What it computes, and where the pages place it
----------------------------------------------
HISA-zh -- "HISA：为什么长文本理解的关键，藏在图书馆的分类索引里？"
(zhichai.net):

* section 二 (DSA 的工作原理): DSA runs in two stages, an indexer that picks k
  tokens per query, then sparse attention computed over those k tokens only;
* section 四 (Drop-in Replacement): the attention operator (Sparse MLA) takes
  the k token indices unchanged, over the unchanged KV cache;
* section 七 (Kernel-level vs End-to-end): the indexer is one part of the
  total latency, and its share grows with the context length.

The pages print no attention formula; the attention over a set of tokens is the
textbook one, for query head h of query t over the listed slots i:

    s[h, i] = scale * (q[t, h] . kv[seq_of[t], idx[t, i]])
    p[h, i] = exp(s[h, i] - max_i s[h, i])
    out[t, h] = sum_i p[h, i] * kv[seq_of[t], idx[t, i], :d_v] / sum_i p[h, i]

Readings taken where the pages are silent (each the plainest one):
* the KV cache holds one latent row per token shared by every query head
  (multi-query form of MLA with the up-projections absorbed into the query, the
  form a DeepSeek-V3.2-shaped model decodes with): keys are the whole row
  (d_qk = 576: 512 latent + 64 rotary), values are its first d_v = 512 entries;
* an index slot of -1 is empty (the indexer's padding) and takes no part; every
  other slot takes part once (the indexer never repeats a token; if a caller
  does, the token counts once per slot);
* a query with no valid slot gets a zero output (and log-sum-exp -inf);
* the scale is an input (the model's softmax scale).

Everything is evaluated in float64 on the values the GPU sees (bf16 inputs
widened to fp64).
"""
from __future__ import annotations

import numpy as np

__all__ = ["sparse_attention", "sparse_attention_abs_weights"]


def _slots(idx_row: np.ndarray, L: int) -> np.ndarray:
    ids = np.asarray(idx_row, dtype=np.int64)
    return ids[(ids >= 0) & (ids < L)]


def sparse_attention(q, kv, seq_of, idx, scale: float, d_v: int):
    """Attention of every query head over its query's listed tokens.

    q [T, Hq, d_qk], kv [nseq, L, d_qk], seq_of [T], idx [T, k] (-1 = empty).
    Returns (out [T, Hq, d_v], lse [T, Hq]) with lse = log sum_i exp(s[h, i]).
    """
    q = np.asarray(q, dtype=np.float64)
    kv = np.asarray(kv, dtype=np.float64)
    T, Hq, _ = q.shape
    L = kv.shape[1]
    out = np.zeros((T, Hq, d_v))
    lse = np.full((T, Hq), -np.inf)
    for t in range(T):
        ids = _slots(idx[t], L)
        if ids.size == 0:
            continue
        rows = kv[int(seq_of[t])][ids]          # [n, d_qk]: keys
        vals = rows[:, :d_v]                    # [n, d_v]: values, the latent part
        s = scale * (q[t] @ rows.T)             # [Hq, n]
        m = s.max(axis=1, keepdims=True)
        p = np.exp(s - m)
        l = p.sum(axis=1)
        out[t] = (p @ vals) / l[:, None]
        lse[t] = m[:, 0] + np.log(l)
    return out, lse


def sparse_attention_abs_weights(q, kv, seq_of, idx, scale: float, d_v: int):
    """sum_i p[h, i] |v_i| / sum_i p[h, i] per output element: the scale of the
    rounding error a weighted average of the values can carry (used to state
    the tolerance of a low-precision evaluation)."""
    q = np.asarray(q, dtype=np.float64)
    kv = np.asarray(kv, dtype=np.float64)
    T, Hq, _ = q.shape
    L = kv.shape[1]
    out = np.zeros((T, Hq, d_v))
    for t in range(T):
        ids = _slots(idx[t], L)
        if ids.size == 0:
            continue
        rows = kv[int(seq_of[t])][ids]
        s = scale * (q[t] @ rows.T)
        p = np.exp(s - s.max(axis=1, keepdims=True))
        out[t] = (p @ np.abs(rows[:, :d_v])) / p.sum(axis=1)[:, None]
    return out

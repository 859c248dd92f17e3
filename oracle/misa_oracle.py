"""Plain fp64 CPU oracle for the MISA / MISA-dagger / HISA token indexer.

TEST INFRASTRUCTURE ONLY.  This module is the checker the CUDA path is compared
against.  Only the test suite, the smoke check and the benchmark's CPU-baseline
(reference) leg may import it; the library itself never does, and there is no
CPU fallback anywhere in the product path.

What it computes, and where the pages define it
------------------------------------------------
Pages cited (short names used throughout this file):

* MISA-gist  -- "MISA: Mixture of Indexer Sparse Attention for Long-Context LLM
  Inference" (gist.science, Spanish / Italian / French editions of one text),
  technical summary: "Problem statement", "Methodology: MISA",
  "Hierarchical variant (MISA-dagger)", "Limitations".
* MISA-zh    -- "MISA：面向长上下文LLM推理的索引器稀疏注意力混合专家机制"
  (zingnex.cn forum thread), sections "DeepSeek稀疏注意力（DSA）的突破",
  "核心架构：轻量级路由器", "层次化变体".
* HISA-zh    -- "HISA：为什么长文本理解的关键，藏在图书馆的分类索引里？"
  (zhichai.net), sections "二、DSA 的工作原理", "三、HISA 的两层搜索"
  (Stage 1 / Stage 2), "四、Drop-in Replacement", "五、选择一致性：IoU 分析".

The pages print no scoring formula.  The indexer score used here is
    S[t, s] = sum over active heads h of  w[t, h] * ReLU(q[t, h] . k[s])
with no extra scale.  Everything is evaluated in float64 on the exact values the
GPU sees (bf16 inputs widened to fp64, fp32 head weights widened to fp64).

Readings taken where the pages are silent (each is the plainest one):
* block statistic = arithmetic mean of the keys of a block; the last, partial
  block averages over the tokens it really holds;
* router affinity of head h with block j = the indexer's own per-head term at
  the block mean, w * ReLU(q . mean_j); head importance = plain (signed) sum over
  the visible blocks and over the queries that share one routing decision;
* a block is visible to a routing decision iff all of its tokens lie inside the
  prefix of the first query of the query block;
* selections are hard top-h / top-m / top-k under the total order
  (value descending, lower index first); selected ids are returned in ascending
  order; -0.0 ranks equal to +0.0;
* key s is visible to query t iff 0 <= s < prefix_len[t]; masked scores are -inf
  and are never selected; when fewer than k entries are valid, all valid ids are
  returned and the rest of the row is -1.

Parity of the router against the paper's own (unpublished) router is unpinned:
the pages do not say how the per-head block affinities are aggregated, so the
reading above is this library's definition of the MISA router.
"""
from __future__ import annotations

import math

import numpy as np

__all__ = [
    "block_means",
    "num_windows",
    "window_stats",
    "visible_blocks",
    "head_block_affinity",
    "route_heads",
    "index_scores",
    "candidate_scores",
    "topk_ascending",
    "topk_rows",
    "dense_indexer",
    "misa_indexer",
    "misa_dagger_indexer",
    "hisa_block_filter",
    "hisa_indexer",
    "iou",
]


# --------------------------------------------------------------------------
# Block statistics
# --------------------------------------------------------------------------
def block_means(keys: np.ndarray, B: int) -> np.ndarray:
    """Mean-pooled key blocks.

    MISA-gist, Methodology (block-aggregated router): the prefix is split into
    M = ceil(L / B) blocks and each block is summarised by the mean of its
    indexer keys.  HISA-zh, Stage 1: each block of B consecutive tokens is
    represented by one mean-pooled vector.

    keys: [L, d] float64.  Returns [M, d] float64.  The last block averages over
    the L - (M-1)*B tokens it holds.
    """
    L, d = keys.shape
    M = (L + B - 1) // B
    out = np.zeros((M, d), dtype=np.float64)
    for j in range(M):
        lo = j * B
        hi = min(lo + B, L)
        out[j] = keys[lo:hi].sum(axis=0) / float(hi - lo)
    return out


def num_windows(L: int, B: int, S: int) -> int:
    """Number of B-token windows that start every S tokens (1 <= S <= B).

    HISA-zh, 七 (局限与未来方向, 潜在改进) names overlapping blocks as a way to
    soften block-boundary effects; the pages give no layout.  Reading: window j
    covers tokens [j*S, min(j*S + B, L)); windows are added while the previous
    one does not reach the end of the cache, so every token is covered and no
    window lies inside another one's extent: M = 1 + ceil(max(L - B, 0) / S).
    With S = B this is the plain M = ceil(L / B) blocks.
    """
    return 1 + (max(L - B, 0) + S - 1) // S


def window_stats(keys: np.ndarray, B: int, S: int | None = None, pool: str = "mean") -> np.ndarray:
    """Block statistics over windows of B tokens starting every S tokens.

    pool = "mean": the arithmetic mean of the window's keys (MISA-gist,
    Methodology; HISA-zh, Stage 1: mean pooling).  pool = "max": the
    coordinate-wise maximum of the window's keys (HISA-zh, 七, 潜在改进: max
    pooling in place of mean pooling; the plainest reading of max pooling a
    set of vectors).  S = None means S = B (non-overlapping blocks).  A window
    cut by the end of the cache pools the tokens it holds.

    keys: [L, d].  Returns [num_windows(L, B, S), d] float64.
    """
    L, d = keys.shape
    S = B if S is None else S
    M = num_windows(L, B, S)
    out = np.zeros((M, d), dtype=np.float64)
    for j in range(M):
        lo = j * S
        hi = min(lo + B, L)
        win = keys[lo:hi]
        out[j] = win.max(axis=0) if pool == "max" else win.sum(axis=0) / float(hi - lo)
    return out


def visible_blocks(prefix_len: int, L: int, B: int, S: int | None = None) -> np.ndarray:
    """Ids of the blocks (windows) a routing decision may look at.

    Block j is visible iff every token it holds is inside the prefix, i.e.
    min((j + 1) * B, L) <= prefix_len.  At decode prefix_len == L, so every block
    (the partial last one included) is visible.  With windows every S tokens
    the same rule holds for window j = [j*S, min(j*S + B, L)).
    """
    S = B if S is None else S
    M = num_windows(L, B, S)
    ends = np.minimum(np.arange(M) * S + B, L)
    return np.nonzero(ends <= prefix_len)[0]


# --------------------------------------------------------------------------
# Router (MISA) and block filter (HISA) share one affinity
# --------------------------------------------------------------------------
def head_block_affinity(q_t: np.ndarray, w_t: np.ndarray, means: np.ndarray) -> np.ndarray:
    """A[h, j] = w[h] * ReLU(q[h] . mean_j).

    MISA-gist, Methodology: the router computes per-head affinities against
    block-aggregated keys instead of individual tokens.  HISA-zh, Stage 1: the
    query is scored against the block representatives only.

    q_t: [H, d], w_t: [H], means: [M, d] -> [H, M].
    """
    dots = q_t @ means.T
    return w_t[:, None] * np.maximum(dots, 0.0)


def _top_ids(values: np.ndarray, count: int) -> np.ndarray:
    """Ids of the `count` largest values (ties: lower id first), ascending."""
    n = values.shape[0]
    if count >= n:
        return np.arange(n, dtype=np.int64)
    order = sorted(range(n), key=lambda i: (-values[i], i))
    return np.sort(np.asarray(order[:count], dtype=np.int64))


def route_heads(q, w, means, seq_of, prefix_len, L, B, q_block, h, S=None):
    """Per-query-block head routing (MISA router).

    MISA-gist, Methodology: the router aggregates the per-head block affinities
    into an importance per head for the current query and keeps the top-h heads;
    MISA-zh, 核心架构 (step 2): 8 of 64 heads are kept per query.

    q: [T, H, d]; w: [T, H]; means: [nseq, M, d]; seq_of, prefix_len: [T].
    Queries [g*q_block, min((g+1)*q_block, T)) share one decision g; block
    visibility follows the first query of the block.  importance[g, h] is the sum
    over the block's queries and the visible blocks of A[h, j].  S: the window
    stride of the statistics (None: S = B, plain blocks).
    Returns heads [G, min(h, H)] (ascending ids) and importance [G, H].
    """
    T, H, _ = q.shape
    G = (T + q_block - 1) // q_block
    keep = min(h, H)
    heads = np.zeros((G, keep), dtype=np.int64)
    importance = np.zeros((G, H), dtype=np.float64)
    for g in range(G):
        t0 = g * q_block
        t1 = min(t0 + q_block, T)
        vis = visible_blocks(int(prefix_len[t0]), L, B, S)
        for t in range(t0, t1):
            A = head_block_affinity(q[t], w[t], means[seq_of[t]][vis])
            importance[g] += A.sum(axis=1)
        heads[g] = _top_ids(importance[g], keep)
    return heads, importance


# --------------------------------------------------------------------------
# Token scoring
# --------------------------------------------------------------------------
def index_scores(q, w, keys, seq_of, prefix_len, heads_of_query):
    """Indexer scores over the whole key cache of each query.

    MISA-gist, Problem statement / Methodology: the indexer scores every prefix
    token; in MISA only the h active heads do so.  HISA-zh, 二: the indexer
    computes one relevance score per (query, historical token).

    heads_of_query: [T, h] head ids (all heads for the dense indexer).
    Returns S [T, L] with S = -inf for s >= prefix_len[t].
    """
    T = q.shape[0]
    L = keys.shape[1]
    S = np.full((T, L), -np.inf, dtype=np.float64)
    for t in range(T):
        hs = np.asarray(heads_of_query[t], dtype=np.int64)
        n_vis = int(min(max(prefix_len[t], 0), L))
        if n_vis == 0:
            continue
        K = keys[seq_of[t], :n_vis]
        dots = q[t, hs] @ K.T  # [h, n_vis]
        S[t, :n_vis] = (w[t, hs][:, None] * np.maximum(dots, 0.0)).sum(axis=0)
    return S


def candidate_scores(q, w, keys, seq_of, prefix_len, heads_of_query, cand):
    """Indexer scores restricted to a candidate list.

    MISA-gist, Hierarchical variant: the full-head indexer re-scores only the k'
    candidates.  HISA-zh, Stage 2: the token-level indexer runs only inside the
    m selected blocks.

    cand: [T, n] token ids (-1 = empty slot).  An entry is scored iff
    0 <= id < prefix_len[t]; every other entry is -inf.
    """
    T, n = cand.shape
    L = keys.shape[1]
    S = np.full((T, n), -np.inf, dtype=np.float64)
    for t in range(T):
        hs = np.asarray(heads_of_query[t], dtype=np.int64)
        ids = cand[t].astype(np.int64)
        ok = (ids >= 0) & (ids < min(int(prefix_len[t]), L))
        if not ok.any():
            continue
        K = keys[seq_of[t], ids[ok]]
        dots = q[t, hs] @ K.T
        S[t, ok] = (w[t, hs][:, None] * np.maximum(dots, 0.0)).sum(axis=0)
    return S


# --------------------------------------------------------------------------
# Top-k
# --------------------------------------------------------------------------
def topk_ascending(scores: np.ndarray, k: int, id_map: np.ndarray | None = None) -> np.ndarray:
    """The k highest-scoring entries of one row, as ascending ids.

    MISA-zh, DSA: the indexer keeps the most relevant token subset for the main
    attention; HISA-zh, 二: the indexer picks the k most relevant tokens per
    query; HISA-zh, 四: the output is k token indices.

    Entries equal to -inf (masked) are never chosen.  Order: larger score first,
    then lower position.  The chosen positions are sorted ascending, mapped
    through id_map (if given) and padded with -1 to length k.
    """
    s = np.asarray(scores, dtype=np.float64)
    valid = np.nonzero(s > -np.inf)[0]
    if valid.size > k:
        # lexsort: last key is primary -> (-score, position)
        order = np.lexsort((valid, -s[valid]))
        chosen = np.sort(valid[order[:k]])
    else:
        chosen = valid
    out = np.full(k, -1, dtype=np.int64)
    ids = chosen if id_map is None else np.asarray(id_map, dtype=np.int64)[chosen]
    out[: ids.size] = ids
    return out


def topk_rows(S: np.ndarray, k: int, id_map: np.ndarray | None = None) -> np.ndarray:
    """topk_ascending applied to every row of S."""
    out = np.empty((S.shape[0], k), dtype=np.int64)
    for t in range(S.shape[0]):
        out[t] = topk_ascending(S[t], k, None if id_map is None else id_map[t])
    return out


# --------------------------------------------------------------------------
# The three indexers, step by step
# --------------------------------------------------------------------------
def dense_indexer(q, w, keys, seq_of, prefix_len, k):
    """DSA dense indexer: all H heads score every prefix token, then top-k.

    MISA-gist, Problem statement: DSA scores every prefix token with all H_I
    heads and keeps the top-k.  Returns (idx [T, k], S [T, L]).
    """
    T, H, _ = q.shape
    all_heads = np.tile(np.arange(H), (T, 1))
    S = index_scores(q, w, keys, seq_of, prefix_len, all_heads)
    return topk_rows(S, k), S


def misa_indexer(q, w, keys, seq_of, prefix_len, B, q_block, h, k, means=None, S=None, pool="mean"):
    """MISA: route h of H heads per query block, score with them, top-k.

    MISA-gist, Methodology (router, then sparse token scoring of the whole prefix
    by the h active heads, then top-k on the reduced scores).  S / pool select
    the block statistic (window_stats); the defaults are the mean-pooled blocks.
    Returns dict with heads, importance, scores, idx.
    """
    T, H, _ = q.shape
    L = keys.shape[1]
    if means is None:
        if S is None and pool == "mean":
            means = np.stack([block_means(keys[b], B) for b in range(keys.shape[0])])
        else:
            means = np.stack([window_stats(keys[b], B, S, pool) for b in range(keys.shape[0])])
    heads, imp = route_heads(q, w, means, seq_of, prefix_len, L, B, q_block, h, S)
    per_query = np.stack([heads[t // q_block] for t in range(T)])
    S = index_scores(q, w, keys, seq_of, prefix_len, per_query)
    return {"heads": heads, "importance": imp, "scores": S, "idx": topk_rows(S, k)}


def misa_dagger_indexer(q, w, keys, seq_of, prefix_len, B, q_block, h, kp, k, means=None):
    """MISA-dagger: routed coarse top-k' candidates, full-head rerank, top-k.

    MISA-gist, Hierarchical variant: the routed pass keeps an enlarged set of k'
    tokens; the original all-head indexer re-scores only those candidates and the
    final top-k is taken among them.  MISA-zh, 层次化变体 (two layers).
    """
    T, H, _ = q.shape
    coarse = misa_indexer(q, w, keys, seq_of, prefix_len, B, q_block, h, kp, means=means)
    cand = coarse["idx"]
    all_heads = np.tile(np.arange(H), (T, 1))
    S_fine = candidate_scores(q, w, keys, seq_of, prefix_len, all_heads, cand)
    idx = topk_rows(S_fine, k, id_map=cand)
    return {"heads": coarse["heads"], "importance": coarse["importance"],
            "coarse_scores": coarse["scores"], "cand": cand,
            "cand_scores": S_fine, "idx": idx}


def hisa_block_filter(q, w, means, seq_of, prefix_len, L, B, m, S=None):
    """HISA Stage 1: score block representatives with all heads, keep top-m.

    HISA-zh, Stage 1: the query is scored only against the mean-pooled block
    representatives and the m best blocks are kept; Stage 2 then looks at the
    at most m*B tokens of those blocks.  HISA keeps every indexer head.

    A block the prefix cuts (some of its tokens visible, some not: a causal
    query's own, partly filled block) has a mean that includes future keys, so it
    is not scored; it is always kept instead (score +inf) and its tokens past the
    prefix are masked like any other -- the other m - 1 blocks are the best
    wholly visible ones.  (The pages do not say how Stage 1 treats a partly
    visible block; keeping the query's local block is the plainest causal
    reading.)

    Overlapping windows (S < B, window j = [j*S, min(j*S + B, L)); HISA-zh, 七,
    潜在改进): the same rules apply per window; every window the prefix cuts is
    kept; a token that an earlier chosen window already lists is listed once
    only (its later slot is -1), so the candidate ids stay distinct and
    ascending.  The chosen windows ascend, so token x of the i-th one is
    already listed iff x < (start of the (i-1)-th) + B.

    Returns blocks [T, m] (ascending, -1 padded), cand [T, m*B] (token ids of the
    chosen blocks in ascending order, -1 where a slot is past the prefix or past
    the cache) and block scores [T, M] (-inf where not visible, +inf for a block
    the prefix cuts).
    """
    T, H, _ = q.shape
    S = B if S is None else S
    M = num_windows(L, B, S)
    bs = np.full((T, M), -np.inf, dtype=np.float64)
    blocks = np.full((T, m), -1, dtype=np.int64)
    cand = np.full((T, m * B), -1, dtype=np.int64)
    for t in range(T):
        plen = int(prefix_len[t])
        vis = visible_blocks(plen, L, B, S)
        if vis.size:
            A = head_block_affinity(q[t], w[t], means[seq_of[t]][vis])
            bs[t, vis] = A.sum(axis=0)
        for jp in range(M):  # the blocks holding token plen, if the prefix cuts them
            if jp * S < plen < min(jp * S + B, L):
                bs[t, jp] = np.inf
        chosen = topk_ascending(bs[t], m)
        blocks[t] = chosen
        limit = min(int(prefix_len[t]), L)
        prev_end = -1
        for i, j in enumerate(chosen):
            if j < 0:
                continue
            ids = np.arange(j * S, j * S + B)
            ids[(ids >= limit) | (ids < prev_end)] = -1
            cand[t, i * B:(i + 1) * B] = ids
            prev_end = j * S + B
    return blocks, cand, bs


def hisa_indexer(q, w, keys, seq_of, prefix_len, B, m, k, means=None, S=None, pool="mean"):
    """HISA: block coarse filter, then all-head token scoring inside, top-k.

    HISA-zh, Stage 1 + Stage 2; cost per query O(L/B + m*B).  S / pool select
    the block statistic (window_stats: overlapping windows, max pooling).
    """
    T, H, _ = q.shape
    L = keys.shape[1]
    if means is None:
        if S is None and pool == "mean":
            means = np.stack([block_means(keys[b], B) for b in range(keys.shape[0])])
        else:
            means = np.stack([window_stats(keys[b], B, S, pool) for b in range(keys.shape[0])])
    blocks, cand, bs = hisa_block_filter(q, w, means, seq_of, prefix_len, L, B, m, S)
    all_heads = np.tile(np.arange(H), (T, 1))
    S = candidate_scores(q, w, keys, seq_of, prefix_len, all_heads, cand)
    idx = topk_rows(S, k, id_map=cand)
    return {"blocks": blocks, "cand": cand, "block_scores": bs, "cand_scores": S, "idx": idx}


# --------------------------------------------------------------------------
# Quality metric
# --------------------------------------------------------------------------
def iou(a, b) -> float:
    """|A n B| / |A u B| of two selected sets (-1 slots ignored).

    HISA-zh, 五 (选择一致性：IoU 分析): intersection over union of the token
    sets two indexers select.
    """
    sa = {int(x) for x in np.asarray(a).ravel() if x >= 0}
    sb = {int(x) for x in np.asarray(b).ravel() if x >= 0}
    if not sa and not sb:
        return 1.0
    return len(sa & sb) / len(sa | sb)


def num_blocks(L: int, B: int) -> int:
    """M = ceil(L / B) (MISA-gist, Methodology)."""
    return int(math.ceil(L / B))

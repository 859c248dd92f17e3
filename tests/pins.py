"""Pins that tie the fp64 oracle to something other than itself.

Every check takes the oracle as a module-like object so that the same checks can
be run against deliberately broken copies of it (see test_oracle_mutations.py):
each plausible slip in the oracle has to make at least one of them fail.

Kinds of pin used here:
* the hand-worked 2-head / 8-token case in tests/golden (exact values);
* closed forms (constant and linear blocks, a partial last block);
* brute force on tiny inputs (top-k by its rank definition, evaluated pairwise);
* invariants that follow from the definitions (all heads routed == dense
  indexer; HISA with m*B >= L == dense; hierarchical rerank with k' >= L ==
  dense).
"""
from __future__ import annotations

import json
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_case_2head_8token.json")


def hand_case():
    with open(GOLDEN, encoding="utf-8") as f:
        g = json.load(f)
    q = np.asarray(g["q"], dtype=np.float64)        # [1, 2, 2]
    w = np.asarray(g["w"], dtype=np.float64)        # [1, 2]
    keys = np.asarray(g["keys"], dtype=np.float64)  # [1, 8, 2]
    return g, q, w, keys


def _one(x):
    return np.asarray(x).ravel().tolist()


# ---------------------------------------------------------------- hand case
def check_hand_dense(orc):
    g, q, w, keys = hand_case()
    seq_of, plen = np.array([0]), np.array([8])
    idx3, S = orc.dense_indexer(q, w, keys, seq_of, plen, 3)
    assert np.array_equal(S[0], np.asarray(g["dense_scores"])), S
    assert _one(idx3) == g["dense_top3"], idx3
    idx4, _ = orc.dense_indexer(q, w, keys, seq_of, plen, 4)
    assert _one(idx4) == g["dense_top4"], idx4


def check_hand_block_means(orc):
    g, q, w, keys = hand_case()
    assert np.allclose(orc.block_means(keys[0], g["B"]), np.asarray(g["block_means"]), rtol=0, atol=0)
    p = g["partial_block_B3"]
    assert np.allclose(orc.block_means(keys[0], 3), np.asarray(p["block_means"]), rtol=0, atol=1e-15)


def check_hand_router(orc):
    g, q, w, keys = hand_case()
    means = orc.block_means(keys[0], g["B"])[None]
    heads, imp = orc.route_heads(q, w, means, np.array([0]), np.array([8]), 8, g["B"], 1, 1)
    assert np.array_equal(imp[0], np.asarray(g["router_importance"])), imp
    assert _one(heads) == g["router_heads_h1"], heads


def check_hand_misa(orc):
    g, q, w, keys = hand_case()
    r = orc.misa_indexer(q, w, keys, np.array([0]), np.array([8]), g["B"], 1, 1, 4)
    assert np.array_equal(r["scores"][0], np.asarray(g["misa1_scores"])), r["scores"]
    assert _one(r["idx"]) == g["misa1_top4"], r["idx"]


def check_hand_dagger(orc):
    g, q, w, keys = hand_case()
    r = orc.misa_dagger_indexer(q, w, keys, np.array([0]), np.array([8]), g["B"], 1, 1, 4, 3)
    assert _one(r["cand"]) == g["dagger_h1_kp4_cand"], r["cand"]
    assert _one(r["idx"]) == g["dagger_h1_kp4_top3"], r["idx"]


def check_hand_hisa(orc):
    g, q, w, keys = hand_case()
    r = orc.hisa_indexer(q, w, keys, np.array([0]), np.array([8]), g["B"], 1, 3)
    assert np.array_equal(r["block_scores"][0], np.asarray(g["hisa_block_scores"])), r["block_scores"]
    assert _one(r["blocks"]) == g["hisa_m1_blocks"], r["blocks"]
    assert _one(r["idx"]) == g["hisa_m1_top3"], r["idx"]


def check_hand_hisa_partial_block(orc):
    g, q, w, keys = hand_case()
    p = g["partial_block_B3"]
    r3 = orc.hisa_indexer(q, w, keys, np.array([0]), np.array([8]), 3, 2, 3)
    assert np.allclose(r3["block_scores"][0], np.asarray(p["hisa_block_scores"]), rtol=0, atol=1e-15)
    assert _one(r3["blocks"]) == p["hisa_m2_blocks"], r3["blocks"]
    assert _one(r3["cand"]) == p["hisa_m2_cand"], r3["cand"]
    assert _one(r3["idx"]) == p["hisa_m2_top3"], r3["idx"]
    r4 = orc.hisa_indexer(q, w, keys, np.array([0]), np.array([8]), 3, 2, 4)
    assert _one(r4["idx"]) == p["hisa_m2_top4"], r4["idx"]


def check_hand_hisa_causal_cut_block(orc):
    """prefix 6 with B = 4: block 0 is wholly visible, block 1 is cut (tokens 4, 5
    visible, 6, 7 in the future).  The cut block is always kept and only its
    visible tokens are candidates; with m = 2 the candidates are tokens 0..5."""
    g, q, w, keys = hand_case()
    dense = np.asarray(g["dense_scores"], dtype=np.float64)
    r1 = orc.hisa_indexer(q, w, keys, np.array([0]), np.array([6]), 4, 1, 3)
    assert _one(r1["blocks"]) == [1], r1["blocks"]
    assert _one(r1["cand"]) == [4, 5, -1, -1], r1["cand"]
    assert r1["block_scores"][0, 1] == np.inf, r1["block_scores"]
    assert _one(r1["idx"]) == [4, 5, -1], r1["idx"]          # two visible candidates for k = 3
    r2 = orc.hisa_indexer(q, w, keys, np.array([0]), np.array([6]), 4, 2, 3)
    assert _one(r2["blocks"]) == [0, 1], r2["blocks"]
    assert _one(r2["cand"]) == [0, 1, 2, 3, 4, 5, -1, -1], r2["cand"]
    # top-3 of the dense scores over tokens 0..5 (score desc, lower id first)
    order = sorted(range(6), key=lambda s: (-dense[s], s))[:3]
    assert _one(r2["idx"]) == sorted(order), (r2["idx"], order)


def check_hand_causal_router(orc):
    """prefix 6 with B = 4: only block 0 is complete; the two heads tie at 0.25
    and the lower head id wins."""
    g, q, w, keys = hand_case()
    means = orc.block_means(keys[0], g["B"])[None]
    heads, imp = orc.route_heads(q, w, means, np.array([0]), np.array([6]), 8, g["B"], 1, 1)
    assert np.array_equal(imp[0], np.asarray(g["causal_prefix6_importance"])), imp
    assert _one(heads) == g["causal_prefix6_heads_h1"], heads


def check_hand_causal_scores(orc):
    """Keys at or past prefix_len are masked to -inf and never selected."""
    g, q, w, keys = hand_case()
    idx, S = orc.dense_indexer(q, w, keys, np.array([0]), np.array([5]), 4)
    exp = np.asarray(g["dense_scores"], dtype=np.float64).copy()
    exp[5:] = -np.inf
    assert np.array_equal(S[0], exp), S
    # valid scores 1, .5, 1.5, 0, 0: top-4 is {2, 0, 1} plus the lower-index zero (3)
    assert _one(idx) == [0, 1, 2, 3], idx
    idx8, _ = orc.dense_indexer(q, w, keys, np.array([0]), np.array([2]), 4)
    assert _one(idx8) == [0, 1, -1, -1], idx8


def check_hand_candidate_scores(orc):
    """Candidate scoring equals the dense scores at the candidate ids; empty
    slots (-1) and ids at or past prefix_len are -inf."""
    g, q, w, keys = hand_case()
    dense = np.asarray(g["dense_scores"])
    cand = np.array([[0, 5, 7, -1, 2]])
    all_heads = np.array([[0, 1]])
    S = orc.candidate_scores(q, w, keys, np.array([0]), np.array([6]), all_heads, cand)
    assert np.array_equal(S[0], np.array([dense[0], dense[5], -np.inf, -np.inf, dense[2]])), S
    S8 = orc.candidate_scores(q, w, keys, np.array([0]), np.array([8]), all_heads, cand)
    assert np.array_equal(S8[0], np.array([dense[0], dense[5], dense[7], -np.inf, dense[2]])), S8


# ---------------------------------------------------------------- closed forms
def check_block_means_closed_form(orc):
    rng = np.random.default_rng(7)
    d, B, L = 5, 4, 11            # 3 blocks, the last holds 3 tokens
    v = rng.standard_normal(d)
    c = rng.standard_normal(d)
    keys = np.zeros((L, d))
    keys[:4] = c                  # constant block -> that constant
    for s in range(4, L):         # linear ramp -> value at the block's midpoint
        keys[s] = s * v
    m = orc.block_means(keys, B)
    assert m.shape == (3, d)
    assert np.allclose(m[0], c, atol=1e-14)
    assert np.allclose(m[1], 5.5 * v, atol=1e-12)       # tokens 4..7
    assert np.allclose(m[2], 9.0 * v, atol=1e-12)       # tokens 8..10 (partial)


def check_visible_blocks(orc):
    assert orc.visible_blocks(8, 8, 4).tolist() == [0, 1]
    assert orc.visible_blocks(7, 8, 4).tolist() == [0]
    assert orc.visible_blocks(4, 8, 4).tolist() == [0]
    assert orc.visible_blocks(3, 8, 4).tolist() == []
    assert orc.visible_blocks(10, 10, 4).tolist() == [0, 1, 2]   # partial last block at decode
    assert orc.visible_blocks(9, 10, 4).tolist() == [0, 1]


def check_router_query_block_sum(orc):
    """A query block of two copies of one query doubles every importance and
    keeps the same heads; a block of one query keeps that query's decision."""
    rng = np.random.default_rng(11)
    T, H, d, L, B = 1, 6, 4, 12, 4
    q = rng.standard_normal((T, H, d))
    w = rng.standard_normal((T, H))
    keys = rng.standard_normal((1, L, d))
    means = orc.block_means(keys[0], B)[None]
    h1, i1 = orc.route_heads(q, w, means, np.array([0]), np.array([L]), L, B, 1, 3)
    q2 = np.concatenate([q, q]); w2 = np.concatenate([w, w])
    h2, i2 = orc.route_heads(q2, w2, means, np.array([0, 0]), np.array([L, L]), L, B, 2, 3)
    assert np.allclose(i2[0], 2 * i1[0], rtol=1e-14, atol=0)
    assert h2[0].tolist() == h1[0].tolist()
    # brute force importance: sum over blocks of w * max(q.mean, 0), scalar loops
    for h in range(H):
        acc = 0.0
        for j in range(means.shape[1]):
            dot = sum(q[0, h, c] * means[0, j, c] for c in range(d))
            acc += w[0, h] * (dot if dot > 0 else 0.0)
        assert abs(acc - i1[0, h]) <= 1e-12 * max(1.0, abs(acc))


# ---------------------------------------------------------------- brute force top-k
def _topk_by_rank_definition(s, k):
    """Entry i (finite) is chosen iff fewer than k valid entries beat it, where
    j beats i iff s_j > s_i, or s_j == s_i and j < i."""
    n = len(s)
    chosen = []
    for i in range(n):
        if not s[i] > -np.inf:
            continue
        beat = 0
        for j in range(n):
            if j == i or not s[j] > -np.inf:
                continue
            if s[j] > s[i] or (s[j] == s[i] and j < i):
                beat += 1
        if beat < k:
            chosen.append(i)
    return chosen + [-1] * (k - len(chosen))


def check_topk_brute_force(orc):
    rng = np.random.default_rng(3)
    for trial in range(60):
        n = int(rng.integers(1, 40))
        k = int(rng.integers(1, 45))
        s = rng.choice(np.array([-1.5, -0.0, 0.0, 0.25, 0.25, 1.0, 3.0, -np.inf]), size=n)
        s = np.where(rng.random(n) < 0.3, rng.standard_normal(n), s)
        got = orc.topk_ascending(s, k).tolist()
        assert got == _topk_by_rank_definition(s, k), (trial, s, k, got)
    # -0.0 and +0.0 rank equal: the lower position wins
    assert orc.topk_ascending(np.array([-1.0, -0.0, 0.0, -2.0]), 1).tolist() == [1]
    assert orc.topk_ascending(np.array([-1.0, 0.0, -0.0, -2.0]), 1).tolist() == [1]
    # id_map: positions are chosen, ids are reported
    assert orc.topk_ascending(np.array([3.0, 1.0, 2.0]), 2, np.array([10, 20, 30])).tolist() == [10, 30]


# ---------------------------------------------------------------- invariants
def _tiny_problem(seed, T=3, H=6, d=8, L=37, nseq=2):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((T, H, d))
    w = rng.standard_normal((T, H)) / 8
    keys = rng.standard_normal((nseq, L, d)) / np.sqrt(d)
    seq_of = rng.integers(0, nseq, size=T)
    plen = np.full(T, L)
    return q, w, keys, seq_of, plen


def check_invariant_all_heads_is_dense(orc):
    for seed in range(4):
        q, w, keys, seq_of, plen = _tiny_problem(seed)
        H = q.shape[1]
        idx_d, S_d = orc.dense_indexer(q, w, keys, seq_of, plen, 9)
        r = orc.misa_indexer(q, w, keys, seq_of, plen, 5, 1, H, 9)
        assert r["heads"].tolist() == [list(range(H))] * q.shape[0]
        assert np.allclose(r["scores"], S_d, rtol=1e-13, atol=0)
        assert np.array_equal(r["idx"], idx_d)


def check_invariant_hisa_covering_is_dense(orc):
    for seed in range(4):
        q, w, keys, seq_of, plen = _tiny_problem(seed + 10)
        L = keys.shape[1]
        idx_d, _ = orc.dense_indexer(q, w, keys, seq_of, plen, 9)
        for B in (4, 5, 37):
            m = (L + B - 1) // B            # m * B >= L: every block kept
            r = orc.hisa_indexer(q, w, keys, seq_of, plen, B, m, 9)
            assert np.array_equal(r["idx"], idx_d), (seed, B)


def check_invariant_hisa_causal_covering_is_dense(orc):
    """Causal prefixes that end inside a block: with every block kept (m*B >= L)
    HISA must still see exactly the dense indexer's tokens, the cut block's
    visible tokens included."""
    for seed in range(4):
        q, w, keys, seq_of, _ = _tiny_problem(seed + 20)
        L = keys.shape[1]
        plen = np.array([5, 22, 36])       # mid-block prefixes for B = 4 and 5
        idx_d, _ = orc.dense_indexer(q, w, keys, seq_of, plen, 9)
        for B in (4, 5):
            m = (L + B - 1) // B
            r = orc.hisa_indexer(q, w, keys, seq_of, plen, B, m, 9)
            assert np.array_equal(r["idx"], idx_d), (seed, B)


def check_invariant_dagger_full_candidates_is_dense(orc):
    for seed in range(4):
        q, w, keys, seq_of, plen = _tiny_problem(seed + 20)
        L = keys.shape[1]
        idx_d, _ = orc.dense_indexer(q, w, keys, seq_of, plen, 9)
        r = orc.misa_dagger_indexer(q, w, keys, seq_of, plen, 5, 1, 2, L, 9)
        assert np.array_equal(r["idx"], idx_d), seed


def check_iou(orc):
    assert orc.iou([1, 2, 3, -1], [2, 3, 4, -1]) == 0.5
    assert orc.iou([5, 6], [6, 5]) == 1.0
    assert orc.iou([-1], [-1]) == 1.0


ALL_CHECKS = [
    check_hand_dense, check_hand_block_means, check_hand_router, check_hand_misa,
    check_hand_dagger, check_hand_hisa, check_hand_hisa_partial_block, check_hand_hisa_causal_cut_block,
    check_hand_causal_router, check_hand_causal_scores, check_hand_candidate_scores, check_block_means_closed_form,
    check_visible_blocks, check_router_query_block_sum, check_topk_brute_force,
    check_invariant_all_heads_is_dense, check_invariant_hisa_covering_is_dense,
    check_invariant_hisa_causal_covering_is_dense,
    check_invariant_dagger_full_candidates_is_dense, check_iou,
]

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
  dense; HISA over overlapping windows, all kept, == dense; a max-pooled
  block score bounds its tokens' scores for nonnegative q and w);
* the same hand case with max pooling and overlapping windows
  (tests/golden/hand_case_window_stats.json), and a hand-counted table of
  window counts, visible and cut windows.
"""
from __future__ import annotations

import json
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_case_2head_8token.json")
GOLDEN_WIN = os.path.join(os.path.dirname(__file__), "golden", "hand_case_window_stats.json")


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


# ---------------------------------------------------------------- max pooling and overlapping windows
def _win_golden():
    with open(GOLDEN_WIN, encoding="utf-8") as f:
        return json.load(f)


def check_hand_max_pool(orc):
    """HISA-zh, 七 (潜在改进): max pooling instead of mean pooling."""
    _, q, w, keys = hand_case()
    g = _win_golden()["max_B4"]
    st = orc.window_stats(keys[0], 4, None, "max")
    assert np.array_equal(st, np.asarray(g["block_max"])), st
    heads, imp = orc.route_heads(q, w, st[None], np.array([0]), np.array([8]), 8, 4, 1, 1)
    assert np.array_equal(imp[0], np.asarray(g["router_importance"])), imp
    assert _one(heads) == g["router_heads_h1"]
    blocks, cand, bs = orc.hisa_block_filter(q, w, st[None], np.array([0]), np.array([8]), 8, 4, 1)
    assert np.array_equal(bs[0], np.asarray(g["hisa_block_scores"])), bs
    assert _one(blocks) == g["hisa_m1_blocks"] and _one(cand) == g["hisa_m1_cand"]
    r = orc.hisa_indexer(q, w, keys, np.array([0]), np.array([8]), 4, 1, 3, pool="max")
    assert _one(r["idx"]) == g["hisa_m1_top3"], r["idx"]


def check_hand_overlap(orc):
    """HISA-zh, 七 (潜在改进): overlapping blocks; windows of B = 4 every S = 2."""
    _, q, w, keys = hand_case()
    g = _win_golden()["overlap_B4_S2"]
    assert orc.num_windows(8, 4, 2) == g["num_windows"]
    st = orc.window_stats(keys[0], 4, 2, "mean")
    assert np.array_equal(st, np.asarray(g["window_means"])), st
    heads, imp = orc.route_heads(q, w, st[None], np.array([0]), np.array([8]), 8, 4, 1, 1, 2)
    assert np.array_equal(imp[0], np.asarray(g["router_importance"])), imp
    assert _one(heads) == g["router_heads_h1"]
    for m in (1, 2):
        blocks, cand, bs = orc.hisa_block_filter(q, w, st[None], np.array([0]), np.array([8]), 8, 4, m, 2)
        assert np.array_equal(bs[0], np.asarray(g["hisa_block_scores"])), bs
        assert _one(blocks) == g[f"hisa_m{m}_blocks"], blocks
        assert _one(cand) == g[f"hisa_m{m}_cand"], cand
    assert _one(orc.hisa_indexer(q, w, keys, np.array([0]), np.array([8]), 4, 1, 3, S=2)["idx"]) == g["hisa_m1_top3"]
    assert _one(orc.hisa_indexer(q, w, keys, np.array([0]), np.array([8]), 4, 2, 3, S=2)["idx"]) == g["hisa_m2_top3"]
    assert _one(orc.hisa_indexer(q, w, keys, np.array([0]), np.array([8]), 4, 2, 4, S=2)["idx"]) == g["hisa_m2_top4"]


def check_hand_overlap_causal(orc):
    _, q, w, keys = hand_case()
    g = _win_golden()["overlap_B4_S2_causal_prefix6"]
    assert orc.visible_blocks(6, 8, 4, 2).tolist() == g["visible_windows"]
    st = orc.window_stats(keys[0], 4, 2, "mean")[None]
    blocks, cand, bs = orc.hisa_block_filter(q, w, st, np.array([0]), np.array([6]), 8, 4, 2, 2)
    exp_bs = [float(x) for x in g["hisa_block_scores"]]
    assert bs[0].tolist() == exp_bs, bs
    assert _one(blocks) == g["hisa_m2_blocks"] and _one(cand) == g["hisa_m2_cand"], (blocks, cand)
    r = orc.hisa_indexer(q, w, keys, np.array([0]), np.array([6]), 4, 2, 3, S=2)
    assert _one(r["idx"]) == g["hisa_m2_top3"]
    _, imp = orc.route_heads(q, w, st, np.array([0]), np.array([6]), 8, 4, 1, 1, 2)
    assert np.array_equal(imp[0], np.asarray(g["router_importance"])), imp


def check_window_counts(orc):
    """Hand-counted windows: [L, B, S, M, start, end of the last window]."""
    for L, B, S, M, s0, s1 in _win_golden()["window_counts"]["cases"]:
        assert orc.num_windows(L, B, S) == M, (L, B, S)
        keys = np.arange(L, dtype=np.float64)[:, None] * np.ones((1, 2))
        st = orc.window_stats(keys, B, S, "max")
        assert st.shape == (M, 2)
        assert st[-1, 0] == s1 - 1                       # the last window ends at token s1 - 1
        mean_last = orc.window_stats(keys, B, S, "mean")[-1, 0]
        assert mean_last == (s0 + s1 - 1) / 2.0          # ... and starts at s0
    for L in range(1, 40):                                # S = B: the plain blocks
        assert orc.num_windows(L, 4, 4) == (L + 3) // 4


def check_window_closed_forms(orc):
    rng = np.random.default_rng(17)
    d = 6
    v = np.abs(rng.standard_normal(d))          # nonnegative ramp direction
    c = rng.standard_normal(d)
    for L, B, S in ((13, 4, 2), (20, 5, 3), (9, 9, 1), (7, 3, 3)):
        ramp = np.arange(L, dtype=np.float64)[:, None] * v[None]
        const = np.tile(c, (L, 1))
        mx, mn = orc.window_stats(ramp, B, S, "max"), orc.window_stats(ramp, B, S, "mean")
        for j in range(mx.shape[0]):
            s0, s1 = j * S, min(j * S + B, L)
            assert np.allclose(mx[j], (s1 - 1) * v, rtol=1e-15, atol=0)          # max of a ramp: its last token
            assert np.allclose(mn[j], 0.5 * (s0 + s1 - 1) * v, rtol=1e-14, atol=0)  # mean: its midpoint
        assert np.allclose(orc.window_stats(const, B, S, "max"), c[None], rtol=0, atol=0)
        assert np.allclose(orc.window_stats(const, B, S, "mean"), c[None], rtol=1e-15, atol=1e-15)


def check_window_stats_brute_force(orc):
    """Each window statistic against a scan that tests every token for
    membership (j*S <= s < j*S + B, s < L) and pools with scalar loops."""
    rng = np.random.default_rng(19)
    for trial in range(12):
        L = int(rng.integers(1, 30)); B = int(rng.integers(1, 9)); S = int(rng.integers(1, B + 1))
        keys = rng.standard_normal((L, 3))
        for pool in ("mean", "max"):
            st = orc.window_stats(keys, B, S, pool)
            for j in range(st.shape[0]):
                members = [s for s in range(L) if j * S <= s < j * S + B]
                assert members, (trial, j)
                for c in range(3):
                    vals = [keys[s, c] for s in members]
                    ref = max(vals) if pool == "max" else sum(vals) / len(vals)
                    assert abs(st[j, c] - ref) <= 1e-14 * max(1.0, abs(ref)), (trial, pool, j, c)
            # every token lies in some window
            covered = {s for j in range(st.shape[0]) for s in range(L) if j * S <= s < j * S + B}
            assert covered == set(range(L)), (trial, L, B, S)


def check_max_pool_bounds_token_scores(orc):
    """With nonnegative q and w, a max-pooled block score bounds the dense score
    of every token of the block from above (q . max_j >= q . k_s, ReLU and the
    weighted sum are monotone); a mean does not."""
    rng = np.random.default_rng(23)
    for seed in range(3):
        T, H, d, L, B, S = 2, 4, 5, 23, 4, 3
        q = np.abs(rng.standard_normal((T, H, d)))
        w = np.abs(rng.standard_normal((T, H)))
        keys = rng.standard_normal((1, L, d))
        st = orc.window_stats(keys[0], B, S, "max")[None]
        _, _, bs = orc.hisa_block_filter(q, w, st, np.zeros(T, np.int64), np.full(T, L), L, B, 1, S)
        _, Sd = orc.dense_indexer(q, w, keys, np.zeros(T, np.int64), np.full(T, L), 1)
        for t in range(T):
            for j in range(bs.shape[1]):
                toks = np.arange(j * S, min(j * S + B, L))
                assert np.all(bs[t, j] >= Sd[t, toks] - 1e-12), (seed, t, j)


def check_invariant_hisa_overlap_covering_is_dense(orc):
    """Overlapping windows with every window kept: each visible token is listed
    once (distinct, ascending candidate ids) and HISA equals the dense indexer,
    at decode and for causal prefixes that end inside windows."""
    for seed in range(3):
        q, w, keys, seq_of, plen = _tiny_problem(seed + 30)
        L = keys.shape[1]
        for B, S in ((6, 2), (5, 3), (8, 5)):
            m = orc.num_windows(L, B, S)
            for pl in (plen, np.array([7, 20, 33])):
                idx_d, _ = orc.dense_indexer(q, w, keys, seq_of, pl, 9)
                r = orc.hisa_indexer(q, w, keys, seq_of, pl, B, m, 9, S=S)
                assert np.array_equal(r["idx"], idx_d), (seed, B, S)
                for t in range(q.shape[0]):
                    ids = r["cand"][t][r["cand"][t] >= 0]
                    assert np.all(np.diff(ids) > 0), (seed, B, S, t)
                    assert ids.tolist() == list(range(min(int(pl[t]), L))), (seed, B, S, t)


def check_window_visibility_and_cuts(orc):
    """Hand-derived: for L = 8, B = 4, S = 2 (windows [0,4), [2,6), [4,8)) and
    L = 11, B = 4, S = 3 (windows [0,4), [3,7), [6,10), [9,11)), which windows a
    prefix sees whole (finite score) and which it cuts (kept, +inf)."""
    table = [  # L, B, S, prefix, visible, cut
        (8, 4, 2, 3, [], [0, 1]), (8, 4, 2, 4, [0], [1]), (8, 4, 2, 5, [0], [1, 2]), (8, 4, 2, 6, [0, 1], [2]),
        (8, 4, 2, 7, [0, 1], [2]), (8, 4, 2, 8, [0, 1, 2], []),
        (11, 4, 3, 5, [0], [1]), (11, 4, 3, 7, [0, 1], [2]), (11, 4, 3, 10, [0, 1, 2], [3]),
        (11, 4, 3, 11, [0, 1, 2, 3], []),
    ]
    rng = np.random.default_rng(29)
    for L, B, S, pl, vis, cut in table:
        assert orc.visible_blocks(pl, L, B, S).tolist() == vis, (L, B, S, pl)
        q = np.abs(rng.standard_normal((1, 2, 3)))
        w = np.abs(rng.standard_normal((1, 2)))
        keys = rng.standard_normal((1, L, 3))
        st = orc.window_stats(keys[0], B, S, "mean")[None]
        _, _, bs = orc.hisa_block_filter(q, w, st, np.array([0]), np.array([pl]), L, B, 1, S)
        got_vis = [j for j in range(bs.shape[1]) if np.isfinite(bs[0, j])]
        got_cut = [j for j in range(bs.shape[1]) if bs[0, j] == np.inf]
        assert got_vis == vis and got_cut == cut, (L, B, S, pl, bs)


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
    check_hand_max_pool, check_hand_overlap, check_hand_overlap_causal, check_window_counts,
    check_window_closed_forms, check_window_stats_brute_force, check_max_pool_bounds_token_scores,
    check_invariant_hisa_overlap_covering_is_dense, check_window_visibility_and_cuts,
]

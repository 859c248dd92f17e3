"""Plant plausible mistakes in a copy of the oracle (on the CPU) and check that
the pins catch every one of them.

Each mutant is the oracle's source with one small edit: a dropped term, a wrong
sign or index, a transposed operand, an off-by-one.  A mutant counts as caught
when at least one pin raises (an assertion or any other error).
"""
import inspect
import types

import numpy as np
import pytest

import oracle.misa_oracle as real
import pins

SRC = inspect.getsource(real)

MUTANTS = {
    "relu_dropped_in_affinity": ("return w_t[:, None] * np.maximum(dots, 0.0)", "return w_t[:, None] * dots"),
    "weight_dropped_in_affinity": ("return w_t[:, None] * np.maximum(dots, 0.0)", "return np.maximum(dots, 0.0)"),
    "relu_dropped_in_scores": ("S[t, :n_vis] = (w[t, hs][:, None] * np.maximum(dots, 0.0)).sum(axis=0)",
                               "S[t, :n_vis] = (w[t, hs][:, None] * dots).sum(axis=0)"),
    "weight_not_per_head": ("S[t, :n_vis] = (w[t, hs][:, None] * np.maximum(dots, 0.0)).sum(axis=0)",
                            "S[t, :n_vis] = (w[t, :][:1, None] * np.maximum(dots, 0.0)).sum(axis=0)"),
    "mean_divides_by_B": ("out[j] = keys[lo:hi].sum(axis=0) / float(hi - lo)",
                          "out[j] = keys[lo:hi].sum(axis=0) / float(B)"),
    "block_off_by_one": ("hi = min(lo + B, L)\n        out[j] = keys", "hi = min(lo + B + 1, L)\n        out[j] = keys"),
    "visibility_strict": ("return np.nonzero(ends <= prefix_len)[0]", "return np.nonzero(ends < prefix_len)[0]"),
    "visibility_by_start": ("ends = np.minimum(np.arange(M) * S + B, L)", "ends = np.arange(M) * S"),
    "head_tie_higher_id": ("order = sorted(range(n), key=lambda i: (-values[i], i))",
                           "order = sorted(range(n), key=lambda i: (-values[i], -i))"),
    "head_pick_smallest": ("order = sorted(range(n), key=lambda i: (-values[i], i))",
                           "order = sorted(range(n), key=lambda i: (values[i], i))"),
    "importance_over_heads": ("importance[g] += A.sum(axis=1)", "importance[g] += A.sum(axis=0)[: A.shape[0]]"),
    "router_last_query_visibility": ("vis = visible_blocks(int(prefix_len[t0]), L, B, S)",
                                     "vis = visible_blocks(int(prefix_len[t1 - 1]) + B, L, B, S)"),
    "topk_tie_higher_index": ("order = np.lexsort((valid, -s[valid]))", "order = np.lexsort((-valid, -s[valid]))"),
    "topk_smallest": ("order = np.lexsort((valid, -s[valid]))", "order = np.lexsort((valid, s[valid]))"),
    "topk_not_ascending": ("chosen = np.sort(valid[order[:k]])", "chosen = valid[order[:k]]"),
    "topk_keeps_masked": ("valid = np.nonzero(s > -np.inf)[0]", "valid = np.arange(s.shape[0])"),
    "prefix_off_by_one": ("n_vis = int(min(max(prefix_len[t], 0), L))", "n_vis = int(min(max(prefix_len[t] + 1, 0), L))"),
    "cand_prefix_ignored": ("ok = (ids >= 0) & (ids < min(int(prefix_len[t]), L))", "ok = (ids >= 0) & (ids < L)"),
    "dagger_rerank_routed_heads": ("S_fine = candidate_scores(q, w, keys, seq_of, prefix_len, all_heads, cand)",
                                   "S_fine = candidate_scores(q, w, keys, seq_of, prefix_len, np.stack([coarse['heads'][t // q_block] for t in range(T)]), cand)"),
    "dagger_no_id_map": ("idx = topk_rows(S_fine, k, id_map=cand)\n    return {\"heads\"",
                         "idx = topk_rows(S_fine, k)\n    return {\"heads\""),
    "hisa_block_sum_over_blocks": ("bs[t, vis] = A.sum(axis=0)", "bs[t, vis] = A.sum(axis=0) * 0 + A.max(axis=0)"),
    "hisa_cand_wrong_block": ("ids = np.arange(j * S, j * S + B)", "ids = np.arange(j * S + 1, j * S + B + 1)"),
    "hisa_partial_not_masked": ("ids[(ids >= limit) | (ids < prev_end)] = -1",
                                "ids[(ids > limit) | (ids < prev_end)] = -1"),
    "hisa_cut_block_not_kept": ("            bs[t, jp] = np.inf", "            pass"),
    "hisa_cut_block_scored_low": ("            bs[t, jp] = np.inf", "            bs[t, jp] = -1.0"),
    "transposed_means": ("dots = q_t @ means.T", "dots = (means @ q_t.T).T[:, ::-1]"),
    # max pooling and overlapping windows (HISA explainer, section 七, 潜在改进)
    "max_pool_is_mean": ('out[j] = win.max(axis=0) if pool == "max"', 'out[j] = win.mean(axis=0) if pool == "max"'),
    "max_pool_is_min": ('out[j] = win.max(axis=0) if pool == "max"', 'out[j] = win.min(axis=0) if pool == "max"'),
    "window_start_by_B": ("        lo = j * S\n", "        lo = j * B\n"),
    "window_count_ceil_L_over_S": ("return 1 + (max(L - B, 0) + S - 1) // S", "return (L + S - 1) // S"),
    "window_count_one_short": ("return 1 + (max(L - B, 0) + S - 1) // S", "return 1 + max(L - B, 0) // S"),
    "window_no_dedup": ("ids[(ids >= limit) | (ids < prev_end)] = -1", "ids[ids >= limit] = -1"),
    "window_dedup_against_first_only": ("            prev_end = j * S + B",
                                        "            prev_end = j * S + B if prev_end < 0 else prev_end"),
    "window_cut_first_only": ("                bs[t, jp] = np.inf", "                bs[t, jp] = np.inf\n                break"),
    "window_stride_dropped_in_router": ("vis = visible_blocks(int(prefix_len[t0]), L, B, S)",
                                        "vis = visible_blocks(int(prefix_len[t0]), L, B)"),
    "window_visibility_by_stride_end": ("ends = np.minimum(np.arange(M) * S + B, L)",
                                        "ends = np.minimum((np.arange(M) + 1) * S, L)"),
    "window_mean_divides_by_B": ("else win.sum(axis=0) / float(hi - lo)", "else win.sum(axis=0) / float(B)"),
    "iou_intersection_as_union": ("return len(sa & sb) / len(sa | sb)", "return len(sa & sb) / max(len(sa), len(sb))"),
}


def _build(name):
    old, new = MUTANTS[name]
    assert SRC.count(old) == 1, f"mutation anchor for {name} must match exactly once"
    mod = types.ModuleType(f"oracle_mutant_{name}")
    mod.__dict__["__builtins__"] = __builtins__
    exec(compile(SRC.replace(old, new), mod.__name__, "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name):
    mutant = _build(name)
    caught = []
    for check in pins.ALL_CHECKS:
        try:
            with np.errstate(all="ignore"):
                check(mutant)
        except Exception:  # noqa: BLE001 - any failure is a catch
            caught.append(check.__name__)
    assert caught, f"no pin catches the planted mistake {name}"

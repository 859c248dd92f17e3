"""Comparison rules between the CUDA path and the fp64 oracle.

Scores: |S_gpu - S_ora| <= 1e-3 * max(|S_ora|, |tau_t|), where tau_t is the
oracle's k-th largest score of row t; masked entries (-inf) must match exactly.

Selections (top-k tokens, routed heads, HISA blocks): for each row with oracle
threshold tau (the k-th largest oracle value) and tol = 1e-3 * max(|tau|, 1e-6)
  * every entry whose oracle value is > tau + tol is selected by the GPU;
  * every entry the GPU selects has oracle value >= tau - tol and is valid;
  * the GPU output is ascending, duplicate-free, -1 only as trailing padding,
    and holds min(k, #valid) entries.
Only entries whose oracle value lies within the tolerance of the threshold may
differ.  Separately, selections are checked bit-exactly against a CPU sort of
the GPU's own values (same precision on both sides of that decision).
"""
from __future__ import annotations

import numpy as np

REL = 1e-3


def kth_threshold(vals: np.ndarray, k: int) -> float:
    v = vals[vals > -np.inf]
    if v.size == 0:
        return 0.0
    if v.size <= k:
        return float(v.min())
    return float(np.partition(v, v.size - k)[v.size - k])


def check_scores(S_gpu: np.ndarray, S_ora: np.ndarray, k: int, what: str = "scores") -> float:
    """Elementwise score parity; returns the worst |diff| / allowance ratio."""
    S_gpu = np.asarray(S_gpu, dtype=np.float64)
    assert S_gpu.shape == S_ora.shape, (what, S_gpu.shape, S_ora.shape)
    worst = 0.0
    for t in range(S_ora.shape[0]):
        mo = S_ora[t] == -np.inf
        mg = S_gpu[t] == -np.inf
        bad = np.nonzero(mo != mg)[0]
        assert bad.size == 0, f"{what} row {t}: mask differs at {bad[:8]} (ora {S_ora[t, bad[:4]]}, gpu {S_gpu[t, bad[:4]]})"
        # +inf marks a forced choice (HISA: the block a causal prefix cuts): exact
        po = S_ora[t] == np.inf
        assert np.array_equal(po, S_gpu[t] == np.inf), f"{what} row {t}: +inf entries differ"
        mo = mo | po
        if mo.all():
            continue
        tau = kth_threshold(S_ora[t], k)
        allow = REL * np.maximum(np.abs(S_ora[t, ~mo]), abs(tau))
        allow = np.maximum(allow, 1e-30)
        diff = np.abs(S_gpu[t, ~mo] - S_ora[t, ~mo])
        assert np.isfinite(S_gpu[t, ~mo]).all(), f"{what} row {t}: non-finite GPU score"
        r = float((diff / allow).max())
        worst = max(worst, r)
        if r > 1.0:
            j = int(np.argmax(diff / allow))
            raise AssertionError(f"{what} row {t}: |diff| {diff[j]:.3e} > allowance {allow[j]:.3e} "
                                 f"(ora {S_ora[t, ~mo][j]!r}, gpu {S_gpu[t, ~mo][j]!r})")
    return worst


def check_selection(sel_gpu: np.ndarray, vals_ora: np.ndarray, k: int, what: str = "selection",
                    ids: np.ndarray | None = None) -> int:
    """One row.  sel_gpu: [k] selected ids (-1 padded).  vals_ora: oracle values
    by position.  ids: position -> id map (None: the id is the position).
    Returns how many selected entries differ from the oracle's own choice."""
    sel = np.asarray(sel_gpu, dtype=np.int64)
    n_valid = int((vals_ora > -np.inf).sum())
    want = min(k, n_valid)
    assert (sel[:want] >= 0).all() and (sel[want:] == -1).all(), f"{what}: padding wrong: {sel[:16]}.. count {want}"
    chosen = sel[:want]
    if ids is None:
        pos = chosen
    else:
        ids = np.asarray(ids, dtype=np.int64)
        lookup = {int(v): i for i, v in enumerate(ids) if v >= 0}
        assert all(int(c) in lookup for c in chosen), f"{what}: id not among the candidates"
        pos = np.array([lookup[int(c)] for c in chosen], dtype=np.int64)
    assert np.all(np.diff(pos) > 0), f"{what}: not strictly ascending"
    if want == 0:
        return 0
    tau = kth_threshold(vals_ora, k)
    tol = REL * max(abs(tau), 1e-6)
    assert np.all(vals_ora[pos] > -np.inf), f"{what}: masked entry selected"
    low = pos[vals_ora[pos] < tau - tol]
    assert low.size == 0, f"{what}: selected entries below tau - tol: {low[:8]} vals {vals_ora[low[:4]]} tau {tau}"
    must = np.nonzero(vals_ora > tau + tol)[0]
    missing = np.setdiff1d(must, pos)
    assert missing.size == 0, f"{what}: entries above tau + tol missing: {missing[:8]} vals {vals_ora[missing[:4]]} tau {tau}"
    # the oracle's own choice (rank order, lower position first)
    valid = np.nonzero(vals_ora > -np.inf)[0]
    order = np.lexsort((valid, -vals_ora[valid]))
    ora_pos = np.sort(valid[order[:want]])
    return int(np.setdiff1d(pos, ora_pos).size)


def cpu_topk_of(vals_f32: np.ndarray, k: int, ids: np.ndarray | None = None) -> np.ndarray:
    """Top-k of one row of fp32 values as the kernel defines it (score desc,
    position asc; -0 == +0; -inf/NaN never chosen), ascending, -1 padded."""
    v = np.asarray(vals_f32, dtype=np.float32).astype(np.float64)
    valid = np.nonzero((v > -np.inf) & ~np.isnan(v))[0]
    order = np.lexsort((valid, -v[valid]))
    chosen = np.sort(valid[order[:k]])
    out = np.full(k, -1, dtype=np.int64)
    mapped = chosen if ids is None else np.asarray(ids, dtype=np.int64)[chosen]
    out[: mapped.size] = mapped
    return out


def check_bit_exact_topk(idx_gpu: np.ndarray, vals_gpu: np.ndarray, k: int, ids: np.ndarray | None = None,
                         what: str = "top-k"):
    for t in range(idx_gpu.shape[0]):
        exp = cpu_topk_of(vals_gpu[t], k, None if ids is None else ids[t])
        got = np.asarray(idx_gpu[t], dtype=np.int64)
        if not np.array_equal(got, exp):
            d = np.nonzero(got != exp)[0]
            raise AssertionError(f"{what} row {t}: differs from a CPU sort of the GPU values at {d[:8]}: "
                                 f"gpu {got[d[:4]]} cpu {exp[d[:4]]}")

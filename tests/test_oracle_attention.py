"""The fp64 sparse-attention oracle against its pins, and planted mistakes in
copies of it (on the CPU) that the pins must catch."""
import inspect
import types

import numpy as np
import pytest

import oracle.attention_oracle as real
import pins_attention as pins

SRC = inspect.getsource(real)

MUTANTS = {
    "scale_dropped": ("s = scale * (q[t] @ rows.T)             # [Hq, n]", "s = (q[t] @ rows.T)             # [Hq, n]"),
    "keys_without_rotary_part": ("s = scale * (q[t] @ rows.T)             # [Hq, n]",
                                 "s = scale * (q[t][:, :d_v] @ rows[:, :d_v].T)             # [Hq, n]"),
    "values_from_tail": ("vals = rows[:, :d_v]                    # [n, d_v]", "vals = rows[:, -d_v:]                    # [n, d_v]"),
    "padding_not_skipped": ("return ids[(ids >= 0) & (ids < L)]", "return ids[ids < L]"),
    "count_instead_of_weight_sum": ("out[t] = (p @ vals) / l[:, None]", "out[t] = (p @ vals) / ids.size"),
    "max_over_heads": ("m = s.max(axis=1, keepdims=True)\n        p = np.exp(s - m)\n        l",
                       "m = s.max(axis=0, keepdims=True)\n        p = np.exp(s - m)\n        l"),
    "lse_without_max": ("lse[t] = m[:, 0] + np.log(l)", "lse[t] = np.log(l)"),
    "weights_not_exponentiated": ("p = np.exp(s - m)\n        l", "p = np.maximum(s - m + 10.0, 0.0)\n        l"),
    "sequence_ignored": ("rows = kv[int(seq_of[t])][ids]          # [n, d_qk]", "rows = kv[0][ids]          # [n, d_qk]"),
}


@pytest.mark.parametrize("check", pins.ATTN_CHECKS, ids=lambda c: c.__name__)
def test_attention_oracle_pin(check):
    check(real)


def _build(name):
    old, new = MUTANTS[name]
    assert SRC.count(old) == 1, f"mutation anchor for {name} must match exactly once"
    mod = types.ModuleType(f"attn_mutant_{name}")
    mod.__dict__["__builtins__"] = __builtins__
    exec(compile(SRC.replace(old, new), mod.__name__, "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_attention_mutant(name):
    mutant = _build(name)
    caught = []
    for check in pins.ATTN_CHECKS:
        try:
            with np.errstate(all="ignore"):
                check(mutant)
        except Exception:  # noqa: BLE001 - any failure is a catch
            caught.append(check.__name__)
    assert caught, f"no pin catches the planted mistake {name}"

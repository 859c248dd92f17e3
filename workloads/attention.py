"""Seeded synthetic inputs for the sparse attention after the indexer.

Inputs only: none of the attention's arithmetic lives here; the CUDA path and
the fp64 oracle consume exactly what these functions return (bf16 values
rounded once, here, round-to-nearest-even).

Shapes stand in for a DeepSeek-V3.2-shaped decode (the pages name the model; its
weights are not available): 128 query heads over one latent KV row of 576
entries per token (512 latent + 64 rotary), values = the first 512 entries.

* latent rows ~ N(0, 1) per entry (a normalised latent), bf16;
* q ~ N(0, 1) per entry, bf16;
* scale = 1 / sqrt(192) (the softmax scale of a 128 + 64 query-key head), so a
  score has a standard deviation near 1.7 and the weights are neither flat nor
  one-hot;
* idx: k distinct token ids per query, ascending (the indexer's output order),
  drawn uniformly from the query's cache, the last n_pad slots -1 (padding).
Each sequence's cache is drawn from its own seed (seed, b), so a test can
rebuild the rows of one sequence without drawing the others.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

DQK = 576
DV = 512
SCALE = 1.0 / float(np.sqrt(192.0))


@dataclass
class MlaBatch:
    q: torch.Tensor        # [T, Hq, 576] bf16
    kv: torch.Tensor       # [nseq, L, 576] bf16
    seq_of: torch.Tensor   # [T] int32
    idx: torch.Tensor      # [T, k] int32, -1 padded
    scale: float
    seed: int


def mla_cache_rows(seed: int, b: int, L: int) -> torch.Tensor:
    """Latent rows [L, 576] bf16 of sequence b."""
    rng = np.random.default_rng([seed, b])
    out = torch.empty((L, DQK), dtype=torch.bfloat16)
    step = 1 << 16
    for s in range(0, L, step):
        e = min(L, s + step)
        out[s:e] = torch.from_numpy(rng.standard_normal((e - s, DQK), dtype=np.float32)).to(torch.bfloat16)
    return out


def make_mla(seed: int, T: int, Hq: int, L: int, nseq: int, k: int, n_pad: int = 0,
             shared_cache: bool = False) -> MlaBatch:
    """T queries; query t reads cache t % nseq (or cache 0 when shared_cache)."""
    rng = np.random.default_rng(seed)
    q = torch.from_numpy(rng.standard_normal((T, Hq, DQK), dtype=np.float32)).to(torch.bfloat16)
    seq_of = np.zeros(T, dtype=np.int32) if shared_cache else (np.arange(T) % nseq).astype(np.int32)
    n_valid = min(k - n_pad, L)
    idx = np.full((T, k), -1, dtype=np.int32)
    for t in range(T):
        idx[t, :n_valid] = np.sort(rng.choice(L, size=n_valid, replace=False))
    kv = torch.empty((nseq, L, DQK), dtype=torch.bfloat16)
    for b in range(nseq):
        kv[b] = mla_cache_rows(seed, b, L)
    return MlaBatch(q=q, kv=kv, seq_of=torch.from_numpy(seq_of), idx=torch.from_numpy(idx), scale=SCALE, seed=seed)

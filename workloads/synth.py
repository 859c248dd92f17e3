"""Seeded synthetic inputs for the token indexer.

This module only draws inputs.  It holds none of the indexer's arithmetic, and
both the CUDA path and the fp64 oracle consume exactly what it returns (bf16
tensors are rounded once, here, with round-to-nearest-even; the oracle widens
those same values to fp64).

The shapes and value distributions stand in for the workloads the pages
measure on (DeepSeek-V3.2 with 64 indexer heads and GLM-5 with 32 heads, 32K to
128K contexts, top-k 2048; the LongBench / needle-in-a-haystack data and the
model weights are not available, so "planted" keys replace needles):

* keys  ~ N(0, 1) / sqrt(d) per coordinate (|k| ~ 1), stored bf16;
* q     ~ N(0, 1) per coordinate, stored bf16;
* w     ~ N(0, 1) / 8, fp32;
* planted key for query t = normalize(mean over heads of q[t, h]) + eps,
  eps ~ N(0, 0.1^2 / d) per coordinate, written at distinct uniform positions;
* the 128K prefill workload clusters 16 regions of 2048 tokens around 16
  centroids: k = c_i + 0.3 * eps with c_i, eps ~ N(0, 1) / sqrt(d).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

D = 128


@dataclass
class Workload:
    """One batch of indexer inputs (host tensors) plus the method's knobs."""

    name: str
    mode: str                  # "misa", "misa_dagger", "hisa" or "dense"
    q: torch.Tensor            # [T, H, d] bf16
    w: torch.Tensor            # [T, H] fp32
    keys: torch.Tensor         # [nseq, L, d] bf16
    seq_of: torch.Tensor       # [T] int32
    prefix_len: torch.Tensor   # [T] int32
    H: int
    h: int
    B: int
    k: int
    q_block: int = 1
    kp: int = 0                # MISA-dagger candidate count k'
    m: int = 0                 # HISA blocks kept
    shared_cache: bool = False  # one cache for every query (key_seq_stride = 0)
    planted: np.ndarray = field(default_factory=lambda: np.zeros((0, 0), np.int64))

    @property
    def T(self) -> int:
        return int(self.q.shape[0])

    @property
    def L(self) -> int:
        return int(self.keys.shape[1])

    @property
    def nseq(self) -> int:
        return int(self.keys.shape[0])

    @property
    def M(self) -> int:
        return (self.L + self.B - 1) // self.B


def _bf16(x: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)


def _planted_key(q_bf16_t: np.ndarray, rng: np.random.Generator) -> np.ndarray:
    """normalize(mean_h q[t, h]) + eps for one query (q given as fp32 values)."""
    u = q_bf16_t.mean(axis=0)
    u = u / np.linalg.norm(u)
    eps = rng.standard_normal(D, dtype=np.float32) * np.float32(0.1 / np.sqrt(D))
    return (u + eps).astype(np.float32)


def make_decode(name: str, seed: int, T: int, L: int, H: int, h: int, B: int, k: int,
                n_planted: int, shared_cache: bool = False, mode: str = "misa",
                kp: int = 0, m: int = 0, planted_range=(0.0, 1.0)) -> Workload:
    """Decode batch: T queries, each at the end of its own cache of L keys.

    With shared_cache=True every query reads one cache (nseq = 1).  Every query
    sees the whole cache (prefix_len = L).  Draw order: keys, q, w, planted
    positions, planted noise.
    """
    rng = np.random.default_rng(seed)
    nseq = 1 if shared_cache else T
    keys = rng.standard_normal((nseq, L, D), dtype=np.float32)
    keys *= np.float32(1.0 / np.sqrt(D))
    q = _bf16(rng.standard_normal((T, H, D), dtype=np.float32))
    w = torch.from_numpy((rng.standard_normal((T, H), dtype=np.float32) / np.float32(8.0)))
    q32 = q.to(torch.float32).numpy()
    lo = int(planted_range[0] * L)
    hi = max(int(planted_range[1] * L), lo + 1)
    planted = np.zeros((T, n_planted), dtype=np.int64)
    if n_planted:
        if shared_cache:
            pos = rng.choice(np.arange(lo, hi), size=T * n_planted, replace=False)
            planted = pos.reshape(T, n_planted)
        else:
            for t in range(T):
                planted[t] = rng.choice(np.arange(lo, hi), size=n_planted, replace=False)
        for t in range(T):
            b = 0 if shared_cache else t
            for p in planted[t]:
                keys[b, p] = _planted_key(q32[t], rng)
    return Workload(
        name=name, mode=mode, q=q, w=w, keys=_bf16(keys),
        seq_of=torch.tensor([0 if shared_cache else t for t in range(T)], dtype=torch.int32),
        prefix_len=torch.full((T,), L, dtype=torch.int32),
        H=H, h=h, B=B, k=k, q_block=1, kp=kp, m=m, shared_cache=shared_cache,
        planted=planted)


def make_prefill(name: str, seed: int, T: int, L: int, H: int, h: int, B: int, k: int,
                 q_block: int, n_regions: int, region_len: int, sigma: float = 0.3,
                 first_pos: int | None = None) -> Workload:
    """Causal prefill chunk: T consecutive queries over one cache of L keys.

    Query i sits at 1-based position first_pos + i and sees that many keys
    (prefix_len = position).  The default places the chunk at the end of the
    cache, so the last query sees all L keys.  Keys are N(0,1)/sqrt(d) except
    n_regions non-overlapping regions of region_len tokens clustered around
    their own centroid (k = c + sigma * eps).  Draw order: keys, region
    offsets, centroids and noise per region, q, w.
    """
    rng = np.random.default_rng(seed)
    keys = rng.standard_normal((1, L, D), dtype=np.float32)
    keys *= np.float32(1.0 / np.sqrt(D))
    slots = L // region_len
    if n_regions:
        chosen = np.sort(rng.choice(slots, size=n_regions, replace=False))
        for r in chosen:
            c = rng.standard_normal(D, dtype=np.float32) / np.float32(np.sqrt(D))
            eps = rng.standard_normal((region_len, D), dtype=np.float32) / np.float32(np.sqrt(D))
            keys[0, r * region_len:(r + 1) * region_len] = c + np.float32(sigma) * eps
    q = _bf16(rng.standard_normal((T, H, D), dtype=np.float32))
    w = torch.from_numpy(rng.standard_normal((T, H), dtype=np.float32) / np.float32(8.0))
    if first_pos is None:
        first_pos = L - T + 1
    prefix = torch.arange(first_pos, first_pos + T, dtype=torch.int32)
    return Workload(
        name=name, mode="misa", q=q, w=w, keys=_bf16(keys),
        seq_of=torch.zeros(T, dtype=torch.int32), prefix_len=prefix,
        H=H, h=h, B=B, k=k, q_block=q_block, shared_cache=True)


def make_local_decode(name: str, seed: int, T: int, L: int, H: int, h: int, B: int, k: int, n_planted: int,
                      region_len=(256, 4096), sigma: float = 0.3, planted_range=(0.0, 1.0)) -> Workload:
    """Decode batch whose keys have locality, with needles the dense score favours.

    Used only for the selection-quality figures (IoU, recall); the timed
    workloads are the ones below.  Each cache is cut into consecutive regions
    of uniform random length in region_len; region r draws a centroid
    c_r ~ N(0, 1) / sqrt(d) and its keys are c_r + sigma * eps (eps ~ N(0, 1) /
    sqrt(d)), so neighbouring keys resemble each other the way text does and a
    block statistic says something about its tokens.  Needle keys for query t
    point along the query rows of its positively weighted heads,
    normalize(sum_h max(w[t, h], 0) * q[t, h]) + N(0, 0.1^2 / d), at distinct
    uniform positions in planted_range.  Draw order: per cache region lengths,
    centroids and noise; then q, w, needle positions and noise.
    """
    rng = np.random.default_rng(seed)
    keys = np.empty((T, L, D), dtype=np.float32)
    for b in range(T):
        s = 0
        while s < L:
            n = int(rng.integers(region_len[0], region_len[1] + 1))
            n = min(n, L - s)
            c = rng.standard_normal(D, dtype=np.float32) / np.float32(np.sqrt(D))
            eps = rng.standard_normal((n, D), dtype=np.float32) / np.float32(np.sqrt(D))
            keys[b, s:s + n] = c + np.float32(sigma) * eps
            s += n
    q = _bf16(rng.standard_normal((T, H, D), dtype=np.float32))
    w = torch.from_numpy(rng.standard_normal((T, H), dtype=np.float32) / np.float32(8.0))
    q32 = q.to(torch.float32).numpy()
    w32 = w.numpy()
    lo = int(planted_range[0] * L)
    hi = max(int(planted_range[1] * L), lo + n_planted)
    planted = np.zeros((T, n_planted), dtype=np.int64)
    for t in range(T):
        planted[t] = rng.choice(np.arange(lo, hi), size=n_planted, replace=False)
        u = (np.maximum(w32[t], 0.0)[:, None] * q32[t]).sum(axis=0)
        u = u / max(float(np.linalg.norm(u)), 1e-12)
        for p_ in planted[t]:
            keys[t, p_] = u + rng.standard_normal(D, dtype=np.float32) * np.float32(0.1 / np.sqrt(D))
    return Workload(
        name=name, mode="misa", q=q, w=w, keys=_bf16(keys),
        seq_of=torch.arange(T, dtype=torch.int32), prefix_len=torch.full((T,), L, dtype=torch.int32),
        H=H, h=h, B=B, k=k, q_block=1, planted=planted)


# The five workloads, by what they are.  Names say the shape.
CONFIG_NAMES = (
    "tiny_decode_L4096",
    "dsv32_decode_L32768",
    "prefill_L131072",
    "glm5_dagger_decode_L65536",
    "hisa_decode_L131072",
)


def make_workload(name: str) -> Workload:
    """Full-size workload by name (see CONFIG_NAMES)."""
    if name == "tiny_decode_L4096":
        return make_decode(name, 1, T=16, L=4096, H=64, h=8, B=128, k=256,
                           n_planted=4, shared_cache=True)
    if name == "dsv32_decode_L32768":
        return make_decode(name, 2, T=32, L=32768, H=64, h=8, B=128, k=2048, n_planted=16)
    if name == "prefill_L131072":
        return make_prefill(name, 3, T=4096, L=131072, H=64, h=8, B=128, k=2048,
                            q_block=64, n_regions=16, region_len=2048)
    if name == "glm5_dagger_decode_L65536":
        return make_decode(name, 4, T=64, L=65536, H=32, h=8, B=128, k=2048,
                           n_planted=32, mode="misa_dagger", kp=8192)
    if name == "hisa_decode_L131072":
        return make_decode(name, 5, T=16, L=131072, H=64, h=64, B=128, k=2048,
                           n_planted=8, mode="hisa", m=64, planted_range=(0.4, 0.6))
    raise KeyError(name)


def random_scores(seed: int, T: int, n: int, tie_frac: float = 0.0,
                  neg_inf_frac: float = 0.0, zero_frac: float = 0.0) -> torch.Tensor:
    """fp32 score rows for exercising top-k on its own.

    A fraction of entries is overwritten with repeated values (ties), with -inf
    (masked) and with +0.0 / -0.0 so that the tie and sign rules are exercised.
    """
    rng = np.random.default_rng(seed)
    s = rng.standard_normal((T, n), dtype=np.float32)
    if tie_frac > 0:
        mask = rng.random((T, n)) < tie_frac
        vals = rng.choice(np.array([0.5, 1.25, 2.0, -0.75], dtype=np.float32), size=(T, n))
        s[mask] = vals[mask]
    if zero_frac > 0:
        mask = rng.random((T, n)) < zero_frac
        signs = rng.random((T, n)) < 0.5
        s[mask & signs] = np.float32(0.0)
        s[mask & ~signs] = np.float32(-0.0)
    if neg_inf_frac > 0:
        mask = rng.random((T, n)) < neg_inf_frac
        s[mask] = -np.inf
    return torch.from_numpy(s)

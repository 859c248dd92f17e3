"""Shared helpers of the GPU parity tests: device copies of a workload and the
matching fp64 arrays for the oracle (both from the same seeded tensors)."""
from __future__ import annotations

import numpy as np
import torch

import sparse_attention_token_misa_b200 as misa


def dev(x: torch.Tensor) -> torch.Tensor:
    return x.contiguous().cuda()


def f64(x: torch.Tensor) -> np.ndarray:
    return x.to(torch.float64).numpy()


def to_gpu(wl):
    return dict(q=dev(wl.q), w=dev(wl.w), keys=dev(wl.keys), seq_of=dev(wl.seq_of), prefix_len=dev(wl.prefix_len))


def to_ora(wl, seqs=None):
    """fp64 oracle arrays; `seqs` keeps only those caches (seq_of remapped)."""
    seq_of = wl.seq_of.numpy().astype(np.int64)
    if seqs is None:
        keys = f64(wl.keys)
    else:
        keys = f64(wl.keys[list(seqs)])
        remap = {int(s): i for i, s in enumerate(seqs)}
        seq_of = np.array([remap.get(int(s), -1) for s in seq_of], dtype=np.int64)
    return dict(q=f64(wl.q), w=wl.w.numpy().astype(np.float64), keys=keys, seq_of=seq_of,
                prefix_len=wl.prefix_len.numpy().astype(np.int64))


def assert_no_device_error(ws: torch.Tensor):
    bits = misa.error_query(ws)
    assert bits == 0, f"device error word = {bits:#x}"


def np_i(x: torch.Tensor) -> np.ndarray:
    return x.cpu().numpy().astype(np.int64)


def np_f(x: torch.Tensor) -> np.ndarray:
    return x.cpu().numpy().astype(np.float64)

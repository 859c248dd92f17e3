"""misa_route_heads_noalloc against misa_route_heads, on the GPU.

The no-workspace router exists for callers that cannot allocate device memory
where they route (an engine that reserved all device memory and gives plug-ins
no allocator; a serving loop where cudaMalloc / cudaFree, which can
synchronise the device, are not allowed).  It runs the same kernels with the
partial importances in a fixed array inside the library, so its heads and
importances must equal those of the workspace version, call after call: the
second call below reuses the array the first call left filled, with a
different shape.  This file is collected last so that a failure here cannot
stop the rest of the suite from running first.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import sparse_attention_token_misa_b200 as misa
from sparse_attention_token_misa_b200 import _native as nat
from workloads import make_decode, make_prefill

pytestmark = pytest.mark.gpu


def _inputs(wl):
    dev = torch.device("cuda", 0)
    q, w, keys = wl.q.to(dev), wl.w.to(dev), wl.keys.to(dev)
    so, pl = wl.seq_of.to(dev), wl.prefix_len.to(dev)
    means = misa.block_stats(keys, wl.B)
    return q, w, means, so, pl


def _takes_persistent_path(wl) -> bool:
    """True when the router runs its persistent (non-cluster) kernel for this
    shape, the path that keeps partial importances and per-decision counters in
    the scratch array.  Same arithmetic as the launcher: a cluster of up to 8
    CTAs per decision is used when a decision has at most 64 work items and one
    wave of clusters covers the batch."""
    shared = wl.nseq == 1
    qpm = 1
    while shared and qpm * 2 * wl.H <= 128 and wl.q_block % (qpm * 2) == 0:
        qpm *= 2
    n_bt = (wl.M + 63) // 64
    items_per_dec = (wl.q_block // qpm) * n_bt
    D = min(items_per_dec, 8)
    G = (wl.T + wl.q_block - 1) // wl.q_block
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    cluster = items_per_dec <= 64 and G * D <= sms
    return not cluster


def _scratch_bytes(wl) -> int:
    """Bytes of the fixed array the call uses (partials, then one counter per decision)."""
    M = (wl.L + wl.B - 1) // wl.B
    part = wl.T * ((M + 31) // 32) * wl.H * 4
    G = (wl.T + wl.q_block - 1) // wl.q_block
    return (part + 255) // 256 * 256 + 4 * G


def _persistent_cases():
    # causal prefill chunks over one shared cache: many work items per decision
    c = make_prefill("na_c", 43, T=256, L=32768, H=64, h=8, B=128, k=16, q_block=64, n_regions=2, region_len=1024)
    d = make_prefill("na_d", 44, T=200, L=40000, H=32, h=6, B=64, k=16, q_block=32, n_regions=1, region_len=512)
    return c, d


def _check_against_workspace_router(wl):
    q, w, means, so, pl = _inputs(wl)
    ref_heads, ref_imp = misa.route_heads(q, w, means, so, pl, wl.L, wl.B, wl.q_block, wl.h)
    heads, imp = nat.route_heads_noalloc(q, w, means, so, pl, wl.L, wl.B, wl.q_block, wl.h)
    torch.cuda.synchronize()
    assert torch.equal(heads, ref_heads)
    assert torch.allclose(imp, ref_imp, rtol=1e-6, atol=0.0)
    imp_np = imp.cpu().numpy()
    for g in range(heads.shape[0]):
        exp = np.sort(np.lexsort((np.arange(wl.H), -imp_np[g].astype(np.float64)))[: wl.h])
        assert np.array_equal(heads[g].cpu().numpy(), exp)


@pytest.mark.parametrize("order", ["c_then_d", "d_then_c"])
def test_noalloc_router_persistent_path_back_to_back(order):
    """Two calls in a row that both take the persistent path, so both use the
    fixed array's partials and counters; the second call finds the array as the
    first left it (different shape, different counter count)."""
    c, d = _persistent_cases()
    cases = [c, d] if order == "c_then_d" else [d, c]
    for wl in cases:
        assert _takes_persistent_path(wl), wl.name
        assert _scratch_bytes(wl) <= nat.ROUTE_NOALLOC_SCRATCH_BYTES, wl.name
        _check_against_workspace_router(wl)


@pytest.mark.parametrize("order", ["large_then_small", "small_then_large"])
def test_noalloc_router_matches_workspace_router(order):
    a = make_decode("na_a", 41, T=32, L=32768, H=64, h=8, B=128, k=16, n_planted=4)
    b = make_prefill("na_b", 42, T=70, L=3000, H=32, h=5, B=64, k=16, q_block=16, n_regions=1, region_len=256)
    cases = [a, b] if order == "large_then_small" else [b, a]
    for wl in cases:  # two calls in a row through the C ABI; the scratch keeps the previous call's data
        q, w, means, so, pl = _inputs(wl)
        ref_heads, ref_imp = misa.route_heads(q, w, means, so, pl, wl.L, wl.B, wl.q_block, wl.h)
        heads, imp = nat.route_heads_noalloc(q, w, means, so, pl, wl.L, wl.B, wl.q_block, wl.h)
        torch.cuda.synchronize()
        assert torch.equal(heads, ref_heads)
        assert torch.allclose(imp, ref_imp, rtol=1e-6, atol=0.0)
        # and the routed heads are a valid top-h of the importances (selection rule sanity)
        imp_np = imp.cpu().numpy()
        for g in range(heads.shape[0]):
            exp = np.sort(np.lexsort((np.arange(wl.H), -imp_np[g].astype(np.float64)))[: wl.h])
            assert np.array_equal(heads[g].cpu().numpy(), exp)


def test_noalloc_router_rejects_sizes_beyond_its_scratch():
    # 4096 queries x 32 chunks x 64 heads x 4 B = 32 MiB > the fixed scratch
    f = nat.lib().misa_route_heads_noalloc
    P, P2 = 1 << 20, (1 << 20) + 4096
    st = f(P, P, P, 1, 0, P, P, 4096, 64, 131072, 128, 64, 8, P2, None, None)
    assert st == 2  # MISA_ERR_UNSUPPORTED, before any launch

"""Host-side checks of the C ABI (no GPU needed).

* the library loads without a GPU and exports every function include/misa.h
  declares (and the binding knows each of them);
* argument validation rejects bad calls with the documented status before
  anything reaches the CUDA runtime (the pointers below are never touched);
* workspace sizing follows its documented formula.
"""
import ctypes
import os
import re

import pytest

import sparse_attention_token_misa_b200 as pkg
from sparse_attention_token_misa_b200 import _native as nat

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "misa.h")

OK, INVALID, UNSUPPORTED, WORKSPACE, CUDA, DEVICE = 0, 1, 2, 3, 4, 5

# fake, 16-byte aligned "device" addresses: validation must fail before use
P = 1 << 20
P2 = (1 << 20) + 4096
MIS = (1 << 20) + 4  # misaligned


def declared_functions():
    text = open(HEADER, encoding="utf-8").read()
    return re.findall(r"MISA_API\s+[\w\s\*]+?\b(\w+)\s*\(", text)


def test_library_loads_and_exports_every_declared_symbol():
    l = pkg.lib()
    names = declared_functions()
    assert len(names) == 24, names
    for n in names:
        assert hasattr(l, n), n
        assert n in nat.SIGNATURES, n
    assert set(nat.SIGNATURES) == set(names)
    assert l.misa_abi_version() == 1


def test_status_strings():
    for code in range(6):
        assert nat.status_string(code) != "unknown status"
    assert nat.status_string(99) == "unknown status"


def test_workspace_formula():
    ws = nat.workspace_bytes
    # router: 256 + (T * ceil(M/32) * H * 4 rounded up to 256) + 4 * T
    assert ws(nat.OP_ROUTE_HEADS, 32, 64, 32768, 128) == 256 + 32 * 8 * 64 * 4 + 4 * 32
    assert ws(nat.OP_ROUTE_HEADS, 3, 5, 100, 7) == 256 + 256 + 4 * 3
    assert ws(nat.OP_INDEX_SCORE, 5, 5, 5, 5) == 256
    assert ws(nat.OP_TOPK, 5, 5, 5, 5) == 256
    assert ws(nat.OP_APPEND_KEYS, 5, 5, 5, 5) == 256
    assert ws(nat.OP_INDEX_DECODE, 32, 64, 32768, 128, 2048) == 256   # the error word only
    assert ws(nat.OP_HIER_RERANK, 64, 32, 65536, 128, 2048, 8192) == 256 + 64 * 8192 * 4
    assert ws(nat.OP_HIER_RERANK, 2, 32, 100, 1, 3, 5) == 256 + 2 * 8 * 4
    assert ws(nat.OP_HISA_BLOCK_FILTER, 16, 64, 131072, 128, 64) == 256 + 16 * 1024 * 4
    assert ws(nat.OP_HISA_BLOCK_FILTER, 1, 2, 8, 3, 2) == 256 + 1 * 4 * 4
    # sparse attention: 256 + T * ceil(k / 256) * Hq * (512 + 2) * 4
    assert ws(nat.OP_SPARSE_MLA, 32, 128, 0, 0, 2048) == 256 + 32 * 8 * 128 * 514 * 4
    assert ws(nat.OP_SPARSE_MLA, 3, 16, 0, 0, 257) == 256 + 3 * 2 * 16 * 514 * 4
    assert ws(nat.OP_SPARSE_MLA, 3, 16, 0, 0, 0) == 0
    assert ws(99, 1, 1, 1, 1) == 0
    assert ws(nat.OP_ROUTE_HEADS, -1, 1, 1, 1) == 0


def topk(scores=P, T=2, n=64, row_stride=64, row_valid=None, id_map=None, id_map_stride=0, k=8, idx=P2,
         ws=P2 + 4096, ws_bytes=256):
    return pkg.lib().misa_topk(scores, T, n, row_stride, row_valid, id_map, id_map_stride, k, idx, ws, ws_bytes, None)


@pytest.mark.parametrize("kw,status", [
    (dict(k=0), INVALID),
    (dict(k=16385), UNSUPPORTED),
    (dict(T=0), INVALID),
    (dict(n=0), INVALID),
    (dict(scores=MIS), INVALID),
    (dict(row_stride=66), INVALID),
    (dict(row_stride=60), INVALID),
    (dict(scores=None), INVALID),
    (dict(idx=None), INVALID),
    (dict(id_map=P, id_map_stride=10), INVALID),
    (dict(ws=None), WORKSPACE),
    (dict(ws_bytes=255), WORKSPACE),
])
def test_topk_rejects(kw, status):
    assert topk(**kw) == status


def score(q=P, w=P, keys=P, nkeyseq=1, stride=0, seq_of=P, plen=P, T=4, H=64, L=1000, heads=P2, h=8, q_block=1,
          cand=None, n_cand=0, scores=P, row_stride=1000, ws=P2, ws_bytes=256):
    return pkg.lib().misa_index_score(q, w, keys, nkeyseq, stride, seq_of, plen, T, H, L, heads, h, q_block, cand,
                                      n_cand, scores, row_stride, ws, ws_bytes, None)


@pytest.mark.parametrize("kw,status", [
    (dict(T=0), INVALID),
    (dict(H=0), INVALID),
    (dict(H=129), UNSUPPORTED),
    (dict(h=0), INVALID),
    (dict(h=65), INVALID),
    (dict(q_block=0), INVALID),
    (dict(L=0), INVALID),
    (dict(q=MIS), INVALID),
    (dict(keys=MIS), INVALID),
    (dict(stride=100, nkeyseq=2), INVALID),
    (dict(stride=128, nkeyseq=2), INVALID),          # sequences would overlap (stride < L*128)
    (dict(row_stride=999), INVALID),
    (dict(cand=P, n_cand=0), INVALID),
    (dict(cand=P, n_cand=300, row_stride=200), INVALID),
    (dict(nkeyseq=0), INVALID),
    (dict(q=None), INVALID),
    (dict(scores=None), INVALID),
    (dict(ws=None), WORKSPACE),
    (dict(ws_bytes=100), WORKSPACE),
    (dict(nkeyseq=70000, stride=1 << 22, L=32768, row_stride=32768), UNSUPPORTED),  # rows beyond int32 TMA coords
])
def test_index_score_rejects(kw, status):
    assert score(**kw) == status


def route(q=P, w=P, means=P, hi=None, lo=None, nseq=1, mstride=0, seq_of=P, plen=P, T=4, H=64, L=1024, B=128,
          q_block=1, h=8, heads=P2, imp=None, ws=P2, ws_bytes=1 << 20):
    return pkg.lib().misa_route_heads(q, w, means, hi, lo, nseq, mstride, seq_of, plen, T, H, L, B, q_block, h, heads,
                                      imp, ws, ws_bytes, None)


@pytest.mark.parametrize("kw,status", [
    (dict(h=0), INVALID),
    (dict(h=65), INVALID),
    (dict(q_block=0), INVALID),
    (dict(B=0), INVALID),
    (dict(H=200), UNSUPPORTED),
    (dict(means=MIS), INVALID),
    (dict(mstride=6, nseq=2), INVALID),
    (dict(mstride=8 * 128 - 4, nseq=2), INVALID),   # M * 128 = 1024 required
    (dict(mstride=8 * 128 + 4, nseq=2), INVALID),   # rows of 128 means
    (dict(heads=None), INVALID),
    (dict(ws_bytes=256), WORKSPACE),
    (dict(ws=None), WORKSPACE),
    (dict(means=None), INVALID),                     # neither fp32 means nor the split
    (dict(hi=P), INVALID),                           # hi without lo
    (dict(lo=P), INVALID),
    (dict(means=None, hi=P, lo=MIS), INVALID),       # misaligned split
])
def test_route_rejects(kw, status):
    assert route(**kw) == status


def test_block_stats_rejects():
    f = pkg.lib().misa_block_stats
    assert f(P, 1, 100, 0, 0, P2, None, None, None) == INVALID
    assert f(P, 1, 100, 0, 5000, P2, None, None, None) == UNSUPPORTED
    assert f(MIS, 1, 100, 0, 4, P2, None, None, None) == INVALID
    assert f(P, 1, 100, 0, 4, MIS, None, None, None) == INVALID
    assert f(P, 2, 100, 4, 4, P2, None, None, None) == INVALID        # stride % 8
    assert f(P, 2, 100, 128, 4, P2, None, None, None) == INVALID      # overlapping sequences
    assert f(None, 1, 100, 0, 4, P2, None, None, None) == INVALID
    assert f(P, 0, 100, 0, 4, P2, None, None, None) == INVALID
    # the bf16 split: both outputs or neither, 16-byte aligned
    assert f(P, 1, 100, 0, 4, P2, P, None, None) == INVALID
    assert f(P, 1, 100, 0, 4, P2, None, P, None) == INVALID
    assert f(P, 1, 100, 0, 4, P2, P, MIS, None) == INVALID


def test_hier_rerank_and_hisa_reject():
    l = pkg.lib()
    r = l.misa_hier_rerank
    # k > kp
    assert r(P, P, P, 1, 0, P, P, 2, 32, 100, P, 4, 5, None, P2, P2, 1 << 20, None) == INVALID
    assert r(P, P, P, 1, 0, P, P, 2, 32, 100, None, 4, 2, None, P2, P2, 1 << 20, None) == INVALID
    assert r(P, P, P, 1, 0, P, P, 2, 32, 100, P, 4, 2, None, P2, P2, 64, None) == WORKSPACE
    hf = l.hisa_block_filter
    N = None
    assert hf(P, P, P, N, N, 1, 0, P, P, 2, 64, 1000, 128, 0, P2, P2, N, P2, 1 << 20, N) == INVALID
    assert hf(P, P, P, N, N, 1, 0, P, P, 2, 64, 1000, 128, 20000, P2, P2, N, P2, 1 << 20, N) == UNSUPPORTED
    assert hf(P, P, P, N, N, 1, 0, P, P, 2, 64, 1000, 128, 4, N, P2, N, P2, 1 << 20, N) == INVALID
    assert hf(P, P, P, N, N, 1, 0, P, P, 2, 64, 1000, 128, 4, P2, P2, N, P2, 256, N) == WORKSPACE
    # sequence stride of the means: whole 128-float rows (TMA rows)
    assert hf(P, P, P, N, N, 2, 8 * 128 + 4, P, P, 2, 64, 1000, 128, 4, P2, P2, N, P2, 1 << 20, N) == INVALID
    # the bf16 split: both or neither; with it the fp32 means may be absent
    assert hf(P, P, N, P, N, 1, 0, P, P, 2, 64, 1000, 128, 4, P2, P2, N, P2, 1 << 20, N) == INVALID
    assert hf(P, P, N, N, N, 1, 0, P, P, 2, 64, 1000, 128, 4, P2, P2, N, P2, 1 << 20, N) == INVALID


def test_error_query_rejects_null():
    bits = ctypes.c_uint32(0)
    assert pkg.lib().misa_error_query(None, None, ctypes.byref(bits)) == INVALID
    assert pkg.lib().misa_error_reset(None, None) == INVALID


def append(keys=P, nseq=2, key_seq_stride=1024 * 128, L_cap=1024, lens=P2, new_keys=P2 + 4096, n_new=1, B=128,
           means=P2 + 8192, hi=None, lo=None, means_seq_stride=8 * 128, ws=P2 + 16384, ws_bytes=256):
    return pkg.lib().misa_append_keys(keys, nseq, key_seq_stride, L_cap, lens, new_keys, n_new, B, means, hi, lo,
                                      means_seq_stride, ws, ws_bytes, None)


def test_append_keys_validation():
    # every case is rejected on the host; nothing is launched
    assert append(keys=None) == INVALID
    assert append(lens=None) == INVALID
    assert append(n_new=0) == INVALID
    assert append(B=0) == INVALID
    assert append(B=5000) == UNSUPPORTED
    assert append(keys=MIS) == INVALID
    assert append(new_keys=MIS) == INVALID
    assert append(key_seq_stride=1023 * 128) == INVALID      # shorter than L_cap rows
    assert append(means_seq_stride=7 * 128) == INVALID       # fewer than ceil(L_cap / B) blocks
    assert append(means_seq_stride=8 * 128 + 4) == INVALID   # not whole 128-float rows
    assert append(ws=None) == WORKSPACE
    assert append(ws_bytes=255) == WORKSPACE
    assert append(hi=P) == INVALID                           # split: both or neither
    assert append(hi=P, lo=MIS) == INVALID


def mla(q=P, kv=P, nseq=1, stride=0, L=1000, seq_of=P, T=2, Hq=128, idx=P2, k=300, idx_stride=300, scale=0.1,
        out=P2 + 4096, lse=None, ws=P2 + 8192, ws_bytes=1 << 22):
    return pkg.lib().misa_sparse_mla(q, kv, nseq, stride, L, seq_of, T, Hq, idx, k, idx_stride, scale, out, lse, ws,
                                     ws_bytes, None)


@pytest.mark.parametrize("kw,status", [
    (dict(q=None), INVALID),
    (dict(kv=None), INVALID),
    (dict(idx=None), INVALID),
    (dict(out=None), INVALID),
    (dict(T=0), INVALID),
    (dict(Hq=0), INVALID),
    (dict(Hq=129), UNSUPPORTED),
    (dict(k=0), INVALID),
    (dict(k=16385, idx_stride=16385), UNSUPPORTED),
    (dict(idx_stride=299), INVALID),              # rows shorter than k
    (dict(q=MIS), INVALID),
    (dict(kv=MIS), INVALID),
    (dict(out=MIS), INVALID),
    (dict(nseq=2, stride=4), INVALID),            # stride % 8
    (dict(nseq=2, stride=576 * 999), INVALID),    # sequences would overlap
    (dict(ws=None), WORKSPACE),
    (dict(ws_bytes=256), WORKSPACE),
])
def test_sparse_mla_rejects(kw, status):
    assert mla(**kw) == status


def test_shard_helpers_reject():
    l = pkg.lib()
    assert l.misa_shard_prefix(None, 4, 0, 100, P2, None) == INVALID
    assert l.misa_shard_prefix(P, 0, 0, 100, P2, None) == INVALID
    assert l.misa_shard_prefix(P, 4, -1, 100, P2, None) == INVALID
    assert l.misa_shard_prefix(P, 4, 0, 0, P2, None) == INVALID
    assert l.misa_shard_prefix(P, 4, 0, 1 << 31, P2, None) == UNSUPPORTED
    g = l.misa_gather_candidates
    assert g(None, 2, 100, 100, P, 8, 0, P2, P2, None) == INVALID
    assert g(P, 2, 100, 99, P, 8, 0, P2, P2, None) == INVALID      # rows shorter than n
    assert g(P, 2, 100, 100, P, 0, 0, P2, P2, None) == INVALID
    assert g(P, 2, 100, 100, P, 8, -5, P2, P2, None) == INVALID
    assert g(P, 2, 100, 100, P, 8, (1 << 31) - 50, P2, P2, None) == UNSUPPORTED


def test_selftest_needs_a_workspace():
    l = pkg.lib()
    assert l.misa_selftest_wait_timeout(None, 256, None) == WORKSPACE
    assert l.misa_selftest_wait_timeout(P, 255, None) == WORKSPACE


def test_window_entry_points_reject_and_count():
    l = pkg.lib()
    # window counts: 1 + ceil(max(L - B, 0) / S); 0 for a bad geometry
    assert l.misa_num_windows(10, 4, 2) == 4 and l.misa_num_windows(11, 4, 2) == 5
    assert l.misa_num_windows(3, 4, 2) == 1 and l.misa_num_windows(32768, 128, 128) == 256
    assert l.misa_num_windows(100, 4, 5) == 0 and l.misa_num_windows(100, 4, 0) == 0
    assert l.misa_num_windows(0, 4, 2) == 0
    f = l.misa_block_stats_ex
    assert f(P, 1, 100, 0, 8, 9, 0, P2, None, None, None) == INVALID     # S > B
    assert f(P, 1, 100, 0, 8, 0, 0, P2, None, None, None) == INVALID     # S < 1
    assert f(P, 1, 100, 0, 8, 4, 2, P2, None, None, None) == INVALID     # unknown pool
    assert f(P, 1, 100, 0, 5000, 4, 0, P2, None, None, None) == UNSUPPORTED
    a = l.misa_append_keys_ex
    assert a(P, 1, 0, 1024, P2, P2, 1, 128, 200, 0, P2, None, None, 8 * 128, P2, 256, None) == INVALID
    assert a(P, 1, 0, 1024, P2, P2, 1, 128, 64, 3, P2, None, None, 16 * 128, P2, 256, None) == INVALID
    # the statistics stride must hold every window of the cache (1024 keys, B 128, S 64: 15 windows)
    assert a(P, 2, 1024 * 128, 1024, P2, P2, 1, 128, 64, 0, P2, None, None, 14 * 128, P2, 256, None) == INVALID
    r = l.misa_route_heads_ex
    N = None
    assert r(P, P, P, N, N, 1, 0, P, P, 2, 64, 1000, 128, 129, 1, 8, P2, N, P2, 1 << 20, N) == INVALID
    assert r(P, P, P, N, N, 1, 0, P, P, 2, 64, 1000, 128, 0, 1, 8, P2, N, P2, 1 << 20, N) == INVALID
    # workspace sized for plain blocks is too small for windows every 32 keys
    need_blocks = nat.workspace_bytes(nat.OP_ROUTE_HEADS, 2, 64, 10000, 128)   # 79 blocks: 3 chunks of 32
    assert need_blocks < nat.workspace_bytes(nat.OP_ROUTE_HEADS, 2, 64, 10000, 32)  # 310 windows: 10 chunks
    assert r(P, P, P, N, N, 1, 0, P, P, 2, 64, 10000, 128, 32, 1, 8, P2, N, P2, need_blocks, N) == WORKSPACE
    hf = l.hisa_block_filter_ex
    assert hf(P, P, P, N, N, 1, 0, P, P, 2, 64, 1000, 128, 256, 4, P2, P2, N, P2, 1 << 20, N) == INVALID
    need = nat.workspace_bytes(nat.OP_HISA_BLOCK_FILTER, 2, 64, 1000, 128, 4)
    assert hf(P, P, P, N, N, 1, 0, P, P, 2, 64, 1000, 128, 32, 4, P2, P2, N, P2, need, N) == WORKSPACE


def test_index_score_blocks_rejects():
    f = pkg.lib().misa_index_score_blocks
    N = None
    good = dict(q=P, w=P, keys=P, nseq=1, stride=0, seq_of=P, pl=P, T=2, H=64, L=1000, blocks=P2, m=4, B=128,
                scores=P2, row_stride=512, ws=P2, ws_bytes=256)

    def call(**kw):
        a = dict(good, **kw)
        return f(a["q"], a["w"], a["keys"], a["nseq"], a["stride"], a["seq_of"], a["pl"], a["T"], a["H"], a["L"],
                 a["blocks"], a["m"], a["B"], a["scores"], a["row_stride"], a["ws"], a["ws_bytes"], N)

    assert call(B=100) == INVALID            # blocks of 64 or 128 keys only
    assert call(m=0) == INVALID
    assert call(blocks=None) == INVALID
    assert call(row_stride=511) == INVALID   # shorter than m * B
    assert call(q=MIS) == INVALID
    assert call(ws_bytes=64) == WORKSPACE


def test_index_decode_rejects():
    """misa_index_decode: shapes outside the fused kernel's limits are
    unsupported (the separate calls cover them); bad pointers, strides and a
    short workspace are rejected before any launch."""
    f = pkg.lib().misa_index_decode
    N = None
    good = dict(q=P, w=P, keys=P, nkeyseq=2, kstride=4096 * 128, hi=P2, lo=P2, nmeanseq=2, mstride=32 * 128,
                seq_of=P, pl=P, T=2, H=64, L=4096, B=128, h=8, k=256, heads=P2, imp=N, scores=P2, sstride=4096,
                idx=P2, ws=P2, ws_bytes=256)

    def call(**kw):
        a = dict(good, **kw)
        return f(a["q"], a["w"], a["keys"], a["nkeyseq"], a["kstride"], a["hi"], a["lo"], a["nmeanseq"],
                 a["mstride"], a["seq_of"], a["pl"], a["T"], a["H"], a["L"], a["B"], a["h"], a["k"], a["heads"],
                 a["imp"], a["scores"], a["sstride"], a["idx"], a["ws"], a["ws_bytes"], N)

    assert call(H=65) == UNSUPPORTED         # more than 64 router columns
    assert call(h=17) == UNSUPPORTED         # more than 16 routed heads
    assert call(L=65537, kstride=65537 * 128, sstride=65540) == UNSUPPORTED
    assert call(k=16385) == UNSUPPORTED
    assert call(h=0) == INVALID
    assert call(heads=None) == INVALID
    assert call(hi=None) == INVALID
    assert call(q=MIS) == INVALID
    assert call(sstride=4095) == INVALID     # shorter than L
    assert call(kstride=4095 * 128) == INVALID
    assert call(ws_bytes=255) == WORKSPACE

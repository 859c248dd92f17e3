"""Stage-by-stage parity of the CUDA kernels (through the C ABI) with the fp64
oracle, at sizes the oracle finishes in seconds that span several tiles and a
ragged tail, plus the edge cases of each stage.  Each stage is fed the same
seeded inputs (and, downstream, the oracle's own upstream decisions), so a
difference points at that stage."""
import numpy as np
import pytest
import torch

import oracle
import sparse_attention_token_misa_b200 as misa
from gpu_helpers import assert_no_device_error, dev, f64, np_f, np_i, to_gpu, to_ora
from parity import check_bit_exact_topk, check_scores, check_selection
from workloads import make_decode, make_prefill, random_scores

pytestmark = pytest.mark.gpu


# ------------------------------------------------------------------ block statistics
@pytest.mark.parametrize("nseq,L,B", [(1, 4096, 128), (3, 1000, 128), (2, 777, 64), (1, 5, 1), (1, 300, 4096),
                                      (2, 129, 128)])
def test_block_stats(nseq, L, B):
    wl = make_decode("bs", 11 + L, T=nseq, L=L, H=2, h=1, B=B, k=1, n_planted=0)
    keys = dev(wl.keys)
    means = misa.block_stats(keys, B)
    torch.cuda.synchronize()
    k64 = f64(wl.keys)
    for b in range(nseq):
        ref = oracle.block_means(k64[b], B)
        got = np_f(means[b])
        M = ref.shape[0]
        for j in range(M):
            blk = k64[b, j * B:min((j + 1) * B, L)]
            allow = 2e-5 * np.abs(blk).mean(axis=0) + 1e-12
            assert np.all(np.abs(got[j] - ref[j]) <= allow), (b, j)


# ------------------------------------------------------------------ top-k on its own
@pytest.mark.parametrize("T,n,k,ties,neg_inf,zeros", [
    (4, 4096, 256, 0.0, 0.0, 0.0),        # one CTA per row, 4 entries per thread
    (3, 32768, 2048, 0.0, 0.0, 0.0),      # cluster of 4 CTAs per row, 8 entries per thread
    (2, 131072, 2048, 0.0, 0.0, 0.0),     # cluster of 8, 16 entries per thread
    (5, 10001, 300, 0.3, 0.1, 0.1),       # ties, masked, +-0, ragged length
    (3, 50000, 100, 0.9, 0.0, 0.0),       # threshold bin far above candidate capacity
    (2, 70000, 9000, 0.0, 0.0, 0.0),      # k above the fast path's list capacity
    (2, 9000, 16384, 0.0, 0.2, 0.0),      # fewer valid entries than k (padding)
    (3, 7, 3, 0.5, 0.3, 0.3),             # tiny row
    (2, 20000, 1, 0.5, 0.0, 0.5),
    (2, 300000, 2048, 0.0, 0.0, 0.0),     # digit-radix cluster kernel (keys re-read from global)
    (3, 16385, 100, 0.2, 0.1, 0.1),       # cluster of 3, the last CTA holds one entry
    (4, 4097, 50, 0.3, 0.0, 0.2),         # 8 entries per thread, one valid in the last group
    (65, 1024, 64, 0.1, 0.0, 0.0),        # many short rows
    (3, 30000, 100, 0.9, 0.0, 0.0),       # the k-th entry's value-range bin holds most of the row
    (2, 12000, 700, 0.35, 0.0, 0.0),      # heavy ties at the threshold
    (2, 5000, 100, 0.0, 0.0, 1.0),        # every entry +-0: no value range, select by position
    (2, 3000, 10, 0.0, 0.0, 1.0),         # same, 4 entries per thread
    (2, 40960, 2048, 0.0, 0.0, 0.0),      # cluster of 5
    (2, 32768, 2048, 0.1, 0.0, 0.0),      # cluster of 4, ties
    (2, 32769, 2048, 0.0, 0.0, 0.0),      # cluster of 5, the last CTA holds one entry
    (2, 65536, 2048, 0.0, 0.1, 0.0),      # cluster of 8, 8 entries per thread
    (2, 131072, 5000, 0.2, 0.0, 0.0),     # cluster of 8, 16 entries per thread, ties
    (2, 65537, 2048, 0.0, 0.0, 0.0),      # 16 entries per thread, cluster of 5
    (3, 40000, 100, 0.0, 0.0, 1.0),       # cluster, every entry +-0: no value range
    (2, 45000, 700, 0.35, 0.0, 0.0),      # cluster per row, heavy ties at the threshold
    (2, 60000, 300, 0.3, 0.1, 0.1),       # cluster per row, ties, masked, +-0
    (2, 200000, 700, 0.35, 0.1, 0.0),     # digit-radix cluster kernel, heavy ties
])
def test_topk_exact(T, n, k, ties, neg_inf, zeros):
    _check_topk(random_scores(1000 + n + k, T, n, tie_frac=ties, neg_inf_frac=neg_inf, zero_frac=zeros), n, k)


@pytest.mark.parametrize("T,n,k,ties,neg_inf,zeros", [
    (300, 20000, 2048, 0.0, 0.0, 0.0),     # one CTA per row (at least two rows per SM)
    (300, 5001, 300, 0.3, 0.1, 0.1),       # ties, masked, +-0, ragged length
    (300, 3000, 100, 0.9, 0.0, 0.0),       # threshold among massive ties: radix over the row
    (300, 2000, 50, 0.0, 0.0, 1.0),        # all +-0
    (300, 700, 1000, 0.0, 0.3, 0.0),       # fewer valid entries than k
    (300, 131072, 2048, 0.1, 0.0, 0.0),    # prefill-length rows
])
def test_topk_many_rows(T, n, k, ties, neg_inf, zeros):
    _check_topk(random_scores(3000 + n + k, T, n, tie_frac=ties, neg_inf_frac=neg_inf, zero_frac=zeros), n, k)


def test_topk_many_rows_valid_and_id_map():
    T, n, k = 320, 6000, 128
    s = random_scores(78, T, n, tie_frac=0.2)
    valid = torch.from_numpy(np.random.default_rng(6).integers(0, n + 1, size=T).astype(np.int32))
    ids = torch.from_numpy(np.random.default_rng(7).integers(0, 10**6, size=(T, n)).astype(np.int32))
    idx = misa.topk(s.cuda(), k, row_valid=valid.cuda(), id_map=ids.cuda())
    torch.cuda.synchronize()
    got = np_i(idx)
    for t in range(T):
        row = s[t].numpy().astype(np.float64).copy()
        row[int(valid[t]):] = -np.inf
        exp = oracle.topk_ascending(row, k, ids[t].numpy())
        assert np.array_equal(got[t], exp), t


def test_topk_unusual_rows():
    """Rows whose first entries are all masked, +-inf entries, a single huge
    outlier that squeezes every other value into one bin."""
    n = 20000
    s = random_scores(5, 4, n)
    s[0, :8000] = float("-inf")
    s[1, 100] = float("inf")
    s[1, 5000] = float("-inf")
    s[2, 7] = 1e30
    s[3, :] = torch.linspace(-1.0, 1.0, n)
    for k in (1, 50, 2048, 15000):
        _check_topk(s, n, k)


def test_topk_register_rows():
    """Rows for the register-resident kernels' range and tie paths (one CTA
    per row up to 8192 entries, a cluster above): NaN entries (never
    selected), values a few ulps apart, a range too wide for fp32, one of
    denormals, values repeating every 16 positions (every lane of a warp in the
    same bin), and exactly 100 selectable entries."""
    rng = np.random.default_rng(11)
    for n in (1000, 4096, 8193, 32768, 65536):
        rows = []
        r = rng.standard_normal(n).astype(np.float32)
        r[rng.random(n) < 0.1] = np.nan
        rows.append(r)
        rows.append((np.float32(1.0) + rng.integers(0, 64, n).astype(np.float32) * np.float32(2.0**-23)))
        r = rng.standard_normal(n).astype(np.float32)
        r[0], r[n // 2] = np.float32(-3e38), np.float32(3e38)
        rows.append(r)
        rows.append((rng.random(n) * 1e-40).astype(np.float32))
        rows.append(np.tile(rng.standard_normal(16).astype(np.float32), n // 16 + 1)[:n])
        r = rng.standard_normal(n).astype(np.float32)
        r[rng.permutation(n)[: n - 100]] = -np.inf
        rows.append(r)
        s = torch.from_numpy(np.stack(rows))
        for k in (1, 100, min(2048, n)):
            _check_topk(s, n, k)


def _check_topk(s, n, k):
    T = s.shape[0]
    stride = (n + 3) // 4 * 4
    buf = torch.full((T, stride), float("nan"), dtype=torch.float32)
    buf[:, :n] = s
    g = buf.cuda()
    idx = misa.topk(g, k, n=n)
    torch.cuda.synchronize()
    got = np_i(idx)
    for t in range(T):
        exp = oracle.topk_ascending(s[t].numpy().astype(np.float64), k)
        assert np.array_equal(got[t], exp), (t, np.nonzero(got[t] != exp)[0][:8])


def test_topk_row_valid_and_id_map():
    T, n, k = 4, 5000, 64
    s = random_scores(77, T, n, tie_frac=0.2)
    valid = torch.tensor([5000, 100, 0, 3], dtype=torch.int32)
    ids = torch.from_numpy(np.random.default_rng(5).integers(0, 10**6, size=(T, n)).astype(np.int32))
    idx = misa.topk(s.cuda(), k, row_valid=valid.cuda(), id_map=ids.cuda())
    torch.cuda.synchronize()
    got = np_i(idx)
    for t in range(T):
        row = s[t].numpy().astype(np.float64).copy()
        row[int(valid[t]):] = -np.inf
        exp = oracle.topk_ascending(row, k, ids[t].numpy())
        assert np.array_equal(got[t], exp), t


# ------------------------------------------------------------------ token scoring
def _heads_from_oracle(wl, o):
    means = np.stack([oracle.block_means(o["keys"][b], wl.B) for b in range(o["keys"].shape[0])])
    heads, imp = oracle.route_heads(o["q"], o["w"], means, o["seq_of"], o["prefix_len"], wl.L, wl.B, wl.q_block, wl.h)
    return heads, imp, means


@pytest.mark.parametrize("T,L,H,h", [(5, 1000, 64, 8), (3, 4096, 32, 8), (2, 300, 64, 64), (4, 129, 16, 3),
                                     (2, 777, 128, 128), (3, 1, 8, 2)])
def test_index_score_decode_routed(T, L, H, h):
    """Per-query caches (TMA path, one query per MMA group), oracle heads as input."""
    wl = make_decode("sc", 100 + T + L, T=T, L=L, H=H, h=h, B=64, k=min(64, L), n_planted=min(2, L))
    g, o = to_gpu(wl), to_ora(wl)
    heads, _, _ = _heads_from_oracle(wl, o)
    ws = misa.alloc_workspace(256)
    S = misa.index_score(g["q"], g["w"], g["keys"], g["seq_of"], g["prefix_len"], heads=dev(torch.from_numpy(heads).int()),
                         h=heads.shape[1], workspace=ws)
    torch.cuda.synchronize()
    assert_no_device_error(ws)
    per_q = np.stack([heads[t] for t in range(T)])
    S_ora = oracle.index_scores(o["q"], o["w"], o["keys"], o["seq_of"], o["prefix_len"], per_q)
    check_scores(np_f(S), S_ora, wl.k)


@pytest.mark.parametrize("T,L,H,h,q_block", [(70, 1000, 64, 8, 64), (33, 2049, 64, 64, 1), (300, 515, 16, 1, 7),
                                             (17, 4096, 32, 4, 16), (5, 260, 128, 128, 2), (40, 384, 64, 2, 8)])
def test_index_score_shared_cache_causal(T, L, H, h, q_block):
    """One shared cache (several queries per MMA group), causal prefixes, ragged T and L."""
    wl = make_prefill("pf", 200 + T + L, T=T, L=L, H=H, h=h, B=64, k=min(128, L), q_block=q_block, n_regions=2,
                      region_len=64, first_pos=max(1, L - T - 37))
    g, o = to_gpu(wl), to_ora(wl)
    heads, _, _ = _heads_from_oracle(wl, o)
    ws = misa.alloc_workspace(256)
    S = misa.index_score(g["q"], g["w"], g["keys"], g["seq_of"], g["prefix_len"], heads=dev(torch.from_numpy(heads).int()),
                         h=h, q_block=q_block, workspace=ws)
    torch.cuda.synchronize()
    assert_no_device_error(ws)
    per_q = np.stack([heads[t // q_block] for t in range(T)])
    S_ora = oracle.index_scores(o["q"], o["w"], o["keys"], o["seq_of"], o["prefix_len"], per_q)
    check_scores(np_f(S), S_ora, wl.k)


@pytest.mark.parametrize("shared", [False, True])
def test_index_score_dense(shared):
    if shared:
        wl = make_prefill("dn", 7, T=9, L=1500, H=64, h=64, B=128, k=100, q_block=1, n_regions=1, region_len=128)
    else:
        wl = make_decode("dn", 8, T=4, L=1500, H=64, h=64, B=128, k=100, n_planted=3)
    g, o = to_gpu(wl), to_ora(wl)
    ws = misa.alloc_workspace(256)
    S = misa.index_score(g["q"], g["w"], g["keys"], g["seq_of"], g["prefix_len"], workspace=ws)
    torch.cuda.synchronize()
    assert_no_device_error(ws)
    _, S_ora = oracle.dense_indexer(o["q"], o["w"], o["keys"], o["seq_of"], o["prefix_len"], wl.k)
    check_scores(np_f(S), S_ora, wl.k)


def test_index_score_candidates():
    """Candidate (gather) mode: -1 slots, ids past the prefix, duplicates, ragged count."""
    T, L, H = 6, 3000, 32
    wl = make_decode("cd", 9, T=T, L=L, H=H, h=H, B=128, k=50, n_planted=2)
    wl.prefix_len[:] = torch.tensor([3000, 2500, 10, 0, 3000, 1], dtype=torch.int32)
    g, o = to_gpu(wl), to_ora(wl)
    rng = np.random.default_rng(3)
    n_cand = 517
    cand = rng.integers(-1, L, size=(T, n_cand)).astype(np.int32)
    cand[:, 5] = cand[:, 4]
    ws = misa.alloc_workspace(256)
    S = misa.index_score(g["q"], g["w"], g["keys"], g["seq_of"], g["prefix_len"], cand=dev(torch.from_numpy(cand)),
                         workspace=ws)
    torch.cuda.synchronize()
    assert_no_device_error(ws)
    S_ora = oracle.candidate_scores(o["q"], o["w"], o["keys"], o["seq_of"], o["prefix_len"],
                                    np.tile(np.arange(H), (T, 1)), cand)
    check_scores(np_f(S), S_ora, wl.k)


# ------------------------------------------------------------------ router
@pytest.mark.parametrize("T,L,H,h,B,q_block", [(16, 4096, 64, 8, 128, 1), (7, 1000, 32, 8, 64, 1),
                                               (130, 2000, 64, 8, 128, 64), (9, 100, 64, 64, 16, 4),
                                               (3, 777, 128, 5, 50, 2)])
def test_route_heads(T, L, H, h, B, q_block):
    if q_block == 1:
        wl = make_decode("rt", 300 + T, T=T, L=L, H=H, h=h, B=B, k=16, n_planted=2)
    else:
        wl = make_prefill("rt", 300 + T, T=T, L=L, H=H, h=h, B=B, k=16, q_block=q_block, n_regions=1,
                          region_len=min(256, L // 2))
    g, o = to_gpu(wl), to_ora(wl)
    means = np.stack([oracle.block_means(o["keys"][b], B) for b in range(o["keys"].shape[0])])
    heads_ora, imp_ora = oracle.route_heads(o["q"], o["w"], means, o["seq_of"], o["prefix_len"], L, B, q_block, h)
    ws = misa.alloc_workspace(misa.workspace_bytes(1, T, H, L, B))
    heads, imp = misa.route_heads(g["q"], g["w"], dev(torch.from_numpy(means).float()), g["seq_of"],
                                  g["prefix_len"], L, B, q_block, h, workspace=ws)
    torch.cuda.synchronize()
    assert_no_device_error(ws)
    imp_g, heads_g = np_f(imp), np_i(heads)
    for gi in range(heads_ora.shape[0]):
        check_selection(heads_g[gi], imp_ora[gi], h, what=f"heads g{gi}")
    check_scores(imp_g, imp_ora, h, what="importance")
    check_bit_exact_topk(heads_g, imp.cpu().numpy(), h, what="heads vs CPU sort of GPU importance")


def test_route_heads_workspace_contents_do_not_matter():
    """The router's workspace may hold anything on entry (a buffer reused from
    another call, or never initialised): fill it with 0xFF bytes (error word
    cleared) and route a prefill-shaped batch that takes the persistent path,
    whose per-decision counters live in the workspace; twice in a row, and
    equal to the result on a zeroed workspace."""
    T, L, H, h, B, q_block = 256, 20000, 64, 8, 128, 64
    wl = make_prefill("rtff", 777, T=T, L=L, H=H, h=h, B=B, k=16, q_block=q_block, n_regions=1, region_len=1024)
    g, o = to_gpu(wl), to_ora(wl)
    means = np.stack([oracle.block_means(o["keys"][b], B) for b in range(o["keys"].shape[0])])
    m_d = dev(torch.from_numpy(means).float())
    nbytes = misa.workspace_bytes(1, T, H, L, B)
    ws0 = misa.alloc_workspace(nbytes)
    ref_heads, ref_imp = misa.route_heads(g["q"], g["w"], m_d, g["seq_of"], g["prefix_len"], L, B, q_block, h,
                                          workspace=ws0)
    ws = misa.alloc_workspace(nbytes)
    ws.fill_(0xFF)
    misa.error_reset(ws)
    for _ in range(2):
        heads, imp = misa.route_heads(g["q"], g["w"], m_d, g["seq_of"], g["prefix_len"], L, B, q_block, h,
                                      workspace=ws)
        torch.cuda.synchronize()
        assert_no_device_error(ws)
        assert torch.equal(heads, ref_heads)
        assert torch.equal(imp, ref_imp)
    heads_ora, imp_ora = oracle.route_heads(o["q"], o["w"], means, o["seq_of"], o["prefix_len"], L, B, q_block, h)
    for gi in range(heads_ora.shape[0]):
        check_selection(np_i(heads)[gi], imp_ora[gi], h, what=f"heads g{gi}")


# ------------------------------------------------------------------ HISA block filter
@pytest.mark.parametrize("T,L,B,m", [(4, 5000, 128, 8), (3, 1000, 64, 40), (2, 777, 100, 3), (2, 300, 128, 9)])
def test_hisa_block_filter(T, L, B, m):
    wl = make_decode("hf", 400 + L, T=T, L=L, H=64, h=64, B=B, k=16, n_planted=3, mode="hisa", m=m)
    wl.prefix_len[-1] = max(1, L // 2)
    g, o = to_gpu(wl), to_ora(wl)
    means = np.stack([oracle.block_means(o["keys"][b], B) for b in range(o["keys"].shape[0])])
    blocks_o, cand_o, bs_o = oracle.hisa_block_filter(o["q"], o["w"], means, o["seq_of"], o["prefix_len"], L, B, m)
    blocks, cand, bs = misa.hisa_block_filter(g["q"], g["w"], dev(torch.from_numpy(means).float()), g["seq_of"],
                                              g["prefix_len"], L, B, m, want_scores=True)
    torch.cuda.synchronize()
    check_scores(np_f(bs), bs_o, m, what="block scores")
    blocks_g = np_i(blocks)
    for t in range(T):
        check_selection(blocks_g[t], bs_o[t], m, what=f"blocks t{t}")
    check_bit_exact_topk(blocks_g, bs.cpu().numpy(), m, what="blocks vs CPU sort of GPU block scores")
    # expansion is exact integer work given the blocks
    cand_g = np_i(cand)
    for t in range(T):
        limit = min(int(o["prefix_len"][t]), L)
        exp = np.full(m * B, -1)
        for i, j in enumerate(blocks_g[t]):
            if j >= 0:
                ids = np.arange(j * B, j * B + B)
                ids[ids >= limit] = -1
                exp[i * B:(i + 1) * B] = ids
        assert np.array_equal(cand_g[t], exp), t


@pytest.mark.parametrize("T,L,H,B,m", [(9, 3000, 32, 128, 6), (6, 1500, 16, 64, 5), (5, 2000, 64, 100, 4)])
def test_hisa_block_filter_shared_cache_causal(T, L, H, B, m):
    """One cache shared by every query (several queries per MMA row group),
    causal prefixes that end inside a block (the cut block is kept, +inf)."""
    wl = make_prefill("hfp", 500 + L, T=T, L=L, H=H, h=H, B=B, k=16, q_block=1, n_regions=0, region_len=1,
                      first_pos=L // 3)
    g, o = to_gpu(wl), to_ora(wl)
    means = oracle.block_means(o["keys"][0], B)[None]
    blocks_o, cand_o, bs_o = oracle.hisa_block_filter(o["q"], o["w"], means, o["seq_of"], o["prefix_len"], L, B, m)
    blocks, cand, bs = misa.hisa_block_filter(g["q"], g["w"], dev(torch.from_numpy(means).float()), g["seq_of"],
                                              g["prefix_len"], L, B, m, want_scores=True)
    torch.cuda.synchronize()
    check_scores(np_f(bs), bs_o, m, what="block scores")
    blocks_g = np_i(blocks)
    for t in range(T):
        check_selection(blocks_g[t], bs_o[t], m, what=f"blocks t{t}")
        p = int(wl.prefix_len[t])
        if p % B and p < L:
            assert p // B in blocks_g[t], (t, p)


# ------------------------------------------------------------------ MISA-dagger rerank
def test_hier_rerank():
    T, L, H, kp, k = 5, 4000, 32, 700, 150
    wl = make_decode("hr", 12, T=T, L=L, H=H, h=8, B=128, k=k, n_planted=4, mode="misa_dagger", kp=kp)
    g, o = to_gpu(wl), to_ora(wl)
    rng = np.random.default_rng(9)
    cand = np.sort(rng.choice(L, size=(T, kp), replace=True), axis=1).astype(np.int32)
    cand = np.array([np.unique(r)[:kp] for r in cand], dtype=object)
    cand = np.stack([np.pad(r, (0, kp - len(r)), constant_values=-1) for r in cand]).astype(np.int32)
    ws = misa.alloc_workspace(misa.workspace_bytes(4, T, H, L, 1, k, kp))
    idx, cs = misa.hier_rerank(g["q"], g["w"], g["keys"], g["seq_of"], g["prefix_len"], dev(torch.from_numpy(cand)),
                               k, want_scores=True, workspace=ws)
    torch.cuda.synchronize()
    assert_no_device_error(ws)
    S_ora = oracle.candidate_scores(o["q"], o["w"], o["keys"], o["seq_of"], o["prefix_len"],
                                    np.tile(np.arange(H), (T, 1)), cand)
    check_scores(np_f(cs), S_ora, k)
    idx_g = np_i(idx)
    for t in range(T):
        check_selection(idx_g[t], S_ora[t], k, what=f"rerank t{t}", ids=cand[t])
    check_bit_exact_topk(idx_g, cs.cpu().numpy(), k, ids=cand, what="rerank vs CPU sort")


# ------------------------------------------------------------------ device-side checks
def test_bad_seq_index_is_recorded_not_faulted():
    wl = make_decode("bad", 13, T=3, L=300, H=16, h=4, B=64, k=8, n_planted=0)
    g = to_gpu(wl)
    g["seq_of"] = dev(torch.tensor([0, 7, 1], dtype=torch.int32))   # 7 is out of range
    ws = misa.alloc_workspace(256)
    heads = dev(torch.tensor([[0, 1, 2, 3]] * 3, dtype=torch.int32))
    misa.index_score(g["q"], g["w"], g["keys"], g["seq_of"], g["prefix_len"], heads=heads, h=4, workspace=ws)
    torch.cuda.synchronize()
    assert misa.error_query(ws) & misa._native.DEVERR_BAD_SEQ
    misa.error_reset(ws)
    assert misa.error_query(ws) == 0

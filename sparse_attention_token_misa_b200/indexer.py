"""The four indexers as sequences of libmisa calls with preallocated buffers.

Each class owns its device buffers (outputs and workspaces) for one batch shape
and issues the C-ABI calls on the current CUDA stream in `run`, so a step
allocates nothing and can be captured in a CUDA graph.  All arithmetic runs in
the library's kernels.  `means` is what `block_stats` returns: the fp32 block
means, or the tuple (means, means_hi, means_lo) with their bf16 split, which
the router and the block filter then read directly.

* MisaIndexer   -- router (h of H heads per query block), routed token scoring,
                   top-k.  MISA page (gist.science), "Methodology: MISA".
* DenseIndexer  -- all H heads score every token, top-k (the DSA indexer).
* MisaDaggerIndexer -- routed coarse top-k', all-head rerank, top-k.  MISA page,
                   "Hierarchical variant (MISA-dagger)".
* HisaIndexer   -- block filter (top-m blocks), all-head scoring of their
                   tokens, top-k.  HISA explainer (zhichai.net), 三, Stage 1/2.
"""
from __future__ import annotations

import torch

from . import _native as nat


def _pad4(n: int) -> int:
    return (n + 3) // 4 * 4


def _means_args(means) -> dict:
    if isinstance(means, tuple):
        m, hi, lo = means
        return dict(means=m, means_hi=hi, means_lo=lo)
    return dict(means=means)


def capture_graph(fn) -> torch.cuda.CUDAGraph:
    """Capture the library calls `fn` issues into a CUDA graph.

    `fn` runs once eagerly on a side stream first (kernel attributes, TMA maps
    and modules are set up outside the capture), then once under capture.  The
    graph replays the same kernels on the same buffers with one launch.
    """
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        fn()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    torch.cuda.synchronize()
    return g


class MisaIndexer:
    """Router + routed token scoring + top-k for one batch shape.

    fused=True runs the step through misa_index_decode (decode: one routing
    decision per query; needs the bf16 split of the block means): router and
    scoring in one kernel, the top-k behind it; route / score / select stay
    available as the three separate calls."""

    def __init__(self, T: int, H: int, h: int, L: int, B: int, k: int, q_block: int = 1, device="cuda",
                 stride: int | None = None, fused: bool = False):
        self.T, self.H, self.h, self.L, self.B, self.k, self.q_block = T, H, h, L, B, k, q_block
        self.fused = fused
        if fused and (q_block != 1 or (stride is not None and stride != B)):
            raise ValueError("the fused decode step routes per query over plain blocks")
        self.stride = B if stride is None else stride   # window stride of the block statistics
        G = (T + q_block - 1) // q_block
        self.heads = torch.empty((G, h), dtype=torch.int32, device=device)
        self.importance = torch.empty((G, H), dtype=torch.float32, device=device)
        self.scores_buf = torch.empty((T, _pad4(L)), dtype=torch.float32, device=device)
        self.scores = self.scores_buf[:, :L]
        self.idx = torch.empty((T, k), dtype=torch.int32, device=device)
        self.ws_route = nat.alloc_workspace(nat.workspace_bytes(nat.OP_ROUTE_HEADS, T, H, L, self.stride), device)
        self.ws = nat.alloc_workspace(256, device)
        if fused:
            self.ws_decode = nat.alloc_workspace(nat.workspace_bytes(nat.OP_INDEX_DECODE, T, H, L, B, k), device)

    def route(self, q, w, means, seq_of, prefix_len, stream=None):
        nat.route_heads(q, w, seq_of=seq_of, prefix_len=prefix_len, L=self.L, B=self.B, q_block=self.q_block,
                        h=self.h, heads=self.heads, importance=self.importance, workspace=self.ws_route,
                        stream=stream, stride=self.stride, **_means_args(means))

    def score(self, q, w, keys, seq_of, prefix_len, stream=None):
        nat.index_score(q, w, keys, seq_of, prefix_len, heads=self.heads, h=self.h, q_block=self.q_block,
                        scores=self.scores_buf, workspace=self.ws, stream=stream)

    def select(self, prefix_len, stream=None):
        nat.topk(self.scores_buf, self.k, n=self.L, row_valid=prefix_len, idx=self.idx, workspace=self.ws,
                 stream=stream)

    def route_score(self, q, w, keys, means, seq_of, prefix_len, stream=None):
        """The fused step without its top-k (heads, importance, scores)."""
        _, hi, lo = means
        nat.index_decode(q, w, keys, hi, lo, seq_of, prefix_len, self.B, self.h, self.k, heads=self.heads,
                         importance=self.importance, scores=self.scores_buf, workspace=self.ws_decode,
                         select=False, stream=stream)

    def run(self, q, w, keys, means, seq_of, prefix_len, stream=None) -> torch.Tensor:
        if self.fused:
            _, hi, lo = means
            nat.index_decode(q, w, keys, hi, lo, seq_of, prefix_len, self.B, self.h, self.k, heads=self.heads,
                             importance=self.importance, scores=self.scores_buf, idx=self.idx,
                             workspace=self.ws_decode, stream=stream)
            return self.idx
        self.route(q, w, means, seq_of, prefix_len, stream)
        self.score(q, w, keys, seq_of, prefix_len, stream)
        self.select(prefix_len, stream)
        return self.idx

    def capture(self, q, w, keys, means, seq_of, prefix_len):
        """Graphs of the whole step and of its three stages, on these buffers."""
        self.g_step = capture_graph(lambda: self.run(q, w, keys, means, seq_of, prefix_len))
        self.g_route = capture_graph(lambda: self.route(q, w, means, seq_of, prefix_len))
        self.g_score = capture_graph(lambda: self.score(q, w, keys, seq_of, prefix_len))
        self.g_select = capture_graph(lambda: self.select(prefix_len))
        return self


class DenseIndexer:
    def __init__(self, T: int, H: int, L: int, k: int, device="cuda"):
        self.T, self.H, self.L, self.k = T, H, L, k
        self.scores_buf = torch.empty((T, _pad4(L)), dtype=torch.float32, device=device)
        self.scores = self.scores_buf[:, :L]
        self.idx = torch.empty((T, k), dtype=torch.int32, device=device)
        self.ws = nat.alloc_workspace(256, device)

    def score(self, q, w, keys, seq_of, prefix_len, stream=None):
        nat.index_score(q, w, keys, seq_of, prefix_len, scores=self.scores_buf, workspace=self.ws, stream=stream)

    def select(self, prefix_len, stream=None):
        nat.topk(self.scores_buf, self.k, n=self.L, row_valid=prefix_len, idx=self.idx, workspace=self.ws,
                 stream=stream)

    def run(self, q, w, keys, seq_of, prefix_len, stream=None) -> torch.Tensor:
        self.score(q, w, keys, seq_of, prefix_len, stream)
        self.select(prefix_len, stream)
        return self.idx

    def capture(self, q, w, keys, seq_of, prefix_len):
        self.g_step = capture_graph(lambda: self.run(q, w, keys, seq_of, prefix_len))
        self.g_score = capture_graph(lambda: self.score(q, w, keys, seq_of, prefix_len))
        self.g_select = capture_graph(lambda: self.select(prefix_len))
        return self


class MisaDaggerIndexer:
    """fused=True runs the coarse stage through misa_index_decode (decode, one
    routing decision per query)."""

    def __init__(self, T: int, H: int, h: int, L: int, B: int, kp: int, k: int, q_block: int = 1, device="cuda",
                 fused: bool = False):
        self.coarse = MisaIndexer(T, H, h, L, B, kp, q_block, device, fused=fused)
        self.T, self.H, self.L, self.kp, self.k = T, H, L, kp, k
        self.idx = torch.empty((T, k), dtype=torch.int32, device=device)
        self.cand_scores = torch.empty((T, kp), dtype=torch.float32, device=device)
        self.ws_rerank = nat.alloc_workspace(nat.workspace_bytes(nat.OP_HIER_RERANK, T, H, L, 1, k, kp), device)

    def run(self, q, w, keys, means, seq_of, prefix_len, stream=None, want_scores=False) -> torch.Tensor:
        cand = self.coarse.run(q, w, keys, means, seq_of, prefix_len, stream)
        nat.hier_rerank(q, w, keys, seq_of, prefix_len, cand, self.k, idx=self.idx,
                        cand_scores=self.cand_scores if want_scores else None, workspace=self.ws_rerank,
                        stream=stream)
        return self.idx

    def capture(self, q, w, keys, means, seq_of, prefix_len):
        self.g_step = capture_graph(lambda: self.run(q, w, keys, means, seq_of, prefix_len))
        return self


class HisaIndexer:
    """`stride` < B: the block statistics are overlapping windows of B keys every
    `stride` keys (as block_stats(..., stride=) writes them); candidates that
    two chosen windows share are listed once."""

    def __init__(self, T: int, H: int, L: int, B: int, m: int, k: int, device="cuda", stride: int | None = None):
        self.T, self.H, self.L, self.B, self.m, self.k = T, H, L, B, m, k
        self.stride = B if stride is None else stride
        self.by_blocks = self.stride == B and B in (64, 128)
        self.blocks = torch.empty((T, m), dtype=torch.int32, device=device)
        self.cand = torch.empty((T, m * B), dtype=torch.int32, device=device)
        self.scores_buf = torch.empty((T, _pad4(m * B)), dtype=torch.float32, device=device)
        self.scores = self.scores_buf[:, : m * B]
        self.idx = torch.empty((T, k), dtype=torch.int32, device=device)
        self.ws_filter = nat.alloc_workspace(nat.workspace_bytes(nat.OP_HISA_BLOCK_FILTER, T, H, L, self.stride, m),
                                             device)
        self.ws = nat.alloc_workspace(256, device)

    def run(self, q, w, keys, means, seq_of, prefix_len, stream=None) -> torch.Tensor:
        nat.hisa_block_filter(q, w, seq_of=seq_of, prefix_len=prefix_len, L=self.L, B=self.B, m=self.m,
                              blocks=self.blocks, cand=self.cand, workspace=self.ws_filter, stream=stream,
                              stride=self.stride, **_means_args(means))
        if self.by_blocks and keys.shape[0] > 1:
            # plain blocks of 64 or 128 keys in per-query caches: score them
            # block by block (a cache shared by every query, as in a causal
            # prefill, is read faster by the candidate gather)
            nat.index_score_blocks(q, w, keys, seq_of, prefix_len, self.blocks, self.B, scores=self.scores_buf,
                                   workspace=self.ws, stream=stream)
        else:
            nat.index_score(q, w, keys, seq_of, prefix_len, cand=self.cand, scores=self.scores_buf,
                            workspace=self.ws, stream=stream)
        nat.topk(self.scores_buf, self.k, n=self.m * self.B, id_map=self.cand, idx=self.idx, workspace=self.ws,
                 stream=stream)
        return self.idx

    def capture(self, q, w, keys, means, seq_of, prefix_len):
        self.g_step = capture_graph(lambda: self.run(q, w, keys, means, seq_of, prefix_len))
        return self

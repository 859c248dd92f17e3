"""Key-sharded (context-parallel) MISA indexer: one process per GPU, rank r
holding keys [s0_r, s1_r) of every sequence.

The pages do not shard the indexer; this is the library's key-sharded form of
the MISA step ("MISA: Mixture of Indexer Sparse Attention for Long-Context LLM
Inference", gist.science, Methodology), resting on two facts of the method:

* a head's importance is a sum over the visible blocks, so the per-shard sums
  add up to it: one all-reduce (sum) of the [decisions x H] partial importances
  gives every rank the same importances, and every rank picks the same h heads
  with the same top-k kernel (ties to the lower head id);
* the top-k of a row is the top-k of the union of the per-shard top-k lists:
  each rank scores its shard with the routed heads, keeps its local top-k as
  (score, global token id) pairs, one all-gather collects the W lists, and a
  top-k over the W*k candidates (ids as the id map) gives the row's top-k; the
  lists are ascending and concatenated in shard order, so a tie goes to the
  lower token id as in the unsharded indexer.

Shard boundaries are multiples of the block size B, so a shard's blocks are the
global blocks.  Every step is a libmisa call; torch.distributed (NCCL) carries
the two exchanges.  The phases are separate methods so that a test can run the
ranks of a group one after the other in one process and do the exchanges
itself.
"""
from __future__ import annotations

import torch

from . import _native as nat


def shard_bounds(L: int, B: int, world: int) -> list[tuple[int, int]]:
    """Split [0, L) into `world` contiguous shards of whole B-blocks (the last
    may end inside a block), as equal as the blocks allow."""
    M = (L + B - 1) // B
    if world < 1 or world > M:
        raise ValueError("need 1 <= world <= number of blocks")
    cuts = [min(L, (M * r // world) * B) for r in range(world + 1)]
    cuts[-1] = L
    return [(cuts[r], cuts[r + 1]) for r in range(world)]


class TorchShardComm:
    """The two exchanges over a torch.distributed process group (NCCL on GPUs)."""

    def __init__(self, group=None):
        import torch.distributed as dist

        self.dist = dist
        self.group = group
        self.world = dist.get_world_size(group)

    def all_reduce_sum_(self, t: torch.Tensor) -> torch.Tensor:
        self.dist.all_reduce(t, op=self.dist.ReduceOp.SUM, group=self.group)
        return t

    def all_gather(self, t: torch.Tensor) -> torch.Tensor:
        """[W, *t.shape]: rank w's tensor at index w (gathered along dim 0)."""
        t = t.contiguous()
        out = torch.empty((self.world * t.shape[0], *t.shape[1:]), dtype=t.dtype, device=t.device)
        self.dist.all_gather_into_tensor(out, t, group=self.group)
        return out.view(self.world, *t.shape)


def candidate_rows(gathered: torch.Tensor, out: torch.Tensor | None = None) -> torch.Tensor:
    """[W, T, k] (rank-major, as gathered) -> [T, W*k] rows in shard order."""
    W, T, k = gathered.shape
    if out is None:
        out = torch.empty((T, W * k), dtype=gathered.dtype, device=gathered.device)
    out.view(T, W, k).copy_(gathered.permute(1, 0, 2))
    return out


class ShardedMisaIndexer:
    """MISA indexer over one key shard; `run` does the whole step with a comm
    object (TorchShardComm in a real group)."""

    def __init__(self, T: int, H: int, h: int, L: int, B: int, k: int, s0: int, s1: int, world: int,
                 q_block: int = 1, device="cuda"):
        if s0 % B != 0 or not (0 <= s0 < s1 <= L):
            raise ValueError("a shard starts on a block boundary and is non-empty")
        if H % 4 != 0 or k % 4 != 0:
            raise ValueError("H and k must be multiples of 4 (importance and candidate rows are top-k rows)")
        self.T, self.H, self.h, self.L, self.B, self.k, self.q_block = T, H, h, L, B, k, q_block
        self.s0, self.s1, self.Ls, self.world = s0, s1, s1 - s0, world
        G = (T + q_block - 1) // q_block
        self.G = G
        self.local_prefix = torch.empty((T,), dtype=torch.int32, device=device)
        self.importance_buf = torch.zeros((G, H), dtype=torch.float32, device=device)
        self.importance = self.importance_buf
        self.route_heads_scratch = torch.empty((G, h), dtype=torch.int32, device=device)
        self.heads = torch.empty((G, h), dtype=torch.int32, device=device)
        self.scores_buf = torch.empty((T, (self.Ls + 3) // 4 * 4), dtype=torch.float32, device=device)
        self.local_idx = torch.empty((T, k), dtype=torch.int32, device=device)
        self.cand_scores = torch.empty((T, k), dtype=torch.float32, device=device)
        self.cand_ids = torch.empty((T, k), dtype=torch.int32, device=device)
        self.all_scores = torch.empty((T, world * k), dtype=torch.float32, device=device)
        self.all_ids = torch.empty((T, world * k), dtype=torch.int32, device=device)
        self.idx = torch.empty((T, k), dtype=torch.int32, device=device)
        self.ws_route = nat.alloc_workspace(nat.workspace_bytes(nat.OP_ROUTE_HEADS, T, H, self.Ls, B), device)
        self.ws = nat.alloc_workspace(256, device)

    # -- phase 1: this shard's partial head importances
    def route_partial(self, q, w, means, seq_of, prefix_len, stream=None, means_hi=None, means_lo=None):
        nat.shard_prefix(prefix_len, self.s0, self.Ls, out=self.local_prefix, stream=stream)
        nat.route_heads(q, w, means, seq_of, self.local_prefix, self.Ls, self.B, self.q_block, self.h,
                        heads=self.route_heads_scratch, importance=self.importance, workspace=self.ws_route,
                        stream=stream, means_hi=means_hi, means_lo=means_lo)
        return self.importance_buf

    # -- phase 2 (after the all-reduce of importance_buf): the same heads on every rank
    def select_heads(self, stream=None):
        nat.topk(self.importance_buf, self.h, n=self.H, idx=self.heads, workspace=self.ws, stream=stream)
        return self.heads

    # -- phase 3: score the shard with the routed heads, keep the local top-k as (score, global id)
    def local_candidates(self, q, w, keys, seq_of, stream=None):
        nat.index_score(q, w, keys, seq_of, self.local_prefix, heads=self.heads, h=self.h, q_block=self.q_block,
                        scores=self.scores_buf, workspace=self.ws, stream=stream)
        nat.topk(self.scores_buf, self.k, n=self.Ls, row_valid=self.local_prefix, idx=self.local_idx,
                 workspace=self.ws, stream=stream)
        nat.gather_candidates(self.scores_buf, self.local_idx, self.Ls, self.s0, out_scores=self.cand_scores,
                              out_ids=self.cand_ids, stream=stream)
        return self.cand_scores, self.cand_ids

    # -- phase 4 (after the all-gather): top-k over the W*k candidates of each row
    def merge(self, gathered_scores, gathered_ids, stream=None):
        W = gathered_scores.shape[0]
        if W != self.world:
            raise ValueError("one candidate list per rank")
        n = W * self.k
        candidate_rows(gathered_scores, out=self.all_scores)
        candidate_rows(gathered_ids, out=self.all_ids)
        nat.topk(self.all_scores, self.k, n=n, id_map=self.all_ids, idx=self.idx, workspace=self.ws, stream=stream)
        return self.idx

    def run(self, q, w, keys, means, seq_of, prefix_len, comm, stream=None) -> torch.Tensor:
        """The whole step on this rank: keys / means are this rank's shard
        ([nseq, s1 - s0, 128] and its block means, or the (means, hi, lo) tuple
        of block_stats)."""
        m = dict(means=means) if not isinstance(means, tuple) else dict(zip(("means", "means_hi", "means_lo"), means))
        imp = self.route_partial(q, w, m["means"], seq_of, prefix_len, stream, m.get("means_hi"), m.get("means_lo"))
        comm.all_reduce_sum_(imp)
        self.select_heads(stream)
        cs, ci = self.local_candidates(q, w, keys, seq_of, stream)
        return self.merge(comm.all_gather(cs), comm.all_gather(ci), stream)

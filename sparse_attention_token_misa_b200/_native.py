"""ctypes binding of libmisa.so (argument marshalling only).

Every function here forwards device pointers, sizes and the current CUDA
stream of torch to the C ABI declared in include/misa.h; all arithmetic runs
in the library's CUDA kernels.  If the library is missing or cannot be
loaded, the first call raises: there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmisa.so")

OP_ROUTE_HEADS = 1
OP_INDEX_SCORE = 2
OP_TOPK = 3
OP_HIER_RERANK = 4
OP_HISA_BLOCK_FILTER = 5
OP_APPEND_KEYS = 6
OP_SPARSE_MLA = 7
OP_INDEX_DECODE = 8

DEVERR_TIMEOUT = 1
DEVERR_BAD_SEQ = 2
DEVERR_BAD_HEAD = 4
DEVERR_BAD_LEN = 8
DEVERR_BAD_INDEX = 16

MLA_DQK = 576   # latent KV row: 512 latent + 64 rotary
MLA_DV = 512    # value part: the first 512 entries of a row

HEAD_DIM = 128
POOL = {"mean": 0, "max": 1}   # MISA_POOL_MEAN, MISA_POOL_MAX
ROUTE_NOALLOC_SCRATCH_BYTES = 2 << 20  # MISA_ROUTE_NOALLOC_SCRATCH_BYTES

_lib = None

c_i64 = ctypes.c_int64
c_int = ctypes.c_int
c_size = ctypes.c_size_t
c_vp = ctypes.c_void_p

# name -> (restype, argtypes), in the order of include/misa.h
SIGNATURES = {
    "misa_status_string": (ctypes.c_char_p, [c_int]),
    "misa_abi_version": (c_int, []),
    "misa_workspace_bytes": (c_size, [c_int, c_int, c_int, c_i64, c_int, c_int, c_int]),
    "misa_error_reset": (c_int, [c_vp, c_vp]),
    "misa_error_query": (c_int, [c_vp, c_vp, ctypes.POINTER(ctypes.c_uint32)]),
    "misa_block_stats": (c_int, [c_vp, c_i64, c_i64, c_i64, c_int, c_vp, c_vp, c_vp, c_vp]),
    "misa_num_windows": (c_i64, [c_i64, c_int, c_int]),
    "misa_block_stats_ex": (c_int, [c_vp, c_i64, c_i64, c_i64, c_int, c_int, c_int, c_vp, c_vp, c_vp, c_vp]),
    "misa_append_keys_ex": (c_int, [c_vp, c_i64, c_i64, c_i64, c_vp, c_vp, c_int, c_int, c_int, c_int, c_vp, c_vp,
                                    c_vp, c_i64, c_vp, c_size, c_vp]),
    "misa_route_heads_ex": (c_int, [c_vp, c_vp, c_vp, c_vp, c_vp, c_i64, c_i64, c_vp, c_vp, c_int, c_int, c_i64,
                                    c_int, c_int, c_int, c_int, c_vp, c_vp, c_vp, c_size, c_vp]),
    "hisa_block_filter_ex": (c_int, [c_vp, c_vp, c_vp, c_vp, c_vp, c_i64, c_i64, c_vp, c_vp, c_int, c_int, c_i64,
                                     c_int, c_int, c_int, c_vp, c_vp, c_vp, c_vp, c_size, c_vp]),
    "misa_append_keys": (c_int, [c_vp, c_i64, c_i64, c_i64, c_vp, c_vp, c_int, c_int, c_vp, c_vp, c_vp, c_i64,
                                 c_vp, c_size, c_vp]),
    "misa_route_heads": (c_int, [c_vp, c_vp, c_vp, c_vp, c_vp, c_i64, c_i64, c_vp, c_vp, c_int, c_int, c_i64,
                                 c_int, c_int, c_int, c_vp, c_vp, c_vp, c_size, c_vp]),
    "misa_route_heads_noalloc": (c_int, [c_vp, c_vp, c_vp, c_i64, c_i64, c_vp, c_vp, c_int, c_int, c_i64, c_int,
                                         c_int, c_int, c_vp, c_vp, c_vp]),
    "misa_index_score": (c_int, [c_vp, c_vp, c_vp, c_i64, c_i64, c_vp, c_vp, c_int, c_int, c_i64, c_vp, c_int,
                                 c_int, c_vp, c_int, c_vp, c_i64, c_vp, c_size, c_vp]),
    "misa_topk": (c_int, [c_vp, c_int, c_i64, c_i64, c_vp, c_vp, c_i64, c_int, c_vp, c_vp, c_size, c_vp]),
    "misa_index_score_blocks": (c_int, [c_vp, c_vp, c_vp, c_i64, c_i64, c_vp, c_vp, c_int, c_int, c_i64, c_vp,
                                        c_int, c_int, c_vp, c_i64, c_vp, c_size, c_vp]),
    "misa_index_decode": (c_int, [c_vp, c_vp, c_vp, c_i64, c_i64, c_vp, c_vp, c_i64, c_i64, c_vp, c_vp, c_int,
                                  c_int, c_i64, c_int, c_int, c_int, c_vp, c_vp, c_vp, c_i64, c_vp, c_vp, c_size,
                                  c_vp]),
    "misa_hier_rerank": (c_int, [c_vp, c_vp, c_vp, c_i64, c_i64, c_vp, c_vp, c_int, c_int, c_i64, c_vp, c_int,
                                 c_int, c_vp, c_vp, c_vp, c_size, c_vp]),
    "misa_selftest_wait_timeout": (c_int, [c_vp, c_size, c_vp]),
    "misa_shard_prefix": (c_int, [c_vp, c_int, c_i64, c_i64, c_vp, c_vp]),
    "misa_gather_candidates": (c_int, [c_vp, c_int, c_i64, c_i64, c_vp, c_int, c_i64, c_vp, c_vp, c_vp]),
    "misa_sparse_mla": (c_int, [c_vp, c_vp, c_i64, c_i64, c_i64, c_vp, c_int, c_int, c_vp, c_int, c_i64,
                                ctypes.c_float, c_vp, c_vp, c_vp, c_size, c_vp]),
    "hisa_block_filter": (c_int, [c_vp, c_vp, c_vp, c_vp, c_vp, c_i64, c_i64, c_vp, c_vp, c_int, c_int, c_i64,
                                  c_int, c_int, c_vp, c_vp, c_vp, c_vp, c_size, c_vp]),
}


class MisaError(RuntimeError):
    """A libmisa call returned a non-OK status."""

    def __init__(self, name: str, status: int):
        self.status = status
        super().__init__(f"{name}: status {status} ({status_string(status)})")


def lib() -> ctypes.CDLL:
    """Load libmisa.so (once).  Raises if it is missing: nothing runs without it."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"libmisa.so not found at {LIB_PATH}; build it with "
                "`python -m sparse_attention_token_misa_b200.build`")
        l = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(l, name)
            f.restype = res
            f.argtypes = args
        _lib = l
    return _lib


def status_string(status: int) -> str:
    return lib().misa_status_string(int(status)).decode()


def _call(name: str, *args) -> None:
    st = getattr(lib(), name)(*args)
    if st != 0:
        raise MisaError(name, st)


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _p(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libmisa takes device tensors")
    return t.data_ptr()


def _req(t: torch.Tensor, dtype, name: str, contiguous: bool = True):
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if contiguous and not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _shape(t, name: str, *dims):
    """Raise unless t has exactly these sizes (None: any).  The library sees
    only pointers, so a tensor smaller than the call implies must be caught
    here, before any launch."""
    if t is None:
        return
    if t.dim() != len(dims) or any(d is not None and t.shape[i] != d for i, d in enumerate(dims)):
        raise ValueError(f"{name}: expected shape {tuple('*' if d is None else d for d in dims)}, "
                         f"got {tuple(t.shape)}")


def _rows(t, name: str, T: int, min_cols: int):
    """A [T, >= min_cols] matrix with contiguous rows."""
    if t.dim() != 2 or t.shape[0] != T or t.shape[1] < min_cols or t.stride(1) != 1:
        raise ValueError(f"{name}: expected [{T}, >= {min_cols}] with contiguous rows, got {tuple(t.shape)}")


def workspace_bytes(op: int, T: int, H: int, L: int, B: int, k: int = 0, kp: int = 0) -> int:
    return int(lib().misa_workspace_bytes(op, T, H, L, B, k, kp))


def alloc_workspace(nbytes: int, device=None) -> torch.Tensor:
    """Zeroed uint8 device buffer of at least nbytes (16-byte aligned by torch)."""
    return torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device=device or "cuda")


def error_reset(workspace: torch.Tensor, stream=None) -> None:
    _call("misa_error_reset", _p(workspace), _stream(stream))


def error_query(workspace: torch.Tensor, stream=None) -> int:
    bits = ctypes.c_uint32(0)
    st = lib().misa_error_query(_p(workspace), _stream(stream), ctypes.byref(bits))
    if st not in (0, 5):
        raise MisaError("misa_error_query", st)
    return int(bits.value)


def _key_stride(keys: torch.Tensor) -> int:
    # one cache for every query -> stride 0 lets the kernel batch queries per MMA
    return 0 if keys.shape[0] == 1 else int(keys.stride(0))


def _split_pair(hi, lo, like: torch.Tensor | None = None):
    """Check the bf16 hi / lo split of the block means (both or neither)."""
    if (hi is None) != (lo is None):
        raise ValueError("means_hi and means_lo go together")
    if hi is None:
        return
    _req(hi, torch.bfloat16, "means_hi"); _req(lo, torch.bfloat16, "means_lo")
    for t in (hi, lo):
        if like is not None and (t.shape != like.shape or t.stride() != like.stride()):
            raise ValueError("the split must be laid out like the fp32 means")


def num_windows(L: int, B: int, stride: int | None = None) -> int:
    """misa_num_windows: windows of B keys every `stride` keys (None: B) over L keys."""
    S = B if stride is None else stride
    M = int(lib().misa_num_windows(L, B, S))
    if M < 1:
        raise ValueError(f"bad window geometry L={L} B={B} S={S}")
    return M


def _pool(pool: str) -> int:
    if pool not in POOL:
        raise ValueError(f"pool must be one of {tuple(POOL)}")
    return POOL[pool]


def block_stats(keys: torch.Tensor, B: int, out: torch.Tensor | None = None, stream=None, split: bool = False,
                out_hi: torch.Tensor | None = None, out_lo: torch.Tensor | None = None,
                stride: int | None = None, pool: str = "mean"):
    """misa_block_stats_ex: keys [nseq, L, 128] bf16 -> block statistics
    [nseq, M, 128] fp32 over windows of B keys every `stride` keys (None: B,
    plain blocks), mean or max pooled; or (stats, hi, lo) with the bf16 split
    when split=True."""
    _req(keys, torch.bfloat16, "keys", contiguous=False)
    _shape(keys, "keys", None, None, HEAD_DIM)
    if keys.stride(2) != 1 or keys.stride(1) != HEAD_DIM:
        raise ValueError("keys rows must be contiguous 128-element rows")
    nseq, L, _ = keys.shape
    S = B if stride is None else stride
    M = num_windows(L, B, S)
    _shape(out, "out", nseq, M, HEAD_DIM)
    _shape(out_hi, "out_hi", nseq, M, HEAD_DIM)
    if out is None:
        out = torch.empty((nseq, M, HEAD_DIM), dtype=torch.float32, device=keys.device)
    if split and out_hi is None:
        out_hi = torch.empty((nseq, M, HEAD_DIM), dtype=torch.bfloat16, device=keys.device)
        out_lo = torch.empty_like(out_hi)
    _split_pair(out_hi, out_lo, out)
    _call("misa_block_stats_ex", _p(keys), nseq, L, _key_stride(keys) if nseq > 1 else 0, B, S, _pool(pool), _p(out),
          _p(out_hi), _p(out_lo), _stream(stream))
    return (out, out_hi, out_lo) if out_hi is not None else out


def append_keys(keys: torch.Tensor, lens: torch.Tensor, new_keys: torch.Tensor, B: int, means: torch.Tensor,
                workspace: torch.Tensor | None = None, stream=None, means_hi=None, means_lo=None,
                stride: int | None = None, pool: str = "mean") -> None:
    """misa_append_keys_ex: new_keys [nseq, n_new, 128] bf16 go to rows
    [lens[b], lens[b] + n_new) of keys [nseq, L_cap, 128]; the statistics
    [nseq, M_cap, 128] fp32 (and their bf16 split, if given) of the touched
    windows are recomputed.  lens is not advanced."""
    _req(keys, torch.bfloat16, "keys", contiguous=False)
    _req(new_keys, torch.bfloat16, "new_keys")
    _req(lens, torch.int32, "lens")
    _req(means, torch.float32, "means", contiguous=False)
    if keys.stride(2) != 1 or keys.stride(1) != HEAD_DIM:
        raise ValueError("keys rows must be contiguous 128-element rows")
    if means.stride(2) != 1 or means.stride(1) != HEAD_DIM:
        raise ValueError("means rows must be contiguous 128-element rows")
    _shape(keys, "keys", None, None, HEAD_DIM)
    nseq, L_cap, _ = keys.shape
    _shape(new_keys, "new_keys", nseq, None, HEAD_DIM)
    S = B if stride is None else stride
    _shape(means, "means", nseq, num_windows(L_cap, B, S), HEAD_DIM)
    n_new = new_keys.shape[1]
    if new_keys.shape[0] != nseq or lens.numel() != nseq or means.shape[0] != nseq:
        raise ValueError("keys, lens, new_keys and means must agree on nseq")
    _split_pair(means_hi, means_lo, means)
    ws = workspace if workspace is not None else alloc_workspace(256, keys.device)
    _call("misa_append_keys_ex", _p(keys), nseq, int(keys.stride(0)) if nseq > 1 else 0, L_cap, _p(lens),
          _p(new_keys), n_new, B, S, _pool(pool), _p(means), _p(means_hi), _p(means_lo), int(means.stride(0)),
          _p(ws), ws.numel(), _stream(stream))


def _means_layout(means, means_hi, means_lo):
    """(nseq, sequence stride) of the block means given as fp32 and/or split."""
    if means is not None:
        _req(means, torch.float32, "means")
    _split_pair(means_hi, means_lo, means)
    ref = means if means is not None else means_hi
    if ref is None:
        raise ValueError("the block means are needed, as fp32 or as the bf16 split")
    return ref.shape[0], int(ref.stride(0))


def route_heads(q, w, means, seq_of, prefix_len, L: int, B: int, q_block: int, h: int,
                heads=None, importance=None, workspace=None, want_importance: bool = True, stream=None,
                means_hi=None, means_lo=None, stride: int | None = None):
    """misa_route_heads_ex -> (heads [G, h] int32, importance [G, H] fp32 or None).
    means may be None when the bf16 split (means_hi, means_lo) is given;
    stride: the window stride of the statistics (None: B, plain blocks)."""
    _req(q, torch.bfloat16, "q"); _req(w, torch.float32, "w")
    nseq, mstride = _means_layout(means, means_hi, means_lo)
    _req(seq_of, torch.int32, "seq_of"); _req(prefix_len, torch.int32, "prefix_len")
    _shape(q, "q", None, None, HEAD_DIM)
    T, H, _ = q.shape
    G = (T + q_block - 1) // q_block
    _shape(w, "w", T, H); _shape(seq_of, "seq_of", T); _shape(prefix_len, "prefix_len", T)
    S = B if stride is None else stride
    M = num_windows(L, B, S)
    for name_, m_ in (("means", means), ("means_hi", means_hi)):
        _shape(m_, name_, nseq, None, HEAD_DIM)
        if m_ is not None and m_.shape[1] < M:
            raise ValueError(f"{name_}: fewer than {M} blocks")
    _shape(heads, "heads", G, h); _shape(importance, "importance", G, H)
    dev = q.device
    if heads is None:
        heads = torch.empty((G, h), dtype=torch.int32, device=dev)
    if importance is None and want_importance:
        importance = torch.empty((G, H), dtype=torch.float32, device=dev)
    need = workspace_bytes(OP_ROUTE_HEADS, T, H, L, S)
    if workspace is None:
        workspace = alloc_workspace(need, dev)
    _call("misa_route_heads_ex", _p(q), _p(w), _p(means), _p(means_hi), _p(means_lo), nseq, mstride, _p(seq_of),
          _p(prefix_len), T, H, L, B, S, q_block, h, _p(heads), _p(importance), _p(workspace),
          workspace.numel(), _stream(stream))
    return heads, importance


def route_heads_noalloc(q, w, means, seq_of, prefix_len, L: int, B: int, q_block: int, h: int,
                        heads=None, importance=None, want_importance: bool = True, stream=None):
    """misa_route_heads_noalloc (no workspace; library-owned fixed scratch)."""
    _req(q, torch.bfloat16, "q"); _req(w, torch.float32, "w"); _req(means, torch.float32, "means")
    _req(seq_of, torch.int32, "seq_of"); _req(prefix_len, torch.int32, "prefix_len")
    _shape(q, "q", None, None, HEAD_DIM)
    T, H, _ = q.shape
    G = (T + q_block - 1) // q_block
    _shape(w, "w", T, H); _shape(seq_of, "seq_of", T); _shape(prefix_len, "prefix_len", T)
    _shape(means, "means", None, None, HEAD_DIM)
    if means.shape[1] < (L + B - 1) // B:
        raise ValueError("means: fewer blocks than ceil(L / B)")
    _shape(heads, "heads", G, h); _shape(importance, "importance", G, H)
    if heads is None:
        heads = torch.empty((G, h), dtype=torch.int32, device=q.device)
    if importance is None and want_importance:
        importance = torch.empty((G, H), dtype=torch.float32, device=q.device)
    _call("misa_route_heads_noalloc", _p(q), _p(w), _p(means), means.shape[0], int(means.stride(0)), _p(seq_of),
          _p(prefix_len), T, H, L, B, q_block, h, _p(heads), _p(importance), _stream(stream))
    return heads, importance


def index_score(q, w, keys, seq_of, prefix_len, heads=None, h: int | None = None, q_block: int = 1,
                cand=None, scores=None, workspace=None, stream=None) -> torch.Tensor:
    """misa_index_score -> scores [T, L] (or [T, n_cand]) fp32."""
    _req(q, torch.bfloat16, "q"); _req(w, torch.float32, "w"); _req(keys, torch.bfloat16, "keys")
    _req(seq_of, torch.int32, "seq_of"); _req(prefix_len, torch.int32, "prefix_len")
    _shape(q, "q", None, None, HEAD_DIM); _shape(keys, "keys", None, None, HEAD_DIM)
    T, H, _ = q.shape
    L = keys.shape[1]
    _shape(w, "w", T, H); _shape(seq_of, "seq_of", T); _shape(prefix_len, "prefix_len", T)
    if heads is not None:
        _req(heads, torch.int32, "heads")
        h = heads.shape[1] if h is None else h
        _shape(heads, "heads", (T + q_block - 1) // q_block, h)
    n_cand = 0
    if cand is not None:
        _req(cand, torch.int32, "cand")
        _shape(cand, "cand", T, None)
        n_cand = cand.shape[1]
    ncol = n_cand if cand is not None else L
    if scores is not None:
        _rows(scores, "scores", T, ncol)
    if scores is None:
        scores = torch.empty((T, ncol), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = alloc_workspace(256, q.device)
    _call("misa_index_score", _p(q), _p(w), _p(keys), keys.shape[0], _key_stride(keys), _p(seq_of),
          _p(prefix_len), T, H, L, _p(heads), int(h or H), q_block, _p(cand), n_cand, _p(scores),
          int(scores.stride(0)), _p(workspace), workspace.numel(), _stream(stream))
    return scores


def index_decode(q, w, keys, means_hi, means_lo, seq_of, prefix_len, B: int, h: int, k: int, heads=None,
                 importance=None, scores=None, idx=None, workspace=None, want_importance: bool = True,
                 select: bool = True, stream=None):
    """misa_index_decode: router + routed scoring in one kernel, the top-k
    behind it -> (heads [T, h], importance [T, H] or None, scores [T, >= L],
    idx [T, k], or None with select=False: no top-k)."""
    _req(q, torch.bfloat16, "q"); _req(w, torch.float32, "w"); _req(keys, torch.bfloat16, "keys")
    _req(seq_of, torch.int32, "seq_of"); _req(prefix_len, torch.int32, "prefix_len")
    _shape(q, "q", None, None, HEAD_DIM); _shape(keys, "keys", None, None, HEAD_DIM)
    T, H, _ = q.shape
    L = keys.shape[1]
    M = (L + B - 1) // B
    _shape(w, "w", T, H); _shape(seq_of, "seq_of", T); _shape(prefix_len, "prefix_len", T)
    _split_pair(means_hi, means_lo)
    if means_hi is None:
        raise ValueError("misa_index_decode reads the bf16 split of the block means")
    _shape(means_hi, "means_hi", None, None, HEAD_DIM)
    if means_hi.shape[1] < M or means_lo.shape != means_hi.shape:
        raise ValueError(f"means_hi / means_lo: expected [nseq, >= {M}, 128]")
    _shape(heads, "heads", T, h); _shape(importance, "importance", T, H); _shape(idx, "idx", T, k)
    dev = q.device
    if heads is None:
        heads = torch.empty((T, h), dtype=torch.int32, device=dev)
    if importance is None and want_importance:
        importance = torch.empty((T, H), dtype=torch.float32, device=dev)
    if scores is None:
        scores = torch.empty((T, (L + 3) // 4 * 4), dtype=torch.float32, device=dev)
    _rows(scores, "scores", T, L)
    if not select:
        idx = None
    elif idx is None:
        idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    need = workspace_bytes(OP_INDEX_DECODE, T, H, L, B, k)
    if workspace is None:
        workspace = alloc_workspace(need, dev)
    _call("misa_index_decode", _p(q), _p(w), _p(keys), keys.shape[0], _key_stride(keys), _p(means_hi),
          _p(means_lo), means_hi.shape[0], int(means_hi.stride(0)) if means_hi.shape[0] > 1 else 0, _p(seq_of),
          _p(prefix_len), T, H, L, B, h, k, _p(heads), _p(importance), _p(scores), int(scores.stride(0)), _p(idx),
          _p(workspace), workspace.numel(), _stream(stream))
    return heads, importance, scores, idx


def index_score_blocks(q, w, keys, seq_of, prefix_len, blocks, B: int, scores=None, workspace=None,
                       stream=None) -> torch.Tensor:
    """misa_index_score_blocks -> scores [T, m * B] fp32 (all heads over the
    tokens of the chosen blocks, -inf for empty slots and past the prefix)."""
    _req(q, torch.bfloat16, "q"); _req(w, torch.float32, "w"); _req(keys, torch.bfloat16, "keys")
    _req(seq_of, torch.int32, "seq_of"); _req(prefix_len, torch.int32, "prefix_len")
    _req(blocks, torch.int32, "blocks")
    _shape(q, "q", None, None, HEAD_DIM); _shape(keys, "keys", None, None, HEAD_DIM)
    T, H, _ = q.shape
    L = keys.shape[1]
    _shape(w, "w", T, H); _shape(seq_of, "seq_of", T); _shape(prefix_len, "prefix_len", T)
    _shape(blocks, "blocks", T, None)
    m = blocks.shape[1]
    if scores is not None:
        _rows(scores, "scores", T, m * B)
    else:
        scores = torch.empty((T, m * B), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = alloc_workspace(256, q.device)
    _call("misa_index_score_blocks", _p(q), _p(w), _p(keys), keys.shape[0], _key_stride(keys), _p(seq_of),
          _p(prefix_len), T, H, L, _p(blocks), m, B, _p(scores), int(scores.stride(0)), _p(workspace),
          workspace.numel(), _stream(stream))
    return scores


def topk(scores, k: int, n: int | None = None, row_valid=None, id_map=None, idx=None, workspace=None,
         stream=None) -> torch.Tensor:
    """misa_topk -> idx [T, k] int32 (ascending positions / ids, -1 padded)."""
    _req(scores, torch.float32, "scores", contiguous=False)
    T = scores.shape[0]
    n = scores.shape[1] if n is None else n
    _rows(scores, "scores", T, n)
    _shape(idx, "idx", T, k)
    if row_valid is not None:
        _req(row_valid, torch.int32, "row_valid"); _shape(row_valid, "row_valid", T)
    if idx is None:
        idx = torch.empty((T, k), dtype=torch.int32, device=scores.device)
    if workspace is None:
        workspace = alloc_workspace(256, scores.device)
    idm_stride = 0
    if id_map is not None:
        _req(id_map, torch.int32, "id_map", contiguous=False)
        if id_map.dim() != 2 or id_map.shape[1] < n or id_map.stride(1) != 1 or id_map.shape[0] not in (1, T):
            raise ValueError(f"id_map: expected [{T} or 1, >= {n}] with contiguous rows, got {tuple(id_map.shape)}")
        idm_stride = int(id_map.stride(0)) if id_map.shape[0] == T else 0
    _call("misa_topk", _p(scores), T, n, int(scores.stride(0)), _p(row_valid), _p(id_map), idm_stride, k, _p(idx),
          _p(workspace), workspace.numel(), _stream(stream))
    return idx


def hier_rerank(q, w, keys, seq_of, prefix_len, cand, k: int, idx=None, cand_scores=None, want_scores=False,
                workspace=None, stream=None):
    """misa_hier_rerank -> (idx [T, k], cand_scores [T, kp] or None)."""
    _req(q, torch.bfloat16, "q"); _req(w, torch.float32, "w"); _req(keys, torch.bfloat16, "keys")
    _shape(q, "q", None, None, HEAD_DIM); _shape(keys, "keys", None, None, HEAD_DIM)
    T, H, _ = q.shape
    L = keys.shape[1]
    _req(cand, torch.int32, "cand")
    _shape(w, "w", T, H); _shape(cand, "cand", T, None); _shape(seq_of, "seq_of", T)
    kp = cand.shape[1]
    _shape(idx, "idx", T, k); _shape(cand_scores, "cand_scores", T, kp)
    if idx is None:
        idx = torch.empty((T, k), dtype=torch.int32, device=q.device)
    if cand_scores is None and want_scores:
        cand_scores = torch.empty((T, kp), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = alloc_workspace(workspace_bytes(OP_HIER_RERANK, T, H, L, 1, k, kp), q.device)
    _call("misa_hier_rerank", _p(q), _p(w), _p(keys), keys.shape[0], _key_stride(keys), _p(seq_of),
          _p(prefix_len), T, H, L, _p(cand), kp, k, _p(cand_scores), _p(idx), _p(workspace), workspace.numel(),
          _stream(stream))
    return idx, cand_scores


def hisa_block_filter(q, w, means, seq_of, prefix_len, L: int, B: int, m: int, blocks=None, cand=None,
                      block_scores=None, want_scores=False, workspace=None, stream=None, means_hi=None,
                      means_lo=None, stride: int | None = None):
    """hisa_block_filter_ex -> (blocks [T, m], cand [T, m*B], block_scores [T, M] or None).
    means may be None when the bf16 split (means_hi, means_lo) is given;
    stride: the window stride of the statistics (None: B, plain blocks)."""
    nseq, mstride = _means_layout(means, means_hi, means_lo)
    _req(q, torch.bfloat16, "q"); _req(w, torch.float32, "w")
    _shape(q, "q", None, None, HEAD_DIM)
    T, H, _ = q.shape
    S = B if stride is None else stride
    M = num_windows(L, B, S)
    _shape(w, "w", T, H); _shape(seq_of, "seq_of", T); _shape(prefix_len, "prefix_len", T)
    for name_, m_ in (("means", means), ("means_hi", means_hi)):
        _shape(m_, name_, nseq, None, HEAD_DIM)
        if m_ is not None and m_.shape[1] < M:
            raise ValueError(f"{name_}: fewer than {M} blocks")
    _shape(blocks, "blocks", T, m); _shape(cand, "cand", T, m * B); _shape(block_scores, "block_scores", T, M)
    dev = q.device
    if blocks is None:
        blocks = torch.empty((T, m), dtype=torch.int32, device=dev)
    if cand is None:
        cand = torch.empty((T, m * B), dtype=torch.int32, device=dev)
    if block_scores is None and want_scores:
        block_scores = torch.empty((T, M), dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = alloc_workspace(workspace_bytes(OP_HISA_BLOCK_FILTER, T, H, L, S, m), dev)
    _call("hisa_block_filter_ex", _p(q), _p(w), _p(means), _p(means_hi), _p(means_lo), nseq, mstride, _p(seq_of),
          _p(prefix_len), T, H, L, B, S, m, _p(blocks), _p(cand), _p(block_scores), _p(workspace),
          workspace.numel(), _stream(stream))
    return blocks, cand, block_scores


def sparse_mla(q, kv, seq_of, idx, scale: float, out=None, lse=None, want_lse: bool = False, workspace=None,
               stream=None):
    """misa_sparse_mla -> (out [T, Hq, 512] bf16, lse [T, Hq] fp32 or None).

    q [T, Hq, 576] bf16; kv [nseq, L, 576] bf16 latent rows (keys = whole row,
    values = the first 512 entries); idx [T, k] int32 token ids, -1 = empty."""
    _req(q, torch.bfloat16, "q"); _req(kv, torch.bfloat16, "kv", contiguous=False)
    _req(seq_of, torch.int32, "seq_of"); _req(idx, torch.int32, "idx", contiguous=False)
    if kv.stride(2) != 1 or kv.stride(1) != MLA_DQK:
        raise ValueError("kv rows must be contiguous 576-element rows")
    if idx.stride(1) != 1:
        raise ValueError("idx rows must be contiguous")
    _shape(q, "q", None, None, MLA_DQK); _shape(kv, "kv", None, None, MLA_DQK)
    T, Hq, _ = q.shape
    nseq, L, _ = kv.shape
    _shape(idx, "idx", T, None); _shape(seq_of, "seq_of", T)
    k = idx.shape[1]
    _shape(out, "out", T, Hq, MLA_DV); _shape(lse, "lse", T, Hq)
    if out is None:
        out = torch.empty((T, Hq, MLA_DV), dtype=torch.bfloat16, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((T, Hq), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = alloc_workspace(workspace_bytes(OP_SPARSE_MLA, T, Hq, 0, 0, k), q.device)
    _call("misa_sparse_mla", _p(q), _p(kv), nseq, int(kv.stride(0)) if nseq > 1 else 0, L, _p(seq_of), T, Hq,
          _p(idx), k, int(idx.stride(0)), float(scale), _p(out), _p(lse), _p(workspace), workspace.numel(),
          _stream(stream))
    return out, lse


def shard_prefix(prefix_len, s0: int, L_shard: int, out=None, stream=None) -> torch.Tensor:
    """misa_shard_prefix -> [T] int32 prefix lengths local to keys [s0, s0 + L_shard)."""
    _req(prefix_len, torch.int32, "prefix_len")
    T = prefix_len.numel()
    if out is None:
        out = torch.empty_like(prefix_len)
    _call("misa_shard_prefix", _p(prefix_len), T, int(s0), int(L_shard), _p(out), _stream(stream))
    return out


def gather_candidates(scores, idx, n: int, id_offset: int, out_scores=None, out_ids=None, stream=None):
    """misa_gather_candidates -> (scores [T, k] fp32, global ids [T, k] int32) of local picks."""
    _req(scores, torch.float32, "scores", contiguous=False)
    _req(idx, torch.int32, "idx")
    T, k = idx.shape
    _rows(scores, "scores", T, n)
    _shape(out_scores, "out_scores", T, k); _shape(out_ids, "out_ids", T, k)
    if out_scores is None:
        out_scores = torch.empty((T, k), dtype=torch.float32, device=idx.device)
    if out_ids is None:
        out_ids = torch.empty((T, k), dtype=torch.int32, device=idx.device)
    _call("misa_gather_candidates", _p(scores), T, int(n), int(scores.stride(0)), _p(idx), k, int(id_offset),
          _p(out_scores), _p(out_ids), _stream(stream))
    return out_scores, out_ids


def selftest_wait_timeout(workspace: torch.Tensor, stream=None) -> None:
    """misa_selftest_wait_timeout: a bounded wait on a barrier nothing completes
    (about two seconds); read the outcome with error_query."""
    _call("misa_selftest_wait_timeout", _p(workspace), workspace.numel(), _stream(stream))

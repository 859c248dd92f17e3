"""The Python binding rejects tensors whose sizes disagree with the call before
anything reaches the library (the C ABI sees only pointers, so a tensor smaller
than the call implies would be read or written past its end).  CPU tensors are
enough: the shape check comes before the device-pointer check."""
import pytest
import torch

from sparse_attention_token_misa_b200 import _native as nat

bf, f32, i32 = torch.bfloat16, torch.float32, torch.int32


def z(*shape, dtype=f32):
    return torch.zeros(shape, dtype=dtype)


def _raises_shape(fn):
    with pytest.raises(ValueError, match="expected"):
        fn()


def test_block_stats_and_append_shapes():
    _raises_shape(lambda: nat.block_stats(z(2, 100, 64, dtype=bf), 16))               # rows of 64, not 128
    _raises_shape(lambda: nat.block_stats(z(2, 100, 128, dtype=bf), 16, out=z(2, 6, 128)))   # 7 blocks needed
    keys = z(2, 256, 128, dtype=bf)
    _raises_shape(lambda: nat.append_keys(keys, z(2, dtype=i32), z(2, 4, 64, dtype=bf), 128, z(2, 2, 128)))
    _raises_shape(lambda: nat.append_keys(keys, z(2, dtype=i32), z(2, 4, 128, dtype=bf), 128, z(2, 1, 128)))


def test_router_and_filter_shapes():
    q, w = z(4, 64, 128, dtype=bf), z(4, 64)
    so, pl = z(4, dtype=i32), z(4, dtype=i32)
    _raises_shape(lambda: nat.route_heads(q, z(4, 32), z(1, 8, 128), so, pl, 1024, 128, 1, 8))     # w
    _raises_shape(lambda: nat.route_heads(q, w, z(1, 8, 128), z(3, dtype=i32), pl, 1024, 128, 1, 8))
    _raises_shape(lambda: nat.route_heads(q, w, z(1, 8, 128), so, pl, 1024, 128, 1, 8,
                                          heads=z(4, 4, dtype=i32)))                                  # h = 8
    _raises_shape(lambda: nat.route_heads_noalloc(q, w, z(1, 8, 64), so, pl, 1024, 128, 1, 8))
    _raises_shape(lambda: nat.hisa_block_filter(q, w, z(1, 8, 128), so, pl, 1024, 128, 4, blocks=z(4, 3, dtype=i32)))
    with pytest.raises(ValueError, match="fewer than"):
        nat.route_heads(q, w, z(1, 7, 128), so, pl, 1024, 128, 1, 8)                                 # 8 blocks needed


def test_scoring_topk_attention_shapes():
    q, w, keys = z(4, 64, 128, dtype=bf), z(4, 64), z(1, 500, 128, dtype=bf)
    so, pl = z(4, dtype=i32), z(4, dtype=i32)
    _raises_shape(lambda: nat.index_score(q, w, keys, so, pl, scores=z(4, 499)))
    _raises_shape(lambda: nat.index_score(q, w, keys, so, pl, heads=z(4, 8, dtype=i32), h=8, q_block=2))
    _raises_shape(lambda: nat.topk(z(3, 100), 10, idx=z(3, 9, dtype=i32)))
    _raises_shape(lambda: nat.topk(z(3, 100), 10, n=101))
    _raises_shape(lambda: nat.topk(z(3, 100), 10, id_map=z(3, 99, dtype=i32)))
    _raises_shape(lambda: nat.hier_rerank(q, w, keys, so, pl, z(4, 50, dtype=i32), 10, idx=z(4, 11, dtype=i32)))
    _raises_shape(lambda: nat.sparse_mla(z(2, 128, 512, dtype=bf), z(1, 100, 576, dtype=bf), z(2, dtype=i32),
                                         z(2, 16, dtype=i32), 0.1))
    _raises_shape(lambda: nat.sparse_mla(z(2, 128, 576, dtype=bf), z(1, 100, 576, dtype=bf), z(2, dtype=i32),
                                         z(2, 16, dtype=i32), 0.1, out=z(2, 128, 576, dtype=bf)))
    _raises_shape(lambda: nat.gather_candidates(z(2, 50), z(2, 8, dtype=i32), 60, 0))


def test_well_formed_cpu_tensors_reach_the_device_check():
    # correct shapes get past the shape checks and stop at the device-tensor check
    with pytest.raises(ValueError, match="device tensors"):
        nat.topk(z(3, 100), 10)

"""PackedKVCache checks every tensor against the layout its call reads before a
pointer reaches the library.  On the CPU (no library state) a call whose
tensors pass reaches the C entry point, which answers BGTQ_ERR_NULL for the
missing state; a call whose tensors do not match is refused in Python with
BGTQ_ERR_INVALID_ARG.  The accepted shapes are the ones the GPU tests and the
benchmark use."""
import numpy as np
import pytest
import torch

from packed_decode_attention_b200 import bgtq
from packed_decode_attention_b200 import build as pkg_build

ERR_INVALID_ARG, ERR_NULL = -1, -2


@pytest.fixture()
def kv(monkeypatch):
    pkg_build.build()
    bgtq.lib()
    monkeypatch.setattr(bgtq, "_stream", lambda s: 0)
    obj = object.__new__(bgtq.PackedKVCache)
    obj.cfg = bgtq.Config(n_layers=3, n_kv_heads=2, n_q_heads=8, max_batch=4, capacity_tokens=300)
    obj.device = torch.device("cpu")
    obj.state = None
    return obj


def status(fn, *args, **kw):
    with pytest.raises(bgtq.BgtqError) as e:
        fn(*args, **kw)
    return e.value.status


def h(*shape):
    return torch.zeros(shape, dtype=torch.float16)


def i32(n, v=0):
    return torch.full((n,), v, dtype=torch.int32)


def test_matching_tensors_reach_the_library(kv):
    L, B = 2, 3
    q, out = h(L, B, 8, 128), h(L, B, 8, 128)
    k = h(L, B, 5, 2, 128)
    s = i32(B)
    bk = h(L, B, 7, 2, 128)
    assert status(kv.allocate, h(3, 16, 8, 128), h(3, 20, 2, 128)) == ERR_NULL
    assert status(kv.set_allocation, np.full((3, 2, 64), 3, dtype=np.int8)) == ERR_NULL
    assert status(kv.encode_append, 0, k, k.clone(), s, s, layer_count=L) == ERR_NULL
    kd = h(L, 40, 2, 128)
    assert status(kv.encode_append, 0, kd[:, None], kd[:, None], i32(1), i32(1), layer_count=L) == ERR_NULL
    assert status(kv.encode_append, 0, k, k, s, s, layer_count=L, rope_base=1e6) == ERR_NULL
    assert status(kv.rotate_query, 0, q, torch.zeros(q.shape), layer_count=L) == ERR_NULL
    assert status(kv.decode_attn, 0, q, s, out, layer_count=L) == ERR_NULL
    assert status(kv.decode_attn, 1, q[1:2], s, out[1:2]) == ERR_NULL
    assert status(kv.decode_attn_static_scratch, 0, q, s, out, layer_count=L) == ERR_NULL
    assert status(kv.decode_step, 0, k, k, s, s, q, s, out, layer_count=L) == ERR_NULL
    assert status(kv.decode_step, 0, None, None, None, None, q, s, out, layer_count=L) == ERR_NULL
    assert status(kv.decode_attn_buffered, 0, q, s, s, bk, bk, s, out, layer_count=L) == ERR_NULL
    assert status(kv.decode_step_buffered, 0, k, k, s, s, q, s, s, bk, bk, s, out, layer_count=L) == ERR_NULL
    assert status(kv.decode_step_buffered, 0, None, None, None, None, q, s, s, bk, bk, s, out,
                  layer_count=L) == ERR_NULL
    assert status(kv.logit_mae, 0, 1, 10, h(L, 50, 8, 128), h(L, 50, 2, 128),
                  torch.zeros((L, 8), dtype=torch.float64), layer_count=L) == ERR_NULL
    assert status(kv.decode_split, 0, torch.zeros((L, B, 8, 128)), s, layer_count=L) == ERR_NULL
    assert status(kv.decode_combine, 0, s, out, layer_count=L) == ERR_NULL
    # a contiguous cache leaves the table to the library, which refuses it
    assert status(kv.set_block_table, torch.zeros((1, 4), dtype=torch.int32)) == ERR_NULL


def test_mismatched_tensors_are_refused_before_the_library(kv):
    L, B = 2, 3
    q, out = h(L, B, 8, 128), h(L, B, 8, 128)
    k = h(L, B, 5, 2, 128)
    s = i32(B)
    bk = h(L, B, 7, 2, 128)
    bad = [
        (kv.allocate, (h(2, 16, 8, 128), h(3, 20, 2, 128)), {}),                # layers
        (kv.allocate, (h(3, 16, 8, 128), h(3, 20, 8, 128)), {}),                # KV heads
        (kv.set_allocation, (np.full((3, 2, 32), 3, dtype=np.int8),), {}),       # too few widths
        (kv.encode_append, (0, k, k, s, s), {}),                                 # layer_count 1 vs 2
        (kv.encode_append, (0, k, h(L, B, 4, 2, 128), s, s), {"layer_count": L}),  # v != k
        (kv.encode_append, (0, k, k, i32(B + 1), s), {"layer_count": L}),       # start length
        (kv.encode_append, (0, k.float(), k.float(), s, s), {"layer_count": L}),  # dtype
        (kv.rotate_query, (0, q, h(L, B, 8, 128)), {"layer_count": L}),          # out must be fp32
        (kv.decode_attn, (0, q, s, h(L, B, 8, 64)), {"layer_count": L}),         # out shape
        (kv.decode_attn, (0, q, i32(B - 1), out), {"layer_count": L}),           # seq_lens length
        (kv.decode_attn, (0, q, s.long(), out), {"layer_count": L}),             # seq_lens dtype
        (kv.decode_attn, (0, h(L, B, 4, 128), s, h(L, B, 4, 128)), {"layer_count": L}),  # query heads
        (kv.decode_attn, (0, q.transpose(2, 3).contiguous().transpose(2, 3), s, out), {"layer_count": L}),
        (kv.decode_attn, (0, q.numpy(), s, out), {"layer_count": L}),            # not a tensor
        (kv.decode_attn_static_scratch, (0, q, s, h(L, B, 8, 64)), {"layer_count": L}),  # out shape
        (kv.decode_attn_static_scratch, (0, q, i32(B + 1), out), {"layer_count": L}),    # seq_lens length
        (kv.decode_attn_static_scratch, (0, q, s, out), {}),                              # layer_count 1 vs 2
        (kv.decode_step, (0, h(L, B + 1, 1, 2, 128), h(L, B + 1, 1, 2, 128), i32(B + 1), i32(B + 1), q, s, out),
         {"layer_count": L}),                                                    # rows of another batch
        (kv.decode_attn_buffered, (0, q, s, s, bk, h(L, B, 6, 2, 128), s, out), {"layer_count": L}),
        (kv.decode_attn_buffered, (0, q, s, i32(B - 1), bk, bk, s, out), {"layer_count": L}),
        (kv.logit_mae, (0, 0, 0, h(L, 50, 8, 128), h(L, 49, 2, 128), torch.zeros((L, 8), dtype=torch.float64)),
         {"layer_count": L}),                                                    # k rows != q rows
        (kv.logit_mae, (0, 0, 0, h(L, 50, 8, 128), h(L, 50, 2, 128), torch.zeros((L, 8))),
         {"layer_count": L}),                                                    # out must be float64
        (kv.decode_split, (0, q, s), {"layer_count": L}),                        # q~ must be fp32
        (kv.decode_combine, (0, s, out.float()), {"layer_count": L}),
    ]
    for fn, args, kw in bad:
        assert status(fn, *args, **kw) == ERR_INVALID_ARG, (fn.__name__, kw)


def test_paged_table_shape_is_checked(kv):
    kv.cfg = bgtq.Config(n_layers=3, n_kv_heads=2, n_q_heads=8, max_batch=4, capacity_tokens=300,
                         page_pool_tiles=20)
    assert status(kv.set_block_table, torch.zeros((4, 5), dtype=torch.int32)) == ERR_NULL
    assert status(kv.set_block_table, torch.zeros((4, 4), dtype=torch.int32)) == ERR_INVALID_ARG
    assert status(kv.set_block_table, torch.zeros((4, 5), dtype=torch.int64)) == ERR_INVALID_ARG
    assert status(kv.set_block_table, None) == ERR_NULL

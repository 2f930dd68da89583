"""Argument checks of the PyTorch wrapper (CPU only: they run before any library call).

The C ABI receives plain pointers and strides and cannot see a tensor's extent,
so ``SegPagedLayer`` refuses tensors that would make a kernel read or write
outside them.  These tests build the wrapper's state by hand (no plan, no GPU)
and check that valid shapes pass and each kind of mistake is refused.
"""
from __future__ import annotations

from types import SimpleNamespace

import pytest
import torch

from head_aware_paged_build_b200.runtime import SegPagedLayer, build_layers


def fake_layer(batch=2, hq=4, hkv=2, d=128, ctx=(100, 70), dtype=torch.bfloat16, num_queries=None,
               kv_dtype=None):
    lay = object.__new__(SegPagedLayer)
    lay.torch_dtype = dtype
    lay.kv_dtype = kv_dtype or "bf16"
    lay.batch, lay.num_q_heads, lay.num_kv_heads, lay.head_dim = batch, hq, hkv, d
    lay.ctx_len = list(ctx)
    lay.sizes = SimpleNamespace(num_queries=batch if num_queries is None else num_queries)
    lay.k_pool = torch.empty(16, dtype=torch.uint8)
    lay.v_pool = torch.empty(16, dtype=torch.uint8)
    lay.plan = None
    return lay


def dense(*shape, dtype=torch.bfloat16):
    return torch.zeros(*shape, dtype=dtype)


def test_dense_shapes_that_cover_the_plan_pass():
    lay = fake_layer()
    lay._check_dense(dense(2, 2, 100, 128), dense(2, 2, 100, 128), False, "build")
    lay._check_dense(dense(3, 4, 128, 128), dense(3, 4, 128, 128), False, "build")  # larger is fine
    k = dense(2, 2, 200, 128)[:, :, :100]  # a strided view
    lay._check_dense(k, dense(2, 2, 200, 128)[:, :, :100], False, "build")
    lay._check_dense(dense(170, 2, 128), dense(170, 2, 128), True, "build")  # varlen [sum L, Hkv, d]


@pytest.mark.parametrize("k_shape,varlen", [
    ((2, 2, 99, 128), False),   # shorter than the longest context
    ((1, 2, 100, 128), False),  # fewer sequences
    ((2, 1, 100, 128), False),  # fewer kv-heads
    ((2, 2, 100, 64), False),   # wrong head_dim
    ((2, 2, 100), False),       # wrong rank
    ((169, 2, 128), True),      # varlen rows short of sum L
    ((2, 2, 100, 128), True),   # padded layout passed as varlen
])
def test_dense_shapes_that_do_not_cover_the_plan_are_refused(k_shape, varlen):
    lay = fake_layer()
    with pytest.raises(ValueError):
        lay._check_dense(dense(*k_shape), dense(*k_shape), varlen, "build")


def test_dense_dtype_layout_and_device_are_checked():
    lay = fake_layer()
    ok = dense(2, 2, 100, 128)
    with pytest.raises(TypeError):
        lay._check_dense(dense(2, 2, 100, 128, dtype=torch.float32), ok, False, "build")
    with pytest.raises(ValueError):  # K and V differ
        lay._check_dense(ok, dense(2, 2, 101, 128), False, "build")
    with pytest.raises(ValueError):  # head_dim not contiguous
        t = dense(2, 2, 128, 100).transpose(2, 3)
        lay._check_dense(t, t, False, "build")
    with pytest.raises(ValueError):  # not where the layer's buffers are
        m = torch.empty(2, 2, 100, 128, dtype=torch.bfloat16, device="meta")
        lay._check_dense(m, m, False, "build")


def test_gather_of_e4m3_pages_takes_byte_codes():
    """E4M3 pages gather their 1-byte codes: uint8 targets pass the checks, bf16 ones are refused."""
    lay = fake_layer(kv_dtype="e4m3")
    codes = torch.zeros(2, 2, 100, 128, dtype=torch.uint8)
    lay._check_dense(codes, codes, False, "gather", torch.uint8)
    with pytest.raises(TypeError):
        lay.gather(dense(2, 2, 100, 128), dense(2, 2, 100, 128))
    with pytest.raises(ValueError):  # shape still checked
        short = torch.zeros(2, 2, 99, 128, dtype=torch.uint8)
        lay.gather(short, short)
    with pytest.raises(TypeError):  # build still takes the bf16 dense K/V
        lay.build(codes, codes)


def test_attention_refuses_wrong_q_out_lse_before_any_call():
    lay = fake_layer()
    q = dense(2, 4, 128)
    with pytest.raises(ValueError):
        lay.attention(dense(3, 4, 128))  # rows != the plan's queries
    with pytest.raises(ValueError):
        lay.attention(dense(2, 4, 256)[:, :, :128])  # not contiguous
    with pytest.raises(TypeError):
        lay.attention(dense(2, 4, 128, dtype=torch.float32))
    with pytest.raises(ValueError):
        lay.attention(q, dense(2, 4, 64))
    with pytest.raises(TypeError):
        lay.attention(q, dense(2, 4, 128), dense(2, 4))  # lse must be fp32
    with pytest.raises(ValueError):
        lay.attention(q, dense(2, 4, 128), torch.zeros(2, 5))


def test_append_refuses_rows_that_do_not_match_the_heads():
    lay = fake_layer()
    with pytest.raises(ValueError):
        lay.append(dense(2, 1, 128), dense(2, 1, 128))
    with pytest.raises(ValueError):
        lay.append(dense(2, 2, 128), dense(2, 2, 64))
    with pytest.raises(TypeError):
        lay.append(dense(2, 2, 128, dtype=torch.float16), dense(2, 2, 128, dtype=torch.float16))


def test_build_layers_needs_one_dense_pair_per_layer_and_shared_pools():
    a, b = fake_layer(), fake_layer()
    k = dense(2, 2, 100, 128)
    with pytest.raises(ValueError):
        build_layers([a, b], [k], [k])
    with pytest.raises(ValueError):
        build_layers([], [], [])
    with pytest.raises(ValueError):  # b has its own pools
        build_layers([a, b], [k, k], [k, k])

"""The Python binding allocates exactly the arrays the library's descriptor describes.

A QuantizedKVCache is built in host memory here (descriptor validation and the footprint
are host arithmetic; no kernel runs), and the bytes of the tensors it allocated are checked
against kvq_cache_bytes for every scheme pair, layout, INT4 group size and rotation."""
import pytest
import torch

from decode_attention_quantize_b200 import kvq

PAIRS = [(kvq.FP8_E4M3_PER_TENSOR, kvq.FP8_E4M3_PER_TENSOR), (kvq.FP8_E5M2_PER_TENSOR, kvq.FP8_E5M2_PER_TENSOR),
         (kvq.INT8_SYM_PER_TENSOR, kvq.UINT8_ASYM_PER_CHANNEL), (kvq.INT8_SYM_PER_TOKEN, kvq.INT8_SYM_PER_TOKEN),
         (kvq.INT8_SYM_PER_CHANNEL, kvq.INT8_SYM_PER_CHANNEL), (kvq.INT4_SYM_PER_GROUP, kvq.INT4_SYM_PER_GROUP),
         (kvq.KIVI_INT4, kvq.KIVI_INT4), (kvq.KIVI_INT2, kvq.KIVI_INT2),
         (kvq.KIVI_INT4_F16, kvq.KIVI_INT4_F16), (kvq.KIVI_INT2_F16, kvq.KIVI_INT2_F16)]


def _bytes(t):
    return t.numel() * t.element_size()


def _check(cache):
    f = cache.footprint()
    t = cache.t
    codes = _bytes(t["k_codes"]) + _bytes(t["v_codes"])
    meta = sum(_bytes(t[n]) for n in ("k_scale", "v_scale", "k_zero", "v_zero", "k_zp", "v_zp") if n in t)
    # a per-tensor scale is allocated as four floats (16-byte alignment); the footprint counts one
    pad = sum(12 for side in ("k", "v")
              if getattr(cache.spec, side + "_scheme") in (kvq.FP8_E4M3_PER_TENSOR, kvq.FP8_E5M2_PER_TENSOR,
                                                           kvq.INT8_SYM_PER_TENSOR))
    res = sum(_bytes(t[n]) for n in ("k_res", "v_res") if n in t)
    assert f.code_bytes == codes
    assert f.meta_bytes == meta - pad
    assert f.residual_bytes == res
    assert f.total_bytes == f.code_bytes + f.meta_bytes + f.residual_bytes


@pytest.mark.parametrize("ks,vs", PAIRS)
def test_dense_allocation_matches_footprint(ks, vs):
    cache = kvq.QuantizedKVCache(kvq.CacheSpec(2, 8, 2, ks, vs, capacity=256), device="cpu")
    _check(cache)
    assert cache.desc.capacity == 256 and cache.desc.rotation == kvq.KVQ_ROTATE_NONE


@pytest.mark.parametrize("ks,vs", [p for p in PAIRS if p[0] not in kvq.KIVI_SCHEMES])
def test_paged_allocation_matches_footprint(ks, vs):
    cache = kvq.QuantizedKVCache(kvq.CacheSpec(3, 8, 2, ks, vs, paged=True, page_size=32, max_pages=4,
                                               num_pages=10), device="cpu")
    _check(cache)
    assert tuple(cache["page_table"].shape) == (3, 4)


@pytest.mark.parametrize("group", [32, 64, 128])
def test_int4_group_scales_and_rotation_flag(group):
    cache = kvq.QuantizedKVCache(kvq.CacheSpec(2, 4, 2, kvq.INT4_SYM_PER_GROUP, kvq.INT4_SYM_PER_GROUP,
                                               capacity=128, group=group, rotate=True), device="cpu")
    _check(cache)
    assert tuple(cache["k_scale"].shape) == (2, 2, 128, 128 // group)
    assert cache.desc.group_size == group and cache.desc.rotation == kvq.KVQ_ROTATE_HADAMARD


def test_rejected_specs_raise():
    with pytest.raises(RuntimeError):   # INT4 groups: 32, 64 or 128
        kvq.QuantizedKVCache(kvq.CacheSpec(1, 1, 1, kvq.INT4_SYM_PER_GROUP, kvq.INT4_SYM_PER_GROUP, capacity=128,
                                           group=16), device="cpu")
    with pytest.raises(RuntimeError):   # no rotation with KIVI
        kvq.QuantizedKVCache(kvq.CacheSpec(1, 1, 1, kvq.KIVI_INT4, kvq.KIVI_INT4, capacity=128, rotate=True),
                             device="cpu")

"""The C-ABI library loads, exports every symbol its header declares, and rejects bad
arguments on the host before touching a device (no compute calls here)."""
import ctypes
import re
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "kvq.h")).read()
    return sorted(set(re.findall(r"KVQ_API\s+[\w\s\*]*?\b(kvq_\w+)\s*\(", src)))


def test_header_declares_the_documented_entry_points():
    names = _declared()
    for must in ("kvq_quantize_append", "kvq_dequantize", "kvq_decode_attention"):
        assert must in names


def test_library_exports_every_declared_symbol():
    from decode_attention_quantize_b200 import kvq
    lib = ctypes.CDLL(kvq.LIB_PATH)
    for name in _declared():
        assert hasattr(lib, name), name
    assert sorted(kvq.EXPORTS) == _declared()
    assert lib.kvq_abi_version() == 3


def _desc(**kw):
    from decode_attention_quantize_b200.kvq import KvqDesc
    d = KvqDesc()
    d.batch, d.num_q_heads, d.num_kv_heads, d.head_dim = 2, 8, 2, 128
    d.k_scheme = d.v_scheme = 0
    d.layout, d.capacity = 0, 256
    d.group_size, d.residual_cap = 32, 128
    fake = 0x10000  # never dereferenced: validation is host-only
    for f in ("k_codes", "v_codes", "k_scale", "v_scale", "dev_status"):
        setattr(d, f, fake)
    for k, v in kw.items():
        setattr(d, k, v)
    return d


def test_validation_is_host_side():
    from decode_attention_quantize_b200 import kvq
    L = kvq.lib
    ok = _desc()
    assert L.kvq_validate(ctypes.byref(ok)) == kvq.KVQ_OK
    cases = [
        (dict(head_dim=64), kvq.KVQ_ERR_UNSUPPORTED),
        (dict(num_q_heads=7), kvq.KVQ_ERR_INVALID_ARG),
        (dict(capacity=200), kvq.KVQ_ERR_INVALID_ARG),
        (dict(k_scheme=11), kvq.KVQ_ERR_INVALID_ARG),
        (dict(k_scheme=5, v_scheme=6), kvq.KVQ_ERR_UNSUPPORTED),
        (dict(rotation=2), kvq.KVQ_ERR_INVALID_ARG),
        (dict(rotation=1, k_scheme=5, v_scheme=5), kvq.KVQ_ERR_UNSUPPORTED),   # no rotation with KIVI
        (dict(k_scheme=8, v_scheme=8, group_size=16), kvq.KVQ_ERR_UNSUPPORTED),   # INT4 groups: 32, 64, 128
        (dict(k_codes=None), kvq.KVQ_ERR_INVALID_ARG),
        (dict(k_codes=0x10004), kvq.KVQ_ERR_INVALID_ARG),   # not 16-byte aligned
        (dict(layout=1, page_size=16, max_pages_per_seq=4, num_pages=8), kvq.KVQ_ERR_INVALID_ARG),
        (dict(layout=1, page_size=24, max_pages_per_seq=4, num_pages=8, page_table=0x10000, seq_lens=0x10000),
         kvq.KVQ_ERR_UNSUPPORTED),
        (dict(v_scheme=4), kvq.KVQ_ERR_INVALID_ARG),          # asym needs a zero-point array
        (dict(k_scheme=5, v_scheme=5), kvq.KVQ_ERR_INVALID_ARG),  # KIVI needs minima and residual
    ]
    for kw, want in cases:
        d = _desc(**kw)
        assert L.kvq_validate(ctypes.byref(d)) == want, kw


def test_append_and_decode_reject_before_launch():
    from decode_attention_quantize_b200 import kvq
    L = kvq.lib
    d = _desc(num_quantized=250)
    buf = 0x20000
    # capacity: 250 + 8 > 256
    st = L.kvq_quantize_append(ctypes.byref(d), buf, buf, kvq.KVQ_BF16, 8, None, 0, None, 0, None)
    assert st == kvq.KVQ_ERR_CAPACITY and d.num_quantized == 250
    # calibration without workspace
    d2 = _desc()
    st = L.kvq_quantize_append(ctypes.byref(d2), buf, buf, kvq.KVQ_BF16, 8, None, kvq.KVQ_APPEND_CALIBRATE,
                               None, 0, None)
    assert st == kvq.KVQ_ERR_WORKSPACE and d2.num_quantized == 0
    # KIVI takes bf16 only
    d3 = _desc(k_scheme=5, v_scheme=5, k_zero=buf, v_zero=buf, k_res=buf, v_res=buf)
    st = L.kvq_quantize_append(ctypes.byref(d3), buf, buf, kvq.KVQ_F32, 8, None, 0, None, 0, None)
    assert st == kvq.KVQ_ERR_UNSUPPORTED
    # per-sequence counts are for the paged layout only
    st = L.kvq_quantize_append(ctypes.byref(d2), buf, buf, kvq.KVQ_BF16, 8, buf, 0, None, 0, None)
    assert st == kvq.KVQ_ERR_INVALID_ARG
    # decode: workspace too small, bad dtype, bad scale
    need = L.kvq_decode_workspace_bytes(ctypes.byref(d2))
    assert need > 0
    assert L.kvq_decode_attention(ctypes.byref(d2), buf, 1, ctypes.c_float(0.088), buf, None, buf, need - 1,
                                  None) == kvq.KVQ_ERR_WORKSPACE
    assert L.kvq_decode_attention(ctypes.byref(d2), buf, 7, ctypes.c_float(0.088), buf, None, buf, need,
                                  None) == kvq.KVQ_ERR_INVALID_ARG
    assert L.kvq_decode_attention(ctypes.byref(d2), buf, 1, ctypes.c_float(-1.0), buf, None, buf, need,
                                  None) == kvq.KVQ_ERR_INVALID_ARG
    # the output is written with 16-byte stores: a misaligned pointer is refused on the host
    assert L.kvq_decode_attention(ctypes.byref(d2), buf, 1, ctypes.c_float(0.088), buf + 4, None, buf, need,
                                  None) == kvq.KVQ_ERR_INVALID_ARG
    # the bounded-wait self-check refuses a null status pointer before launching
    assert L.kvq_check_bounded_wait(None, None) == kvq.KVQ_ERR_INVALID_ARG
    # dequantize needs room for every token
    d4 = _desc(num_quantized=100)
    assert L.kvq_dequantize(ctypes.byref(d4), 0, buf, 99, None) == kvq.KVQ_ERR_INVALID_ARG
    assert L.kvq_status_string(kvq.KVQ_ERR_CAPACITY) == b"cache capacity exceeded"


def test_footprint_matches_the_pages_per_token_bytes():
    # 70B shape, one layer: 8 KV heads x 128 channels. BF16 would take 2 * 2 * 8 * 128 bytes per
    # token per layer; FP8 codes take half of that and INT4 a quarter (memory table, infra.bea.ai).
    from decode_attention_quantize_b200 import kvq
    L = kvq.lib
    d = _desc(batch=1, num_q_heads=64, num_kv_heads=8, capacity=4096)
    f = kvq.KvqFootprint()
    assert L.kvq_cache_bytes(ctypes.byref(d), ctypes.byref(f)) == kvq.KVQ_OK
    assert f.code_bytes == 4096 * 2 * 8 * 128 and f.bytes_per_token == 2 * 128
    assert f.code_bytes * 80 / 4096 == 163840  # FP8 row of the memory table: 160 KiB per token
    buf = 0x30000
    d5 = _desc(batch=1, num_q_heads=64, num_kv_heads=8, capacity=4096, k_scheme=5, v_scheme=5, k_zero=buf,
               v_zero=buf, k_res=buf, v_res=buf)
    assert L.kvq_cache_bytes(ctypes.byref(d5), ctypes.byref(f)) == kvq.KVQ_OK
    assert f.code_bytes * 80 / 4096 == 81920  # INT4 codes: 80 KiB per token for 80 layers
    assert f.bytes_per_token == 2 * 64 + 2 * 8 * 4  # codes + fp32 (scale, min) per 32 elements


def test_rescale_flag_is_checked_on_the_host():
    from decode_attention_quantize_b200 import kvq
    L = kvq.lib
    d = _desc()
    cal = L.kvq_append_workspace_bytes(ctypes.byref(d), kvq.KVQ_APPEND_CALIBRATE)
    res = L.kvq_append_workspace_bytes(ctypes.byref(d), kvq.KVQ_APPEND_RESCALE)
    assert L.kvq_append_workspace_bytes(ctypes.byref(d), 0) == 0
    # the rescaling workspace holds the calibration keys plus the old scales, zero points and flags
    assert res >= cal + 2 * 2 * 128 * 5 + 16 and res % 256 == 0
    buf = 0x20000
    both = kvq.KVQ_APPEND_CALIBRATE | kvq.KVQ_APPEND_RESCALE
    assert L.kvq_quantize_append(ctypes.byref(d), buf, buf, kvq.KVQ_BF16, 4, None, both, buf, res,
                                 None) == kvq.KVQ_ERR_INVALID_ARG
    assert L.kvq_quantize_append(ctypes.byref(d), buf, buf, kvq.KVQ_BF16, 4, None, 0x4, buf, res,
                                 None) == kvq.KVQ_ERR_INVALID_ARG
    assert L.kvq_quantize_append(ctypes.byref(d), buf, buf, kvq.KVQ_BF16, 4, None, kvq.KVQ_APPEND_RESCALE,
                                 buf, cal, None) == kvq.KVQ_ERR_WORKSPACE
    assert d.num_quantized == 0  # nothing was accepted
    # statistics need one block row per (sequence, kv head): refused on the host past 65535
    big = _desc(batch=40000, num_q_heads=4, num_kv_heads=2, capacity=128)
    need = L.kvq_append_workspace_bytes(ctypes.byref(big), kvq.KVQ_APPEND_CALIBRATE)
    assert L.kvq_quantize_append(ctypes.byref(big), buf, buf, kvq.KVQ_BF16, 1, None, kvq.KVQ_APPEND_CALIBRATE,
                                 buf, need, None) == kvq.KVQ_ERR_UNSUPPORTED


def test_rescale_schedule_counts_tokens():
    # every 1024 appended tokens one append rescales (n4n.ai Step 7); a calibration restarts the count
    from decode_attention_quantize_b200.kvq import RescaleSchedule
    s = RescaleSchedule(1024)
    fired = [s.step(1) for _ in range(3000)]
    assert [i for i, f in enumerate(fired) if f] == [1023, 2047]
    s = RescaleSchedule(1024)
    assert not s.step(1000) and s.step(100) and s.pending == 0
    s.step(500)
    s.reset()
    assert s.pending == 0 and not s.step(1023) and s.step(1)
    with pytest.raises(ValueError):
        RescaleSchedule(0)


def test_validation_bounds_the_decode_plan_integers():
    # the decode's split plan counts pairs and tiles in 32-bit integers: refused on the host
    from decode_attention_quantize_b200 import kvq
    L = kvq.lib
    buf = 0x10000
    paged = dict(layout=1, page_table=buf, seq_lens=buf, num_pages=8)
    cases = [
        dict(num_q_heads=16384, num_kv_heads=2),                                   # > 8192 query heads
        dict(batch=1000, num_q_heads=8192, num_kv_heads=1, capacity=1 << 20),     # 2^20 pairs x 8196 tiles
        dict(page_size=64, max_pages_per_seq=(1 << 25) + 1, **paged),              # longest length >= 2^31
        dict(batch=65535, num_q_heads=8, num_kv_heads=8, page_size=64, max_pages_per_seq=8200, **paged),
    ]
    for kw in cases:
        assert L.kvq_validate(ctypes.byref(_desc(**kw))) == kvq.KVQ_ERR_UNSUPPORTED, kw
    assert L.kvq_validate(ctypes.byref(_desc(num_q_heads=8192, num_kv_heads=1))) == kvq.KVQ_OK


def test_binding_checks_shapes_before_any_device_call():
    # a wrong-shaped tensor would make the kernels read or write past a buffer: the binding
    # refuses it on the host (CPU tensors here; nothing reaches the library)
    import torch
    from decode_attention_quantize_b200 import kvq
    cache = kvq.QuantizedKVCache(kvq.CacheSpec(2, 8, 2, kvq.FP8_E4M3_PER_TENSOR, kvq.FP8_E4M3_PER_TENSOR,
                                               capacity=256), device="cpu")
    good_kv = torch.zeros(2, 2, 4, 128, dtype=torch.bfloat16)
    bad = [
        (torch.zeros(2, 2, 4, 64, dtype=torch.bfloat16), good_kv),      # head_dim
        (torch.zeros(1, 2, 4, 128, dtype=torch.bfloat16), good_kv),     # batch
        (good_kv, torch.zeros(2, 2, 5, 128, dtype=torch.bfloat16)),     # v_new tokens differ
        (good_kv, torch.zeros(2, 2, 4, 128, dtype=torch.float32)),      # dtypes differ
        (torch.zeros(2, 4, 128, dtype=torch.bfloat16), good_kv),        # not 4-D
    ]
    for k, v in bad:
        with pytest.raises(ValueError):
            cache.append(k, v)
    with pytest.raises(ValueError):
        cache.append(good_kv, good_kv, new_lens=torch.zeros(2, dtype=torch.int32))  # dense: counts refused
    for q in (torch.zeros(2, 4, 128, dtype=torch.bfloat16), torch.zeros(2, 8, 64, dtype=torch.bfloat16),
              torch.zeros(3, 8, 128, dtype=torch.bfloat16)):
        with pytest.raises(ValueError, match="q: shape"):
            cache.decode(q)
    q = torch.zeros(2, 8, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="out: shape"):
        cache.decode(q, out=torch.zeros(2, 8, 127))
    with pytest.raises(ValueError, match="out: float32"):
        cache.decode(q, out=torch.zeros(2, 8, 128, dtype=torch.float64))
    with pytest.raises(ValueError, match="lse: shape"):
        cache.decode(q, lse=torch.zeros(2, 4))
    with pytest.raises(ValueError, match="out: shape"):
        kvq.kvq_dequantize(cache.desc, 0, 10, out=torch.zeros(2, 2, 9, 128))
    paged = kvq.QuantizedKVCache(kvq.CacheSpec(2, 8, 2, kvq.INT8_SYM_PER_TENSOR, kvq.INT8_SYM_PER_TENSOR, paged=True,
                                               max_pages=4, num_pages=8), device="cpu")
    with pytest.raises(ValueError, match="new_lens"):
        paged.append(good_kv, good_kv, new_lens=torch.zeros(3, dtype=torch.int32))
    with pytest.raises(ValueError, match="new_lens: int32"):
        paged.append(good_kv, good_kv, new_lens=torch.zeros(2, dtype=torch.int64))
    # the one-call step checks the new rows and the query before anything is launched
    for k, v in bad:
        with pytest.raises(ValueError):
            cache.append_decode(k, v, q)
    with pytest.raises(ValueError, match="q: shape"):
        cache.append_decode(good_kv, good_kv, torch.zeros(2, 4, 128, dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="out: shape"):
        cache.append_decode(good_kv, good_kv, q, out=torch.zeros(2, 8, 127))
    scheduled = kvq.QuantizedKVCache(kvq.CacheSpec(2, 8, 2, kvq.FP8_E4M3_PER_TENSOR, kvq.FP8_E4M3_PER_TENSOR,
                                                   capacity=256), device="cpu", rescale_every=1024)
    with pytest.raises(ValueError, match="rescaling schedule"):
        scheduled.append_decode(good_kv, good_kv, q)
    assert cache.num_quantized == 0  # nothing was appended


def test_fp16_kivi_metadata_halves_the_metadata_bytes():
    # fp16 scale and minimum per 32 elements: KIVI INT2 takes 2 + 16 * 2 / 32 = 3 bits per element
    # and INT4 takes 5, against 4 and 6 with fp32 metadata
    from decode_attention_quantize_b200 import kvq
    L = kvq.lib
    buf = 0x30000
    f = kvq.KvqFootprint()
    bits = {}
    for sch in (kvq.KIVI_INT2, kvq.KIVI_INT2_F16, kvq.KIVI_INT4, kvq.KIVI_INT4_F16):
        d = _desc(batch=1, num_q_heads=64, num_kv_heads=8, capacity=4096, k_scheme=sch, v_scheme=sch, k_zero=buf,
                  v_zero=buf, k_res=buf, v_res=buf)
        assert L.kvq_cache_bytes(ctypes.byref(d), ctypes.byref(f)) == kvq.KVQ_OK
        bits[sch] = f.bytes_per_token * 8 / (2 * 128)
        meta_elems = 2 * 2 * 8 * (4096 // 32) * 128  # (K + V) x (scale + min)
        assert f.meta_bytes == meta_elems * (2 if sch in (kvq.KIVI_INT2_F16, kvq.KIVI_INT4_F16) else 4)
    assert bits == {kvq.KIVI_INT2: 4.0, kvq.KIVI_INT2_F16: 3.0, kvq.KIVI_INT4: 6.0, kvq.KIVI_INT4_F16: 5.0}


def test_prerope_validation():
    # keys cached before RoPE: a finite base >= 0, 8-bit key codes, not with the Hadamard rotation
    from decode_attention_quantize_b200 import kvq
    L = kvq.lib
    buf = 0x30000
    assert L.kvq_validate(ctypes.byref(_desc(rope_theta=500000.0))) == kvq.KVQ_OK
    assert L.kvq_validate(ctypes.byref(_desc(rope_theta=-1.0))) == kvq.KVQ_ERR_INVALID_ARG
    assert L.kvq_validate(ctypes.byref(_desc(rope_theta=float("nan")))) == kvq.KVQ_ERR_INVALID_ARG
    assert L.kvq_validate(ctypes.byref(_desc(rope_theta=float("inf")))) == kvq.KVQ_ERR_INVALID_ARG
    assert L.kvq_validate(ctypes.byref(_desc(rope_theta=1e4, rotation=1))) == kvq.KVQ_ERR_UNSUPPORTED
    kivi = dict(k_scheme=5, v_scheme=5, k_zero=buf, v_zero=buf, k_res=buf, v_res=buf)
    assert L.kvq_validate(ctypes.byref(_desc(rope_theta=1e4, **kivi))) == kvq.KVQ_ERR_UNSUPPORTED
    assert L.kvq_validate(ctypes.byref(_desc(rope_theta=1e4, k_scheme=8, v_scheme=8))) == kvq.KVQ_ERR_UNSUPPORTED
    # a pair with no pre-RoPE decode kernel is refused before anything is launched
    d = _desc(rope_theta=1e4, k_scheme=2, v_scheme=2)
    need = L.kvq_decode_workspace_bytes(ctypes.byref(d))
    assert L.kvq_decode_attention(ctypes.byref(d), buf, 1, ctypes.c_float(0.088), buf, None, buf, need,
                                  None) == kvq.KVQ_ERR_UNSUPPORTED


def test_append_decode_checks_both_calls_before_launch():
    # every check of the append and of the decode runs before anything is launched: a failing
    # decode argument leaves the descriptor's length unchanged (no append happened)
    from decode_attention_quantize_b200 import kvq
    L = kvq.lib
    buf = 0x20000
    d = _desc(num_quantized=100)
    need = L.kvq_decode_workspace_bytes(ctypes.byref(d))

    def call(n_new=1, q_dtype=1, scale=0.088, out=buf, ws_bytes=None, in_dtype=kvq.KVQ_BF16, k=buf):
        return L.kvq_append_decode(ctypes.byref(d), k, buf, in_dtype, n_new, buf, q_dtype, ctypes.c_float(scale),
                                   out, None, buf, need if ws_bytes is None else ws_bytes, None)

    assert call(ws_bytes=need - 1) == kvq.KVQ_ERR_WORKSPACE
    assert call(q_dtype=7) == kvq.KVQ_ERR_INVALID_ARG
    assert call(scale=-1.0) == kvq.KVQ_ERR_INVALID_ARG
    assert call(out=buf + 4) == kvq.KVQ_ERR_INVALID_ARG
    assert call(n_new=-1) == kvq.KVQ_ERR_INVALID_ARG
    assert call(in_dtype=5) == kvq.KVQ_ERR_INVALID_ARG
    assert call(k=buf + 2) == kvq.KVQ_ERR_INVALID_ARG  # misaligned new keys
    assert call(n_new=157) == kvq.KVQ_ERR_CAPACITY      # 100 + 157 > 256
    assert d.num_quantized == 100
    # KIVI appends take bf16 only
    d3 = _desc(k_scheme=5, v_scheme=5, k_zero=buf, v_zero=buf, k_res=buf, v_res=buf)
    need3 = L.kvq_decode_workspace_bytes(ctypes.byref(d3))
    assert L.kvq_append_decode(ctypes.byref(d3), buf, buf, kvq.KVQ_F32, 1, buf, 1, ctypes.c_float(0.088), buf,
                               None, buf, need3, None) == kvq.KVQ_ERR_UNSUPPORTED

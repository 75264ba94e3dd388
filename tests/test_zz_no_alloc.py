"""The allocation-free decode entry point against the regular one.

kvq_decode_attention_noalloc serves callers that cannot call cudaMalloc (an engine plugin
that only receives its input and output buffers, code running during CUDA graph capture,
a serving loop that forbids allocation after start-up). It runs the same kernels with the
same launch shape as kvq_decode_attention given a caller workspace, so its output and lse
must be bit-identical to that call's, call after call: for dense and paged caches, for a
large cache followed by a smaller one (the shared scratch keeps the larger call's data), and
for a cache whose workspace is just under the scratch size. Caches whose partials would not
fit the scratch are rejected on the host. This file is collected last so a failure here
cannot hide a failure elsewhere; it also passes on its own.
"""
import ctypes
import math

import pytest
import torch

import synth
from tests import harness as H

pytestmark = pytest.mark.gpu
SCALE = 1.0 / math.sqrt(128.0)


def _noalloc(kvq, desc, q, out, lse):
    return kvq.lib.kvq_decode_attention_noalloc(
        ctypes.byref(desc), ctypes.c_void_p(q.data_ptr()), kvq.KVQ_BF16, ctypes.c_float(SCALE),
        ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(lse.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _cache(kvq, ks, vs, B, Hq, Hkv, T, seed):
    w = H.workload(B, Hq, Hkv, ks, vs, seed=seed)
    K = synth.keys(w, 0, B, 0, Hkv, 0, T)
    V = synth.values(w, 0, B, 0, Hkv, 0, T)
    gc = kvq.QuantizedKVCache(kvq.CacheSpec(B, Hq, Hkv, ks, vs, capacity=(T + 127) // 128 * 128))
    gc.append(H.dev(K, True), H.dev(V, True), calibrate=ks in H.CALIBRATED)
    return gc, H.dev(synth.queries(w, 0, 0, B), True)


def _same_as_workspace_decode(kvq, gc, q, calls=2, where=""):
    """Two no-alloc calls, each bit-identical to the workspace decode of the same cache."""
    ref_lse = torch.empty(q.shape[:2], dtype=torch.float32, device="cuda")
    ref, _ = gc.decode(q, SCALE, lse=ref_lse)
    for call in range(calls):
        out = torch.full(tuple(q.shape), float("nan"), dtype=torch.float32, device="cuda")
        lse = torch.full(q.shape[:2], float("nan"), dtype=torch.float32, device="cuda")
        assert _noalloc(kvq, gc.desc, q, out, lse) == kvq.KVQ_OK
        torch.cuda.synchronize()
        assert torch.equal(out, ref), f"{where} call {call}: output differs from the workspace decode"
        assert torch.equal(lse, ref_lse), f"{where} call {call}: lse differs from the workspace decode"
    assert gc.status()[0] == 0


@pytest.mark.parametrize("ks,vs", [(synth.FP8_E4M3_PER_TENSOR, synth.FP8_E4M3_PER_TENSOR),
                                   (synth.KIVI_INT4, synth.KIVI_INT4)])
def test_noalloc_matches_workspace_decode_on_two_calls(ks, vs):
    kvq = H.kvq()
    gc, q = _cache(kvq, ks, vs, B=4, Hq=32, Hkv=4, T=1000, seed=31)
    _same_as_workspace_decode(kvq, gc, q, where=f"schemes {ks}/{vs}")


def test_noalloc_paged_int8():
    # the paged plan also lives in the scratch array
    kvq = H.kvq()
    B, Hq, Hkv = 4, 16, 4
    w, oc, gc, K, V, lens, calib, nl = H.paged_case(B, Hq, Hkv, synth.INT8_SYM_PER_TENSOR,
                                                    synth.UINT8_ASYM_PER_CHANNEL, lens=[37, 1000, 5, 640], steps=0)
    gc.append(H.dev(K, True), H.dev(V, True), new_lens=nl, calibrate=True)
    _same_as_workspace_decode(kvq, gc, H.dev(synth.queries(w, 0, 0, B), True), where="paged int8")


def test_noalloc_large_then_small_then_large():
    # a smaller cache after a larger one finds the larger call's partials in the shared scratch
    kvq = H.kvq()
    big = _cache(kvq, synth.FP8_E4M3_PER_TENSOR, synth.FP8_E4M3_PER_TENSOR, B=16, Hq=64, Hkv=8, T=3000, seed=41)
    small = _cache(kvq, synth.INT8_SYM_PER_TOKEN, synth.INT8_SYM_PER_TOKEN, B=2, Hq=8, Hkv=2, T=300, seed=42)
    _same_as_workspace_decode(kvq, *big, calls=1, where="large")
    _same_as_workspace_decode(kvq, *small, calls=1, where="small after large")
    _same_as_workspace_decode(kvq, *big, calls=1, where="large after small")


def _noalloc_fits(kvq, B):
    from decode_attention_quantize_b200.kvq import KvqDesc
    d = KvqDesc()
    d.batch, d.num_q_heads, d.num_kv_heads, d.head_dim = B, 8, 1, 128
    return kvq.lib.kvq_decode_workspace_bytes(ctypes.byref(d)) <= kvq.NOALLOC_SCRATCH_BYTES


def test_noalloc_just_under_the_scratch_size():
    kvq = H.kvq()
    B = 1
    while _noalloc_fits(kvq, B + 1):
        B += 1
    assert not _noalloc_fits(kvq, B + 1)
    gc, q = _cache(kvq, synth.FP8_E4M3_PER_TENSOR, synth.FP8_E4M3_PER_TENSOR, B=B, Hq=8, Hkv=1, T=300, seed=43)
    need = kvq.lib.kvq_decode_workspace_bytes(ctypes.byref(gc.desc))
    assert kvq.NOALLOC_SCRATCH_BYTES - 8192 < need <= kvq.NOALLOC_SCRATCH_BYTES
    _same_as_workspace_decode(kvq, gc, q, where=f"batch {B}, workspace {need} bytes")


def test_noalloc_rejects_a_cache_too_large_for_its_scratch():
    kvq = H.kvq()
    from decode_attention_quantize_b200.kvq import KvqDesc
    d = KvqDesc()
    d.batch, d.num_q_heads, d.num_kv_heads, d.head_dim = 4096, 64, 8, 128
    d.k_scheme = d.v_scheme = synth.FP8_E4M3_PER_TENSOR
    d.layout, d.capacity = kvq.KVQ_DENSE, 128
    d.group_size, d.residual_cap = 32, 128
    for f in ("k_codes", "v_codes", "k_scale", "v_scale", "dev_status"):
        setattr(d, f, 0x10000)  # rejected on the host before any device access
    assert kvq.lib.kvq_decode_workspace_bytes(ctypes.byref(d)) > kvq.NOALLOC_SCRATCH_BYTES
    st = kvq.lib.kvq_decode_attention_noalloc(ctypes.byref(d), ctypes.c_void_p(0x20000), kvq.KVQ_BF16,
                                              ctypes.c_float(0.088), ctypes.c_void_p(0x20000), None, None)
    assert st == kvq.KVQ_ERR_WORKSPACE

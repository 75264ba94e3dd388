"""The allocation-free decode entry point against the regular one.

kvq_decode_attention_noalloc serves callers that cannot call cudaMalloc (an engine plugin
that only receives its input and output buffers, code running during CUDA graph capture,
a serving loop that forbids allocation after start-up). It must give the same attention
output as kvq_decode_attention with a caller workspace, call after call, and must reject
caches whose partials would not fit its static scratch array. This file is collected last
so a failure here cannot hide a failure elsewhere; it also passes on its own.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

import synth
from tests import harness as H

pytestmark = pytest.mark.gpu


def _noalloc(kvq, desc, q, out, lse):
    return kvq.lib.kvq_decode_attention_noalloc(
        ctypes.byref(desc), ctypes.c_void_p(q.data_ptr()), kvq.KVQ_BF16, ctypes.c_float(1.0 / math.sqrt(128.0)),
        ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(lse.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _cache(kvq, ks, vs, B, Hq, Hkv, T, seed):
    w = H.workload(B, Hq, Hkv, ks, vs, seed=seed)
    K = synth.keys(w, 0, B, 0, Hkv, 0, T)
    V = synth.values(w, 0, B, 0, Hkv, 0, T)
    gc = kvq.QuantizedKVCache(kvq.CacheSpec(B, Hq, Hkv, ks, vs, capacity=(T + 127) // 128 * 128))
    gc.append(H.dev(K, True), H.dev(V, True), calibrate=ks in H.CALIBRATED)
    return gc, H.dev(synth.queries(w, 0, 0, B), True)


@pytest.mark.parametrize("ks,vs", [(synth.FP8_E4M3_PER_TENSOR, synth.FP8_E4M3_PER_TENSOR),
                                   (synth.KIVI_INT4, synth.KIVI_INT4)])
def test_noalloc_matches_workspace_decode_on_two_calls(ks, vs):
    kvq = H.kvq()
    gc, q = _cache(kvq, ks, vs, B=4, Hq=32, Hkv=4, T=1000, seed=31)
    ref_lse = torch.empty(q.shape[:2], dtype=torch.float32, device="cuda")
    ref, _ = gc.decode(q, 1.0 / math.sqrt(128.0), lse=ref_lse)
    torch.cuda.synchronize()
    ref = ref.cpu().numpy().astype(np.float64)
    for call in range(2):
        out = torch.full_like(q, float("nan"), dtype=torch.float32)
        lse = torch.full(q.shape[:2], float("nan"), dtype=torch.float32, device="cuda")
        assert _noalloc(kvq, gc.desc, q, out, lse) == kvq.KVQ_OK
        torch.cuda.synchronize()
        H.attn_check(out, ref, lse, ref_lse.cpu().numpy().astype(np.float64), where=f"noalloc call {call}")


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

"""GPU parity for keys cached before RoPE, with RoPE applied at decode.

KVQuant quantizes keys before the rotary embedding ("KV Cache Quantization in Production LLM
Serving", llms.blog, §4): the cache holds the keys as they come, and decode rotates each
dequantized key at its position t in the sequence (pairs (i, i + 64), angle t * base^(-2i/128))
before the scores; the queries arrive rotated. The oracle does the rotation in fp64 on its own
dequantized keys; the library rotates in fp32 with angles reduced modulo 2 pi in fp64. Codes
are the plain schemes' (bit for bit); attention within 2e-4 * max|ref| of the fp64 oracle,
including positions near 131072 where an angle formed in fp32 alone would be off by ~1e-2 rad.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import OracleCache
from tests import harness as H

pytestmark = pytest.mark.gpu
S = synth
THETA = 500000.0
PAIRS = [(S.FP8_E4M3_PER_TENSOR, S.FP8_E4M3_PER_TENSOR), (S.INT8_SYM_PER_CHANNEL, S.UINT8_ASYM_PER_CHANNEL),
         (S.INT8_SYM_PER_TENSOR, S.UINT8_ASYM_PER_CHANNEL)]


@pytest.mark.parametrize("ks,vs", PAIRS)
def test_prerope_dense(ks, vs):
    H.dense_case(B=2, Hq=16, Hkv=2, ks=ks, vs=vs, prefill=300, steps=2, rope=0.0, prerope=THETA, outlier=100.0)


@pytest.mark.parametrize("G", [1, 4, 8, 16])
def test_prerope_gqa_sizes(G):
    H.dense_case(B=2, Hq=2 * G, Hkv=2, ks=S.FP8_E4M3_PER_TENSOR, vs=S.FP8_E4M3_PER_TENSOR, prefill=200, steps=1,
                 rope=0.0, prerope=THETA)


def test_prerope_fp32_queries_and_other_base():
    # fp32 queries take the hi/lo query split as well; a base of 10000 turns the angles faster
    H.dense_case(B=2, Hq=8, Hkv=2, ks=S.INT8_SYM_PER_CHANNEL, vs=S.UINT8_ASYM_PER_CHANNEL, prefill=257, steps=1,
                 bf16=True, q_bf16=False, rope=0.0, prerope=10000.0)
    H.dense_case(B=1, Hq=4, Hkv=1, ks=S.FP8_E4M3_PER_TENSOR, vs=S.FP8_E4M3_PER_TENSOR, prefill=130, steps=1,
                 bf16=False, rope=0.0, prerope=10000.0)


@pytest.mark.parametrize("ks,vs", PAIRS)
@pytest.mark.parametrize("ps", [16, 64])
def test_prerope_paged(ks, vs, ps):
    B, Hq, Hkv = 4, 16, 4
    w, oc, gc, K, V, lens, calib, nl = H.paged_case(B, Hq, Hkv, ks, vs, lens=[37, 300, 5, 64], page_size=ps,
                                                    steps=2, prerope=THETA)
    oc.append(K, V, True, calibrate=calib, new_lens=lens)
    gc.append(H.dev(K, True), H.dev(V, True), new_lens=nl, calibrate=calib)
    torch.cuda.synchronize()
    H.compare_paged(oc, gc, "pre-RoPE paged prefill")
    H.decode_both(oc, gc, synth.queries(w, 0, 0, B), True, "pre-RoPE paged decode 0")
    for s in range(2):
        kk = np.stack([synth.keys(w, b, b + 1, 0, Hkv, int(lens[b]) + s, int(lens[b]) + s + 1)[0] for b in range(B)])
        vv = np.stack([synth.values(w, b, b + 1, 0, Hkv, int(lens[b]) + s, int(lens[b]) + s + 1)[0] for b in range(B)])
        oc.append(kk, vv, True)
        gc.append(H.dev(kk, True), H.dev(vv, True))
        torch.cuda.synchronize()
        H.compare_paged(oc, gc, f"pre-RoPE paged step {s}")
        H.decode_both(oc, gc, synth.queries(w, s + 1, 0, B), True, f"pre-RoPE paged decode {s + 1}")
    assert gc.status()[0] == 0


def test_prerope_positions_near_131072():
    # the keys past position 130900 are 100x larger, so the softmax weight sits on the far
    # positions, where the angle t * theta_0 is ~1.3e5 rad
    B, Hq, Hkv, T = 1, 4, 1, 131072 + 200
    ks = vs = S.FP8_E4M3_PER_TENSOR
    w = H.workload(B, Hq, Hkv, ks, vs, rope=0.0, seed=17)
    K = synth.bf16_bits_to_f32(synth.keys(w, 0, B, 0, Hkv, 0, T))
    V = synth.bf16_bits_to_f32(synth.values(w, 0, B, 0, Hkv, 0, T))
    K[:, :, 130900:] *= np.float32(10.0)
    K[:, :, :130900] *= np.float32(0.1)
    K, V = np.ascontiguousarray(K, np.float32), np.ascontiguousarray(V, np.float32)
    cap = (T + 127) // 128 * 128
    oc = OracleCache(B, Hq, Hkv, 128, ks, vs, cap=cap, rope_theta=THETA)
    gc = H.kvq().QuantizedKVCache(H.kvq().CacheSpec(B, Hq, Hkv, ks, vs, capacity=cap, rope_theta=THETA))
    oc.append(K, V, False, calibrate=True)
    gc.append(H.dev(K, False), H.dev(V, False), calibrate=True)
    torch.cuda.synchronize()
    H.compare_dense(oc, gc, "long pre-RoPE cache")
    for step in range(2):
        H.decode_both(oc, gc, synth.queries(w, step, 0, B), True, f"pre-RoPE decode at 131k, query {step}")
    assert gc.status()[0] == 0


def test_prerope_dequantize_returns_the_stored_keys():
    oc, gc, _ = H.dense_case(B=2, Hq=8, Hkv=2, ks=S.FP8_E4M3_PER_TENSOR, vs=S.FP8_E4M3_PER_TENSOR, prefill=150,
                             steps=0, rope=0.0, prerope=THETA)
    for which in (0, 1):
        got = gc.dequantize(which, 150).cpu().numpy()
        assert np.array_equal(got.view(np.uint32), oc.dequantize(which, 150).view(np.uint32))

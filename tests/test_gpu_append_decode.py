"""GPU parity of the one-call decode step (kvq_append_decode): a plain append, then decode over
the updated cache, the decode of a dense 8-bit / INT4 cache reading the cached tiles while the
append runs ("KV Cache Quantization" (infra.bea.ai), §4 FP8 KV cache: the cache is appended to
and read at every step). Codes bit-exact against the oracle after every step; attention within
2e-4 * max|ref| of the fp64 oracle over the updated cache. Steps land on and across tile
boundaries (the decode waits for the append exactly before the tiles holding new positions)."""
import numpy as np
import pytest
import torch

import synth
from oracle import OracleCache
from tests import harness as H

pytestmark = pytest.mark.gpu
S = synth


def fused_steps(ks, vs, prefill, news, B=2, Hq=8, Hkv=2, bf16=True, q_bf16=None, group=32, rotate=False,
                prerope=0.0, seed=31):
    q_bf16 = bf16 if q_bf16 is None else q_bf16
    w = H.workload(B, Hq, Hkv, ks, vs, bf16=bf16, seed=seed, rope=0.0 if prerope else 500000.0)
    total = prefill + sum(news)
    cap = max(128, (total + 127) // 128 * 128)
    K = synth.keys(w, 0, B, 0, Hkv, 0, total)
    V = synth.values(w, 0, B, 0, Hkv, 0, total)
    oc = OracleCache(B, Hq, Hkv, 128, ks, vs, cap=cap, rotate=rotate, group=group, rope_theta=prerope)
    gc = H.kvq().QuantizedKVCache(H.kvq().CacheSpec(B, Hq, Hkv, ks, vs, capacity=cap, rotate=rotate, group=group,
                                                    rope_theta=prerope))
    calib = ks in H.CALIBRATED or vs in H.CALIBRATED
    oc.append(K[:, :, :prefill], V[:, :, :prefill], bf16, calibrate=calib)
    gc.append(H.dev(K[:, :, :prefill], bf16), H.dev(V[:, :, :prefill], bf16), calibrate=calib)
    torch.cuda.synchronize()
    qw = H.workload(B, Hq, Hkv, ks, vs, bf16=q_bf16, seed=seed)
    pos = prefill
    for s, n in enumerate(news):
        kk = np.ascontiguousarray(K[:, :, pos:pos + n])
        vv = np.ascontiguousarray(V[:, :, pos:pos + n])
        q = synth.queries(qw, s, 0, B)
        oc.append(kk, vv, bf16)
        lse = torch.empty((B, Hq), dtype=torch.float32, device="cuda")
        out, _ = gc.append_decode(H.dev(kk, bf16), H.dev(vv, bf16), H.dev(q, q_bf16), float(H.SCALE), lse=lse)
        torch.cuda.synchronize()
        H.compare_dense(oc, gc, f"step {s} (positions {pos}..{pos + n - 1})")
        ref, ref_lse = oc.decode(q, q_bf16, float(H.SCALE))
        H.attn_check(out, ref, lse, ref_lse, f"fused decode step {s}")
        pos += n
    assert gc.status()[0] == 0
    return oc, gc


# prefills that put the appended positions at the end of a tile, at the start of the next one,
# and across a tile boundary (multi-token steps)
STEPS = [(126, [1, 1, 1, 3]), (255, [1, 2]), (300, [5, 1])]


@pytest.mark.parametrize("prefill,news", STEPS)
@pytest.mark.parametrize("ks,vs", [(S.FP8_E4M3_PER_TENSOR, S.FP8_E4M3_PER_TENSOR),
                                   (S.FP8_E5M2_PER_TENSOR, S.FP8_E5M2_PER_TENSOR),
                                   (S.INT8_SYM_PER_TENSOR, S.UINT8_ASYM_PER_CHANNEL),
                                   (S.INT8_SYM_PER_TOKEN, S.INT8_SYM_PER_TOKEN),
                                   (S.INT8_SYM_PER_CHANNEL, S.UINT8_ASYM_PER_CHANNEL),
                                   (S.INT4_SYM_PER_GROUP, S.INT4_SYM_PER_GROUP)])
def test_fused_step_dense(ks, vs, prefill, news):
    fused_steps(ks, vs, prefill, news)


def test_fused_step_variants():
    fused_steps(S.INT4_SYM_PER_GROUP, S.INT4_SYM_PER_GROUP, 129, [1, 2], group=128, rotate=True)
    fused_steps(S.FP8_E4M3_PER_TENSOR, S.FP8_E4M3_PER_TENSOR, 200, [1, 1], bf16=False)           # fp32 rows
    fused_steps(S.FP8_E4M3_PER_TENSOR, S.FP8_E4M3_PER_TENSOR, 127, [1, 2], prerope=500000.0)    # pre-RoPE keys
    fused_steps(S.INT8_SYM_PER_TENSOR, S.UINT8_ASYM_PER_CHANNEL, 64, [1, 1], B=3, Hq=24, Hkv=3)  # G = 8


def test_fused_step_without_new_tokens():
    # n_new = 0: nothing is appended, so the decode is not a dependent of an append and waits at
    # its start as the plain decode does
    fused_steps(S.FP8_E4M3_PER_TENSOR, S.FP8_E4M3_PER_TENSOR, 200, [1, 0, 1])


def test_fused_step_kivi_runs_in_sequence():
    # KIVI (the flush may rewrite a whole group) takes the two calls one after the other
    fused_steps(S.KIVI_INT4, S.KIVI_INT4, 250, [3, 4, 1])


def test_fused_step_paged_runs_in_sequence():
    B, Hq, Hkv = 3, 8, 2
    ks, vs = S.INT8_SYM_PER_TENSOR, S.UINT8_ASYM_PER_CHANNEL
    w, oc, gc, K, V, lens, calib, nl = H.paged_case(B, Hq, Hkv, ks, vs, lens=[40, 100, 17], page_size=16, steps=2)
    oc.append(K, V, True, calibrate=calib, new_lens=lens)
    gc.append(H.dev(K, True), H.dev(V, True), new_lens=nl, calibrate=calib)
    torch.cuda.synchronize()
    for s in range(2):
        kk = np.stack([synth.keys(w, b, b + 1, 0, Hkv, int(lens[b]) + s, int(lens[b]) + s + 1)[0] for b in range(B)])
        vv = np.stack([synth.values(w, b, b + 1, 0, Hkv, int(lens[b]) + s, int(lens[b]) + s + 1)[0] for b in range(B)])
        q = synth.queries(w, s, 0, B)
        oc.append(kk, vv, True)
        lse = torch.empty((B, Hq), dtype=torch.float32, device="cuda")
        out, _ = gc.append_decode(H.dev(kk, True), H.dev(vv, True), H.dev(q, True), float(H.SCALE), lse=lse)
        torch.cuda.synchronize()
        H.compare_paged(oc, gc, f"paged fused step {s}")
        ref, ref_lse = oc.decode(q, True, float(H.SCALE))
        H.attn_check(out, ref, lse, ref_lse, f"paged fused decode {s}")
    assert gc.status()[0] == 0

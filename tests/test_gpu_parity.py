"""GPU parity: the CUDA library (through its C ABI) against the CPU oracle.

Codes, scales, zero points and residual tokens must match bit for bit; decode attention
must satisfy max|err| <= 2e-4 * max|ref| against the fp64 oracle on the same cache.
Sizes span several tiles with ragged tails; every scheme pair, both layouts, GQA group
sizes 1, 4, 8 and 16, streaming appends and the KIVI flush boundary are covered.
"""
import numpy as np
import pytest
import torch

import synth
from tests import harness as H

pytestmark = pytest.mark.gpu

S = synth


# ------------------------------------------------------------------ dense, 8-bit schemes
@pytest.mark.parametrize("ks,vs", [
    (S.FP8_E4M3_PER_TENSOR, S.FP8_E4M3_PER_TENSOR),
    (S.FP8_E5M2_PER_TENSOR, S.FP8_E5M2_PER_TENSOR),
    (S.INT8_SYM_PER_TENSOR, S.INT8_SYM_PER_TENSOR),
    (S.INT8_SYM_PER_TOKEN, S.INT8_SYM_PER_TOKEN),
    (S.INT8_SYM_PER_CHANNEL, S.INT8_SYM_PER_CHANNEL),
    (S.UINT8_ASYM_PER_CHANNEL, S.UINT8_ASYM_PER_CHANNEL),
    (S.INT8_SYM_PER_TENSOR, S.UINT8_ASYM_PER_CHANNEL),
    (S.INT8_SYM_PER_CHANNEL, S.UINT8_ASYM_PER_CHANNEL),
])
def test_dense_8bit_schemes(ks, vs):
    H.dense_case(B=2, Hq=16, Hkv=2, ks=ks, vs=vs, prefill=300, steps=2)


@pytest.mark.parametrize("G", [1, 4, 8, 16])
def test_gqa_group_sizes(G):
    H.dense_case(B=2, Hq=2 * G, Hkv=2, ks=S.FP8_E4M3_PER_TENSOR, vs=S.FP8_E4M3_PER_TENSOR, prefill=200, steps=1)


def test_fp32_inputs_and_queries():
    # fp32 K/V/Q (the tiny configuration's input type); Q needs the hi/lo split
    H.dense_case(B=1, Hq=4, Hkv=1, ks=S.INT8_SYM_PER_TOKEN, vs=S.INT8_SYM_PER_TOKEN, prefill=257, steps=2,
                 bf16=False, rope=0.0)
    H.dense_case(B=2, Hq=8, Hkv=2, ks=S.FP8_E4M3_PER_TENSOR, vs=S.FP8_E4M3_PER_TENSOR, prefill=130, steps=1,
                 bf16=True, q_bf16=False)


def test_tiny_int8_configuration_full_size():
    w = synth.workloads()["tiny_int8"]
    _, _, err = H.dense_case(B=w.B, Hq=w.Hq, Hkv=w.Hkv, ks=w.k_scheme, vs=w.v_scheme, prefill=w.context,
                             steps=0, bf16=False, seed=w.seed, outlier=w.outlier_scale, rope=w.rope_theta)
    assert err <= H.ATTN_RTOL


def test_single_token_and_chunked_prefill():
    H.dense_case(B=1, Hq=8, Hkv=1, ks=S.FP8_E4M3_PER_TENSOR, vs=S.FP8_E4M3_PER_TENSOR, prefill=1, steps=3)
    H.dense_case(B=2, Hq=8, Hkv=2, ks=S.INT8_SYM_PER_TOKEN, vs=S.INT8_SYM_PER_TOKEN, prefill=333, steps=1,
                 chunks=[17, 200])


def test_outliers_x100_int8_per_channel():
    H.dense_case(B=2, Hq=16, Hkv=2, ks=S.INT8_SYM_PER_CHANNEL, vs=S.UINT8_ASYM_PER_CHANNEL, prefill=190, steps=1,
                 outlier=100.0)


# ------------------------------------------------------------------ bulk prefill (four rows per thread)
# 4 x 2 x 9600 rows is past the size where the append switches to its bulk form; every pair
# the library accepts goes through it, the oracle recomputing every code bit for bit.
BULK_PAIRS = [
    (S.FP8_E4M3_PER_TENSOR, S.FP8_E4M3_PER_TENSOR), (S.INT8_SYM_PER_TENSOR, S.INT8_SYM_PER_TENSOR),
    (S.INT8_SYM_PER_TOKEN, S.INT8_SYM_PER_TOKEN), (S.INT8_SYM_PER_CHANNEL, S.INT8_SYM_PER_CHANNEL),
    (S.UINT8_ASYM_PER_CHANNEL, S.UINT8_ASYM_PER_CHANNEL), (S.INT8_SYM_PER_TENSOR, S.UINT8_ASYM_PER_CHANNEL),
    (S.INT8_SYM_PER_CHANNEL, S.UINT8_ASYM_PER_CHANNEL), (S.INT8_SYM_PER_TOKEN, S.UINT8_ASYM_PER_CHANNEL),
    (S.INT8_SYM_PER_TENSOR, S.INT8_SYM_PER_TOKEN), (S.FP8_E4M3_PER_TENSOR, S.INT8_SYM_PER_TENSOR),
    (S.INT8_SYM_PER_TENSOR, S.FP8_E4M3_PER_TENSOR), (S.FP8_E5M2_PER_TENSOR, S.FP8_E5M2_PER_TENSOR),
]


@pytest.mark.parametrize("ks,vs", BULK_PAIRS)
def test_bulk_prefill_every_pair(ks, vs):
    H.dense_case(B=4, Hq=8, Hkv=2, ks=ks, vs=vs, prefill=9600, steps=1, outlier=100.0)


def test_bulk_prefill_fp32_inputs():
    H.dense_case(B=4, Hq=8, Hkv=2, ks=S.INT8_SYM_PER_CHANNEL, vs=S.UINT8_ASYM_PER_CHANNEL, prefill=9600, steps=1,
                 bf16=False)


def test_bulk_prefill_paged():
    B, Hq, Hkv = 4, 8, 2
    w, oc, gc, K, V, lens, calib, nl = H.paged_case(B, Hq, Hkv, S.INT8_SYM_PER_TENSOR, S.UINT8_ASYM_PER_CHANNEL,
                                                    lens=[9600, 5000, 1, 9001], steps=0)
    oc.append(K, V, True, calibrate=True, new_lens=lens)
    gc.append(H.dev(K, True), H.dev(V, True), new_lens=nl, calibrate=True)
    torch.cuda.synchronize()
    H.compare_paged(oc, gc, "bulk paged prefill")
    H.decode_both(oc, gc, synth.queries(w, 0, 0, B), True, "bulk paged decode")
    assert gc.status()[0] == 0


# ------------------------------------------------------------------ KIVI
@pytest.mark.parametrize("scheme", [S.KIVI_INT4, S.KIVI_INT2, S.KIVI_INT4_F16, S.KIVI_INT2_F16])
@pytest.mark.parametrize("prefill", [44, 128, 129, 300, 384, 385])
def test_kivi_prefill_and_stream(scheme, prefill):
    H.dense_case(B=2, Hq=16, Hkv=2, ks=scheme, vs=scheme, prefill=prefill, steps=2, cap=640)


@pytest.mark.parametrize("scheme", [S.KIVI_INT4, S.KIVI_INT2, S.KIVI_INT4_F16, S.KIVI_INT2_F16])
def test_kivi_flush_on_stream_boundary(scheme):
    # 127 + 1 fills the residual; the next token flushes 128 tokens into 4 key groups
    H.dense_case(B=1, Hq=8, Hkv=1, ks=scheme, vs=scheme, prefill=127, steps=3, cap=256)
    H.dense_case(B=2, Hq=8, Hkv=2, ks=scheme, vs=scheme, prefill=256, steps=2, cap=512, outlier=100.0)


def test_kivi_chunked_appends_match_bulk():
    H.dense_case(B=1, Hq=16, Hkv=2, ks=S.KIVI_INT4, vs=S.KIVI_INT4, prefill=400, steps=1, cap=512,
                 chunks=[5, 100, 260])


# ------------------------------------------------------------------ paged
@pytest.mark.parametrize("ks,vs,ps", [
    (S.INT8_SYM_PER_TENSOR, S.UINT8_ASYM_PER_CHANNEL, 16),
    (S.INT8_SYM_PER_TENSOR, S.UINT8_ASYM_PER_CHANNEL, 32),
    (S.FP8_E4M3_PER_TENSOR, S.FP8_E4M3_PER_TENSOR, 16),
    (S.FP8_E5M2_PER_TENSOR, S.FP8_E5M2_PER_TENSOR, 32),
    (S.INT8_SYM_PER_TOKEN, S.INT8_SYM_PER_TOKEN, 64),
    (S.INT8_SYM_PER_CHANNEL, S.INT8_SYM_PER_CHANNEL, 16),
])
def test_paged(ks, vs, ps):
    B, Hq, Hkv = 4, 16, 4
    w, oc, gc, K, V, lens, calib, nl = H.paged_case(B, Hq, Hkv, ks, vs, lens=[37, 100, 5, 64], page_size=ps,
                                                    steps=3)
    oc.append(K, V, True, calibrate=calib, new_lens=lens)
    gc.append(H.dev(K, True), H.dev(V, True), new_lens=nl, calibrate=calib)
    torch.cuda.synchronize()
    H.compare_paged(oc, gc, "prefill")
    H.decode_both(oc, gc, synth.queries(w, 0, 0, B), True, "paged decode 0")
    for s in range(3):
        kk = np.stack([synth.keys(w, b, b + 1, 0, Hkv, int(lens[b]) + s, int(lens[b]) + s + 1)[0] for b in range(B)])
        vv = np.stack([synth.values(w, b, b + 1, 0, Hkv, int(lens[b]) + s, int(lens[b]) + s + 1)[0] for b in range(B)])
        oc.append(kk, vv, True)
        gc.append(H.dev(kk, True), H.dev(vv, True))
        torch.cuda.synchronize()
        H.compare_paged(oc, gc, f"step {s}")
        H.decode_both(oc, gc, synth.queries(w, s + 1, 0, B), True, f"paged decode {s + 1}")
    assert gc.status()[0] == 0


def test_paged_empty_sequence_and_variable_lengths():
    B, Hq, Hkv = 3, 8, 2
    w, oc, gc, K, V, lens, calib, nl = H.paged_case(B, Hq, Hkv, S.INT8_SYM_PER_TENSOR, S.UINT8_ASYM_PER_CHANNEL,
                                                    lens=[0, 250, 1], steps=0)
    oc.append(K, V, True, calibrate=True, new_lens=lens)
    gc.append(H.dev(K, True), H.dev(V, True), new_lens=nl, calibrate=True)
    torch.cuda.synchronize()
    H.compare_paged(oc, gc)
    q = synth.queries(w, 0, 0, B)
    lse = torch.empty((B, Hq), dtype=torch.float32, device="cuda")
    out, _ = gc.decode(H.dev(q, True), float(H.SCALE), lse=lse)
    ref, ref_lse = oc.decode(q, True, float(H.SCALE))
    torch.cuda.synchronize()
    assert torch.all(out[0] == 0) and torch.all(torch.isneginf(lse[0]))  # empty sequence
    H.attn_check(out, ref, lse, ref_lse, "variable lengths")
    assert np.abs(ref[1]).max() > 0


def test_bad_page_id_is_flagged_not_dereferenced():
    # sequence 1's second page is outside the pool: its append is refused on the device (its
    # length stays 0, the rows written to its good pages stay invisible), sequence 0 is appended
    B, Hq, Hkv = 2, 8, 2
    w, oc, gc, K, V, lens, calib, nl = H.paged_case(B, Hq, Hkv, S.INT8_SYM_PER_TENSOR, S.UINT8_ASYM_PER_CHANNEL,
                                                    lens=[40, 40], steps=0, bad_page=(1, 1))
    gc.append(H.dev(K, True), H.dev(V, True), new_lens=nl, calibrate=True)
    q = synth.queries(w, 0, 0, B)
    lse = torch.empty((B, Hq), dtype=torch.float32, device="cuda")
    out, _ = gc.decode(H.dev(q, True), float(H.SCALE), lse=lse)
    torch.cuda.synchronize()
    st = gc.status(clear=True)
    assert st[0] & H.kvq().KVQ_DEV_BAD_PAGE
    assert H.np_of(gc["seq_lens"]).tolist() == [40, 0]
    assert torch.all(out[1] == 0) and torch.all(torch.isneginf(lse[1]))
    # the oracle over the same statistics, with sequence 1 holding no tokens (the calibration
    # reads the whole block: the device saw both sequences' rows)
    oc.calibrate(K, V, True, new_lens=lens)
    oc.append(K, V, True, new_lens=np.array([40, 0], np.int32))  # the calibrated scales, sequence 0 only
    H.compare_paged(oc, gc, "after a refused sequence")
    ref, ref_lse = oc.decode(q, True, float(H.SCALE))
    H.attn_check(out, ref, lse, ref_lse, "decode after a refused sequence")
    assert gc.status()[0] == 0


def test_saturation_is_counted():
    # fixed per-tensor scale from a small prefill; a later token 50x larger saturates
    B, Hq, Hkv = 1, 8, 1
    gc = H.kvq().QuantizedKVCache(H.kvq().CacheSpec(B, Hq, Hkv, S.INT8_SYM_PER_TENSOR, S.INT8_SYM_PER_TENSOR,
                                                    capacity=128))
    x = torch.randn(B, Hkv, 4, 128, device="cuda", dtype=torch.float32)
    gc.append(x, x, calibrate=True)
    big = x[:, :, :1] * 50
    gc.append(big.contiguous(), big.contiguous())
    torch.cuda.synchronize()
    assert gc.status()[1] > 0


@pytest.mark.parametrize("scheme", [S.FP8_E4M3_PER_TENSOR, S.FP8_E5M2_PER_TENSOR, S.INT8_SYM_PER_TENSOR])
def test_saturated_codes_match_oracle(scheme):
    # a per-tensor scale calibrated on a small prefill, then tokens up to 50x past its range:
    # the saturated codes (largest finite of the format) must still match bit for bit
    B, Hq, Hkv = 2, 8, 2
    w = H.workload(B, Hq, Hkv, scheme, scheme, bf16=False)  # fp32 inputs, scaled below
    K = synth.keys(w, 0, B, 0, Hkv, 0, 70)
    V = synth.values(w, 0, B, 0, Hkv, 0, 70)
    oc = H.OracleCache(B, Hq, Hkv, 128, scheme, scheme, cap=128)
    gc = H.kvq().QuantizedKVCache(H.kvq().CacheSpec(B, Hq, Hkv, scheme, scheme, capacity=128))
    oc.append(K[:, :, :64], V[:, :, :64], False, calibrate=True)
    gc.append(H.dev(K[:, :, :64], False), H.dev(V[:, :, :64], False), calibrate=True)
    for t, f in zip(range(64, 70), (1.5, 3.0, 7.0, 20.0, 50.0, -50.0)):
        kk = np.ascontiguousarray(K[:, :, t:t + 1] * np.float32(f))
        vv = np.ascontiguousarray(V[:, :, t:t + 1] * np.float32(f))
        oc.append(kk, vv, False)
        gc.append(H.dev(kk, False), H.dev(vv, False))
    torch.cuda.synchronize()
    H.compare_dense(oc, gc, "saturated tokens")
    assert gc.status()[1] > 0
    H.decode_both(oc, gc, synth.queries(w, 0, 0, B), False, "decode over saturated codes")


# ------------------------------------------------------------------ INT4 symmetric per group
# keys: every MMA sums one 32-channel group and takes its (token, group) scale afterwards;
# values: one scaled P' per group; ragged tails, GQA group sizes, both input types, paged.
@pytest.mark.parametrize("prefill", [1, 100, 128, 300, 9600])
def test_int4_group_dense(prefill):
    H.dense_case(B=2, Hq=16, Hkv=2, ks=S.INT4_SYM_PER_GROUP, vs=S.INT4_SYM_PER_GROUP, prefill=prefill, steps=2,
                 outlier=100.0)


@pytest.mark.parametrize("G", [1, 4, 8, 16])
def test_int4_group_gqa_sizes(G):
    H.dense_case(B=2, Hq=2 * G, Hkv=2, ks=S.INT4_SYM_PER_GROUP, vs=S.INT4_SYM_PER_GROUP, prefill=200, steps=1)


def test_int4_group_fp32_inputs_and_queries():
    H.dense_case(B=1, Hq=4, Hkv=1, ks=S.INT4_SYM_PER_GROUP, vs=S.INT4_SYM_PER_GROUP, prefill=257, steps=2,
                 bf16=False, rope=0.0)
    H.dense_case(B=2, Hq=8, Hkv=2, ks=S.INT4_SYM_PER_GROUP, vs=S.INT4_SYM_PER_GROUP, prefill=130, steps=1,
                 bf16=True, q_bf16=False)


@pytest.mark.parametrize("group", [64, 128])
def test_int4_larger_groups(group):
    # groups of 64 and 128 channels (128: one scale per token): dense with ragged tails, paged,
    # rotated, and dequantize
    H.dense_case(B=2, Hq=16, Hkv=2, ks=S.INT4_SYM_PER_GROUP, vs=S.INT4_SYM_PER_GROUP, prefill=300, steps=2,
                 outlier=100.0, group=group)
    oc, gc, _ = H.dense_case(B=2, Hq=8, Hkv=2, ks=S.INT4_SYM_PER_GROUP, vs=S.INT4_SYM_PER_GROUP, prefill=9600,
                             steps=1, group=group, rotate=True)
    for which in (0, 1):
        got = gc.dequantize(which, 9601).cpu().numpy()
        assert np.array_equal(got.view(np.uint32), oc.dequantize(which, 9601).view(np.uint32))
    B, Hq, Hkv, sch = 4, 16, 4, S.INT4_SYM_PER_GROUP
    w, oc, gc, K, V, lens, calib, nl = H.paged_case(B, Hq, Hkv, sch, sch, lens=[37, 100, 5, 64], page_size=32,
                                                    steps=0, group=group)
    oc.append(K, V, True, new_lens=lens)
    gc.append(H.dev(K, True), H.dev(V, True), new_lens=nl)
    torch.cuda.synchronize()
    H.compare_paged(oc, gc, f"paged, groups of {group}")
    H.decode_both(oc, gc, synth.queries(w, 0, 0, B), True, f"paged decode, groups of {group}")
    assert gc.status()[0] == 0


@pytest.mark.parametrize("ps", [16, 32, 64])
def test_int4_group_paged(ps):
    B, Hq, Hkv, sch = 4, 16, 4, S.INT4_SYM_PER_GROUP
    w, oc, gc, K, V, lens, calib, nl = H.paged_case(B, Hq, Hkv, sch, sch, lens=[37, 100, 5, 64], page_size=ps,
                                                    steps=2)
    oc.append(K, V, True, new_lens=lens)
    gc.append(H.dev(K, True), H.dev(V, True), new_lens=nl)
    torch.cuda.synchronize()
    H.compare_paged(oc, gc, "int4 paged prefill")
    H.decode_both(oc, gc, synth.queries(w, 0, 0, B), True, "int4 paged decode 0")
    for s in range(2):
        kk = np.stack([synth.keys(w, b, b + 1, 0, Hkv, int(lens[b]) + s, int(lens[b]) + s + 1)[0] for b in range(B)])
        vv = np.stack([synth.values(w, b, b + 1, 0, Hkv, int(lens[b]) + s, int(lens[b]) + s + 1)[0] for b in range(B)])
        oc.append(kk, vv, True)
        gc.append(H.dev(kk, True), H.dev(vv, True))
        torch.cuda.synchronize()
        H.compare_paged(oc, gc, f"int4 paged step {s}")
        H.decode_both(oc, gc, synth.queries(w, s + 1, 0, B), True, f"int4 paged decode {s + 1}")
    assert gc.status()[0] == 0


# ------------------------------------------------------------------ Walsh-Hadamard rotation
# K/V rows rotated before quantization (codes and scales bit for bit), the query rotated and
# the output rotated back in decode, dequantized rows rotated back.
@pytest.mark.parametrize("ks,vs", [
    (S.INT4_SYM_PER_GROUP, S.INT4_SYM_PER_GROUP), (S.INT8_SYM_PER_TOKEN, S.INT8_SYM_PER_TOKEN),
    (S.FP8_E4M3_PER_TENSOR, S.FP8_E4M3_PER_TENSOR), (S.INT8_SYM_PER_CHANNEL, S.UINT8_ASYM_PER_CHANNEL),
])
def test_rotation_dense(ks, vs):
    H.dense_case(B=2, Hq=16, Hkv=2, ks=ks, vs=vs, prefill=300, steps=2, outlier=100.0, rotate=True)


def test_rotation_bulk_fp32_and_gqa():
    H.dense_case(B=4, Hq=8, Hkv=2, ks=S.INT4_SYM_PER_GROUP, vs=S.INT4_SYM_PER_GROUP, prefill=9600, steps=1,
                 rotate=True)
    H.dense_case(B=1, Hq=4, Hkv=1, ks=S.INT8_SYM_PER_TOKEN, vs=S.INT8_SYM_PER_TOKEN, prefill=257, steps=1,
                 bf16=False, rope=0.0, rotate=True)
    H.dense_case(B=2, Hq=32, Hkv=2, ks=S.INT4_SYM_PER_GROUP, vs=S.INT4_SYM_PER_GROUP, prefill=130, steps=1,
                 rotate=True)


def test_rotation_paged_and_dequantize():
    B, Hq, Hkv, sch = 4, 16, 4, S.INT4_SYM_PER_GROUP
    w, oc, gc, K, V, lens, calib, nl = H.paged_case(B, Hq, Hkv, sch, sch, lens=[37, 100, 5, 64], page_size=16,
                                                    steps=0, rotate=True)
    oc.append(K, V, True, new_lens=lens)
    gc.append(H.dev(K, True), H.dev(V, True), new_lens=nl)
    torch.cuda.synchronize()
    H.compare_paged(oc, gc, "rotated paged prefill")
    H.decode_both(oc, gc, synth.queries(w, 0, 0, B), True, "rotated paged decode")
    for which in (0, 1):
        got = gc.dequantize(which, 101).cpu().numpy()
        ref = oc.dequantize(which, 101)
        assert np.array_equal(got.view(np.uint32), ref.view(np.uint32)), f"rotated dequantize side {which}"


# ------------------------------------------------------------------ rescaling append
# Scales merged with each block's (they only grow) and the cached codes whose scale changed
# requantized, bit for bit against the oracle; blocks inside the range, a grown single
# token, a grown bulk block; dense and paged.
RESCALE_PAIRS = [
    (S.FP8_E4M3_PER_TENSOR, S.FP8_E4M3_PER_TENSOR), (S.FP8_E5M2_PER_TENSOR, S.FP8_E5M2_PER_TENSOR),
    (S.INT8_SYM_PER_TENSOR, S.UINT8_ASYM_PER_CHANNEL), (S.INT8_SYM_PER_CHANNEL, S.UINT8_ASYM_PER_CHANNEL),
    (S.INT8_SYM_PER_TENSOR, S.INT8_SYM_PER_TOKEN),
]
RESCALE_SPANS = [(300, 340, 0.5), (340, 341, 3.0), (341, 345, 1.0), (345, 420, -1.75)]


def _f32(a, bf16):
    return synth.bf16_bits_to_f32(a) if bf16 else a


@pytest.mark.parametrize("ks,vs", RESCALE_PAIRS)
def test_rescale_dense(ks, vs):
    B, Hq, Hkv = 2, 8, 2
    w = H.workload(B, Hq, Hkv, ks, vs, bf16=False)
    K = synth.keys(w, 0, B, 0, Hkv, 0, 420)
    V = synth.values(w, 0, B, 0, Hkv, 0, 420)
    oc = H.OracleCache(B, Hq, Hkv, 128, ks, vs, cap=512)
    gc = H.kvq().QuantizedKVCache(H.kvq().CacheSpec(B, Hq, Hkv, ks, vs, capacity=512))
    # the first block rescales a fresh cache (zero scales): the same as a calibration
    oc.append(K[:, :, :300], V[:, :, :300], False, rescale=True)
    gc.append(H.dev(K[:, :, :300], False), H.dev(V[:, :, :300], False), rescale=True)
    torch.cuda.synchronize()
    H.compare_dense(oc, gc, "rescaling prefill")
    for a, b, f in RESCALE_SPANS:
        kk = np.ascontiguousarray(K[:, :, a:b] * np.float32(f))
        vv = np.ascontiguousarray(V[:, :, a:b] * np.float32(-f))
        oc.append(kk, vv, False, rescale=True)
        gc.append(H.dev(kk, False), H.dev(vv, False), rescale=True)
        torch.cuda.synchronize()
        H.compare_dense(oc, gc, f"rescale at {a}")
        H.decode_both(oc, gc, synth.queries(w, a, 0, B), False, f"decode after rescale at {a}")
    assert gc.status()[0] == 0


def test_rescale_paged():
    B, Hq, Hkv, ks, vs = 4, 16, 4, S.INT8_SYM_PER_CHANNEL, S.UINT8_ASYM_PER_CHANNEL
    w, oc, gc, K, V, lens, calib, nl = H.paged_case(B, Hq, Hkv, ks, vs, lens=[37, 100, 5, 64], page_size=16,
                                                    steps=8)
    oc.append(K, V, True, calibrate=True, new_lens=lens)
    gc.append(H.dev(K, True), H.dev(V, True), new_lens=nl, calibrate=True)
    for s, f in enumerate((0.25, 4.0, 1.0, -3.0)):
        kk = np.stack([_f32(synth.keys(w, b, b + 1, 0, Hkv, int(lens[b]) + s, int(lens[b]) + s + 1)[0], True)
                       for b in range(B)]) * np.float32(f)
        vv = np.stack([_f32(synth.values(w, b, b + 1, 0, Hkv, int(lens[b]) + s, int(lens[b]) + s + 1)[0], True)
                       for b in range(B)]) * np.float32(-f)
        kk, vv = np.ascontiguousarray(kk, np.float32), np.ascontiguousarray(vv, np.float32)
        oc.append(kk, vv, False, rescale=True)
        gc.append(H.dev(kk, False), H.dev(vv, False), rescale=True)
        torch.cuda.synchronize()
        H.compare_paged(oc, gc, f"paged rescale {s}")
        H.decode_both(oc, gc, synth.queries(w, s, 0, B), True, f"paged decode after rescale {s}")
    assert gc.status()[0] == 0


def test_rescale_schedule_every_1024_tokens():
    # a cache built token by token with rescale_every=64 (the policy's period, shortened)
    B, Hq, Hkv, ks, vs = 1, 8, 2, S.INT8_SYM_PER_TENSOR, S.INT8_SYM_PER_TENSOR
    w = H.workload(B, Hq, Hkv, ks, vs, bf16=False)
    K = synth.keys(w, 0, B, 0, Hkv, 0, 200)
    V = synth.values(w, 0, B, 0, Hkv, 0, 200)
    oc = H.OracleCache(B, Hq, Hkv, 128, ks, vs, cap=256)
    gc = H.kvq().QuantizedKVCache(H.kvq().CacheSpec(B, Hq, Hkv, ks, vs, capacity=256), rescale_every=64)
    oc.append(K[:, :, :8], V[:, :, :8], False, calibrate=True)
    gc.append(H.dev(K[:, :, :8], False), H.dev(V[:, :, :8], False), calibrate=True)
    growth = np.float32(1.0)
    for t in range(8, 200):
        growth *= np.float32(1.01)
        kk = np.ascontiguousarray(K[:, :, t:t + 1] * growth)
        vv = np.ascontiguousarray(V[:, :, t:t + 1] * growth)
        oc.append(kk, vv, False, rescale=(t - 8 + 1) % 64 == 0)
        gc.append(H.dev(kk, False), H.dev(vv, False))
    torch.cuda.synchronize()
    H.compare_dense(oc, gc, "scheduled rescales")
    H.decode_both(oc, gc, synth.queries(w, 0, 0, B), False, "decode after scheduled rescales")


# ------------------------------------------------------------------ dequantize
@pytest.mark.parametrize("ks,vs", [(S.FP8_E4M3_PER_TENSOR, S.FP8_E4M3_PER_TENSOR), (S.KIVI_INT2, S.KIVI_INT2),
                                   (S.KIVI_INT4_F16, S.KIVI_INT4_F16), (S.KIVI_INT2_F16, S.KIVI_INT2_F16),
                                   (S.INT8_SYM_PER_TENSOR, S.UINT8_ASYM_PER_CHANNEL),
                                   (S.FP8_E5M2_PER_TENSOR, S.FP8_E5M2_PER_TENSOR),
                                   (S.INT4_SYM_PER_GROUP, S.INT4_SYM_PER_GROUP)])
def test_dequantize_matches_oracle(ks, vs):
    oc, gc, _ = H.dense_case(B=2, Hq=8, Hkv=2, ks=ks, vs=vs, prefill=200, steps=1, cap=384)
    T = oc.tokens()
    for which in (0, 1):
        got = gc.dequantize(which, T + 3).cpu().numpy()
        ref = oc.dequantize(which, T + 3)
        assert np.array_equal(got.view(np.uint32), ref.view(np.uint32)), f"dequantize side {which}"

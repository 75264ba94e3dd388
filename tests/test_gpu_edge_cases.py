"""GPU parity on the method's edge cases: planted inputs that take the kernels' special branches.

The pages are silent on a zero range (their cache code divides by zero) and on the sign of
zero; the readings taken are: a zero range gives scale 0 and code 0 (dequantized as 0, or as
the minimum for KIVI), E4M3 / E5M2 keep the sign of a zero quotient, KIVI stores +-0 extremes as
+0 ("How KV cache quantization reduces GPU memory", n4n.ai, Step 3; "KV Cache Quantization",
infra.bea.ai, §3). Scales outside 2^-60 .. 2^60 and quotients that may overflow the exact
quotient's range take element-by-element IEEE division in the kernels. Every case below plants
inputs that reach those branches - all-zero rows, +-0 rows, subnormal fp32 (or bf16) values,
rows scaled by 1e-25, whole blocks scaled by 1e-25 or 1e25 (scales leave 2^+-60), constant KIVI
key columns and value groups - and checks codes, scales, zero points and minima bit for bit
against the oracle, dense and paged, then a decode within 2e-4 * max|ref| of the fp64 oracle.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import OracleCache
from tests import harness as H

S = synth
gpu = pytest.mark.gpu

KINDS = ["mixed", "zeros", "tiny", "huge"]


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns, round to nearest even (finite inputs)."""
    u = np.ascontiguousarray(x, np.float32).view(np.uint32).astype(np.uint64)
    return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)


def planted(B, Hkv, T, kind, seed, bf16, by_group=False):
    """Inputs [B, Hkv, T, 128] (float32, or bf16 bits) of one edge-case kind.

    mixed: token classes cycle over normal rows, all-zero rows, +-0 rows, rows whose even
    channels are subnormal, wholly subnormal rows, rows scaled by 1e-25, and constant rows
    (every token of the class equal; for values, each 32-channel group one value). The class
    changes per token, or per 32-token group when by_group (KIVI key groups then see one class).
    zeros / tiny / huge: the whole block zero, or N(0, 1) scaled by 1e-25 / 1e25."""
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((B, Hkv, T, 128)).astype(np.float32)
    if kind == "zeros":
        X[...] = 0.0
    elif kind == "tiny":
        X *= np.float32(1e-25)
    elif kind == "huge":
        X *= np.float32(1e25)
    else:
        cls = (np.arange(T) // 32 if by_group else np.arange(T)) % 8
        # subnormal magnitudes: m * 2^-149 in fp32, m * 2^-133 in bf16 (both exact)
        if bf16:
            sub = rng.integers(1, 128, size=X.shape).astype(np.float32) * np.float32(2.0 ** -133)
        else:
            sub = rng.integers(1, 1 << 23, size=X.shape).astype(np.float32) * np.float32(2.0 ** -149)
        sub *= np.where(rng.random(X.shape) < 0.5, np.float32(-1), np.float32(1))
        zero_pm = np.where(rng.random(X.shape) < 0.5, np.float32(-0.0), np.float32(0.0))
        for t in range(T):
            c = cls[t]
            if c == 1:
                X[:, :, t] = 0.0
            elif c == 2:
                X[:, :, t] = zero_pm[:, :, t]
            elif c == 3:
                X[:, :, t, ::2] = sub[:, :, t, ::2]
            elif c == 4:
                X[:, :, t] = sub[:, :, t]
            elif c == 5:
                X[:, :, t] *= np.float32(1e-25)
            elif c == 6:
                first = t - (t % 32 if by_group else 0)
                X[:, :, t] = X[:, :, first]
                X[:, :, t] = np.repeat(X[:, :, t, ::32], 32, axis=-1)  # constant 32-channel groups
    return bf16_bits(X) if bf16 else X


def run_dense(ks, vs, K, V, bf16, Hq, prefill, steps, group=32, where="", allow_zero=False):
    B, Hkv, T, _ = K.shape
    cap = max(128, (T + 127) // 128 * 128)
    kivi = ks in S.KIVI_SCHEMES
    if kivi:
        cap = max(cap, (T // 128 + 1) * 128)
    oc = OracleCache(B, Hq, Hkv, 128, ks, vs, cap=cap, group=group)
    gc = H.kvq().QuantizedKVCache(H.kvq().CacheSpec(B, Hq, Hkv, ks, vs, capacity=cap, group=group))
    calib = ks in H.CALIBRATED or vs in H.CALIBRATED
    oc.append(K[:, :, :prefill], V[:, :, :prefill], bf16, calibrate=calib)
    gc.append(H.dev(K[:, :, :prefill], bf16), H.dev(V[:, :, :prefill], bf16), calibrate=calib)
    torch.cuda.synchronize()
    H.compare_dense(oc, gc, f"{where} prefill")
    qw = H.workload(B, Hq, Hkv, ks, vs, bf16=bf16, seed=5)
    H.decode_both(oc, gc, synth.queries(qw, 0, 0, B), bf16, f"{where} decode", allow_zero)
    for s in range(steps):
        t = prefill + s
        oc.append(K[:, :, t:t + 1], V[:, :, t:t + 1], bf16)
        gc.append(H.dev(K[:, :, t:t + 1], bf16), H.dev(V[:, :, t:t + 1], bf16))
        torch.cuda.synchronize()
        H.compare_dense(oc, gc, f"{where} step {s}")
        H.decode_both(oc, gc, synth.queries(qw, s + 1, 0, B), bf16, f"{where} decode {s}", allow_zero)
    assert gc.status()[0] == 0
    return oc, gc


DENSE = [
    (S.FP8_E4M3_PER_TENSOR, S.FP8_E4M3_PER_TENSOR, 32), (S.FP8_E5M2_PER_TENSOR, S.FP8_E5M2_PER_TENSOR, 32),
    (S.INT8_SYM_PER_TENSOR, S.INT8_SYM_PER_TENSOR, 32), (S.INT8_SYM_PER_TOKEN, S.INT8_SYM_PER_TOKEN, 32),
    (S.INT8_SYM_PER_CHANNEL, S.UINT8_ASYM_PER_CHANNEL, 32), (S.UINT8_ASYM_PER_CHANNEL, S.UINT8_ASYM_PER_CHANNEL, 32),
    (S.INT4_SYM_PER_GROUP, S.INT4_SYM_PER_GROUP, 32), (S.INT4_SYM_PER_GROUP, S.INT4_SYM_PER_GROUP, 128),
]


@pytest.mark.parametrize("kind", KINDS)
@pytest.mark.parametrize("ks,vs,group", DENSE)
@gpu
def test_dense_edge_cases_fp32_inputs(ks, vs, group, kind):
    B, Hkv, T = 2, 2, 300
    K = planted(B, Hkv, T + 2, kind, 100 + ks, False)
    V = planted(B, Hkv, T + 2, kind, 200 + vs, False)
    run_dense(ks, vs, K, V, False, 16, T, 2, group=group, where=f"{kind} fp32", allow_zero=kind == "zeros")


@pytest.mark.parametrize("ks,vs,group", DENSE)
@gpu
def test_dense_edge_cases_bf16_inputs(ks, vs, group):
    B, Hkv, T = 2, 2, 300
    K = planted(B, Hkv, T + 1, "mixed", 300 + ks, True)
    V = planted(B, Hkv, T + 1, "mixed", 400 + vs, True)
    run_dense(ks, vs, K, V, True, 16, T, 1, group=group, where="mixed bf16")


@gpu
def test_dense_edge_cases_bulk_form():
    # a block past the size where the append switches to its four-rows-per-thread form
    B, Hkv, T = 4, 2, 9600
    for ks, vs in ((S.INT8_SYM_PER_TOKEN, S.UINT8_ASYM_PER_CHANNEL), (S.FP8_E4M3_PER_TENSOR, S.FP8_E4M3_PER_TENSOR),
                   (S.INT4_SYM_PER_GROUP, S.INT4_SYM_PER_GROUP)):
        K = planted(B, Hkv, T, "mixed", 500 + ks, True)
        V = planted(B, Hkv, T, "mixed", 600 + vs, True)
        run_dense(ks, vs, K, V, True, 8, T, 0, where=f"bulk mixed {ks}/{vs}")


@pytest.mark.parametrize("kind", KINDS)
@pytest.mark.parametrize("scheme", [S.KIVI_INT4, S.KIVI_INT2, S.KIVI_INT4_F16, S.KIVI_INT2_F16])
@gpu
def test_kivi_edge_cases(scheme, kind):
    # classes per 32-token group: zero-range key groups (zeros, +-0, constant columns) and
    # value groups (constant 32-channel groups), subnormal and tiny groups, flushed and residual
    B, Hkv, T = 2, 2, 300
    K = planted(B, Hkv, T + 2, kind, 700 + scheme, True, by_group=True)
    V = planted(B, Hkv, T + 2, kind, 800 + scheme, True, by_group=True)
    run_dense(scheme, scheme, K, V, True, 16, T, 2, where=f"kivi {kind}", allow_zero=kind == "zeros")


PAGED = [(S.INT8_SYM_PER_TENSOR, S.UINT8_ASYM_PER_CHANNEL, 16), (S.INT8_SYM_PER_TOKEN, S.INT8_SYM_PER_TOKEN, 32),
         (S.FP8_E4M3_PER_TENSOR, S.FP8_E4M3_PER_TENSOR, 16), (S.INT4_SYM_PER_GROUP, S.INT4_SYM_PER_GROUP, 64)]


@pytest.mark.parametrize("kind", KINDS)
@pytest.mark.parametrize("ks,vs,ps", PAGED)
@gpu
def test_paged_edge_cases(ks, vs, ps, kind):
    B, Hq, Hkv = 4, 16, 4
    w, oc, gc, _, _, lens, calib, nl = H.paged_case(B, Hq, Hkv, ks, vs, lens=[37, 200, 5, 64], page_size=ps,
                                                    steps=2)
    n_max = int(lens.max())
    K = planted(B, Hkv, n_max + 2, kind, 900 + ks, True)
    V = planted(B, Hkv, n_max + 2, kind, 950 + vs, True)
    Kp, Vp = K[:, :, :n_max].copy(), V[:, :, :n_max].copy()
    oc.append(Kp, Vp, True, calibrate=calib, new_lens=lens)
    gc.append(H.dev(Kp, True), H.dev(Vp, True), new_lens=nl, calibrate=calib)
    torch.cuda.synchronize()
    H.compare_paged(oc, gc, f"paged {kind} prefill")
    H.decode_both(oc, gc, synth.queries(w, 0, 0, B), True, f"paged {kind} decode", kind == "zeros")
    for s in range(2):
        kk = np.stack([K[b, :, int(lens[b]) + s:int(lens[b]) + s + 1] for b in range(B)])
        vv = np.stack([V[b, :, int(lens[b]) + s:int(lens[b]) + s + 1] for b in range(B)])
        oc.append(kk, vv, True)
        gc.append(H.dev(kk, True), H.dev(vv, True))
        torch.cuda.synchronize()
        H.compare_paged(oc, gc, f"paged {kind} step {s}")
        H.decode_both(oc, gc, synth.queries(w, s + 1, 0, B), True, f"paged {kind} decode {s}", kind == "zeros")
    assert gc.status()[0] == 0


def test_planted_inputs_reach_the_branches():
    # the planted classes are what they claim (host-side check of the generator)
    X = planted(1, 1, 16, "mixed", 1, False)
    assert np.all(X[0, 0, 1] == 0) and np.all(X[0, 0, 9] == 0)
    assert np.any(np.signbit(X[0, 0, 2])) and np.all(X[0, 0, 2] == 0)
    sub = X[0, 0, 4]
    assert np.all((np.abs(sub) > 0) & (np.abs(sub) < np.finfo(np.float32).tiny))
    assert np.all(np.abs(X[0, 0, 5]) < 1e-20)
    assert np.all(X[0, 0, 6, :32] == X[0, 0, 6, 0])
    Xb = planted(1, 1, 64, "mixed", 1, True, by_group=True)
    assert np.all(Xb[0, 0, 32:64] == Xb[0, 0, 32])  # a whole 32-token group of zeros
    assert np.all((planted(1, 1, 4, "huge", 1, False) == 0) | (np.abs(planted(1, 1, 4, "huge", 1, False)) > 1e18))

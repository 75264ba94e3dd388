"""Full-size parity at the benchmark workloads' shapes.

The CUDA library builds each workload's cache exactly as the benchmark does (same shapes,
calibration, the streamed tokens, the library's own grid choice) and the oracle builds the
same cache from the same inputs. Codes, scales, zero points, minima and residual tokens of
EVERY (sequence, kv head) pair must match bit for bit; attention rows of sampled pairs (the
oracle's fp64 attention costs seconds per pair at these lengths) must be within 2e-4 * max|ref|.

The paged workload streams all of its 128 steps (one token per sequence appended, then a
decode): attention is compared on steps 0, 1, 63 and 127 for sampled sequences and on every
step for four seeded sequences (drawn among the shortest quarter, so the oracle keeps up), and
every sequence's codes at every position after the last step.
"""
import math

import numpy as np
import pytest
import torch

import synth
from oracle import OracleCache
from tests import harness as H

pytestmark = [pytest.mark.gpu, pytest.mark.slow]
SCALE = 1.0 / math.sqrt(128.0)
CAL = H.CALIBRATED


def _pairs(w, n=6, seed=0):
    rng = np.random.default_rng(seed + w.seed)
    allp = [(b, h) for b in range(w.B) for h in range(w.Hkv)]
    idx = rng.choice(len(allp), size=min(n, len(allp)), replace=False)
    return sorted(set([allp[i] for i in idx] + [allp[0], allp[-1]]))


def _dense_full(name):
    w = synth.workloads()[name]
    kvq = H.kvq()
    total = w.prefill_tokens()
    append = name != "tiny_int8"
    pre = total - 1 if append else total
    cap = (total + 127) // 128 * 128
    K = synth.keys(w, 0, w.B, 0, w.Hkv, 0, total)
    V = synth.values(w, 0, w.B, 0, w.Hkv, 0, total)
    gc = kvq.QuantizedKVCache(kvq.CacheSpec(w.B, w.Hq, w.Hkv, w.k_scheme, w.v_scheme, capacity=cap,
                                            rotate=w.rotate, group=w.group, rope_theta=w.prerope_theta))
    oc = OracleCache(w.B, w.Hq, w.Hkv, 128, w.k_scheme, w.v_scheme, cap=cap, rotate=w.rotate, group=w.group,
                     rope_theta=w.prerope_theta)
    calib = w.k_scheme in CAL or w.v_scheme in CAL
    gc.append(H.dev(K[:, :, :pre], w.bf16), H.dev(V[:, :, :pre], w.bf16), calibrate=calib)
    oc.append(K[:, :, :pre], V[:, :, :pre], w.bf16, calibrate=calib)
    if append:
        gc.append(H.dev(K[:, :, pre:], w.bf16), H.dev(V[:, :, pre:], w.bf16))
        oc.append(K[:, :, pre:], V[:, :, pre:], w.bf16)
    del K, V
    q = synth.queries(w, 0, 0, w.B)
    lse = torch.empty((w.B, w.Hq), dtype=torch.float32, device="cuda")
    out, _ = gc.decode(H.dev(q, w.bf16), SCALE, lse=lse)
    torch.cuda.synchronize()
    assert gc.status()[0] == 0
    H.compare_dense(oc, gc, f"{name}: every pair")
    pairs = _pairs(w)
    ref, ref_lse = oc.decode_pairs(q, w.bf16, SCALE, pairs)
    G = w.G
    got = torch.stack([out[b, h * G:(h + 1) * G] for b, h in pairs])
    got_lse = torch.stack([lse[b, h * G:(h + 1) * G] for b, h in pairs])
    H.attn_check(got, ref, got_lse, ref_lse, where=f"{name} sampled pairs")


def test_tiny_int8_full():
    _dense_full("tiny_int8")


def test_fp8_8b_full():
    _dense_full("fp8_8b")


def test_e5m2_8b_full():
    _dense_full("e5m2_8b")


def test_fp8_8b_prerope_full():
    _dense_full("fp8_8b_prerope")


def test_int4g_70b_full():
    _dense_full("int4g_70b")


def test_int4g_rot_70b_full():
    _dense_full("int4g_rot_70b")


def test_int4g128_70b_full():
    _dense_full("int4g128_70b")


def test_kivi4_70b_full():
    _dense_full("kivi4_70b")


def test_kivi2_131k_full():
    _dense_full("kivi2_131k")


def test_kivi4f16_70b_full():
    _dense_full("kivi4f16_70b")


def test_kivi2f16_131k_full():
    _dense_full("kivi2f16_131k")


def _step_tokens(w, lens, s):
    kk = np.stack([synth.keys(w, b, b + 1, 0, w.Hkv, int(lens[b]) + s, int(lens[b]) + s + 1)[0] for b in range(w.B)])
    vv = np.stack([synth.values(w, b, b + 1, 0, w.Hkv, int(lens[b]) + s, int(lens[b]) + s + 1)[0]
                   for b in range(w.B)])
    return kk, vv


def test_paged_int8_full():
    """64 sequences of 1k..32k tokens in 16-token pages; a calibrating prefill over all of them,
    then the workload's 128 streamed steps."""
    w = synth.workloads()["paged_int8"]
    kvq = H.kvq()
    steps = w.steps
    lens = w.prefill_lengths()
    table, pool = w.page_table(max_pages=(int(lens.max()) + steps + 15) // 16 + 1)
    n_max = int(lens.max())
    K = np.zeros((w.B, w.Hkv, n_max, 128), np.uint16)
    V = np.zeros_like(K)
    for b in range(w.B):
        L = int(lens[b])
        K[b:b + 1, :, :L] = synth.keys(w, b, b + 1, 0, w.Hkv, 0, L)
        V[b:b + 1, :, :L] = synth.values(w, b, b + 1, 0, w.Hkv, 0, L)
    spec = kvq.CacheSpec(w.B, w.Hq, w.Hkv, w.k_scheme, w.v_scheme, paged=True, page_size=16,
                         max_pages=table.shape[1], num_pages=pool)
    gc = kvq.QuantizedKVCache(spec, page_table=torch.from_numpy(table))
    oc = OracleCache(w.B, w.Hq, w.Hkv, 128, w.k_scheme, w.v_scheme, paged=True, page_size=16,
                     max_pages=table.shape[1], num_pages=pool, page_table=table)
    gc.append(H.dev(K, True), H.dev(V, True), new_lens=torch.from_numpy(lens).cuda(), calibrate=True)
    oc.append(K, V, True, calibrate=True, new_lens=lens)
    del K, V
    rng = np.random.default_rng(5)
    sampled = sorted(set(rng.choice(w.B, 5, replace=False).tolist() + [int(np.argmax(lens))]))
    shorter = np.argsort(lens)[: w.B // 4]
    every = sorted(rng.choice(shorter, 4, replace=False).tolist())
    checkpoints = {0, 1, 63, steps - 1}
    G = w.G
    for s in range(steps):
        kk, vv = _step_tokens(w, lens, s)
        gc.append(H.dev(kk, True), H.dev(vv, True))
        oc.append(kk, vv, True)
        q = synth.queries(w, s, 0, w.B)
        lse = torch.empty((w.B, w.Hq), dtype=torch.float32, device="cuda")
        out, _ = gc.decode(H.dev(q, True), SCALE, lse=lse)
        seqs = sorted(set(every) | (set(sampled) if s in checkpoints else set()))
        pairs = [(b, h) for b in seqs for h in range(w.Hkv)]
        ref, ref_lse = oc.decode_pairs(q, True, SCALE, pairs)
        torch.cuda.synchronize()
        got = torch.stack([out[b, h * G:(h + 1) * G] for b, h in pairs])
        got_lse = torch.stack([lse[b, h * G:(h + 1) * G] for b, h in pairs])
        H.attn_check(got, ref, got_lse, ref_lse, where=f"paged_int8 step {s}, sequences {seqs}")
    assert gc.status()[0] == 0
    assert np.array_equal(H.np_of(gc["seq_lens"]), lens + steps)
    # every sequence's codes at every position, and the batch-wide scales and zero points
    for side in ("k", "v"):
        pool_g, pool_o = H.np_of(gc[side + "_codes"]), oc[side + "_codes"]
        for b in range(w.B):
            L = int(lens[b]) + steps
            pages = table[b, :(L + 15) // 16]
            g = pool_g[pages].transpose(0, 2, 1, 3).reshape(-1, w.Hkv, 128)[:L]
            o = pool_o[pages].transpose(0, 2, 1, 3).reshape(-1, w.Hkv, 128)[:L]
            assert np.array_equal(g, o), f"{side} codes of sequence {b}"
        assert np.array_equal(H.np_of(gc[side + "_scale"]).reshape(-1)[:oc[side + "_scale"].size].view(np.uint32),
                              oc[side + "_scale"].reshape(-1).view(np.uint32)), side
    assert np.array_equal(H.np_of(gc["v_zp"]), oc["v_zp"])

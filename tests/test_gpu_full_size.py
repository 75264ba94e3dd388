"""Full-size parity at the five workload shapes.

The CUDA library builds each workload's cache exactly as the benchmark does (same shapes,
calibration, one streamed token, the library's own grid choice) and the oracle recomputes
sampled (sequence, kv_head) pairs one by one: their codes, scales, minima and residual
tokens must match bit for bit and their attention rows must be within 2e-4 * max|ref|.
Scales that span the whole batch (per-tensor, per-channel) come from an oracle calibration
over the full prefill block.
"""
import math

import numpy as np
import pytest
import torch

import oracle
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
    return [allp[i] for i in sorted(idx)] + [allp[0], allp[-1]]


def _copy_scales(dst: OracleCache, src: OracleCache, h: int):
    """Give a one-head oracle cache the batch-wide scales an oracle calibration computed:
    the per-tensor scale, or kv head h's row of a per-channel scale (and zero point)."""
    for side in ("k", "v"):
        s = src[side + "_scale"]
        if s.size == 1:
            dst[side + "_scale"][...] = s
        elif s.ndim == 2 and s.shape[1] == 128:  # [Hkv, D]
            dst[side + "_scale"][...] = s[h:h + 1]
            if src[side + "_zp"] is not None:
                dst[side + "_zp"][...] = src[side + "_zp"][h:h + 1]


def _check_pair_dense(w, gc, oc, b, h, out_gpu, q):
    """Bit-exact slice comparison and attention for one (b, h) pair."""
    L = oc.length
    G = w.G
    for side in ("k", "v"):
        got = H.np_of(gc[side + "_codes"][b, h, :L])
        assert np.array_equal(got, oc[side + "_codes"][0, 0, :L]), f"pair {(b, h)}: {side} codes"
        sch = w.k_scheme if side == "k" else w.v_scheme
        if sch in (synth.INT8_SYM_PER_TOKEN, synth.INT4_SYM_PER_GROUP):
            assert np.array_equal(H.np_of(gc[side + "_scale"][b, h, :L]).view(np.uint32),
                                  oc[side + "_scale"][0, 0, :L].view(np.uint32))
        if sch in (synth.KIVI_INT4, synth.KIVI_INT2):
            rows = L // 32 if side == "k" else L
            for name in ("_scale", "_zero"):
                assert np.array_equal(H.np_of(gc[side + name][b, h, :rows]).view(np.uint32),
                                      oc[side + name][0, 0, :rows].view(np.uint32)), f"pair {(b, h)} {side}{name}"
            r = oc.residual
            assert np.array_equal(H.np_of(gc[side + "_res"][b, h, :r]).view(np.uint16), oc[side + "_res"][0, 0, :r])
    ref, ref_lse = oc.decode(q[b:b + 1, h * G:(h + 1) * G], w.bf16, SCALE)
    return ref[0]


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
                                            rotate=w.rotate, group=w.group))
    calib = w.k_scheme in CAL or w.v_scheme in CAL
    gc.append(H.dev(K[:, :, :pre], w.bf16), H.dev(V[:, :, :pre], w.bf16), calibrate=calib)
    if append:
        gc.append(H.dev(K[:, :, pre:], w.bf16), H.dev(V[:, :, pre:], w.bf16))
    q = synth.queries(w, 0, 0, w.B)
    out, _ = gc.decode(H.dev(q, w.bf16), SCALE)
    torch.cuda.synchronize()
    out = out.cpu().numpy()
    assert gc.status()[0] == 0
    full_cal = None
    if calib:
        full_cal = OracleCache(w.B, w.Hq, w.Hkv, 128, w.k_scheme, w.v_scheme, cap=128, rotate=w.rotate)
        full_cal.calibrate(K[:, :, :pre], V[:, :, :pre], w.bf16)
        for side in ("k", "v"):
            assert np.array_equal(H.np_of(gc[side + "_scale"]).reshape(-1)[:full_cal[side + "_scale"].size]
                                  .view(np.uint32), full_cal[side + "_scale"].reshape(-1).view(np.uint32))
    refs, gots = [], []
    for b, h in _pairs(w):
        oc = OracleCache(1, w.G, 1, 128, w.k_scheme, w.v_scheme, cap=cap, rotate=w.rotate, group=w.group)
        if full_cal is not None:
            _copy_scales(oc, full_cal, h)
        oc.append(K[b:b + 1, h:h + 1, :pre], V[b:b + 1, h:h + 1, :pre], w.bf16)
        if append:
            oc.append(K[b:b + 1, h:h + 1, pre:], V[b:b + 1, h:h + 1, pre:], w.bf16)
        assert gc.num_quantized == oc.length and gc.num_residual == oc.residual
        refs.append(_check_pair_dense(w, gc, oc, b, h, None, q))
        gots.append(out[b, h * w.G:(h + 1) * w.G])
    H.attn_check(torch.from_numpy(np.stack(gots)), np.stack(refs), where=f"{name} sampled pairs")


def test_tiny_int8_full():
    _dense_full("tiny_int8")


def test_fp8_8b_full():
    _dense_full("fp8_8b")


def test_e5m2_8b_full():
    _dense_full("e5m2_8b")


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


def test_paged_int8_full():
    """64 sequences of 1k..32k tokens in 16-token pages; calibrating prefill over all of
    them, then 3 streamed tokens per sequence; sampled sequences recomputed by the oracle."""
    w = synth.workloads()["paged_int8"]
    kvq = H.kvq()
    steps = 3
    lens = w.prefill_lengths()
    table, pool = w.page_table(max_pages=(int(lens.max()) + w.steps + 15) // 16 + 1)
    # the workload's table covers prefill + its 128 streamed steps
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
    nl = torch.from_numpy(lens).cuda()
    gc.append(H.dev(K, True), H.dev(V, True), new_lens=nl, calibrate=True)
    toks = []
    for s in range(steps):
        kk = np.stack([synth.keys(w, b, b + 1, 0, w.Hkv, int(lens[b]) + s, int(lens[b]) + s + 1)[0] for b in range(w.B)])
        vv = np.stack([synth.values(w, b, b + 1, 0, w.Hkv, int(lens[b]) + s, int(lens[b]) + s + 1)[0] for b in range(w.B)])
        toks.append((kk, vv))
        gc.append(H.dev(kk, True), H.dev(vv, True))
    q = synth.queries(w, steps, 0, w.B)
    out, _ = gc.decode(H.dev(q, True), SCALE)
    torch.cuda.synchronize()
    out = out.cpu().numpy()
    assert gc.status()[0] == 0
    assert np.array_equal(H.np_of(gc["seq_lens"]), lens + steps)
    cal = OracleCache(w.B, w.Hq, w.Hkv, 128, w.k_scheme, w.v_scheme, paged=True, page_size=16,
                      max_pages=table.shape[1], num_pages=1, page_table=table)
    cal.calibrate(K, V, True, new_lens=lens)
    del K, V
    for side in ("k", "v"):
        assert np.array_equal(H.np_of(gc[side + "_scale"]).reshape(-1)[:cal[side + "_scale"].size].view(np.uint32),
                              cal[side + "_scale"].reshape(-1).view(np.uint32)), side
    assert np.array_equal(H.np_of(gc["v_zp"]), cal["v_zp"])
    refs, gots = [], []
    seqs = sorted(set(np.random.default_rng(5).choice(w.B, 5, replace=False).tolist() + [int(np.argmax(lens))]))
    pool_k, pool_v = H.np_of(gc["k_codes"]), H.np_of(gc["v_codes"])
    for b in seqs:
        L = int(lens[b])
        npg = (L + steps + 15) // 16
        own = np.arange(npg, dtype=np.int32)[None]  # the oracle keeps this sequence in a compact pool
        oc = OracleCache(1, w.Hq, w.Hkv, 128, w.k_scheme, w.v_scheme, paged=True, page_size=16,
                         max_pages=npg, num_pages=npg, page_table=own)
        for side in ("k", "v"):
            oc[side + "_scale"][...] = cal[side + "_scale"]
        oc["v_zp"][...] = cal["v_zp"]
        oc.append(synth.keys(w, b, b + 1, 0, w.Hkv, 0, L), synth.values(w, b, b + 1, 0, w.Hkv, 0, L), True)
        for kk, vv in toks:
            oc.append(kk[b:b + 1], vv[b:b + 1], True)
        for t in range(L + steps):
            page, slot = table[b, t // 16], t % 16
            assert np.array_equal(pool_k[page, :, slot], oc["k_codes"][t // 16, :, slot]), (b, t)
            assert np.array_equal(pool_v[page, :, slot], oc["v_codes"][t // 16, :, slot]), (b, t)
        ref, _ = oc.decode(q[b:b + 1], True, SCALE)
        refs.append(ref[0])
        gots.append(out[b])
    H.attn_check(torch.from_numpy(np.stack(gots)), np.stack(refs), where="paged_int8 sampled sequences")

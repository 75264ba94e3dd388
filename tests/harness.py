"""Shared GPU-vs-oracle harness for the parity tests (test infrastructure).

The same seeded synthetic inputs go to the CUDA library (through its C ABI) and to the CPU
oracle; codes, scales and zero points are compared bit for bit, attention outputs against
the fp64 oracle with max|err| <= 2e-4 * max|ref| over the whole output.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle
import synth
from oracle import OracleCache

ATTN_RTOL = 2e-4          # max|out - ref| <= ATTN_RTOL * max|ref|
CALIBRATED = (synth.FP8_E4M3_PER_TENSOR, synth.FP8_E5M2_PER_TENSOR, synth.INT8_SYM_PER_TENSOR, synth.INT8_SYM_PER_CHANNEL,
              synth.UINT8_ASYM_PER_CHANNEL)
SCALE = np.float32(1.0 / math.sqrt(128.0))


def kvq():
    from decode_attention_quantize_b200 import kvq as mod
    return mod


def dev(a: np.ndarray, bf16: bool) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a)).cuda()
    return t.view(torch.bfloat16) if bf16 else t


def workload(B, Hq, Hkv, ks, vs, bf16=True, seed=11, outlier=20.0, rope=500000.0):
    return synth.Workload(name="case", seed=seed, B=B, Hq=Hq, Hkv=Hkv, D=128, k_scheme=ks, v_scheme=vs,
                          bf16=bf16, outlier_scale=outlier, rope_theta=rope)


ERRORS = []  # (where, relative error) of every attention comparison, for the report


def attn_check(out_gpu: torch.Tensor, ref: np.ndarray, lse_gpu=None, lse_ref=None, where="", allow_zero=False):
    got = out_gpu.detach().cpu().numpy().astype(np.float64)
    err = np.abs(got - ref).max()
    scale = np.abs(ref).max()
    assert np.isfinite(got).all(), f"{where}: non-finite output"
    assert allow_zero or scale > 0, f"{where}: reference is all zero"
    assert err <= ATTN_RTOL * scale, f"{where}: max err {err:.3e} > {ATTN_RTOL} * {scale:.3e}"
    if lse_gpu is not None:
        lg = lse_gpu.detach().cpu().numpy().astype(np.float64)
        fin = np.isfinite(lse_ref)
        assert np.array_equal(np.isfinite(lg), fin), f"{where}: lse finiteness differs"
        if fin.any():
            lerr = np.abs(lg[fin] - lse_ref[fin]).max()
            assert lerr <= 1e-4 * max(1.0, np.abs(lse_ref[fin]).max()), f"{where}: lse err {lerr:.3e}"
    rel = err / max(scale, 1e-30)
    ERRORS.append((where, float(rel)))
    return rel


def np_of(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        t = t.view(torch.uint16) if hasattr(torch, "uint16") else t.view(torch.int16)
    return t.numpy()


def compare_dense(oc: OracleCache, gc, where=""):
    """Bit-exact comparison of the valid part of a dense cache."""
    L = oc.length
    assert gc.num_quantized == L, f"{where}: length {gc.num_quantized} != {L}"
    assert gc.num_residual == oc.residual, f"{where}: residual {gc.num_residual} != {oc.residual}"
    for side in ("k", "v"):
        assert np.array_equal(np_of(gc[side + "_codes"])[:, :, :L], oc[side + "_codes"][:, :, :L]), \
            f"{where}: {side} codes differ"
        sch = oc.k_scheme if side == "k" else oc.v_scheme
        s_g, s_o = np_of(gc[side + "_scale"]), oc[side + "_scale"]
        if sch in (synth.FP8_E4M3_PER_TENSOR, synth.FP8_E5M2_PER_TENSOR, synth.INT8_SYM_PER_TENSOR):
            assert s_g.view(np.uint32)[0] == s_o.view(np.uint32)[0], f"{where}: {side} scale differs"
        elif sch in (synth.INT8_SYM_PER_TOKEN, synth.INT4_SYM_PER_GROUP):
            assert np.array_equal(s_g[:, :, :L].view(np.uint32), s_o[:, :, :L].view(np.uint32)), \
                f"{where}: {side} token scales differ"
        elif sch in (synth.INT8_SYM_PER_CHANNEL, synth.UINT8_ASYM_PER_CHANNEL):
            assert np.array_equal(s_g.view(np.uint32), s_o.view(np.uint32)), f"{where}: {side} channel scales"
            if sch == synth.UINT8_ASYM_PER_CHANNEL:
                assert np.array_equal(np_of(gc[side + "_zp"]), oc[side + "_zp"]), f"{where}: {side} zero points"
        else:
            # KIVI: fp32 scale and minimum, or fp16 ones (the oracle holds the stored fp16 values
            # as fp32, exactly)
            rows = L // 32 if side == "k" else L
            z_g = np_of(gc[side + "_zero"])
            s_g, z_g = s_g.astype(np.float32), z_g.astype(np.float32)
            assert np.array_equal(s_g[:, :, :rows].view(np.uint32), s_o[:, :, :rows].view(np.uint32)), \
                f"{where}: {side} KIVI scales differ"
            assert np.array_equal(z_g[:, :, :rows].view(np.uint32), oc[side + "_zero"][:, :, :rows].view(np.uint32)), \
                f"{where}: {side} KIVI minima differ"
    if oc.k_scheme in synth.KIVI_SCHEMES:
        r = oc.residual
        for side in ("k", "v"):
            got = np_of(gc[side + "_res"]).view(np.uint16)[:, :, :r]
            assert np.array_equal(got, oc[side + "_res"][:, :, :r]), f"{where}: {side} residual differs"


def compare_paged(oc: OracleCache, gc, where=""):
    lens = oc["seq_lens"]
    assert np.array_equal(np_of(gc["seq_lens"]), lens), f"{where}: seq_lens differ"
    table = oc["page_table"]
    ps = oc.page_size
    for side in ("k", "v"):
        pool_g, pool_o = np_of(gc[side + "_codes"]), oc[side + "_codes"]
        sch = oc.k_scheme if side == "k" else oc.v_scheme
        for b in range(oc.B):
            for t in range(int(lens[b])):
                page, slot = table[b, t // ps], t % ps
                assert np.array_equal(pool_g[page, :, slot], pool_o[page, :, slot]), \
                    f"{where}: {side} codes differ at seq {b} token {t}"
                if sch in (synth.INT8_SYM_PER_TOKEN, synth.INT4_SYM_PER_GROUP):
                    assert np.array_equal(np_of(gc[side + "_scale"])[page, :, slot].view(np.uint32),
                                          oc[side + "_scale"][page, :, slot].view(np.uint32))
        s_g, s_o = np_of(gc[side + "_scale"]), oc[side + "_scale"]
        if sch in (synth.FP8_E4M3_PER_TENSOR, synth.FP8_E5M2_PER_TENSOR, synth.INT8_SYM_PER_TENSOR):
            assert s_g.view(np.uint32)[0] == s_o.view(np.uint32)[0], f"{where}: {side} scale differs"
        elif sch in (synth.INT8_SYM_PER_CHANNEL, synth.UINT8_ASYM_PER_CHANNEL):
            assert np.array_equal(s_g.view(np.uint32), s_o.view(np.uint32)), f"{where}: {side} channel scales"
            if sch == synth.UINT8_ASYM_PER_CHANNEL:
                assert np.array_equal(np_of(gc[side + "_zp"]), oc[side + "_zp"])


def decode_both(oc: OracleCache, gc, q: np.ndarray, bf16: bool, where="", allow_zero=False):
    qd = dev(q, bf16)
    lse = torch.empty(q.shape[:2], dtype=torch.float32, device="cuda")
    out, _ = gc.decode(qd, float(SCALE), lse=lse)
    ref, ref_lse = oc.decode(q, bf16, float(SCALE))
    torch.cuda.synchronize()
    return attn_check(out, ref, lse, ref_lse, where, allow_zero=allow_zero)


def dense_case(B, Hq, Hkv, ks, vs, prefill, steps=2, cap=None, bf16=True, q_bf16=None, seed=11, outlier=20.0,
               rope=500000.0, chunks=None, rotate=False, group=32, prerope=0.0):
    """Prefill (calibrating when the scheme needs it), then `steps` one-token appends each
    followed by a decode; codes and attention compared after every call. rope: RoPE the input
    generator applies to the keys; prerope > 0: the cache holds keys before RoPE and decode
    applies RoPE with this base (pass rope=0 for such keys)."""
    q_bf16 = bf16 if q_bf16 is None else q_bf16
    w = workload(B, Hq, Hkv, ks, vs, bf16=bf16, seed=seed, outlier=outlier, rope=rope)
    total = prefill + steps
    if cap is None:
        cap = max(128, (total + 127) // 128 * 128)
    K = synth.keys(w, 0, B, 0, Hkv, 0, total)
    V = synth.values(w, 0, B, 0, Hkv, 0, total)
    oc = OracleCache(B, Hq, Hkv, 128, ks, vs, cap=cap, rotate=rotate, group=group, rope_theta=prerope)
    gc = kvq().QuantizedKVCache(kvq().CacheSpec(B, Hq, Hkv, ks, vs, capacity=cap, rotate=rotate, group=group,
                                                rope_theta=prerope))
    calib = ks in CALIBRATED or vs in CALIBRATED
    bounds = [0, prefill] if chunks is None else [0, *chunks, prefill]
    for i, (a, b) in enumerate(zip(bounds, bounds[1:])):
        kk, vv = K[:, :, a:b], V[:, :, a:b]
        oc.append(kk, vv, bf16, calibrate=calib and i == 0)
        gc.append(dev(kk, bf16), dev(vv, bf16), calibrate=calib and i == 0)
    torch.cuda.synchronize()
    compare_dense(oc, gc, "prefill")
    errs = []
    qw = workload(B, Hq, Hkv, ks, vs, bf16=q_bf16, seed=seed)
    errs.append(decode_both(oc, gc, synth.queries(qw, 0, 0, B), q_bf16, "decode after prefill"))
    for s in range(steps):
        kk, vv = K[:, :, prefill + s:prefill + s + 1], V[:, :, prefill + s:prefill + s + 1]
        oc.append(kk, vv, bf16)
        gc.append(dev(kk, bf16), dev(vv, bf16))
        torch.cuda.synchronize()
        compare_dense(oc, gc, f"step {s}")
        errs.append(decode_both(oc, gc, synth.queries(qw, s + 1, 0, B), q_bf16, f"decode step {s}"))
    st = gc.status()
    assert st[0] == 0, f"device status {st}"
    return oc, gc, max(errs)


def paged_case(B, Hq, Hkv, ks, vs, lens, page_size=16, steps=2, seed=21, extra_pages=5, bad_page=None,
               rotate=False, group=32, prerope=0.0):
    w = workload(B, Hq, Hkv, ks, vs, bf16=True, seed=seed, rope=0.0 if prerope else 500000.0)
    lens = np.asarray(lens, np.int32)
    n_max = int(lens.max()) if len(lens) else 0
    need = [(int(L) + steps + page_size - 1) // page_size for L in lens]
    max_pages = max(need) + 1
    num_pages = int(sum(need)) + extra_pages
    perm = synth.permutation(seed, num_pages)
    table = np.full((B, max_pages), -1, np.int32)
    off = 0
    for b, n in enumerate(need):
        table[b, :n] = perm[off:off + n]
        off += n
    if bad_page is not None:
        b, i = bad_page
        table[b, i] = num_pages + 7  # outside the pool: must be flagged, never dereferenced
    K = np.zeros((B, Hkv, max(n_max, 1), 128), np.uint16)
    V = np.zeros_like(K)
    for b in range(B):
        if lens[b]:
            K[b:b + 1, :, :lens[b]] = synth.keys(w, b, b + 1, 0, Hkv, 0, int(lens[b]))
            V[b:b + 1, :, :lens[b]] = synth.values(w, b, b + 1, 0, Hkv, 0, int(lens[b]))
    oc = OracleCache(B, Hq, Hkv, 128, ks, vs, paged=True, page_size=page_size, max_pages=max_pages,
                     num_pages=num_pages, page_table=table if bad_page is None else _clean(table, num_pages),
                     rotate=rotate, group=group, rope_theta=prerope)
    spec = kvq().CacheSpec(B, Hq, Hkv, ks, vs, paged=True, page_size=page_size, max_pages=max_pages,
                           num_pages=num_pages, rotate=rotate, group=group, rope_theta=prerope)
    gc = kvq().QuantizedKVCache(spec, page_table=torch.from_numpy(table))
    calib = ks in CALIBRATED or vs in CALIBRATED
    nl = torch.from_numpy(lens).cuda()
    return w, oc, gc, K, V, lens, calib, nl


def _clean(table, num_pages):
    t = table.copy()
    t[(t < 0) | (t >= num_pages)] = -1
    return t

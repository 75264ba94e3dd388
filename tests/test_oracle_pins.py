"""Pins of the CPU oracle against what the pages and the mathematics fix.

Each test checks the oracle against something other than itself: a worked example the
pages print, a closed form, an invariant, an independent library routine, or brute force.
"""
import decimal
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from oracle import OracleCache

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
F32 = np.float32


def _read_golden(name):
    sections, cur = {}, None
    with open(os.path.join(GOLDEN, name)) as fh:
        for line in fh:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            if line in ("tokens", "codes"):
                cur = sections.setdefault(line, [])
                continue
            cur.append(line.split())
    return sections


def _rne(fr: Fraction) -> int:
    """Round a rational half to even."""
    fl = math.floor(fr)
    rem = fr - fl
    if rem > Fraction(1, 2):
        return fl + 1
    if rem < Fraction(1, 2):
        return fl
    return fl if fl % 2 == 0 else fl + 1


def _sym_exact(xs, absmax):
    s = Fraction(absmax) / 127
    return [max(-127, min(127, _rne(Fraction(x) / s))) for x in xs]


# --------------------------------------------------------------- worked examples
def test_key_worked_example_per_channel():
    g = _read_golden("key_per_channel_example.txt")
    X = np.array([[float(v) for v in row[1:]] for row in g["tokens"]], np.float32)  # [3 tok, 4 ch]
    c = OracleCache(1, 1, 1, 4, oracle.INT8_SYM_PER_CHANNEL, oracle.INT8_SYM_PER_CHANNEL, cap=8)
    x = X[None, None]  # [B=1, H=1, T=3, D=4]
    c.append(x, x, bf16=False, calibrate=True)
    codes = c["k_codes"][0, 0, :3].view(np.int8)
    for row in g["codes"]:
        ch, num, want = int(row[0]) - 1, row[1], [int(v) for v in row[2:]]
        col = [str(r[1 + ch]) for r in g["tokens"]]
        assert _sym_exact(col, max(Fraction(v) for v in col)) == want  # fixture is exact math
        assert list(codes[:, ch]) == want
        # the per-channel scale is max|column| / 127; channel 3 prints s = 9.0/127
        assert c["k_scale"][0, ch] == F32(float(num)) / F32(127)
    assert c["k_scale"][0, 2] == F32(9.0) / F32(127)
    # each column has its own scale: channel 3's outliers do not touch channels 1, 2, 4
    assert len(set(c["k_scale"][0].tolist())) == 3


def test_value_worked_example_per_token():
    g = _read_golden("value_per_token_example.txt")
    X = np.array([[float(v) for v in row[1:]] for row in g["tokens"]], np.float32)
    c = OracleCache(1, 1, 1, 4, oracle.INT8_SYM_PER_TOKEN, oracle.INT8_SYM_PER_TOKEN, cap=8)
    c.append(X[None, None], X[None, None], bf16=False)
    codes = c["v_codes"][0, 0, :3].view(np.int8)
    for row in g["codes"]:
        t, num, want = int(row[0]) - 1, row[1], [int(v) for v in row[2:]]
        tok = g["tokens"][t][1:]
        assert _sym_exact(tok, max(Fraction(v) for v in tok)) == want
        assert list(codes[t]) == want
        assert c["v_scale"][0, 0, t] == F32(float(num)) / F32(127)


# --------------------------------------------------------------- byte arithmetic
def test_memory_table_and_formula():
    table = []
    with open(os.path.join(GOLDEN, "memory_table.txt")) as fh:
        for line in fh:
            if line.strip() and not line.startswith("#"):
                table.append(line.split())
    per_tok = {}
    for name, bpe, kb, gb, req in table:
        b = oracle.kv_bytes_per_token(80, 8, 128, float(bpe))
        per_tok[name] = b
        assert b / 1024 == float(kb)                       # 320 / 160 / 80 KiB
        assert abs(b * 4096 / 2**30 - float(gb)) < 0.0051  # 1.25 / 0.63 / 0.31 GiB
        exact = int(45 * 2**30 // (b * 4096))
        assert abs(exact - int(req)) <= 1                  # 36/72/144 vs printed 36/71/145
    assert per_tok["BF16"] == 327680.0 == 2 * 2 * 80 * 8 * 128
    assert per_tok["FP8"] == 163840.0 and per_tok["INT4"] == 81920.0
    assert per_tok["BF16"] * 4096 == 1.25 * 2**30


# --------------------------------------------------------------- E4M3 codec
def test_e4m3_decode_matches_torch():
    torch = pytest.importorskip("torch")
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).float().numpy()
    for c in codes:
        got = oracle.e4m3_decode(int(c))
        if np.isnan(ref[c]):
            assert np.isnan(got)
        else:
            assert got == ref[c] and np.signbit(got) == np.signbit(ref[c])


def test_e4m3_roundtrip_all_codes():
    for c in range(256):
        if c & 0x7F == 0x7F:
            continue  # NaN
        assert oracle.e4m3_encode(oracle.e4m3_decode(c)) == c


def test_e4m3_encode_matches_torch_in_range():
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(7)
    x = np.concatenate([
        rng.uniform(-448, 448, 20000), rng.normal(0, 1, 20000), rng.normal(0, 0.01, 20000),
        np.ldexp(rng.uniform(-1, 1, 5000), -8),
    ]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_encode(v) for v in x], np.uint8)
    assert np.array_equal(got, ref)


def test_e4m3_ties_saturation_and_zero():
    assert oracle.e4m3_encode(1.0 + 1 / 16) == oracle.e4m3_encode(1.0)        # tie -> even (m=0)
    assert oracle.e4m3_decode(oracle.e4m3_encode(1.0 + 3 / 16)) == 1.25         # tie -> even (m=2)
    assert oracle.e4m3_encode(2.0**-10) == 0x00                                 # subnormal tie -> 0
    assert oracle.e4m3_decode(oracle.e4m3_encode(3 * 2.0**-10)) == 2.0**-8      # -> even code 2
    for big in (448.0, 449.0, 464.0, 500.0, 1e30, float("inf")):
        assert oracle.e4m3_encode(big) == 0x7E
        assert oracle.e4m3_encode(-big) == 0xFE
    assert oracle.e4m3_decode(0x7E) == 448.0
    assert oracle.e4m3_encode(-0.0) == 0x80 and oracle.e4m3_encode(0.0) == 0x00


def test_e4m3_nearest_by_brute_force():
    finite = [(c, oracle.e4m3_decode(c)) for c in range(128) if c != 0x7F]
    rng = np.random.default_rng(3)
    for x in rng.uniform(0, 448, 3000).astype(np.float32):
        code = oracle.e4m3_encode(float(x))
        best = min(abs(v - float(x)) for _, v in finite)
        assert abs(oracle.e4m3_decode(code) - float(x)) == best


# --------------------------------------------------------------- FP8 E5M2 (a next-row format)
def test_e5m2_decode_matches_torch():
    torch = pytest.importorskip("torch")
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes.copy()).view(torch.float8_e5m2).float().numpy()
    for c in codes:
        got = oracle.e5m2_decode(int(c))
        if np.isnan(ref[c]):
            assert np.isnan(got)
        else:
            assert got == ref[c] and np.signbit(got) == np.signbit(ref[c])


def test_e5m2_roundtrip_all_finite_codes():
    for c in range(256):
        if (c >> 2) & 0x1F == 0x1F:
            continue  # infinity and NaN
        assert oracle.e5m2_encode(oracle.e5m2_decode(c)) == c


def test_e5m2_encode_matches_torch_in_range():
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(8)
    x = np.concatenate([
        rng.uniform(-57344, 57344, 20000), rng.normal(0, 1, 20000), rng.normal(0, 1e-3, 20000),
        np.ldexp(rng.uniform(-1, 1, 5000), -15),
    ]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e5m2).view(torch.uint8).numpy()
    got = np.array([oracle.e5m2_encode(v) for v in x], np.uint8)
    assert np.array_equal(got, ref)


def test_e5m2_ties_saturation_and_zero():
    assert oracle.e5m2_encode(1.125) == oracle.e5m2_encode(1.0)                 # tie -> even (m=0)
    assert oracle.e5m2_decode(oracle.e5m2_encode(1.375)) == 1.5                 # tie -> even (m=2)
    assert oracle.e5m2_encode(2.0**-17) == 0x00                                 # subnormal tie -> 0
    assert oracle.e5m2_decode(oracle.e5m2_encode(3 * 2.0**-17)) == 2.0**-15     # -> even code 2
    for big in (57344.0, 57345.0, 61440.0, 70000.0, 1e30, float("inf")):
        assert oracle.e5m2_encode(big) == 0x7B
        assert oracle.e5m2_encode(-big) == 0xFB
    assert oracle.e5m2_decode(0x7B) == 57344.0
    assert oracle.e5m2_encode(-0.0) == 0x80 and oracle.e5m2_encode(0.0) == 0x00


def test_e5m2_nearest_by_brute_force():
    finite = [(c, oracle.e5m2_decode(c)) for c in range(124)]
    rng = np.random.default_rng(4)
    for x in np.concatenate([rng.uniform(0, 57344, 1500), rng.uniform(0, 4, 1500)]).astype(np.float32):
        code = oracle.e5m2_encode(float(x))
        best = min(abs(v - float(x)) for _, v in finite)
        assert abs(oracle.e5m2_decode(code) - float(x)) == best


def test_e5m2_per_tensor_scale_and_codes():
    rng = np.random.default_rng(5)
    x = rng.normal(0, 2, (1, 2, 6, 16)).astype(np.float32)
    c = OracleCache(1, 2, 2, 16, oracle.FP8_E5M2_PER_TENSOR, oracle.FP8_E5M2_PER_TENSOR, cap=8)
    c.append(x, x, bf16=False, calibrate=True)
    s = F32(np.abs(x).max()) / F32(57344)
    assert c["k_scale"][0] == s and c["v_scale"][0] == s
    deq = c.dequantize(1, 8)[:, :, :6]
    # E5M2 relative step is 2^-2: nearest-value error <= 2^-3 relative (normal range)
    err = np.abs(deq - x)
    bound = np.maximum(np.abs(x) * 2.0**-3, float(s) * 2.0**-17) * (1 + 2**-20)
    assert np.all(err <= bound)
    assert np.abs(deq).max() == np.abs(x).max()  # the absmax element maps to 57344 exactly


# --------------------------------------------------------------- symmetric INT8
def test_sym_round_half_even_tie():
    s = 0.125
    assert oracle.sym_code(62.5 * s, s) == 62   # half-away would give 63
    assert oracle.sym_code(63.5 * s, s) == 64
    assert oracle.sym_code(-62.5 * s, s) == -62
    assert oracle.sym_code(5.0, 0.0) == 0       # zero range
    assert oracle.sym_code(1000.0, 1.0) == 127 and oracle.sym_code(-1000.0, 1.0) == -127


def test_sym_exact_roundtrip_and_half_step_bound():
    for s in (2.0**-7, 0.25, 1.0, 8.0):
        for k in range(-127, 128):
            assert oracle.sym_code(k * s, s) == k
    rng = np.random.default_rng(11)
    x = rng.normal(0, 3, 4000).astype(np.float32)
    s = F32(np.abs(x).max()) / F32(127)
    for v in x:
        q = oracle.sym_code(float(v), float(s))
        xh = F32(q) * s
        assert abs(float(xh) - float(v)) <= float(s) / 2 * (1 + 2**-22)


def test_per_tensor_scale_covers_all_rows_and_heads():
    B, H, T, D = 2, 3, 5, 8
    rng = np.random.default_rng(1)
    x = rng.normal(0, 1, (B, H, T, D)).astype(np.float32)
    x[1, 2, 4, 7] = -50.0  # the largest magnitude sits in the last row / head / token / channel
    c = OracleCache(B, H, H, D, oracle.INT8_SYM_PER_TENSOR, oracle.INT8_SYM_PER_TENSOR, cap=16)
    c.append(x, x, bf16=False, calibrate=True)
    assert c["k_scale"][0] == F32(50.0) / F32(127)
    assert c["k_codes"][1, 2, 4, 7].view(np.int8) == -127
    # a second, non-calibrating append keeps the scale and saturates out-of-range values
    y = np.full((B, H, 1, D), 100.0, np.float32)
    c.append(y, y, bf16=False)
    assert c["k_scale"][0] == F32(50.0) / F32(127)
    assert np.all(c["k_codes"][:, :, T].view(np.int8) == 127)


def test_fp8_per_tensor_scale_and_codes():
    rng = np.random.default_rng(2)
    x = rng.normal(0, 2, (1, 2, 6, 16)).astype(np.float32)
    c = OracleCache(1, 2, 2, 16, oracle.FP8_E4M3_PER_TENSOR, oracle.FP8_E4M3_PER_TENSOR, cap=8)
    c.append(x, x, bf16=False, calibrate=True)
    s = F32(np.abs(x).max()) / F32(448)
    assert c["k_scale"][0] == s
    deq = c.dequantize(0, 8)[:, :, :6]
    # E4M3 relative step is 2^-3: nearest-value error <= 2^-4 relative (normal range)
    err = np.abs(deq - x)
    bound = np.maximum(np.abs(x) * 2.0**-4, float(s) * 2.0**-10) * (1 + 2**-20)
    assert np.all(err <= bound)
    assert np.abs(deq).max() == np.abs(x).max()  # the absmax element maps to 448 exactly


# --------------------------------------------------------------- asymmetric uint8
def test_asym_affine_roundtrip_and_bounds():
    s_pow2 = 2.0**-4
    mn, mx = -100 * s_pow2, 155 * s_pow2
    s, zp = oracle.asym_params(mn, mx)
    assert s == F32(mx - mn) / F32(255) and zp == 100
    for k in range(256):
        x = (k - zp) * float(s)
        q = oracle.asym_code(x, s, zp)
        assert q == k and (q - zp) * s == F32(x)
    rng = np.random.default_rng(5)
    x = rng.normal(0.3, 2.0, 3000).astype(np.float32)
    s, zp = oracle.asym_params(float(x.min()), float(x.max()))
    for v in x:
        q = oracle.asym_code(float(v), s, zp)
        err = abs(float(F32(q - zp) * F32(s)) - float(v))
        assert err <= float(s) * (1 + 2**-20)  # <= s/2 inside, <= s at a clamped edge


def test_asym_range_without_zero_is_widened():
    # The page's literal form (zp clamped to 0, codes from (x - min)/s, dequant
    # (q - zp) * s) decodes the range [1, 2] onto [0, 1]; the affine reading keeps it.
    s, zp = oracle.asym_params(1.0, 2.0)
    assert zp == 0 and s == F32(2.0) / F32(255)
    for v in (1.0, 1.5, 2.0):
        q = oracle.asym_code(v, s, zp)
        assert abs(float(F32(q) * F32(s)) - v) <= float(s) / 2 * (1 + 2**-20)


def test_per_channel_asym_calibration_axis():
    # One (scale, zp) per (kv_head, channel), reduced over batch rows and tokens.
    B, H, T, D = 3, 2, 4, 8
    rng = np.random.default_rng(9)
    x = rng.normal(0, 1, (B, H, T, D)).astype(np.float32)
    c = OracleCache(B, H, H, D, oracle.INT8_SYM_PER_TENSOR, oracle.UINT8_ASYM_PER_CHANNEL, cap=8)
    c.append(x, x, bf16=False, calibrate=True)
    for h in range(H):
        for d in range(D):
            col = x[:, h, :, d]
            s, zp = oracle.asym_params(float(col.min()), float(col.max()))
            assert c["v_scale"][h, d] == s and c["v_zp"][h, d] == zp


# --------------------------------------------------------------- KIVI
@pytest.mark.parametrize("bits", [4, 2])
def test_kivi_group_extremes_and_nearest_level(bits):
    qmax = 2**bits - 1
    rng = np.random.default_rng(bits)
    for _ in range(200):
        x = rng.normal(0, 1, 32).astype(np.float32)
        codes, s, mn = oracle.kivi_group(x, bits)
        assert mn == x.min() and s == F32(F32(x.max()) - F32(x.min())) / F32(qmax)
        assert codes[np.argmin(x)] == 0 and codes[np.argmax(x)] == qmax
        for xi, qi in zip(x, codes):
            levels = [oracle.kivi_value(k, s, mn) for k in range(qmax + 1)]
            dists = [abs(float(L) - float(xi)) for L in levels]
            # the chosen level is a nearest one (brute force over all 2^bits codes)
            assert dists[qi] <= min(dists) + float(s) * 2**-20
            assert dists[qi] <= float(s) / 2 * (1 + 2**-22) + abs(float(mn)) * 2**-23


@pytest.mark.parametrize("bits", [4, 2])
def test_kivi_exact_grid_and_zero_range(bits):
    qmax = 2**bits - 1
    s, mn = 2.0**-3, -1.5
    ks = np.arange(32) % (qmax + 1)
    ks[0], ks[1] = 0, qmax
    x = (mn + ks * s).astype(np.float32)
    codes, s_o, mn_o = oracle.kivi_group(x, bits)
    assert s_o == s and mn_o == mn and list(codes) == list(ks)
    for k in range(qmax + 1):
        assert oracle.kivi_value(k, s_o, mn_o) == F32(mn + k * s)
    z = np.full(32, 0.75, np.float32)
    codes, s_o, mn_o = oracle.kivi_group(z, bits)
    assert s_o == 0 and mn_o == F32(0.75) and not codes.any()
    neg0 = np.array([-0.0] * 32, np.float32)
    _, s_o, mn_o = oracle.kivi_group(neg0, bits)
    assert not np.signbit(mn_o) and not np.signbit(s_o)


def _kivi_cache(B, H, D, cap, bits, group=32, rcap=128):
    sch = oracle.KIVI_INT4 if bits == 4 else oracle.KIVI_INT2
    return OracleCache(B, H, H, D, sch, sch, cap=cap, group=group, rcap=rcap)


def _bf16(a):
    return (np.ascontiguousarray(a, np.float32).view(np.uint32) >> 16).astype(np.uint16)


def test_kivi_residual_page_example():
    # The page's streaming example: with groups of 64 tokens, 200 tokens leave tokens
    # 1..192 quantized (three groups) and tokens 193..200 in the bf16 residual.
    rng = np.random.default_rng(4)
    x = _bf16(rng.normal(0, 1, (1, 1, 200, 128)))
    c = _kivi_cache(1, 1, 128, 256, 4, group=64, rcap=64)
    c.append(x, x, bf16=True)
    assert (c.length, c.residual) == (192, 8)
    assert np.array_equal(c["k_res"][0, 0, :8], x[0, 0, 192:200])


@pytest.mark.parametrize("n", [1, 127, 128, 129, 256, 257, 300])
def test_kivi_bulk_equals_streaming(n):
    rng = np.random.default_rng(n)
    k = _bf16(rng.normal(0, 1, (2, 2, n, 64)))
    v = _bf16(rng.normal(0, 1, (2, 2, n, 64)))
    a = _kivi_cache(2, 2, 64, 512, 2)
    a.append(k, v, bf16=True)
    b = _kivi_cache(2, 2, 64, 512, 2)
    for t in range(n):
        b.append(k[:, :, t:t + 1], v[:, :, t:t + 1], bf16=True)
    assert a.length == b.length == 128 * ((n - 1) // 128)
    assert a.residual == b.residual == n - a.length
    for name in ("k_codes", "v_codes", "k_scale", "k_zero", "v_scale", "v_zero"):
        assert np.array_equal(a[name], b[name]), name
    for name in ("k_res", "v_res"):  # only the first `residual` slots are state
        assert np.array_equal(a[name][:, :, :a.residual], b[name][:, :, :b.residual]), name


def test_kivi_axes_key_per_channel_value_per_token():
    # Keys: one (scale, min) per channel per 32-token group; values: one per token per
    # 32-channel group. A key outlier channel must not change other channels' scales;
    # a large value token must not change other tokens' scales.
    rng = np.random.default_rng(8)
    k = rng.normal(0, 1, (1, 1, 129, 64)).astype(np.float32)
    v = rng.normal(0, 1, (1, 1, 129, 64)).astype(np.float32)
    k2, v2 = k.copy(), v.copy()
    k2[0, 0, :, 5] *= 100.0
    v2[0, 0, 17, :] *= 100.0
    outs = []
    for kk, vv in ((k, v), (k2, v2)):
        c = _kivi_cache(1, 1, 64, 256, 4)
        c.append(_bf16(kk), _bf16(vv), bf16=True)
        outs.append(c)
    a, b = outs
    diff_k = (a["k_scale"] != b["k_scale"])[:, :, :4]  # [1,1,groups,D]; 128 tokens flushed
    assert diff_k[0, 0, :, 5].all() and not np.delete(diff_k[0, 0], 5, axis=1).any()
    diff_v = a["v_scale"] != b["v_scale"]          # [1,1,T,D/32]
    assert diff_v[0, 0, 17].all() and not np.delete(diff_v[0, 0], 17, axis=0).any()
    # the scale of channel d in group gi is (max - min)/15 of that column slice
    xk = _bf16(k).astype(np.uint32) << 16
    col = xk.view(np.float32)[0, 0, 32:64, 9]
    assert a["k_scale"][0, 0, 1, 9] == F32(F32(col.max()) - F32(col.min())) / F32(15)


def test_kivi_packing_low_index_low_bits():
    x = np.zeros((1, 1, 129, 64), np.float32)
    ramp = np.arange(32) % 4
    x[0, 0, 0, :32] = ramp           # value token 0, channel group 0: codes 0,1,2,3,0,1,...
    c = _kivi_cache(1, 1, 64, 256, 2)
    c.append(_bf16(x), _bf16(x), bf16=True)
    row = c["v_codes"][0, 0, 0]
    assert row[0] == (0 | 1 << 2 | 2 << 4 | 3 << 6)


# --------------------------------------------------------------- attention (fp64)
def _attn(q, k, v, scale):
    return oracle.attention_row(np.asarray(q, np.float32), np.asarray(k, np.float32),
                                np.asarray(v, np.float32), scale)


def test_attention_closed_forms():
    rng = np.random.default_rng(0)
    D = 16
    q = rng.normal(0, 1, D).astype(np.float32)
    k = rng.normal(0, 1, (5, D)).astype(np.float32)
    v = rng.normal(0, 1, (5, D)).astype(np.float32)
    out, lse = _attn(q, k[:1], v[:1], 0.3)
    assert np.array_equal(out, v[0].astype(np.float64))      # T = 1 -> that value row
    out, _ = _attn(np.zeros(D), k, v, 0.3)
    assert np.allclose(out, v.astype(np.float64).mean(0), rtol=0, atol=1e-15)  # q = 0 -> mean
    kk = np.repeat(k[:1], 5, 0)
    out, lse = _attn(q, kk, v, 0.3)
    assert np.allclose(out, v.astype(np.float64).mean(0), rtol=0, atol=1e-15)  # equal keys
    s0 = float(np.dot(q.astype(np.float64), kk[0].astype(np.float64))) * np.float64(F32(0.3))
    assert abs(lse - (s0 + math.log(5))) < 1e-12
    # one score larger by >= 800 -> exactly that value row (exp(-800) underflows)
    k3 = np.zeros((4, D), np.float32)
    q3 = np.zeros(D, np.float32)
    q3[0] = 1.0
    k3[2, 0] = 1000.0
    out, _ = _attn(q3, k3, v[:4], 1.0)
    assert np.array_equal(out, v[2].astype(np.float64))


def test_attention_shift_invariance_and_empty():
    rng = np.random.default_rng(1)
    D = 8
    q = np.zeros(D, np.float32)
    q[0] = 2.0
    k = (np.round(rng.normal(0, 1, (6, D)) * 1024) / 1024).astype(np.float32)  # k + 3 is exact
    v = rng.normal(0, 1, (6, D)).astype(np.float32)
    a, la = _attn(q, k, v, 0.5)
    k2 = k.copy()
    k2[:, 0] += 3.0  # adds 2 * 3 * 0.5 = 3 to every score exactly
    b, lb = _attn(q, k2, v, 0.5)
    assert np.allclose(a, b, rtol=0, atol=1e-13) and abs((lb - la) - 3.0) < 1e-12
    out, lse = _attn(q, np.zeros((0, D)), np.zeros((0, D)), 0.5)
    assert not out.any() and lse == -math.inf


def test_attention_against_high_precision_brute_force():
    decimal.getcontext().prec = 50
    rng = np.random.default_rng(2)
    for T in (1, 3, 17, 64):
        D = 8
        q = rng.normal(0, 1, D).astype(np.float32)
        k = (rng.normal(0, 3, (T, D))).astype(np.float32)
        v = rng.normal(0, 1, (T, D)).astype(np.float32)
        scale = F32(1 / math.sqrt(D))
        out, lse = _attn(q, k, v, float(scale))
        Dd = decimal.Decimal
        s = [sum(Dd(float(q[d])) * Dd(float(k[t, d])) for d in range(D)) * Dd(float(scale)) for t in range(T)]
        m = max(s)
        p = [(x - m).exp() for x in s]
        l = sum(p)
        ref = [float(sum(p[t] * Dd(float(v[t, d])) for t in range(T)) / l) for d in range(D)]
        assert np.allclose(out, ref, rtol=1e-13, atol=1e-13)
        assert abs(lse - float(m + l.ln())) < 1e-12


def test_attention_split_merge_equals_whole():
    # LSE merge of any split of the token axis equals attention over all tokens.
    rng = np.random.default_rng(3)
    D, T = 16, 40
    q = rng.normal(0, 1, D).astype(np.float32)
    k = rng.normal(0, 2, (T, D)).astype(np.float32)
    v = rng.normal(0, 1, (T, D)).astype(np.float32)
    whole, lw = _attn(q, k, v, 0.25)
    for cuts in ([13], [1, 2, 39], [10, 20, 30]):
        bounds = [0, *cuts, T]
        parts = [_attn(q, k[a:b], v[a:b], 0.25) for a, b in zip(bounds, bounds[1:])]
        M = max(l for _, l in parts)
        w = [math.exp(l - M) for _, l in parts]
        merged = sum(wi * o for wi, (o, _) in zip(w, parts)) / sum(w)
        assert np.allclose(merged, whole, rtol=1e-13, atol=1e-13)
        assert abs(M + math.log(sum(w)) - lw) < 1e-12


# --------------------------------------------------------------- cache plumbing
def test_paged_gather_matches_dense():
    rng = np.random.default_rng(6)
    B, H, D, ps = 3, 2, 16, 4
    lens = np.array([5, 9, 1], np.int32)
    maxp = 4
    perm = rng.permutation(12).astype(np.int32)
    table = perm.reshape(B, maxp)
    n = int(lens.max())
    k = rng.normal(0, 1, (B, H, n, D)).astype(np.float32)
    v = rng.normal(0, 1, (B, H, n, D)).astype(np.float32)
    pg = OracleCache(B, H, H, D, oracle.INT8_SYM_PER_TENSOR, oracle.UINT8_ASYM_PER_CHANNEL,
                     paged=True, page_size=ps, max_pages=maxp, num_pages=12, page_table=table)
    pg.append(k, v, bf16=False, calibrate=True, new_lens=lens)
    assert list(pg["seq_lens"]) == list(lens)
    for b in range(B):
        dn = OracleCache(1, H, H, D, oracle.INT8_SYM_PER_TENSOR, oracle.UINT8_ASYM_PER_CHANNEL, cap=16)
        dn["k_scale"][:] = pg["k_scale"]
        dn["v_scale"][:] = pg["v_scale"]
        dn["v_zp"][:] = pg["v_zp"]
        dn.append(k[b:b + 1, :, :lens[b]], v[b:b + 1, :, :lens[b]], bf16=False)
        for t in range(lens[b]):
            page, slot = table[b, t // ps], t % ps
            assert np.array_equal(pg["k_codes"][page, :, slot], dn["k_codes"][0, :, t])
            assert np.array_equal(pg["v_codes"][page, :, slot], dn["v_codes"][0, :, t])
        a = pg.dequantize(1, 12)[b, :, :lens[b]]
        assert np.array_equal(a, dn.dequantize(1, 12)[0, :, :lens[b]])


def test_gqa_head_mapping_and_decode():
    # Query head h reads kv head h // G: with G = 2, heads 0,1 -> kv 0 and 2,3 -> kv 1.
    rng = np.random.default_rng(12)
    B, Hq, H, D, T = 1, 4, 2, 8, 6
    k = rng.normal(0, 1, (B, H, T, D)).astype(np.float32)
    v = rng.normal(0, 1, (B, H, T, D)).astype(np.float32)
    c = OracleCache(B, Hq, H, D, oracle.INT8_SYM_PER_TOKEN, oracle.INT8_SYM_PER_TOKEN, cap=8)
    c.append(k, v, bf16=False)
    q = rng.normal(0, 1, (B, Hq, D)).astype(np.float32)
    out, lse = c.decode(q, bf16=False, scale=0.35)
    K, V = c.dequantize(0, T), c.dequantize(1, T)
    for h in range(Hq):
        ref, lr = _attn(q[0, h], K[0, h // 2], V[0, h // 2], 0.35)
        assert np.array_equal(out[0, h], ref) and lse[0, h] == lr


def test_capacity_errors():
    c = OracleCache(1, 1, 1, 8, oracle.INT8_SYM_PER_TOKEN, oracle.INT8_SYM_PER_TOKEN, cap=4)
    x = np.zeros((1, 1, 5, 8), np.float32)
    with pytest.raises(ValueError):
        c.append(x, x, bf16=False)


def test_calibrate_only_equals_calibrating_append():
    rng = np.random.default_rng(13)
    B, H, T, D = 3, 2, 9, 16
    k = rng.normal(0, 2, (B, H, T, D)).astype(np.float32)
    v = rng.normal(0.5, 1, (B, H, T, D)).astype(np.float32)
    lens = np.array([9, 4, 0], np.int32)
    table = np.arange(3 * 4, dtype=np.int32).reshape(3, 4)
    mk = lambda: OracleCache(B, H, H, D, oracle.INT8_SYM_PER_TENSOR, oracle.UINT8_ASYM_PER_CHANNEL, paged=True,
                             page_size=4, max_pages=4, num_pages=12, page_table=table)
    a, b = mk(), mk()
    a.append(k, v, bf16=False, calibrate=True, new_lens=lens)
    b.calibrate(k, v, bf16=False, new_lens=lens)
    for name in ("k_scale", "v_scale", "v_zp"):
        assert np.array_equal(a[name], b[name]), name
    assert not b["k_codes"].any() and not b["seq_lens"].any()


# --------------------------------------------------------------- rescaling append
# n4n.ai Step 3 merges each new block's scale into the cached one with a running maximum;
# Step 7 asks for scales that only grow, or are recomputed as the cache grows. The oracle's
# rescaling append merges and requantizes the cached codes whose scale changed.
BATCH_WIDE = [oracle.FP8_E4M3_PER_TENSOR, oracle.FP8_E5M2_PER_TENSOR, oracle.INT8_SYM_PER_TENSOR,
              oracle.INT8_SYM_PER_CHANNEL, oracle.UINT8_ASYM_PER_CHANNEL]


def _exact(x) -> Fraction:
    return Fraction(float(x))


def _nearest_sym(x: Fraction, s: Fraction, qmax=127):
    """All integers k in [-qmax, qmax] at the least distance |x - k s| (brute force)."""
    d = [abs(x - k * s) for k in range(-qmax, qmax + 1)]
    m = min(d)
    return [k - qmax for k, v in enumerate(d) if v == m], m


@pytest.mark.parametrize("scheme", BATCH_WIDE)
def test_rescale_on_empty_cache_equals_calibration(scheme):
    # merging into the zero scale (or the empty range) of a fresh cache is a calibration
    rng = np.random.default_rng(40 + scheme)
    B, H, T, D = 2, 2, 5, 16
    k = rng.normal(0, 2, (B, H, T, D)).astype(np.float32)
    v = rng.normal(0.4, 1, (B, H, T, D)).astype(np.float32)
    a = OracleCache(B, H, H, D, oracle.INT8_SYM_PER_TENSOR, scheme, cap=8)
    b = OracleCache(B, H, H, D, oracle.INT8_SYM_PER_TENSOR, scheme, cap=8)
    a.append(k, v, bf16=False, rescale=True)
    b.append(k, v, bf16=False, calibrate=True)
    for name in ("k_scale", "v_scale", "k_codes", "v_codes"):
        assert np.array_equal(a[name], b[name]), name
    if scheme == oracle.UINT8_ASYM_PER_CHANNEL:
        assert np.array_equal(a["v_zp"], b["v_zp"])
    assert a["v_scale"].any() and a["v_codes"].any()


@pytest.mark.parametrize("scheme", BATCH_WIDE)
def test_rescale_inside_range_changes_nothing(scheme):
    rng = np.random.default_rng(50 + scheme)
    B, H, T, D = 2, 2, 6, 16
    x = rng.normal(0.2, 2, (B, H, T, D)).astype(np.float32)
    y = (x[:, :, :2] * F32(0.5)).astype(np.float32)  # inside every per-channel / per-tensor range
    a = OracleCache(B, H, H, D, scheme, scheme, cap=8)
    b = OracleCache(B, H, H, D, scheme, scheme, cap=8)
    for c in (a, b):
        c.append(x, x, bf16=False, calibrate=True)
    before = {n: a[n].copy() for n in ("k_scale", "k_codes", "v_zp") if a[n] is not None}
    a.append(y, y, bf16=False, rescale=True)
    b.append(y, y, bf16=False)  # plain append with the cached scales
    for n, old in before.items():
        assert np.array_equal(a[n][..., :T, :] if n == "k_codes" else a[n],
                              old[..., :T, :] if n == "k_codes" else old), n
    assert np.array_equal(a["k_codes"], b["k_codes"]) and np.array_equal(a["v_codes"], b["v_codes"])


def test_rescale_per_tensor_int8_grows_and_requantizes_to_nearest():
    rng = np.random.default_rng(60)
    B, H, T, D = 1, 2, 6, 16
    x = rng.normal(0, 1, (B, H, T, D)).astype(np.float32)
    amax = F32(np.abs(x).max())
    y = np.zeros((B, H, 1, D), np.float32)
    y[0, 1, 0, 3] = F32(4) * amax
    c = OracleCache(B, H, H, D, oracle.INT8_SYM_PER_TENSOR, oracle.INT8_SYM_PER_TENSOR, cap=8)
    c.append(x, x, bf16=False, calibrate=True)
    s0 = c["k_scale"][0]
    q0 = c["k_codes"][:, :, :T].view(np.int8).astype(int)
    c.append(y, y, bf16=False, rescale=True)
    s1 = c["k_scale"][0]
    assert s1 == F32(F32(4) * amax) / F32(127) and s1 > s0  # the block's scale wins
    q1 = c["k_codes"][:, :, :T].view(np.int8).astype(int)
    assert c["k_codes"][0, 1, T, 3].view(np.int8) == 127
    S1 = _exact(s1)
    for old, new in zip(q0.ravel(), q1.ravel()):
        xo = _exact(F32(old) * s0)                  # the cached value before the rescale
        best, dist = _nearest_sym(xo, S1)
        r = xo / S1
        half = math.floor(r) + Fraction(1, 2)
        if len(best) > 1:                           # an exact tie between two levels: the even one
            assert new in best and new % 2 == 0
        elif abs(r - half) <= abs(r) * Fraction(1, 2**24):
            # within the fp32 rounding of x / s of a tie: the rounded quotient decides
            assert new in (math.floor(r), math.floor(r) + 1)
        else:
            assert new == best[0]
        assert abs(new) <= abs(old)


def test_rescale_fp8_requantizes_like_torch_cast():
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(61)
    B, H, T, D = 1, 2, 8, 16
    x = rng.normal(0, 1, (B, H, T, D)).astype(np.float32)
    y = (x[:, :, :1] * F32(3)).astype(np.float32)
    c = OracleCache(B, H, H, D, oracle.FP8_E4M3_PER_TENSOR, oracle.FP8_E4M3_PER_TENSOR, cap=16)
    c.append(x, x, bf16=False, calibrate=True)
    s0 = c["v_scale"][0]
    old = c["v_codes"][:, :, :T].copy()
    c.append(y, y, bf16=False, rescale=True)
    s1 = c["v_scale"][0]
    assert s1 == F32(np.abs(y).max()) / F32(448)
    xo = torch.from_numpy(old.copy()).view(torch.float8_e4m3fn).float() * float(s0)   # fp32 product
    want = (xo / float(s1)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(c["v_codes"][:, :, :T], want)


def test_rescale_asym_union_of_ranges():
    rng = np.random.default_rng(62)
    B, H, T, D = 2, 1, 6, 8
    x = rng.normal(0.5, 1, (B, H, T, D)).astype(np.float32)
    y = np.zeros((B, H, 1, D), np.float32)
    y[0, 0, 0, :4] = F32(5)                      # channels 0..3 grow upwards only
    y[1, 0, 0, 4:6] = F32(-7)                    # channels 4, 5 grow downwards only
    c = OracleCache(B, H, H, D, oracle.INT8_SYM_PER_TENSOR, oracle.UINT8_ASYM_PER_CHANNEL, cap=8)
    c.append(x, x, bf16=False, calibrate=True)
    s0, z0 = c["v_scale"].copy(), c["v_zp"].copy()
    old = c["v_codes"][:, :, :T].copy()
    c.append(y, y, bf16=False, rescale=True)
    s1, z1 = c["v_scale"], c["v_zp"]
    for d in range(D):
        lo_o = float(F32(0 - int(z0[0, d])) * s0[0, d])
        hi_o = float(F32(255 - int(z0[0, d])) * s0[0, d])
        col = y[:, 0, 0, d]
        lo, hi = min(lo_o, float(col.min()), 0.0), max(hi_o, float(col.max()), 0.0)
        if d >= 6:
            assert s1[0, d] == s0[0, d] and z1[0, d] == z0[0, d]   # untouched channels
            assert np.array_equal(c["v_codes"][:, :, :T, d], old[:, :, :, d])
            continue
        s, z = float(s1[0, d]), int(z1[0, d])
        assert abs(s - (hi - lo) / 255) <= 1e-6 * s                 # 255 steps over the union
        assert -z * s <= lo + s / 2 and (255 - z) * s >= hi - s / 2  # the union is represented
        S1 = _exact(s1[0, d])
        for b in range(B):
            for t in range(T):
                xo = _exact(F32(int(old[b, 0, t, d]) - int(z0[0, d])) * s0[0, d])
                q = int(c["v_codes"][b, 0, t, d])
                dist = [abs(xo - (k - z) * S1) for k in range(256)]
                assert dist[q] == min(dist)                          # nearest representable level


def test_rescale_per_channel_sym_only_grown_channels_move():
    rng = np.random.default_rng(63)
    B, H, T, D = 2, 2, 5, 8
    x = rng.normal(0, 1, (B, H, T, D)).astype(np.float32)
    y = np.zeros((B, H, 1, D), np.float32)
    y[1, 1, 0, 2] = F32(9)
    c = OracleCache(B, H, H, D, oracle.INT8_SYM_PER_CHANNEL, oracle.INT8_SYM_PER_CHANNEL, cap=8)
    c.append(x, x, bf16=False, calibrate=True)
    s0, old = c["k_scale"].copy(), c["k_codes"][:, :, :T].copy()
    c.append(y, y, bf16=False, rescale=True)
    moved = c["k_scale"] != s0
    assert moved.sum() == 1 and moved[1, 2] and c["k_scale"][1, 2] == F32(9) / F32(127)
    keep = np.ones((H, D), bool)
    keep[1, 2] = False
    for h in range(H):
        for d in range(D):
            same = np.array_equal(c["k_codes"][:, h, :T, d], old[:, h, :, d])
            assert same == bool(keep[h, d]) or (not keep[h, d] and same and not old[:, h, :, d].any())


def test_rescale_scales_never_shrink():
    rng = np.random.default_rng(64)
    B, H, D = 1, 2, 16
    c = OracleCache(B, H, H, D, oracle.FP8_E5M2_PER_TENSOR, oracle.UINT8_ASYM_PER_CHANNEL, cap=64)
    prev_k, prev_lo, prev_hi = 0.0, np.zeros((H, D)), np.zeros((H, D))
    for i in range(8):
        blk = rng.normal(0, float(rng.uniform(0.2, 3)), (B, H, 4, D)).astype(np.float32)
        c.append(blk, blk, bf16=False, rescale=True)
        sk = float(c["k_scale"][0])
        lo = (0 - c["v_zp"].astype(float)) * c["v_scale"]
        hi = (255 - c["v_zp"].astype(float)) * c["v_scale"]
        assert sk >= prev_k
        # the represented range only widens, up to the half step the integer zero point
        # rounds away at one end
        half = c["v_scale"] / 2 * (1 + 1e-5)
        assert np.all(lo <= prev_lo + half) and np.all(hi >= prev_hi - half)
        prev_k, prev_lo, prev_hi = sk, lo, hi


def test_rescale_paged_matches_dense():
    rng = np.random.default_rng(65)
    B, H, D, ps, maxp = 2, 2, 16, 4, 3
    table = rng.permutation(8)[:6].astype(np.int32).reshape(B, maxp)
    k = rng.normal(0, 1, (B, H, 7, D)).astype(np.float32)
    v = rng.normal(0, 1, (B, H, 7, D)).astype(np.float32)
    y = (k[:, :, :2] * F32(2.5)).astype(np.float32)
    w = (v[:, :, :2] * F32(-3)).astype(np.float32)
    pg = OracleCache(B, H, H, D, oracle.INT8_SYM_PER_TENSOR, oracle.UINT8_ASYM_PER_CHANNEL, paged=True,
                     page_size=ps, max_pages=maxp, num_pages=8, page_table=table)
    dn = OracleCache(B, H, H, D, oracle.INT8_SYM_PER_TENSOR, oracle.UINT8_ASYM_PER_CHANNEL, cap=12)
    pg.append(k, v, bf16=False, calibrate=True, new_lens=np.array([7, 7], np.int32))
    dn.append(k, v, bf16=False, calibrate=True)
    pg.append(y, w, bf16=False, rescale=True, new_lens=np.array([2, 2], np.int32))
    dn.append(y, w, bf16=False, rescale=True)
    for n in ("k_scale", "v_scale", "v_zp"):
        assert np.array_equal(pg[n], dn[n]), n
    for b in range(B):
        for t in range(9):
            page, slot = table[b, t // ps], t % ps
            assert np.array_equal(pg["k_codes"][page, :, slot], dn["k_codes"][b, :, t])
            assert np.array_equal(pg["v_codes"][page, :, slot], dn["v_codes"][b, :, t])


# --------------------------------------------------------------- INT4 symmetric per group
# llms.blog §2 "INT4 Group-Wise": groups of 32-128 elements along the channel dimension;
# n4n.ai Step 2 "Per-group INT4" and its Step 3 code: scale = max|x| / 7, codes clamped to the
# signed 4-bit range. Groups here are 32 consecutive channels of one token.
def _int4_cache(B, H, cap=8, **kw):
    return OracleCache(B, H, H, 32 * 4, oracle.INT4_SYM_PER_GROUP, oracle.INT4_SYM_PER_GROUP, cap=cap, **kw)


def test_int4_group_scale_exact_grid_and_packing():
    s = 2.0**-3
    x = np.zeros((1, 1, 1, 128), np.float32)
    ks = np.array([(i % 15) - 7 for i in range(128)])
    x[0, 0, 0] = ks * s                          # every group holds -7..7, so absmax = 7 s
    c = _int4_cache(1, 1)
    c.append(x, x, bf16=False)
    assert np.all(c["k_scale"][0, 0, 0] == F32(s))   # (7 s) / 7 = s exactly
    row = c["k_codes"][0, 0, 0]
    assert row.shape == (64,)
    for d in range(128):
        nib = (int(row[d // 2]) >> (4 * (d % 2))) & 0xF  # lower channel in the low nibble
        val = nib - 16 if nib >= 8 else nib          # two's complement
        assert val == ks[d], d
    assert np.array_equal(c.dequantize(0, 8)[0, 0, 0], x[0, 0, 0])


def test_int4_code_is_nearest_level_and_clamped():
    rng = np.random.default_rng(70)
    for _ in range(300):
        s = float(F32(rng.uniform(0.01, 3)))
        v = float(F32(rng.normal(0, 6 * s)))
        q = oracle.int4_code(v, s)
        r = Fraction(v) / Fraction(s)
        d = [abs(r - k) for k in range(-8, 8)]
        m = min(d)
        best = [k - 8 for k, e in enumerate(d) if e == m]
        half = math.floor(r) + Fraction(1, 2)
        if len(best) > 1:
            assert q in best and q % 2 == 0
        elif abs(r - half) <= abs(r) * Fraction(1, 2**24) and -8 < math.floor(r) < 7:
            assert q in (math.floor(r), math.floor(r) + 1)
        else:
            assert q == best[0]
    assert oracle.int4_code(100.0, 1.0) == 7 and oracle.int4_code(-100.0, 1.0) == -8
    assert oracle.int4_code(3.0, 0.0) == 0


def test_int4_groups_are_channel_slices_of_one_token():
    rng = np.random.default_rng(71)
    B, H, T = 2, 2, 5
    x = rng.normal(0, 1, (B, H, T, 128)).astype(np.float32)
    y = x.copy()
    y[1, 0, 3, 70] = 40.0                        # group 2 of token 3 of (b=1, h=0)
    a, b = _int4_cache(B, H), _int4_cache(B, H)
    a.append(x, x, bf16=False)
    b.append(y, y, bf16=False)
    diff = a["k_scale"] != b["k_scale"]
    assert diff.sum() == 1 and diff[1, 0, 3, 2]
    assert b["k_scale"][1, 0, 3, 2] == F32(40.0) / F32(7)
    changed = np.argwhere(a["k_codes"] != b["k_codes"])
    assert len(changed) and all((r[0], r[1], r[2]) == (1, 0, 3) and 64 <= 2 * r[3] < 96 for r in changed)
    for g in range(4):                           # per-group scale is the group's absmax / 7
        amax = np.abs(x[0, 1, 2, 32 * g:32 * (g + 1)]).max()
        assert a["k_scale"][0, 1, 2, g] == F32(amax) / F32(7)


def test_int4_dequant_within_half_step_and_zero_group():
    rng = np.random.default_rng(72)
    x = rng.normal(0, 2, (1, 2, 6, 128)).astype(np.float32)
    x[0, 1, 4, 96:] = 0.0                        # an all-zero group
    c = _int4_cache(1, 2)
    c.append(x, x, bf16=False)
    deq = c.dequantize(1, 8)[:, :, :6]
    s = np.repeat(c["v_scale"][:, :, :6], 32, axis=-1)
    assert np.all(np.abs(deq - x) <= s / 2 * (1 + 2**-20))
    assert c["v_scale"][0, 1, 4, 3] == 0 and not deq[0, 1, 4, 96:].any()


def test_int4_paged_matches_dense():
    rng = np.random.default_rng(73)
    B, H, ps, maxp = 2, 2, 4, 3
    table = rng.permutation(8)[:6].astype(np.int32).reshape(B, maxp)
    lens = np.array([7, 3], np.int32)
    x = rng.normal(0, 1, (B, H, 7, 128)).astype(np.float32)
    pg = _int4_cache(B, H, cap=0, paged=True, page_size=ps, max_pages=maxp, num_pages=8, page_table=table)
    dn = _int4_cache(B, H, cap=8)
    pg.append(x, x, bf16=False, new_lens=lens)
    dn.append(x, x, bf16=False)
    for b in range(B):
        for t in range(lens[b]):
            page, slot = table[b, t // ps], t % ps
            assert np.array_equal(pg["k_codes"][page, :, slot], dn["k_codes"][b, :, t])
            assert np.array_equal(pg["v_scale"][page, :, slot], dn["v_scale"][b, :, t])


# --------------------------------------------------------------- Walsh-Hadamard rotation
# llms.blog §5 (QuaRot / RotateKV): an orthogonal Hadamard rotation of K, V and Q spreads
# outlier channels before low-bit quantization and leaves q.k unchanged.
def _walsh(n, j):
    return np.array([(-1) ** bin(i & j).count("1") for i in range(n)], np.float64)


def test_fwht_basis_vectors_are_walsh_functions():
    c = F32(1.0 / math.sqrt(128.0))
    for j in (0, 1, 5, 64, 77, 127):
        e = np.zeros(128, np.float32)
        e[j] = 1.0
        assert np.array_equal(oracle.fwht(e), (_walsh(128, j) * float(c)).astype(np.float32)), j


def test_fwht_matches_the_hadamard_matrix_and_is_orthogonal():
    scipy_linalg = pytest.importorskip("scipy.linalg")
    Hm = scipy_linalg.hadamard(128).astype(np.float64) / math.sqrt(128.0)
    rng = np.random.default_rng(80)
    for _ in range(20):
        x = rng.normal(0, 3, 128).astype(np.float32)
        y = oracle.fwht(x).astype(np.float64)
        ref = Hm @ x.astype(np.float64)
        assert np.max(np.abs(y - ref)) <= 1e-6 * np.abs(x).sum()
        assert abs(np.linalg.norm(y) - np.linalg.norm(x)) <= 1e-6 * np.linalg.norm(x)   # Parseval
        z = oracle.fwht(oracle.fwht(x)).astype(np.float64)                              # own inverse
        assert np.max(np.abs(z - x)) <= 1e-6 * np.abs(x).max()


def test_rotated_cache_quantizes_the_rotated_rows():
    # codes and scales of a rotating cache are those of a plain cache fed H x
    rng = np.random.default_rng(81)
    B, H, T = 2, 2, 9
    k = rng.normal(0, 1, (B, H, T, 128)).astype(np.float32)
    v = rng.normal(0, 1, (B, H, T, 128)).astype(np.float32)
    k[..., 3] *= 30                              # an outlier channel
    kr = np.apply_along_axis(oracle.fwht, -1, k)
    vr = np.apply_along_axis(oracle.fwht, -1, v)
    for sch in (oracle.INT8_SYM_PER_TOKEN, oracle.INT4_SYM_PER_GROUP, oracle.FP8_E4M3_PER_TENSOR):
        a = OracleCache(B, H, H, 128, sch, sch, cap=16, rotate=True)
        b = OracleCache(B, H, H, 128, sch, sch, cap=16)
        a.append(k, v, bf16=False, calibrate=True)
        b.append(kr, vr, bf16=False, calibrate=True)
        for n in ("k_codes", "v_codes", "k_scale", "v_scale"):
            assert np.array_equal(a[n], b[n]), (sch, n)
        # dequantize returns the original domain: H applied to the rotated values
        back = np.apply_along_axis(oracle.fwht, -1, b.dequantize(0, 16)[:, :, :T])
        assert np.array_equal(a.dequantize(0, 16)[:, :, :T], back)


def test_rotated_decode_equals_attention_in_the_original_domain():
    rng = np.random.default_rng(82)
    B, Hq, H, T = 1, 4, 2, 40
    k = rng.normal(0, 1, (B, H, T, 128)).astype(np.float32)
    v = rng.normal(0, 1, (B, H, T, 128)).astype(np.float32)
    k[..., 7] *= 20
    c = OracleCache(B, Hq, H, 128, oracle.INT8_SYM_PER_TOKEN, oracle.INT8_SYM_PER_TOKEN, cap=64, rotate=True)
    c.append(k, v, bf16=False)
    q = rng.normal(0, 1, (B, Hq, 128)).astype(np.float32)
    out, lse = c.decode(q, bf16=False, scale=0.09)
    K, V = c.dequantize(0, T).astype(np.float64), c.dequantize(1, T).astype(np.float64)
    for h in range(Hq):
        s = K[0, h // 2] @ q[0, h].astype(np.float64) * float(F32(0.09))
        p = np.exp(s - s.max())
        ref = (p / p.sum()) @ V[0, h // 2]
        assert np.max(np.abs(out[0, h] - ref)) <= 1e-5 * np.abs(ref).max()
        assert abs(lse[0, h] - (s.max() + math.log(p.sum()))) <= 1e-5



@pytest.mark.parametrize("group", [64, 128])
def test_int4_larger_groups_share_one_scale(group):
    # groups of 64 or 128 channels (128: one scale per token, the page code's default)
    rng = np.random.default_rng(74 + group)
    B, H, T = 1, 2, 4
    x = rng.normal(0, 1, (B, H, T, 128)).astype(np.float32)
    c = OracleCache(B, H, H, 128, oracle.INT4_SYM_PER_GROUP, oracle.INT4_SYM_PER_GROUP, cap=8, group=group)
    c.append(x, x, bf16=False)
    assert c["k_scale"].shape == (B, H, 8, 128 // group)
    for h in range(H):
        for t in range(T):
            for j in range(128 // group):
                amax = np.abs(x[0, h, t, group * j:group * (j + 1)]).max()
                assert c["k_scale"][0, h, t, j] == F32(amax) / F32(7)
    d = c.dequantize(0, 8)[:, :, :T]
    s = np.repeat(c["k_scale"][:, :, :T], group, axis=-1)
    assert np.all(np.abs(d - x) <= s / 2 * (1 + 2**-20))


# --------------------------------------------------------------- KIVI with fp16 metadata
# Scale and minimum stored in fp16 (the tensor precision of the pages' cache code, n4n.ai
# Step 3), which halves KIVI's metadata: INT2 then takes 2 + 2 * 16 / 32 = 3 bits per element.
def test_f16_codec_matches_numpy():
    rng = np.random.default_rng(90)
    vals = np.concatenate([rng.normal(0, 1, 3000), rng.normal(0, 1e-5, 1000), rng.uniform(-65000, 65000, 1000),
                           [0.0, -0.0, 2.0**-24, 2.0**-25, 3 * 2.0**-26, 65504.0, 2.0**-14, 1 + 2.0**-11]])
    for v in vals.astype(np.float32):
        want = np.array([v], np.float32).astype(np.float16).view(np.uint16)[0]
        assert oracle.f16_encode(float(v)) == want, v
        assert oracle.f16_decode(int(want)) == np.float32(np.array([want], np.uint16).view(np.float16)[0])
    assert oracle.f16_encode(1e6) == 0x7BFF and oracle.f16_encode(-65520.0) == 0xFBFF  # saturating


@pytest.mark.parametrize("bits", [4, 2])
def test_kivi_f16_meta_is_the_rounded_fp32_meta_with_nearest_codes(bits):
    qmax = 2**bits - 1
    rng = np.random.default_rng(91 + bits)
    for _ in range(200):
        x = (rng.normal(0.3, 1.5, 32) * rng.uniform(0.01, 50)).astype(np.float32)
        _, s32, mn32 = oracle.kivi_group(x, bits)
        codes, s16, mn16 = oracle.kivi_group(x, bits, f16_meta=True)
        assert s16 == np.float32(np.float16(s32)) and mn16 == np.float32(np.float16(mn32))
        S, M = Fraction(float(s16)), Fraction(float(mn16))
        for v, q in zip(x, codes):
            d = [abs(Fraction(float(v)) - (k * S + M)) for k in range(qmax + 1)]
            # nearest level of the stored grid, up to the fp32 rounding of (x - min) / s
            assert d[q] <= min(d) + S * Fraction(1, 2**20), (v, q)


def test_kivi_f16_cache_layout_and_dequant():
    rng = np.random.default_rng(93)
    B, H = 1, 2
    x = rng.normal(0, 1, (B, H, 200, 128)).astype(np.float32)
    xb = (x.view(np.uint32) >> 16).astype(np.uint16)          # bf16 bits (truncated; any bf16 will do)
    a = OracleCache(B, 4, H, 128, oracle.KIVI_INT2_F16, oracle.KIVI_INT2_F16, cap=256)
    b = OracleCache(B, 4, H, 128, oracle.KIVI_INT2, oracle.KIVI_INT2, cap=256)
    a.append(xb, xb, bf16=True)
    b.append(xb, xb, bf16=True)
    assert a.length == b.length == 128 and a.residual == b.residual == 72
    for side in ("k", "v"):
        s16, s32 = a[side + "_scale"], b[side + "_scale"]
        assert np.array_equal(s16, s32.astype(np.float16).astype(np.float32))
        z16, z32 = a[side + "_zero"], b[side + "_zero"]
        assert np.array_equal(z16, z32.astype(np.float16).astype(np.float32))
    # the residual (bf16) is untouched by the metadata precision
    assert np.array_equal(a["k_res"], b["k_res"])
    d = a.dequantize(1, 256)[:, :, :128].astype(np.float64)
    xf = synth_bf16(xb)[:, :, :128]
    s = np.repeat(a["v_scale"][:, :, :128], 32, axis=-1)
    assert np.all(np.abs(d - xf) <= s * 0.5 + np.abs(xf) * 2.0**-10 + 2.0**-24)


def synth_bf16(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


# --------------------------------------------------------------- pre-RoPE keys (KVQuant)
# llms.blog §4: KVQuant quantizes keys before the rotary embedding, whose position-dependent
# rotation would otherwise mix the outlier channels; decode rotates each dequantized key.
def test_rope_equals_the_complex_rotation():
    rng = np.random.default_rng(100)
    theta = 500000.0
    for pos in (0, 1, 7, 4095, 131071):
        x = rng.normal(0, 1, 128)
        z = (x[:64] + 1j * x[64:]) * np.exp(1j * pos * theta ** (-np.arange(64) * 2.0 / 128))
        y = oracle.rope(x, pos, theta)
        assert np.max(np.abs(y - np.concatenate([z.real, z.imag]))) <= 1e-12 * np.abs(x).sum()
        assert abs(np.linalg.norm(y) - np.linalg.norm(x)) <= 1e-12 * np.linalg.norm(x)
    assert np.array_equal(oracle.rope(np.arange(128.0), 0, theta), np.arange(128.0))   # position 0


def test_rope_scores_depend_on_relative_position():
    rng = np.random.default_rng(101)
    q, k = rng.normal(0, 1, 128), rng.normal(0, 1, 128)
    a = oracle.rope(q, 1000, 10000.0) @ oracle.rope(k, 990, 10000.0)
    b = oracle.rope(q, 10, 10000.0) @ oracle.rope(k, 0, 10000.0)
    assert abs(a - b) <= 1e-9 * np.abs(q).sum() * np.abs(k).sum()


@pytest.mark.parametrize("scheme", [oracle.INT8_SYM_PER_CHANNEL, oracle.KIVI_INT4])
def test_pre_rope_decode_rotates_each_dequantized_key_at_its_position(scheme):
    rng = np.random.default_rng(102)
    B, Hq, H, T = 1, 4, 2, 150
    k = rng.normal(0, 1, (B, H, T, 128)).astype(np.float32)
    v = rng.normal(0, 1, (B, H, T, 128)).astype(np.float32)
    k[..., 5] *= 20
    bf16 = scheme == oracle.KIVI_INT4
    if bf16:  # KIVI takes bf16 inputs
        k = (k.view(np.uint32) >> 16).astype(np.uint16)
        v = (v.view(np.uint32) >> 16).astype(np.uint16)
    c = OracleCache(B, Hq, H, 128, scheme, scheme, cap=256, rope_theta=10000.0)
    c.append(k, v, bf16=bf16, calibrate=scheme != oracle.KIVI_INT4)
    q = rng.normal(0, 1, (B, Hq, 128)).astype(np.float32)
    out, lse = c.decode(q, bf16=False, scale=0.09)
    K, V = c.dequantize(0, T).astype(np.float64), c.dequantize(1, T).astype(np.float64)
    Kr = np.stack([np.stack([oracle.rope(K[0, h, t], t, 10000.0) for t in range(T)]) for h in range(H)])
    for h in range(Hq):
        s = Kr[h // 2] @ q[0, h].astype(np.float64) * float(F32(0.09))
        p = np.exp(s - s.max())
        ref = (p / p.sum()) @ V[0, h // 2]
        assert np.max(np.abs(out[0, h] - ref)) <= 1e-9 * np.abs(ref).max()
        assert abs(lse[0, h] - (s.max() + math.log(p.sum()))) <= 1e-9
    # the cache itself holds the keys as given (dequantize returns pre-RoPE values)
    plain = OracleCache(B, Hq, H, 128, scheme, scheme, cap=256)
    plain.append(k, v, bf16=bf16, calibrate=scheme != oracle.KIVI_INT4)
    assert np.array_equal(plain["k_codes"], c["k_codes"])

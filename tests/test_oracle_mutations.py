"""Planted mistakes in the oracle must fail its pins.

Each case copies kvq_oracle.c, applies one plausible mistake (a wrong constant, a
dropped term, a wrong sign, a transposed operand, a wrong index), compiles the copy on
the CPU and runs the pin tests against it. A mutation no pin catches would mean the
pins do not constrain that part of the oracle.
"""
import inspect
import os
import subprocess

import pytest

import oracle
from tests import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "kvq_oracle.c")

MUTATIONS = [
    ("per-tensor qmax 128", "scheme == OQ_FP8_E5M2_PER_TENSOR ? 57344.0f : 127.0f);",
     "scheme == OQ_FP8_E5M2_PER_TENSOR ? 57344.0f : 128.0f);"),
    ("per-token qmax 128", "tok_scale = amax / 127.0f;", "tok_scale = amax / 128.0f;"),
    ("per-channel qmax 255", "scale[h * D + d] = amax / 127.0f;", "scale[h * D + d] = amax / 255.0f;"),
    ("round half away", "  float y = x / s;\n  float r = rintf(y);", "  float y = x / s;\n  float r = roundf(y);"),
    ("clamp -128", "if (r < (float)-qmax) r = (float)-qmax;", "if (r < (float)(-qmax - 1)) r = (float)(-qmax - 1);"),
    ("fp8 scale 240", "OQ_FP8_E4M3_PER_TENSOR ? 448.0f :", "OQ_FP8_E4M3_PER_TENSOR ? 240.0f :"),
    ("e5m2 scale 61440", "57344.0f : 127.0f", "61440.0f : 127.0f"),
    ("e5m2 bias", "v = ldexpf(1.0f + (float)M / 4.0f, E - 15);", "v = ldexpf(1.0f + (float)M / 4.0f, E - 14);"),
    ("e5m2 subnormal grid", "v = ldexpf((float)M, -16);", "v = ldexpf((float)M, -15);"),
    ("e4m3 bias", "v = ldexpf((float)(8 + m), e - 10);", "v = ldexpf((float)(8 + m), e - 9);"),
    ("e4m3 no saturation", "if (a > 448.0f) return (uint8_t)(sign | 0x7E);", "if (a > 480.0f) return (uint8_t)(sign | 0x7F);"),
    ("asym zp sign", "float z = rintf(-lo / sc);", "float z = rintf(lo / sc);"),
    ("asym 256 levels", "float sc = (hi - lo) / 255.0f;", "float sc = (hi - lo) / 256.0f;"),
    ("asym page form", "float r = rintf(x / s) + (float)zp;", "float r = rintf(x / s);"),
    ("kivi dequant sign", "  return a + mn;", "  return a - mn;"),
    ("kivi no min shift", "float diff = x[(size_t)i * stride] - lo;", "float diff = x[(size_t)i * stride];"),
    ("kivi key axis transposed",
     "(kh ? oq_kivi_group_f16 : oq_kivi_group)(xk + (size_t)gi * g * D + d, g, D, kb, codes, &s, &mn);",
     "(kh ? oq_kivi_group_f16 : oq_kivi_group)(xk + (size_t)gi * g * D + (size_t)d * g % (g * D), g, 1, kb, codes, "
     "&s, &mn);"),
    ("kivi flush rule", "const int r_new = ((total - 1) % R) + 1;", "const int r_new = total % R;"),
    ("kivi pack order", "const int byte = d / per, sh = (d % per) * bits;",
     "const int byte = d / per, sh = (per - 1 - d % per) * bits;"),
    ("paged slot", "(size_t)(t % c->page_size);\n}", "(size_t)((t + 1) % c->page_size);\n}"),
    ("calibration skips last head", "      for (int h = 0; h < H; ++h)\n        for (int t = 0; t < block_len(k, b); ++t)\n          for (int d = 0; d < D; ++d) {\n            float a = fabsf",
     "      for (int h = 0; h < H - 1; ++h)\n        for (int t = 0; t < block_len(k, b); ++t)\n          for (int d = 0; d < D; ++d) {\n            float a = fabsf"),
    ("attention drops scale", "s[t] = acc * (double)scale;", "s[t] = acc;"),
    ("attention no max shift", "const double p = exp(s[t] - m);", "const double p = exp(s[t]);"),
    ("attention lse", "*lse = m + log(l);", "*lse = log(l);"),
    ("gqa mapping", "const int hq = hk * G + j;", "const int hq = j * c->Hkv + hk;"),
    ("bytes formula", "return 2.0 * bytes_per_elem *", "return bytes_per_elem *"),
    ("rescale keeps the smaller scale", "if (s_blk[i] > scale[i]) scale[i] = s_blk[i];",
     "if (s_blk[i] < scale[i]) scale[i] = s_blk[i];"),
    ("rescale keeps old codes", "put_code(codes, scheme, D, row, d, code_for(scheme, x, scale[i], z_new));",
     "(void)x;"),
    ("rescale requantizes with the old scale", "code_for(scheme, x, scale[i], z_new)",
     "code_for(scheme, x, s_old[i], z_new)"),
    ("rescale old range top", "(float)(255 - (int)zp_old[i]) * s_old[i]", "(float)(255 + (int)zp_old[i]) * s_old[i]"),
    ("rescale drops old low end", "lo_b < lo_o ? lo_b : lo_o", "lo_b"),
    ("int4 qmax 8", "const float s = amax / 7.0f;", "const float s = amax / 8.0f;"),
    ("int4 no sign extension", "(float)(q >= 8 ? q - 16 : q)", "(float)q"),
    ("int4 clamp -7", "if (r < -8.0f) r = -8.0f;", "if (r < -7.0f) r = -7.0f;"),
    ("int4 group amax from group 0", "for (int d = j * g; d < (j + 1) * g; ++d) {\n        float a = fabsf",
     "for (int d = 0; d < g; ++d) {\n        float a = fabsf"),
    ("fwht sign", "        x[j] = a + b;\n        x[j + h] = a - b;\n      }\n  const float c",
     "        x[j] = a + b;\n        x[j + h] = b - a;\n      }\n  const float c"),
    ("fwht unnormalised", "const float c = (float)(1.0 / sqrt((double)n));", "const float c = 1.0f;"),
    ("fwht skips last stage", "  for (int h = 1; h < n; h *= 2)\n    for (int i = 0; i < n; i += 2 * h)\n      for (int j = i; j < i + h; ++j) {\n        const float a",
     "  for (int h = 1; h < n / 2; h *= 2)\n    for (int i = 0; i < n; i += 2 * h)\n      for (int j = i; j < i + h; ++j) {\n        const float a"),
    ("decode query not rotated", "    if (c->rotate) oq_fwht(qr, D);", "    (void)0;"),
    ("decode output not rotated back", "    if (c->rotate) fwht_d(out + (size_t)j * D, D);", "    (void)0;"),
    ("dequantize not rotated back", "        if (c->rotate && t < T) oq_fwht(row, D);", "        (void)row;"),
    ("f16 exponent bias", "return (uint16_t)(sign | (uint16_t)(((E + 15) << 10) | ((int)m - 1024)));",
     "return (uint16_t)(sign | (uint16_t)(((E + 14) << 10) | ((int)m - 1024)));"),
    ("f16 subnormal grid", "    v = ldexpf((float)M, -24);", "    v = ldexpf((float)M, -23);"),
    ("kivi f16 codes from fp32 parameters", "float r = rintf((x[(size_t)i * stride] - mn16) / s16);",
     "float r = rintf((x[(size_t)i * stride] - lo) / sc);"),
    ("rope sine sign", "    x[i] = a * c - b * s;\n    x[i + half] = b * c + a * s;",
     "    x[i] = a * c + b * s;\n    x[i + half] = b * c - a * s;"),
    ("rope frequency exponent", "const double inv_freq = pow(theta, -2.0 * (double)i / (double)D);\n    const double ang = (double)pos",
     "const double inv_freq = pow(theta, -1.0 * (double)i / (double)D);\n    const double ang = (double)pos"),
    ("pre-rope position off by one", "oq_rope(kd + (size_t)t * D, D, t, (double)c->rope_theta);",
     "oq_rope(kd + (size_t)t * D, D, t + 1, (double)c->rope_theta);"),
    ("pre-rope keys not rotated", "  if (c->rope_theta > 0.0f) {  /* pre-RoPE keys", "  if (0) {  /* pre-RoPE keys"),
    ("rescale paged length", "const int len = c->paged ? c->seq_lens[b] : c->len;",
     "const int len = c->paged ? c->seq_lens[b] - 1 : c->len;"),
]


def _pin_tests():
    out = []
    for name, fn in inspect.getmembers(pins, inspect.isfunction):
        if not name.startswith("test_"):
            continue
        marks = getattr(fn, "pytestmark", [])
        params = [m for m in marks if m.name == "parametrize"]
        if params:
            argname, values = params[0].args
            for v in values:
                out.append((f"{name}[{v}]", lambda fn=fn, a=argname, v=v: fn(**{a: v})))
        else:
            out.append((name, fn))
    return out


@pytest.mark.parametrize("label,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_pins_catch_mutation(label, old, new, tmp_path):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor not unique or missing: {label}"
    mut = tmp_path / "kvq_oracle.c"
    mut.write_text(src.replace(old, new))
    (tmp_path / "kvq_oracle.h").write_text(open(SRC[:-2] + ".h").read())
    so = tmp_path / "libmut.so"
    subprocess.check_call(["gcc", *oracle.CFLAGS, "-o", str(so), str(mut), "-lm"])
    saved = oracle._lib
    oracle._lib = oracle.load(str(so))
    caught = []
    try:
        for name, fn in _pin_tests():
            try:
                fn()
            except (AssertionError, ValueError):
                caught.append(name)
                break
    finally:
        oracle._lib = saved
    assert caught, f"no pin failed for planted mistake: {label}"

"""CPU oracle for KV-cache quantize-on-append and decode attention.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this package.
The product path (``decode_attention_quantize_b200``) never imports it and has no CPU
fallback.

The arithmetic lives in ``kvq_oracle.c`` (single-threaded C, strict IEEE fp32 for
quantization, fp64 for attention); this module compiles it and holds the cache arrays
as numpy buffers laid out like the library's:

* dense codes ``[B, Hkv, cap, row_bytes]``; paged codes ``[num_pages, Hkv, page, row_bytes]``
* per-tensor scale ``[1]``; per-token scale ``[B, Hkv, cap]`` (paged ``[P, Hkv, page]``);
  per-channel scale ``[Hkv, D]`` (+ uint8 zero point ``[Hkv, D]``)
* KIVI key scale / minimum ``[B, Hkv, cap/32, D]``; value scale / minimum
  ``[B, Hkv, cap, D/32]``; bf16 residual ``[B, Hkv, 128, D]``
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "liboracle.so")
CFLAGS = ["-O2", "-ffp-contract=off", "-fno-fast-math", "-std=c11", "-fPIC", "-shared"]

FP8_E4M3_PER_TENSOR = 0
INT8_SYM_PER_TENSOR = 1
INT8_SYM_PER_TOKEN = 2
INT8_SYM_PER_CHANNEL = 3
UINT8_ASYM_PER_CHANNEL = 4
KIVI_INT4 = 5
KIVI_INT2 = 6
FP8_E5M2_PER_TENSOR = 7
INT4_SYM_PER_GROUP = 8
KIVI_INT4_F16 = 9   # KIVI with fp16 scale and minimum
KIVI_INT2_F16 = 10
APPEND_CALIBRATE, APPEND_RESCALE = 1, 2  # append modes (oq_append)

_lib = None


def build(force: bool = False) -> str:
    src = os.path.join(_HERE, "kvq_oracle.c")
    hdr = os.path.join(_HERE, "kvq_oracle.h")
    newest = max(os.path.getmtime(src), os.path.getmtime(hdr))
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < newest:
        subprocess.check_call(["gcc", *CFLAGS, "-o", _SO, src, "-lm"])
    return _SO


class _Cache(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int), ("Hq", ctypes.c_int), ("Hkv", ctypes.c_int), ("D", ctypes.c_int),
        ("k_scheme", ctypes.c_int), ("v_scheme", ctypes.c_int),
        ("paged", ctypes.c_int), ("cap", ctypes.c_int),
        ("page_size", ctypes.c_int), ("max_pages", ctypes.c_int), ("num_pages", ctypes.c_int),
        ("group", ctypes.c_int), ("rcap", ctypes.c_int),
        ("len", ctypes.c_int), ("res", ctypes.c_int),
        ("k_codes", ctypes.c_void_p), ("v_codes", ctypes.c_void_p),
        ("k_scale", ctypes.c_void_p), ("k_zero", ctypes.c_void_p),
        ("v_scale", ctypes.c_void_p), ("v_zero", ctypes.c_void_p),
        ("k_zp", ctypes.c_void_p), ("v_zp", ctypes.c_void_p),
        ("k_res", ctypes.c_void_p), ("v_res", ctypes.c_void_p),
        ("page_table", ctypes.c_void_p), ("seq_lens", ctypes.c_void_p),
        ("rotate", ctypes.c_int),
        ("rope_theta", ctypes.c_float),
    ]


def lib():
    global _lib
    if _lib is None:
        _lib = load(build())
    return _lib


def load(path: str):
    """Load a compiled oracle library and declare its C signatures."""
    L = ctypes.CDLL(path)
    vp, i32, f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    L.oq_e4m3_encode.argtypes = [f32]
    L.oq_e4m3_encode.restype = ctypes.c_uint8
    L.oq_e4m3_decode.argtypes = [ctypes.c_uint8]
    L.oq_e4m3_decode.restype = f32
    L.oq_e5m2_encode.argtypes = [f32]
    L.oq_e5m2_encode.restype = ctypes.c_uint8
    L.oq_e5m2_decode.argtypes = [ctypes.c_uint8]
    L.oq_e5m2_decode.restype = f32
    L.oq_sym_code.argtypes = [f32, f32, i32]
    L.oq_sym_code.restype = i32
    L.oq_int4_code.argtypes = [f32, f32]
    L.oq_int4_code.restype = i32
    L.oq_asym_params.argtypes = [f32, f32, vp, vp]
    L.oq_asym_code.argtypes = [f32, f32, ctypes.c_uint8]
    L.oq_asym_code.restype = i32
    L.oq_kivi_group.argtypes = [vp, i32, i32, i32, vp, vp, vp]
    L.oq_kivi_group_f16.argtypes = [vp, i32, i32, i32, vp, vp, vp]
    L.oq_f16_encode.argtypes = [f32]
    L.oq_f16_encode.restype = ctypes.c_uint16
    L.oq_f16_decode.argtypes = [ctypes.c_uint16]
    L.oq_f16_decode.restype = f32
    L.oq_kivi_value.argtypes = [i32, f32, f32]
    L.oq_kivi_value.restype = f32
    L.oq_append.argtypes = [ctypes.POINTER(_Cache), vp, vp, i32, i32, vp, i32]
    L.oq_append.restype = i32
    L.oq_calibrate.argtypes = [ctypes.POINTER(_Cache), vp, vp, i32, i32, vp]
    L.oq_fwht.argtypes = [vp, i32]
    L.oq_rope.argtypes = [vp, i32, i32, ctypes.c_double]
    L.oq_rope.restype = None
    L.oq_fwht.restype = None
    L.oq_calibrate.restype = i32
    L.oq_tokens.argtypes = [ctypes.POINTER(_Cache), i32]
    L.oq_tokens.restype = i32
    L.oq_dequantize.argtypes = [ctypes.POINTER(_Cache), i32, vp, i32]
    L.oq_attention_row.argtypes = [vp, vp, vp, i32, i32, f32, vp, vp]
    L.oq_decode.argtypes = [ctypes.POINTER(_Cache), vp, i32, f32, vp, vp]
    L.oq_decode_pairs.argtypes = [ctypes.POINTER(_Cache), vp, i32, f32, vp, i32, vp, vp]
    L.oq_kv_bytes_per_token.argtypes = [i32, i32, i32, ctypes.c_double]
    L.oq_kv_bytes_per_token.restype = ctypes.c_double
    return L


def _ptr(a):
    return None if a is None else a.ctypes.data


# ---------------------------------------------------------------- element codecs
def e4m3_encode(x: float) -> int:
    return int(lib().oq_e4m3_encode(float(x)))


def e4m3_decode(code: int) -> float:
    return float(lib().oq_e4m3_decode(int(code)))


def e5m2_encode(x: float) -> int:
    return int(lib().oq_e5m2_encode(float(x)))


def e5m2_decode(code: int) -> float:
    return float(lib().oq_e5m2_decode(int(code)))


def sym_code(x: float, s: float, qmax: int = 127) -> int:
    return int(lib().oq_sym_code(float(x), float(s), qmax))


def int4_code(x: float, s: float) -> int:
    return int(lib().oq_int4_code(float(x), float(s)))


def rope(x, pos: int, theta: float) -> np.ndarray:
    """Rotate-half RoPE of a row at position pos (fp64)."""
    y = np.array(x, np.float64, copy=True)
    lib().oq_rope(y.ctypes.data, int(y.size), int(pos), float(theta))
    return y


def fwht(x) -> np.ndarray:
    """Normalised Walsh-Hadamard transform of a float32 vector (length a power of two)."""
    y = np.array(x, np.float32, copy=True)
    lib().oq_fwht(y.ctypes.data, int(y.size))
    return y


def asym_params(mn: float, mx: float):
    s = np.zeros(1, np.float32)
    zp = np.zeros(1, np.uint8)
    lib().oq_asym_params(float(mn), float(mx), s.ctypes.data, zp.ctypes.data)
    return s[0], int(zp[0])


def asym_code(x: float, s: float, zp: int) -> int:
    return int(lib().oq_asym_code(float(x), float(s), int(zp)))


def kivi_group(x: np.ndarray, bits: int, f16_meta: bool = False):
    x = np.ascontiguousarray(x, dtype=np.float32)
    codes = np.zeros(x.size, np.int32)
    s = np.zeros(1, np.float32)
    mn = np.zeros(1, np.float32)
    fn = lib().oq_kivi_group_f16 if f16_meta else lib().oq_kivi_group
    fn(x.ctypes.data, x.size, 1, bits, codes.ctypes.data, s.ctypes.data, mn.ctypes.data)
    return codes, s[0], mn[0]


def f16_encode(x: float) -> int:
    return int(lib().oq_f16_encode(float(x)))


def f16_decode(h: int) -> float:
    return float(lib().oq_f16_decode(int(h)))


def kivi_value(code: int, s: float, mn: float) -> float:
    return float(lib().oq_kivi_value(int(code), float(s), float(mn)))


def attention_row(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float):
    q = np.ascontiguousarray(q, np.float32)
    k = np.ascontiguousarray(k, np.float32)
    v = np.ascontiguousarray(v, np.float32)
    T, D = k.shape
    out = np.zeros(D, np.float64)
    lse = np.zeros(1, np.float64)
    lib().oq_attention_row(q.ctypes.data, k.ctypes.data, v.ctypes.data, T, D, float(scale),
                           out.ctypes.data, lse.ctypes.data)
    return out, lse[0]


def kv_bytes_per_token(n_layers: int, n_kv_heads: int, d_head: int, bytes_per_elem: float) -> float:
    return float(lib().oq_kv_bytes_per_token(n_layers, n_kv_heads, d_head, float(bytes_per_elem)))


def _bits(scheme):
    return {KIVI_INT4: 4, KIVI_INT2: 2, INT4_SYM_PER_GROUP: 4, KIVI_INT4_F16: 4, KIVI_INT2_F16: 2}.get(scheme, 8)


# ---------------------------------------------------------------- cache
class OracleCache:
    """Oracle cache with numpy arrays in the library's layouts (see module docstring)."""

    def __init__(self, B, Hq, Hkv, D, k_scheme, v_scheme, cap=0, paged=False, page_size=16,
                 max_pages=0, num_pages=0, page_table=None, group=32, rcap=128, rotate=False,
                 rope_theta=0.0):
        self.B, self.Hq, self.Hkv, self.D = B, Hq, Hkv, D
        self.k_scheme, self.v_scheme = k_scheme, v_scheme
        self.paged, self.cap, self.page_size = paged, cap, page_size
        self.max_pages, self.num_pages = max_pages, num_pages
        self.group, self.rcap = group, rcap
        self.arrays = {}
        for side, scheme in (("k", k_scheme), ("v", v_scheme)):
            rb = D * _bits(scheme) // 8
            if paged:
                self.arrays[side + "_codes"] = np.zeros((num_pages, Hkv, page_size, rb), np.uint8)
            else:
                self.arrays[side + "_codes"] = np.zeros((B, Hkv, cap, rb), np.uint8)
            scale = zero = zp = None
            if scheme in (FP8_E4M3_PER_TENSOR, FP8_E5M2_PER_TENSOR, INT8_SYM_PER_TENSOR):
                scale = np.zeros(1, np.float32)
            elif scheme == INT8_SYM_PER_TOKEN:
                scale = np.zeros((num_pages, Hkv, page_size) if paged else (B, Hkv, cap), np.float32)
            elif scheme in (INT8_SYM_PER_CHANNEL, UINT8_ASYM_PER_CHANNEL):
                scale = np.zeros((Hkv, D), np.float32)
                if scheme == UINT8_ASYM_PER_CHANNEL:
                    zp = np.zeros((Hkv, D), np.uint8)
            elif scheme == INT4_SYM_PER_GROUP:
                rows = (num_pages, Hkv, page_size) if paged else (B, Hkv, cap)
                scale = np.zeros((*rows, D // group), np.float32)
            else:
                shape = (B, Hkv, cap // group, D) if side == "k" else (B, Hkv, cap, D // group)
                scale = np.zeros(shape, np.float32)
                zero = np.zeros(shape, np.float32)
            self.arrays[side + "_scale"] = scale
            self.arrays[side + "_zero"] = zero
            self.arrays[side + "_zp"] = zp
        kivi = k_scheme in (KIVI_INT4, KIVI_INT2, KIVI_INT4_F16, KIVI_INT2_F16)
        self.arrays["k_res"] = np.zeros((B, Hkv, rcap, D), np.uint16) if kivi else None
        self.arrays["v_res"] = np.zeros((B, Hkv, rcap, D), np.uint16) if kivi else None
        self.arrays["page_table"] = (np.ascontiguousarray(page_table, np.int32)
                                     if paged else None)
        self.arrays["seq_lens"] = np.zeros(B, np.int32) if paged else None
        self.c = _Cache(B, Hq, Hkv, D, k_scheme, v_scheme, int(paged), cap, page_size,
                        max_pages, num_pages, group, rcap, 0, 0)
        for name, arr in self.arrays.items():
            setattr(self.c, name, _ptr(arr))
        self.c.rotate = int(bool(rotate))
        self.rotate = bool(rotate)
        self.c.rope_theta = float(rope_theta)

    def __getitem__(self, name):
        return self.arrays[name]

    @property
    def length(self):
        return self.c.len

    @property
    def residual(self):
        return self.c.res

    def tokens(self, b=0):
        return int(lib().oq_tokens(ctypes.byref(self.c), b))

    def append(self, k, v, bf16: bool, calibrate=False, new_lens=None, rescale=False):
        """calibrate: scales from this block; rescale: merge this block's scales into the
        cached ones and requantize the cached codes whose scale grew (not both)."""
        if calibrate and rescale:
            raise ValueError("calibrate and rescale are exclusive")
        k = np.ascontiguousarray(k)
        v = np.ascontiguousarray(v)
        n_new = k.shape[2]
        nl = None if new_lens is None else np.ascontiguousarray(new_lens, np.int32)
        mode = APPEND_CALIBRATE if calibrate else (APPEND_RESCALE if rescale else 0)
        rc = lib().oq_append(ctypes.byref(self.c), k.ctypes.data, v.ctypes.data, int(bf16), n_new,
                             _ptr(nl), mode)
        if rc != 0:
            raise ValueError("oracle append rejected the call (capacity or arguments)")

    def calibrate(self, k, v, bf16: bool, new_lens=None):
        """Scales of the calibrating append for block k, v (nothing is quantized)."""
        k = np.ascontiguousarray(k)
        v = np.ascontiguousarray(v)
        nl = None if new_lens is None else np.ascontiguousarray(new_lens, np.int32)
        if lib().oq_calibrate(ctypes.byref(self.c), k.ctypes.data, v.ctypes.data, int(bf16), k.shape[2],
                              _ptr(nl)) != 0:
            raise ValueError("oracle calibrate rejected the call")

    def dequantize(self, which: int, T_out: int) -> np.ndarray:
        out = np.zeros((self.B, self.Hkv, T_out, self.D), np.float32)
        lib().oq_dequantize(ctypes.byref(self.c), which, out.ctypes.data, T_out)
        return out

    def decode(self, q, bf16: bool, scale: float):
        q = np.ascontiguousarray(q)
        out = np.zeros((self.B, self.Hq, self.D), np.float64)
        lse = np.zeros((self.B, self.Hq), np.float64)
        lib().oq_decode(ctypes.byref(self.c), q.ctypes.data, int(bf16), float(scale),
                        out.ctypes.data, lse.ctypes.data)
        return out, lse

    def decode_pairs(self, q, bf16: bool, scale: float, pairs):
        q = np.ascontiguousarray(q)
        pairs = np.ascontiguousarray(pairs, np.int32).reshape(-1, 2)
        G = self.Hq // self.Hkv
        out = np.zeros((len(pairs), G, self.D), np.float64)
        lse = np.zeros((len(pairs), G), np.float64)
        lib().oq_decode_pairs(ctypes.byref(self.c), q.ctypes.data, int(bf16), float(scale),
                              pairs.ctypes.data, len(pairs), out.ctypes.data, lse.ctypes.data)
        return out, lse

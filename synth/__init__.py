"""Seeded synthetic inputs shared by the oracle harness and the CUDA library harness.

Nothing here quantizes, dequantizes or attends: the module draws K, V, Q, sequence
lengths, residual lengths and page tables from a counter-based generator (``synth.c``)
and describes the five benchmark workloads by their shapes. Every array is a pure
function of the seed and the coordinates, so any slice (one batch row, one head) can
be regenerated independently of the rest.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "libkvqsynth.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile synth.c into libkvqsynth.so next to it (gcc, OpenMP)."""
    src = os.path.join(_HERE, "synth.c")
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(src):
        subprocess.check_call(
            ["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-std=c11", "-o", _SO, src, "-lm"]
        )
    return _SO


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_SO)
        u64, i32, dbl, vp = ctypes.c_uint64, ctypes.c_int, ctypes.c_double, ctypes.c_void_p
        lib.syn_keys.argtypes = [u64, i32, i32, i32, i32, i32, i32, i32, vp, i32, dbl, dbl, i32, vp]
        lib.syn_values.argtypes = [u64, i32, i32, i32, i32, i32, i32, i32, i32, vp]
        lib.syn_queries.argtypes = [u64, i32, i32, i32, i32, i32, i32, vp]
        lib.syn_lengths.argtypes = [u64, i32, i32, i32, vp]
        lib.syn_outlier_channels.argtypes = [u64, i32, i32, vp]
        lib.syn_uniform_int.argtypes = [u64, u64, i32]
        lib.syn_uniform_int.restype = i32
        lib.syn_permutation.argtypes = [u64, i32, vp]
        _lib = lib
    return _lib


def _out(shape, bf16: bool):
    return np.empty(shape, dtype=np.uint16 if bf16 else np.float32)


def outlier_channels(seed: int, D: int = 128, n: int = 4) -> np.ndarray:
    out = np.empty(n, dtype=np.int32)
    _load().syn_outlier_channels(seed, D, n, out.ctypes.data)
    return out


def keys(w: "Workload", b0, b1, h0, h1, t0, t1) -> np.ndarray:
    """Keys [b1-b0, h1-h0, t1-t0, D]; uint16 bf16 bits or float32 per ``w.bf16``."""
    out = _out((b1 - b0, h1 - h0, t1 - t0, w.D), w.bf16)
    outl = outlier_channels(w.seed, w.D, w.n_outliers)
    _load().syn_keys(w.seed, b0, b1, h0, h1, t0, t1, w.D, outl.ctypes.data, w.n_outliers,
                     float(w.outlier_scale), float(w.rope_theta), int(w.bf16), out.ctypes.data)
    return out


def values(w: "Workload", b0, b1, h0, h1, t0, t1) -> np.ndarray:
    out = _out((b1 - b0, h1 - h0, t1 - t0, w.D), w.bf16)
    _load().syn_values(w.seed, b0, b1, h0, h1, t0, t1, w.D, int(w.bf16), out.ctypes.data)
    return out


def queries(w: "Workload", step: int, b0: int, b1: int) -> np.ndarray:
    out = _out((b1 - b0, w.Hq, w.D), w.bf16)
    _load().syn_queries(w.seed, step, b0, b1, w.Hq, w.D, int(w.bf16), out.ctypes.data)
    return out


def lengths(seed: int, B: int, lo: int, hi: int) -> np.ndarray:
    out = np.empty(B, dtype=np.int32)
    _load().syn_lengths(seed, B, lo, hi, out.ctypes.data)
    return out


def uniform_int(seed: int, tag: int, n: int) -> int:
    return int(_load().syn_uniform_int(seed, tag, n))


def permutation(seed: int, n: int) -> np.ndarray:
    out = np.empty(n, dtype=np.int32)
    _load().syn_permutation(seed, n, out.ctypes.data)
    return out


def bf16_bits_to_f32(a: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to float32 (exact: the low 16 bits become zero)."""
    return (a.astype(np.uint32) << 16).view(np.float32)


# Scheme numbering used by every harness (the library header and the oracle each
# define the same integers independently).
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
KIVI_SCHEMES = (KIVI_INT4, KIVI_INT2, KIVI_INT4_F16, KIVI_INT2_F16)


@dataclass
class Workload:
    """Shape and generator recipe of one synthetic decode workload."""
    name: str
    seed: int
    B: int
    Hq: int
    Hkv: int
    D: int
    k_scheme: int
    v_scheme: int
    bf16: bool                      # inputs (K, V, Q) in bf16, else fp32
    outlier_scale: float
    n_outliers: int = 4
    rope_theta: float = 0.0         # 0 disables RoPE
    context: int = 0                # uniform prefill length (dense)
    paged: bool = False
    page_size: int = 16
    len_lo: int = 0                 # paged: lengths uniform on [len_lo, len_hi]
    len_hi: int = 0
    steps: int = 1                  # decode steps (each appends one token when append_per_step)
    append_per_step: bool = False
    residual_cap: int = 128
    group: int = 32
    rotate: bool = False            # Walsh-Hadamard rotation of K, V and Q
    prerope_theta: float = 0.0      # > 0: keys cached before RoPE (generated with rope_theta = 0),
                                    # RoPE with this base applied at decode
    extra: dict = field(default_factory=dict)

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def kivi(self) -> bool:
        return self.k_scheme in KIVI_SCHEMES

    def prefill_lengths(self) -> np.ndarray:
        """Prefill tokens per sequence."""
        if self.paged:
            return lengths(self.seed, self.B, self.len_lo, self.len_hi)
        return np.full(self.B, self.prefill_tokens(), dtype=np.int32)

    def prefill_tokens(self) -> int:
        """Dense prefill length. KIVI config 3 adds a seeded residual length r0 in [0,127]."""
        if self.kivi and self.extra.get("seeded_residual"):
            return self.context + uniform_int(self.seed, 0, self.residual_cap)
        return self.context + self.extra.get("prefill_extra", 0)

    def page_table(self, max_pages: int):
        """Seeded random page table: a permutation of a pool sized for prefill + steps."""
        lens = self.prefill_lengths()
        need = [(int(L) + self.steps + self.page_size - 1) // self.page_size for L in lens]
        pool = int(sum(need))
        perm = permutation(self.seed, pool)
        table = np.full((self.B, max_pages), -1, dtype=np.int32)
        off = 0
        for b, n in enumerate(need):
            table[b, :n] = perm[off:off + n]
            off += n
        return table, pool


_OVERRIDES: dict = {}


def register_workload(w: "Workload") -> None:
    """Replace a named workload's shape for this process (e.g. a reduced batch for profiling)."""
    _OVERRIDES[w.name] = w


def workloads() -> dict:
    table = _base_workloads()
    table.update(_OVERRIDES)
    return table


def _base_workloads() -> dict:
    """The workloads: tiny INT8, FP8 E4M3 and FP8 E5M2 8B-shaped, KIVI-4 and INT4 per-group
    70B-shaped (INT4 with groups of 32, also with the Walsh-Hadamard rotation, and with groups
    of 128; same inputs), KIVI-2 131K, the two KIVI shapes with fp16 scale and minimum (same
    inputs as their fp32-metadata twins), the FP8 8B shape with keys cached before RoPE (RoPE
    applied at decode), paged INT8."""
    return {
        "tiny_int8": Workload(
            name="tiny_int8", seed=1, B=1, Hq=1, Hkv=1, D=128,
            k_scheme=INT8_SYM_PER_TOKEN, v_scheme=INT8_SYM_PER_TOKEN, bf16=False,
            outlier_scale=20.0, context=256),
        "fp8_8b": Workload(
            name="fp8_8b", seed=2, B=32, Hq=32, Hkv=8, D=128,
            k_scheme=FP8_E4M3_PER_TENSOR, v_scheme=FP8_E4M3_PER_TENSOR, bf16=True,
            outlier_scale=20.0, rope_theta=500000.0, context=4096),
        "e5m2_8b": Workload(
            name="e5m2_8b", seed=6, B=32, Hq=32, Hkv=8, D=128,
            k_scheme=FP8_E5M2_PER_TENSOR, v_scheme=FP8_E5M2_PER_TENSOR, bf16=True,
            outlier_scale=20.0, rope_theta=500000.0, context=4096),
        "fp8_8b_prerope": Workload(
            name="fp8_8b_prerope", seed=2, B=32, Hq=32, Hkv=8, D=128,
            k_scheme=FP8_E4M3_PER_TENSOR, v_scheme=FP8_E4M3_PER_TENSOR, bf16=True,
            outlier_scale=20.0, rope_theta=0.0, prerope_theta=500000.0, context=4096),
        "kivi4_70b": Workload(
            name="kivi4_70b", seed=3, B=16, Hq=64, Hkv=8, D=128,
            k_scheme=KIVI_INT4, v_scheme=KIVI_INT4, bf16=True,
            outlier_scale=20.0, rope_theta=500000.0, context=32768,
            extra={"seeded_residual": True}),
        "int4g_70b": Workload(
            name="int4g_70b", seed=7, B=16, Hq=64, Hkv=8, D=128,
            k_scheme=INT4_SYM_PER_GROUP, v_scheme=INT4_SYM_PER_GROUP, bf16=True,
            outlier_scale=20.0, rope_theta=500000.0, context=32768),
        "int4g_rot_70b": Workload(
            name="int4g_rot_70b", seed=7, B=16, Hq=64, Hkv=8, D=128,
            k_scheme=INT4_SYM_PER_GROUP, v_scheme=INT4_SYM_PER_GROUP, bf16=True,
            outlier_scale=20.0, rope_theta=500000.0, context=32768, rotate=True),
        "int4g128_70b": Workload(
            name="int4g128_70b", seed=7, B=16, Hq=64, Hkv=8, D=128,
            k_scheme=INT4_SYM_PER_GROUP, v_scheme=INT4_SYM_PER_GROUP, bf16=True,
            outlier_scale=20.0, rope_theta=500000.0, context=32768, group=128),
        "kivi4f16_70b": Workload(
            name="kivi4f16_70b", seed=3, B=16, Hq=64, Hkv=8, D=128,
            k_scheme=KIVI_INT4_F16, v_scheme=KIVI_INT4_F16, bf16=True,
            outlier_scale=20.0, rope_theta=500000.0, context=32768,
            extra={"seeded_residual": True}),
        "kivi2f16_131k": Workload(
            name="kivi2f16_131k", seed=4, B=4, Hq=64, Hkv=8, D=128,
            k_scheme=KIVI_INT2_F16, v_scheme=KIVI_INT2_F16, bf16=True,
            outlier_scale=100.0, rope_theta=500000.0, context=131072,
            extra={"prefill_extra": 128}),
        "kivi2_131k": Workload(
            name="kivi2_131k", seed=4, B=4, Hq=64, Hkv=8, D=128,
            k_scheme=KIVI_INT2, v_scheme=KIVI_INT2, bf16=True,
            outlier_scale=100.0, rope_theta=500000.0, context=131072,
            extra={"prefill_extra": 128}),
        "paged_int8": Workload(
            name="paged_int8", seed=5, B=64, Hq=32, Hkv=8, D=128,
            k_scheme=INT8_SYM_PER_TENSOR, v_scheme=UINT8_ASYM_PER_CHANNEL, bf16=True,
            outlier_scale=20.0, rope_theta=500000.0, paged=True, page_size=16,
            len_lo=1024, len_hi=32768, steps=128, append_per_step=True),
    }

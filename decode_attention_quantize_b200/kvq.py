"""Thin ctypes binding of libkvq (argument marshalling only).

Every step of the path runs in the CUDA library: this module turns torch tensors into
device pointers and calls the C entry points of the same names. PyTorch provides device
memory and streams. There is no CPU fallback: if ``libkvq.so`` is missing the import
fails, and every call requires CUDA tensors.
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libkvq.so")

# enums (mirror include/kvq.h)
KVQ_OK, KVQ_ERR_INVALID_ARG, KVQ_ERR_UNSUPPORTED, KVQ_ERR_CAPACITY, KVQ_ERR_WORKSPACE, KVQ_ERR_CUDA = range(6)
FP8_E4M3_PER_TENSOR = 0
INT8_SYM_PER_TENSOR = 1
INT8_SYM_PER_TOKEN = 2
INT8_SYM_PER_CHANNEL = 3
UINT8_ASYM_PER_CHANNEL = 4
KIVI_INT4 = 5
KIVI_INT2 = 6
FP8_E5M2_PER_TENSOR = 7
INT4_SYM_PER_GROUP = 8
KIVI_INT4_F16 = 9    # KIVI with fp16 scale and minimum
KIVI_INT2_F16 = 10
KIVI_SCHEMES = (KIVI_INT4, KIVI_INT2, KIVI_INT4_F16, KIVI_INT2_F16)
KVQ_F32, KVQ_BF16 = 0, 1
KVQ_DENSE, KVQ_PAGED = 0, 1
KVQ_ROTATE_NONE, KVQ_ROTATE_HADAMARD = 0, 1
KVQ_APPEND_CALIBRATE = 0x1
KVQ_APPEND_RESCALE = 0x2
KVQ_DEV_BAD_PAGE, KVQ_DEV_BAD_LENGTH, KVQ_DEV_TIMEOUT = 0x1, 0x2, 0x4

EXPORTS = [
    "kvq_abi_version", "kvq_status_string", "kvq_validate", "kvq_cache_bytes",
    "kvq_append_workspace_bytes", "kvq_quantize_append", "kvq_dequantize",
    "kvq_decode_workspace_bytes", "kvq_decode_attention", "kvq_get_device_status", "kvq_launch_count",
    "kvq_decode_attention_noalloc", "kvq_check_bounded_wait", "kvq_append_decode",
]
NOALLOC_SCRATCH_BYTES = 8 << 20


class KvqDesc(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32), ("num_q_heads", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32), ("k_scheme", ctypes.c_int32), ("v_scheme", ctypes.c_int32),
        ("layout", ctypes.c_int32), ("capacity", ctypes.c_int32), ("page_size", ctypes.c_int32),
        ("max_pages_per_seq", ctypes.c_int32), ("num_pages", ctypes.c_int32),
        ("group_size", ctypes.c_int32), ("residual_cap", ctypes.c_int32),
        ("num_quantized", ctypes.c_int32), ("num_residual", ctypes.c_int32),
        ("k_codes", ctypes.c_void_p), ("v_codes", ctypes.c_void_p),
        ("k_scale", ctypes.c_void_p), ("k_zero", ctypes.c_void_p),
        ("v_scale", ctypes.c_void_p), ("v_zero", ctypes.c_void_p),
        ("k_zp", ctypes.c_void_p), ("v_zp", ctypes.c_void_p),
        ("k_res", ctypes.c_void_p), ("v_res", ctypes.c_void_p),
        ("page_table", ctypes.c_void_p), ("seq_lens", ctypes.c_void_p),
        ("dev_status", ctypes.c_void_p),
        ("rotation", ctypes.c_int32),
        ("rope_theta", ctypes.c_float),
    ]


class KvqFootprint(ctypes.Structure):
    _fields_ = [("code_bytes", ctypes.c_uint64), ("meta_bytes", ctypes.c_uint64),
                ("residual_bytes", ctypes.c_uint64), ("total_bytes", ctypes.c_uint64),
                ("bytes_per_token", ctypes.c_double)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libkvq.so is not built ({LIB_PATH}); run decode_attention_quantize_b200/build.py")
    L = ctypes.CDLL(LIB_PATH)
    P = ctypes.POINTER(KvqDesc)
    vp, i32, u32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_uint32, ctypes.c_size_t
    L.kvq_abi_version.restype = ctypes.c_int
    L.kvq_status_string.argtypes = [ctypes.c_int]
    L.kvq_status_string.restype = ctypes.c_char_p
    L.kvq_validate.argtypes = [P]
    L.kvq_cache_bytes.argtypes = [P, ctypes.POINTER(KvqFootprint)]
    L.kvq_append_workspace_bytes.argtypes = [P, u32]
    L.kvq_append_workspace_bytes.restype = sz
    L.kvq_quantize_append.argtypes = [P, vp, vp, i32, i32, vp, u32, vp, sz, vp]
    L.kvq_dequantize.argtypes = [P, i32, vp, i32, vp]
    L.kvq_decode_workspace_bytes.argtypes = [P]
    L.kvq_decode_workspace_bytes.restype = sz
    L.kvq_decode_attention.argtypes = [P, vp, i32, ctypes.c_float, vp, vp, vp, sz, vp]
    L.kvq_get_device_status.argtypes = [P, vp, i32, vp]
    L.kvq_launch_count.restype = ctypes.c_uint64
    L.kvq_append_decode.argtypes = [P, vp, vp, i32, i32, vp, i32, ctypes.c_float, vp, vp, vp, sz, vp]
    L.kvq_decode_attention_noalloc.argtypes = [P, vp, i32, ctypes.c_float, vp, vp, vp]
    L.kvq_decode_attention_noalloc.restype = ctypes.c_int
    L.kvq_check_bounded_wait.argtypes = [vp, vp]
    L.kvq_check_bounded_wait.restype = ctypes.c_int
    for name in ("kvq_validate", "kvq_cache_bytes", "kvq_quantize_append", "kvq_dequantize",
                 "kvq_decode_attention", "kvq_get_device_status", "kvq_append_decode"):
        getattr(L, name).restype = ctypes.c_int
    return L


lib = _load()


class KvqError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {lib.kvq_status_string(status).decode()} (status {status})")
        self.status = status


def _check(status: int, where: str):
    if status != KVQ_OK:
        raise KvqError(status, where)


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libkvq takes CUDA tensors only")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _dtype_code(t):
    if t.dtype == torch.bfloat16:
        return KVQ_BF16
    if t.dtype == torch.float32:
        return KVQ_F32
    raise ValueError(f"unsupported dtype {t.dtype}: bf16 or fp32")


def _need(cond: bool, what: str):
    if not cond:
        raise ValueError(what)


def _check_shape(t, shape, name):
    _need(t is not None and tuple(t.shape) == tuple(shape), f"{name}: shape {None if t is None else tuple(t.shape)}, "
                                                           f"expected {tuple(shape)}")


def _check_device(tensors, device):
    for name, t in tensors:
        if t is not None and t.is_cuda and device is not None and t.device != device:
            raise ValueError(f"{name} is on {t.device}, expected {device}")


def row_bytes(scheme: int, D: int = 128) -> int:
    return D * {KIVI_INT4: 4, KIVI_INT2: 2, INT4_SYM_PER_GROUP: 4, KIVI_INT4_F16: 4, KIVI_INT2_F16: 2}.get(scheme, 8) // 8


# ---------------------------------------------------------------- entry points
def kvq_quantize_append(desc: KvqDesc, k_new, v_new, new_lens=None, calibrate=False, workspace=None,
                        stream=None, rescale=False):
    """Quantize [B, Hkv, n, D] K/V (bf16 or fp32) and append them to the cache.
    calibrate: scales from this block; rescale: grow the scales to cover this block and
    requantize the cached codes whose scale changed."""
    flags = (KVQ_APPEND_CALIBRATE if calibrate else 0) | (KVQ_APPEND_RESCALE if rescale else 0)
    # the kernels index k_new / v_new / new_lens by the descriptor's shape: check them first
    _need(k_new is not None and v_new is not None and k_new.dim() == 4, "k_new, v_new: [B, Hkv, n, D] tensors")
    n = int(k_new.shape[2])
    _check_shape(k_new, (desc.batch, desc.num_kv_heads, n, desc.head_dim), "k_new")
    _check_shape(v_new, (desc.batch, desc.num_kv_heads, n, desc.head_dim), "v_new")
    _need(k_new.dtype == v_new.dtype, f"k_new and v_new dtypes differ ({k_new.dtype}, {v_new.dtype})")
    if new_lens is not None:
        _check_shape(new_lens, (desc.batch,), "new_lens")
        _need(new_lens.dtype == torch.int32, "new_lens: int32")
    _check_device([("v_new", v_new), ("new_lens", new_lens), ("workspace", workspace)], k_new.device)
    need = lib.kvq_append_workspace_bytes(ctypes.byref(desc), flags)
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=k_new.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.kvq_quantize_append(ctypes.byref(desc), _ptr(k_new), _ptr(v_new), _dtype_code(k_new),
                                   int(k_new.shape[2]), _ptr(new_lens), flags, _ptr(workspace), ws_bytes,
                                   _stream(stream)), "kvq_quantize_append")


def kvq_dequantize(desc: KvqDesc, which: int, out_tokens: int, out=None, stream=None, device="cuda"):
    if out is None:
        out = torch.empty((desc.batch, desc.num_kv_heads, out_tokens, desc.head_dim), dtype=torch.float32,
                          device=device)
    _check_shape(out, (desc.batch, desc.num_kv_heads, out_tokens, desc.head_dim), "out")
    _need(out.dtype == torch.float32, "out: float32")
    _check(lib.kvq_dequantize(ctypes.byref(desc), which, _ptr(out), out_tokens, _stream(stream)),
           "kvq_dequantize")
    return out


def kvq_decode_workspace_bytes(desc: KvqDesc) -> int:
    return int(lib.kvq_decode_workspace_bytes(ctypes.byref(desc)))


def decode_workspace(desc: KvqDesc, device) -> torch.Tensor:
    """A decode workspace for this descriptor (split partials and the paged plan; no contents
    need to be kept between calls)."""
    return torch.empty(kvq_decode_workspace_bytes(desc), dtype=torch.uint8, device=device)


def _check_decode_args(desc: KvqDesc, q, out, lse):
    _check_shape(q, (desc.batch, desc.num_q_heads, desc.head_dim), "q")
    _check_shape(out, (desc.batch, desc.num_q_heads, desc.head_dim), "out")
    _need(out.dtype == torch.float32, "out: float32")
    if lse is not None:
        _check_shape(lse, (desc.batch, desc.num_q_heads), "lse")
        _need(lse.dtype == torch.float32, "lse: float32")
    _check_device([("out", out), ("lse", lse)], q.device)


def kvq_decode_attention(desc: KvqDesc, q, softmax_scale: float, out=None, lse=None, workspace=None,
                         stream=None):
    """Decode attention of q [B, Hq, D] over the quantized cache; returns (out, lse)."""
    _need(q is not None and q.dim() == 3, "q: [B, Hq, D] tensor")
    if out is None:
        out = torch.empty(tuple(q.shape), dtype=torch.float32, device=q.device)
    _check_decode_args(desc, q, out, lse)
    if workspace is None:
        workspace = decode_workspace(desc, q.device)
    _check_device([("workspace", workspace)], q.device)
    _check(lib.kvq_decode_attention(ctypes.byref(desc), _ptr(q), _dtype_code(q), float(softmax_scale),
                                    _ptr(out), _ptr(lse), _ptr(workspace),
                                    workspace.numel() * workspace.element_size(), _stream(stream)),
           "kvq_decode_attention")
    return out, lse


def kvq_append_decode(desc: KvqDesc, k_new, v_new, q, softmax_scale: float, out=None, lse=None, workspace=None,
                      stream=None):
    """One decode step: a plain append of k_new / v_new [B, Hkv, n, D], then decode attention of
    q [B, Hq, D] over the updated cache; returns (out, lse)."""
    _need(k_new is not None and v_new is not None and k_new.dim() == 4, "k_new, v_new: [B, Hkv, n, D] tensors")
    n = int(k_new.shape[2])
    _check_shape(k_new, (desc.batch, desc.num_kv_heads, n, desc.head_dim), "k_new")
    _check_shape(v_new, (desc.batch, desc.num_kv_heads, n, desc.head_dim), "v_new")
    _need(k_new.dtype == v_new.dtype, f"k_new and v_new dtypes differ ({k_new.dtype}, {v_new.dtype})")
    _need(q is not None and q.dim() == 3, "q: [B, Hq, D] tensor")
    if out is None:
        out = torch.empty(tuple(q.shape), dtype=torch.float32, device=q.device)
    _check_decode_args(desc, q, out, lse)
    if workspace is None:
        workspace = decode_workspace(desc, q.device)
    _check_device([("k_new", k_new), ("v_new", v_new), ("workspace", workspace)], q.device)
    _check(lib.kvq_append_decode(ctypes.byref(desc), _ptr(k_new), _ptr(v_new), _dtype_code(k_new), n, _ptr(q),
                                 _dtype_code(q), float(softmax_scale), _ptr(out), _ptr(lse), _ptr(workspace),
                                 workspace.numel() * workspace.element_size(), _stream(stream)),
           "kvq_append_decode")
    return out, lse


def kvq_decode_attention_noalloc(desc: KvqDesc, q, softmax_scale: float, out=None, lse=None, stream=None):
    """kvq_decode_attention without a workspace: for callers that cannot allocate device
    memory (the library's static scratch array holds the partials; see include/kvq.h)."""
    _need(q is not None and q.dim() == 3, "q: [B, Hq, D] tensor")
    if out is None:
        out = torch.empty(tuple(q.shape), dtype=torch.float32, device=q.device)
    _check_decode_args(desc, q, out, lse)
    _check(lib.kvq_decode_attention_noalloc(ctypes.byref(desc), _ptr(q), _dtype_code(q), float(softmax_scale),
                                            _ptr(out), _ptr(lse), _stream(stream)),
           "kvq_decode_attention_noalloc")
    return out, lse


def kvq_get_device_status(desc: KvqDesc, clear=False, stream=None):
    buf = (ctypes.c_uint32 * 2)()
    _check(lib.kvq_get_device_status(ctypes.byref(desc), ctypes.cast(buf, ctypes.c_void_p), int(clear),
                                     _stream(stream)), "kvq_get_device_status")
    return int(buf[0]), int(buf[1])


def kvq_check_bounded_wait(status, stream=None):
    """Run the library's bounded-wait self-check (a wait that nothing completes); it sets
    KVQ_DEV_TIMEOUT in status[0] after about a second. `status`: CUDA int32/uint32 tensor [2]."""
    _check(lib.kvq_check_bounded_wait(_ptr(status), _stream(stream)), "kvq_check_bounded_wait")


def kvq_launch_count() -> int:
    return int(lib.kvq_launch_count())


def kvq_cache_bytes(desc: KvqDesc) -> KvqFootprint:
    f = KvqFootprint()
    _check(lib.kvq_cache_bytes(ctypes.byref(desc), ctypes.byref(f)), "kvq_cache_bytes")
    return f


# ---------------------------------------------------------------- cache allocation
@dataclass
class CacheSpec:
    B: int
    Hq: int
    Hkv: int
    k_scheme: int
    v_scheme: int
    capacity: int = 0            # dense tokens per row (multiple of 128)
    paged: bool = False
    page_size: int = 16
    max_pages: int = 0
    num_pages: int = 0
    D: int = 128
    rotate: bool = False         # Walsh-Hadamard rotation of K, V and Q (not with KIVI)
    group: int = 32              # INT4 per group: channels per group (32, 64 or 128); KIVI: 32
    rope_theta: float = 0.0      # > 0: keys cached before RoPE, rotated at decode (8-bit key schemes)


class RescaleSchedule:
    """When to rescale: n4n.ai Step 7 recomputes the scales of a growing cache every 1024
    new tokens. ``step(n)`` counts appended tokens and answers whether this append is the
    one that rescales (the count restarts there, and at a calibration)."""

    def __init__(self, every: int = 1024):
        if every <= 0:
            raise ValueError("every must be positive")
        self.every = every
        self.pending = 0

    def step(self, n_new: int) -> bool:
        self.pending += int(n_new)
        if self.pending >= self.every:
            self.pending = 0
            return True
        return False

    def reset(self):
        self.pending = 0


class QuantizedKVCache:
    """One layer's quantized cache in caller-owned (torch) device memory plus its descriptor.
    ``rescale_every`` > 0 makes every append that completes that many tokens a rescaling one."""

    def __init__(self, spec: CacheSpec, device="cuda", page_table=None, rescale_every: int = 0):
        s = spec
        self.spec = s
        self.schedule = RescaleSchedule(rescale_every) if rescale_every > 0 else None
        dev = torch.device(device)
        self.t = {}
        kivi = s.k_scheme in KIVI_SCHEMES
        rows = (s.num_pages, s.Hkv, s.page_size) if s.paged else (s.B, s.Hkv, s.capacity)
        for side, sch in (("k", s.k_scheme), ("v", s.v_scheme)):
            self.t[side + "_codes"] = torch.zeros(*rows, row_bytes(sch, s.D), dtype=torch.uint8, device=dev)
            if sch in (FP8_E4M3_PER_TENSOR, FP8_E5M2_PER_TENSOR, INT8_SYM_PER_TENSOR):
                self.t[side + "_scale"] = torch.zeros(4, dtype=torch.float32, device=dev)
            elif sch == INT8_SYM_PER_TOKEN:
                self.t[side + "_scale"] = torch.zeros(*rows, dtype=torch.float32, device=dev)
            elif sch == INT4_SYM_PER_GROUP:
                self.t[side + "_scale"] = torch.zeros(*rows, s.D // s.group, dtype=torch.float32, device=dev)
            elif sch in (INT8_SYM_PER_CHANNEL, UINT8_ASYM_PER_CHANNEL):
                self.t[side + "_scale"] = torch.zeros(s.Hkv, s.D, dtype=torch.float32, device=dev)
                if sch == UINT8_ASYM_PER_CHANNEL:
                    self.t[side + "_zp"] = torch.zeros(s.Hkv, s.D, dtype=torch.uint8, device=dev)
            else:
                shape = (s.B, s.Hkv, s.capacity // 32, s.D) if side == "k" else (s.B, s.Hkv, s.capacity, s.D // 32)
                meta = torch.float16 if sch in (KIVI_INT4_F16, KIVI_INT2_F16) else torch.float32
                self.t[side + "_scale"] = torch.zeros(*shape, dtype=meta, device=dev)
                self.t[side + "_zero"] = torch.zeros(*shape, dtype=meta, device=dev)
        if kivi:
            self.t["k_res"] = torch.zeros(s.B, s.Hkv, 128, s.D, dtype=torch.bfloat16, device=dev)
            self.t["v_res"] = torch.zeros(s.B, s.Hkv, 128, s.D, dtype=torch.bfloat16, device=dev)
        if s.paged:
            pt = torch.full((s.B, s.max_pages), -1, dtype=torch.int32) if page_table is None else page_table
            self.t["page_table"] = torch.as_tensor(pt, dtype=torch.int32).to(dev).contiguous()
            self.t["seq_lens"] = torch.zeros(s.B, dtype=torch.int32, device=dev)
        self.t["dev_status"] = torch.zeros(4, dtype=torch.int32, device=dev)
        d = KvqDesc()
        d.batch, d.num_q_heads, d.num_kv_heads, d.head_dim = s.B, s.Hq, s.Hkv, s.D
        d.k_scheme, d.v_scheme = s.k_scheme, s.v_scheme
        d.layout = KVQ_PAGED if s.paged else KVQ_DENSE
        d.capacity = s.capacity
        d.page_size, d.max_pages_per_seq, d.num_pages = s.page_size, s.max_pages, s.num_pages
        d.group_size, d.residual_cap = s.group, 128
        d.rotation = KVQ_ROTATE_HADAMARD if s.rotate else KVQ_ROTATE_NONE
        d.rope_theta = float(s.rope_theta)
        for name, tensor in self.t.items():
            setattr(d, name, tensor.data_ptr())
        self.desc = d
        self.device = dev
        self._decode_ws = None
        _check(lib.kvq_validate(ctypes.byref(d)), "kvq_validate")

    def __getitem__(self, name):
        return self.t[name]

    @property
    def num_quantized(self):
        return self.desc.num_quantized

    @property
    def num_residual(self):
        return self.desc.num_residual

    def append(self, k, v, new_lens=None, calibrate=False, workspace=None, stream=None, rescale=None):
        """rescale: True / False, or None to follow ``rescale_every`` (never when calibrating)."""
        if calibrate:
            if self.schedule is not None:
                self.schedule.reset()
            rescale = False
        elif rescale is None:
            rescale = self.schedule.step(k.shape[2]) if self.schedule is not None else False
        kvq_quantize_append(self.desc, k, v, new_lens=new_lens, calibrate=calibrate, workspace=workspace,
                            stream=stream, rescale=rescale)

    def dequantize(self, which: int, out_tokens: int, stream=None):
        return kvq_dequantize(self.desc, which, out_tokens, stream=stream, device=self.device)

    def decode(self, q, softmax_scale=None, out=None, lse=None, workspace=None, stream=None):
        """Without a workspace the cache's own (allocated at the first decode, kept) is used."""
        if softmax_scale is None:
            softmax_scale = 1.0 / math.sqrt(self.spec.D)
        if workspace is None:
            if self._decode_ws is None:
                self._decode_ws = decode_workspace(self.desc, self.device)
            workspace = self._decode_ws
        return kvq_decode_attention(self.desc, q, softmax_scale, out=out, lse=lse, workspace=workspace,
                                    stream=stream)

    def append_decode(self, k, v, q, softmax_scale=None, out=None, lse=None, workspace=None, stream=None):
        """One decode step: append k, v with the cache's scales as they are, then decode q. The
        decode of a dense 8-bit or INT4 cache starts reading the cached tiles while the append
        runs. Not with a rescaling schedule (use append, then decode)."""
        _need(self.schedule is None, "append_decode: the cache has a rescaling schedule")
        if softmax_scale is None:
            softmax_scale = 1.0 / math.sqrt(self.spec.D)
        if workspace is None:
            if self._decode_ws is None:
                self._decode_ws = decode_workspace(self.desc, self.device)
            workspace = self._decode_ws
        return kvq_append_decode(self.desc, k, v, q, softmax_scale, out=out, lse=lse, workspace=workspace,
                                 stream=stream)

    def status(self, clear=False):
        return kvq_get_device_status(self.desc, clear=clear)

    def footprint(self) -> KvqFootprint:
        return kvq_cache_bytes(self.desc)

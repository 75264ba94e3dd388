"""The algorithmic bytes behind bench.py's roofline figures, checked against the library's
own footprint formula (kvq_cache_bytes, computed in C from the descriptor) for every
workload, with no GPU: the per-token bytes a decode call must read are the codes plus the
per-token metadata of both sides."""
import ctypes
import os
import sys

import numpy as np
import pytest

import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _footprint(w):
    from decode_attention_quantize_b200 import kvq
    d = kvq.KvqDesc()
    d.batch, d.num_q_heads, d.num_kv_heads, d.head_dim = w.B, w.Hq, w.Hkv, 128
    d.k_scheme, d.v_scheme = w.k_scheme, w.v_scheme
    d.layout, d.capacity = kvq.KVQ_DENSE, 4096
    d.group_size, d.residual_cap = w.group, 128
    d.rotation = kvq.KVQ_ROTATE_HADAMARD if w.rotate else kvq.KVQ_ROTATE_NONE
    fake = 0x10000  # never dereferenced: the footprint is host arithmetic
    for f in ("k_codes", "v_codes", "k_scale", "v_scale", "k_zero", "v_zero", "k_zp", "v_zp", "k_res", "v_res",
              "dev_status"):
        setattr(d, f, fake)
    f = kvq.KvqFootprint()
    assert kvq.lib.kvq_cache_bytes(ctypes.byref(d), ctypes.byref(f)) == kvq.KVQ_OK
    return f


@pytest.mark.parametrize("name", [n for n, w in synth.workloads().items() if not w.paged])
def test_decode_bytes_match_the_library_footprint(name):
    w = synth.workloads()[name]
    f = _footprint(w)
    L = 1000
    lens = np.full(w.B, L)
    got = bench.decode_bytes(w, lens, 0)
    fixed = bench.fixed_meta_bytes(w.k_scheme, w.Hkv) + bench.fixed_meta_bytes(w.v_scheme, w.Hkv)
    qo = w.B * w.Hq * 128 * ((2 if w.bf16 else 4) + 4)
    assert got - fixed - qo == pytest.approx(w.B * w.Hkv * L * f.bytes_per_token, rel=1e-12)


def test_headline_decode_bytes():
    # fp8_8b: 32 x 8 x 4096 token rows of 128 + 128 code bytes, the two scales, bf16 Q, fp32 out
    w = synth.workloads()["fp8_8b"]
    got = bench.decode_bytes(w, np.full(w.B, 4096), 0)
    assert got == 32 * 8 * 4096 * 256 + 8 + 32 * 32 * 128 * (2 + 4)

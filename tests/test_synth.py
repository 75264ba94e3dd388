"""The shared input generator: deterministic, slice-independent, right shapes."""
import numpy as np

import synth


def test_slices_are_independent_of_the_request():
    w = synth.workloads()["fp8_8b"]
    full = synth.keys(w, 0, 2, 0, 3, 0, 40)
    part = synth.keys(w, 1, 2, 2, 3, 17, 23)
    assert np.array_equal(full[1:2, 2:3, 17:23], part)
    v = synth.values(w, 0, 2, 0, 3, 0, 40)
    assert np.array_equal(v[0:1, 1:2, 5:9], synth.values(w, 0, 1, 1, 2, 5, 9))
    q = synth.queries(w, 3, 0, 4)
    assert np.array_equal(q[2:4], synth.queries(w, 3, 2, 4))
    assert not np.array_equal(q, synth.queries(w, 4, 0, 4))


def test_outliers_and_sigma_recipe():
    w = synth.workloads()["tiny_int8"]          # fp32, no RoPE, outliers x20
    k = synth.keys(w, 0, 1, 0, 1, 0, 4096)[0, 0]
    outl = synth.outlier_channels(w.seed, 128, 4)
    assert len(set(outl.tolist())) == 4
    std = k.std(axis=0)
    assert np.all(std[outl] > 15) and np.all(np.delete(std, outl) < 1.2)
    v = synth.values(w, 0, 1, 0, 1, 0, 4096)[0, 0]
    row_std = v.std(axis=1)
    assert row_std.min() > 0.05 and row_std.max() < 15


def test_lengths_pages_and_residual():
    w = synth.workloads()["paged_int8"]
    L = w.prefill_lengths()
    assert L.min() >= 1024 and L.max() <= 32768 and len(L) == 64
    table, pool = w.page_table(max_pages=(32768 + 128) // 16 + 1)
    used = table[table >= 0]
    assert len(np.unique(used)) == len(used) == pool
    w3 = synth.workloads()["kivi4_70b"]
    assert 32768 <= w3.prefill_tokens() < 32768 + 128
    assert synth.workloads()["kivi2_131k"].prefill_tokens() == 131200


def test_bf16_rounding_is_exact_widening():
    w = synth.workloads()["fp8_8b"]
    k = synth.keys(w, 0, 1, 0, 1, 0, 8)
    f = synth.bf16_bits_to_f32(k)
    assert np.array_equal((f.view(np.uint32) >> 16).astype(np.uint16), k)

"""The seeded input generator (long_context_sparse_cca_b200/synth.py): the
same workload always gives the same bits; a reduced batch, length or head
count holds exactly the corresponding slices of the full inputs (the
benchmark's CPU baselines rely on this); the value distributions are the
ones the workloads state."""

import dataclasses

import numpy as np

from long_context_sparse_cca_b200 import synth


def test_deterministic_and_slice_consistent():
    wl = synth.GQA_16K
    a = synth.generate(wl, T=512, B=2)
    b = synth.generate(wl, T=512, B=2)
    for x, y in zip((a.q, a.k, a.v), (b.q, b.k, b.v)):
        assert np.array_equal(x, y)
    # fewer batch rows: the leading rows
    c = synth.generate(wl, T=512, B=1)
    assert np.array_equal(c.q, a.q[:1]) and np.array_equal(c.k, a.k[:1])
    # shorter: the leading tokens of every slice
    s = synth.generate(wl, T=256, B=2)
    assert np.array_equal(s.v, a.v[:, :, :256])


def test_single_head_workload_is_head_zero():
    dw = synth.DECODE_64K
    full = synth.generate(dw, T=300, B=2)
    one = synth.generate(dataclasses.replace(dw, B=1, Hq=1, Hkv=1), T=300)
    assert np.array_equal(one.q[0, 0], full.q[0, 0])
    assert np.array_equal(one.k[0, 0], full.k[0, 0])
    assert np.array_equal(one.v[0, 0], full.v[0, 0])


def test_value_distributions():
    wl = synth.PREFILL_32K
    x = synth.generate(wl, T=8192)
    q = synth.bf16_bits_to_f64(x.q)
    assert abs(q.mean()) < 0.01 and abs(q.std() - 1.0) < 0.01
    # heavy-hitter key rows: about 1% of rows, scaled by 4
    frac = x.heavy.mean()
    assert 0.008 < frac < 0.012
    k = synth.bf16_bits_to_f64(x.k)
    rows_std = k.std(axis=-1)
    assert rows_std[x.heavy].mean() > 3.5 and rows_std[~x.heavy].mean() < 1.2
    # per-head scales of the GQA workload lie in [0.5, 2]
    g = synth.generate(synth.GQA_16K, T=2048, B=1)
    stds = synth.bf16_bits_to_f64(g.q).std(axis=(0, 2, 3))
    assert stds.min() > 0.45 and stds.max() < 2.1 and stds.max() / stds.min() > 1.5


def test_bf16_rounding_is_nearest_even():
    x = np.array([1.0, 1.00390625, 1.005859375, -2.5, 3.0e38], dtype=np.float32)
    bits = synth.f32_to_bf16_bits(x)
    back = synth.bf16_bits_to_f32(bits)
    # 1 + 2^-8 is halfway between 1 and 1 + 2^-7: ties to even (1.0)
    assert back[0] == 1.0 and back[1] == 1.0
    assert back[2] == np.float32(1.0078125)  # above the tie: rounds up
    assert back[3] == -2.5

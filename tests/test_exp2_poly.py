"""The FMA-pipe exp2 of the prefill kernel, replayed in float32 on the CPU.

The kernel can compute a share of its softmax exponentials (kPolyPerEight
of every eight pairs; currently none) as 2^y = 2^n * p(f)
with n = rint(y) taken from the low mantissa bits of y + 1.5*2^23,
f = y - n in [-1/2, 1/2], p a degree-3 polynomial, and n added to the
exponent field of p(f).  This test reads the polynomial's coefficients and
the clamp from the kernel source, replays the same steps in float32 (each
step rounded like the GPU's IEEE fp32 operations, with a fused multiply-add
emulated in float64 and rounded once) and checks the result against 2^y.
"""

import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "long_context_sparse_cca_b200", "csrc", "prefill.cu")


def _constants():
    src = open(SRC).read()
    c = {k: np.float32(float(v)) for k, v in
         re.findall(r"constexpr float (kP[0-3]|kRoundMagic) = ([0-9.e+-]+)f;", src)}
    clamp = float(re.search(r"fmaxf\(y\.x, (-[0-9.]+)f\)", src).group(1))
    return c, np.float32(clamp)


def _fma(a, b, c):
    return (a.astype(np.float64) * b + c).astype(np.float32)


def _exp2_poly(y):
    c, clamp = _constants()
    y = np.maximum(y.astype(np.float32), clamp)
    t = (y + c["kRoundMagic"]).astype(np.float32)
    n = (t - c["kRoundMagic"]).astype(np.float32)
    f = _fma(n, np.float32(-1.0), y)
    q = _fma(np.full_like(f, c["kP3"]), f, np.float32(c["kP2"]))
    q = _fma(q, f, np.float32(c["kP1"]))
    q = _fma(q, f, np.float32(c["kP0"]))
    bits = q.view(np.int32) + (t.view(np.int32) << np.int32(23))
    return bits.view(np.float32)


def test_relative_error_over_the_softmax_range():
    # exponent arguments of the kernel: masked/small (-125..) up to the lazy
    # rescale bound (+8)
    y = np.concatenate([np.linspace(-125.0, 8.0, 2_000_001),
                        np.array([0.0, -0.5, 0.5, -1.0, 8.0, -124.5])]).astype(np.float32)
    got = _exp2_poly(y).astype(np.float64)
    ref = np.exp2(y.astype(np.float64))
    rel = np.abs(got - ref) / ref
    assert rel.max() < 1.0e-4, rel.max()
    # below half an fp16 spacing (2^-11 relative): invisible after packing P
    assert rel.max() < 2.0 ** -12


def test_masked_logits_give_tiny_positive_weights():
    got = _exp2_poly(np.array([-np.inf, -1e30, -200.0, -125.0], dtype=np.float32))
    assert np.all(got >= 0) and np.all(np.isfinite(got))
    assert got.max() < 1e-37  # no sign flip or exponent wrap-around

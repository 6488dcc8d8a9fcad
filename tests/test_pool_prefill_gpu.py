"""Parity of cca_pool and cca_attn_prefill (CUDA, through the C ABI) with the
fp64 oracle, on small cases computed in full: several tiles and ragged
tails, grouped-query heads, g = 1, w = 0, a window wider than the sequence,
a one-token sequence, d = 64 and 128."""

import numpy as np
import pytest

import oracle
from gpu_util import assert_close, to_cuda, to_f64, to_bits
from long_context_sparse_cca_b200 import synth

pytestmark = pytest.mark.gpu

# (B, Hq, Hkv, T, d, g, w)
CASES = [
    (1, 2, 2, 256, 64, 16, 64),     # the tiny workload's shape
    (1, 2, 2, 300, 128, 16, 64),    # ragged last query tile
    (2, 4, 2, 200, 128, 8, 40),     # grouped-query heads, B = 2
    (1, 4, 1, 130, 64, 4, 0),       # w = 0, one key/value head
    (1, 2, 2, 100, 128, 1, 10),     # g = 1: full causal attention
    (1, 2, 2, 90, 128, 16, 1000),   # window wider than the sequence
    (1, 2, 2, 1, 128, 16, 64),      # one token, no group
    (1, 2, 2, 1000, 128, 4, 50),    # core stream spans two key tiles
    (1, 2, 2, 517, 128, 5, 37),     # g not dividing w or T
    (1, 3, 1, 700, 64, 32, 100),    # r = 3
    (8, 16, 8, 384, 128, 16, 64),   # 384 work items: several per CTA, 1-4 tiles each
    (4, 32, 8, 1100, 128, 32, 200), # grouped heads, many items with and without core
]


def _inputs(B, Hq, Hkv, T, d, seed, heavy=False):
    q = synth.random_bf16((B, Hq, T, d), seed)
    k = synth.random_bf16((B, Hkv, T, d), seed + 1, scale=2.0 if heavy else 1.0)
    v = synth.random_bf16((B, Hkv, T, d), seed + 2)
    return q, k, v


@pytest.fixture(scope="module")
def cca():
    from long_context_sparse_cca_b200 import build
    build.build()
    import long_context_sparse_cca_b200 as m
    return m


@pytest.mark.parametrize("case", CASES, ids=[str(c) for c in CASES])
def test_pool_and_prefill_match_oracle(cca, case):
    import torch
    B, Hq, Hkv, T, d, g, w = case
    q, k, v = _inputs(B, Hq, Hkv, T, d, seed=sum(case))
    Q, K, V = to_cuda(q), to_cuda(k), to_cuda(v)
    Kc, Vc = cca.cca_pool(Q, K, V, g)
    O32 = cca.cca_attn_prefill(Q, K, V, Kc, Vc, g, w, out_dtype=torch.float32)
    O16 = cca.cca_attn_prefill(Q, K, V, Kc, Vc, g, w)
    assert cca.cca_device_status() == cca.CCA_OK
    qf, kf, vf = (synth.bf16_bits_to_f64(x) for x in (q, k, v))
    Kc_ref, Vc_ref = oracle.pool(qf, kf, vf, g)
    O_ref = oracle.attend_rows(qf, kf, vf, Kc_ref, Vc_ref, g, w)
    if T // g > 0:
        assert_close(Kc, Kc_ref, None, "Kc")
        assert_close(Vc, Vc_ref, None, "Vc")
    assert_close(O32, O_ref, None, "O fp32")
    assert_close(O16, O_ref, None, "O bf16")


def test_heavy_hitter_values(cca):
    """The 32K workload's value distribution (1% of keys x4) at T = 2048."""
    import torch
    wl = synth.PREFILL_32K
    x = synth.generate(wl, T=2048, B=1)
    Q, K, V = to_cuda(x.q), to_cuda(x.k), to_cuda(x.v)
    Kc, Vc = cca.cca_pool(Q, K, V, wl.g)
    O = cca.cca_attn_prefill(Q, K, V, Kc, Vc, wl.g, wl.w, out_dtype=torch.float32)
    assert cca.cca_device_status() == cca.CCA_OK
    qf, kf, vf = (synth.bf16_bits_to_f64(a) for a in (x.q, x.k, x.v))
    Kc_ref, Vc_ref = oracle.pool(qf, kf, vf, wl.g)
    O_ref = oracle.attend_rows(qf, kf, vf, Kc_ref, Vc_ref, wl.g, wl.w)
    assert_close(Kc, Kc_ref, None, "Kc")
    assert_close(Vc, Vc_ref, None, "Vc")
    assert_close(O, O_ref, None, "O")


def test_repeatable_bitwise(cca):
    """The kernels are deterministic: two runs give identical bits."""
    B, Hq, Hkv, T, d, g, w = 1, 4, 2, 700, 128, 16, 64
    q, k, v = _inputs(B, Hq, Hkv, T, d, seed=7)
    Q, K, V = to_cuda(q), to_cuda(k), to_cuda(v)
    Kc1, Vc1 = cca.cca_pool(Q, K, V, g)
    O1 = cca.cca_attn_prefill(Q, K, V, Kc1, Vc1, g, w)
    Kc2, Vc2 = cca.cca_pool(Q, K, V, g)
    O2 = cca.cca_attn_prefill(Q, K, V, Kc2, Vc2, g, w)
    assert np.array_equal(to_bits(Kc1), to_bits(Kc2))
    assert np.array_equal(to_bits(O1), to_bits(O2))


def test_output_rows_outside_sequence_untouched(cca):
    """Guard bands around O stay untouched (no writes past the last row)."""
    import torch
    B, Hq, Hkv, T, d, g, w = 1, 2, 2, 130, 128, 16, 64
    q, k, v = _inputs(B, Hq, Hkv, T, d, seed=11)
    Q, K, V = to_cuda(q), to_cuda(k), to_cuda(v)
    Kc, Vc = cca.cca_pool(Q, K, V, g)
    n = B * Hq * T * d
    buf = torch.full((n + 2 * 4096,), 7.0, dtype=torch.float32, device="cuda")
    O = buf[4096:4096 + n].view(B, Hq, T, d)
    cca.cca_attn_prefill(Q, K, V, Kc, Vc, g, w, O=O)
    torch.cuda.synchronize()
    assert torch.all(buf[:4096] == 7.0) and torch.all(buf[4096 + n:] == 7.0)

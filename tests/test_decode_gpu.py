"""Parity of the decode path (cca_cache_prefill, cca_cache_append,
cca_attn_decode through the C ABI) with the fp64 oracle on small cases:
every generated token's output equals row t of the fused attention over the
whole sequence; core slots hold the pooled groups; ring slots hold the raw
tokens bit for bit."""

import numpy as np
import pytest

import oracle
from gpu_util import assert_close, to_bits, to_cuda, to_f64
from long_context_sparse_cca_b200 import synth

pytestmark = pytest.mark.gpu

# (B, Hq, Hkv, d, g, w, prefix, steps, extra ring slots)
CASES = [
    (2, 4, 2, 128, 16, 64, 300, 40, 0),
    (1, 2, 2, 64, 4, 10, 0, 60, 0),      # from an empty cache
    (1, 2, 2, 128, 1, 0, 5, 20, 0),      # g = 1, w = 0
    (1, 4, 1, 128, 8, 20, 100, 50, 13),  # ring longer than w + g
    (1, 8, 2, 128, 32, 64, 1000, 70, 0), # r = 4, g = 32
    (3, 2, 2, 64, 16, 1024, 200, 30, 0), # window wider than the sequence
]


@pytest.fixture(scope="module")
def cca():
    from long_context_sparse_cca_b200 import build
    build.build()
    import long_context_sparse_cca_b200 as m
    return m


def _run_decode(cca, q, k, v, g, w, prefix, extra, out_dtype):
    import torch
    B, Hq, total, d = q.shape
    Hkv = k.shape[1]
    Q, K, V = to_cuda(q), to_cuda(k), to_cuda(v)
    cache = cca.Cache(B, Hq, Hkv, d, g, w, core_cap=total // g + 1,
                      tail_cap=w + g + extra)
    cca.cca_cache_prefill(cache, Q[:, :, :prefix].contiguous(),
                          K[:, :, :prefix].contiguous(), V[:, :, :prefix].contiguous())
    assert cache.len == prefix
    outs = []
    for t in range(prefix, total):
        qt = Q[:, :, t].contiguous()
        cca.cca_cache_append(cache, qt, K[:, :, t].contiguous(), V[:, :, t].contiguous())
        outs.append(cca.cca_attn_decode(cache, qt, out_dtype=out_dtype))
    assert cca.cca_device_status() == cca.CCA_OK
    assert cache.len == total
    return cache, torch.stack(outs, dim=2)


@pytest.mark.parametrize("case", CASES, ids=[str(c) for c in CASES])
def test_decode_matches_oracle(cca, case):
    import torch
    B, Hq, Hkv, d, g, w, prefix, steps, extra = case
    total = prefix + steps
    seed = 100 + sum(case)
    q = synth.random_bf16((B, Hq, total, d), seed)
    k = synth.random_bf16((B, Hkv, total, d), seed + 1, scale=1.5)
    v = synth.random_bf16((B, Hkv, total, d), seed + 2)
    cache, O = _run_decode(cca, q, k, v, g, w, prefix, extra, torch.float32)
    qf, kf, vf = (synth.bf16_bits_to_f64(x) for x in (q, k, v))
    rows = np.arange(prefix, total)
    O_ref = oracle.prefill(qf, kf, vf, g, w, rows)
    assert_close(O, O_ref, None, "decode output")
    m = total // g
    if m:
        Kc_ref, Vc_ref = oracle.pool(qf, kf, vf, g)
        assert_close(cache.k_core[:, :, :m], Kc_ref, None, "core keys")
        assert_close(cache.v_core[:, :, :m], Vc_ref, None, "core values")
    cap = cache.tail_cap
    kt, vt = to_bits(cache.k_tail), to_bits(cache.v_tail)
    for p in range(max(0, total - cap), total):
        assert np.array_equal(kt[:, :, p % cap], k[:, :, p]), p
        assert np.array_equal(vt[:, :, p % cap], v[:, :, p]), p


def test_decode_bf16_output(cca):
    import torch
    B, Hq, Hkv, d, g, w, prefix, steps = 1, 4, 2, 128, 16, 64, 200, 20
    total = prefix + steps
    q = synth.random_bf16((B, Hq, total, d), 5)
    k = synth.random_bf16((B, Hkv, total, d), 6)
    v = synth.random_bf16((B, Hkv, total, d), 7)
    _, O = _run_decode(cca, q, k, v, g, w, prefix, 0, torch.bfloat16)
    qf, kf, vf = (synth.bf16_bits_to_f64(x) for x in (q, k, v))
    O_ref = oracle.prefill(qf, kf, vf, g, w, np.arange(prefix, total))
    assert_close(O, O_ref, None, "decode output bf16")


def test_cache_prefill_equals_appends(cca):
    """Filling the cache from a prefix gives the same core and ring contents
    as appending the prefix token by token."""
    B, Hq, Hkv, d, g, w, T = 1, 2, 2, 128, 8, 24, 150
    q = synth.random_bf16((B, Hq, T, d), 21)
    k = synth.random_bf16((B, Hkv, T, d), 22)
    v = synth.random_bf16((B, Hkv, T, d), 23)
    Q, K, V = to_cuda(q), to_cuda(k), to_cuda(v)
    a = cca.Cache(B, Hq, Hkv, d, g, w, core_cap=T // g + 1)
    cca.cca_cache_prefill(a, Q, K, V)
    b = cca.Cache(B, Hq, Hkv, d, g, w, core_cap=T // g + 1)
    for t in range(T):
        cca.cca_cache_append(b, Q[:, :, t].contiguous(), K[:, :, t].contiguous(),
                             V[:, :, t].contiguous())
    assert cca.cca_device_status() == cca.CCA_OK
    m = T // g
    assert np.array_equal(to_bits(a.k_tail), to_bits(b.k_tail))
    assert np.array_equal(to_bits(a.v_tail), to_bits(b.v_tail))
    # same arithmetic in both kernels: identical bits
    assert np.array_equal(to_bits(a.k_core[:, :, :m]), to_bits(b.k_core[:, :, :m]))
    assert np.array_equal(to_bits(a.v_core[:, :, :m]), to_bits(b.v_core[:, :, :m]))

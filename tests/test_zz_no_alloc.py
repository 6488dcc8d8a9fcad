"""cca_attn_decode_noalloc: the decode attention for callers that cannot
allocate device memory, with the library's fixed scratch in place of a
caller-provided workspace.  Its output must match cca_attn_decode's (with a
workspace) on consecutive decode steps, through the C ABI (the refusal of an
oversized cache is a host-side check, tested on the CPU in test_abi.py).
This file is collected last so that, should it fail, every other test has
already run.
"""

import pytest

from gpu_util import assert_close, to_cuda, to_f64
from long_context_sparse_cca_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def cca():
    from long_context_sparse_cca_b200 import build
    build.build()
    import long_context_sparse_cca_b200 as m
    return m


def test_noalloc_decode_matches_workspace_decode(cca):
    import torch
    B, Hq, Hkv, d, g, w, prefix = 2, 8, 2, 128, 16, 64, 1000
    total = prefix + 2
    q = synth.random_bf16((B, Hq, total, d), 71)
    k = synth.random_bf16((B, Hkv, total, d), 72)
    v = synth.random_bf16((B, Hkv, total, d), 73)
    Q, K, V = to_cuda(q), to_cuda(k), to_cuda(v)
    cache = cca.Cache(B, Hq, Hkv, d, g, w, core_cap=total // g + 1)
    cca.cca_cache_prefill(cache, Q[:, :, :prefix].contiguous(), K[:, :, :prefix].contiguous(),
                          V[:, :, :prefix].contiguous())
    assert 0 < cca.cca_decode_workspace_bytes(cache) <= cca.NOALLOC_SCRATCH_BYTES
    for t in (prefix, prefix + 1):  # two calls in a row
        qt = Q[:, :, t].contiguous()
        cca.cca_cache_append(cache, qt, K[:, :, t].contiguous(), V[:, :, t].contiguous())
        ref = cca.cca_attn_decode(cache, qt, out_dtype=torch.float32)
        got = cca.cca_attn_decode_noalloc(cache, qt, out_dtype=torch.float32)
        assert cca.cca_device_status() == cca.CCA_OK
        assert_close(to_f64(got), to_f64(ref), None, f"noalloc decode t={t}")


def _decode_case(cca, B, Hq, Hkv, d, g, w, prefix, seed):
    """A cache filled from a prefix, with the inputs of the next two tokens."""
    total = prefix + 2
    q = synth.random_bf16((B, Hq, total, d), seed)
    k = synth.random_bf16((B, Hkv, total, d), seed + 1)
    v = synth.random_bf16((B, Hkv, total, d), seed + 2)
    Q, K, V = to_cuda(q), to_cuda(k), to_cuda(v)
    cache = cca.Cache(B, Hq, Hkv, d, g, w, core_cap=total // g + 1)
    cca.cca_cache_prefill(cache, Q[:, :, :prefix].contiguous(), K[:, :, :prefix].contiguous(),
                          V[:, :, :prefix].contiguous())
    new = [(Q[:, :, t].contiguous(), K[:, :, t].contiguous(), V[:, :, t].contiguous())
           for t in (prefix, prefix + 1)]
    return dict(cache=cache, q=q, k=k, v=v, new=new, g=g, w=w, prefix=prefix)


def _oracle_row(case, t, heads):
    """fp64 oracle output of token t for the given query heads, one
    key/value head at a time (the plain definition over that head's whole
    sequence, pooled with all r query heads that share it)."""
    import numpy as np
    import oracle
    r = case["q"].shape[1] // case["k"].shape[1]
    out = []
    for b in range(case["q"].shape[0]):
        per_head = []
        for h in heads:
            kv = h // r
            qf = synth.bf16_bits_to_f64(case["q"][b:b + 1, kv * r:(kv + 1) * r, :t + 1])
            kf = synth.bf16_bits_to_f64(case["k"][b:b + 1, kv:kv + 1, :t + 1])
            vf = synth.bf16_bits_to_f64(case["v"][b:b + 1, kv:kv + 1, :t + 1])
            per_head.append(oracle.prefill(qf, kf, vf, case["g"], case["w"],
                                           np.array([t]))[0, h - kv * r, 0])
        out.append(per_head)
    return np.array(out)  # [B, len(heads), d]


def test_noalloc_near_limit_and_alternating_shapes(cca):
    """One cache whose decode workspace fills most of the fixed scratch
    (g = 1, a 60000-token prefix: 235 splits for each of 32 query heads)
    and one small cache of another shape (d = 64, grouped heads), decoded in
    turn: leftover partial results or counters of one shape must not reach
    the other's output.  Every output is checked against the workspace path
    and, on sampled heads, against the fp64 oracle."""
    import torch
    big = _decode_case(cca, 1, 32, 8, 128, 1, 16, 60000, 81)
    small = _decode_case(cca, 2, 4, 2, 64, 16, 64, 1000, 91)
    need = cca.cca_decode_workspace_bytes(big["cache"])
    assert 0.9 * cca.NOALLOC_SCRATCH_BYTES < need <= cca.NOALLOC_SCRATCH_BYTES
    assert cca.cca_decode_workspace_bytes(small["cache"]) < need
    for step in range(2):
        for case, heads in ((big, (0, 13, 31)), (small, (0, 1, 2, 3))):
            cache = case["cache"]
            qt, kt, vt = case["new"][step]
            cca.cca_cache_append(cache, qt, kt, vt)
            got = cca.cca_attn_decode_noalloc(cache, qt, out_dtype=torch.float32)
            ref = cca.cca_attn_decode(cache, qt, out_dtype=torch.float32)
            assert cca.cca_device_status() == cca.CCA_OK
            assert_close(to_f64(got), to_f64(ref), None, "noalloc vs workspace decode")
            t = case["prefix"] + step
            assert_close(to_f64(got)[:, list(heads)], _oracle_row(case, t, heads), None,
                         f"noalloc decode vs oracle, t={t}")

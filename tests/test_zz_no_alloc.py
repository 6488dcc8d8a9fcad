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

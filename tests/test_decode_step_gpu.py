"""cca_decode_step: append + decode attention of one token in one launch.

Checked through the C ABI against the fp64 oracle (every output equals row
t of the fused attention over the whole sequence; pooled core slots equal
the oracle's pooling), and against the two separate calls cca_cache_append
+ cca_attn_decode: the raw ring slots bit for bit, the outputs within 2e-3
(the fused step pools a completed group with a whole CTA, in another
summation order than the separate append).  The ticket counters the fused
call leaves at zero are exercised by interleaving it with cca_attn_decode on
one workspace.
"""

import numpy as np
import pytest

import oracle
from gpu_util import assert_close, to_bits, to_cuda
from long_context_sparse_cca_b200 import synth

pytestmark = pytest.mark.gpu

# (B, Hq, Hkv, d, g, w, prefix, steps, extra ring slots)
CASES = [
    (2, 4, 2, 128, 16, 64, 300, 40, 0),
    (1, 2, 2, 64, 4, 10, 0, 60, 0),       # from an empty cache
    (1, 2, 2, 128, 1, 0, 5, 20, 0),       # g = 1, w = 0: a group completes every step
    (1, 4, 1, 128, 8, 20, 100, 50, 13),   # ring longer than w + g
    (1, 8, 2, 128, 32, 64, 1000, 70, 0),  # r = 4, g = 32
    (3, 2, 2, 64, 16, 1024, 200, 30, 0),  # window wider than the sequence
    (1, 32, 2, 128, 16, 64, 600, 20, 0),  # r = 16
]


@pytest.fixture(scope="module")
def cca():
    from long_context_sparse_cca_b200 import build
    build.build()
    import long_context_sparse_cca_b200 as m
    return m


def _inputs(case):
    B, Hq, Hkv, d, g, w, prefix, steps, extra = case
    total = prefix + steps
    seed = 300 + sum(case)
    q = synth.random_bf16((B, Hq, total, d), seed)
    k = synth.random_bf16((B, Hkv, total, d), seed + 1, scale=1.5)
    v = synth.random_bf16((B, Hkv, total, d), seed + 2)
    return q, k, v


def _new_cache(cca, case, Q, K, V):
    B, Hq, Hkv, d, g, w, prefix, steps, extra = case
    total = prefix + steps
    cache = cca.Cache(B, Hq, Hkv, d, g, w, core_cap=total // g + 1, tail_cap=w + g + extra)
    cca.cca_cache_prefill(cache, Q[:, :, :prefix].contiguous(), K[:, :, :prefix].contiguous(),
                          V[:, :, :prefix].contiguous())
    return cache


@pytest.mark.parametrize("case", CASES, ids=[str(c) for c in CASES])
def test_decode_step_matches_oracle_and_separate_calls(cca, case):
    import torch
    B, Hq, Hkv, d, g, w, prefix, steps, extra = case
    total = prefix + steps
    q, k, v = _inputs(case)
    Q, K, V = to_cuda(q), to_cuda(k), to_cuda(v)
    fused = _new_cache(cca, case, Q, K, V)
    separate = _new_cache(cca, case, Q, K, V)
    out_f, out_s = [], []
    for t in range(prefix, total):
        qt, kt, vt = (X[:, :, t].contiguous() for X in (Q, K, V))
        out_f.append(cca.cca_decode_step(fused, qt, kt, vt, out_dtype=torch.float32))
        cca.cca_cache_append(separate, qt, kt, vt)
        out_s.append(cca.cca_attn_decode(separate, qt, out_dtype=torch.float32))
    assert cca.cca_device_status() == cca.CCA_OK
    assert fused.len == total
    # raw ring slots: exact copies
    for name in ("k_tail", "v_tail"):
        assert np.array_equal(to_bits(getattr(fused, name)), to_bits(getattr(separate, name))), name
    qf, kf, vf = (synth.bf16_bits_to_f64(x) for x in (q, k, v))
    # pooled core slots: the fused step pools with the whole CTA (another
    # summation order than the separate append), so both are held to the
    # oracle rather than to each other's bits
    m = total // g
    if m:
        Kc_ref, Vc_ref = oracle.pool(qf, kf, vf, g)
        assert_close(fused.k_core[:, :, :m], Kc_ref, None, "core keys")
        assert_close(fused.v_core[:, :, :m], Vc_ref, None, "core values")
    Of, Os = torch.stack(out_f, dim=2), torch.stack(out_s, dim=2)
    O_ref = oracle.prefill(qf, kf, vf, g, w, np.arange(prefix, total))
    assert_close(Of, O_ref, None, "fused decode step")
    assert float((Of - Os).abs().max()) < 2e-3, "fused step far from append + decode"


def test_decode_step_bf16_output(cca):
    import torch
    case = (2, 8, 2, 128, 16, 64, 500, 24, 0)
    B, Hq, Hkv, d, g, w, prefix, steps, extra = case
    q, k, v = _inputs(case)
    Q, K, V = to_cuda(q), to_cuda(k), to_cuda(v)
    cache = _new_cache(cca, case, Q, K, V)
    outs = [cca.cca_decode_step(cache, *(X[:, :, t].contiguous() for X in (Q, K, V)))
            for t in range(prefix, prefix + steps)]
    assert cca.cca_device_status() == cca.CCA_OK
    O = torch.stack(outs, dim=2)
    assert O.dtype == torch.bfloat16
    qf, kf, vf = (synth.bf16_bits_to_f64(x) for x in (q, k, v))
    O_ref = oracle.prefill(qf, kf, vf, g, w, np.arange(prefix, prefix + steps))
    assert_close(O, O_ref, None, "fused decode step, bf16 output")


def test_decode_step_interleaved_with_decode_on_one_workspace(cca):
    """The fused step does not clear the ticket counters; every decode call
    leaves them at zero.  Alternating the fused step with plain decodes of
    the same token on one workspace must keep giving the same outputs: the
    two plain decodes bit for bit, the fused step within 1e-5 (it adds the
    new token's share after its loop, so its fp32 sums run in another
    order)."""
    import torch
    case = (1, 4, 2, 128, 8, 32, 400, 30, 0)
    B, Hq, Hkv, d, g, w, prefix, steps, extra = case
    q, k, v = _inputs(case)
    Q, K, V = to_cuda(q), to_cuda(k), to_cuda(v)
    cache = _new_cache(cca, case, Q, K, V)
    ws = torch.zeros(cca.cca_decode_workspace_bytes(cache), dtype=torch.uint8, device="cuda")
    for t in range(prefix, prefix + steps):
        qt, kt, vt = (X[:, :, t].contiguous() for X in (Q, K, V))
        a = cca.cca_decode_step(cache, qt, kt, vt, out_dtype=torch.float32, workspace=ws)
        b = cca.cca_attn_decode(cache, qt, out_dtype=torch.float32, workspace=ws)
        c = cca.cca_attn_decode(cache, qt, out_dtype=torch.float32, workspace=ws)
        assert torch.equal(b, c), t
        assert float((a - b).abs().max()) < 1e-5, t
    assert cca.cca_device_status() == cca.CCA_OK
    tickets = ws[-256:].view(torch.int32)  # the counters: the workspace's last part
    assert int(tickets.abs().sum()) == 0


def test_decode_step_capacity(cca):
    """A token without a free core slot is refused before any launch, and
    the cache is left as it was."""
    import torch
    B, Hq, Hkv, d, g, w = 1, 2, 2, 64, 4, 8
    cache = cca.Cache(B, Hq, Hkv, d, g, w, core_cap=2)
    x = torch.zeros((B, Hq, d), dtype=torch.bfloat16, device="cuda")
    kv = torch.zeros((B, Hkv, d), dtype=torch.bfloat16, device="cuda")
    for _ in range(8):
        cca.cca_decode_step(cache, x, kv, kv)
    assert cache.len == 8
    with pytest.raises(cca.CCAError) as e:
        cca.cca_decode_step(cache, x, kv, kv)
    assert e.value.status == cca.CCA_ERR_CAPACITY
    assert cache.len == 8

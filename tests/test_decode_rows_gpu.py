"""Per-row decode lengths in device memory (cca_cache_append_rows,
cca_attn_decode_rows), through the C ABI:

- with equal lengths they reproduce cca_cache_append / cca_attn_decode bit
  for bit;
- rows of different lengths each match the fp64 oracle's fused attention
  over their own sequence;
- a run of decode steps captured once in a CUDA graph and replayed gives the
  same bits as the eager calls;
- empty rows give zero output, rows longer than the cache give zero output
  and CCA_ERR_CAPACITY.
"""

import numpy as np
import pytest

import oracle
from gpu_util import assert_close, to_cuda
from long_context_sparse_cca_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def cca():
    from long_context_sparse_cca_b200 import build
    build.build()
    import long_context_sparse_cca_b200 as m
    return m


def _inputs(B, Hq, Hkv, total, d, seed):
    q = synth.random_bf16((B, Hq, total, d), seed)
    k = synth.random_bf16((B, Hkv, total, d), seed + 1, scale=1.5)
    v = synth.random_bf16((B, Hkv, total, d), seed + 2)
    return q, k, v


@pytest.mark.parametrize("d", [128, 64])
def test_rows_equal_lengths_match_host_length_path(cca, d):
    import torch
    B, Hq, Hkv, g, w, prefix, steps = 2, 4, 2, 16, 64, 300, 40
    total = prefix + steps
    q, k, v = _inputs(B, Hq, Hkv, total, d, 7000 + d)
    Q, K, V = to_cuda(q), to_cuda(k), to_cuda(v)
    caches = [cca.Cache(B, Hq, Hkv, d, g, w, core_cap=total // g + 1) for _ in range(2)]
    for c in caches:
        cca.cca_cache_prefill(c, Q[:, :, :prefix].contiguous(), K[:, :, :prefix].contiguous(),
                              V[:, :, :prefix].contiguous())
    lens = torch.full((B,), prefix, dtype=torch.int64, device="cuda")
    for t in range(prefix, total):
        qt, kt, vt = (X[:, :, t].contiguous() for X in (Q, K, V))
        cca.cca_cache_append(caches[0], qt, kt, vt)
        o_host = cca.cca_attn_decode(caches[0], qt, out_dtype=torch.float32)
        cca.cca_cache_append_rows(caches[1], lens, qt, kt, vt)
        o_rows = cca.cca_attn_decode_rows(caches[1], lens, qt, out_dtype=torch.float32)
        assert torch.equal(o_host, o_rows), t
    assert cca.cca_device_status() == cca.CCA_OK
    assert lens.tolist() == [total] * B
    for a, b in zip((caches[0].k_core, caches[0].v_core, caches[0].k_tail, caches[0].v_tail),
                    (caches[1].k_core, caches[1].v_core, caches[1].k_tail, caches[1].v_tail)):
        assert torch.equal(a, b)


def test_rows_of_different_lengths_match_oracle(cca):
    import torch
    B, Hq, Hkv, d, g, w, steps = 3, 4, 2, 128, 16, 64, 24
    prefixes = [200, 257, 0]
    total = max(prefixes) + steps
    q, k, v = _inputs(B, Hq, Hkv, total, d, 7300)
    Q, K, V = to_cuda(q), to_cuda(k), to_cuda(v)
    cache = cca.Cache(B, Hq, Hkv, d, g, w, core_cap=total // g + 1)
    for b, n in enumerate(prefixes):
        if n:
            cca.cca_cache_prefill(cache.row(b), Q[b:b + 1, :, :n].contiguous(),
                                  K[b:b + 1, :, :n].contiguous(),
                                  V[b:b + 1, :, :n].contiguous())
    lens = torch.tensor(prefixes, dtype=torch.int64, device="cuda")
    outs = []
    for s in range(steps):
        # row b's next token is its own token prefixes[b] + s
        idx = torch.tensor([n + s for n in prefixes], device="cuda")
        ar = torch.arange(B, device="cuda")
        qt = Q[ar, :, idx].contiguous()
        kt = K[ar, :, idx].contiguous()
        vt = V[ar, :, idx].contiguous()
        cca.cca_cache_append_rows(cache, lens, qt, kt, vt)
        outs.append(cca.cca_attn_decode_rows(cache, lens, qt, out_dtype=torch.float32))
    assert cca.cca_device_status() == cca.CCA_OK
    assert lens.tolist() == [n + steps for n in prefixes]
    O = torch.stack(outs, dim=2)  # [B, Hq, steps, d]
    qf, kf, vf = (synth.bf16_bits_to_f64(x) for x in (q, k, v))
    for b, n in enumerate(prefixes):
        L = n + steps
        sl = (slice(b, b + 1), slice(None), slice(0, L))
        ref = oracle.prefill(qf[sl], kf[sl], vf[sl], g, w, np.arange(n, L))
        assert_close(O[b:b + 1], ref, None, f"row {b}")


def test_graph_replay_matches_eager(cca):
    import torch
    B, Hq, Hkv, d, g, w, prefix, steps = 2, 4, 2, 128, 16, 64, 150, 12
    total = prefix + steps
    q, k, v = _inputs(B, Hq, Hkv, total, d, 7600)
    Q, K, V = to_cuda(q), to_cuda(k), to_cuda(v)
    step_in = [tuple(X[:, :, t].contiguous() for X in (Q, K, V)) for t in range(prefix, total)]

    def fresh():
        c = cca.Cache(B, Hq, Hkv, d, g, w, core_cap=total // g + 1)
        cca.cca_cache_prefill(c, Q[:, :, :prefix].contiguous(), K[:, :, :prefix].contiguous(),
                              V[:, :, :prefix].contiguous())
        c.workspace = torch.empty(cca.cca_decode_workspace_bytes(c), dtype=torch.uint8,
                                  device="cuda")
        return c

    # eager
    c1 = fresh()
    lens1 = torch.full((B,), prefix, dtype=torch.int64, device="cuda")
    eager = []
    for qt, kt, vt in step_in:
        cca.cca_cache_append_rows(c1, lens1, qt, kt, vt)
        eager.append(cca.cca_attn_decode_rows(c1, lens1, qt, out_dtype=torch.float32))
    # one capture of all steps, replayed twice from the same start
    c2 = fresh()
    lens2 = torch.full((B,), prefix, dtype=torch.int64, device="cuda")
    outs = [torch.empty((B, Hq, d), dtype=torch.float32, device="cuda") for _ in step_in]
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for (qt, kt, vt), o in zip(step_in, outs):
            cca.cca_cache_append_rows(c2, lens2, qt, kt, vt)
            cca.cca_attn_decode_rows(c2, lens2, qt, o_t=o, workspace=c2.workspace)
    # the appends overwrite ring slots that the first steps read, so every
    # replay starts from a copy of the cache as the prefill left it
    snap = [t.clone() for t in (c2.k_core, c2.v_core, c2.k_tail, c2.v_tail)]
    for _ in range(2):
        for t, s0 in zip((c2.k_core, c2.v_core, c2.k_tail, c2.v_tail), snap):
            t.copy_(s0)
        lens2.fill_(prefix)
        for o in outs:
            o.zero_()
        graph.replay()
        torch.cuda.synchronize()
        for a, b in zip(eager, outs):
            assert torch.equal(a, b)
        assert lens2.tolist() == [total] * B
    assert cca.cca_device_status() == cca.CCA_OK
    del graph


def test_empty_and_overfull_rows(cca):
    import torch
    B, Hq, Hkv, d, g, w = 2, 2, 2, 64, 4, 8
    q, k, v = _inputs(B, Hq, Hkv, 40, d, 7900)
    Q, K, V = to_cuda(q), to_cuda(k), to_cuda(v)
    cache = cca.Cache(B, Hq, Hkv, d, g, w, core_cap=4)  # holds 16 tokens' groups
    qt = Q[:, :, 0].contiguous()
    lens = torch.tensor([0, 40], dtype=torch.int64, device="cuda")
    o = torch.full((B, Hq, d), 7.0, dtype=torch.float32, device="cuda")
    cca.cca_attn_decode_rows(cache, lens, qt, o_t=o)
    assert cca.cca_device_status() == cca.CCA_ERR_CAPACITY
    assert torch.count_nonzero(o) == 0
    # appending to a row past the cache leaves it unchanged and is reported
    cca.cca_cache_append_rows(cache, lens, qt, K[:, :, 0].contiguous(), V[:, :, 0].contiguous())
    assert cca.cca_device_status() == cca.CCA_ERR_CAPACITY
    assert lens.tolist() == [1, 40]
    assert cca.cca_device_status() == cca.CCA_OK

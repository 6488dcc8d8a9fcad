"""Parity at the benchmark's full sizes, in the launch configuration the
benchmark times (bf16 O), against the fp64 oracle on sampled outputs the
oracle computes one by one:

  prefill 32K  (B=1, H=32, d=128, g=16, w=1024, 1% heavy keys)
  prefill 128K (same layer, T = 131072)
  GQA 16K      (B=4, Hq=32, Hkv=8, g=32, w=2048, per-head scales)
  decode       (B=8, H=32, 65536-token prefix + 256 steps)

Pooling is checked in full (every core row); attention on sampled query
rows (window and group edges, tile edges, the last 64 rows, 256 seeded
random rows) for every batch entry and head; decode at every step for batch
row 0 and at 16 sampled steps for all rows, in fp32 and in bf16 (the
benchmark's output type).
"""

import numpy as np
import pytest

import oracle
from gpu_util import assert_close, sample_rows, to_bits, to_cuda
from long_context_sparse_cca_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def cca():
    from long_context_sparse_cca_b200 import build
    build.build()
    import long_context_sparse_cca_b200 as m
    return m


def _prefill_case(cca, wl):
    import torch
    x = synth.generate(wl)
    Q, K, V = to_cuda(x.q), to_cuda(x.k), to_cuda(x.v)
    Kc, Vc = cca.cca_pool(Q, K, V, wl.g)
    O = cca.cca_attn_prefill(Q, K, V, Kc, Vc, wl.g, wl.w)  # bf16, as benchmarked
    O32 = cca.cca_attn_prefill(Q, K, V, Kc, Vc, wl.g, wl.w, out_dtype=torch.float32)
    assert cca.cca_device_status() == cca.CCA_OK
    rows = sample_rows(wl.T, wl.g, wl.w, n_random=256, seed=wl.seed)
    O_rows = O[:, :, torch.from_numpy(rows).cuda()]
    O32_rows = O32[:, :, torch.from_numpy(rows).cuda()]
    Kc_h, Vc_h = Kc.cpu(), Vc.cpu()
    del O, O32, Q, K, V, Kc, Vc
    torch.cuda.empty_cache()
    qf, kf, vf = (synth.bf16_bits_to_f64(a) for a in (x.q, x.k, x.v))
    del x
    Kc_ref, Vc_ref = oracle.pool(qf, kf, vf, wl.g)
    assert_close(Kc_h, Kc_ref, None, "Kc")
    assert_close(Vc_h, Vc_ref, None, "Vc")
    O_ref = oracle.attend_rows(qf, kf, vf, Kc_ref, Vc_ref, wl.g, wl.w, rows)
    e16 = assert_close(O_rows, O_ref, None, "O bf16")
    e32 = assert_close(O32_rows, O_ref, None, "O fp32")
    print(f"{wl.name}: rows {rows.size}, O bf16 {e16}, O fp32 {e32}")


def test_prefill_32k(cca):
    _prefill_case(cca, synth.PREFILL_32K)


def test_prefill_128k(cca):
    _prefill_case(cca, synth.PREFILL_128K)


def test_prefill_gqa_16k(cca):
    _prefill_case(cca, synth.GQA_16K)


def test_decode_64k_256_steps(cca):
    import torch
    wl = synth.DECODE_64K
    y = synth.generate(wl)
    total = wl.T + wl.steps
    cache = cca.Cache(wl.B, wl.Hq, wl.Hkv, wl.d, wl.g, wl.w, core_cap=total // wl.g)
    pre = [to_cuda(np.ascontiguousarray(a[:, :, :wl.T])) for a in (y.q, y.k, y.v)]
    cca.cca_cache_prefill(cache, *pre)
    del pre
    nq, nk, nv = (to_cuda(np.ascontiguousarray(a[:, :, wl.T:].transpose(2, 0, 1, 3)))
                  for a in (y.q, y.k, y.v))
    outs, outs16 = [], []
    for s in range(wl.steps):
        cca.cca_cache_append(cache, nq[s], nk[s], nv[s])
        outs.append(cca.cca_attn_decode(cache, nq[s], out_dtype=torch.float32))
        # bf16, as benchmarked
        outs16.append(cca.cca_attn_decode(cache, nq[s], out_dtype=torch.bfloat16))
    assert cca.cca_device_status() == cca.CCA_OK
    O = torch.stack(outs, dim=2).cpu()  # [B, Hq, steps, d]
    O16 = torch.stack(outs16, dim=2).cpu()
    m = total // wl.g
    k_core, v_core = cache.k_core[:, :, :m].cpu(), cache.v_core[:, :, :m].cpu()
    kt, vt = to_bits(cache.k_tail), to_bits(cache.v_tail)
    del cache, nq, nk, nv
    torch.cuda.empty_cache()
    cap = wl.w + wl.g
    for p in range(total - cap, total):
        assert np.array_equal(kt[:, :, p % cap], y.k[:, :, p]), p
        assert np.array_equal(vt[:, :, p % cap], y.v[:, :, p]), p
    rows_all = np.arange(wl.T, total)
    sampled = np.sort(np.random.default_rng(5).choice(wl.steps, 16, replace=False))
    for b in range(wl.B):
        qf, kf, vf = (synth.bf16_bits_to_f64(a[b:b + 1]) for a in (y.q, y.k, y.v))
        Kc_ref, Vc_ref = oracle.pool(qf, kf, vf, wl.g)
        assert_close(k_core[b:b + 1], Kc_ref, None, f"core keys b={b}")
        assert_close(v_core[b:b + 1], Vc_ref, None, f"core values b={b}")
        steps = np.arange(wl.steps) if b == 0 else sampled
        O_ref = oracle.attend_rows(qf, kf, vf, Kc_ref, Vc_ref, wl.g, wl.w, rows_all[steps])
        assert_close(O[b:b + 1, :, steps].numpy(), O_ref, None, f"decode b={b}")
        assert_close(O16[b:b + 1, :, steps], O_ref, None, f"decode bf16 b={b}")

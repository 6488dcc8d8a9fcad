"""Values beyond the fp16 range.

Core keys/values and the query copy that scores them are fp16, so a pooled
value or a query element above 65504 in magnitude cannot be stored as it is.
The library clamps it to +-65504 and reports CCA_ERR_RANGE through
cca_device_status().  These cases plant such values in bf16 inputs (bf16
reaches 3.4e38) and check, for every call that clamps:

  - the status is CCA_ERR_RANGE, and it clears after one read;
  - every output is finite;
  - the clamped element is exactly +-65504 (pooling, append);
  - everything the planted value does not reach still matches the fp64
    oracle within the usual tolerance.
"""

import numpy as np
import pytest

import oracle
from gpu_util import assert_close, to_cuda, to_f64
from long_context_sparse_cca_b200 import synth

pytestmark = pytest.mark.gpu

BIG = 7.0e4          # above the fp16 maximum; bf16 holds it (70144 after rounding)
F16_MAX = 65504.0


@pytest.fixture(scope="module")
def cca():
    from long_context_sparse_cca_b200 import build
    build.build()
    import long_context_sparse_cca_b200 as m
    return m


def _bits(x: float) -> int:
    """bf16 bit pattern of one value."""
    return int(synth.f32_to_bf16_bits(np.array([x], dtype=np.float32))[0])


def _plant_group_value(v_bits: np.ndarray, b: int, h: int, j: int, g: int, dim: int):
    """Every value row of group j of (b, h) gets BIG in column `dim`: the
    pooled value of that column is then BIG whatever the weights are."""
    out = v_bits.copy()
    out[b, h, j * g:(j + 1) * g, dim] = _bits(BIG)
    return out


def test_pool_clamps_and_reports(cca):
    B, Hq, Hkv, T, d, g = 1, 4, 2, 256, 128, 16
    q = synth.random_bf16((B, Hq, T, d), 31)
    k = synth.random_bf16((B, Hkv, T, d), 32)
    v = _plant_group_value(synth.random_bf16((B, Hkv, T, d), 33), 0, 1, 5, g, 7)
    assert cca.cca_device_status() == cca.CCA_OK
    Kc, Vc = cca.cca_pool(to_cuda(q), to_cuda(k), to_cuda(v), g)
    assert cca.cca_device_status() == cca.CCA_ERR_RANGE
    assert cca.cca_device_status() == cca.CCA_OK  # the record was cleared
    kc, vc = to_f64(Kc), to_f64(Vc)
    assert np.all(np.isfinite(kc)) and np.all(np.isfinite(vc))
    assert vc[0, 1, 5, 7] == F16_MAX
    Kc_ref, Vc_ref = oracle.pool(*(synth.bf16_bits_to_f64(x) for x in (q, k, v)), g)
    assert Vc_ref[0, 1, 5, 7] > F16_MAX  # the plain definition is not clamped
    assert_close(kc, Kc_ref, None, "Kc")
    mask = np.ones(vc.shape, dtype=bool)
    mask[0, 1, 5, 7] = False
    assert_close(vc[mask], Vc_ref[mask], None, "Vc away from the clamped element")


def test_cache_append_clamps_and_reports(cca):
    import torch
    B, Hq, Hkv, d, g, w, T = 2, 2, 2, 64, 8, 16, 64
    q = synth.random_bf16((B, Hq, T, d), 41)
    k = synth.random_bf16((B, Hkv, T, d), 42)
    v = _plant_group_value(synth.random_bf16((B, Hkv, T, d), 43), 1, 0, 3, g, 2)
    Q, K, V = to_cuda(q), to_cuda(k), to_cuda(v)
    cache = cca.Cache(B, Hq, Hkv, d, g, w, core_cap=T // g)
    outs = []
    for t in range(T):
        qt = Q[:, :, t].contiguous()
        cca.cca_cache_append(cache, qt, K[:, :, t].contiguous(), V[:, :, t].contiguous())
        if t == 3 * g - 1:  # before the planted group completes: nothing clamped
            assert cca.cca_device_status() == cca.CCA_OK
        outs.append(cca.cca_attn_decode(cache, qt, out_dtype=torch.float32))
    assert cca.cca_device_status() == cca.CCA_ERR_RANGE
    assert cca.cca_device_status() == cca.CCA_OK
    vcore = to_f64(cache.v_core)
    assert vcore[1, 0, 3, 2] == F16_MAX
    O = to_f64(torch.stack(outs, dim=2))
    assert np.all(np.isfinite(O))
    qf, kf, vf = (synth.bf16_bits_to_f64(x) for x in (q, k, v))
    Kc_ref, Vc_ref = oracle.pool(qf, kf, vf, g)
    mask = np.ones(Vc_ref.shape, dtype=bool)
    mask[1, 0, 3, 2] = False
    assert_close(vcore[mask], Vc_ref[mask], None, "core values away from the clamp")
    # Column 2 of the values reaches only column 2 of the outputs (the
    # softmax weights come from the keys): every other column matches the
    # oracle everywhere, and column 2 until group 3 first enters a core set.
    O_ref = oracle.prefill(qf, kf, vf, g, w, np.arange(T))
    assert_close(O[0], O_ref[0], None, "decode, batch row 0")
    cols = np.arange(d) != 2
    assert_close(O[1][..., cols], O_ref[1][..., cols], None, "decode, batch row 1")
    first_core3 = next(t for t in range(T) if oracle.window_start(t, g, w) // g > 3)
    assert 3 * g < first_core3 < T
    assert_close(O[1, :, :3 * g, 2], O_ref[1, :, :3 * g, 2], None,
                 "decode, batch row 1, column 2 before the planted group")


def test_prefill_clamps_query_copy_and_reports(cca):
    import torch
    B, Hq, Hkv, T, d, g, w = 1, 2, 2, 600, 128, 16, 64
    q = synth.random_bf16((B, Hq, T, d), 51)
    k = synth.random_bf16((B, Hkv, T, d), 52)
    v = synth.random_bf16((B, Hkv, T, d), 53)
    t_big = 400          # has core tokens (ws(400) = 336, 21 groups)
    assert (t_big + 1) % g != 0  # not a scoring query: pooling is unaffected
    q[0, 1, t_big, 9] = _bits(BIG)
    Q, K, V = to_cuda(q), to_cuda(k), to_cuda(v)
    Kc, Vc = cca.cca_pool(Q, K, V, g)
    assert cca.cca_device_status() == cca.CCA_OK
    O = cca.cca_attn_prefill(Q, K, V, Kc, Vc, g, w, out_dtype=torch.float32)
    assert cca.cca_device_status() == cca.CCA_ERR_RANGE
    assert cca.cca_device_status() == cca.CCA_OK
    o = to_f64(O)
    assert np.all(np.isfinite(o))
    qf, kf, vf = (synth.bf16_bits_to_f64(x) for x in (q, k, v))
    Kc_ref, Vc_ref = oracle.pool(qf, kf, vf, g)
    O_ref = oracle.attend_rows(qf, kf, vf, Kc_ref, Vc_ref, g, w)
    assert_close(o[0, 0], O_ref[0, 0], None, "head 0 (no planted value)")
    keep = np.arange(T) != t_big
    assert_close(o[0, 1, keep], O_ref[0, 1, keep], None, "head 1, other rows")

"""The backward pass on the GPU (cca_attn_prefill_lse + cca_attn_backward,
through the C ABI) against the fp64 gradient oracle (oracle/cca_backward.py,
itself pinned to finite differences of the C oracle's forward): dQ, dK, dV
of L = sum(dO * O) on the same bf16 inputs and upstream gradient.

Cases cover grouped-query heads, g = 1, a window wider than the sequence
(no core stream), T mod g != 0, several core tiles (so that the core
tiles' query ranges are cut into chunks), d = 64 and 128, and a 4K-context
case.  The tolerance is relative to each gradient's own scale (see
gpu_util.grad_errors): the kernels round P and dS to 16 bits for the
tensor cores and take the pooled rows in fp16, as the forward does.
"""

import numpy as np
import pytest

from gpu_util import grad_errors, to_cuda
from long_context_sparse_cca_b200 import synth
from oracle import cca_backward as bw

pytestmark = pytest.mark.gpu

# (B, Hq, Hkv, T, d, g, w)
CASES = [
    (1, 2, 2, 200, 64, 16, 64),
    (1, 4, 2, 300, 128, 16, 64),     # grouped heads, ragged last tile
    (1, 2, 2, 130, 128, 1, 10),      # g = 1: every token is a core token
    (1, 2, 2, 100, 64, 16, 1000),    # window wider than the sequence: no core
    (1, 4, 1, 333, 64, 8, 40),       # r = 4, T mod g != 0
    (2, 2, 1, 2500, 64, 8, 64),      # three core tiles, chunked query ranges
    (1, 8, 1, 700, 128, 32, 64),     # r = 8, g = 32
    (1, 24, 1, 600, 64, 256, 64),    # r = 24, g = 256: pooling scratch for 7 warps a block
]


@pytest.fixture(scope="module")
def cca():
    from long_context_sparse_cca_b200 import build
    build.build()
    import long_context_sparse_cca_b200 as m
    return m


def _run(cca, case, seed):
    import torch
    B, Hq, Hkv, T, d, g, w = case
    q = synth.random_bf16((B, Hq, T, d), seed)
    k = synth.random_bf16((B, Hkv, T, d), seed + 1, scale=1.5)
    v = synth.random_bf16((B, Hkv, T, d), seed + 2)
    do = synth.random_bf16((B, Hq, T, d), seed + 3)
    Q, K, V, dO = (to_cuda(x) for x in (q, k, v, do))
    Kc, Vc = cca.cca_pool(Q, K, V, g)
    O, lse = cca.cca_attn_prefill_lse(Q, K, V, Kc, Vc, g, w)
    dQ, dK, dV = cca.cca_attn_backward(Q, K, V, Kc, Vc, O, lse, dO, g, w)
    assert cca.cca_device_status() == cca.CCA_OK
    got = tuple(x.double().cpu().numpy() for x in (dQ, dK, dV))
    ref = bw.backward(*(synth.bf16_bits_to_f64(x) for x in (q, k, v)), g, w,
                      synth.bf16_bits_to_f64(do))
    return got, ref


@pytest.mark.parametrize("case", CASES, ids=[str(c) for c in CASES])
def test_backward_matches_gradient_oracle(cca, case):
    got, ref = _run(cca, case, seed=40 + sum(case))
    for name, a, b in zip(("dQ", "dK", "dV"), got, ref):
        e = grad_errors(a, b)
        print(name, e)
        assert e["ok"], f"{name}: {e}"


def test_backward_4k_context(cca):
    case = (1, 4, 2, 4096, 128, 16, 1024)
    got, ref = _run(cca, case, seed=77)
    for name, a, b in zip(("dQ", "dK", "dV"), got, ref):
        e = grad_errors(a, b)
        print(name, e)
        assert e["ok"], f"{name}: {e}"


def test_backward_repeatable(cca):
    """Raw-key and query gradients are plain stores (bitwise repeatable);
    the core keys' partial sums are added atomically in an order that may
    vary, so dK, dV of grouped rows are compared within rounding."""
    import torch
    B, Hq, Hkv, T, d, g, w = 1, 2, 2, 700, 128, 16, 64
    q, k, v, do = (synth.random_bf16((B, H, T, d), 90 + i)
                   for i, H in enumerate((Hq, Hkv, Hkv, Hq)))
    Q, K, V, dO = (to_cuda(x) for x in (q, k, v, do))
    Kc, Vc = cca.cca_pool(Q, K, V, g)
    O, lse = cca.cca_attn_prefill_lse(Q, K, V, Kc, Vc, g, w)
    a = cca.cca_attn_backward(Q, K, V, Kc, Vc, O, lse, dO, g, w)
    b = cca.cca_attn_backward(Q, K, V, Kc, Vc, O, lse, dO, g, w)
    assert cca.cca_device_status() == cca.CCA_OK
    for x, y in zip(a, b):
        assert float((x - y).abs().max()) <= 1e-5 * float(x.abs().max())


def test_backward_poisoned_buffers(cca):
    """Outputs pre-filled with NaN and a workspace of 0xFF bytes, three calls
    in a row on a shape with partial key tiles and several core tiles: every
    gradient element is written, and each call matches the oracle (a read of
    an accumulator before its last products landed showed up exactly here,
    on partial key tiles)."""
    import torch
    case = (2, 2, 1, 2500, 64, 8, 64)
    B, Hq, Hkv, T, d, g, w = case
    seed = 40 + sum(case)
    q = synth.random_bf16((B, Hq, T, d), seed)
    k = synth.random_bf16((B, Hkv, T, d), seed + 1, scale=1.5)
    v = synth.random_bf16((B, Hkv, T, d), seed + 2)
    do = synth.random_bf16((B, Hq, T, d), seed + 3)
    Q, K, V, dO = (to_cuda(x) for x in (q, k, v, do))
    Kc, Vc = cca.cca_pool(Q, K, V, g)
    O, lse = cca.cca_attn_prefill_lse(Q, K, V, Kc, Vc, g, w)
    ref = bw.backward(*(synth.bf16_bits_to_f64(x) for x in (q, k, v)), g, w,
                      synth.bf16_bits_to_f64(do))
    nb = cca.cca_attn_backward_workspace_bytes(B, Hq, Hkv, T, d, g)
    for _ in range(3):
        outs = [torch.full(shape, float("nan"), device="cuda")
                for shape in ((B, Hq, T, d), (B, Hkv, T, d), (B, Hkv, T, d))]
        ws = torch.full((nb,), 255, dtype=torch.uint8, device="cuda")
        cca.cca_attn_backward(Q, K, V, Kc, Vc, O, lse, dO, g, w, *outs, workspace=ws)
        assert cca.cca_device_status() == cca.CCA_OK
        for name, a, b in zip(("dQ", "dK", "dV"), outs, ref):
            a = a.double().cpu().numpy()
            assert not np.isnan(a).any(), f"{name}: unwritten elements"
            e = grad_errors(a, b)
            assert e["ok"], f"{name}: {e}"

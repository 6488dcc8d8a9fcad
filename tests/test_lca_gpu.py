"""The LCA variant on the GPU (cca_lca_pool, cca_lca_cache_prefill,
cca_lca_cache_append; then cca_attn_prefill and cca_attn_decode on the
condensed rows), through the C ABI, against the fp64 oracle's lca_pool and
fused attention.

The anchor (the group's highest-weight token) is an integer that floating
point decides.  Where the oracle's two largest weights differ by more than
ANCHOR_MARGIN, the kernel must pick the oracle's token; closer than that, any
token whose oracle weight is within the margin of the largest is valid.  The
kernel's choice is read back from the positional entries of the core key,
which are the anchor's own (bf16 -> fp16, an exact conversion here).  The
content entries and the values are held to the usual tolerance.
"""

import numpy as np
import pytest

import oracle
from gpu_util import assert_close, to_bits, to_cuda, to_f64
from long_context_sparse_cca_b200 import synth

pytestmark = pytest.mark.gpu

# fp32 softmax weights carry relative errors of a few 1e-7; a margin of 1e-5
# separates a real choice from rounding.
ANCHOR_MARGIN = 1e-5

# (B, Hq, Hkv, T, d, g, d_rope)
POOL_CASES = [
    (1, 2, 2, 16 * 40 + 7, 128, 16, 64),   # register path g = 16, ragged tail
    (2, 8, 2, 32 * 20 + 5, 128, 32, 64),   # register path g = 32, r = 4
    (1, 4, 4, 300, 64, 16, 32),            # d = 64
    (1, 4, 4, 300, 64, 32, 8),             # d = 64, g = 32
    (1, 4, 1, 333, 64, 8, 16),             # generic path, r = 4
    (1, 2, 2, 100, 128, 5, 0),             # odd g, no positional part
    (1, 2, 2, 256, 128, 16, 128),          # all positional: selection
    (1, 2, 2, 64, 128, 1, 64),             # g = 1: the token itself
    (1, 32, 2, 512, 128, 16, 64),          # r = 16
    (1, 2, 2, 15, 128, 16, 64),            # no complete group
]


@pytest.fixture(scope="module")
def cca():
    from long_context_sparse_cca_b200 import build
    build.build()
    import long_context_sparse_cca_b200 as m
    return m


def _inputs(B, Hq, Hkv, T, d, seed):
    q = synth.random_bf16((B, Hq, T, d), seed)
    k = synth.random_bf16((B, Hkv, T, d), seed + 1, scale=1.5)
    v = synth.random_bf16((B, Hkv, T, d), seed + 2)
    return q, k, v


def _f16_rows(x: np.ndarray) -> np.ndarray:
    """fp16 bit patterns of float64 values that are exactly bf16 numbers
    (round to nearest even, as the kernel's conversion)."""
    return x.astype(np.float16).view(np.uint16)


def check_anchors(Kc_bits, kf, A, anchor_ref, g, d_rope, what):
    """Kc_bits [B, Hkv, m, d] fp16 bits from the GPU; kf [B, Hkv, T, d]
    float64 keys; A [B, Hkv, m, g] and anchor_ref [B, Hkv, m] from the
    oracle.  Returns the kernel's anchors."""
    B, Hkv, m, d = Kc_bits.shape
    got = np.full((B, Hkv, m), -1, dtype=np.int64)
    if d_rope == 0 or m == 0:
        return got
    rows = _f16_rows(kf[:, :, :m * g, d - d_rope:]).reshape(B, Hkv, m, g, d_rope)
    pos = Kc_bits[..., d - d_rope:]
    match = np.all(rows == pos[:, :, :, None, :], axis=-1)  # [B, Hkv, m, g]
    assert match.any(-1).all(), f"{what}: a positional part matches no token of its group"
    if g > 1:
        top2 = np.sort(A, axis=-1)[..., -2:]
        gap = top2[..., 1] - top2[..., 0]
    else:
        gap = np.full(A.shape[:-1], np.inf)
    amax = A.max(-1)
    for idx in np.ndindex(B, Hkv, m):
        cand = np.flatnonzero(match[idx])
        if gap[idx] > ANCHOR_MARGIN:
            assert anchor_ref[idx] in cand, (what, idx, cand, anchor_ref[idx])
            got[idx] = anchor_ref[idx]
        else:
            ok = [i for i in cand if A[idx][i] >= amax[idx] - ANCHOR_MARGIN]
            assert ok, (what, idx, cand, A[idx])
            got[idx] = ok[0]
    return got


def check_condensed(Kc, Vc, qf, kf, vf, g, d_rope, what):
    """Kc, Vc: GPU fp16 tensors.  Checks anchors, content and values."""
    Kc_ref, Vc_ref, A, anchor_ref = oracle.lca_pool(qf, kf, vf, g, d_rope, want_weights=True)
    d = kf.shape[-1]
    check_anchors(to_bits(Kc), kf, A, anchor_ref, g, d_rope, what)
    got_k = to_f64(Kc)
    assert_close(got_k[..., :d - d_rope], Kc_ref[..., :d - d_rope], "f16", what + " content")
    assert_close(Vc, Vc_ref, None, what + " values")
    return Kc_ref, Vc_ref, A


def _min_gap(A):
    if A.shape[-1] < 2 or A.size == 0:
        return np.inf
    s = np.sort(A, axis=-1)
    return float((s[..., -1] - s[..., -2]).min())


@pytest.mark.parametrize("case", POOL_CASES, ids=[str(c) for c in POOL_CASES])
def test_lca_pool_matches_oracle(cca, case):
    B, Hq, Hkv, T, d, g, d_rope = case
    q, k, v = _inputs(B, Hq, Hkv, T, d, 500 + sum(case))
    Kc, Vc = cca.cca_lca_pool(to_cuda(q), to_cuda(k), to_cuda(v), g, d_rope)
    assert cca.cca_device_status() == cca.CCA_OK
    assert Kc.shape == (B, Hkv, T // g, d)
    if T // g == 0:
        return
    qf, kf, vf = (synth.bf16_bits_to_f64(x) for x in (q, k, v))
    check_condensed(Kc, Vc, qf, kf, vf, g, d_rope, f"lca_pool {case}")


def test_lca_pool_deterministic(cca):
    q, k, v = _inputs(2, 8, 2, 1024 + 9, 128, 77)
    Q, K, V = to_cuda(q), to_cuda(k), to_cuda(v)
    a = cca.cca_lca_pool(Q, K, V, 16, 64)
    b = cca.cca_lca_pool(Q, K, V, 16, 64)
    assert all(np.array_equal(to_bits(x), to_bits(y)) for x, y in zip(a, b))


# (B, Hq, Hkv, T, d, g, w, d_rope), seed.  The seeds give no anchor
# near-tie (two largest oracle weights closer than 5e-5) in any group, so
# that the attention, which sees whole core rows, has one right answer.
PREFILL_CASES = [
    ((1, 2, 2, 1100, 128, 16, 256, 64), 2169),
    ((1, 8, 2, 900, 128, 32, 128, 64), 1870),
    ((1, 4, 4, 700, 64, 8, 64, 32), 1478),
]


@pytest.mark.parametrize("case,seed", PREFILL_CASES, ids=[str(c[0]) for c in PREFILL_CASES])
def test_lca_prefill_attention(cca, case, seed):
    """cca_lca_pool then cca_attn_prefill on its rows equals the oracle's
    fused attention over the oracle's condensed rows."""
    import torch
    B, Hq, Hkv, T, d, g, w, d_rope = case
    q, k, v = _inputs(B, Hq, Hkv, T, d, seed)
    Q, K, V = to_cuda(q), to_cuda(k), to_cuda(v)
    Kc, Vc = cca.cca_lca_pool(Q, K, V, g, d_rope)
    O = cca.cca_attn_prefill(Q, K, V, Kc, Vc, g, w, out_dtype=torch.float32)
    assert cca.cca_device_status() == cca.CCA_OK
    qf, kf, vf = (synth.bf16_bits_to_f64(x) for x in (q, k, v))
    Kc_ref, Vc_ref, A = check_condensed(Kc, Vc, qf, kf, vf, g, d_rope, f"lca prefill {case}")
    # the attention is compared where the anchors are unambiguous
    assert _min_gap(A) > ANCHOR_MARGIN, "seed gives a near-tie; the fixture needs another seed"
    O_ref = oracle.attend_rows(qf, kf, vf, Kc_ref, Vc_ref, g, w)
    assert_close(O, O_ref, None, f"lca prefill attention {case}")


# (B, Hq, Hkv, d, g, w, d_rope, prefix, steps), seed (no anchor near-tie,
# as above)
DECODE_CASES = [
    ((2, 4, 2, 128, 16, 64, 64, 300, 40), 1321),
    ((1, 2, 2, 64, 4, 10, 16, 0, 60), 859),       # from an empty cache
    ((1, 2, 2, 128, 1, 0, 64, 5, 20), 923),       # g = 1
    ((1, 8, 2, 128, 32, 64, 128, 1000, 70), 2137),
]


@pytest.mark.parametrize("case,seed", DECODE_CASES, ids=[str(c[0]) for c in DECODE_CASES])
def test_lca_decode_cache(cca, case, seed):
    """Prefix fill, then append + decode token by token: the core slots
    equal the oracle's condensation of the whole sequence (the running query
    sums give each group its average query), and every decode output equals
    row t of the oracle's fused attention over those rows."""
    import torch
    B, Hq, Hkv, d, g, w, d_rope, prefix, steps = case
    total = prefix + steps
    q, k, v = _inputs(B, Hq, Hkv, total, d, seed)
    Q, K, V = to_cuda(q), to_cuda(k), to_cuda(v)
    cache = cca.Cache(B, Hq, Hkv, d, g, w, core_cap=total // g + 1)
    q_sum = cca.lca_query_sums(cache)
    cca.cca_lca_cache_prefill(cache, q_sum, Q[:, :, :prefix].contiguous(),
                              K[:, :, :prefix].contiguous(), V[:, :, :prefix].contiguous(),
                              d_rope)
    outs = []
    for t in range(prefix, total):
        qt, kt, vt = (X[:, :, t].contiguous() for X in (Q, K, V))
        cca.cca_lca_cache_append(cache, q_sum, qt, kt, vt, d_rope)
        outs.append(cca.cca_attn_decode(cache, qt, out_dtype=torch.float32))
    assert cca.cca_device_status() == cca.CCA_OK
    assert cache.len == total
    qf, kf, vf = (synth.bf16_bits_to_f64(x) for x in (q, k, v))
    m = total // g
    Kc_ref, Vc_ref, A = check_condensed(cache.k_core[:, :, :m], cache.v_core[:, :, :m], qf, kf,
                                        vf, g, d_rope, f"lca cache {case}")
    # the open group's query sums
    rest = total - m * g
    qs_ref = qf[:, :, m * g:].sum(axis=2) if rest else np.zeros((B, Hq, d))
    np.testing.assert_allclose(q_sum.cpu().numpy(), qs_ref, rtol=1e-5, atol=1e-4)
    assert _min_gap(A) > ANCHOR_MARGIN, "seed gives a near-tie; the fixture needs another seed"
    O = torch.stack(outs, dim=2)
    O_ref = oracle.attend_rows(qf, kf, vf, Kc_ref, Vc_ref, g, w, np.arange(prefix, total))
    assert_close(O, O_ref, None, f"lca decode {case}")


def test_lca_fullsize_sampled_groups(cca):
    """The 128K-context shape (B1 H32 d128 g16, 64 positional entries),
    condensed at full size in one launch; sampled groups checked one by one
    against the oracle run on each group's own rows (a group's condensed
    token depends on nothing else)."""
    B, H, T, d, g, d_rope = 1, 32, 131072, 128, 16, 64
    q, k, v = _inputs(B, H, H, T, d, 901)
    Q, K, V = to_cuda(q), to_cuda(k), to_cuda(v)
    Kc, Vc = cca.cca_lca_pool(Q, K, V, g, d_rope)
    assert cca.cca_device_status() == cca.CCA_OK
    Kb, Vf = to_bits(Kc), to_f64(Vc)
    rng = np.random.default_rng(5)
    m = T // g
    groups = sorted({0, 1, m // 2, m - 1} | set(int(x) for x in rng.integers(0, m, 60)))
    heads = [0, 7, 31]
    for h in heads:
        for j in groups:
            sl = slice(j * g, (j + 1) * g)
            qf, kf, vf = (synth.bf16_bits_to_f64(x[:, h:h + 1, sl]) for x in (q, k, v))
            Kr, Vr, A, an = oracle.lca_pool(qf, kf, vf, g, d_rope, want_weights=True)
            what = f"full-size group (h={h}, j={j})"
            check_anchors(Kb[:, h:h + 1, j:j + 1], kf, A, an, g, d_rope, what)
            Kg = Kb[:, h:h + 1, j:j + 1].view(np.float16).astype(np.float64)
            assert_close(Kg[..., :d - d_rope], Kr[..., :d - d_rope], "f16", what)
            assert_close(Vf[:, h:h + 1, j:j + 1], Vr, "f16", what)

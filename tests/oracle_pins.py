"""Pins of the CPU oracle: checks against facts fixed outside the oracle.

Each ``pin_*`` function takes an ``oracle.Oracle`` and raises AssertionError
if that oracle disagrees with something the pages or the mathematics fix:
closed forms, reductions to textbook causal attention (computed by
``torch.nn.functional.scaled_dot_product_attention`` in float64), invariants
the write-up states, brute force from the prose on tiny inputs, and the one
number the pages print for the cache.  The same functions run against the
committed oracle (test_oracle_pins.py) and against copies with a planted
mistake (test_oracle_mutants.py), which must each fail at least one pin.

The write-up cited is "ICML 2025 | 全局池化+局部保留，CCA-Attention为LLM长文本建模
带来突破性进展" (a summary of "Core Context Aware Transformers for Long
Context Language Modeling").
"""

from __future__ import annotations

import math
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def _sdpa_causal(Q, K, V):
    """Textbook causal attention (float64, library routine), GQA by
    repeating each key/value head over its query heads."""
    import torch
    import torch.nn.functional as F

    r = Q.shape[1] // K.shape[1]
    q = torch.from_numpy(np.ascontiguousarray(Q))
    k = torch.from_numpy(np.repeat(K, r, axis=1))
    v = torch.from_numpy(np.repeat(V, r, axis=1))
    return F.scaled_dot_product_attention(q, k, v, is_causal=True).numpy()


def _prose_window_start(t, g, w):
    """Window start found by search from the prose of section 局部保留模块:
    the start must leave at least w raw predecessors of t in the window (all
    of them when t < w) and be a multiple of g; the window is the smallest
    such one, i.e. the start is the largest admissible multiple of g."""
    need = max(t - w, 0)
    best = None
    s = 0
    while s <= need:
        best = s
        s += g
    return best


# ---------------------------------------------------------------------------
# window (section 局部保留模块)
# ---------------------------------------------------------------------------

def pin_window_matches_prose(orc):
    for g in (1, 2, 3, 4, 16):
        for w in (0, 1, 5, 8, 16, 64):
            for t in range(0, 150):
                s = orc.window_start(t, g, w)
                assert s == _prose_window_start(t, g, w), (t, g, w, s)
                assert 0 <= s <= t and s % g == 0


# ---------------------------------------------------------------------------
# pooling (section 全局感知池化)
# ---------------------------------------------------------------------------

def pin_pool_single_token_groups(orc):
    """g = 1: each core token is its own single token."""
    r = _rng(1)
    for Hq, Hkv in ((2, 2), (4, 2)):
        Q = r.standard_normal((2, Hq, 9, 8))
        K = r.standard_normal((2, Hkv, 9, 8))
        V = r.standard_normal((2, Hkv, 9, 8))
        Kc, Vc = orc.pool(Q, K, V, 1)
        np.testing.assert_allclose(Kc, K, rtol=0, atol=1e-14)
        np.testing.assert_allclose(Vc, V, rtol=0, atol=1e-14)


def pin_pool_two_token_closed_form(orc):
    """One group of two tokens, d = 4: the last query (2,0,0,0) scores
    k0 = e0 at 2/sqrt(4) = 1 and k1 = e1 at 0, so the weights are
    e/(e+1) and 1/(e+1)."""
    Q = np.zeros((1, 1, 2, 4))
    Q[0, 0, 0] = (-5.0, 3.0, 1.0, 0.5)  # first query: not the scorer
    Q[0, 0, 1] = (2.0, 0.0, 0.0, 0.0)
    K = np.zeros((1, 1, 2, 4))
    K[0, 0, 0, 0] = 1.0
    K[0, 0, 1, 1] = 1.0
    V = np.array([[[[1.0, 2.0, 3.0, 4.0], [5.0, 6.0, 7.0, 8.0]]]])
    a0 = math.e / (math.e + 1.0)
    a1 = 1.0 / (math.e + 1.0)
    Kc, Vc, A = orc.pool(Q, K, V, 2, want_weights=True)
    np.testing.assert_allclose(A[0, 0, 0], [a0, a1], rtol=1e-14)
    np.testing.assert_allclose(Kc[0, 0, 0], [a0, a1, 0.0, 0.0], atol=1e-15)
    np.testing.assert_allclose(
        Vc[0, 0, 0], [a0 * 1 + a1 * 5, a0 * 2 + a1 * 6, a0 * 3 + a1 * 7,
                      a0 * 4 + a1 * 8], rtol=1e-14)


def pin_pool_zero_query_is_group_mean(orc):
    """A zero scoring query gives equal weights: the core token is the plain
    mean of the group."""
    r = _rng(2)
    B, H, T, d, g = 1, 3, 20, 6, 5
    Q = r.standard_normal((B, H, T, d))
    Q[:, :, g - 1::g] = 0.0
    K = r.standard_normal((B, H, T, d))
    V = r.standard_normal((B, H, T, d))
    Kc, Vc = orc.pool(Q, K, V, g)
    np.testing.assert_allclose(Kc, K.reshape(B, H, T // g, g, d).mean(3),
                               atol=1e-14)
    np.testing.assert_allclose(Vc, V.reshape(B, H, T // g, g, d).mean(3),
                               atol=1e-14)


def pin_pool_scored_by_last_query(orc):
    """Only the query of the group's last token scores the group."""
    r = _rng(3)
    B, H, T, d, g = 2, 2, 24, 8, 4
    Q = r.standard_normal((B, H, T, d))
    K = r.standard_normal((B, H, T, d))
    V = r.standard_normal((B, H, T, d))
    Kc, Vc = orc.pool(Q, K, V, g)
    Q2 = Q.copy()
    mask = np.ones(T, bool)
    mask[g - 1::g] = False
    Q2[:, :, mask] = r.standard_normal(Q2[:, :, mask].shape) * 3
    Kc2, Vc2 = orc.pool(Q2, K, V, g)
    np.testing.assert_array_equal(Kc, Kc2)
    np.testing.assert_array_equal(Vc, Vc2)
    Q3 = Q.copy()
    Q3[:, :, g - 1::g] = r.standard_normal(Q3[:, :, g - 1::g].shape) * 3
    Kc3, _ = orc.pool(Q3, K, V, g)
    assert np.all(np.abs(Kc3 - Kc).max(-1) > 1e-6)


def pin_pool_identical_keys(orc):
    """If every key (and value) of a group is the same vector, the core
    token is that vector, whatever the scores."""
    r = _rng(4)
    B, Hq, Hkv, T, d, g = 1, 4, 2, 18, 5, 6
    base_k = r.standard_normal((B, Hkv, T // g, 1, d))
    base_v = r.standard_normal((B, Hkv, T // g, 1, d))
    K = np.broadcast_to(base_k, (B, Hkv, T // g, g, d)).reshape(B, Hkv, T, d)
    V = np.broadcast_to(base_v, (B, Hkv, T // g, g, d)).reshape(B, Hkv, T, d)
    Q = r.standard_normal((B, Hq, T, d)) * 4
    Kc, Vc = orc.pool(Q, K, V, g)
    np.testing.assert_allclose(Kc, base_k[:, :, :, 0], atol=1e-13)
    np.testing.assert_allclose(Vc, base_v[:, :, :, 0], atol=1e-13)


def pin_pool_weights_are_distributions(orc):
    r = _rng(5)
    for Hq, Hkv in ((3, 3), (6, 2)):
        Q = r.standard_normal((2, Hq, 35, 8)) * 3
        K = r.standard_normal((2, Hkv, 35, 8))
        V = r.standard_normal((2, Hkv, 35, 8))
        _, _, A = orc.pool(Q, K, V, 7, want_weights=True)
        assert A.shape == (2, Hkv, 5, 7)
        assert np.all(A >= 0)
        np.testing.assert_allclose(A.sum(-1), 1.0, atol=1e-13)


def pin_pool_gqa_mean_of_head_softmaxes(orc):
    """Two query heads share one key/value head (g = 3, d = 2).  Keys
    k0 = (1,0), k1 = k2 = 0.  Head 0's last query (L*sqrt2, 0) gives logits
    (L,0,0); head 1's gives (-L,0,0).  The core weights are the mean of the
    two softmax vectors (the reading taken for grouped-query attention)."""
    L = 3.0
    Q = np.zeros((1, 2, 3, 2))
    Q[0, 0, 2] = (L * math.sqrt(2.0), 0.0)
    Q[0, 1, 2] = (-L * math.sqrt(2.0), 0.0)
    K = np.zeros((1, 1, 3, 2))
    K[0, 0, 0] = (1.0, 0.0)
    V = np.array([[[[1.0, 0.0], [0.0, 1.0], [0.0, 0.0]]]])
    e = math.exp(L)
    p0 = np.array([e, 1.0, 1.0]) / (e + 2.0)
    p1 = np.array([1.0 / e, 1.0, 1.0]) / (1.0 / e + 2.0)
    a = (p0 + p1) / 2
    Kc, Vc, A = orc.pool(Q, K, V, 3, want_weights=True)
    np.testing.assert_allclose(A[0, 0, 0], a, rtol=1e-14)
    np.testing.assert_allclose(Kc[0, 0, 0], [a[0], 0.0], rtol=1e-14)
    np.testing.assert_allclose(Vc[0, 0, 0], [a[0], a[1]], rtol=1e-14)


def pin_pool_gqa_identical_queries_is_mha(orc):
    """With all query heads of a key/value head equal, grouped-query pooling
    equals pooling with that single head."""
    r = _rng(6)
    B, Hkv, rr, T, d, g = 2, 2, 3, 20, 8, 4
    Q1 = r.standard_normal((B, Hkv, T, d))
    Q = np.repeat(Q1, rr, axis=1)
    K = r.standard_normal((B, Hkv, T, d))
    V = r.standard_normal((B, Hkv, T, d))
    Kc, Vc = orc.pool(Q, K, V, g)
    Kc1, Vc1 = orc.pool(Q1, K, V, g)
    np.testing.assert_allclose(Kc, Kc1, atol=1e-14)
    np.testing.assert_allclose(Vc, Vc1, atol=1e-14)


def pin_pool_then_project_equals_project_then_pool(orc):
    """Section 全局感知池化 pools the tokens and then projects the core
    tokens with the shared W_K, W_V.  Pooling the raw tokens X with the
    weights the scores give (obtained by pooling X as the 'values') and then
    projecting must equal pooling K = X W_K and V = X W_V."""
    r = _rng(7)
    T, d, g = 32, 8, 4
    dm = d  # the oracle pools vectors of the head width
    X = r.standard_normal((1, 1, T, dm))
    WK = r.standard_normal((dm, d)) / 3
    WV = r.standard_normal((dm, d)) / 3
    WQ = r.standard_normal((dm, d)) / 3
    Q, K, V = X @ WQ, X @ WK, X @ WV
    Kc, Vc = orc.pool(Q, K, V, g)
    # pooling X itself: the scores depend on Q and K only
    _, C = orc.pool(Q, K, X, g)
    np.testing.assert_allclose(C @ WK, Kc, atol=1e-13)
    np.testing.assert_allclose(C @ WV, Vc, atol=1e-13)


# ---------------------------------------------------------------------------
# latent-condensed pooling, the LCA variant (page "Latent-Condensed
# Transformer for Efficient Long Context Modeling", section 2 方法论:
# 语义凝聚, 位置锚定)
# ---------------------------------------------------------------------------

def _lca_anchor_group():
    """One group of four tokens, d = 4, one head.  Queries (8,0,0,0), 0, 0, 0
    average to (2,0,0,0), so token i scores x_i * 2 / sqrt(4) = x_i for a
    key whose first entry is x_i.  With x = (0, ln 2, ln 4, 0) the weights
    are (1, 2, 4, 1) / 8 and token 2 is the anchor.  The last query is zero:
    it would give equal weights."""
    x = np.array([0.0, math.log(2.0), math.log(4.0), 0.0])
    Q = np.zeros((1, 1, 4, 4))
    Q[0, 0, 0, 0] = 8.0
    K = np.zeros((1, 1, 4, 4))
    K[0, 0, :, 0] = x
    K[0, 0, :, 1] = (1.0, -1.0, 0.5, 2.0)
    K[0, 0, :, 2] = (3.0, 5.0, -7.0, 11.0)
    K[0, 0, :, 3] = (-0.25, 0.75, 1.25, 0.5)
    V = np.arange(16.0).reshape(1, 1, 4, 4) - 6.0
    a = np.array([1.0, 2.0, 4.0, 1.0]) / 8.0
    return Q, K, V, a


def pin_lca_average_query_closed_form(orc):
    """Weights from the group's average query (not its last query, not the
    sum of its queries): (1, 2, 4, 1) / 8 for the group above."""
    Q, K, V, a = _lca_anchor_group()
    Kc, Vc, A, anchor = orc.lca_pool(Q, K, V, 4, 0, want_weights=True)
    np.testing.assert_allclose(A[0, 0, 0], a, rtol=1e-14)
    assert anchor[0, 0, 0] == 2
    np.testing.assert_allclose(Kc[0, 0, 0], a @ K[0, 0], rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(Vc[0, 0, 0], a @ V[0, 0], rtol=1e-13, atol=1e-15)


def pin_lca_anchor_keeps_positional_part(orc):
    """d_rope = 2: the last two entries of the core key are the anchor's
    own, (-7, 1.25) of token 2, copied, not pooled; the first two are
    pooled; the value is pooled in full."""
    Q, K, V, a = _lca_anchor_group()
    Kc, Vc = orc.lca_pool(Q, K, V, 4, 2)
    np.testing.assert_array_equal(Kc[0, 0, 0, 2:], [-7.0, 1.25])
    np.testing.assert_allclose(Kc[0, 0, 0, :2], (a @ K[0, 0])[:2], rtol=1e-13)
    np.testing.assert_allclose(Vc[0, 0, 0], a @ V[0, 0], rtol=1e-13, atol=1e-15)


def pin_lca_all_positional_is_selection(orc):
    """d_rope = d: the core key is the anchor's key row itself."""
    Q, K, V, a = _lca_anchor_group()
    Kc, Vc = orc.lca_pool(Q, K, V, 4, 4)
    np.testing.assert_array_equal(Kc[0, 0, 0], K[0, 0, 2])
    np.testing.assert_allclose(Vc[0, 0, 0], a @ V[0, 0], rtol=1e-13, atol=1e-15)


def pin_lca_only_the_query_mean_matters(orc):
    """Replacing a group's queries by others with the same mean changes
    nothing; changing the mean changes the result."""
    r = _rng(21)
    B, H, T, d, g = 2, 2, 24, 8, 4
    Q = r.standard_normal((B, H, T, d))
    K = r.standard_normal((B, H, T, d))
    V = r.standard_normal((B, H, T, d))
    Kc, Vc = orc.lca_pool(Q, K, V, g, 4)
    noise = r.standard_normal((B, H, T // g, g, d)) * 3
    noise -= noise.mean(axis=3, keepdims=True)
    Q2 = Q + noise.reshape(B, H, T, d)
    Kc2, Vc2 = orc.lca_pool(Q2, K, V, g, 4)
    np.testing.assert_allclose(Kc2, Kc, atol=1e-12)
    np.testing.assert_allclose(Vc2, Vc, atol=1e-12)
    Q3 = Q.copy()
    Q3[:, :, g - 1::g] += r.standard_normal(Q3[:, :, g - 1::g].shape) * 3
    _, Vc3 = orc.lca_pool(Q3, K, V, g, 4)
    assert np.all(np.abs(Vc3 - Vc).max(-1) > 1e-6)


def pin_lca_gqa_mean_of_head_softmaxes(orc):
    """Two query heads on one key/value head, g = 2, d = 2.  Head 0's
    queries average to (L sqrt2, 0), head 1's to (-L sqrt2, 0); with
    k0 = (1, 0), k1 = 0 the heads' softmaxes are (e^L, 1)/(e^L + 1) and
    (e^-L, 1)/(e^-L + 1), and the weights are their mean."""
    L = 2.0
    c = L * math.sqrt(2.0)
    Q = np.zeros((1, 2, 2, 2))
    Q[0, 0, 0] = (2 * c + 1.0, 3.0)
    Q[0, 0, 1] = (-1.0, -3.0)
    Q[0, 1, 0] = (-2 * c, 0.5)
    Q[0, 1, 1] = (0.0, -0.5)
    K = np.zeros((1, 1, 2, 2))
    K[0, 0, 0] = (1.0, 0.0)
    V = np.array([[[[1.0, 0.0], [0.0, 1.0]]]])
    e = math.exp(L)
    a = (np.array([e, 1.0]) / (e + 1.0) + np.array([1.0 / e, 1.0]) / (1.0 / e + 1.0)) / 2
    Kc, Vc, A, anchor = orc.lca_pool(Q, K, V, 2, 0, want_weights=True)
    np.testing.assert_allclose(A[0, 0, 0], a, rtol=1e-14)
    np.testing.assert_allclose(Vc[0, 0, 0], a, rtol=1e-14)
    assert anchor[0, 0, 0] == (0 if a[0] > a[1] else 1)


def pin_lca_permutation_within_group(orc):
    """Permuting a group's tokens (query, key and value rows together)
    leaves its core token unchanged: the average query and the weighted sums
    do not depend on the order, and the anchor moves with its token."""
    r = _rng(22)
    B, Hq, Hkv, T, d, g = 1, 4, 2, 30, 8, 6
    Q = r.standard_normal((B, Hq, T, d))
    K = r.standard_normal((B, Hkv, T, d))
    V = r.standard_normal((B, Hkv, T, d))
    perm = np.concatenate([j * g + r.permutation(g) for j in range(T // g)])
    Kc, Vc = orc.lca_pool(Q, K, V, g, 4)
    Kc2, Vc2 = orc.lca_pool(Q[:, :, perm], K[:, :, perm], V[:, :, perm], g, 4)
    np.testing.assert_allclose(Kc2, Kc, atol=1e-12)
    np.testing.assert_allclose(Vc2, Vc, atol=1e-12)


def pin_lca_tie_takes_first_token(orc):
    """Identical keys give equal weights: the anchor is the first token and
    the core key is that key."""
    r = _rng(23)
    Q = r.standard_normal((1, 1, 5, 8))
    K = np.broadcast_to(r.standard_normal((1, 1, 1, 8)), (1, 1, 5, 8)).copy()
    V = r.standard_normal((1, 1, 5, 8))
    Kc, Vc, A, anchor = orc.lca_pool(Q, K, V, 5, 3, want_weights=True)
    assert anchor[0, 0, 0] == 0
    np.testing.assert_allclose(A[0, 0, 0], 0.2, rtol=1e-14)
    np.testing.assert_allclose(Kc[0, 0, 0], K[0, 0, 0], atol=1e-14)
    np.testing.assert_allclose(Vc[0, 0, 0], V[0, 0].mean(0), atol=1e-14)


def pin_lca_one_query_per_group_is_cca(orc):
    """If every query of a group equals the group's last query, the average
    query is that query, and with no positional part the condensed token is
    CCA's pooled token (the earlier method of the same group, section
    全局感知池化 of the CCA write-up)."""
    r = _rng(24)
    B, Hq, Hkv, T, d, g = 2, 4, 2, 27, 8, 3
    Q = r.standard_normal((B, Hq, T, d))
    Ql = Q.reshape(B, Hq, T // g, g, d)[:, :, :, g - 1:g]
    Qs = np.broadcast_to(Ql, (B, Hq, T // g, g, d)).reshape(B, Hq, T, d)
    K = r.standard_normal((B, Hkv, T, d))
    V = r.standard_normal((B, Hkv, T, d))
    Kc, Vc = orc.lca_pool(Qs, K, V, g, 0)
    Kc1, Vc1 = orc.pool(Qs, K, V, g)
    np.testing.assert_allclose(Kc, Kc1, atol=1e-13)
    np.testing.assert_allclose(Vc, Vc1, atol=1e-13)


def pin_lca_trailing_partial_group(orc):
    """Tokens after the last complete group get no core token and do not
    change the complete groups' core tokens."""
    r = _rng(25)
    B, H, d, g = 1, 2, 8, 4
    Q = r.standard_normal((B, H, 23, d))
    K = r.standard_normal((B, H, 23, d))
    V = r.standard_normal((B, H, 23, d))
    Kc, Vc = orc.lca_pool(Q, K, V, g, 4)
    Kc2, Vc2 = orc.lca_pool(Q[:, :, :20], K[:, :, :20], V[:, :, :20], g, 4)
    assert Kc.shape == (B, H, 5, d)
    np.testing.assert_array_equal(Kc, Kc2)
    np.testing.assert_array_equal(Vc, Vc2)


def pin_lca_cache_condenses_as_lca_pool(orc):
    """The LCA decode cache (推理流程: groups condensed as tokens arrive,
    with the running sums of the open group's queries) ends with the same
    core tokens as condensing the whole sequence at once, keeps the open
    group's query sums, and its decode of token t is row t of the fused
    attention over those core tokens.  The ring (w + g slots) wraps."""
    r = _rng(26)
    B, Hq, Hkv, T, d, g, w, d_rope = 2, 4, 2, 75, 8, 4, 10, 4
    Q = r.standard_normal((B, Hq, T, d))
    K = r.standard_normal((B, Hkv, T, d))
    V = r.standard_normal((B, Hkv, T, d))
    Kc, Vc = orc.lca_pool(Q, K, V, g, d_rope)
    m = T // g
    c = orc.cache(B, Hq, Hkv, d, g, w, core_cap=m + 1)
    q_sum = np.zeros((B, Hq, d))
    for t in range(T):
        c.lca_append(q_sum, Q[:, :, t], K[:, :, t], V[:, :, t], d_rope)
        if t >= 40:
            np.testing.assert_allclose(c.decode(Q[:, :, t]),
                                       orc.attend_rows(Q, K, V, Kc, Vc, g, w, [t])[:, :, 0],
                                       atol=1e-12)
    np.testing.assert_allclose(c.k_core[:, :, :m], Kc, atol=1e-12)
    np.testing.assert_allclose(c.v_core[:, :, :m], Vc, atol=1e-12)
    np.testing.assert_allclose(q_sum, Q[:, :, m * g:].sum(axis=2), atol=1e-12)


# ---------------------------------------------------------------------------
# fused attention (sections 局部保留模块, 全局-局部模块可微融合)
# ---------------------------------------------------------------------------

def pin_prefill_g1_is_causal_attention(orc):
    """g = 1 makes every core token a raw token: whatever the window, the
    fused attention is ordinary causal attention."""
    r = _rng(8)
    for (Hq, Hkv, w) in ((2, 2, 0), (2, 2, 3), (4, 2, 7), (2, 1, 100)):
        Q = r.standard_normal((2, Hq, 23, 8))
        K = r.standard_normal((2, Hkv, 23, 8))
        V = r.standard_normal((2, Hkv, 23, 8))
        O = orc.prefill(Q, K, V, 1, w)
        np.testing.assert_allclose(O, _sdpa_causal(Q, K, V), atol=1e-12)


def pin_prefill_wide_window_is_causal_attention(orc):
    """A window covering the whole sequence leaves no core token in use."""
    r = _rng(9)
    for (T, g, w) in ((37, 4, 37), (40, 8, 64), (33, 5, 40)):
        Q = r.standard_normal((1, 2, T, 8))
        K = r.standard_normal((1, 2, T, 8))
        V = r.standard_normal((1, 2, T, 8))
        O = orc.prefill(Q, K, V, g, w)
        np.testing.assert_allclose(O, _sdpa_causal(Q, K, V), atol=1e-12)


def pin_prefill_constant_values(orc):
    """Attention averages values: constant values give that constant."""
    r = _rng(10)
    T, d = 50, 6
    Q = r.standard_normal((1, 2, T, d)) * 3
    K = r.standard_normal((1, 2, T, d)) * 3
    c = r.standard_normal(d)
    V = np.broadcast_to(c, (1, 2, T, d)).copy()
    O = orc.prefill(Q, K, V, 4, 9)
    np.testing.assert_allclose(O, np.broadcast_to(c, O.shape), atol=1e-13)


def pin_prefill_reachability_probe(orc):
    """Zero keys give every visible key the same logit, and one-hot values
    (V[i] = e_i) make output entry i the weight that token i receives.  So
    O[t] shows exactly which tokens query t reaches and how: raw tokens of
    the window get 1/n each, tokens inside a core token get 1/(g n) (a core
    token with equal weights is its group's mean), where n counts keys.
    Every token 0..t must be reached exactly once (introduction:
    "reachability"; section 全局-局部模块可微融合) and none after t; the raw
    ones must form the window the prose of section 局部保留模块 defines."""
    r = _rng(11)
    for (T, g, w) in ((64, 4, 10), (50, 8, 12), (48, 16, 16), (30, 3, 0)):
        Q = r.standard_normal((1, 1, T, T))
        K = np.zeros((1, 1, T, T))
        V = np.eye(T).reshape(1, 1, T, T)
        O = orc.prefill(Q, K, V, g, w)[0, 0]
        for t in range(T):
            s = _prose_window_start(t, g, w)
            n = s // g + (t - s + 1)
            expect = np.zeros(T)
            expect[:s] = 1.0 / (g * n)
            expect[s:t + 1] = 1.0 / n
            np.testing.assert_allclose(O[t], expect, atol=1e-14,
                                       err_msg=f"T={T} g={g} w={w} t={t}")


def _bruteforce_prefill(Q, K, V, Kc, Vc, g, w):
    """Dense masked attention over the extended key list [core ; raw], with
    the mask built from the prose: a core token of group j is visible to t
    if the whole group lies before t's window; raw token i if it lies in the
    window [s, t]."""
    B, Hq, T, d = Q.shape
    Hkv = K.shape[1]
    r = Hq // Hkv
    m = Kc.shape[2]
    O = np.zeros_like(Q)
    for b in range(B):
        for hq in range(Hq):
            h = hq // r
            keys = np.concatenate([Kc[b, h], K[b, h]], 0)
            vals = np.concatenate([Vc[b, h], V[b, h]], 0)
            mask = np.zeros((T, m + T), bool)
            for t in range(T):
                s = _prose_window_start(t, g, w)
                for j in range(m):
                    mask[t, j] = (j * g + g - 1) < s
                for i in range(T):
                    mask[t, m + i] = s <= i <= t
            logits = Q[b, hq] @ keys.T / math.sqrt(d)
            logits = np.where(mask, logits, -np.inf)
            logits -= logits.max(1, keepdims=True)
            p = np.exp(logits)
            p /= p.sum(1, keepdims=True)
            O[b, hq] = p @ vals
    return O


def pin_prefill_bruteforce(orc):
    r = _rng(12)
    for (B, Hq, Hkv, T, g, w) in ((1, 2, 2, 40, 4, 8), (2, 4, 2, 45, 4, 6),
                                  (1, 1, 1, 33, 5, 7), (1, 3, 1, 26, 2, 3),
                                  (1, 2, 2, 20, 8, 0)):
        d = 8
        Q = r.standard_normal((B, Hq, T, d))
        K = r.standard_normal((B, Hkv, T, d)) * 2
        V = r.standard_normal((B, Hkv, T, d))
        Kc, Vc = orc.pool(Q, K, V, g)
        O = orc.attend_rows(Q, K, V, Kc, Vc, g, w)
        np.testing.assert_allclose(
            O, _bruteforce_prefill(Q, K, V, Kc, Vc, g, w), atol=1e-12)
        rows = [T - 1, 0, g, w]
        O2 = orc.attend_rows(Q, K, V, Kc, Vc, g, w, rows)
        np.testing.assert_allclose(O2, O[:, :, rows], atol=0, rtol=0)


# ---------------------------------------------------------------------------
# decode cache (sections 基于 Triton 的底层加速, 计算和存储效率对比)
# ---------------------------------------------------------------------------

def pin_decode_matches_prefill(orc):
    """Generating token t against the cache gives the same output as row t
    of the fused attention over the whole sequence."""
    r = _rng(13)
    for (B, Hq, Hkv, T, d, g, w, extra) in ((2, 4, 2, 45, 8, 4, 6, 0),
                                            (1, 2, 2, 40, 8, 4, 6, 3),
                                            (1, 2, 2, 20, 4, 1, 0, 0),
                                            (1, 3, 1, 37, 4, 5, 3, 0),
                                            (1, 2, 2, 30, 4, 3, 7, 11)):
        Q = r.standard_normal((B, Hq, T, d))
        K = r.standard_normal((B, Hkv, T, d)) * 2
        V = r.standard_normal((B, Hkv, T, d))
        full = orc.prefill(Q, K, V, g, w)
        c = orc.cache(B, Hq, Hkv, d, g, w, core_cap=T // g + 1,
                      tail_cap=w + g + extra)
        for t in range(T):
            c.append(Q[:, :, t], K[:, :, t], V[:, :, t])
            assert c.len == t + 1
            o = c.decode(Q[:, :, t])
            np.testing.assert_allclose(o, full[:, :, t], atol=1e-12,
                                       err_msg=f"t={t}")


def pin_cache_slots(orc):
    """Core slot j holds the pooled group j; tail slot p mod tail_cap holds
    raw token p."""
    r = _rng(14)
    B, Hq, Hkv, T, d, g, w = 2, 4, 2, 43, 8, 4, 5
    Q = r.standard_normal((B, Hq, T, d))
    K = r.standard_normal((B, Hkv, T, d))
    V = r.standard_normal((B, Hkv, T, d))
    c = orc.cache(B, Hq, Hkv, d, g, w, core_cap=T // g + 2)
    for t in range(T):
        c.append(Q[:, :, t], K[:, :, t], V[:, :, t])
    Kc, Vc = orc.pool(Q, K, V, g)
    m = T // g
    np.testing.assert_allclose(c.k_core[:, :, :m], Kc, atol=1e-13)
    np.testing.assert_allclose(c.v_core[:, :, :m], Vc, atol=1e-13)
    for p in range(T - c.tail_cap, T):
        np.testing.assert_array_equal(c.k_tail[:, :, p % c.tail_cap],
                                      K[:, :, p])
        np.testing.assert_array_equal(c.v_tail[:, :, p % c.tail_cap],
                                      V[:, :, p])


def pin_cache_capacity(orc):
    """Appending a token whose group has no core slot is refused and leaves
    the cache as it was."""
    import oracle as _o

    B, Hq, Hkv, d, g, w = 1, 2, 2, 4, 4, 3
    c = orc.cache(B, Hq, Hkv, d, g, w, core_cap=2)
    z = np.ones((B, Hq, d))
    for _ in range(8):
        assert c.try_append(z, z, z) == _o.OK
    k_before = c.k_tail.copy()
    assert c.try_append(z * 2, z * 2, z * 2) == _o.ECAPACITY
    assert c.len == 8
    np.testing.assert_array_equal(c.k_tail, k_before)


def _read_golden(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                k, v = line.split("=")
                vals[k.strip()] = float(v)
    return vals


def pin_kv_cache_reduction_matches_page(orc):
    """The printed 93% KV-cache reduction at 128K: a cache of core slots for
    all groups plus a raw tail of w + g tokens, against a full cache of
    every token, rounds to the page's whole percent."""
    gv = _read_golden("kv_cache_reduction_128k.txt")
    T, g, w = int(gv["context_tokens"]), int(gv["g"]), int(gv["w"])
    c = orc.cache(1, 1, 1, 2, g, w, core_cap=T // g)
    cache_bytes = (c.k_core.nbytes + c.v_core.nbytes + c.k_tail.nbytes +
                   c.v_tail.nbytes)
    full_bytes = 2 * T * 2 * 8
    reduction = 100.0 * (1.0 - cache_bytes / full_bytes)
    assert round(reduction) == gv["reduction_percent"], reduction


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]

"""Pins of the fp64 gradient oracle (oracle/cca_backward.py).

Its forward is checked against the C oracle's forward (an independent
implementation of the same definitions), and its gradients against central
finite differences of the C oracle's forward:
    dL/dX[i] ~ (L(X + e_i h) - L(X - e_i h)) / 2h,  L = sum(dO * O).
The coordinates probed include the pooling queries (the last row of each
group), keys and values of groups that only reach the output through the
core stream, and window keys, so that a dropped path or a wrong sign in
either the attention or the pooling backward fails.
"""

import numpy as np
import pytest

import oracle
from oracle import cca_backward as bw

# (B, Hq, Hkv, T, d, g, w)
CASES = [
    (1, 2, 1, 37, 8, 4, 8),     # GQA r = 2, T mod g != 0
    (1, 2, 2, 24, 8, 1, 3),     # g = 1: the core keys are the tokens
    (1, 1, 1, 20, 4, 4, 64),    # window wider than the sequence: no core
    (2, 4, 2, 33, 8, 8, 8),     # two rows, r = 2
]


def _inputs(case, seed):
    B, Hq, Hkv, T, d, g, w = case
    rng = np.random.default_rng(seed)
    Q = rng.standard_normal((B, Hq, T, d))
    K = rng.standard_normal((B, Hkv, T, d)) * 1.5
    V = rng.standard_normal((B, Hkv, T, d))
    dO = rng.standard_normal((B, Hq, T, d))
    return Q, K, V, dO


@pytest.mark.parametrize("case", CASES, ids=[str(c) for c in CASES])
def test_forward_matches_c_oracle(case):
    Q, K, V, _ = _inputs(case, 11)
    g, w = case[5], case[6]
    np.testing.assert_allclose(bw.forward(Q, K, V, g, w), oracle.prefill(Q, K, V, g, w),
                               rtol=0, atol=1e-12)


def _probe_coords(case, rng, n=12):
    B, Hq, Hkv, T, d, g, w = case
    coords = {"Q": [], "K": [], "V": []}
    lasts = [i * g + g - 1 for i in range(T // g)]
    for _ in range(n):
        b = rng.integers(B)
        # queries: pooling rows first, then any row
        t = int(rng.choice(lasts)) if lasts and rng.random() < 0.6 else int(rng.integers(T))
        coords["Q"].append((b, rng.integers(Hq), t, rng.integers(d)))
        # keys/values: early groups (core path) and late rows (window)
        t = int(rng.integers(max(1, T // 3))) if rng.random() < 0.5 else int(rng.integers(T))
        coords["K"].append((b, rng.integers(Hkv), t, rng.integers(d)))
        t = int(rng.integers(max(1, T // 3))) if rng.random() < 0.5 else int(rng.integers(T))
        coords["V"].append((b, rng.integers(Hkv), t, rng.integers(d)))
    return coords


@pytest.mark.parametrize("case", CASES, ids=[str(c) for c in CASES])
def test_gradients_match_finite_differences(case):
    Q, K, V, dO = _inputs(case, 23)
    g, w = case[5], case[6]
    dQ, dK, dV = bw.backward(Q, K, V, g, w, dO)
    grads = {"Q": dQ, "K": dK, "V": dV}

    def loss(Qx, Kx, Vx):
        return float(np.sum(dO * oracle.prefill(Qx, Kx, Vx, g, w)))

    h = 1e-5
    coords = _probe_coords(case, np.random.default_rng(5))
    for name, idxs in coords.items():
        for idx in idxs:
            X = {"Q": Q, "K": K, "V": V}
            Xp = {k: v.copy() for k, v in X.items()}
            Xm = {k: v.copy() for k, v in X.items()}
            Xp[name][idx] += h
            Xm[name][idx] -= h
            fd = (loss(Xp["Q"], Xp["K"], Xp["V"]) - loss(Xm["Q"], Xm["K"], Xm["V"])) / (2 * h)
            an = grads[name][idx]
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(fd)), (name, idx, fd, an)


def test_pooling_path_carries_gradient():
    # a query row that is the last of a group gets gradient through the
    # pooling even when it attends only to itself and its window
    case = (1, 1, 1, 24, 4, 4, 4)
    Q, K, V, dO = _inputs(case, 31)
    dO[:, :, :12] = 0.0  # no gradient reaches rows < 12 directly
    dQ, _, _ = bw.backward(Q, K, V, 4, 4, dO)
    # rows 3 and 7 are pooling queries of groups 0 and 1, which rows >= 12
    # see as core keys; other early rows have no gradient at all
    assert np.abs(dQ[0, 0, 3]).max() > 1e-6 and np.abs(dQ[0, 0, 7]).max() > 1e-6
    for t in (0, 1, 2, 4, 5, 6, 8, 9, 10):
        assert np.abs(dQ[0, 0, t]).max() == 0.0


# Plausible mistakes, each planted in a copy of the gradient oracle's source:
# every one must be caught by the finite-difference pin above.
MUTANTS = [
    ("dK[b, h, sl] += np.outer(a, dKc[b, h, i])", "pass"),       # drops Kc -> K
    ("dV[b, h, sl] += np.outer(a, dVc[b, h, i])", "pass"),       # drops Vc -> V
    ("ds = da / r", "ds = da"),                                  # mean over heads
    ("dz = s * (ds - s @ ds)", "dz = s * ds"),                   # softmax Jacobian
    ("dx = p * (dp - p @ dp)", "dx = p * (dp + p @ dp)"),        # sign
    ("dKc[b, h, :nc] += dkeys[:nc]", "pass"),                    # core-key path
    ("dQ[b, h * r + k, l] += (dz @ Kg) * sc", "pass"),           # pooling query path
]


@pytest.mark.parametrize("mutant", MUTANTS, ids=[m[1] + " <- " + m[0][:20] for m in MUTANTS])
def test_finite_differences_catch_planted_mistakes(mutant):
    import types
    src = open(bw.__file__).read()
    old, new = mutant
    assert src.count(old) == 1, old
    mod = types.ModuleType("cca_backward_mutant")
    exec(compile(src.replace(old, new), "cca_backward_mutant", "exec"), mod.__dict__)
    case = (1, 2, 1, 37, 8, 4, 8)
    Q, K, V, dO = _inputs(case, 23)
    g, w = case[5], case[6]
    dQ, dK, dV = mod.backward(Q, K, V, g, w, dO)
    good = bw.backward(Q, K, V, g, w, dO)
    # the pin compares against finite differences; the correct gradients
    # pass it (test above), so a mutant that changes any probed value fails
    diffs = [np.abs(a - b).max() for a, b in zip((dQ, dK, dV), good)]
    assert max(diffs) > 1e-6, mutant
    coords = _probe_coords(case, np.random.default_rng(5))
    grads = {"Q": dQ, "K": dK, "V": dV}
    goodg = {"Q": good[0], "K": good[1], "V": good[2]}
    assert any(abs(grads[n][i] - goodg[n][i]) > 1e-6
               for n, idxs in coords.items() for i in idxs), ("not probed", mutant)

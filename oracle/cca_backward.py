"""Gradients of CCA-Attention in fp64 (test infrastructure, as the rest of
this package: only tests may use it; the CUDA library never does).

The write-up "ICML 2025 | 全局池化+局部保留，CCA-Attention为LLM长文本建模带来突破性
进展" calls the fusion of the global (core) and local streams differentiable
(section 全局-局部模块可微融合), and the authors' fused operator serves
training as well as inference (section 基于 Triton 的底层加速).  This module
gives, for upstream gradients dO of the fused attention output O, the
gradients dQ, dK, dV of L = sum(dO * O), where O depends on Q, K, V both
directly (local keys and values, and the queries) and through the pooled
core keys and values (section 全局感知池化: each group's last query scores
the group's keys; with grouped-query attention the weights are the mean of
the r mapped query heads' softmax vectors).

Everything is the chain rule written out step by step, in numpy fp64 with
plain loops over rows, for small cases.  `forward` restates the definition
so that the backward can reuse its intermediate values; the tests pin it to
the C oracle's forward, and pin `backward` to central finite differences of
that C forward.  No tensor-core blocking, online softmax or recomputation
tricks: this is the reference a backward kernel would be checked against.
"""

from __future__ import annotations

import numpy as np


def window_start(t: int, g: int, w: int) -> int:
    """ws(t) = g * floor(max(t - w, 0) / g) (section 局部保留模块)."""
    return g * (max(t - w, 0) // g)


def _softmax(x: np.ndarray) -> np.ndarray:
    e = np.exp(x - x.max())
    return e / e.sum()


def pool_forward(Q, K, V, g: int):
    """Pooled core keys/values and, per (b, kv head, group), the r query
    heads' softmax vectors (kept for the backward)."""
    B, Hq, T, d = Q.shape
    Hkv = K.shape[1]
    r = Hq // Hkv
    m = T // g
    Kc = np.zeros((B, Hkv, m, d))
    Vc = np.zeros((B, Hkv, m, d))
    S = np.zeros((B, Hkv, m, r, g))
    for b in range(B):
        for h in range(Hkv):
            for i in range(m):
                l = i * g + g - 1
                Kg, Vg = K[b, h, i * g:(i + 1) * g], V[b, h, i * g:(i + 1) * g]
                for k in range(r):
                    S[b, h, i, k] = _softmax(Kg @ Q[b, h * r + k, l] / np.sqrt(d))
                a = S[b, h, i].mean(axis=0)
                Kc[b, h, i] = a @ Kg
                Vc[b, h, i] = a @ Vg
    return Kc, Vc, S


def forward(Q, K, V, g: int, w: int):
    """O [B, Hq, T, d]: for each row t one softmax over the core keys of the
    groups before ws(t) and the raw keys ws(t) .. t (sections 局部保留模块 and
    全局-局部模块可微融合)."""
    B, Hq, T, d = Q.shape
    r = Hq // K.shape[1]
    Kc, Vc, _ = pool_forward(Q, K, V, g)
    O = np.zeros_like(Q)
    for b in range(B):
        for hq in range(Hq):
            h = hq // r
            for t in range(T):
                ws = window_start(t, g, w)
                nc = ws // g
                keys = np.concatenate([Kc[b, h, :nc], K[b, h, ws:t + 1]])
                vals = np.concatenate([Vc[b, h, :nc], V[b, h, ws:t + 1]])
                p = _softmax(keys @ Q[b, hq, t] / np.sqrt(d))
                O[b, hq, t] = p @ vals
    return O


def backward(Q, K, V, g: int, w: int, dO):
    """(dQ, dK, dV) of L = sum(dO * forward(Q, K, V, g, w))."""
    B, Hq, T, d = Q.shape
    Hkv = K.shape[1]
    r = Hq // Hkv
    sc = 1.0 / np.sqrt(d)
    Kc, Vc, S = pool_forward(Q, K, V, g)
    dQ, dK, dV = np.zeros_like(Q), np.zeros_like(K), np.zeros_like(V)
    dKc, dVc = np.zeros_like(Kc), np.zeros_like(Vc)
    # 1. the fused attention, row by row
    for b in range(B):
        for hq in range(Hq):
            h = hq // r
            for t in range(T):
                ws = window_start(t, g, w)
                nc = ws // g
                keys = np.concatenate([Kc[b, h, :nc], K[b, h, ws:t + 1]])
                vals = np.concatenate([Vc[b, h, :nc], V[b, h, ws:t + 1]])
                p = _softmax(keys @ Q[b, hq, t] * sc)
                dp = vals @ dO[b, hq, t]             # dL/dp
                dx = p * (dp - p @ dp)               # through the softmax
                dQ[b, hq, t] += (dx @ keys) * sc
                dkeys = np.outer(dx, Q[b, hq, t]) * sc
                dvals = np.outer(p, dO[b, hq, t])
                dKc[b, h, :nc] += dkeys[:nc]
                dVc[b, h, :nc] += dvals[:nc]
                dK[b, h, ws:t + 1] += dkeys[nc:]
                dV[b, h, ws:t + 1] += dvals[nc:]
    # 2. the pooling, group by group
    m = Kc.shape[2]
    for b in range(B):
        for h in range(Hkv):
            for i in range(m):
                l = i * g + g - 1
                sl = slice(i * g, (i + 1) * g)
                Kg, Vg = K[b, h, sl], V[b, h, sl]
                a = S[b, h, i].mean(axis=0)
                # Kc = a Kg, Vc = a Vg
                dK[b, h, sl] += np.outer(a, dKc[b, h, i])
                dV[b, h, sl] += np.outer(a, dVc[b, h, i])
                da = Kg @ dKc[b, h, i] + Vg @ dVc[b, h, i]
                # a = mean over the r heads of s_k = softmax(Kg q_k c)
                for k in range(r):
                    s = S[b, h, i, k]
                    ds = da / r
                    dz = s * (ds - s @ ds)
                    dQ[b, h * r + k, l] += (dz @ Kg) * sc
                    dK[b, h, sl] += np.outer(dz, Q[b, h * r + k, l]) * sc
    return dQ, dK, dV

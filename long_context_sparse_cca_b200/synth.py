"""Seeded synthetic inputs for the CCA-Attention hot path.

This module is shared by the GPU tests, the benchmark and the CPU oracle's
tests.  It holds no arithmetic of the method itself (no scoring, softmax,
pooling or attention): only random numbers, the bf16 storage format and the
workload shapes.

The shapes stand in for the workloads of the CCA write-up ("ICML 2025 |
全局池化+局部保留，CCA-Attention为LLM长文本建模带来突破性进展", section 实验设置):
single attention layers of LLaMA2-7B (32 heads, head dim 128) at 16K-128K
context.  The pages evaluate on LongBench-E, multi-document QA and
SlimPajama; none of those datasets is used here.  Values are N(0,1) with the
structure described per workload below.

Every tensor is generated with numpy's PCG64 generator from a fixed seed
(one stream per tensor, batch row and head), as float32, and rounded once to
bf16 (round to nearest even).  The GPU receives the bf16 bits; the
oracle receives exactly the same values widened to float64.
"""

from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np


# ----------------------------------------------------------------------------
# bf16 storage format
# ----------------------------------------------------------------------------

def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (round to nearest, ties to even).

    Returns the 16-bit patterns as uint16.  Inputs here are finite.
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    # add 0x7FFF plus the lowest kept bit, then truncate: round-half-even
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = (u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to float32 (exact)."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to float64 (exact)."""
    return bf16_bits_to_f32(b).astype(np.float64)


def f16_half_ulp(x: np.ndarray) -> np.ndarray:
    """Half the spacing of fp16 numbers around |x| (11 significant bits;
    spacing 2^-24 below the smallest normal 2^-14)."""
    a = np.abs(np.asarray(x, dtype=np.float64))
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -14)))
    return np.ldexp(1.0, (e - 11).astype(np.int64))


def bf16_half_ulp(x: np.ndarray) -> np.ndarray:
    """Half the spacing of bf16 numbers around |x| (the largest rounding error
    of a correctly rounded bf16 store of a value near x).

    bf16 keeps 8 significant bits, so values in [2^e, 2^(e+1)) are spaced
    2^(e-7) apart.
    """
    a = np.abs(np.asarray(x, dtype=np.float64))
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -126)))
    return np.ldexp(1.0, (e - 8).astype(np.int64))


# ----------------------------------------------------------------------------
# workloads
# ----------------------------------------------------------------------------

@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic workload.

    name        short identifier
    B, Hq, Hkv  batch, query heads, key/value heads (Hq % Hkv == 0)
    T           sequence length (prefill) or cached prefix length (decode)
    d           head dimension
    g, w        group size and local window of CCA-Attention
    steps       decode steps after the prefix (0 for prefill workloads)
    heavy_frac  fraction of (b, h, t) key rows multiplied by ``heavy_scale``
    head_scale  per-head scale drawn from U[lo, hi] (None: no scaling)
    seed        PCG64 seed
    """

    name: str
    B: int
    Hq: int
    Hkv: int
    T: int
    d: int
    g: int
    w: int
    steps: int = 0
    heavy_frac: float = 0.0
    heavy_scale: float = 4.0
    head_scale: Optional[tuple] = None
    seed: int = 1234

    @property
    def r(self) -> int:
        return self.Hq // self.Hkv

    @property
    def total_len(self) -> int:
        """Tokens in the generated sequence (prefix plus decode steps)."""
        return self.T + self.steps


# The five workloads.  Seeds are 1234 + index.
TINY = Workload("tiny_B1_H2_d64_T256_g16_w64", B=1, Hq=2, Hkv=2, T=256, d=64,
                g=16, w=64, seed=1235)
PREFILL_32K = Workload("prefill_B1_H32_d128_T32768_g16_w1024", B=1, Hq=32,
                       Hkv=32, T=32768, d=128, g=16, w=1024, heavy_frac=0.01,
                       seed=1236)
PREFILL_128K = Workload("prefill_B1_H32_d128_T131072_g16_w1024", B=1, Hq=32,
                        Hkv=32, T=131072, d=128, g=16, w=1024,
                        heavy_frac=0.01, seed=1237)
DECODE_64K = Workload("decode_B8_H32_d128_ctx65536_g16_w1024_steps256", B=8,
                      Hq=32, Hkv=32, T=65536, d=128, g=16, w=1024, steps=256,
                      seed=1238)
GQA_16K = Workload("gqa_B4_Hq32_Hkv8_d128_T16384_g32_w2048", B=4, Hq=32,
                   Hkv=8, T=16384, d=128, g=32, w=2048,
                   head_scale=(0.5, 2.0), seed=1239)

WORKLOADS = {wl.name: wl for wl in (TINY, PREFILL_32K, PREFILL_128K,
                                    DECODE_64K, GQA_16K)}


@dataclasses.dataclass
class Inputs:
    """Generated tensors as bf16 bit patterns, layout [B, H, T, d]."""

    q: np.ndarray  # uint16 [B, Hq, T, d]
    k: np.ndarray  # uint16 [B, Hkv, T, d]
    v: np.ndarray  # uint16 [B, Hkv, T, d]
    heavy: Optional[np.ndarray] = None  # bool [B, Hkv, T] rows scaled


_TENSOR_ID = {"q": 0, "k": 1, "v": 2}


def _slice_rng(seed: int, tensor: str, b: int, h: int) -> np.random.Generator:
    """Independent PCG64 stream for one (tensor, batch, head) slice."""
    return np.random.Generator(np.random.PCG64(
        np.random.SeedSequence([seed, _TENSOR_ID[tensor], b, h])))


def _fill_slice(out: np.ndarray, seed: int, tensor: str, b: int, h: int,
                scale: float, heavy_frac: float, heavy_scale: float,
                heavy_out: Optional[np.ndarray]) -> None:
    rng = _slice_rng(seed, tensor, b, h)
    T, d = out.shape
    rows = None
    if heavy_frac > 0:
        rows = rng.random(size=T) < heavy_frac
        heavy_out[:] = rows
    x = rng.standard_normal(size=(T, d), dtype=np.float32)
    if scale != 1.0:
        x *= np.float32(scale)
    if rows is not None:
        x[rows] *= np.float32(heavy_scale)
    out[:] = f32_to_bf16_bits(x)


def generate(wl: Workload, T: Optional[int] = None, B: Optional[int] = None,
             threads: Optional[int] = None) -> Inputs:
    """Generate Q, K, V for a workload.

    Each (tensor, batch, head) slice [T, d] has its own PCG64 stream seeded
    from (seed, tensor, b, h), so slices are generated in parallel and a
    reduced-B case holds exactly the leading batch rows of the full one.  In
    a K slice with heavy hitters, the row mask (Bernoulli(heavy_frac) per
    row) is drawn before the values.  Per-head scales (workloads with
    ``head_scale``) come from one extra stream seeded from (seed, 3): first
    the Hq query-head scales, then the Hkv key/value-head scales.

    ``T`` and ``B`` override the length / batch (reduced-size parity cases
    with the same value distribution).  For decode workloads the default
    length is prefix + steps.
    """
    import concurrent.futures as cf
    import os

    T = wl.total_len if T is None else int(T)
    B = wl.B if B is None else int(B)
    sq = np.ones(wl.Hq, dtype=np.float32)
    skv = np.ones(wl.Hkv, dtype=np.float32)
    if wl.head_scale is not None:
        lo, hi = wl.head_scale
        rng = np.random.Generator(np.random.PCG64(
            np.random.SeedSequence([wl.seed, 3])))
        sq = rng.uniform(lo, hi, size=wl.Hq).astype(np.float32)
        skv = rng.uniform(lo, hi, size=wl.Hkv).astype(np.float32)
    q = np.empty((B, wl.Hq, T, wl.d), dtype=np.uint16)
    k = np.empty((B, wl.Hkv, T, wl.d), dtype=np.uint16)
    v = np.empty((B, wl.Hkv, T, wl.d), dtype=np.uint16)
    heavy = (np.zeros((B, wl.Hkv, T), dtype=bool) if wl.heavy_frac > 0
             else None)
    jobs = []
    for b in range(B):
        for h in range(wl.Hq):
            jobs.append((q[b, h], "q", b, h, float(sq[h]), 0.0, None))
        for h in range(wl.Hkv):
            hv = heavy[b, h] if heavy is not None else None
            jobs.append((k[b, h], "k", b, h, float(skv[h]), wl.heavy_frac, hv))
            jobs.append((v[b, h], "v", b, h, float(skv[h]), 0.0, None))
    n = threads or min(32, os.cpu_count() or 1)
    with cf.ThreadPoolExecutor(max_workers=n) as ex:
        futs = [ex.submit(_fill_slice, out, wl.seed, t, b, h, s, hf,
                          wl.heavy_scale, hv)
                for (out, t, b, h, s, hf, hv) in jobs]
        for f in futs:
            f.result()
    return Inputs(q=q, k=k, v=v, heavy=heavy)


def random_bf16(shape, seed: int, scale: float = 1.0) -> np.ndarray:
    """N(0, scale^2) values rounded to bf16, as bit patterns."""
    rng = np.random.Generator(np.random.PCG64(seed))
    x = rng.standard_normal(size=shape, dtype=np.float32) * np.float32(scale)
    return f32_to_bf16_bits(x)

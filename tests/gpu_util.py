"""Helpers of the GPU parity tests: moving bf16 bit patterns to and from the
device, row sampling, and the comparison against the fp64 oracle.

Tolerances: max-abs 1e-2 and mean-abs 1e-3 between the CUDA result and the
oracle, on the same bf16 inputs.  For a tensor the library stores in a
16-bit format (fp16 Kc, Vc and core cache rows; bf16 O when asked for) the
check applies to the value before that final rounding: the stored value must
be the rounding of some number within the bounds of the oracle, i.e. the
error beyond half a spacing of the format at the stored value is held to
1e-2 (max) and 1e-3 (mean).  fp32 outputs are held to the bounds as they
are.
"""

from __future__ import annotations

import numpy as np

from long_context_sparse_cca_b200 import synth

TOL_MAX = 1e-2
TOL_MEAN = 1e-3


def to_cuda(bits: np.ndarray):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.to("cuda").view(torch.bfloat16)


def to_f64(t) -> np.ndarray:
    import torch
    if t.dtype == torch.bfloat16:
        return synth.bf16_bits_to_f64(t.view(torch.int16).cpu().numpy().view(np.uint16))
    return t.detach().double().cpu().numpy()


def stored_format(t):
    """'bf16', 'f16' or None (fp32) for a CUDA result tensor."""
    import torch
    return {torch.bfloat16: "bf16", torch.float16: "f16"}.get(t.dtype)


def to_bits(t) -> np.ndarray:
    """Bit patterns of a 16-bit (bf16 or fp16) CUDA tensor."""
    import torch
    assert t.dtype in (torch.bfloat16, torch.float16)
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def errors(got: np.ndarray, ref: np.ndarray, stored) -> dict:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), "non-finite values in the CUDA result"
    d = np.abs(got - ref)
    out = {"max_abs": float(d.max()) if d.size else 0.0,
           "mean_abs": float(d.mean()) if d.size else 0.0}
    if stored:
        half = synth.bf16_half_ulp(got) if stored == "bf16" else synth.f16_half_ulp(got)
        ex = np.maximum(d - half, 0.0)
        out["max_excess"] = float(ex.max()) if ex.size else 0.0
        out["mean_excess"] = float(ex.mean()) if ex.size else 0.0
    return out


def assert_close(got, ref, stored, what: str) -> dict:
    """``got`` is a CUDA tensor (its dtype gives the storage format) or an
    array with ``stored`` in (None, 'bf16', 'f16')."""
    if hasattr(got, "dtype") and not isinstance(got, np.ndarray):
        stored = stored_format(got)
        got = to_f64(got)
    e = errors(got, ref, stored)
    mx = e["max_excess"] if stored else e["max_abs"]
    mn = e["mean_excess"] if stored else e["mean_abs"]
    assert mx <= TOL_MAX and mn <= TOL_MEAN, f"{what}: {e}"
    return e


def sample_rows(T: int, g: int, w: int, n_random: int = 256, seed: int = 0):
    """Query rows for a full-size parity check: sequence start, group and
    window edges (every residue mod g around the window boundary), 128-row
    tile edges, the last 64 rows and seeded random rows."""
    rows = {0, 1, g - 1, g, g + 1, w - 1, w, w + 1, w + g - 1, w + g, w + g + 1,
            127, 128, 255, 256}
    for k in range(-g, 2 * g + 1):
        rows.add(w + k)
    for k in range(-2, 3):
        rows.add(T // 2 + k)
    rows.update(range(max(0, T - 64), T))
    rng = np.random.default_rng(seed)
    rows.update(int(x) for x in rng.integers(0, T, size=n_random))
    return np.array(sorted(r for r in rows if 0 <= r < T), dtype=np.int64)


# Gradient tolerance.  Gradients have no fixed scale (they grow with the
# upstream gradient and the number of keys a row attends to), so the error
# is measured against the reference's own size: the largest error at most
# 1% of the largest |reference| entry, the mean error at most 0.5% of the
# mean |reference|.  The GPU rounds P and dS to 16 bits before the tensor
# cores (relative error 2^-9 per term for bf16) and takes core keys and
# values in fp16, as the forward does; the forward's own bound (1e-2 on
# values of size ~1) is of the same order.
GRAD_TOL_MAX = 1e-2
GRAD_TOL_MEAN = 5e-3


def grad_errors(got: np.ndarray, ref: np.ndarray) -> dict:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    finite = bool(np.all(np.isfinite(got)))
    d = np.abs(got - ref)
    scale_max = float(np.abs(ref).max()) if ref.size else 0.0
    scale_mean = float(np.abs(ref).mean()) if ref.size else 0.0
    out = {"max_abs": float(d.max()) if d.size else 0.0,
           "mean_abs": float(d.mean()) if d.size else 0.0,
           "ref_max": scale_max, "ref_mean": scale_mean}
    out["ok"] = finite and out["max_abs"] <= GRAD_TOL_MAX * max(scale_max, 1e-12) and \
        out["mean_abs"] <= GRAD_TOL_MEAN * max(scale_mean, 1e-12)
    return out

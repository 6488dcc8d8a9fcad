"""CCA-Attention CPU oracle: test infrastructure only.

A ctypes front end over ``cca_oracle.c`` (fp64, OpenMP), the plain
restatement of CCA-Attention against which the CUDA library is checked.
``cca_backward.py`` adds the fp64 gradients (dQ, dK, dV through the fused
attention and the pooling), pinned to finite differences of the C forward.
Only the tests, the package's smoke check and the benchmark's CPU-baseline
leg may import this package; the CUDA library and its Python binding never
do, and the two share no code.

The method follows the write-up "ICML 2025 | 全局池化+局部保留，CCA-Attention
为LLM长文本建模带来突破性进展" (sections 全局感知池化, 局部保留模块,
全局-局部模块可微融合, 基于 Triton 的底层加速); the C source states, function
by function, the passage followed and the reading taken where it is open.
"""

from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "cca_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")

OK, EINVAL, ECAPACITY = 0, 1, 3


def build(force: bool = False) -> str:
    """Compile ``liboracle.so`` next to the source (gcc, -O2, OpenMP)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= max(
                os.path.getmtime(_SRC),
                os.path.getmtime(os.path.join(_HERE, "cca_oracle.h")))):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-std=c11", "-O2", "-fopenmp", "-fPIC", "-shared",
           "-Wall", "-Wextra", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


class _Cache(ctypes.Structure):
    _fields_ = [("k_core", ctypes.c_void_p), ("v_core", ctypes.c_void_p),
                ("k_tail", ctypes.c_void_p), ("v_tail", ctypes.c_void_p),
                ("B", ctypes.c_int), ("Hq", ctypes.c_int),
                ("Hkv", ctypes.c_int), ("d", ctypes.c_int),
                ("g", ctypes.c_int), ("w", ctypes.c_int),
                ("core_cap", ctypes.c_long), ("tail_cap", ctypes.c_long),
                ("len", ctypes.c_long)]


def _bind(path: str):
    L = ctypes.CDLL(path)
    P = ctypes.c_void_p
    i, l = ctypes.c_int, ctypes.c_long
    L.cca_oracle_set_threads.argtypes = [i]
    L.cca_oracle_set_threads.restype = i
    L.cca_oracle_threads.argtypes = []
    L.cca_oracle_threads.restype = i
    L.cca_oracle_window_start.argtypes = [l, l, l]
    L.cca_oracle_window_start.restype = l
    L.cca_oracle_pool.argtypes = [P, P, P, P, P, P, i, i, i, l, i, i]
    L.cca_oracle_pool.restype = i
    L.cca_oracle_lca_pool.argtypes = [P, P, P, P, P, P, P, i, i, i, l, i, i, i]
    L.cca_oracle_lca_pool.restype = i
    L.cca_oracle_attend_rows.argtypes = [P, P, P, P, P, i, i, i, l, i, i, i,
                                         P, l, P]
    L.cca_oracle_attend_rows.restype = i
    L.cca_oracle_cache_append.argtypes = [ctypes.POINTER(_Cache), P, P, P]
    L.cca_oracle_cache_append.restype = i
    L.cca_oracle_lca_cache_append.argtypes = [ctypes.POINTER(_Cache), P, P, P, P, i]
    L.cca_oracle_lca_cache_append.restype = i
    L.cca_oracle_decode.argtypes = [ctypes.POINTER(_Cache), P, P]
    L.cca_oracle_decode.restype = i
    return L


def _f64(x) -> np.ndarray:
    return np.ascontiguousarray(x, dtype=np.float64)


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


class OracleError(RuntimeError):
    pass


def _check(rc: int, what: str) -> None:
    if rc != OK:
        raise OracleError(f"{what}: oracle status {rc}")


class Oracle:
    """The oracle's entry points over one compiled copy of ``cca_oracle.c``
    (the default copy, or a test's deliberately altered one)."""

    def __init__(self, path: str):
        self.path = path
        self.lib = _bind(path)

    def set_threads(self, n: int) -> int:
        return self.lib.cca_oracle_set_threads(int(n))

    def threads(self) -> int:
        return self.lib.cca_oracle_threads()

    def window_start(self, t: int, g: int, w: int) -> int:
        """Start of the group-aligned local window of query t."""
        return int(self.lib.cca_oracle_window_start(int(t), int(g), int(w)))

    def pool(self, Q, K, V, g: int, want_weights: bool = False):
        """Globally-aware pooling.  Q [B,Hq,T,d], K/V [B,Hkv,T,d].

        Returns (Kc, Vc) [B,Hkv,m,d], plus the weights [B,Hkv,m,g] if asked.
        """
        Q, K, V = _f64(Q), _f64(K), _f64(V)
        B, Hq, T, d = Q.shape
        Hkv = K.shape[1]
        m = T // g
        Kc = np.empty((B, Hkv, m, d))
        Vc = np.empty((B, Hkv, m, d))
        A = np.empty((B, Hkv, m, g)) if want_weights else None
        _check(self.lib.cca_oracle_pool(_ptr(Q), _ptr(K), _ptr(V), _ptr(Kc),
                                        _ptr(Vc), _ptr(A), B, Hq, Hkv, T, d,
                                        g), "pool")
        return (Kc, Vc, A) if want_weights else (Kc, Vc)

    def lca_pool(self, Q, K, V, g: int, d_rope: int, want_weights: bool = False):
        """Latent-condensed pooling (the LCA variant).  Q [B,Hq,T,d],
        K/V [B,Hkv,T,d]; the last d_rope entries of a key row are its
        positional part.

        Returns (Kc, Vc) [B,Hkv,m,d], plus the weights [B,Hkv,m,g] and the
        anchor index per group [B,Hkv,m] if asked.
        """
        Q, K, V = _f64(Q), _f64(K), _f64(V)
        B, Hq, T, d = Q.shape
        Hkv = K.shape[1]
        m = T // g
        Kc = np.empty((B, Hkv, m, d))
        Vc = np.empty((B, Hkv, m, d))
        A = np.empty((B, Hkv, m, g)) if want_weights else None
        anchor = np.empty((B, Hkv, m), dtype=np.int64) if want_weights else None
        _check(self.lib.cca_oracle_lca_pool(_ptr(Q), _ptr(K), _ptr(V), _ptr(Kc),
                                            _ptr(Vc), _ptr(A), _ptr(anchor), B, Hq,
                                            Hkv, T, d, g, int(d_rope)), "lca_pool")
        return (Kc, Vc, A, anchor) if want_weights else (Kc, Vc)

    def attend_rows(self, Q, K, V, Kc, Vc, g: int, w: int,
                    rows: Optional[Sequence[int]] = None) -> np.ndarray:
        """Fused core + local attention at the listed query rows (all rows if
        None).  Returns O [B, Hq, len(rows), d]."""
        Q, K, V, Kc, Vc = _f64(Q), _f64(K), _f64(V), _f64(Kc), _f64(Vc)
        B, Hq, T, d = Q.shape
        Hkv = K.shape[1]
        if rows is None:
            rows = np.arange(T, dtype=np.int64)
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        O = np.empty((B, Hq, rows.size, d))
        _check(self.lib.cca_oracle_attend_rows(
            _ptr(Q), _ptr(K), _ptr(V), _ptr(Kc), _ptr(Vc), B, Hq, Hkv, T, d,
            g, w, _ptr(rows), rows.size, _ptr(O)), "attend_rows")
        return O

    def prefill(self, Q, K, V, g: int, w: int, rows=None) -> np.ndarray:
        """Pooling followed by the fused attention (all rows, or ``rows``)."""
        Kc, Vc = self.pool(Q, K, V, g)
        return self.attend_rows(Q, K, V, Kc, Vc, g, w, rows)

    def cache(self, B: int, Hq: int, Hkv: int, d: int, g: int, w: int,
              core_cap: int, tail_cap: Optional[int] = None) -> "Cache":
        return Cache(self, B, Hq, Hkv, d, g, w, core_cap, tail_cap)


class Cache:
    """The decode cache: core slots of completed groups plus a raw ring."""

    def __init__(self, orc: Oracle, B: int, Hq: int, Hkv: int, d: int,
                 g: int, w: int, core_cap: int,
                 tail_cap: Optional[int] = None):
        tail_cap = w + g if tail_cap is None else tail_cap
        self._lib = orc.lib
        self.k_core = np.zeros((B, Hkv, core_cap, d))
        self.v_core = np.zeros((B, Hkv, core_cap, d))
        self.k_tail = np.zeros((B, Hkv, tail_cap, d))
        self.v_tail = np.zeros((B, Hkv, tail_cap, d))
        self._c = _Cache(_ptr(self.k_core), _ptr(self.v_core),
                         _ptr(self.k_tail), _ptr(self.v_tail), B, Hq, Hkv, d,
                         g, w, core_cap, tail_cap, 0)

    @property
    def len(self) -> int:
        return int(self._c.len)

    @len.setter
    def len(self, n: int) -> None:
        self._c.len = int(n)

    @property
    def tail_cap(self) -> int:
        return int(self._c.tail_cap)

    @property
    def core_cap(self) -> int:
        return int(self._c.core_cap)

    def try_append(self, q, k, v) -> int:
        """q [B,Hq,d], k/v [B,Hkv,d]; returns the oracle status."""
        q, k, v = _f64(q), _f64(k), _f64(v)
        return self._lib.cca_oracle_cache_append(ctypes.byref(self._c),
                                                 _ptr(q), _ptr(k), _ptr(v))

    def append(self, q, k, v) -> None:
        _check(self.try_append(q, k, v), "append")

    def lca_append(self, q_sum: np.ndarray, q, k, v, d_rope: int) -> None:
        """LCA variant: append one token, condensing the group it completes
        with the open group's average queries.  q_sum [B,Hq,d] float64, the
        open group's query sums, is updated in place."""
        assert q_sum.dtype == np.float64 and q_sum.flags.c_contiguous
        q, k, v = _f64(q), _f64(k), _f64(v)
        _check(self._lib.cca_oracle_lca_cache_append(ctypes.byref(self._c), _ptr(q_sum),
                                                     _ptr(q), _ptr(k), _ptr(v), int(d_rope)),
               "lca_append")

    def decode(self, q) -> np.ndarray:
        q = _f64(q)
        o = np.empty(q.shape)
        _check(self._lib.cca_oracle_decode(ctypes.byref(self._c), _ptr(q),
                                           _ptr(o)), "decode")
        return o


_default: Optional[Oracle] = None


def default() -> Oracle:
    """The oracle built from the committed source."""
    global _default
    if _default is None:
        _default = Oracle(build())
    return _default


def build_variant(source: str, out_path: str) -> Oracle:
    """Compile an altered copy of the oracle source (used by the tests that
    check that each pin catches a planted mistake) and load it."""
    src = out_path + ".c"
    with open(src, "w") as f:
        f.write(source)
    cmd = ["gcc", "-std=c11", "-O2", "-fopenmp", "-fPIC", "-shared",
           "-I", _HERE, "-o", out_path, src, "-lm"]
    subprocess.run(cmd, check=True, capture_output=True)
    return Oracle(out_path)


def source() -> str:
    with open(_SRC) as f:
        return f.read()


# Module-level shortcuts to the default oracle.
def set_threads(n: int) -> int:
    return default().set_threads(n)


def threads() -> int:
    return default().threads()


def window_start(t: int, g: int, w: int) -> int:
    return default().window_start(t, g, w)


def pool(Q, K, V, g: int, want_weights: bool = False):
    return default().pool(Q, K, V, g, want_weights)


def lca_pool(Q, K, V, g: int, d_rope: int, want_weights: bool = False):
    return default().lca_pool(Q, K, V, g, d_rope, want_weights)


def attend_rows(Q, K, V, Kc, Vc, g: int, w: int, rows=None):
    return default().attend_rows(Q, K, V, Kc, Vc, g, w, rows)


def prefill(Q, K, V, g: int, w: int, rows=None):
    return default().prefill(Q, K, V, g, w, rows)


def new_cache(B, Hq, Hkv, d, g, w, core_cap, tail_cap=None) -> Cache:
    return default().cache(B, Hq, Hkv, d, g, w, core_cap, tail_cap)

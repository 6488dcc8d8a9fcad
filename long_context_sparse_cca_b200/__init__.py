"""CCA-Attention on NVIDIA B200: Python binding of the C library libcca.

Thin ctypes layer over ``include/cca.h``: it checks tensor devices, dtypes
and layouts, allocates outputs with PyTorch when the caller passes none, and
hands raw device pointers and the current CUDA stream to the library.  Every
step of the computation runs in the library's CUDA kernels; there is no
other code path.  If ``libcca.so`` is missing, every call raises.

Build the library with ``python -m long_context_sparse_cca_b200.build``.

Entry points (same names as the C ABI):
    cca_pool, cca_attn_prefill, cca_cache_prefill, cca_cache_append,
    cca_attn_prefill_lse (forward that keeps each row's log-sum-exp),
    cca_attn_backward, cca_attn_backward_workspace_bytes (training),
    cca_attn_decode, cca_decode_step (append + decode in one launch),
    cca_decode_workspace_bytes, cca_attn_decode_noalloc,
    cca_cache_append_rows, cca_attn_decode_rows (per-row lengths in device
    memory), cca_lca_pool, cca_lca_cache_prefill, cca_lca_cache_append (the
    LCA variant's condensation; ``lca_query_sums`` allocates the running
    query sums its cache calls keep), cca_selftest_wait_timeout,
    cca_device_status
and the ``Cache`` class holding a decode cache's device buffers.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libcca.so")

CCA_OK = 0
CCA_ERR_INVALID_ARG = 1
CCA_ERR_UNSUPPORTED = 2
CCA_ERR_CAPACITY = 3
CCA_ERR_CUDA = 4
CCA_ERR_TIMEOUT = 5
CCA_ERR_RANGE = 6
CCA_ERR_SCRATCH = 7
CCA_BF16 = 0
CCA_F32 = 1
NOALLOC_SCRATCH_BYTES = 4 << 20  # CCA_NOALLOC_SCRATCH_BYTES of include/cca.h

# Every symbol include/cca.h declares.
EXPORTS = ("cca_pool", "cca_attn_prefill", "cca_cache_prefill",
           "cca_cache_append", "cca_decode_workspace_bytes", "cca_attn_decode",
           "cca_device_status", "cca_status_string", "cca_version", "cca_last_error",
           "cca_attn_decode_noalloc", "cca_selftest_wait_timeout",
           "cca_cache_append_rows", "cca_attn_decode_rows", "cca_decode_step",
           "cca_attn_prefill_lse", "cca_attn_backward", "cca_attn_backward_workspace_bytes",
           "cca_lca_pool", "cca_lca_cache_prefill", "cca_lca_cache_append")


class CCAError(RuntimeError):
    """A nonzero status from libcca."""

    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)}")


class _CacheStruct(ctypes.Structure):
    _fields_ = [("k_core", ctypes.c_void_p), ("v_core", ctypes.c_void_p),
                ("k_tail", ctypes.c_void_p), ("v_tail", ctypes.c_void_p),
                ("B", ctypes.c_int), ("Hq", ctypes.c_int), ("Hkv", ctypes.c_int),
                ("d", ctypes.c_int), ("g", ctypes.c_int), ("w", ctypes.c_int),
                ("core_cap", ctypes.c_int64), ("tail_cap", ctypes.c_int64),
                ("len", ctypes.c_int64)]


_lib = None


def lib():
    """Load libcca.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"libcca.so not found at {LIB_PATH}; build it with "
            "`python -m long_context_sparse_cca_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    P, i, i64, st = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_int
    CP = ctypes.POINTER(_CacheStruct)
    L.cca_pool.argtypes = [P, P, P, P, P, i, i, i, i64, i, i, P]
    L.cca_pool.restype = st
    L.cca_attn_prefill.argtypes = [P, P, P, P, P, P, i, i, i, i, i64, i, i, i, P]
    L.cca_attn_prefill.restype = st
    L.cca_attn_prefill_lse.argtypes = [P, P, P, P, P, P, i, P, i, i, i, i64, i, i, i, P]
    L.cca_attn_prefill_lse.restype = st
    L.cca_attn_backward_workspace_bytes.argtypes = [i, i, i, i64, i, i]
    L.cca_attn_backward_workspace_bytes.restype = ctypes.c_size_t
    L.cca_attn_backward.argtypes = [P, P, P, P, P, P, i, P, P, P, P, P, i, i, i, i64, i, i, i,
                                    P, ctypes.c_size_t, P]
    L.cca_attn_backward.restype = st
    L.cca_lca_pool.argtypes = [P, P, P, P, P, i, i, i, i64, i, i, i, P]
    L.cca_lca_pool.restype = i
    L.cca_lca_cache_prefill.argtypes = [CP, P, P, P, P, i64, i, P]
    L.cca_lca_cache_prefill.restype = i
    L.cca_lca_cache_append.argtypes = [CP, P, P, P, P, i, P]
    L.cca_lca_cache_append.restype = i
    L.cca_cache_prefill.argtypes = [CP, P, P, P, i64, P]
    L.cca_cache_prefill.restype = st
    L.cca_cache_append.argtypes = [CP, P, P, P, P]
    L.cca_cache_append.restype = st
    L.cca_decode_workspace_bytes.argtypes = [CP]
    L.cca_decode_workspace_bytes.restype = ctypes.c_size_t
    L.cca_attn_decode.argtypes = [CP, P, P, i, P, ctypes.c_size_t, P]
    L.cca_attn_decode.restype = st
    L.cca_attn_decode_noalloc.argtypes = [CP, P, P, i, P]
    L.cca_attn_decode_noalloc.restype = st
    L.cca_decode_step.argtypes = [CP, P, P, P, P, i, P, ctypes.c_size_t, P]
    L.cca_decode_step.restype = st
    L.cca_cache_append_rows.argtypes = [CP, P, P, P, P, P]
    L.cca_cache_append_rows.restype = st
    L.cca_attn_decode_rows.argtypes = [CP, P, P, P, i, P, ctypes.c_size_t, P]
    L.cca_attn_decode_rows.restype = st
    L.cca_selftest_wait_timeout.argtypes = [ctypes.c_uint, P]
    L.cca_selftest_wait_timeout.restype = st
    L.cca_device_status.argtypes = [P]
    L.cca_device_status.restype = st
    L.cca_status_string.argtypes = [i]
    L.cca_status_string.restype = ctypes.c_char_p
    L.cca_version.argtypes = []
    L.cca_version.restype = ctypes.c_char_p
    L.cca_last_error.argtypes = []
    L.cca_last_error.restype = ctypes.c_char_p
    _lib = L
    return L


def status_string(status: int) -> str:
    return lib().cca_status_string(int(status)).decode()


def version() -> str:
    return lib().cca_version().decode()


def last_error() -> str:
    """CUDA error text behind this thread's last CCA_ERR_CUDA."""
    return lib().cca_last_error().decode()


def _check(status: int, what: str) -> None:
    if status != CCA_OK:
        if status == CCA_ERR_CUDA:
            what = f"{what} ({last_error()})"
        raise CCAError(status, what)


def _torch():
    import torch
    return torch


def _stream(stream) -> ctypes.c_void_p:
    torch = _torch()
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dev(t, name: str, dtype=None):
    """Pointer of a contiguous CUDA tensor (None passes NULL)."""
    if t is None:
        return None
    torch = _torch()
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    want = dtype or torch.bfloat16
    if t.dtype != want:
        raise ValueError(f"{name} must be {want}, got {t.dtype}")
    return ctypes.c_void_p(t.data_ptr())


def _odtype(out_dtype) -> int:
    torch = _torch()
    if out_dtype in (torch.bfloat16, "bf16"):
        return CCA_BF16
    if out_dtype in (torch.float32, "f32", "fp32"):
        return CCA_F32
    raise ValueError(f"unsupported output dtype {out_dtype}")


def cca_pool(Q, K, V, g: int, Kc=None, Vc=None, stream=None):
    """Globally-aware pooling: Q [B,Hq,T,d], K/V [B,Hkv,T,d] (bf16, CUDA).

    Returns (Kc, Vc) [B, Hkv, T // g, d] fp16.
    """
    torch = _torch()
    B, Hq, T, d = Q.shape
    Hkv = K.shape[1]
    m = T // g
    if Kc is None:
        Kc = torch.empty((B, Hkv, m, d), dtype=torch.float16, device=Q.device)
    if Vc is None:
        Vc = torch.empty((B, Hkv, m, d), dtype=torch.float16, device=Q.device)
    if tuple(K.shape) != (B, Hkv, T, d) or tuple(V.shape) != (B, Hkv, T, d):
        raise ValueError("K and V must be [B, Hkv, T, d]")
    if tuple(Kc.shape) != (B, Hkv, m, d) or tuple(Vc.shape) != (B, Hkv, m, d):
        raise ValueError("Kc and Vc must be [B, Hkv, T // g, d]")
    _check(lib().cca_pool(_dev(Q, "Q"), _dev(K, "K"), _dev(V, "V"),
                          _dev(Kc, "Kc", torch.float16), _dev(Vc, "Vc", torch.float16),
                          B, Hq, Hkv, T, d,
                          int(g), _stream(stream)), "cca_pool")
    return Kc, Vc


def cca_attn_prefill(Q, K, V, Kc, Vc, g: int, w: int, O=None,
                     out_dtype=None, stream=None):
    """Fused core + local attention over the whole sequence.

    Q [B,Hq,T,d], K/V [B,Hkv,T,d] (bf16), Kc/Vc [B,Hkv,T//g,d] (fp16).
    Returns O [B, Hq, T, d] in ``out_dtype`` (bf16 default, or fp32).
    """
    torch = _torch()
    B, Hq, T, d = Q.shape
    Hkv = K.shape[1]
    if O is None:
        dt = torch.bfloat16 if out_dtype is None else out_dtype
        O = torch.empty((B, Hq, T, d), dtype=dt, device=Q.device)
    od = _odtype(O.dtype)
    if tuple(O.shape) != (B, Hq, T, d):
        raise ValueError("O must be [B, Hq, T, d]")
    _check(lib().cca_attn_prefill(
        _dev(Q, "Q"), _dev(K, "K"), _dev(V, "V"), _dev(Kc, "Kc", torch.float16),
        _dev(Vc, "Vc", torch.float16), _dev(O, "O", O.dtype), od, B, Hq, Hkv, T, d, int(g),
        int(w), _stream(stream)), "cca_attn_prefill")
    return O


def cca_attn_prefill_lse(Q, K, V, Kc, Vc, g: int, w: int, O=None, out_dtype=None,
                         lse=None, stream=None):
    """cca_attn_prefill that also returns each row's log-sum-exp (fp32
    [B, Hq, T], log2 units), as cca_attn_backward needs: (O, lse)."""
    torch = _torch()
    B, Hq, T, d = Q.shape
    Hkv = K.shape[1]
    if O is None:
        dt = torch.bfloat16 if out_dtype is None else out_dtype
        O = torch.empty((B, Hq, T, d), dtype=dt, device=Q.device)
    if lse is None:
        lse = torch.empty((B, Hq, T), dtype=torch.float32, device=Q.device)
    od = _odtype(O.dtype)
    if tuple(O.shape) != (B, Hq, T, d) or tuple(lse.shape) != (B, Hq, T):
        raise ValueError("O must be [B, Hq, T, d] and lse [B, Hq, T]")
    _check(lib().cca_attn_prefill_lse(
        _dev(Q, "Q"), _dev(K, "K"), _dev(V, "V"), _dev(Kc, "Kc", torch.float16),
        _dev(Vc, "Vc", torch.float16), _dev(O, "O", O.dtype), od,
        _dev(lse, "lse", torch.float32), B, Hq, Hkv, T, d, int(g), int(w), _stream(stream)),
        "cca_attn_prefill_lse")
    return O, lse


def cca_attn_backward_workspace_bytes(B: int, Hq: int, Hkv: int, T: int, d: int, g: int) -> int:
    return int(lib().cca_attn_backward_workspace_bytes(int(B), int(Hq), int(Hkv), int(T),
                                                       int(d), int(g)))


def cca_attn_backward(Q, K, V, Kc, Vc, O, lse, dO, g: int, w: int, dQ=None, dK=None,
                      dV=None, workspace=None, stream=None):
    """Gradients (dQ, dK, dV), fp32, of sum(dO * O) for the CCA attention
    O = attention(Q, K, V) with its pooled Kc, Vc (from cca_pool) and the
    forward's O and lse (from cca_attn_prefill_lse).  dO: bf16 like Q."""
    torch = _torch()
    B, Hq, T, d = Q.shape
    Hkv = K.shape[1]
    f32 = dict(dtype=torch.float32, device=Q.device)
    dQ = torch.empty((B, Hq, T, d), **f32) if dQ is None else dQ
    dK = torch.empty((B, Hkv, T, d), **f32) if dK is None else dK
    dV = torch.empty((B, Hkv, T, d), **f32) if dV is None else dV
    nbytes = cca_attn_backward_workspace_bytes(B, Hq, Hkv, T, d, g)
    if workspace is None:
        workspace = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=Q.device)
    _check(lib().cca_attn_backward(
        _dev(Q, "Q"), _dev(K, "K"), _dev(V, "V"), _dev(Kc, "Kc", torch.float16),
        _dev(Vc, "Vc", torch.float16), _dev(O, "O", O.dtype), _odtype(O.dtype),
        _dev(lse, "lse", torch.float32), _dev(dO, "dO"), _dev(dQ, "dQ", torch.float32),
        _dev(dK, "dK", torch.float32), _dev(dV, "dV", torch.float32), B, Hq, Hkv, T, d, int(g),
        int(w), ctypes.c_void_p(workspace.data_ptr()), workspace.numel(), _stream(stream)),
        "cca_attn_backward")
    return dQ, dK, dV


class Cache:
    """A decode cache: core slots of completed groups (fp16) plus a raw ring
    of ``tail_cap`` tokens (bf16, default w + g), device buffers owned here."""

    def __init__(self, B: int, Hq: int, Hkv: int, d: int, g: int, w: int,
                 core_cap: int, tail_cap: Optional[int] = None, device="cuda"):
        torch = _torch()
        tail_cap = w + g if tail_cap is None else int(tail_cap)
        kw = dict(dtype=torch.bfloat16, device=device)
        kh = dict(dtype=torch.float16, device=device)
        self.k_core = torch.zeros((B, Hkv, core_cap, d), **kh)
        self.v_core = torch.zeros((B, Hkv, core_cap, d), **kh)
        self.k_tail = torch.zeros((B, Hkv, tail_cap, d), **kw)
        self.v_tail = torch.zeros((B, Hkv, tail_cap, d), **kw)
        self.struct = _CacheStruct(self.k_core.data_ptr(), self.v_core.data_ptr(),
                                   self.k_tail.data_ptr(), self.v_tail.data_ptr(),
                                   B, Hq, Hkv, d, g, w, core_cap, tail_cap, 0)
        self.workspace = None

    def row(self, b: int) -> "Cache":
        """Row b alone: a B = 1 cache over the same device buffers (for
        example to fill rows from prefixes of different lengths with
        cca_cache_prefill before decoding them with per-row lengths)."""
        v = object.__new__(Cache)
        v.k_core, v.v_core = self.k_core[b:b + 1], self.v_core[b:b + 1]
        v.k_tail, v.v_tail = self.k_tail[b:b + 1], self.v_tail[b:b + 1]
        st = self.struct
        v.struct = _CacheStruct(v.k_core.data_ptr(), v.v_core.data_ptr(),
                                v.k_tail.data_ptr(), v.v_tail.data_ptr(),
                                1, st.Hq, st.Hkv, st.d, st.g, st.w, st.core_cap,
                                st.tail_cap, 0)
        v.workspace = None
        return v

    def state_dict(self) -> dict:
        """Host copy of the cache (core slots, ring, shape, length), for
        saving and later restoring a decode session."""
        st = self.struct
        return {"shape": {n: int(getattr(st, n)) for n in
                          ("B", "Hq", "Hkv", "d", "g", "w", "core_cap", "tail_cap")},
                "len": int(st.len),
                "k_core": self.k_core.cpu(), "v_core": self.v_core.cpu(),
                "k_tail": self.k_tail.cpu(), "v_tail": self.v_tail.cpu()}

    @classmethod
    def from_state_dict(cls, state: dict, device="cuda") -> "Cache":
        """A cache on ``device`` holding what ``state_dict`` saved."""
        sh = state["shape"]
        c = cls(sh["B"], sh["Hq"], sh["Hkv"], sh["d"], sh["g"], sh["w"], sh["core_cap"],
                sh["tail_cap"], device=device)
        for n in ("k_core", "v_core", "k_tail", "v_tail"):
            getattr(c, n).copy_(state[n])
        c.len = state["len"]
        return c

    @property
    def len(self) -> int:
        return int(self.struct.len)

    @len.setter
    def len(self, n: int) -> None:
        self.struct.len = int(n)

    def __getattr__(self, name):
        if name in ("B", "Hq", "Hkv", "d", "g", "w", "core_cap", "tail_cap"):
            return getattr(self.struct, name)
        raise AttributeError(name)

    def nbytes(self) -> int:
        return sum(t.numel() * t.element_size() for t in
                   (self.k_core, self.v_core, self.k_tail, self.v_tail))


def cca_cache_prefill(cache: Cache, Q, K, V, stream=None) -> None:
    """Fill ``cache`` from a prefix Q [B,Hq,T,d], K/V [B,Hkv,T,d]."""
    T = Q.shape[2]
    _check(lib().cca_cache_prefill(ctypes.byref(cache.struct), _dev(Q, "Q"),
                                   _dev(K, "K"), _dev(V, "V"), T,
                                   _stream(stream)), "cca_cache_prefill")


def cca_cache_append(cache: Cache, q_t, k_t, v_t, stream=None) -> None:
    """Append one token: q_t [B,Hq,d], k_t/v_t [B,Hkv,d] (bf16, CUDA)."""
    _check(lib().cca_cache_append(ctypes.byref(cache.struct), _dev(q_t, "q_t"),
                                  _dev(k_t, "k_t"), _dev(v_t, "v_t"),
                                  _stream(stream)), "cca_cache_append")


# ---- the LCA variant: latent-condensed pooling with a positional anchor

def cca_lca_pool(Q, K, V, g: int, d_rope: int, Kc=None, Vc=None, stream=None):
    """LCA condensation: Q [B,Hq,T,d], K/V [B,Hkv,T,d] (bf16, CUDA); the last
    d_rope entries of a key row are its positional part.

    Returns (Kc, Vc) [B, Hkv, T // g, d] fp16, for cca_attn_prefill.
    """
    torch = _torch()
    B, Hq, T, d = Q.shape
    Hkv = K.shape[1]
    m = T // g
    if Kc is None:
        Kc = torch.empty((B, Hkv, m, d), dtype=torch.float16, device=Q.device)
    if Vc is None:
        Vc = torch.empty((B, Hkv, m, d), dtype=torch.float16, device=Q.device)
    if tuple(K.shape) != (B, Hkv, T, d) or tuple(V.shape) != (B, Hkv, T, d):
        raise ValueError("K and V must be [B, Hkv, T, d]")
    if tuple(Kc.shape) != (B, Hkv, m, d) or tuple(Vc.shape) != (B, Hkv, m, d):
        raise ValueError("Kc and Vc must be [B, Hkv, T // g, d]")
    _check(lib().cca_lca_pool(_dev(Q, "Q"), _dev(K, "K"), _dev(V, "V"),
                              _dev(Kc, "Kc", torch.float16), _dev(Vc, "Vc", torch.float16),
                              B, Hq, Hkv, T, d, int(g), int(d_rope), _stream(stream)),
           "cca_lca_pool")
    return Kc, Vc


def lca_query_sums(cache: Cache):
    """A zeroed q_sum [B, Hq, d] fp32 buffer for the LCA cache calls."""
    torch = _torch()
    return torch.zeros((cache.B, cache.Hq, cache.d), dtype=torch.float32, device="cuda")


def _qsum(cache: Cache, q_sum):
    torch = _torch()
    if tuple(q_sum.shape) != (cache.B, cache.Hq, cache.d):
        raise ValueError("q_sum must be [B, Hq, d]")
    return _dev(q_sum, "q_sum", torch.float32)


def cca_lca_cache_prefill(cache: Cache, q_sum, Q, K, V, d_rope: int, stream=None) -> None:
    """Fill ``cache`` from a prefix with LCA condensation; sets q_sum to the
    open group's query sums."""
    T = Q.shape[2]
    _check(lib().cca_lca_cache_prefill(ctypes.byref(cache.struct), _qsum(cache, q_sum),
                                       _dev(Q, "Q"), _dev(K, "K"), _dev(V, "V"), T,
                                       int(d_rope), _stream(stream)), "cca_lca_cache_prefill")


def cca_lca_cache_append(cache: Cache, q_sum, q_t, k_t, v_t, d_rope: int, stream=None) -> None:
    """Append one token with LCA condensation of the group it completes."""
    _check(lib().cca_lca_cache_append(ctypes.byref(cache.struct), _qsum(cache, q_sum),
                                      _dev(q_t, "q_t"), _dev(k_t, "k_t"), _dev(v_t, "v_t"),
                                      int(d_rope), _stream(stream)), "cca_lca_cache_append")


def cca_decode_workspace_bytes(cache: Cache) -> int:
    return int(lib().cca_decode_workspace_bytes(ctypes.byref(cache.struct)))


def cca_attn_decode(cache: Cache, q_t, o_t=None, out_dtype=None,
                    workspace=None, stream=None):
    """Attention of the newest token: q_t [B,Hq,d] -> o_t [B,Hq,d]."""
    torch = _torch()
    if o_t is None:
        dt = torch.bfloat16 if out_dtype is None else out_dtype
        o_t = torch.empty(tuple(q_t.shape), dtype=dt, device=q_t.device)
    od = _odtype(o_t.dtype)
    if workspace is None:
        workspace = _cache_workspace(cache, q_t.device)
    _check(lib().cca_attn_decode(
        ctypes.byref(cache.struct), _dev(q_t, "q_t"), _dev(o_t, "o_t", o_t.dtype),
        od, ctypes.c_void_p(workspace.data_ptr()), workspace.numel(),
        _stream(stream)), "cca_attn_decode")
    return o_t


def _cache_workspace(cache: Cache, device):
    """The cache's own decode workspace, zero-filled when (re)allocated, as
    cca_decode_step requires before its first use."""
    torch = _torch()
    nbytes = cca_decode_workspace_bytes(cache)
    if cache.workspace is None or cache.workspace.numel() < nbytes:
        cache.workspace = torch.zeros(max(nbytes, 256), dtype=torch.uint8, device=device)
    return cache.workspace


def cca_decode_step(cache: Cache, q_t, k_t, v_t, o_t=None, out_dtype=None,
                    workspace=None, stream=None):
    """Append token t = cache.len and return its attention output, in one
    launch: q_t [B,Hq,d], k_t/v_t [B,Hkv,d] (bf16) -> o_t [B,Hq,d].  A
    caller-provided workspace must have been zero-filled before its first
    use with this cache."""
    torch = _torch()
    if o_t is None:
        dt = torch.bfloat16 if out_dtype is None else out_dtype
        o_t = torch.empty(tuple(q_t.shape), dtype=dt, device=q_t.device)
    od = _odtype(o_t.dtype)
    if workspace is None:
        workspace = _cache_workspace(cache, q_t.device)
    _check(lib().cca_decode_step(
        ctypes.byref(cache.struct), _dev(q_t, "q_t"), _dev(k_t, "k_t"), _dev(v_t, "v_t"),
        _dev(o_t, "o_t", o_t.dtype), od, ctypes.c_void_p(workspace.data_ptr()),
        workspace.numel(), _stream(stream)), "cca_decode_step")
    return o_t


def _lens(lens):
    torch = _torch()
    if not (isinstance(lens, torch.Tensor) and lens.is_cuda and lens.dtype == torch.int64
            and lens.is_contiguous()):
        raise ValueError("lens must be a contiguous int64 CUDA tensor of B entries")
    return ctypes.c_void_p(lens.data_ptr())


def cca_cache_append_rows(cache: Cache, lens, q_t, k_t, v_t, stream=None) -> None:
    """Append one token per row, row b at position lens[b]; lens (int64,
    CUDA, [B]) is advanced on the device.  cache.len is not used."""
    if lens.numel() != cache.B:
        raise ValueError("lens needs one entry per batch row")
    _check(lib().cca_cache_append_rows(ctypes.byref(cache.struct), _lens(lens),
                                       _dev(q_t, "q_t"), _dev(k_t, "k_t"), _dev(v_t, "v_t"),
                                       _stream(stream)), "cca_cache_append_rows")


def cca_attn_decode_rows(cache: Cache, lens, q_t, o_t=None, out_dtype=None,
                         workspace=None, stream=None):
    """Attention of token lens[b] - 1 of every row b (lens: int64, CUDA, [B]):
    q_t [B,Hq,d] -> o_t [B,Hq,d].  Capturable in a CUDA graph."""
    torch = _torch()
    if lens.numel() != cache.B:
        raise ValueError("lens needs one entry per batch row")
    if o_t is None:
        dt = torch.bfloat16 if out_dtype is None else out_dtype
        o_t = torch.empty(tuple(q_t.shape), dtype=dt, device=q_t.device)
    od = _odtype(o_t.dtype)
    if workspace is None:
        workspace = _cache_workspace(cache, q_t.device)
    _check(lib().cca_attn_decode_rows(
        ctypes.byref(cache.struct), _lens(lens), _dev(q_t, "q_t"),
        _dev(o_t, "o_t", o_t.dtype), od, ctypes.c_void_p(workspace.data_ptr()),
        workspace.numel(), _stream(stream)), "cca_attn_decode_rows")
    return o_t


def cca_attn_decode_noalloc(cache: Cache, q_t, o_t=None, out_dtype=None, stream=None):
    """As cca_attn_decode, with the library's fixed device scratch in place
    of a workspace (for callers that cannot allocate device memory)."""
    torch = _torch()
    if o_t is None:
        dt = torch.bfloat16 if out_dtype is None else out_dtype
        o_t = torch.empty(tuple(q_t.shape), dtype=dt, device=q_t.device)
    od = _odtype(o_t.dtype)
    _check(lib().cca_attn_decode_noalloc(
        ctypes.byref(cache.struct), _dev(q_t, "q_t"), _dev(o_t, "o_t", o_t.dtype), od,
        _stream(stream)), "cca_attn_decode_noalloc")
    return o_t


def cca_selftest_wait_timeout(limit_us: int = 1000, stream=None) -> None:
    """Launch the failure-path self-test kernel: a bounded wait on a barrier
    that nothing completes.  cca_device_status() afterwards returns
    CCA_ERR_TIMEOUT; the context stays usable."""
    _check(lib().cca_selftest_wait_timeout(int(limit_us), _stream(stream)),
           "cca_selftest_wait_timeout")


def cca_device_status(stream=None) -> int:
    """Synchronise the stream; return the library's device status
    (CCA_OK, CCA_ERR_TIMEOUT, CCA_ERR_RANGE or CCA_ERR_CUDA)."""
    return int(lib().cca_device_status(_stream(stream)))

"""The C-ABI library on the CPU: it builds, loads without a GPU, exports
every entry point include/cca.h declares, and rejects bad arguments on the
host before any launch (so these calls never reach the GPU)."""

import ctypes
import os
import re

import pytest

import long_context_sparse_cca_b200 as cca
from long_context_sparse_cca_b200 import build as cca_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FAKE = 0x10000  # aligned, never dereferenced: every call below fails its checks


@pytest.fixture(scope="module")
def L():
    cca_build.build()
    return cca.lib()


def _declared():
    with open(os.path.join(ROOT, "include", "cca.h")) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(cca_[a-z_]+)\s*\(", text)))


def test_exports_every_declared_symbol(L):
    declared = _declared()
    assert len(declared) >= 9
    for name in declared:
        assert hasattr(L, name), name
    assert sorted(declared) == sorted(cca.EXPORTS)


def test_status_strings(L):
    assert cca.status_string(cca.CCA_OK) == "CCA_OK"
    assert cca.status_string(cca.CCA_ERR_TIMEOUT) == "CCA_ERR_TIMEOUT"
    assert cca.status_string(99) == "CCA_ERR_UNKNOWN"
    assert re.match(r"\d+\.\d+\.\d+", cca.version())


def _pool(L, Q=FAKE, K=FAKE, V=FAKE, Kc=FAKE + 4096, Vc=FAKE + 8192, B=1,
          Hq=2, Hkv=2, T=64, d=128, g=16):
    P = ctypes.c_void_p
    return L.cca_pool(P(Q), P(K), P(V), P(Kc), P(Vc), B, Hq, Hkv, T, d, g, None)


def test_pool_argument_checks(L):
    assert _pool(L, Q=0) == cca.CCA_ERR_INVALID_ARG
    assert _pool(L, K=FAKE + 2) == cca.CCA_ERR_INVALID_ARG  # misaligned
    assert _pool(L, d=96) == cca.CCA_ERR_UNSUPPORTED
    assert _pool(L, Hq=3, Hkv=2) == cca.CCA_ERR_INVALID_ARG
    assert _pool(L, g=0) == cca.CCA_ERR_INVALID_ARG
    assert _pool(L, g=257) == cca.CCA_ERR_UNSUPPORTED
    assert _pool(L, T=-1) == cca.CCA_ERR_INVALID_ARG
    assert _pool(L, B=0) == cca.CCA_ERR_INVALID_ARG
    # output overlapping an input
    assert _pool(L, Kc=FAKE) == cca.CCA_ERR_INVALID_ARG
    # no complete group: nothing to do, null pointers allowed
    assert _pool(L, Q=0, K=0, V=0, Kc=0, Vc=0, T=15) == cca.CCA_OK


def test_prefill_argument_checks(L):
    P = ctypes.c_void_p

    def call(O=FAKE + (1 << 24), od=0, d=128, T=300, g=16, w=64, Kc=FAKE + (1 << 20)):
        return L.cca_attn_prefill(P(FAKE), P(FAKE), P(FAKE), P(Kc), P(Kc + 4096), P(O),
                                  od, 1, 2, 2, T, d, g, w, None)

    assert call(od=7) == cca.CCA_ERR_INVALID_ARG
    assert call(O=0) == cca.CCA_ERR_INVALID_ARG
    assert call(O=FAKE) == cca.CCA_ERR_INVALID_ARG  # O aliases Q
    assert call(d=32) == cca.CCA_ERR_UNSUPPORTED
    assert call(w=-1) == cca.CCA_ERR_INVALID_ARG
    assert call(T=0, O=0) == cca.CCA_OK  # empty sequence
    assert call(Kc=0) == cca.CCA_ERR_INVALID_ARG  # T // g > 0 needs Kc
    assert call(Kc=FAKE + (1 << 20) + 8) == cca.CCA_ERR_INVALID_ARG  # misaligned
    assert call(O=FAKE + (1 << 24) + 16) == cca.CCA_ERR_INVALID_ARG  # O not 32-byte aligned


def _cache(B=1, Hq=2, Hkv=2, d=128, g=16, w=64, core_cap=8, tail_cap=80, length=0,
           ptrs=True):
    base = FAKE if ptrs else 0
    return cca._CacheStruct(base, base + (1 << 20), base + (2 << 20), base + (3 << 20),
                            B, Hq, Hkv, d, g, w, core_cap, tail_cap, length)


def test_cache_checks(L):
    P = ctypes.c_void_p
    c = _cache(tail_cap=79)  # below w + g
    assert L.cca_cache_append(ctypes.byref(c), P(FAKE), P(FAKE), P(FAKE),
                              None) == cca.CCA_ERR_INVALID_ARG
    c = _cache(core_cap=2, length=32)  # token 32 belongs to group 2: no slot
    assert L.cca_cache_append(ctypes.byref(c), P(FAKE), P(FAKE), P(FAKE),
                              None) == cca.CCA_ERR_CAPACITY
    assert c.len == 32
    c = _cache(core_cap=2)
    assert L.cca_cache_prefill(ctypes.byref(c), P(FAKE), P(FAKE), P(FAKE), 33,
                               None) == cca.CCA_ERR_CAPACITY
    assert c.len == 0
    c = _cache(Hq=64, Hkv=2)
    assert L.cca_decode_workspace_bytes(ctypes.byref(c)) == 0  # r > 16
    c = _cache()
    ws = L.cca_decode_workspace_bytes(ctypes.byref(c))
    assert ws > 0
    c.len = 0
    assert L.cca_attn_decode(ctypes.byref(c), P(FAKE), P(FAKE + 4096), 0, P(FAKE),
                             ws, None) == cca.CCA_ERR_INVALID_ARG  # empty cache
    c.len = 10
    assert L.cca_attn_decode(ctypes.byref(c), P(FAKE), P(FAKE + 4096), 0, P(FAKE),
                             ws - 1, None) == cca.CCA_ERR_INVALID_ARG  # small ws
    assert L.cca_attn_decode(ctypes.byref(c), P(FAKE), P(FAKE + 4096), 0,
                             P(FAKE + 16), ws, None) == cca.CCA_ERR_INVALID_ARG
    assert L.cca_attn_decode(ctypes.byref(c), P(FAKE), P(FAKE + 4096), 3, P(FAKE),
                             ws, None) == cca.CCA_ERR_INVALID_ARG  # dtype


def test_decode_step_argument_checks(L):
    """cca_decode_step refuses bad arguments and a full cache before any
    launch, and leaves the cache length unchanged."""
    P = ctypes.c_void_p
    c = _cache(length=10)
    ws = L.cca_decode_workspace_bytes(ctypes.byref(c))
    args = lambda q=FAKE, k=FAKE + 8192, v=FAKE + 16384, o=FAKE + 4096, dt=0, w=FAKE, n=ws: (  # noqa: E731
        ctypes.byref(c), P(q), P(k), P(v), P(o), dt, P(w), n, None)
    assert L.cca_decode_step(*args(q=0)) == cca.CCA_ERR_INVALID_ARG
    assert L.cca_decode_step(*args(k=FAKE + 8)) == cca.CCA_ERR_INVALID_ARG  # misaligned
    assert L.cca_decode_step(*args(n=ws - 1)) == cca.CCA_ERR_INVALID_ARG
    assert L.cca_decode_step(*args(w=FAKE + 16)) == cca.CCA_ERR_INVALID_ARG  # 256-byte
    assert L.cca_decode_step(*args(dt=3)) == cca.CCA_ERR_INVALID_ARG
    assert L.cca_decode_step(*args(o=FAKE)) == cca.CCA_ERR_INVALID_ARG  # o_t overlaps q_t
    assert c.len == 10
    c = _cache(core_cap=2, length=32)  # token 32 belongs to group 2: no slot
    ws = L.cca_decode_workspace_bytes(ctypes.byref(c))
    assert L.cca_decode_step(ctypes.byref(c), P(FAKE), P(FAKE + 8192), P(FAKE + 16384),
                             P(FAKE + 4096), 0, P(FAKE + (8 << 20)), ws,
                             None) == cca.CCA_ERR_CAPACITY
    assert c.len == 32
    bad = _cache(tail_cap=10)
    assert L.cca_decode_step(ctypes.byref(bad), P(FAKE), P(FAKE + 8192), P(FAKE + 16384),
                             P(FAKE + 4096), 0, P(FAKE), 1 << 20,
                             None) == cca.CCA_ERR_INVALID_ARG


def test_noalloc_decode_refuses_oversized_cache(L):
    """A cache whose decode workspace exceeds the library's fixed scratch is
    refused before anything touches the GPU."""
    P = ctypes.c_void_p
    c = _cache(B=64, Hq=32, Hkv=32, core_cap=2048, length=100)
    need = L.cca_decode_workspace_bytes(ctypes.byref(c))
    assert need > cca.NOALLOC_SCRATCH_BYTES
    st = L.cca_attn_decode_noalloc(ctypes.byref(c), P(FAKE), P(FAKE + 4096), 1, None)
    assert st == cca.CCA_ERR_SCRATCH
    assert cca.status_string(st) == "CCA_ERR_SCRATCH"
    bad = _cache(tail_cap=10)  # invalid cache: the cache's own error
    assert L.cca_attn_decode_noalloc(ctypes.byref(bad), P(FAKE), P(FAKE + 4096), 1,
                                     None) == cca.CCA_ERR_INVALID_ARG


def test_noalloc_scratch_size_matches_header():
    with open(os.path.join(ROOT, "include", "cca.h")) as f:
        m = re.search(r"#define CCA_NOALLOC_SCRATCH_BYTES \((\d+)u << (\d+)\)", f.read())
    assert m and int(m.group(1)) << int(m.group(2)) == cca.NOALLOC_SCRATCH_BYTES


def test_workspace_grows_with_capacity(L):
    a = _cache(core_cap=8)
    b = _cache(core_cap=4096)
    assert L.cca_decode_workspace_bytes(ctypes.byref(b)) > \
        L.cca_decode_workspace_bytes(ctypes.byref(a))


def test_binding_refuses_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(cca, "_lib", None)
    monkeypatch.setattr(cca, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="libcca.so not found"):
        cca.lib()


def test_selftest_limit_checks(L):
    # out-of-range limits are refused on the host, before any launch
    assert L.cca_selftest_wait_timeout(0, None) == cca.CCA_ERR_INVALID_ARG
    assert L.cca_selftest_wait_timeout(2000001, None) == cca.CCA_ERR_INVALID_ARG


def test_cache_state_round_trip():
    # save/restore of a decode session is a host copy of the caller-owned
    # buffers plus the length (tensors on the CPU here; no kernel runs)
    import torch
    c = cca.Cache(2, 4, 2, 64, 16, 32, core_cap=8, device="cpu")
    for t in (c.k_core, c.v_core, c.k_tail, c.v_tail):
        t.copy_(torch.randn(t.shape).to(t.dtype))
    c.len = 77
    st = c.state_dict()
    d = cca.Cache.from_state_dict(st, device="cpu")
    assert d.len == 77 and (d.B, d.Hq, d.Hkv, d.d, d.g, d.w, d.core_cap, d.tail_cap) == \
        (2, 4, 2, 64, 16, 32, 8, 48)
    for n in ("k_core", "v_core", "k_tail", "v_tail"):
        assert torch.equal(getattr(c, n), getattr(d, n))
        assert getattr(d, n).data_ptr() != getattr(c, n).data_ptr()


def test_rows_argument_checks(L):
    """The per-row calls check their arguments on the host, before any
    launch: every call below fails there."""
    P = ctypes.c_void_p
    c = _cache()
    ws = L.cca_decode_workspace_bytes(ctypes.byref(c))
    lens = FAKE + (5 << 20)
    # lens missing or misaligned
    for bad in (0, lens + 4):
        assert L.cca_cache_append_rows(ctypes.byref(c), P(bad), P(FAKE), P(FAKE), P(FAKE),
                                       None) == cca.CCA_ERR_INVALID_ARG
        assert L.cca_attn_decode_rows(ctypes.byref(c), P(bad), P(FAKE), P(FAKE + 4096), 0,
                                      P(FAKE), ws, None) == cca.CCA_ERR_INVALID_ARG
    # invalid cache, output dtype, workspace size and alignment
    bad = _cache(tail_cap=10)
    assert L.cca_cache_append_rows(ctypes.byref(bad), P(lens), P(FAKE), P(FAKE), P(FAKE),
                                   None) == cca.CCA_ERR_INVALID_ARG
    assert L.cca_attn_decode_rows(ctypes.byref(c), P(lens), P(FAKE), P(FAKE + 4096), 3,
                                  P(FAKE), ws, None) == cca.CCA_ERR_INVALID_ARG
    assert L.cca_attn_decode_rows(ctypes.byref(c), P(lens), P(FAKE), P(FAKE + 4096), 0,
                                  P(FAKE), ws - 1, None) == cca.CCA_ERR_INVALID_ARG
    assert L.cca_attn_decode_rows(ctypes.byref(c), P(lens), P(FAKE), P(FAKE + 4096), 0,
                                  P(FAKE + 16), ws, None) == cca.CCA_ERR_INVALID_ARG
    # one block per row holds one warp per key/value head: at most 32
    wide = _cache(Hq=64, Hkv=64)
    assert L.cca_cache_append_rows(ctypes.byref(wide), P(lens), P(FAKE), P(FAKE), P(FAKE),
                                   None) == cca.CCA_ERR_UNSUPPORTED


def test_rows_binding_checks_lens():
    import torch
    c = cca.Cache(2, 2, 2, 64, 16, 32, core_cap=4, device="cpu")
    q = torch.zeros((2, 2, 64), dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        cca.cca_cache_append_rows(c, torch.zeros(3, dtype=torch.int64), q, q, q)
    with pytest.raises(ValueError):
        cca.cca_attn_decode_rows(c, torch.zeros(2, dtype=torch.int32), q)


def test_lca_argument_checks(L):
    """The LCA calls refuse a bad d_rope, bad pointers and a full cache on
    the host, before any launch; a refused append leaves the length."""
    P = ctypes.c_void_p

    def lpool(Q=FAKE, Kc=FAKE + 4096, d_rope=64, T=64, d=128):
        return L.cca_lca_pool(P(Q), P(FAKE), P(FAKE), P(Kc), P(FAKE + 8192), 1, 2, 2, T, d,
                              16, d_rope, None)

    assert lpool(d_rope=4) == cca.CCA_ERR_INVALID_ARG   # not a multiple of 8
    assert lpool(d_rope=-8) == cca.CCA_ERR_INVALID_ARG
    assert lpool(d_rope=136) == cca.CCA_ERR_INVALID_ARG  # beyond d
    assert lpool(Q=0) == cca.CCA_ERR_INVALID_ARG
    assert lpool(Kc=FAKE) == cca.CCA_ERR_INVALID_ARG     # output overlaps an input
    assert lpool(d=96) == cca.CCA_ERR_UNSUPPORTED
    assert L.cca_lca_pool(None, None, None, None, None, 1, 2, 2, 15, 128, 16, 0,
                          None) == cca.CCA_OK            # no complete group

    QS = FAKE + (8 << 20)
    c = _cache(length=10)
    app = lambda qs=QS, q=FAKE, d_rope=64: L.cca_lca_cache_append(  # noqa: E731
        ctypes.byref(c), P(qs), P(q), P(FAKE + 8192), P(FAKE + 16384), d_rope, None)
    assert app(qs=0) == cca.CCA_ERR_INVALID_ARG
    assert app(qs=QS + 4) == cca.CCA_ERR_INVALID_ARG     # misaligned sums
    assert app(q=0) == cca.CCA_ERR_INVALID_ARG
    assert app(d_rope=12) == cca.CCA_ERR_INVALID_ARG
    assert c.len == 10
    c = _cache(core_cap=2, length=32)  # token 32 belongs to group 2: no slot
    assert app() == cca.CCA_ERR_CAPACITY
    assert c.len == 32
    c = _cache(core_cap=2)
    assert L.cca_lca_cache_prefill(ctypes.byref(c), P(QS), P(FAKE), P(FAKE), P(FAKE), 33, 0,
                                   None) == cca.CCA_ERR_CAPACITY
    assert L.cca_lca_cache_prefill(ctypes.byref(c), None, P(FAKE), P(FAKE), P(FAKE), 20, 0,
                                   None) == cca.CCA_ERR_INVALID_ARG
    assert L.cca_lca_cache_prefill(ctypes.byref(c), P(QS), P(FAKE), P(FAKE), P(FAKE), 20, 130,
                                   None) == cca.CCA_ERR_INVALID_ARG
    assert c.len == 0


def test_backward_argument_checks(L):
    """cca_attn_backward refuses bad shapes, outputs that are not 32-byte
    aligned, a short workspace and aliasing, all before any launch."""
    P = ctypes.c_void_p
    B, Hq, Hkv, T, d, g, w = 1, 2, 2, 256, 128, 16, 64
    nb = L.cca_attn_backward_workspace_bytes(B, Hq, Hkv, T, d, g)
    assert nb > 0
    base = FAKE
    step = 1 << 24  # every buffer 16 MiB apart: no overlaps unless asked
    names = ("Q", "K", "V", "Kc", "Vc", "O", "lse", "dO", "dQ", "dK", "dV", "ws")
    addr = {n: base + i * step for i, n in enumerate(names)}

    def call(**kw):
        a = dict(addr)
        a.update({k: v for k, v in kw.items() if k in addr})
        return L.cca_attn_backward(P(a["Q"]), P(a["K"]), P(a["V"]), P(a["Kc"]), P(a["Vc"]),
                                   P(a["O"]), 0, P(a["lse"]), P(a["dO"]), P(a["dQ"]), P(a["dK"]),
                                   P(a["dV"]), B, kw.get("Hq", Hq), Hkv, T, d, g, w,
                                   P(a["ws"]), kw.get("nb", nb), None)

    assert call(dK=addr["dK"] + 16) == cca.CCA_ERR_INVALID_ARG   # 16- but not 32-byte aligned
    assert call(dQ=addr["dQ"] + 16) == cca.CCA_ERR_INVALID_ARG
    assert call(ws=addr["ws"] + 128) == cca.CCA_ERR_INVALID_ARG  # workspace 256-byte aligned
    assert call(nb=nb - 1) == cca.CCA_ERR_INVALID_ARG
    assert call(dV=addr["Q"]) == cca.CCA_ERR_INVALID_ARG          # output aliases an input
    assert call(Hq=3) == cca.CCA_ERR_INVALID_ARG                  # Hq % Hkv != 0
    assert call(Hq=66) == cca.CCA_ERR_UNSUPPORTED                 # r = 33 > 32


class _FakeCuda:
    """A stand-in for a contiguous CUDA tensor: enough for the binding's
    argument checks, which run before any library call."""

    def __init__(self, shape, dtype):
        self.shape, self.dtype, self.is_cuda = shape, dtype, True

    def is_contiguous(self):
        return True

    def data_ptr(self):
        return FAKE


def test_core_rows_are_fp16():
    """Core keys/values (Kc, Vc and the cache's core slots) are fp16: the
    header names that layout and the binding refuses bf16 core rows before
    calling the library."""
    import torch
    with open(os.path.join(ROOT, "include", "cca.h")) as f:
        text = f.read()
    assert "Kc, Vc [B, Hkv, m, d], m = floor(T / g)  (fp16, written)" in text
    assert "(fp16, from cca_pool)" in text
    B, H, T, d, g = 1, 2, 64, 128, 16
    qkv = [_FakeCuda((B, H, T, d), torch.bfloat16) for _ in range(3)]
    bad = _FakeCuda((B, H, T // g, d), torch.bfloat16)
    with pytest.raises(ValueError, match="float16"):
        cca.cca_pool(*qkv, g, Kc=bad, Vc=bad)
    with pytest.raises(ValueError, match="float16"):
        cca.cca_attn_prefill(*qkv, bad, bad, g, 64, O=_FakeCuda((B, H, T, d), torch.bfloat16))

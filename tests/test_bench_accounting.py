"""The workload arithmetic bench.py reports against (algorithmic FLOPs and
bytes, KV-cache sizes), checked against direct counting and against the
numbers the method's definitions give for the benchmark shapes."""

import os
import sys

import numpy as np
import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402
from long_context_sparse_cca_b200 import synth  # noqa: E402


@pytest.mark.parametrize("T,g,w", [(300, 16, 64), (97, 4, 10), (50, 1, 0), (40, 8, 100)])
def test_keys_per_query_counts_the_attended_set(T, g, w):
    got = bench.keys_per_query(T, g, w)
    for t in range(T):
        ws = oracle.window_start(t, g, w)
        core = set(range(ws // g))          # pooled groups before the window
        raw = set(range(ws, t + 1))         # the window, the query included
        assert got[t] == len(core) + len(raw), t


def test_prefill_flops_of_the_benchmark_shapes():
    # 4 d per attended (query, key) pair; sums counted row by row
    for wl, expect in ((synth.PREFILL_32K, 1.061e12), (synth.PREFILL_128K, 1.087e13),
                       (synth.GQA_16K, 2.287e12)):
        n = sum(int(oracle.window_start(t, wl.g, wl.w)) // wl.g
                + t - int(oracle.window_start(t, wl.g, wl.w)) + 1 for t in range(wl.T))
        assert bench.prefill_flops(wl) == 4.0 * wl.d * n * wl.B * wl.Hq
        assert abs(bench.prefill_flops(wl) / expect - 1) < 1e-3


def test_pool_and_decode_bytes():
    assert abs(bench.pool_bytes(synth.PREFILL_128K) - 2.349e9) < 1e6
    assert abs(bench.pool_bytes(synth.PREFILL_32K) - 5.87e8) < 1e6
    dw = synth.DECODE_64K
    n = [int(bench.keys_per_query(t + 1, dw.g, dw.w, t)[0])
         for t in range(dw.T, dw.T + dw.steps)]
    assert min(n) == 5057 and max(n) == 5087
    mean = np.mean([bench.decode_bytes(dw, t) for t in range(dw.T, dw.T + dw.steps)])
    assert abs(mean / 664.9e6 - 1) < 1e-3


def test_kv_cache_reduction_at_128k():
    c = bench.cache_bytes(synth.PREFILL_128K, 131072)
    assert c["full_cache_bytes"] == 2 * 32 * 131072 * 128 * 2
    assert c["cca_cache_bytes"] == 2 * 32 * (8192 + 1040) * 128 * 2
    assert abs(c["reduction"] - 0.9296) < 1e-4


def test_backward_flops_and_lca_bytes():
    # backward: 10 d per attended pair (S, dP, dV, dK, dQ at 2 d each)
    wl = synth.PREFILL_32K
    assert bench.backward_flops(wl) == pytest.approx(10.0 / 4.0 * bench.prefill_flops(wl))
    assert bench.backward_flops(wl) == pytest.approx(2.653e12, rel=1e-3)
    # LCA condensation: every query row, K and V read; Kc, Vc written (2 bytes)
    w = synth.PREFILL_128K
    m = w.T // w.g
    expect = 2 * (w.B * w.Hq * w.T * w.d + 2 * w.B * w.Hkv * w.T * w.d + 2 * w.B * w.Hkv * m * w.d)
    assert bench.lca_pool_bytes(w) == expect
    assert bench.lca_pool_bytes(w) == pytest.approx(3.355e9, rel=1e-3)
    # it reads all queries where CCA's pooling reads one per group
    assert bench.lca_pool_bytes(w) - bench.pool_bytes(w) == 2 * w.B * w.Hq * (w.T - m) * w.d


def test_measured_traffic_is_tied_to_the_kernel_sources(tmp_path, monkeypatch):
    """A traffic line counts only while the prefill sources hash to the value
    recorded with it; another workload or a stale hash reads as unmeasured."""
    h = bench.prefill_source_hash()
    assert len(h) == 16
    assert "long_context_sparse_cca_b200/csrc/tma_map.h" in bench.PREFILL_SOURCES
    prof = tmp_path / "traffic.md"
    prof.write_text(f"# summary\n`traffic wlA 4.5e9 {h}`\n`traffic wlB 1.0e9 0123456789abcdef`\n")
    monkeypatch.setattr(bench, "TRAFFIC_PROFILE", str(prof))
    assert bench.measured_traffic("wlA") == 4.5e9
    assert bench.measured_traffic("wlB") is None   # recorded on other sources
    assert bench.measured_traffic("wlC") is None   # never captured
    monkeypatch.setattr(bench, "TRAFFIC_PROFILE", str(tmp_path / "missing.md"))
    assert bench.measured_traffic("wlA") is None


def test_committed_traffic_lines_match_the_current_sources():
    """The committed summary carries a line for each timed prefill workload,
    taken on the present kernel sources."""
    for name in (synth.PREFILL_128K.name,) + bench.EXTRA_PREFILL:
        t = bench.measured_traffic(name)
        assert t is not None, name
        assert t >= bench.prefill_bytes(synth.WORKLOADS[name]) * 0.9, name

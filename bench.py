"""Benchmark of the CCA-Attention hot path on B200.

One step is one pass of the whole hot path over synthetic inputs:
  prefill  cca_pool + cca_attn_prefill on a LLaMA2-7B-shaped layer at 128K
           context (B=1, H=32, d=128, T=131072, g=16, w=1024; bf16 N(0,1)
           inputs, 1% of key rows x4);
  decode   256 x cca_decode_step (append + attention, one launch) with B=8, H=32,
           d=128, g=16, w=1024 against a cache built from a 65536-token
           prefix (4096 core slots + a 1040-token raw ring).
value = prefill tokens/s (whole job, all ranks); decode latency per token
step is reported beside it.  Inputs (3 GB prefill, 0.67 GB cache) are larger
than L2, so no flush is needed between steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl cuda|reference]

Profiling runs use smaller pieces of the same harness: --parts prefill or
--parts decode runs one half, --prefill-workload picks the 32K or GQA
prefill workload, --no-e2e skips the host-buffer pass.

With --gpus N > 1 launch under torch.distributed.run: every rank runs the
same workload on its own GPU (independent sequences: weak scaling, no data
exchange); timing is the max over ranks.  --impl reference times the fp64
CPU oracle on a bounded sample of the same workload instead.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import shutil
import subprocess
import threading
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from long_context_sparse_cca_b200 import synth  # noqa: E402

METRIC = "CCA prefill tokens/s and decode µs/step at 128K on 1 B200; % of roofline"
UNIT = "tokens/s"
PREFILL = synth.PREFILL_128K
DECODE = synth.DECODE_64K
L2_BYTES = 126 * 2 ** 20
# the other prefill workloads of the method's evaluation shapes, timed beside
# the headline one
EXTRA_PREFILL = (synth.PREFILL_32K.name, synth.GQA_16K.name)
# LCA variant: positional entries per key row (the rotary part of a
# latent-attention key is 64 of its 192 entries in DeepSeek-V2; half of a
# 128-entry head here)
LCA_D_ROPE = 64
TRAFFIC_PROFILE = os.path.join(ROOT, "profiles", "prefill_kernel_dram_traffic.md")
# the sources of the prefill kernel: DRAM counters taken on another version
# of them do not describe this one
PREFILL_SOURCES = ("long_context_sparse_cca_b200/csrc/prefill.cu",
                   "long_context_sparse_cca_b200/csrc/sm100.cuh",
                   "long_context_sparse_cca_b200/csrc/common.cuh",
                   "long_context_sparse_cca_b200/csrc/tma_map.h")


# ----------------------------------------------------------------- workload arithmetic

def keys_per_query(T: int, g: int, w: int, t0: int = 0) -> np.ndarray:
    """Number of keys (core + raw) query t attends to, for t in [t0, T)."""
    t = np.arange(t0, T, dtype=np.int64)
    ws = (np.maximum(t - w, 0) // g) * g
    return ws // g + (t - ws + 1)


def prefill_flops(wl) -> float:
    """Algorithmic FLOPs of the fused attention: 4 d per (query, key) pair
    the method attends to (QK^T and PV), every batch row and query head."""
    n = keys_per_query(wl.T, wl.g, wl.w).sum()
    return 4.0 * wl.d * float(n) * wl.B * wl.Hq


def pool_bytes(wl) -> float:
    """Algorithmic bytes of pooling: read K, V and the scoring queries,
    write Kc, Vc (2-byte elements)."""
    m = wl.T // wl.g
    return 2.0 * (2 * wl.B * wl.Hkv * wl.T * wl.d + wl.B * wl.Hq * m * wl.d +
                  2 * wl.B * wl.Hkv * m * wl.d)


def lca_pool_bytes(wl) -> float:
    """Algorithmic bytes of the LCA condensation: read every query row (the
    group averages), K and V; write Kc, Vc (2-byte elements)."""
    m = wl.T // wl.g
    return 2.0 * (wl.B * wl.Hq * wl.T * wl.d + 2 * wl.B * wl.Hkv * wl.T * wl.d +
                  2 * wl.B * wl.Hkv * m * wl.d)


def lca_entry(wl, t: dict, pk: dict, world: int) -> dict:
    """The LCA variant on one workload: condensation against HBM, then the
    shared fused attention on the condensed rows."""
    gbs = lca_pool_bytes(wl) / (t["lca_pool_ms"] * 1e-3) / 1e9
    tf = prefill_flops(wl) / (t["prefill_ms"] * 1e-3) / 1e12
    return {"tokens_per_s": world * wl.B * wl.T / ((t["lca_pool_ms"] + t["prefill_ms"]) * 1e-3),
            "lca_pool_ms": t["lca_pool_ms"], "lca_pool_gbs": gbs,
            "lca_pool_frac": gbs / pk["hbm_gbs"], "lca_pool_bytes": lca_pool_bytes(wl),
            "prefill_ms": t["prefill_ms"], "prefill_tflops": tf,
            "prefill_frac_burst": tf / pk["bf16_tflops"], "d_rope": LCA_D_ROPE,
            "what": "cca_lca_pool (average-query weights, positional anchor) + "
                    "cca_attn_prefill on the condensed rows"}


def prefill_bytes(wl) -> float:
    """Algorithmic DRAM bytes of the fused attention: Q, K, V and the core
    keys/values read once, O written once (2-byte elements)."""
    m = wl.T // wl.g
    return 2.0 * (2 * wl.B * wl.Hq * wl.T * wl.d + 2 * wl.B * wl.Hkv * wl.T * wl.d +
                  2 * wl.B * wl.Hkv * m * wl.d)


def prefill_entry(wl, t: dict, pk: dict, world: int) -> dict:
    """Tokens/s and roofline fractions of one prefill workload from its
    pool and prefill times (ms)."""
    flops = prefill_flops(wl)
    tf = flops / (t["prefill_ms"] * 1e-3) / 1e12
    gbs = pool_bytes(wl) / (t["pool_ms"] * 1e-3) / 1e9
    out = {"tokens_per_s": world * wl.B * wl.T / ((t["pool_ms"] + t["prefill_ms"]) * 1e-3),
           "pool_ms": t["pool_ms"], "prefill_ms": t["prefill_ms"],
           "prefill_tflops": tf, "algorithmic_flops": flops,
           "prefill_frac_burst": tf / pk["bf16_tflops"],
           "prefill_frac_sustained": (tf / pk["bf16_tflops_sustained"]
                                      if pk["bf16_tflops_sustained"] else None),
           "pool_gbs": gbs, "pool_frac": gbs / pk["hbm_gbs"],
           "traffic": measured_traffic(wl.name),
           "algorithmic_bytes": prefill_bytes(wl)}
    return out


def backward_flops(wl) -> float:
    """Algorithmic FLOPs of the attention backward: 10 d per attended
    (query, key) pair (S recomputed, dP, dV, dK, dQ), every batch row and
    query head; the pooling's chain rule is not counted."""
    return 2.5 * prefill_flops(wl)


def backward_entry(wl, t: dict, pk: dict, world: int) -> dict:
    """Time and tensor-core fraction of the backward pass on one workload."""
    flops = backward_flops(wl)
    tf = flops / (t["backward_ms"] * 1e-3) / 1e12
    return {"backward_ms": t["backward_ms"], "forward_lse_ms": t["forward_ms"],
            "tflops": tf, "algorithmic_flops": flops,
            "frac_burst": tf / pk["bf16_tflops"],
            "frac_sustained": (tf / pk["bf16_tflops_sustained"]
                               if pk["bf16_tflops_sustained"] else None),
            "what": "cca_attn_backward: row sums + tcgen05 dQ + tcgen05 dK/dV + pooling "
                    "chain rule; FLOPs 10 d per attended (query, key) pair"}


def decode_bytes(wl, t: int) -> float:
    """Algorithmic bytes of one decode step at token t: every key and value
    row the token attends to, plus its query and output rows."""
    n = int(keys_per_query(t + 1, wl.g, wl.w, t)[0])
    return float(wl.B * wl.Hkv * n * 2 * wl.d * 2 + wl.B * wl.Hq * 2 * wl.d * 2)


def append_bytes(wl, t: int) -> float:
    """Algorithmic bytes of one append: the new k, v rows (and on a group's
    last token the group's g keys/values read back and one core row pair
    written)."""
    b = wl.B * wl.Hkv * 2 * wl.d * 2 * 2  # read + write of k_t, v_t
    if (t + 1) % wl.g == 0:
        b += wl.B * wl.Hkv * (2 * wl.g * wl.d * 2 + 2 * wl.d * 2) + wl.B * wl.Hq * wl.d * 2
    return float(b)


def cache_bytes(wl, T: int) -> dict:
    core = 2 * wl.B * wl.Hkv * (T // wl.g) * wl.d * 2
    tail = 2 * wl.B * wl.Hkv * (wl.w + wl.g) * wl.d * 2
    full = 2 * wl.B * wl.Hkv * T * wl.d * 2
    return {"full_cache_bytes": full, "cca_cache_bytes": core + tail,
            "reduction": 1.0 - (core + tail) / full}


def peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0,
            "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def prefill_source_hash() -> str:
    import hashlib
    h = hashlib.sha256()
    for rel in PREFILL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def measured_traffic(workload: str):
    """DRAM bytes (read + write) of one prefill-kernel launch on `workload`,
    from the committed ncu summary, or None when that summary is missing,
    names another workload, or was taken on other kernel sources.  The
    summary holds machine-readable lines `traffic <workload> <bytes>
    <source hash>`."""
    if not os.path.exists(TRAFFIC_PROFILE):
        return None
    want = prefill_source_hash()
    with open(TRAFFIC_PROFILE) as f:
        for line in f:
            parts = line.strip().strip("`").split()
            if len(parts) == 4 and parts[0] == "traffic" and parts[1] == workload:
                return float(parts[2]) if parts[3] == want else None
    return None


# ----------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu_index = gpu_index
        self.proc = None

    def __enter__(self):
        self.lines = []
        self.proc = None
        self.reader = None
        cmd = ["nvidia-smi", "-i", str(self.gpu_index), f"--query-gpu={self.FIELDS}",
               "--format=csv,noheader,nounits", "-lms", "100"]
        # nvidia-smi block-buffers a pipe: line-buffer it so that samples
        # arrive while the timed region runs, and read them on a thread
        if shutil.which("stdbuf"):
            cmd = ["stdbuf", "-oL"] + cmd
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
            # start timing only once the sampler is producing samples
            first = self.proc.stdout.readline()
            if first:
                self.lines.append(first)
            self.reader = threading.Thread(target=self._read, daemon=True)
            self.reader.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line)

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.15)  # one more sample of the end of the timed region
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.proc.wait()
            if self.reader is not None:
                self.reader.join(timeout=5)
        self.out = "".join(self.lines)
        return False

    def summary(self) -> dict:
        rows = [r.split(",") for r in getattr(self, "out", "").strip().splitlines() if r.strip()]
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            if len(r) < 9:
                continue
            try:
                sm.append(float(r[1]))
                mx = float(r[2])
            except ValueError:
                continue
            for name, val in zip(names, r[5:9]):
                if val.strip().lower() == "active":
                    reasons.add(name)
        loaded = [s for s in sm if mx and s > 0.3 * mx] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


def max_over_ranks(values, world: int, device) -> list:
    """Element-wise maximum of each rank's timings, by one all-reduce over
    the process group (the identity for a single rank).  Every rank must
    call it with the same number of values."""
    if world == 1:
        return [float(v) for v in values]
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


# ----------------------------------------------------------------- CUDA arm

def _dev(bits, torch):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(
        torch.bfloat16)


def run_cuda(args, rank: int, world: int, local_rank: int) -> dict:
    import torch
    import torch.distributed as dist
    import long_context_sparse_cca_b200 as cca
    from long_context_sparse_cca_b200 import build as cca_build

    if rank == 0 or world == 1:
        cca_build.build()
    if world > 1:
        dist.barrier()
    torch.cuda.set_device(local_rank)
    cca.lib()
    stream = torch.cuda.current_stream()

    do_prefill = "prefill" in args.parts
    do_decode = "decode" in args.parts
    pw = args.prefill_wl
    dw = DECODE
    if do_prefill:
        # prefill inputs resident in HBM, pinned host copies for the e2e pass
        x = synth.generate(pw)
        Q, K, V = _dev(x.q, torch), _dev(x.k, torch), _dev(x.v, torch)
        if not args.no_e2e:
            hQ, hK, hV = (torch.from_numpy(a.view(np.int16)).view(torch.bfloat16)
                          .pin_memory() for a in (x.q, x.k, x.v))
        del x
        m = pw.T // pw.g
        Kc = torch.empty((pw.B, pw.Hkv, m, pw.d), dtype=torch.float16, device="cuda")
        Vc = torch.empty_like(Kc)
        O = torch.empty((pw.B, pw.Hq, pw.T, pw.d), dtype=torch.bfloat16, device="cuda")
        if not args.no_e2e:
            hO = torch.empty(O.shape, dtype=torch.bfloat16).pin_memory()
    if do_decode:
        # decode cache from a 65536-token prefix, then 256 new tokens
        y = synth.generate(dw)
        cache = cca.Cache(dw.B, dw.Hq, dw.Hkv, dw.d, dw.g, dw.w,
                          core_cap=(dw.T + dw.steps) // dw.g)
        pre = [_dev(np.ascontiguousarray(a[:, :, :dw.T]), torch) for a in (y.q, y.k, y.v)]
        cca.cca_cache_prefill(cache, *pre)
        torch.cuda.synchronize()
        del pre
        torch.cuda.empty_cache()  # the prefix is not part of the workload
        new_q = _dev(np.ascontiguousarray(y.q[:, :, dw.T:].transpose(2, 0, 1, 3)), torch)
        new_k = _dev(np.ascontiguousarray(y.k[:, :, dw.T:].transpose(2, 0, 1, 3)), torch)
        new_v = _dev(np.ascontiguousarray(y.v[:, :, dw.T:].transpose(2, 0, 1, 3)), torch)
        del y
        o_t = torch.empty((dw.B, dw.Hq, dw.d), dtype=torch.bfloat16, device="cuda")
        ws_bytes = cca.cca_decode_workspace_bytes(cache)
        # zero-filled once, as cca_decode_step requires of a new workspace
        workspace = torch.zeros(ws_bytes, dtype=torch.uint8, device="cuda")
    st = cca.cca_device_status()
    assert st == cca.CCA_OK, cca.status_string(st)

    def prefill_part(evs):
        if not do_prefill:
            return
        evs[0].record(stream)
        cca.cca_pool(Q, K, V, pw.g, Kc, Vc)
        evs[1].record(stream)
        cca.cca_attn_prefill(Q, K, V, Kc, Vc, pw.g, pw.w, O=O)
        evs[2].record(stream)

    def decode_part(evs):
        if not do_decode:
            return
        cache.len = dw.T  # same 256 steps every time (slots rewritten identically)
        evs[0].record(stream)
        for s in range(dw.steps):
            # append + decode attention of the token, one launch
            cca.cca_decode_step(cache, new_q[s], new_k[s], new_v[s], o_t, workspace=workspace)
        evs[1].record(stream)

    def step(ev_p, ev_d):
        prefill_part(ev_p)
        decode_part(ev_d)

    mk = lambda n: [torch.cuda.Event(enable_timing=True) for _ in range(n)]  # noqa: E731
    for _ in range(args.warmup):
        step(mk(3), mk(2))
    torch.cuda.synchronize()
    st = cca.cca_device_status()
    assert st == cca.CCA_OK, cca.status_string(st)

    # --- timed region
    evp = [mk(3) for _ in range(args.steps)]
    evd = [mk(2) for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        t_start.record(stream)
        for i in range(args.steps):
            step(evp[i], evd[i])
        t_end.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    total_ms = t_start.elapsed_time(t_end)
    pool_ms = [e[0].elapsed_time(e[1]) for e in evp] if do_prefill else [0.0]
    prefill_ms = [e[1].elapsed_time(e[2]) for e in evp] if do_prefill else [0.0]
    decode_ms = [e[0].elapsed_time(e[1]) for e in evd] if do_decode else [0.0]
    st = cca.cca_device_status()
    assert st == cca.CCA_OK, cca.status_string(st)

    # --- end to end through host buffers (prefill; H2D of Q, K, V and D2H of O)
    e2e_ms = []
    n_e2e = 0 if (args.no_e2e or not do_prefill) else max(2, min(args.steps, 3)) + 1
    if n_e2e:
        O_resident = O.clone()  # the timed steps' output: the e2e pass must match it
    for i in range(n_e2e):
        ms = e2e_pass(cca, Q, K, V, Kc, Vc, O, hQ, hK, hV, hO, pw, stream, torch)
        if i > 0:  # first one warms the pinned paths
            e2e_ms.append(ms)
    if n_e2e:
        assert torch.equal(O, O_resident), "e2e output differs from the resident run"
        del O_resident

    # --- the other prefill workloads, each timed on its own after the
    # headline step (kernels entries, not the bench value)
    extra = {}
    for name in ([] if args.no_extra else EXTRA_PREFILL):
        if not do_prefill:
            break
        extra[name] = time_prefill(cca, synth.WORKLOADS[name], args.steps, args.warmup,
                                   stream, torch)

    # --- the backward pass (training) on the 32K workload: the forward with
    # log-sum-exp, then cca_attn_backward (four launches)
    if do_prefill and not args.no_backward:
        extra["backward"] = time_backward(cca, synth.PREFILL_32K, args.steps, args.warmup,
                                          stream, torch)

    # --- the LCA variant on the headline inputs: condensation, then the
    # shared fused attention (overwrites Kc, Vc, O after the timed region)
    if do_prefill and not args.no_extra:
        extra["lca"] = time_lca(cca, Q, K, V, Kc, Vc, O, pw, args.steps, args.warmup, stream,
                                torch)

    # one all-reduce of every timing, the same on all ranks (no e2e: -1)
    total_ms, mean_pool, mean_prefill, mean_decode, mean_e2e = max_over_ranks(
        [total_ms, float(np.mean(pool_ms)), float(np.mean(prefill_ms)),
         float(np.mean(decode_ms)), float(np.mean(e2e_ms)) if e2e_ms else -1.0],
        world, "cuda")
    mean_e2e = mean_e2e if mean_e2e >= 0 else None
    for name in list(extra):
        keys = sorted(extra[name])
        extra[name] = dict(zip(keys, max_over_ranks([extra[name][k] for k in keys], world,
                                                    "cuda")))
    h2d = 3 * Q.numel() * 2 if do_prefill else 0
    d2h = O.numel() * 2 if do_prefill else 0
    return dict(total_ms=total_ms, pool_ms=mean_pool, prefill_ms=mean_prefill,
                decode_ms=mean_decode, e2e_ms=mean_e2e, clocks=clk.summary(),
                h2d=h2d, d2h=d2h, extra=extra)


E2E_CHUNKS = 4  # head chunks of the pipelined host-buffer pass


def e2e_pass(cca, Q, K, V, Kc, Vc, O, hQ, hK, hV, hO, wl, stream, torch) -> float:
    """One prefill through the public API from pinned host Q, K, V to host O,
    device-timed on `stream`.  With B = 1 and the heads divisible into
    E2E_CHUNKS chunks (every chunk's rows are contiguous), it pipelines: the
    copy in of a chunk of heads (one stream), its pooling and prefill
    (another) and the copy out of its output (a third) overlap those of the
    neighbouring chunks.  Otherwise: copy in, compute, copy out."""
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n = E2E_CHUNKS
    chunked = wl.B == 1 and wl.Hkv % n == 0 and wl.Hq % n == 0
    torch.cuda.synchronize()
    a.record(stream)
    if not chunked:
        Q.copy_(hQ, non_blocking=True)
        K.copy_(hK, non_blocking=True)
        V.copy_(hV, non_blocking=True)
        cca.cca_pool(Q, K, V, wl.g, Kc, Vc)
        cca.cca_attn_prefill(Q, K, V, Kc, Vc, wl.g, wl.w, O=O)
        hO.copy_(O, non_blocking=True)
    else:
        s_in, s_cmp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
        for s_ in (s_in, s_cmp, s_out):
            s_.wait_event(a)
        hq, hk = wl.Hq // n, wl.Hkv // n
        for c in range(n):
            qs, ks = slice(c * hq, (c + 1) * hq), slice(c * hk, (c + 1) * hk)
            with torch.cuda.stream(s_in):
                Q[:, qs].copy_(hQ[:, qs], non_blocking=True)
                K[:, ks].copy_(hK[:, ks], non_blocking=True)
                V[:, ks].copy_(hV[:, ks], non_blocking=True)
            ev_in = torch.cuda.Event()
            ev_in.record(s_in)
            s_cmp.wait_event(ev_in)
            cca.cca_pool(Q[:, qs], K[:, ks], V[:, ks], wl.g, Kc[:, ks], Vc[:, ks], stream=s_cmp)
            cca.cca_attn_prefill(Q[:, qs], K[:, ks], V[:, ks], Kc[:, ks], Vc[:, ks], wl.g,
                                 wl.w, O=O[:, qs], stream=s_cmp)
            ev_cmp = torch.cuda.Event()
            ev_cmp.record(s_cmp)
            s_out.wait_event(ev_cmp)
            with torch.cuda.stream(s_out):
                hO[:, qs].copy_(O[:, qs], non_blocking=True)
        ev_out = torch.cuda.Event()
        ev_out.record(s_out)
        stream.wait_event(ev_out)
    b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b)


def time_backward(cca, wl, steps: int, warmup: int, stream, torch) -> dict:
    """Mean CUDA-event times (ms) of cca_attn_prefill_lse and of
    cca_attn_backward on one workload (synthetic upstream gradient dO,
    N(0,1) bf16), inputs resident in HBM."""
    x = synth.generate(wl)
    Q, K, V = _dev(x.q, torch), _dev(x.k, torch), _dev(x.v, torch)
    dO = _dev(synth.random_bf16(x.q.shape, wl.seed + 100), torch)
    del x
    Kc, Vc = cca.cca_pool(Q, K, V, wl.g)
    O = torch.empty((wl.B, wl.Hq, wl.T, wl.d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((wl.B, wl.Hq, wl.T), dtype=torch.float32, device="cuda")
    dQ = torch.empty((wl.B, wl.Hq, wl.T, wl.d), dtype=torch.float32, device="cuda")
    dK = torch.empty((wl.B, wl.Hkv, wl.T, wl.d), dtype=torch.float32, device="cuda")
    dV = torch.empty_like(dK)
    ws = torch.empty(cca.cca_attn_backward_workspace_bytes(wl.B, wl.Hq, wl.Hkv, wl.T, wl.d,
                                                           wl.g), dtype=torch.uint8,
                     device="cuda")
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)]
           for _ in range(warmup + steps)]
    for e in evs:
        e[0].record(stream)
        cca.cca_attn_prefill_lse(Q, K, V, Kc, Vc, wl.g, wl.w, O=O, lse=lse)
        e[1].record(stream)
        cca.cca_attn_backward(Q, K, V, Kc, Vc, O, lse, dO, wl.g, wl.w, dQ, dK, dV, workspace=ws)
        e[2].record(stream)
    torch.cuda.synchronize()
    st = cca.cca_device_status()
    assert st == cca.CCA_OK, cca.status_string(st)
    timed = evs[warmup:]
    out = {"forward_ms": float(np.mean([e[0].elapsed_time(e[1]) for e in timed])),
           "backward_ms": float(np.mean([e[1].elapsed_time(e[2]) for e in timed]))}
    del Q, K, V, dO, Kc, Vc, O, lse, dQ, dK, dV, ws
    torch.cuda.empty_cache()
    return out


def time_lca(cca, Q, K, V, Kc, Vc, O, wl, steps: int, warmup: int, stream, torch) -> dict:
    """Mean CUDA-event times (ms) of cca_lca_pool and of cca_attn_prefill on
    its rows, on resident inputs of workload wl."""
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)]
           for _ in range(warmup + steps)]
    for e in evs:
        e[0].record(stream)
        cca.cca_lca_pool(Q, K, V, wl.g, LCA_D_ROPE, Kc, Vc)
        e[1].record(stream)
        cca.cca_attn_prefill(Q, K, V, Kc, Vc, wl.g, wl.w, O=O)
        e[2].record(stream)
    torch.cuda.synchronize()
    st = cca.cca_device_status()
    assert st == cca.CCA_OK, cca.status_string(st)
    timed = evs[warmup:]
    return {"lca_pool_ms": float(np.mean([e[0].elapsed_time(e[1]) for e in timed])),
            "prefill_ms": float(np.mean([e[1].elapsed_time(e[2]) for e in timed]))}


def time_prefill(cca, wl, steps: int, warmup: int, stream, torch) -> dict:
    """Mean CUDA-event times (ms) of cca_pool and cca_attn_prefill on one
    prefill workload, inputs resident in HBM, after `warmup` untimed
    passes; the buffers are freed afterwards."""
    x = synth.generate(wl)
    Q, K, V = _dev(x.q, torch), _dev(x.k, torch), _dev(x.v, torch)
    del x
    m = wl.T // wl.g
    Kc = torch.empty((wl.B, wl.Hkv, m, wl.d), dtype=torch.float16, device="cuda")
    Vc = torch.empty_like(Kc)
    O = torch.empty((wl.B, wl.Hq, wl.T, wl.d), dtype=torch.bfloat16, device="cuda")
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)]
           for _ in range(warmup + steps)]
    for e in evs:
        e[0].record(stream)
        cca.cca_pool(Q, K, V, wl.g, Kc, Vc)
        e[1].record(stream)
        cca.cca_attn_prefill(Q, K, V, Kc, Vc, wl.g, wl.w, O=O)
        e[2].record(stream)
    torch.cuda.synchronize()
    st = cca.cca_device_status()
    assert st == cca.CCA_OK, cca.status_string(st)
    timed = evs[warmup:]
    out = {"pool_ms": float(np.mean([e[0].elapsed_time(e[1]) for e in timed])),
           "prefill_ms": float(np.mean([e[1].elapsed_time(e[2]) for e in timed]))}
    del Q, K, V, Kc, Vc, O
    torch.cuda.empty_cache()
    return out


# ----------------------------------------------------------------- oracle (CPU) arm

_SAMPLE = None


def oracle_sample(budget_s: float = 20.0) -> dict:
    """Time the fp64 oracle on a bounded sample of the prefill workload:
    pooling of one head's whole sequence plus the fused attention of seeded
    random rows of that head, scaled to tokens/s of the full workload (all
    heads, all rows)."""
    import oracle

    wl = PREFILL
    global _SAMPLE
    if _SAMPLE is None:
        x = synth.generate(wl, B=1)
        h = 0
        _SAMPLE = tuple(synth.bf16_bits_to_f64(a[:, h:h + 1]) for a in (x.q, x.k, x.v))
        del x
    q, k, v = _SAMPLE
    t0 = time.perf_counter()
    Kc, Vc = oracle.pool(q, k, v, wl.g)
    pool_s = time.perf_counter() - t0
    rng = np.random.default_rng(99)
    rows_done, attend_s, n_keys = 0, 0.0, 0
    while attend_s < budget_s and rows_done < wl.T:
        rows = np.sort(rng.integers(0, wl.T, size=64))
        t0 = time.perf_counter()
        oracle.attend_rows(q, k, v, Kc, Vc, wl.g, wl.w, rows)
        attend_s += time.perf_counter() - t0
        rows_done += rows.size
        n_keys += int(keys_per_query(wl.T, wl.g, wl.w)[rows].sum())
    # cost per token of the full workload: pooling per token plus the mean
    # attention cost per row (sampled rows are uniform in t), all heads
    per_token = (pool_s / wl.T + attend_s / rows_done) * wl.Hq * wl.B
    return {"value": 1.0 / per_token, "unit": UNIT, "cores": oracle.threads(),
            "kind": "oracle",
            "sample": (f"prefill 128K workload, head 0 of {wl.Hq}: full pooling "
                       f"({pool_s:.2f} s) + fused attention of {rows_done} seeded random "
                       f"rows ({attend_s:.2f} s); scaled to all rows and heads"),
            "seconds": pool_s + attend_s}


def oracle_decode_sample(budget_s: float = 4.0) -> dict:
    """Time the fp64 oracle's decode step (append + decode) on head 0 of
    batch row 0 of the decode workload: the cache is built from the
    65536-token prefix (pooled core slots and the ring), then steps run
    until the budget or the 256 steps are spent.  Scaled to all rows and
    heads of the workload."""
    import dataclasses

    import oracle

    dw = DECODE
    one = dataclasses.replace(dw, B=1, Hq=1, Hkv=1)  # the same values as head 0 of row 0
    y = synth.generate(one)
    q, k, v = (synth.bf16_bits_to_f64(a) for a in (y.q, y.k, y.v))
    T = dw.T
    c = oracle.new_cache(1, 1, 1, dw.d, dw.g, dw.w, core_cap=(T + dw.steps) // dw.g)
    Kc, Vc = oracle.pool(q[:, :, :T], k[:, :, :T], v[:, :, :T], dw.g)
    m = Kc.shape[2]
    c.k_core[:, :, :m] = Kc
    c.v_core[:, :, :m] = Vc
    cap = c.tail_cap
    for p in range(T - cap, T):
        c.k_tail[:, :, p % cap] = k[:, :, p]
        c.v_tail[:, :, p % cap] = v[:, :, p]
    c.len = T
    n = 0
    t0 = time.perf_counter()
    while n < dw.steps and (n == 0 or time.perf_counter() - t0 < budget_s):
        t = T + n
        c.append(q[:, :, t], k[:, :, t], v[:, :, t])
        c.decode(q[:, :, t])
        n += 1
    sec = time.perf_counter() - t0
    return {"us_per_step": sec / n * 1e6 * dw.B * dw.Hq, "unit": "us/step",
            "cores": oracle.threads(), "kind": "oracle",
            "sample": (f"decode workload, row 0 head 0 of {dw.B} x {dw.Hq}: {n} steps of "
                       f"append + decode after the 65536-token prefix ({sec:.2f} s); "
                       "scaled to all rows and heads")}


def oracle_single_thread_value(budget_s: float = 3.0) -> float:
    """The prefill oracle sample on one thread (tokens/s of the full
    workload), the thread count restored afterwards."""
    import oracle

    n = oracle.threads()
    oracle.set_threads(1)
    try:
        return oracle_sample(budget_s=budget_s)["value"]
    finally:
        oracle.set_threads(n)


# ----------------------------------------------------------------- main

def config_dict(args, world: int) -> dict:
    """The workload description both arms print (the same keys and values,
    so the two lines describe one configuration)."""
    pw = args.prefill_wl
    return {"workload": pw.name, "decode_workload": DECODE.name,
            "parts": args.parts,
            "global_batch": pw.B * world, "seq_len": pw.T,
            "parallelism": f"replicas{world}", "core_dtype": "f16",
            "o_dtype": "bf16",
            "l2": "inputs larger than L2 (no flush)"}


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__,
                                 formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("cuda", "reference"), default="cuda")
    ap.add_argument("--no-cpu-baseline", action="store_true",
                    help="skip timing the CPU oracle (rank 0, N=1)")
    ap.add_argument("--parts", default="prefill,decode",
                    help="comma list of prefill, decode (profiling runs)")
    ap.add_argument("--prefill-workload", default=PREFILL.name,
                    choices=[w.name for w in synth.WORKLOADS.values() if w.steps == 0],
                    help="prefill workload (profiling runs; the default is the headline)")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer pass")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip timing the 32K and GQA prefill workloads")
    ap.add_argument("--no-backward", action="store_true",
                    help="skip timing the backward pass on the 32K workload")
    args = ap.parse_args(argv)
    args.prefill_wl = synth.WORKLOADS[args.prefill_workload]
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.gpus != world and world > 1:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE {world}", file=sys.stderr)

    if args.impl == "reference":
        if rank != 0:
            return 0
        res = []
        for _ in range(args.warmup + args.steps):
            res.append(oracle_sample(budget_s=max(2.0, 60.0 / (args.warmup + args.steps))))
        timed = res[args.warmup:]
        val = float(np.mean([r["value"] for r in timed]))
        sec = float(np.mean([r["seconds"] for r in timed]))
        cb = dict(timed[-1])
        cb["value"] = val
        cb.pop("seconds", None)
        line = {"metric": METRIC, "value": val, "unit": UNIT, "n_gpus": 0,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec * 1e3,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "f64", "data": "synthetic", "impl": "reference",
                "config": config_dict(args, world),
                "cpu_baseline": cb,
                "e2e": {"value": val, "unit": UNIT, "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        return 0

    if world > 1:
        import torch
        import torch.distributed as dist
        from datetime import timedelta
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=timedelta(seconds=600))

    r = run_cuda(args, rank, world, local_rank)

    pk = peaks()
    pw = args.prefill_wl
    do_prefill = "prefill" in args.parts
    do_decode = "decode" in args.parts
    nz = lambda v: v if v else float("nan")  # noqa: E731
    tokens = pw.B * pw.T
    prefill_s = nz((r["pool_ms"] + r["prefill_ms"]) * 1e-3)
    value = world * tokens / prefill_s if do_prefill else None
    dec_us = r["decode_ms"] * 1e3 / DECODE.steps if do_decode else None
    flops = prefill_flops(pw)
    achieved_tf = flops / (nz(r["prefill_ms"]) * 1e-3) / 1e12
    pbytes = pool_bytes(pw)
    dbytes = float(np.mean([decode_bytes(DECODE, t) + append_bytes(DECODE, t)
                            for t in range(DECODE.T, DECODE.T + DECODE.steps)]))
    dec_gbs = dbytes / (nz(dec_us) * 1e-6) / 1e9
    pool_gbs = pbytes / (nz(r["pool_ms"]) * 1e-3) / 1e9
    launches = args.steps * ((2 if do_prefill else 0) + (DECODE.steps if do_decode else 0))
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": r["total_ms"] / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": config_dict(args, world),
        "decode_us_per_step": dec_us,
        "roofline": {"bound": "tensor", "kernel": "cca_attn_prefill",
                     "achieved": achieved_tf, "peak": pk["bf16_tflops"],
                     "unit": "TFLOP/s", "frac": achieved_tf / pk["bf16_tflops"],
                     "traffic": measured_traffic(pw.name),
                     "peak_source": pk["source"] + " (burst)",
                     "algorithmic_flops": flops,
                     "algorithmic_bytes": prefill_bytes(pw)},
        "kernels": {
            "cca_attn_prefill": {"ms": r["prefill_ms"], "tflops": achieved_tf,
                                 "frac_burst": achieved_tf / pk["bf16_tflops"],
                                 "frac_sustained": (achieved_tf / pk["bf16_tflops_sustained"]
                                                    if pk["bf16_tflops_sustained"] else None)},
            "cca_pool": {"ms": r["pool_ms"], "gbs": pool_gbs,
                         "frac": pool_gbs / pk["hbm_gbs"], "bytes": pbytes},
            "decode_step": {"us": dec_us, "gbs": dec_gbs, "frac": dec_gbs / pk["hbm_gbs"],
                            "bytes": dbytes,
                            "launches": "cca_decode_step: one kernel per token (append, split-K attention, merge)"},
            **{f"prefill[{name}]": prefill_entry(synth.WORKLOADS[name], t, pk, world)
               for name, t in r["extra"].items() if name not in ("backward", "lca")},
            **({"lca[" + args.prefill_wl.name + "]": lca_entry(args.prefill_wl, r["extra"]["lca"],
                                                              pk, world)}
               if "lca" in r["extra"] else {}),
            **({"backward[" + synth.PREFILL_32K.name + "]": backward_entry(
                synth.PREFILL_32K, r["extra"]["backward"], pk, world)}
               if "backward" in r["extra"] else {}),
        },
        "kv_cache": cache_bytes(pw, pw.T),
        "clocks": r["clocks"],
        "e2e": {"value": world * tokens / (r["e2e_ms"] * 1e-3) if r["e2e_ms"] else None,
                "unit": UNIT,
                "h2d_bytes_per_step": r["h2d"], "d2h_bytes_per_step": r["d2h"],
                "what": "prefill through cca_pool + cca_attn_prefill from pinned host Q/K/V "
                        "to host O, in head chunks whose copy in, compute and copy out "
                        "overlap on three streams"},
        "gpu_launches": launches,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cb = oracle_sample()
        cb.pop("seconds", None)
        cb["single_thread_value"] = oracle_single_thread_value()
        cb["decode"] = oracle_decode_sample()
        line["cpu_baseline"] = cb
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())

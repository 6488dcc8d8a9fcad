"""CPU models of the mbarrier protocols of the three warp-specialised
tcgen05 kernels (prefill_kernel, bw_dq_kernel, bw_dkv_kernel).

Each model restates, role by role, the order in which a kernel's warps wait
on and arrive at its barriers: TMA producer, MMA issuer(s) (whose
tcgen05.commit arrivals are modelled as arrivals at issue time) and the
element-wise warp groups.  A barrier counts completed phases.  The kernels
wait with parity tests, which only tell the phase in progress from the one
before it, so a wait on phase k is sound only while exactly k or k + 1
phases have completed.  The checker runs seeded random interleavings of the
roles and reports:

  * a wait begun when phase k - 1 has not completed (the parity test would
    return at once: the wait "runs ahead");
  * a wait begun when phase k + 1 has already completed (parity aliasing);
  * deadlock (no role can move).

The tile geometry of each work item mirrors the kernel's; work items are
dealt to a CTA as the kernel deals them.  Models are host logic only: they
run no GPU code.
"""

from __future__ import annotations

import random


class ProtocolError(AssertionError):
    pass


class Barrier:
    def __init__(self, count: int):
        self.count, self.arrived, self.done = count, 0, 0

    def arrive(self):
        self.arrived += 1
        if self.arrived == self.count:
            self.arrived = 0
            self.done += 1


class Sim:
    def __init__(self):
        self.bars = {}

    def bar(self, name: str, count: int = 1) -> Barrier:
        self.bars[name] = Barrier(count)
        return self.bars[name]

    def arrive(self, name: str):
        self.bars[name].arrive()

    def ready(self, name: str, phase: int) -> bool:
        """True once phase `phase` (0-based) of barrier `name` completed."""
        b = self.bars[name]
        if b.done >= phase + 2:
            raise ProtocolError(f"parity aliasing on {name}: waiting for phase {phase}, "
                                f"{b.done} completed")
        if b.done < phase:
            raise ProtocolError(f"parity wait runs ahead on {name}: waiting for phase {phase}, "
                                f"only {b.done} completed")
        return b.done > phase

    def wait(self, name: str, phase: int):
        """Generator: yields until the phase completed (checked at the first
        poll, as the kernel's parity test would see it)."""
        while not self.ready(name, phase):
            yield

    def run(self, roles, seed: int, limit: int = 200000):
        rng = random.Random(seed)
        live = list(range(len(roles)))
        idle = 0
        state = lambda: tuple((b.done, b.arrived) for b in self.bars.values())  # noqa: E731
        while live:
            i = rng.choice(live)
            before = state()
            try:
                next(roles[i])
            except StopIteration:
                live.remove(i)
                idle = 0
                continue
            idle = 0 if state() != before else idle + 1
            if idle > limit:
                raise ProtocolError(f"deadlock: roles {live} cannot move")


def ws_of(t: int, g: int, w: int) -> int:
    return (max(t - w, 0) // g) * g


# ---------------------------------------------------------------- prefill

def prefill_items(T, g, w, B, Hq, cta, grid):
    """(n_local, n_core) of the 256-row blocks dealt to CTA `cta`, in the
    kernel's order (latest block first; round-robin over the CTAs)."""
    nb = (T + 255) // 256
    n_items = nb * B * Hq
    out = []
    for item in range(cta, n_items, grid):
        blk = nb - 1 - item // (B * Hq)
        t0 = blk * 256
        tlast = min(t0 + 255, T - 1)
        n_core = (ws_of(tlast, g, w) // g + 127) // 128
        n_local = (tlast - ws_of(t0, g, w) + 1 + 127) // 128
        out.append((n_local, n_core))
    return out


def prefill_roles(sim: Sim, items, KST=3, VST=2):
    for n in ("q_full", "q_empty"):
        sim.bar(n)
    for s in range(KST):
        sim.bar(f"k_full{s}")
        sim.bar(f"k_empty{s}")
    for s in range(VST):
        sim.bar(f"v_full{s}")
        sim.bar(f"v_empty{s}")
    for h in range(2):
        for n in ("s_full", "s_free", "p_full", "o_bar", "o_empty", "qh_full"):
            sim.bar(f"{n}{h}")

    def producer():
        qc = kc = vc = 0
        for nl, nc in items:
            if qc > 0:
                yield from sim.wait("q_empty", qc - 1)
            sim.arrive("q_full")
            qc += 1
            for _ in range(nl + nc):
                if kc >= KST:
                    yield from sim.wait(f"k_empty{kc % KST}", kc // KST - 1)
                sim.arrive(f"k_full{kc % KST}")
                kc += 1
                if vc >= VST:
                    yield from sim.wait(f"v_empty{vc % VST}", vc // VST - 1)
                sim.arrive(f"v_full{vc % VST}")
                vc += 1

    def qk_issuer():
        kc = cq = it = 0
        for k, (nl, nc) in enumerate(items):
            yield from sim.wait("q_full", k)
            for j in range(nl + nc):
                core = j >= nl
                yield from sim.wait(f"k_full{kc % KST}", kc // KST)
                for h in range(2):
                    if h == 1 or it > 0:
                        yield from sim.wait(f"s_free{h ^ 1}", it - 1 if h == 0 else it)
                    if core and j == nl:
                        yield from sim.wait(f"qh_full{h}", cq)
                    sim.arrive(f"s_full{h}")
                sim.arrive(f"k_empty{kc % KST}")
                kc += 1
                if j == nl + nc - 1:
                    sim.arrive("q_empty")
                it += 1
            if nc > 0:
                cq += 1

    def pv_issuer():
        vc = it = 0
        for k, (nl, nc) in enumerate(items):
            for j in range(nl + nc):
                for h in range(2):
                    yield from sim.wait(f"p_full{h}", it)
                    if j == 0 and k > 0:
                        yield from sim.wait(f"o_empty{h}", k - 1)
                    if h == 0:
                        yield from sim.wait(f"v_full{vc % VST}", vc // VST)
                    sim.arrive(f"o_bar{h}")
                sim.arrive(f"v_empty{vc % VST}")
                vc += 1
                it += 1

    def softmax(h):
        it = 0
        for nl, nc in items:
            for j in range(nl + nc):
                yield from sim.wait(f"s_full{h}", it)
                sim.arrive(f"s_free{h}")
                yield
                if it > 0:
                    yield from sim.wait(f"o_bar{h}", it - 1)
                sim.arrive(f"p_full{h}")
                if nc > 0 and j == nl - 1:
                    sim.arrive(f"qh_full{h}")
                it += 1
            yield from sim.wait(f"o_bar{h}", it - 1)
            sim.arrive(f"o_empty{h}")

    return [producer(), qk_issuer(), pv_issuer(), softmax(0), softmax(1)]


# ---------------------------------------------------------------- dQ

def dq_items(T, g, w, bhq, cta, grid):
    """(n_local, n_core) of the 128-row query tiles dealt to CTA `cta`."""
    nqt = (T + 127) // 128
    out = []
    for item in range(cta, nqt * bhq, grid):
        qt = nqt - 1 - item // bhq
        t0 = qt * 128
        tl = min(t0 + 127, T - 1)
        nl = (tl - ws_of(t0, g, w) + 1 + 127) // 128
        nc = (ws_of(tl, g, w) // g + 127) // 128
        out.append((nl, nc))
    return out


def dq_roles(sim: Sim, items, KST=3, VST=2, NW=8):
    for n in ("q_full", "q_empty", "s_full", "mm_done"):
        sim.bar(n)
    for n in ("s_free", "p_full", "acc_empty"):
        sim.bar(n, NW)
    for s in range(KST):
        sim.bar(f"k_full{s}")
        sim.bar(f"k_empty{s}")
    for s in range(VST):
        sim.bar(f"v_full{s}")
        sim.bar(f"v_empty{s}")
    seq = [(k, j, nl, nl + nc) for k, (nl, nc) in enumerate(items) for j in range(nl + nc)]

    def producer():
        qc = kc = vc = 0
        for nl, nc in items:
            for j in range(-1, nl + nc):
                if j == -1 or (nc > 0 and j == nl):  # bf16 Q, then its fp16 copy
                    if qc > 0:
                        yield from sim.wait("q_empty", qc - 1)
                    sim.arrive("q_full")
                    qc += 1
                    if j == -1:
                        continue
                if kc >= KST:
                    yield from sim.wait(f"k_empty{kc % KST}", kc // KST - 1)
                sim.arrive(f"k_full{kc % KST}")
                kc += 1
                if vc >= VST:
                    yield from sim.wait(f"v_empty{vc % VST}", vc // VST - 1)
                sim.arrive(f"v_full{vc % VST}")
                vc += 1

    def issuer():
        na = nb = qc = 0

        def issue_a():
            nonlocal na, qc
            k, j, nl, nt = seq[na]
            core = j >= nl
            if j == 0 or (core and j == nl):
                yield from sim.wait("q_full", qc)
                qc += 1
            yield from sim.wait(f"k_full{na % KST}", na // KST)
            yield from sim.wait(f"v_full{na % VST}", na // VST)
            if na > 0:
                yield from sim.wait("s_free", na - 1)
            sim.arrive("s_full")
            sim.arrive(f"v_empty{na % VST}")
            if j + 1 == nt or (not core and j + 1 == nl):
                sim.arrive("q_empty")
            na += 1

        def issue_b():
            nonlocal nb
            k, j, _, _ = seq[nb]
            yield from sim.wait("p_full", nb)
            if j == 0 and k > 0:
                yield from sim.wait("acc_empty", k - 1)
            sim.arrive("mm_done")
            sim.arrive(f"k_empty{nb % KST}")
            nb += 1

        if seq:
            yield from issue_a()
        while nb < na:
            if na < len(seq):
                yield from issue_a()
            yield from issue_b()

    def ds_warp():
        it = 0
        for nl, nc in items:
            for _ in range(nl + nc):
                yield from sim.wait("s_full", it)
                yield
                sim.arrive("s_free")
                if it > 0:
                    yield from sim.wait("mm_done", it - 1)
                sim.arrive("p_full")
                it += 1
            yield from sim.wait("mm_done", it - 1)
            sim.arrive("acc_empty")

    return [producer(), issuer()] + [ds_warp() for _ in range(NW)]


# ---------------------------------------------------------------- dK/dV

def dkv_items(T, g, w, B, Hkv, r, cta, grid, chunk=16):
    """Query tiles per work item (r x query-tile range) for CTA `cta`: core
    items (query ranges cut into chunks) first, then one item per raw key
    tile, as the kernel deals them."""
    nqt = (T + 127) // 128
    m = T // g
    nct = (m + 127) // 128
    pairs = B * Hkv
    tiles = []
    for ct in range(nct):
        qs = ((ct * 128 + 1) * g + w) // 128
        nch = (nqt - qs + chunk - 1) // chunk if qs < nqt else 0
        for c in range(nch):
            qa = qs + c * chunk
            tiles += [r * (min(qa + chunk, nqt) - qa)] * pairs
    for kt in range(nqt):
        klast = min(kt * 128 + 127, T - 1)
        tmax = min((klast // g + 1) * g + w - 1, T - 1)
        tiles += [r * (tmax // 128 + 1 - kt)] * pairs
    return [tiles[i] for i in range(cta, len(tiles), grid)]


def dkv_roles(sim: Sim, items, QST=2, epilogue_waits=(0, 1)):
    """`epilogue_waits`: the halves whose product barriers the epilogue waits
    on, in order (the kernel: half 0, then half 1)."""
    for n in ("kv_full", "kv_empty", "hs_full0", "hs_full1", "hmm_done0", "hmm_done1"):
        sim.bar(n)
    sim.bar("hp_full0", 4)
    sim.bar("hp_full1", 4)
    sim.bar("acc_empty", 8)
    for s in range(QST):
        sim.bar(f"q_full{s}")
        sim.bar(f"q_empty{s}")

    def producer():
        qc = kvc = 0
        for nt in items:
            if kvc > 0:
                yield from sim.wait("kv_empty", kvc - 1)
            sim.arrive("kv_full")
            kvc += 1
            for _ in range(nt):
                if qc >= QST:
                    yield from sim.wait(f"q_empty{qc % QST}", qc // QST - 1)
                sim.arrive(f"q_full{qc % QST}")
                qc += 1

    def issuer():
        kvc = base = 0

        def issue_a(h, n):
            if n > 0:
                yield from sim.wait(f"hmm_done{h}", n - 1)
            sim.arrive(f"hs_full{h}")

        def issue_b(h, n, first, k):
            yield from sim.wait(f"hp_full{h}", n)
            if h == 0 and first and k > 0:
                yield from sim.wait("acc_empty", k - 1)
            sim.arrive(f"hmm_done{h}")

        for k, nt in enumerate(items):
            yield from sim.wait("kv_full", kvc)
            kvc += 1
            yield from sim.wait(f"q_full{base % QST}", base // QST)
            yield from issue_a(0, base)
            yield from issue_a(1, base)
            for i in range(nt):
                n = base + i
                yield from issue_b(0, n, i == 0, k)
                if i + 1 < nt:
                    yield from sim.wait(f"q_full{(n + 1) % QST}", (n + 1) // QST)
                    yield from issue_a(0, n + 1)
                yield from issue_b(1, n, i == 0, k)
                sim.arrive(f"q_empty{n % QST}")
                if i + 1 < nt:
                    yield from issue_a(1, n + 1)
            base += nt
            sim.arrive("kv_empty")

    def warp(h):
        it = 0
        for nt in items:
            for _ in range(nt):
                yield  # stage this tile's per-column values
                yield from sim.wait(f"hs_full{h}", it)
                yield
                sim.arrive(f"hp_full{h}")
                it += 1
            for e in epilogue_waits:
                yield from sim.wait(f"hmm_done{e}", it - 1)
            sim.arrive("acc_empty")

    return [producer(), issuer()] + [warp(h) for h in (0, 0, 0, 0, 1, 1, 1, 1)]

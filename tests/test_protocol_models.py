"""The barrier protocols of the tcgen05 kernels, model-checked on the CPU
(tests/protocol_models.py): random interleavings of every role over work
items of the kernels' own geometry, for deadlock and for parity waits that
run ahead or alias.  A model of the dK/dV epilogue as it first was (waiting
only on the second half's product barrier) must be caught: the checker
found that bug's cause after the GPU suite had shown its symptom."""

import pytest

import protocol_models as pm

PREFILL_CASES = [(256, 16, 64, 1, 2), (300, 16, 64, 1, 2), (200, 8, 40, 2, 4), (130, 4, 0, 1, 4),
                 (100, 1, 10, 1, 2), (90, 16, 1000, 1, 2), (1, 16, 64, 1, 2), (1000, 4, 50, 1, 2),
                 (517, 5, 37, 1, 2), (384, 16, 64, 8, 16), (2048, 16, 1024, 1, 4),
                 (8192, 16, 1024, 1, 2), (129, 16, 64, 1, 1), (5000, 7, 333, 1, 2)]
BW_CASES = [(200, 16, 64, 1, 2), (300, 16, 64, 2, 2), (130, 1, 10, 1, 2), (100, 16, 1000, 1, 2),
            (333, 8, 40, 1, 4), (2500, 8, 64, 2, 1), (4096, 16, 1024, 1, 2), (1000, 4, 100, 1, 3)]


def _ctas(n_items):
    grid = max(1, min(n_items, 148))
    for grid_ in sorted({1, 2, 3, grid}):
        for cta in sorted({0, grid_ - 1, grid_ // 2}):
            yield cta, grid_


@pytest.mark.parametrize("case", PREFILL_CASES, ids=[str(c) for c in PREFILL_CASES])
def test_prefill_protocol(case):
    T, g, w, B, Hq = case
    n_items = ((T + 255) // 256) * B * Hq
    for cta, grid in _ctas(n_items):
        items = pm.prefill_items(T, g, w, B, Hq, cta, grid)
        for seed in range(2):
            sim = pm.Sim()
            sim.run(pm.prefill_roles(sim, items), seed)


@pytest.mark.parametrize("case", BW_CASES, ids=[str(c) for c in BW_CASES])
def test_dq_protocol(case):
    T, g, w, bhq, _ = case
    n_items = ((T + 127) // 128) * bhq
    for cta, grid in _ctas(n_items):
        items = pm.dq_items(T, g, w, bhq, cta, grid)
        for seed in range(2):
            sim = pm.Sim()
            sim.run(pm.dq_roles(sim, items), seed)


@pytest.mark.parametrize("case", BW_CASES, ids=[str(c) for c in BW_CASES])
def test_dkv_protocol(case):
    T, g, w, B, r = case
    n_items = len(pm.dkv_items(T, g, w, B, 1, r, 0, 1))
    for cta, grid in _ctas(n_items):
        items = pm.dkv_items(T, g, w, B, 1, r, cta, grid)
        for seed in range(2):
            sim = pm.Sim()
            sim.run(pm.dkv_roles(sim, items), seed)


def test_dkv_epilogue_on_second_half_only_is_caught():
    caught = False
    for seed in range(40):
        sim = pm.Sim()
        try:
            sim.run(pm.dkv_roles(sim, [2, 4, 1], epilogue_waits=(1,)), seed)
        except pm.ProtocolError as e:
            assert "runs ahead" in str(e)
            caught = True
            break
    assert caught


def test_checker_sees_a_missing_arrival():
    """A consumer that waits for a phase nobody completes is a deadlock."""
    sim = pm.Sim()
    sim.bar("never")

    def waiter():
        yield from sim.wait("never", 0)

    with pytest.raises(pm.ProtocolError, match="deadlock"):
        sim.run([waiter()], 0, limit=1000)

"""The failure path on the GPU, without a fault.

A kernel whose barrier never completes must end its wait after the bound,
record a timeout that cca_device_status() reports as CCA_ERR_TIMEOUT, and
leave the context usable.  cca_selftest_wait_timeout launches exactly such
a wait (a barrier nothing arrives at) with a 1 ms bound; nothing faults,
traps or hangs.
"""

import numpy as np
import pytest
import torch

import long_context_sparse_cca_b200 as cca
from long_context_sparse_cca_b200 import synth

pytestmark = pytest.mark.gpu


def test_stuck_wait_reports_timeout_and_context_survives():
    assert cca.cca_device_status() == cca.CCA_OK
    cca.cca_selftest_wait_timeout(1000)
    assert cca.cca_device_status() == cca.CCA_ERR_TIMEOUT
    # the record is cleared by reading it
    assert cca.cca_device_status() == cca.CCA_OK
    # and the context still runs the library's kernels correctly
    wl = synth.TINY
    x = synth.generate(wl)
    dev = lambda a: torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)  # noqa: E731
    Q, K, V = dev(x.q), dev(x.k), dev(x.v)
    Kc1, Vc1 = cca.cca_pool(Q, K, V, wl.g)
    O1 = cca.cca_attn_prefill(Q, K, V, Kc1, Vc1, wl.g, wl.w)
    assert cca.cca_device_status() == cca.CCA_OK
    cca.cca_selftest_wait_timeout(1000)
    Kc2, Vc2 = cca.cca_pool(Q, K, V, wl.g)
    O2 = cca.cca_attn_prefill(Q, K, V, Kc2, Vc2, wl.g, wl.w)
    assert cca.cca_device_status() == cca.CCA_ERR_TIMEOUT
    assert torch.equal(O1, O2) and torch.equal(Kc1, Kc2) and torch.equal(Vc1, Vc2)
    assert cca.cca_device_status() == cca.CCA_OK

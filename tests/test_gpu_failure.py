"""Failure detection on the GPU without a fault.

Every spin-wait of the library is bounded: when a signal never comes, the
kernel latches a timeout in the device's error word and returns, and the host
reads SBL_ERR_TIMEOUT from sbl_check.  sbl_selftest_wait_timeout takes that
path on purpose (a barrier phase that nothing completes, a 20 ms limit); the
test checks the status, that reading it clears it, and that the context still
runs the path correctly afterwards.
"""
import time

import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu


def test_expired_wait_reports_timeout_and_context_survives(lib):
    from semi_structured_sparsity_step_b200._binding import SblError, STATUS
    from semi_structured_sparsity_step_b200.layer import act_quant
    lib.sbl_check()  # nothing pending before the test
    t0 = time.perf_counter()
    lib.sbl_selftest_wait_timeout(20000)
    with pytest.raises(SblError) as e:
        lib.sbl_check()
    waited = time.perf_counter() - t0
    assert STATUS[e.value.status] == "SBL_ERR_TIMEOUT"
    assert waited >= 0.02
    lib.sbl_check()  # the latched error was cleared by the read
    x = synth.activations(33, 272, seed=9, tensor_id=1)
    xq = torch.empty(33, 272, dtype=torch.int8, device="cuda")
    amax = torch.empty(33, dtype=torch.float32, device="cuda")
    act_quant(x.cuda(), xq, amax)
    lib.sbl_check()
    ref_q, ref_a = oracle.act_quant(synth.bits(x))
    assert np.array_equal(xq.cpu().numpy(), ref_q)
    assert np.array_equal(amax.cpu().numpy(), ref_a)

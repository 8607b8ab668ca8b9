"""Failure detection on the device, without a GPU fault: a bounded wait runs out and
the host reads the error from the status word.

pact_selftest_wait_timeout makes one kernel thread wait, through the same bounded
mbarrier wait every libpact kernel uses, on a barrier that nothing completes, with
a short limit.  The wait gives up, the kernel records PACT_ERR_TIMEOUT in the
per-device status word and returns with nothing in flight.  The test checks that
pact_get_device_status reports it once (reading clears it), that the wait took at
least its limit, and that the context stays usable: a normal call afterwards runs
and matches the oracle, and the status is clean again."""
import numpy as np
import pytest
import torch

import synth
from tests.util import assert_nvfp4_equal, to_dev

pytestmark = pytest.mark.gpu

PACT_OK, PACT_ERR_TIMEOUT = 0, 5


def test_bounded_wait_runs_out_and_is_reported(orc):
    import nvfp4_gemm_b200 as P
    torch.cuda.set_device(0)
    assert P.pact_get_device_status() == PACT_OK, P.pact_last_error()      # clean start
    limit = 20_000_000                                                      # ~10 ms of SM cycles
    waited = torch.zeros(1, dtype=torch.int64, device="cuda")
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    P.pact_selftest_wait_timeout(limit, waited)
    t1.record()
    torch.cuda.synchronize()
    assert P.pact_get_device_status() == PACT_ERR_TIMEOUT
    assert "bounded wait" in P.pact_last_error()
    assert P.pact_get_device_status() == PACT_OK                            # reading cleared it
    assert int(waited.item()) > limit
    assert t0.elapsed_time(t1) > 1.0                                        # it really waited (ms)
    # the context is usable: a normal call runs and is right
    x = synth.gaussian_bf16(7, (130, 256))
    xq = P.pact_quantize_nvfp4(to_dev(x))
    torch.cuda.synchronize()
    assert P.pact_get_device_status() == PACT_OK, P.pact_last_error()
    assert_nvfp4_equal(xq, orc.quantize(x), orc, "quantize after a timeout")


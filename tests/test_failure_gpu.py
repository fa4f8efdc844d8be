"""Failure detection on the GPU without a fault: a kernel waits, through the same bounded wait
every kernel of the path uses, on an mbarrier that nothing completes.  The wait must give up after
its limit, record a timeout (kind 5, site 30) in the device status word, and leave the context
usable: the next forward call still matches the oracle and reports no error."""
import pytest
import torch

import causal_sliding_window_swa_b200 as swa
import workloads
from tests import parity

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)
    yield


def test_bounded_wait_expires_and_context_stays_usable():
    assert swa.swa_attn_last_device_status()[0] == swa.SWA_OK    # clear anything pending
    assert swa.swa_attn_selftest_wait(50, None) == swa.SWA_OK
    rc, detail = swa.swa_attn_last_device_status()
    assert rc == swa.SWA_ERR_TIMEOUT, (rc, hex(detail))
    assert detail & 0xff == 5 and (detail >> 8) & 0xff == 30, hex(detail)
    # the status word was cleared by the read
    assert swa.swa_attn_last_device_status() == (swa.SWA_OK, 0)
    # the device still runs the path correctly
    err = parity.check_full(workloads.TINY)
    assert err["max_abs"] <= parity.OUT_MAX_ABS
    assert swa.swa_attn_last_device_status() == (swa.SWA_OK, 0)

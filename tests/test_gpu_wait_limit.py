"""Failure detection on the device without a fault: the bounded barrier wait that every
GEMM pipeline role uses gives up after its limit, records TIMEOUT in the device status
word, makes the CTA's other waits give up too, and returns, leaving the context usable.
The wait runs out because nothing ever arrives on its barrier; no fault, trap or endless
loop is involved (each wait ends by the global timer)."""
import pytest
import torch

import mxfp4_microscaled_bit_b200 as fl
import synthetic_inputs as si
from gpu_util import DEV, check_nvfp4, status_ok

pytestmark = pytest.mark.gpu

TIMEOUT = 5  # FP4LIN_ERR_TIMEOUT


def test_waits_complete_when_the_barrier_is_arrived_on():
    status_ok()
    r = fl.wait_selftest(2_000_000, arrive=True, device=DEV).cpu().tolist()
    assert r[0] == 1 and r[1] == 1, r
    assert r[2] < 1_000_000 and r[3] < 1_000_000, r  # no time spent near the limit
    status_ok()


@pytest.mark.parametrize("limit_ns", [10_000, 2_000_000])
def test_wait_expires_reports_timeout_and_releases_the_cta(limit_ns, orc):
    status_ok()
    r = fl.wait_selftest(limit_ns, arrive=False, device=DEV).cpu().tolist()
    done0, done1, ns0, ns1 = r
    assert done1 == 0 and done0 == 0, r
    # the limited wait ran at least its limit, and far less than the library's 1 s limit
    assert limit_ns <= ns1 < 500_000_000, r
    # the other wait gave up on the abort flag, not by its own 1 s limit
    assert ns0 < 500_000_000, r
    assert fl.device_status() == TIMEOUT
    status_ok()  # reading the status cleared it
    # the context still runs the library: a quantisation matches the oracle bit for bit
    check_nvfp4(orc, si.normal_bf16(5, 256, 512), hadamard=16)
    status_ok()


def test_status_keeps_the_first_error_until_read():
    fl.wait_selftest(10_000, arrive=False, device=DEV)
    fl.wait_selftest(10_000, arrive=True, device=DEV)  # a later clean run does not clear it
    assert fl.device_status() == TIMEOUT
    status_ok()

"""The failure path of the library's bounded device waits, exercised without
faulting or hanging the GPU: a kernel waits on a barrier that nothing
signals, its wait expires, the status flag reports ZQ_ERR_TIMEOUT on the
host, the flag clears, and the context keeps computing correctly."""
import time

import numpy as np
import pytest
import torch

import oracle
from tests.gpu_helpers import dev, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def zq():
    from w8a8_post_quantized_b200 import zq as m
    m.lib()
    return m


def test_expired_wait_reports_timeout_and_context_survives(zq):
    zq.zq_device_status()                       # start from a clear flag
    t0 = time.monotonic()
    zq.zq_watchdog_selftest()
    with pytest.raises(zq.ZQError) as e:
        zq.zq_device_status()
    assert e.value.status == zq.ZQ_ERR_TIMEOUT
    waited = time.monotonic() - t0
    assert 1.0 < waited < 30.0                  # the wait limit is about 2 s
    assert "0x7e57" in zq.lib().zq_last_cuda_error().decode()
    zq.zq_device_status()                       # the flag was cleared
    # the context still computes: a quantizer call matches the oracle bit for bit
    rng = np.random.default_rng(5)
    x = rng.standard_normal((33, 256)).astype(np.float32)
    q, s = zq.zq_act_quant(dev(x))
    q_ref, s_ref = oracle.quantize_rows(x)
    np.testing.assert_array_equal(host(q), q_ref)
    np.testing.assert_array_equal(host(s), s_ref)
    zq.zq_device_status()

"""GPU: failure detection without a fault.  A bounded wait that can never
complete (mxfp4_selftest_wait_timeout) expires after its budget, records a
timeout for its role in the device status word, ends the other waiter
through the abort flag (no second record), and leaves the context usable: a
quantisation right after it is still bit-exact against the oracle."""
import numpy as np
import pytest
import torch

import oracle
from fp4_precision_numerics_b200 import mxfp4, synth
from tests.gpu_util import dev_bf16, host

pytestmark = pytest.mark.gpu


def test_expired_wait_is_reported_and_the_context_stays_usable():
    mxfp4.mxfp4_check_device_status()                      # clean start
    mxfp4.mxfp4_selftest_wait_timeout()
    with pytest.raises(mxfp4.MXFP4Error) as e:
        mxfp4.mxfp4_check_device_status()
    assert e.value.status == -5                            # MXFP4_ERR_DEVICE_TIMEOUT
    msg = mxfp4.last_error()
    assert "mma" in msg and "epilogue" not in msg, msg
    mxfp4.mxfp4_check_device_status()                      # read once, then cleared
    rng = np.random.default_rng(3)
    x = synth.bf16_bits(rng.standard_normal((64, 256)).astype(np.float32))
    q = mxfp4.quantize(dev_bf16(x), scales=True)
    torch.cuda.synchronize()
    c, s = oracle.quantize_1d(x)
    assert np.array_equal(host(q["codes"][0]), c) and np.array_equal(host(q["scales"][0]), s)

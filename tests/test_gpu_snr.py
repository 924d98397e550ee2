"""The operator-level SNR report (fp4_precision_numerics_b200.snr) runs
through the library's kernels and shows the properties its techniques are
for: stochastic rounding costs SNR against nearest rounding (it trades
variance for unbiasedness), the RHT helps on the outlier layer and on
heavy-tailed activations, and de-oscillation lowers how often codes change
between steps at a small SNR cost."""
import numpy as np
import pytest

from fp4_precision_numerics_b200 import snr

pytestmark = pytest.mark.gpu


def test_snr_db_closed_form():
    ref = np.ones(100)
    assert abs(snr.snr_db(ref, ref * 1.1) - 20.0) < 1e-9      # noise power 1% -> 20 dB


def test_single_layer_and_activation_snr():
    c1 = snr.config1()
    assert c1[(True, False)] > c1[(False, False)] + 3.0        # outliers: the RHT spreads them
    assert c1[(False, True)] < c1[(False, False)]
    c2 = snr.config2(1024, 2880)
    assert 10.0 < c2[(False, False)] < 25.0
    assert c2[(True, False)] > c2[(False, False)]              # Student-t tails
    assert c2[(False, True)] < c2[(False, False)] and c2[(True, True)] < c2[(True, False)]


def test_deosc_lowers_code_changes():
    d = snr.deosc(steps=12)
    assert d[True][1] < d[False][1]
    assert abs(d[True][0] - d[False][0]) < 2.0

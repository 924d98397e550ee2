"""CPU: the bench's algorithmic work per launch (the roofline numerators)
equals the per-unit figures: 2 r N K FLOP per GEMM over the 65,536 routed
rows (9.78 TFLOP per step), 3.0625 B per element for the dual quantiser
(2 B in, 1/2 + 1/32 B out in each direction) and 7.0625 B per weight for
de-oscillation (4 B master + 1 B state in; 1 B state, 1/2 + 1/2 B W and W^T
codes, 2/32 B scales out)."""
import os
import sys

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402


def test_algorithmic_work_of_the_moe_layer_step():
    rows, M, E, D, F = 65536, 67584, 32, 2880, 5760
    flops, qbytes = bench.algorithmic_work(rows, M, E)
    assert set(flops) | set(qbytes) == set(bench.KERNELS)
    assert sum(flops.values()) == 3 * 2 * rows * D * (F + D)
    assert abs(sum(flops.values()) - 9.78e12) < 0.005e12
    assert flops["wgrad_up"] == flops["fprop_up"] == flops["dgrad_up"] == 2 * rows * F * D
    assert qbytes["deosc_up"] == E * F * D * 7.0625 and qbytes["deosc_down"] == E * D * D * 7.0625
    for k, cols in (("dual_x", D), ("dual_h", D), ("dual_dy_up", F), ("dual_dy_down", D)):
        assert qbytes[k] == M * cols * 3.0625

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


def test_gemm_roofline_takes_the_longer_roof():
    rows, M, E = 65536, 67584, 32
    flops, _ = bench.algorithmic_work(rows, M, E)
    D, F = 2880, 5760
    per = 0.5 + 1.0 / 32
    # wgrad_up: operands (F + D) x tokens once, binary32 dW [E, F, D] once
    wgrad_bytes = (F + D) * M * per + E * F * D * 4
    # fprop_up: X [M, D] and W_up [E, F, D] codes once, binary32 Y [M, F] once
    fprop_bytes = (M * D + E * F * D) * per + M * F * 4
    peak_t, peak_h = 6665.6, 6551.0
    w = bench.gemm_roofline(flops["wgrad_up"], wgrad_bytes, 0.74, peak_t, 5455.0, peak_h, "t", "h")
    f = bench.gemm_roofline(flops["fprop_up"], fprop_bytes, 0.65, peak_t, 5455.0, peak_h, "t", "h")
    # wgrad: 2.43 GB at 6551 GB/s (0.371 ms) outlasts 2.17 TFLOP at 6666 TFLOP/s (0.326 ms)
    assert w["bound"] == "hbm" and w["unit"] == "GB/s" and w["peak"] == peak_h
    assert abs(w["roof_ms"]["hbm"] - 0.3715) < 1e-3 and abs(w["roof_ms"]["tensor"] - 0.3262) < 1e-3
    assert abs(w["frac"] - wgrad_bytes / 0.74e-3 / 1e9 / peak_h) < 1e-12
    assert abs(w["frac_tensor"] - flops["wgrad_up"] / 0.74e-3 / 1e12 / peak_t) < 1e-12
    # fprop: the tensor roof is the longer one
    assert f["bound"] == "tensor" and f["unit"] == "TFLOP/s" and f["roof_ms"]["tensor"] > f["roof_ms"]["hbm"]
    assert abs(f["frac"] - f["frac_tensor"]) < 1e-15

"""Benchmark: one MXFP4 training step of a GPT-OSS-20B-shaped MoE expert
layer through libmxfp4 (the ALTO recipe's quantise-and-contract hot path).

A step, all on one GPU and one stream:
  1. de-oscillation re-quantisation of the fp32 master weights W_up
     [32, 5760, 2880] and W_down [32, 2880, 2880] (2D 32x32 blocks; emits W
     and W^T codes and tensor-core scales),
  2. quantise X and H (1x32 along K, nearest) -> fprop GEMMs Y_up, Y_down,
  3. quantise dY_up, dY_down (1x32 along N, SR) -> dgrad GEMMs dX, dH,
  4. quantise X^T, H^T, dY_up^T, dY_down^T along tokens (RHT-16; SR on
     gradients) -> wgrad GEMMs dW_up, dW_down (fp32).
16384 tokens routed top-4 over 32 experts with Zipf(1.1) skew (65536 routed
rows, segments padded to 128).  Inputs are synthetic (seeded), bigger than
L2, resident in HBM when the timed region starts.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
For N > 1 launch with torchrun (one process per GPU); every rank runs its
own replica of the layer (the path has no exchange step), so per-GPU work is
fixed and the result line reports weak scaling.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "MXFP4 grouped-GEMM TFLOPS + quantise GB/s, % of FP4/HBM roofline, 1 B200"
WORKLOAD = ("GPT-OSS-20B-shaped MoE expert layer, full MXFP4 training step (fprop + dgrad + wgrad, "
            "2D de-oscillation weight re-quantisation), 32 experts, d_model 2880, W_up 5760x2880, "
            "W_down 2880x2880, 16384 tokens top-4 Zipf(1.1)")
E, D, F = 32, 2880, 5760
NOMINAL_FP4_OVER_BF16 = 4.0          # dense FP4 / dense BF16 tensor rate, B200 datasheet (9 / 2.25 PFLOP/s)
NOMINAL_HBM_GBS = 8000.0             # B200 HBM3e, datasheet
NOMINAL_FP4_TFLOPS = 9000.0          # B200 dense FP4, datasheet


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return dict(hbm_gbs=float(j["hbm_gbs"]), bf16_burst=float(j["bf16_tflops"]),
                    bf16_sustained=float(j.get("bf16_tflops_sustained", j["bf16_tflops"])), source="measured")
    return dict(hbm_gbs=6650.0, bf16_burst=1590.0, bf16_sustained=1400.0, source="fallback")


# ---------------------------------------------------------------------------
# Workload
# ---------------------------------------------------------------------------
def algorithmic_work(rows_real, M, n_experts):
    """Per-launch algorithmic work of the step's kernels, the roofline
    numerators.  GEMMs: 2 r N K FLOP over the r real (routed) rows.  The dual
    quantiser reads its bf16 input once and writes codes (1/2 B) and scales
    (1/32 B) in each direction: 3.0625 B per element of the padded [M, cols]
    input.  De-oscillation reads the fp32 master and the state byte and
    writes the state, the W and W^T codes and both scale layouts: 7.0625 B
    per weight."""
    r = rows_real
    gemm_flops = {
        "fprop_up": 2.0 * r * F * D, "fprop_down": 2.0 * r * D * D,
        "dgrad_up": 2.0 * r * F * D, "dgrad_down": 2.0 * r * D * D,
        "wgrad_up": 2.0 * r * F * D, "wgrad_down": 2.0 * r * D * D,
    }
    q2 = 2.0 + 2 * (0.5 + 1.0 / 32)
    per_weight = 4 + 1 + 1 + 0.5 + 0.5 + 2.0 / 32
    quant_bytes = {
        "deosc_up": n_experts * F * D * per_weight,
        "deosc_down": n_experts * D * D * per_weight,
        "dual_x": M * D * q2, "dual_h": M * D * q2, "dual_dy_up": M * F * q2, "dual_dy_down": M * D * q2,
    }
    return gemm_flops, quant_bytes


class Layer:
    """Device buffers of one MoE layer replica and its training step."""

    def __init__(self, dev, seed=0, n_experts=32, n_tokens=16384):
        import numpy as np
        import torch

        from fp4_precision_numerics_b200 import mxfp4, synth
        self.mx = mxfp4
        global E
        E = n_experts
        self.n_tokens = n_tokens
        routing = synth.zipf_routing(n_tokens=n_tokens, n_experts=n_experts, seed=2)
        counts, offsets, tor = synth.expert_layout(routing, n_experts)
        self.counts = counts
        self.M = int(offsets[-1])
        self.rows_real = int(counts.sum())
        self.offsets = torch.tensor(offsets.astype(np.int32), device=dev)
        M = self.M
        g = torch.Generator(device=dev)
        g.manual_seed(1000 + seed)
        pad = torch.from_numpy(tor < 0).to(dev)

        def act(shape, std):
            t = torch.randn(shape, generator=g, device=dev, dtype=torch.float32).mul_(std).to(torch.bfloat16)
            t[pad] = 0
            return t

        # token activations are gathered into expert order (each token appears top-4 times)
        x_tok = torch.randn((n_tokens, D), generator=g, device=dev, dtype=torch.float32).to(torch.bfloat16)
        idx = torch.from_numpy(np.where(tor < 0, 0, tor)).to(dev)
        self.x = x_tok[idx]
        self.x[pad] = 0
        self.h = act((M, D), 1.0)
        self.dy_up = act((M, F), 1e-3)
        self.dy_down = act((M, D), 1e-3)
        self.w_up = torch.randn((E, F, D), generator=g, device=dev, dtype=torch.float32).mul_(0.02)
        self.w_down = torch.randn((E, D, D), generator=g, device=dev, dtype=torch.float32).mul_(0.02)
        self.st_up = torch.zeros((E, F, D), dtype=torch.uint8, device=dev)
        self.st_down = torch.zeros((E, D, D), dtype=torch.uint8, device=dev)
        u8 = dict(dtype=torch.uint8, device=dev)
        f32 = dict(dtype=torch.float32, device=dev)
        sb = mxfp4.mxfp4_mma_scale_bytes
        self.q = {
            "w_up": dict(codes=torch.empty((E, F, D // 2), **u8), scales_mma=torch.empty((E, sb(F, D // 32)), **u8),
                         codes_t=torch.empty((E, D, F // 2), **u8), scales_mma_t=torch.empty((E, sb(D, F // 32)), **u8)),
            "w_down": dict(codes=torch.empty((E, D, D // 2), **u8), scales_mma=torch.empty((E, sb(D, D // 32)), **u8),
                           codes_t=torch.empty((E, D, D // 2), **u8), scales_mma_t=torch.empty((E, sb(D, D // 32)), **u8)),
            "x": dict(codes=torch.empty((1, M, D // 2), **u8), scales_mma=torch.empty((1, sb(M, D // 32)), **u8)),
            "h": dict(codes=torch.empty((1, M, D // 2), **u8), scales_mma=torch.empty((1, sb(M, D // 32)), **u8)),
            "dy_up": dict(codes=torch.empty((1, M, F // 2), **u8), scales_mma=torch.empty((1, sb(M, F // 32)), **u8)),
            "dy_down": dict(codes=torch.empty((1, M, D // 2), **u8), scales_mma=torch.empty((1, sb(M, D // 32)), **u8)),
            "xt": dict(codes=torch.empty((1, D, M // 2), **u8), scales_mma=torch.empty((1, sb(D, M // 32)), **u8)),
            "ht": dict(codes=torch.empty((1, D, M // 2), **u8), scales_mma=torch.empty((1, sb(D, M // 32)), **u8)),
            "dy_up_t": dict(codes=torch.empty((1, F, M // 2), **u8), scales_mma=torch.empty((1, sb(F, M // 32)), **u8)),
            "dy_down_t": dict(codes=torch.empty((1, D, M // 2), **u8), scales_mma=torch.empty((1, sb(D, M // 32)), **u8)),
        }
        self.y_up = torch.empty((M, F), **f32)
        self.y_down = torch.empty((M, D), **f32)
        self.dx = torch.empty((M, D), **f32)
        self.dh = torch.empty((M, D), **f32)
        self.dw_up = torch.empty((E, F, D), **f32)
        self.dw_down = torch.empty((E, D, D), **f32)
        self.step_idx = 0
        self.launches_per_step = 12
        self.gemm_flops, self.quant_bytes = algorithmic_work(self.rows_real, M, E)
        self.gemm_dims = {
            "fprop_up": (M, F, D), "fprop_down": (M, D, D), "dgrad_up": (M, D, F), "dgrad_down": (M, D, D),
            "wgrad_up": (F, D, M), "wgrad_down": (D, D, M),
        }

    FUSED = ("fprop_up", "fprop_down", "dgrad_up", "dgrad_down")

    def alloc_fused(self):
        """Outputs of the fused-epilogue variant of the fprop/dgrad GEMMs:
        bf16 Y and its 1x32-along-N codes and tensor-core scales."""
        import torch
        sb = self.mx.mxfp4_mma_scale_bytes
        self.fused_out = {}
        for name in self.FUSED:
            Mg, N, _ = self.gemm_dims[name]
            self.fused_out[name] = (torch.empty((Mg, N), dtype=torch.bfloat16, device=self.offsets.device),
                                    dict(codes=torch.empty((Mg, N // 2), dtype=torch.uint8, device=self.offsets.device),
                                         scales_mma=torch.empty((sb(Mg, N // 32),), dtype=torch.uint8,
                                                                device=self.offsets.device)))

    def fused_out_bytes(self, name):
        """Algorithmic HBM bytes of one fused fprop/dgrad launch: operands read
        once, bf16 output plus its codes and scales written once."""
        Mg, N, K = self.gemm_dims[name]
        per = 0.5 + 1.0 / 32
        return (Mg * K + E * N * K) * per + Mg * N * (2 + per)

    def gemm_out_bytes(self, name):
        """Algorithmic HBM bytes of one GEMM launch: each operand's codes and
        scales read once, the binary32 output written once."""
        Mg, N, K = self.gemm_dims[name]
        per = 0.5 + 1.0 / 32
        if name.startswith("wgrad"):
            return (Mg + N) * K * per + E * Mg * N * 4
        return (Mg * K + E * N * K) * per + Mg * N * 4

    def step(self, ev=None, fused=False):
        """One training step.  `ev` (optional) maps a kernel name to a pair of
        CUDA events recorded around its launch on the current stream.  With
        `fused`, fprop and dgrad write bf16 outputs and their MXFP4
        quantisation (the fused epilogue; SR for dgrad's gradient outputs)
        instead of binary32."""
        import torch
        mx = self.mx
        q = self.q

        def gemm(name, op, a, b, b_codes, b_scales, Mg, N, K, out):
            if fused:
                # dgrad's output is a gradient: its codes take SR (own offsets)
                y, qo = self.fused_out[name]
                sr = dict(sr_seed=1, sr_offset=2000 + 2 * self.step_idx + (name == "dgrad_down")) \
                    if op == mx.GEMM_DGRAD else {}
                mx.grouped_gemm_fused(op, self.offsets, q[a]["codes"], q[a]["scales_mma"], q[b][b_codes],
                                      q[b][b_scales], Mg, N, K, scales=False, y=y, out=qo, **sr)
            else:
                mx.grouped_gemm(op, self.offsets, q[a]["codes"], q[a]["scales_mma"], q[b][b_codes], q[b][b_scales],
                                Mg, N, K, out=out)

        def rec(name, i):
            # an NVTX range per launch (for profiler timelines) and, when
            # asked, CUDA events around it
            if i == 0:
                torch.cuda.nvtx.range_push(name)
            if ev is not None:
                ev[name][i].record()
            if i == 1:
                torch.cuda.nvtx.range_pop()

        s = self.step_idx
        rec("deosc_up", 0)
        mx.deosc_update(self.w_up, s, self.st_up, scales=False, scales_mma=True, transposed=True, out=q["w_up"])
        rec("deosc_up", 1)
        rec("deosc_down", 0)
        mx.deosc_update(self.w_down, s, self.st_down, scales=False, scales_mma=True, transposed=True,
                        out=q["w_down"])
        rec("deosc_down", 1)
        M = self.M
        # activations and gradients: one dual-direction quantisation each gives
        # the contraction-dim operand (fprop/dgrad) and the token-dim RHT operand (wgrad)
        rec("dual_x", 0)
        mx.quantize_dual(self.x, col_rht_seed=1, scales=False, scales_mma=True, out_row=q["x"], out_col=q["xt"])
        rec("dual_x", 1)
        rec("fprop_up", 0)
        gemm("fprop_up", mx.GEMM_FPROP, "x", "w_up", "codes", "scales_mma", M, F, D, self.y_up)
        rec("fprop_up", 1)
        rec("dual_h", 0)
        mx.quantize_dual(self.h, col_rht_seed=1, scales=False, scales_mma=True, out_row=q["h"], out_col=q["ht"])
        rec("dual_h", 1)
        rec("fprop_down", 0)
        gemm("fprop_down", mx.GEMM_FPROP, "h", "w_down", "codes", "scales_mma", M, D, D, self.y_down)
        rec("fprop_down", 1)
        rec("dual_dy_up", 0)
        mx.quantize_dual(self.dy_up, col_rht_seed=1, sr_seed=1, row_sr_offset=2 * s, col_sr_offset=1000 + 2 * s,
                         scales=False, scales_mma=True, out_row=q["dy_up"], out_col=q["dy_up_t"])
        rec("dual_dy_up", 1)
        rec("dgrad_up", 0)
        gemm("dgrad_up", mx.GEMM_DGRAD, "dy_up", "w_up", "codes_t", "scales_mma_t", M, D, F, self.dx)
        rec("dgrad_up", 1)
        rec("dual_dy_down", 0)
        mx.quantize_dual(self.dy_down, col_rht_seed=1, sr_seed=1, row_sr_offset=2 * s + 1,
                         col_sr_offset=1001 + 2 * s, scales=False, scales_mma=True, out_row=q["dy_down"],
                         out_col=q["dy_down_t"])
        rec("dual_dy_down", 1)
        rec("dgrad_down", 0)
        gemm("dgrad_down", mx.GEMM_DGRAD, "dy_down", "w_down", "codes_t", "scales_mma_t", M, D, D, self.dh)
        rec("dgrad_down", 1)
        rec("wgrad_up", 0)
        mx.grouped_gemm(mx.GEMM_WGRAD, self.offsets, q["dy_up_t"]["codes"], q["dy_up_t"]["scales_mma"],
                        q["xt"]["codes"], q["xt"]["scales_mma"], F, D, M, out=self.dw_up)
        rec("wgrad_up", 1)
        rec("wgrad_down", 0)
        mx.grouped_gemm(mx.GEMM_WGRAD, self.offsets, q["dy_down_t"]["codes"], q["dy_down_t"]["scales_mma"],
                        q["ht"]["codes"], q["ht"]["scales_mma"], D, D, M, out=self.dw_down)
        rec("wgrad_down", 1)
        self.step_idx += 1


# DRAM bytes per launch on the full workload (32 experts, 16384 tokens):
# ncu dram__bytes_read.sum + dram__bytes_write.sum of each launch of the
# 8-expert / 4096-token layer, whose every tensor is exactly a quarter of the
# full one, times 4; one kernel and at most three launches per capture (the
# commands are in profiles/moe_layer_small_dram_counters.md).  An entry must
# go back to None when its kernel changes.
DRAM_BYTES_FULL = {
    "deosc_up": 4 * (663.90e6 + 242.47e6), "deosc_down": 4 * (332.08e6 + 102.85e6),
    "dual_x": 4 * (97.39e6 + 19.04e6), "dual_h": 4 * (97.39e6 + 13.97e6),
    "dual_dy_up": 4 * (194.73e6 + 67.89e6), "dual_dy_down": 4 * (97.43e6 + 11.64e6),
    "fprop_up": 4 * (97.13e6 + 332.59e6), "fprop_down": 4 * (61.32e6 + 135.22e6),
    "dgrad_up": 4 * (122.53e6 + 149.11e6), "dgrad_down": 4 * (61.32e6 + 137.45e6),
    "wgrad_up": 4 * (78.72e6 + 467.04e6), "wgrad_down": 4 * (51.96e6 + 202.02e6),
}

def gemm_roofline(flops, alg_bytes, ms, fp4_peak, fp4_sustained, hbm_gbs, tensor_src, hbm_src):
    """Roofline entry of one GEMM launch.  The kernel is bound by whichever
    roof takes longer for its algorithmic work: its flops at the FP4 peak
    (TFLOP/s), or its bytes (operand codes and scales once, the binary32
    output once) at the HBM peak (GB/s).  That roof gives `bound`, `achieved`,
    `peak` and `frac`; the fractions against the other roof are kept beside
    them."""
    tflops = flops / (ms / 1e3) / 1e12
    gbs = alg_bytes / (ms / 1e3) / 1e9
    t_tensor_ms = flops / (fp4_peak * 1e12) * 1e3
    t_hbm_ms = alg_bytes / (hbm_gbs * 1e9) * 1e3
    if t_hbm_ms > t_tensor_ms:
        roof = {"bound": "hbm", "achieved": gbs, "peak": hbm_gbs, "unit": "GB/s", "frac": gbs / hbm_gbs,
                "peak_source": hbm_src, "peak_nominal": NOMINAL_HBM_GBS, "frac_nominal": gbs / NOMINAL_HBM_GBS}
    else:
        roof = {"bound": "tensor", "achieved": tflops, "peak": fp4_peak, "unit": "TFLOP/s", "frac": tflops / fp4_peak,
                "peak_source": tensor_src, "peak_nominal": NOMINAL_FP4_TFLOPS,
                "frac_nominal": tflops / NOMINAL_FP4_TFLOPS}
    roof.update({"alg_bytes": alg_bytes, "roof_ms": {"tensor": round(t_tensor_ms, 4), "hbm": round(t_hbm_ms, 4)},
                 "tflops": tflops, "frac_tensor": tflops / fp4_peak, "peak_tensor": fp4_peak,
                 "peak_tensor_source": tensor_src, "frac_tensor_sustained": tflops / fp4_sustained,
                 "frac_tensor_nominal": tflops / NOMINAL_FP4_TFLOPS, "gbs": gbs, "frac_hbm": gbs / hbm_gbs})
    return roof


KERNELS = ["deosc_up", "deosc_down", "dual_x", "fprop_up", "dual_h", "fprop_down", "dual_dy_up", "dgrad_up",
           "dual_dy_down", "dgrad_down", "wgrad_up", "wgrad_down"]


# Thread instructions per element of the stochastic-rounding quantisers:
# ncu smsp__inst_executed.sum x 32 / elements of one launch (profiles/ gives
# the commands).  An entry must go back to None when its kernel changes.
SR_INST_PER_ELEMENT = {"dual_dy_up": 20.59, "dual_dy_down": 20.94, "rows_sr": 10.39}
SMSP_PER_SM = 4          # warp schedulers per SM, each issuing one warp instruction per cycle


def issue_roof_ms(inst_per_element, elements, n_sms, sm_mhz):
    """Time to issue `inst_per_element` thread instructions for every element
    at one warp instruction per scheduler per cycle on every SM at the given
    clock: the ALU roof of an instruction-bound kernel."""
    warp_inst = inst_per_element * elements / 32.0
    return warp_inst / (n_sms * SMSP_PER_SM) / (sm_mhz * 1e6) * 1e3



# ---------------------------------------------------------------------------
# Clock sampling
# ---------------------------------------------------------------------------
class ClockSampler:
    """SM clock and clock-event (throttle) reasons of one GPU, sampled during
    the timed region: through NVML every ~5 ms, else `nvidia-smi -lms 50`.
    It only reads; no setting of the GPU is touched."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")
    # NVML clock-event reason bits (every one NVML defines, so a slow clock is never left unexplained)
    REASON_BITS = {"gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4, "hw_slowdown": 0x8,
                   "sync_boost": 0x10, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
                   "hw_power_brake_slowdown": 0x80, "display_clock_setting": 0x100}

    def __init__(self, gpu_id):
        self.gpu_id = gpu_id
        self.samples = []          # (time, sm_mhz, max_mhz, set of reasons)
        self.proc = None
        self.thread = None
        self.stop_flag = threading.Event()

    def start(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            uuid = str(self.gpu_id)
            h = (pynvml.nvmlDeviceGetHandleByUUID(uuid) if uuid.startswith("GPU-")
                 else pynvml.nvmlDeviceGetHandleByIndex(int(uuid)))
            self.thread = threading.Thread(target=self._nvml, args=(pynvml, h), daemon=True)
            self.thread.start()
            return
        except Exception:
            pass
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu_id), "--query-gpu=" + self.FIELDS,
                                          "--format=csv,noheader,nounits", "-lms", "50"], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _nvml(self, pynvml, h):
        get_reasons = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
        max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
        while not self.stop_flag.is_set():
            try:
                mhz = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
                bits = get_reasons(h)
            except Exception:
                break
            reasons = {n for n, b in self.REASON_BITS.items() if bits & b}
            self.samples.append((time.time(), float(mhz), float(max_mhz), reasons))
            time.sleep(0.005)

    def _read(self):
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.strip().split(",")]
            if len(parts) < 8:
                continue
            try:
                mhz, maxmhz = float(parts[0]), float(parts[1])
            except ValueError:
                continue
            reasons = {n for n, v in zip(names, parts[4:8]) if v.lower().startswith("active")}
            self.samples.append((time.time(), mhz, maxmhz, reasons))

    def stop(self):
        self.stop_flag.set()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=2)

    def summary_windows(self, windows):
        """Summary of the samples taken inside any of the (t0, t1) windows."""
        rows = [r for r in self.samples if any(a <= r[0] <= b for a, b in windows)]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        reasons = set()
        for r in rows:
            reasons |= r[3]
        return {"sm_mhz": statistics.median(r[1] for r in rows), "sm_max_mhz": max(r[2] for r in rows),
                "sm_mhz_min": min(r[1] for r in rows), "reasons": sorted(reasons), "samples": len(rows)}

    def summary(self, t0, t1):
        rows = [r for r in self.samples if t0 <= r[0] <= t1] or self.samples
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        reasons = set()
        for r in rows:
            reasons |= r[3]
        return {"sm_mhz": statistics.median(r[1] for r in rows), "sm_max_mhz": max(r[2] for r in rows),
                "sm_mhz_min": min(r[1] for r in rows), "reasons": sorted(reasons), "samples": len(rows)}


# ---------------------------------------------------------------------------
# Distributed plumbing
# ---------------------------------------------------------------------------
def dist_setup(n_gpus):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != n_gpus and world > 1:
        raise SystemExit("WORLD_SIZE %d != --gpus %d" % (world, n_gpus))
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
        pg = dist
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return rank, world, local, pg


def max_over_ranks(value, pg, device):
    """Max of a float over all ranks (identity for one rank)."""
    if pg is None:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def barrier(pg):
    if pg is not None:
        pg.barrier()


# ---------------------------------------------------------------------------
# CPU baseline: the oracle on a bounded sample of the same step
# ---------------------------------------------------------------------------
CPU_SAMPLE_ROWS = 24576   # ~10 s of oracle work on the GPU machine's host cores


def cpu_baseline_sample(rows=256, expert=0):
    """Time the oracle (as it stands) on a bounded sample of the step: the
    first `rows` routed rows of one expert through the up-projection's three
    GEMMs with the quantisations they need (1x32 X, SR dY, 2D W with
    de-oscillation state, RHT-16 transposed operands for wgrad).  Returns
    (TFLOP/s of GEMM work over the sample's wall time, seconds, threads)."""
    import numpy as np

    import oracle
    from fp4_precision_numerics_b200 import synth
    rng = np.random.default_rng(0)
    x = synth.bf16_bits(rng.standard_normal((rows, D)).astype(np.float32))
    dy = synth.bf16_bits((rng.standard_normal((rows, F)) * 1e-3).astype(np.float32))
    w = (rng.standard_normal((F, D)) * 0.02).astype(np.float32)
    oracle.lib()
    t0 = time.perf_counter()
    st = np.zeros((1, F, D), dtype=np.uint8)
    cw, sw = oracle.deosc_update(w[None], 0, st)
    Wq = oracle.dequant_2d(cw[0], sw[0])
    cx, sx = oracle.quantize_1d(x)
    Xq = oracle.dequant_1d(cx, sx)
    y = oracle.gemm_f64(Xq, Wq)                                        # fprop
    cdy, sdy = oracle.quantize_1d(dy, sr=True, sr_seed=1)
    dYq = oracle.dequant_1d(cdy, sdy)
    dx = dYq @ Wq                                                      # dgrad (binary64)
    cxt, sxt = oracle.quantize_1d_transposed(x, rht_d=16, rht_seed=1)
    cdt, sdt = oracle.quantize_1d_transposed(dy, rht_d=16, rht_seed=1, sr=True, sr_seed=1)
    dw = oracle.gemm_f64(oracle.dequant_1d(cdt, sdt), oracle.dequant_1d(cxt, sxt))   # wgrad
    secs = time.perf_counter() - t0
    del y, dx, dw
    flops = 3 * 2.0 * rows * F * D
    return flops / secs / 1e12, secs, oracle.num_threads(), flops


def oracle_timing():
    """A fuller timing report of the oracle (part of the CPU-baseline leg):
    the 1x32 quantisation of the three sweep shapes at full size with every
    host thread, the smallest shape on one thread, the plain binary64 GEMM
    loop on the single layer and on the smallest expert of the MoE layer,
    and the numpy binary64 GEMMs of the layer's fprop (up and down)."""
    import subprocess

    import numpy as np

    import oracle
    from fp4_precision_numerics_b200 import synth
    oracle.lib()
    rep = {"threads": oracle.num_threads(), "host_cores": os.cpu_count()}
    qs = []
    for (R, C) in synth.QUANT_SWEEP_SHAPES:
        x = synth.student_t_activations(R, C, seed=0)
        for sr in (False, True):
            t0 = time.perf_counter()
            oracle.quantize_1d(x, rht_d=16, rht_seed=1, sr=sr, sr_seed=1)
            dt = time.perf_counter() - t0
            qs.append({"shape": [R, C], "sr": sr, "s": round(dt, 3), "gbs": round(R * C * 2.53125 / dt / 1e9, 3)})
        del x
    rep["quantise_all_threads"] = qs
    R, C = synth.QUANT_SWEEP_SHAPES[0]
    code = ("import time, sys; sys.path.insert(0, %r); import oracle; from fp4_precision_numerics_b200 import synth; "
            "x = synth.student_t_activations(%d, %d, seed=0); oracle.lib(); t0 = time.perf_counter(); "
            "oracle.quantize_1d(x, rht_d=16, rht_seed=1, sr=True, sr_seed=1); print(time.perf_counter() - t0)"
            % (ROOT, R, C))
    env = dict(os.environ, OMP_NUM_THREADS="1")
    out = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, check=True)
    dt1 = float(out.stdout.strip().splitlines()[-1])
    rep["quantise_one_thread"] = {"shape": [R, C], "sr": True, "s": round(dt1, 3),
                                  "gbs": round(R * C * 2.53125 / dt1 / 1e9, 3)}
    x, w = synth.single_layer(seed=0)
    A, B = synth.bf16_to_f32(x).astype(np.float64), synth.bf16_to_f32(w).astype(np.float64)
    t0 = time.perf_counter()
    oracle.gemm_f64_loop(A, B)
    dt = time.perf_counter() - t0
    rep["gemm_loop_single_layer"] = {"flop": 2 * 256 ** 3, "s": round(dt, 4), "gflops": round(2 * 256 ** 3 / dt / 1e9, 3)}
    L = synth.moe_layer(with_grads=False)
    off, counts = L["offsets"], L["counts"]
    e = int(np.argmin(counts))
    lo, hi = int(off[e]), int(off[e + 1])
    cx, sx = oracle.quantize_1d(L["x"][lo:hi])
    Xq = oracle.dequant_1d(cx, sx)
    cw, sw = oracle.quantize_2d(L["w_up"][e])
    Wq = oracle.dequant_2d(cw, sw)
    fl = 2.0 * (hi - lo) * Wq.shape[0] * Wq.shape[1]
    t0 = time.perf_counter()
    oracle.gemm_f64_loop(Xq, Wq)
    dt = time.perf_counter() - t0
    rep["gemm_loop_smallest_expert"] = {"expert": e, "rows": hi - lo, "routed_rows": int(counts[e]), "flop": fl,
                                        "s": round(dt, 2), "gflops": round(fl / dt / 1e9, 3)}
    cx, sx = oracle.quantize_1d(L["x"])
    Xq = oracle.dequant_1d(cx, sx)
    ch, sh = oracle.quantize_1d(L["h"])
    Hq = oracle.dequant_1d(ch, sh)
    E = len(counts)
    Wu = np.stack([oracle.dequant_2d(*oracle.quantize_2d(L["w_up"][g])) for g in range(E)])
    Wd = np.stack([oracle.dequant_2d(*oracle.quantize_2d(L["w_down"][g])) for g in range(E)])
    fl = 2.0 * float(counts.sum()) * (Wu.shape[1] * Wu.shape[2] + Wd.shape[1] * Wd.shape[2])
    t0 = time.perf_counter()
    oracle.grouped_gemm_f64(Xq, Wu, off)
    oracle.grouped_gemm_f64(Hq, Wd, off)
    dt = time.perf_counter() - t0
    rep["numpy_fprop_up_down"] = {"flop": fl, "s": round(dt, 2), "tflops": round(fl / dt / 1e12, 4),
                                  "note": "numpy binary64 matmul on dequantised operands; the training step is 3x "
                                          "this work (dgrad and wgrad have the same FLOPs)"}
    return rep


def quant_sweep(iters=20, warmup=3, stream=None):
    """GPU timing of the 1x32 quantiser alone on the quantise-sweep shapes
    (bf16 Gaussian draws on the device -- the kernels' time does not depend
    on the values --, RHT-16, nearest and stochastic rounding):
    median of `iters` CUDA-event timings after `warmup`, with L2 flushed
    (a 256 MB write) before every timed launch and the GPU held by a short
    spin until the launch is queued.  Bytes per element: 2 in,
    1/2 + 1/32 out.  The launch floor is the same measurement on a single
    32 x 32 block (one CTA): what a launch costs with no data to move."""
    import numpy as np
    import torch

    from fp4_precision_numerics_b200 import mxfp4, synth
    peaks = load_peaks()
    dev = torch.device("cuda", torch.cuda.current_device())
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def timed(x, out, sr):
        ts = []
        for i in range(warmup + iters):
            flush.zero_()
            # hold the GPU (a spin of ~0.1 ms) so the launch and both events
            # are queued before the GPU reaches the first event: the interval
            # then holds the kernel alone, not the host's time to launch it
            torch.cuda._sleep(200000)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            mxfp4.quantize(x, rht_seed=1, sr_seed=1 if sr else None, sr_offset=i, scales=True, out=out)
            e1.record()
            torch.cuda.synchronize()
            if i >= warmup:
                ts.append(e0.elapsed_time(e1))
        return float(np.median(ts))

    rows = []
    for (R, C) in synth.QUANT_SWEEP_SHAPES:
        g = torch.Generator(device=dev)
        g.manual_seed(R + C)
        x = torch.randn((R, C), generator=g, device=dev).to(torch.bfloat16)
        out = dict(codes=torch.empty((1, R, C // 2), dtype=torch.uint8, device=dev),
                   scales=torch.empty((1, R, C // 32), dtype=torch.uint8, device=dev))
        for sr in (False, True):
            ms = timed(x, out, sr)
            gbs = R * C * (2 + 0.5 + 1.0 / 32) / (ms / 1e3) / 1e9
            rows.append({"shape": [R, C], "sr": sr, "ms": round(ms, 4), "gbs": round(gbs, 1),
                         "frac_hbm": round(gbs / peaks["hbm_gbs"], 4), "frac_hbm_nominal": round(gbs / NOMINAL_HBM_GBS, 4),
                         "hbm_roof_us": round(R * C * (2 + 0.5 + 1.0 / 32) / (peaks["hbm_gbs"] * 1e9) * 1e6, 2)})
        del x, out
    x = torch.zeros((32, 32), dtype=torch.bfloat16, device=dev)
    out = dict(codes=torch.empty((1, 32, 16), dtype=torch.uint8, device=dev),
               scales=torch.empty((1, 32, 1), dtype=torch.uint8, device=dev))
    floor = {"rn_us": round(1e3 * timed(x, out, False), 2), "sr_us": round(1e3 * timed(x, out, True), 2),
             "what": "one 32x32 block (one CTA), same timing method: the cost of a launch with no data to move"}
    mxfp4.mxfp4_check_device_status()
    return {"quant_sweep": rows, "launch_floor": floor, "l2": "flushed (256 MB write) before every timed launch",
            "iters": iters, "warmup": warmup, "peak_source": peaks["source"] + " copy bandwidth"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    samples = []
    threads = None
    flops = None
    for _ in range(args.warmup):
        cpu_baseline_sample(rows=64)
    t_all = 0.0
    for _ in range(args.steps):
        v, secs, threads, flops = cpu_baseline_sample(rows=64)
        samples.append(v)
        t_all += secs
    value = sum(flops for _ in samples) / t_all / 1e12
    sample = ("oracle on 64 routed rows of expert 0 per step: up-projection fprop/dgrad/wgrad binary64 GEMMs "
              "plus the quantisations they need (5760x2880 W with de-oscillation)")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 * t_all / max(1, args.steps),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD + " (bounded CPU sample)", "l2": "n/a (CPU)"},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


# ---------------------------------------------------------------------------
# Main (our arm)
# ---------------------------------------------------------------------------
def fp4_mma_probe(mx, stream, mmas=16384, launches=10, warmup=3):
    """The tensor pipe alone: the GEMM's own block-scaled MMA (M = 256,
    N = 192, K = 64) issued back to back on operands resident in shared
    memory (`mxfp4_mma_peak_probe`); median TFLOP/s of `launches` launches
    after `warmup`, each timed with CUDA events on `stream`."""
    import torch
    for _ in range(warmup):
        mx.mxfp4_mma_peak_probe(mmas, stream)
    rates = []
    for _ in range(launches):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        flops = mx.mxfp4_mma_peak_probe(mmas, stream)
        e1.record(stream)
        e1.synchronize()
        rates.append(flops / (e0.elapsed_time(e1) / 1e3) / 1e12)
    mx.mxfp4_check_device_status(stream)
    return statistics.median(rates)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=40)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=8)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-quant-sweep", action="store_true",
                    help="skip the quantise-sweep leg after the step measurements")
    ap.add_argument("--quant-sweep", action="store_true",
                    help="time the 1x32 quantiser alone on the quantise-sweep shapes (L2 flushed) and exit")
    ap.add_argument("--oracle-timing", action="store_true",
                    help="print a fuller timing report of the CPU oracle (host only) and exit")
    ap.add_argument("--fused-steps", type=int, default=10,
                    help="steps of each variant (binary32 / fused epilogue) timed interleaved after the main region "
                         "(0: skip)")
    ap.add_argument("--experts", type=int, default=32,
                    help="smaller layers are for profiler captures only; the result line names the size")
    ap.add_argument("--tokens", type=int, default=16384)
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    if args.oracle_timing:
        print(json.dumps({"oracle_timing": oracle_timing()}))
        return 0
    if args.quant_sweep:
        print(json.dumps(quant_sweep()))
        return 0

    import torch
    rank, world, local, pg = dist_setup(args.gpus)
    dev = torch.device("cuda", local)
    peaks = load_peaks()
    layer = Layer(dev, seed=rank, n_experts=args.experts, n_tokens=args.tokens)
    torch.cuda.synchronize()

    stream = torch.cuda.current_stream()
    gpu_uuid = None
    try:
        gpu_uuid = str(torch.cuda.get_device_properties(dev).uuid)
        if not gpu_uuid.startswith("GPU-"):
            gpu_uuid = "GPU-" + gpu_uuid
    except Exception:
        gpu_uuid = str(local)
    # the clock sampler runs from before the warm-up steps, so the GPU does
    # not sit idle (and drop its clocks) between the warm-up and the region
    clocks = ClockSampler(gpu_uuid)
    clocks.start()
    for _ in range(args.warmup):
        layer.step()
    layer.mx.mxfp4_check_device_status()
    torch.cuda.synchronize()

    # per-kernel events over the timed steps
    evs = [{k: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for k in KERNELS}
           for _ in range(args.steps)]
    barrier(pg)
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0 = time.time()
    start.record(stream)
    for i in range(args.steps):
        layer.step(evs[i])
    end.record(stream)
    torch.cuda.synchronize()
    t1 = time.time()
    barrier(pg)
    clocks.stop()
    layer.mx.mxfp4_check_device_status()
    ms_local = start.elapsed_time(end)
    ms = max_over_ranks(ms_local, pg, dev)

    per_kernel = {k: statistics.mean(e[k][0].elapsed_time(e[k][1]) for e in evs) for k in KERNELS}
    step_flops = sum(layer.gemm_flops.values())
    value = step_flops * args.steps * world / (ms / 1e3) / 1e12
    gemm_ms = sum(per_kernel[k] for k in layer.gemm_flops)
    quant_ms = sum(per_kernel[k] for k in layer.quant_bytes)
    quant_gbs = sum(layer.quant_bytes.values()) / (quant_ms / 1e3) / 1e9
    # kernels timed with events inside a sub-second region: the burst bf16
    # peak (x 4, the datasheet's dense FP4:BF16 ratio) is the denominator
    fp4_peak = peaks["bf16_burst"] * NOMINAL_FP4_OVER_BF16
    fp4_sustained = peaks["bf16_sustained"] * NOMINAL_FP4_OVER_BF16
    region_s = ms / 1e3
    dominant = max(per_kernel, key=lambda k: per_kernel[k])
    dom_ms = per_kernel[dominant]
    full_size = (args.experts, args.tokens) == (32, 16384)
    dom_traffic = DRAM_BYTES_FULL.get(dominant) if full_size else None
    if dominant in layer.gemm_flops:
        tensor_src = ("%s burst bf16 x %.0f (nominal FP4:BF16 dense ratio); the kernel is timed with CUDA events "
                      "inside a %.2f s region" % (peaks["source"], NOMINAL_FP4_OVER_BF16, region_s))
        roof = gemm_roofline(layer.gemm_flops[dominant], layer.gemm_out_bytes(dominant), dom_ms, fp4_peak,
                             fp4_sustained, peaks["hbm_gbs"], tensor_src, peaks["source"] + " copy bandwidth")
        roof.update({"kernel": dominant, "traffic": dom_traffic})
    else:
        achieved = layer.quant_bytes[dominant] / (dom_ms / 1e3) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"], "peak_source": peaks["source"] + " copy bandwidth",
                "kernel": dominant, "traffic": dom_traffic,
                "peak_nominal": NOMINAL_HBM_GBS, "frac_nominal": achieved / NOMINAL_HBM_GBS}
    components = {}
    for k in KERNELS:
        t = per_kernel[k]
        if k in layer.gemm_flops:
            tf = layer.gemm_flops[k] / (t / 1e3) / 1e12
            gbs = layer.gemm_out_bytes(k) / (t / 1e3) / 1e9
            components[k] = {"ms": round(t, 4), "tflops": round(tf, 1), "frac_fp4": round(tf / fp4_peak, 4),
                             "alg_gbs": round(gbs, 1), "frac_hbm": round(gbs / peaks["hbm_gbs"], 4)}
        else:
            gbs = layer.quant_bytes[k] / (t / 1e3) / 1e9
            components[k] = {"ms": round(t, 4), "gbs": round(gbs, 1), "frac_hbm": round(gbs / peaks["hbm_gbs"], 4)}
    ck = clocks.summary(t0, t1)

    # ---------------- fused-epilogue variant, interleaved with the binary32 step
    # The same step with fprop/dgrad writing bf16 outputs plus their MXFP4
    # quantisation straight from the accumulator instead of binary32.  The
    # two variants alternate step by step (the order flips every pair) in one
    # region, each step synchronised so the clock samples taken during it are
    # attributed to its variant.
    fused = None
    if args.fused_steps > 0:
        layer.alloc_fused()
        clocks = ClockSampler(gpu_uuid)       # started before this section's warm-up steps
        clocks.start()
        for _ in range(3):
            layer.step()
            layer.step(fused=True)
        layer.mx.mxfp4_check_device_status()
        torch.cuda.synchronize()
        res = {"binary32": {"win": [], "ms": [], "k": []}, "fused": {"win": [], "ms": [], "k": []}}
        for i in range(args.fused_steps):
            order = (("binary32", False), ("fused", True)) if i % 2 == 0 else (("fused", True), ("binary32", False))
            for name, fz in order:
                ev = {k: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for k in KERNELS}
                a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                # a spin of ~1 ms holds the GPU until the whole step is queued,
                # so the host's launch time stays out of the step's interval
                torch.cuda._sleep(2000000)
                w0 = time.time()
                a0.record(stream)
                layer.step(ev, fused=fz)
                a1.record(stream)
                torch.cuda.synchronize()
                res[name]["win"].append((w0, time.time()))
                res[name]["ms"].append(a0.elapsed_time(a1))
                res[name]["k"].append({k: ev[k][0].elapsed_time(ev[k][1]) for k in layer.FUSED})
        clocks.stop()
        layer.mx.mxfp4_check_device_status()

        def kmed(name, k):
            return statistics.median(r[k] for r in res[name]["k"])
        fused = {"steps_each": args.fused_steps, "interleaved": True,
                 "ms_per_step": statistics.median(res["fused"]["ms"]),
                 "ms_per_step_binary32": statistics.median(res["binary32"]["ms"]),
                 "clocks_fused": clocks.summary_windows(res["fused"]["win"]),
                 "clocks_binary32": clocks.summary_windows(res["binary32"]["win"]),
                 "kernels": {k: {"ms": round(kmed("fused", k), 4), "ms_binary32_out": round(kmed("binary32", k), 4),
                                 "tflops": round(layer.gemm_flops[k] / (kmed("fused", k) / 1e3) / 1e12, 1),
                                 "alg_gbs": round(layer.fused_out_bytes(k) / (kmed("fused", k) / 1e3) / 1e9, 1)}
                             for k in layer.FUSED},
                 "what": "medians over steps; each step synchronised; per-step ms from CUDA events around the step"}
        del layer.fused_out

    # ---------------- end to end through the C ABI with host buffers
    # Every step uploads its inputs (X, H, dY_up, dY_down) from pinned host
    # memory and reads every output of the step back (Y_up, Y_down, dX, dH,
    # dW_up, dW_down).  The fp32 master weights and their de-oscillation
    # state persist on the device between steps, as an optimizer keeps them.
    # Two sets of device I/O buffers and three streams let the upload of step
    # i+1, the step-i kernels and the download of step i-1 run at once (PCIe
    # moves both directions concurrently).
    io_in, io_out = ("x", "h", "dy_up", "dy_down"), ("y_up", "y_down", "dx", "dh", "dw_up", "dw_down")
    sets = [{n: getattr(layer, n) for n in io_in + io_out},
            {n: torch.empty_like(getattr(layer, n)) for n in io_in + io_out}]
    for n in io_in:
        sets[1][n].copy_(getattr(layer, n))
    h2d_bytes = sum(sets[0][n].numel() * sets[0][n].element_size() for n in io_in)
    host_in = {n: sets[0][n].cpu().pin_memory() for n in io_in}
    host_out = {n: torch.empty(sets[0][n].shape, dtype=torch.float32).pin_memory() for n in io_out}
    d2h_bytes = sum(t.numel() * t.element_size() for t in host_out.values())
    s_up, s_dn = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    up_done = [torch.cuda.Event(), torch.cuda.Event()]
    comp_done = [torch.cuda.Event(), torch.cuda.Event()]
    dn_done = [torch.cuda.Event(), torch.cuda.Event()]

    def e2e_pipeline(nsteps, e_start=None, e_end=None):
        if e_start is not None:
            e_start.record(s_up)
        for i in range(nsteps):
            b = i % 2
            with torch.cuda.stream(s_up):
                if i >= 2:
                    s_up.wait_event(comp_done[b])          # step i-2 no longer reads buffer set b
                for n in io_in:
                    sets[b][n].copy_(host_in[n], non_blocking=True)
                up_done[b].record(s_up)
            stream.wait_event(up_done[b])
            if i >= 2:
                stream.wait_event(dn_done[b])              # results of step i-2 are on the host
            for n in io_in + io_out:
                setattr(layer, n, sets[b][n])
            layer.step()
            comp_done[b].record(stream)
            with torch.cuda.stream(s_dn):
                s_dn.wait_event(comp_done[b])
                for n in io_out:
                    host_out[n].copy_(sets[b][n], non_blocking=True)
                dn_done[b].record(s_dn)
        if e_end is not None:
            e_end.record(s_dn)

    e2e_pipeline(2)                                          # untimed pass through the pipeline
    torch.cuda.synchronize()
    barrier(pg)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_pipeline(args.e2e_steps, e0, e1)
    torch.cuda.synchronize()
    barrier(pg)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), pg, dev)
    e2e_value = step_flops * args.e2e_steps * world / (e2e_ms / 1e3) / 1e12
    for n in io_in + io_out:
        setattr(layer, n, sets[0][n])
    del sets, host_in, host_out

    # ---------------- quantise sweep (the 1x32 quantiser alone, L2 flushed)
    # and the issue-rate (ALU) roof of the stochastic-rounding kernels
    qs = None
    if not args.no_quant_sweep:
        qs = quant_sweep()
    n_sms = torch.cuda.get_device_properties(dev).multi_processor_count
    mhz = ck["sm_mhz"] or peaks.get("sm_max_mhz", 1965.0)
    alu = {"sm_mhz": mhz, "issue": "%d SMs x %d schedulers x 1 warp instruction per cycle" % (n_sms, SMSP_PER_SM),
           "kernels": {}}
    for k, elems in (("dual_dy_up", layer.M * F), ("dual_dy_down", layer.M * D)):
        ipe = SR_INST_PER_ELEMENT[k]
        hbm_ms = layer.quant_bytes[k] / (peaks["hbm_gbs"] * 1e9) * 1e3
        ent = {"elements": elems, "inst_per_element": ipe, "hbm_ms": round(hbm_ms, 4), "ms": round(per_kernel[k], 4)}
        if ipe is not None:
            alu_ms = issue_roof_ms(ipe, elems, n_sms, mhz)
            ent.update(alu_ms=round(alu_ms, 4), roof_ms=round(max(alu_ms, hbm_ms), 4),
                       frac_roof=round(max(alu_ms, hbm_ms) / per_kernel[k], 4))
        alu["kernels"][k] = ent
    if qs is not None:
        for row in qs["quant_sweep"]:
            if not row["sr"]:
                continue
            R, C = row["shape"]
            ipe = SR_INST_PER_ELEMENT["rows_sr"]
            hbm_ms = row["hbm_roof_us"] / 1e3
            ent = {"elements": R * C, "inst_per_element": ipe, "hbm_ms": round(hbm_ms, 4), "ms": row["ms"]}
            if ipe is not None:
                alu_ms = issue_roof_ms(ipe, R * C, n_sms, mhz)
                ent.update(alu_ms=round(alu_ms, 4), roof_ms=round(max(alu_ms, hbm_ms), 4),
                           frac_roof=round(max(alu_ms, hbm_ms) / row["ms"], 4))
            alu["kernels"]["quantise_sr_%dx%d" % (R, C)] = ent

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, secs, threads, _ = cpu_baseline_sample(rows=CPU_SAMPLE_ROWS)
        cpu = {"value": v, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
               "sample": "%d routed rows of expert 0: up-projection fprop/dgrad/wgrad binary64 GEMMs plus their "
                         % CPU_SAMPLE_ROWS +
                         "quantisations (2D de-oscillation W, SR dY, RHT-16 transposed operands); %.1f s on %d "
                         "threads of %d host cores" % (secs, threads, os.cpu_count() or 0)}
    probe = fp4_mma_probe(layer.mx, stream)
    if "tflops" in roof:
        roof["peak_probe"] = probe
        roof["frac_tensor_probe"] = roof["tflops"] / probe
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "e2m1+ue8m0 (fp32 accumulate)", "data": "synthetic",
        "config": {"workload": WORKLOAD if (args.experts, args.tokens) == (32, 16384) else
                   "reduced MoE layer for profiling: %d experts, %d tokens" % (args.experts, args.tokens),
                   "tokens": args.tokens, "routed_rows": layer.rows_real, "padded_rows": layer.M,
                   "experts": E, "parallelism": "replica per GPU" if world > 1 else "single GPU",
                   "l2": "inputs larger than L2 (working set ~14 GB per step)"},
        "quantise_gbs": quant_gbs, "quantise_frac_hbm": quant_gbs / peaks["hbm_gbs"],
        "quantise_frac_hbm_nominal": quant_gbs / NOMINAL_HBM_GBS,
        "gemm_frac_fp4_nominal": step_flops / (gemm_ms / 1e3) / 1e12 / NOMINAL_FP4_TFLOPS,
        "gemm_tflops": step_flops / (gemm_ms / 1e3) / 1e12, "gemm_frac_fp4": step_flops / (gemm_ms / 1e3) / 1e12 / fp4_peak,
        "fp4_mma_probe": {"tflops": probe, "mmas_per_pair": 16384, "launches": 10,
                          "what": "the GEMM's block-scaled MMA alone on resident operands, after the timed region"},
        "gemm_frac_fp4_probe": step_flops / (gemm_ms / 1e3) / 1e12 / probe,
        "roofline": roof, "components": components,
        "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": int(h2d_bytes),
                "d2h_bytes_per_step": int(d2h_bytes), "steps": args.e2e_steps,
                "what": "inputs X, H, dY_up, dY_down uploaded and every output (Y_up, Y_down, dX, dH, dW_up, dW_down) "
                        "read back each step; masters and de-oscillation state resident"},
        "gpu_launches": layer.launches_per_step * args.steps,
        "clocks": {"sm_mhz": ck["sm_mhz"], "sm_max_mhz": ck["sm_max_mhz"], "sm_mhz_min": ck.get("sm_mhz_min"),
                   "reasons": ck["reasons"], "samples": ck["samples"]},
        "cpu_baseline": cpu,
        "fused_epilogue": fused,
        "quantise_sweep": qs,
        "sr_alu_roof": alu,
    }
    if rank == 0:
        print(json.dumps(line))
    if pg is not None:
        pg.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())

"""Operator-level signal-to-noise report of the MXFP4 path on synthetic data.

The pages report operator-level SNR only qualitatively (for techniques they
rejected); this report measures the same kind of quantity for the recipe's
own operators, through the library's kernels:

  - config 1, single layer (X, W 256x256 with 1% x20 outliers): SNR of
    Y = deq(Q(X)) deq(Q(W))^T against the binary64 X W^T, for nearest and
    stochastic rounding of X, with and without the RHT-16 (applied to both
    operands, so it cancels in the product);
  - config 2, activation sweep (Student-t, 4096 x 2880): SNR of the
    dequantised tensor against the input (in the RHT domain when the RHT is
    on; the transform is orthogonal, so the numbers compare);
  - config 3, MoE up-projection fprop on the first experts: SNR of the
    grouped GEMM output against binary64;
  - de-oscillation: over steps of small updates to fp32 masters with weights
    near bin boundaries, the SNR of the emitted weights against the masters
    and the fraction of codes that change per step, with the pass on and off.

SNR = 10 log10(sum ref^2 / sum (out - ref)^2).

    python -m fp4_precision_numerics_b200.snr [--small]
"""
from __future__ import annotations

import argparse

import numpy as np
import torch

from fp4_precision_numerics_b200 import mxfp4, synth

_GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0, -0.0, -0.5, -1.0, -1.5, -2.0, -3.0, -4.0, -6.0])


def snr_db(ref: np.ndarray, out: np.ndarray) -> float:
    ref = np.asarray(ref, dtype=np.float64)
    err = np.asarray(out, dtype=np.float64) - ref
    return float(10.0 * np.log10(np.sum(ref * ref) / max(np.sum(err * err), 1e-300)))


def _decode(codes: np.ndarray, scales: np.ndarray, block_rows: int = 1) -> np.ndarray:
    """Packed E2M1 codes [R, C/2] and UE8M0 scales ([R, C/32], or [R/32, C/32]
    for 2D blocks with block_rows = 32) -> binary64 values [R, C]."""
    lo, hi = codes & 0x0F, codes >> 4
    c = np.stack([lo, hi], axis=-1).reshape(codes.shape[0], -1)
    s = np.repeat(np.repeat(scales.astype(np.int64) - 127, 32, axis=1), block_rows, axis=0)
    return np.ldexp(_GRID[c], s)


def _bf16_dev(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _gemm_snr(x_bits, w_bits, rht: bool, sr: bool) -> float:
    xd, wd = _bf16_dev(x_bits), _bf16_dev(w_bits)
    seed = 1 if rht else None
    qx = mxfp4.quantize(xd, rht_seed=seed, sr_seed=1 if sr else None, scales=False, scales_mma=True)
    qw = mxfp4.quantize(wd, block="32x32", rht_seed=seed, scales=False, scales_mma=True)
    M, K = x_bits.shape
    N = w_bits.shape[0]
    offs = torch.tensor([0, M], dtype=torch.int32, device="cuda")
    y = mxfp4.grouped_gemm(mxfp4.GEMM_FPROP, offs, qx["codes"], qx["scales_mma"], qw["codes"], qw["scales_mma"],
                           M, N, K).cpu().numpy()
    ref = synth.bf16_to_f32(x_bits).astype(np.float64) @ synth.bf16_to_f32(w_bits).astype(np.float64).T
    return snr_db(ref, y)


def config1() -> dict:
    x, w = synth.single_layer(seed=0)
    return {(r, s): _gemm_snr(x, w, r, s) for r in (False, True) for s in (False, True)}


def config2(rows: int = 4096, cols: int = 2880) -> dict:
    x = synth.student_t_activations(rows, cols, seed=0)
    xd = _bf16_dev(x)
    out = {}
    for rht in (False, True):
        ref = mxfp4.rht(xd, seed=1).cpu().numpy() if rht else synth.bf16_to_f32(x)
        for sr in (False, True):
            q = mxfp4.quantize(xd, rht_seed=1 if rht else None, sr_seed=1 if sr else None, scales=True)
            out[(rht, sr)] = snr_db(ref, _decode(q["codes"][0].cpu().numpy(), q["scales"][0].cpu().numpy()))
    return out


def config3(n_experts: int = 4) -> dict:
    L = synth.moe_layer()
    off = L["offsets"]
    rows = int(off[n_experts])
    x, w = L["x"][:rows], L["w_up"][:n_experts]
    out = {}
    for rht in (False, True):
        for sr in (False, True):
            seed = 1 if rht else None
            qx = mxfp4.quantize(_bf16_dev(x), rht_seed=seed, sr_seed=1 if sr else None, scales=False,
                                scales_mma=True)
            qw = mxfp4.quantize(_bf16_dev(w), block="32x32", rht_seed=seed, scales=False, scales_mma=True)
            offs = torch.tensor(off[:n_experts + 1].astype(np.int32), device="cuda")
            F, D = w.shape[1], w.shape[2]
            y = mxfp4.grouped_gemm(mxfp4.GEMM_FPROP, offs, qx["codes"], qx["scales_mma"], qw["codes"],
                                   qw["scales_mma"], rows, F, D).cpu().numpy()
            xf = synth.bf16_to_f32(x).astype(np.float64)
            wf = synth.bf16_to_f32(w).astype(np.float64)
            ref = np.concatenate([xf[off[e]:off[e + 1]] @ wf[e].T for e in range(n_experts)])
            out[(rht, sr)] = snr_db(ref, y)
    return out


def deosc(steps: int = 30, groups: int = 2, rows: int = 256, cols: int = 512) -> dict:
    out = {}
    for on in (False, True):
        w = synth.deosc_master(groups=groups, rows=rows, cols=cols, seed=5)
        wd = torch.from_numpy(w).cuda()
        st = torch.zeros(w.shape, dtype=torch.uint8, device="cuda")
        prev, snrs, flips = None, [], []
        for t in range(steps):
            if t:
                w = (w + synth.deosc_update_noise(w.shape, t, std=2e-4)).astype(np.float32)
                wd.copy_(torch.from_numpy(w))
            if on:
                q = mxfp4.deosc_update(wd, t, st, flip_threshold=4, scales=True)
            else:
                q = mxfp4.quantize(wd, block="32x32", scales=True)
            codes = q["codes"].cpu().numpy()
            deq = np.stack([_decode(codes[g], q["scales"][g].cpu().numpy(), 32) for g in range(groups)])
            snrs.append(snr_db(w, deq))
            if prev is not None:
                flips.append(float(np.mean(((codes ^ prev) & 0x0F) != 0) + np.mean(((codes ^ prev) >> 4) != 0)) / 2)
            prev = codes
        out[on] = (float(np.mean(snrs)), float(np.mean(flips)))
    return out


def report(small: bool = False) -> str:
    c1 = config1()
    c2 = config2(*((1024, 2880) if small else (4096, 2880)))
    c3 = config3(2 if small else 4)
    d = deosc(steps=12 if small else 30)
    lines = ["| operator | RN | SR | RN + RHT | SR + RHT |", "|---|---|---|---|---|"]
    for name, c in (("config 1: single-layer GEMM output", c1), ("config 2: 1x32 quantised activations", c2),
                    ("config 3: MoE up-projection fprop output", c3)):
        lines.append("| %s | %.2f dB | %.2f dB | %.2f dB | %.2f dB |" % (
            name, c[(False, False)], c[(False, True)], c[(True, False)], c[(True, True)]))
    lines += ["", "| 2D weight re-quantisation over %d steps | mean SNR vs masters | codes changing per step |"
              % (12 if small else 30), "|---|---|---|",
              "| de-oscillation off | %.2f dB | %.4f%% |" % (d[False][0], 100 * d[False][1]),
              "| de-oscillation on (threshold 4) | %.2f dB | %.4f%% |" % (d[True][0], 100 * d[True][1])]
    return "\n".join(lines)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--small", action="store_true")
    args = ap.parse_args()
    print(report(small=args.small))


if __name__ == "__main__":
    main()

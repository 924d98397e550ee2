"""Test-side helpers: host <-> device marshalling and layout unpacking.

Written independently of the CUDA kernels: the tensor-core scale layout is
decoded here from its definition in include/mxfp4.h."""
import numpy as np
import torch

import oracle


def dev_bf16(bits: np.ndarray) -> torch.Tensor:
    """uint16 bf16 bit patterns -> CUDA bfloat16 tensor (same bits)."""
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def dev_f32(x: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).cuda()


def host(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy()


def mma_scales_to_rows(buf: np.ndarray, R: int, S: int) -> np.ndarray:
    """Decode a tensor-core scale buffer into the [R, S] per-row scale matrix:
    byte of (r, s) at ((r/128)*ceil(S/4) + s/4)*512 + (r%32)*16 + ((r/32)%4)*4 + s%4."""
    buf = np.asarray(buf).reshape(-1)
    r = np.arange(R)[:, None]
    s = np.arange(S)[None, :]
    nchunk = (S + 3) // 4
    off = ((r // 128) * nchunk + s // 4) * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4 + s % 4
    return buf[off]


def nibbles(codes: np.ndarray) -> np.ndarray:
    codes = np.asarray(codes)
    lo = codes & 0x0F
    hi = codes >> 4
    return np.stack([lo, hi], axis=-1).reshape(*codes.shape[:-1], codes.shape[-1] * 2)


def gemm_errors(y: np.ndarray, y_ref: np.ndarray, abs_prod: np.ndarray):
    """(componentwise max |y - ref| / (|A||B|^T), normwise max|dy| / max|ref|)."""
    d = np.abs(y.astype(np.float64) - y_ref)
    denom = abs_prod + 1e-300
    comp = float(np.max(np.where(abs_prod > 0, d / denom, np.where(d > 0, np.inf, 0.0))))
    norm = float(d.max() / max(np.abs(y_ref).max(), 1e-300))
    return comp, norm


def oracle_operand_1d(x_bits, **kw):
    """Oracle quantisation of an activation/gradient (1x32 along the last
    dim) and its binary64 dequantisation."""
    c, s = oracle.quantize_1d(x_bits, **kw)
    return c, s, oracle.dequant_1d(c, s)

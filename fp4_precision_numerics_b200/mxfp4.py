"""Thin Python binding of libmxfp4 (C ABI in include/mxfp4.h).

Argument marshalling only: every step of the path runs in the library's
sm_100a kernels.  PyTorch supplies device memory and the current CUDA stream.
There is no fallback: if the shared library is missing or fails to load, the
first call raises.

Raw entry points keep the C names (``mxfp4_quantize``, ``mxfp4_rht``,
``mxfp4_deosc_update``, ``mxfp4_grouped_gemm``, ...).  The lower-case helpers
(``quantize``, ``rht``, ``deosc_update``, ``grouped_gemm``) allocate outputs
with torch and call the raw entry points.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmxfp4.so")

MXFP4_OK = 0
STATUS_NAMES = {0: "OK", -1: "INVALID_ARG", -2: "UNSUPPORTED_SHAPE", -3: "MISALIGNED", -4: "CUDA_ERROR",
                -5: "DEVICE_TIMEOUT", -6: "DEVICE_BAD_INPUT"}
DTYPE_BF16, DTYPE_F32 = 0, 1
BLOCK_1X32, BLOCK_32X32 = 0, 1
ROUND_NEAREST, ROUND_STOCHASTIC = 0, 1
GEMM_FPROP, GEMM_DGRAD, GEMM_WGRAD = 0, 1, 2


class QuantParams(ctypes.Structure):
    _fields_ = [("block", ctypes.c_int), ("along_rows", ctypes.c_int), ("rht_d", ctypes.c_int),
                ("rht_seed", ctypes.c_uint64), ("rounding", ctypes.c_int), ("sr_seed", ctypes.c_uint64),
                ("sr_offset", ctypes.c_uint32)]


class QuantOutputs(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("scales_mma", ctypes.c_void_p),
                ("codes_t", ctypes.c_void_p), ("scales_mma_t", ctypes.c_void_p)]


class DeoscParams(ctypes.Structure):
    _fields_ = [("flip_threshold", ctypes.c_uint32), ("reset_period", ctypes.c_uint32),
                ("freeze_lower", ctypes.c_uint32)]


class Operand(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("scales_mma", ctypes.c_void_p)]


class MXFP4Error(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__("%s (%d): %s" % (STATUS_NAMES.get(status, "?"), status, message))
        self.status = status


_lib = None
_lock = threading.Lock()


def lib() -> ctypes.CDLL:
    """Load libmxfp4.so (raises if it is absent: there is no fallback)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError("libmxfp4.so not built (%s); run python -m fp4_precision_numerics_b200.build"
                                   % LIB_PATH)
            L = ctypes.CDLL(LIB_PATH)
            vp, i64, st = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
            L.mxfp4_quantize.argtypes = [vp, st, i64, i64, i64, i64, ctypes.POINTER(QuantParams),
                                         ctypes.POINTER(QuantOutputs), vp]
            L.mxfp4_quantize.restype = st
            L.mxfp4_quantize_dual.argtypes = [vp, st, i64, i64, i64, i64, ctypes.POINTER(QuantParams),
                                              ctypes.POINTER(QuantParams), ctypes.POINTER(QuantOutputs),
                                              ctypes.POINTER(QuantOutputs), vp]
            L.mxfp4_quantize_dual.restype = st
            L.mxfp4_rht.argtypes = [vp, st, i64, i64, i64, st, st, ctypes.c_uint64, vp, st, vp]
            L.mxfp4_rht.restype = st
            L.mxfp4_deosc_update.argtypes = [vp, i64, i64, i64, ctypes.c_uint32, ctypes.POINTER(DeoscParams), vp,
                                             ctypes.POINTER(QuantOutputs), vp]
            L.mxfp4_deosc_update.restype = st
            L.mxfp4_grouped_gemm.argtypes = [st, st, vp, Operand, Operand, i64, i64, i64, vp, i64, vp]
            L.mxfp4_grouped_gemm.restype = st
            L.mxfp4_grouped_gemm_fused.argtypes = [st, st, vp, Operand, Operand, i64, i64, i64, vp, i64,
                                                   ctypes.POINTER(QuantOutputs), ctypes.POINTER(QuantParams), vp]
            L.mxfp4_grouped_gemm_fused.restype = st
            L.mxfp4_mma_peak_probe.argtypes = [i64, ctypes.POINTER(ctypes.c_double), vp]
            L.mxfp4_mma_peak_probe.restype = st
            L.mxfp4_selftest_wait_timeout.argtypes = [vp]
            L.mxfp4_selftest_wait_timeout.restype = st
            L.mxfp4_mma_scale_bytes.argtypes = [i64, i64]
            L.mxfp4_mma_scale_bytes.restype = ctypes.c_size_t
            L.mxfp4_last_error.argtypes = [ctypes.c_char_p, ctypes.c_size_t]
            L.mxfp4_last_error.restype = ctypes.c_size_t
            L.mxfp4_check_device_status.argtypes = [vp]
            L.mxfp4_check_device_status.restype = st
            L.mxfp4_version.restype = ctypes.c_char_p
            _lib = L
    return _lib


def last_error() -> str:
    buf = ctypes.create_string_buffer(1024)
    lib().mxfp4_last_error(buf, len(buf))
    return buf.value.decode(errors="replace")


def _check(status: int):
    if status != MXFP4_OK:
        raise MXFP4Error(status, last_error())


def _stream(stream=None) -> ctypes.c_void_p:
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t) -> ctypes.c_void_p:
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return DTYPE_BF16
    if t.dtype == torch.float32:
        return DTYPE_F32
    raise TypeError("expected bfloat16 or float32, got %s" % t.dtype)


# ---------------------------------------------------------------------------
# Raw entry points (same names as the C ABI)
# ---------------------------------------------------------------------------
def mxfp4_mma_scale_bytes(rows: int, nscales: int) -> int:
    return int(lib().mxfp4_mma_scale_bytes(rows, nscales))


def mxfp4_quantize(x_ptr, in_dtype, groups, rows, cols, ld, params: QuantParams, outputs: QuantOutputs,
                   stream=None):
    _check(lib().mxfp4_quantize(x_ptr, in_dtype, groups, rows, cols, ld, ctypes.byref(params),
                                ctypes.byref(outputs), _stream(stream)))


def mxfp4_quantize_dual(x_ptr, in_dtype, groups, rows, cols, ld, row_params: QuantParams, col_params: QuantParams,
                        row_outputs: QuantOutputs, col_outputs: QuantOutputs, stream=None):
    _check(lib().mxfp4_quantize_dual(x_ptr, in_dtype, groups, rows, cols, ld, ctypes.byref(row_params),
                                     ctypes.byref(col_params), ctypes.byref(row_outputs), ctypes.byref(col_outputs),
                                     _stream(stream)))


def mxfp4_rht(x_ptr, in_dtype, rows, cols, ld, axis, d, seed, out_ptr, out_dtype, stream=None):
    _check(lib().mxfp4_rht(x_ptr, in_dtype, rows, cols, ld, axis, d, seed, out_ptr, out_dtype, _stream(stream)))


def mxfp4_deosc_update(master_ptr, groups, rows, cols, step, params: DeoscParams, state_ptr,
                       outputs: QuantOutputs, stream=None):
    _check(lib().mxfp4_deosc_update(master_ptr, groups, rows, cols, step, ctypes.byref(params), state_ptr,
                                    ctypes.byref(outputs), _stream(stream)))


def mxfp4_grouped_gemm(op, num_groups, offsets_ptr, a: Operand, b: Operand, M, N, K, out_ptr, ldo, stream=None):
    _check(lib().mxfp4_grouped_gemm(op, num_groups, offsets_ptr, a, b, M, N, K, out_ptr, ldo, _stream(stream)))


def mxfp4_grouped_gemm_fused(op, num_groups, offsets_ptr, a: Operand, b: Operand, M, N, K, y_ptr, ldy,
                             q: QuantOutputs, qp: QuantParams | None = None, stream=None):
    _check(lib().mxfp4_grouped_gemm_fused(op, num_groups, offsets_ptr, a, b, M, N, K, y_ptr, ldy, ctypes.byref(q),
                                          ctypes.byref(qp) if qp is not None else None, _stream(stream)))


def mxfp4_mma_peak_probe(mmas_per_pair: int, stream=None) -> float:
    """Launch the tensor-pipe peak probe on `stream`; returns the launch's
    floating-point operations (the caller times the launch)."""
    flops = ctypes.c_double(0.0)
    _check(lib().mxfp4_mma_peak_probe(int(mmas_per_pair), ctypes.byref(flops), _stream(stream)))
    return flops.value


def mxfp4_selftest_wait_timeout(stream=None):
    """Launch the failure-detection self-test (a bounded wait that expires
    after about 2 s); read its result with mxfp4_check_device_status."""
    _check(lib().mxfp4_selftest_wait_timeout(_stream(stream)))


def mxfp4_check_device_status(stream=None):
    _check(lib().mxfp4_check_device_status(_stream(stream)))


def version() -> str:
    return lib().mxfp4_version().decode()


# ---------------------------------------------------------------------------
# Tensor helpers
# ---------------------------------------------------------------------------
def _require(cond: bool, msg: str) -> None:
    """Argument checks of the tensor helpers.  They raise (and survive
    `python -O`): a wrong dtype, layout or size would otherwise reach the
    library as a pointer and become an out-of-bounds device access."""
    if not cond:
        raise ValueError(msg)


def _check_buf(t, nbytes: int, name: str, dtype=torch.uint8) -> None:
    """`t` is a contiguous CUDA tensor of `dtype` holding at least `nbytes`."""
    _require(isinstance(t, torch.Tensor) and t.is_cuda and t.dtype == dtype and t.is_contiguous(),
             "%s: a contiguous CUDA %s tensor is required" % (name, dtype))
    have = t.numel() * t.element_size()
    _require(have >= nbytes, "%s: %d bytes, at least %d required" % (name, have, nbytes))


def _check_input(x: torch.Tensor, name: str = "x") -> torch.Tensor:
    if isinstance(x, torch.Tensor) and x.dim() == 2:
        x = x.unsqueeze(0)
    _require(isinstance(x, torch.Tensor) and x.is_cuda and x.dim() == 3 and x.stride(2) == 1,
             "%s: a [rows, cols] or [groups, rows, cols] CUDA tensor with unit column stride is required" % name)
    _require(x.dtype in (torch.bfloat16, torch.float32), "%s: bf16 or float32 required" % name)
    _require(x.shape[0] == 1 or x.stride(0) == x.shape[1] * x.stride(1), "%s: groups must be back to back" % name)
    return x


def _check_offsets(offsets) -> None:
    _require(isinstance(offsets, torch.Tensor) and offsets.is_cuda and offsets.dtype == torch.int32
             and offsets.dim() == 1 and offsets.is_contiguous() and offsets.numel() >= 1,
             "offsets: a contiguous 1D int32 CUDA tensor of G + 1 entries")


def _check_quant_outputs(o: dict, G: int, Ro: int, Co: int, two_d: bool, R: int, C: int) -> None:
    """Sizes of a quantiser's output buffers (those present in `o`): codes
    [G, Ro, Co/2]; scales [G, Ro, Co/32] (2D: [G, R/32, C/32]); tensor-core
    scales per group; for 2D the transpose's codes [G, C, R/2] and scales."""
    _check_buf(o["codes"], G * Ro * (Co // 2), "codes")
    if o.get("scales") is not None:
        _check_buf(o["scales"], G * ((R // 32) * (C // 32) if two_d else Ro * (Co // 32)), "scales")
    if o.get("scales_mma") is not None:
        _check_buf(o["scales_mma"], G * mxfp4_mma_scale_bytes(Ro, Co // 32), "scales_mma")
    if o.get("codes_t") is not None:
        _check_buf(o["codes_t"], G * C * (R // 2), "codes_t")
    if o.get("scales_mma_t") is not None:
        _check_buf(o["scales_mma_t"], G * mxfp4_mma_scale_bytes(C, R // 32), "scales_mma_t")


def _check_operands(op: int, G: int, M: int, N: int, K: int, a_codes, a_scales, b_codes, b_scales) -> None:
    """Sizes of the GEMM operands as include/mxfp4.h lays them out."""
    _check_buf(a_codes, M * K // 2, "a_codes")
    _check_buf(a_scales, mxfp4_mma_scale_bytes(M, K // 32), "a_scales_mma")
    groups_b = 1 if op == GEMM_WGRAD else G
    _check_buf(b_codes, groups_b * N * K // 2, "b_codes")
    _check_buf(b_scales, groups_b * mxfp4_mma_scale_bytes(N, K // 32), "b_scales_mma")


def quantize(x: torch.Tensor, block: str = "1x32", along_rows: bool = False, rht_seed=None, sr_seed=None,
             sr_offset: int = 0, scales: bool = True, scales_mma: bool = False, transposed: bool = False,
             out: dict | None = None, stream=None) -> dict:
    """Quantise a [rows, cols] or [groups, rows, cols] bf16/f32 CUDA tensor.

    Returns a dict with 'codes', and as requested 'scales' (canonical),
    'scales_mma', 'codes_t' and 'scales_mma_t' (2D: the transpose's codes
    and tensor-core scales).  `out` may supply preallocated tensors."""
    x = _check_input(x)
    G, R, C = x.shape
    ld = x.stride(1)
    two_d = block == "32x32"
    p = QuantParams(BLOCK_32X32 if two_d else BLOCK_1X32, int(bool(along_rows) and not two_d),
                    16 if rht_seed is not None else 0, int(rht_seed or 0),
                    ROUND_STOCHASTIC if sr_seed is not None else ROUND_NEAREST, int(sr_seed or 0), int(sr_offset))
    Ro, Co = (C, R) if (along_rows and not two_d) else (R, C)
    o = dict(out or {})
    dev = x.device
    if "codes" not in o:
        o["codes"] = torch.empty((G, Ro, Co // 2), dtype=torch.uint8, device=dev)
    if scales and "scales" not in o:
        shape = (G, R // 32, C // 32) if two_d else (G, Ro, Co // 32)
        o["scales"] = torch.empty(shape, dtype=torch.uint8, device=dev)
    if scales_mma and "scales_mma" not in o:
        o["scales_mma"] = torch.empty((G, mxfp4_mma_scale_bytes(Ro, Co // 32)), dtype=torch.uint8, device=dev)
    if transposed and two_d:
        if "codes_t" not in o:
            o["codes_t"] = torch.empty((G, C, R // 2), dtype=torch.uint8, device=dev)
        if scales_mma and "scales_mma_t" not in o:
            o["scales_mma_t"] = torch.empty((G, mxfp4_mma_scale_bytes(C, R // 32)), dtype=torch.uint8, device=dev)
    _check_quant_outputs(o, G, Ro, Co, two_d, R, C)
    outs = QuantOutputs(o["codes"].data_ptr(), _ptr(o.get("scales")), _ptr(o.get("scales_mma")),
                        _ptr(o.get("codes_t")), _ptr(o.get("scales_mma_t")))
    mxfp4_quantize(ctypes.c_void_p(x.data_ptr()), _dtype_code(x), G, R, C, ld, p, outs, stream)
    return o


def quantize_dual(x: torch.Tensor, row_rht_seed=None, col_rht_seed=None, sr_seed=None, row_sr_offset: int = 0,
                  col_sr_offset: int = 0, scales: bool = True, scales_mma: bool = False, out_row: dict | None = None,
                  out_col: dict | None = None, stream=None) -> tuple:
    """Quantise a [rows, cols] or [groups, rows, cols] bf16/f32 CUDA tensor
    in both 1D directions from one read: returns (row, col), the outputs of
    quantize(x, ...) along the last dim and quantize(x, along_rows=True, ...),
    each a dict like quantize's."""
    x = _check_input(x)
    G, R, C = x.shape
    rounding = ROUND_STOCHASTIC if sr_seed is not None else ROUND_NEAREST
    rp = QuantParams(BLOCK_1X32, 0, 16 if row_rht_seed is not None else 0, int(row_rht_seed or 0), rounding,
                     int(sr_seed or 0), int(row_sr_offset))
    cp = QuantParams(BLOCK_1X32, 1, 16 if col_rht_seed is not None else 0, int(col_rht_seed or 0), rounding,
                     int(sr_seed or 0), int(col_sr_offset))
    dev = x.device
    outs = []
    for (o, Ro, Co) in ((dict(out_row or {}), R, C), (dict(out_col or {}), C, R)):
        if "codes" not in o:
            o["codes"] = torch.empty((G, Ro, Co // 2), dtype=torch.uint8, device=dev)
        if scales and "scales" not in o:
            o["scales"] = torch.empty((G, Ro, Co // 32), dtype=torch.uint8, device=dev)
        if scales_mma and "scales_mma" not in o:
            o["scales_mma"] = torch.empty((G, mxfp4_mma_scale_bytes(Ro, Co // 32)), dtype=torch.uint8, device=dev)
        _check_quant_outputs(o, G, Ro, Co, False, R, C)
        outs.append(o)
    ro, co = outs
    qo_r = QuantOutputs(ro["codes"].data_ptr(), _ptr(ro.get("scales")), _ptr(ro.get("scales_mma")), None, None)
    qo_c = QuantOutputs(co["codes"].data_ptr(), _ptr(co.get("scales")), _ptr(co.get("scales_mma")), None, None)
    mxfp4_quantize_dual(ctypes.c_void_p(x.data_ptr()), _dtype_code(x), G, R, C, x.stride(1), rp, cp, qo_r, qo_c,
                        stream)
    return ro, co


def rht(x: torch.Tensor, seed: int, out_dtype=torch.float32, axis: int = 1, stream=None) -> torch.Tensor:
    """RHT-16 of a 2D tensor along the last dim (axis 1) or along dim 0
    (axis 0); the output keeps x's shape."""
    _require(isinstance(x, torch.Tensor) and x.is_cuda and x.dim() == 2 and x.stride(1) == 1
             and x.dtype in (torch.bfloat16, torch.float32), "x: a 2D bf16/float32 CUDA tensor with unit column stride")
    _require(axis in (0, 1), "axis: 0 or 1")
    R, C = x.shape
    y = torch.empty((R, C), dtype=out_dtype, device=x.device)
    mxfp4_rht(ctypes.c_void_p(x.data_ptr()), _dtype_code(x), R, C, x.stride(0), int(axis), 16, int(seed),
              ctypes.c_void_p(y.data_ptr()), _dtype_code(y), stream)
    return y


def deosc_update(master: torch.Tensor, step: int, state: torch.Tensor, flip_threshold: int = 4,
                 reset_period: int = 0, scales: bool = True, scales_mma: bool = False, transposed: bool = False,
                 out: dict | None = None, stream=None, freeze_lower: bool = False) -> dict:
    if isinstance(master, torch.Tensor) and master.dim() == 2:
        master = master.unsqueeze(0)
    _require(isinstance(master, torch.Tensor) and master.is_cuda and master.dtype == torch.float32
             and master.dim() == 3 and master.is_contiguous(), "master: a contiguous float32 CUDA tensor")
    _check_buf(state, master.numel(), "state")
    _require(state.numel() == master.numel(), "state: one byte per weight")
    G, R, C = master.shape
    o = dict(out or {})
    dev = master.device
    if "codes" not in o:
        o["codes"] = torch.empty((G, R, C // 2), dtype=torch.uint8, device=dev)
    if scales and "scales" not in o:
        o["scales"] = torch.empty((G, R // 32, C // 32), dtype=torch.uint8, device=dev)
    if scales_mma and "scales_mma" not in o:
        o["scales_mma"] = torch.empty((G, mxfp4_mma_scale_bytes(R, C // 32)), dtype=torch.uint8, device=dev)
    if transposed:
        if "codes_t" not in o:
            o["codes_t"] = torch.empty((G, C, R // 2), dtype=torch.uint8, device=dev)
        if scales_mma and "scales_mma_t" not in o:
            o["scales_mma_t"] = torch.empty((G, mxfp4_mma_scale_bytes(C, R // 32)), dtype=torch.uint8, device=dev)
    _check_quant_outputs(o, G, R, C, True, R, C)
    outs = QuantOutputs(o["codes"].data_ptr(), _ptr(o.get("scales")), _ptr(o.get("scales_mma")),
                        _ptr(o.get("codes_t")), _ptr(o.get("scales_mma_t")))
    mxfp4_deosc_update(ctypes.c_void_p(master.data_ptr()), G, R, C, int(step),
                       DeoscParams(int(flip_threshold), int(reset_period), int(bool(freeze_lower))),
                       ctypes.c_void_p(state.data_ptr()), outs,
                       stream)
    return o


def grouped_gemm(op: int, offsets: torch.Tensor, a_codes, a_scales_mma, b_codes, b_scales_mma, M: int, N: int,
                 K: int, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """FPROP/DGRAD: out [M, N]; WGRAD: out [G, M, N] (see include/mxfp4.h)."""
    _check_offsets(offsets)
    G = offsets.numel() - 1
    if out is None:
        shape = (G, M, N) if op == GEMM_WGRAD else (M, N)
        out = torch.empty(shape, dtype=torch.float32, device=offsets.device)
    _require(isinstance(out, torch.Tensor) and out.is_cuda and out.dtype == torch.float32 and out.stride(-1) == 1,
             "out: a float32 CUDA tensor with unit column stride")
    ldo = out.stride(-2)
    if op == GEMM_WGRAD:
        _require(out.dim() == 3 and out.shape[0] >= G and out.shape[1] == M and out.shape[2] >= N
                 and (G <= 1 or out.stride(0) == M * ldo), "out: [G, M, >= N] with group stride M * row stride")
    else:
        _require(out.dim() == 2 and out.shape[0] >= M and out.shape[1] >= N, "out: [>= M, >= N]")
    _check_operands(op, G, M, N, K, a_codes, a_scales_mma, b_codes, b_scales_mma)
    mxfp4_grouped_gemm(op, G, ctypes.c_void_p(offsets.data_ptr()),
                       Operand(a_codes.data_ptr(), a_scales_mma.data_ptr()),
                       Operand(b_codes.data_ptr(), b_scales_mma.data_ptr()), M, N, K,
                       ctypes.c_void_p(out.data_ptr()), ldo, stream)
    return out


def grouped_gemm_fused(op: int, offsets: torch.Tensor, a_codes, a_scales_mma, b_codes, b_scales_mma, M: int, N: int,
                       K: int, scales: bool = True, scales_mma: bool = True, y: torch.Tensor | None = None,
                       out: dict | None = None, sr_seed=None, sr_offset: int = 0, stream=None) -> tuple:
    """FPROP/DGRAD with the fused epilogue: returns (y, q) with y the [M, N]
    bf16 output and q the dict ('codes', 'scales', 'scales_mma') of its
    1x32-along-N MXFP4 quantisation, nearest rounding or, with sr_seed,
    stochastic rounding as quantize(y, sr_seed=..., sr_offset=...)."""
    _check_offsets(offsets)
    G = offsets.numel() - 1
    dev = offsets.device
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    _require(isinstance(y, torch.Tensor) and y.is_cuda and y.dtype == torch.bfloat16 and y.dim() == 2
             and y.stride(-1) == 1 and y.shape[0] >= M and y.shape[1] >= N,
             "y: a [>= M, >= N] bf16 CUDA tensor with unit column stride")
    _check_operands(op, G, M, N, K, a_codes, a_scales_mma, b_codes, b_scales_mma)
    o = dict(out or {})
    if "codes" not in o:
        o["codes"] = torch.empty((M, N // 2), dtype=torch.uint8, device=dev)
    if scales and "scales" not in o:
        o["scales"] = torch.empty((M, N // 32), dtype=torch.uint8, device=dev)
    if scales_mma and "scales_mma" not in o:
        o["scales_mma"] = torch.empty((mxfp4_mma_scale_bytes(M, N // 32),), dtype=torch.uint8, device=dev)
    _check_quant_outputs(o, 1, M, N, False, M, N)
    q = QuantOutputs(o["codes"].data_ptr(), _ptr(o.get("scales")), _ptr(o.get("scales_mma")), None, None)
    qp = QuantParams(BLOCK_1X32, 0, 0, 0, ROUND_STOCHASTIC if sr_seed is not None else ROUND_NEAREST,
                     int(sr_seed or 0), int(sr_offset))
    mxfp4_grouped_gemm_fused(op, G, ctypes.c_void_p(offsets.data_ptr()),
                             Operand(a_codes.data_ptr(), a_scales_mma.data_ptr()),
                             Operand(b_codes.data_ptr(), b_scales_mma.data_ptr()), M, N, K,
                             ctypes.c_void_p(y.data_ptr()), y.stride(0), q, qp, stream)
    return y, o

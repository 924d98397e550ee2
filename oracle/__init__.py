"""Plain CPU oracle for the MXFP4 quantise-and-contract path (ALTO recipe).

TEST INFRASTRUCTURE ONLY: the test-suite, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` are the only callers.  The product library
(``fp4_precision_numerics_b200``) never imports this package, and this package
never imports the product.

The arithmetic lives in ``mxfp4_oracle.c`` (scalar C, binary32 ops rounded to
nearest-even, no FMA contraction, no flush-to-zero); this module builds it
with gcc on first use and marshals numpy arrays.  The GEMM reference is a
binary64 matrix product of the dequantised operands (``numpy.matmul`` for
large cases, cross-checked against the C triple loop).

Which passage each step follows is cited in ``mxfp4_oracle.c``.  Parity of
the de-oscillation rule is unpinned by the pages (the rule is a reading of
its own, pinned only by hand-worked traces).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mxfp4_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_SO = os.path.join(_BUILD, "libmxfp4_oracle.so")
_lock = threading.Lock()
_lib = None

BF16 = 0
F32 = 1

E2M1_GRID = (0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0)


def build(force: bool = False) -> str:
    """Compile the oracle shared library (gcc, OpenMP, no fast-math)."""
    os.makedirs(_BUILD, exist_ok=True)
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + ".tmp%d" % os.getpid()
        cmd = ["gcc", "-O2", "-std=gnu11", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
               "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"]
        subprocess.check_call(cmd)
        os.replace(tmp, _SO)
    return _SO


def lib():
    global _lib
    with _lock:
        if _lib is None:
            build()
            L = ctypes.CDLL(_SO)
            u32p = ctypes.POINTER(ctypes.c_uint32)
            L.oracle_philox4x32_10.argtypes = [u32p, u32p, u32p]
            L.oracle_sr_bits16.argtypes = [ctypes.c_uint64, ctypes.c_uint32, ctypes.c_uint64]
            L.oracle_sr_bits16.restype = ctypes.c_uint32
            L.oracle_rht_signs.argtypes = [ctypes.c_uint64, ctypes.c_int, ctypes.c_void_p]
            L.oracle_e2m1_value.argtypes = [ctypes.c_int]
            L.oracle_e2m1_value.restype = ctypes.c_double
            L.oracle_scale_exponent.argtypes = [ctypes.c_float]
            L.oracle_scale_exponent.restype = ctypes.c_int
            L.oracle_e2m1_rn.argtypes = [ctypes.c_float]
            L.oracle_e2m1_rn.restype = ctypes.c_int
            L.oracle_e2m1_sr.argtypes = [ctypes.c_float, ctypes.c_uint32]
            L.oracle_e2m1_sr.restype = ctypes.c_int
            L.oracle_rht16.argtypes = [ctypes.c_void_p] * 3
            L.oracle_rht16_dense_f64.argtypes = [ctypes.c_void_p] * 3
            i64 = ctypes.c_int64
            L.oracle_rht_rows.argtypes = [ctypes.c_void_p, ctypes.c_int, i64, i64, i64, ctypes.c_uint64,
                                          ctypes.c_void_p]
            qargs = [ctypes.c_void_p, ctypes.c_int, i64, i64, i64, ctypes.c_int, ctypes.c_uint64, ctypes.c_int,
                     ctypes.c_uint64, ctypes.c_uint32]
            L.oracle_quantize_1d.argtypes = qargs + [i64, ctypes.c_void_p, ctypes.c_void_p]
            L.oracle_quantize_1d_transposed.argtypes = qargs + [i64, ctypes.c_void_p, ctypes.c_void_p]
            L.oracle_quantize_2d.argtypes = qargs + [ctypes.c_void_p, ctypes.c_void_p]
            L.oracle_deosc_update.argtypes = [ctypes.c_void_p, i64, i64, i64, ctypes.c_uint32, ctypes.c_uint32,
                                              ctypes.c_uint32, ctypes.c_uint32, ctypes.c_void_p, ctypes.c_void_p,
                                              ctypes.c_void_p]
            L.oracle_dequant_1d.argtypes = [ctypes.c_void_p, ctypes.c_void_p, i64, i64, ctypes.c_void_p]
            L.oracle_dequant_2d.argtypes = [ctypes.c_void_p, ctypes.c_void_p, i64, i64, ctypes.c_void_p]
            L.oracle_gemm_f64.argtypes = [ctypes.c_void_p, ctypes.c_void_p, i64, i64, i64, ctypes.c_void_p]
            L.oracle_num_threads.restype = ctypes.c_int
            _lib = L
    return _lib


def _ptr(a: np.ndarray) -> ctypes.c_void_p:
    assert a.flags["C_CONTIGUOUS"]
    return ctypes.c_void_p(a.ctypes.data)


def _input(x: np.ndarray):
    """bf16 inputs travel as uint16 bit patterns, float32 as float32."""
    x = np.ascontiguousarray(x)
    if x.dtype == np.uint16:
        return x, BF16
    if x.dtype == np.float32:
        return x, F32
    raise TypeError("oracle input must be bf16 bits (uint16) or float32, got %s" % x.dtype)


# --------------------------------------------------------------------------
# Scalar pieces
# --------------------------------------------------------------------------
def philox4x32_10(counter, key) -> np.ndarray:
    c = (ctypes.c_uint32 * 4)(*[int(v) & 0xFFFFFFFF for v in counter])
    k = (ctypes.c_uint32 * 2)(*[int(v) & 0xFFFFFFFF for v in key])
    o = (ctypes.c_uint32 * 4)()
    lib().oracle_philox4x32_10(c, k, o)
    return np.array(list(o), dtype=np.uint32)


def sr_bits16(seed: int, offset: int, n: int) -> int:
    return int(lib().oracle_sr_bits16(seed, offset, n))


def rht_signs(seed: int, d: int = 16) -> np.ndarray:
    s = np.zeros(d, dtype=np.float32)
    lib().oracle_rht_signs(seed, d, _ptr(s))
    return s


def e2m1_value(code: int) -> float:
    return float(lib().oracle_e2m1_value(int(code)))


def scale_exponent(amax: float) -> int:
    return int(lib().oracle_scale_exponent(float(amax)))


def e2m1_rn(v: float) -> int:
    return int(lib().oracle_e2m1_rn(float(v)))


def e2m1_sr(v: float, r16: int) -> int:
    return int(lib().oracle_e2m1_sr(float(v), int(r16)))


def rht16(x: np.ndarray, s: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    s = np.ascontiguousarray(s, dtype=np.float32)
    y = np.zeros(16, dtype=np.float32)
    lib().oracle_rht16(_ptr(x), _ptr(s), _ptr(y))
    return y


def rht16_dense_f64(x: np.ndarray, s: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float64)
    s = np.ascontiguousarray(s, dtype=np.float64)
    y = np.zeros(16, dtype=np.float64)
    lib().oracle_rht16_dense_f64(_ptr(x), _ptr(s), _ptr(y))
    return y


# --------------------------------------------------------------------------
# Tensor-level operations
# --------------------------------------------------------------------------
def rht_rows(x: np.ndarray, seed: int) -> np.ndarray:
    x, dt = _input(x)
    rows, cols = x.shape
    out = np.zeros((rows, cols), dtype=np.float32)
    lib().oracle_rht_rows(_ptr(x), dt, rows, cols, cols, seed, _ptr(out))
    return out


def quantize_1d(x: np.ndarray, rht_d: int = 0, rht_seed: int = 0, sr: bool = False, sr_seed: int = 0,
                sr_offset: int = 0, row0: int = 0):
    """1x32 blocks along the last dim.  Returns (codes [R, C/2], scales [R, C/32])."""
    x, dt = _input(x)
    rows, cols = x.shape
    codes = np.zeros((rows, cols // 2), dtype=np.uint8)
    scales = np.zeros((rows, cols // 32), dtype=np.uint8)
    lib().oracle_quantize_1d(_ptr(x), dt, rows, cols, cols, rht_d, rht_seed, int(sr), sr_seed, sr_offset, row0,
                             _ptr(codes), _ptr(scales))
    return codes, scales


def quantize_1d_transposed(x: np.ndarray, rht_d: int = 0, rht_seed: int = 0, sr: bool = False,
                           sr_seed: int = 0, sr_offset: int = 0, col0: int = 0):
    """1x32 blocks along dim 0; output in the transposed layout
    (codes [C, R/2], scales [C, R/32]).  `col0` is the global index of x's
    first column (= first output row), so a column slice draws the same SR
    bits as the whole tensor."""
    x, dt = _input(x)
    rows, cols = x.shape
    codes = np.zeros((cols, rows // 2), dtype=np.uint8)
    scales = np.zeros((cols, rows // 32), dtype=np.uint8)
    lib().oracle_quantize_1d_transposed(_ptr(x), dt, rows, cols, cols, rht_d, rht_seed, int(sr), sr_seed,
                                        sr_offset, col0, _ptr(codes), _ptr(scales))
    return codes, scales


def quantize_2d(x: np.ndarray, rht_d: int = 0, rht_seed: int = 0, sr: bool = False, sr_seed: int = 0,
                sr_offset: int = 0):
    """32x32 blocks.  Returns (codes [R, C/2], scales [R/32, C/32])."""
    x, dt = _input(x)
    rows, cols = x.shape
    codes = np.zeros((rows, cols // 2), dtype=np.uint8)
    scales = np.zeros((rows // 32, cols // 32), dtype=np.uint8)
    lib().oracle_quantize_2d(_ptr(x), dt, rows, cols, cols, rht_d, rht_seed, int(sr), sr_seed, sr_offset,
                             _ptr(codes), _ptr(scales))
    return codes, scales


def deosc_update(master: np.ndarray, step: int, state: np.ndarray, flip_threshold: int = 4,
                 reset_period: int = 0, freeze_lower: bool = False):
    """One de-oscillation step over fp32 master weights [G, R, C].  Updates
    ``state`` in place; returns (codes [G, R, C/2], scales [G, R/32, C/32])."""
    master = np.ascontiguousarray(master, dtype=np.float32)
    if master.ndim == 2:
        master = master[None]
    g, rows, cols = master.shape
    assert state.dtype == np.uint8 and state.shape == (g, rows, cols) and state.flags["C_CONTIGUOUS"]
    codes = np.zeros((g, rows, cols // 2), dtype=np.uint8)
    scales = np.zeros((g, rows // 32, cols // 32), dtype=np.uint8)
    lib().oracle_deosc_update(_ptr(master), g, rows, cols, step, flip_threshold, reset_period,
                              int(bool(freeze_lower)), _ptr(state), _ptr(codes), _ptr(scales))
    return codes, scales


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Binary64 values -> bfloat16 bit patterns (uint16), rounded once to
    nearest with ties to even: 8 significant bits, the binary32 exponent
    range, spacing 2^-133 below 2^-126 (subnormals), and a result at or past
    2^128 becomes infinity.  This is how a GEMM output is stored when the
    next layer reads it as a bf16 activation (the recipe trains against a
    BF16 baseline: abstract; roboaidigest "What ALTO Actually Does")."""
    x = np.asarray(x, dtype=np.float64)
    _, e = np.frexp(x)                        # |x| in [2^(e-1), 2^e)
    q = np.maximum(e - 8, -133)               # exponent of one bf16 step at x
    y = np.ldexp(np.round(np.ldexp(x, -q)), q)  # np.round: halves to even
    y = np.where(np.abs(y) >= 2.0 ** 128, np.copysign(np.inf, x), y)
    return (y.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)


def dequant_1d(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    codes = np.ascontiguousarray(codes)
    scales = np.ascontiguousarray(scales)
    rows, half = codes.shape
    out = np.zeros((rows, half * 2), dtype=np.float64)
    lib().oracle_dequant_1d(_ptr(codes), _ptr(scales), rows, half * 2, _ptr(out))
    return out


def dequant_2d(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    codes = np.ascontiguousarray(codes)
    scales = np.ascontiguousarray(scales)
    rows, half = codes.shape
    out = np.zeros((rows, half * 2), dtype=np.float64)
    lib().oracle_dequant_2d(_ptr(codes), _ptr(scales), rows, half * 2, _ptr(out))
    return out


def gemm_f64_loop(A: np.ndarray, B: np.ndarray) -> np.ndarray:
    """C = A @ B^T by the plain C triple loop (binary64)."""
    A = np.ascontiguousarray(A, dtype=np.float64)
    B = np.ascontiguousarray(B, dtype=np.float64)
    M, K = A.shape
    N = B.shape[0]
    C = np.zeros((M, N), dtype=np.float64)
    lib().oracle_gemm_f64(_ptr(A), _ptr(B), M, N, K, _ptr(C))
    return C


def gemm_f64(A: np.ndarray, B: np.ndarray) -> np.ndarray:
    """C = A @ B^T in binary64 (numpy matmul; pinned against the loop)."""
    return np.asarray(A, dtype=np.float64) @ np.asarray(B, dtype=np.float64).T


def grouped_gemm_f64(A: np.ndarray, B: np.ndarray, offsets) -> np.ndarray:
    """Per group g: C[o_g:o_{g+1}] = A[o_g:o_{g+1}] @ B[g]^T (binary64).
    A: [M_total, K]; B: [G, N, K]."""
    G = len(offsets) - 1
    C = np.zeros((A.shape[0], B.shape[1]), dtype=np.float64)
    for g in range(G):
        lo, hi = int(offsets[g]), int(offsets[g + 1])
        if hi > lo:
            C[lo:hi] = gemm_f64(A[lo:hi], B[g])
    return C


def num_threads() -> int:
    return int(lib().oracle_num_threads())

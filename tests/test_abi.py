"""CPU checks of the boundary: libmxfp4.so builds for sm_100a, loads, and
exports every entry point include/mxfp4.h declares; host-side argument
validation runs without a GPU (no compute call is made)."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mxfp4.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(mxfp4_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def libpath():
    from fp4_precision_numerics_b200 import build
    return build.build()


def test_header_declares_the_four_calls():
    fns = declared_functions()
    for name in ("mxfp4_quantize", "mxfp4_rht", "mxfp4_deosc_update", "mxfp4_grouped_gemm"):
        assert name in fns


def test_library_exports_every_declared_symbol(libpath):
    out = subprocess.run(["nm", "-D", "--defined-only", libpath], capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\bT (\w+)", out))
    missing = [f for f in declared_functions() if f not in exported]
    assert not missing, missing
    # nothing else leaks out with the mxfp4_ prefix
    extra = [s for s in exported if s.startswith("mxfp4_") and s not in declared_functions()]
    assert not extra, extra


def test_library_loads_and_reports_version(libpath):
    L = ctypes.CDLL(libpath)
    L.mxfp4_version.restype = ctypes.c_char_p
    assert b"sm_100a" in L.mxfp4_version()
    L.mxfp4_mma_scale_bytes.argtypes = [ctypes.c_int64, ctypes.c_int64]
    L.mxfp4_mma_scale_bytes.restype = ctypes.c_size_t
    assert L.mxfp4_mma_scale_bytes(128, 4) == 512
    assert L.mxfp4_mma_scale_bytes(2880, 90) == 23 * 23 * 512
    assert L.mxfp4_mma_scale_bytes(0, 4) == 0


def test_host_validation_without_gpu(libpath):
    from fp4_precision_numerics_b200 import mxfp4
    L = mxfp4.lib()
    p = mxfp4.QuantParams(mxfp4.BLOCK_1X32, 0, 0, 0, 0, 0, 0)
    o = mxfp4.QuantOutputs(None, None, None, None, None)
    # null input
    assert L.mxfp4_quantize(None, 0, 1, 4, 32, 32, ctypes.byref(p), ctypes.byref(o), None) == -1
    # null codes output
    assert L.mxfp4_quantize(ctypes.c_void_p(16), 0, 1, 4, 32, 32, ctypes.byref(p), ctypes.byref(o), None) == -1
    o.codes = 16
    # cols not a multiple of 32
    assert L.mxfp4_quantize(ctypes.c_void_p(16), 0, 1, 4, 48, 48, ctypes.byref(p), ctypes.byref(o), None) == -2
    # misaligned input
    assert L.mxfp4_quantize(ctypes.c_void_p(18), 0, 1, 4, 32, 32, ctypes.byref(p), ctypes.byref(o), None) == -3
    # bad enum
    p.rounding = 9
    assert L.mxfp4_quantize(ctypes.c_void_p(16), 0, 1, 4, 32, 32, ctypes.byref(p), ctypes.byref(o), None) == -1
    assert "rounding" in mxfp4.last_error()
    # rht with unsupported d
    assert L.mxfp4_rht(ctypes.c_void_p(16), 0, 4, 32, 32, 1, 8, 0, ctypes.c_void_p(16), 1, None) == -1
    # gemm: bad op, null operands
    a = mxfp4.Operand(None, None)
    assert L.mxfp4_grouped_gemm(7, 1, ctypes.c_void_p(16), a, a, 128, 192, 128, ctypes.c_void_p(16), 192, None) == -1
    assert L.mxfp4_grouped_gemm(0, 1, ctypes.c_void_p(16), a, a, 128, 192, 128, ctypes.c_void_p(16), 192, None) == -1
    d = mxfp4.DeoscParams(9, 0)
    assert L.mxfp4_deosc_update(ctypes.c_void_p(16), 1, 32, 32, 0, ctypes.byref(d), ctypes.c_void_p(16),
                                ctypes.byref(o), None) == -1


def test_dual_host_validation_without_gpu(libpath):
    from fp4_precision_numerics_b200 import mxfp4
    L = mxfp4.lib()
    rp = mxfp4.QuantParams(mxfp4.BLOCK_1X32, 0, 0, 0, 0, 0, 0)
    cp = mxfp4.QuantParams(mxfp4.BLOCK_1X32, 1, 0, 0, 0, 0, 0)
    o = mxfp4.QuantOutputs(None, None, None, None, None)
    args = lambda r, c: (None, 0, 1, 32, 32, 32, ctypes.byref(r), ctypes.byref(c), ctypes.byref(o), ctypes.byref(o),
                         None)
    assert L.mxfp4_quantize_dual(*args(rp, cp)) == -1                      # null input
    assert L.mxfp4_quantize_dual(*args(cp, rp)) == -1                      # directions swapped
    bad = mxfp4.QuantParams(mxfp4.BLOCK_1X32, 1, 0, 0, mxfp4.ROUND_STOCHASTIC, 0, 0)
    assert L.mxfp4_quantize_dual(*args(rp, bad)) == -1                     # rounding differs
    assert L.mxfp4_quantize_dual(None, 0, 0, 32, 32, 32, ctypes.byref(rp), ctypes.byref(cp), ctypes.byref(o),
                                 ctypes.byref(o), None) == 0                # empty: nothing to do



def test_fused_gemm_host_validation_without_gpu(libpath):
    from fp4_precision_numerics_b200 import mxfp4
    L = mxfp4.lib()
    a = mxfp4.Operand(16, 16)
    q = mxfp4.QuantOutputs(16, None, None, None, None)
    off, y = ctypes.c_void_p(16), ctypes.c_void_p(16)

    def call(op=0, G=1, M=128, N=192, K=128, y=y, ldy=192, q=q, qp=None):
        return L.mxfp4_grouped_gemm_fused(op, G, off, a, a, M, N, K, y, ldy, ctypes.byref(q),
                                          ctypes.byref(qp) if qp is not None else None, None)

    assert call(op=mxfp4.GEMM_WGRAD) == -1                                  # wgrad has no fused epilogue
    assert call(y=None) == -1                                               # null y
    assert call(N=200, ldy=200) == -2                                       # N % 32 != 0
    assert call(K=0) == -2                                                  # nothing to contract
    assert call(ldy=100) == -1                                              # ldy < N
    assert call(ldy=196) == -3                                              # ldy % 8 != 0
    assert call(y=ctypes.c_void_p(18)) == -3                                # misaligned y
    assert call(G=300) == -2                                                # CTA-pair kernel only
    assert call(q=mxfp4.QuantOutputs(16, None, None, 16, None)) == -1      # 2D-only outputs given
    assert call(q=mxfp4.QuantOutputs(None, None, None, None, None)) == -1  # null codes
    assert call(qp=mxfp4.QuantParams(mxfp4.BLOCK_32X32, 0, 0, 0, 0, 0, 0)) == -1     # 2D blocks
    assert call(qp=mxfp4.QuantParams(mxfp4.BLOCK_1X32, 1, 0, 0, 0, 0, 0)) == -1      # along rows
    assert call(qp=mxfp4.QuantParams(mxfp4.BLOCK_1X32, 0, 16, 1, 0, 0, 0)) == -1     # RHT
    assert call(qp=mxfp4.QuantParams(mxfp4.BLOCK_1X32, 0, 0, 0, 9, 0, 0)) == -1      # bad rounding
    assert "fused" in mxfp4.last_error()


def test_index_range_is_checked_before_launch(libpath):
    """The quantisers index rows and features of all groups in 32 bits:
    2^31 rows are rejected on the host (no device memory is touched)."""
    from fp4_precision_numerics_b200 import mxfp4
    L = mxfp4.lib()
    o = mxfp4.QuantOutputs(16, None, None, None, None)
    for along in (0, 1):
        p = mxfp4.QuantParams(mxfp4.BLOCK_1X32, along, 0, 0, 0, 0, 0)
        assert L.mxfp4_quantize(ctypes.c_void_p(16), 0, 1, 1 << 31, 32, 32, ctypes.byref(p), ctypes.byref(o),
                                None) == -2
        assert "2^31" in mxfp4.last_error()
    rp = mxfp4.QuantParams(mxfp4.BLOCK_1X32, 0, 0, 0, 0, 0, 0)
    cp = mxfp4.QuantParams(mxfp4.BLOCK_1X32, 1, 0, 0, 0, 0, 0)
    assert L.mxfp4_quantize_dual(ctypes.c_void_p(16), 0, 2, 1 << 30, 32, 32, ctypes.byref(rp), ctypes.byref(cp),
                                 ctypes.byref(o), ctypes.byref(o), None) == -2


def test_mma_peak_probe_host_validation_without_gpu(libpath):
    """The peak probe rejects an MMA count outside [1, 2^22] and a null
    result pointer before any CUDA call."""
    from fp4_precision_numerics_b200 import mxfp4
    L = mxfp4.lib()
    f = ctypes.c_double(-1.0)
    for n in (0, -5, (1 << 22) + 1):
        assert L.mxfp4_mma_peak_probe(n, ctypes.byref(f), None) == -1
    assert L.mxfp4_mma_peak_probe(16, None, None) == -1
    assert "mmas_per_pair" in mxfp4.last_error()
    assert f.value == -1.0


def test_every_host_check_returns_its_status(libpath):
    """Each host-side check of include/mxfp4.h returns its documented status
    before any CUDA call (pointers are fake, aligned or not as the case
    needs; nothing is dereferenced on the host)."""
    from fp4_precision_numerics_b200 import mxfp4
    L = mxfp4.lib()
    INV, SHAPE, ALIGN = -1, -2, -3
    P = lambda *a: mxfp4.QuantParams(*a)
    ok_p = P(mxfp4.BLOCK_1X32, 0, 0, 0, 0, 0, 0)
    outs = mxfp4.QuantOutputs(16, None, None, None, None)

    def quant(in_ptr=16, dtype=0, G=1, R=64, C=64, ld=64, p=ok_p, o=outs):
        return L.mxfp4_quantize(ctypes.c_void_p(in_ptr), dtype, G, R, C, ld, ctypes.byref(p), ctypes.byref(o), None)

    assert quant(dtype=7) == INV                                             # in_dtype
    assert quant(ld=32) == INV                                               # ld < cols
    assert quant(p=P(5, 0, 0, 0, 0, 0, 0)) == INV                            # block
    assert quant(p=P(mxfp4.BLOCK_1X32, 0, 8, 1, 0, 0, 0)) == INV             # rht_d
    assert quant(p=P(mxfp4.BLOCK_32X32, 0, 0, 0, 0, 0, 0), R=48) == SHAPE    # 2D rows % 32
    assert quant(p=P(mxfp4.BLOCK_1X32, 1, 0, 0, 0, 0, 0), R=48) == SHAPE     # along rows, rows % 32
    assert quant(o=mxfp4.QuantOutputs(24, None, None, None, None)) == ALIGN  # codes misaligned
    assert quant(o=mxfp4.QuantOutputs(16, None, None, 16, None)) == INV      # codes_t with 1D blocks
    assert quant(p=P(mxfp4.BLOCK_32X32, 0, 0, 0, 0, 0, 0),
                 o=mxfp4.QuantOutputs(16, None, None, None, 16)) == INV      # scales_mma_t without codes_t
    assert quant(G=0) == 0 and quant(R=0) == 0                               # empty: nothing to do

    rp, cp = ok_p, P(mxfp4.BLOCK_1X32, 1, 0, 0, 0, 0, 0)

    def dual(R=64, C=64, r=rp, c=cp, in_ptr=16):
        return L.mxfp4_quantize_dual(ctypes.c_void_p(in_ptr), 0, 1, R, C, C, ctypes.byref(r), ctypes.byref(c),
                                     ctypes.byref(outs), ctypes.byref(outs), None)

    assert dual(c=P(mxfp4.BLOCK_32X32, 1, 0, 0, 0, 0, 0)) == INV             # 2D blocks
    assert dual(c=P(mxfp4.BLOCK_1X32, 1, 8, 1, 0, 0, 0)) == INV              # rht_d
    sr = mxfp4.ROUND_STOCHASTIC
    assert dual(r=P(mxfp4.BLOCK_1X32, 0, 0, 0, sr, 1, 0), c=P(mxfp4.BLOCK_1X32, 1, 0, 0, sr, 2, 0)) == INV  # seeds
    assert dual(R=48) == SHAPE and dual(C=48) == SHAPE                       # multiples of 32
    assert dual(in_ptr=18) == ALIGN                                          # input misaligned

    def rht(in_ptr=16, out_ptr=16, dtype=0, out_dtype=1, R=4, C=32, ld=32, axis=1):
        return L.mxfp4_rht(ctypes.c_void_p(in_ptr), dtype, R, C, ld, axis, 16, 1, ctypes.c_void_p(out_ptr), out_dtype,
                           None)

    assert rht(dtype=5) == INV and rht(out_dtype=5) == INV                   # dtypes
    assert rht(axis=2) == INV and rht(axis=-1) == INV                        # axis 0 or 1
    assert rht(C=24, ld=24) == SHAPE                                         # cols % 16 along the last dim
    assert rht(axis=0, R=24) == SHAPE                                        # rows % 16 along dim 0
    assert rht(axis=0, R=4, C=24, ld=24) == SHAPE                            # (cols need not be)
    assert rht(out_ptr=20) == ALIGN                                          # output misaligned

    def deosc(thr=4, freeze_lower=0, R=64, C=64, master=16):
        d = mxfp4.DeoscParams(thr, 0, freeze_lower)
        return L.mxfp4_deosc_update(ctypes.c_void_p(master), 1, R, C, 1, ctypes.byref(d), ctypes.c_void_p(16),
                                    ctypes.byref(outs), None)

    assert deosc(thr=0) == INV and deosc(thr=8) == INV                       # threshold in 1..7
    assert deosc(freeze_lower=2) == INV
    assert deosc(R=48) == SHAPE and deosc(C=40) == SHAPE                     # 32x32 blocks
    assert deosc(master=8) == ALIGN

    A = mxfp4.Operand(16, 16)

    def gemm(op=0, G=1, M=128, N=192, K=128, ldo=192, out=16, a=A):
        return L.mxfp4_grouped_gemm(op, G, ctypes.c_void_p(16), a, a, M, N, K, ctypes.c_void_p(out), ldo, None)

    assert gemm(N=0) == INV and gemm(ldo=100) == INV                         # geometry, ldo < N
    assert gemm(G=5000) == SHAPE                                             # group count
    assert gemm(op=mxfp4.GEMM_WGRAD, K=192) == SHAPE                         # wgrad tokens % 128
    assert gemm(K=96) == SHAPE and gemm(M=192) == SHAPE                      # K % 64, M % 128
    assert gemm(ldo=194) == ALIGN                                            # ldo % 4
    assert gemm(out=24) == ALIGN and gemm(a=mxfp4.Operand(16, 40)) == ALIGN  # pointer alignment


C_CONSUMER = r'''
#include "mxfp4.h"
#include <stdio.h>
int main(void) {
    mxfp4_quant_params p = {0};
    mxfp4_quant_outputs o = {0};
    char msg[256];
    int st = mxfp4_quantize(NULL, MXFP4_DTYPE_BF16, 1, 32, 32, 32, &p, &o, NULL);
    mxfp4_last_error(msg, sizeof msg);
    printf("%s|%zu|%d|%s\n", mxfp4_version(), mxfp4_mma_scale_bytes(128, 4), st, msg);
    return 0;
}
'''


def test_header_is_plain_c_and_a_c_program_uses_the_library(libpath):
    """include/mxfp4.h is a C ABI: it compiles as strict C99, and a C program
    links against libmxfp4.so and calls it (version, a layout helper and a
    host-side check; none needs a GPU)."""
    d = os.path.join(ROOT, "tests", "_build")
    os.makedirs(d, exist_ok=True)
    src, exe = os.path.join(d, "c_consumer.c"), os.path.join(d, "c_consumer")
    with open(src, "w") as f:
        f.write(C_CONSUMER)
    libdir = os.path.dirname(libpath)
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", os.path.join(ROOT, "include"),
                    src, "-o", exe, "-L", libdir, "-lmxfp4", "-Wl,-rpath," + libdir], check=True)
    out = subprocess.run([exe], capture_output=True, text=True, check=True).stdout.strip().split("|")
    assert "sm_100a" in out[0] and out[1] == "512" and out[2] == "-1" and "null" in out[3]


def test_tensor_core_scale_layout_is_a_bijection(libpath):
    """The tensor-core scale layout of include/mxfp4.h (the decoder the GPU
    tests use) sends distinct (row, scale) pairs to distinct bytes inside
    mxfp4_mma_scale_bytes(R, S), and fills that buffer exactly when R and S
    are whole chunks (128 rows x 4 scales)."""
    import numpy as np
    from fp4_precision_numerics_b200 import mxfp4
    from tests.gpu_util import mma_scales_to_rows
    for R, S in ((128, 4), (256, 8), (2880, 90), (200, 5), (33, 3), (67584, 180)):
        size = mxfp4.mxfp4_mma_scale_bytes(R, S)
        assert size == ((R + 127) // 128) * ((S + 3) // 4) * 512
        off = mma_scales_to_rows(np.arange(size, dtype=np.int64), R, S)
        assert off.shape == (R, S) and off.min() >= 0 and off.max() < size
        assert len(np.unique(off)) == R * S
        if R % 128 == 0 and S % 4 == 0:
            assert R * S == size


def test_pair_gemm_unit_walk_matches_direct_decomposition(tmp_path):
    """The pair GEMM's division-free unit walk visits, for every cluster,
    exactly the units of the direct decomposition of u = cluster, cluster +
    step, ... (random expert layouts with empty experts, both modes); checked
    by a host program built from the kernel's own header."""
    src = os.path.join(ROOT, "tests", "native", "unit_walk_check.cu")
    exe = str(tmp_path / "unit_walk_check")
    subprocess.run(["nvcc", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-I",
                    os.path.join(ROOT, "fp4_precision_numerics_b200", "csrc"), "-I", os.path.join(ROOT, "include"),
                    "-o", exe, src, "-lcuda"], check=True)
    out = subprocess.run([exe], capture_output=True, text=True, check=True).stdout
    assert out.startswith("ok") and int(out.split()[1]) > 10 ** 6, out


def test_staging_index_maps_match_the_direct_stores(tmp_path):
    """The shared-memory staging of the token-dim codes (quant1d_cols_kernel)
    and of the W^T codes (quant2d_coal_kernel): every piece lands in its own
    16-byte slot, and the cooperative store writes each slot to the row and
    bytes of the direct store of the lane that filled it; checked by a host
    program built from the kernels' header."""
    src = os.path.join(ROOT, "tests", "native", "staging_check.cu")
    exe = str(tmp_path / "staging_check")
    subprocess.run(["nvcc", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-I",
                    os.path.join(ROOT, "fp4_precision_numerics_b200", "csrc"), "-I", os.path.join(ROOT, "include"),
                    "-o", exe, src, "-lcuda"], check=True)
    out = subprocess.run([exe], capture_output=True, text=True, check=True).stdout
    assert out.startswith("ok") and int(out.split()[1]) > 3000, out

"""GPU parity: the grouped GEMM with the fused epilogue (bf16 output plus its
1x32-along-N MXFP4 quantisation, nearest or stochastic rounding).

Exact regime: operands on the E2M1 grid with block exponents in {-1, 0, 1}
(every block holds a +-6 * 2^e entry, so quantisation is lossless) keep
every product and partial sum of the contraction exact in binary32 (sums
below 2^17 on a 2^-4 lattice).  The binary32 accumulation then equals the
oracle's binary64 product whatever the order, so the bf16 output and its
codes and scales are compared bit for bit with the oracle's rounding and
quantisation of that product.

Realistic regime (Gaussian activations and weights): the bf16 output is the
binary32 path's output rounded by torch, lies within the GEMM bound of the
oracle plus half a bf16 step, and the codes and scales equal the library's
quantisation of that bf16 output.

Groups: one single-tile group (the pair's second tile idle), an empty group,
a three-tile group and a two-tile group; N = 448 and 640 leave a partial
192-column tile at the edge."""
import numpy as np
import pytest
import torch

import oracle
from fp4_precision_numerics_b200 import mxfp4, synth
from tests.gpu_util import dev_bf16, host, mma_scales_to_rows

pytestmark = pytest.mark.gpu
TOL = 1e-3
SEG = [128, 0, 384, 256]
OFFS = np.concatenate([[0], np.cumsum(SEG)]).astype(np.int64)
G, M = len(SEG), int(OFFS[-1])
NW, KW = 448, 640                       # W_g is [NW, KW]: fprop N = NW, K = KW; dgrad N = KW, K = NW
GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def _grid_blocks(rng, shape, brows):
    """Values g * 2^e, g on the signed E2M1 grid, one exponent e in {-1, 0, 1}
    per brows x 32 block, and one +-6 * 2^e entry in every block."""
    *lead, R, C = shape
    v = rng.choice(GRID, size=shape) * rng.choice([-1.0, 1.0], size=shape)
    e = rng.integers(-1, 2, size=(*lead, R // brows, C // 32))
    v[..., :, ::32] = 6.0 * rng.choice([-1.0, 1.0], size=(*lead, R, C // 32))
    v = v * np.exp2(np.repeat(np.repeat(e, brows, axis=-2), 32, axis=-1))
    return synth.bf16_bits(v.astype(np.float32))


def _bits(y: torch.Tensor) -> np.ndarray:
    return host(y.view(torch.int16)).view(np.uint16)


def _offs_dev():
    return torch.tensor(OFFS.astype(np.int32), device="cuda")


def _run(op, a_bits, w_bits, sr_seed=None, sr_offset=0):
    """Quantise (library) and run both epilogues; returns y fused, q, y fp32."""
    qa = mxfp4.quantize(dev_bf16(a_bits), scales=False, scales_mma=True)
    qw = mxfp4.quantize(dev_bf16(w_bits), block="32x32", scales=False, scales_mma=True, transposed=True)
    if op == mxfp4.GEMM_FPROP:
        b, bs, N, K = qw["codes"], qw["scales_mma"], NW, KW
    else:
        b, bs, N, K = qw["codes_t"], qw["scales_mma_t"], KW, NW
    y, q = mxfp4.grouped_gemm_fused(op, _offs_dev(), qa["codes"], qa["scales_mma"], b, bs, M, N, K,
                                    sr_seed=sr_seed, sr_offset=sr_offset)
    y32 = mxfp4.grouped_gemm(op, _offs_dev(), qa["codes"], qa["scales_mma"], b, bs, M, N, K)
    mxfp4.mxfp4_check_device_status()
    torch.cuda.synchronize()
    return y, q, y32, N


def _oracle_product(op, a_bits, w_bits):
    ca, sa = oracle.quantize_1d(a_bits)
    A = oracle.dequant_1d(ca, sa)
    cw, sw = oracle.quantize_2d(w_bits.reshape(G * NW, KW))
    W = oracle.dequant_2d(cw, sw).reshape(G, NW, KW)
    B = W if op == mxfp4.GEMM_FPROP else np.ascontiguousarray(W.transpose(0, 2, 1))
    return oracle.grouped_gemm_f64(A, B, OFFS), oracle.grouped_gemm_f64(np.abs(A), np.abs(B), OFFS)


@pytest.mark.parametrize("op", [mxfp4.GEMM_FPROP, mxfp4.GEMM_DGRAD])
def test_fused_epilogue_exact_regime_bit_exact(op):
    rng = np.random.default_rng(21 + op)
    a = _grid_blocks(rng, (M, NW if op == mxfp4.GEMM_DGRAD else KW), 1)
    w = _grid_blocks(rng, (G, NW, KW), 32)
    y, q, y32, N = _run(op, a, w)
    ref, _ = _oracle_product(op, a, w)
    assert np.array_equal(host(y32).astype(np.float64), ref), "binary32 accumulation is not exact here"
    y_ref = oracle.bf16_round(ref)
    c_ref, s_ref = oracle.quantize_1d(y_ref)
    assert np.array_equal(_bits(y), y_ref)
    assert np.array_equal(host(q["codes"]), c_ref)
    assert np.array_equal(host(q["scales"]), s_ref)
    assert np.array_equal(mma_scales_to_rows(host(q["scales_mma"]), M, N // 32), s_ref)


@pytest.mark.parametrize("op", [mxfp4.GEMM_FPROP, mxfp4.GEMM_DGRAD])
def test_fused_epilogue_realistic_inputs(op):
    rng = np.random.default_rng(31 + op)
    a = synth.bf16_bits(rng.standard_normal((M, NW if op == mxfp4.GEMM_DGRAD else KW)).astype(np.float32))
    w = synth.bf16_bits((rng.standard_normal((G, NW, KW)) * 0.02).astype(np.float32))
    y, q, y32, N = _run(op, a, w)
    assert np.array_equal(_bits(y), _bits(y32.to(torch.bfloat16)))
    ref, absprod = _oracle_product(op, a, w)
    yf = synth.bf16_to_f32(_bits(y)).astype(np.float64)
    assert np.all(np.abs(yf - ref) <= TOL * absprod + 2.0 ** -8 * np.abs(yf) + 1e-30)
    ql = mxfp4.quantize(y, scales=True, scales_mma=True)
    assert torch.equal(q["codes"], ql["codes"][0])
    assert torch.equal(q["scales"], ql["scales"][0])
    assert np.array_equal(mma_scales_to_rows(host(q["scales_mma"]), M, N // 32),
                          mma_scales_to_rows(host(ql["scales_mma"][0]), M, N // 32))


def test_fused_epilogue_strided_output_leaves_padding():
    """ldy > N: columns past N of each row keep what the caller put there."""
    rng = np.random.default_rng(41)
    a = synth.bf16_bits(rng.standard_normal((M, KW)).astype(np.float32))
    w = synth.bf16_bits((rng.standard_normal((G, NW, KW)) * 0.02).astype(np.float32))
    qa = mxfp4.quantize(dev_bf16(a), scales=False, scales_mma=True)
    qw = mxfp4.quantize(dev_bf16(w), block="32x32", scales=False, scales_mma=True)
    ybuf = torch.full((M, NW + 64), 7.0, dtype=torch.bfloat16, device="cuda")
    y, q = mxfp4.grouped_gemm_fused(mxfp4.GEMM_FPROP, _offs_dev(), qa["codes"], qa["scales_mma"], qw["codes"],
                                    qw["scales_mma"], M, NW, KW, y=ybuf[:, :NW])
    y32 = mxfp4.grouped_gemm(mxfp4.GEMM_FPROP, _offs_dev(), qa["codes"], qa["scales_mma"], qw["codes"],
                             qw["scales_mma"], M, NW, KW)
    mxfp4.mxfp4_check_device_status()
    assert torch.equal(ybuf[:, NW:], torch.full((M, 64), 7.0, dtype=torch.bfloat16, device="cuda"))
    assert np.array_equal(_bits(ybuf[:, :NW].contiguous()), _bits(y32.to(torch.bfloat16)))


def test_fused_epilogue_stochastic_rounding_exact_regime():
    """SR codes of the dgrad output (a gradient): in the exact regime the
    oracle's SR quantisation of its bf16-rounded binary64 product, bit for
    bit (element n = row * N + col of the output, the given seed and offset)."""
    op = mxfp4.GEMM_DGRAD
    rng = np.random.default_rng(51)
    a = _grid_blocks(rng, (M, NW), 1)
    w = _grid_blocks(rng, (G, NW, KW), 32)
    y, q, y32, N = _run(op, a, w, sr_seed=0x1234ABCD5678, sr_offset=17)
    ref, _ = _oracle_product(op, a, w)
    assert np.array_equal(host(y32).astype(np.float64), ref)
    y_ref = oracle.bf16_round(ref)
    c_ref, s_ref = oracle.quantize_1d(y_ref, sr=True, sr_seed=0x1234ABCD5678, sr_offset=17)
    assert np.array_equal(_bits(y), y_ref)
    assert np.array_equal(host(q["codes"]), c_ref)
    assert np.array_equal(host(q["scales"]), s_ref)


@pytest.mark.parametrize("op", [mxfp4.GEMM_FPROP, mxfp4.GEMM_DGRAD])
def test_fused_epilogue_stochastic_rounding_matches_quantiser(op):
    rng = np.random.default_rng(61 + op)
    a = synth.bf16_bits(rng.standard_normal((M, NW if op == mxfp4.GEMM_DGRAD else KW)).astype(np.float32))
    w = synth.bf16_bits((rng.standard_normal((G, NW, KW)) * 0.02).astype(np.float32))
    y, q, y32, N = _run(op, a, w, sr_seed=7, sr_offset=3)
    ql = mxfp4.quantize(y, sr_seed=7, sr_offset=3, scales=True, scales_mma=True)
    assert torch.equal(q["codes"], ql["codes"][0])
    assert torch.equal(q["scales"], ql["scales"][0])
    rn = mxfp4.quantize(y, scales=False)
    assert not torch.equal(q["codes"], rn["codes"][0]), "SR codes identical to nearest rounding"

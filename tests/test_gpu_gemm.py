"""GPU parity: the grouped block-scaled MXFP4 GEMM (tcgen05) versus a
binary64 GEMM of the oracle's own dequantised operands.  Bar: componentwise
|y - y_ref| / (|A| |B|^T) <= 1e-3 (the accumulation-order bound for binary32
sums of exact products), normwise max|dy| / max|y_ref| reported too.

Expert linears dominate compute and memory (roboaidigest "What ALTO
Actually Does"); fprop, dgrad and wgrad are the three contractions."""
import numpy as np
import pytest
import torch

import oracle
from fp4_precision_numerics_b200 import mxfp4, synth
from tests.gpu_util import dev_bf16, gemm_errors, host

pytestmark = pytest.mark.gpu
TOL = 1e-3


def _offsets_dev(offs):
    return torch.tensor(np.asarray(offs, dtype=np.int32), device="cuda")


def _fprop_case(x_bits, w_bits, offs, rht_seed=None, sr=(None, None)):
    """x_bits [M, K] (rows grouped by offs), w_bits [G, N, K]."""
    G, N, K = w_bits.shape
    M = x_bits.shape[0]
    qx = mxfp4.quantize(dev_bf16(x_bits), rht_seed=rht_seed, sr_seed=sr[0], sr_offset=0, scales=False,
                        scales_mma=True)
    qw = mxfp4.quantize(dev_bf16(w_bits), block="32x32", rht_seed=rht_seed, sr_seed=sr[1], sr_offset=1,
                        scales=False, scales_mma=True)
    y = mxfp4.grouped_gemm(mxfp4.GEMM_FPROP, _offsets_dev(offs), qx["codes"], qx["scales_mma"], qw["codes"],
                           qw["scales_mma"], M, N, K)
    mxfp4.mxfp4_check_device_status()
    y = host(y)
    # oracle: its own quantisation of the same inputs, then binary64 GEMM
    rd = 16 if rht_seed is not None else 0
    cx, sx = oracle.quantize_1d(x_bits, rht_d=rd, rht_seed=rht_seed or 0, sr=sr[0] is not None,
                                sr_seed=sr[0] or 0, sr_offset=0)
    A = oracle.dequant_1d(cx, sx)
    wr = w_bits.reshape(G * N, K)
    cw, sw = oracle.quantize_2d(wr, rht_d=rd, rht_seed=rht_seed or 0, sr=sr[1] is not None, sr_seed=sr[1] or 0,
                                sr_offset=1)
    B = oracle.dequant_2d(cw, sw).reshape(G, N, K)
    ref = oracle.grouped_gemm_f64(A, B, offs)
    absprod = oracle.grouped_gemm_f64(np.abs(A), np.abs(B), offs)
    return y, ref, absprod


@pytest.mark.parametrize("rht,sr", [(None, (None, None)), (1, (None, None)), (1, (1, 1))])
def test_single_layer_fprop(rht, sr):
    """256 x 256 layer with 1% x20 outliers: 1x32 blocks on X, 32x32 on W,
    RHT-16 on both along K; Y = X W^T, one expert, a partial N tile."""
    x, w = synth.single_layer(seed=0)
    y, ref, ap = _fprop_case(x, w[None], [0, 256], rht_seed=rht, sr=sr)
    comp, norm = gemm_errors(y, ref, ap)
    assert comp <= TOL and norm <= TOL, (comp, norm)


def test_uniform_scales_isolate_codes():
    """All-equal block scales: a mismatch here is in code layout or
    descriptors, not in the scale path."""
    rng = np.random.default_rng(3)
    grid = np.array([0, .5, 1, 1.5, 2, 3, 4, 6, -0.5, -1, -2, -6], dtype=np.float32)
    x = rng.choice(grid, size=(128, 256)).astype(np.float32)
    w = rng.choice(grid, size=(192, 256)).astype(np.float32)
    x[:, ::32] = 6.0
    w[::32, ::32] = 6.0
    w[:, ::32] = 6.0
    y, ref, ap = _fprop_case(synth.bf16_bits(x), synth.bf16_bits(w)[None], [0, 128])
    assert np.array_equal(y.astype(np.float64), ref)       # small integer sums: exact


def test_grouped_fprop_with_empty_and_ragged_groups():
    rng = np.random.default_rng(4)
    seg = [128, 0, 384, 256, 128]
    offs = np.concatenate([[0], np.cumsum(seg)])
    M, N, K = int(offs[-1]), 384, 576
    x = synth.bf16_bits(rng.standard_normal((M, K)).astype(np.float32))
    w = synth.bf16_bits((rng.standard_normal((len(seg), N, K)) * 0.02).astype(np.float32))
    y, ref, ap = _fprop_case(x, w, offs)
    comp, norm = gemm_errors(y, ref, ap)
    assert comp <= TOL and norm <= TOL, (comp, norm)


def test_dgrad_uses_transposed_weight_codes():
    """dX = dY W: B is W^T, taken from the 2D quantiser's transposed output."""
    rng = np.random.default_rng(5)
    seg = [256, 128, 0, 384]
    offs = np.concatenate([[0], np.cumsum(seg)])
    M, Nw, Kw = int(offs[-1]), 384, 320
    dy = synth.bf16_bits((rng.standard_normal((M, Nw)) * 1e-3).astype(np.float32))
    w = synth.bf16_bits((rng.standard_normal((len(seg), Nw, Kw)) * 0.02).astype(np.float32))
    qdy = mxfp4.quantize(dev_bf16(dy), sr_seed=1, sr_offset=2, scales=False, scales_mma=True)
    qw = mxfp4.quantize(dev_bf16(w), block="32x32", scales=False, scales_mma=True, transposed=True)
    dx = mxfp4.grouped_gemm(mxfp4.GEMM_DGRAD, _offsets_dev(offs), qdy["codes"], qdy["scales_mma"], qw["codes_t"],
                            qw["scales_mma_t"], M, Kw, Nw)
    mxfp4.mxfp4_check_device_status()
    cdy, sdy = oracle.quantize_1d(dy, sr=True, sr_seed=1, sr_offset=2)
    A = oracle.dequant_1d(cdy, sdy)
    Bs = []
    for g in range(len(seg)):
        cw, sw = oracle.quantize_2d(w[g])
        Bs.append(oracle.dequant_2d(cw, sw).T)                 # W^T: [Kw, Nw]
    B = np.stack(Bs)
    ref = oracle.grouped_gemm_f64(A, B, offs)
    ap = oracle.grouped_gemm_f64(np.abs(A), np.abs(B), offs)
    comp, norm = gemm_errors(host(dx), ref, ap)
    assert comp <= TOL and norm <= TOL, (comp, norm)


def test_wgrad_contracts_over_each_experts_tokens():
    """dW_g = dY_g^T X_g with RHT-16 along tokens on both operands and SR on
    dY; an empty expert gives zeros; M (= 320) leaves a ragged row tile."""
    rng = np.random.default_rng(6)
    seg = [256, 0, 128, 640]
    offs = np.concatenate([[0], np.cumsum(seg)])
    T, Nw, Kw = int(offs[-1]), 320, 192
    x = synth.bf16_bits(rng.standard_normal((T, Kw)).astype(np.float32))
    dy = synth.bf16_bits((rng.standard_normal((T, Nw)) * 1e-3).astype(np.float32))
    qx = mxfp4.quantize(dev_bf16(x), along_rows=True, rht_seed=1, sr_offset=3, scales=False, scales_mma=True)
    qdy = mxfp4.quantize(dev_bf16(dy), along_rows=True, rht_seed=1, sr_seed=1, sr_offset=4, scales=False,
                         scales_mma=True)
    dw = mxfp4.grouped_gemm(mxfp4.GEMM_WGRAD, _offsets_dev(offs), qdy["codes"], qdy["scales_mma"], qx["codes"],
                            qx["scales_mma"], Nw, Kw, T)
    mxfp4.mxfp4_check_device_status()
    cx, sx = oracle.quantize_1d_transposed(x, rht_d=16, rht_seed=1, sr_offset=3)
    cdy, sdy = oracle.quantize_1d_transposed(dy, rht_d=16, rht_seed=1, sr=True, sr_seed=1, sr_offset=4)
    Xt = oracle.dequant_1d(cx, sx)                          # [Kw, T]
    Dt = oracle.dequant_1d(cdy, sdy)                        # [Nw, T]
    dw = host(dw)
    for g in range(len(seg)):
        lo, hi = int(offs[g]), int(offs[g + 1])
        ref = Dt[:, lo:hi] @ Xt[:, lo:hi].T
        ap = np.abs(Dt[:, lo:hi]) @ np.abs(Xt[:, lo:hi]).T
        if hi == lo:
            assert np.all(dw[g] == 0.0)
            continue
        comp, norm = gemm_errors(dw[g], ref, ap)
        assert comp <= TOL and norm <= TOL, (g, comp, norm)


def test_more_than_255_groups_fprop_and_wgrad():
    """300 groups: beyond the CTA-pair kernel's group table, so the call runs
    the one-CTA kernel (128 x 192 tiles); empty and 1-3 tile groups."""
    rng = np.random.default_rng(9)
    seg = [int(v) * 128 for v in rng.choice([0, 1, 1, 2, 3], size=300)]
    offs = np.concatenate([[0], np.cumsum(seg)])
    M, N, K = int(offs[-1]), 224, 128
    x = synth.bf16_bits(rng.standard_normal((M, K)).astype(np.float32))
    w = synth.bf16_bits((rng.standard_normal((len(seg), N, K)) * 0.02).astype(np.float32))
    y, ref, ap = _fprop_case(x, w, offs)
    comp, norm = gemm_errors(y, ref, ap)
    assert comp <= TOL and norm <= TOL, (comp, norm)
    # wgrad over the same 300 token groups
    Nw, Kw = 96, 64
    a = synth.bf16_bits(rng.standard_normal((M, Nw)).astype(np.float32))
    b = synth.bf16_bits(rng.standard_normal((M, Kw)).astype(np.float32))
    qa = mxfp4.quantize(dev_bf16(a), along_rows=True, scales=False, scales_mma=True)
    qb = mxfp4.quantize(dev_bf16(b), along_rows=True, scales=False, scales_mma=True)
    dw = host(mxfp4.grouped_gemm(mxfp4.GEMM_WGRAD, _offsets_dev(offs), qa["codes"], qa["scales_mma"], qb["codes"],
                                 qb["scales_mma"], Nw, Kw, M))
    mxfp4.mxfp4_check_device_status()
    ca, sa = oracle.quantize_1d_transposed(a)
    cb, sb = oracle.quantize_1d_transposed(b)
    At, Bt = oracle.dequant_1d(ca, sa), oracle.dequant_1d(cb, sb)
    for g in range(len(seg)):
        lo, hi = int(offs[g]), int(offs[g + 1])
        if hi == lo:
            assert np.all(dw[g] == 0.0)
            continue
        comp, norm = gemm_errors(dw[g], At[:, lo:hi] @ Bt[:, lo:hi].T, np.abs(At[:, lo:hi]) @ np.abs(Bt[:, lo:hi]).T)
        assert comp <= TOL and norm <= TOL, (g, comp, norm)


def test_bad_group_offsets_flag_the_device_status():
    rng = np.random.default_rng(7)
    x = synth.bf16_bits(rng.standard_normal((256, 256)).astype(np.float32))
    w = synth.bf16_bits(rng.standard_normal((2, 192, 256)).astype(np.float32))
    qx = mxfp4.quantize(dev_bf16(x), scales=False, scales_mma=True)
    qw = mxfp4.quantize(dev_bf16(w), block="32x32", scales=False, scales_mma=True)
    bad = _offsets_dev([0, 100, 256])                        # not a multiple of 128
    mxfp4.grouped_gemm(mxfp4.GEMM_FPROP, bad, qx["codes"], qx["scales_mma"], qw["codes"], qw["scales_mma"],
                       256, 192, 256)
    with pytest.raises(mxfp4.MXFP4Error) as e:
        mxfp4.mxfp4_check_device_status()
    assert e.value.status == -6
    mxfp4.mxfp4_check_device_status()                        # cleared after reading


def test_host_rejects_bad_shapes_without_launch():
    # buffers large enough for the claimed shapes, so the library's shape
    # checks (not the binding's size checks) are what rejects the calls
    z = torch.zeros(1 << 20, dtype=torch.uint8, device="cuda")
    offs = _offsets_dev([0, 128])
    with pytest.raises(mxfp4.MXFP4Error) as e:
        mxfp4.grouped_gemm(mxfp4.GEMM_FPROP, offs, z, z, z, z, 128, 192, 100)   # K % 64
    assert e.value.status == -2
    with pytest.raises(mxfp4.MXFP4Error) as e:
        mxfp4.grouped_gemm(mxfp4.GEMM_FPROP, offs, z, z, z, z, 100, 192, 128)   # M % 128
    assert e.value.status == -2


def test_binding_rejects_undersized_or_mistyped_buffers():
    """The tensor helpers check dtype, layout and size before any call: an
    undersized operand or a wrong-dtype output raises ValueError instead of
    reaching the library as a pointer."""
    offs = _offsets_dev([0, 128])
    small = torch.zeros(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(ValueError):
        mxfp4.grouped_gemm(mxfp4.GEMM_FPROP, offs, small, small, small, small, 128, 192, 128)
    big = torch.zeros(1 << 20, dtype=torch.uint8, device="cuda")
    with pytest.raises(ValueError):
        mxfp4.grouped_gemm(mxfp4.GEMM_FPROP, offs, big, big, big, big, 128, 192, 128,
                           out=torch.zeros((128, 192), dtype=torch.bfloat16, device="cuda"))
    with pytest.raises(ValueError):
        mxfp4.grouped_gemm(mxfp4.GEMM_WGRAD, offs, big, big, big, big, 192, 192, 128,
                           out=torch.zeros((1, 96, 192), dtype=torch.float32, device="cuda"))
    x = torch.zeros((64, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError):
        mxfp4.quantize(x, out={"codes": small})
    with pytest.raises(ValueError):
        mxfp4.quantize(x.float().t(), scales=False)          # column stride != 1
    torch.cuda.synchronize()
    mxfp4.mxfp4_check_device_status()

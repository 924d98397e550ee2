"""GPU parity of the dual-direction quantiser (mxfp4_quantize_dual): one
read of an activation or gradient tensor gives the contraction-dim codes
(1x32 along the last dim) and the token-dim codes (1x32 along dim 0, with
the RHT), which must equal bit for bit the two separate quantisations, and
on a small case the oracle.  Inputs follow the MoE layer's shapes (the
abstract's hybrid 1D blocks for activations and gradients)."""
import numpy as np
import pytest
import torch

import oracle
from fp4_precision_numerics_b200 import mxfp4, synth
from tests.gpu_util import dev_bf16, dev_f32, host, mma_scales_to_rows

pytestmark = pytest.mark.gpu


def _separate(x, row_rht, col_rht, sr_seed, row_off, col_off):
    r = mxfp4.quantize(x, rht_seed=row_rht, sr_seed=sr_seed, sr_offset=row_off, scales=True, scales_mma=True)
    c = mxfp4.quantize(x, along_rows=True, rht_seed=col_rht, sr_seed=sr_seed, sr_offset=col_off, scales=True,
                       scales_mma=True)
    return r, c


def _compare(x, row_rht=None, col_rht=1, sr_seed=None, row_off=0, col_off=7):
    ro, co = mxfp4.quantize_dual(x, row_rht_seed=row_rht, col_rht_seed=col_rht, sr_seed=sr_seed,
                                 row_sr_offset=row_off, col_sr_offset=col_off, scales=True, scales_mma=True)
    r, c = _separate(x, row_rht, col_rht, sr_seed, row_off, col_off)
    torch.cuda.synchronize()
    G, T, F = (1,) + tuple(x.shape) if x.dim() == 2 else tuple(x.shape)
    for name, got, want, (Ro, Co) in (("row", ro, r, (T, F)), ("col", co, c, (F, T))):
        for k in ("codes", "scales"):
            a, b = host(got[k]), host(want[k])
            bad = np.argwhere(a != b)
            assert bad.size == 0, (name, k, bad[:5].tolist())
        for g in range(G):   # the tensor-core layout pads each 4-scale chunk: compare the defined bytes
            a = mma_scales_to_rows(host(got["scales_mma"])[g], Ro, Co // 32)
            b = mma_scales_to_rows(host(want["scales_mma"])[g], Ro, Co // 32)
            assert np.array_equal(a, b), (name, "scales_mma", g)
    return ro, co


@pytest.mark.parametrize("sr", [False, True])
@pytest.mark.parametrize("shape", [(4096, 2880), (1024, 5760), (96, 64), (4160, 2880)])
def test_dual_equals_separate_bf16(shape, sr):
    T, F = shape
    x = synth.student_t_activations(T, F, seed=3)
    _compare(dev_bf16(x), sr_seed=1 if sr else None, row_off=2, col_off=1000)


def test_dual_row_rht_and_no_col_rht():
    x = synth.student_t_activations(2048, 2880, seed=4)
    _compare(dev_bf16(x), row_rht=5, col_rht=None, sr_seed=9, row_off=1, col_off=2)


def test_dual_groups_and_f32_input():
    rng = np.random.default_rng(8)
    x = (rng.standard_normal((3, 256, 160)) * 0.3).astype(np.float32)
    for sr in (None, 4):
        _compare(dev_f32(x), sr_seed=sr)


def test_dual_moe_activation_full_size():
    """The MoE layer's routed activations (67,584 padded rows x 2880) and the
    up-projection output gradients (x 5760), as the step quantises them."""
    L = synth.moe_layer()
    _compare(dev_bf16(L["x"]), col_rht=1, row_off=0, col_off=0)
    _compare(dev_bf16(L["dy_up"]), col_rht=1, sr_seed=1, row_off=2, col_off=1000)


def test_dual_against_oracle_small():
    x = synth.student_t_activations(128, 96, seed=11)
    ro, co = mxfp4.quantize_dual(dev_bf16(x), col_rht_seed=1, sr_seed=3, row_sr_offset=4, col_sr_offset=5,
                                 scales=True, scales_mma=True)
    torch.cuda.synchronize()
    c_ref, s_ref = oracle.quantize_1d(x, sr=True, sr_seed=3, sr_offset=4)
    assert np.array_equal(host(ro["codes"])[0], c_ref)
    assert np.array_equal(host(ro["scales"])[0], s_ref)
    ct_ref, st_ref = oracle.quantize_1d_transposed(x, rht_d=16, rht_seed=1, sr=True, sr_seed=3, sr_offset=5)
    assert np.array_equal(host(co["codes"])[0], ct_ref)
    assert np.array_equal(host(co["scales"])[0], st_ref)
    assert np.array_equal(mma_scales_to_rows(host(co["scales_mma"])[0], 96, 128 // 32), st_ref)


def test_dual_rejects_bad_arguments():
    x = torch.zeros((64, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(mxfp4.MXFP4Error):
        mxfp4.quantize_dual(torch.zeros((48, 64), dtype=torch.bfloat16, device="cuda"))   # rows % 32
    L = mxfp4.lib()
    import ctypes
    rp = mxfp4.QuantParams(mxfp4.BLOCK_1X32, 0, 0, 0, mxfp4.ROUND_STOCHASTIC, 1, 0)
    cp = mxfp4.QuantParams(mxfp4.BLOCK_1X32, 1, 0, 0, mxfp4.ROUND_STOCHASTIC, 2, 0)   # different sr_seed
    o = dict(codes=torch.empty((1, 64, 32), dtype=torch.uint8, device="cuda"))
    qo = mxfp4.QuantOutputs(o["codes"].data_ptr(), None, None, None, None)
    st = L.mxfp4_quantize_dual(ctypes.c_void_p(x.data_ptr()), mxfp4.DTYPE_BF16, 1, 64, 64, 64, ctypes.byref(rp),
                               ctypes.byref(cp), ctypes.byref(qo), ctypes.byref(qo), None)
    assert st == -1   # MXFP4_ERR_INVALID_ARG

"""GPU parity at full size, in the launch configuration bench.py times: the
GPT-OSS-20B-shaped MoE expert layer (32 experts, d_model 2880, W_up
5760x2880, W_down 2880x2880, 16384 tokens top-4 with Zipf(1.1) skew), the
fused bf16 + MXFP4 epilogue of its fprop and dgrad, and the 200-step
de-oscillation stress on 32x5760x2880 fp32 masters.

The oracle cannot run the whole layer, so it checks sampled outputs one by
one: for each sampled GEMM output it quantises exactly the rows (1x32), the
32-row / 32-column slabs (2D) or the token columns (RHT + 1x32 along tokens)
that the output depends on, with the same SR counters as the full tensors,
and takes a binary64 dot product of the dequantised operands."""
import numpy as np
import pytest
import torch

import oracle
from fp4_precision_numerics_b200 import mxfp4, synth
from tests.gpu_util import dev_bf16, dev_f32, host, mma_scales_to_rows

pytestmark = pytest.mark.gpu
TOL = 1e-3
D, F = synth.D_MODEL, synth.D_FF_FUSED


def _check(y, ref, absref, what):
    err = abs(float(y) - ref)
    assert err <= TOL * absref + 1e-30, (what, float(y), ref, absref)


@pytest.fixture(scope="module")
def layer():
    return synth.moe_layer()


def test_moe_layer_full_size_sampled(layer):
    L = layer
    offs_h = L["offsets"]
    M = int(offs_h[-1])
    offs = torch.tensor(offs_h.astype(np.int32), device="cuda")
    E = len(offs_h) - 1
    rng = np.random.default_rng(11)
    x, h, dy_up, dy_down = (dev_bf16(L[k]) for k in ("x", "h", "dy_up", "dy_down"))
    w_up, w_down = dev_bf16(L["w_up"]), dev_bf16(L["w_down"])
    qwu = mxfp4.quantize(w_up, block="32x32", scales=False, scales_mma=True, transposed=True)
    qwd = mxfp4.quantize(w_down, block="32x32", scales=False, scales_mma=True, transposed=True)
    qx = mxfp4.quantize(x, scales=False, scales_mma=True)
    qh = mxfp4.quantize(h, scales=False, scales_mma=True)
    qdu = mxfp4.quantize(dy_up, sr_seed=1, sr_offset=2, scales=False, scales_mma=True)
    qdd = mxfp4.quantize(dy_down, sr_seed=1, sr_offset=3, scales=False, scales_mma=True)
    qxt = mxfp4.quantize(x, along_rows=True, rht_seed=1, scales=False, scales_mma=True)
    qht = mxfp4.quantize(h, along_rows=True, rht_seed=1, scales=False, scales_mma=True)
    qdut = mxfp4.quantize(dy_up, along_rows=True, rht_seed=1, sr_seed=1, sr_offset=1000, scales=False,
                          scales_mma=True)
    qddt = mxfp4.quantize(dy_down, along_rows=True, rht_seed=1, sr_seed=1, sr_offset=1001, scales=False,
                          scales_mma=True)
    g = mxfp4.grouped_gemm
    y_up = g(mxfp4.GEMM_FPROP, offs, qx["codes"], qx["scales_mma"], qwu["codes"], qwu["scales_mma"], M, F, D)
    y_dn = g(mxfp4.GEMM_FPROP, offs, qh["codes"], qh["scales_mma"], qwd["codes"], qwd["scales_mma"], M, D, D)
    dx = g(mxfp4.GEMM_DGRAD, offs, qdu["codes"], qdu["scales_mma"], qwu["codes_t"], qwu["scales_mma_t"], M, D, F)
    dh = g(mxfp4.GEMM_DGRAD, offs, qdd["codes"], qdd["scales_mma"], qwd["codes_t"], qwd["scales_mma_t"], M, D, D)
    dwu = g(mxfp4.GEMM_WGRAD, offs, qdut["codes"], qdut["scales_mma"], qxt["codes"], qxt["scales_mma"], F, D, M)
    dwd = g(mxfp4.GEMM_WGRAD, offs, qddt["codes"], qddt["scales_mma"], qht["codes"], qht["scales_mma"], D, D, M)
    mxfp4.mxfp4_check_device_status()
    torch.cuda.synchronize()

    def group_of(row):
        return int(np.searchsorted(offs_h, row, side="right") - 1)

    def deq_row_1d(a, row, **kw):
        c, s = oracle.quantize_1d(a[row:row + 1], row0=row, **kw)
        return oracle.dequant_1d(c, s)[0]

    def deq_w_row(w, grp, n):                       # row n of W_grp (2D blocks, 32-row slab)
        r0 = 32 * (n // 32)
        c, s = oracle.quantize_2d(w[grp, r0:r0 + 32])
        return oracle.dequant_2d(c, s)[n - r0]

    def deq_w_col(w, grp, k):                       # column k of W_grp = row k of W^T (32-column slab)
        c0 = 32 * (k // 32)
        c, s = oracle.quantize_2d(np.ascontiguousarray(w[grp][:, c0:c0 + 32]))
        return oracle.dequant_2d(c, s)[:, k - c0]

    def deq_token_col(a, col, **kw):                 # column of a, quantised along tokens with RHT
        c, s = oracle.quantize_1d_transposed(np.ascontiguousarray(a[:, col:col + 1]), rht_d=16, rht_seed=1,
                                             col0=col, **kw)
        return oracle.dequant_1d(c, s)[0]

    n_samples = 24
    rows = rng.integers(0, M, size=n_samples)
    for (name, yd, a, w, Ncols, kw_a) in (("fprop_up", y_up, L["x"], L["w_up"], F, {}),
                                          ("fprop_down", y_dn, L["h"], L["w_down"], D, {})):
        yh = host(yd[torch.from_numpy(rows).cuda()])
        cols = rng.integers(0, Ncols, size=n_samples)
        for i, (m, n) in enumerate(zip(rows, cols)):
            A = deq_row_1d(a, int(m), **kw_a)
            B = deq_w_row(w, group_of(int(m)), int(n))
            _check(yh[i, n], float(A @ B), float(np.abs(A) @ np.abs(B)), (name, m, n))
    for (name, yd, dy, w, off) in (("dgrad_up", dx, L["dy_up"], L["w_up"], 2), ("dgrad_down", dh, L["dy_down"],
                                                                                     L["w_down"], 3)):
        yh = host(yd[torch.from_numpy(rows).cuda()])
        cols = rng.integers(0, D, size=n_samples)
        for i, (m, k) in enumerate(zip(rows, cols)):
            A = deq_row_1d(dy, int(m), sr=True, sr_seed=1, sr_offset=off)
            B = deq_w_col(w, group_of(int(m)), int(k))
            _check(yh[i, k], float(A @ B), float(np.abs(A) @ np.abs(B)), (name, m, k))
    for (name, dwd_, dy, a, Mrows, off) in (("wgrad_up", dwu, L["dy_up"], L["x"], F, 1000),
                                             ("wgrad_down", dwd, L["dy_down"], L["h"], D, 1001)):
        for _ in range(8):
            grp = int(rng.integers(0, E))
            n, k = int(rng.integers(0, Mrows)), int(rng.integers(0, D))
            lo, hi = int(offs_h[grp]), int(offs_h[grp + 1])
            Dt = deq_token_col(dy, n, sr=True, sr_seed=1, sr_offset=off)[lo:hi]
            Xt = deq_token_col(a, k)[lo:hi]
            got = float(dwd_[grp, n, k].item())
            _check(got, float(Dt @ Xt), float(np.abs(Dt) @ np.abs(Xt)), (name, grp, n, k))
    # the largest and an empty-or-smallest expert both produced finite results
    assert torch.isfinite(y_up).all() and torch.isfinite(dwu).all()


def test_deosc_full_size_200_steps():
    G, R, C = synth.N_EXPERTS, F, D
    w = synth.deosc_master(groups=G, rows=R, cols=C, seed=5)
    wd = dev_f32(w)
    del w
    st = torch.zeros((G, R, C), dtype=torch.uint8, device="cuda")
    rng = np.random.default_rng(3)
    nb = 48
    blocks = [(int(rng.integers(0, G)), int(rng.integers(0, R // 32)), int(rng.integers(0, C // 32))) for _ in range(nb)]
    st_ref = np.zeros((nb, 32, 32), dtype=np.uint8)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(6)
    out = None
    for step in range(200):
        if step > 0:
            wd.add_(torch.randn(wd.shape, generator=gen, device="cuda").mul_(1e-5))
        out = mxfp4.deosc_update(wd, step, st, flip_threshold=4, scales=True, transposed=True, out=out)
        torch.cuda.synchronize()
        mb = np.stack([host(wd[g, 32 * bi:32 * bi + 32, 32 * bj:32 * bj + 32]) for g, bi, bj in blocks])
        c_ref, s_ref = oracle.deosc_update(mb, step, st_ref, flip_threshold=4)
        for i, (g, bi, bj) in enumerate(blocks):
            assert np.array_equal(host(st[g, 32 * bi:32 * bi + 32, 32 * bj:32 * bj + 32]), st_ref[i]), (step, i)
            assert np.array_equal(host(out["codes"][g, 32 * bi:32 * bi + 32, 16 * bj:16 * bj + 16]), c_ref[i]), (step, i)
            assert int(out["scales"][g, bi, bj].item()) == int(s_ref[i, 0, 0]), (step, i)
    frozen = int((st >> 7).sum().item())
    assert frozen > 0, "near-boundary weights never froze"


def test_fused_epilogue_full_size(layer):
    """fprop_up and dgrad_up of the full layer with the fused epilogue: the
    bf16 output equals the binary32 path's output rounded to bf16 and its
    codes and scales equal the library's 1x32 quantisation of that output,
    over every element; sampled outputs lie within the GEMM bound of the
    oracle's binary64 product plus half a bf16 step."""
    L = layer
    offs_h = L["offsets"]
    M = int(offs_h[-1])
    offs = torch.tensor(offs_h.astype(np.int32), device="cuda")
    x, dy_up, w_up = dev_bf16(L["x"]), dev_bf16(L["dy_up"]), dev_bf16(L["w_up"])
    qwu = mxfp4.quantize(w_up, block="32x32", scales=False, scales_mma=True, transposed=True)
    qx = mxfp4.quantize(x, scales=False, scales_mma=True)
    qdu = mxfp4.quantize(dy_up, sr_seed=1, sr_offset=2, scales=False, scales_mma=True)
    cases = (("fprop_up", mxfp4.GEMM_FPROP, qx, qwu["codes"], qwu["scales_mma"], F, D),
             ("dgrad_up", mxfp4.GEMM_DGRAD, qdu, qwu["codes_t"], qwu["scales_mma_t"], D, F))
    rng = np.random.default_rng(12)
    for name, op, qa, bc, bs, N, K in cases:
        y, q = mxfp4.grouped_gemm_fused(op, offs, qa["codes"], qa["scales_mma"], bc, bs, M, N, K)
        y32 = mxfp4.grouped_gemm(op, offs, qa["codes"], qa["scales_mma"], bc, bs, M, N, K)
        mxfp4.mxfp4_check_device_status()
        assert torch.equal(y.view(torch.int16), y32.to(torch.bfloat16).view(torch.int16)), name
        del y32
        ql = mxfp4.quantize(y, scales=True, scales_mma=True)
        assert torch.equal(q["codes"], ql["codes"][0]) and torch.equal(q["scales"], ql["scales"][0]), name
        S = N // 32   # the tensor-core layout pads the last 4-scale chunk: compare the defined bytes
        assert np.array_equal(mma_scales_to_rows(host(q["scales_mma"]), M, S),
                              mma_scales_to_rows(host(ql["scales_mma"][0]), M, S)), name
        del ql
        rows = rng.integers(0, M, size=12)
        cols = rng.integers(0, N, size=12)
        yh = host(y[torch.from_numpy(rows).cuda()].float())
        for i, (m, n) in enumerate(zip(rows, cols)):
            g = int(np.searchsorted(offs_h, m, side="right") - 1)
            if op == mxfp4.GEMM_FPROP:
                c, s = oracle.quantize_1d(L["x"][m:m + 1], row0=int(m))
                A = oracle.dequant_1d(c, s)[0]
                r0 = 32 * (n // 32)
                cw, sw = oracle.quantize_2d(L["w_up"][g, r0:r0 + 32])
                B = oracle.dequant_2d(cw, sw)[n - r0]
            else:
                c, s = oracle.quantize_1d(L["dy_up"][m:m + 1], row0=int(m), sr=True, sr_seed=1, sr_offset=2)
                A = oracle.dequant_1d(c, s)[0]
                c0 = 32 * (n // 32)
                cw, sw = oracle.quantize_2d(np.ascontiguousarray(L["w_up"][g][:, c0:c0 + 32]))
                B = oracle.dequant_2d(cw, sw)[:, n - c0]
            ref, absref = float(A @ B), float(np.abs(A) @ np.abs(B))
            err = abs(float(yh[i, n]) - ref)
            assert err <= TOL * absref + 2.0 ** -8 * abs(float(yh[i, n])) + 1e-30, (name, m, n, float(yh[i, n]), ref)
        del y, q

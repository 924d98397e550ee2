"""GPU parity at full size, in the launch configuration bench.py times: the
GPT-OSS-20B-shaped MoE expert layer (32 experts, d_model 2880, W_up
5760x2880, W_down 2880x2880, 16384 tokens top-4 with Zipf(1.1) skew), the
fused bf16 + MXFP4 epilogue of its fprop and dgrad, and the 200-step
de-oscillation stress on 32x5760x2880 fp32 masters.

Every element is compared.  The operands come from the bench's calls (the
de-oscillation re-quantisation of fp32 masters for the weights, the
dual-direction quantiser for activations and gradients) and must equal the
oracle's codes and scales bit for bit.  Every output of the six GEMMs is
checked against the binary64 product of the oracle's dequantised operands
with the componentwise bound |y - ref| <= 1e-3 (|A| |B|^T)_ij (the bound of
binary32 accumulation of exact products)."""
import numpy as np
import pytest
import torch

import oracle
from fp4_precision_numerics_b200 import mxfp4, synth
from tests.gpu_util import dev_bf16, dev_f32, host, mma_scales_to_rows, nibbles

pytestmark = pytest.mark.gpu
TOL = 1e-3
D, F = synth.D_MODEL, synth.D_FF_FUSED


@pytest.fixture(scope="module")
def layer():
    return synth.moe_layer()


@pytest.fixture(scope="module")
def step(layer):
    """The bench's launch sequence for one training step, on the layer's
    tensors: de-oscillation step 0 of the fp32 masters (the bf16 weights
    widened), the dual quantiser on X, H, dY_up, dY_down with the bench's
    seeds and offsets, and the six grouped GEMMs."""
    L = layer
    offs = torch.tensor(L["offsets"].astype(np.int32), device="cuda")
    M = int(L["offsets"][-1])
    q = {}
    for name, w in (("w_up", L["w_up"]), ("w_down", L["w_down"])):
        master = dev_bf16(w).float()
        st = torch.zeros(master.shape, dtype=torch.uint8, device="cuda")
        q[name] = mxfp4.deosc_update(master, 0, st, scales=True, scales_mma=True, transposed=True)
        q[name]["state"] = st
        del master
    kw = dict(scales=True, scales_mma=True, col_rht_seed=1)
    q["x"], q["xt"] = mxfp4.quantize_dual(dev_bf16(L["x"]), **kw)
    q["h"], q["ht"] = mxfp4.quantize_dual(dev_bf16(L["h"]), **kw)
    q["dy_up"], q["dy_up_t"] = mxfp4.quantize_dual(dev_bf16(L["dy_up"]), sr_seed=1, row_sr_offset=0,
                                                   col_sr_offset=1000, **kw)
    q["dy_down"], q["dy_down_t"] = mxfp4.quantize_dual(dev_bf16(L["dy_down"]), sr_seed=1, row_sr_offset=1,
                                                       col_sr_offset=1001, **kw)
    g = mxfp4.grouped_gemm
    out = {
        "fprop_up": g(mxfp4.GEMM_FPROP, offs, q["x"]["codes"], q["x"]["scales_mma"], q["w_up"]["codes"],
                      q["w_up"]["scales_mma"], M, F, D),
        "fprop_down": g(mxfp4.GEMM_FPROP, offs, q["h"]["codes"], q["h"]["scales_mma"], q["w_down"]["codes"],
                        q["w_down"]["scales_mma"], M, D, D),
        "dgrad_up": g(mxfp4.GEMM_DGRAD, offs, q["dy_up"]["codes"], q["dy_up"]["scales_mma"], q["w_up"]["codes_t"],
                      q["w_up"]["scales_mma_t"], M, D, F),
        "dgrad_down": g(mxfp4.GEMM_DGRAD, offs, q["dy_down"]["codes"], q["dy_down"]["scales_mma"],
                        q["w_down"]["codes_t"], q["w_down"]["scales_mma_t"], M, D, D),
        "wgrad_up": g(mxfp4.GEMM_WGRAD, offs, q["dy_up_t"]["codes"], q["dy_up_t"]["scales_mma"], q["xt"]["codes"],
                      q["xt"]["scales_mma"], F, D, M),
        "wgrad_down": g(mxfp4.GEMM_WGRAD, offs, q["dy_down_t"]["codes"], q["dy_down_t"]["scales_mma"],
                        q["ht"]["codes"], q["ht"]["scales_mma"], D, D, M),
    }
    mxfp4.mxfp4_check_device_status()
    torch.cuda.synchronize()
    return q, out


@pytest.fixture(scope="module")
def ref_operands(layer):
    """The oracle's quantisation of every operand (same seeds and offsets as
    the step): 1x32 codes/scales for both directions of the four activation
    and gradient tensors, 2D codes/scales of the weights."""
    L = layer
    r = {}
    r["x"] = oracle.quantize_1d(L["x"])
    r["h"] = oracle.quantize_1d(L["h"])
    r["dy_up"] = oracle.quantize_1d(L["dy_up"], sr=True, sr_seed=1, sr_offset=0)
    r["dy_down"] = oracle.quantize_1d(L["dy_down"], sr=True, sr_seed=1, sr_offset=1)
    r["xt"] = oracle.quantize_1d_transposed(L["x"], rht_d=16, rht_seed=1)
    r["ht"] = oracle.quantize_1d_transposed(L["h"], rht_d=16, rht_seed=1)
    r["dy_up_t"] = oracle.quantize_1d_transposed(L["dy_up"], rht_d=16, rht_seed=1, sr=True, sr_seed=1,
                                                 sr_offset=1000)
    r["dy_down_t"] = oracle.quantize_1d_transposed(L["dy_down"], rht_d=16, rht_seed=1, sr=True, sr_seed=1,
                                                   sr_offset=1001)
    for name in ("w_up", "w_down"):
        w = synth.bf16_to_f32(L[name])
        st = np.zeros(w.shape, dtype=np.uint8)
        c, s = oracle.deosc_update(w, 0, st)
        r[name] = (c, s, st)
    return r


def test_full_size_operands_bit_exact(step, ref_operands):
    """Codes and both scale layouts of every operand, all elements: the
    dual-direction quantiser (contraction dim and token dim with RHT, SR on
    the gradients) and the de-oscillation re-quantisation of the weights
    (W and W^T codes, state)."""
    q, _ = step
    r = ref_operands
    for name in ("x", "h", "dy_up", "dy_down", "xt", "ht", "dy_up_t", "dy_down_t"):
        c_ref, s_ref = r[name]
        assert np.array_equal(host(q[name]["codes"])[0], c_ref), name
        assert np.array_equal(host(q[name]["scales"])[0], s_ref), name
        Ro, S = s_ref.shape
        assert np.array_equal(mma_scales_to_rows(host(q[name]["scales_mma"])[0], Ro, S), s_ref), name
    for name in ("w_up", "w_down"):
        c_ref, s_ref, st_ref = r[name]
        G, R, C2 = c_ref.shape
        C = 2 * C2
        assert np.array_equal(host(q[name]["codes"]), c_ref), name
        assert np.array_equal(host(q[name]["scales"]), s_ref), name
        assert np.array_equal(host(q[name]["state"]), st_ref), name
        ct = host(q[name]["codes_t"])
        sm, smt = host(q[name]["scales_mma"]), host(q[name]["scales_mma_t"])
        for g in range(G):
            assert np.array_equal(nibbles(ct[g]), nibbles(c_ref[g]).T), (name, g)
            assert np.array_equal(mma_scales_to_rows(sm[g], R, C // 32), np.repeat(s_ref[g], 32, axis=0)), (name, g)
            assert np.array_equal(mma_scales_to_rows(smt[g], C, R // 32), np.repeat(s_ref[g].T, 32, axis=0)), (name, g)


def _check_every_element(y, A, B, what):
    """y (binary32, from the GPU) against A B^T in binary64, componentwise."""
    ref = A @ B.T
    bound = TOL * (np.abs(A) @ np.abs(B).T)
    err = np.abs(y.astype(np.float64) - ref)
    bad = err > bound
    if bad.any():
        i, j = np.argwhere(bad)[0]
        raise AssertionError("%s: %d of %d outputs outside the bound; first at (%d, %d): %r vs %r (bound %r)"
                             % (what, int(bad.sum()), bad.size, i, j, float(y[i, j]), ref[i, j], bound[i, j]))


def test_full_size_gemms_every_element(layer, step, ref_operands):
    """All six GEMMs of the step, every output element, per expert: fprop
    Y_e = X_e W_e^T, dgrad dX_e = dY_e W_e, wgrad dW_e = dY^T_e X^T_e^T over
    the expert's tokens (RHT on both operands along the tokens; an empty
    expert gives zeros).  Padding rows are zero inputs, so their outputs
    must be exactly zero."""
    _, out = step
    r = ref_operands
    offs = layer["offsets"]
    E = len(offs) - 1
    deq_w = {name: (lambda g, name=name: oracle.dequant_2d(r[name][0][g], r[name][1][g])) for name in ("w_up", "w_down")}
    for name, a, w, transpose in (("fprop_up", "x", "w_up", False), ("fprop_down", "h", "w_down", False),
                                  ("dgrad_up", "dy_up", "w_up", True), ("dgrad_down", "dy_down", "w_down", True)):
        y = host(out[name])
        for g in range(E):
            lo, hi = int(offs[g]), int(offs[g + 1])
            if hi == lo:
                continue
            A = oracle.dequant_1d(r[a][0][lo:hi], r[a][1][lo:hi])
            Wg = deq_w[w](g)
            _check_every_element(y[lo:hi], A, Wg.T.copy() if transpose else Wg, (name, g))
        del y
    for name, a, b in (("wgrad_up", "dy_up_t", "xt"), ("wgrad_down", "dy_down_t", "ht")):
        dw = host(out[name])
        ca, sa = r[a]
        cb, sb = r[b]
        for g in range(E):
            lo, hi = int(offs[g]), int(offs[g + 1])
            if hi == lo:
                assert not dw[g].any(), (name, g)
                continue
            A = oracle.dequant_1d(np.ascontiguousarray(ca[:, lo // 2:hi // 2]), np.ascontiguousarray(sa[:, lo // 32:hi // 32]))
            B = oracle.dequant_1d(np.ascontiguousarray(cb[:, lo // 2:hi // 2]), np.ascontiguousarray(sb[:, lo // 32:hi // 32]))
            _check_every_element(dw[g], A, B, (name, g))
        del dw


def test_deosc_full_size_200_steps():
    """The de-oscillation stress at full size: 200 steps of N(0, 1e-5)
    updates on 32x5760x2880 fp32 masters with 5% of the weights placed next
    to a bin boundary.  The oracle runs every step on the whole tensor; the
    state bytes, codes, W^T codes and both scale layouts are compared in full
    at steps 0, 1, 2, 50, 100, 150 and 199, and on 48 sampled blocks at every
    other step."""
    G, R, C = synth.N_EXPERTS, F, D
    w = synth.deosc_master(groups=G, rows=R, cols=C, seed=5)
    wd = dev_f32(w)
    del w
    st = torch.zeros((G, R, C), dtype=torch.uint8, device="cuda")
    w_host = torch.empty((G, R, C), dtype=torch.float32).pin_memory()
    wh = w_host.numpy()
    st_ref = np.zeros((G, R, C), dtype=np.uint8)
    rng = np.random.default_rng(3)
    nb = 48
    blocks = [(int(rng.integers(0, G)), int(rng.integers(0, R // 32)), int(rng.integers(0, C // 32))) for _ in range(nb)]
    full_steps = {0, 1, 2, 50, 100, 150, 199}
    gen = torch.Generator(device="cuda")
    gen.manual_seed(6)
    out = None
    for t in range(200):
        if t > 0:
            wd.add_(torch.randn(wd.shape, generator=gen, device="cuda").mul_(1e-5))
        out = mxfp4.deosc_update(wd, t, st, flip_threshold=4, scales=True, scales_mma=True, transposed=True, out=out)
        w_host.copy_(wd, non_blocking=True)
        torch.cuda.synchronize()
        c_ref, s_ref = oracle.deosc_update(wh, t, st_ref, flip_threshold=4)
        if t in full_steps:
            assert np.array_equal(host(st), st_ref), t
            assert np.array_equal(host(out["codes"]), c_ref), t
            assert np.array_equal(host(out["scales"]), s_ref), t
            ct, sm, smt = host(out["codes_t"]), host(out["scales_mma"]), host(out["scales_mma_t"])
            for g in range(G):
                assert np.array_equal(nibbles(ct[g]), nibbles(c_ref[g]).T), (t, g)
                assert np.array_equal(mma_scales_to_rows(sm[g], R, C // 32), np.repeat(s_ref[g], 32, axis=0)), (t, g)
                assert np.array_equal(mma_scales_to_rows(smt[g], C, R // 32), np.repeat(s_ref[g].T, 32, axis=0)), (t, g)
            del ct, sm, smt
        else:
            for i, (g, bi, bj) in enumerate(blocks):
                rs, cs = slice(32 * bi, 32 * bi + 32), slice(32 * bj, 32 * bj + 32)
                assert np.array_equal(host(st[g, rs, cs]), st_ref[g, rs, cs]), (t, i)
                assert np.array_equal(host(out["codes"][g, rs, 16 * bj:16 * bj + 16]), c_ref[g, rs, 16 * bj:16 * bj + 16]), (t, i)
                assert int(out["scales"][g, bi, bj].item()) == int(s_ref[g, bi, bj]), (t, i)
    mxfp4.mxfp4_check_device_status()
    frozen = int((st_ref >> 7).astype(np.int64).sum())
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

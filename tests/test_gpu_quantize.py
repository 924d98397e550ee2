"""GPU parity: fused quantisation kernels versus the CPU oracle, bit for bit
(codes, scales in both layouts, SR decisions, RHT outputs).  Inputs are the
seeded synthetic workloads of the ALTO recipe's expert layers plus edge
cases; every call goes through the C ABI of libmxfp4."""
import numpy as np
import pytest
import torch

import oracle
from fp4_precision_numerics_b200 import mxfp4, synth
from tests.gpu_util import dev_bf16, dev_f32, host, mma_scales_to_rows, nibbles

pytestmark = pytest.mark.gpu


def _check_1d(x_host, x_dev, **kw):
    rht_seed = kw.get("rht_seed")
    sr_seed = kw.get("sr_seed")
    sr_offset = kw.get("sr_offset", 0)
    out = mxfp4.quantize(x_dev, rht_seed=rht_seed, sr_seed=sr_seed, sr_offset=sr_offset, scales=True,
                         scales_mma=True)
    torch.cuda.synchronize()
    R, C = x_host.shape
    c_ref, s_ref = oracle.quantize_1d(x_host, rht_d=16 if rht_seed is not None else 0, rht_seed=rht_seed or 0,
                                      sr=sr_seed is not None, sr_seed=sr_seed or 0, sr_offset=sr_offset)
    codes = host(out["codes"])[0]
    scales = host(out["scales"])[0]
    assert np.array_equal(scales, s_ref)
    bad = np.argwhere(codes != c_ref)
    assert bad.size == 0, "first mismatches (row, byte): %s gpu %s ref %s" % (
        bad[:5].tolist(), codes[tuple(bad[:5].T)], c_ref[tuple(bad[:5].T)])
    assert np.array_equal(mma_scales_to_rows(host(out["scales_mma"])[0], R, C // 32), s_ref)


@pytest.mark.parametrize("rht", [False, True])
@pytest.mark.parametrize("sr", [False, True])
def test_single_layer_activation(rht, sr):
    x, _ = synth.single_layer(seed=0)
    _check_1d(x, dev_bf16(x), rht_seed=1 if rht else None, sr_seed=1 if sr else None, sr_offset=0)


@pytest.mark.parametrize("sr", [False, True])
def test_student_t_sweep_smallest_shape(sr):
    R, C = synth.QUANT_SWEEP_SHAPES[0]
    x = synth.student_t_activations(R, C, seed=0)
    _check_1d(x, dev_bf16(x), rht_seed=1, sr_seed=1 if sr else None, sr_offset=3)


@pytest.mark.parametrize("sr", [False, True])
def test_student_t_sweep_middle_shape(sr):
    """16384 x 2880, every element against the oracle."""
    R, C = synth.QUANT_SWEEP_SHAPES[1]
    x = synth.student_t_activations(R, C, seed=1)
    _check_1d(x, dev_bf16(x), rht_seed=1, sr_seed=1 if sr else None, sr_offset=4)


def test_student_t_largest_shape_sampled_rows():
    """65536 x 5760 at full size (the bench's launch shape), oracle on 48
    sampled rows (SR counters use the global row index)."""
    R, C = synth.QUANT_SWEEP_SHAPES[2]
    x = synth.student_t_activations(R, C, seed=0)
    xd = dev_bf16(x)
    for sr in (False, True):
        out = mxfp4.quantize(xd, rht_seed=1, sr_seed=1 if sr else None, sr_offset=5, scales=True)
        torch.cuda.synchronize()
        rows = np.sort(np.random.default_rng(0).choice(R, size=48, replace=False))
        rows[-1] = R - 1
        codes = host(out["codes"][0][torch.from_numpy(rows).cuda()])
        scales = host(out["scales"][0][torch.from_numpy(rows).cuda()])
        for i, r in enumerate(rows):
            c_ref, s_ref = oracle.quantize_1d(x[r:r + 1], rht_d=16, rht_seed=1, sr=sr, sr_seed=1, sr_offset=5,
                                              row0=int(r))
            assert np.array_equal(codes[i:i + 1], c_ref) and np.array_equal(scales[i:i + 1], s_ref), r


def test_float32_input_and_edge_values():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((64, 96)).astype(np.float32)
    x[0, :32] = 0.0                                         # all-zero block
    x[1, :32] = -0.0
    x[2, :32] = np.float32(1e-42)                           # subnormal block
    x[3, :32] = np.float32(3.0e38)                          # near the top of binary32
    x[3, 0] = -3.0e38
    x[4, :12] = [6, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.25, -5.0, 7.99, -6.01]  # ties and saturation
    x[5, 32:64] = np.float32(2.0 ** -130)
    x[5, 40] = np.float32(-2.0 ** -126)
    # with the RHT the top-of-range row would overflow binary32 (out of
    # contract: the transform must stay finite), so it is replaced there
    xr = x.copy()
    xr[3] = rng.standard_normal(96).astype(np.float32) * 1e30
    for sr in (None, 7):
        _check_1d(x, dev_f32(x), sr_seed=sr)
        _check_1d(xr, dev_f32(xr), rht_seed=11, sr_seed=sr)


def test_bf16_edge_values():
    vals = np.array([0.0, -0.0, 1e-40, -1e-40, 2.0 ** -133, 3.3e37, -3.3e37, 0.25, 0.75, 5.0, 6.0, 7.5],
                    dtype=np.float32)
    rng = np.random.default_rng(5)
    x = rng.choice(vals, size=(33, 64)).astype(np.float32)
    bits = synth.bf16_bits(x)
    for rht in (None, 2):
        for sr in (None, 3):
            _check_1d(bits, dev_bf16(bits), rht_seed=rht, sr_seed=sr)


def test_tiny_and_ragged_shapes():
    rng = np.random.default_rng(6)
    for R, C in [(1, 32), (3, 32), (5, 64), (129, 160), (257, 2880)]:
        x = synth.bf16_bits(rng.standard_normal((R, C)).astype(np.float32) * 3)
        _check_1d(x, dev_bf16(x), rht_seed=9, sr_seed=4, sr_offset=1)
        _check_1d(x, dev_bf16(x))


def test_empty_input_is_a_no_op():
    x = torch.empty((0, 64), dtype=torch.bfloat16, device="cuda")
    out = mxfp4.quantize(x)
    assert out["codes"].numel() == 0


def test_row_stride_is_honoured():
    rng = np.random.default_rng(7)
    big = synth.bf16_bits(rng.standard_normal((40, 128)).astype(np.float32))
    xd = dev_bf16(big)[:, :64]                    # ld = 128 elements
    out = mxfp4.quantize(xd, rht_seed=5, sr_seed=2)
    torch.cuda.synchronize()
    c_ref, s_ref = oracle.quantize_1d(np.ascontiguousarray(big[:, :64]), rht_d=16, rht_seed=5, sr=True, sr_seed=2)
    assert np.array_equal(host(out["codes"])[0], c_ref) and np.array_equal(host(out["scales"])[0], s_ref)


def test_grouped_rows_share_one_sr_stream():
    """[G, R, C] input: groups are back to back in the output and in the SR
    element index; tensor-core scales restart per group."""
    rng = np.random.default_rng(8)
    G, R, C = 3, 160, 96
    x = synth.bf16_bits(rng.standard_normal((G, R, C)).astype(np.float32))
    out = mxfp4.quantize(dev_bf16(x), rht_seed=1, sr_seed=6, scales_mma=True)
    torch.cuda.synchronize()
    c_ref, s_ref = oracle.quantize_1d(x.reshape(G * R, C), rht_d=16, rht_seed=1, sr=True, sr_seed=6)
    assert np.array_equal(host(out["codes"]).reshape(G * R, -1), c_ref)
    smma = host(out["scales_mma"])
    for g in range(G):
        assert np.array_equal(mma_scales_to_rows(smma[g], R, C // 32), s_ref[g * R:(g + 1) * R])


# ----------------------------------------------------------- along the token dim
@pytest.mark.parametrize("shape", [(256, 192), (1024, 2880), (384, 104), (96, 64)])
def test_transposed_quantise(shape):
    T, F = shape
    rng = np.random.default_rng(T + F)
    x = synth.bf16_bits(rng.standard_normal((T, F)).astype(np.float32) * 0.001)
    for rht, sr in [(None, None), (1, None), (1, 1), (None, 2)]:
        out = mxfp4.quantize(dev_bf16(x), along_rows=True, rht_seed=rht, sr_seed=sr, sr_offset=4, scales_mma=True)
        torch.cuda.synchronize()
        c_ref, s_ref = oracle.quantize_1d_transposed(x, rht_d=16 if rht else 0, rht_seed=rht or 0, sr=sr is not None,
                                                     sr_seed=sr or 0, sr_offset=4)
        assert np.array_equal(host(out["codes"])[0], c_ref), (rht, sr)
        assert np.array_equal(host(out["scales"])[0], s_ref), (rht, sr)
        assert np.array_equal(mma_scales_to_rows(host(out["scales_mma"])[0], F, T // 32), s_ref)


# ----------------------------------------------------------- 2D weights
@pytest.mark.parametrize("rht,sr", [(None, None), (1, None), (1, 1)])
def test_2d_weights_and_transpose(rht, sr):
    _, w = synth.single_layer(seed=0)
    rng = np.random.default_rng(1)
    w2 = synth.bf16_bits(rng.standard_normal((2, 96, 160)).astype(np.float32) * 0.02)
    for wb in (w[None], w2):
        G, R, C = wb.shape
        out = mxfp4.quantize(dev_bf16(wb), block="32x32", rht_seed=rht, sr_seed=sr, sr_offset=1, scales_mma=True,
                             transposed=True)
        torch.cuda.synchronize()
        for g in range(G):
            c_ref, s_ref = oracle.quantize_2d(wb[g], rht_d=16 if rht else 0, rht_seed=rht or 0, sr=sr is not None,
                                              sr_seed=sr or 0, sr_offset=1)
            if sr is not None and g > 0:
                # the SR element index runs over all groups back to back
                c_all, _ = oracle.quantize_2d(wb.reshape(G * R, C), rht_d=16 if rht else 0, rht_seed=rht or 0,
                                              sr=True, sr_seed=sr, sr_offset=1)
                c_ref = c_all[g * R:(g + 1) * R]
            assert np.array_equal(host(out["codes"])[g], c_ref)
            assert np.array_equal(host(out["scales"])[g], s_ref)
            per_row = np.repeat(s_ref, 32, axis=0)
            assert np.array_equal(mma_scales_to_rows(host(out["scales_mma"])[g], R, C // 32), per_row)
            assert np.array_equal(nibbles(host(out["codes_t"])[g]), nibbles(c_ref).T)
            assert np.array_equal(mma_scales_to_rows(host(out["scales_mma_t"])[g], C, R // 32),
                                  np.repeat(s_ref.T, 32, axis=0))


# ----------------------------------------------------------- standalone RHT
def _rht_ref(xh, seed, axis):
    """Oracle RHT along the last dim, or along dim 0 as the oracle's RHT of the transpose."""
    if axis == 1:
        return oracle.rht_rows(xh, seed=seed)
    return np.ascontiguousarray(oracle.rht_rows(np.ascontiguousarray(xh.T), seed=seed).T)


def _bf16_out_matches(yb, ref):
    """bf16 output against the oracle's nearest-even rounding of the binary32
    result: bit-equal where the result is a number, a NaN where it is NaN."""
    want = oracle.bf16_round(ref.astype(np.float64))
    nan = np.isnan(ref)
    got_nan = ((yb & 0x7F80) == 0x7F80) & ((yb & 0x7F) != 0)
    return np.array_equal(yb[~nan], want[~nan]) and bool(got_nan[nan].all())


@pytest.mark.parametrize("axis", [1, 0])
def test_rht_standalone(axis):
    """RHT-16 along either dim, binary32 and bf16 outputs, bf16 and binary32
    inputs, a ragged tail (77 rows along the last dim; 320 columns, not a
    multiple of the 256-thread block, along dim 0)."""
    rng = np.random.default_rng(12)
    shape = (77, 320) if axis == 1 else (96, 320)
    xf = rng.standard_normal(shape).astype(np.float32)
    xb = synth.bf16_bits(xf)
    for xh, xd in ((xb, dev_bf16(xb)), (xf, dev_f32(xf))):
        y = host(mxfp4.rht(xd, seed=21, axis=axis))
        ref = _rht_ref(xh, 21, axis)
        assert np.array_equal(y.view(np.uint32), ref.view(np.uint32))
        yb = host(mxfp4.rht(xd, seed=21, out_dtype=torch.bfloat16, axis=axis).view(torch.int16)).view(np.uint16)
        assert _bf16_out_matches(yb, ref)


@pytest.mark.parametrize("axis", [1, 0])
def test_rht_non_finite_and_overflow(axis):
    """NaN and infinity propagate through the butterfly as the oracle's
    binary32 arithmetic says, a NaN stays a NaN in the bf16 output, and
    binary32 results past the largest bf16 round to infinity there."""
    rng = np.random.default_rng(13)
    x = rng.standard_normal((64, 64)).astype(np.float32)
    x[3, 5] = np.nan
    x[17, 40] = np.inf
    x[30, 2] = -np.inf
    # chunks x_i = s_i * c (s the RHT signs): output 0 of the chunk is exactly
    # 16 c / 4 = 4c, the others 0.  4 * 0.8495e38 lies past the bf16 rounding
    # edge to infinity (3.3961e38), 4 * 0.8472e38 just below the largest bf16
    s = oracle.rht_signs(3)
    for j, c in enumerate((0.8495e38, 0.8472e38)):
        x[44, 16 * j:16 * j + 16] = (s * np.float32(c)).astype(np.float32)
        x[16 * j:16 * j + 16, 50] = (s * np.float32(c)).astype(np.float32)
    xd = dev_f32(x)
    y = host(mxfp4.rht(xd, seed=3, axis=axis))
    ref = _rht_ref(x, 3, axis)
    nan = np.isnan(ref)
    assert nan.any() and np.isinf(ref).any()
    assert np.array_equal(np.isnan(y), nan)
    assert np.array_equal(y[~nan].view(np.uint32), ref[~nan].view(np.uint32))
    yb = host(mxfp4.rht(xd, seed=3, out_dtype=torch.bfloat16, axis=axis).view(torch.int16)).view(np.uint16)
    assert _bf16_out_matches(yb, ref)
    finite = np.isfinite(ref)
    assert (np.abs(ref[finite]) >= 3.3961e38).any(), "no binary32 result rounds to a bf16 infinity"


# ----------------------------------------------------------- de-oscillation
@pytest.mark.parametrize("freeze_lower", [False, True])
@pytest.mark.parametrize("shape", [(2, 256, 512), (3, 160, 96)])
def test_deosc_steps_bit_exact(freeze_lower, shape):
    # (3, 160, 96): 5 block rows, so the kernel's last column of 8 blocks is ragged
    G, R, C = shape
    w = synth.deosc_master(groups=G, rows=R, cols=C, seed=5)
    st_ref = np.zeros((G, R, C), dtype=np.uint8)
    wd = dev_f32(w)
    st = torch.zeros((G, R, C), dtype=torch.uint8, device="cuda")
    for step in range(24):
        if step > 0:
            upd = synth.deosc_update_noise(w.shape, step, std=2e-4)
            w = (w + upd).astype(np.float32)
            wd.copy_(dev_f32(w))
        out = mxfp4.deosc_update(wd, step, st, flip_threshold=4, reset_period=10, scales_mma=True, transposed=True,
                                 freeze_lower=freeze_lower)
        torch.cuda.synchronize()
        c_ref, s_ref = oracle.deosc_update(w, step, st_ref, flip_threshold=4, reset_period=10,
                                           freeze_lower=freeze_lower)
        assert np.array_equal(host(st), st_ref), step
        assert np.array_equal(host(out["codes"]), c_ref), step
        assert np.array_equal(host(out["scales"]), s_ref), step
        for g in range(G):
            assert np.array_equal(nibbles(host(out["codes_t"])[g]), nibbles(c_ref[g]).T)
    frozen = (st_ref >> 7).sum()
    assert frozen > 0                     # the boundary weights did oscillate and freeze


@pytest.mark.parametrize("freeze_lower", [False, True])
def test_deosc_resume_bit_exact(tmp_path, freeze_lower):
    """Through the library: stop after step k, write the fp32 masters and
    the state bytes to a file, read them into fresh device buffers and
    continue.  Every later step's codes (W and W^T), scales and state equal
    the uninterrupted run's and the oracle's; the reset period falls inside
    the resumed part."""
    G, R, C = 2, 256, 512
    w0 = synth.deosc_master(groups=G, rows=R, cols=C, seed=7)
    n_steps, k = 16, 7
    kw = dict(flip_threshold=3, reset_period=10, freeze_lower=freeze_lower)

    def upd(step):
        return synth.deosc_update_noise(w0.shape, step, std=2e-4)

    wd, st = dev_f32(w0), torch.zeros((G, R, C), dtype=torch.uint8, device="cuda")
    w_ref, st_ref = w0.copy(), np.zeros((G, R, C), dtype=np.uint8)
    run = []
    for step in range(n_steps):
        if step:
            w_ref = (w_ref + upd(step)).astype(np.float32)
            wd.copy_(dev_f32(w_ref))
        out = mxfp4.deosc_update(wd, step, st, scales=True, transposed=True, **kw)
        c_ref, s_ref = oracle.deosc_update(w_ref, step, st_ref, **kw)
        torch.cuda.synchronize()
        run.append({n: host(t).copy() for n, t in out.items() if n in ("codes", "scales", "codes_t")})
        run[-1]["state"] = host(st).copy()
        assert np.array_equal(run[-1]["codes"], c_ref) and np.array_equal(run[-1]["state"], st_ref), step
    assert (run[k]["state"] >> 7).any(), "no weight froze before the checkpoint"
    del wd, st

    wd, st = dev_f32(w0), torch.zeros((G, R, C), dtype=torch.uint8, device="cuda")
    w = w0.copy()
    for step in range(k + 1):
        if step:
            w = (w + upd(step)).astype(np.float32)
            wd.copy_(dev_f32(w))
        mxfp4.deosc_update(wd, step, st, scales=True, transposed=True, **kw)
    path = tmp_path / ("deosc_step%d.npz" % k)
    np.savez(path, master=host(wd), state=host(st), step=k)
    del wd, st
    ck = np.load(path)
    wd = dev_f32(ck["master"])
    st = torch.from_numpy(ck["state"].copy()).cuda()
    w = ck["master"].copy()
    for step in range(int(ck["step"]) + 1, n_steps):
        w = (w + upd(step)).astype(np.float32)
        wd.copy_(dev_f32(w))
        out = mxfp4.deosc_update(wd, step, st, scales=True, transposed=True, **kw)
        torch.cuda.synchronize()
        for n in ("codes", "scales", "codes_t"):
            assert np.array_equal(host(out[n]), run[step][n]), (step, n)
        assert np.array_equal(host(st), run[step]["state"]), step
    mxfp4.mxfp4_check_device_status()


def test_misaligned_rows_are_rejected():
    x = torch.zeros((64, 100), dtype=torch.bfloat16, device="cuda")      # 200-byte rows
    with pytest.raises(mxfp4.MXFP4Error) as e:
        mxfp4.quantize(x, along_rows=True)
    assert e.value.status == -3


def test_bad_arguments_are_rejected_before_launch():
    x = torch.zeros((4, 48), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(mxfp4.MXFP4Error) as e:
        mxfp4.quantize(x)
    assert e.value.status == -2
    y = torch.zeros((4, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(mxfp4.MXFP4Error) as e:
        mxfp4.quantize(y, block="32x32")
    assert e.value.status == -2

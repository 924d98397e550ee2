"""Pins for the oracle's tensor-level quantisation (hybrid 1D/2D blocks of
the abstract), de-oscillation traces and binary64 GEMM.  Hand-worked
examples, invariants and the textbook matrix product."""
import numpy as np
import pytest

import oracle
from fp4_precision_numerics_b200 import synth


def nib(codes: np.ndarray) -> np.ndarray:
    """Unpack [R, C/2] bytes into [R, C] 4-bit codes (low nibble = even col)."""
    lo = codes & 0x0F
    hi = codes >> 4
    return np.stack([lo, hi], axis=-1).reshape(codes.shape[0], -1)


def test_hand_worked_block():
    # amax 6 -> E = 0, scale byte 127; values on the grid map to their codes
    row = np.zeros((1, 32), dtype=np.float32)
    row[0, :8] = [6.0, -3.0, 1.5, 0.5, -0.5, 0.0, -0.0, 4.0]
    row[0, 8:12] = [0.25, 0.75, 2.5, -5.0]           # ties to the even code
    codes, scales = oracle.quantize_1d(row)
    assert scales[0, 0] == 127
    c = nib(codes)[0]
    assert list(c[:8]) == [7, 8 | 5, 3, 1, 8 | 1, 0, 8, 6]
    assert list(c[8:12]) == [0, 2, 4, 8 | 6]
    # amax 12 -> floor(log2 12) = 3 -> E = 1, values halve before rounding
    row2 = row * 2
    codes2, scales2 = oracle.quantize_1d(row2)
    assert scales2[0, 0] == 128
    assert np.array_equal(codes2, codes)
    # all-zero block: scale byte 0 (E = -127), codes zero
    z = np.zeros((1, 32), dtype=np.float32)
    cz, sz = oracle.quantize_1d(z)
    assert sz[0, 0] == 0 and np.all(cz == 0)


def test_bf16_input_widens_exactly():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((16, 64)).astype(np.float32)
    bits = synth.bf16_bits(x)
    c1, s1 = oracle.quantize_1d(bits)
    c2, s2 = oracle.quantize_1d(synth.bf16_to_f32(bits))
    assert np.array_equal(c1, c2) and np.array_equal(s1, s2)


def test_requantising_dequantised_values_is_identity():
    rng = np.random.default_rng(2)
    x = (rng.standard_normal((32, 128)) * 3).astype(np.float32)
    codes, scales = oracle.quantize_1d(x)
    deq = oracle.dequant_1d(codes, scales).astype(np.float32)
    c2, s2 = oracle.quantize_1d(deq)
    # the block max (|v| in [4, 8)) dequantises to 4 or 6 times the scale, so
    # the scale is re-derived unchanged and on-grid values keep their codes
    assert np.array_equal(oracle.dequant_1d(c2, s2), oracle.dequant_1d(codes, scales))
    assert np.array_equal(c2, codes) and np.array_equal(s2, scales)


def test_slices_draw_the_same_sr_bits():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((64, 96)).astype(np.float32)
    full_c, full_s = oracle.quantize_1d(x, rht_d=16, rht_seed=5, sr=True, sr_seed=1, sr_offset=2)
    part_c, part_s = oracle.quantize_1d(x[20:37], rht_d=16, rht_seed=5, sr=True, sr_seed=1, sr_offset=2,
                                        row0=20)
    assert np.array_equal(full_c[20:37], part_c) and np.array_equal(full_s[20:37], part_s)


def test_transposed_is_quantise_of_transpose():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((64, 48)).astype(np.float32)
    ct, st = oracle.quantize_1d_transposed(x, rht_d=16, rht_seed=7, sr=True, sr_seed=1, sr_offset=3)
    c, s = oracle.quantize_1d(np.ascontiguousarray(x.T), rht_d=16, rht_seed=7, sr=True, sr_seed=1, sr_offset=3)
    assert np.array_equal(ct, c) and np.array_equal(st, s)


def test_2d_blocks_share_codes_with_transpose():
    """32x32 blocks: quantising W^T gives the nibble-transpose of W's codes
    and the transpose of its scale grid (W and W^T share codes)."""
    rng = np.random.default_rng(5)
    w = (rng.standard_normal((96, 160)) * 0.02).astype(np.float32)
    c, s = oracle.quantize_2d(w)
    ct, stt = oracle.quantize_2d(np.ascontiguousarray(w.T))
    assert np.array_equal(nib(ct), nib(c).T)
    assert np.array_equal(stt, s.T)


def test_2d_scale_is_block_max_rule():
    rng = np.random.default_rng(6)
    w = (rng.standard_normal((64, 64)) * 0.02).astype(np.float32)
    _, s = oracle.quantize_2d(w)
    for bi in range(2):
        for bj in range(2):
            amax = float(np.abs(w[32 * bi:32 * bi + 32, 32 * bj:32 * bj + 32]).max())
            m, e = np.frexp(amax)
            assert s[bi, bj] == (e - 1) - 2 + 127


def _block_with(value_at_0_0: float, amax: float = 6.0) -> np.ndarray:
    w = np.zeros((1, 32, 32), dtype=np.float32)
    w[0, 31, 31] = amax                   # pins the block scale at 1
    w[0, 0, 0] = value_at_0_0
    return w


def test_deosc_freezes_after_threshold_flips():
    """A weight alternating across the 1.25 boundary (codes 2 <-> 3) flips on
    every step; with threshold 4 it freezes at the 4th flip and then keeps
    emitting the code it froze at."""
    st = np.zeros((1, 32, 32), dtype=np.uint8)
    seq = [1.2, 1.3, 1.2, 1.3, 1.2, 1.3, 1.2]
    emitted = []
    for t, v in enumerate(seq):
        codes, scales = oracle.deosc_update(_block_with(v), t, st, flip_threshold=4)
        assert scales[0, 0, 0] == 127
        emitted.append(int(codes[0, 0, 0] & 0x0F))
        if t == 0:
            assert st[0, 0, 0] == 2                        # initial: RN code, count 0
    # t=1..4 flip (count 1..4); frozen after t=4 holding code 2
    assert emitted == [2, 3, 2, 3, 2, 2, 2]
    assert (st[0, 0, 0] >> 7) == 1 and ((st[0, 0, 0] >> 4) & 7) == 4 and (st[0, 0, 0] & 0xF) == 2


def test_deosc_monotone_drift_does_not_freeze():
    st = np.zeros((1, 32, 32), dtype=np.uint8)
    for t, v in enumerate([0.9, 1.3, 1.8, 2.6, 3.6]):     # codes 2, 3, 4, 5, 6: 4 changes
        codes, _ = oracle.deosc_update(_block_with(v), t, st, flip_threshold=5)
        assert (codes[0, 0, 0] & 0xF) == [2, 3, 4, 5, 6][t]
    assert (st[0, 0, 0] >> 7) == 0 and ((st[0, 0, 0] >> 4) & 7) == 4


def test_deosc_reset_period_unfreezes():
    st = np.zeros((1, 32, 32), dtype=np.uint8)
    seq = [1.2, 1.3, 1.2, 1.3]
    for t, v in enumerate(seq):
        oracle.deosc_update(_block_with(v), t, st, flip_threshold=2, reset_period=0)
    assert (st[0, 0, 0] >> 7) == 1
    codes, _ = oracle.deosc_update(_block_with(1.3), 4, st, flip_threshold=2, reset_period=4)
    assert (codes[0, 0, 0] & 0xF) == 3 and (st[0, 0, 0] >> 7) == 0


def test_deosc_frozen_code_follows_new_scale():
    """Frozen weights keep their code; the scale tracks the master weights."""
    st = np.zeros((1, 32, 32), dtype=np.uint8)
    for t, v in enumerate([1.2, 1.3, 1.2]):
        oracle.deosc_update(_block_with(v), t, st, flip_threshold=2)
    w = _block_with(1.3, amax=12.0)                      # scale doubles
    codes, scales = oracle.deosc_update(w, 3, st, flip_threshold=2)
    assert scales[0, 0, 0] == 128 and (codes[0, 0, 0] & 0xF) == 2


def test_deosc_freeze_lower_keeps_the_smaller_code():
    """Variant: a weight alternating 1.3 / 1.2 (codes 3 <-> 2) freezes at its
    4th flip (t = 4, new code 3, old code 2).  The default rule freezes the
    new code 3; freeze_lower freezes 2, the lower magnitude, and emits it
    from the freezing step on."""
    seq = [1.3, 1.2, 1.3, 1.2, 1.3, 1.2, 1.3]
    for lower, want_frozen in ((False, 3), (True, 2)):
        st = np.zeros((1, 32, 32), dtype=np.uint8)
        emitted = []
        for t, v in enumerate(seq):
            codes, _ = oracle.deosc_update(_block_with(v), t, st, flip_threshold=4, freeze_lower=lower)
            emitted.append(int(codes[0, 0, 0] & 0x0F))
        assert emitted == [3, 2, 3, 2, want_frozen, want_frozen, want_frozen]
        assert (st[0, 0, 0] >> 7) == 1 and (st[0, 0, 0] & 0xF) == want_frozen


def test_deosc_freeze_lower_tie_keeps_the_new_code():
    """+-0.5 (codes 1 and 9) have equal magnitude: the new code is kept."""
    st = np.zeros((1, 32, 32), dtype=np.uint8)
    emitted = []
    for t, v in enumerate([0.4, -0.4, 0.4, -0.4]):
        codes, _ = oracle.deosc_update(_block_with(v), t, st, flip_threshold=2, freeze_lower=True)
        emitted.append(int(codes[0, 0, 0] & 0x0F))
    assert emitted == [1, 9, 1, 1]                       # freezes at t = 2 on the new code (+0.5)
    assert (st[0, 0, 0] >> 7) == 1 and (st[0, 0, 0] & 0xF) == 1


def test_dequant_closed_form():
    codes = np.array([[0x7F, 0x08]], dtype=np.uint8)           # codes 15, 7, 8, 0
    d = oracle.dequant_1d(np.tile(codes, (1, 8)), np.array([[130]], dtype=np.uint8))
    assert list(d[0, :4]) == [-6 * 8.0, 6 * 8.0, -0.0, 0.0]
    assert np.signbit(d[0, 2]) and not np.signbit(d[0, 3])
    d2 = oracle.dequant_2d(np.full((32, 16), 0x21, dtype=np.uint8), np.array([[125]], dtype=np.uint8))
    assert np.all(d2[:, 0::2] == 0.5 * 0.25) and np.all(d2[:, 1::2] == 1.0 * 0.25)


def test_gemm_loop_matches_numpy_and_hand_dot():
    x, w = synth.single_layer(seed=0, n=64)
    cx, sx = oracle.quantize_1d(x, rht_d=16, rht_seed=1)
    cw, sw = oracle.quantize_2d(w, rht_d=16, rht_seed=1)
    A = oracle.dequant_1d(cx, sx)
    B = oracle.dequant_2d(cw, sw)
    C_loop = oracle.gemm_f64_loop(A, B)
    C_np = oracle.gemm_f64(A, B)
    assert np.allclose(C_loop, C_np, rtol=1e-12, atol=1e-12)
    hand = sum(float(A[3, k]) * float(B[5, k]) for k in range(64))
    assert abs(C_loop[3, 5] - hand) <= 1e-12 * max(1.0, abs(hand))


def test_grouped_gemm_segments():
    rng = np.random.default_rng(9)
    A = rng.standard_normal((10, 8))
    B = rng.standard_normal((3, 5, 8))
    offs = [0, 4, 4, 10]
    C = oracle.grouped_gemm_f64(A, B, offs)
    assert np.allclose(C[:4], A[:4] @ B[0].T) and np.allclose(C[4:], A[4:] @ B[2].T)


def test_oracle_is_unchanged_at_O0():
    """The C oracle built at -O0 gives the same bits as the -O2 build on every
    step (RHT, 1D/2D quantisation with RN and SR, the transposed layout,
    de-oscillation over three steps, the binary64 GEMM loop): no result
    depends on undefined behaviour, uninitialised memory or optimisation."""
    import os
    import subprocess

    def run_all():
        rng = np.random.default_rng(11)
        x = synth.bf16_bits((rng.standard_normal((64, 96)) * 3).astype(np.float32))
        out = [oracle.rht_rows(x, 5)]
        out += list(oracle.quantize_1d(x, rht_d=16, rht_seed=5, sr=True, sr_seed=9, sr_offset=2))
        out += list(oracle.quantize_1d_transposed(x, rht_d=16, rht_seed=5, sr=True, sr_seed=9, sr_offset=3))
        out += list(oracle.quantize_2d(x))
        m = (rng.standard_normal((2, 64, 64)) * 0.02).astype(np.float32)
        st = np.zeros(m.shape, dtype=np.uint8)
        for step in range(3):
            out += list(oracle.deosc_update(m + np.float32(1e-3 * step), step, st))
            out.append(st.copy())
        A, B = rng.standard_normal((8, 64)), rng.standard_normal((5, 64))
        out.append(oracle.gemm_f64_loop(A, B))
        return out

    ref = run_all()
    so0 = os.path.join(oracle._BUILD, "libmxfp4_oracle_O0.so")
    subprocess.check_call(["gcc", "-O0", "-std=gnu11", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-fPIC",
                           "-shared", "-o", so0, oracle._SRC, "-lm"])
    saved = (oracle._SO, oracle._lib)
    try:
        oracle._SO, oracle._lib = so0, None
        got = run_all()
    finally:
        oracle._SO, oracle._lib = saved
    assert len(got) == len(ref)
    for a, b in zip(ref, got):
        assert a.dtype == b.dtype and np.array_equal(a.view(np.uint8), b.view(np.uint8))


@pytest.mark.parametrize("freeze_lower", [False, True])
def test_deosc_resume_equivalence(tmp_path, freeze_lower):
    """The fp32 master weights and the one state byte per weight are the whole
    de-oscillation state: stopping after step k, writing both to a file,
    reading them back into fresh arrays and continuing gives, at every later
    step, the same codes, scales and state as the run that never stopped
    (the reset period falls inside the resumed part, so the step number is
    carried too)."""
    G, R, C = 2, 64, 96
    w0 = synth.deosc_master(groups=G, rows=R, cols=C, seed=7)
    n_steps, k, kw = 15, 7, dict(flip_threshold=3, reset_period=10, freeze_lower=freeze_lower)

    def update(w, step):
        return (w + synth.deosc_update_noise(w.shape, step, std=2e-4)).astype(np.float32)

    w, st = w0.copy(), np.zeros((G, R, C), dtype=np.uint8)
    ref = []
    for step in range(n_steps):
        if step:
            w = update(w, step)
        c, s = oracle.deosc_update(w, step, st, **kw)
        ref.append((c, s, st.copy()))
    assert (ref[-1][2] >> 7).any() and (ref[k][2] >> 7).any(), "no weight froze: the test would not exercise the state"

    w, st = w0.copy(), np.zeros((G, R, C), dtype=np.uint8)
    for step in range(k + 1):
        if step:
            w = update(w, step)
        oracle.deosc_update(w, step, st, **kw)
    path = tmp_path / ("deosc_step%d.npz" % k)
    np.savez(path, master=w, state=st, step=k)
    del w, st
    ck = np.load(path)
    w, st, k2 = ck["master"].copy(), ck["state"].copy(), int(ck["step"])
    assert k2 == k
    for step in range(k + 1, n_steps):
        w = update(w, step)
        c, s = oracle.deosc_update(w, step, st, **kw)
        assert np.array_equal(c, ref[step][0]) and np.array_equal(s, ref[step][1]), step
        assert np.array_equal(st, ref[step][2]), step

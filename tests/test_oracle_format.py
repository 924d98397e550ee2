"""Pins for the oracle's E2M1 element format, scale rule and nearest
rounding (MX format named on roboaidigest "What ALTO Actually Does": E2M1
values with one UE8M0 scale per block).  Each check compares the oracle with
something other than itself: the bit-level definition of E2M1, CUDA's own
host conversion in cuda_fp4.h, Python's binary64 frexp, and brute force."""
import math

import numpy as np
import pytest

import oracle
from fp4_precision_numerics_b200 import synth


def e2m1_decode_bits(code: int) -> float:
    """E2M1 from its bit fields: 1 sign, 2 exponent (bias 1), 1 mantissa bit;
    exponent field 0 is subnormal (0 or 0.5)."""
    s = (code >> 3) & 1
    e = (code >> 1) & 3
    m = code & 1
    mag = m * 0.5 if e == 0 else (1.0 + m / 2.0) * 2.0 ** (e - 1)
    return -mag if s else mag


def test_grid_matches_bit_definition():
    for code in range(16):
        assert oracle.e2m1_value(code) == e2m1_decode_bits(code)
    mags = sorted({abs(e2m1_decode_bits(c)) for c in range(16)})
    assert mags == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def test_grid_points_roundtrip_rn_and_sr():
    for code in range(16):
        v = e2m1_decode_bits(code)
        assert oracle.e2m1_rn(v) == code
        for r in (0, 1, 0x7FFF, 0xFFFF):
            assert oracle.e2m1_sr(v, r) == code     # on the grid: f = 0, never rounds up


def test_rn_ties_to_even_code():
    # midpoints between adjacent magnitudes: the even code wins
    expect = {0.25: 0, 0.75: 2, 1.25: 2, 1.75: 4, 2.5: 4, 3.5: 6, 5.0: 6}
    for v, c in expect.items():
        assert oracle.e2m1_rn(v) == c
        assert oracle.e2m1_rn(-v) == c | 8


def test_rn_saturates_and_keeps_sign_of_zero():
    assert oracle.e2m1_rn(6.0) == 7
    assert oracle.e2m1_rn(7.999) == 7
    assert oracle.e2m1_rn(-1e30) == 15
    assert oracle.e2m1_rn(0.0) == 0
    assert oracle.e2m1_rn(-0.0) == 8
    assert oracle.e2m1_rn(-0.1) == 8
    assert oracle.e2m1_rn(1e-45) == 0


def test_rn_matches_cuda_fp4_host_conversion(cuda_fp4_rn):
    rng = np.random.default_rng(123)
    dense = np.linspace(-8.0, 8.0, 40001, dtype=np.float32)
    near = np.array([m + d for m in (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0)
                     for d in (-2e-7, -1e-7, 0.0, 1e-7, 2e-7)], dtype=np.float32)
    special = np.array([0.0, -0.0, 1e-45, -1e-45, 1e-38, -1e-38, 6.0, -6.0, 7.9999, 100.0, -100.0],
                       dtype=np.float32)
    rand = rng.uniform(-8, 8, size=20000).astype(np.float32)
    xs = np.concatenate([dense, near, -near, special, rand])
    ref = cuda_fp4_rn(xs)
    ours = np.array([oracle.e2m1_rn(float(v)) for v in xs], dtype=np.uint8)
    bad = np.nonzero(ref != ours)[0]
    assert bad.size == 0, list(zip(xs[bad][:10], ours[bad][:10], ref[bad][:10]))


def test_rn_brute_force_nearest():
    rng = np.random.default_rng(7)
    for v in rng.uniform(-7.5, 7.5, size=3000).astype(np.float32):
        a = min(abs(float(v)), 6.0)
        dists = [abs(a - abs(e2m1_decode_bits(c))) for c in range(8)]
        best = min(dists)
        cands = [c for c in range(8) if dists[c] == best]
        want = [c for c in cands if c % 2 == 0][0] if len(cands) > 1 else cands[0]
        got = oracle.e2m1_rn(float(v))
        assert got & 7 == want
        assert (got >> 3) == (1 if math.copysign(1.0, float(v)) < 0 else 0)


def _floor_log2(a: float) -> int:
    m, e = math.frexp(a)
    return e - 1


@pytest.mark.parametrize("amax", [
    1.0, 4.0, 6.0, 7.99999, 8.0, 0.5, 0.75, 1e-3, 3.0e38,
    float(np.float32(2.0 ** -133)),           # smallest bf16 subnormal
    float(np.float32(2.0 ** -126)),           # smallest fp32 normal
    float(np.float32(1.5 * 2.0 ** -140)),     # fp32 subnormal
    float(np.float32(6.0 * 2.0 ** 20)), float(np.nextafter(np.float32(8.0 * 2 ** 20), np.float32(0))),
])
def test_scale_rule_closed_form(amax):
    want = max(-127, min(127, _floor_log2(amax) - 2))
    assert oracle.scale_exponent(amax) == want


def test_scale_rule_special_cases():
    assert oracle.scale_exponent(0.0) == -127            # all-zero block: smallest scale
    assert oracle.scale_exponent(6.0) == 0                # 6 = 1.5 * 2^2 maps to scale 1
    assert oracle.scale_exponent(1.0) == -2
    assert oracle.scale_exponent(float(np.float32(2.0 ** -133))) == -127   # clamped
    bf16_max = float(np.float32((2 - 2 ** -7) * 2.0 ** 127))
    assert oracle.scale_exponent(bf16_max) == 125


def test_scaled_block_max_in_4_to_8():
    """After scaling by 2^-E the block maximum lies in [4, 8): saturation
    only ever touches |v| in (6, 8)."""
    rng = np.random.default_rng(3)
    for amax in np.exp(rng.uniform(-80, 80, size=2000)).astype(np.float32):
        if not np.isfinite(amax) or amax == 0:
            continue
        E = oracle.scale_exponent(float(amax))
        v = float(np.float32(np.ldexp(np.float32(amax), -E)))
        assert 4.0 <= v < 8.0


def test_rn_error_bound_on_tensor():
    """Nearest rounding: every element within half a grid step (times the
    block scale) of its input, or saturated."""
    rng = np.random.default_rng(11)
    x = rng.standard_normal((64, 256)).astype(np.float32)
    codes, scales = oracle.quantize_1d(x)
    deq = oracle.dequant_1d(codes, scales)
    E = scales.astype(np.int64) - 127
    scale = np.repeat(np.ldexp(1.0, E), 32, axis=1)
    v = x / scale
    err = np.abs(deq - x) / scale
    halfstep = np.where(np.abs(v) < 2, 0.25, np.where(np.abs(v) < 4, 0.5, 1.0))
    sat = np.abs(v) > 6
    assert np.all(err[~sat] <= halfstep[~sat] + 1e-12)
    assert np.all(np.abs(deq[sat]) == 6 * scale[sat])


# ---------------------------------------------------------------- bf16 output rounding
def test_bf16_round_fixes_every_finite_bf16():
    """Every finite bf16 value is already representable: it maps to itself."""
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    vals = (bits.astype(np.uint32) << 16).view(np.float32)
    keep = np.isfinite(vals)
    assert np.array_equal(oracle.bf16_round(vals[keep].astype(np.float64)), bits[keep])


def test_bf16_round_matches_torch_conversion_of_binary32():
    """On binary32 inputs (exact in binary64) the rounding is torch's
    float32 -> bfloat16 conversion: random bit patterns over the whole
    exponent range, exact halfway cases of both parities, subnormals and the
    overflow edge."""
    import torch
    rng = np.random.default_rng(17)
    u = rng.integers(0, 1 << 32, size=200000, dtype=np.uint64).astype(np.uint32)
    ties = (rng.integers(0, 1 << 16, size=20000, dtype=np.uint64).astype(np.uint32) << 16) | 0x8000
    sub = rng.integers(0, 1 << 23, size=20000, dtype=np.uint64).astype(np.uint32)
    edge = np.array([0x7F7F7FFF, 0x7F7F8000, 0x7F7FFFFF, 0x7F7F0000, 0x00000000, 0x80000000, 0x00008000,
                     0x00018000, 0x3F808000, 0x3F818000], dtype=np.uint32)
    u = np.concatenate([u, ties, sub, sub | 0x80000000, edge])
    x = u.view(np.float32)
    x = x[np.isfinite(x)]
    ref = torch.from_numpy(x.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(oracle.bf16_round(x.astype(np.float64)), ref)


def test_bf16_round_rounds_once_from_binary64():
    """A binary64 value just above a bf16 halfway point rounds up, where a
    detour through binary32 would land on the tie and round to even."""
    t = 2.0 ** -30
    cases = {1 + 2 ** -8 + t: 0x3F81, 1 + 2 ** -8: 0x3F80, 1 + 3 * 2 ** -8: 0x3F82, -(1 + 2 ** -8 + t): 0xBF81,
             2.0 ** 128 - 2.0 ** 119: 0x7F80, 2.0 ** 128 - 2.0 ** 119 - 2.0 ** 100: 0x7F7F,
             2.0 ** -134 + 2.0 ** -160: 0x0001, 2.0 ** -134: 0x0000}
    got = oracle.bf16_round(np.array(list(cases), dtype=np.float64))
    assert [int(g) for g in got] == list(cases.values())


def test_operand_footprint_is_a_quarter_of_bf16():
    """roboaidigest "What ALTO Actually Does": E2M1 values with per-block
    UE8M0 scales give a theoretical 4x smaller operand than BF16.  The
    oracle's packing: two codes per byte (exactly a quarter of the bf16
    bytes), plus one scale byte per 32 elements (4.25 bits per element, a
    16/4.25 = 3.76x reduction with scales; 1/1024 byte per element for the
    32x32 weight blocks)."""
    rng = np.random.default_rng(3)
    x = synth.bf16_bits(rng.standard_normal((64, 256)).astype(np.float32))
    codes, scales = oracle.quantize_1d(x)
    assert codes.dtype == np.uint8 and scales.dtype == np.uint8
    assert codes.nbytes * 4 == x.nbytes
    assert (codes.nbytes + scales.nbytes) * 8 == x.size * 4.25
    assert abs(x.nbytes / (codes.nbytes + scales.nbytes) - 16 / 4.25) < 1e-12
    c2, s2 = oracle.quantize_2d(x)
    assert c2.nbytes * 4 == x.nbytes and s2.nbytes * 1024 == x.size

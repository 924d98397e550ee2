"""Pins for the oracle's Philox stream, randomized Hadamard transform and
stochastic rounding (both named by the abstract as recipe techniques).
References: curand's host-side Philox4x32-10, the closed-form Sylvester
matrix, binary64 arithmetic and statistics."""
import numpy as np

import oracle


def test_philox_matches_curand(curand_philox):
    rng = np.random.default_rng(0)
    n = 10000
    ctr = rng.integers(0, 2 ** 32, size=(n, 4), dtype=np.uint64)
    key = rng.integers(0, 2 ** 32, size=(n, 2), dtype=np.uint64)
    ctr[:8] = 0
    key[:8] = 0
    ctr[8] = 0xFFFFFFFF
    key[8] = 0xFFFFFFFF
    ref = curand_philox(ctr, key)
    ours = np.stack([oracle.philox4x32_10(c, k) for c, k in zip(ctr, key)])
    assert np.array_equal(ref, ours)


def _rev16(u):
    return int(format(u, "016b")[::-1], 2)


def test_sr_bits_are_curand_words(curand_philox):
    """Element n draws 16 bits of word (n>>2)&3 of Philox(key=seed,
    ctr=(n>>4 lo, hi, offset, 0)): with bytes b0..b3 of that word, elements
    4m..4m+3 take b2:b0, its bit reversal, b3:b1, its bit reversal."""
    seed, offset = 0x1234_5678_9ABC_DEF0, 7
    ns = [0, 1, 2, 3, 4, 5, 6, 7, 12, 13, 14, 15, 16, 31, 1 << 33, (1 << 40) + 5, (1 << 40) + 10]
    ctr = np.array([[(n >> 4) & 0xFFFFFFFF, (n >> 4) >> 32, offset, 0] for n in ns], dtype=np.uint64)
    key = np.array([[seed & 0xFFFFFFFF, seed >> 32]] * len(ns), dtype=np.uint64)
    words = curand_philox(ctr, key)
    for n, w in zip(ns, words):
        word = int(w[(n >> 2) & 3])
        b = [(word >> (8 * i)) & 0xFF for i in range(4)]
        even, odd = (b[2] << 8) | b[0], (b[3] << 8) | b[1]
        want = [even, _rev16(even), odd, _rev16(odd)][n & 3]
        assert oracle.sr_bits16(seed, offset, n) == want, n


def test_sr_bits_uniform_and_pairwise_uncorrelated():
    """Every element's 16-bit draw is uniform (each bit is set half the time)
    and the bit-reversed partner is uncorrelated with it in value."""
    seed, offset = 5, 3
    n = np.arange(0, 4 * 20000)
    r = np.array([oracle.sr_bits16(seed, offset, int(i)) for i in n], dtype=np.float64)
    for j in range(4):
        rj = r[j::4]
        assert abs(rj.mean() / 65536 - 0.5) < 0.01
        for bit in (0, 7, 15):
            assert abs(np.mean((rj.astype(np.int64) >> bit) & 1) - 0.5) < 0.02
    for a, b in ((0, 1), (2, 3), (0, 2)):
        c = np.corrcoef(r[a::4], r[b::4])[0, 1]
        assert abs(c) < 0.03, (a, b, c)


def test_rht_signs_are_curand_bits(curand_philox):
    for seed in (0, 1, 0xDEADBEEF, (1 << 40) + 3):
        w = curand_philox(np.array([[0, 0, 0, 1]], dtype=np.uint64),
                          np.array([[seed & 0xFFFFFFFF, seed >> 32]], dtype=np.uint64))[0]
        want = np.array([-1.0 if (int(w[0]) >> i) & 1 else 1.0 for i in range(16)], dtype=np.float32)
        assert np.array_equal(oracle.rht_signs(seed), want)


def sylvester16():
    i = np.arange(16)
    par = np.array([[bin(a & b).count("1") & 1 for b in i] for a in i])
    return np.where(par == 1, -1.0, 1.0)


def test_rht_unit_vectors_give_hadamard_rows():
    """With all signs +1, e_i maps to row i of H16/4 exactly; H H^T = 16 I."""
    H = sylvester16()
    assert np.array_equal(H @ H.T, 16 * np.eye(16))
    ones = np.ones(16, dtype=np.float32)
    for i in range(16):
        e = np.zeros(16, dtype=np.float32)
        e[i] = 1.0
        assert np.array_equal(oracle.rht16(e, ones), (H[i] / 4).astype(np.float32))


def test_rht_matches_dense_f64_within_rounding_bound():
    rng = np.random.default_rng(5)
    u = 2.0 ** -24
    for _ in range(500):
        x = (rng.standard_normal(16) * np.exp(rng.uniform(-20, 20))).astype(np.float32)
        s = np.where(rng.random(16) < 0.5, -1.0, 1.0).astype(np.float32)
        y = oracle.rht16(x, s).astype(np.float64)
        yd = oracle.rht16_dense_f64(x.astype(np.float64), s.astype(np.float64))
        yref = (s.astype(np.float64) * x.astype(np.float64)) @ sylvester16() / 4
        assert np.allclose(yd, yref, rtol=0, atol=1e-300 + 1e-15 * np.abs(x).sum())
        bound = 4 * u * np.abs(x.astype(np.float64)).sum() / 4 * (1 + 4 * u)
        assert np.all(np.abs(y - yref) <= bound)


def test_rht_preserves_norm():
    rng = np.random.default_rng(6)
    x = rng.standard_normal((200, 64)).astype(np.float32)
    y = oracle.rht_rows(x, seed=9).astype(np.float64)
    nx = np.linalg.norm(x.astype(np.float64).reshape(-1, 16), axis=1)
    ny = np.linalg.norm(y.reshape(-1, 16), axis=1)
    assert np.all(np.abs(ny - nx) <= 16 * 2.0 ** -24 * nx + 1e-30)


def test_rht_cancels_in_the_product():
    """(X R)(W R)^T = X W^T: the same signed Hadamard on both operands along
    the contraction dim leaves the product unchanged (up to fp32 rounding)."""
    rng = np.random.default_rng(8)
    X = rng.standard_normal((48, 128)).astype(np.float32)
    W = rng.standard_normal((40, 128)).astype(np.float32)
    XR = oracle.rht_rows(X, seed=3).astype(np.float64)
    WR = oracle.rht_rows(W, seed=3).astype(np.float64)
    ref = X.astype(np.float64) @ W.astype(np.float64).T
    bound = 16 * 2.0 ** -24 * (np.abs(X).astype(np.float64) @ np.abs(W).astype(np.float64).T) * 4
    assert np.all(np.abs(XR @ WR.T - ref) <= bound)


def test_rht_butterfly_order_independent_check():
    """An in-place radix-2 butterfly (strides 1, 2, 4, 8; (a, b) -> (a+b,
    a-b) in float32) written here with numpy scalars agrees bit for bit with
    the oracle's product of explicit Kronecker factors."""
    rng = np.random.default_rng(10)
    for _ in range(300):
        x = (rng.standard_normal(16) * np.exp(rng.uniform(-30, 30))).astype(np.float32)
        x[rng.random(16) < 0.1] = np.float32(0.0)
        s = np.where(rng.random(16) < 0.5, -1.0, 1.0).astype(np.float32)
        t = [np.float32(np.float32(si * xi) * np.float32(0.25)) for si, xi in zip(s, x)]
        h = 1
        while h < 16:
            for base in range(0, 16, 2 * h):
                for i in range(base, base + h):
                    a, b = t[i], t[i + h]
                    t[i], t[i + h] = np.float32(a + b), np.float32(a - b)
            h *= 2
        y = oracle.rht16(x, s)
        assert np.array_equal(np.array(t, dtype=np.float32).view(np.uint32), y.view(np.uint32))


def test_sr_exhaustive_over_r16():
    """For fixed v the number of r16 in [0, 2^16) that round up is
    floor(f * 2^16): the draws whose sum with the kept 16-bit position
    carries out of 16 bits.  f is computed here in binary64 from the grid."""
    grid = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    rng = np.random.default_rng(12)
    for i in range(7):
        lo, hi = grid[i], grid[i + 1]
        for frac in (0.0, 1 / 3, 0.5, 0.9, float(rng.random()), 2.0 ** -20):
            v = np.float32(lo + frac * (hi - lo))
            f = (float(v) - lo) / (hi - lo)
            ups = sum(1 for r in range(0, 65536) if (oracle.e2m1_sr(float(v), r) & 7) == i + 1)
            assert ups == int(np.floor(f * 65536))
            # and they are the top F draws
            F = int(np.floor(f * 65536))
            if 0 < F < 65536:
                assert (oracle.e2m1_sr(float(v), 65536 - F) & 7) == i + 1
                assert (oracle.e2m1_sr(float(v), 65535 - F) & 7) == i


def test_sr_unbiased_over_1e6_draws():
    """Mean of dequantised SR values equals v within 5 sigma plus the 2^-16
    resolution bias, for v at fractions {1/3, 0.5, 0.9} of each interval."""
    grid = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    rows = 32768                               # 31 draws per row -> ~1.0e6 draws
    for i in range(7):
        lo, hi = grid[i], grid[i + 1]
        for frac in (1 / 3, 0.5, 0.9):
            v = np.float32(lo + frac * (hi - lo))
            x = np.full((rows, 32), v, dtype=np.float32)
            x[:, 0] = 6.0                      # fixes the block scale at 1
            codes, scales = oracle.quantize_1d(x, sr=True, sr_seed=99, sr_offset=i)
            assert np.all(scales == 127)
            deq = oracle.dequant_1d(codes, scales)[:, 1:]
            n = deq.size
            p = (float(v) - lo) / (hi - lo)
            sigma = (hi - lo) * np.sqrt(p * (1 - p) / n)
            assert abs(deq.mean() - float(v)) <= 5 * sigma + (hi - lo) * 2.0 ** -16


def test_philox_known_answer_vectors():
    """The oracle's Philox4x32-10 reproduces the published known-answer
    vectors (tests/golden/philox4x32_10_kat.txt, cited there): an input of
    all zeros, all ones and the digits of pi."""
    import os
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "philox4x32_10_kat.txt")
    rows = [ln.split() for ln in open(path) if ln.strip() and not ln.startswith("#")]
    assert len(rows) == 3
    for r in rows:
        w = [int(v, 16) for v in r]
        assert [int(v) for v in oracle.philox4x32_10(w[0:4], w[4:6])] == w[6:10]


# Largest |P(both round up) - P(first up) P(second up)| over every pair of
# kept positions (F1, F2) for the two elements of a word that draw a 16-bit
# value and its bit reversal (elements 4m, 4m+1 and 4m+2, 4m+3): 8.31e-5,
# reached at F1 = F2 = 43691 (f = 2/3).  It is found by counting, for every
# (F1, F2), the draws r in [0, 2^16) with F1 + r >= 2^16 and
# F2 + reverse16(r) >= 2^16.  Elements drawing disjoint bytes are independent.
SR_PAIR_DEPENDENCE_BOUND = 8.31e-5


def test_sr_pair_decisions_are_nearly_independent():
    """Joint behaviour of the SR decisions inside one Philox word, measured
    through the oracle's quantiser over 2^20 blocks (one counter pair per
    block): every element rounds up with frequency F/2^16, and every pair of
    elements of a word rounds up together with frequency P1 P2 within the
    layout's dependence bound (zero for elements on disjoint bytes) plus 5
    standard deviations.  A layout that handed two elements the same or
    overlapping random bits would fail: at f = 1/2 a shared draw gives a
    joint frequency of 1/2 instead of 1/4."""
    nb = 1 << 20
    # block scale 2^0 (block max 6 at element 31); elements 0..27 sit in
    # [1, 1.5) at kept positions F (value 1 + F/2^17, exact in binary32)
    Fs = np.array([43691, 32768, 21845, 58982, 6554, 43691, 32768,
                   16384, 49152, 43691, 21845, 32768, 65535, 1,
                   43691, 43691, 32768, 32768, 21845, 43691, 5000,
                   60000, 40000, 20000, 43691, 21845, 50000, 32768], dtype=np.int64)
    row = np.zeros(32, dtype=np.float32)
    row[:28] = (1.0 + Fs / 131072.0).astype(np.float32)
    assert np.all(((row[:28].astype(np.float64) - 1.0) * 131072.0) == Fs)
    row[31] = 6.0
    x = np.broadcast_to(row, (nb, 32)).copy()
    codes, scales = oracle.quantize_1d(x, sr=True, sr_seed=0xC0FFEE, sr_offset=11)
    assert np.all(scales == 127)
    nib = np.stack([codes & 0xF, codes >> 4], axis=-1).reshape(nb, 32)
    assert np.all(np.isin(nib[:, :28], (2, 3)))
    up = (nib[:, :28] == 3)
    p = Fs / 65536.0
    freq = up.mean(axis=0)
    sig = np.sqrt(p * (1 - p) / nb)
    assert np.all(np.abs(freq - p) <= 5 * sig + 1e-12), np.abs(freq - p) / np.maximum(sig, 1e-12)
    for w in range(7):
        for a, b in ((0, 1), (2, 3), (0, 2), (0, 3), (1, 2), (1, 3)):
            i, j = 4 * w + a, 4 * w + b
            q = p[i] * p[j]
            joint = float(np.mean(up[:, i] & up[:, j]))
            shared = (a, b) in ((0, 1), (2, 3))
            bound = (SR_PAIR_DEPENDENCE_BOUND if shared else 0.0) + 5 * np.sqrt(max(q * (1 - q), 1e-12) / nb)
            assert abs(joint - q) <= bound, (w, a, b, joint, q)

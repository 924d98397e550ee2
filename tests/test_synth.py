"""CPU: the seeded synthetic inputs have the recipe's stated properties
(shapes, routing counts and padding, the de-oscillation stress positions,
bf16 rounding), so every parity case and the bench read the workload the
recipe describes."""
import numpy as np

from fp4_precision_numerics_b200 import synth


def test_bf16_bits_round_to_nearest_even():
    x = np.array([1.0, 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -2.0, 1.0 + 2.0 ** -8 + 2.0 ** -20, 0.0, -0.0],
                 dtype=np.float32)
    assert synth.bf16_bits(x).tolist() == [0x3F80, 0x3F80, 0x3F82, 0xC000, 0x3F81, 0x0000, 0x8000]
    b = synth.bf16_bits(np.array([3.140625], dtype=np.float32))
    assert synth.bf16_to_f32(b)[0] == np.float32(3.140625)


def test_zipf_routing_counts_and_distinct_experts():
    r = synth.zipf_routing()
    assert r.shape == (synth.N_TOKENS, synth.TOP_K) and r.dtype == np.int32
    assert r.min() >= 0 and r.max() < synth.N_EXPERTS
    s = np.sort(r, axis=1)
    assert np.all(s[:, 1:] != s[:, :-1])                       # top-k distinct experts per token
    counts, offsets, tor = synth.expert_layout(r)
    assert counts.sum() == synth.N_TOKENS * synth.TOP_K == 65536
    # p_i proportional to i^-1.1: the heaviest expert takes about a fifth of the rows
    assert counts[0] == 12715 and counts.min() >= 450
    assert counts[0] > counts[1] > counts[2] > counts[3]
    assert np.all(offsets % synth.SEGMENT_ALIGN == 0) and offsets[0] == 0 and offsets[-1] == 67584


def test_expert_layout_rows_are_the_routed_tokens():
    r = synth.zipf_routing(n_tokens=512, n_experts=8, top_k=2, seed=9)
    counts, offsets, tor = synth.expert_layout(r, n_experts=8)
    assert np.all(np.diff(offsets) >= counts) and np.all(np.diff(offsets) - counts < synth.SEGMENT_ALIGN)
    for e in range(8):
        seg = tor[offsets[e]:offsets[e + 1]]
        toks = seg[seg >= 0]
        assert len(toks) == counts[e]
        assert np.all(seg[len(toks):] == -1)                   # padding after the expert's tokens
        assert np.array_equal(toks, np.nonzero((r == e).any(axis=1))[0])
    x = synth.normal_bf16((512, 64), 1.0, seed=1)
    g = synth.gather_rows(x, tor)
    assert np.all(g[tor < 0] == 0) and np.array_equal(g[tor >= 0], x[tor[tor >= 0]])


def test_deosc_master_moves_positions_next_to_bin_boundaries():
    w = synth.deosc_master(groups=2, rows=64, cols=96, seed=5)
    base = np.random.default_rng(5).standard_normal((2, 64, 96), dtype=np.float32) * np.float32(0.02)
    moved = w != base
    assert 0.03 < moved.mean() < 0.06                          # 5% minus the skipped block maxima
    bw = np.abs(w.reshape(2, 2, 32, 3, 32))
    bb = np.abs(base.reshape(2, 2, 32, 3, 32))
    assert np.array_equal(bw.max(axis=(2, 4)), bb.max(axis=(2, 4)))   # block maxima (hence scales) unchanged
    amax = bb.max(axis=(2, 4))
    S = np.ldexp(1.0, np.frexp(amax.astype(np.float64))[1] - 1) / 4.0
    g, r, c = np.nonzero(moved)
    m = np.abs(w[g, r, c]).astype(np.float64) / S[g, r // 32, c // 32]
    mids = np.array(synth.BOUNDARY_MIDPOINTS)
    dist = np.abs(m[:, None] - mids[None, :]).min(axis=1)
    assert np.all(dist * S[g, r // 32, c // 32] <= 1e-4 + 1e-9)      # within the jitter of a midpoint


def test_student_t_activations_are_heavy_tailed():
    x = synth.bf16_to_f32(synth.student_t_activations(4096, 64, seed=0)).astype(np.float64)
    assert x.shape == (4096, 64)
    z = x / x.std(axis=0, keepdims=True)
    kurt = (z ** 4).mean(axis=0)
    assert np.median(kurt) > 4.0                               # Gaussian: 3
    spread = x.std(axis=0)
    assert spread.max() / spread.min() > 10.0                  # per-column scales over two decades


def test_single_layer_outliers():
    x, w = synth.single_layer(seed=0)
    for a in (x, w):
        v = np.abs(synth.bf16_to_f32(a))
        big = (v > 8.0).sum()                                  # N(0,1) alone: P(|z| > 8) ~ 1e-15
        assert 0.006 * v.size < big <= 0.01 * v.size

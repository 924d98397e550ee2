"""Seeded synthetic inputs with the shapes and value distributions of the
GPT-OSS-20B MoE expert layers the ALTO recipe trains (abstract; roboaidigest
"What ALTO Actually Does": expert matrices dominate compute and memory).

Both the CUDA path and the CPU oracle read these arrays; this module holds
none of the quantisation arithmetic.  Everything is drawn on the host with
``numpy.random.default_rng(seed)`` (PCG64) and rounded to bfloat16 with
round-to-nearest-even; bf16 tensors travel as uint16 bit patterns.

No dataset is used: C4, the MLPerf benchmark and trained weights stand
behind the pages' numbers and are replaced by these draws.
"""
from __future__ import annotations

import numpy as np

D_MODEL = 2880
D_FF_FUSED = 5760          # gate/up fused: W_up is [5760, 2880] per expert
N_EXPERTS = 32
TOP_K = 4
N_TOKENS = 16384
ZIPF_S = 1.1
SEGMENT_ALIGN = 128         # expert segments start on 128-row boundaries


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 bit patterns (uint16), round to nearest even."""
    f = np.ascontiguousarray(x, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


# ---------------------------------------------------------------- config 1
def single_layer(seed: int = 0, n: int = 256, outlier_frac: float = 0.01, outlier_mult: float = 20.0):
    """X[n x n], W[n x n] ~ N(0,1) with outlier_frac of the entries (chosen
    without replacement) multiplied by outlier_mult.  Returns bf16 bits."""
    rng = np.random.default_rng(seed)
    out = []
    for _ in range(2):
        a = rng.standard_normal((n, n), dtype=np.float32)
        k = int(round(outlier_frac * a.size))
        idx = rng.choice(a.size, size=k, replace=False)
        a.reshape(-1)[idx] *= outlier_mult
        out.append(bf16_bits(a))
    return out[0], out[1]


# ---------------------------------------------------------------- config 2
QUANT_SWEEP_SHAPES = ((4096, 2880), (16384, 2880), (65536, 5760))


def student_t_activations(rows: int, cols: int, seed: int = 0, nu: float = 4.0):
    """Student-t(nu) entries times a per-column scale drawn log-uniform in
    [0.1, 10].  Returns bf16 bits [rows, cols]."""
    rng = np.random.default_rng(seed)
    col_scale = np.exp(rng.uniform(np.log(0.1), np.log(10.0), size=cols)).astype(np.float32)
    out = np.empty((rows, cols), dtype=np.uint16)
    step = max(1, (1 << 24) // cols)
    for r0 in range(0, rows, step):
        r1 = min(rows, r0 + step)
        t = rng.standard_t(nu, size=(r1 - r0, cols)).astype(np.float32)
        out[r0:r1] = bf16_bits(t * col_scale[None, :])
    return out


# ---------------------------------------------------------------- config 3/4
def zipf_routing(n_tokens: int = N_TOKENS, n_experts: int = N_EXPERTS, top_k: int = TOP_K,
                 s: float = ZIPF_S, seed: int = 2):
    """Top-k distinct experts per token by Gumbel-top-k on log p_i with
    p_i proportional to i^-s (i = 1..E).  Returns an int32 [n_tokens, top_k]
    expert-id matrix."""
    rng = np.random.default_rng(seed)
    logp = -s * np.log(np.arange(1, n_experts + 1, dtype=np.float64))
    g = rng.gumbel(size=(n_tokens, n_experts))
    return np.argsort(-(logp[None, :] + g), axis=1)[:, :top_k].astype(np.int32)


def expert_layout(routing: np.ndarray, n_experts: int = N_EXPERTS, align: int = SEGMENT_ALIGN):
    """Expert-sorted row layout.  Returns (counts[E], offsets[E+1] padded to
    `align`, token_of_row[M_pad] with -1 on padding rows)."""
    counts = np.bincount(routing.reshape(-1), minlength=n_experts).astype(np.int64)
    padded = (counts + align - 1) // align * align
    offsets = np.zeros(n_experts + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(padded)
    token_of_row = np.full(int(offsets[-1]), -1, dtype=np.int64)
    for e in range(n_experts):
        toks = np.nonzero((routing == e).any(axis=1))[0]
        token_of_row[offsets[e]:offsets[e] + len(toks)] = toks
    return counts, offsets, token_of_row


def gather_rows(x_bits: np.ndarray, token_of_row: np.ndarray) -> np.ndarray:
    """Rows of x in expert-sorted order; padding rows are +0."""
    out = np.zeros((len(token_of_row), x_bits.shape[1]), dtype=x_bits.dtype)
    valid = token_of_row >= 0
    out[valid] = x_bits[token_of_row[valid]]
    return out


def normal_bf16(shape, std: float, seed: int) -> np.ndarray:
    rng = np.random.default_rng(seed)
    out = np.empty(shape, dtype=np.uint16)
    flat = out.reshape(-1)
    step = 1 << 24
    for i in range(0, flat.size, step):
        j = min(flat.size, i + step)
        flat[i:j] = bf16_bits(rng.standard_normal(j - i, dtype=np.float32) * np.float32(std))
    return out


def zero_padding_rows(x_bits: np.ndarray, token_of_row: np.ndarray) -> np.ndarray:
    x_bits[token_of_row < 0] = 0
    return x_bits


def moe_layer(seed_route: int = 2, seed_x: int = 0, seed_w: int = 1, seed_h: int = 3, seed_dy: int = 4,
              n_tokens: int = N_TOKENS, n_experts: int = N_EXPERTS, d_model: int = D_MODEL,
              d_ff: int = D_FF_FUSED, with_grads: bool = True):
    """GPT-OSS-20B-shaped MoE expert layer, expert-sorted and padded.

    Returns a dict of host arrays (bf16 as uint16 bits):
      offsets [E+1] (int64, multiples of 128), counts [E],
      x      [M_pad, d_model]  routed token activations N(0,1), zero padding rows
      w_up   [E, d_ff, d_model] N(0, 0.02)
      w_down [E, d_model, d_model] N(0, 0.02)   (expert intermediate 2880)
      h      [M_pad, d_model]  down-proj input, fresh N(0,1)
      dy_up  [M_pad, d_ff], dy_down [M_pad, d_model]  N(0, 1e-3) output grads
    """
    routing = zipf_routing(n_tokens, n_experts, seed=seed_route)
    counts, offsets, tor = expert_layout(routing, n_experts)
    m_pad = int(offsets[-1])
    x_tok = normal_bf16((n_tokens, d_model), 1.0, seed_x)
    out = dict(offsets=offsets, counts=counts, token_of_row=tor)
    out["x"] = gather_rows(x_tok, tor)
    out["w_up"] = normal_bf16((n_experts, d_ff, d_model), 0.02, seed_w)
    out["w_down"] = normal_bf16((n_experts, d_model, d_model), 0.02, seed_w + 100)
    out["h"] = zero_padding_rows(normal_bf16((m_pad, d_model), 1.0, seed_h), tor)
    if with_grads:
        out["dy_up"] = zero_padding_rows(normal_bf16((m_pad, d_ff), 1e-3, seed_dy), tor)
        out["dy_down"] = zero_padding_rows(normal_bf16((m_pad, d_model), 1e-3, seed_dy + 100), tor)
    return out


# ---------------------------------------------------------------- config 5
BOUNDARY_MIDPOINTS = (0.25, 0.75, 1.25, 1.75, 2.5, 3.5)   # halfway between E2M1 magnitudes


def deosc_master(groups: int = N_EXPERTS, rows: int = D_FF_FUSED, cols: int = D_MODEL, seed: int = 5,
                 frac: float = 0.05, jitter: float = 1e-4, std: float = 0.02):
    """fp32 master weights N(0, std) with `frac` of the positions moved next
    to an E2M1 bin boundary of their 32x32 block: w = +-m*S + U(-jitter,
    jitter), m a boundary midpoint and S = P/4 where P is the largest power
    of two at or below the block's largest magnitude.  The block's largest
    element is never moved, and m*S + jitter < P, so P is unchanged."""
    rng = np.random.default_rng(seed)
    w = (rng.standard_normal((groups, rows, cols), dtype=np.float32) * np.float32(std))
    blk = w.reshape(groups, rows // 32, 32, cols // 32, 32)
    amax = np.abs(blk).max(axis=(2, 4))                        # [g, rb, cb]
    mant, ex = np.frexp(amax.astype(np.float64))                 # amax = mant*2^ex, mant in [0.5,1)
    P = np.ldexp(1.0, ex - 1)                                    # largest power of two <= amax
    S = (P / 4.0).astype(np.float32)
    n = w.size
    k = int(round(frac * n))
    idx = rng.choice(n, size=k, replace=False)
    g_i, rem = np.divmod(idx, rows * cols)
    r_i, c_i = np.divmod(rem, cols)
    # never move the element that holds its block's maximum magnitude
    blk_max_here = np.abs(w[g_i, r_i, c_i]) == amax[g_i, r_i // 32, c_i // 32]
    keep = ~blk_max_here
    g_i, r_i, c_i = g_i[keep], r_i[keep], c_i[keep]
    m = np.asarray(BOUNDARY_MIDPOINTS, dtype=np.float32)[rng.integers(0, len(BOUNDARY_MIDPOINTS), size=len(g_i))]
    sign = np.where(rng.random(len(g_i)) < 0.5, np.float32(-1.0), np.float32(1.0))
    jit = rng.uniform(-jitter, jitter, size=len(g_i)).astype(np.float32)
    w[g_i, r_i, c_i] = sign * m * S[g_i, r_i // 32, c_i // 32] + jit
    return w


def deosc_update_noise(shape, step: int, std: float = 1e-5) -> np.ndarray:
    """The synthetic optimizer update of step `step` (seed 6 + step)."""
    rng = np.random.default_rng(6 + step)
    return rng.standard_normal(shape, dtype=np.float32) * np.float32(std)

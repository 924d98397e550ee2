// quantize.cuh -- fused MXFP4 quantisation kernels for sm_100a.
//
// One pass over the input per kernel: widen -> (random signs, 1/4, 16-point
// Hadamard butterfly) -> block amax -> UE8M0 scale -> nearest or stochastic
// rounding (Philox4x32-10) -> nibble packing -> codes + scales, with the
// de-oscillation state update fused into the 2D weight path.  The
// arithmetic follows the readings stated in include/mxfp4.h; every float
// operation is an explicitly rounded binary32 op (no contraction, no FTZ).
//
// Recipe sources: abstract of "Training an MoE LLM in MXFP4: How We Closed
// the Gap to BF16" (hybrid 1D/2D block quantisation, RHT, SR, simplified
// de-oscillation) and roboaidigest "What ALTO Actually Does" (E2M1 values
// with UE8M0 block scales; why de-oscillation is needed).
#pragma once

#include "common.cuh"

namespace mxfp4 {

// Byte offset of scale (r, s) in the tensor-core scale layout of a [R, S]
// scale matrix: 512-byte chunks of 128 rows x 4 scales, chunks ordered
// (row block, scale chunk) with the scale chunk fastest.
__host__ __device__ __forceinline__ int64_t mma_scale_offset(int64_t r, int64_t s, int64_t S) {
    const int64_t nchunk = (S + 3) / 4;
    return ((r >> 7) * nchunk + (s >> 2)) * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4 + (s & 3);
}

__host__ __device__ __forceinline__ int64_t mma_scale_bytes(int64_t R, int64_t S) {
    return ((R + 127) / 128) * ((S + 3) / 4) * 512;
}

struct QuantArgs {
    const void* in;
    int64_t groups, rows, cols, ld;   // input geometry (per group: rows x cols, row stride ld)
    uint32_t rht_signs;               // bit i set -> sign i is -1 (only used with RHT)
    uint32_t sr_key0, sr_key1, sr_offset;
    uint8_t* codes;
    uint8_t* scales;                  // canonical, may be null
    uint8_t* scales_mma;              // tensor-core layout, may be null
    uint8_t* codes_t;                 // 2D only
    uint8_t* scales_mma_t;            // 2D only
    // de-oscillation
    uint8_t* state;
    uint32_t step, flip_threshold, reset_period;
};

// ---------------------------------------------------------------------------
// Loading 16 consecutive elements as binary32.
// ---------------------------------------------------------------------------
template <typename T>
struct Loader;

template <>
struct Loader<uint16_t> {  // bfloat16 bit patterns
    __device__ __forceinline__ static void load16(const uint16_t* p, float (&x)[16]) {
        const uint4* q = reinterpret_cast<const uint4*>(p);
        const uint4 a = __ldg(q);
        const uint4 b = __ldg(q + 1);
        const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            x[2 * i] = __uint_as_float(w[i] << 16);
            x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
        }
    }
};

template <>
struct Loader<float> {
    __device__ __forceinline__ static void load16(const float* p, float (&x)[16]) {
        const float4* q = reinterpret_cast<const float4*>(p);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float4 v = __ldg(q + i);
            x[4 * i] = v.x;
            x[4 * i + 1] = v.y;
            x[4 * i + 2] = v.z;
            x[4 * i + 3] = v.w;
        }
    }
};

// Randomized Hadamard transform of one 16-element chunk in registers:
// t = (s .* x) * 1/4, then the radix-2 butterfly with strides 1, 2, 4, 8.
__device__ __forceinline__ void rht16(float (&x)[16], uint32_t signs) {
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const float s = __uint_as_float(__float_as_uint(x[i]) ^ (((signs >> i) & 1u) << 31));
        x[i] = __fmul_rn(s, 0.25f);
    }
#pragma unroll
    for (int h = 1; h < 16; h <<= 1) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            if ((i & h) == 0) {
                const float a = x[i], b = x[i + h];
                x[i] = __fadd_rn(a, b);
                x[i + h] = __fsub_rn(a, b);
            }
        }
    }
}

__device__ __forceinline__ float amax16(const float (&x)[16]) {
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) m = fmaxf(m, fabsf(x[i]));
    return m;
}

// Scale 16 values by 2^-E and round them to 8 bytes of packed codes.
// `n0` is the SR element index of x[0] (multiple of 8).
template <bool SR>
__device__ __forceinline__ uint2 quant16(const float (&x)[16], float inv_scale, uint64_t n0, uint32_t key0,
                                         uint32_t key1, uint32_t offset) {
    float v[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __fmul_rn(x[i], inv_scale);
    if constexpr (SR) {
        const uint64_t g0 = n0 >> 3;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            const uint64_t g = g0 + half;
            const Philox4 r = philox4x32_10(uint32_t(g), uint32_t(g >> 32), offset, 0u, key0, key1);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const uint32_t r16 = (r.w[j >> 1] >> (16 * (j & 1))) & 0xFFFFu;
                v[8 * half + j] = e2m1_sr_value(v[8 * half + j], r16);
            }
        }
    }
    uint32_t b[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) b[i] = e2m1x2_rn(v[2 * i], v[2 * i + 1]);
    uint2 out;
    out.x = b[0] | (b[1] << 8) | (b[2] << 16) | (b[3] << 24);
    out.y = b[4] | (b[5] << 8) | (b[6] << 16) | (b[7] << 24);
    return out;
}

// ---------------------------------------------------------------------------
// 1D blocks along the last dim.  One thread per 16-element chunk; the two
// threads of a 32-element block are adjacent lanes and combine their maxima
// with one shuffle.  Output rows = input rows (groups back to back).
// ---------------------------------------------------------------------------
template <typename InT, bool RHT, bool SR>
__global__ void __launch_bounds__(256) quant1d_rows_kernel(QuantArgs a) {
    const int64_t C = a.cols;
    const int64_t chunks_per_row = C >> 4;
    const int64_t total_rows = a.groups * a.rows;
    const int64_t total = total_rows * chunks_per_row;
    const int64_t S = C >> 5;
    const int64_t mma_group_bytes = mma_scale_bytes(a.rows, S);
    const InT* in = static_cast<const InT*>(a.in);
    const int64_t stride = int64_t(gridDim.x) * blockDim.x;
    // Whole warps iterate together (the pair shuffle uses the full mask);
    // `total` is even, so the two lanes of a block are valid together.
    const int64_t first = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
    const int lane = threadIdx.x & 31;
    for (int64_t i = first; i - lane < total; i += stride) {
        const bool valid = i < total;
        const int64_t ic = valid ? i : total - 2 + (lane & 1);
        const int64_t row = ic / chunks_per_row;
        const int64_t col0 = (ic - row * chunks_per_row) << 4;
        float x[16];
        Loader<InT>::load16(in + row * a.ld + col0, x);
        if constexpr (RHT) rht16(x, a.rht_signs);
        float m = amax16(x);
        m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
        if (!valid) continue;
        const int sb = scale_byte_from_amax(m);
        const uint2 q = quant16<SR>(x, inv_scale_from_byte(sb), uint64_t(row) * uint64_t(C) + uint64_t(col0),
                                    a.sr_key0, a.sr_key1, a.sr_offset);
        *reinterpret_cast<uint2*>(a.codes + row * (C >> 1) + (col0 >> 1)) = q;
        if ((col0 & 16) == 0) {
            const int64_t s = col0 >> 5;
            if (a.scales) a.scales[row * S + s] = uint8_t(sb);
            if (a.scales_mma) {
                const int64_t g = row / a.rows, r = row - g * a.rows;
                a.scales_mma[g * mma_group_bytes + mma_scale_offset(r, s, S)] = uint8_t(sb);
            }
        }
    }
}

// ---------------------------------------------------------------------------
// 1D blocks along dim 0 (the token dim), output transposed: input [T, F]
// (per group), output [F, T].  A CTA stages a 128-token x 64-feature tile in
// shared memory with coalesced row loads; each thread then owns one
// (feature, 32-token block): RHT on its two chunks, amax, scale, rounding,
// and one 16-byte store of codes into output row `feature`.
// ---------------------------------------------------------------------------
constexpr int kTT = 128;  // tokens per tile
constexpr int kTF = 64;   // features per tile

template <typename InT, bool RHT, bool SR>
__global__ void __launch_bounds__(256) quant1d_cols_kernel(QuantArgs a) {
    __shared__ __align__(16) InT tile[kTT][kTF + 16 / sizeof(InT)];
    const int64_t T = a.rows, F = a.cols;
    const int64_t g = blockIdx.z;
    const int64_t t0 = int64_t(blockIdx.x) * kTT;
    const int64_t f0 = int64_t(blockIdx.y) * kTF;
    const InT* in = static_cast<const InT*>(a.in) + g * T * a.ld;
    // stage: 16-byte vectors along the feature dim
    constexpr int kVec = 16 / sizeof(InT);
    constexpr int kVecPerRow = kTF / kVec;
    for (int idx = threadIdx.x; idx < kTT * kVecPerRow; idx += blockDim.x) {
        const int tr = idx / kVecPerRow;
        const int fv = (idx - tr * kVecPerRow) * kVec;
        const int64_t t = t0 + tr, f = f0 + fv;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (t < T) {
            if (f + kVec <= F) {
                v = __ldg(reinterpret_cast<const uint4*>(in + t * a.ld + f));
            } else {
                InT tmp[kVec];
#pragma unroll
                for (int k = 0; k < kVec; ++k) tmp[k] = (f + k < F) ? in[t * a.ld + f + k] : InT(0);
                v = *reinterpret_cast<const uint4*>(tmp);
            }
        }
        *reinterpret_cast<uint4*>(&tile[tr][fv]) = v;
    }
    __syncthreads();
    // one (feature, block) per thread: 64 features x 4 blocks
    const int fl = threadIdx.x & 63;
    const int blk = threadIdx.x >> 6;
    const int64_t f = f0 + fl;
    const int64_t tb = t0 + blk * 32;
    if (f >= F || tb >= T) return;
    float x0[16], x1[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) {
        if constexpr (sizeof(InT) == 2) {
            x0[k] = __uint_as_float(uint32_t(tile[blk * 32 + k][fl]) << 16);
            x1[k] = __uint_as_float(uint32_t(tile[blk * 32 + 16 + k][fl]) << 16);
        } else {
            x0[k] = tile[blk * 32 + k][fl];
            x1[k] = tile[blk * 32 + 16 + k][fl];
        }
    }
    if constexpr (RHT) {
        rht16(x0, a.rht_signs);
        rht16(x1, a.rht_signs);
    }
    const float m = fmaxf(amax16(x0), amax16(x1));
    const int sb = scale_byte_from_amax(m);
    const float inv = inv_scale_from_byte(sb);
    const int64_t orow = g * F + f;  // output row (groups back to back)
    const uint64_t n0 = uint64_t(orow) * uint64_t(T) + uint64_t(tb);
    const uint2 q0 = quant16<SR>(x0, inv, n0, a.sr_key0, a.sr_key1, a.sr_offset);
    const uint2 q1 = quant16<SR>(x1, inv, n0 + 16, a.sr_key0, a.sr_key1, a.sr_offset);
    *reinterpret_cast<uint4*>(a.codes + orow * (T >> 1) + (tb >> 1)) = make_uint4(q0.x, q0.y, q1.x, q1.y);
    const int64_t S = T >> 5;
    const int64_t s = tb >> 5;
    if (a.scales) a.scales[orow * S + s] = uint8_t(sb);
    if (a.scales_mma) a.scales_mma[g * mma_scale_bytes(F, S) + mma_scale_offset(f, s, S)] = uint8_t(sb);
}

// ---------------------------------------------------------------------------
// 2D 32x32 blocks (weights), optionally with the de-oscillation update.
// One warp per block; lane l owns row l of the block (32 elements).  The
// codes of the transpose are produced through a padded shared-memory copy
// of the block's 32x32 code bytes.
// ---------------------------------------------------------------------------
template <typename InT, bool RHT, bool SR, bool DEOSC>
__global__ void __launch_bounds__(256) quant2d_kernel(QuantArgs a) {
    __shared__ uint32_t tcodes[8][32 * 9];  // per warp: 32 rows x 36 bytes
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t R = a.rows, C = a.cols;
    const int64_t nbr = R >> 5, nbc = C >> 5;
    const int64_t nblocks = a.groups * nbr * nbc;
    const int64_t bid = int64_t(blockIdx.x) * 8 + warp;
    if (bid >= nblocks) return;
    const int64_t g = bid / (nbr * nbc);
    const int64_t rem = bid - g * nbr * nbc;
    const int64_t bi = rem / nbc, bj = rem - bi * nbc;
    const int64_t r = bi * 32 + lane;
    const int64_t c0 = bj * 32;
    const InT* in = static_cast<const InT*>(a.in) + g * R * a.ld;
    float x0[16], x1[16];
    Loader<InT>::load16(in + r * a.ld + c0, x0);
    Loader<InT>::load16(in + r * a.ld + c0 + 16, x1);
    if constexpr (RHT) {
        rht16(x0, a.rht_signs);
        rht16(x1, a.rht_signs);
    }
    float m = fmaxf(amax16(x0), amax16(x1));
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    const int sb = scale_byte_from_amax(m);
    const float inv = inv_scale_from_byte(sb);
    const uint64_t n0 = (uint64_t(g) * uint64_t(R) + uint64_t(r)) * uint64_t(C) + uint64_t(c0);
    uint2 q0 = quant16<SR>(x0, inv, n0, a.sr_key0, a.sr_key1, a.sr_offset);
    uint2 q1 = quant16<SR>(x1, inv, n0 + 16, a.sr_key0, a.sr_key1, a.sr_offset);
    uint32_t w[4] = {q0.x, q0.y, q1.x, q1.y};  // 32 codes of row r, nibble k = element k
    const int64_t widx = (g * R + r) * C + c0;  // weight index of element 0 of this row
    if constexpr (DEOSC) {
        uint4 st0 = *reinterpret_cast<const uint4*>(a.state + widx);
        uint4 st1 = *reinterpret_cast<const uint4*>(a.state + widx + 16);
        uint32_t s[8] = {st0.x, st0.y, st0.z, st0.w, st1.x, st1.y, st1.z, st1.w};
        const bool reset = a.step > 0 && a.reset_period > 0 && (a.step % a.reset_period) == 0;
#pragma unroll
        for (int k = 0; k < 32; ++k) {
            const uint32_t q = (w[k >> 3] >> (4 * (k & 7))) & 0xFu;
            uint32_t st = (s[k >> 2] >> (8 * (k & 3))) & 0xFFu;
            uint32_t outc;
            if (a.step == 0) {
                st = q;
                outc = q;
            } else {
                uint32_t prev = st & 0xFu, cnt = (st >> 4) & 7u, frz = st >> 7;
                if (reset) {
                    cnt = 0;
                    frz = 0;
                }
                if (frz) {
                    outc = prev;
                } else {
                    if (q != prev) {
                        cnt = cnt < 7u ? cnt + 1u : 7u;
                        prev = q;
                        if (cnt >= a.flip_threshold) frz = 1;
                    }
                    outc = q;
                }
                st = prev | (cnt << 4) | (frz << 7);
            }
            s[k >> 2] = (s[k >> 2] & ~(0xFFu << (8 * (k & 3)))) | (st << (8 * (k & 3)));
            w[k >> 3] = (w[k >> 3] & ~(0xFu << (4 * (k & 7)))) | (outc << (4 * (k & 7)));
        }
        *reinterpret_cast<uint4*>(a.state + widx) = make_uint4(s[0], s[1], s[2], s[3]);
        *reinterpret_cast<uint4*>(a.state + widx + 16) = make_uint4(s[4], s[5], s[6], s[7]);
    }
    *reinterpret_cast<uint4*>(a.codes + (widx >> 1)) = make_uint4(w[0], w[1], w[2], w[3]);
    const int64_t S = nbc;  // scales per row
    if (a.scales && lane == 0) a.scales[g * nbr * nbc + bi * nbc + bj] = uint8_t(sb);
    if (a.scales_mma) a.scales_mma[g * mma_scale_bytes(R, S) + mma_scale_offset(r, bj, S)] = uint8_t(sb);
    if (a.codes_t) {
        // byte k of row `lane` = code of element k (0..31), row pitch 36 bytes
        uint32_t* t = tcodes[warp];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const uint32_t src = w[j >> 1] >> (16 * (j & 1));  // codes 4j..4j+3
            t[lane * 9 + j] = (src & 0xFu) | (((src >> 4) & 0xFu) << 8) | (((src >> 8) & 0xFu) << 16) |
                              (((src >> 12) & 0xFu) << 24);
        }
        __syncwarp();
        const uint8_t* tb = reinterpret_cast<const uint8_t*>(t);
        uint32_t o[4] = {0, 0, 0, 0};
#pragma unroll
        for (int i = 0; i < 32; ++i) o[i >> 3] |= uint32_t(tb[i * 36 + lane]) << (4 * (i & 7));
        // row (c0 + lane) of W^T, columns r0..r0+31 of it are rows of this block
        const int64_t tr = g * C + c0 + lane;
        *reinterpret_cast<uint4*>(a.codes_t + tr * (R >> 1) + (bi * 16)) = make_uint4(o[0], o[1], o[2], o[3]);
        if (a.scales_mma_t)
            a.scales_mma_t[g * mma_scale_bytes(C, nbr) + mma_scale_offset(c0 + lane, bi, nbr)] = uint8_t(sb);
    }
}

// ---------------------------------------------------------------------------
// Standalone RHT along the last dim: one thread per 16-element chunk.
// ---------------------------------------------------------------------------
template <typename InT, bool OUT_BF16>
__global__ void __launch_bounds__(256) rht_kernel(const InT* __restrict__ in, int64_t rows, int64_t cols, int64_t ld,
                                                  uint32_t signs, void* __restrict__ out) {
    const int64_t cpr = cols >> 4;
    const int64_t total = rows * cpr;
    const int64_t stride = int64_t(gridDim.x) * blockDim.x;
    for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < total; i += stride) {
        const int64_t row = i / cpr;
        const int64_t col0 = (i - row * cpr) << 4;
        float x[16];
        Loader<InT>::load16(in + row * ld + col0, x);
        rht16(x, signs);
        if constexpr (OUT_BF16) {
            uint32_t w[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const uint32_t lo = __float_as_uint(x[2 * k]), hi = __float_as_uint(x[2 * k + 1]);
                const uint32_t rlo = (lo + 0x7FFFu + ((lo >> 16) & 1u)) >> 16;
                const uint32_t rhi = (hi + 0x7FFFu + ((hi >> 16) & 1u)) >> 16;
                w[k] = rlo | (rhi << 16);
            }
            uint4* o = reinterpret_cast<uint4*>(static_cast<uint16_t*>(out) + row * cols + col0);
            o[0] = make_uint4(w[0], w[1], w[2], w[3]);
            o[1] = make_uint4(w[4], w[5], w[6], w[7]);
        } else {
            float4* o = reinterpret_cast<float4*>(static_cast<float*>(out) + row * cols + col0);
#pragma unroll
            for (int k = 0; k < 4; ++k) o[k] = make_float4(x[4 * k], x[4 * k + 1], x[4 * k + 2], x[4 * k + 3]);
        }
    }
}

}  // namespace mxfp4

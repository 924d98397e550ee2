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

// Byte offset of scale (r, s) in the tensor-core layout of one group whose
// scale matrix has `nchunk` 4-scale chunks per row (32-bit form of
// mma_scale_offset, for groups below 4 GB of scales).
__device__ __forceinline__ uint32_t mma_off32(uint32_t r, uint32_t s, uint32_t nchunk) {
    return ((r >> 7) * nchunk + (s >> 2)) * 512u + (r & 31u) * 16u + ((r >> 3) & 12u) + (s & 3u);
}


struct QuantArgs {
    const void* in;
    int64_t groups, rows, cols, ld;   // input geometry (per group: rows x cols, row stride ld)
    uint32_t rht_signs;               // bit i set -> sign i is -1 (only used with RHT)
    uint64_t rht_mul2[16];            // packed (s_i / 4, s_i / 4): sign and 1/4 of RHT index i
    uint32_t sr_key0, sr_key1, sr_offset;
    PhiloxKeys sr_keys;               // the ten round keys of (sr_key0, sr_key1), filled by the host
    uint8_t* codes;
    uint8_t* scales;                  // canonical, may be null
    uint8_t* scales_mma;              // tensor-core layout, may be null
    uint8_t* codes_t;                 // 2D only
    uint8_t* scales_mma_t;            // 2D only
    // de-oscillation
    uint8_t* state;
    uint32_t step, flip_threshold, reset_period, freeze_lower;
    // dual-direction quantisation: the 1x32-along-cols outputs of the same
    // input (codes [groups*rows, cols/2], scales, tensor-core scales)
    uint8_t* r_codes;
    uint8_t* r_scales;
    uint8_t* r_scales_mma;
    uint32_t r_rht_signs;
    uint64_t r_rht_mul2[16];          // packed (s_i / 4, s_i / 4) of the row-direction RHT
    uint32_t r_sr_offset;
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

// rht16 on two independent 16-element chunks at once, held as packed pairs
// (chunk A in the low halves, chunk B in the high halves): every operation
// is the scalar one of rht16 applied to both halves.
// `mul2[i]` holds s_i / 4 in both halves, so the sign and the 1/4 of index i
// are one packed multiplication (s_i x / 4 is exactly (s_i x) * 1/4).
__device__ __forceinline__ void rht16x2(uint64_t (&p)[16], const uint64_t (&mul2)[16]) {
#pragma unroll
    for (int i = 0; i < 16; ++i) p[i] = f2_mul(p[i], mul2[i]);
#pragma unroll
    for (int h = 1; h < 16; h <<= 1) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            if ((i & h) == 0) {
                const uint64_t a = p[i], b = p[i + h];
                p[i] = f2_add(a, b);
                p[i + h] = f2_sub(a, b);
            }
        }
    }
}

// rht16 of a 32-element block's two 16-element chunks, run two-wide as
// packed pairs (x0[i], x1[i]); `mul2` as for rht16x2.
__device__ __forceinline__ void rht16_pair(float (&x0)[16], float (&x1)[16], const uint64_t (&mul2)[16]) {
    uint64_t p[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) p[k] = f2_pack(x0[k], x1[k]);
    rht16x2(p, mul2);
#pragma unroll
    for (int k = 0; k < 16; ++k) f2_unpack(p[k], x0[k], x1[k]);
}

__device__ __forceinline__ float amax16(const float (&x)[16]) {
    float m = fmax3_abs(x[0], x[1], x[2]);
#pragma unroll
    for (int i = 3; i < 15; i += 2) m = fmax3_abs(m, x[i], x[i + 1]);
    return fmaxf(m, fabsf(x[15]));
}

// Scale 16 values by 2^-E and round them to 8 bytes of packed codes.
// `n0` is the SR element index of x[0] (a multiple of 16): one Philox call
// covers the 16 elements, word j the four elements 4j..4j+3, consumed by the
// four-element stochastic-rounding conversion (see e2m1x4_sr).
template <bool SR>
__device__ __forceinline__ uint2 quant16_scaled(const float (&v)[16], uint64_t n0, const PhiloxKeys& keys,
                                                uint32_t offset) {
    uint2 out;
    if constexpr (SR) {
        const uint64_t g = n0 >> 4;
        const Philox4 r = philox4x32_10(uint32_t(g), uint32_t(g >> 32), offset, 0u, keys);
        const uint32_t q0 = e2m1x4_sr(v[0], v[1], v[2], v[3], r.w[0]);
        const uint32_t q1 = e2m1x4_sr(v[4], v[5], v[6], v[7], r.w[1]);
        const uint32_t q2 = e2m1x4_sr(v[8], v[9], v[10], v[11], r.w[2]);
        const uint32_t q3 = e2m1x4_sr(v[12], v[13], v[14], v[15], r.w[3]);
        out.x = q0 | (q1 << 16);
        out.y = q2 | (q3 << 16);
    } else {
        out.x = e2m1x8_rn(v[0], v[1], v[2], v[3], v[4], v[5], v[6], v[7]);
        out.y = e2m1x8_rn(v[8], v[9], v[10], v[11], v[12], v[13], v[14], v[15]);
    }
    return out;
}

template <bool SR>
__device__ __forceinline__ uint2 quant16(const float (&x)[16], float inv_scale, uint64_t n0, const PhiloxKeys& keys,
                                         uint32_t offset) {
    float v[16];
    const uint64_t inv2 = f2_pack(inv_scale, inv_scale);
#pragma unroll
    for (int i = 0; i < 16; i += 2) f2_unpack(f2_mul(f2_pack(x[i], x[i + 1]), inv2), v[i], v[i + 1]);
    return quant16_scaled<SR>(v, n0, keys, offset);
}

// ---------------------------------------------------------------------------
// 1D blocks along the last dim.  One thread per 32-element block: two
// 16-element RHT chunks in registers, the block maximum, scale, rounding,
// and one 16-byte store of codes (consecutive threads write consecutive
// blocks, so a warp's code stores are contiguous).  Output rows = input rows
// (groups back to back).
// ---------------------------------------------------------------------------
template <typename InT, bool RHT, bool SR>
__global__ void __launch_bounds__(256) quant1d_rows_kernel(const __grid_constant__ QuantArgs a) {
    // block i = (row, s) of the [groups * rows, cols / 32] block grid, and the
    // row's group g and row r inside it, are advanced by the grid stride with
    // adds and one conditional wrap each (no division in the loop; the host
    // keeps groups * rows below 2^31)
    const uint32_t C = uint32_t(a.cols), S = C >> 5, R = uint32_t(a.rows);
    const uint64_t total = uint64_t(a.groups) * R * S;
    const uint32_t stride = gridDim.x * blockDim.x;
    const uint32_t i0 = blockIdx.x * blockDim.x + threadIdx.x;
    if (i0 >= total) return;
    uint32_t row = i0 / S, s = i0 - row * S;
    uint32_t g = row / R, r = row - g * R;
    const uint32_t drow = stride / S, ds = stride - drow * S;
    const uint32_t dg = drow / R, dr = drow - dg * R;
    const uint32_t nchunk = (S + 3) >> 2;
    const uint64_t mma_group_bytes = uint64_t((R + 127) >> 7) * nchunk * 512u;
    const InT* in = static_cast<const InT*>(a.in);
    const PhiloxKeys& keys = a.sr_keys;   // kernel parameters: read from the constant bank
    for (uint64_t i = i0; i < total; i += stride) {
        const uint32_t col0 = s << 5;
        float x0[16], x1[16];
        const InT* src = in + uint64_t(row) * uint64_t(a.ld) + col0;
        Loader<InT>::load16(src, x0);
        Loader<InT>::load16(src + 16, x1);
        if constexpr (RHT) {
            // the block's two 16-element chunks take the same butterflies
            rht16_pair(x0, x1, a.rht_mul2);
        }
        const int sb = scale_byte_from_amax(fmaxf(amax16(x0), amax16(x1)));
        const float inv = inv_scale_from_byte(sb);
        const uint64_t n0 = uint64_t(row) * C + col0;
        const uint2 q0 = quant16<SR>(x0, inv, n0, keys, a.sr_offset);
        const uint2 q1 = quant16<SR>(x1, inv, n0 + 16, keys, a.sr_offset);
        *reinterpret_cast<uint4*>(a.codes + uint64_t(row) * (C >> 1) + (col0 >> 1)) = make_uint4(q0.x, q0.y, q1.x, q1.y);
        if (a.scales) a.scales[i] = uint8_t(sb);
        if (a.scales_mma) a.scales_mma[g * mma_group_bytes + mma_off32(r, s, nchunk)] = uint8_t(sb);
        // advance by the grid stride
        s += ds;
        const uint32_t cs = s >= S ? 1u : 0u;
        s -= cs * S;
        row += drow + cs;
        r += dr + cs;
        const uint32_t cr = r >= R ? 1u : 0u;
        r -= cr * R;
        g += dg + cr;
    }
}

// ---------------------------------------------------------------------------
// 1D blocks along dim 0 (the token dim), output transposed: input [T, F]
// (per group), output [F, T].  Persistent CTAs walk tiles of 128 features x
// (128 tokens for bf16, 64 for binary32), 32 KB each; a 3-deep ring of
// shared-memory buffers is filled by TMA (zero fill at the ragged edges), so
// the next tiles stream in while the current one is quantised.  Each thread
// owns two neighbouring features of one 32-token block: one 4-byte (bf16) or
// 8-byte (binary32) shared load per token gives both, and the RHT and the
// scaling run on packed pairs (two-wide fp32); then per feature the amax,
// scale, rounding and a 16-byte store of codes.
// ---------------------------------------------------------------------------
constexpr int kColsTF = 128;   // features per tile
constexpr int kColsRing = 3;

template <typename InT>
__host__ __device__ constexpr int cols_tt() { return sizeof(InT) == 2 ? 128 : 64; }   // tokens per tile

template <typename InT>
__host__ __device__ constexpr int cols_threads() { return (kColsTF / 2) * (cols_tt<InT>() / 32); }

template <typename InT>
__host__ __device__ constexpr uint32_t cols_tile_bytes() { return uint32_t(cols_tt<InT>() * kColsTF * sizeof(InT)); }

template <typename InT>
__host__ __device__ constexpr uint32_t cols_stage_bytes() { return uint32_t(kColsTF * (cols_tt<InT>() / 2)); }

// Token-dim code staging: byte offset, inside one tile's buffer, of the 16
// code bytes of the tile's feature row fl and 32-token block c.  Rows are
// kTT/2 bytes; chunk c of row fl sits at chunk c ^ ((fl >> 1) & (kTT/32 - 1)).
template <typename InT>
__host__ __device__ constexpr int cols_stage_off(int fl, int c) {
    return fl * (cols_tt<InT>() / 2) + 16 * (c ^ ((fl >> 1) & (cols_tt<InT>() / 32 - 1)));
}

// the ring, its barriers and the abort flag, and two token-dim code buffers
template <typename InT>
__host__ __device__ constexpr uint32_t cols_smem_bytes() {
    return kColsRing * cols_tile_bytes<InT>() + 64 + 128 + 2 * cols_stage_bytes<InT>();
}

// Tile walk of a persistent CTA: tiles first, first + step, ... of a
// [groups][token tiles][feature tiles] grid, kept as (g, tt, tf) and advanced
// with adds and one conditional wrap per level (no division in the loop).
struct TileWalk {
    uint32_t g, tt, tf;
    uint32_t sg, stt, stf;   // the step, decomposed the same way
    uint32_t ntt, ntf;
    __device__ void init(uint32_t t, uint32_t step, uint32_t ntt_, uint32_t ntf_) {
        ntt = ntt_;
        ntf = ntf_;
        const uint32_t per = ntt * ntf;
        g = t / per;
        tt = (t - g * per) / ntf;
        tf = t - g * per - tt * ntf;
        sg = step / per;
        stt = (step - sg * per) / ntf;
        stf = step - sg * per - stt * ntf;
    }
    __device__ __forceinline__ void advance() {
        tf += stf;
        const uint32_t c1 = tf >= ntf ? 1u : 0u;
        tf -= c1 * ntf;
        tt += stt + c1;
        const uint32_t c2 = tt >= ntt ? 1u : 0u;
        tt -= c2 * ntt;
        g += sg + c2;
    }
};

// Dual mode (DUAL): every tile is also quantised in 1x32 blocks along the
// features (the layout of quant1d_rows_kernel) into a.r_*, so one read of
// the input feeds both the contraction-dim codes and the token-dim codes.
// Each thread takes two of the tile's (token row, 32-feature block) pairs.
// Indices are 32-bit (the host keeps groups * rows and groups * cols below
// 2^31); products that address memory or count elements are widened.
template <typename InT, bool RHT, bool SR, bool DUAL = false, bool RHT_R = false>
__global__ void __launch_bounds__(256, 2) quant1d_cols_kernel(const __grid_constant__ CUtensorMap tm_in, const __grid_constant__ QuantArgs a,
                                                           uint32_t* status) {
    constexpr int kTT = cols_tt<InT>();
    constexpr int kTF = kColsTF;
    constexpr int kPairs = kTF / 2;
    extern __shared__ uint8_t cols_smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(cols_smem_raw) + 127) & ~uintptr_t(127));
    constexpr uint32_t kTile = cols_tile_bytes<InT>();
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kColsRing * kTile);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kColsRing * kTile + 8 * kColsRing);
    // Token-dim codes: a lane's 16 bytes go to its own feature row, so the
    // warp's direct store covers 32 rows with half sectors.  Except in the
    // dual SR kernel (issue-bound, where the extra instructions cost more than
    // the stores save), each tile's codes are staged as [feature][kTT / 2
    // bytes] (cols_stage_off, two buffers) and written after the tile's
    // barrier as whole row segments.
    constexpr bool kStageCodes = !(DUAL && SR);
    constexpr uint32_t kStage = cols_stage_bytes<InT>();
    constexpr int kCh = kTT / 32;
    uint8_t* stage_base = smem + kColsRing * kTile + 64 + 128;
    const uint32_t T = uint32_t(a.rows), F = uint32_t(a.cols);
    const uint32_t ntt = (T + kTT - 1) / kTT, ntf = (F + kTF - 1) / kTF;
    const uint32_t ntiles = uint32_t(a.groups) * ntt * ntf;
    const uint32_t first = blockIdx.x, step = gridDim.x;
    if (ntiles == 0) return;
    const uint32_t mine = first < ntiles ? (ntiles - first + step - 1) / step : 0u;
    if (threadIdx.x == 0) {
        for (int b = 0; b < kColsRing; ++b) mbar_init(&full[b], 1);
        *abort_flag = 0;
        fence_barrier_init();
        prefetch_tensormap(&tm_in);
        TileWalk w;
        w.init(first, step, ntt, ntf);
        for (uint32_t i = 0; i < mine && i < uint32_t(kColsRing); ++i) {
            mbar_arrive_expect_tx(&full[i], kTile);
            tma_load_3d(smem + i * kTile, &tm_in, &full[i], int32_t(w.tf * kTF), int32_t(w.tt * kTT), int32_t(w.g));
            w.advance();
        }
    }
    __syncthreads();
    TileWalk cur;                 // the tile being quantised
    cur.init(first, step, ntt, ntf);
    TileWalk nxt;                 // thread 0: the tile the freed buffer is refilled with
    if (threadIdx.x == 0) nxt.init(first + uint32_t(kColsRing) * step, step, ntt, ntf);
    const PhiloxKeys& keys = a.sr_keys;   // kernel parameters: read from the constant bank
    const int pr = threadIdx.x % kPairs;   // features 2 pr, 2 pr + 1 of the tile
    const int blk = threadIdx.x / kPairs;  // 32-token block of the tile
    const uint32_t S = T >> 5, SF = F >> 5;
    const uint32_t nchunk_c = (S + 3) >> 2, nchunk_r = (SF + 3) >> 2;
    const uint64_t mma_group_c = uint64_t((F + 127) >> 7) * nchunk_c * 512u;   // scale bytes of one group (col)
    const uint64_t mma_group_r = uint64_t((T + 127) >> 7) * nchunk_r * 512u;   // (row direction)
    for (uint32_t i = 0; i < mine; ++i) {
        const int b = int(i % kColsRing);
        const uint32_t phase = (i / kColsRing) & 1u;
        const bool got = mbar_wait_bounded(&full[b], phase, abort_flag, status, kRoleProducer);
        const uint32_t g = cur.g, t0 = cur.tt * kTT, f0 = cur.tf * kTF;
        const uint32_t f = f0 + 2 * pr;
        const uint32_t tb = t0 + blk * 32;
        if (got && f < F && tb < T) {
            const uint8_t* tile = smem + b * kTile;   // [kTT][kTF] of InT, dense
            uint64_t p[32];                            // token k: (feature f, feature f + 1)
#pragma unroll
            for (int k = 0; k < 32; ++k) {
                const int e = (blk * 32 + k) * kTF + 2 * pr;
                if constexpr (sizeof(InT) == 2) {
                    const uint32_t w = *reinterpret_cast<const uint32_t*>(tile + 2 * e);
                    p[k] = f2_pack(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
                } else {
                    p[k] = *reinterpret_cast<const uint64_t*>(tile + 4 * e);
                }
            }
            if constexpr (RHT) {
                rht16x2(*reinterpret_cast<uint64_t(*)[16]>(&p[0]), a.rht_mul2);
                rht16x2(*reinterpret_cast<uint64_t(*)[16]>(&p[16]), a.rht_mul2);
            }
            float m0 = 0.0f, m1 = 0.0f;
#pragma unroll
            for (int k = 0; k < 32; k += 2) {
                float lo0, hi0, lo1, hi1;
                f2_unpack(p[k], lo0, hi0);
                f2_unpack(p[k + 1], lo1, hi1);
                m0 = fmax3_abs(m0, lo0, lo1);
                m1 = fmax3_abs(m1, hi0, hi1);
            }
            const int sb0 = scale_byte_from_amax(m0), sb1 = scale_byte_from_amax(m1);
            const uint64_t inv = f2_pack(inv_scale_from_byte(sb0), inv_scale_from_byte(sb1));
            float v0[32], v1[32];
#pragma unroll
            for (int k = 0; k < 32; ++k) f2_unpack(f2_mul(p[k], inv), v0[k], v1[k]);
            const bool two = f + 1 < F;
            const uint32_t orow = g * F + f;   // output row of feature f (groups back to back)
            const uint32_t s = tb >> 5;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                if (h == 1 && !two) break;
                const float* v = h ? v1 : v0;
                const uint64_t n0 = uint64_t(orow + h) * T + tb;
                const uint2 q0 = quant16_scaled<SR>(*reinterpret_cast<const float(*)[16]>(v), n0, keys, a.sr_offset);
                const uint2 q1 = quant16_scaled<SR>(*reinterpret_cast<const float(*)[16]>(v + 16), n0 + 16, keys,
                                                    a.sr_offset);
                if constexpr (kStageCodes) {
                    const int fl = 2 * pr + h;
                    *reinterpret_cast<uint4*>(stage_base + (i & 1u) * kStage + cols_stage_off<InT>(fl, blk)) =
                        make_uint4(q0.x, q0.y, q1.x, q1.y);
                } else {
                    *reinterpret_cast<uint4*>(a.codes + uint64_t(orow + h) * (T >> 1) + (tb >> 1)) =
                        make_uint4(q0.x, q0.y, q1.x, q1.y);
                }
                const int sb = h ? sb1 : sb0;
                if (a.scales) a.scales[uint64_t(orow + h) * S + s] = uint8_t(sb);
                if (a.scales_mma) a.scales_mma[g * mma_group_c + mma_off32(f + h, s, nchunk_c)] = uint8_t(sb);
            }
        }
        if constexpr (DUAL) {
            // the same tile, 1x32 blocks along the features
            constexpr int kChunks16 = 32 * int(sizeof(InT)) / 16;   // 16-byte chunks per 32-element block
            const uint8_t* tile = smem + b * kTile;
#pragma unroll   // compile-time trip count (the launch has cols_threads threads)
            for (int e = int(threadIdx.x); e < kTT * (kTF / 32); e += cols_threads<InT>()) {
                const int rr = e / (kTF / 32), fb = e % (kTF / 32);
                const uint32_t t = t0 + rr, fc = f0 + 32 * fb;
                if (!got || t >= T || fc >= F) continue;
                const uint8_t* src = tile + (rr * kTF + 32 * fb) * int(sizeof(InT));
                // bf16: a block is 4 chunks of 16 bytes and half a 128-byte bank
                // row.  Lane l of an 8-lane phase reads chunk j ^ m at step j,
                // m = (fb >> 1) | 2 (rr & 1), so the phase covers 8 distinct
                // 16-byte bank groups; two predicated swap stages restore the
                // order (no register array indexed at run time).
                uint4 w[kChunks16];
                const int m = sizeof(InT) == 2 ? (((fb >> 1) | ((rr & 1) << 1)) & 3) : 0;
#pragma unroll
                for (int j = 0; j < kChunks16; ++j) w[j] = *reinterpret_cast<const uint4*>(src + 16 * (j ^ m));
                const uint32_t row = g * T + t;   // output row (groups back to back)
                const uint64_t n0 = uint64_t(row) * F + fc;
                int sb;
                uint32_t cw[4];                   // codes of elements 8j .. 8j + 7
                if constexpr (sizeof(InT) == 2 && !RHT_R) {
                    // Slot j holds chunk j ^ m.  The block maximum and the
                    // scaling do not depend on the order, so the data stay
                    // in slot order and only the four code words (and, for
                    // SR, the chunks' random words) are permuted.
                    float x[32];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const uint32_t ww[4] = {w[j].x, w[j].y, w[j].z, w[j].w};
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            x[8 * j + 2 * q] = __uint_as_float(ww[q] << 16);
                            x[8 * j + 2 * q + 1] = __uint_as_float(ww[q] & 0xFFFF0000u);
                        }
                    }
                    sb = scale_byte_from_amax(fmaxf(amax16(*reinterpret_cast<float(*)[16]>(&x[0])),
                                                    amax16(*reinterpret_cast<float(*)[16]>(&x[16]))));
                    const uint64_t inv2 = f2_pack(inv_scale_from_byte(sb), inv_scale_from_byte(sb));
                    float v[32];
#pragma unroll
                    for (int i = 0; i < 32; i += 2) f2_unpack(f2_mul(f2_pack(x[i], x[i + 1]), inv2), v[i], v[i + 1]);
                    if constexpr (SR) {
                        // chunk c takes words 2c, 2c + 1 of the block's two
                        // Philox calls (elements 0-15 and 16-31)
                        const uint64_t gq = n0 >> 4;
                        const Philox4 r0 = philox4x32_10(uint32_t(gq), uint32_t(gq >> 32), a.r_sr_offset, 0u, keys);
                        const Philox4 r1 =
                            philox4x32_10(uint32_t(gq + 1), uint32_t((gq + 1) >> 32), a.r_sr_offset, 0u, keys);
                        uint32_t R[8] = {r0.w[0], r0.w[1], r0.w[2], r0.w[3], r1.w[0], r1.w[1], r1.w[2], r1.w[3]};
                        if (m & 1) {
                            uint32_t tq;
                            tq = R[0]; R[0] = R[2]; R[2] = tq;
                            tq = R[1]; R[1] = R[3]; R[3] = tq;
                            tq = R[4]; R[4] = R[6]; R[6] = tq;
                            tq = R[5]; R[5] = R[7]; R[7] = tq;
                        }
                        if (m & 2) {
                            uint32_t tq;
                            tq = R[0]; R[0] = R[4]; R[4] = tq;
                            tq = R[1]; R[1] = R[5]; R[5] = tq;
                            tq = R[2]; R[2] = R[6]; R[6] = tq;
                            tq = R[3]; R[3] = R[7]; R[7] = tq;
                        }
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            cw[j] = e2m1x4_sr(v[8 * j], v[8 * j + 1], v[8 * j + 2], v[8 * j + 3], R[2 * j]) |
                                    (e2m1x4_sr(v[8 * j + 4], v[8 * j + 5], v[8 * j + 6], v[8 * j + 7], R[2 * j + 1])
                                     << 16);
                    } else {
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            cw[j] = e2m1x8_rn(v[8 * j], v[8 * j + 1], v[8 * j + 2], v[8 * j + 3], v[8 * j + 4],
                                              v[8 * j + 5], v[8 * j + 6], v[8 * j + 7]);
                    }
                    // chunk c's codes sit in cw[c ^ m]
                    if (m & 1) {
                        uint32_t tq;
                        tq = cw[0]; cw[0] = cw[1]; cw[1] = tq;
                        tq = cw[2]; cw[2] = cw[3]; cw[3] = tq;
                    }
                    if (m & 2) {
                        uint32_t tq;
                        tq = cw[0]; cw[0] = cw[2]; cw[2] = tq;
                        tq = cw[1]; cw[1] = cw[3]; cw[3] = tq;
                    }
                } else {
                    if constexpr (sizeof(InT) == 2) {
                        if (m & 1) {
                            const uint4 t01 = w[0], t23 = w[2];
                            w[0] = w[1]; w[1] = t01; w[2] = w[3]; w[3] = t23;
                        }
                        if (m & 2) {
                            const uint4 tq0 = w[0], tq1 = w[1];
                            w[0] = w[2]; w[1] = w[3]; w[2] = tq0; w[3] = tq1;
                        }
                    }
                    float x[32];
#pragma unroll
                    for (int j = 0; j < kChunks16; ++j) {
                        const uint32_t ww[4] = {w[j].x, w[j].y, w[j].z, w[j].w};
                        if constexpr (sizeof(InT) == 2) {
#pragma unroll
                            for (int q = 0; q < 4; ++q) {
                                x[8 * j + 2 * q] = __uint_as_float(ww[q] << 16);
                                x[8 * j + 2 * q + 1] = __uint_as_float(ww[q] & 0xFFFF0000u);
                            }
                        } else {
#pragma unroll
                            for (int q = 0; q < 4; ++q) x[4 * j + q] = __uint_as_float(ww[q]);
                        }
                    }
                    float (&x0)[16] = *reinterpret_cast<float(*)[16]>(&x[0]);
                    float (&x1)[16] = *reinterpret_cast<float(*)[16]>(&x[16]);
                    if constexpr (RHT_R) rht16_pair(x0, x1, a.r_rht_mul2);
                    sb = scale_byte_from_amax(fmaxf(amax16(x0), amax16(x1)));
                    const float inv = inv_scale_from_byte(sb);
                    const uint2 q0 = quant16<SR>(x0, inv, n0, keys, a.r_sr_offset);
                    const uint2 q1 = quant16<SR>(x1, inv, n0 + 16, keys, a.r_sr_offset);
                    cw[0] = q0.x;
                    cw[1] = q0.y;
                    cw[2] = q1.x;
                    cw[3] = q1.y;
                }
                *reinterpret_cast<uint4*>(a.r_codes + uint64_t(row) * (F >> 1) + (fc >> 1)) =
                    make_uint4(cw[0], cw[1], cw[2], cw[3]);
                const uint32_t sc = fc >> 5;
                if (a.r_scales) a.r_scales[uint64_t(row) * SF + sc] = uint8_t(sb);
                if (a.r_scales_mma) a.r_scales_mma[g * mma_group_r + mma_off32(t, sc, nchunk_r)] = uint8_t(sb);
            }
        }
        __syncthreads();  // buffer b fully read: refill it with tile i + kColsRing
        if (kStageCodes && !*abort_flag) {
            // the tile's token-dim codes: whole kTT/2-byte row segments; the
            // buffer is written again two tiles later, after the next barrier
            const uint8_t* stg = stage_base + (i & 1u) * kStage;
#pragma unroll
            for (int it = 0; it < kTF * kCh / cols_threads<InT>(); ++it) {
                const int idx = it * cols_threads<InT>() + int(threadIdx.x);
                const int fl = idx / kCh, c = idx % kCh;
                if (f0 + fl < F && t0 + 32 * c < T)
                    *reinterpret_cast<uint4*>(a.codes + uint64_t(g * F + f0 + fl) * (T >> 1) + ((t0 >> 1) + 16 * c)) =
                        *reinterpret_cast<const uint4*>(stg + cols_stage_off<InT>(fl, c));
            }
        }
        if (threadIdx.x == 0 && i + kColsRing < mine) {
            mbar_arrive_expect_tx(&full[b], kTile);
            tma_load_3d(smem + b * kTile, &tm_in, &full[b], int32_t(nxt.tf * kTF), int32_t(nxt.tt * kTT),
                        int32_t(nxt.g));
            nxt.advance();
        }
        cur.advance();
    }
}

// ---------------------------------------------------------------------------
// 2D 32x32 blocks (weights), optionally with the de-oscillation update.
// One warp per block; lane l owns row l of the block (32 elements), and the
// warps of a CTA take neighbouring blocks of a block row, so the row
// segments they read together share DRAM pages.  The codes of the transpose
// come from a register transpose across the warp (five shuffle stages).
// ---------------------------------------------------------------------------
// Transpose a 32 x 32 matrix of 4-bit codes held one row per lane (nibble k
// of word m of lane r = element (r, 8m + k)) so that lane c ends up with
// column c in the same format.  Five butterfly stages exchange blocks of 16,
// 8, 4, 2 and 1 codes with the lane at distance 16, 8, 4, 2, 1.
__device__ __forceinline__ void transpose32x32_nibbles(uint32_t (&w)[4], int lane) {
    constexpr uint32_t kAll = 0xFFFFFFFFu;
#pragma unroll
    for (int j = 0; j < 2; ++j) {   // 16 codes: words (j) <-> (j + 2)
        const bool up = lane & 16;
        const uint32_t r = __shfl_xor_sync(kAll, up ? w[j] : w[j + 2], 16);
        if (up) w[j] = r;
        else w[j + 2] = r;
    }
#pragma unroll
    for (int j = 0; j < 4; j += 2) {   // 8 codes: words (j) <-> (j + 1)
        const bool up = lane & 8;
        const uint32_t r = __shfl_xor_sync(kAll, up ? w[j] : w[j + 1], 8);
        if (up) w[j] = r;
        else w[j + 1] = r;
    }
#pragma unroll
    for (int j = 0; j < 4; j += 2) {   // 4 codes: 16-bit halves, two words per shuffle
        const uint32_t a = w[j], b = w[j + 1];
        const bool up = lane & 4;
        const uint32_t r = __shfl_xor_sync(kAll, up ? __byte_perm(a, b, 0x5410) : __byte_perm(a, b, 0x7632), 4);
        w[j] = up ? __byte_perm(a, r, 0x3254) : __byte_perm(a, r, 0x5410);
        w[j + 1] = up ? __byte_perm(b, r, 0x3276) : __byte_perm(b, r, 0x7610);
    }
#pragma unroll
    for (int j = 0; j < 4; j += 2) {   // 2 codes: bytes
        const uint32_t a = w[j], b = w[j + 1];
        const bool up = lane & 2;
        const uint32_t r = __shfl_xor_sync(kAll, up ? __byte_perm(a, b, 0x6420) : __byte_perm(a, b, 0x7531), 2);
        w[j] = up ? __byte_perm(a, r, 0x3514) : __byte_perm(a, r, 0x5240);
        w[j + 1] = up ? __byte_perm(b, r, 0x3716) : __byte_perm(b, r, 0x7260);
    }
#pragma unroll
    for (int j = 0; j < 4; j += 2) {   // 1 code: nibbles inside each byte
        const uint32_t a = w[j], b = w[j + 1];
        const bool up = lane & 1;
        // the low (up) or high (!up) nibble of every byte, four per 16 bits
        const uint32_t ta = up ? (a & 0x0F0F0F0Fu) : ((a >> 4) & 0x0F0F0F0Fu);
        const uint32_t tb = up ? (b & 0x0F0F0F0Fu) : ((b >> 4) & 0x0F0F0F0Fu);
        const uint32_t r = __shfl_xor_sync(kAll, __byte_perm(ta | (ta >> 4), tb | (tb >> 4), 0x6420), 1);
        const uint32_t va = __byte_perm(r, 0u, 0x1100), vb = __byte_perm(r, 0u, 0x3322);
        const uint32_t sa = (va & 0x000F000Fu) | ((va >> 4) & 0x0F000F00u);   // nibble k -> low nibble of byte k
        const uint32_t sb = (vb & 0x000F000Fu) | ((vb >> 4) & 0x0F000F00u);
        w[j] = up ? ((a & 0xF0F0F0F0u) | sa) : ((a & 0x0F0F0F0Fu) | (sa << 4));
        w[j + 1] = up ? ((b & 0xF0F0F0F0u) | sb) : ((b & 0x0F0F0F0Fu) | (sb << 4));
    }
}

template <typename InT, bool RHT, bool SR, bool DEOSC>
__device__ __forceinline__ void quant2d_block(const QuantArgs& a, int64_t g, int64_t bi, int64_t bj, int lane,
                                              float (&x0)[16], float (&x1)[16], uint32_t (&s)[8]) {
    const int64_t R = a.rows, C = a.cols;
    const int64_t nbr = R >> 5, nbc = C >> 5;
    const int64_t r = bi * 32 + lane;
    const int64_t c0 = bj * 32;
    if constexpr (RHT) rht16_pair(x0, x1, a.rht_mul2);
    float m = fmaxf(amax16(x0), amax16(x1));
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    const int sb = scale_byte_from_amax(m);
    const float inv = inv_scale_from_byte(sb);
    const uint64_t n0 = (uint64_t(g) * uint64_t(R) + uint64_t(r)) * uint64_t(C) + uint64_t(c0);
    const PhiloxKeys& keys = a.sr_keys;   // kernel parameters: read from the constant bank
    uint2 q0 = quant16<SR>(x0, inv, n0, keys, a.sr_offset);
    uint2 q1 = quant16<SR>(x1, inv, n0 + 16, keys, a.sr_offset);
    uint32_t w[4] = {q0.x, q0.y, q1.x, q1.y};  // 32 codes of row r, nibble k = element k
    const int64_t widx = (g * R + r) * C + c0;  // weight index of element 0 of this row
    if constexpr (DEOSC) {
        // Byte-parallel state update: four weights per 32-bit word.  The
        // codes of 8 weights (one nibble each) are spread to two words of
        // 4 bytes, updated with carry-free byte arithmetic, and packed back.
        const bool reset = a.step > 0 && a.reset_period > 0 && (a.step % a.reset_period) == 0;
        const uint32_t thr_bias = (0x80u - a.flip_threshold) * 0x01010101u;
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            const uint32_t ev = w[m] & 0x0F0F0F0Fu;          // codes 8m+0, +2, +4, +6
            const uint32_t od = (w[m] >> 4) & 0x0F0F0F0Fu;   // codes 8m+1, +3, +5, +7
            uint32_t q[2] = {__byte_perm(ev, od, 0x5140), __byte_perm(ev, od, 0x7362)};
            uint32_t o[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const uint32_t S = s[2 * m + h], Q = q[h];
                if (a.step == 0) {
                    s[2 * m + h] = Q;
                    o[h] = Q;
                    continue;
                }
                const uint32_t prev = S & 0x0F0F0F0Fu;
                uint32_t cnt = (S >> 4) & 0x07070707u;
                uint32_t frz = S & 0x80808080u;
                if (reset) {
                    cnt = 0u;
                    frz = 0u;
                }
                const uint32_t ne = ((Q ^ prev) + 0x7F7F7F7Fu) & 0x80808080u;  // 0x80 where q != prev
                const uint32_t upd = ne & ~frz;                                 // 0x80 where the weight flips
                uint32_t c2 = cnt + (upd >> 7);
                c2 -= (c2 >> 3) & 0x01010101u;                                  // saturate 8 -> 7
                const uint32_t updm = (upd >> 7) * 0xFFu;
                const uint32_t frzm = (frz >> 7) * 0xFFu;
                uint32_t prev2 = (Q & updm) | (prev & ~updm);
                const uint32_t frz2 = frz | (upd & ((c2 + thr_bias) & 0x80808080u));
                o[h] = (prev & frzm) | (Q & ~frzm);                             // frozen: stored code
                if (a.freeze_lower) {
                    // weights freezing now keep the lower-magnitude code of this
                    // flip (magnitudes 0..7 per byte; ties keep Q)
                    const uint32_t nfm = ((frz2 & ~frz) >> 7) * 0xFFu;
                    const uint32_t mp = prev & 0x07070707u, mq = Q & 0x07070707u;
                    const uint32_t ltm = ((((mq | 0x80808080u) - mp - 0x01010101u) & 0x80808080u) >> 7) * 0xFFu;
                    const uint32_t keep = (prev & ltm) | (Q & ~ltm);           // prev where |prev| < |Q|
                    prev2 = (keep & nfm) | (prev2 & ~nfm);
                    o[h] = (keep & nfm) | (o[h] & ~nfm);
                }
                s[2 * m + h] = prev2 | (c2 << 4) | frz2;
            }
            w[m] = __byte_perm(o[0], o[1], 0x6420) | (__byte_perm(o[0], o[1], 0x7531) << 4);
        }
    }
    *reinterpret_cast<uint4*>(a.codes + (widx >> 1)) = make_uint4(w[0], w[1], w[2], w[3]);
    const int64_t S = nbc;  // scales per row
    if (a.scales && lane == 0) a.scales[g * nbr * nbc + bi * nbc + bj] = uint8_t(sb);
    if (a.scales_mma) a.scales_mma[g * mma_scale_bytes(R, S) + mma_scale_offset(r, bj, S)] = uint8_t(sb);
    if (a.codes_t) {
        uint32_t o[4] = {w[0], w[1], w[2], w[3]};
        transpose32x32_nibbles(o, lane);
        // row (c0 + lane) of W^T, columns r0..r0+31 of it are rows of this block
        const int64_t tr = g * C + c0 + lane;
        *reinterpret_cast<uint4*>(a.codes_t + tr * (R >> 1) + (bi * 16)) = make_uint4(o[0], o[1], o[2], o[3]);
        if (a.scales_mma_t)
            a.scales_mma_t[g * mma_scale_bytes(C, nbr) + mma_scale_offset(c0 + lane, bi, nbr)] = uint8_t(sb);
    }
}

constexpr int kQ2dWarps = 8;   // warps (blocks) per CTA
constexpr int kCoalBlkRows = 8, kCoalBlkCols = 1;   // the coalesced kernel's CTA: a column of 8 blocks
constexpr int kCoalWarps = kCoalBlkRows * kCoalBlkCols;   // one warp per block

template <typename InT, bool RHT, bool SR, bool DEOSC>
__global__ void __launch_bounds__(kQ2dWarps * 32, 4) quant2d_kernel(const __grid_constant__ QuantArgs a) {
    // Per warp: the block as 32 rows x 8 chunks of 4 binary32 (chunk c of row
    // r at slot c ^ (r & 7)), and its 32 x 32 state bytes (word c of row r at
    // slot c ^ ((r >> 2) & 7)); both swizzles keep the row-of-4-rows writes
    // and the row-per-lane reads free of bank conflicts.
    __shared__ float4 xs[kQ2dWarps][32 * 8];
    __shared__ uint32_t ss[kQ2dWarps][DEOSC ? 32 * 8 : 1];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t R = a.rows, C = a.cols;
    const int64_t nbr = R >> 5, nbc = C >> 5;
    const int64_t nblocks = a.groups * nbr * nbc;
    const int64_t bid = int64_t(blockIdx.x) * kQ2dWarps + warp;
    if (bid >= nblocks) return;
    const int64_t g = bid / (nbr * nbc);
    const int64_t rem = bid - g * nbr * nbc;
    const int64_t bi = rem / nbc, bj = rem - bi * nbc;
    const int64_t c0 = bj * 32;
    const InT* in = static_cast<const InT*>(a.in) + g * R * a.ld;
    // Coalesced loads: instruction k covers rows 4k..4k+3 of the block, eight
    // lanes per row (lane = 8 q + c: row 4k + q, elements 4c..4c+3).  One warp
    // instruction touching 32 rows at once (a row per lane) reads DRAM at
    // about two thirds of this rate.
    const int q = lane >> 3, c = lane & 7;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const int rr = 4 * k + q;
        const InT* src = in + (bi * 32 + rr) * a.ld + c0 + 4 * c;
        float4 v;
        if constexpr (sizeof(InT) == 4) {
            v = __ldg(reinterpret_cast<const float4*>(src));
        } else {
            const uint2 u = __ldg(reinterpret_cast<const uint2*>(src));
            v = make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xFFFF0000u),
                            __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xFFFF0000u));
        }
        xs[warp][rr * 8 + (c ^ (rr & 7))] = v;
        if constexpr (DEOSC)
            ss[warp][rr * 8 + (c ^ k)] =
                __ldg(reinterpret_cast<const uint32_t*>(a.state + (g * R + bi * 32 + rr) * C + c0 + 4 * c));
    }
    __syncwarp();
    float x0[16], x1[16];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const float4 v = xs[warp][lane * 8 + (j ^ (lane & 7))];
        float* dst = j < 4 ? &x0[4 * j] : &x1[4 * (j - 4)];
        dst[0] = v.x; dst[1] = v.y; dst[2] = v.z; dst[3] = v.w;
    }
    uint32_t s[8];
    if constexpr (DEOSC) {
#pragma unroll
        for (int j = 0; j < 8; ++j) s[j] = ss[warp][lane * 8 + (j ^ ((lane >> 2) & 7))];
    }
    quant2d_block<InT, RHT, SR, DEOSC>(a, g, bi, bj, lane, x0, x1, s);
    if constexpr (DEOSC) {
        // the updated state goes back through the same swizzled tile and out
        // in the coalesced layout (rows 4k..4k+3 per instruction)
#pragma unroll
        for (int j = 0; j < 8; ++j) ss[warp][lane * 8 + (j ^ ((lane >> 2) & 7))] = s[j];
        __syncwarp();
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const int rr = 4 * k + q;
            *reinterpret_cast<uint32_t*>(a.state + (g * R + bi * 32 + rr) * C + c0 + 4 * c) = ss[warp][rr * 8 + (c ^ k)];
        }
    }
}

// ---------------------------------------------------------------------------
// 2D 32x32 blocks with nearest rounding (weights), optionally with the
// de-oscillation update, computed in the coalesced layout: lane l = 8 q + c
// holds rows 4k + q (k = 0..7), elements 4c..4c+3 of its block, so every
// load and store instruction of the warp covers 4 rows x 8 lanes of
// contiguous bytes.  One 32-bit state word per row feeds the byte-parallel
// de-oscillation update directly.  Codes leave as 16-bit pieces; the W^T
// codes are built by an in-lane nibble transpose, a 4 x 4 word transpose
// across the lanes 8 apart, and a second in-lane nibble transpose.
// ---------------------------------------------------------------------------
// Nibble-index bit swap on a 32-nibble vector in four 32-bit words (nibble
// i = word i >> 3, position i & 7): exchanges index bits A < B, i.e. swaps
// the nibbles at p and p + 2^B - 2^A for every p with bit A set and bit B
// clear.  Bits 0-2 index inside a word, bits 3-4 the word.
__host__ __device__ constexpr uint32_t nib_mask_pairs(int a, int b) {
    uint32_t m = 0;
    for (int n = 0; n < 8; ++n)
        if (((n >> a) & 1) && !((n >> b) & 1)) m |= 0xFu << (4 * n);
    return m;
}

__host__ __device__ constexpr uint32_t nib_mask_clear(int a) {
    uint32_t m = 0;
    for (int n = 0; n < 8; ++n)
        if (!((n >> a) & 1)) m |= 0xFu << (4 * n);
    return m;
}

template <int A, int B>
__device__ __forceinline__ void nib_swap(uint32_t (&w)[4]) {
    static_assert(A < B && B <= 4, "index bits");
    if constexpr (B <= 2) {
        constexpr int d = 4 * ((1 << B) - (1 << A));
        constexpr uint32_t M = nib_mask_pairs(A, B);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t t = ((w[i] >> d) ^ w[i]) & M;
            w[i] ^= t ^ (t << d);
        }
    } else if constexpr (A <= 2) {
        constexpr int bb = B - 3, sh = 4 << A;
        constexpr uint32_t M = nib_mask_clear(A);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            if ((i >> bb) & 1) continue;
            const int j = i + (1 << bb);
            const uint32_t t = ((w[i] >> sh) ^ w[j]) & M;
            w[j] ^= t;
            w[i] ^= t << sh;
        }
    } else {
        // both bits index the words (A = 3, B = 4): swap words 1 and 2
        const uint32_t t = w[1];
        w[1] = w[2];
        w[2] = t;
    }
}

// W^T staging of the column-of-blocks CTA.  Lane l of the warp of block row
// bil (block column bjl) leaves its 16 W^T bytes in slot
// coal_wt_slot(bjl, l, bil); thread t writes slot t out, which holds piece
// t % kCoalBlkRows of the row pair index t / kCoalBlkRows.  The piece of lane
// l of block column bj is W^T row coal_wt_row(bj, l) of its group.
__host__ __device__ constexpr int coal_wt_slot(int bjl, int lane, int bil) {
    return (bjl * 32 + lane) * kCoalBlkRows + bil;
}
__host__ __device__ constexpr int64_t coal_wt_row(int64_t bj, int lane) {
    return bj * 32 + 4 * (lane & 7) + (lane >> 3);
}

// One 32x32 block of the coalesced layout (lane 8q + c holds rows 4k + q,
// elements 4c..4c+3): block maximum, scale, codes, de-oscillation state,
// and the block's W^T codes, which go to *ct (16 bytes of W^T row
// c0 + 4c + q) for the CTA to write out.
template <typename InT, bool DEOSC>
__device__ __forceinline__ void coal_block(const QuantArgs& a, int64_t g, int64_t bi, int64_t bj, int lane,
                                           uint4* ct) {
    const int q = lane >> 3, c = lane & 7;
    const int64_t R = a.rows, C = a.cols;
    const int64_t nbr = R >> 5, nbc = C >> 5;
    const int64_t c0 = bj * 32;
    const InT* in = static_cast<const InT*>(a.in) + g * R * a.ld;
    const int64_t row0 = g * R + bi * 32;   // global row of the block's row 0
    float v[8][4];
    uint32_t st[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const int rr = 4 * k + q;
        const InT* src = in + (bi * 32 + rr) * a.ld + c0 + 4 * c;
        if constexpr (sizeof(InT) == 4) {
            const float4 x = __ldg(reinterpret_cast<const float4*>(src));
            v[k][0] = x.x; v[k][1] = x.y; v[k][2] = x.z; v[k][3] = x.w;
        } else {
            const uint2 u = __ldg(reinterpret_cast<const uint2*>(src));
            v[k][0] = __uint_as_float(u.x << 16); v[k][1] = __uint_as_float(u.x & 0xFFFF0000u);
            v[k][2] = __uint_as_float(u.y << 16); v[k][3] = __uint_as_float(u.y & 0xFFFF0000u);
        }
        if constexpr (DEOSC) st[k] = __ldg(reinterpret_cast<const uint32_t*>(a.state + (row0 + rr) * C + c0 + 4 * c));
    }
    float m = 0.0f;
#pragma unroll
    for (int k = 0; k < 8; ++k) m = fmax3_abs(fmax3_abs(m, v[k][0], v[k][1]), v[k][2], v[k][3]);
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    const int sb = scale_byte_from_amax(m);
    const float inv = inv_scale_from_byte(sb);
    uint32_t cw[8];   // codes of row 4k + q, elements 4c..4c+3 (nibble j = element 4c + j)
#pragma unroll
    for (int k = 0; k < 8; ++k)
        cw[k] = e2m1x4_rn(__fmul_rn(v[k][0], inv), __fmul_rn(v[k][1], inv), __fmul_rn(v[k][2], inv),
                          __fmul_rn(v[k][3], inv));
    if constexpr (DEOSC) {
        const bool reset = a.step > 0 && a.reset_period > 0 && (a.step % a.reset_period) == 0;
        const uint32_t thr_bias = (0x80u - a.flip_threshold) * 0x01010101u;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            // the four codes spread to bytes (byte j = element 4c + j)
            const uint32_t Q = __byte_perm(cw[k] & 0x0F0Fu, (cw[k] >> 4) & 0x0F0Fu, 0x5140);
            uint32_t o;
            if (a.step == 0) {
                st[k] = Q;
                o = Q;
            } else {
                const uint32_t S = st[k];
                const uint32_t prev = S & 0x0F0F0F0Fu;
                uint32_t cnt = (S >> 4) & 0x07070707u;
                uint32_t frz = S & 0x80808080u;
                if (reset) {
                    cnt = 0u;
                    frz = 0u;
                }
                const uint32_t ne = ((Q ^ prev) + 0x7F7F7F7Fu) & 0x80808080u;   // 0x80 where q != prev
                const uint32_t upd = ne & ~frz;                                  // 0x80 where the weight flips
                uint32_t c2 = cnt + (upd >> 7);
                c2 -= (c2 >> 3) & 0x01010101u;                                   // saturate 8 -> 7
                const uint32_t updm = (upd >> 7) * 0xFFu;
                const uint32_t frzm = (frz >> 7) * 0xFFu;
                uint32_t prev2 = (Q & updm) | (prev & ~updm);
                const uint32_t frz2 = frz | (upd & ((c2 + thr_bias) & 0x80808080u));
                o = (prev & frzm) | (Q & ~frzm);                                 // frozen: stored code
                if (a.freeze_lower) {
                    const uint32_t nfm = ((frz2 & ~frz) >> 7) * 0xFFu;
                    const uint32_t mp = prev & 0x07070707u, mq = Q & 0x07070707u;
                    const uint32_t ltm = ((((mq | 0x80808080u) - mp - 0x01010101u) & 0x80808080u) >> 7) * 0xFFu;
                    const uint32_t keep = (prev & ltm) | (Q & ~ltm);
                    prev2 = (keep & nfm) | (prev2 & ~nfm);
                    o = (keep & nfm) | (o & ~nfm);
                }
                st[k] = prev2 | (c2 << 4) | frz2;
            }
            const uint32_t t = (o & 0x0F0F0F0Fu) | ((o & 0x0F0F0F0Fu) >> 4);   // byte 0: n0 n1, byte 2: n2 n3
            cw[k] = __byte_perm(t, 0u, 0x4420) & 0xFFFFu;
            *reinterpret_cast<uint32_t*>(a.state + (row0 + 4 * k + q) * C + c0 + 4 * c) = st[k];
        }
    }
#pragma unroll
    for (int k = 0; k < 8; ++k)
        *reinterpret_cast<uint16_t*>(a.codes + (row0 + 4 * k + q) * (C >> 1) + (c0 >> 1) + 2 * c) = uint16_t(cw[k]);
    if (a.scales && lane == 0) a.scales[g * nbr * nbc + bi * nbc + bj] = uint8_t(sb);
    if (a.scales_mma) a.scales_mma[g * mma_scale_bytes(R, nbc) + mma_scale_offset(bi * 32 + lane, bj, nbc)] = uint8_t(sb);
    if (a.codes_t) {
        // rows 8 m .. 8 m + 7 of this lane's 8 x 4 code matrix (row k, column j) -> words
        uint32_t w[4] = {cw[0] | (cw[1] << 16), cw[2] | (cw[3] << 16), cw[4] | (cw[5] << 16), cw[6] | (cw[7] << 16)};
        // nibble 4k + j -> 8j + k: word j = column 4c + j over rows 4k + q
        nib_swap<0, 2>(w);
        nib_swap<1, 3>(w);
        nib_swap<2, 4>(w);
        nib_swap<3, 4>(w);
        // lane (q, c) gathers column 4c + q from the lanes (q', c), q' = 0..3
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const bool up = lane & 16;
            const uint32_t r = __shfl_xor_sync(0xFFFFFFFFu, up ? w[j] : w[j + 2], 16);
            if (up) w[j] = r;
            else w[j + 2] = r;
        }
#pragma unroll
        for (int j = 0; j < 4; j += 2) {
            const bool up = lane & 8;
            const uint32_t r = __shfl_xor_sync(0xFFFFFFFFu, up ? w[j] : w[j + 1], 8);
            if (up) w[j] = r;
            else w[j + 1] = r;
        }
        // word q' = rows 4k + q' (nibble k) -> nibble 4k + q' = row-ordered W^T codes
        nib_swap<0, 3>(w);
        nib_swap<1, 4>(w);
        nib_swap<2, 3>(w);
        nib_swap<3, 4>(w);
        *ct = make_uint4(w[0], w[1], w[2], w[3]);   // W^T row c0 + 4c + q, bytes 16 bi .. 16 bi + 15
        if (a.scales_mma_t)
            a.scales_mma_t[g * mma_scale_bytes(C, nbr) + mma_scale_offset(c0 + lane, bi, nbr)] = uint8_t(sb);
    }
}


// A CTA takes a grid-aligned column of kCoalBlkRows blocks, one warp each.
// Their W^T codes are 16-byte pieces of the same 32 W^T rows at consecutive
// offsets, so they are staged in shared memory and written as whole
// 128-byte row segments (a 16-byte piece per lane per block leaves half
// sectors scattered over 32 rows and made the W^T stores the launch's
// costliest part).  The masters are read in 128-byte row segments.
template <typename InT, bool DEOSC>
__global__ void __launch_bounds__(kCoalWarps * 32) quant2d_coal_kernel(const __grid_constant__ QuantArgs a) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t R = a.rows, C = a.cols;
    const int64_t nbr = R >> 5, nbc = C >> 5;
    const uint32_t tiles_c = uint32_t((nbc + kCoalBlkCols - 1) / kCoalBlkCols);
    const uint32_t tiles_r = uint32_t((nbr + kCoalBlkRows - 1) / kCoalBlkRows);
    const uint32_t per_g = tiles_r * tiles_c;
    const uint32_t cta = blockIdx.x;
    const int64_t g = cta / per_g;
    const uint32_t rem = cta - uint32_t(g) * per_g;
    const uint32_t ti = rem / tiles_c, tj = rem - ti * tiles_c;
    const int bil = warp / kCoalBlkCols, bjl = warp % kCoalBlkCols;
    const int64_t bi = int64_t(ti) * kCoalBlkRows + bil;
    const int64_t bj = int64_t(tj) * kCoalBlkCols + bjl;
    __shared__ uint4 s_ct[kCoalBlkCols * 32 * kCoalBlkRows];   // W^T pieces, by coal_wt_slot
    if (g < a.groups && bi < nbr && bj < nbc) coal_block<InT, DEOSC>(a, g, bi, bj, lane, &s_ct[coal_wt_slot(bjl, lane, bil)]);
    if (!a.codes_t || g >= a.groups) return;   // uniform over the CTA
    __syncthreads();
    // thread t writes piece t % kCoalBlkRows of W^T row t / kCoalBlkRows, so
    // each warp's store covers whole row segments
    static_assert(kCoalBlkCols * 32 * kCoalBlkRows == kCoalWarps * 32, "one W^T piece per thread");
    const int p = int(threadIdx.x) % kCoalBlkRows, pr = int(threadIdx.x) / kCoalBlkRows;
    const int wb = pr >> 5, l = pr & 31;
    const int64_t bis = int64_t(ti) * kCoalBlkRows + p;
    const int64_t bjs = int64_t(tj) * kCoalBlkCols + wb;
    if (bis >= nbr || bjs >= nbc) return;
    const int64_t tr = g * C + coal_wt_row(bjs, l);   // row of W^T
    *reinterpret_cast<uint4*>(a.codes_t + tr * (R >> 1) + bis * 16) = s_ct[threadIdx.x];   // slot (wb, l, p)
}

// ---------------------------------------------------------------------------
// Standalone RHT.  bf16 output: round-to-nearest-even of the binary32 result
// by cvt.rn.bf16x2.f32 (a NaN stays a NaN, infinities and overflow give
// infinities).
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t bf16x2_rn(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// Along the last dim: one thread per 16-element chunk of a row.
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
            for (int k = 0; k < 8; ++k) w[k] = bf16x2_rn(x[2 * k], x[2 * k + 1]);
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

// Along dim 0: one thread per (16-row chunk, column).  Consecutive threads
// take consecutive columns, so every load and store of a warp covers one
// contiguous row segment.  The output keeps the input's [rows, cols] layout.
template <typename InT, bool OUT_BF16>
__global__ void __launch_bounds__(256) rht_dim0_kernel(const InT* __restrict__ in, int64_t rows, int64_t cols,
                                                       int64_t ld, uint32_t signs, void* __restrict__ out) {
    const int64_t total = (rows >> 4) * cols;
    const int64_t stride = int64_t(gridDim.x) * blockDim.x;
    for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < total; i += stride) {
        const int64_t rb = i / cols;
        const int64_t col = i - rb * cols;
        const int64_t r0 = rb << 4;
        float x[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            if constexpr (sizeof(InT) == 2)
                x[k] = __uint_as_float(uint32_t(__ldg(reinterpret_cast<const unsigned short*>(in) + (r0 + k) * ld + col)) << 16);
            else
                x[k] = __ldg(reinterpret_cast<const float*>(in) + (r0 + k) * ld + col);
        }
        rht16(x, signs);
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            if constexpr (OUT_BF16)
                static_cast<uint16_t*>(out)[(r0 + k) * cols + col] = uint16_t(bf16x2_rn(x[k], 0.0f) & 0xFFFFu);
            else
                static_cast<float*>(out)[(r0 + k) * cols + col] = x[k];
        }
    }
}

}  // namespace mxfp4

// gemm.cuh -- grouped block-scaled MXFP4 GEMM for sm_100a (tcgen05).
//
// D_g = deq(A_g) * deq(B_g)^T for the expert linears of an MoE layer: the
// expert matrices dominate compute and memory (roboaidigest "What ALTO
// Actually Does"), and the GEMM sees only the quantised values.
//
// Per CTA (persistent, one per SM, static round-robin over output tiles):
//   warp 0      TMA producer: A/B code tiles (128B-swizzled, K-major) and
//               the UE8M0 scale chunks (bulk copies) into a 4-stage ring.
//   warp 1      tcgen05 issuer (one thread): tcgen05.mma kind::mxf4
//               block_scale (K = 64) into a double-buffered binary32 TMEM
//               accumulator; nothing but MMAs and commits enters its pipe.
//   warps 2-5   epilogue: tcgen05.ld 32 lanes x 32 columns -> swizzled smem
//               -> TMA tensor store, overlapped with the next tile's MMAs.
//   warps 6-9   scale loaders: each stage's UE8M0 chunks smem -> registers
//               -> tcgen05.st into its own TMEM lane quarter (the layout the
//               MMA reads replicates every 32-row chunk into all four
//               quarters).  Staging scales with tcgen05.cp from the MMA
//               thread would serialise with the MMAs: more than three copies
//               per four MMAs stall the tensor pipe on sm_100a, and this tile
//               needs six.
// Tile 128 x 192 (192 divides both expert widths, 2880 and 5760; other N
// are handled by TMA zero fill and store clipping), K-tile
// 256 elements (128 bytes per row, one swizzle atom).  TMEM: accumulators at
// columns [0, 192) and [192, 384); scale slots from column 384 (per stage 8
// columns for A, 16 for B).
//
// Every mbarrier wait is bounded (%globaltimer); an expired wait sets the
// device status word and all roles drain and exit, freeing tensor memory.
#pragma once

#include "common.cuh"
#include "quantize.cuh"

namespace mxfp4 {

namespace gemm {

constexpr int BM = 128;
constexpr int BN = 192;
constexpr int BK = 256;                       // elements per K-tile
constexpr int kStages = 4;
constexpr int kThreads = 320;                 // 10 warps
constexpr uint32_t kABytes = BM * BK / 2;     // 16384
constexpr uint32_t kBBytes = BN * BK / 2;     // 24576
constexpr uint32_t kSFABytes = 1024;          // 2 chunks of (128 rows x 4 scales)
constexpr uint32_t kSFBBytes = 2048;          // 2 row blocks x 2 chunks
constexpr uint32_t kEpiBufBytes = 32 * 32 * 4;  // one 32x32 fp32 box
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAccCols = BN;             // per accumulator
constexpr uint32_t kSfCol0 = 2 * kAccCols;    // 384
constexpr uint32_t kSfColsPerStage = 24;      // 8 (A) + 16 (B)

// shared memory map (offsets from a 1024-aligned base)
constexpr uint32_t kOffA = 0;
constexpr uint32_t kOffB = kOffA + kStages * kABytes;        // 65536
constexpr uint32_t kOffSFA = kOffB + kStages * kBBytes;      // 163840
constexpr uint32_t kOffSFB = kOffSFA + kStages * kSFABytes;  // 167936
constexpr uint32_t kOffEpi = kOffSFB + kStages * kSFBBytes;  // 176128 (1024-aligned)
constexpr uint32_t kOffBar = kOffEpi + 4 * 2 * kEpiBufBytes;  // 208896
constexpr uint32_t kNumBars = 3 * kStages + 2 + 2 + 1;       // full, empty, sfready, tfull, tempty, drain
constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;
constexpr int kMaxGroups = 1023;                               // group offsets staged in smem
constexpr uint32_t kOffGroups = kOffMisc + 64;
constexpr uint32_t kSmemBytes = kOffGroups + (kMaxGroups + 1) * 4 + 1024;  // + alignment slack
static_assert(kOffEpi % 1024 == 0, "epilogue staging must be 1024-aligned");
static_assert(kSfCol0 + kStages * kSfColsPerStage <= kTmemCols, "TMEM budget");

__device__ __forceinline__ int64_t imin64(int64_t x, int64_t y) { return x < y ? x : y; }

struct Args {
    int mode;                 // 0: groups split rows of A (fprop/dgrad); 1: groups split K (wgrad)
    int num_groups;
    const int32_t* offsets;   // [G+1] device
    int64_t M, N, K;          // mode 0: M = rows of A, K = contraction; mode 1: M = rows of A, K = total tokens
    const uint8_t* sfa;
    const uint8_t* sfb;
    int64_t nchunk_a;         // scale chunks per 128-row block of A (ceil(S_a / 4))
    int64_t nchunk_b;
    int64_t nrb_b;            // 128-row blocks of B (per group)
    int64_t sfb_group_bytes;  // mode 0: per-group stride of B's scales
    int m_tiles, n_tiles;     // mode 0: over all rows of A; mode 1: per group
    int64_t total_tiles;
    uint32_t* status;
    // CTA-pair kernel: a K-step loads A and B with one box each through views
    // [chunk][row][256 bytes] of the codes (chunk stride 128 B); k_chunks is
    // the number of chunk positions whose 256 bytes lie inside a row, 0 if
    // the views are not used
    int32_t k_chunks;
    // CTA-pair kernel, binary32 epilogue: store two 32-column chunks per TMA
    // box through a view [column block][row][32 floats] of D (N % 32 == 0)
    int32_t d_pairs;
    // fused epilogue (CTA-pair kernel, mode 0 only): bf16 output and its MXFP4
    // quantisation in 1x32 blocks along N, in place of the binary32 output
    // (bf16 [M][ldy] and codes [M][N/2] leave through tensor maps)
    uint8_t* qscales;         // canonical [M][N/32], may be null
    uint8_t* qscales_mma;     // tensor-core layout of the [M, N/32] scales, may be null
    int32_t q_sr;             // fused epilogue rounding: 0 nearest, 1 stochastic
    uint32_t q_sr_offset;     // Philox counter word 2 of the fused codes (SR)
    PhiloxKeys q_sr_keys;     // round keys of the fused codes' SR seed
};

struct Tile {
    int g;
    int64_t m0, n0;
    int64_t kbeg, kend;       // contraction range (elements)
};

// Map a linear tile index to its group, origin and contraction range, from
// the group offsets staged (and validated) in shared memory.  Every role
// calls this with the same index and sees the same offsets.
__device__ __forceinline__ Tile tile_info(const Args& a, const int32_t* s_off, int64_t t) {
    Tile ti;
    if (a.mode == 0) {
        const int64_t mt = t / a.n_tiles;
        ti.m0 = mt * BM;
        ti.n0 = (t - mt * a.n_tiles) * BN;
        ti.kbeg = 0;
        ti.kend = a.K;
        // last group g with off[g] <= m0 (segments are non-empty where m0 lands)
        int lo = 0, hi = a.num_groups - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (s_off[mid] <= ti.m0) lo = mid;
            else hi = mid - 1;
        }
        ti.g = lo;
    } else {
        const int64_t per = int64_t(a.m_tiles) * a.n_tiles;
        const int g = int(t / per);
        const int64_t rem = t - int64_t(g) * per;
        const int64_t mt = rem / a.n_tiles;
        ti.g = g;
        ti.m0 = mt * BM;
        ti.n0 = (rem - mt * a.n_tiles) * BN;
        ti.kbeg = s_off[g];
        ti.kend = s_off[g + 1];
    }
    return ti;
}

// One pass over the offsets: non-decreasing, multiples of 128, starting at
// 0; mode 0 ends at M, mode 1 at most at K.
__device__ __forceinline__ bool offsets_valid(const Args& a, const int32_t* s_off) {
    if (s_off[0] != 0) return false;
    for (int i = 0; i < a.num_groups; ++i)
        if (s_off[i + 1] < s_off[i] || (s_off[i + 1] & 127) != 0) return false;
    return a.mode == 0 ? s_off[a.num_groups] == int32_t(a.M) : s_off[a.num_groups] <= int32_t(a.K);
}

// UMMA shared-memory descriptor, K-major operand with 128-byte swizzle:
// start address >> 4, leading offset 16 B (unused for swizzled K-major),
// stride 1024 B between 8-row groups, descriptor version 1, layout 2.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
    return uint64_t((saddr & 0x3FFFFu) >> 4) | (uint64_t(1) << 16) | (uint64_t(1024 >> 4) << 32) |
           (uint64_t(1) << 46) | (uint64_t(2) << 61);
}

// Instruction descriptor, kind::mxf4: E2M1 x E2M1, UE8M0 scales, K-major
// A and B, M = 128, N = 192, dense K = 64; scale-factor byte selectors for
// A (bits 29-30) and B (bits 4-5).
__device__ __forceinline__ uint32_t mxf4_idesc(uint32_t sf_id) {
    return (sf_id << 4) | (1u << 7) | (1u << 10) | (uint32_t(BN >> 3) << 17) | (1u << 23) |
           (uint32_t(BM >> 4) << 24) | (sf_id << 29);
}

__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                        const __grid_constant__ CUtensorMap tmD, const Args a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
    uint64_t* full = bars;
    uint64_t* empty = bars + kStages;
    uint64_t* sfready = bars + 2 * kStages;
    uint64_t* tfull = bars + 3 * kStages;
    uint64_t* tempty = bars + 3 * kStages + 2;
    uint64_t* drain = bars + 3 * kStages + 4;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 8);
    volatile int* offsets_ok = reinterpret_cast<volatile int*>(smem + kOffMisc + 16);
    int32_t* s_off = reinterpret_cast<int32_t*>(smem + kOffGroups);
    for (int i = threadIdx.x; i <= a.num_groups; i += blockDim.x) s_off[i] = __ldg(a.offsets + i);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
            mbar_init(&sfready[s], 4);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&tfull[i], 1);
            mbar_init(&tempty[i], 4);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_barrier_init();
        prefetch_tensormap(&tmA);
        prefetch_tensormap(&tmB);
        prefetch_tensormap(&tmD);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    if (threadIdx.x == 0) {
        const bool v = offsets_valid(a, s_off);
        *offsets_ok = v ? 1 : 0;
        if (!v && blockIdx.x == 0) atomicOr(a.status, kStatusBadInput);
    }
    __syncthreads();
    // a rejected offsets array: every role skips every tile, nothing is written
    const int64_t total_tiles = *offsets_ok ? a.total_tiles : 0;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            uint32_t stage = 0, phase = 0;
            bool pend[kStages];
            uint32_t pend_phase[kStages];
            for (int s = 0; s < kStages; ++s) {
                pend[s] = false;
                pend_phase[s] = 0;
            }
            bool ok = true;
            for (int64_t t = blockIdx.x; t < total_tiles && ok; t += gridDim.x) {
                const Tile ti = tile_info(a, s_off, t);
                const int64_t rba = ti.m0 / BM;
                const int64_t rbb = ti.n0 / BM;
                const bool has_rb1 = rbb + 1 < a.nrb_b;
                const uint8_t* sfb_g = a.sfb + (a.mode == 0 ? int64_t(ti.g) * a.sfb_group_bytes : 0);
                for (int64_t k = ti.kbeg; k < ti.kend; k += BK) {
                    if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, abort_flag, a.status, kRoleProducer)) {
                        ok = false;
                        break;
                    }
                    const int64_t chunk = k >> 7;  // 128 elements per scale chunk
                    const uint32_t nca = uint32_t(imin64(2, a.nchunk_a - chunk));
                    const uint32_t ncb = uint32_t(imin64(2, a.nchunk_b - chunk));
                    const uint32_t bytes = kABytes + kBBytes + nca * 512u + ncb * 512u * (has_rb1 ? 2u : 1u);
                    mbar_arrive_expect_tx(&full[stage], bytes);
                    const int32_t xk = int32_t(k >> 1);
                    uint8_t* sA = smem + kOffA + stage * kABytes;
                    uint8_t* sB = smem + kOffB + stage * kBBytes;
                    if (a.mode == 0) {
                        tma_load_2d(sA, &tmA, &full[stage], xk, int32_t(ti.m0));
                        tma_load_3d(sB, &tmB, &full[stage], xk, int32_t(ti.n0), ti.g);
                    } else {
                        tma_load_2d(sA, &tmA, &full[stage], xk, int32_t(ti.m0));
                        tma_load_2d(sB, &tmB, &full[stage], xk, int32_t(ti.n0));
                    }
                    bulk_load(smem + kOffSFA + stage * kSFABytes, a.sfa + (rba * a.nchunk_a + chunk) * 512,
                              nca * 512u, &full[stage]);
                    bulk_load(smem + kOffSFB + stage * kSFBBytes, sfb_g + (rbb * a.nchunk_b + chunk) * 512,
                              ncb * 512u, &full[stage]);
                    if (has_rb1)
                        bulk_load(smem + kOffSFB + stage * kSFBBytes + 1024,
                                  sfb_g + ((rbb + 1) * a.nchunk_b + chunk) * 512, ncb * 512u, &full[stage]);
                    pend[stage] = true;
                    pend_phase[stage] = phase;
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            // drain: every issued copy has landed before the CTA may exit
            for (int s = 0; s < kStages; ++s) {
                if (!pend[s]) continue;
                const uint64_t t0 = globaltimer_ns();
                while (!mbar_try_wait(&full[s], pend_phase[s])) {
                    if (globaltimer_ns() - t0 > kWaitBudgetNs) {
                        atomicOr(a.status, kStatusTimeout | kRoleTeardown);
                        break;
                    }
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            uint32_t stage = 0, phase = 0;
            uint32_t acc = 0, acc_phase = 0;
            bool ok = true;
            for (int64_t t = blockIdx.x; t < total_tiles && ok; t += gridDim.x) {
                const Tile ti = tile_info(a, s_off, t);
                if (ti.kend <= ti.kbeg) continue;
                if (!mbar_wait_bounded(&tempty[acc], acc_phase ^ 1u, abort_flag, a.status, kRoleMma)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + acc * kAccCols;
                const uint32_t sfb_shift = uint32_t((ti.n0 & 127) >> 5);  // 0 or 2 columns
                bool first = true;
                for (int64_t k = ti.kbeg; k < ti.kend; k += BK) {
                    // sfready completes only after all four loader warps observed `full` for this
                    // stage (operand tiles landed) and stored its scales: one wait covers both
                    if (!mbar_wait_bounded(&sfready[stage], phase, abort_flag, a.status, kRoleMma)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sf_cols = tmem_base + kSfCol0 + stage * kSfColsPerStage;
                    const int nmma = int(imin64(BK, ti.kend - k) >> 6);
                    const uint64_t adesc = sw128_desc(smem_u32(smem + kOffA + stage * kABytes));
                    const uint64_t bdesc = sw128_desc(smem_u32(smem + kOffB + stage * kBBytes));
                    for (int kk = 0; kk < nmma; ++kk) {
                        const uint32_t sf_id = uint32_t(kk & 1) * 2u;
                        const uint32_t cl = uint32_t(kk >> 1);
                        tc_mma_mxf4(d_tmem, adesc + uint64_t(2 * kk), bdesc + uint64_t(2 * kk), mxf4_idesc(sf_id),
                                    sf_cols + 4 * cl, sf_cols + 8 + 8 * cl + sfb_shift, first ? 0u : 1u);
                        first = false;
                    }
                    tc_commit(&empty[stage]);
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                tc_commit(&tfull[acc]);
                if (++acc == 2) {
                    acc = 0;
                    acc_phase ^= 1u;
                }
            }
            // drain: all issued tcgen05 operations complete before TMEM is freed
            tc_commit(drain);
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(drain, 0)) {
                if (globaltimer_ns() - t0 > kWaitBudgetNs) {
                    atomicOr(a.status, kStatusTimeout | kRoleTeardown);
                    break;
                }
            }
        }
        __syncwarp();
    } else if (warp >= 6) {
        // ------------------------------------------------------------ scale loaders
        // TMEM scale slot of a stage: A chunks c at columns 4c..4c+3; B row
        // blocks rb0 / rb1 of chunk c at 8 + 8c + {0..3, 4..7}.  Lane r of a
        // quarter receives row r of each 512-byte chunk (16 bytes = the four
        // 32-bit columns of rows r, r+32, r+64, r+96).
        const int q = warp & 3;
        uint32_t stage = 0, phase = 0;
        bool ok = true;
        for (int64_t t = blockIdx.x; t < total_tiles && ok; t += gridDim.x) {
            const Tile ti = tile_info(a, s_off, t);
            for (int64_t k = ti.kbeg; k < ti.kend; k += BK) {
                const bool got = mbar_wait_bounded(&full[stage], phase, abort_flag, a.status, kRoleScales);
                if (!__all_sync(0xFFFFFFFFu, got)) {
                    ok = false;
                    break;
                }
                const uint8_t* sfa_s = smem + kOffSFA + stage * kSFABytes + lane * 16;
                const uint8_t* sfb_s = smem + kOffSFB + stage * kSFBBytes + lane * 16;
                uint32_t ra[8], rb[16];
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    const uint4 va = *reinterpret_cast<const uint4*>(sfa_s + 512 * c);
                    const uint4 v0 = *reinterpret_cast<const uint4*>(sfb_s + 512 * c);
                    const uint4 v1 = *reinterpret_cast<const uint4*>(sfb_s + 1024 + 512 * c);
                    ra[4 * c + 0] = va.x; ra[4 * c + 1] = va.y; ra[4 * c + 2] = va.z; ra[4 * c + 3] = va.w;
                    rb[8 * c + 0] = v0.x; rb[8 * c + 1] = v0.y; rb[8 * c + 2] = v0.z; rb[8 * c + 3] = v0.w;
                    rb[8 * c + 4] = v1.x; rb[8 * c + 5] = v1.y; rb[8 * c + 6] = v1.z; rb[8 * c + 7] = v1.w;
                }
                const uint32_t sf_cols = tmem_base + (uint32_t(32 * q) << 16) + kSfCol0 + stage * kSfColsPerStage;
                tmem_st_32x32b_x8(sf_cols, ra);
                tmem_st_32x32b_x16(sf_cols + 8, rb);
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sfready[stage]);
                if (++stage == kStages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;          // TMEM lane quarter this warp may access (warps 2-5)
        const int ew = warp - 2;         // staging buffers of this warp
        uint8_t* stg = smem + kOffEpi + ew * 2 * kEpiBufBytes;
        uint32_t acc = 0, acc_phase = 0;
        uint32_t buf = 0;
        bool ok = true;
        for (int64_t t = blockIdx.x; t < total_tiles && ok; t += gridDim.x) {
            const Tile ti = tile_info(a, s_off, t);
            const bool zero = ti.kend <= ti.kbeg;
            if (!zero) {
                bool got = true;
                if (lane == 0) got = mbar_wait_bounded(&tfull[acc], acc_phase, abort_flag, a.status, kRoleEpilogue);
                got = __shfl_sync(0xFFFFFFFFu, got ? 1 : 0, 0) != 0;
                if (!got) {
                    ok = false;
                    break;
                }
                tc_fence_after();
            }
            const int32_t row = int32_t(ti.m0 + 32 * q);
            for (int c = 0; c < BN / 32; ++c) {
                uint32_t r[32];
                if (!zero) {
                    tmem_ld_32x32b_x32(tmem_base + (uint32_t(32 * q) << 16) + acc * kAccCols + 32 * c, r);
                    tmem_ld_wait();
                    if (c == BN / 32 - 1) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&tempty[acc]);
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) r[i] = 0u;
                }
                // the staging buffer about to be written must be free
                if (lane == 0) bulk_wait_read<1>();
                __syncwarp();
                uint8_t* sb = stg + buf * kEpiBufBytes;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int pos = j ^ (lane & 7);
                    *reinterpret_cast<uint4*>(sb + lane * 128 + pos * 16) =
                        make_uint4(r[4 * j], r[4 * j + 1], r[4 * j + 2], r[4 * j + 3]);
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    const int32_t col = int32_t(ti.n0 + 32 * c);
                    // boxes wholly outside D are skipped; partial ones are clipped by the TMA unit
                    if (col < a.N && row < a.M) {
                        if (a.mode == 0)
                            tma_store_2d(&tmD, sb, col, row);
                        else
                            tma_store_3d(&tmD, sb, col, row, ti.g);
                    }
                    bulk_commit();
                }
                buf ^= 1u;
            }
            if (!zero) {
                if (++acc == 2) {
                    acc = 0;
                    acc_phase ^= 1u;
                }
            }
        }
        if (lane == 0) bulk_wait_all<0>();
        __syncwarp();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

}  // namespace gemm
}  // namespace mxfp4

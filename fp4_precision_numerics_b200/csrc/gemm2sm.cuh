// gemm2sm.cuh -- grouped block-scaled MXFP4 GEMM on CTA pairs (tcgen05
// cta_group::2), sm_100a.
//
// Same contract as the one-CTA kernel in gemm.cuh (D_g = deq(A_g) deq(B_g)^T,
// binary32 accumulation in tensor memory), with each output tile computed by
// a cluster of two CTAs on neighbouring SMs:
//   - the pair owns two 128-row tiles of A of the same group (an m-tile
//     pair; an odd last tile leaves the second half idle) and one 192-column
//     tile of the output; each CTA stages its own 128 rows of A and its half
//     (96 rows) of B.  A K-step is 512 elements (8 MMAs per barrier round):
//     56 KB per CTA in three stages, A and B each in one TMA box through a
//     [chunk][row][256 bytes] view of the codes (chunk stride 128 B);
//   - the leader CTA's single MMA thread issues tcgen05.mma.cta_group::2
//     (M = 256, N = 192, K = 64) over both CTAs' shared memory and tensor
//     memory, and its commits are multicast to both CTAs' barriers;
//   - warp 0 issues the operand boxes; warp 10 issues the UE8M0 scale copies
//     into a ring of four slots of their own, so they run ahead of the
//     operand ring;
//   - four loader warps read a scale slot (and free it at once), wait until
//     the stage's tensor-memory scale columns are free, and write them with
//     tcgen05.st in the layout of a 128 x 256 one-CTA MMA (every CTA holds its
//     own rows of A's scales and all of B's); the odd-tile offset of the
//     192-wide B window is applied by the loaders, so a stage needs 40 scale
//     columns and two 192-column accumulators still fit in TMEM.  The loaders
//     arrive on the stage's full barrier, so the MMA thread waits once;
//   - every role walks the cluster's units (group, m-tile pair, n-tile)
//     with adds and bounded wraps, no division per unit;
//   - four epilogue warps drain the accumulator: binary32 output in 8 KB TMA
//     stores (two 32-column chunks through a [column block][row][32 floats]
//     view of D), or with FUSED the bf16 output and its 1x32 MXFP4 codes;
//   - every wait is bounded; both CTAs meet at a cluster barrier before the
//     pair's tensor memory is released.
// No TMA multicast is used: every load reads global memory of this GPU into
// the issuing CTA's own shared memory.
#pragma once

#include "common.cuh"
#include "gemm.cuh"
#include "quantize.cuh"

namespace mxfp4 {
namespace gemm2 {

using gemm::Args;
using gemm::imin64;
using gemm::sw128_desc;

constexpr int BM = 128;                          // rows of A per CTA (256 per pair)
constexpr int BN = 192;                          // output columns per tile
constexpr int BNH = BN / 2;                      // rows of B per CTA
constexpr int BK = 512;                          // elements per K-step (one barrier round, 8 MMAs)
constexpr int kSub = BK / 256;                   // 128-byte-wide swizzled boxes per operand and K-step
constexpr int kChunks = BK / 128;                // 4-scale chunks per K-step
constexpr int kStages = 3;
constexpr int kSfStages = 4;                     // scale ring: copies run ahead of the operand ring
constexpr int kThreads = 352;
constexpr uint32_t kABox = BM * 128;             // 16384: 128 rows x 256 elements
constexpr uint32_t kBBox = BNH * 128;            // 12288:  96 rows x 256 elements
constexpr uint32_t kABytes = kSub * kABox;
constexpr uint32_t kBBytes = kSub * kBBox;
constexpr uint32_t kSFABytes = kChunks * 512;    // chunks of 128 rows x 4 scales
constexpr uint32_t kSFBBytes = 2 * kChunks * 512;  // two 128-row blocks of B
constexpr uint32_t kEpiBufBytes = 32 * 32 * 4;
constexpr uint32_t kEpiCodesOff = 32 * 32 * 2;   // fused epilogue: codes after the bf16 rows
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAccCols = BN;
constexpr uint32_t kSfCol0 = 2 * kAccCols;       // 384
constexpr uint32_t kSfColsPerStage = kChunks * (4 + 6);   // per chunk: A 4 columns, B 6 columns
constexpr uint32_t kSfbCol = kChunks * 4;        // B's scales follow A's inside a stage
constexpr int kMaxGroups = 255;

constexpr uint32_t kOffA = 0;
constexpr uint32_t kOffB = kOffA + kStages * kABytes;
constexpr uint32_t kOffSFA = kOffB + kStages * kBBytes;
constexpr uint32_t kOffSFB = kOffSFA + kSfStages * kSFABytes;
constexpr uint32_t kOffEpi = kOffSFB + kSfStages * kSFBBytes;
constexpr uint32_t kOffBar = kOffEpi + 4 * 2 * kEpiBufBytes;
// full, empty (operand stages); sffull, sfempty (scale slots); tfull, tempty; drain
constexpr uint32_t kNumBars = 2 * kStages + 2 * kSfStages + 2 + 2 + 1;
constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;
constexpr uint32_t kOffGroups = kOffMisc + 64;
constexpr uint32_t kSmemBytes = kOffGroups + (kMaxGroups + 1) * 4 + 1024;
static_assert(kOffB % 1024 == 0 && kOffEpi % 1024 == 0, "swizzled tiles must be 1024-aligned");
static_assert(kABox % 1024 == 0 && kBBox % 1024 == 0, "boxes must hold whole swizzle atoms");
static_assert(kSfCol0 + kStages * kSfColsPerStage <= kTmemCols, "TMEM budget");
static_assert(kSmemBytes <= 232448, "shared-memory budget");

// kind::mxf4 instruction descriptor for the pair: M = 256, N = 192.
__device__ __forceinline__ uint32_t idesc_pair(uint32_t sf_id) {
    return (sf_id << 4) | (1u << 7) | (1u << 10) | (uint32_t(BN >> 3) << 17) | (1u << 23) |
           (uint32_t((2 * BM) >> 4) << 24) | (sf_id << 29);
}

struct Unit {
    int g;
    int64_t ma, mb;       // the pair's two 128-row tiles of A (mb may be idle)
    bool vb;              // mb holds rows of this group
    int64_t n0;
    int64_t kbeg, kend;
};

// Units of work: (group, m-tile pair, n-tile), n-tile fastest.  Mode 0 pairs
// the 128-row tiles inside each group (a group of t tiles has (t + 1) / 2
// pairs); mode 1 pairs the row tiles of A, the same for every group, and the
// groups split the contraction.  A cluster takes the units u = first,
// first + step, ...; the walk advances (group g, pair p, n-tile n) by the
// step with adds and bounded wraps -- a group's units are its pairs x
// n_tiles, so the index carries from n into p and from p into the next group
// with pairs (empty groups have none) -- with no division per unit.
struct UnitWalk {
    int g;
    int32_t p, n, dp, dn;
    __host__ __device__ static int32_t pairs_in(const Args& a, const int32_t* s_off, int g) {
        return a.mode == 0 ? (((s_off[g + 1] - s_off[g]) / BM) + 1) / 2 : (a.m_tiles + 1) / 2;
    }
    __host__ __device__ void init(const Args& a, const int32_t* s_off, int64_t u, int64_t step) {
        dp = int32_t(step / a.n_tiles);
        dn = int32_t(step - int64_t(dp) * a.n_tiles);
        int64_t local = u;
        g = 0;
        while (g < a.num_groups) {
            const int64_t units = int64_t(pairs_in(a, s_off, g)) * a.n_tiles;
            if (local < units) break;
            local -= units;
            ++g;
        }
        p = int32_t(local / a.n_tiles);
        n = int32_t(local - int64_t(p) * a.n_tiles);
    }
    __host__ __device__ void advance(const Args& a, const int32_t* s_off) {
        n += dn;
        if (n >= a.n_tiles) {
            n -= a.n_tiles;
            ++p;
        }
        p += dp;
        while (g < a.num_groups) {
            const int32_t pg = pairs_in(a, s_off, g);
            if (p < pg) break;
            p -= pg;
            ++g;
        }
    }
    __host__ __device__ Unit unit(const Args& a, const int32_t* s_off) const {
        Unit un;
        un.g = g;
        un.n0 = int64_t(n) * BN;
        if (a.mode == 0) {
            un.ma = s_off[g] / BM + 2 * int64_t(p);
            un.mb = un.ma + 1;
            un.vb = un.mb * BM < s_off[g + 1];
            un.kbeg = 0;
            un.kend = a.K;
        } else {
            un.ma = 2 * int64_t(p);
            un.mb = un.ma + 1;
            un.vb = un.mb < a.m_tiles;
            un.kbeg = s_off[g];
            un.kend = s_off[g + 1];
        }
        return un;
    }
};

// FUSED (mode 0): the epilogue writes each output element as bf16 (round to
// nearest even) and quantises every 32-column chunk of a row -- one lane's
// registers -- as one 1x32 MXFP4 block of the bf16 values (nearest or
// stochastic rounding), i.e. exactly what mxfp4_quantize gives for the bf16
// output.
template <bool FUSED>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    grouped_gemm_2sm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                            const __grid_constant__ CUtensorMap tmD, const __grid_constant__ CUtensorMap tmQ,
                            const __grid_constant__ CUtensorMap tmA2, const __grid_constant__ CUtensorMap tmB2,
                            const __grid_constant__ CUtensorMap tmD2, const Args a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
    // full (leader): the stage is ready for the pair's MMAs -- A/B of both
    // CTAs landed (2 producer arrivals + bytes) and both CTAs' scales are in
    // tensor memory (8 loader-warp arrivals); one wait per K-step
    uint64_t* full = bars;
    uint64_t* empty = bars + kStages;             // both: the pair's MMAs released the stage
    uint64_t* sffull = bars + 2 * kStages;        // both: a scale slot's chunks landed
    uint64_t* sfempty = sffull + kSfStages;       // both: the 4 loader warps have read a scale slot
    uint64_t* tfull = sfempty + kSfStages;        // both: accumulator ready
    uint64_t* tempty = tfull + 2;                 // leader: both CTAs drained the accumulator (8 warps)
    uint64_t* drain = tempty + 2;                 // both: all of the pair's MMAs completed
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 8);
    volatile int* offsets_ok = reinterpret_cast<volatile int*>(smem + kOffMisc + 16);
    int64_t* s_total = reinterpret_cast<int64_t*>(smem + kOffMisc + 24);
    int32_t* s_off = reinterpret_cast<int32_t*>(smem + kOffGroups);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int64_t cluster = blockIdx.x >> 1, nclusters = gridDim.x >> 1;

    for (int i = threadIdx.x; i <= a.num_groups; i += blockDim.x) s_off[i] = __ldg(a.offsets + i);
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 2 + 8);
            mbar_init(&empty[s], 1);
        }
        for (int s = 0; s < kSfStages; ++s) {
            mbar_init(&sffull[s], 1);
            mbar_init(&sfempty[s], 4);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&tfull[i], 1);
            mbar_init(&tempty[i], 8);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_barrier_init();
        prefetch_tensormap(&tmA);
        prefetch_tensormap(&tmB);
        prefetch_tensormap(&tmD);
        if constexpr (FUSED) prefetch_tensormap(&tmQ);
        if (a.k_chunks > 0) {
            prefetch_tensormap(&tmA2);
            prefetch_tensormap(&tmB2);
        }
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0) {
        const bool v = gemm::offsets_valid(a, s_off);
        *offsets_ok = v ? 1 : 0;
        if (!v && blockIdx.x == 0) atomicOr(a.status, kStatusBadInput);
        int64_t units = 0;
        if (v)
            for (int g = 0; g < a.num_groups; ++g) units += int64_t(UnitWalk::pairs_in(a, s_off, g)) * a.n_tiles;
        *s_total = units;
    }
    __syncthreads();
    cluster_sync_all();   // both CTAs' barriers initialised and TMEM allocated before any cross-CTA traffic
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int64_t total = *s_total;   // 0 when the offsets were rejected

    if (warp == 0) {
        // ------------------------------------------------------------ producer (both CTAs)
        if (lane == 0) {
            uint32_t stage = 0, phase = 0;
            bool pend[kStages];
            uint32_t pend_phase[kStages];
            for (int s = 0; s < kStages; ++s) {
                pend[s] = false;
                pend_phase[s] = 0;
            }
            bool ok = true;
            UnitWalk uw;
            uw.init(a, s_off, cluster, nclusters);
            for (int64_t u = cluster; u < total && ok; u += nclusters, uw.advance(a, s_off)) {
                const Unit un = uw.unit(a, s_off);
                const int64_t mt = (leader || !un.vb) ? un.ma : un.mb;   // an idle half reloads ma (never stored)
                for (int64_t k = un.kbeg; k < un.kend; k += BK) {
                    if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, abort_flag, a.status, kRoleProducer)) {
                        ok = false;
                        break;
                    }
                    const int nsub = un.kend - k > 256 ? 2 : 1;   // boxes of 256 elements this K-step needs
                    const uint32_t full_c = mapa_shared(smem_u32(&full[stage]), 0);
                    mbar_arrive_expect_tx_cluster(full_c, uint32_t(nsub) * (kABox + kBBox));
                    uint8_t* sA = smem + kOffA + stage * kABytes;
                    uint8_t* sB = smem + kOffB + stage * kBBytes;
                    const int32_t brow = int32_t(un.n0 + BNH * int64_t(rank));
                    // the K-step's 256 bytes per row start at byte k/2: chunk kc,
                    // offset xo (0 or 64) inside it
                    const int32_t kc = int32_t(k >> 8), xo = int32_t((k >> 1) & 127);
                    if (nsub == 2 && kc + 2 <= a.k_chunks) {
                        // both halves in one box each for A and B
                        tma_load_3d_pair(sA, &tmA2, full_c, xo, int32_t(mt * BM), kc);
                        if (a.mode == 0)
                            tma_load_4d_pair(sB, &tmB2, full_c, xo, brow, kc, un.g);
                        else
                            tma_load_3d_pair(sB, &tmB2, full_c, xo, brow, kc);
                    } else {
                        for (int j = 0; j < nsub; ++j) {
                            const int32_t xk = int32_t((k + 256 * j) >> 1);
                            tma_load_2d_pair(sA + j * kABox, &tmA, full_c, xk, int32_t(mt * BM));
                            if (a.mode == 0)
                                tma_load_3d_pair(sB + j * kBBox, &tmB, full_c, xk, brow, un.g);
                            else
                                tma_load_2d_pair(sB + j * kBBox, &tmB, full_c, xk, brow);
                        }
                    }
                    pend[stage] = true;
                    pend_phase[stage] = phase;
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            // drain: the leader waits for the operand tiles of both CTAs (they
            // complete on its `full` barriers)
            for (int s = 0; s < kStages; ++s) {
                if (!pend[s] || !leader) continue;
                const uint64_t t1 = globaltimer_ns();
                while (!mbar_try_wait(&full[s], pend_phase[s])) {
                    if (globaltimer_ns() - t1 > kWaitBudgetNs) {
                        atomicOr(a.status, kStatusTimeout | kRoleTeardown);
                        break;
                    }
                }
            }
        }
        __syncwarp();
    } else if (warp == 10) {
        // ------------------------------------------------------------ scale copies (both CTAs)
        // The UE8M0 scales of each K-step go into a ring of kSfStages slots of
        // their own, freed as soon as the loader warps have read them, so the
        // copies run ahead of the operand ring and the scales are in registers
        // by the time a stage's tensor-memory columns are free.
        if (lane == 0) {
            uint32_t slot = 0, sphase = 0;
            bool pend[kSfStages];
            uint32_t pend_phase[kSfStages];
            for (int i = 0; i < kSfStages; ++i) {
                pend[i] = false;
                pend_phase[i] = 0;
            }
            bool ok = true;
            UnitWalk uw;
            uw.init(a, s_off, cluster, nclusters);
            for (int64_t u = cluster; u < total && ok; u += nclusters, uw.advance(a, s_off)) {
                const Unit un = uw.unit(a, s_off);
                const int64_t mt = (leader || !un.vb) ? un.ma : un.mb;
                const int64_t rbb = un.n0 / 128;
                const bool has_rb1 = rbb + 1 < a.nrb_b;
                const uint8_t* sfb_g = a.sfb + (a.mode == 0 ? int64_t(un.g) * a.sfb_group_bytes : 0);
                for (int64_t k = un.kbeg; k < un.kend; k += BK) {
                    if (!mbar_wait_bounded(&sfempty[slot], sphase ^ 1u, abort_flag, a.status, kRoleScales)) {
                        ok = false;
                        break;
                    }
                    const int64_t chunk = k >> 7;
                    const uint32_t nca = uint32_t(imin64(kChunks, a.nchunk_a - chunk));
                    const uint32_t ncb = uint32_t(imin64(kChunks, a.nchunk_b - chunk));
                    mbar_arrive_expect_tx(&sffull[slot], nca * 512u + ncb * 512u * (has_rb1 ? 2u : 1u));
                    bulk_load(smem + kOffSFA + slot * kSFABytes, a.sfa + (mt * a.nchunk_a + chunk) * 512, nca * 512u,
                              &sffull[slot]);
                    bulk_load(smem + kOffSFB + slot * kSFBBytes, sfb_g + (rbb * a.nchunk_b + chunk) * 512,
                              ncb * 512u, &sffull[slot]);
                    if (has_rb1)
                        bulk_load(smem + kOffSFB + slot * kSFBBytes + kChunks * 512,
                                  sfb_g + ((rbb + 1) * a.nchunk_b + chunk) * 512, ncb * 512u, &sffull[slot]);
                    pend[slot] = true;
                    pend_phase[slot] = sphase;
                    if (++slot == kSfStages) {
                        slot = 0;
                        sphase ^= 1u;
                    }
                }
            }
            // drain: every copy this thread issued has landed before the CTA
            // may exit (the loaders consume every slot on a normal exit; after
            // an abort some may still be in flight)
            for (int i = 0; i < kSfStages; ++i) {
                if (!pend[i]) continue;
                const uint64_t t0 = globaltimer_ns();
                while (!mbar_try_wait(&sffull[i], pend_phase[i])) {
                    if (globaltimer_ns() - t0 > kWaitBudgetNs) {
                        atomicOr(a.status, kStatusTimeout | kRoleTeardown);
                        break;
                    }
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer (leader) / drain (both)
        if (lane == 0) {
            if (leader) {
                uint32_t stage = 0, phase = 0;
                uint32_t acc = 0, acc_phase = 0;
                bool ok = true;
                UnitWalk uw;
                uw.init(a, s_off, cluster, nclusters);
                for (int64_t u = cluster; u < total && ok; u += nclusters, uw.advance(a, s_off)) {
                    const Unit un = uw.unit(a, s_off);
                    if (un.kend <= un.kbeg) continue;
                    if (!mbar_wait_bounded(&tempty[acc], acc_phase ^ 1u, abort_flag, a.status, kRoleMma)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t d_tmem = tmem_base + acc * kAccCols;
                    bool first = true;
                    for (int64_t k = un.kbeg; k < un.kend; k += BK) {
                        if (!mbar_wait_bounded(&full[stage], phase, abort_flag, a.status, kRoleMma)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t sf_cols = tmem_base + kSfCol0 + stage * kSfColsPerStage;
                        const int nmma = int(imin64(BK, un.kend - k) >> 6);
                        const uint32_t a_s = smem_u32(smem + kOffA + stage * kABytes);
                        const uint32_t b_s = smem_u32(smem + kOffB + stage * kBBytes);
                        for (int kk = 0; kk < nmma; ++kk) {
                            const uint32_t sf_id = uint32_t(kk & 1) * 2u;
                            const uint32_t cl = uint32_t(kk >> 1);   // 4-scale chunk
                            const uint32_t j = uint32_t(kk >> 2);    // 256-element box
                            const uint64_t koff = uint64_t(2 * (kk & 3));
                            tc_mma_mxf4_pair(d_tmem, sw128_desc(a_s + j * kABox) + koff,
                                             sw128_desc(b_s + j * kBBox) + koff, idesc_pair(sf_id),
                                             sf_cols + 4 * cl, sf_cols + kSfbCol + 6 * cl, first ? 0u : 1u);
                            first = false;
                        }
                        tc_commit_pair_mc(&empty[stage], uint16_t(0x3));
                        if (++stage == kStages) {
                            stage = 0;
                            phase ^= 1u;
                        }
                    }
                    if (!ok) break;
                    tc_commit_pair_mc(&tfull[acc], uint16_t(0x3));
                    if (++acc == 2) {
                        acc = 0;
                        acc_phase ^= 1u;
                    }
                }
                tc_commit_pair_mc(drain, uint16_t(0x3));
            }
        }
        __syncwarp();
    } else if (warp >= 6) {
        // ------------------------------------------------------------ scale loaders (both CTAs)
        // Per K-step: read the scale slot into registers and free it, wait
        // until the pair's MMAs of the stage's previous round have completed
        // (its tensor-memory scale columns are then free), write them, and
        // arrive on the leader's `full` barrier of the stage.
        const int q = warp & 3;
        uint32_t stage = 0, phase = 0;     // operand / tensor-memory stage
        uint32_t slot = 0, sphase = 0;     // scale slot
        bool ok = true;
        UnitWalk uw;
        uw.init(a, s_off, cluster, nclusters);
        for (int64_t u = cluster; u < total && ok; u += nclusters, uw.advance(a, s_off)) {
            const Unit un = uw.unit(a, s_off);
            const int shift = int((un.n0 & 127) >> 5);   // 0 or 2: the 192-wide window inside 256 rows of B
            for (int64_t k = un.kbeg; k < un.kend; k += BK) {
                const bool got = mbar_wait_bounded(&sffull[slot], sphase, abort_flag, a.status, kRoleScales);
                if (!__all_sync(0xFFFFFFFFu, got)) {
                    ok = false;
                    break;
                }
                const uint8_t* sfa_s = smem + kOffSFA + slot * kSFABytes + lane * 16;
                const uint8_t* sfb_s = smem + kOffSFB + slot * kSFBBytes + lane * 16;
                uint32_t ra[16], rb[24];
#pragma unroll
                for (int c = 0; c < kChunks; ++c) {
                    const uint4 va = *reinterpret_cast<const uint4*>(sfa_s + 512 * c);
                    const uint4 v0 = *reinterpret_cast<const uint4*>(sfb_s + 512 * c);                 // rows 0..127
                    const uint4 v1 = *reinterpret_cast<const uint4*>(sfb_s + kChunks * 512 + 512 * c); // 128..255
                    ra[4 * c + 0] = va.x; ra[4 * c + 1] = va.y; ra[4 * c + 2] = va.z; ra[4 * c + 3] = va.w;
                    const uint32_t w8[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
                    for (int j = 0; j < 6; ++j) rb[6 * c + j] = shift ? w8[j + 2] : w8[j];
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&sfempty[slot]);
                if (++slot == kSfStages) {
                    slot = 0;
                    sphase ^= 1u;
                }
                const bool free_cols = mbar_wait_bounded(&empty[stage], phase ^ 1u, abort_flag, a.status, kRoleScales);
                if (!__all_sync(0xFFFFFFFFu, free_cols)) {
                    ok = false;
                    break;
                }
                tc_fence_after();   // the tensor-memory writes follow the MMAs that read these columns
                const uint32_t sf_cols = tmem_base + (uint32_t(32 * q) << 16) + kSfCol0 + stage * kSfColsPerStage;
                tmem_st_32x32b_x16(sf_cols, ra);
                uint32_t rb_lo[16], rb_hi[8];
#pragma unroll
                for (int j = 0; j < 16; ++j) rb_lo[j] = rb[j];
#pragma unroll
                for (int j = 0; j < 8; ++j) rb_hi[j] = rb[16 + j];
                tmem_st_32x32b_x16(sf_cols + kSfbCol, rb_lo);
                tmem_st_32x32b_x8(sf_cols + kSfbCol + 16, rb_hi);
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&full[stage]), 0));
                if (++stage == kStages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue (both CTAs, warps 2-5)
        const int q = warp & 3;
        const int ew = warp - 2;
        uint8_t* stg = smem + kOffEpi + ew * 2 * kEpiBufBytes;
        uint32_t acc = 0, acc_phase = 0;
        uint32_t buf = 0;
        bool ok = true;
        UnitWalk uw;
        uw.init(a, s_off, cluster, nclusters);
        for (int64_t u = cluster; u < total && ok; u += nclusters, uw.advance(a, s_off)) {
            const Unit un = uw.unit(a, s_off);
            const bool zero = un.kend <= un.kbeg;
            const bool valid = leader || un.vb;
            const int64_t mt = leader ? un.ma : un.mb;
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
            const int64_t row = mt * BM + 32 * q;
            for (int c = 0; c < BN / 32; ++c) {
                uint32_t r[32];
                if (!zero) {
                    tmem_ld_32x32b_x32(tmem_base + (uint32_t(32 * q) << 16) + acc * kAccCols + 32 * c, r);
                    tmem_ld_wait();
                    if (c == BN / 32 - 1) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&tempty[acc]), 0));
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) r[i] = 0u;
                }
                if (!valid) continue;
                if constexpr (FUSED) {
                    // bf16 pairs (element 2i in the low half) and the block
                    // maximum of the rounded values
                    uint32_t hb[16];
                    float m = 0.0f;
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        asm("cvt.rn.bf16x2.f32 %0, %1, %2;"
                            : "=r"(hb[i])
                            : "f"(__uint_as_float(r[2 * i + 1])), "f"(__uint_as_float(r[2 * i])));
                        m = fmax3_abs(m, __uint_as_float(hb[i] << 16), __uint_as_float(hb[i] & 0xFFFF0000u));
                    }
                    const int sbyte = scale_byte_from_amax(m);
                    const float inv = inv_scale_from_byte(sbyte);
                    float y[32];   // scaled bf16 values in element order
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        y[2 * i] = __fmul_rn(__uint_as_float(hb[i] << 16), inv);
                        y[2 * i + 1] = __fmul_rn(__uint_as_float(hb[i] & 0xFFFF0000u), inv);
                    }
                    uint32_t qb[4];
                    if (a.q_sr) {
                        // SR as mxfp4_quantize: element n = row * N + col of the
                        // output, one Philox call per 16 elements, word w for
                        // elements 4w..4w+3 of the 16
                        const uint64_t gq = (uint64_t(row + lane) * uint64_t(a.N) + uint64_t(un.n0 + 32 * c)) >> 4;
                        const Philox4 r0 = philox4x32_10(uint32_t(gq), uint32_t(gq >> 32), a.q_sr_offset, 0u,
                                                         a.q_sr_keys);
                        const Philox4 r1 = philox4x32_10(uint32_t(gq + 1), uint32_t((gq + 1) >> 32), a.q_sr_offset,
                                                         0u, a.q_sr_keys);
                        const uint32_t R[8] = {r0.w[0], r0.w[1], r0.w[2], r0.w[3], r1.w[0], r1.w[1], r1.w[2], r1.w[3]};
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            qb[j] = e2m1x4_sr(y[8 * j], y[8 * j + 1], y[8 * j + 2], y[8 * j + 3], R[2 * j]) |
                                    (e2m1x4_sr(y[8 * j + 4], y[8 * j + 5], y[8 * j + 6], y[8 * j + 7], R[2 * j + 1])
                                     << 16);
                    } else {
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            qb[j] = e2m1x8_rn(y[8 * j], y[8 * j + 1], y[8 * j + 2], y[8 * j + 3], y[8 * j + 4],
                                              y[8 * j + 5], y[8 * j + 6], y[8 * j + 7]);
                    }
                    if (lane == 0) bulk_wait_read<1>();
                    __syncwarp();
                    // staging: 32 rows x 64 B of bf16 in the 64-byte swizzle
                    // (16-byte chunk j of row r at chunk j ^ ((r >> 1) & 3)),
                    // then 32 rows x 16 B of codes
                    uint8_t* sbuf = stg + buf * kEpiBufBytes;
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int pos = j ^ ((lane >> 1) & 3);
                        *reinterpret_cast<uint4*>(sbuf + lane * 64 + pos * 16) =
                            make_uint4(hb[4 * j], hb[4 * j + 1], hb[4 * j + 2], hb[4 * j + 3]);
                    }
                    *reinterpret_cast<uint4*>(sbuf + kEpiCodesOff + lane * 16) = make_uint4(qb[0], qb[1], qb[2], qb[3]);
                    fence_proxy_async_smem();
                    __syncwarp();
                    const int64_t col = un.n0 + 32 * c;
                    if (lane == 0) {
                        if (col < a.N && row < a.M) {   // N % 32 == 0: a chunk is all in or all out
                            tma_store_2d(&tmD, sbuf, int32_t(col), int32_t(row));
                            tma_store_2d(&tmQ, sbuf + kEpiCodesOff, int32_t(col >> 1), int32_t(row));
                        }
                        bulk_commit();
                    }
                    const int64_t grow = row + lane;
                    if (grow < a.M && col < a.N) {
                        const int64_t SN = a.N >> 5, s = col >> 5;
                        if (a.qscales) a.qscales[grow * SN + s] = uint8_t(sbyte);
                        if (a.qscales_mma) a.qscales_mma[mma_scale_offset(grow, s, SN)] = uint8_t(sbyte);
                    }
                    buf ^= 1u;
                    continue;
                }
                if (a.d_pairs) {
                    // two 32-column chunks per store: chunk c into buffer c & 1,
                    // one 8 KB box [2][32 rows][32 floats] after the odd chunk
                    if ((c & 1) == 0 && lane == 0) bulk_wait_read<0>();
                    __syncwarp();
                    uint8_t* sb = stg + (c & 1) * kEpiBufBytes;
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const int pos = j ^ (lane & 7);
                        *reinterpret_cast<uint4*>(sb + lane * 128 + pos * 16) =
                            make_uint4(r[4 * j], r[4 * j + 1], r[4 * j + 2], r[4 * j + 3]);
                    }
                    if (c & 1) {
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) {
                            const int64_t col = un.n0 + 32 * (c - 1);
                            if (col < a.N && row < a.M) {
                                if (a.mode == 0)
                                    tma_store_3d(&tmD2, stg, 0, int32_t(row), int32_t(col >> 5));
                                else
                                    tma_store_4d(&tmD2, stg, 0, int32_t(row), int32_t(col >> 5), un.g);
                            }
                            bulk_commit();
                        }
                    }
                    continue;
                }
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
                    const int64_t col = un.n0 + 32 * c;
                    if (col < a.N && row < a.M) {
                        if (a.mode == 0)
                            tma_store_2d(&tmD, sb, int32_t(col), int32_t(row));
                        else
                            tma_store_3d(&tmD, sb, int32_t(col), int32_t(row), un.g);
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
    if (threadIdx.x == 32) {
        // every MMA of the pair (which reads this CTA's shared memory and
        // writes its tensor memory) has completed; timed from here, after
        // this CTA's epilogue has drained its last accumulator
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(drain, 0)) {
            if (globaltimer_ns() - t0 > kWaitBudgetNs) {
                atomicOr(a.status, kStatusTimeout | kRoleTeardown);
                break;
            }
        }
    }
    __syncthreads();
    cluster_sync_all();   // the peer no longer touches this CTA's shared or tensor memory
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, kTmemCols);
    }
}

}  // namespace gemm2
}  // namespace mxfp4

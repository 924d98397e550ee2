// peak.cuh -- tensor-pipe peak probe for the FP4 roofline, sm_100a.
//
// The grouped GEMM's own instruction -- tcgen05.mma.cta_group::2
// kind::mxf4.block_scale (M = 256, N = 192, K = 64, UE8M0 scales in tensor
// memory) -- issued back to back by one thread per CTA pair on operands that
// stay in shared memory, with no loads and no epilogue, so the launch time
// is the tensor pipe's.  The operands are a fixed pseudo-random byte pattern
// (every byte is two finite E2M1 values) and the scales are 2^0, so the
// switching activity resembles real data under the power cap.  The
// accumulator's value is not an output.  It is a measurement helper, not a
// step of the path; the launch shape (one CTA per SM, CTA pairs) is the
// GEMM's.
#pragma once

#include "common.cuh"
#include "gemm2sm.cuh"

namespace mxfp4 {
namespace peak {

constexpr int kThreads = 128;
constexpr uint32_t kOffA = 0;                                   // 128 rows x 128 B (SW128 atoms)
constexpr uint32_t kOffB = gemm2::kABox;                        //  96 rows x 128 B
constexpr uint32_t kOffBar = gemm2::kABox + gemm2::kBBox;
constexpr uint32_t kSmemBytes = gemm2::kSmemBytes;             // as the GEMM: one CTA per SM

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    mma_peak_kernel(int64_t mmas, uint32_t* status) {
    extern __shared__ uint8_t peak_smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(peak_smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* done = reinterpret_cast<uint64_t*>(smem + kOffBar);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffBar + 8);
    const int warp = threadIdx.x >> 5;
    const bool leader = cluster_ctarank() == 0;

    for (uint32_t i = threadIdx.x; i < kOffBar / 4; i += blockDim.x)
        reinterpret_cast<uint32_t*>(smem)[i] = (i + 1u) * 0x9E3779B9u;
    fence_proxy_async_smem();   // the operands are read by the tensor core
    if (threadIdx.x == 0) {
        mbar_init(done, 1);
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc_pair(tmem_slot, gemm2::kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    {
        // scale bytes 127 (2^0) in the columns of the first stage's scales:
        // A's 16 columns, then B's 24
        uint32_t s16[16], s8[8];
#pragma unroll
        for (int i = 0; i < 16; ++i) s16[i] = 0x7F7F7F7Fu;
#pragma unroll
        for (int i = 0; i < 8; ++i) s8[i] = 0x7F7F7F7Fu;
        const uint32_t cols = tmem + (uint32_t(32 * warp) << 16) + gemm2::kSfCol0;
        tmem_st_32x32b_x16(cols, s16);
        tmem_st_32x32b_x16(cols + gemm2::kSfbCol, s16);
        tmem_st_32x32b_x8(cols + gemm2::kSfbCol + 16, s8);
        tmem_st_wait();
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();   // both CTAs' operands, scales and barrier ready
    tc_fence_after();
    if (leader && threadIdx.x == 0) {
        const uint64_t a_desc = gemm::sw128_desc(smem_u32(smem + kOffA));
        const uint64_t b_desc = gemm::sw128_desc(smem_u32(smem + kOffB));
        const uint32_t sf = tmem + gemm2::kSfCol0;
        for (int64_t i = 0; i < mmas; ++i) {
            // the GEMM's K-step pattern: 32-byte K offset inside the 128-byte
            // row, scale chunk and byte selector as for MMA i of a K-step
            const uint32_t kk = uint32_t(i & 7);
            tc_mma_mxf4_pair(tmem, a_desc + uint64_t(2 * (kk & 3)), b_desc + uint64_t(2 * (kk & 3)),
                             gemm2::idesc_pair((kk & 1) * 2u), sf + 4 * (kk >> 1),
                             sf + gemm2::kSfbCol + 6 * (kk >> 1), i > 0 ? 1u : 0u);
        }
        tc_commit_pair_mc(done, uint16_t(0x3));
    }
    if (threadIdx.x == 0) {
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(done, 0)) {
            if (globaltimer_ns() - t0 > kWaitBudgetNs) {
                atomicOr(status, kStatusTimeout | kRoleTeardown);
                break;
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();   // the pair's MMAs no longer read either CTA's memory
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, gemm2::kTmemCols);
    }
}

}  // namespace peak
}  // namespace mxfp4

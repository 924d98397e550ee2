// mxfp4_api.cu -- the C ABI of libmxfp4 (declared in include/mxfp4.h):
// argument validation, tensor-map encoding and kernel launches on the
// caller's stream.  No allocation, no exceptions across the boundary.
#include <cstdarg>
#include <cstdlib>
#include <cstdio>
#include <cstring>
#include <atomic>
#include <map>
#include <mutex>
#include <tuple>
#include <string>

#include "../../include/mxfp4.h"
#include "common.cuh"
#include "gemm.cuh"
#include "gemm2sm.cuh"
#include "peak.cuh"
#include "selftest.cuh"
#include "quantize.cuh"

namespace {

thread_local std::string g_last_error;

__device__ uint32_t g_device_status;

// Snapshots of the status word taken by mxfp4_check_device_status: each
// check reads and clears the word in one atomic exchange on the caller's
// stream and leaves the value it took in its own slot, so checks running at
// the same time on different streams or threads do not overwrite each
// other's result (up to kStatusSlots concurrent checks).
constexpr uint32_t kStatusSlots = 64;
__device__ uint32_t g_status_taken[kStatusSlots];

__global__ void status_take_kernel(uint32_t slot) { g_status_taken[slot] = atomicExch(&g_device_status, 0u); }

mxfp4_status fail(mxfp4_status st, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return st;
}

mxfp4_status ok() { return MXFP4_OK; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

mxfp4_status check_launch(const char* what) {
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(MXFP4_ERR_CUDA, "%s: launch failed: %s", what, cudaGetErrorString(e));
    return ok();
}

int num_sms() {
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n;
}

// CTAs of a persistent kernel that fit on the device at once (every SM
// filled to its occupancy limit), at least one per SM.  Cached per (kernel,
// block size, shared memory, device) under a lock: kernels of one signature
// may differ in registers and hence occupancy.
int64_t resident_ctas_of(const void* kern, int threads, size_t smem) {
    static std::mutex mu;
    static std::map<std::tuple<const void*, int, size_t, int>, int> cache;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) dev = -1;
    const auto key = std::make_tuple(kern, threads, smem, dev);
    {
        std::lock_guard<std::mutex> lock(mu);
        const auto it = cache.find(key);
        if (it != cache.end()) return int64_t(num_sms()) * it->second;
    }
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, threads, smem) != cudaSuccess || n <= 0) {
        cudaGetLastError();
        n = 1;
    }
    std::lock_guard<std::mutex> lock(mu);
    cache[key] = n;
    return int64_t(num_sms()) * n;
}

template <typename K>
int64_t resident_ctas(K kern, int threads, size_t smem) {
    return resident_ctas_of(reinterpret_cast<const void*>(kern), threads, smem);
}

// The pair GEMM's binary32 epilogue stores two 32-column chunks per TMA box.
constexpr bool kEpiPairStores = true;

// Clusters of two CTAs of the pair GEMM that can be resident at once (one
// CTA per SM; an SM left without a partner in its GPC stays idle).
int pair_clusters() {
    static std::atomic<int> cached[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return num_sms() / 2;
    const int c = cached[dev].load();
    if (c > 0) return c;
    int n = 0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * unsigned(num_sms() / 2), 1, 1);
    cfg.blockDim = dim3(mxfp4::gemm2::kThreads, 1, 1);
    cfg.dynamicSmemBytes = mxfp4::gemm2::kSmemBytes;
    if (cudaOccupancyMaxActiveClusters(&n, mxfp4::gemm2::grouped_gemm_2sm_kernel<false>, &cfg) != cudaSuccess ||
        n <= 0) {
        cudaGetLastError();
        n = num_sms() / 2;
    }
    cached[dev] = n;
    return n;
}

// The one-CTA GEMM serves more than gemm2::kMaxGroups groups, and is also
// chosen for every call when MXFP4_GEMM_CTA_PAIRS=0 is set in the
// environment (for side-by-side measurement).
bool pairs_enabled() {
    static const bool on = [] {
        const char* v = getenv("MXFP4_GEMM_CTA_PAIRS");
        return !(v && v[0] == '0');
    }();
    return on;
}

uint32_t* status_word() {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) return nullptr;
    return static_cast<uint32_t*>(p);
}

// Host-side Philox4x32-10 (SC'11 constants) for the RHT sign word: bit i of
// word 0 of Philox(key = seed, counter = (0, 0, 0, 1)).
// (s_i / 4, s_i / 4) as two binary32 in one 64-bit word, for the packed RHT.
void fill_rht_mul2(uint64_t (&m)[16], uint32_t signs) {
    for (int i = 0; i < 16; ++i) {
        const uint64_t w = 0x3E800000u | (((signs >> i) & 1u) << 31);   // +-0.25
        m[i] = w | (w << 32);
    }
}

uint32_t rht_sign_mask(uint64_t seed) {
    uint32_t c[4] = {0u, 0u, 0u, 1u};
    uint32_t k0 = uint32_t(seed), k1 = uint32_t(seed >> 32);
    for (int round = 0; round < 10; ++round) {
        const uint64_t p0 = uint64_t(0xD2511F53u) * c[0];
        const uint64_t p1 = uint64_t(0xCD9E8D57u) * c[2];
        const uint32_t n0 = uint32_t(p1 >> 32) ^ c[1] ^ k0;
        const uint32_t n2 = uint32_t(p0 >> 32) ^ c[3] ^ k1;
        c[0] = n0;
        c[1] = uint32_t(p1);
        c[2] = n2;
        c[3] = uint32_t(p0);
        k0 += 0x9E3779B9u;
        k1 += 0xBB67AE85u;
    }
    return c[0] & 0xFFFFu;
}

unsigned grid_for(int64_t work, int threads) {
    const int64_t blocks = (work + threads - 1) / threads;
    const int64_t cap = int64_t(num_sms()) * 16;
    return unsigned(blocks < 1 ? 1 : (blocks > cap ? cap : blocks));
}

// --- quantisation launchers --------------------------------------------------
template <typename InT>
mxfp4_status launch_rows(const mxfp4::QuantArgs& qa, bool rht, bool sr, cudaStream_t st) {
    // the kernel indexes the rows of all groups in 32 bits
    if (qa.groups * qa.rows >= (int64_t(1) << 31))
        return fail(MXFP4_ERR_UNSUPPORTED_SHAPE, "mxfp4_quantize: groups * rows must be < 2^31");
    const int64_t work = qa.groups * qa.rows * (qa.cols / 32);
    // Grid: a tensor of at most 16 CTAs of work per resident CTA slot runs as
    // one grid-stride pass of exactly the resident CTAs (no last wave of
    // CTAs to wait for: 4096 x 2880 and 16384 x 2880 ran 8-10% faster); a
    // larger one keeps 16 CTAs per SM, which the block scheduler backfills
    // (65536 x 5760 with SR ran 5% slower as one resident pass).
    auto go = [&](auto kern) -> mxfp4_status {
        const int64_t blocks = (work + 255) / 256;
        const int64_t resident = resident_ctas(kern, 256, 0);
        const int64_t cap = blocks <= 16 * resident ? resident : int64_t(num_sms()) * 16;
        const unsigned grid = unsigned(blocks < 1 ? 1 : (blocks < cap ? blocks : cap));
        kern<<<grid, 256, 0, st>>>(qa);
        return check_launch("mxfp4_quantize(1d)");
    };
    if (rht && sr) return go(mxfp4::quant1d_rows_kernel<InT, true, true>);
    if (rht) return go(mxfp4::quant1d_rows_kernel<InT, true, false>);
    if (sr) return go(mxfp4::quant1d_rows_kernel<InT, false, true>);
    return go(mxfp4::quant1d_rows_kernel<InT, false, false>);
}

bool make_map_plain(CUtensorMap* m, CUtensorMapDataType dt, int rank, const void* base, const uint64_t* dims,
                    const uint64_t* strides_bytes, const uint32_t* box,
                    CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_NONE);

template <typename InT>
mxfp4_status launch_cols(const mxfp4::QuantArgs& qa, bool rht, bool sr, cudaStream_t st) {
    // input [groups][rows = T][cols = F] with row stride ld: box = 128 features x (128 or 64) tokens
    // the kernel indexes rows and features of all groups in 32 bits
    if (qa.groups * qa.rows >= (int64_t(1) << 31) || qa.groups * qa.cols >= (int64_t(1) << 31))
        return fail(MXFP4_ERR_UNSUPPORTED_SHAPE, "mxfp4_quantize: groups * rows and groups * cols must be < 2^31");
    CUtensorMap tm;
    const uint64_t esz = sizeof(InT);
    const uint64_t dims[3] = {uint64_t(qa.cols), uint64_t(qa.rows), uint64_t(qa.groups)};
    const uint64_t strides[2] = {uint64_t(qa.ld) * esz, uint64_t(qa.ld) * esz * uint64_t(qa.rows)};
    const uint32_t box[3] = {uint32_t(mxfp4::kColsTF), uint32_t(mxfp4::cols_tt<InT>()), 1u};
    if (!make_map_plain(&tm, sizeof(InT) == 2 ? CU_TENSOR_MAP_DATA_TYPE_UINT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3,
                        qa.in, dims, strides, box))
        return fail(MXFP4_ERR_CUDA, "mxfp4_quantize(along rows): tensor map encode failed");
    uint32_t* status = status_word();
    if (!status) return fail(MXFP4_ERR_CUDA, "mxfp4_quantize: cannot resolve the device status word");
    const int64_t tt = mxfp4::cols_tt<InT>(), tf = mxfp4::kColsTF;
    const int64_t tiles = qa.groups * ((qa.rows + tt - 1) / tt) * ((qa.cols + tf - 1) / tf);
    const uint32_t smem = mxfp4::cols_smem_bytes<InT>();
    auto go = [&](auto kern) -> mxfp4_status {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
            return fail(MXFP4_ERR_CUDA, "mxfp4_quantize(along rows): shared-memory attribute");
        const int64_t cap = resident_ctas(kern, mxfp4::cols_threads<InT>(), smem);
        const unsigned grid = unsigned(tiles < cap ? tiles : cap);
        kern<<<grid, mxfp4::cols_threads<InT>(), smem, st>>>(tm, qa, status);
        return check_launch("mxfp4_quantize(1d along rows)");
    };
    if (rht && sr) return go(mxfp4::quant1d_cols_kernel<InT, true, true>);
    if (rht) return go(mxfp4::quant1d_cols_kernel<InT, true, false>);
    if (sr) return go(mxfp4::quant1d_cols_kernel<InT, false, true>);
    return go(mxfp4::quant1d_cols_kernel<InT, false, false>);
}

template <typename InT>
mxfp4_status launch_dual(const mxfp4::QuantArgs& qa, bool rht_col, bool rht_row, bool sr, cudaStream_t st) {
    // the kernel indexes rows and features of all groups in 32 bits
    if (qa.groups * qa.rows >= (int64_t(1) << 31) || qa.groups * qa.cols >= (int64_t(1) << 31))
        return fail(MXFP4_ERR_UNSUPPORTED_SHAPE, "mxfp4_quantize: groups * rows and groups * cols must be < 2^31");
    CUtensorMap tm;
    const uint64_t esz = sizeof(InT);
    const uint64_t dims[3] = {uint64_t(qa.cols), uint64_t(qa.rows), uint64_t(qa.groups)};
    const uint64_t strides[2] = {uint64_t(qa.ld) * esz, uint64_t(qa.ld) * esz * uint64_t(qa.rows)};
    const uint32_t box[3] = {uint32_t(mxfp4::kColsTF), uint32_t(mxfp4::cols_tt<InT>()), 1u};
    if (!make_map_plain(&tm, sizeof(InT) == 2 ? CU_TENSOR_MAP_DATA_TYPE_UINT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3,
                        qa.in, dims, strides, box))
        return fail(MXFP4_ERR_CUDA, "mxfp4_quantize_dual: tensor map encode failed");
    uint32_t* status = status_word();
    if (!status) return fail(MXFP4_ERR_CUDA, "mxfp4_quantize_dual: cannot resolve the device status word");
    const int64_t tt = mxfp4::cols_tt<InT>(), tf = mxfp4::kColsTF;
    const int64_t tiles = qa.groups * ((qa.rows + tt - 1) / tt) * ((qa.cols + tf - 1) / tf);
    const uint32_t smem = mxfp4::cols_smem_bytes<InT>();
    auto go = [&](auto kern) -> mxfp4_status {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
            return fail(MXFP4_ERR_CUDA, "mxfp4_quantize_dual: shared-memory attribute");
        const int64_t cap = resident_ctas(kern, mxfp4::cols_threads<InT>(), smem);
        const unsigned grid = unsigned(tiles < cap ? tiles : cap);
        kern<<<grid, mxfp4::cols_threads<InT>(), smem, st>>>(tm, qa, status);
        return check_launch("mxfp4_quantize_dual");
    };
    using namespace mxfp4;
    if (sr) {
        if (rht_col && rht_row) return go(quant1d_cols_kernel<InT, true, true, true, true>);
        if (rht_col) return go(quant1d_cols_kernel<InT, true, true, true, false>);
        if (rht_row) return go(quant1d_cols_kernel<InT, false, true, true, true>);
        return go(quant1d_cols_kernel<InT, false, true, true, false>);
    }
    if (rht_col && rht_row) return go(quant1d_cols_kernel<InT, true, false, true, true>);
    if (rht_col) return go(quant1d_cols_kernel<InT, true, false, true, false>);
    if (rht_row) return go(quant1d_cols_kernel<InT, false, false, true, true>);
    return go(quant1d_cols_kernel<InT, false, false, true, false>);
}

template <typename InT, bool DEOSC>
mxfp4_status launch_2d(const mxfp4::QuantArgs& qa, bool rht, bool sr, cudaStream_t st) {
    const int64_t nblocks = qa.groups * (qa.rows / 32) * (qa.cols / 32);
    constexpr int kThreads2d = mxfp4::kQ2dWarps * 32;   // warps of a CTA take neighbouring blocks of a block row
    const unsigned grid = unsigned((nblocks + mxfp4::kQ2dWarps - 1) / mxfp4::kQ2dWarps);
    // the coalesced kernel: one CTA per tile of kCoalBlkRows x kCoalBlkCols blocks in every group
    const int64_t tiles2 = ((qa.rows / 32 + mxfp4::kCoalBlkRows - 1) / mxfp4::kCoalBlkRows) *
                           ((qa.cols / 32 + mxfp4::kCoalBlkCols - 1) / mxfp4::kCoalBlkCols);
    const unsigned grid_coal = unsigned(qa.groups * tiles2);
    if constexpr (DEOSC) {
        mxfp4::quant2d_coal_kernel<InT, true><<<grid_coal, mxfp4::kCoalWarps * 32, 0, st>>>(qa);
    } else {
        if (rht && sr) mxfp4::quant2d_kernel<InT, true, true, false><<<grid, kThreads2d, 0, st>>>(qa);
        else if (rht) mxfp4::quant2d_kernel<InT, true, false, false><<<grid, kThreads2d, 0, st>>>(qa);
        else if (sr) mxfp4::quant2d_kernel<InT, false, true, false><<<grid, kThreads2d, 0, st>>>(qa);
        else mxfp4::quant2d_coal_kernel<InT, false><<<grid_coal, mxfp4::kCoalWarps * 32, 0, st>>>(qa);
    }
    return check_launch(DEOSC ? "mxfp4_deosc_update" : "mxfp4_quantize(2d)");
}

mxfp4_status check_outputs(const mxfp4_quant_outputs* out, bool two_d) {
    if (!out || !out->codes) return fail(MXFP4_ERR_INVALID_ARG, "outputs: codes pointer is null");
    if (!aligned16(out->codes)) return fail(MXFP4_ERR_MISALIGNED, "outputs: codes not 16-byte aligned");
    if (!two_d && (out->codes_t || out->scales_mma_t))
        return fail(MXFP4_ERR_INVALID_ARG, "outputs: codes_t / scales_mma_t are for 2D blocks only");
    if (out->scales_mma_t && !out->codes_t)
        return fail(MXFP4_ERR_INVALID_ARG, "outputs: scales_mma_t needs codes_t");
    if (out->codes_t && !aligned16(out->codes_t)) return fail(MXFP4_ERR_MISALIGNED, "outputs: codes_t misaligned");
    return ok();
}

// --- tensor maps ---------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

bool make_map(CUtensorMap* m, CUtensorMapDataType dt, int rank, const void* base, const uint64_t* dims,
              const uint64_t* strides_bytes, const uint32_t* box) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    if (rank < 1 || rank > 5) return false;
    cuuint64_t d[5], s[4];
    cuuint32_t b[5], e[5] = {1, 1, 1, 1, 1};
    for (int i = 0; i < rank; ++i) {
        d[i] = dims[i];
        b[i] = box[i];
    }
    for (int i = 0; i + 1 < rank; ++i) s[i] = strides_bytes[i];
    return fn(m, dt, cuuint32_t(rank), const_cast<void*>(base), d, s, b, e, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_map_plain(CUtensorMap* m, CUtensorMapDataType dt, int rank, const void* base, const uint64_t* dims,
                    const uint64_t* strides_bytes, const uint32_t* box, CUtensorMapSwizzle swizzle) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    if (rank < 1 || rank > 5) return false;
    cuuint64_t d[5], s[4];
    cuuint32_t b[5], e[5] = {1, 1, 1, 1, 1};
    for (int i = 0; i < rank; ++i) {
        d[i] = dims[i];
        b[i] = box[i];
    }
    for (int i = 0; i + 1 < rank; ++i) s[i] = strides_bytes[i];
    return fn(m, dt, cuuint32_t(rank), const_cast<void*>(base), d, s, b, e, CU_TENSOR_MAP_INTERLEAVE_NONE,
              swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct FusedOut {
    uint16_t* y;
    int64_t ldy;
    uint8_t* codes;
    uint8_t* scales;
    uint8_t* scales_mma;
    bool sr;
    uint64_t sr_seed;
    uint32_t sr_offset;
};

// Shared by the binary32-output and the fused (bf16 + MXFP4) entry points:
// argument checks, tensor maps, kernel choice and launch.  f != null selects
// the fused epilogue of the CTA-pair kernel (out is then unused).
mxfp4_status grouped_gemm_impl(int op, int num_groups, const int32_t* group_offsets, mxfp4_operand A,
                               mxfp4_operand B, int64_t M, int64_t N, int64_t K, float* out, int64_t ldo,
                               const FusedOut* f, void* stream) {
    using namespace mxfp4::gemm;
    if (op != MXFP4_GEMM_FPROP && op != MXFP4_GEMM_DGRAD && op != MXFP4_GEMM_WGRAD)
        return fail(MXFP4_ERR_INVALID_ARG, "mxfp4_grouped_gemm: bad op %d", op);
    if (num_groups <= 0 || !group_offsets || !A.codes || !A.scales_mma || !B.codes || !B.scales_mma)
        return fail(MXFP4_ERR_INVALID_ARG, "mxfp4_grouped_gemm: null pointer or num_groups <= 0");
    if (M < 0 || N <= 0 || K < 0 || ldo < N) return fail(MXFP4_ERR_INVALID_ARG, "mxfp4_grouped_gemm: bad geometry");
    if (num_groups > kMaxGroups)
        return fail(MXFP4_ERR_UNSUPPORTED_SHAPE, "mxfp4_grouped_gemm: at most %d groups", kMaxGroups);
    if (K % 128 && op == MXFP4_GEMM_WGRAD)
        return fail(MXFP4_ERR_UNSUPPORTED_SHAPE, "mxfp4_grouped_gemm(wgrad): total tokens must be a multiple of 128");
    if (K % 64) return fail(MXFP4_ERR_UNSUPPORTED_SHAPE, "mxfp4_grouped_gemm: K %% 64 != 0");
    if (op != MXFP4_GEMM_WGRAD && M % 128)
        return fail(MXFP4_ERR_UNSUPPORTED_SHAPE, "mxfp4_grouped_gemm: M must be a multiple of 128 (padded groups)");
    if (ldo % 4) return fail(MXFP4_ERR_MISALIGNED, "mxfp4_grouped_gemm: ldo must be a multiple of 4");
    if (!aligned16(A.codes) || !aligned16(B.codes) || !aligned16(A.scales_mma) || !aligned16(B.scales_mma) ||
        (out && !aligned16(out)) || (reinterpret_cast<uintptr_t>(group_offsets) & 3u))
        return fail(MXFP4_ERR_MISALIGNED, "mxfp4_grouped_gemm: pointer not 16-byte aligned");
    if (M == 0) return ok();
    if (K == 0) {
        if (op != MXFP4_GEMM_WGRAD) return ok();
        // every group is empty: dW_g = 0
        const cudaError_t e = cudaMemset2DAsync(out, size_t(ldo) * 4, 0, size_t(N) * 4, size_t(M) * num_groups,
                                                static_cast<cudaStream_t>(stream));
        if (e != cudaSuccess) return fail(MXFP4_ERR_CUDA, "mxfp4_grouped_gemm: %s", cudaGetErrorString(e));
        return ok();
    }
    uint32_t* status = status_word();
    if (!status) return fail(MXFP4_ERR_CUDA, "mxfp4_grouped_gemm: cannot resolve the device status word");

    Args a{};
    a.mode = op == MXFP4_GEMM_WGRAD ? 1 : 0;
    a.num_groups = num_groups;
    a.offsets = group_offsets;
    a.M = M;
    a.N = N;
    a.K = K;
    a.sfa = A.scales_mma;
    a.sfb = B.scales_mma;
    const int64_t S = (K + 31) / 32;
    a.nchunk_a = (S + 3) / 4;
    a.nchunk_b = (S + 3) / 4;
    a.nrb_b = (N + 127) / 128;
    a.sfb_group_bytes = mxfp4::mma_scale_bytes(N, S);
    a.m_tiles = int((M + BM - 1) / BM);
    a.n_tiles = int((N + BN - 1) / BN);
    a.total_tiles = a.mode == 0 ? int64_t(a.m_tiles) * a.n_tiles : int64_t(num_groups) * a.m_tiles * a.n_tiles;
    a.status = status;
    if (f) {
        a.qscales = f->scales;
        a.q_sr = f->sr ? 1 : 0;
        a.q_sr_offset = f->sr_offset;
        a.q_sr_keys = mxfp4::philox_keys(uint32_t(f->sr_seed), uint32_t(f->sr_seed >> 32));
        a.qscales_mma = f->scales_mma;
    }

    const bool pair = pairs_enabled() && num_groups <= mxfp4::gemm2::kMaxGroups;
    const uint32_t b_rows = pair ? uint32_t(mxfp4::gemm2::BNH) : uint32_t(BN);
    CUtensorMap tmA, tmB, tmD, tmQ;
    const uint64_t kb = uint64_t(K / 2);
    {
        const uint64_t dims[2] = {kb, uint64_t(M)};
        const uint64_t str[1] = {kb};
        const uint32_t box[2] = {128, BM};
        if (!make_map(&tmA, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, A.codes, dims, str, box))
            return fail(MXFP4_ERR_CUDA, "mxfp4_grouped_gemm: tensor map for A failed");
    }
    if (a.mode == 0) {
        const uint64_t dims[3] = {kb, uint64_t(N), uint64_t(num_groups)};
        const uint64_t str[2] = {kb, kb * uint64_t(N)};
        const uint32_t box[3] = {128, b_rows, 1};
        if (!make_map(&tmB, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, B.codes, dims, str, box))
            return fail(MXFP4_ERR_CUDA, "mxfp4_grouped_gemm: tensor map for B failed");
        const uint64_t ddims[2] = {uint64_t(N), uint64_t(M)};
        const uint64_t dstr[1] = {uint64_t(ldo) * 4};
        const uint32_t dbox[2] = {32, 32};
        if (f) {
            // bf16 Y in 32 x 32 boxes (64-byte rows, 64-byte swizzle) and
            // its codes in 32-row x 16-byte boxes
            const uint64_t ydims[2] = {uint64_t(N), uint64_t(M)};
            const uint64_t ystr[1] = {uint64_t(f->ldy) * 2};
            const uint32_t ybox[2] = {32, 32};
            if (!make_map_plain(&tmD, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, f->y, ydims, ystr, ybox,
                                CU_TENSOR_MAP_SWIZZLE_64B))
                return fail(MXFP4_ERR_CUDA, "mxfp4_grouped_gemm_fused: tensor map for y failed");
            const uint64_t qdims[2] = {uint64_t(N / 2), uint64_t(M)};
            const uint64_t qstr[1] = {uint64_t(N / 2)};
            const uint32_t qbox[2] = {16, 32};
            if (!make_map_plain(&tmQ, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, f->codes, qdims, qstr, qbox))
                return fail(MXFP4_ERR_CUDA, "mxfp4_grouped_gemm_fused: tensor map for codes failed");
        } else if (!make_map(&tmD, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, out, ddims, dstr, dbox)) {
            return fail(MXFP4_ERR_CUDA, "mxfp4_grouped_gemm: tensor map for D failed");
        }
    } else {
        const uint64_t dims[2] = {kb, uint64_t(N)};
        const uint64_t str[1] = {kb};
        const uint32_t box[2] = {128, b_rows};
        if (!make_map(&tmB, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, B.codes, dims, str, box))
            return fail(MXFP4_ERR_CUDA, "mxfp4_grouped_gemm: tensor map for B failed");
        const uint64_t ddims[3] = {uint64_t(N), uint64_t(M), uint64_t(num_groups)};
        const uint64_t dstr[2] = {uint64_t(ldo) * 4, uint64_t(ldo) * 4 * uint64_t(M)};
        const uint32_t dbox[3] = {32, 32, 1};
        if (!make_map(&tmD, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, out, ddims, dstr, dbox))
            return fail(MXFP4_ERR_CUDA, "mxfp4_grouped_gemm: tensor map for D failed");
    }
    if (pair) {
        namespace g2 = mxfp4::gemm2;
        if (!f) tmQ = tmA;   // unused by the binary32 epilogue
        // two-chunk views: each row of K/2 bytes seen as [chunk][row][256
        // bytes] with a chunk stride of 128 B, so one 128-byte-wide box of two
        // chunks carries both 256-element halves of a K-step, starting at byte
        // offset 0 or 64 of its first chunk (wgrad's expert ranges start on
        // 128-token boundaries).  Only chunk positions whose 256 bytes lie
        // inside the row are in the view.
        CUtensorMap tmA2 = tmA, tmB2 = tmB;
        const uint64_t nch = kb >= 256 ? (kb - 256) / 128 + 1 : 0;
        a.k_chunks = int32_t(nch >= 2 ? nch : 0);
        if (a.k_chunks > 0) {
            const uint64_t dimsA[3] = {256, uint64_t(M), nch};
            const uint64_t strA[2] = {kb, 128};
            const uint32_t boxA[3] = {128, BM, 2};
            if (!make_map(&tmA2, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, A.codes, dimsA, strA, boxA))
                return fail(MXFP4_ERR_CUDA, "mxfp4_grouped_gemm: tensor map for A (whole chunks) failed");
            if (a.mode == 0) {
                const uint64_t dimsB[4] = {256, uint64_t(N), nch, uint64_t(num_groups)};
                const uint64_t strB[3] = {kb, 128, kb * uint64_t(N)};
                const uint32_t boxB[4] = {128, b_rows, 2, 1};
                if (!make_map(&tmB2, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, B.codes, dimsB, strB, boxB))
                    return fail(MXFP4_ERR_CUDA, "mxfp4_grouped_gemm: tensor map for B (whole chunks) failed");
            } else {
                const uint64_t dimsB[3] = {256, uint64_t(N), nch};
                const uint64_t strB[2] = {kb, 128};
                const uint32_t boxB[3] = {128, b_rows, 2};
                if (!make_map(&tmB2, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, B.codes, dimsB, strB, boxB))
                    return fail(MXFP4_ERR_CUDA, "mxfp4_grouped_gemm: tensor map for B (whole chunks) failed");
            }
        }
        // binary32 output seen as [column block][row][32 floats] (column-block
        // stride 128 B), so one 32 x 32 x 2 box stores two chunks
        CUtensorMap tmD2 = tmD;
        a.d_pairs = 0;
        if (!f && N % 32 == 0 && kEpiPairStores) {
            bool okm;
            if (a.mode == 0) {
                const uint64_t dd[3] = {32, uint64_t(M), uint64_t(N / 32)};
                const uint64_t ds[2] = {uint64_t(ldo) * 4, 128};
                const uint32_t db[3] = {32, 32, 2};
                okm = make_map(&tmD2, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, out, dd, ds, db);
            } else {
                const uint64_t dd[4] = {32, uint64_t(M), uint64_t(N / 32), uint64_t(num_groups)};
                const uint64_t ds[3] = {uint64_t(ldo) * 4, 128, uint64_t(ldo) * 4 * uint64_t(M)};
                const uint32_t db[4] = {32, 32, 2, 1};
                okm = make_map(&tmD2, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, out, dd, ds, db);
            }
            if (!okm) return fail(MXFP4_ERR_CUDA, "mxfp4_grouped_gemm: tensor map for D (chunk pairs) failed");
            a.d_pairs = 1;
        }
        void (*kern)(const CUtensorMap, const CUtensorMap, const CUtensorMap, const CUtensorMap, const CUtensorMap,
                     const CUtensorMap, const CUtensorMap, const Args) =
            f ? g2::grouped_gemm_2sm_kernel<true> : g2::grouped_gemm_2sm_kernel<false>;
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, g2::kSmemBytes) != cudaSuccess)
            return fail(MXFP4_ERR_CUDA, "mxfp4_grouped_gemm: cannot raise the shared-memory limit");
        // upper bound on the units (group, m-tile pair, n-tile): the exact
        // count depends on the device-side offsets
        const int64_t units = a.mode == 0 ? (int64_t(a.m_tiles) / 2 + num_groups) * a.n_tiles
                                          : int64_t(num_groups) * ((a.m_tiles + 1) / 2) * a.n_tiles;
        if (units == 0) return ok();
        const int64_t clusters = pair_clusters();
        const unsigned grid = 2u * unsigned(units < clusters ? units : clusters);
        kern<<<grid, g2::kThreads, g2::kSmemBytes, static_cast<cudaStream_t>(stream)>>>(tmA, tmB, tmD, tmQ, tmA2, tmB2,
                                                                                       tmD2, a);
        return check_launch("mxfp4_grouped_gemm");
    }
    if (f) return fail(MXFP4_ERR_UNSUPPORTED_SHAPE, "mxfp4_grouped_gemm_fused: needs the CTA-pair kernel");
    if (cudaFuncSetAttribute(grouped_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) !=
        cudaSuccess)
        return fail(MXFP4_ERR_CUDA, "mxfp4_grouped_gemm: cannot raise the shared-memory limit");
    if (a.total_tiles == 0) return ok();
    const int64_t sms = num_sms();
    const unsigned grid = unsigned(a.total_tiles < sms ? a.total_tiles : sms);
    grouped_gemm_kernel<<<grid, kThreads, kSmemBytes, static_cast<cudaStream_t>(stream)>>>(tmA, tmB, tmD, a);
    return check_launch("mxfp4_grouped_gemm");
}

}  // namespace

extern "C" {

size_t mxfp4_mma_scale_bytes(int64_t rows, int64_t nscales) {
    if (rows <= 0 || nscales <= 0) return 0;
    return size_t(mxfp4::mma_scale_bytes(rows, nscales));
}

const char* mxfp4_version(void) { return "mxfp4-b200 0.1 (sm_100a)"; }

size_t mxfp4_last_error(char* buf, size_t len) {
    const size_t n = g_last_error.size();
    if (buf && len) {
        const size_t c = n < len - 1 ? n : len - 1;
        memcpy(buf, g_last_error.data(), c);
        buf[c] = 0;
    }
    return n;
}

mxfp4_status mxfp4_check_device_status(void* stream) {
    static std::atomic<uint32_t> next_slot{0};
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const uint32_t slot = next_slot.fetch_add(1u) % kStatusSlots;
    uint32_t v = 0;
    status_take_kernel<<<1, 1, 0, st>>>(slot);
    cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess)
        e = cudaMemcpyFromSymbolAsync(&v, g_status_taken, sizeof(v), sizeof(uint32_t) * slot, cudaMemcpyDeviceToHost,
                                      st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return fail(MXFP4_ERR_CUDA, "check_device_status: %s", cudaGetErrorString(e));
    if (v == 0) return ok();
    if (v & mxfp4::kStatusTimeout)
        return fail(MXFP4_ERR_DEVICE_TIMEOUT, "device wait timed out (status 0x%08x: roles %s%s%s%s%s)", v,
                    (v & mxfp4::kRoleProducer) ? "producer " : "", (v & mxfp4::kRoleMma) ? "mma " : "",
                    (v & mxfp4::kRoleEpilogue) ? "epilogue " : "", (v & mxfp4::kRoleScales) ? "scales " : "",
                    (v & mxfp4::kRoleTeardown) ? "teardown" : "");
    return fail(MXFP4_ERR_DEVICE_BAD_INPUT, "device rejected group offsets (status 0x%08x)", v);
}

mxfp4_status mxfp4_quantize(const void* in, int in_dtype, int64_t groups, int64_t rows, int64_t cols, int64_t ld,
                            const mxfp4_quant_params* p, const mxfp4_quant_outputs* out, void* stream) {
    if (!p) return fail(MXFP4_ERR_INVALID_ARG, "mxfp4_quantize: null params");
    if (in_dtype != MXFP4_DTYPE_BF16 && in_dtype != MXFP4_DTYPE_F32)
        return fail(MXFP4_ERR_INVALID_ARG, "mxfp4_quantize: bad in_dtype %d", in_dtype);
    if (groups < 0 || rows < 0 || cols < 0 || ld < cols)
        return fail(MXFP4_ERR_INVALID_ARG, "mxfp4_quantize: bad geometry groups=%lld rows=%lld cols=%lld ld=%lld",
                    (long long)groups, (long long)rows, (long long)cols, (long long)ld);
    const bool empty = groups == 0 || rows == 0 || cols == 0;
    if (!in && !empty) return fail(MXFP4_ERR_INVALID_ARG, "mxfp4_quantize: null input");
    if (p->block != MXFP4_BLOCK_1X32 && p->block != MXFP4_BLOCK_32X32)
        return fail(MXFP4_ERR_INVALID_ARG, "mxfp4_quantize: bad block %d", p->block);
    if (p->rht_d != 0 && p->rht_d != 16) return fail(MXFP4_ERR_INVALID_ARG, "mxfp4_quantize: rht_d must be 0 or 16");
    if (p->rounding != MXFP4_ROUND_NEAREST && p->rounding != MXFP4_ROUND_STOCHASTIC)
        return fail(MXFP4_ERR_INVALID_ARG, "mxfp4_quantize: bad rounding %d", p->rounding);
    const bool two_d = p->block == MXFP4_BLOCK_32X32;
    if (empty) return ok();  // nothing to read or write; output pointers may be null
    mxfp4_status s = check_outputs(out, two_d);
    if (s != MXFP4_OK) return s;
    const bool along_rows = !two_d && p->along_rows;
    if (two_d) {
        if (rows % 32 || cols % 32)
            return fail(MXFP4_ERR_UNSUPPORTED_SHAPE, "mxfp4_quantize(2d): rows and cols must be multiples of 32");
    } else if (along_rows) {
        if (rows % 32) return fail(MXFP4_ERR_UNSUPPORTED_SHAPE, "mxfp4_quantize(along rows): rows %% 32 != 0");
    } else if (cols % 32) {
        return fail(MXFP4_ERR_UNSUPPORTED_SHAPE, "mxfp4_quantize: cols %% 32 != 0");
    }
    const int esz = in_dtype == MXFP4_DTYPE_BF16 ? 2 : 4;
    if (!aligned16(in) || (ld * esz) % 16) return fail(MXFP4_ERR_MISALIGNED, "mxfp4_quantize: input rows not 16-byte aligned");
    mxfp4::QuantArgs qa{};
    qa.in = in;
    qa.groups = groups;
    qa.rows = rows;
    qa.cols = cols;
    qa.ld = ld;
    qa.rht_signs = p->rht_d == 16 ? rht_sign_mask(p->rht_seed) : 0u;
    fill_rht_mul2(qa.rht_mul2, qa.rht_signs);
    qa.sr_key0 = uint32_t(p->sr_seed);
    qa.sr_keys = mxfp4::philox_keys(uint32_t(p->sr_seed), uint32_t(p->sr_seed >> 32));
    qa.sr_key1 = uint32_t(p->sr_seed >> 32);
    qa.sr_offset = p->sr_offset;
    qa.codes = out->codes;
    qa.scales = out->scales;
    qa.scales_mma = out->scales_mma;
    qa.codes_t = out->codes_t;
    qa.scales_mma_t = out->scales_mma_t;
    const bool rht = p->rht_d == 16, sr = p->rounding == MXFP4_ROUND_STOCHASTIC;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (two_d)
        return in_dtype == MXFP4_DTYPE_BF16 ? launch_2d<uint16_t, false>(qa, rht, sr, st)
                                            : launch_2d<float, false>(qa, rht, sr, st);
    if (along_rows)
        return in_dtype == MXFP4_DTYPE_BF16 ? launch_cols<uint16_t>(qa, rht, sr, st) : launch_cols<float>(qa, rht, sr, st);
    return in_dtype == MXFP4_DTYPE_BF16 ? launch_rows<uint16_t>(qa, rht, sr, st) : launch_rows<float>(qa, rht, sr, st);
}

mxfp4_status mxfp4_quantize_dual(const void* in, int in_dtype, int64_t groups, int64_t rows, int64_t cols, int64_t ld,
                                 const mxfp4_quant_params* rp, const mxfp4_quant_params* cp,
                                 const mxfp4_quant_outputs* row_out, const mxfp4_quant_outputs* col_out, void* stream) {
    if (!rp || !cp) return fail(MXFP4_ERR_INVALID_ARG, "mxfp4_quantize_dual: null params");
    if (in_dtype != MXFP4_DTYPE_BF16 && in_dtype != MXFP4_DTYPE_F32)
        return fail(MXFP4_ERR_INVALID_ARG, "mxfp4_quantize_dual: bad in_dtype %d", in_dtype);
    if (groups < 0 || rows < 0 || cols < 0 || ld < cols)
        return fail(MXFP4_ERR_INVALID_ARG, "mxfp4_quantize_dual: bad geometry");
    if (rp->block != MXFP4_BLOCK_1X32 || cp->block != MXFP4_BLOCK_1X32)
        return fail(MXFP4_ERR_INVALID_ARG, "mxfp4_quantize_dual: both directions use 1x32 blocks");
    if (rp->along_rows != 0 || cp->along_rows != 1)
        return fail(MXFP4_ERR_INVALID_ARG, "mxfp4_quantize_dual: row_params.along_rows must be 0, col_params 1");
    if ((rp->rht_d != 0 && rp->rht_d != 16) || (cp->rht_d != 0 && cp->rht_d != 16))
        return fail(MXFP4_ERR_INVALID_ARG, "mxfp4_quantize_dual: rht_d must be 0 or 16");
    if ((rp->rounding != MXFP4_ROUND_NEAREST && rp->rounding != MXFP4_ROUND_STOCHASTIC) ||
        rp->rounding != cp->rounding)
        return fail(MXFP4_ERR_INVALID_ARG, "mxfp4_quantize_dual: both directions need the same valid rounding");
    const bool sr = rp->rounding == MXFP4_ROUND_STOCHASTIC;
    if (sr && rp->sr_seed != cp->sr_seed)
        return fail(MXFP4_ERR_INVALID_ARG, "mxfp4_quantize_dual: both directions need the same sr_seed");
    const bool empty = groups == 0 || rows == 0 || cols == 0;
    if (!in && !empty) return fail(MXFP4_ERR_INVALID_ARG, "mxfp4_quantize_dual: null input");
    if (empty) return ok();
    mxfp4_status s = check_outputs(row_out, false);
    if (s != MXFP4_OK) return s;
    s = check_outputs(col_out, false);
    if (s != MXFP4_OK) return s;
    if (rows % 32 || cols % 32)
        return fail(MXFP4_ERR_UNSUPPORTED_SHAPE, "mxfp4_quantize_dual: rows and cols must be multiples of 32");
    const int esz = in_dtype == MXFP4_DTYPE_BF16 ? 2 : 4;
    if (!aligned16(in) || (ld * esz) % 16)
        return fail(MXFP4_ERR_MISALIGNED, "mxfp4_quantize_dual: input rows not 16-byte aligned");
    mxfp4::QuantArgs qa{};
    qa.in = in;
    qa.groups = groups;
    qa.rows = rows;
    qa.cols = cols;
    qa.ld = ld;
    qa.rht_signs = cp->rht_d == 16 ? rht_sign_mask(cp->rht_seed) : 0u;
    fill_rht_mul2(qa.rht_mul2, qa.rht_signs);
    qa.sr_key0 = uint32_t(cp->sr_seed);
    qa.sr_keys = mxfp4::philox_keys(uint32_t(cp->sr_seed), uint32_t(cp->sr_seed >> 32));
    qa.sr_key1 = uint32_t(cp->sr_seed >> 32);
    qa.sr_offset = cp->sr_offset;
    qa.codes = col_out->codes;
    qa.scales = col_out->scales;
    qa.scales_mma = col_out->scales_mma;
    qa.r_codes = row_out->codes;
    qa.r_scales = row_out->scales;
    qa.r_scales_mma = row_out->scales_mma;
    qa.r_rht_signs = rp->rht_d == 16 ? rht_sign_mask(rp->rht_seed) : 0u;
    fill_rht_mul2(qa.r_rht_mul2, qa.r_rht_signs);
    qa.r_sr_offset = rp->sr_offset;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    return in_dtype == MXFP4_DTYPE_BF16 ? launch_dual<uint16_t>(qa, cp->rht_d == 16, rp->rht_d == 16, sr, st)
                                        : launch_dual<float>(qa, cp->rht_d == 16, rp->rht_d == 16, sr, st);
}

mxfp4_status mxfp4_rht(const void* in, int in_dtype, int64_t rows, int64_t cols, int64_t ld, int axis, int d,
                       uint64_t seed, void* out, int out_dtype, void* stream) {
    if (!in || !out) return fail(MXFP4_ERR_INVALID_ARG, "mxfp4_rht: null pointer");
    if (axis != 0 && axis != 1) return fail(MXFP4_ERR_INVALID_ARG, "mxfp4_rht: axis must be 0 or 1");
    if (d != 16) return fail(MXFP4_ERR_INVALID_ARG, "mxfp4_rht: only d = 16 is supported");
    if ((in_dtype != MXFP4_DTYPE_BF16 && in_dtype != MXFP4_DTYPE_F32) ||
        (out_dtype != MXFP4_DTYPE_BF16 && out_dtype != MXFP4_DTYPE_F32))
        return fail(MXFP4_ERR_INVALID_ARG, "mxfp4_rht: bad dtype");
    if (rows < 0 || cols < 0 || ld < cols) return fail(MXFP4_ERR_INVALID_ARG, "mxfp4_rht: bad geometry");
    if (axis == 1 && cols % 16) return fail(MXFP4_ERR_UNSUPPORTED_SHAPE, "mxfp4_rht: cols %% 16 != 0");
    if (axis == 0 && rows % 16) return fail(MXFP4_ERR_UNSUPPORTED_SHAPE, "mxfp4_rht(axis 0): rows %% 16 != 0");
    const int esz = in_dtype == MXFP4_DTYPE_BF16 ? 2 : 4;
    if (!aligned16(in) || !aligned16(out) || (ld * esz) % 16)
        return fail(MXFP4_ERR_MISALIGNED, "mxfp4_rht: pointers/rows not 16-byte aligned");
    if (rows == 0 || cols == 0) return ok();
    const uint32_t signs = rht_sign_mask(seed);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (axis == 0) {
        const unsigned grid = grid_for((rows / 16) * cols, 256);
        if (in_dtype == MXFP4_DTYPE_BF16) {
            if (out_dtype == MXFP4_DTYPE_BF16)
                mxfp4::rht_dim0_kernel<uint16_t, true><<<grid, 256, 0, st>>>(static_cast<const uint16_t*>(in), rows, cols, ld, signs, out);
            else
                mxfp4::rht_dim0_kernel<uint16_t, false><<<grid, 256, 0, st>>>(static_cast<const uint16_t*>(in), rows, cols, ld, signs, out);
        } else {
            if (out_dtype == MXFP4_DTYPE_BF16)
                mxfp4::rht_dim0_kernel<float, true><<<grid, 256, 0, st>>>(static_cast<const float*>(in), rows, cols, ld, signs, out);
            else
                mxfp4::rht_dim0_kernel<float, false><<<grid, 256, 0, st>>>(static_cast<const float*>(in), rows, cols, ld, signs, out);
        }
        return check_launch("mxfp4_rht(axis 0)");
    }
    const unsigned grid = grid_for(rows * (cols / 16), 256);
    if (in_dtype == MXFP4_DTYPE_BF16) {
        if (out_dtype == MXFP4_DTYPE_BF16)
            mxfp4::rht_kernel<uint16_t, true><<<grid, 256, 0, st>>>(static_cast<const uint16_t*>(in), rows, cols, ld, signs, out);
        else
            mxfp4::rht_kernel<uint16_t, false><<<grid, 256, 0, st>>>(static_cast<const uint16_t*>(in), rows, cols, ld, signs, out);
    } else {
        if (out_dtype == MXFP4_DTYPE_BF16)
            mxfp4::rht_kernel<float, true><<<grid, 256, 0, st>>>(static_cast<const float*>(in), rows, cols, ld, signs, out);
        else
            mxfp4::rht_kernel<float, false><<<grid, 256, 0, st>>>(static_cast<const float*>(in), rows, cols, ld, signs, out);
    }
    return check_launch("mxfp4_rht");
}

mxfp4_status mxfp4_deosc_update(const float* master, int64_t groups, int64_t rows, int64_t cols, uint32_t step,
                                const mxfp4_deosc_params* dp, uint8_t* state, const mxfp4_quant_outputs* out,
                                void* stream) {
    if (!master || !state || !dp) return fail(MXFP4_ERR_INVALID_ARG, "mxfp4_deosc_update: null pointer");
    if (dp->flip_threshold < 1 || dp->flip_threshold > 7)
        return fail(MXFP4_ERR_INVALID_ARG, "mxfp4_deosc_update: flip_threshold must be in 1..7");
    if (dp->freeze_lower > 1) return fail(MXFP4_ERR_INVALID_ARG, "mxfp4_deosc_update: freeze_lower must be 0 or 1");
    if (groups < 0 || rows < 0 || cols < 0) return fail(MXFP4_ERR_INVALID_ARG, "mxfp4_deosc_update: bad geometry");
    mxfp4_status s = check_outputs(out, true);
    if (s != MXFP4_OK) return s;
    if (rows % 32 || cols % 32) return fail(MXFP4_ERR_UNSUPPORTED_SHAPE, "mxfp4_deosc_update: rows, cols must be multiples of 32");
    if (!aligned16(master) || !aligned16(state))
        return fail(MXFP4_ERR_MISALIGNED, "mxfp4_deosc_update: master/state not 16-byte aligned");
    if (groups == 0 || rows == 0 || cols == 0) return ok();
    mxfp4::QuantArgs qa{};
    qa.in = master;
    qa.groups = groups;
    qa.rows = rows;
    qa.cols = cols;
    qa.ld = cols;
    qa.codes = out->codes;
    qa.scales = out->scales;
    qa.scales_mma = out->scales_mma;
    qa.codes_t = out->codes_t;
    qa.scales_mma_t = out->scales_mma_t;
    qa.state = state;
    qa.step = step;
    qa.flip_threshold = dp->flip_threshold;
    qa.reset_period = dp->reset_period;
    qa.freeze_lower = dp->freeze_lower;
    return launch_2d<float, true>(qa, false, false, static_cast<cudaStream_t>(stream));
}

mxfp4_status mxfp4_grouped_gemm(int op, int num_groups, const int32_t* group_offsets, mxfp4_operand A,
                                mxfp4_operand B, int64_t M, int64_t N, int64_t K, float* out, int64_t ldo,
                                void* stream) {
    if (!out) return fail(MXFP4_ERR_INVALID_ARG, "mxfp4_grouped_gemm: null pointer or num_groups <= 0");
    return grouped_gemm_impl(op, num_groups, group_offsets, A, B, M, N, K, out, ldo, nullptr, stream);
}

mxfp4_status mxfp4_grouped_gemm_fused(int op, int num_groups, const int32_t* group_offsets, mxfp4_operand A,
                                      mxfp4_operand B, int64_t M, int64_t N, int64_t K, uint16_t* y, int64_t ldy,
                                      const mxfp4_quant_outputs* q, const mxfp4_quant_params* qp, void* stream) {
    if (op != MXFP4_GEMM_FPROP && op != MXFP4_GEMM_DGRAD)
        return fail(MXFP4_ERR_INVALID_ARG, "mxfp4_grouped_gemm_fused: op must be FPROP or DGRAD");
    if (!y || !q || !q->codes)
        return fail(MXFP4_ERR_INVALID_ARG, "mxfp4_grouped_gemm_fused: null output pointer");
    if (q->codes_t || q->scales_mma_t)
        return fail(MXFP4_ERR_INVALID_ARG, "mxfp4_grouped_gemm_fused: codes_t / scales_mma_t are for 2D blocks only");
    if (qp && (qp->block != MXFP4_BLOCK_1X32 || qp->along_rows != 0 || qp->rht_d != 0 ||
               (qp->rounding != MXFP4_ROUND_NEAREST && qp->rounding != MXFP4_ROUND_STOCHASTIC)))
        return fail(MXFP4_ERR_INVALID_ARG,
                    "mxfp4_grouped_gemm_fused: params must be 1x32 along the last dim, no RHT, RN or SR");
    if (N % 32 || K <= 0) return fail(MXFP4_ERR_UNSUPPORTED_SHAPE, "mxfp4_grouped_gemm_fused: N %% 32 != 0 or K <= 0");
    if (ldy < N) return fail(MXFP4_ERR_INVALID_ARG, "mxfp4_grouped_gemm_fused: ldy < N");
    if (ldy % 8) return fail(MXFP4_ERR_MISALIGNED, "mxfp4_grouped_gemm_fused: ldy must be a multiple of 8");
    if (!aligned16(y) || !aligned16(q->codes))
        return fail(MXFP4_ERR_MISALIGNED, "mxfp4_grouped_gemm_fused: output pointer not 16-byte aligned");
    if (num_groups > mxfp4::gemm2::kMaxGroups || !pairs_enabled())
        return fail(MXFP4_ERR_UNSUPPORTED_SHAPE, "mxfp4_grouped_gemm_fused: at most %d groups, CTA pairs enabled",
                    mxfp4::gemm2::kMaxGroups);
    const bool sr = qp && qp->rounding == MXFP4_ROUND_STOCHASTIC;
    FusedOut f{y, ldy, q->codes, q->scales, q->scales_mma, sr, sr ? qp->sr_seed : 0u, sr ? qp->sr_offset : 0u};
    return grouped_gemm_impl(op, num_groups, group_offsets, A, B, M, N, K, nullptr, N, &f, stream);
}

mxfp4_status mxfp4_mma_peak_probe(int64_t mmas_per_pair, double* flops, void* stream) {
    if (mmas_per_pair < 1 || mmas_per_pair > (int64_t(1) << 22) || !flops)
        return fail(MXFP4_ERR_INVALID_ARG, "mxfp4_mma_peak_probe: mmas_per_pair must lie in [1, 2^22], flops non-null");
    uint32_t* status = status_word();
    if (!status) return fail(MXFP4_ERR_CUDA, "mxfp4_mma_peak_probe: no device status word");
    if (cudaFuncSetAttribute(mxfp4::peak::mma_peak_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             mxfp4::peak::kSmemBytes) != cudaSuccess)
        return fail(MXFP4_ERR_CUDA, "mxfp4_mma_peak_probe: cannot raise the shared-memory limit");
    const int64_t clusters = pair_clusters();
    mxfp4::peak::mma_peak_kernel<<<unsigned(2 * clusters), mxfp4::peak::kThreads, mxfp4::peak::kSmemBytes,
                                   static_cast<cudaStream_t>(stream)>>>(mmas_per_pair, status);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess)
        return fail(MXFP4_ERR_CUDA, "mxfp4_mma_peak_probe: launch failed: %s", cudaGetErrorString(e));
    *flops = double(clusters) * double(mmas_per_pair) * 2.0 * 256.0 * 192.0 * 64.0;
    return ok();
}

mxfp4_status mxfp4_selftest_wait_timeout(void* stream) {
    uint32_t* status = status_word();
    if (!status) return fail(MXFP4_ERR_CUDA, "mxfp4_selftest_wait_timeout: no device status word");
    mxfp4::selftest::wait_timeout_kernel<<<1, 64, 0, static_cast<cudaStream_t>(stream)>>>(status);
    return check_launch("mxfp4_selftest_wait_timeout");
}

}  // extern "C"

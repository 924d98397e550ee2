// Host-side check of the shared-memory staging index arithmetic of two
// kernels, against the addresses their direct stores would use:
//  - the token-dim quantiser (quant1d_cols_kernel): the staging offset of
//    (feature row fl, token block c) is a bijection onto the 16-byte chunks of
//    a tile's buffer, and the chunk the cooperative store reads for (fl, c)
//    is the one its writer (feature 2 pr + h, block blk) left there, written
//    to that writer's output row and token bytes;
//  - the 2D / de-oscillation kernel (quant2d_coal_kernel): thread t of the
//    W^T write-out reads slot t, which the lane of the matching block row and
//    column filled, and writes it to the W^T row and byte column the lane's
//    own direct store used.
// Built with nvcc as a host program; no GPU is used.
#include <cstdio>
#include <vector>

#include "quantize.cuh"

using namespace mxfp4;

template <typename InT>
static long check_cols(int& bad) {
    constexpr int kTT = cols_tt<InT>(), kCh = kTT / 32, kPairs = kColsTF / 2;
    constexpr int kStage = int(cols_stage_bytes<InT>());
    constexpr int kThreads = cols_threads<InT>();
    long n = 0;
    // writer of each chunk: (pr, blk, h) -> offset
    std::vector<int> owner(kStage / 16, -1);
    for (int t = 0; t < kThreads; ++t) {
        const int pr = t % kPairs, blk = t / kPairs;
        for (int h = 0; h < 2; ++h) {
            const int fl = 2 * pr + h;
            const int off = cols_stage_off<InT>(fl, blk);
            if (off % 16 || off < 0 || off + 16 > kStage || owner[off / 16] != -1) { ++bad; continue; }
            owner[off / 16] = fl * kCh + blk;   // the writer's (row, block)
            ++n;
        }
    }
    for (int o : owner) bad += o < 0;
    // the cooperative store: thread t, iteration it
    for (int it = 0; it < kColsTF * kCh / kThreads; ++it)
        for (int t = 0; t < kThreads; ++t) {
            const int idx = it * kThreads + t;
            const int fl = idx / kCh, c = idx % kCh;
            const int off = cols_stage_off<InT>(fl, c);
            // read chunk written by (row fl, block c); its direct store went to
            // row f0 + fl, bytes t0/2 + 16c -- the cooperative store's target
            bad += owner[off / 16] != fl * kCh + c;
            ++n;
        }
    return n;
}

static long check_coal(int& bad) {
    constexpr int kThreads = kCoalWarps * 32;
    long n = 0;
    std::vector<int> filled(kThreads, -1);
    for (int warp = 0; warp < kCoalWarps; ++warp)
        for (int lane = 0; lane < 32; ++lane) {
            const int bil = warp / kCoalBlkCols, bjl = warp % kCoalBlkCols;
            const int slot = coal_wt_slot(bjl, lane, bil);
            if (slot < 0 || slot >= kThreads || filled[slot] != -1) { ++bad; continue; }
            filled[slot] = (bil * kCoalBlkCols + bjl) * 32 + lane;
        }
    for (int tj = 0; tj < 3; ++tj)
        for (int ti = 0; ti < 3; ++ti)
            for (int t = 0; t < kThreads; ++t) {
                // the write-out of thread t (as in the kernel)
                const int p = t % kCoalBlkRows, pr = t / kCoalBlkRows;
                const int wb = pr >> 5, l = pr & 31;
                const int64_t bis = int64_t(ti) * kCoalBlkRows + p, bjs = int64_t(tj) * kCoalBlkCols + wb;
                const int64_t row = coal_wt_row(bjs, l), byte = bis * 16;
                // the lane that filled slot t and its direct store
                const int w = filled[t] / 32, lane = filled[t] % 32;
                const int64_t bi = int64_t(ti) * kCoalBlkRows + w / kCoalBlkCols;
                const int64_t bj = int64_t(tj) * kCoalBlkCols + w % kCoalBlkCols;
                const int q = lane >> 3, c = lane & 7;
                const int64_t row_direct = bj * 32 + 4 * c + q, byte_direct = bi * 16;
                bad += row != row_direct || byte != byte_direct;
                ++n;
            }
    return n;
}

int main() {
    int bad = 0;
    long n = check_cols<uint16_t>(bad) + check_cols<float>(bad) + check_coal(bad);
    if (bad) {
        printf("FAIL %d of %ld\n", bad, n);
        return 1;
    }
    printf("ok %ld\n", n);
    return 0;
}

// Host-side check of the pair GEMM's unit walk (UnitWalk in gemm2sm.cuh):
// for random expert layouts (empty experts included), cluster counts and
// tile counts, the units a cluster visits with the walk equal the direct
// decomposition of u = cluster, cluster + step, ... into (group, m-tile pair,
// n-tile).  Built with nvcc as a host program; no GPU is used.
#include <cstdio>
#include <cstdlib>
#include <vector>

#include "gemm2sm.cuh"

using namespace mxfp4;
using namespace mxfp4::gemm2;

// Direct decomposition: mode 0 counts ((tiles + 1) / 2) * n_tiles units per
// group and walks the groups; mode 1 has the same count for every group.
static Unit direct(const Args& a, const std::vector<int32_t>& off, int64_t u) {
    int g = 0;
    int64_t local = u;
    for (;; ++g) {
        const int64_t pairs = a.mode == 0 ? ((off[g + 1] - off[g]) / 128 + 1) / 2 : (a.m_tiles + 1) / 2;
        if (local < pairs * a.n_tiles) break;
        local -= pairs * a.n_tiles;
    }
    const int64_t p = local / a.n_tiles, n = local % a.n_tiles;
    Unit un;
    un.g = g;
    un.n0 = n * 192;
    if (a.mode == 0) {
        un.ma = off[g] / 128 + 2 * p;
        un.mb = un.ma + 1;
        un.vb = un.mb * 128 < off[g + 1];
        un.kbeg = 0;
        un.kend = a.K;
    } else {
        un.ma = 2 * p;
        un.mb = 2 * p + 1;
        un.vb = un.mb < a.m_tiles;
        un.kbeg = off[g];
        un.kend = off[g + 1];
    }
    return un;
}

int main() {
    srand(7);
    long checked = 0;
    for (int trial = 0; trial < 2000; ++trial) {
        Args a{};
        a.mode = trial & 1;
        a.num_groups = 1 + rand() % 40;
        std::vector<int32_t> off(a.num_groups + 1, 0);
        for (int g = 0; g < a.num_groups; ++g) off[g + 1] = off[g] + 128 * (rand() % 5 == 0 ? 0 : rand() % 12);
        a.n_tiles = 1 + rand() % 31;
        a.m_tiles = 1 + rand() % 45;
        a.K = 2880;
        int64_t total = 0;
        for (int g = 0; g < a.num_groups; ++g) total += int64_t(UnitWalk::pairs_in(a, off.data(), g)) * a.n_tiles;
        const int step = 1 + rand() % 80;
        for (int c = 0; c < step; ++c) {
            UnitWalk w;
            w.init(a, off.data(), c, step);
            for (int64_t u = c; u < total; u += step, w.advance(a, off.data())) {
                const Unit x = w.unit(a, off.data()), y = direct(a, off, u);
                if (x.g != y.g || x.ma != y.ma || x.mb != y.mb || x.vb != y.vb || x.n0 != y.n0 || x.kbeg != y.kbeg ||
                    x.kend != y.kend) {
                    printf("mismatch: trial %d mode %d unit %lld\n", trial, a.mode, (long long)u);
                    return 1;
                }
                ++checked;
            }
        }
    }
    printf("ok %ld\n", checked);
    return 0;
}

// Independent reference for the oracle's Philox4x32-10: calls the host path
// of curand's header-only Philox (curand_Philox4x32_10).  Reads lines
// "c0 c1 c2 c3 k0 k1" (hex) on stdin, prints the four output words (hex).
#define QUALIFIERS static inline __host__ __device__
#include <cstdio>
#include <vector_types.h>
#include <curand_philox4x32_x.h>

int main() {
    unsigned c0, c1, c2, c3, k0, k1;
    while (std::scanf("%x %x %x %x %x %x", &c0, &c1, &c2, &c3, &k0, &k1) == 6) {
        uint4 c = make_uint4(c0, c1, c2, c3);
        uint2 k = make_uint2(k0, k1);
        uint4 r = curand_Philox4x32_10(c, k);
        std::printf("%08x %08x %08x %08x\n", r.x, r.y, r.z, r.w);
    }
    return 0;
}

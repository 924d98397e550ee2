// Independent reference for the oracle's round-to-nearest E2M1 conversion:
// calls the host path of cuda_fp4.h (__nv_cvt_float_to_fp4, E2M1,
// round-to-nearest).  Reads float32 bit patterns (hex) on stdin, prints the
// 4-bit code (hex) per line.
#include <cstdio>
#include <cstring>
#include <cuda_fp4.h>

int main() {
    unsigned bits;
    while (std::scanf("%x", &bits) == 1) {
        float f;
        std::memcpy(&f, &bits, 4);
        __nv_fp4_storage_t q = __nv_cvt_float_to_fp4(f, __NV_E2M1, cudaRoundNearest);
        std::printf("%x\n", (unsigned)q & 0xF);
    }
    return 0;
}

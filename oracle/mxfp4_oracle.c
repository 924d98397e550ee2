/*
 * mxfp4_oracle.c -- plain, slow, scalar CPU oracle for the MXFP4
 * quantise-and-contract path of the ALTO training recipe.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test-suite, the smoke check and the
 * CPU-baseline leg of the benchmark may load this library.  It shares no
 * code, header, table or constant generator with the CUDA library.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math -fopenmp
 * (no FMA contraction, no flush-to-zero; every float operation below is a
 * single IEEE-754 binary32 operation rounded to nearest-even).
 *
 * Sources (all pages are about "Training an MoE LLM in MXFP4: How We Closed
 * the Gap to BF16", the ALTO recipe):
 *  - MX format, E2M1 elements with one UE8M0 scale per block:
 *    roboaidigest, "What ALTO Actually Does" (also the OCP MX spec named in
 *    the article's introduction).
 *  - hybrid 1D/2D block quantisation, randomized Hadamard transform,
 *    stochastic rounding, simplified weight de-oscillation: the abstract
 *    (foxai.news / scholarbro / paperdot) and roboaidigest "What ALTO
 *    Actually Does".
 *  - why de-oscillation exists (master weight vs quantised value, bin
 *    flipping near a boundary): roboaidigest "What ALTO Actually Does".
 * The pages fix no bit-level detail; the readings used here are listed in
 * the repository design notes and repeated at each function:
 *  block size 32, scale rule E = floor(log2(amax)) - 2 clamped to the UE8M0
 *  range, saturation to +-6, Hadamard size 16 with Philox signs, SR with 16
 *  Philox bits per element added to the position kept to 16 bits (the rule
 *  and bit layout of the sm_100 stochastic-rounding conversion),
 *  de-oscillation = per-weight flip counter with a frozen-code mask.
 *
 * Parity status: quantise/RHT/Philox/SR/GEMM are pinned by CPU tests against
 * library routines, closed forms and brute force.  The de-oscillation rule is
 * a reading of its own (the pages give only its motivation): parity
 * unpinned by the pages; pinned only by hand-worked traces.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* Philox4x32-10 counter-based generator.                                    */
/* Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as easy as 1, 2, 3" */
/* (SC'11): 10 rounds of the Philox-4x32 S-box; the two 32-bit multipliers   */
/* and the two Weyl key increments are the published ones.                   */
/* ------------------------------------------------------------------------ */
static const uint32_t PHILOX_MUL_A = 0xD2511F53u;
static const uint32_t PHILOX_MUL_B = 0xCD9E8D57u;
static const uint32_t PHILOX_WEYL_A = 0x9E3779B9u;
static const uint32_t PHILOX_WEYL_B = 0xBB67AE85u;

void oracle_philox4x32_10(const uint32_t ctr_in[4], const uint32_t key_in[2], uint32_t out[4])
{
    uint32_t c[4] = {ctr_in[0], ctr_in[1], ctr_in[2], ctr_in[3]};
    uint32_t k0 = key_in[0], k1 = key_in[1];
    for (int round = 0; round < 10; ++round) {
        if (round > 0) { /* key schedule: bump between rounds */
            k0 += PHILOX_WEYL_A;
            k1 += PHILOX_WEYL_B;
        }
        uint64_t p0 = (uint64_t)PHILOX_MUL_A * (uint64_t)c[0];
        uint64_t p1 = (uint64_t)PHILOX_MUL_B * (uint64_t)c[2];
        uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
        uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
        uint32_t n0 = hi1 ^ c[1] ^ k0;
        uint32_t n1 = lo1;
        uint32_t n2 = hi0 ^ c[3] ^ k1;
        uint32_t n3 = lo0;
        c[0] = n0; c[1] = n1; c[2] = n2; c[3] = n3;
    }
    out[0] = c[0]; out[1] = c[1]; out[2] = c[2]; out[3] = c[3];
}

/* Stream layout (reading): key = (seed mod 2^32, seed >> 32);
 * counter = (group lo, group hi, offset, tag); tag 0 = stochastic rounding,
 * tag 1 = Hadamard signs. */
enum { TAG_SR = 0, TAG_RHT = 1 };

/* Bit reversal of a 16-bit value. */
static uint32_t reverse16(uint32_t u)
{
    uint32_t r = 0;
    for (int b = 0; b < 16; ++b)
        if (u & (1u << b)) r |= 1u << (15 - b);
    return r;
}

/* 16 random bits for output element n of an SR stream (reading): one Philox
 * call serves 16 consecutive elements, word q = (n >> 2) & 3 serves the four
 * elements 4m..4m+3 (m = n >> 2), and with bytes b0..b3 of that word (b0 the
 * least significant):
 *   element 4m + 0 : b2 * 256 + b0          element 4m + 2 : b3 * 256 + b1
 *   element 4m + 1 : reverse16(b2*256 + b0) element 4m + 3 : reverse16(b3*256 + b1)
 * This is the way the sm_100 four-element stochastic-rounding conversion
 * consumes one 32-bit random word, so the device path can hand it the Philox
 * word unchanged. */
uint32_t oracle_sr_bits16(uint64_t seed, uint32_t offset, uint64_t n)
{
    uint64_t g = n >> 4;
    unsigned q = (unsigned)((n >> 2) & 3u), j = (unsigned)(n & 3u);
    uint32_t ctr[4] = {(uint32_t)g, (uint32_t)(g >> 32), offset, TAG_SR};
    uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
    uint32_t w[4];
    oracle_philox4x32_10(ctr, key, w);
    uint32_t b0 = w[q] & 0xFFu, b1 = (w[q] >> 8) & 0xFFu, b2 = (w[q] >> 16) & 0xFFu, b3 = w[q] >> 24;
    uint32_t even = (b2 << 8) | b0, odd = (b3 << 8) | b1;
    switch (j) {
    case 0: return even;
    case 1: return reverse16(even);
    case 2: return odd;
    default: return reverse16(odd);
    }
}

/* Random Hadamard signs (reading): s_i = -1 iff bit i of word 0 of
 * Philox(key = rht_seed, counter = (0, 0, 0, tag 1)), i = 0..d-1, d <= 32. */
void oracle_rht_signs(uint64_t seed, int d, float* s)
{
    uint32_t ctr[4] = {0u, 0u, 0u, TAG_RHT};
    uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
    uint32_t w[4];
    oracle_philox4x32_10(ctr, key, w);
    for (int i = 0; i < d; ++i) s[i] = ((w[0] >> i) & 1u) ? -1.0f : 1.0f;
}

/* ------------------------------------------------------------------------ */
/* E2M1 element format (MX spec, as named on roboaidigest "What ALTO        */
/* Actually Does"): sign bit, 2 exponent bits, 1 mantissa bit.  Code c has  */
/* magnitude GRID[c & 7] and is negative iff bit 3 is set.                  */
/* ------------------------------------------------------------------------ */
static const double E2M1_GRID[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

double oracle_e2m1_value(int code)
{
    double m = E2M1_GRID[code & 7];
    return (code & 8) ? -m : m;
}

/* Block scale exponent (reading of the MX rule): E = floor(log2(amax)) - 2,
 * where 2 is the exponent of the largest E2M1 magnitude (6 = 1.5 * 2^2),
 * clamped to the UE8M0 range [-127, 127].  amax == 0 gives -127 (the
 * smallest scale; every element then encodes as zero).  frexp gives
 * amax = m * 2^x with m in [0.5, 1), exact for subnormals, so
 * floor(log2(amax)) = x - 1. */
int oracle_scale_exponent(float amax)
{
    if (amax == 0.0f) return -127;
    int x;
    (void)frexpf(amax, &x);
    int e = (x - 1) - 2;
    if (e < -127) e = -127;
    if (e > 127) e = 127;
    return e;
}

/* Scale an element into the block's E2M1 range: v = y * 2^-E, one binary32
 * rounding (exact unless the product is subnormal). */
static float scale_down(float y, int E)
{
    return ldexpf(y, -E);
}

/* Round-to-nearest onto the E2M1 grid: saturate |v| to 6, take the nearest
 * grid magnitude, ties to the even code; the sign is kept (so a negative
 * value that rounds to zero gives code 8, "-0"). */
int oracle_e2m1_rn(float v)
{
    int neg = signbit(v) ? 1 : 0;
    double a = fabs((double)v);
    if (a > 6.0) a = 6.0;
    int best = 0;
    double bestd = fabs(a - E2M1_GRID[0]);
    for (int i = 1; i < 8; ++i) {
        double d = fabs(a - E2M1_GRID[i]);
        if (d < bestd || (d == bestd && (i % 2) == 0)) {
            best = i;
            bestd = d;
        }
    }
    return (neg << 3) | best;
}

/* Stochastic rounding onto the E2M1 grid (reading): |v| >= 6 gives 6;
 * otherwise lo <= |v| < hi are adjacent grid magnitudes, f = (|v| - lo) /
 * (hi - lo), F = floor(f * 2^16) (the position kept to 16 bits), and the
 * magnitude rounds up iff F + r16 >= 2^16 (a carry out of 16 bits when the
 * random draw is added to the kept position).  r16 is a uniform 16-bit draw,
 * so P(up) = F / 2^16, within 2^-16 of f.  The sign is kept (-0 included). */
int oracle_e2m1_sr(float v, uint32_t r16)
{
    int neg = signbit(v) ? 1 : 0;
    double a = fabs((double)v);
    int mag;
    if (a >= 6.0) {
        mag = 7;
    } else {
        int i = 0;
        while (!(E2M1_GRID[i] <= a && a < E2M1_GRID[i + 1])) ++i;
        double f = (a - E2M1_GRID[i]) / (E2M1_GRID[i + 1] - E2M1_GRID[i]);   /* exact in binary64 */
        uint32_t F = (uint32_t)floor(f * 65536.0);                         /* exact: scaling by 2^16 */
        mag = (F + (r16 & 0xFFFFu) >= 65536u) ? i + 1 : i;
    }
    return (neg << 3) | mag;
}

/* ------------------------------------------------------------------------ */
/* Randomized Hadamard transform on one 16-element chunk (reading of the    */
/* RHT the abstract names, with d = 16):                                     */
/*   t = (s .* x) * 1/4            (exact)                                   */
/*   y = t * F1 * F2 * F4 * F8     each factor applied in binary32           */
/* where F_h = I_{16/2h} (x) H2 (x) I_h with H2 = [[1,1],[1,-1]].  Each      */
/* output of a factor has exactly two non-zero terms, so it is the single    */
/* rounded value a+b or a-b; the product of the four factors is the          */
/* Sylvester Hadamard matrix H16 (natural order) and H16/4 is orthogonal.    */
/* ------------------------------------------------------------------------ */
static void build_factor(int h, int F[16][16])
{
    for (int i = 0; i < 16; ++i)
        for (int j = 0; j < 16; ++j) {
            int same_outer = (i / (2 * h)) == (j / (2 * h));
            int same_inner = (i % h) == (j % h);
            int p = (i / h) % 2, q = (j / h) % 2;
            int h2 = (p == 1 && q == 1) ? -1 : 1;
            F[i][j] = (same_outer && same_inner) ? h2 : 0;
        }
}

static void apply_factor(const float* t, int h, float* out)
{
    int F[16][16];
    build_factor(h, F);
    for (int j = 0; j < 16; ++j) {
        /* sum over the non-zero entries of column j in increasing row order;
         * no accumulator starts from +0, so signed zeros survive */
        int have = 0;
        float acc = 0.0f;
        for (int i = 0; i < 16; ++i) {
            if (F[i][j] == 0) continue;
            float term = (F[i][j] > 0) ? t[i] : -t[i];
            if (!have) { acc = term; have = 1; }
            else acc = acc + term;
        }
        out[j] = acc;
    }
}

void oracle_rht16(const float* x, const float* s, float* y)
{
    float a[16], b[16];
    for (int i = 0; i < 16; ++i) a[i] = (s[i] * x[i]) * 0.25f;
    apply_factor(a, 1, b);
    apply_factor(b, 2, a);
    apply_factor(a, 4, b);
    apply_factor(b, 8, a);
    for (int i = 0; i < 16; ++i) y[i] = a[i];
}

/* Mathematical check: y = (s .* x) * H16 / 4 in binary64 with the dense
 * Sylvester matrix H16[i][j] = (-1)^popcount(i & j). */
void oracle_rht16_dense_f64(const double* x, const double* s, double* y)
{
    for (int j = 0; j < 16; ++j) {
        double acc = 0.0;
        for (int i = 0; i < 16; ++i) {
            int par = __builtin_popcount((unsigned)(i & j)) & 1;
            acc += s[i] * x[i] * (par ? -1.0 : 1.0);
        }
        y[j] = acc / 4.0;
    }
}

/* ------------------------------------------------------------------------ */
/* Input widening.  dtype 0 = bfloat16 (uint16 bit patterns), 1 = float32.  */
/* ------------------------------------------------------------------------ */
static float load_elem(const void* in, int dtype, int64_t idx)
{
    if (dtype == 0) {
        uint32_t bits = (uint32_t)((const uint16_t*)in)[idx] << 16;
        float f;
        memcpy(&f, &bits, 4);
        return f;
    }
    return ((const float*)in)[idx];
}

/* RHT of a whole row of `cols` elements, chunk by chunk. */
static void rht_row(const float* row, int64_t cols, const float* s, float* out)
{
    for (int64_t c0 = 0; c0 < cols; c0 += 16) oracle_rht16(row + c0, s, out + c0);
}

/* Standalone RHT (along the last dim), output binary32 [rows, cols]. */
void oracle_rht_rows(const void* in, int dtype, int64_t rows, int64_t cols, int64_t ld,
                     uint64_t seed, float* out)
{
    float s[16];
    oracle_rht_signs(seed, 16, s);
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        float* x = (float*)malloc(sizeof(float) * (size_t)cols);
        for (int64_t c = 0; c < cols; ++c) x[c] = load_elem(in, dtype, r * ld + c);
        rht_row(x, cols, s, out + r * cols);
        free(x);
    }
}

/* ------------------------------------------------------------------------ */
/* 1D quantisation: 1x32 blocks along the last dim (hybrid 1D/2D blocks of  */
/* the abstract; 1D for activations and gradients).                         */
/*   rows x cols input (row stride ld), cols % 32 == 0.                      */
/*   codes : rows x cols/2 bytes, element c in nibble (c & 1) of byte c/2    */
/*           (low nibble = even column).                                     */
/*   scales: rows x cols/32 bytes, E + 127.                                  */
/*   rht_d : 0 (off) or 16.  sr: 0 = nearest, 1 = stochastic.                */
/*   row0  : global index of the first row, so that a slice of rows draws    */
/*           the same SR bits as the whole tensor (n = (row0+r)*cols + c).   */
/* ------------------------------------------------------------------------ */
void oracle_quantize_1d(const void* in, int dtype, int64_t rows, int64_t cols, int64_t ld,
                        int rht_d, uint64_t rht_seed, int sr, uint64_t sr_seed, uint32_t sr_offset,
                        int64_t row0, uint8_t* codes, uint8_t* scales)
{
    float s[16];
    if (rht_d == 16) oracle_rht_signs(rht_seed, 16, s);
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        float* y = (float*)malloc(sizeof(float) * (size_t)cols);
        for (int64_t c = 0; c < cols; ++c) y[c] = load_elem(in, dtype, r * ld + c);
        if (rht_d == 16) {
            float* t = (float*)malloc(sizeof(float) * (size_t)cols);
            rht_row(y, cols, s, t);
            memcpy(y, t, sizeof(float) * (size_t)cols);
            free(t);
        }
        for (int64_t b = 0; b < cols / 32; ++b) {
            float amax = 0.0f;
            for (int k = 0; k < 32; ++k) {
                float a = fabsf(y[b * 32 + k]);
                if (a > amax) amax = a;
            }
            int E = oracle_scale_exponent(amax);
            scales[r * (cols / 32) + b] = (uint8_t)(E + 127);
            for (int k = 0; k < 32; ++k) {
                int64_t c = b * 32 + k;
                float v = scale_down(y[c], E);
                int code;
                if (sr) {
                    uint64_t n = (uint64_t)(row0 + r) * (uint64_t)cols + (uint64_t)c;
                    code = oracle_e2m1_sr(v, oracle_sr_bits16(sr_seed, sr_offset, n));
                } else {
                    code = oracle_e2m1_rn(v);
                }
                uint8_t* byte = &codes[r * (cols / 2) + c / 2];
                if ((c & 1) == 0) *byte = (uint8_t)((*byte & 0xF0) | code);
                else *byte = (uint8_t)((*byte & 0x0F) | (code << 4));
            }
        }
        free(y);
    }
}

/* 1D quantisation along dim 0 (the token dim of the weight-gradient
 * operands): the rows x cols input is transposed first, then quantised as a
 * cols x rows matrix with blocks along its last dim.  The output (codes,
 * scales, SR element index) is in that transposed layout; col0 plays the
 * role of row0. */
void oracle_quantize_1d_transposed(const void* in, int dtype, int64_t rows, int64_t cols, int64_t ld,
                                   int rht_d, uint64_t rht_seed, int sr, uint64_t sr_seed,
                                   uint32_t sr_offset, int64_t col0, uint8_t* codes, uint8_t* scales)
{
    float* t = (float*)malloc(sizeof(float) * (size_t)rows * (size_t)cols);
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < cols; ++c) t[c * rows + r] = load_elem(in, dtype, r * ld + c);
    oracle_quantize_1d(t, 1, cols, rows, rows, rht_d, rht_seed, sr, sr_seed, sr_offset, col0, codes, scales);
    free(t);
}

/* ------------------------------------------------------------------------ */
/* 2D quantisation: 32x32 blocks aligned at (0,0) (weights; W and W^T then  */
/* share codes and scales).  Optional RHT-16 along the last dim first.       */
/*   codes : rows x cols/2 (same packing as 1D); scales: rows/32 x cols/32.  */
/* ------------------------------------------------------------------------ */
void oracle_quantize_2d(const void* in, int dtype, int64_t rows, int64_t cols, int64_t ld,
                        int rht_d, uint64_t rht_seed, int sr, uint64_t sr_seed, uint32_t sr_offset,
                        uint8_t* codes, uint8_t* scales)
{
    float s[16];
    if (rht_d == 16) oracle_rht_signs(rht_seed, 16, s);
    float* y = (float*)malloc(sizeof(float) * (size_t)rows * (size_t)cols);
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t c = 0; c < cols; ++c) y[r * cols + c] = load_elem(in, dtype, r * ld + c);
        if (rht_d == 16) {
            float* t = (float*)malloc(sizeof(float) * (size_t)cols);
            rht_row(y + r * cols, cols, s, t);
            memcpy(y + r * cols, t, sizeof(float) * (size_t)cols);
            free(t);
        }
    }
    int64_t nbr = rows / 32, nbc = cols / 32;
#pragma omp parallel for schedule(static)
    for (int64_t bi = 0; bi < nbr; ++bi) {
        for (int64_t bj = 0; bj < nbc; ++bj) {
            float amax = 0.0f;
            for (int i = 0; i < 32; ++i)
                for (int j = 0; j < 32; ++j) {
                    float a = fabsf(y[(bi * 32 + i) * cols + bj * 32 + j]);
                    if (a > amax) amax = a;
                }
            int E = oracle_scale_exponent(amax);
            scales[bi * nbc + bj] = (uint8_t)(E + 127);
            for (int i = 0; i < 32; ++i)
                for (int j = 0; j < 32; ++j) {
                    int64_t r = bi * 32 + i, c = bj * 32 + j;
                    float v = scale_down(y[r * cols + c], E);
                    int code;
                    if (sr) {
                        uint64_t n = (uint64_t)r * (uint64_t)cols + (uint64_t)c;
                        code = oracle_e2m1_sr(v, oracle_sr_bits16(sr_seed, sr_offset, n));
                    } else {
                        code = oracle_e2m1_rn(v);
                    }
                    uint8_t* byte = &codes[r * (cols / 2) + c / 2];
                    if ((c & 1) == 0) *byte = (uint8_t)((*byte & 0xF0) | code);
                    else *byte = (uint8_t)((*byte & 0x0F) | (code << 4));
                }
        }
    }
    free(y);
}

/* ------------------------------------------------------------------------ */
/* Weight de-oscillation (reading; the pages give the motivation on         */
/* roboaidigest "What ALTO Actually Does"; the abstract says only that the  */
/* scheme is a simplified one derived from TetraJet-v2, not the rule).       */
/* Per weight, one state byte: bits 0-3 previous code, bits 4-6 flip count  */
/* (saturating at 7), bit 7 frozen.                                          */
/*  step == 0 : initialise state = (RN code, count 0, not frozen).           */
/*  step  > 0 : if reset_period > 0 and step % reset_period == 0, clear      */
/*              count and frozen first.  q = RN code under the block scale   */
/*              recomputed from the current master weights.  Frozen: emit    */
/*              the stored code, state unchanged.  Otherwise: if q differs   */
/*              from the stored code, count = min(count+1, 7), store q, and  */
/*              freeze once count >= flip_threshold; emit q.                 */
/*  freeze_lower (variant): at the flip that freezes a weight, store and     */
/*              emit the lower-magnitude of the two codes of that flip (the  */
/*              stored one and q; magnitude = code & 7, ties keep q).        */
/* Scales are always those of the current master weights (2D, 32x32).        */
/* master: groups x rows x cols binary32; state/codes per weight;            */
/* scales: groups x rows/32 x cols/32.                                       */
/* ------------------------------------------------------------------------ */
void oracle_deosc_update(const float* master, int64_t groups, int64_t rows, int64_t cols, uint32_t step,
                         uint32_t flip_threshold, uint32_t reset_period, uint32_t freeze_lower, uint8_t* state,
                         uint8_t* codes, uint8_t* scales)
{
    int64_t per = rows * cols;
    int64_t nbr = rows / 32, nbc = cols / 32;
#pragma omp parallel for schedule(static) collapse(2)
    for (int64_t g = 0; g < groups; ++g) {
        for (int64_t bi = 0; bi < nbr; ++bi) {
            const float* W = master + g * per;
            for (int64_t bj = 0; bj < nbc; ++bj) {
                float amax = 0.0f;
                for (int i = 0; i < 32; ++i)
                    for (int j = 0; j < 32; ++j) {
                        float a = fabsf(W[(bi * 32 + i) * cols + bj * 32 + j]);
                        if (a > amax) amax = a;
                    }
                int E = oracle_scale_exponent(amax);
                scales[g * nbr * nbc + bi * nbc + bj] = (uint8_t)(E + 127);
                for (int i = 0; i < 32; ++i)
                    for (int j = 0; j < 32; ++j) {
                        int64_t r = bi * 32 + i, c = bj * 32 + j;
                        int64_t idx = g * per + r * cols + c;
                        int q = oracle_e2m1_rn(scale_down(W[r * cols + c], E));
                        int out;
                        uint8_t st = state[idx];
                        if (step == 0) {
                            st = (uint8_t)q;
                            out = q;
                        } else {
                            int prev = st & 0x0F;
                            int count = (st >> 4) & 0x7;
                            int frozen = (st >> 7) & 1;
                            if (reset_period > 0 && (step % reset_period) == 0) {
                                count = 0;
                                frozen = 0;
                            }
                            if (frozen) {
                                out = prev;
                            } else {
                                out = q;
                                if (q != prev) {
                                    count = count < 7 ? count + 1 : 7;
                                    int keep = q;
                                    if ((uint32_t)count >= flip_threshold) {
                                        frozen = 1;
                                        /* variant: freeze to the lower-magnitude code of
                                         * this flip (ties keep the new code) */
                                        if (freeze_lower && (prev & 7) < (q & 7)) keep = prev;
                                        out = keep;
                                    }
                                    prev = keep;
                                }
                            }
                            st = (uint8_t)(prev | (count << 4) | (frozen << 7));
                        }
                        state[idx] = st;
                        uint8_t* byte = &codes[g * (per / 2) + r * (cols / 2) + c / 2];
                        if ((c & 1) == 0) *byte = (uint8_t)((*byte & 0xF0) | out);
                        else *byte = (uint8_t)((*byte & 0x0F) | (out << 4));
                    }
            }
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Dequantisation (binary64): value = grid(code) * 2^(scale - 127).         */
/* ------------------------------------------------------------------------ */
void oracle_dequant_1d(const uint8_t* codes, const uint8_t* scales, int64_t rows, int64_t cols, double* out)
{
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < cols; ++c) {
            uint8_t byte = codes[r * (cols / 2) + c / 2];
            int code = (c & 1) ? (byte >> 4) : (byte & 0x0F);
            int E = (int)scales[r * (cols / 32) + c / 32] - 127;
            out[r * cols + c] = ldexp(oracle_e2m1_value(code), E);
        }
}

void oracle_dequant_2d(const uint8_t* codes, const uint8_t* scales, int64_t rows, int64_t cols, double* out)
{
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < cols; ++c) {
            uint8_t byte = codes[r * (cols / 2) + c / 2];
            int code = (c & 1) ? (byte >> 4) : (byte & 0x0F);
            int E = (int)scales[(r / 32) * (cols / 32) + c / 32] - 127;
            out[r * cols + c] = ldexp(oracle_e2m1_value(code), E);
        }
}

/* Plain triple-loop binary64 GEMM: C[M,N] = A[M,K] * B[N,K]^T. */
void oracle_gemm_f64(const double* A, const double* B, int64_t M, int64_t N, int64_t K, double* C)
{
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k) acc += A[m * K + k] * B[n * K + k];
            C[m * N + n] = acc;
        }
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}

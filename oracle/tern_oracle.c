/*
 * tern_oracle.c -- fp64 CPU oracle for the ternary-g128 weight-only matmul.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It shares no source,
 * header, table or helper with the CUDA library, and the CUDA library never
 * calls it.
 *
 * What it computes, and where the definition comes from:
 *
 *   - The number format.  Every weight is a ternary code t in {-1, 0, +1};
 *     every 128 consecutive weights share one FP16 scale s_g, and the real
 *     weight is w_i = s_g * t_i.  ("Bonsai 27B ternary / 1-bit quantization",
 *     ThakiCloud blog, section "How compression works" (압축은 어떻게
 *     작동하는가); "Ternary-Bonsai-27B" model summary, aitrends.kr, section
 *     "Technical features" (기술적 특징); "Ternary quantization: 27B in 7 GB",
 *     devnsb blog, section "What ternary quantization is".)
 *   - The group runs along K, the reduction axis, inside one output row
 *     (plainest reading: the scale is "applied in the matrix multiply").
 *   - The 2-bit slot layout is this library's own contract (the pages say only
 *     that ternary values are stored in 2-bit slots, devnsb blog section
 *     "Limits" (한계)): code c = t + 1 in {0,1,2}, 3 is invalid; weight (n,k)
 *     sits in byte n*K/4 + k/4 at bits 2*(k%4) and 2*(k%4)+1 (least
 *     significant pair first); scales are a separate fp16 array [N][K/128].
 *   - The matmul is y[m][n] = sum_k x[m][k] * w[n][k]   (y = x * W^T),
 *     evaluated here naively in fp64, k in increasing order.
 *
 * Everything is written out plainly: no blocking, no reordering, no vector
 * code.  fp16 values are decoded from the IEEE-754 binary16 definition.
 *
 * ORC_MUTANT (compile-time, tests only) plants one deliberate mistake so the
 * tests can show that the pins catch it.  The default build has none.
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#ifndef ORC_MUTANT
#define ORC_MUTANT 0
#endif

#define ORC_GROUP 128

/* IEEE-754 binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits.
 * exponent 0: subnormal, value = fraction * 2^-24;
 * exponent 31: infinity (fraction 0) or NaN;
 * otherwise value = (1024 + fraction) * 2^(exponent - 25). */
double orc_half_to_double(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int expo = (h >> 10) & 31;
    int frac = h & 1023;
    double v;
    if (expo == 0) {
#if ORC_MUTANT == 6
        v = ldexp(1024.0 + (double)frac, -25); /* planted: subnormals decoded as normals */
#else
        v = ldexp((double)frac, -24);
#endif
    } else if (expo == 31) {
        v = frac ? NAN : INFINITY;
    } else {
        v = ldexp(1024.0 + (double)frac, expo - 25);
    }
    return sign ? -v : v;
}

/* Bytes of the two packed buffers (the "2-bit slot" storage plus one fp16
 * scale per 128 weights).  Together: K*N/4 + 2*K*N/128 = 2.125 bits/weight. */
int64_t orc_slots_bytes(int64_t N, int64_t K) { return N * (K / 4); }
int64_t orc_scales_bytes(int64_t N, int64_t K) { return N * (K / ORC_GROUP) * 2; }

/* Bit position of weight k inside its byte. */
static int orc_shift(int64_t k)
{
#if ORC_MUTANT == 1
    return 6 - 2 * (int)(k % 4); /* planted: most significant pair first */
#else
    return 2 * (int)(k % 4);
#endif
}

/* code c for ternary value t; 3 for anything outside {-1,0,+1} */
static int orc_code_of(int t)
{
    if (t < -1 || t > 1) return 3;
#if ORC_MUTANT == 2
    return 1 - t; /* planted: sign of the code mapping flipped */
#else
    return t + 1;
#endif
}

/* ternary value for code c (c == 3 has none; the caller handles it) */
static int orc_value_of(int c)
{
#if ORC_MUTANT == 2
    return 1 - c;
#else
    return c - 1;
#endif
}

/* Pack codes [N][K] (int8 t) and scales [N][K/128] (fp16 bits) into the slot
 * layout.  An input outside {-1,0,+1} is stored as code 3 and counted.
 * Returns the number of invalid codes (or -1 if K is not a multiple of 128);
 * *first_bad receives the flat index of the first one (or -1). */
int64_t orc_pack_g128(const int8_t *codes, const uint16_t *scales_in, int64_t N, int64_t K,
                      uint8_t *slots, uint16_t *scales_out, int64_t *first_bad)
{
    int64_t bad = 0, first = -1;
    if (K <= 0 || N <= 0 || K % ORC_GROUP != 0) return -1;
    for (int64_t i = 0; i < N * (K / 4); i++) slots[i] = 0;
    for (int64_t n = 0; n < N; n++) {
        for (int64_t k = 0; k < K; k++) {
            int t = codes[n * K + k];
            int c = orc_code_of(t);
            if (c == 3) {
                if (first < 0) first = n * K + k;
                bad++;
            }
            slots[n * (K / 4) + k / 4] |= (uint8_t)(c << orc_shift(k));
        }
    }
    for (int64_t i = 0; i < N * (K / ORC_GROUP); i++) scales_out[i] = scales_in[i];
    if (first_bad) *first_bad = first;
    return bad;
}

/* Slot value of weight (n,k). */
static int orc_slot(const uint8_t *slots, int64_t K, int64_t n, int64_t k)
{
    return (slots[n * (K / 4) + k / 4] >> orc_shift(k)) & 3;
}

/* Unpack slots [N][K/4] into codes [N][K] (int8 t).  Slot value 3 is written
 * as the sentinel 2 and counted.  Returns the count (or -1 for a bad K). */
int64_t orc_unpack_g128(const uint8_t *slots, int64_t N, int64_t K, int8_t *codes_out)
{
    int64_t bad = 0;
    if (K <= 0 || N <= 0 || K % ORC_GROUP != 0) return -1;
    for (int64_t n = 0; n < N; n++) {
        for (int64_t k = 0; k < K; k++) {
            int c = orc_slot(slots, K, n, k);
            if (c == 3) {
                codes_out[n * K + k] = 2;
                bad++;
            } else {
                codes_out[n * K + k] = (int8_t)orc_value_of(c);
            }
        }
    }
    return bad;
}

/* Group index of weight k: one scale per 128 consecutive weights along K. */
static int64_t orc_group_of(int64_t k)
{
#if ORC_MUTANT == 3
    return k / 64; /* planted: wrong group size */
#else
    return k / ORC_GROUP;
#endif
}

/* Dequantised weight w[n][k] = s[n][k/128] * t[n][k] in fp64 (exact).
 * An invalid slot (3) yields NaN. */
double orc_weight(const uint8_t *slots, const uint16_t *scales, int64_t K, int64_t n, int64_t k)
{
    int64_t G = K / ORC_GROUP;
    int64_t g = orc_group_of(k);
    int c = orc_slot(slots, K, n, k);
    if (c == 3) return NAN;
    if (g >= G) g = G - 1; /* only reachable by mutant 3; keeps it in bounds */
    return orc_half_to_double(scales[n * G + g]) * (double)orc_value_of(c);
}

/* W dequantised to fp64 [N][K]. */
void orc_dequant(const uint8_t *slots, const uint16_t *scales, int64_t N, int64_t K, double *w)
{
    for (int64_t n = 0; n < N; n++)
        for (int64_t k = 0; k < K; k++) w[n * K + k] = orc_weight(slots, scales, K, n, k);
}

/* One output element: y = sum_k x[m][k] * w[n][k], bound = sum_k |x[m][k] * w[n][k]|. */
static void orc_dot(const uint16_t *x, int64_t M, int64_t K, const uint8_t *slots,
                    const uint16_t *scales, int64_t m, int64_t n, double *y, double *bound)
{
    double acc = 0.0, b = 0.0;
#if ORC_MUTANT == 5
    int64_t kend = K - 1; /* planted: last term dropped */
#else
    int64_t kend = K;
#endif
    for (int64_t k = 0; k < kend; k++) {
#if ORC_MUTANT == 4
        int64_t xi = k * M + m; /* planted: x read as if stored [K][M] */
#else
        int64_t xi = m * K + k;
#endif
        double p = orc_half_to_double(x[xi]) * orc_weight(slots, scales, K, n, k);
        acc += p;
        b += fabs(p);
    }
    *y = acc;
    *bound = b;
}

/* Full product y[M][N] = x[M][K] * W^T, plus the per-element bound
 * sum_k |x*w| that the acceptance tolerance is stated against.
 * nthreads > 1 spreads independent output elements over OpenMP threads
 * (each element is still one sequential sum).  Returns the thread count used. */
int orc_matmul(const uint16_t *x, int64_t M, int64_t K, const uint8_t *slots,
               const uint16_t *scales, int64_t N, double *y, double *bound, int nthreads)
{
    int used = 1;
#ifdef _OPENMP
    if (nthreads < 1) nthreads = 1;
#pragma omp parallel for num_threads(nthreads) schedule(static)
    for (int64_t i = 0; i < M * N; i++) {
        if (i == 0) used = omp_get_num_threads();
        orc_dot(x, M, K, slots, scales, i / N, i % N, &y[i], &bound[i]);
    }
#else
    (void)nthreads;
    for (int64_t i = 0; i < M * N; i++) orc_dot(x, M, K, slots, scales, i / N, i % N, &y[i], &bound[i]);
#endif
    return used;
}

/* Selected output elements (m_idx[i], n_idx[i]) only: for spot checks of
 * shapes too large to evaluate in full.  Returns the thread count used. */
int orc_matmul_at(const uint16_t *x, int64_t M, int64_t K, const uint8_t *slots,
                  const uint16_t *scales, int64_t N, const int64_t *m_idx, const int64_t *n_idx,
                  int64_t count, double *y, double *bound, int nthreads)
{
    int used = 1;
    (void)N;
#ifdef _OPENMP
    if (nthreads < 1) nthreads = 1;
#pragma omp parallel for num_threads(nthreads) schedule(dynamic, 16)
    for (int64_t i = 0; i < count; i++) {
        if (i == 0) used = omp_get_num_threads();
        orc_dot(x, M, K, slots, scales, m_idx[i], n_idx[i], &y[i], &bound[i]);
    }
#else
    (void)nthreads;
    for (int64_t i = 0; i < count; i++)
        orc_dot(x, M, K, slots, scales, m_idx[i], n_idx[i], &y[i], &bound[i]);
#endif
    return used;
}

/* Row-sampled product for K-row slices of one matrix whose rows are passed
 * individually: rows_slots[r] / rows_scales[r] point at row r's packed bytes
 * and scales (K/4 bytes, K/128 fp16).  y[m][r] over m in [0,M).  Used when
 * only some rows of a very large matrix are on the host. */
int orc_matvec_rows(const uint16_t *x, int64_t M, int64_t K, const uint8_t *const *rows_slots,
                    const uint16_t *const *rows_scales, int64_t R, double *y, double *bound,
                    int nthreads)
{
    int used = 1;
#ifdef _OPENMP
    if (nthreads < 1) nthreads = 1;
#pragma omp parallel for num_threads(nthreads) schedule(static)
    for (int64_t i = 0; i < M * R; i++) {
        if (i == 0) used = omp_get_num_threads();
        int64_t m = i / R, r = i % R;
        orc_dot(x, M, K, rows_slots[r], rows_scales[r], m, 0, &y[i], &bound[i]);
    }
#else
    (void)nthreads;
    for (int64_t i = 0; i < M * R; i++) {
        int64_t m = i / R, r = i % R;
        orc_dot(x, M, K, rows_slots[r], rows_scales[r], m, 0, &y[i], &bound[i]);
    }
#endif
    return used;
}

/* Embedding lookup: out[m][k] = s[id][k/128] * t[id][k] for the table row
 * id = ids[m] (the same fp64 weight orc_weight gives, so the sign of a zero
 * follows IEEE multiplication by the scale); an id outside [0, V) gives a row
 * of +0.  Returns the number of such ids.  (Embeddings are among the ternary
 * matrices: "Ternary-Bonsai-27B" model summary, aitrends.kr, section
 * "Differentiators".) */
int64_t orc_embed(const uint8_t *slots, const uint16_t *scales, int64_t V, int64_t K, const int32_t *ids,
                  int64_t M, double *out)
{
    int64_t bad = 0;
    for (int64_t m = 0; m < M; m++) {
        int64_t id = ids[m];
        if (id < 0 || id >= V) {
            bad++;
            for (int64_t k = 0; k < K; k++) out[m * K + k] = 0.0;
            continue;
        }
        for (int64_t k = 0; k < K; k++) out[m * K + k] = orc_weight(slots, scales, K, id, k);
    }
    return bad;
}

/* ------------------------------------------------------------------------
 * The 1-bit variant ("Bonsai 27B ternary / 1-bit quantization", ThakiCloud
 * blog, sections "What it is" and "How compression works": weights in
 * {-1, +1} with one FP16 scale per 128 weights, 1 + 16/128 = 1.125
 * bits/weight).  The pages give no bit layout; this library's: bit b =
 * (t + 1) / 2 (0 -> -1, 1 -> +1), weight (n,k) in byte n*K/8 + k/8 at bit
 * k%8 (least significant bit first); scales fp16 [N][K/128] as for the
 * ternary slots.
 * ------------------------------------------------------------------------ */

int64_t orc_b1_slots_bytes(int64_t N, int64_t K) { return N * (K / 8); }

/* Pack codes [N][K] (int8, -1 or +1) and scales into the 1-bit layout.  Any
 * other input is stored as bit 0 and counted.  Returns the count (or -1 for
 * a bad K); *first_bad receives the flat index of the first one (or -1). */
int64_t orc_pack_b1(const int8_t *codes, const uint16_t *scales_in, int64_t N, int64_t K, uint8_t *bits,
                    uint16_t *scales_out, int64_t *first_bad)
{
    int64_t bad = 0, first = -1;
    if (K <= 0 || N <= 0 || K % ORC_GROUP != 0) return -1;
    for (int64_t i = 0; i < N * (K / 8); i++) bits[i] = 0;
    for (int64_t n = 0; n < N; n++) {
        for (int64_t k = 0; k < K; k++) {
            int t = codes[n * K + k];
            int b = 0;
            if (t == 1) {
                b = 1;
            } else if (t != -1) {
                if (first < 0) first = n * K + k;
                bad++;
            }
            bits[n * (K / 8) + k / 8] |= (uint8_t)(b << (k % 8));
        }
    }
    for (int64_t i = 0; i < N * (K / ORC_GROUP); i++) scales_out[i] = scales_in[i];
    if (first_bad) *first_bad = first;
    return bad;
}

/* Bit of weight (n,k) -> t in {-1, +1}. */
static int orc_b1_value(const uint8_t *bits, int64_t K, int64_t n, int64_t k)
{
#if ORC_MUTANT == 7
    return ((bits[n * (K / 8) + k / 8] >> (7 - k % 8)) & 1) ? 1 : -1; /* planted: bits MSB first */
#elif ORC_MUTANT == 8
    return ((bits[n * (K / 8) + k / 8] >> (k % 8)) & 1) ? -1 : 1; /* planted: bit meaning swapped */
#else
    return ((bits[n * (K / 8) + k / 8] >> (k % 8)) & 1) ? 1 : -1;
#endif
}

int64_t orc_unpack_b1(const uint8_t *bits, int64_t N, int64_t K, int8_t *codes_out)
{
    if (K <= 0 || N <= 0 || K % ORC_GROUP != 0) return -1;
    for (int64_t n = 0; n < N; n++)
        for (int64_t k = 0; k < K; k++) codes_out[n * K + k] = (int8_t)orc_b1_value(bits, K, n, k);
    return 0;
}

/* w[n][k] = s[n][k/128] * t[n][k] in fp64 (exact). */
double orc_b1_weight(const uint8_t *bits, const uint16_t *scales, int64_t K, int64_t n, int64_t k)
{
#if ORC_MUTANT == 9
    return orc_half_to_double(scales[n * (K / ORC_GROUP)]) * (double)orc_b1_value(bits, K, n, k); /* planted: one scale per row */
#else
    return orc_half_to_double(scales[n * (K / ORC_GROUP) + k / ORC_GROUP]) * (double)orc_b1_value(bits, K, n, k);
#endif
}

/* y[M][N] = x[M][K] * W^T with the 1-bit weights, naive fp64 in k order, and
 * the bound sum_k |x*w|.  Returns the thread count used. */
int orc_b1_matmul(const uint16_t *x, int64_t M, int64_t K, const uint8_t *bits, const uint16_t *scales,
                  int64_t N, double *y, double *bound, int nthreads)
{
    int used = 1;
#ifdef _OPENMP
    if (nthreads < 1) nthreads = 1;
#pragma omp parallel for num_threads(nthreads) schedule(static)
#else
    (void)nthreads;
#endif
    for (int64_t i = 0; i < M * N; i++) {
#ifdef _OPENMP
        if (i == 0) used = omp_get_num_threads();
#endif
        int64_t m = i / N, n = i % N;
        double acc = 0.0, b = 0.0;
        for (int64_t k = 0; k < K; k++) {
            double p = orc_half_to_double(x[m * K + k]) * orc_b1_weight(bits, scales, K, n, k);
            acc += p;
            b += fabs(p);
        }
        y[i] = acc;
        bound[i] = b;
    }
    return used;
}

/* ------------------------------------------------------------------------
 * Dense ternary packing, five trits per byte.  The pages expect a "native
 * ternary" kernel near the log2(3) + 16/128 ~= 1.71 bits/weight ideal instead
 * of 2-bit slots, without a layout ("Ternary-Bonsai-27B" model summary,
 * aitrends.kr, sections "TL;DR" and "Technical features"; "Ternary
 * quantization: 27B in 7 GB", devnsb blog, section "Limits").  Reading
 * taken: 3^5 = 243 <= 256, so a byte holds five codes as base-3 digits,
 *   byte value v = sum_{i=0..4} c_i * 3^i,  c = t + 1 (0 -> -1, 1 -> 0, 2 -> +1),
 * least significant digit first, inside each 128-weight scale group: weight j
 * of group g is digit j % 5 of byte 26 g + j / 5 of the row (25 full bytes
 * and one byte holding weights 125..127, whose digits 3 and 4 are 0); each
 * row is padded with zero bytes to a multiple of 16 bytes (R = 26 K / 128
 * rounded up to 16); scales fp16 [N][K/128] as for the 2-bit slots.
 * 26 * 8 / 128 + 16/128 = 1.75 bits/weight.  Byte values 243..255 are
 * invalid.
 * ------------------------------------------------------------------------ */

int64_t orc_t5_row_bytes(int64_t K)
{
    if (K <= 0) return 0;
#if ORC_MUTANT == 12
    return 26 * (K / ORC_GROUP); /* planted: no padding to 16 bytes */
#else
    return (26 * (K / ORC_GROUP) + 15) / 16 * 16;
#endif
}

/* Byte of weight k inside its row. */
static int64_t orc_t5_byte(int64_t k)
{
#if ORC_MUTANT == 13
    return k / 5; /* planted: digits continue across groups */
#else
    return 26 * (k / ORC_GROUP) + (k % ORC_GROUP) / 5;
#endif
}

/* power of three of digit position d (0..4) */
static int orc_pow3(int d)
{
    int p = 1;
    for (int i = 0; i < d; i++) p *= 3;
    return p;
}

/* Digit position of weight k inside its byte. */
static int orc_t5_pos(int64_t k)
{
    const int j = (int)(k % ORC_GROUP);
#if ORC_MUTANT == 10
    return 4 - j % 5; /* planted: most significant digit first */
#elif ORC_MUTANT == 13
    return (int)(k % 5);
#else
    return j % 5;
#endif
}

/* Code c of weight (n,k), or -1 for an invalid byte (243..255). */
static int orc_t5_code(const uint8_t *bytes, int64_t K, int64_t n, int64_t k)
{
    int v = bytes[n * orc_t5_row_bytes(K) + orc_t5_byte(k)];
    if (v >= 243) return -1;
#if ORC_MUTANT == 11
    return (v >> (2 * orc_t5_pos(k))) & 3; /* planted: base 4 instead of 3 */
#else
    return (v / orc_pow3(orc_t5_pos(k))) % 3;
#endif
}

/* Pack codes [N][K] (int8 in {-1,0,+1}) and scales.  Any other code is
 * stored as digit 1 (t = 0) and counted; returns the count (or -1 for a bad
 * K); *first_bad receives the flat index of the first one (or -1). */
int64_t orc_pack_t5(const int8_t *codes, const uint16_t *scales_in, int64_t N, int64_t K, uint8_t *bytes,
                    uint16_t *scales_out, int64_t *first_bad)
{
    int64_t bad = 0, first = -1;
    if (K <= 0 || N <= 0 || K % ORC_GROUP != 0) return -1;
    const int64_t R = orc_t5_row_bytes(K);
    for (int64_t i = 0; i < N * R; i++) bytes[i] = 0;
    for (int64_t n = 0; n < N; n++) {
        for (int64_t k = 0; k < K; k++) {
            int t = codes[n * K + k];
            int c = t + 1;
            if (t < -1 || t > 1) {
                c = 1;
                if (first < 0) first = n * K + k;
                bad++;
            }
            bytes[n * R + orc_t5_byte(k)] = (uint8_t)(bytes[n * R + orc_t5_byte(k)] + c * orc_pow3(orc_t5_pos(k)));
        }
    }
    for (int64_t i = 0; i < N * (K / ORC_GROUP); i++) scales_out[i] = scales_in[i];
    if (first_bad) *first_bad = first;
    return bad;
}

/* codes_out [N][K]: t = c - 1, or the sentinel 2 for weights of an invalid byte. */
int64_t orc_unpack_t5(const uint8_t *bytes, int64_t N, int64_t K, int8_t *codes_out)
{
    if (K <= 0 || N <= 0 || K % ORC_GROUP != 0) return -1;
    for (int64_t n = 0; n < N; n++)
        for (int64_t k = 0; k < K; k++) {
            int c = orc_t5_code(bytes, K, n, k);
            codes_out[n * K + k] = (int8_t)(c < 0 ? 2 : c - 1);
        }
    return 0;
}

/* w[n][k] = s[n][k/128] * t[n][k] in fp64 (exact); an invalid byte gives 0. */
double orc_t5_weight(const uint8_t *bytes, const uint16_t *scales, int64_t K, int64_t n, int64_t k)
{
    int c = orc_t5_code(bytes, K, n, k);
    if (c < 0) return 0.0;
    return orc_half_to_double(scales[n * (K / ORC_GROUP) + k / ORC_GROUP]) * (double)(c - 1);
}

/* y[M][N] = x[M][K] * W^T with the five-per-byte weights, naive fp64 in k
 * order, and the bound sum_k |x*w|.  Returns the thread count used. */
int orc_t5_matmul(const uint16_t *x, int64_t M, int64_t K, const uint8_t *bytes, const uint16_t *scales,
                  int64_t N, double *y, double *bound, int nthreads)
{
    int used = 1;
#ifdef _OPENMP
    if (nthreads < 1) nthreads = 1;
#pragma omp parallel for num_threads(nthreads) schedule(static)
#else
    (void)nthreads;
#endif
    for (int64_t i = 0; i < M * N; i++) {
#ifdef _OPENMP
        if (i == 0) used = omp_get_num_threads();
#endif
        int64_t m = i / N, n = i % N;
        double acc = 0.0, b = 0.0;
        for (int64_t k = 0; k < K; k++) {
            double p = orc_half_to_double(x[m * K + k]) * orc_t5_weight(bytes, scales, K, n, k);
            acc += p;
            b += fabs(p);
        }
        y[i] = acc;
        bound[i] = b;
    }
    return used;
}

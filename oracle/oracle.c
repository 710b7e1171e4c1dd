/*
 * oracle.c -- plain, slow CPU reference for groupwise affine low-bit weight
 * quantization and for the matmul Y = X * What^T that decode runs.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It shares no code,
 * header, table or helper with the CUDA library.
 *
 * Sources (the three web pages on the subject):
 *   [P1] "vLLM 量化与推测解码" -- section 1 (affine equations q = clamp(round(x/s)+z,
 *        qmin, qmax), x^ = s(q - z); min-max scale s = (xmax-xmin)/(qmax-qmin),
 *        zero z = round(qmin - xmin/s); unsigned range qmin = 0, qmax = 2^b - 1;
 *        the per-tensor / per-group executable example, whose range is widened
 *        to contain 0, whose degenerate range gets scale 1.0 and whose zero is
 *        clamped); section 2 (weight payload = Nparam*b/8 + metadata, two INT4
 *        codes per byte, 2-byte scale + 2-byte zero per group).
 *   [P2] "量化" (llminference s08) -- "解法" (symmetric per-group quantizer:
 *        z = 0, s = absmax/qmax with qmax = 2^(b-1) - 1, codes clipped to
 *        [-qmax-1, qmax], scale stored as fp16); "实现" (fused dequant inside
 *        the accumulation).
 *   [P3] "量化：为何加速推理与精度权衡" -- "直接答案" (error bound scale/2) and
 *        "深入原理" (real 0 is represented exactly).
 *
 * Readings taken where the pages leave a step open (each is listed in the
 * design notes):
 *   - round() is round-half-to-even (Python round / numpy round); here it is
 *     nearbyint() under the default FE_TONEAREST mode.
 *   - The arithmetic is done in double precision, the precision the pages'
 *     Python code uses.  Inputs are binary16 weights, so every quotient the
 *     method rounds is decided exactly (see the tests' exact-rational pins).
 *   - The scale is stored as binary16, rounded toward +infinity, and codes
 *     are computed with the stored scale, so that the stored metadata
 *     reproduces the codes and the bound |x - x^| <= s/2 holds for the
 *     stored s.
 *   - The zero point is stored as a binary16 holding an integer.
 *   - Symmetric codes are stored offset-binary: u = q + 2^(b-1).
 *   - 4-bit packing: byte j of a row holds k = 2j in its low nibble and
 *     k = 2j + 1 in its high nibble.
 *
 * Build: gcc -O2 -fopenmp -ffp-contract=off -fno-fast-math -shared -fPIC.
 */
#include <math.h>
#include <omp.h>
#include <stdint.h>
#include <string.h>

/* ---- binary16 / bfloat16 decoding, from the IEEE-754 field definitions ---- */

/* value of a binary16 bit pattern: sign, 5-bit exponent (bias 15), 10-bit
 * fraction; exponent 0 is subnormal (fraction * 2^-24). */
static double half_bits_to_double(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int f = h & 0x3ff;
    double v;
    if (e == 0)
        v = ldexp((double)f, -24);
    else if (e == 31)
        v = f ? NAN : INFINITY;
    else
        v = ldexp((double)(f + 1024), e - 25);
    return sign ? -v : v;
}

/* bfloat16 is the upper half of a binary32 pattern. */
static double bf16_bits_to_double(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Smallest binary16 value >= x, for x > 0: binary search over the positive
 * finite patterns 0x0001..0x7bff, whose values increase with the pattern.
 * Returns +inf (0x7c00) above the largest finite value. */
static uint16_t half_round_up_positive(double x)
{
    if (x > half_bits_to_double(0x7bff))
        return 0x7c00;
    uint16_t lo = 0x0001, hi = 0x7bff; /* answer lies in [lo, hi] */
    while (lo < hi) {
        uint16_t mid = (uint16_t)(lo + (hi - lo) / 2);
        if (half_bits_to_double(mid) >= x)
            hi = mid;
        else
            lo = (uint16_t)(mid + 1);
    }
    return lo;
}

/* binary16 pattern of a small non-negative integer (exact for 0..2048). */
static uint16_t half_bits_of_small_int(int z)
{
    if (z == 0)
        return 0;
    int e = 0;
    while ((z >> (e + 1)) != 0)
        e++;                                   /* 2^e <= z < 2^(e+1) */
    int frac = (z << (10 - e)) & 0x3ff;        /* e <= 10 here */
    return (uint16_t)(((e + 15) << 10) | frac);
}

static double clampd(double v, double lo, double hi)
{
    return v < lo ? lo : (v > hi ? hi : v);
}

/* ---- quantize ----------------------------------------------------------- */

/* Quantize W[N][K] (binary16 bit patterns, row-major) in groups of `group`
 * consecutive weights along K.
 *   q_out     : int32 codes, [N][K] (the unpacked codes; may be NULL)
 *   codes     : packed codes, [N][K*bits/8] bytes (may be NULL)
 *   scales    : binary16 scale per (row, group), [N][K/group]
 *   zeros     : binary16 integer zero per (row, group), [N][K/group]
 *               (asymmetric only; ignored when symmetric)
 * Asymmetric follows [P1] section 1: range widened to contain 0, scale from
 * the min-max formula, scale 1.0 when the range is degenerate, zero rounded
 * then clamped, code = clamp(round(w/s) + z).  Symmetric follows [P2] "解法":
 * s = max|w| / (2^(b-1)-1), code = clip(round(w/s), -2^(b-1), 2^(b-1)-1). */
void oracle_quantize(const uint16_t *W, int64_t N, int64_t K, int bits,
                     int group, int symmetric, int32_t *q_out, uint8_t *codes,
                     uint16_t *scales, uint16_t *zeros)
{
    const int64_t ngroups = K / group;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; n++) {
        for (int64_t g = 0; g < ngroups; g++) {
            const uint16_t *w = W + n * K + g * group;
            double s;
            uint16_t s16;
            double z;      /* zero point (integer valued) */
            double qmin, qmax;
            if (!symmetric) {
                qmin = 0.0;
                qmax = (double)((1 << bits) - 1);
                double lo = 0.0, hi = 0.0; /* range must contain real 0 */
                for (int i = 0; i < group; i++) {
                    double v = half_bits_to_double(w[i]);
                    if (v < lo) lo = v;
                    if (v > hi) hi = v;
                }
                if (hi == lo) {
                    s16 = 0x3c00; /* 1.0 */
                    s = 1.0;
                    z = 0.0;
                } else {
                    s16 = half_round_up_positive((hi - lo) / (qmax - qmin));
                    s = half_bits_to_double(s16);
                    z = clampd(nearbyint(qmin - lo / s), qmin, qmax);
                }
                zeros[n * ngroups + g] = half_bits_of_small_int((int)z);
            } else {
                double qm = (double)((1 << (bits - 1)) - 1);
                qmin = -qm - 1.0;
                qmax = qm;
                double a = 0.0;
                for (int i = 0; i < group; i++) {
                    double v = fabs(half_bits_to_double(w[i]));
                    if (v > a) a = v;
                }
                if (a == 0.0) {
                    s16 = 0x3c00;
                    s = 1.0;
                } else {
                    s16 = half_round_up_positive(a / qm);
                    s = half_bits_to_double(s16);
                }
                z = 0.0;
            }
            scales[n * ngroups + g] = s16;

            for (int i = 0; i < group; i++) {
                int64_t k = g * group + i;
                double v = half_bits_to_double(w[i]);
                double q = clampd(nearbyint(v / s) + z, qmin, qmax);
                int u = symmetric ? (int)q + (1 << (bits - 1)) : (int)q;
                if (q_out)
                    q_out[n * K + k] = (int32_t)q;
                if (codes) {
                    if (bits == 8) {
                        codes[n * K + k] = (uint8_t)u;
                    } else { /* bits == 4: even k low nibble, odd k high */
                        uint8_t *byte = &codes[n * (K / 2) + k / 2];
                        if ((k & 1) == 0)
                            *byte = (uint8_t)((*byte & 0xf0) | (u & 0x0f));
                        else
                            *byte = (uint8_t)((*byte & 0x0f) | ((u & 0x0f) << 4));
                    }
                }
            }
        }
    }
}

/* ---- dequantize --------------------------------------------------------- */

/* Decode the stored code of weight (n, k) back to its integer q. */
static int code_at(const uint8_t *codes, int64_t K, int bits, int symmetric,
                   int64_t n, int64_t k)
{
    int u;
    if (bits == 8)
        u = codes[n * K + k];
    else {
        uint8_t byte = codes[n * (K / 2) + k / 2];
        u = (k & 1) ? (byte >> 4) : (byte & 0x0f);
    }
    return symmetric ? u - (1 << (bits - 1)) : u;
}

/* What[N][K] = s * (q - z) in double (exact: an 11-bit scale times a code
 * difference of at most 9 bits).  [P1] section 1, x^ = s(q - z). */
void oracle_dequantize(const uint8_t *codes, const uint16_t *scales,
                       const uint16_t *zeros, int64_t N, int64_t K, int bits,
                       int group, int symmetric, double *What)
{
    const int64_t ngroups = K / group;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; n++) {
        for (int64_t k = 0; k < K; k++) {
            int64_t g = k / group;
            double s = half_bits_to_double(scales[n * ngroups + g]);
            double z = symmetric ? 0.0 : half_bits_to_double(zeros[n * ngroups + g]);
            int q = code_at(codes, K, bits, symmetric, n, k);
            What[n * K + k] = s * ((double)q - z);
        }
    }
}

/* ---- matmul ------------------------------------------------------------- */

/* Y[m][n] = sum_k X[m][k] * What[n][k] and Yabs[m][n] = sum_k |X[m][k] *
 * What[n][k]|, both in double, What decoded from the stored codes row by row.
 * X is bfloat16 bit patterns, [M][K] row-major.  ([P1] section 2, Y = X W^T;
 * the dequantized weights are the ones the stored metadata define.) */
void oracle_matmul(const uint16_t *X, int64_t M, const uint8_t *codes,
                   const uint16_t *scales, const uint16_t *zeros, int64_t N,
                   int64_t K, int bits, int group, int symmetric, double *Y,
                   double *Yabs)
{
    const int64_t ngroups = K / group;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; n++) {
        for (int64_t m = 0; m < M; m++) {
            double acc = 0.0, accabs = 0.0;
            for (int64_t k = 0; k < K; k++) {
                int64_t g = k / group;
                double s = half_bits_to_double(scales[n * ngroups + g]);
                double z = symmetric ? 0.0 : half_bits_to_double(zeros[n * ngroups + g]);
                double w = s * ((double)code_at(codes, K, bits, symmetric, n, k) - z);
                double p = bf16_bits_to_double(X[m * K + k]) * w;
                acc += p;
                accabs += fabs(p);
            }
            Y[m * N + n] = acc;
            Yabs[m * N + n] = accabs;
        }
    }
}

/* The same sum for a list of (m, n) output coordinates only: y[i] for
 * (ms[i], ns[i]).  Used to check large outputs one element at a time. */
void oracle_matmul_at(const uint16_t *X, int64_t M, const uint8_t *codes,
                      const uint16_t *scales, const uint16_t *zeros, int64_t N,
                      int64_t K, int bits, int group, int symmetric,
                      const int64_t *ms, const int64_t *ns, int64_t count,
                      double *y, double *yabs)
{
    (void)M;
    (void)N;
    const int64_t ngroups = K / group;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < count; i++) {
        int64_t m = ms[i], n = ns[i];
        double acc = 0.0, accabs = 0.0;
        for (int64_t k = 0; k < K; k++) {
            int64_t g = k / group;
            double s = half_bits_to_double(scales[n * ngroups + g]);
            double z = symmetric ? 0.0 : half_bits_to_double(zeros[n * ngroups + g]);
            double w = s * ((double)code_at(codes, K, bits, symmetric, n, k) - z);
            double p = bf16_bits_to_double(X[m * K + k]) * w;
            acc += p;
            accabs += fabs(p);
        }
        y[i] = acc;
        yabs[i] = accabs;
    }
}

/* Dense reference: Y[m][n] = sum_k X[m][k] * B[n][k] with B given as
 * bfloat16 bit patterns (the unfused path's materialised weights). */
void oracle_matmul_dense_bf16(const uint16_t *X, int64_t M, const uint16_t *B,
                              int64_t N, int64_t K, double *Y)
{
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; n++) {
        for (int64_t m = 0; m < M; m++) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; k++)
                acc += bf16_bits_to_double(X[m * K + k]) *
                       bf16_bits_to_double(B[n * K + k]);
            Y[m * N + n] = acc;
        }
    }
}

/* Exposed for the tests' independent checks of the decoders. */
/* ---- nested superblocks (Q4_K-style), 4.5 bits per weight ---------------
 *
 * [P2] "量化", the Q4_K superblock figure: 256 weights in 8 subblocks of 32;
 * every subblock has a 6-bit scale and a 6-bit minimum, themselves quantized
 * against a binary16 super-scale d and super-minimum dmin; 4-bit codes;
 * 4.5 bits per weight.  The page fixes only the nesting and the bit counts.
 * The plain reading taken here (listed in the design notes):
 *   subblock j:  lo = min(0, min w), hi = max(0, max w)  (P1's range),
 *                s_j = (hi - lo) / 15,  m_j = -lo;
 *   d    = smallest binary16 >= max_j s_j / 63  (0 when every s_j is 0),
 *   dmin = smallest binary16 >= max_j m_j / 63  (0 when every m_j is 0);
 *   sc_j = clamp(round(s_j / d), 1, 63)     (1 when d = 0),
 *   mq_j = clamp(round(m_j / dmin), 0, 63)  (0 when dmin = 0);
 *   S_j = d sc_j,  M_j = dmin mq_j  (exact);
 *   q = clamp(round((w + M_j) / S_j), 0, 15)  (0 when S_j = 0);
 *   w^ = S_j q - M_j.
 * Every rounding is round-half-to-even of the exact quotient: the operands
 * are binary16 values and products of them with small integers, so the
 * double-precision quotients land on the right side of every half-integer
 * and exact ties stay exact.
 * Block layout (144 bytes): d (binary16, little-endian), dmin, 12 bytes
 * holding sc_0..sc_7 then mq_0..mq_7 as 6-bit fields, least significant bit
 * first (field f in bits 6f .. 6f+5 of the 96-bit little-endian value), then
 * 128 bytes of codes (byte i: weight 2i in the low nibble, 2i+1 in the high).
 * Blocks run along K: block b of row n covers k = 256 b .. 256 b + 255, and
 * row n's blocks are contiguous (K/256 blocks per row). */
void oracle_q4k_quantize(const uint16_t *W, int64_t N, int64_t K, uint8_t *blocks)
{
    const int64_t nb = K / 256;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; n++) {
        for (int64_t b = 0; b < nb; b++) {
            const uint16_t *w = W + n * K + b * 256;
            uint8_t *blk = blocks + (n * nb + b) * 144;
            double s[8], m[8], smax = 0.0, mmax = 0.0;
            for (int j = 0; j < 8; j++) {
                double lo = 0.0, hi = 0.0;
                for (int i = 0; i < 32; i++) {
                    double v = half_bits_to_double(w[32 * j + i]);
                    if (v < lo) lo = v;
                    if (v > hi) hi = v;
                }
                s[j] = (hi - lo) / 15.0;
                m[j] = -lo;
                if (s[j] > smax) smax = s[j];
                if (m[j] > mmax) mmax = m[j];
            }
            uint16_t d16 = smax > 0.0 ? half_round_up_positive(smax / 63.0) : 0;
            uint16_t dm16 = mmax > 0.0 ? half_round_up_positive(mmax / 63.0) : 0;
            double d = half_bits_to_double(d16), dmin = half_bits_to_double(dm16);
            int sc[8], mq[8];
            for (int j = 0; j < 8; j++) {
                sc[j] = d > 0.0 ? (int)clampd(nearbyint(s[j] / d), 1.0, 63.0) : 1;
                mq[j] = dmin > 0.0 ? (int)clampd(nearbyint(m[j] / dmin), 0.0, 63.0) : 0;
            }
            memset(blk, 0, 144);
            blk[0] = (uint8_t)(d16 & 0xff);
            blk[1] = (uint8_t)(d16 >> 8);
            blk[2] = (uint8_t)(dm16 & 0xff);
            blk[3] = (uint8_t)(dm16 >> 8);
            for (int f = 0; f < 16; f++) {
                int v = f < 8 ? sc[f] : mq[f - 8];
                for (int bit = 0; bit < 6; bit++) {
                    if ((v >> bit) & 1) {
                        int pos = 6 * f + bit;
                        blk[4 + pos / 8] |= (uint8_t)(1u << (pos % 8));
                    }
                }
            }
            for (int k = 0; k < 256; k++) {
                int j = k / 32;
                double S = d * sc[j], M = dmin * mq[j];
                double v = half_bits_to_double(w[k]);
                int q = S > 0.0 ? (int)clampd(nearbyint((v + M) / S), 0.0, 15.0) : 0;
                blk[16 + k / 2] |= (uint8_t)((k & 1) ? (q << 4) : q);
            }
        }
    }
}

/* w^ = S_j q - M_j for every weight of the blocks written by
 * oracle_q4k_quantize (fields read back from the bytes); out is [N][K]. */
void oracle_q4k_dequantize(const uint8_t *blocks, int64_t N, int64_t K, double *out)
{
    const int64_t nb = K / 256;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; n++) {
        for (int64_t b = 0; b < nb; b++) {
            const uint8_t *blk = blocks + (n * nb + b) * 144;
            double d = half_bits_to_double((uint16_t)(blk[0] | (blk[1] << 8)));
            double dmin = half_bits_to_double((uint16_t)(blk[2] | (blk[3] << 8)));
            int field[16];
            for (int f = 0; f < 16; f++) {
                int v = 0;
                for (int bit = 0; bit < 6; bit++) {
                    int pos = 6 * f + bit;
                    v |= ((blk[4 + pos / 8] >> (pos % 8)) & 1) << bit;
                }
                field[f] = v;
            }
            for (int k = 0; k < 256; k++) {
                int j = k / 32;
                int q = (blk[16 + k / 2] >> ((k & 1) * 4)) & 0x0f;
                out[n * K + b * 256 + k] = d * field[j] * q - dmin * field[8 + j];
            }
        }
    }
}

double oracle_half_to_double(uint16_t h) { return half_bits_to_double(h); }
uint16_t oracle_half_round_up(double x) { return half_round_up_positive(x); }
double oracle_bf16_to_double(uint16_t b) { return bf16_bits_to_double(b); }

/* Thread count of the OpenMP loops above (timing the oracle at one thread
 * and at all threads); not part of the arithmetic. */
void oracle_set_threads(int n) { omp_set_num_threads(n > 0 ? n : 1); }
int oracle_max_threads(void) { return omp_get_max_threads(); }

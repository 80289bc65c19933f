/*
 * lowbit_oracle.c -- the CPU oracle for the packed low-bit products.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the plain, slow, obviously-correct
 * statement of what the GPU library computes.  Only the test-suite, the smoke
 * check and the benchmark's CPU-baseline leg may load it.  It shares no code,
 * header, table or constant with the CUDA library, and the CUDA library never
 * calls it.
 *
 * Style rules kept on purpose:
 *   - single-threaded, no SIMD intrinsics, no blocking, no reordering;
 *   - floating point products are formed and summed in IEEE double, with the
 *     reduction index ascending, exactly as the defining sums are written;
 *   - integer products are summed in int64 and only then reduced mod 2^16.
 *
 * Sources (web pages; section named after the page title):
 *   [Z80]    "Show HN: Z80-uLM, a conversational AI that fits in 40KB"
 *            -- feature list (2-bit weights {-2,-1,0,+1}, 4 per byte; 16-bit
 *            integer inference), architecture list (128 query + 128 context
 *            trigram buckets, hidden layers, ReLU between hidden layers, one
 *            output neuron per character), the "unpack 2-bit weight" listing,
 *            the MULADD listing, and the per-layer arithmetic shift listing.
 *   [BONSAI] "Bonsai-27B-gguf technical white paper digest", section
 *            "technical architecture highlights" (one sign bit per weight,
 *            -1 or +1; one FP16 scale shared by every 128 weights; 1.125 bits
 *            per weight; 14.2x smaller than FP16).
 *   [ACORN]  "acorn-llm 0.11.4" project page, section "int4 quantisation
 *            quality: group quantisation" (one scale per group of values along
 *            the input dimension; symmetric round-to-nearest int4; the scale
 *            changes every 64 values).
 *
 * Readings taken where the pages are silent:
 *   - Q1 bit polarity: bit 1 -> +1, bit 0 -> -1.
 *   - Q1 bit order: weight k of a row is bit (k % 8) of byte (k / 8), LSB first
 *     (the same LSB-first order the Z80 listing uses for its 2-bit fields).
 *   - Q1 scale group: 128 consecutive weights along K of one row.
 *   - INT4: two's-complement nibble, even k in the low nibble, no zero point,
 *     group of 64 consecutive weights along K with one FP16 scale.
 *   - Q2 weight matrix is row-major [out][in], codes packed along `in`.
 *   - Shift after the output layer too; argmax ties go to the lowest index.
 *   - Trigram hash: FNV-1a 32-bit of the three bytes, bucket = hash mod 128,
 *     +32 per trigram, words padded with one space on each side.
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* Scalar decoders, written from the IEEE 754 / bfloat16 bit layouts.        */
/* ------------------------------------------------------------------------ */

/* binary16: 1 sign, 5 exponent (bias 15), 10 fraction bits. */
double orc_f16_to_f64(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int expo = (h >> 10) & 0x1F;
    int frac = h & 0x3FF;
    double v;
    if (expo == 0)
        v = ldexp((double)frac, -24);                 /* subnormal: frac * 2^-24 */
    else if (expo == 31)
        v = frac ? NAN : INFINITY;
    else
        v = ldexp((double)(frac + 1024), expo - 25);  /* (1.frac) * 2^(expo-15) */
    return sign ? -v : v;
}

/* bfloat16: 1 sign, 8 exponent (bias 127), 7 fraction bits. */
double orc_bf16_to_f64(uint16_t b)
{
    int sign = (b >> 15) & 1;
    int expo = (b >> 7) & 0xFF;
    int frac = b & 0x7F;
    double v;
    if (expo == 0)
        v = ldexp((double)frac, -133);                /* subnormal: frac * 2^-133 */
    else if (expo == 255)
        v = frac ? NAN : INFINITY;
    else
        v = ldexp((double)(frac + 128), expo - 134);  /* (1.frac) * 2^(expo-127) */
    return sign ? -v : v;
}

/* ------------------------------------------------------------------------ */
/* Q1_0_g128 [BONSAI]: one sign bit per weight, FP16 scale per 128 weights.  */
/* ------------------------------------------------------------------------ */

/* codes[r][c] in {0,1} -> packed[r][c/8], bit (c%8).  Returns 0, or -1 when
   cols is not a multiple of 8 or a code is out of range. */
int orc_q1_pack(const int8_t *codes, int64_t rows, int64_t cols, uint8_t *packed)
{
    if (cols % 8 != 0) return -1;
    for (int64_t r = 0; r < rows; r++) {
        for (int64_t j = 0; j < cols / 8; j++) {
            unsigned byte = 0;
            for (int i = 0; i < 8; i++) {
                int8_t c = codes[r * cols + 8 * j + i];
                if (c != 0 && c != 1) return -1;
                byte |= (unsigned)c << i;
            }
            packed[r * (cols / 8) + j] = (uint8_t)byte;
        }
    }
    return 0;
}

int orc_q1_unpack(const uint8_t *packed, int64_t rows, int64_t cols, int8_t *codes)
{
    if (cols % 8 != 0) return -1;
    for (int64_t r = 0; r < rows; r++)
        for (int64_t c = 0; c < cols; c++)
            codes[r * cols + c] = (int8_t)((packed[r * (cols / 8) + c / 8] >> (c % 8)) & 1);
    return 0;
}

/* The dequantised weight w[n][k] = (bit ? +1 : -1) * d[n][k/128]. */
double orc_q1_weight(const uint8_t *bits, const uint16_t *scales, int64_t K, int64_t n, int64_t k)
{
    int bit = (bits[n * (K / 8) + k / 8] >> (k % 8)) & 1;
    double d = orc_f16_to_f64(scales[n * (K / 128) + k / 128]);
    return bit ? d : -d;
}

/* y[m][n] = sum_k w[n][k] * x[m][k], in double, k ascending.
   absdot[m][n] = sum_k |w[n][k] * x[m][k]| (may be NULL). */
int orc_q1_gemv(const uint8_t *bits, const uint16_t *scales, const uint16_t *x,
                int64_t M, int64_t N, int64_t K, double *y, double *absdot)
{
    if (K % 128 != 0) return -1;
    for (int64_t m = 0; m < M; m++) {
        for (int64_t n = 0; n < N; n++) {
            double acc = 0.0, aacc = 0.0;
            for (int64_t k = 0; k < K; k++) {
                double p = orc_q1_weight(bits, scales, K, n, k) * orc_bf16_to_f64(x[m * K + k]);
                acc += p;
                aacc += fabs(p);
            }
            y[m * N + n] = acc;
            if (absdot) absdot[m * N + n] = aacc;
        }
    }
    return 0;
}

/* The same definition evaluated only at the listed (m, n) output elements. */
int orc_q1_gemv_at(const uint8_t *bits, const uint16_t *scales, const uint16_t *x,
                   int64_t K, const int64_t *ms, const int64_t *ns, int64_t count,
                   double *y, double *absdot)
{
    if (K % 128 != 0) return -1;
    for (int64_t i = 0; i < count; i++) {
        double acc = 0.0, aacc = 0.0;
        for (int64_t k = 0; k < K; k++) {
            double p = orc_q1_weight(bits, scales, K, ns[i], k) * orc_bf16_to_f64(x[ms[i] * K + k]);
            acc += p;
            aacc += fabs(p);
        }
        y[i] = acc;
        if (absdot) absdot[i] = aacc;
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* INT4, symmetric, FP16 scale per 64 weights along K [ACORN].               */
/* ------------------------------------------------------------------------ */

/* codes[r][c] in [-8,7] -> packed[r][c/2]; even c in the low nibble. */
int orc_int4_pack(const int8_t *codes, int64_t rows, int64_t cols, uint8_t *packed)
{
    if (cols % 2 != 0) return -1;
    for (int64_t r = 0; r < rows; r++) {
        for (int64_t j = 0; j < cols / 2; j++) {
            int8_t lo = codes[r * cols + 2 * j];
            int8_t hi = codes[r * cols + 2 * j + 1];
            if (lo < -8 || lo > 7 || hi < -8 || hi > 7) return -1;
            unsigned lo4 = (unsigned)(lo < 0 ? lo + 16 : lo);   /* two's complement in 4 bits */
            unsigned hi4 = (unsigned)(hi < 0 ? hi + 16 : hi);
            packed[r * (cols / 2) + j] = (uint8_t)(lo4 | (hi4 << 4));
        }
    }
    return 0;
}

static int nibble_value(unsigned nib)
{
    return nib >= 8 ? (int)nib - 16 : (int)nib;
}

int orc_int4_unpack(const uint8_t *packed, int64_t rows, int64_t cols, int8_t *codes)
{
    if (cols % 2 != 0) return -1;
    for (int64_t r = 0; r < rows; r++) {
        for (int64_t c = 0; c < cols; c++) {
            uint8_t byte = packed[r * (cols / 2) + c / 2];
            unsigned nib = (c % 2 == 0) ? (byte & 0xF) : (byte >> 4);
            codes[r * cols + c] = (int8_t)nibble_value(nib);
        }
    }
    return 0;
}

/* w[n][k] = q[n][k] * d[n][k/64]. */
double orc_int4_weight(const uint8_t *q, const uint16_t *scales, int64_t K, int64_t n, int64_t k)
{
    uint8_t byte = q[n * (K / 2) + k / 2];
    unsigned nib = (k % 2 == 0) ? (byte & 0xF) : (byte >> 4);
    return (double)nibble_value(nib) * orc_f16_to_f64(scales[n * (K / 64) + k / 64]);
}

int orc_int4_gemv(const uint8_t *q, const uint16_t *scales, const uint16_t *x,
                  int64_t M, int64_t N, int64_t K, double *y, double *absdot)
{
    if (K % 64 != 0) return -1;
    for (int64_t m = 0; m < M; m++) {
        for (int64_t n = 0; n < N; n++) {
            double acc = 0.0, aacc = 0.0;
            for (int64_t k = 0; k < K; k++) {
                double p = orc_int4_weight(q, scales, K, n, k) * orc_bf16_to_f64(x[m * K + k]);
                acc += p;
                aacc += fabs(p);
            }
            y[m * N + n] = acc;
            if (absdot) absdot[m * N + n] = aacc;
        }
    }
    return 0;
}

int orc_int4_gemv_at(const uint8_t *q, const uint16_t *scales, const uint16_t *x,
                     int64_t K, const int64_t *ms, const int64_t *ns, int64_t count,
                     double *y, double *absdot)
{
    if (K % 64 != 0) return -1;
    for (int64_t i = 0; i < count; i++) {
        double acc = 0.0, aacc = 0.0;
        for (int64_t k = 0; k < K; k++) {
            double p = orc_int4_weight(q, scales, K, ns[i], k) * orc_bf16_to_f64(x[ms[i] * K + k]);
            acc += p;
            aacc += fabs(p);
        }
        y[i] = acc;
        if (absdot) absdot[i] = aacc;
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Z80-style 2-bit integer MLP [Z80].                                        */
/* ------------------------------------------------------------------------ */

/* codes[r][c] in {0,1,2,3} -> packed[r][c/4], code of c at bits 2*(c%4). */
int orc_q2_pack(const int8_t *codes, int64_t rows, int64_t cols, uint8_t *packed)
{
    if (cols % 4 != 0) return -1;
    for (int64_t r = 0; r < rows; r++) {
        for (int64_t j = 0; j < cols / 4; j++) {
            unsigned byte = 0;
            for (int i = 0; i < 4; i++) {
                int8_t c = codes[r * cols + 4 * j + i];
                if (c < 0 || c > 3) return -1;
                byte |= (unsigned)c << (2 * i);
            }
            packed[r * (cols / 4) + j] = (uint8_t)byte;
        }
    }
    return 0;
}

int orc_q2_unpack(const uint8_t *packed, int64_t rows, int64_t cols, int8_t *codes)
{
    if (cols % 4 != 0) return -1;
    for (int64_t r = 0; r < rows; r++)
        for (int64_t c = 0; c < cols; c++)
            codes[r * cols + c] = (int8_t)((packed[r * (cols / 4) + c / 4] >> (2 * (c % 4))) & 3);
    return 0;
}

/* Code -> weight: the "sub 2" step of the unpack listing maps 0,1,2,3 to
   -2,-1,0,+1. */
int orc_q2_weight(const uint8_t *packed, int64_t in_dim, int64_t o, int64_t i)
{
    int code = (packed[o * (in_dim / 4) + i / 4] >> (2 * (i % 4))) & 3;
    return code - 2;
}

/* Reduce an exact integer sum to the 16-bit two's-complement register it
   would leave in a wrapping 16-bit accumulator. */
static int16_t wrap16(int64_t v)
{
    uint16_t u = (uint16_t)((uint64_t)v & 0xFFFFu);
    return (int16_t)(u >= 0x8000u ? (int32_t)u - 0x10000 : (int32_t)u);
}

/* Arithmetic right shift by 2 of a 16-bit register: the listing's
   "sra h / rr l" pair done twice.  Written as floor division by 4, which is
   what a sign-preserving shift of a two's-complement value computes. */
static int16_t sra2(int16_t v)
{
    int32_t q = v / 4;
    if ((v % 4) != 0 && v < 0) q -= 1;   /* C division truncates; floor it */
    return (int16_t)q;
}

/* One layer, exact form: acc = sum_i w[o][i] * a[i] in int64, then wrapped
   to 16 bits, then shifted.  Hidden layers apply ReLU; the output layer does
   not.  out[] receives the post-shift (and post-ReLU for hidden) values. */
void orc_q2_layer(const uint8_t *packed, int64_t in_dim, int64_t out_dim,
                  const int16_t *a, int is_hidden, int16_t *out)
{
    for (int64_t o = 0; o < out_dim; o++) {
        int64_t acc = 0;
        for (int64_t i = 0; i < in_dim; i++)
            acc += (int64_t)orc_q2_weight(packed, in_dim, o, i) * (int64_t)a[i];
        int16_t z = sra2(wrap16(acc));
        out[o] = (is_hidden && z < 0) ? 0 : z;
    }
}

/* One layer, register-level form: the MULADD listing taken literally in its
   arithmetic meaning -- weight 0 skips, +1 adds the activation once, -1
   subtracts it once, -2 subtracts it twice -- with the 16-bit accumulator
   wrapping after every single add or subtract. */
void orc_q2_layer_muladd16(const uint8_t *packed, int64_t in_dim, int64_t out_dim,
                           const int16_t *a, int is_hidden, int16_t *out)
{
    for (int64_t o = 0; o < out_dim; o++) {
        int16_t hl = 0;
        for (int64_t i = 0; i < in_dim; i++) {
            int w = orc_q2_weight(packed, in_dim, o, i);
            int16_t de = a[i];
            if (w == 0) continue;
            if (w == 1) { hl = wrap16((int64_t)hl + de); continue; }
            hl = wrap16((int64_t)hl - de);
            if (w == -2) hl = wrap16((int64_t)hl - de);
        }
        int16_t z = sra2(hl);
        out[o] = (is_hidden && z < 0) ? 0 : z;
    }
}

/* Smallest index of the maximum. */
int32_t orc_argmax16(const int16_t *v, int64_t n)
{
    int32_t best = 0;
    for (int64_t i = 1; i < n; i++)
        if (v[i] > v[best]) best = (int32_t)i;
    return best;
}

/* Whole network for a batch of input vectors.
   packed_layers[l] is [dims[l+1]][dims[l]/4].  logits[b][dims[n_layers]];
   argmax may be NULL.  use_muladd16 selects the register-level form.
   dims[] must not exceed 4096. */
int orc_q2_mlp_forward(const uint8_t *const *packed_layers, const int32_t *dims, int n_layers,
                       const int16_t *x, int64_t batch, int16_t *logits, int32_t *argmax,
                       int use_muladd16)
{
    static int16_t bufa[4096], bufb[4096];
    if (n_layers < 1) return -1;
    for (int l = 0; l <= n_layers; l++)
        if (dims[l] < 1 || dims[l] > 4096 || (l < n_layers && dims[l] % 4 != 0)) return -1;
    for (int64_t b = 0; b < batch; b++) {
        memcpy(bufa, x + b * dims[0], sizeof(int16_t) * (size_t)dims[0]);
        int16_t *cur = bufa, *nxt = bufb;
        for (int l = 0; l < n_layers; l++) {
            int hidden = (l < n_layers - 1);
            if (use_muladd16)
                orc_q2_layer_muladd16(packed_layers[l], dims[l], dims[l + 1], cur, hidden, nxt);
            else
                orc_q2_layer(packed_layers[l], dims[l], dims[l + 1], cur, hidden, nxt);
            int16_t *t = cur; cur = nxt; nxt = t;
        }
        int64_t nout = dims[n_layers];
        memcpy(logits + b * nout, cur, sizeof(int16_t) * (size_t)nout);
        if (argmax) argmax[b] = orc_argmax16(cur, nout);
    }
    return 0;
}

/* Trigram-bucket encoder [Z80 "trigram hash encoding"]: the text is lower-
   cased and split on spaces; each word, padded with one space on each side,
   contributes +32 to bucket (FNV-1a-32 of each 3-byte window) mod 128.  Word
   order does not change the result, because every trigram lies inside one
   word. */
static uint32_t fnv1a3(const unsigned char *p)
{
    uint32_t h = 2166136261u;
    for (int i = 0; i < 3; i++) {
        h ^= p[i];
        h *= 16777619u;
    }
    return h;
}

void orc_trigram_encode(const char *text, int16_t *buckets /* [128] */)
{
    unsigned char word[258];
    memset(buckets, 0, 128 * sizeof(int16_t));
    size_t n = strlen(text), i = 0;
    while (i < n) {
        while (i < n && text[i] == ' ') i++;
        size_t len = 0;
        word[len++] = ' ';
        while (i < n && text[i] != ' ' && len < 256) {
            unsigned char c = (unsigned char)text[i++];
            if (c >= 'A' && c <= 'Z') c = (unsigned char)(c - 'A' + 'a');
            word[len++] = c;
        }
        while (i < n && text[i] != ' ') i++;   /* overlong word: rest ignored */
        if (len == 1) break;                     /* no more words */
        word[len++] = ' ';
        for (size_t t = 0; t + 3 <= len; t++)
            buckets[fnv1a3(word + t) % 128] += 32;
    }
}

/* ------------------------------------------------------------------------ */
/* Glue between the projections of a layer stack: RMS normalisation.         */
/* r[m][d] = v[m][d] / sqrt(mean_d v[m][d]^2 + eps), v = a (+ b when b is     */
/* given), in double.  The caller rounds r to bfloat16.                       */
/* ------------------------------------------------------------------------ */
void orc_rmsnorm(const float *a, const float *b, int64_t M, int64_t D, double eps, double *r)
{
    for (int64_t m = 0; m < M; m++) {
        double ss = 0.0;
        for (int64_t d = 0; d < D; d++) {
            double v = (double)a[m * D + d] + (b ? (double)b[m * D + d] : 0.0);
            ss += v * v;
        }
        double inv = 1.0 / sqrt(ss / (double)D + eps);
        for (int64_t d = 0; d < D; d++) {
            double v = (double)a[m * D + d] + (b ? (double)b[m * D + d] : 0.0);
            r[m * D + d] = v * inv;
        }
    }
}


/* ------------------------------------------------------------------------
 * Quantisers: float weights -> the packed formats' codes and FP16 scales.
 *
 * [BONSAI] "technical architecture highlights" fixes only the result (one
 * sign per weight, one FP16 scale per 128 weights).  Reading: the sign is
 * w >= 0 -> +1 (so -0.0 -> +1 and NaN -> -1), and the scale is the group's
 * mean |w|, the value of d that minimises sum (w - d s)^2 with s = sign(w).
 * [ACORN] "int4 quantisation quality: group quantisation": round-to-nearest
 * int4 with one scale per group along the input dimension (64 values here).
 * Reading: symmetric, d = max |w| / 7, q = w / d rounded to nearest with
 * ties to even, clamped to [-8, 7] (so -8 never occurs), q = 0 where d = 0
 * or w is NaN.
 * Every step is an IEEE double operation in a fixed order (sums with k
 * ascending), and FP16 rounding is to nearest, ties to even, with values at
 * or above 65504 saturating to 65504.
 * ---------------------------------------------------------------------- */

/* double -> FP16 bits: round to nearest, ties to even; |v| >= 65504 gives
 * +-65504 (the largest finite half); NaN gives 0. */
uint16_t orc_f64_to_f16(double v)
{
    if (v != v) return 0;
    const uint16_t sign = signbit(v) ? 0x8000u : 0u;
    double a = fabs(v);
    if (a >= 65504.0) return (uint16_t)(sign | 0x7BFFu);
    if (a == 0.0) return sign;
    /* the spacing of halves near a: 2^-24 below 2^-14, else 2^(e-10) */
    int e;
    frexp(a, &e);           /* a = f * 2^e, 0.5 <= f < 1: a in [2^(e-1), 2^e) */
    int ex = e - 1;         /* a in [2^ex, 2^(ex+1)) */
    if (ex < -14) ex = -14; /* subnormal range shares the spacing of 2^-14 */
    const double quantum = ldexp(1.0, ex - 10);
    const double r = rint(a / quantum) * quantum; /* a / quantum is exact; rint: ties to even */
    if (r >= 65504.0) return (uint16_t)(sign | 0x7BFFu);
    if (r < ldexp(1.0, -14)) return (uint16_t)(sign | (uint16_t)(r / ldexp(1.0, -24)));
    int er;
    const double fr = frexp(r, &er); /* r = fr * 2^er */
    const int exp16 = er - 1 + 15;
    const unsigned mant = (unsigned)((fr * 2.0 - 1.0) * 1024.0);
    return (uint16_t)(sign | ((unsigned)exp16 << 10) | mant);
}

int orc_q1_quantize(const float *w, int64_t rows, int64_t cols, int8_t *codes, uint16_t *scales)
{
    if (cols % 128 != 0) return 1;
    const int64_t G = cols / 128;
    for (int64_t n = 0; n < rows; ++n)
        for (int64_t g = 0; g < G; ++g) {
            double s = 0.0;
            for (int64_t k = g * 128; k < (g + 1) * 128; ++k) {
                const float v = w[n * cols + k];
                s += fabs((double)v);
                codes[n * cols + k] = (int8_t)(v >= 0.0f ? 1 : 0);
            }
            scales[n * G + g] = orc_f64_to_f16(s / 128.0);
        }
    return 0;
}

int orc_int4_quantize(const float *w, int64_t rows, int64_t cols, int8_t *codes, uint16_t *scales)
{
    if (cols % 64 != 0) return 1;
    const int64_t G = cols / 64;
    for (int64_t n = 0; n < rows; ++n)
        for (int64_t g = 0; g < G; ++g) {
            double amax = 0.0;
            for (int64_t k = g * 64; k < (g + 1) * 64; ++k) {
                const double a = fabs((double)w[n * cols + k]);
                if (a > amax) amax = a;
            }
            const uint16_t dh = orc_f64_to_f16(amax / 7.0);
            scales[n * G + g] = dh;
            const double d = orc_f16_to_f64(dh);
            for (int64_t k = g * 64; k < (g + 1) * 64; ++k) {
                const double v = (double)w[n * cols + k];
                double q = 0.0;
                if (d > 0.0 && v == v) {
                    q = rint(v / d);
                    if (q < -8.0) q = -8.0;
                    if (q > 7.0) q = 7.0;
                }
                codes[n * cols + k] = (int8_t)q;
            }
        }
    return 0;
}

/* ------------------------------------------------------------------------
 * Autoregressive reply loop [Z80]: architecture list (128 query + 128
 * context trigram buckets in, one output neuron per character of the
 * character set, ReLU between hidden layers) and feature list (autoregressive
 * generation, one character at a time).
 *
 * Reading (the page names the loop but not its state): the query buckets are
 * the trigram encoding of the user's text; the context buckets are the
 * trigram encoding of the reply generated so far in this turn (empty at the
 * start).  Each step feeds [query, context] through the network, takes the
 * argmax output, and maps it through the character set; the character-set
 * byte 0 marks the end of the reply.  A reply also ends after max_new
 * characters.  Every step re-encodes the whole reply from its text.
 *
 *   queries  [batch][qlen] bytes; a query ends at its first 0 byte or at qlen
 *   charset  [dims[n_layers]] bytes
 *   reply    [batch][max_new] bytes written; bytes past a reply's end are 0
 *   reply_len[batch]
 * dims[0] must be 256; max_new at most 250 (so no reply word is longer than
 * the encoder's 255-character word limit).  Returns 0, or -1 on bad sizes.
 * ---------------------------------------------------------------------- */
int orc_z80_generate(const uint8_t *const *packed_layers, const int32_t *dims, int n_layers,
                     const uint8_t *queries, int64_t batch, int64_t qlen, const uint8_t *charset,
                     int64_t max_new, uint8_t *reply, int32_t *reply_len)
{
    static char qtext[4097];
    static char rtext[251];
    int16_t x[256], logit[4096];
    int32_t am = 0;
    if (n_layers < 1 || dims[0] != 256 || qlen < 1 || qlen > 4096 || max_new < 0 || max_new > 250) return -1;
    for (int64_t b = 0; b < batch; b++) {
        memcpy(qtext, queries + b * qlen, (size_t)qlen);
        qtext[qlen] = 0;                        /* the query ends at its first 0 byte */
        int16_t qb[128];
        orc_trigram_encode(qtext, qb);
        int64_t t = 0;
        rtext[0] = 0;
        for (; t < max_new; t++) {
            orc_trigram_encode(rtext, x + 128);  /* context: the reply so far */
            memcpy(x, qb, sizeof qb);
            if (orc_q2_mlp_forward(packed_layers, dims, n_layers, x, 1, logit, &am, 0) != 0) return -1;
            const uint8_t ch = charset[am];
            if (ch == 0) break;                  /* end of reply */
            reply[b * max_new + t] = ch;
            rtext[t] = (char)ch;
            rtext[t + 1] = 0;
        }
        reply_len[b] = (int32_t)t;
        for (int64_t i = t; i < max_new; i++) reply[b * max_new + i] = 0;
    }
    return 0;
}

/* ------------------------------------------------------------------------
 * Ternary weights with an FP16 scale per 128 ("Bonsai-27B-gguf technical
 * white paper digest", section on intelligence density: the ternary model of
 * the same 27B network is 5.9 GB where the 1-bit Q1_0_g128 one is 3.79 GB).
 * The page gives no layout.  Reading: weights w in {-1, 0, +1}, one FP16
 * scale per 128 consecutive weights of a row (as Q1_0_g128), and the 128
 * trits t = w + 1 of a group packed five per byte in base 3 -- byte j < 25
 * holds k = 5j .. 5j+4 of the group as sum_i t_i 3^i, byte 25 holds
 * k = 125..127 as t_0 + 3 t_1 + 9 t_2 -- so a group is 26 bytes plus 2 of
 * scale: 1.75 bits per weight, and 3.79 GB x 1.75 / 1.125 = 5.90 GB.
 * Row n's packed bytes are [n][26 * K/128], its scales [n][K/128].
 * Decoding takes digit i of a byte b as floor(b / 3^i) mod 3 (i < 5, or
 * i < 3 in byte 25); the packer only writes bytes below 243 (below 27 in
 * byte 25).
 * ---------------------------------------------------------------------- */

static int64_t t3_byte_of(int64_t k, int *digit)
{
    int64_t g = k / 128, r = k % 128;
    *digit = (int)(r % 5);
    return 26 * g + r / 5;     /* r = 125..127 -> byte 25, digits 0..2 */
}

int orc_t3_pack(const int8_t *codes, int64_t rows, int64_t cols, uint8_t *packed)
{
    if (cols % 128 != 0) return -1;
    const int64_t rb = 26 * (cols / 128);
    for (int64_t r = 0; r < rows; r++) {
        for (int64_t j = 0; j < rb; j++) packed[r * rb + j] = 0;
        for (int64_t k = 0; k < cols; k++) {
            int8_t c = codes[r * cols + k];
            if (c < -1 || c > 1) return -1;
            int digit;
            int64_t j = t3_byte_of(k, &digit);
            int p = 1;
            for (int i = 0; i < digit; i++) p *= 3;
            packed[r * rb + j] = (uint8_t)(packed[r * rb + j] + (c + 1) * p);
        }
    }
    return 0;
}

/* Weight value (-1, 0 or +1) of column k of a packed row. */
static int t3_code(const uint8_t *row, int64_t k)
{
    int digit;
    int64_t j = t3_byte_of(k, &digit);
    int v = row[j];
    for (int i = 0; i < digit; i++) v /= 3;
    return v % 3 - 1;
}

int orc_t3_unpack(const uint8_t *packed, int64_t rows, int64_t cols, int8_t *codes)
{
    if (cols % 128 != 0) return -1;
    const int64_t rb = 26 * (cols / 128);
    for (int64_t r = 0; r < rows; r++)
        for (int64_t k = 0; k < cols; k++) codes[r * cols + k] = (int8_t)t3_code(packed + r * rb, k);
    return 0;
}

/* w[n][k] = code * d[n][k/128]. */
double orc_t3_weight(const uint8_t *packed, const uint16_t *scales, int64_t K, int64_t n, int64_t k)
{
    return (double)t3_code(packed + n * 26 * (K / 128), k) * orc_f16_to_f64(scales[n * (K / 128) + k / 128]);
}

int orc_t3_gemv(const uint8_t *packed, const uint16_t *scales, const uint16_t *x,
                int64_t M, int64_t N, int64_t K, double *y, double *absdot)
{
    if (K % 128 != 0) return -1;
    for (int64_t m = 0; m < M; m++) {
        for (int64_t n = 0; n < N; n++) {
            double acc = 0.0, aacc = 0.0;
            for (int64_t k = 0; k < K; k++) {
                double p = orc_t3_weight(packed, scales, K, n, k) * orc_bf16_to_f64(x[m * K + k]);
                acc += p;
                aacc += fabs(p);
            }
            y[m * N + n] = acc;
            if (absdot) absdot[m * N + n] = aacc;
        }
    }
    return 0;
}

int orc_t3_gemv_at(const uint8_t *packed, const uint16_t *scales, const uint16_t *x,
                   int64_t K, const int64_t *ms, const int64_t *ns, int64_t count,
                   double *y, double *absdot)
{
    if (K % 128 != 0) return -1;
    for (int64_t i = 0; i < count; i++) {
        double acc = 0.0, aacc = 0.0;
        for (int64_t k = 0; k < K; k++) {
            double p = orc_t3_weight(packed, scales, K, ns[i], k) * orc_bf16_to_f64(x[ms[i] * K + k]);
            acc += p;
            aacc += fabs(p);
        }
        y[i] = acc;
        if (absdot) absdot[i] = aacc;
    }
    return 0;
}

/*
 * nf4_oracle.c -- plain, slow CPU oracle for the QLoRA frozen-base linear layer.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path may call, link or load
 * this file: only the tests, the smoke check and the benchmark's cpu_baseline
 * leg and reference arm use it. It shares no code, header, table or helper with the CUDA library.
 *
 * What it computes, step by step, with the passage each step follows:
 *
 *  - NF4 table: the 16 values printed in "QLoRA paper notes" (tqpw.cn),
 *    section "Method / NormalFloat Quantization (NF4)". They are typed below as
 *    printed; each is an exact fp32 value.
 *  - Blocks of 64 consecutive weights of the row-major flattened W, absmax per
 *    block, weights normalised into [-1, 1] by that absmax: same section
 *    ("g64", weights normalised to [-1,1] before quantisation) and "How QLoRA
 *    works" (aivaro.ru) section 5 (one constant per 64 weights, stored fp32).
 *  - Nearest code: "QLoRA & PEFT family" (ai-reference-codex) section 3.1
 *    (remember which of the 16 values each weight is closest to). Ties go to
 *    the lower index; an all-zero block gets code 7 (the value 0).
 *  - Double quantisation: "QLoRA paper notes", section "Double Quantization"
 *    (block constants quantised to FP8 in groups of 256 after subtracting
 *    their mean, then symmetric quantisation). FP8 is E4M3 (finite variant,
 *    max 448); the group absmax maps to 448; one fp32 scale per group; one
 *    fp32 mean per tensor, the exact mean rounded once to fp32.
 *  - Dequantisation to the compute type and the LoRA sum h = W x + B A x:
 *    "Quantized LoRA (QLoRA) and 4-bit training" (apxml.com), equations
 *    h = Wx + BAx and h = dequant(W_NF4) x + BAx; shapes W (d x k),
 *    B (d x r), A (r x k) from "How QLoRA works" section 2; the LoRA branch is
 *    scaled by alpha/r (lora_alpha is the scaling factor, LoRA/QLoRA talk
 *    summary, "QLoRA ... practice guide").
 *  - Input gradient through the frozen, dequantised base: "How QLoRA works"
 *    section 7 (the 4-bit weights are dequantised on the fly to compute
 *    gradients and are not updated).
 *  - Gradients of the adapter weights A and B, the only trained parameters:
 *    "How QLoRA works" sections 2 (W frozen; B and A trained) and 7; they
 *    are the derivatives of h = W'x + s B (A x) with respect to B and A.
 *  - Merging the adapter into a 16-bit weight, W' + s B A (the weight cannot
 *    stay NF4 once merged): "QLoRA & PEFT family" section 3.6
 *    (merge_and_unload) and "QLoRA paper notes", Introduction.
 *  - LoRA dropout on the adapter's input (training): "QLoRA & PEFT family"
 *    section 3.4 (dropout 0.05-0.1) and the lora_dropout setting of the
 *    configuration in "How does QLoRA work for training?". The pages give the
 *    rate only; the reading taken: inverted dropout of x on the adapter branch
 *    only (the base path sees x), element (m, k) of x kept when the 32-bit
 *    output of a counter-based generator is >= floor(p 2^32), kept elements
 *    scaled by 1 / (1 - p); the generator is Philox4x32-10 (Salmon, Moraes,
 *    Dror and Shaw, "Parallel random numbers: as easy as 1, 2, 3", SC 2011),
 *    written here from that definition.
 *  - The two other settings of the 4-bit load: the quant type (NF4 or the
 *    standard 4-bit float; "Quantized LoRA (QLoRA) and 4-bit training", the
 *    four configuration knobs, and the bnb_4bit_quant_type setting of "How
 *    does QLoRA work for training?" section 6; NF4 measured better than FP4 in
 *    "QLoRA paper notes", Experiments) and double quantisation on or off (the
 *    same knobs; without it the block constants stay fp32, 0.5 bit per
 *    parameter in "QLoRA & PEFT family" section 3.3). The pages do not define
 *    the 4-bit float; the reading taken: E2M1 (sign, two exponent bits with
 *    bias 1, one mantissa bit, no infinities or NaN), magnitudes 0, 0.5, 1,
 *    1.5, 2, 3, 4, 6, normalised onto [-1, 1] like NF4 by the largest, 6, and
 *    rounded to fp32; code = sign bit (bit 3) and magnitude index (bits 0-2),
 *    so code 8 is -0. Codes are chosen, as for NF4, as the nearest table
 *    value to w / c with ties to the lower code index (so -0 never occurs and
 *    ties go toward zero); an all-zero block gets the lowest code of value 0.
 *    Without double quantisation the block constant is the exact absmax c_b.
 *
 * All sums of the linear layer are taken in fp64 in plain loop order.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define OR_BLOCK 64
#define OR_GROUP 256
#define OR_E4M3_MAX 448.0f

/* The NF4 code values exactly as printed on the page (ascending). */
static const double OR_NF4[16] = {
    -1.0,
    -0.6961928009986877,
    -0.5250730514526367,
    -0.39491748809814453,
    -0.28444138169288635,
    -0.18477343022823334,
    -0.09105003625154495,
    0.0,
    0.07958029955625534,
    0.16093020141124725,
    0.24611230194568634,
    0.33791524171829224,
    0.44070982933044434,
    0.5626170039176941,
    0.7229568362236023,
    1.0,
};

/* The 4-bit float (E2M1) values in code order: codes 0-7 are +m/6 for the
 * magnitudes m = 0, 0.5, 1, 1.5, 2, 3, 4, 6; codes 8-15 are their negatives
 * (code 8 is -0). Each is the fp32 value nearest to m/6. */
#define OR_E2M1(m) ((double)(float)((m) / 6.0))
static const double OR_FP4[16] = {
    OR_E2M1(0.0),  OR_E2M1(0.5),  OR_E2M1(1.0),  OR_E2M1(1.5),  OR_E2M1(2.0),  OR_E2M1(3.0),
    OR_E2M1(4.0),  OR_E2M1(6.0),  -OR_E2M1(0.0), -OR_E2M1(0.5), -OR_E2M1(1.0), -OR_E2M1(1.5),
    -OR_E2M1(2.0), -OR_E2M1(3.0), -OR_E2M1(4.0), -OR_E2M1(6.0),
};

#define OR_QT_NF4 0
#define OR_QT_FP4 1

static const double *table_of(int qtype) { return qtype == OR_QT_FP4 ? OR_FP4 : OR_NF4; }

/* A quantised weight: codes, the quant type's table, and its block constants,
 * either double quantised (q, sigma, mu) or fp32 (absmax). */
typedef struct {
    int qtype; /* OR_QT_NF4 or OR_QT_FP4 */
    int dq;    /* 1: q, sigma, mu; 0: absmax */
    const uint8_t *codes;
    const uint8_t *q;
    const float *sigma;
    float mu;
    const float *absmax;
} or_weight;

/* ------------------------------------------------------------------ scalars */

void or_nf4_table(double *out16) {
    for (int i = 0; i < 16; ++i) out16[i] = OR_NF4[i];
}

void or_4bit_table(int qtype, double *out16) {
    const double *T = table_of(qtype);
    for (int i = 0; i < 16; ++i) out16[i] = T[i];
}

int or_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

static float bf16_bits_to_float(uint16_t b) {
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* fp32 -> bf16, round to nearest, ties to even (finite inputs). */
uint16_t or_f32_to_bf16(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7f800000u) == 0x7f800000u) return (uint16_t)(u >> 16); /* inf/nan: truncate */
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7fffu + lsb;
    return (uint16_t)(u >> 16);
}

/* E4M3 (finite variant): 1 sign, 4 exponent (bias 7), 3 mantissa bits.
 * 0x7f / 0xff are NaN; the largest finite magnitude is 448 (0x7e). */
double or_e4m3_decode(uint8_t v) {
    int s = v >> 7, e = (v >> 3) & 15, m = v & 7;
    double mag;
    if (e == 15 && m == 7) return NAN;
    if (e == 0)
        mag = ldexp((double)m, -9);
    else
        mag = ldexp(1.0 + m / 8.0, e - 7);
    return s ? -mag : mag;
}

/* fp32 -> E4M3 by exhaustive search over the 127 finite magnitudes: nearest
 * value, ties to the even code, magnitudes above 448 saturate to 448, the sign
 * is kept (a negative value that rounds to zero gives 0x80). */
uint8_t or_e4m3_encode(float f) {
    if (f != f) return 0x7f;
    uint8_t sign = (f < 0.0f || (f == 0.0f && signbit(f))) ? 0x80 : 0x00;
    double a = fabs((double)f);
    if (a >= 448.0) return sign | 0x7e;
    int best = 0;
    double best_err = a; /* code 0 is +0 */
    for (int c = 1; c <= 0x7e; ++c) {
        double err = fabs(or_e4m3_decode((uint8_t)c) - a);
        if (err < best_err || (err == best_err && (c & 1) == 0 && (best & 1) == 1)) {
            best = c;
            best_err = err;
        }
    }
    return sign | (uint8_t)best;
}

/* ------------------------------------------------------- exact tensor mean */

/* 320-bit unsigned fixed-point accumulator; unit = 2^-133 (the smallest
 * positive bf16 subnormal), so every bf16 absmax is an integer in it. */
typedef struct { uint64_t limb[5]; } or_big;

static void big_add_shifted(or_big *acc, uint64_t m, int pos) {
    /* acc += m << pos, m < 2^9 */
    int li = pos / 64, sh = pos % 64;
    unsigned __int128 v = ((unsigned __int128)m) << sh;
    uint64_t carry = 0;
    for (int i = li; i < 5; ++i) {
        unsigned __int128 add = (i == li) ? (uint64_t)v : (i == li + 1 ? (uint64_t)(v >> 64) : 0);
        unsigned __int128 s = (unsigned __int128)acc->limb[i] + add + carry;
        acc->limb[i] = (uint64_t)s;
        carry = (uint64_t)(s >> 64);
    }
}

static int big_bitlen(const or_big *a) {
    for (int i = 4; i >= 0; --i)
        if (a->limb[i]) return i * 64 + (64 - __builtin_clzll(a->limb[i]));
    return 0;
}

static int big_bit(const or_big *a, int pos) {
    if (pos < 0 || pos >= 320) return 0;
    return (int)((a->limb[pos / 64] >> (pos % 64)) & 1u);
}

/* Correctly rounded fp32 of (S * 2^-133) / n, S the big integer. */
static float big_div_round_f32(const or_big *S, uint64_t n) {
    const int W = 100;
    int bl = big_bitlen(S);
    if (bl == 0 || n == 0) return 0.0f;
    int sh = bl - W;
    unsigned __int128 top = 0;
    int sticky0 = 0;
    for (int b = W - 1; b >= 0; --b) {
        top = (top << 1) | (unsigned __int128)big_bit(S, b + sh);
    }
    for (int b = 0; b < sh; ++b)
        if (big_bit(S, b)) { sticky0 = 1; break; }
    unsigned __int128 Q = top / n, R = top % n;
    int rem_nz = (R != 0) || sticky0;
    int e0 = sh - 133; /* value = (Q + frac) * 2^e0 */
    int qb = 0;
    for (unsigned __int128 t = Q; t; t >>= 1) ++qb;
    int e_lead = qb - 1 + e0;
    int lsb_exp = e_lead - 23;
    if (lsb_exp < -149) lsb_exp = -149;
    int s2 = lsb_exp - e0;
    unsigned __int128 mant = (s2 >= 128) ? 0 : (Q >> s2);
    int rbit = (s2 - 1 >= 0 && s2 - 1 < 128) ? (int)((Q >> (s2 - 1)) & 1) : 0;
    int sticky = rem_nz;
    for (int b = 0; b < s2 - 1 && b < 128; ++b)
        if ((Q >> b) & 1) { sticky = 1; break; }
    if (rbit && (sticky || (mant & 1))) mant += 1;
    return (float)ldexp((double)(uint64_t)mant, lsb_exp);
}

/* mu = fl32( (sum of the nb fp32 block absmaxes, exactly) / nb ).
 * Each absmax must be an exactly representable bf16 value (it is the absolute
 * value of a bf16 weight). */
float or_exact_mean_f32(const float *c, int64_t nb) {
    or_big S;
    memset(&S, 0, sizeof S);
    for (int64_t b = 0; b < nb; ++b) {
        uint32_t u;
        memcpy(&u, &c[b], 4);
        u &= 0x7fffffffu;
        uint32_t E = u >> 23, frac7 = (u >> 16) & 0x7f;
        if (E == 0) {
            big_add_shifted(&S, frac7, 0);
        } else {
            big_add_shifted(&S, 128u + frac7, (int)E - 1);
        }
    }
    return big_div_round_f32(&S, (uint64_t)nb);
}

/* ------------------------------------------------------------- quantiser */

static int nearest_code(const double *T, float x) {
    int best = 0;
    double best_err = fabs((double)x - T[0]);
    for (int i = 1; i < 16; ++i) {
        double err = fabs((double)x - T[i]);
        if (err < best_err) { /* strict: ties keep the lower index */
            best = i;
            best_err = err;
        }
    }
    return best;
}

/* Code of one bf16 weight w in a block with absmax c under quant type qtype:
 * the nearest value to fl32(w / c); an all-zero block takes the lowest code of
 * the value 0 (7 for NF4, 0 for the 4-bit float). Exposed for tests. */
int or_4bit_code(int qtype, float w, float c) {
    const double *T = table_of(qtype);
    if (c == 0.0f) return nearest_code(T, 0.0f);
    float x = w / c;
    return nearest_code(T, x);
}

int or_nf4_code(float w, float c) { return or_4bit_code(OR_QT_NF4, w, c); }

int64_t or_num_blocks(int64_t n, int64_t k) { return n * k / OR_BLOCK; }
int64_t or_num_groups(int64_t n, int64_t k) { return (or_num_blocks(n, k) + OR_GROUP - 1) / OR_GROUP; }

/* W: n x k bf16 bits, row-major; qtype OR_QT_NF4 or OR_QT_FP4. Outputs: codes
 * (n*k/2 bytes, element e in the low nibble of byte e/2 when e is even, high
 * nibble when odd); with dq: q (nb bytes E4M3), sigma (ng floats), mu (1 float);
 * absmax (nb floats): required without dq, may be NULL with it. Returns 0, or
 * -1 when k is not a multiple of 64. */
int or_quantize4(int qtype, int dq, const uint16_t *W, int64_t n, int64_t k, uint8_t *codes, uint8_t *q,
                 float *sigma, float *mu, float *absmax) {
    if (k % OR_BLOCK != 0 || n < 0 || k < 0) return -1;
    int64_t nb = or_num_blocks(n, k), ng = or_num_groups(n, k);
    float *c = (float *)malloc(sizeof(float) * (size_t)(nb > 0 ? nb : 1));
    if (!c) return -2;

#pragma omp parallel for schedule(static)
    for (int64_t b = 0; b < nb; ++b) {
        const uint16_t *w = W + b * OR_BLOCK;
        float m = 0.0f;
        for (int i = 0; i < OR_BLOCK; ++i) {
            float a = fabsf(bf16_bits_to_float(w[i]));
            if (a > m) m = a;
        }
        c[b] = m;
        for (int i = 0; i < OR_BLOCK; i += 2) {
            int lo = or_4bit_code(qtype, bf16_bits_to_float(w[i]), m);
            int hi = or_4bit_code(qtype, bf16_bits_to_float(w[i + 1]), m);
            codes[(b * OR_BLOCK + i) / 2] = (uint8_t)(lo | (hi << 4));
        }
    }
    if (!dq) {
        memcpy(absmax, c, sizeof(float) * (size_t)nb);
        free(c);
        return 0;
    }

    float m_all = or_exact_mean_f32(c, nb);
    *mu = m_all;

#pragma omp parallel for schedule(static)
    for (int64_t g = 0; g < ng; ++g) {
        int64_t b0 = g * OR_GROUP, b1 = b0 + OR_GROUP < nb ? b0 + OR_GROUP : nb;
        float S = 0.0f;
        for (int64_t b = b0; b < b1; ++b) {
            float d = c[b] - m_all;
            float a = fabsf(d);
            if (a > S) S = a;
        }
        float sg = S / OR_E4M3_MAX;
        sigma[g] = sg;
        for (int64_t b = b0; b < b1; ++b) {
            float d = c[b] - m_all;
            q[b] = (sg == 0.0f) ? (uint8_t)0 : or_e4m3_encode(d / sg);
        }
    }
    if (absmax) memcpy(absmax, c, sizeof(float) * (size_t)nb);
    free(c);
    return 0;
}

int or_nf4_quantize(const uint16_t *W, int64_t n, int64_t k, uint8_t *codes, uint8_t *q,
                    float *sigma, float *mu, float *absmax) {
    return or_quantize4(OR_QT_NF4, 1, W, n, k, codes, q, sigma, mu, absmax);
}

/* ---------------------------------------------------------- dequantiser */

/* c'_b = fma(decode(q_b), sigma_g, mu), one rounding, fp32. */
float or_block_constant(uint8_t qb, float sg, float mu) {
    return fmaf((float)or_e4m3_decode(qb), sg, mu);
}

/* The block constants the dequantiser multiplies by: c'_b with double
 * quantisation, else the stored fp32 absmax c_b itself. */
static void block_constants(const or_weight *w, int64_t nb, float *cp) {
    if (!w->dq) {
        memcpy(cp, w->absmax, sizeof(float) * (size_t)nb);
        return;
    }
#pragma omp parallel for schedule(static)
    for (int64_t b = 0; b < nb; ++b) cp[b] = or_block_constant(w->q[b], w->sigma[b / OR_GROUP], w->mu);
}

static int code_at(const uint8_t *codes, int64_t e) {
    uint8_t byte = codes[e / 2];
    return (e & 1) ? (byte >> 4) : (byte & 15);
}

/* Dequantise into bf16: bf16_rn( fl32( T32[code] * c'_b ) ). */
void or_dequant_bf16(const or_weight *w, int64_t n, int64_t k, uint16_t *out) {
    int64_t nb = or_num_blocks(n, k);
    const double *T = table_of(w->qtype);
    float *cp = (float *)malloc(sizeof(float) * (size_t)(nb > 0 ? nb : 1));
    block_constants(w, nb, cp);
#pragma omp parallel for schedule(static)
    for (int64_t e = 0; e < n * k; ++e) {
        float t = (float)T[code_at(w->codes, e)];
        float v = t * cp[e / OR_BLOCK];
        out[e] = or_f32_to_bf16(v);
    }
    free(cp);
}

/* Dequantise into fp64 without rounding: T[code] * c'_b. */
void or_dequant_f64(const or_weight *w, int64_t n, int64_t k, double *out) {
    int64_t nb = or_num_blocks(n, k);
    const double *T = table_of(w->qtype);
    float *cp = (float *)malloc(sizeof(float) * (size_t)(nb > 0 ? nb : 1));
    block_constants(w, nb, cp);
#pragma omp parallel for schedule(static)
    for (int64_t e = 0; e < n * k; ++e) out[e] = T[code_at(w->codes, e)] * (double)cp[e / OR_BLOCK];
    free(cp);
}

/* ---------------------------------------------------------------- dropout */

/* Philox4x32 with 10 rounds: each round multiplies words 0 and 2 of the counter
 * by the two round multipliers, mixes the high and low halves of the products
 * with words 1 and 3 and the key, and the key is bumped by the two Weyl
 * constants between rounds. */
void or_philox4x32_10(const uint32_t ctr_in[4], const uint32_t key_in[2], uint32_t out[4]) {
    const uint32_t M0 = 0xD2511F53u, M1 = 0xCD9E8D57u, W0 = 0x9E3779B9u, W1 = 0xBB67AE85u;
    uint32_t c0 = ctr_in[0], c1 = ctr_in[1], c2 = ctr_in[2], c3 = ctr_in[3];
    uint32_t k0 = key_in[0], k1 = key_in[1];
    for (int round = 0; round < 10; ++round) {
        if (round > 0) {
            k0 += W0;
            k1 += W1;
        }
        const uint64_t p0 = (uint64_t)M0 * c0, p1 = (uint64_t)M1 * c2;
        const uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
        const uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
        const uint32_t n0 = hi1 ^ c1 ^ k0, n2 = hi0 ^ c3 ^ k1;
        c0 = n0;
        c1 = lo1;
        c2 = n2;
        c3 = lo0;
    }
    out[0] = c0;
    out[1] = c1;
    out[2] = c2;
    out[3] = c3;
}

/* Keep threshold of rate p (0 <= p < 1): floor(p * 2^32), computed in fp64. */
uint32_t or_dropout_threshold(double p) {
    if (!(p > 0.0)) return 0u;
    return (uint32_t)floor(p * 4294967296.0);
}

/* 32-bit generator output for element index e (already offset): word e % 4 of
 * Philox4x32-10 at counter (e / 4 low word, e / 4 high word, 0, 0), key (seed
 * low word, seed high word). */
uint32_t or_dropout_bits(uint64_t seed, uint64_t e) {
    const uint64_t blk = e >> 2;
    const uint32_t ctr[4] = {(uint32_t)blk, (uint32_t)(blk >> 32), 0u, 0u};
    const uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
    uint32_t out[4];
    or_philox4x32_10(ctr, key, out);
    return out[e & 3];
}

/* 1 when element (m, kk) of the M x k activation survives dropout. */
static int keep_at(uint64_t seed, uint64_t offset, uint32_t thr, int64_t m, int64_t k, int64_t kk) {
    if (thr == 0u) return 1;
    return or_dropout_bits(seed, offset + (uint64_t)(m * k + kk)) >= thr;
}

/* ------------------------------------------------------ linear layer */

/* h[i, j] for the selected token rows rows[i] (i < nsel) of x (m x k):
 *   h = sum_k W'[j,k] x[row,k] + s * sum_r B[j,r] * (sum_k A[r,k] x[row,k])
 * with W' = T[code] * c' in fp64, s = fl32(alpha / r). A (r x k) and B (n x r)
 * may be NULL when r == 0. With dropout (p_drop > 0) the adapter's x[row,k] is
 * kept or zeroed by keep_at(seed, offset, row, k) and s becomes s / (1 - p).
 * Output h is nsel x n, fp64. */
void or_qlora_fwd(const or_weight *w, int64_t n, int64_t k, const uint16_t *x, const int64_t *rows,
                  int64_t nsel, const uint16_t *A, const uint16_t *B, int r, float alpha, double p_drop,
                  uint64_t seed, uint64_t offset, double *h) {
    int64_t nb = or_num_blocks(n, k);
    const double *T = table_of(w->qtype);
    const uint8_t *codes = w->codes;
    float *cp = (float *)malloc(sizeof(float) * (size_t)(nb > 0 ? nb : 1));
    block_constants(w, nb, cp);
    double s = (r > 0) ? (double)(alpha / (float)r) : 0.0;
    const uint32_t thr = or_dropout_threshold(p_drop);
    if (thr != 0u) s = s / (1.0 - p_drop);
    double *xs = (double *)malloc(sizeof(double) * (size_t)(nsel * k + 1));
    double *t = (double *)malloc(sizeof(double) * (size_t)(nsel * (r > 0 ? r : 1) + 1));
    for (int64_t i = 0; i < nsel; ++i)
        for (int64_t kk = 0; kk < k; ++kk) xs[i * k + kk] = bf16_bits_to_float(x[rows[i] * k + kk]);
    /* t[i, rr] = sum_k A[rr, k] x[row_i, k] keep(row_i, k) (the dropout scale is in s) */
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < nsel; ++i)
        for (int rr = 0; rr < r; ++rr) {
            double acc = 0.0;
            for (int64_t kk = 0; kk < k; ++kk)
                if (keep_at(seed, offset, thr, rows[i], k, kk))
                    acc += bf16_bits_to_float(A[rr * k + kk]) * xs[i * k + kk];
            t[i * r + rr] = acc;
        }
#pragma omp parallel
    {
        double *wrow = (double *)malloc(sizeof(double) * (size_t)(k + 1));
#pragma omp for schedule(static)
        for (int64_t j = 0; j < n; ++j) {
            for (int64_t kk = 0; kk < k; ++kk)
                wrow[kk] = T[code_at(codes, j * k + kk)] * (double)cp[(j * k + kk) / OR_BLOCK];
            for (int64_t i = 0; i < nsel; ++i) {
                double acc = 0.0;
                for (int64_t kk = 0; kk < k; ++kk) acc += wrow[kk] * xs[i * k + kk];
                double lora = 0.0;
                for (int rr = 0; rr < r; ++rr) lora += bf16_bits_to_float(B[j * r + rr]) * t[i * r + rr];
                h[i * n + j] = acc + s * lora;
            }
        }
        free(wrow);
    }
    free(t);
    free(xs);
    free(cp);
}

/* grad_x[i, kk] for the selected rows of grad_h (m x n):
 *   grad_x = sum_j grad_h[row,j] W'[j,kk] + s * sum_r A[r,kk] * (sum_j grad_h[row,j] B[j,r])
 * With dropout the adapter term of (row, kk) is zeroed where the forward's mask
 * zeroed x[row, kk], and s becomes s / (1 - p). Output nsel x k, fp64. */
void or_qlora_bwd_x(const or_weight *w, int64_t n, int64_t k, const uint16_t *gh, const int64_t *rows,
                    int64_t nsel, const uint16_t *A, const uint16_t *B, int r, float alpha, double p_drop,
                    uint64_t seed, uint64_t offset, double *gx) {
    int64_t nb = or_num_blocks(n, k);
    const double *T = table_of(w->qtype);
    const uint8_t *codes = w->codes;
    float *cp = (float *)malloc(sizeof(float) * (size_t)(nb > 0 ? nb : 1));
    block_constants(w, nb, cp);
    double s = (r > 0) ? (double)(alpha / (float)r) : 0.0;
    const uint32_t thr = or_dropout_threshold(p_drop);
    if (thr != 0u) s = s / (1.0 - p_drop);
    double *gs = (double *)malloc(sizeof(double) * (size_t)(nsel * n + 1));
    double *u = (double *)malloc(sizeof(double) * (size_t)(nsel * (r > 0 ? r : 1) + 1));
    for (int64_t i = 0; i < nsel; ++i)
        for (int64_t j = 0; j < n; ++j) gs[i * n + j] = bf16_bits_to_float(gh[rows[i] * n + j]);
    /* u[i, rr] = sum_j grad_h[row_i, j] B[j, rr] */
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < nsel; ++i)
        for (int rr = 0; rr < r; ++rr) {
            double acc = 0.0;
            for (int64_t j = 0; j < n; ++j) acc += gs[i * n + j] * bf16_bits_to_float(B[j * r + rr]);
            u[i * r + rr] = acc;
        }
    /* Each thread owns a slice of columns kk and walks all rows j. */
    const int64_t CH = 256;
    int64_t nch = (k + CH - 1) / CH;
#pragma omp parallel
    {
        double *acc = (double *)malloc(sizeof(double) * (size_t)(nsel * CH + 1));
        double *wseg = (double *)malloc(sizeof(double) * (size_t)(CH + 1));
#pragma omp for schedule(dynamic, 1)
        for (int64_t ch = 0; ch < nch; ++ch) {
            int64_t k0 = ch * CH, k1 = k0 + CH < k ? k0 + CH : k;
            int64_t w = k1 - k0;
            memset(acc, 0, sizeof(double) * (size_t)(nsel * CH));
            for (int64_t j = 0; j < n; ++j) {
                for (int64_t kk = k0; kk < k1; ++kk)
                    wseg[kk - k0] = T[code_at(codes, j * k + kk)] * (double)cp[(j * k + kk) / OR_BLOCK];
                for (int64_t i = 0; i < nsel; ++i) {
                    double g = gs[i * n + j];
                    for (int64_t kk = 0; kk < w; ++kk) acc[i * CH + kk] += g * wseg[kk];
                }
            }
            for (int64_t i = 0; i < nsel; ++i)
                for (int64_t kk = k0; kk < k1; ++kk) {
                    double lora = 0.0;
                    for (int rr = 0; rr < r; ++rr) lora += bf16_bits_to_float(A[rr * k + kk]) * u[i * r + rr];
                    if (!keep_at(seed, offset, thr, rows[i], k, kk)) lora = 0.0;
                    gx[i * k + kk] = acc[i * CH + (kk - k0)] + s * lora;
                }
        }
        free(wseg);
        free(acc);
    }
    free(u);
    free(gs);
    free(cp);
}

/* ------------------------------------------------- adapter weight gradients */

/* Gradients of the adapter for M token rows (all of them):
 *   t[m, j]      = sum_k A[j,k] x[m,k]          (the unscaled down-projection)
 *   grad_B[n, j] = s * sum_m grad_h[m,n] t[m,j]
 *   u[m, j]      = sum_n grad_h[m,n] B[n,j]
 *   grad_A[j, k] = s * sum_m u[m,j] x[m,k]
 * with s = fl32(alpha / r); with dropout x is the forward's masked x and s
 * becomes s / (1 - p). x is M x k, grad_h M x n, A r x k, B n x r (bf16
 * bits); grad_A (r x k) and grad_B (n x r) are fp64, all sums in fp64 in plain
 * loop order. */
void or_lora_grads(const uint16_t *x, const uint16_t *gh, int64_t M, int64_t n, int64_t k,
                   const uint16_t *A, const uint16_t *B, int r, float alpha, double p_drop, uint64_t seed,
                   uint64_t offset, double *grad_A, double *grad_B) {
    double s = (r > 0) ? (double)(alpha / (float)r) : 0.0;
    const uint32_t thr = or_dropout_threshold(p_drop);
    if (thr != 0u) s = s / (1.0 - p_drop);
    double *t = (double *)malloc(sizeof(double) * (size_t)(M * (r > 0 ? r : 1) + 1));
    double *u = (double *)malloc(sizeof(double) * (size_t)(M * (r > 0 ? r : 1) + 1));
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int j = 0; j < r; ++j) {
            double ta = 0.0, ua = 0.0;
            for (int64_t kk = 0; kk < k; ++kk)
                if (keep_at(seed, offset, thr, m, k, kk))
                    ta += bf16_bits_to_float(A[j * k + kk]) * (double)bf16_bits_to_float(x[m * k + kk]);
            for (int64_t nn = 0; nn < n; ++nn)
                ua += bf16_bits_to_float(gh[m * n + nn]) * (double)bf16_bits_to_float(B[nn * r + j]);
            t[m * r + j] = ta;
            u[m * r + j] = ua;
        }
#pragma omp parallel for schedule(static)
    for (int64_t nn = 0; nn < n; ++nn)
        for (int j = 0; j < r; ++j) {
            double acc = 0.0;
            for (int64_t m = 0; m < M; ++m) acc += bf16_bits_to_float(gh[m * n + nn]) * t[m * r + j];
            grad_B[nn * r + j] = s * acc;
        }
#pragma omp parallel for schedule(static)
    for (int j = 0; j < r; ++j)
        for (int64_t kk = 0; kk < k; ++kk) {
            double acc = 0.0;
            for (int64_t m = 0; m < M; ++m)
                if (keep_at(seed, offset, thr, m, k, kk)) acc += u[m * r + j] * bf16_bits_to_float(x[m * k + kk]);
            grad_A[(int64_t)j * k + kk] = s * acc;
        }
    free(u);
    free(t);
}

/* ------------------------------------------------------------------ merge */

/* fp64 -> bf16, round to nearest, ties to even, in one step (no fp32 on the way);
 * finite inputs, overflow to infinity, bf16 subnormals kept. */
uint16_t or_f64_to_bf16(double v) {
    uint16_t sign = (v < 0.0 || (v == 0.0 && signbit(v))) ? 0x8000 : 0x0000;
    double a = fabs(v);
    if (a == 0.0) return sign;
    /* a = f * 2^e with f in [1, 2) */
    int e;
    double f = frexp(a, &e) * 2.0;
    e -= 1;
    if (e < -126) { /* subnormal range of bf16: units of 2^-133 */
        double units = ldexp(a, 133);
        double fl = floor(units), rem = units - fl;
        uint32_t m = (uint32_t)fl;
        if (rem > 0.5 || (rem == 0.5 && (m & 1u))) m += 1;
        return (uint16_t)(sign | m); /* m == 128 becomes the smallest normal */
    }
    double scaled = ldexp(f, 7); /* in [128, 256) */
    double fl = floor(scaled), rem = scaled - fl;
    uint32_t m = (uint32_t)fl;
    if (rem > 0.5 || (rem == 0.5 && (m & 1u))) m += 1;
    if (m == 256) {
        m = 128;
        e += 1;
    }
    if (e > 127) return (uint16_t)(sign | 0x7f80);
    return (uint16_t)(sign | ((uint32_t)(e + 127) << 7) | (m - 128));
}

/* W_merged[n, k] = bf16_rn( W'32[n,k] + s * sum_j B[n,j] A[j,k] ):
 * W'32 = fl32(T[code] * c'_b), the dequantised weight as or_nf4_dequant rounds it to
 * fp32, the adapter sum exact in fp64 (r products of bf16 values), one rounding of
 * the fp64 total to bf16. A (r x k), B (n x r) bf16 bits; r == 0 gives the plain
 * dequantised weight. */
void or_merge_bf16(const or_weight *wq, int64_t n, int64_t k, const uint16_t *A, const uint16_t *B, int r,
                   float alpha, uint16_t *out) {
    int64_t nb = or_num_blocks(n, k);
    const double *T = table_of(wq->qtype);
    const uint8_t *codes = wq->codes;
    float *cp = (float *)malloc(sizeof(float) * (size_t)(nb > 0 ? nb : 1));
    block_constants(wq, nb, cp);
    double s = (r > 0) ? (double)(alpha / (float)r) : 0.0;
#pragma omp parallel for schedule(static)
    for (int64_t nn = 0; nn < n; ++nn)
        for (int64_t kk = 0; kk < k; ++kk) {
            int64_t e = nn * k + kk;
            float w = (float)T[code_at(codes, e)] * cp[e / OR_BLOCK];
            double ad = 0.0;
            for (int j = 0; j < r; ++j)
                ad += (double)bf16_bits_to_float(B[nn * r + j]) * (double)bf16_bits_to_float(A[(int64_t)j * k + kk]);
            out[e] = or_f64_to_bf16((double)w + s * ad);
        }
    free(cp);
}

/*
 * nf4_oracle.c -- plain, slow CPU oracle for NF4 quantization with double
 * quantization of the block constants.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference legs of bench.py may load this library.  It shares
 * no source, header, table or constant with the CUDA library.
 *
 * Built with  gcc -O2 -ffp-contract=off -fno-fast-math  so that every float
 * expression below is one IEEE-754 round-to-nearest-even operation.
 *
 * Every rule follows the pages (titles cited below) step by step:
 *   - codebook: quantiles of N(0,1), sampled uniformly in probability and
 *     normalized to [-1,1]            -- "从LoRA到QLoRA" §2.3;
 *                                       "QLoRA 原理精讲" §2.1 (核心机制)
 *   - blockwise absmax, 64 weights per block, normalize by the absmax, then
 *     nearest codebook entry         -- "QLoRA 原理精讲" §2.1 (示意代码)
 *   - double quantization: the per-block scale1 values are quantized to FP8
 *     in groups of 256 with one FP32 scale2 per group
 *                                     -- "QLoRA 原理精讲" §2.2 (核心机制, 流程图)
 *   - dequantize in reverse order: scale2 restores scale1, scale1 restores w
 *                                     -- "QLoRA 原理精讲" §2.2 (last paragraph)
 * Readings where the pages are silent are stated beside each function.
 *
 * Parity status: every function here is pinned by a -m "not gpu" test
 * (tests/test_oracle_*.py) against closed forms, invariants, an independent
 * library routine or exact rational brute force.  The choice of the 16 table
 * values themselves is a reading (the construction's numeric details are not
 * printed on the pages); the table is pinned by its defining invariants.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define ORC_BLOCK 64   /* weights per first-level block  ("QLoRA 原理精讲" §2.1, §2.2) */
#define ORC_GROUP 256  /* blocks per second-level group  ("QLoRA 原理精讲" §2.2) */

/* ------------------------------------------------------------------ */
/* bit helpers                                                          */
/* ------------------------------------------------------------------ */
static float f32_from_bits(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t bits_from_f32(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

/* bf16 is the upper half of an fp32 bit pattern: decoding is exact. */
double oracle_bf16_to_f64(uint16_t b) { return (double)f32_from_bits(((uint32_t)b) << 16); }

/* Round a real (given exactly as a double) to the nearest bf16, ties to the
 * even significand, written from the definition: find the two bf16 values
 * that bracket |x| and take the nearer one. bf16 = 1 sign, 8 exponent (bias
 * 127), 7 stored significand bits; subnormal spacing 2^-133; max finite
 * (2-2^-7)*2^127; anything at or above the midpoint to 2^128 becomes inf. */
uint16_t oracle_bf16_round(double x)
{
    if (isnan(x)) return 0x7FC0;
    uint16_t sign = signbit(x) ? 0x8000 : 0;
    double a = fabs(x);
    if (isinf(a)) return sign | 0x7F80;
    if (a == 0.0) return sign;
    double ulp;                       /* spacing of bf16 values around a */
    int e;
    frexp(a, &e);                     /* a = m * 2^e, m in [0.5,1) */
    if (e - 1 < -126) ulp = ldexp(1.0, -133);
    else              ulp = ldexp(1.0, (e - 1) - 7);
    double lo = floor(a / ulp) * ulp; /* exact: power-of-two scaling */
    double hi = lo + ulp;
    double dlo = a - lo, dhi = hi - a; /* exact in double */
    double r;
    if (dlo < dhi) r = lo;
    else if (dhi < dlo) r = hi;
    else {
        /* tie: the candidate whose last significand bit is 0 */
        double k = lo / ulp;          /* integer multiple count */
        r = (fmod(k, 2.0) == 0.0) ? lo : hi;
    }
    if (r >= ldexp(1.0, 128)) return sign | 0x7F80;
    float rf = (float)r;              /* exact: r is a bf16 value */
    return sign | (uint16_t)(bits_from_f32(rf) >> 16);
}

/* ------------------------------------------------------------------ */
/* FP8 E4M3 (OCP "E4M3FN": bias 7, no infinities, max 448, 0x7F = NaN)  */
/* The 8-bit format of the quantized scale1 is FP8 per "QLoRA 原理精讲" */
/* §2.2; the E4M3 variant, round-to-nearest-even and saturation to the */
/* largest finite value are readings (the pages do not say).           */
/* ------------------------------------------------------------------ */
double oracle_e4m3_decode(uint8_t c)
{
    int s = c >> 7, e = (c >> 3) & 0xF, m = c & 7;
    if (e == 15 && m == 7) return NAN;
    double v = (e == 0) ? ldexp((double)m, -9)            /* m/8 * 2^-6   */
                        : ldexp(8.0 + m, e - 10);         /* (1+m/8)*2^(e-7) */
    return s ? -v : v;
}

/* Encode by enumeration: the nearest of the 127 non-negative finite codes,
 * ties to the code with an even last bit; everything above 448 (and +inf)
 * saturates to 448; NaN -> 0x7F. Only non-negative inputs occur here
 * (scale1/scale2 >= 0); a negative input is encoded by symmetry. */
uint8_t oracle_e4m3_encode(float x)
{
    if (isnan(x)) return 0x7F;
    uint8_t sign = signbit(x) ? 0x80 : 0;
    double a = fabs((double)x);
    if (a >= 448.0) return sign | 0x7E;
    int best = 0;
    double bestd = INFINITY;
    for (int c = 0; c <= 0x7E; c++) {
        double d = fabs(a - oracle_e4m3_decode((uint8_t)c));
        if (d < bestd || (d == bestd && (c & 1) == 0)) { bestd = d; best = c; }
    }
    return sign | (uint8_t)best;
}

/* ------------------------------------------------------------------ */
/* NF4 codebook                                                         */
/* ------------------------------------------------------------------ */
static long double std_normal_cdf(long double z) { return 0.5L * erfcl(-z / sqrtl(2.0L)); }

/* Inverse of the standard normal CDF by bisection until the bracket stops
 * shrinking (extended precision). Slow and obviously monotone. */
static long double std_normal_quantile(long double p)
{
    long double lo = -40.0L, hi = 40.0L;
    for (int i = 0; i < 400; i++) {
        long double mid = 0.5L * (lo + hi);
        if (mid == lo || mid == hi) break;
        if (std_normal_cdf(mid) < p) lo = mid; else hi = mid;
    }
    return 0.5L * (lo + hi);
}

/* The 16 NF4 values (reading of "从LoRA到QLoRA" §2.3 and "QLoRA 原理精讲" §2.1):
 * quantiles of N(0,1) at probabilities spaced uniformly between delta and
 * 1/2 -- 8 on the positive side, 7 on the negative side -- plus an exact
 * zero, normalized by the largest magnitude to [-1, 1].  delta is the mean of
 * 1 - 1/(2*15) and 1 - 1/(2*16), the two end-probabilities of an equal-mass
 * split into 15 and 16 bins.  Computed in extended precision, rounded once to
 * fp32.  Output is ascending. */
void oracle_codebook(float codes[16])
{
    const long double delta = 0.5L * ((1.0L - 1.0L / 30.0L) + (1.0L - 1.0L / 32.0L));
    long double v[16];
    int n = 0;
    for (int i = 0; i < 8; i++)   /* probabilities delta, ..., toward 1/2 (exclusive) */
        v[n++] = std_normal_quantile(delta + (0.5L - delta) * (long double)i / 8.0L);
    v[n++] = 0.0L;
    for (int i = 0; i < 7; i++)
        v[n++] = -std_normal_quantile(delta + (0.5L - delta) * (long double)i / 7.0L);
    for (int i = 0; i < 16; i++)                  /* selection sort, ascending */
        for (int j = i + 1; j < 16; j++)
            if (v[j] < v[i]) { long double t = v[i]; v[i] = v[j]; v[j] = t; }
    long double mx = 0.0L;
    for (int i = 0; i < 16; i++) if (fabsl(v[i]) > mx) mx = fabsl(v[i]);
    for (int i = 0; i < 16; i++) codes[i] = (float)(v[i] / mx);
}

/* Nearest code to the exact real quotient w / absmax, ties to the lower
 * index ("lookup_nearest", "QLoRA 原理精讲" §2.1; the tie rule is a reading).
 * Since codes ascend, the nearest index is the number of midpoints that the
 * quotient exceeds.  w/absmax > mid  <=>  w > mid*absmax for absmax > 0, and
 * mid*absmax is exact in double (25-bit mid times 24-bit absmax), so every
 * comparison here is exact.  absmax == 0 (an all-zero block) gives the code
 * of 0.0. */
int oracle_nearest_code(const float codes[16], float w, float absmax)
{
    int zero_idx = 0;
    for (int i = 0; i < 16; i++) if (codes[i] == 0.0f) zero_idx = i;
    if (absmax == 0.0f) return zero_idx;
    int q = 0;
    for (int i = 0; i < 15; i++) {
        double mid = ((double)codes[i] + (double)codes[i + 1]) / 2.0;   /* exact */
        if ((double)w > mid * (double)absmax) q++;
    }
    return q;
}

/* ------------------------------------------------------------------ */
/* sizes                                                                */
/* ------------------------------------------------------------------ */
int64_t oracle_nblocks(int64_t numel) { return (numel + ORC_BLOCK - 1) / ORC_BLOCK; }
int64_t oracle_ngroups(int64_t numel) { return (oracle_nblocks(numel) + ORC_GROUP - 1) / ORC_GROUP; }
int64_t oracle_packed_bytes(int64_t numel) { return (numel + 1) / 2; }

/* ------------------------------------------------------------------ */
/* quantize + double quantization                                       */
/* ------------------------------------------------------------------ */
/* W: numel bf16 bit patterns, the weight flattened row-major (blocks run
 * over consecutive elements; the last block and last group may be short --
 * reading).  Outputs: packed[ceil(numel/2)] (element e in byte e/2, even e
 * in the low nibble, pad nibble 0 -- reading), c1q[nblocks] (E4M3 codes of
 * scale1/scale2), c2[ngroups] (fp32 scale2).  Returns 1 when W holds a NaN
 * or an infinity (outputs then unspecified), else 0. */
int oracle_quantize(const uint16_t* W, int64_t numel,
                    uint8_t* packed, uint8_t* c1q, float* c2)
{
    float codes[16];
    oracle_codebook(codes);
    int64_t nb = oracle_nblocks(numel), ng = oracle_ngroups(numel);
    int nonfinite = 0;

    for (int64_t g = 0; g < ng; g++) {
        int64_t b0 = g * ORC_GROUP, b1 = b0 + ORC_GROUP;
        if (b1 > nb) b1 = nb;
        /* first level: absmax of each block of 64 ("QLoRA 原理精讲" §2.1 step 1) */
        float absmax[ORC_GROUP];
        float gmax = 0.0f;
        for (int64_t b = b0; b < b1; b++) {
            float m = 0.0f;
            int64_t e0 = b * ORC_BLOCK, e1 = e0 + ORC_BLOCK;
            if (e1 > numel) e1 = numel;
            for (int64_t e = e0; e < e1; e++) {
                float w = (float)oracle_bf16_to_f64(W[e]);
                if (!isfinite(w)) nonfinite = 1;
                float a = fabsf(w);
                if (a > m) m = a;
            }
            absmax[b - b0] = m;
            if (m > gmax) gmax = m;
        }
        /* second level: scale2 maps the group's largest scale1 onto the
         * largest E4M3 value; scale1 is stored as E4M3(scale1 / scale2)
         * ("QLoRA 原理精讲" §2.2; the absmax-to-448 rule is a reading). */
        float s2 = gmax / 448.0f;
        c2[g] = s2;
        for (int64_t b = b0; b < b1; b++) {
            float m = absmax[b - b0];
            c1q[b] = (m == 0.0f) ? (uint8_t)0 : oracle_e4m3_encode(m / s2);
        }
        /* 4-bit codes: normalize by the block absmax, take the nearest code
         * ("QLoRA 原理精讲" §2.1 steps 2-3) */
        for (int64_t b = b0; b < b1; b++) {
            int64_t e0 = b * ORC_BLOCK, e1 = e0 + ORC_BLOCK;
            if (e1 > numel) e1 = numel;
            for (int64_t e = e0; e < e1; e++) {
                float w = (float)oracle_bf16_to_f64(W[e]);
                int q = oracle_nearest_code(codes, w, absmax[b - b0]);
                if ((e & 1) == 0) packed[e >> 1] = (uint8_t)q;
                else              packed[e >> 1] = (uint8_t)(packed[e >> 1] | (q << 4));
            }
        }
    }
    return nonfinite;
}

/* ------------------------------------------------------------------ */
/* double dequantization                                                */
/* ------------------------------------------------------------------ */
/* Reverse order ("QLoRA 原理精讲" §2.2): scale1' = fp32(E4M3(c1q) * scale2),
 * then w' = bf16(fp32(code[q] * scale1')): one fp32 multiply each, one final
 * rounding to the BF16 compute type ("从LoRA到QLoRA" §3.1). */
void oracle_dequant(const uint8_t* packed, const uint8_t* c1q, const float* c2,
                    int64_t numel, uint16_t* out)
{
    float codes[16];
    oracle_codebook(codes);
    for (int64_t e = 0; e < numel; e++) {
        int64_t b = e / ORC_BLOCK, g = b / ORC_GROUP;
        float s1 = (float)oracle_e4m3_decode(c1q[b]) * c2[g];
        int q = (e & 1) ? (packed[e >> 1] >> 4) : (packed[e >> 1] & 0xF);
        float v = codes[q] * s1;
        out[e] = oracle_bf16_round((double)v);
    }
}

/* Vector helpers for the Python side. */
void oracle_bf16_round_array(const double* x, int64_t n, uint16_t* out)
{
    for (int64_t i = 0; i < n; i++) out[i] = oracle_bf16_round(x[i]);
}
void oracle_bf16_decode_array(const uint16_t* b, int64_t n, double* out)
{
    for (int64_t i = 0; i < n; i++) out[i] = oracle_bf16_to_f64(b[i]);
}
void oracle_e4m3_encode_array(const float* x, int64_t n, uint8_t* out)
{
    for (int64_t i = 0; i < n; i++) out[i] = oracle_e4m3_encode(x[i]);
}
void oracle_classify_array(const float* w, const float* absmax, int64_t n, int32_t* q)
{
    float codes[16];
    oracle_codebook(codes);
    for (int64_t i = 0; i < n; i++) q[i] = oracle_nearest_code(codes, w[i], absmax[i]);
}

/* ================================================================== */
/* Format variants, the FP16 compute type                              */
/* ================================================================== */

/* Round a real (given exactly as a double) to the nearest IEEE binary16
 * value, ties to the even significand, written from the definition like
 * oracle_bf16_round: 1 sign, 5 exponent (bias 15), 10 stored significand
 * bits; subnormal spacing 2^-24; largest finite 65504; a value whose rounding
 * reaches 2^16 becomes inf.  FP16 is the compute type the pages name for
 * GPUs without BF16 ("QLoRA 原理精讲" §三 误区4). */
uint16_t oracle_f16_round(double x)
{
    if (isnan(x)) return 0x7E00;
    uint16_t sign = signbit(x) ? 0x8000 : 0;
    double a = fabs(x);
    if (isinf(a)) return sign | 0x7C00;
    if (a == 0.0) return sign;
    int e;
    frexp(a, &e);                     /* a = m * 2^e, m in [0.5,1) */
    double ulp = (e - 1 < -14) ? ldexp(1.0, -24) : ldexp(1.0, (e - 1) - 10);
    double lo = floor(a / ulp) * ulp, hi = lo + ulp;
    double dlo = a - lo, dhi = hi - a;
    double r;
    if (dlo < dhi) r = lo;
    else if (dhi < dlo) r = hi;
    else r = (fmod(lo / ulp, 2.0) == 0.0) ? lo : hi;
    if (r >= 65536.0) return sign | 0x7C00;
    /* encode r exactly */
    if (r < ldexp(1.0, -14)) return sign | (uint16_t)(r / ldexp(1.0, -24));      /* subnormal or 0 */
    frexp(r, &e);
    int E = e - 1;                                  /* r = 1.f * 2^E */
    uint16_t frac = (uint16_t)((r / ldexp(1.0, E) - 1.0) * 1024.0);
    return sign | (uint16_t)((E + 15) << 10) | frac;
}

double oracle_f16_to_f64(uint16_t h)
{
    int s = h >> 15, e = (h >> 10) & 0x1F, f = h & 0x3FF;
    double v;
    if (e == 31) v = f ? NAN : INFINITY;
    else if (e == 0) v = ldexp((double)f, -24);
    else v = ldexp(1.0 + f / 1024.0, e - 15);
    return s ? -v : v;
}

/* Uniform INT4 table ("QLoRA 原理精讲" §2.1: INT4 maps the values onto the 16
 * integers [-8, 7], evenly spaced).  Reading: the integers are divided by the
 * largest magnitude, 8, so that the table lies in [-1, 1] like NF4's and the
 * same absmax normalization applies: codes[i] = (i - 8) / 8. */
void oracle_codebook_int4(float codes[16])
{
    for (int i = 0; i < 16; i++) codes[i] = (float)(i - 8) / 8.0f;
}

/* quant_type: 0 = NF4, 1 = INT4 (uniform).  double_quant: 0 = FP8 E4M3
 * scale1 + FP32 scale2 per 256 blocks (the default of the pages), 1 = none
 * (FP32 scale1 per block, "QLoRA 原理精讲" §2.2 工程动机: 0.5 bit per weight),
 * 2 = unsigned 8-bit linear scale1 + FP32 scale2 per 256 blocks (the
 * "8 bit" of "LoRA、Q-LoRA 与 PortLLM" §3.2 read as an integer code). */
static void codebook_of(int quant_type, float codes[16])
{
    if (quant_type == 1) oracle_codebook_int4(codes);
    else oracle_codebook(codes);
}

/* Unsigned 8-bit linear code of a non-negative fp32 ratio: nearest integer,
 * ties to even, clamped to [0, 255]. */
static uint8_t u8_encode(float t)
{
    if (!(t > 0.0f)) return 0;
    if (t >= 255.0f) return 255;
    double fl = floor((double)t), d = (double)t - fl;
    double q = (d > 0.5) ? fl + 1.0 : (d < 0.5) ? fl : ((fmod(fl, 2.0) == 0.0) ? fl : fl + 1.0);
    return (uint8_t)q;
}

/* Quantize with a chosen table and first-level-constant format.  Same block
 * and group layout, codes and packing as oracle_quantize.  c1 receives
 * nblocks bytes (double_quant 0 or 2) or nblocks fp32 values (double_quant 1);
 * c2 receives ngroups fp32 values (unused, may be NULL, for double_quant 1).
 * Returns 1 when W holds a NaN or an infinity. */
int oracle_quantize_fmt(const uint16_t* W, int64_t numel, int quant_type, int double_quant,
                        uint8_t* packed, void* c1, float* c2)
{
    float codes[16];
    codebook_of(quant_type, codes);
    int64_t nb = oracle_nblocks(numel), ng = oracle_ngroups(numel);
    int nonfinite = 0;
    for (int64_t g = 0; g < ng; g++) {
        int64_t b0 = g * ORC_GROUP, b1 = b0 + ORC_GROUP;
        if (b1 > nb) b1 = nb;
        float absmax[ORC_GROUP];
        float gmax = 0.0f;
        for (int64_t b = b0; b < b1; b++) {            /* scale1 = block absmax */
            float m = 0.0f;
            int64_t e0 = b * ORC_BLOCK, e1 = e0 + ORC_BLOCK;
            if (e1 > numel) e1 = numel;
            for (int64_t e = e0; e < e1; e++) {
                float w = (float)oracle_bf16_to_f64(W[e]);
                if (!isfinite(w)) nonfinite = 1;
                float a = fabsf(w);
                if (a > m) m = a;
            }
            absmax[b - b0] = m;
            if (m > gmax) gmax = m;
        }
        if (double_quant == 1) {                       /* FP32 scale1, no second level */
            for (int64_t b = b0; b < b1; b++) ((float*)c1)[b] = absmax[b - b0];
        } else if (double_quant == 2) {                /* uint8 scale1 / FP32 scale2 */
            float s2 = gmax / 255.0f;
            c2[g] = s2;
            for (int64_t b = b0; b < b1; b++) {
                float m = absmax[b - b0];
                ((uint8_t*)c1)[b] = (m == 0.0f) ? (uint8_t)0 : u8_encode(m / s2);
            }
        } else {                                       /* E4M3 scale1 / FP32 scale2 */
            float s2 = gmax / 448.0f;
            c2[g] = s2;
            for (int64_t b = b0; b < b1; b++) {
                float m = absmax[b - b0];
                ((uint8_t*)c1)[b] = (m == 0.0f) ? (uint8_t)0 : oracle_e4m3_encode(m / s2);
            }
        }
        for (int64_t b = b0; b < b1; b++) {            /* 4-bit codes, packed */
            int64_t e0 = b * ORC_BLOCK, e1 = e0 + ORC_BLOCK;
            if (e1 > numel) e1 = numel;
            for (int64_t e = e0; e < e1; e++) {
                float w = (float)oracle_bf16_to_f64(W[e]);
                int q = oracle_nearest_code(codes, w, absmax[b - b0]);
                if ((e & 1) == 0) packed[e >> 1] = (uint8_t)q;
                else              packed[e >> 1] = (uint8_t)(packed[e >> 1] | (q << 4));
            }
        }
    }
    return nonfinite;
}

/* Dequantize a weight stored in any of the formats above into the compute
 * type (dtype 0 = bf16, 1 = fp16): scale1' = the stored FP32 scale1, or
 * fp32(decoded 8-bit code * scale2); w' = round_dtype(fp32(code * scale1')). */
void oracle_dequant_fmt(const uint8_t* packed, const void* c1, const float* c2, int64_t numel,
                        int quant_type, int double_quant, int dtype, uint16_t* out)
{
    float codes[16];
    codebook_of(quant_type, codes);
    for (int64_t e = 0; e < numel; e++) {
        int64_t b = e / ORC_BLOCK, g = b / ORC_GROUP;
        float s1;
        if (double_quant == 1) s1 = ((const float*)c1)[b];
        else if (double_quant == 2) s1 = (float)((const uint8_t*)c1)[b] * c2[g];
        else s1 = (float)oracle_e4m3_decode(((const uint8_t*)c1)[b]) * c2[g];
        int q = (e & 1) ? (packed[e >> 1] >> 4) : (packed[e >> 1] & 0xF);
        float v = codes[q] * s1;
        out[e] = dtype ? oracle_f16_round((double)v) : oracle_bf16_round((double)v);
    }
}

void oracle_f16_round_array(const double* x, int64_t n, uint16_t* out)
{
    for (int64_t i = 0; i < n; i++) out[i] = oracle_f16_round(x[i]);
}
void oracle_f16_decode_array(const uint16_t* h, int64_t n, double* out)
{
    for (int64_t i = 0; i < n; i++) out[i] = oracle_f16_to_f64(h[i]);
}
void oracle_classify_fmt_array(int quant_type, const float* w, const float* absmax, int64_t n, int32_t* q)
{
    float codes[16];
    codebook_of(quant_type, codes);
    for (int64_t i = 0; i < n; i++) q[i] = oracle_nearest_code(codes, w[i], absmax[i]);
}

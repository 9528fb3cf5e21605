/*
 * damp_oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, single-threaded CPU statement of one decode step of a
 * DAMP-style mixed-precision recurrent state for Gated DeltaNet (GDN) and
 * Kimi Delta Attention (KDA).  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg load it.  The CUDA library never calls it, and
 * the two share no source, header, table or helper.
 *
 * Sources (web pages, cited by title and section):
 *   [DAMP-v1] "DAMP: Decay-Aware Mixed-Precision Recurrent-State Quantization",
 *             arXiv 2608.27513v1 abstract: recurrent states are FP32 by
 *             default and their update is memory-bandwidth bound; high-risk
 *             channels are kept at higher precision and the rest in INT8, at
 *             9.9 bits per state value and 69.1 % less storage.
 *   [DAMP-v2] the same paper's later abstract (mlsanity.com index page):
 *             the high-risk *key channels* are kept in FP16 and the remainder
 *             in INT8 under a fixed storage budget.
 *   [STEP-C2] "STEPQuant: When and Where Errors Matter in Delta-Rule Recurrent
 *             State Quantization", Appendix Table C2 (one persistent decode
 *             step): step 1 reconstructs the state from integer codes and
 *             scales, or from FP16 values; step 2 forms
 *             X = D S^ + beta k (v^T - k^T D S^); step 3 emits X^T q *before*
 *             requantization; step 6 packs codes and scales and stores the
 *             FP16 values.
 *
 * Readings where the pages are silent (each is used once, where stated):
 *   R1 state layout: S is d_k x d_v, row i = key channel i, readout o = S^T q.
 *   R2 INT8 rows: symmetric per-row absmax with one FP32 scale per row,
 *      s = a/127 and codes in [-127, 127] (FP32 scales are the reading that
 *      reproduces 9.9 bits/value and 69.1 % at d = 128 with 27 FP16 rows).
 *   R3 quantizer: inv = fl32(127/a) once per row; code = the integer nearest
 *      to the exact product x*inv, ties to even.  A row whose absmax is 0, or
 *      so small that 127/a overflows FP32, is stored as scale 0, codes 0.
 *   R4 dequantize then decay, each an FP32 rounding: S' = fl(alpha_i*fl(c*s)).
 *   R5 u_j = k^T S'_{:,j} is summed over the key rows in recursive pairwise
 *      order (halves summed first, left before right) of the rounded
 *      products fl(k_i * S'_ij); all of it in FP32.
 *   R6 delta_j = fl(v_j - u_j); b_i = fl(beta*k_i); X_ij = fma(b_i, delta_j,
 *      S'_ij) (one rounding).
 *   R7 the readout o_j = sum_i q_i X_ij is returned in double precision (the
 *      FP32 state X read out exactly, up to double rounding).
 *   R8 FP16 rows are rounded to nearest, ties to even, with IEEE overflow to
 *      infinity; subnormals are kept.
 *
 * FP8 comparison format ([DAMP-v1] names uniform FP8 as a baseline that
 * already loses accuracy; it does not fix the variant or the scaling):
 *   F1 every row is FP8 E4M3 as defined by the OCP 8-bit floating point
 *      specification: sign, 4 exponent bits with bias 7, 3 mantissa bits,
 *      subnormals, no infinities, S.1111.111 is NaN, largest finite 448.
 *   F2 per-row absmax scaling as for INT8 rows: scale = fl(a/448),
 *      inv = fl(448/a); a == 0 or inv == +inf -> scale 0, codes 0.
 *   F3 code = the E4M3 value nearest to the FP32 product fl(x*inv), ties to
 *      the even mantissa; magnitudes above 448 saturate to 448.  (The
 *      product is rounded to FP32 first, as a conversion from FP32 does.)
 *   F4 dequantize: fl(value(code) * scale).
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_FMT_FP32 0   /* plain FP32 state, no quantization            */
#define ORACLE_FMT_QUANT 1  /* FP16 rows where is_fp16[i], INT8 rows elsewhere */
#define ORACLE_FMT_FP8 2    /* every row FP8 E4M3 with an FP32 scale (F1-F4)   */

#define ORACLE_GATE_SCALAR 0 /* GDN: one decay per (slot, head)             */
#define ORACLE_GATE_VECTOR 1 /* KDA: one decay per key channel               */

#define ORACLE_OK 0
#define ORACLE_EINVAL (-1)
#define ORACLE_ESLOT (-2)
#define ORACLE_ENOMEM (-3)

/* ------------------------------------------------------------------------ */
/* IEEE 754 binary16 <-> binary32 (R8)                                       */
/* ------------------------------------------------------------------------ */

/* binary32 -> binary16, round to nearest, ties to even.  The magnitude is
 * scaled (exactly, by a power of two) to units of the binary16 quantum at its
 * exponent, rounded with nearbyint() in the default rounding mode, and then
 * encoded.  Values at or above 65520 = 65504 + half a quantum round to
 * infinity. */
uint16_t oracle_f16_from_f32(float x)
{
    uint32_t bits;
    memcpy(&bits, &x, sizeof bits);
    uint16_t sign = (uint16_t)((bits >> 16) & 0x8000u);
    if (isnan(x)) return (uint16_t)(sign | 0x7e00u);
    double a = fabs((double)x);
    if (a >= 65520.0) return (uint16_t)(sign | 0x7c00u);
    int e;
    (void)frexp(a, &e); /* a = m 2^e, m in [0.5, 1): floor(log2 a) = e - 1 */
    int q_exp = (a < ldexp(1.0, -14)) ? -24 : (e - 1) - 10;
    double n = nearbyint(ldexp(a, -q_exp));
    double r = ldexp(n, q_exp);
    if (r == 0.0) return sign;
    if (r < ldexp(1.0, -14)) return (uint16_t)(sign | (uint16_t)n); /* subnormal */
    (void)frexp(r, &e);
    int E = e - 1; /* r in [2^E, 2^(E+1)) */
    uint32_t mant = (uint32_t)(ldexp(r, 10 - E) - 1024.0);
    return (uint16_t)(sign | (uint16_t)(((uint32_t)(E + 15) << 10) | mant));
}

/* binary16 -> binary32, exact. */
float oracle_f32_from_f16(uint16_t h)
{
    int s = (h >> 15) & 1, E = (h >> 10) & 31, m = h & 1023;
    double v;
    if (E == 0)
        v = ldexp((double)m, -24);
    else if (E == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + m), E - 25);
    return (float)(s ? -v : v);
}

void oracle_f16_from_f32_array(const float* x, uint16_t* out, long n)
{
    for (long i = 0; i < n; ++i) out[i] = oracle_f16_from_f32(x[i]);
}

void oracle_f32_from_f16_array(const uint16_t* h, float* out, long n)
{
    for (long i = 0; i < n; ++i) out[i] = oracle_f32_from_f16(h[i]);
}

/* ------------------------------------------------------------------------ */
/* INT8 row quantizer (R2, R3)                                               */
/* ------------------------------------------------------------------------ */

void oracle_quantize_row(const float* x, int n, int8_t* code, float* scale)
{
    float amax = 0.0f;
    for (int j = 0; j < n; ++j) {
        float t = fabsf(x[j]);
        if (t > amax) amax = t;
    }
    float inv = 127.0f / amax;
    if (amax == 0.0f || isinf(inv)) {
        *scale = 0.0f;
        for (int j = 0; j < n; ++j) code[j] = 0;
        return;
    }
    *scale = amax / 127.0f;
    for (int j = 0; j < n; ++j) {
        /* a 24-bit by 24-bit product is exact in double */
        double t = (double)x[j] * (double)inv;
        double r = nearbyint(t);
        if (r > 127.0) r = 127.0;
        if (r < -127.0) r = -127.0;
        code[j] = (int8_t)r;
    }
}

/* Exposes R3's pre-rounding value x*inv (exact, in double) for tests that
 * measure the distance of each code to a rounding boundary. */
void oracle_quantize_row_prerounding(const float* x, int n, double* t_out)
{
    float amax = 0.0f;
    for (int j = 0; j < n; ++j) {
        float t = fabsf(x[j]);
        if (t > amax) amax = t;
    }
    float inv = 127.0f / amax;
    int zero = (amax == 0.0f || isinf(inv));
    for (int j = 0; j < n; ++j) t_out[j] = zero ? 0.0 : (double)x[j] * (double)inv;
}

/* ------------------------------------------------------------------------ */
/* FP8 E4M3 (F1-F4)                                                          */
/* ------------------------------------------------------------------------ */

/* Value of an E4M3 code (F1). */
float oracle_f32_from_e4m3(uint8_t c)
{
    int sign = c >> 7, e = (c >> 3) & 15, m = c & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m, -9);             /* subnormal: m * 2^-6 / 8 */
    else v = ldexp(1.0 + m / 8.0, e - 7);
    return (float)(sign ? -v : v);
}

/* Nearest E4M3 code to y, ties to even mantissa, saturating at 448 (F3).
 * The magnitude is scaled (exactly, by a power of two) to units of the E4M3
 * quantum at its exponent and rounded with nearbyint(). */
uint8_t oracle_e4m3_from_f32(float y)
{
    uint8_t sign = signbit(y) ? 0x80u : 0u;
    if (isnan(y)) return (uint8_t)(sign | 0x7fu);
    double a = fabs((double)y);
    if (a >= 448.0) return (uint8_t)(sign | 0x7eu);
    if (a < ldexp(1.0, -6)) {
        double m = nearbyint(ldexp(a, 9));            /* quantum 2^-9 */
        return (uint8_t)(sign | (uint8_t)m);          /* m == 8 is the smallest normal */
    }
    int e;
    frexp(a, &e);                                     /* a = f * 2^e, f in [0.5, 1) */
    int E = e - 1;                                    /* a in [2^E, 2^(E+1)) */
    double r = nearbyint(ldexp(a, 3 - E));            /* in [8, 16] */
    if (r == 16.0) {
        r = 8.0;
        E += 1;
    }
    return (uint8_t)(sign | (uint8_t)((E + 7) << 3) | (uint8_t)(r - 8.0));
}

void oracle_e4m3_from_f32_array(const float* x, uint8_t* out, long n)
{
    for (long i = 0; i < n; ++i) out[i] = oracle_e4m3_from_f32(x[i]);
}

void oracle_f32_from_e4m3_array(const uint8_t* c, float* out, long n)
{
    for (long i = 0; i < n; ++i) out[i] = oracle_f32_from_e4m3(c[i]);
}

/* F2, F3 for one row; codes are stored as the E4M3 bit patterns. */
void oracle_quantize_row_fp8(const float* x, int n, uint8_t* code, float* scale)
{
    float amax = 0.0f;
    for (int j = 0; j < n; ++j) {
        float t = fabsf(x[j]);
        if (t > amax) amax = t;
    }
    float inv = 448.0f / amax;
    if (amax == 0.0f || isinf(inv)) {
        *scale = 0.0f;
        for (int j = 0; j < n; ++j) code[j] = 0;
        return;
    }
    *scale = amax / 448.0f;
    for (int j = 0; j < n; ++j) code[j] = oracle_e4m3_from_f32(x[j] * inv);
}

/* ------------------------------------------------------------------------ */
/* Pairwise FP32 sum (R5)                                                    */
/* ------------------------------------------------------------------------ */

float oracle_pairwise_sum(const float* x, int n)
{
    if (n == 1) return x[0];
    int h = n / 2;
    float left = oracle_pairwise_sum(x, h);
    float right = oracle_pairwise_sum(x + h, n - h);
    return left + right;
}

/* ------------------------------------------------------------------------ */
/* Pack / unpack one (slot, head) state                                      */
/* ------------------------------------------------------------------------ */
/*
 * Logical representation of one quantized state, rows in key-channel order:
 *   scale[d_k]        FP32 scale of each INT8 row (0 for FP16 rows)
 *   half[d_k*d_v]     binary16 bits of each FP16 row (0 for INT8 rows)
 *   code[d_k*d_v]     INT8 codes of each INT8 row (0 for FP16 rows)
 * and of an FP32 state:
 *   f32[d_k*d_v]
 */

int oracle_pack_unit(int fmt, int dk, int dv, const uint8_t* is_fp16, const float* S,
                     float* scale, uint16_t* half, int8_t* code, float* f32)
{
    if (dk <= 0 || dv <= 0) return ORACLE_EINVAL;
    if (fmt == ORACLE_FMT_FP32) {
        memcpy(f32, S, sizeof(float) * (size_t)dk * (size_t)dv);
        return ORACLE_OK;
    }
    if (fmt == ORACLE_FMT_FP8) {
        for (int i = 0; i < dk; ++i) {
            oracle_quantize_row_fp8(S + (size_t)i * dv, dv, (uint8_t*)code + (size_t)i * dv,
                                    &scale[i]);
            for (int j = 0; j < dv; ++j) half[(size_t)i * dv + j] = 0;
        }
        return ORACLE_OK;
    }
    if (fmt != ORACLE_FMT_QUANT) return ORACLE_EINVAL;
    for (int i = 0; i < dk; ++i) {
        const float* row = S + (size_t)i * dv;
        if (is_fp16[i]) {
            scale[i] = 0.0f;
            for (int j = 0; j < dv; ++j) {
                half[(size_t)i * dv + j] = oracle_f16_from_f32(row[j]);
                code[(size_t)i * dv + j] = 0;
            }
        } else {
            oracle_quantize_row(row, dv, code + (size_t)i * dv, &scale[i]);
            for (int j = 0; j < dv; ++j) half[(size_t)i * dv + j] = 0;
        }
    }
    return ORACLE_OK;
}

/* Step 1 of [STEP-C2]: reconstruct S^ (FP32) from the stored representation. */
int oracle_unpack_unit(int fmt, int dk, int dv, const uint8_t* is_fp16, const float* scale,
                       const uint16_t* half, const int8_t* code, const float* f32, float* S)
{
    if (dk <= 0 || dv <= 0) return ORACLE_EINVAL;
    if (fmt == ORACLE_FMT_FP32) {
        memcpy(S, f32, sizeof(float) * (size_t)dk * (size_t)dv);
        return ORACLE_OK;
    }
    if (fmt == ORACLE_FMT_FP8) {
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j) {
                size_t e = (size_t)i * dv + j;
                S[e] = oracle_f32_from_e4m3((uint8_t)code[e]) * scale[i];
            }
        return ORACLE_OK;
    }
    if (fmt != ORACLE_FMT_QUANT) return ORACLE_EINVAL;
    for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dv; ++j) {
            size_t e = (size_t)i * dv + j;
            S[e] = is_fp16[i] ? oracle_f32_from_f16(half[e]) : (float)code[e] * scale[i];
        }
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------ */
/* One decode step of one (slot, head)                                       */
/* ------------------------------------------------------------------------ */
/*
 * alpha: GDN -> alpha[0] (scalar decay); KDA -> alpha[0..d_k-1] (Diag(alpha)).
 * The new state is written back in place.  o[d_v] receives the readout of the
 * FP32 state X before requantization (R7).  X_out, when not NULL, receives X.
 */
int oracle_step_unit(int fmt, int gate, int dk, int dv, const uint8_t* is_fp16,
                     float* scale, uint16_t* half, int8_t* code, float* f32,
                     const float* q, const float* k, const float* v,
                     const float* alpha, float beta, double* o, float* X_out)
{
    if (dk <= 0 || dv <= 0) return ORACLE_EINVAL;
    if (fmt != ORACLE_FMT_FP32 && fmt != ORACLE_FMT_QUANT && fmt != ORACLE_FMT_FP8)
        return ORACLE_EINVAL;
    if (gate != ORACLE_GATE_SCALAR && gate != ORACLE_GATE_VECTOR) return ORACLE_EINVAL;
    size_t ne = (size_t)dk * dv;
    float* Shat = malloc(sizeof(float) * ne);
    float* Sp = malloc(sizeof(float) * ne);
    float* X = malloc(sizeof(float) * ne);
    float* prod = malloc(sizeof(float) * (size_t)dk);
    float* delta = malloc(sizeof(float) * (size_t)dv);
    float* b = malloc(sizeof(float) * (size_t)dk);
    if (!Shat || !Sp || !X || !prod || !delta || !b) {
        free(Shat); free(Sp); free(X); free(prod); free(delta); free(b);
        return ORACLE_ENOMEM;
    }

    /* [STEP-C2] step 1: reconstruct S^ */
    oracle_unpack_unit(fmt, dk, dv, is_fp16, scale, half, code, f32, Shat);

    /* decay D_t S^ (R4): row i scaled by alpha_i (GDN: D_t = alpha I) */
    for (int i = 0; i < dk; ++i) {
        float a = (gate == ORACLE_GATE_VECTOR) ? alpha[i] : alpha[0];
        for (int j = 0; j < dv; ++j) Sp[(size_t)i * dv + j] = a * Shat[(size_t)i * dv + j];
    }

    /* [STEP-C2] step 2: X = D S^ + beta k (v^T - k^T D S^)  (R5, R6) */
    for (int j = 0; j < dv; ++j) {
        for (int i = 0; i < dk; ++i) prod[i] = k[i] * Sp[(size_t)i * dv + j];
        float u = oracle_pairwise_sum(prod, dk);
        delta[j] = v[j] - u;
    }
    for (int i = 0; i < dk; ++i) b[i] = beta * k[i];
    for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dv; ++j)
            X[(size_t)i * dv + j] = fmaf(b[i], delta[j], Sp[(size_t)i * dv + j]);

    /* [STEP-C2] step 3: readout X^T q before requantization (R7) */
    for (int j = 0; j < dv; ++j) {
        double acc = 0.0;
        for (int i = 0; i < dk; ++i) acc += (double)q[i] * (double)X[(size_t)i * dv + j];
        o[j] = acc;
    }
    if (X_out) memcpy(X_out, X, sizeof(float) * ne);

    /* [STEP-C2] step 6 / [DAMP-v2]: requantize in place (FP16 rows, INT8 rows;
     * FP8 rows for the comparison format) */
    oracle_pack_unit(fmt, dk, dv, is_fp16, X, scale, half, code, f32);

    free(Shat); free(Sp); free(X); free(prod); free(delta); free(b);
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------ */
/* One decode step over a batch of (slot, head) units                        */
/* ------------------------------------------------------------------------ */
/*
 * Pool arrays are indexed [slot][head]:  scale [n_slots][H][dk],
 * half/code/f32 [n_slots][H][dk][dv].  is_fp16 is [H][dk] (the frozen
 * precision map, shared by all slots).  Batch arrays are indexed [b][head]:
 * q, k [n][H][dk], v [n][H][dv], alpha [n][H] (GDN) or [n][H][dk] (KDA),
 * beta [n][H], o [n][H][dv].  slot_idx[b] < 0 marks a padding entry whose
 * readout is zero and whose state is untouched; slot_idx[b] >= n_slots is an
 * error (nothing after it is processed).
 */
int oracle_decode_step(int fmt, int gate, int n, int H, int dk, int dv, int n_slots,
                       const uint8_t* is_fp16, const int32_t* slot_idx,
                       float* scale, uint16_t* half, int8_t* code, float* f32,
                       const float* q, const float* k, const float* v,
                       const float* alpha, const float* beta, double* o)
{
    size_t ne = (size_t)dk * dv;
    for (int bi = 0; bi < n; ++bi) {
        int slot = slot_idx[bi];
        for (int h = 0; h < H; ++h) {
            size_t u = (size_t)bi * H + h;
            double* ou = o + u * dv;
            if (slot < 0) {
                for (int j = 0; j < dv; ++j) ou[j] = 0.0;
                continue;
            }
            if (slot >= n_slots) return ORACLE_ESLOT;
            size_t s = (size_t)slot * H + h;
            const float* au = (gate == ORACLE_GATE_VECTOR) ? alpha + u * dk : alpha + u;
            int rc = oracle_step_unit(fmt, gate, dk, dv, is_fp16 + (size_t)h * dk,
                                      scale ? scale + s * dk : NULL,
                                      half ? half + s * ne : NULL,
                                      code ? code + s * ne : NULL,
                                      f32 ? f32 + s * ne : NULL,
                                      q + u * dk, k + u * dk, v + u * dv, au, beta[u], ou, NULL);
            if (rc != ORACLE_OK) return rc;
        }
    }
    return ORACLE_OK;
}

/*
 * calib_oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * Plain CPU statement of the offline calibration that picks the high-risk key
 * rows of a DAMP-style mixed-precision state.  Part of the oracle library
 * (liboracle.so) next to damp_oracle.c, whose INT8 row quantizer it reuses;
 * the CUDA library never calls it and the two share no code.
 *
 * Sources (web pages, cited by title and section):
 *   [DAMP-v1] "DAMP: Decay-Aware Mixed-Precision Recurrent-State Quantization",
 *             arXiv 2608.27513v1 abstract: quantization-error energy is
 *             concentrated in a few channels; the relative decay strength of
 *             channels is stable across prompts; offline calibration uses both
 *             the error energy and decay-based persistence to find the
 *             high-risk channels.
 *   [DAMP-v2] the later abstract (mlsanity.com index page): the selection
 *             weighs quantization error together with decay-based error
 *             retention, keeps the high-risk key channels in FP16 and the rest
 *             in INT8, under a fixed storage budget.
 *
 * Readings (the pages give no formula):
 *   C1 Error energy.  Calibration records the FP32 state X after each step of
 *      the unquantized recurrence.  For every recorded (slot, head) and key
 *      row i the INT8 quantizer of the decode step (damp_oracle.c, R2/R3) is
 *      applied to the row and e_i = sum_j (X_ij - fl(c_ij * s_i))^2 is formed
 *      in double (each difference is exact in double).  energy_i is the sum
 *      of e_i over the records.
 *   C2 Retention.  A state error in row i is multiplied by the row's decay
 *      alpha_i at the next step, so its energy by alpha_i^2; retention_i is
 *      the sum of alpha_i^2 (double) over the same records (GDN: the scalar
 *      decay of the (slot, head); KDA: channel i of the decay vector).
 *   C3 Score.  With c records per head, rho_i = retention_i / c and
 *      E_i = energy_i / c, error injected at every step accumulates as a
 *      geometric series, so score_i = E_i / max(1 - rho_i, 2^-30).
 *      (The projection (I - beta k k^T) is not counted: the pages call the
 *      persistence decay-based.)
 *   C4 Per-head selection.  The hp rows with the largest score are FP16;
 *      among equal scores the lower row index wins.  Indices are returned in
 *      ascending order.
 *
 * Accumulator layout (double): energy[H][d_k], retention[H][d_k], count[H].
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <string.h>

void oracle_quantize_row(const float* x, int n, int8_t* code, float* scale);

#define CAL_OK 0
#define CAL_EINVAL (-1)
#define CAL_ESLOT (-2)

/* C1 for one row. */
double oracle_row_quant_error(const float* x, int n)
{
    int8_t code[256];
    float scale;
    if (n <= 0 || n > 256) return -1.0;
    oracle_quantize_row(x, n, code, &scale);
    double e = 0.0;
    for (int j = 0; j < n; ++j) {
        float dq = (float)code[j] * scale;
        double diff = (double)x[j] - (double)dq;
        e += diff * diff;
    }
    return e;
}

/*
 * Adds one step's records to acc.  f32_pool [n_slots][H][dk][dv] holds the
 * FP32 states after the step; slot_idx [n] names the slots stepped (negative:
 * padding, skipped); alpha [n][H] (gate 0) or [n][H][dk] (gate 1) is the
 * decay the step used.
 */
int oracle_calib_accumulate(int gate, int n, int H, int dk, int dv, int n_slots,
                            const float* f32_pool, const int32_t* slot_idx,
                            const float* alpha, double* acc)
{
    if (n < 0 || H <= 0 || dk <= 0 || dv <= 0 || dv > 256) return CAL_EINVAL;
    double* energy = acc;
    double* retention = acc + (size_t)H * dk;
    double* count = acc + 2 * (size_t)H * dk;
    for (int b = 0; b < n; ++b) {
        int slot = slot_idx[b];
        if (slot < 0) continue;
        if (slot >= n_slots) return CAL_ESLOT;
        for (int h = 0; h < H; ++h) {
            const float* S = f32_pool + ((size_t)slot * H + h) * dk * dv;
            for (int i = 0; i < dk; ++i) {
                double a = gate == 1 ? (double)alpha[((size_t)b * H + h) * dk + i]
                                     : (double)alpha[(size_t)b * H + h];
                energy[(size_t)h * dk + i] += oracle_row_quant_error(S + (size_t)i * dv, dv);
                retention[(size_t)h * dk + i] += a * a;
            }
            count[h] += 1.0;
        }
    }
    return CAL_OK;
}

/* C3 for every (head, row); score[H][dk]. */
int oracle_calib_scores(int H, int dk, const double* acc, double* score)
{
    if (H <= 0 || dk <= 0) return CAL_EINVAL;
    const double* energy = acc;
    const double* retention = acc + (size_t)H * dk;
    const double* count = acc + 2 * (size_t)H * dk;
    const double floor_ = ldexp(1.0, -30);
    for (int h = 0; h < H; ++h)
        for (int i = 0; i < dk; ++i) {
            size_t e = (size_t)h * dk + i;
            if (count[h] <= 0.0) {
                score[e] = 0.0;
                continue;
            }
            double E = energy[e] / count[h];
            double keep = 1.0 - retention[e] / count[h];
            if (keep < floor_) keep = floor_;
            score[e] = E / keep;
        }
    return CAL_OK;
}

/* C4: idx_out [H][hp], ascending within each head. */
int oracle_calib_select(int H, int dk, int hp, const double* score, uint16_t* idx_out)
{
    if (H <= 0 || dk <= 0 || hp < 0 || hp > dk || dk > 256) return CAL_EINVAL;
    for (int h = 0; h < H; ++h) {
        const double* s = score + (size_t)h * dk;
        uint8_t taken[256];
        memset(taken, 0, sizeof taken);
        for (int k = 0; k < hp; ++k) {
            int best = -1;
            for (int i = 0; i < dk; ++i) {
                if (taken[i]) continue;
                if (best < 0 || s[i] > s[best]) best = i;   /* strict: lower index wins ties */
            }
            taken[best] = 1;
        }
        int w = 0;
        for (int i = 0; i < dk; ++i)
            if (taken[i]) idx_out[(size_t)h * hp + w++] = (uint16_t)i;
    }
    return CAL_OK;
}

/*
 * Budget selection (the "fixed storage budget" of [DAMP-v2], read as a total
 * number of FP16 rows shared by all heads of a layer): the `budget` (head,
 * row) pairs with the largest score are FP16; equal scores go to the lower
 * head, then the lower row.  is_fp16_out [H][dk] (0/1); hp_out [H] counts the
 * FP16 rows each head received.
 */
int oracle_calib_select_budget(int H, int dk, int budget, const double* score,
                               uint8_t* is_fp16_out, int32_t* hp_out)
{
    if (H <= 0 || dk <= 0 || budget < 0 || (long)budget > (long)H * dk) return CAL_EINVAL;
    size_t total = (size_t)H * dk;
    memset(is_fp16_out, 0, total);
    for (int k = 0; k < budget; ++k) {
        size_t best = total;
        for (size_t e = 0; e < total; ++e) {
            if (is_fp16_out[e]) continue;
            if (best == total || score[e] > score[best]) best = e;
        }
        is_fp16_out[best] = 1;
    }
    for (int h = 0; h < H; ++h) {
        int c = 0;
        for (int i = 0; i < dk; ++i) c += is_fp16_out[(size_t)h * dk + i];
        hp_out[h] = c;
    }
    return CAL_OK;
}

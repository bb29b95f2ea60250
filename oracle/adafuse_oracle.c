/*
 * adafuse_oracle.c -- CPU oracle for the AdaFuse adapter-switch hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the plain, slow, fp64 statement of
 * what the hot path computes.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load it.  It shares no code, header, table
 * or helper with the CUDA library in weight_merge_b200/csrc, and neither side
 * includes or links the other.
 *
 * Sources (page title, then the section the step follows):
 *   [P1] "AdaFuse: Accelerating Dynamic Adapter Inference via Token-Level
 *        Pre-Gating and Fused Kernel Optimization", shd-paper.top summary,
 *        English abstract (one routing decision per token for all adapter
 *        layers; one fused switch that merges the selected LoRA adapters into
 *        the backbone in a single pass).
 *   [P2] same title, gist.science technical summary:
 *        section 2-ga "Token-Level Pre-Gating" items 1-3 (a top-2 router in
 *        the first layer picks the token's experts; the choice is applied to
 *        every later layer);
 *        section 2-na "Fused Adapter Switching via the SGMM kernel" (remove
 *        the previous token's adapters, merge the current token's, all
 *        layers, in place).
 *
 * Readings where the pages are silent (each listed in the design notes):
 *   - router input is the fp32 hidden state entering the first layer, no
 *     bias and no norm: z_e = sum_i h_i * Wr[i,e];
 *   - the two experts are the first two under the order (z descending,
 *     index ascending), so ties go to the lower index;
 *   - gates are the full softmax over all E experts renormalised over the
 *     two picks (equal to the softmax of the two logits);
 *   - merge scale s = alpha / r;
 *   - W_new = bf16_rne(W + dW), one rounding, with
 *     dW = s * sum_{e in cur} g_e B_e A_e  -  s * sum_{e in prev} g_e B_e A_e
 *     (each set summed in slot order, so prev == cur cancels exactly).
 *
 * Layouts (row-major everywhere):
 *   h  [T, d] fp32, Wr [d, E] fp32
 *   W  [out, in] bf16 (as uint16 bit patterns)
 *   A  [E, r, in] bf16, B [E, out, r] bf16
 *   route: idx[k] int32 (-1 = no expert), gate[k] fp32; k = 2 for the
 *   pages' top-2 router, 1..4 for the top-k widening
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ---- bf16 <-> double ---------------------------------------------------- */

/* bf16 is the top 16 bits of an IEEE binary32; widening is exact. */
double orc_bf16_to_double(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Round a double to the nearest bf16, ties to even, in ONE step (no detour
 * through binary32, which would round twice).  bf16 keeps 8 significant bits,
 * has binary32's exponent range (normals down to 2^-126) and subnormals with
 * spacing 2^-133.  Overflow past the largest finite value goes to infinity. */
uint16_t orc_bf16_from_double(double x) {
    uint16_t sign = signbit(x) ? 0x8000u : 0u;
    if (isnan(x)) return 0x7fc0u;
    if (isinf(x)) return (uint16_t)(sign | 0x7f80u);
    double ax = fabs(x);
    int e2 = 0;
    frexp(ax, &e2);                    /* ax = m * 2^e2, m in [0.5, 1) */
    int lead = e2 - 1;                 /* weight of the leading bit */
    if (lead < -126) lead = -126;      /* subnormal range: fixed spacing */
    double q = ldexp(1.0, lead - 7);   /* spacing of bf16 values near ax */
    double y = nearbyint(ax / q) * q;  /* default rounding mode: to nearest even */
    if (y >= ldexp(1.0, 128)) return (uint16_t)(sign | 0x7f80u);
    float f = (float)y;                /* exact: y has <= 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(sign | (uint16_t)(u >> 16));
}

void orc_bf16_from_double_array(const double* x, int64_t n, uint16_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = orc_bf16_from_double(x[i]);
}

/* ---- token-level pre-gating ([P2] 2-ga, items 1-3) ---------------------- */

/* For each token t: logits z_e = sum_i h[t,i] Wr[i,e] in fp64; the two
 * experts first in (z desc, index asc); p = softmax(z) over all E (max
 * subtracted); g_j = p_{e_j} / (p_{e_0} + p_{e_1}), rounded to fp32.
 * With E == 1 the second slot is empty: idx = {0, -1}, gate = {1, 0}.
 * Also returns the fp64 logits when z_out is not NULL ([T, E]). */
void orc_pregate(const float* h, int64_t T, int64_t d, const float* Wr,
                 int32_t E, int32_t* idx_out, float* gate_out, double* z_out) {
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        double* z = (double*)malloc(sizeof(double) * (size_t)E);
        for (int32_t e = 0; e < E; ++e) {
            double acc = 0.0;
            for (int64_t i = 0; i < d; ++i)
                acc += (double)h[t * d + i] * (double)Wr[i * E + e];
            z[e] = acc;
        }
        /* first pick: largest z, lowest index among equals */
        int32_t e0 = 0;
        for (int32_t e = 1; e < E; ++e)
            if (z[e] > z[e0]) e0 = e;
        /* second pick: same rule over the remaining experts */
        int32_t e1 = -1;
        for (int32_t e = 0; e < E; ++e) {
            if (e == e0) continue;
            if (e1 < 0 || z[e] > z[e1]) e1 = e;
        }
        /* softmax over all E, then renormalise over the two picks */
        double zmax = z[e0];
        double denom = 0.0;
        for (int32_t e = 0; e < E; ++e) denom += exp(z[e] - zmax);
        double p0 = exp(z[e0] - zmax) / denom;
        double p1 = (e1 >= 0) ? exp(z[e1] - zmax) / denom : 0.0;
        idx_out[2 * t + 0] = e0;
        idx_out[2 * t + 1] = e1;
        gate_out[2 * t + 0] = (float)(p0 / (p0 + p1));
        gate_out[2 * t + 1] = (float)(p1 / (p0 + p1));
        if (z_out)
            for (int32_t e = 0; e < E; ++e) z_out[t * E + e] = z[e];
        free(z);
    }
}

/* Top-k pre-gating, k in [1, 4]: the same rule with k picks.  A reading of
 * [P2] 2-ga beyond its top-2 router (the pages fix k = 2; larger k is the
 * natural widening of the same router):
 *   pick j = the largest z among the experts not yet picked, lowest index
 *   among equals; p = softmax(z) over all E (max subtracted);
 *   g_j = p_{e_j} / sum_{i < k} p_{e_i}, rounded to fp32.
 * Slots past E hold idx -1 and gate 0.  idx_out / gate_out are [T, k]. */
void orc_pregate_topk(const float* h, int64_t T, int64_t d, const float* Wr,
                      int32_t E, int32_t k, int32_t* idx_out, float* gate_out,
                      double* z_out) {
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        double* z = (double*)malloc(sizeof(double) * (size_t)E);
        char* taken = (char*)calloc((size_t)E, 1);
        for (int32_t e = 0; e < E; ++e) {
            double acc = 0.0;
            for (int64_t i = 0; i < d; ++i)
                acc += (double)h[t * d + i] * (double)Wr[i * E + e];
            z[e] = acc;
        }
        int32_t pick[4] = {-1, -1, -1, -1};
        for (int32_t j = 0; j < k; ++j) {
            int32_t best = -1;
            for (int32_t e = 0; e < E; ++e) {
                if (taken[e]) continue;
                if (best < 0 || z[e] > z[best]) best = e;
            }
            if (best < 0) break;
            pick[j] = best;
            taken[best] = 1;
        }
        double zmax = z[pick[0]];
        double denom = 0.0;
        for (int32_t e = 0; e < E; ++e) denom += exp(z[e] - zmax);
        double p[4] = {0.0, 0.0, 0.0, 0.0}, psum = 0.0;
        for (int32_t j = 0; j < k; ++j)
            if (pick[j] >= 0) {
                p[j] = exp(z[pick[j]] - zmax) / denom;
                psum += p[j];
            }
        for (int32_t j = 0; j < k; ++j) {
            idx_out[t * k + j] = pick[j];
            gate_out[t * k + j] = pick[j] >= 0 ? (float)(p[j] / psum) : 0.0f;
        }
        if (z_out)
            for (int32_t e = 0; e < E; ++e) z_out[t * E + e] = z[e];
        free(taken);
        free(z);
    }
}

/* Batch pre-gating: ONE routing decision for a decode batch of T tokens
 * that shares one merged weight.  A reading beyond [P2] 2-ga, which makes
 * one decision per token: a batch whose tokens would pick different experts
 * can carry only one expert set in W, so the batch's router logits are
 * averaged and the token rule is applied to the mean:
 *   z_t,e  = sum_i h[t,i] Wr[i,e]           (each token's logits, fp64)
 *   zbar_e = (1/T) sum_t z_t,e
 *   pick j = the largest zbar among the experts not yet picked, lowest
 *            index among equals, j < k (k in [1, 4]);
 *   g_j    = softmax(zbar) over all E renormalised over the k picks,
 *            rounded to fp32.
 * Slots past E hold idx -1 and gate 0.  idx_out / gate_out are [k]; the
 * mean logits go to zbar_out ([E]) when it is not NULL.  T >= 1. */
void orc_pregate_batch(const float* h, int64_t T, int64_t d, const float* Wr,
                       int32_t E, int32_t k, int32_t* idx_out, float* gate_out,
                       double* zbar_out) {
    double* zbar = (double*)calloc((size_t)E, sizeof(double));
    char* taken = (char*)calloc((size_t)E, 1);
    for (int64_t t = 0; t < T; ++t)
        for (int32_t e = 0; e < E; ++e) {
            double acc = 0.0;
            for (int64_t i = 0; i < d; ++i)
                acc += (double)h[t * d + i] * (double)Wr[i * E + e];
            zbar[e] += acc;
        }
    for (int32_t e = 0; e < E; ++e) zbar[e] /= (double)T;
    int32_t pick[4] = {-1, -1, -1, -1};
    for (int32_t j = 0; j < k; ++j) {
        int32_t best = -1;
        for (int32_t e = 0; e < E; ++e) {
            if (taken[e]) continue;
            if (best < 0 || zbar[e] > zbar[best]) best = e;
        }
        if (best < 0) break;
        pick[j] = best;
        taken[best] = 1;
    }
    double zmax = zbar[pick[0]];
    double denom = 0.0;
    for (int32_t e = 0; e < E; ++e) denom += exp(zbar[e] - zmax);
    double p[4] = {0.0, 0.0, 0.0, 0.0}, psum = 0.0;
    for (int32_t j = 0; j < k; ++j)
        if (pick[j] >= 0) {
            p[j] = exp(zbar[pick[j]] - zmax) / denom;
            psum += p[j];
        }
    for (int32_t j = 0; j < k; ++j) {
        idx_out[j] = pick[j];
        gate_out[j] = pick[j] >= 0 ? (float)(p[j] / psum) : 0.0f;
    }
    if (zbar_out)
        for (int32_t e = 0; e < E; ++e) zbar_out[e] = zbar[e];
    free(taken);
    free(zbar);
}

/* ---- fused adapter switch ([P1] abstract, [P2] 2-na) -------------------- */

/* The experts a route of `slots` slots names (slots holding -1 are empty).
 * Returns how many entries were written (0..slots). */
static int route_experts(const int32_t* idx, const float* gate, int32_t slots,
                        int32_t* e_out, double* g_out) {
    int n = 0;
    if (!idx) return 0;
    for (int j = 0; j < slots; ++j) {
        if (idx[j] < 0) continue;
        e_out[n] = idx[j];
        g_out[n] = (double)gate[j];
        ++n;
    }
    return n;
}

/* (B_e A_e)[i, j] = sum_k B_e[i, k] A_e[k, j], operands widened to fp64. */
static double lora_product(const uint16_t* A, const uint16_t* B, int64_t out,
                           int64_t in, int32_t r, int32_t e, int64_t i,
                           int64_t j) {
    const uint16_t* Brow = B + ((int64_t)e * out + i) * r;
    const uint16_t* Ae = A + (int64_t)e * r * in;
    double acc = 0.0;
    for (int32_t k = 0; k < r; ++k)
        acc += orc_bf16_to_double(Brow[k]) * orc_bf16_to_double(Ae[(int64_t)k * in + j]);
    return acc;
}

/* One switch of one (layer, target) weight, on a chosen set of rows.
 *   W_rows   [n_rows, in]  the rows' values before the switch
 *   row_ids  [n_rows]      which rows of the [out, in] matrix they are
 *   prev_*, cur_*          a route (idx[slots], gate[slots]) or NULL for "none"
 *   slots                  route slots, 1..4 (the top-k of the router)
 *   W_new    [n_rows, in]  bf16_rne(W + dW)          (may be NULL)
 *   W_exact  [n_rows, in]  W + dW in fp64, unrounded (may be NULL)
 * dW = s * sum_{e in cur} g_e (B_e A_e) - s * sum_{e in prev} g_e (B_e A_e),
 * each sum taken in slot order, so equal routes cancel exactly. */
void orc_switch_rows_k(const uint16_t* W_rows, const int64_t* row_ids,
                       int64_t n_rows, int64_t out, int64_t in,
                       const uint16_t* A, const uint16_t* B, int32_t r, double s,
                       int32_t slots,
                       const int32_t* prev_idx, const float* prev_gate,
                       const int32_t* cur_idx, const float* cur_gate,
                       uint16_t* W_new, double* W_exact) {
    int32_t pe[4], ce[4];
    double pg[4], cg[4];
    if (slots < 1) slots = 1;
    if (slots > 4) slots = 4;
    int np = route_experts(prev_idx, prev_gate, slots, pe, pg);
    int nc = route_experts(cur_idx, cur_gate, slots, ce, cg);
#pragma omp parallel for schedule(static)
    for (int64_t q = 0; q < n_rows; ++q) {
        int64_t i = row_ids[q];
        for (int64_t j = 0; j < in; ++j) {
            double plus = 0.0, minus = 0.0;
            for (int a = 0; a < nc; ++a)
                plus += cg[a] * lora_product(A, B, out, in, r, ce[a], i, j);
            for (int a = 0; a < np; ++a)
                minus += pg[a] * lora_product(A, B, out, in, r, pe[a], i, j);
            double dW = s * plus - s * minus;
            double w = orc_bf16_to_double(W_rows[q * in + j]) + dW;
            if (W_exact) W_exact[q * in + j] = w;
            if (W_new) W_new[q * in + j] = orc_bf16_from_double(w);
        }
    }
}

/* The top-2 switch: routes of two slots. */
void orc_switch_rows(const uint16_t* W_rows, const int64_t* row_ids,
                     int64_t n_rows, int64_t out, int64_t in,
                     const uint16_t* A, const uint16_t* B, int32_t r, double s,
                     const int32_t* prev_idx, const float* prev_gate,
                     const int32_t* cur_idx, const float* cur_gate,
                     uint16_t* W_new, double* W_exact) {
    orc_switch_rows_k(W_rows, row_ids, n_rows, out, in, A, B, r, s, 2, prev_idx,
                      prev_gate, cur_idx, cur_gate, W_new, W_exact);
}

/* Threads the oracle's parallel loops use (1 when built without OpenMP). */
int orc_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void orc_set_num_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

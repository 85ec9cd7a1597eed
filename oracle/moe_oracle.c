/*
 * moe_oracle.c -- plain, slow, single-threaded CPU oracle for the forward pass of a
 * Qwen-family sparse MoE FFN block (and, for the training-side entry points, the Switch
 * balance loss and the block's backward pass).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or calls this file:
 * only the tests, the package's smoke check and the benchmark's CPU-baseline leg do.  It
 * shares no code, header or table with the CUDA library.
 *
 * What it computes (sources, by page title and section):
 *  - "27. Mixture of experts" (inference.shantanugoel.com), section "The router":
 *      logits = W_r x, an FP32 softmax over all E experts, keep the k largest
 *      probabilities and their indices, and when norm_topk_prob is set divide the kept
 *      weights by their sum.  Ties in top-k are broken by expert index (the paragraph
 *      after the TopKRouter listing).  Worked example: probabilities [0.1, 0.5, 0.3, 0.1],
 *      k = 2 -> experts 1 and 2 with weights 0.625 and 0.375.
 *  - same page, section "Dispatch": experts are stored stacked, gate_up_proj [E, 2I, D]
 *      with the I gate rows first, down_proj [E, D, I]; expert(x) =
 *      down(silu(gate x) * up x).  The grouped dispatch sorts the N*k assignments by
 *      expert with a stable sort and counts them per expert (bincount).
 *  - same page, section "The shared expert": y = sum_{top-k} w_i expert_i(x)
 *      + sigmoid(w_s . x) shared(x).
 *  - "Qwen3-VL and Mixture of Experts" (gopikrishnatummala.com), section "What a
 *      mixture-of-experts layer is": y = sum_{i in top-k} g_i(x) E_i(x).
 *
 * Arithmetic: every dot product and the SwiGLU chain are evaluated in IEEE double with no
 * intermediate rounding.  The router logit is rounded once to FP32 (the pages compute the
 * softmax in FP32 on FP32-or-narrower logits); probabilities and weights are computed in
 * double from those FP32 logits and stored as FP32.  bf16 inputs are passed as their raw
 * 16-bit patterns and widened exactly.
 *
 * Readings taken where the pages are silent (each is listed in the design notes):
 *  - selection ranks experts by FP32 logit (softmax is strictly increasing, so the set is
 *    the same as ranking the probabilities), ties -> lower expert index; -0.0 == +0.0;
 *  - the softmax subtracts the row maximum before exponentiating;
 *  - an optional FP32 bias b[e] is added to the logit (in FP32) before the softmax;
 *  - the k weighted expert outputs are summed in slot order j = 0..k-1;
 *  - within an expert segment assignments keep their flat order a = t*k + j (stable).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* Exact widening of a bf16 bit pattern. */
static double bf16_to_double(uint16_t h) {
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* ---------------------------------------------------------------- router ------------- */

/* logits[t, e] = fl32( sum_d x[t, d] * W_r[e, d] ), then + bias[e] in FP32 if given.
 * x: [T, D] bf16, W_r: [E, D] bf16 (nn.Linear layout), bias: [E] float or NULL. */
int oracle_router_logits(const uint16_t *x, const uint16_t *W_r, const float *bias,
                         int T, int D, int E, float *logits) {
    if (!x || !W_r || !logits || T < 0 || D <= 0 || E <= 0) return 1;
    for (int t = 0; t < T; ++t) {
        for (int e = 0; e < E; ++e) {
            double s = 0.0;
            for (int d = 0; d < D; ++d)
                s += bf16_to_double(x[(size_t)t * D + d]) * bf16_to_double(W_r[(size_t)e * D + d]);
            float l = (float)s;
            if (bias) l = l + bias[e];
            logits[(size_t)t * E + e] = l;
        }
    }
    return 0;
}

/* Does expert a rank before expert b?  Higher logit first; equal logits -> lower index. */
static int ranks_before(float la, int a, float lb, int b) {
    if (la > lb) return 1;
    if (la < lb) return 0;      /* -0.0 and +0.0 compare equal here, as required */
    return a < b;
}

/* Softmax over all E logits of one token, in double from the FP32 logits, max-subtracted.
 * probs_out[e] receives the double probabilities. */
static void softmax_row(const float *l, int E, double *probs_out) {
    double m = (double)l[0];
    for (int e = 1; e < E; ++e)
        if ((double)l[e] > m) m = (double)l[e];
    double s = 0.0;
    for (int e = 0; e < E; ++e) {
        probs_out[e] = exp((double)l[e] - m);
        s += probs_out[e];
    }
    for (int e = 0; e < E; ++e) probs_out[e] /= s;
}

/* Selection and weights from given FP32 logits [T, E]:
 * idx[t, j] = the j-th ranked expert; w[t, j] = pi(idx) or pi(idx) / sum_j pi(idx_j). */
int oracle_select(const float *logits, int T, int E, int k, int norm, int32_t *idx, float *w) {
    if (!logits || !idx || !w || T < 0 || E <= 0 || k <= 0 || k > E) return 1;
    double *p = (double *)malloc(sizeof(double) * (size_t)E);
    int *order = (int *)malloc(sizeof(int) * (size_t)E);
    if (!p || !order) { free(p); free(order); return 2; }
    for (int t = 0; t < T; ++t) {
        const float *l = logits + (size_t)t * E;
        softmax_row(l, E, p);
        /* insertion sort of all E experts by the ranking rule (O(E^2), deliberately plain) */
        for (int e = 0; e < E; ++e) {
            int pos = e;
            while (pos > 0 && ranks_before(l[e], e, l[order[pos - 1]], order[pos - 1])) {
                order[pos] = order[pos - 1];
                --pos;
            }
            order[pos] = e;
        }
        double kept = 0.0;
        for (int j = 0; j < k; ++j) kept += p[order[j]];
        for (int j = 0; j < k; ++j) {
            idx[(size_t)t * k + j] = order[j];
            double wj = norm ? p[order[j]] / kept : p[order[j]];
            w[(size_t)t * k + j] = (float)wj;
        }
    }
    free(p);
    free(order);
    return 0;
}

/* Router: logits, then selection. */
int oracle_route(const uint16_t *x, const uint16_t *W_r, const float *bias, int T, int D,
                 int E, int k, int norm, float *logits, int32_t *idx, float *w) {
    int rc = oracle_router_logits(x, W_r, bias, T, D, E, logits);
    if (rc) return rc;
    return oracle_select(logits, T, E, k, norm, idx, w);
}

/* ---------------------------------------------------------------- permute ------------ */

/* Stable counting sort of the T*k assignments a = t*k + j by expert:
 *   counts[e]   = #{a : idx[a] == e}
 *   offsets[0]  = 0, offsets[e+1] = offsets[e] + ceil(counts[e] / tile_m) * tile_m
 *   row r in [offsets[e], offsets[e] + counts[e]) holds the assignments of expert e in
 *   increasing a; row_token[r] = a / k; slot_row[a] = r; padding rows get row_token = -1.
 * cap is the length of row_token.  Returns 3 when cap < offsets[E]. */
int oracle_permute(const int32_t *idx, int T, int k, int E, int tile_m, int32_t *counts,
                   int32_t *offsets, int32_t *row_token, int32_t *slot_row, int cap) {
    if (!idx || !counts || !offsets || !row_token || !slot_row || T < 0 || k <= 0 || E <= 0 ||
        tile_m <= 0)
        return 1;
    long n = (long)T * k;
    for (int e = 0; e < E; ++e) counts[e] = 0;
    for (long a = 0; a < n; ++a) {
        int e = idx[a];
        if (e < 0 || e >= E) return 1;
        counts[e] += 1;
    }
    offsets[0] = 0;
    for (int e = 0; e < E; ++e) {
        int padded = (counts[e] + tile_m - 1) / tile_m * tile_m;
        offsets[e + 1] = offsets[e] + padded;
    }
    if (offsets[E] > cap) return 3;
    for (int r = 0; r < cap; ++r) row_token[r] = -1;
    int *fill = (int *)calloc((size_t)E, sizeof(int));
    if (!fill) return 2;
    for (long a = 0; a < n; ++a) {
        int e = idx[a];
        int r = offsets[e] + fill[e]++;
        row_token[r] = (int32_t)(a / k);
        slot_row[a] = r;
    }
    free(fill);
    return 0;
}

/* ---------------------------------------------------------------- experts ------------ */

/* One SwiGLU expert on one token, all in double:
 *   g_i = sum_d W_gu[i, d] x_d,  u_i = sum_d W_gu[I + i, d] x_d   (gate rows first)
 *   h_i = silu(g_i) * u_i,       silu(z) = z / (1 + exp(-z))
 *   out_d = sum_i W_dn[d, i] h_i
 * W_gu: [2I, D] bf16, W_dn: [D, I] bf16.  h is caller scratch of length I. */
static void swiglu_expert(const uint16_t *x_row, const uint16_t *W_gu, const uint16_t *W_dn,
                          int D, int I, double *h, double *out) {
    for (int i = 0; i < I; ++i) {
        double g = 0.0, u = 0.0;
        for (int d = 0; d < D; ++d) {
            double xd = bf16_to_double(x_row[d]);
            g += bf16_to_double(W_gu[(size_t)i * D + d]) * xd;
            u += bf16_to_double(W_gu[(size_t)(I + i) * D + d]) * xd;
        }
        h[i] = g / (1.0 + exp(-g)) * u;
    }
    for (int d = 0; d < D; ++d) {
        double s = 0.0;
        for (int i = 0; i < I; ++i) s += bf16_to_double(W_dn[(size_t)d * I + i]) * h[i];
        out[d] = s;
    }
}

/* y for the listed token rows, given the routing (idx, w) of every token:
 *   y[t] = sum_{j<k} w[t,j] * expert_{idx[t,j]}(x[t])
 *          (+ sigmoid(w_s . x[t]) * shared(x[t])  when shared_gate_up is given;
 *             the sigmoid factor is 1 when shared_gate is NULL)
 *          (+ residual[t] when given)
 * rows: nrows token indices; y_out: [nrows, D] double. */
int oracle_combine_rows(const uint16_t *x, const int32_t *idx, const float *w,
                        const int32_t *rows, int nrows, int T, int D, int E, int k, int I,
                        const uint16_t *W_gu, const uint16_t *W_dn,
                        const uint16_t *shared_gate_up, const uint16_t *shared_down,
                        const uint16_t *shared_gate, int I_s, const uint16_t *residual,
                        double *y_out) {
    if (!x || !idx || !w || !rows || !W_gu || !W_dn || !y_out || D <= 0 || I <= 0 || k <= 0)
        return 1;
    if (shared_gate_up && (!shared_down || I_s <= 0)) return 1;
    int hmax = I > I_s ? I : I_s;
    double *h = (double *)malloc(sizeof(double) * (size_t)hmax);
    double *o = (double *)malloc(sizeof(double) * (size_t)D);
    if (!h || !o) { free(h); free(o); return 2; }
    for (int n = 0; n < nrows; ++n) {
        int t = rows[n];
        if (t < 0 || t >= T) { free(h); free(o); return 1; }
        const uint16_t *xr = x + (size_t)t * D;
        double *y = y_out + (size_t)n * D;
        for (int d = 0; d < D; ++d) y[d] = 0.0;
        for (int j = 0; j < k; ++j) {
            int e = idx[(size_t)t * k + j];
            if (e < 0 || e >= E) { free(h); free(o); return 1; }
            swiglu_expert(xr, W_gu + (size_t)e * 2 * I * D, W_dn + (size_t)e * D * I, D, I, h, o);
            double wj = (double)w[(size_t)t * k + j];
            for (int d = 0; d < D; ++d) y[d] += wj * o[d];
        }
        if (shared_gate_up) {
            double gate = 1.0;
            if (shared_gate) {
                double z = 0.0;
                for (int d = 0; d < D; ++d)
                    z += bf16_to_double(shared_gate[d]) * bf16_to_double(xr[d]);
                gate = 1.0 / (1.0 + exp(-z));
            }
            swiglu_expert(xr, shared_gate_up, shared_down, D, I_s, h, o);
            for (int d = 0; d < D; ++d) y[d] += gate * o[d];
        }
        if (residual)
            for (int d = 0; d < D; ++d) y[d] += bf16_to_double(residual[(size_t)t * D + d]);
    }
    free(h);
    free(o);
    return 0;
}

/* The whole block for the listed rows: route each listed token, then combine.
 * idx_out/w_out/logits_out ([nrows, k], [nrows, k], [nrows, E]) may be NULL. */
int oracle_forward_rows(const uint16_t *x, const uint16_t *W_r, const float *bias,
                        const uint16_t *W_gu, const uint16_t *W_dn,
                        const int32_t *rows, int nrows, int T, int D, int E, int k, int I,
                        int norm, const uint16_t *shared_gate_up, const uint16_t *shared_down,
                        const uint16_t *shared_gate, int I_s, const uint16_t *residual,
                        double *y_out, int32_t *idx_out, float *w_out, float *logits_out) {
    if (!x || !W_r || !rows || !y_out || nrows < 0 || T < 0 || k <= 0 || k > E) return 1;
    int rc = 0;
    /* route one row at a time into a full-size routing table so combine can index it */
    int32_t *idx_all = (int32_t *)malloc(sizeof(int32_t) * (size_t)T * k);
    float *w_all = (float *)malloc(sizeof(float) * (size_t)T * k);
    float *l = (float *)malloc(sizeof(float) * (size_t)E);
    if (!idx_all || !w_all || !l) { rc = 2; goto done; }
    for (long a = 0; a < (long)T * k; ++a) { idx_all[a] = 0; w_all[a] = 0.0f; }
    for (int n = 0; n < nrows; ++n) {
        int t = rows[n];
        if (t < 0 || t >= T) { rc = 1; goto done; }
        rc = oracle_router_logits(x + (size_t)t * D, W_r, bias, 1, D, E, l);
        if (rc) goto done;
        rc = oracle_select(l, 1, E, k, norm, idx_all + (size_t)t * k, w_all + (size_t)t * k);
        if (rc) goto done;
        if (idx_out) memcpy(idx_out + (size_t)n * k, idx_all + (size_t)t * k, sizeof(int32_t) * k);
        if (w_out) memcpy(w_out + (size_t)n * k, w_all + (size_t)t * k, sizeof(float) * k);
        if (logits_out) memcpy(logits_out + (size_t)n * E, l, sizeof(float) * E);
    }
    rc = oracle_combine_rows(x, idx_all, w_all, rows, nrows, T, D, E, k, I, W_gu, W_dn,
                             shared_gate_up, shared_down, shared_gate, I_s, residual, y_out);
done:
    free(idx_all);
    free(w_all);
    free(l);
    return rc;
}

/* The loop dispatch of "27. Mixture of experts", section "Dispatch" (forward_loop): for
 * each expert that any token chose, gather its tokens, run the expert on the gathered rows
 * as a small matrix product, scale by the routing weight and scatter-add into y.  Written
 * independently of swiglu_expert so that "loop dispatch == per-token definition" is a
 * real cross-check.  y_out: [T, D] double (all tokens). */
int oracle_loop_dispatch(const uint16_t *x, const int32_t *idx, const float *w, int T, int D,
                         int E, int k, int I, const uint16_t *W_gu, const uint16_t *W_dn,
                         double *y_out) {
    if (!x || !idx || !w || !W_gu || !W_dn || !y_out) return 1;
    for (long q = 0; q < (long)T * D; ++q) y_out[q] = 0.0;
    int *tok = (int *)malloc(sizeof(int) * (size_t)(T > 0 ? T : 1));
    int *slot = (int *)malloc(sizeof(int) * (size_t)(T > 0 ? T : 1));
    double *G = (double *)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1) * 2 * I);
    double *H = (double *)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1) * I);
    if (!tok || !slot || !G || !H) { free(tok); free(slot); free(G); free(H); return 2; }
    for (int e = 0; e < E; ++e) {
        int m = 0;                                   /* gather: torch.where(experts == e) */
        for (int t = 0; t < T; ++t)
            for (int j = 0; j < k; ++j)
                if (idx[(size_t)t * k + j] == e) { tok[m] = t; slot[m] = j; ++m; }
        if (m == 0) continue;
        const uint16_t *Wg = W_gu + (size_t)e * 2 * I * D;
        const uint16_t *Wd = W_dn + (size_t)e * D * I;
        /* G = X_e W_gu^T : [m, 2I] */
        for (int r = 0; r < m; ++r)
            for (int c = 0; c < 2 * I; ++c) {
                double s = 0.0;
                for (int d = 0; d < D; ++d)
                    s += bf16_to_double(x[(size_t)tok[r] * D + d]) * bf16_to_double(Wg[(size_t)c * D + d]);
                G[(size_t)r * 2 * I + c] = s;
            }
        /* chunk(2): first I columns gate, last I columns up */
        for (int r = 0; r < m; ++r)
            for (int i = 0; i < I; ++i) {
                double g = G[(size_t)r * 2 * I + i], u = G[(size_t)r * 2 * I + I + i];
                H[(size_t)r * I + i] = (g / (1.0 + exp(-g))) * u;
            }
        /* out = H W_dn^T, scaled by the routing weight, index_add_ into y */
        for (int r = 0; r < m; ++r) {
            double wr = (double)w[(size_t)tok[r] * k + slot[r]];
            for (int d = 0; d < D; ++d) {
                double s = 0.0;
                for (int i = 0; i < I; ++i) s += H[(size_t)r * I + i] * bf16_to_double(Wd[(size_t)d * I + i]);
                y_out[(size_t)tok[r] * D + d] += wr * s;
            }
        }
    }
    free(tok); free(slot); free(G); free(H);
    return 0;
}

/* ---------------------------------------------------------------- FP8 weight-only experts */

/* Low-precision experts ("27. Mixture of experts", section "The economics of MoE
 * inference"; "Qwen3-VL and Mixture of Experts", section "Deploying it").  The pages fix no
 * format; the reading taken is per-row E4M3 (OCP "e4m3fn": sign, 4 exponent bits with bias 7,
 * 3 mantissa bits; no infinities, largest value 448):
 *   scale[r] = amax_c |W[r, c]| / 448 in FP32 (1 when the row is all zero),
 *   q[r, c]  = E4M3 of the FP32 quotient W[r, c] / scale[r], nearest-even, saturated to 448,
 *   weight   = scale[r] * value(q[r, c]).                                                   */

/* The value of an E4M3 code (NaN for the two NaN codes). */
double oracle_e4m3_value(uint8_t code) {
    int s = code >> 7, e = (code >> 3) & 15, m = code & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m, -9);                 /* subnormal: m / 8 * 2^(1 - 7) */
    else v = ldexp(1.0 + m / 8.0, e - 7);
    return s ? -v : v;
}

/* The E4M3 code of a finite FP32 value: nearest, ties to even mantissa, saturated to 448. */
static uint8_t e4m3_encode(float f) {
    uint8_t sign = signbit(f) ? 0x80 : 0x00;
    double a = fabs((double)f);
    if (a >= 448.0) return sign | 0x7E;                  /* 448 = 2^8 * 1.75 */
    if (a < ldexp(1.0, -6)) {                            /* below the smallest normal: steps of 2^-9 */
        double m = nearbyint(ldexp(a, 9));               /* 0..8; 8 is the smallest normal's code */
        return sign | (uint8_t)m;
    }
    int E;
    double f2 = frexp(a, &E);                            /* a = f2 * 2^E, f2 in [0.5, 1) */
    int e = E - 1;                                       /* a = (2 f2) * 2^e, 2 f2 in [1, 2) */
    double m = nearbyint((2.0 * f2 - 1.0) * 8.0);        /* mantissa step, ties to even */
    if (m == 8.0) { m = 0.0; e += 1; }
    if (e > 8 || (e == 8 && m > 6.0)) return sign | 0x7E;
    return sign | (uint8_t)(((e + 7) << 3) | (int)m);
}

int oracle_quantize_fp8_rows(const uint16_t *W, long rows, int cols, uint8_t *q, float *scale) {
    if (!W || !q || !scale || rows < 0 || cols <= 0) return 1;
    for (long r = 0; r < rows; ++r) {
        const uint16_t *w = W + (size_t)r * cols;
        float amax = 0.0f;
        for (int c = 0; c < cols; ++c) {
            float a = fabsf((float)bf16_to_double(w[c]));
            if (a > amax) amax = a;
        }
        volatile float s = amax > 0.0f ? amax / 448.0f : 1.0f;   /* one FP32 division */
        scale[r] = s;
        for (int c = 0; c < cols; ++c) {
            volatile float v = (float)bf16_to_double(w[c]) / s;  /* one FP32 division */
            q[(size_t)r * cols + c] = e4m3_encode(v);
        }
    }
    return 0;
}

/* One SwiGLU expert with FP8 weights (as swiglu_expert; weight = scale[row] * value(q)). */
static void swiglu_expert_fp8(const uint16_t *x_row, const uint8_t *q_gu, const float *s_gu,
                              const uint8_t *q_dn, const float *s_dn, int D, int I, double *h,
                              double *out) {
    for (int i = 0; i < I; ++i) {
        double g = 0.0, u = 0.0;
        for (int d = 0; d < D; ++d) {
            double xd = bf16_to_double(x_row[d]);
            g += oracle_e4m3_value(q_gu[(size_t)i * D + d]) * xd;
            u += oracle_e4m3_value(q_gu[(size_t)(I + i) * D + d]) * xd;
        }
        g *= (double)s_gu[i];
        u *= (double)s_gu[I + i];
        h[i] = g / (1.0 + exp(-g)) * u;
    }
    for (int d = 0; d < D; ++d) {
        double s = 0.0;
        for (int i = 0; i < I; ++i) s += oracle_e4m3_value(q_dn[(size_t)d * I + i]) * h[i];
        out[d] = s * (double)s_dn[d];
    }
}

/* y for the listed token rows with FP8 routed experts (no shared expert):
 *   y[t] = sum_{j<k} w[t,j] * expert_{idx[t,j]}(x[t]) (+ residual[t]);
 * q_gu [E, 2I, D], s_gu [E * 2I], q_dn [E, D, I], s_dn [E * D]. */
int oracle_combine_rows_fp8(const uint16_t *x, const int32_t *idx, const float *w,
                            const int32_t *rows, int nrows, int T, int D, int E, int k, int I,
                            const uint8_t *q_gu, const float *s_gu, const uint8_t *q_dn,
                            const float *s_dn, const uint16_t *residual, double *y_out) {
    if (!x || !idx || !w || !rows || !q_gu || !s_gu || !q_dn || !s_dn || !y_out || D <= 0 || I <= 0 || k <= 0)
        return 1;
    double *h = (double *)malloc(sizeof(double) * (size_t)I);
    double *o = (double *)malloc(sizeof(double) * (size_t)D);
    if (!h || !o) { free(h); free(o); return 2; }
    for (int n = 0; n < nrows; ++n) {
        int t = rows[n];
        if (t < 0 || t >= T) { free(h); free(o); return 1; }
        const uint16_t *xr = x + (size_t)t * D;
        double *y = y_out + (size_t)n * D;
        for (int d = 0; d < D; ++d) y[d] = 0.0;
        for (int j = 0; j < k; ++j) {
            int e = idx[(size_t)t * k + j];
            if (e < 0 || e >= E) { free(h); free(o); return 1; }
            swiglu_expert_fp8(xr, q_gu + (size_t)e * 2 * I * D, s_gu + (size_t)e * 2 * I,
                              q_dn + (size_t)e * D * I, s_dn + (size_t)e * D, D, I, h, o);
            double wj = (double)w[(size_t)t * k + j];
            for (int d = 0; d < D; ++d) y[d] += wj * o[d];
        }
        if (residual)
            for (int d = 0; d < D; ++d) y[d] += bf16_to_double(residual[(size_t)t * D + d]);
    }
    free(h);
    free(o);
    return 0;
}

/* ---------------------------------------------------------------- Switch balance loss
 *
 * "Qwen3-VL and Mixture of Experts" (gopikrishnatummala.com), the list of fixes for expert
 * collapse, "An auxiliary balance loss": L = alpha * N * sum_i f_i P_i over the N experts,
 * f_i the fraction of tokens sent to expert i and P_i the router's average probability for
 * it.  The Qwen3-VL MoE walk-through (agent.csdn.net), "load_balancing_loss_func": the
 * probabilities are the softmax of the gate logits, f comes from the one-hot of the top-k
 * selection averaged over tokens (so each token adds 1/T for each of its k experts:
 * f_i = count_i / T), P_i is the mean probability over tokens, and the sum of their products
 * is multiplied by the number of experts.
 * Reading taken: alpha is the caller's coefficient; the selection is the given top-k
 * (the forward's); the gradient treats f as a constant (the selection is not
 * differentiable): dL/dl[t, e] = alpha * N / T * p[t, e] * (f_e - sum_i f_i p[t, i]).
 * Everything in double from the FP32 logits. */
int oracle_aux_loss(const float *logits, const int32_t *idx, int T, int E, int k, double alpha,
                    double *loss, double *dlogits) {
    if (T < 1 || E < 1 || k < 1) return 1;
    double *f = (double *)calloc((size_t)E, sizeof(double));
    double *P = (double *)calloc((size_t)E, sizeof(double));
    double *p = (double *)malloc((size_t)E * sizeof(double));
    if (!f || !P || !p) { free(f); free(P); free(p); return 1; }
    for (int t = 0; t < T; ++t) {
        for (int j = 0; j < k; ++j) {
            int e = idx[(size_t)t * k + j];
            if (e < 0 || e >= E) { free(f); free(P); free(p); return 1; }
            f[e] += 1.0;
        }
        softmax_row(logits + (size_t)t * E, E, p);
        for (int e = 0; e < E; ++e) P[e] += p[e];
    }
    double sum = 0.0;
    for (int e = 0; e < E; ++e) {
        f[e] /= (double)T;
        P[e] /= (double)T;
        sum += f[e] * P[e];
    }
    *loss = alpha * (double)E * sum;
    if (dlogits) {
        const double c = alpha * (double)E / (double)T;
        for (int t = 0; t < T; ++t) {
            softmax_row(logits + (size_t)t * E, E, p);
            double q = 0.0;
            for (int i = 0; i < E; ++i) q += f[i] * p[i];
            for (int e = 0; e < E; ++e) dlogits[(size_t)t * E + e] = c * p[e] * (f[e] - q);
        }
    }
    free(f);
    free(P);
    free(p);
    return 0;
}

/* ---------------------------------------------------------------- backward ----------- */

/* The backward pass of the routed block for a given routing, all in double.
 * "Qwen3-VL and Mixture of Experts", "How the router and experts learn", "What gets trained":
 * only the experts a token chose receive its gradient, and the router learns through the
 * gate weights; the selection itself is held fixed (it is piecewise constant).  The function
 * differentiated is the plain definition (unrounded logits, double softmax, SwiGLU experts),
 * with loss sum_t dy[t] . y[t].  Per token t with routing idx[t, 0..k-1]:
 *   p = softmax(W_r x + b);  S = sum_j p[idx_j];  w_j = p[idx_j] / S  (norm)  or  p[idx_j]
 *   for each slot j, e = idx_j:   g = W_gate[e] x,  u = W_up[e] x,  s = sigmoid(g),
 *                                 h = g s u,        y += w_j W_down[e] h
 *     z   = W_down[e]^T dy            dw_j = h . z           dh = w_j z
 *     dg  = dh u s (1 + g (1 - s))    du   = dh g s
 *     dx += W_gate[e]^T dg + W_up[e]^T du
 *     dW_down[e] += (w_j dy) h^T,  dW_gate[e] += dg x^T,  dW_up[e] += du x^T
 *   dp_j = (dw_j - sum_m dw_m w_m) / S  (norm)  or  dw_j
 *   dl_e = p_e (dp_e - sum_j p[idx_j] dp_j)   (dp_e = 0 for experts not chosen)
 *          (+ dlogits_add[t, e], e.g. the balance loss's gradient)
 *   dW_r += dl x^T,  db += dl,  dx += W_r^T dl   (+ dy when residual)
 * Inputs: x [T, D], W_r [E, D], W_gu [E, 2I, D], W_dn [E, D, I], dy [T, D] as bf16 bit
 * patterns; bias [E] float or NULL; idx [T, k]; dlogits_add [T, E] double or NULL.
 * Outputs (double, overwritten; any may be NULL): dx [T, D], dW_r [E, D], db [E],
 * dlogits [T, E], dw [T, k], and the weight gradients of the n_exp experts listed in
 * experts[]: dW_gu [n_exp, 2I, D], dW_dn [n_exp, D, I]. */
int oracle_backward(const uint16_t *x, const uint16_t *W_r, const float *bias,
                    const uint16_t *W_gu, const uint16_t *W_dn, const uint16_t *dy,
                    const int32_t *idx, int T, int D, int E, int k, int I, int norm, int residual,
                    const double *dlogits_add, double *dx, double *dW_r, double *db,
                    double *dlogits, double *dw, const int32_t *experts, int n_exp,
                    double *dW_gu, double *dW_dn) {
    if (T < 1 || D < 1 || E < 1 || k < 1 || k > E || I < 1 || n_exp < 0) return 1;
    double *xd = (double *)malloc((size_t)D * sizeof(double));
    double *dyd = (double *)malloc((size_t)D * sizeof(double));
    double *dxt = (double *)malloc((size_t)D * sizeof(double));
    double *l = (double *)malloc((size_t)E * sizeof(double));
    double *p = (double *)malloc((size_t)E * sizeof(double));
    double *dl = (double *)malloc((size_t)E * sizeof(double));
    double *dpe = (double *)malloc((size_t)E * sizeof(double));
    double *g = (double *)malloc((size_t)I * sizeof(double));
    double *u = (double *)malloc((size_t)I * sizeof(double));
    double *z = (double *)malloc((size_t)I * sizeof(double));
    double *dg = (double *)malloc((size_t)I * sizeof(double));
    double *du = (double *)malloc((size_t)I * sizeof(double));
    double *h = (double *)malloc((size_t)I * sizeof(double));
    double *wj = (double *)malloc((size_t)k * sizeof(double));
    double *dwj = (double *)malloc((size_t)k * sizeof(double));
    int *slot_of = (int *)malloc((size_t)E * sizeof(int));
    int rc = 0;
    if (!xd || !dyd || !dxt || !l || !p || !dl || !dpe || !g || !u || !z || !dg || !du || !h || !wj ||
        !dwj || !slot_of) { rc = 1; goto done; }
    for (int e = 0; e < E; ++e) slot_of[e] = -1;
    for (int m = 0; m < n_exp; ++m) {
        if (experts[m] < 0 || experts[m] >= E) { rc = 1; goto done; }
        slot_of[experts[m]] = m;
    }
    if (dW_r) memset(dW_r, 0, (size_t)E * D * sizeof(double));
    if (db) memset(db, 0, (size_t)E * sizeof(double));
    if (dW_gu) memset(dW_gu, 0, (size_t)n_exp * 2 * I * D * sizeof(double));
    if (dW_dn) memset(dW_dn, 0, (size_t)n_exp * D * I * sizeof(double));
    for (int t = 0; t < T; ++t) {
        const int32_t *it = idx + (size_t)t * k;
        for (int j = 0; j < k; ++j)
            if (it[j] < 0 || it[j] >= E) { rc = 1; goto done; }
        for (int d = 0; d < D; ++d) {
            xd[d] = bf16_to_double(x[(size_t)t * D + d]);
            dyd[d] = bf16_to_double(dy[(size_t)t * D + d]);
            dxt[d] = residual ? dyd[d] : 0.0;
        }
        /* router: unrounded logits, softmax over all E, the given selection's weights */
        double mx = -INFINITY;
        for (int e = 0; e < E; ++e) {
            double s = 0.0;
            for (int d = 0; d < D; ++d) s += bf16_to_double(W_r[(size_t)e * D + d]) * xd[d];
            if (bias) s += (double)bias[e];
            l[e] = s;
            if (s > mx) mx = s;
        }
        double Z = 0.0;
        for (int e = 0; e < E; ++e) { p[e] = exp(l[e] - mx); Z += p[e]; }
        for (int e = 0; e < E; ++e) p[e] /= Z;
        double S = 0.0;
        for (int j = 0; j < k; ++j) S += p[it[j]];
        for (int j = 0; j < k; ++j) wj[j] = norm ? p[it[j]] / S : p[it[j]];
        /* experts */
        for (int j = 0; j < k; ++j) {
            const int e = it[j];
            const uint16_t *Wg = W_gu + (size_t)e * 2 * I * D, *Wu = Wg + (size_t)I * D;
            const uint16_t *Wd = W_dn + (size_t)e * D * I;
            for (int i = 0; i < I; ++i) {
                double gs = 0.0, us = 0.0;
                for (int d = 0; d < D; ++d) {
                    gs += bf16_to_double(Wg[(size_t)i * D + d]) * xd[d];
                    us += bf16_to_double(Wu[(size_t)i * D + d]) * xd[d];
                }
                g[i] = gs;
                u[i] = us;
                z[i] = 0.0;
            }
            for (int d = 0; d < D; ++d)
                for (int i = 0; i < I; ++i) z[i] += bf16_to_double(Wd[(size_t)d * I + i]) * dyd[d];
            double dws = 0.0;
            for (int i = 0; i < I; ++i) {
                const double s = 1.0 / (1.0 + exp(-g[i]));
                h[i] = g[i] * s * u[i];
                dws += h[i] * z[i];
                const double dh = wj[j] * z[i];
                dg[i] = dh * u[i] * s * (1.0 + g[i] * (1.0 - s));
                du[i] = dh * g[i] * s;
            }
            dwj[j] = dws;
            for (int i = 0; i < I; ++i)
                for (int d = 0; d < D; ++d)
                    dxt[d] += bf16_to_double(Wg[(size_t)i * D + d]) * dg[i] +
                              bf16_to_double(Wu[(size_t)i * D + d]) * du[i];
            const int m = slot_of[e];
            if (m >= 0 && dW_gu)
                for (int i = 0; i < I; ++i)
                    for (int d = 0; d < D; ++d) {
                        dW_gu[((size_t)m * 2 * I + i) * D + d] += dg[i] * xd[d];
                        dW_gu[((size_t)m * 2 * I + I + i) * D + d] += du[i] * xd[d];
                    }
            if (m >= 0 && dW_dn)
                for (int d = 0; d < D; ++d)
                    for (int i = 0; i < I; ++i) dW_dn[((size_t)m * D + d) * I + i] += wj[j] * dyd[d] * h[i];
        }
        if (dw)
            for (int j = 0; j < k; ++j) dw[(size_t)t * k + j] = dwj[j];
        /* routing weights -> chosen probabilities -> logits */
        double sdw = 0.0;
        for (int j = 0; j < k; ++j) sdw += dwj[j] * wj[j];
        for (int e = 0; e < E; ++e) dpe[e] = 0.0;
        for (int j = 0; j < k; ++j) dpe[it[j]] += norm ? (dwj[j] - sdw) / S : dwj[j];
        double pdp = 0.0;
        for (int e = 0; e < E; ++e) pdp += p[e] * dpe[e];
        for (int e = 0; e < E; ++e) {
            dl[e] = p[e] * (dpe[e] - pdp);
            if (dlogits_add) dl[e] += dlogits_add[(size_t)t * E + e];
            if (dlogits) dlogits[(size_t)t * E + e] = dl[e];
            if (db) db[e] += dl[e];
        }
        for (int e = 0; e < E; ++e)
            for (int d = 0; d < D; ++d) {
                const double wr = bf16_to_double(W_r[(size_t)e * D + d]);
                dxt[d] += wr * dl[e];
                if (dW_r) dW_r[(size_t)e * D + d] += dl[e] * xd[d];
            }
        if (dx) memcpy(dx + (size_t)t * D, dxt, (size_t)D * sizeof(double));
    }
done:
    free(xd); free(dyd); free(dxt); free(l); free(p); free(dl); free(dpe); free(g); free(u); free(z);
    free(dg); free(du); free(h); free(wj); free(dwj); free(slot_of);
    return rc;
}

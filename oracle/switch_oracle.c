/*
 * switch_oracle.c -- plain fp64 CPU oracle for the Switch Transformer sparse
 * FFN layer forward pass.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file; only the test-suite, the smoke check and the benchmark's
 * CPU-baseline leg use it.  It shares no code, header or helper with the CUDA
 * library.
 *
 * Every step is the plain definition, in the order the sources give it, in
 * double precision, with no blocking, fusion or reordering:
 *
 *   logits     h(x) = W_r . x                       (llm-papers-study
 *              "精读 06 | Switch Transformers", §3.1, router logits; Incredible.AI
 *              "Switch Transformer - Scaling to Trillion Parameter Models",
 *              section "Router Implementation")
 *   gate       p_i(x) = exp(h_i) / sum_j exp(h_j)   (llm-papers-study §3.1,
 *              softmax formula), evaluated with the row maximum subtracted,
 *              which leaves every p_i unchanged in exact arithmetic
 *   top-1      i* = argmax_i p_i(x), lowest index on ties (llm-papers-study
 *              §3.2; the tie rule is not stated by the sources)
 *   capacity   C = ceil(T / N * c)                  (llm-papers-study §3.4
 *              expert-capacity formula; rounding reading: ceil)
 *   overflow   tokens beyond the first C routed to an expert, in token order,
 *              are dropped (Incredible.AI "MoE Layer"; kasblo "Expert
 *              Capacityはtokenの受付上限"; byhand.ai "Switch Transformer by
 *              Hand", walkthrough step 7)
 *   aux        N * sum_i f_i P_i, f_i = count_i / T before capacity,
 *              P_i = mean over all T tokens of p_i  (llm-papers-study §3.3)
 *   output     y = p_{i*}(x) * E_{i*}(x),  E(x) = W_out . ReLU(W_in . x);
 *              y = 0 for a dropped token (llm-papers-study §3.2 and §3.4)
 *
 * Element types: activations and expert weights are read either as IEEE
 * binary32 (dtype 0) or as bfloat16 bit patterns (dtype 1); both convert to
 * double exactly.  The router weight and the optional logit bias are binary32.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_F32 0
#define ORACLE_BF16 1

/* Exact conversion of element i of a binary32 or bfloat16 array to double. */
static double load_elem(const void *base, int dtype, int64_t i)
{
    if (dtype == ORACLE_BF16) {
        uint16_t bits = ((const uint16_t *)base)[i];
        uint32_t wide = (uint32_t)bits << 16;
        float f;
        memcpy(&f, &wide, sizeof f);
        return (double)f;
    }
    return (double)((const float *)base)[i];
}

/* Expert capacity C = ceil(T / N * c).  A product within 1e-9 of an integer is
 * taken as that integer, so that e.g. 512/8*1.5 gives 96 whatever the binary
 * rounding of c.  At least 1.  Returns -1 for arguments without meaning. */
int64_t oracle_capacity(int64_t T, int32_t N, double c)
{
    if (T < 0 || N < 1 || !(c > 0.0) || !isfinite(c))
        return -1;
    double exact = (double)T / (double)N * c;
    double nearest = floor(exact + 0.5);
    double cap = fabs(exact - nearest) <= 1e-9 ? nearest : ceil(exact);
    if (cap < 1.0)
        cap = 1.0;
    return (int64_t)cap;
}

/* Router logits h[t,i] = sum_k x[t,k] * W_r[i,k] (+ bias[i]), all in double.
 * x is [T,d] row-major, W_r is [N,d] row-major, h is [T,N]. */
void oracle_router_logits(int64_t T, int32_t d, int32_t N, const void *x, int x_dtype,
                          const float *w_r, const float *bias, double *h)
{
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        for (int32_t i = 0; i < N; ++i) {
            double acc = 0.0;
            for (int32_t k = 0; k < d; ++k)
                acc += load_elem(x, x_dtype, t * (int64_t)d + k) * (double)w_r[(int64_t)i * d + k];
            if (bias)
                acc += (double)bias[i];
            h[t * (int64_t)N + i] = acc;
        }
    }
}

/* Softmax, top-1 and gate for every row of h[T,N].
 *   expert[t] = lowest i with h[t,i] equal to the row maximum
 *   gate[t]   = p[t, expert[t]]
 *   margin[t] = row maximum minus the largest logit of any other expert
 *               (+inf when N == 1)
 *   prob_sum[i] = sum over t of p[t,i], accumulated in token order
 *   probs (optional, [T,N]) receives every p[t,i]. */
void oracle_softmax_top1(int64_t T, int32_t N, const double *h, int32_t *expert, double *gate,
                         double *margin, double *prob_sum, double *probs)
{
    double *p = probs ? probs : (double *)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1) * (size_t)N);
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        const double *row = h + t * (int64_t)N;
        double m = row[0];
        int32_t arg = 0;
        for (int32_t i = 1; i < N; ++i) {
            if (row[i] > m) {
                m = row[i];
                arg = i;
            }
        }
        double runner_up = -INFINITY;
        for (int32_t i = 0; i < N; ++i)
            if (i != arg && row[i] > runner_up)
                runner_up = row[i];
        double denom = 0.0;
        for (int32_t i = 0; i < N; ++i)
            denom += exp(row[i] - m);
        for (int32_t i = 0; i < N; ++i)
            p[t * (int64_t)N + i] = exp(row[i] - m) / denom;
        expert[t] = arg;
        gate[t] = p[t * (int64_t)N + arg];
        margin[t] = (N == 1) ? INFINITY : m - runner_up;
    }
    for (int32_t i = 0; i < N; ++i)
        prob_sum[i] = 0.0;
    for (int64_t t = 0; t < T; ++t)
        for (int32_t i = 0; i < N; ++i)
            prob_sum[i] += p[t * (int64_t)N + i];
    if (!probs)
        free(p);
}

/* Capacity assignment in token order.
 *   counts[i]         = number of tokens routed to expert i (before capacity)
 *   slot[t]           = number of earlier tokens routed to the same expert,
 *                       or -1 when that number is >= C (dropped)
 *   slot_token[i*C+s] = the token holding slot s of expert i, -1 if empty. */
void oracle_assign(int64_t T, int32_t N, int64_t C, const int32_t *expert, int32_t *slot,
                   int32_t *counts, int32_t *slot_token)
{
    for (int32_t i = 0; i < N; ++i)
        counts[i] = 0;
    for (int64_t s = 0; s < (int64_t)N * C; ++s)
        slot_token[s] = -1;
    for (int64_t t = 0; t < T; ++t) {
        int32_t e = expert[t];
        int32_t position = counts[e];
        counts[e] = position + 1;
        if (position < C) {
            slot[t] = position;
            slot_token[(int64_t)e * C + position] = (int32_t)t;
        } else {
            slot[t] = -1;
        }
    }
}

/* Load-balancing loss without the alpha weight: N * sum_i f_i * P_i with
 * f_i = counts[i] / T and P_i = prob_sum[i] / T. */
double oracle_aux(int64_t T, int32_t N, const int32_t *counts, const double *prob_sum)
{
    double total = 0.0;
    for (int32_t i = 0; i < N; ++i) {
        double f = (double)counts[i] / (double)T;
        double P = prob_sum[i] / (double)T;
        total += f * P;
    }
    return (double)N * total;
}

/* One expert FFN applied to one token and scaled by its gate:
 *   u[j] = max(0, sum_k W_in[j,k] * x[k]),   j < F
 *   y[k] = gate * sum_j W_out[k,j] * u[j],   k < d
 * W_in is [F,d] and W_out is [d,F], both row-major (nn.Linear layout). */
void oracle_expert_row(int32_t d, int32_t F, const void *x_row, int x_dtype, const void *w_in,
                       const void *w_out, int w_dtype, double gate, double *y_row)
{
    double *x = (double *)malloc(sizeof(double) * (size_t)d);
    double *u = (double *)malloc(sizeof(double) * (size_t)F);
    for (int32_t k = 0; k < d; ++k)
        x[k] = load_elem(x_row, x_dtype, k);
    for (int32_t j = 0; j < F; ++j) {
        double acc = 0.0;
        for (int32_t k = 0; k < d; ++k)
            acc += load_elem(w_in, w_dtype, (int64_t)j * d + k) * x[k];
        u[j] = acc > 0.0 ? acc : 0.0;
    }
    for (int32_t k = 0; k < d; ++k) {
        double acc = 0.0;
        for (int32_t j = 0; j < F; ++j)
            acc += load_elem(w_out, w_dtype, (int64_t)k * F + j) * u[j];
        y_row[k] = gate * acc;
    }
    free(x);
    free(u);
}

/* Layer outputs for a list of tokens: row r of y (shape [n_rows, d]) is the
 * output of token rows[r].  Kept tokens go through their expert and are
 * scaled by their gate; dropped tokens (slot -1) get an all-zero row.
 * w_in is [N,F,d] and w_out is [N,d,F]. */
void oracle_output_rows(int32_t d, int32_t F, int64_t n_rows, const int64_t *rows, const void *x,
                        int x_dtype, const void *w_in, const void *w_out, int w_dtype,
                        const int32_t *expert, const int32_t *slot, const double *gate, double *y)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < n_rows; ++r) {
        int64_t t = rows[r];
        double *out = y + r * (int64_t)d;
        if (slot[t] < 0) {
            for (int32_t k = 0; k < d; ++k)
                out[k] = 0.0;
            continue;
        }
        int64_t e = expert[t];
        size_t esize = (w_dtype == ORACLE_BF16) ? 2 : 4;
        const char *win_e = (const char *)w_in + (size_t)e * (size_t)F * (size_t)d * esize;
        const char *wout_e = (const char *)w_out + (size_t)e * (size_t)d * (size_t)F * esize;
        const char *x_t = (const char *)x + (size_t)t * (size_t)d * (x_dtype == ORACLE_BF16 ? 2 : 4);
        oracle_expert_row(d, F, x_t, x_dtype, win_e, wout_e, w_dtype, gate[t], out);
    }
}

/* ------------------------------------------------------------------------
 * Top-2 routing: the classic mixture-of-experts layer that the Switch layer
 * simplifies (Incredible.AI "Switch Transformer - Scaling to Trillion
 * Parameter Models", section "Mixture of Experts Routing"; llm-papers-study
 * "精读 06 | Switch Transformers" §3.1): softmax over the N logits, the k = 2
 * largest probabilities select the experts, and the output is the sum of the
 * selected experts' outputs, each weighted by its own probability (no
 * renormalisation over the selected pair):  y = sum_{i in top-2} p_i(x) E_i(x).
 *
 * Readings where the sources are silent:
 *   - ties: the first choice is the lowest index attaining the largest
 *     logit, the second the lowest index attaining the largest logit among
 *     the other experts;
 *   - capacity applies to (token, choice) assignments: each expert keeps its
 *     first C assignments in the order "every first choice in token order,
 *     then every second choice in token order", so that first choices get
 *     exactly the slots of top-1 routing;
 *   - the aux loss keeps its definition, f_i counting the tokens whose argmax
 *     (first choice) is expert i (llm-papers-study §3.3).
 * ------------------------------------------------------------------------ */

/* Softmax and top-2 for every row of h[T,N] (N >= 2).
 *   expert2[2t], expert2[2t+1] = first and second choice of token t
 *   gate2[2t],   gate2[2t+1]   = their probabilities p[t, choice]
 *   margin2[2t]   = largest logit minus the second largest (first choice gap)
 *   margin2[2t+1] = second largest minus the third largest (+inf when N == 2)
 *   prob_sum[i]   = sum over t of p[t,i], in token order
 *   probs (optional, [T,N]) receives every p[t,i]. */
void oracle_softmax_top2(int64_t T, int32_t N, const double *h, int32_t *expert2, double *gate2,
                         double *margin2, double *prob_sum, double *probs)
{
    double *p = probs ? probs : (double *)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1) * (size_t)N);
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        const double *row = h + t * (int64_t)N;
        int32_t first = 0;
        for (int32_t i = 1; i < N; ++i)
            if (row[i] > row[first])
                first = i;
        int32_t second = -1;
        for (int32_t i = 0; i < N; ++i)
            if (i != first && (second < 0 || row[i] > row[second]))
                second = i;
        double third = -INFINITY;
        for (int32_t i = 0; i < N; ++i)
            if (i != first && i != second && row[i] > third)
                third = row[i];
        double m = row[first];
        double denom = 0.0;
        for (int32_t j = 0; j < N; ++j)
            denom += exp(row[j] - m);
        for (int32_t j = 0; j < N; ++j)
            p[t * (int64_t)N + j] = exp(row[j] - m) / denom;
        expert2[2 * t] = first;
        expert2[2 * t + 1] = second;
        gate2[2 * t] = p[t * (int64_t)N + first];
        gate2[2 * t + 1] = p[t * (int64_t)N + second];
        margin2[2 * t] = row[first] - row[second];
        margin2[2 * t + 1] = (N == 2) ? INFINITY : row[second] - third;
    }
    for (int32_t i = 0; i < N; ++i)
        prob_sum[i] = 0.0;
    for (int64_t t = 0; t < T; ++t)
        for (int32_t i = 0; i < N; ++i)
            prob_sum[i] += p[t * (int64_t)N + i];
    if (!probs)
        free(p);
}

/* Capacity assignment of top-2 choices.  Assignments are taken in the order
 * (t = 0, first), (t = 1, first), ..., (t = T-1, first), (t = 0, second), ...,
 * (t = T-1, second); each takes the next slot of its expert, or is dropped
 * (slot -1) when the expert already holds C assignments.
 *   counts[i]       = assignments routed to expert i over both choices,
 *                     before capacity
 *   counts_first[i] = tokens whose first choice is expert i
 *   slot2[2t+c]     = slot of choice c of token t, or -1
 *   slot_token[i*C+s] = the token holding slot s of expert i, -1 if empty. */
void oracle_assign_top2(int64_t T, int32_t N, int64_t C, const int32_t *expert2, int32_t *slot2,
                        int32_t *counts, int32_t *counts_first, int32_t *slot_token)
{
    for (int32_t i = 0; i < N; ++i) {
        counts[i] = 0;
        counts_first[i] = 0;
    }
    for (int64_t s = 0; s < (int64_t)N * C; ++s)
        slot_token[s] = -1;
    for (int c = 0; c < 2; ++c) {
        for (int64_t t = 0; t < T; ++t) {
            int32_t e = expert2[2 * t + c];
            int32_t position = counts[e];
            counts[e] = position + 1;
            if (c == 0)
                counts_first[e] += 1;
            if (position < C) {
                slot2[2 * t + c] = position;
                slot_token[(int64_t)e * C + position] = (int32_t)t;
            } else {
                slot2[2 * t + c] = -1;
            }
        }
    }
}

/* Top-2 layer outputs for a list of tokens: row r of y is
 *   sum over the kept choices c of token rows[r] of gate2[2t+c] * E_{expert2[2t+c]}(x_t),
 * first choice first, all in double; an all-zero row when both were dropped. */
void oracle_output_rows_top2(int32_t d, int32_t F, int64_t n_rows, const int64_t *rows, const void *x,
                             int x_dtype, const void *w_in, const void *w_out, int w_dtype,
                             const int32_t *expert2, const int32_t *slot2, const double *gate2, double *y)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < n_rows; ++r) {
        int64_t t = rows[r];
        double *out = y + r * (int64_t)d;
        double *part = (double *)malloc(sizeof(double) * (size_t)d);
        for (int32_t k = 0; k < d; ++k)
            out[k] = 0.0;
        size_t esize = (w_dtype == ORACLE_BF16) ? 2 : 4;
        const char *x_t = (const char *)x + (size_t)t * (size_t)d * (x_dtype == ORACLE_BF16 ? 2 : 4);
        for (int c = 0; c < 2; ++c) {
            if (slot2[2 * t + c] < 0)
                continue;
            int64_t e = expert2[2 * t + c];
            const char *win_e = (const char *)w_in + (size_t)e * (size_t)F * (size_t)d * esize;
            const char *wout_e = (const char *)w_out + (size_t)e * (size_t)d * (size_t)F * esize;
            oracle_expert_row(d, F, x_t, x_dtype, win_e, wout_e, w_dtype, gate2[2 * t + c], part);
            for (int32_t k = 0; k < d; ++k)
                out[k] += part[k];
        }
        free(part);
    }
}

/* Router statistics that the sources list for monitoring a Switch layer
 * next to its loss (kasblo "Switch Transformerとは？", end of section "補助
 * 負荷分散lossは何を均等にするのか": tokens per expert, use of capacity, the
 * overflow / dropped-token rate, the entropy of the router probabilities):
 *   out[0] = mean over the T tokens of -sum_i p_i ln p_i   (0 ln 0 = 0)
 *   out[1] = dropped-token fraction  sum_i max(0, counts_i - C) / T
 *   out[2] = capacity utilisation    sum_i min(counts_i, C) / (N C)
 *   out[3] = busiest expert's load over the uniform load, max_i counts_i N / T
 * probs is [T,N]; every value is 0 when T == 0. */
void oracle_router_stats(int64_t T, int32_t N, int64_t C, const double *probs, const int32_t *counts, double *out)
{
    for (int k = 0; k < 4; ++k)
        out[k] = 0.0;
    if (T <= 0)
        return;
    double entropy = 0.0;
    for (int64_t t = 0; t < T; ++t) {
        double h = 0.0;
        for (int32_t i = 0; i < N; ++i) {
            double p = probs[t * (int64_t)N + i];
            if (p > 0.0)
                h -= p * log(p);
        }
        entropy += h;
    }
    int64_t dropped = 0, kept = 0, busiest = 0;
    for (int32_t i = 0; i < N; ++i) {
        int64_t c = counts[i];
        dropped += c > C ? c - C : 0;
        kept += c < C ? c : C;
        if (c > busiest)
            busiest = c;
    }
    out[0] = entropy / (double)T;
    out[1] = (double)dropped / (double)T;
    out[2] = (double)kept / ((double)N * (double)C);
    out[3] = (double)busiest * (double)N / (double)T;
}

/* ------------------------------------------------------------------------
 * Backward pass of the top-1 layer.  The forward's loss enters as the
 * upstream gradient dy[T,d] of the layer output y and a scalar g_aux, the
 * upstream gradient of aux (the training loss adds alpha * aux, so g_aux is
 * alpha).  The argmax and the capacity assignment are piecewise constant and
 * pass no gradient; the gradient reaches the router through the selected
 * probability p_{i*}(x) that scales the expert output (kasblo "Switch
 * Transformerとは？", section "argmaxは離散なのに、Routerはなぜ学習できるのか")
 * and, for the aux loss, through P_i only, f_i being a count
 * (llm-papers-study "精读 06 | Switch Transformers" §3.3).  With z = W_in x,
 * u = ReLU(z), o = W_out u and y = p_{i*} o for a kept token:
 *   g_gate = dy . o,   do = p_{i*} dy
 *   dW_out[i*] += do u^T,   du = W_out[i*]^T do,   dz = du (z > 0), 0 elsewhere
 *   dW_in[i*]  += dz x^T,   dx += W_in[i*]^T dz
 *   dp_i = [i = i*] g_gate + g_aux N f_i / T      (g_gate = 0 for a dropped token)
 *   dh_i = p_i (dp_i - sum_j p_j dp_j)             (softmax backward)
 *   dW_r += dh x^T,   db += dh,   dx += W_r^T dh
 * All in double; gradients of weights are summed over tokens in token order.
 * ------------------------------------------------------------------------ */
void oracle_layer_bwd(int64_t T, int32_t d, int32_t F, int32_t N, int64_t C, const void *x, int x_dtype,
                      const float *w_r, const float *bias, const void *w_in, const void *w_out, int w_dtype,
                      const double *dy, double g_aux, double *dx, double *dw_r, double *dbias, double *dw_in,
                      double *dw_out)
{
    int64_t Tn = T > 0 ? T : 1;
    double *h = (double *)malloc(sizeof(double) * (size_t)Tn * (size_t)N);
    double *p = (double *)malloc(sizeof(double) * (size_t)Tn * (size_t)N);
    int32_t *expert = (int32_t *)malloc(sizeof(int32_t) * (size_t)Tn);
    double *gate = (double *)malloc(sizeof(double) * (size_t)Tn);
    double *margin = (double *)malloc(sizeof(double) * (size_t)Tn);
    double *prob_sum = (double *)malloc(sizeof(double) * (size_t)N);
    int32_t *slot = (int32_t *)malloc(sizeof(int32_t) * (size_t)Tn);
    int32_t *counts = (int32_t *)malloc(sizeof(int32_t) * (size_t)N);
    int32_t *slot_token = (int32_t *)malloc(sizeof(int32_t) * (size_t)((int64_t)N * C > 0 ? (int64_t)N * C : 1));
    double *g_gate = (double *)calloc((size_t)Tn, sizeof(double));

    /* forward routing, exactly as the forward pass defines it */
    oracle_router_logits(T, d, N, x, x_dtype, w_r, bias, h);
    oracle_softmax_top1(T, N, h, expert, gate, margin, prob_sum, p);
    oracle_assign(T, N, C, expert, slot, counts, slot_token);

    for (int64_t i = 0; i < T * (int64_t)d; ++i)
        dx[i] = 0.0;
    for (int64_t i = 0; i < (int64_t)N * d; ++i)
        dw_r[i] = 0.0;
    if (dbias)
        for (int32_t i = 0; i < N; ++i)
            dbias[i] = 0.0;
    for (int64_t i = 0; i < (int64_t)N * F * d; ++i) {
        dw_in[i] = 0.0;
        dw_out[i] = 0.0;
    }

    size_t esize = (w_dtype == ORACLE_BF16) ? 2 : 4;
    /* expert path: one expert per thread, its tokens in token order */
#pragma omp parallel for schedule(dynamic, 1)
    for (int32_t e = 0; e < N; ++e) {
        const char *win_e = (const char *)w_in + (size_t)e * (size_t)F * (size_t)d * esize;
        const char *wout_e = (const char *)w_out + (size_t)e * (size_t)d * (size_t)F * esize;
        double *dwin_e = dw_in + (int64_t)e * F * d;
        double *dwout_e = dw_out + (int64_t)e * d * F;
        double *xt = (double *)malloc(sizeof(double) * (size_t)d);
        double *z = (double *)malloc(sizeof(double) * (size_t)F);
        double *u = (double *)malloc(sizeof(double) * (size_t)F);
        double *o = (double *)malloc(sizeof(double) * (size_t)d);
        double *dout = (double *)malloc(sizeof(double) * (size_t)d);
        double *dz = (double *)malloc(sizeof(double) * (size_t)F);
        for (int64_t t = 0; t < T; ++t) {
            if (expert[t] != e || slot[t] < 0)
                continue;
            for (int32_t k = 0; k < d; ++k)
                xt[k] = load_elem(x, x_dtype, t * (int64_t)d + k);
            for (int32_t j = 0; j < F; ++j) {
                double acc = 0.0;
                for (int32_t k = 0; k < d; ++k)
                    acc += load_elem(win_e, w_dtype, (int64_t)j * d + k) * xt[k];
                z[j] = acc;
                u[j] = z[j] > 0.0 ? z[j] : 0.0;
            }
            double gg = 0.0;
            for (int32_t k = 0; k < d; ++k) {
                double acc = 0.0;
                for (int32_t j = 0; j < F; ++j)
                    acc += load_elem(wout_e, w_dtype, (int64_t)k * F + j) * u[j];
                o[k] = acc;
                gg += dy[t * (int64_t)d + k] * acc;
                dout[k] = gate[t] * dy[t * (int64_t)d + k];
            }
            g_gate[t] = gg;
            for (int32_t k = 0; k < d; ++k)
                for (int32_t j = 0; j < F; ++j)
                    dwout_e[(int64_t)k * F + j] += dout[k] * u[j];
            for (int32_t j = 0; j < F; ++j) {
                double acc = 0.0;
                for (int32_t k = 0; k < d; ++k)
                    acc += load_elem(wout_e, w_dtype, (int64_t)k * F + j) * dout[k];
                dz[j] = z[j] > 0.0 ? acc : 0.0;
            }
            for (int32_t j = 0; j < F; ++j)
                for (int32_t k = 0; k < d; ++k)
                    dwin_e[(int64_t)j * d + k] += dz[j] * xt[k];
            for (int32_t k = 0; k < d; ++k) {
                double acc = 0.0;
                for (int32_t j = 0; j < F; ++j)
                    acc += load_elem(win_e, w_dtype, (int64_t)j * d + k) * dz[j];
                dx[t * (int64_t)d + k] += acc;
            }
        }
        free(xt);
        free(z);
        free(u);
        free(o);
        free(dout);
        free(dz);
    }

    /* router: softmax backward per token, then dh into dx, dW_r and db */
    double *dh = (double *)malloc(sizeof(double) * (size_t)Tn * (size_t)N);
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        const double *pt = p + t * (int64_t)N;
        double *dht = dh + t * (int64_t)N;
        double dot = 0.0;
        for (int32_t i = 0; i < N; ++i) {
            double dp = g_aux * (double)N * ((double)counts[i] / (double)T) / (double)T;
            if (i == expert[t])
                dp += g_gate[t];
            dht[i] = dp;
            dot += pt[i] * dp;
        }
        for (int32_t i = 0; i < N; ++i)
            dht[i] = pt[i] * (dht[i] - dot);
        for (int32_t k = 0; k < d; ++k) {
            double router_part = 0.0;
            for (int32_t i = 0; i < N; ++i)
                router_part += dht[i] * w_r[(int64_t)i * d + k]; /* float -> double, exact */
            dx[t * (int64_t)d + k] += router_part;
        }
    }
#pragma omp parallel for schedule(static)
    for (int32_t i = 0; i < N; ++i) {
        for (int64_t t = 0; t < T; ++t) {
            double g = dh[t * (int64_t)N + i];
            for (int32_t k = 0; k < d; ++k)
                dw_r[(int64_t)i * d + k] += g * load_elem(x, x_dtype, t * (int64_t)d + k);
            if (dbias)
                dbias[i] += g;
        }
    }
    free(dh);
    free(h);
    free(p);
    free(expert);
    free(gate);
    free(margin);
    free(prob_sum);
    free(slot);
    free(counts);
    free(slot_token);
    free(g_gate);
}

/* Set the number of OpenMP threads the parallel loops above use (no effect
 * without OpenMP).  Used to time the oracle on one core and on all cores. */
void oracle_set_threads(int n)
{
#ifdef _OPENMP
    extern void omp_set_num_threads(int);
    if (n > 0)
        omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* Number of OpenMP threads the parallel loops above use (1 without OpenMP). */
int oracle_threads(void)
{
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}

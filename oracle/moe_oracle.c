/*
 * moe_oracle.c -- plain, slow CPU reference of one top-k MoE SwiGLU layer forward.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or call this
 * file; only the tests, the smoke check and the benchmark's CPU-baseline leg do.  It
 * shares no code with the CUDA library (no headers, helpers or tables).
 *
 * Precision: the inputs are bf16 bit patterns, widened exactly to double; every sum,
 * exp and product below is in double, with no intermediate rounding.
 *
 * Sources (page title, section, equation):
 *   "MoE" (llm.rainlin.net), section 2 "Router":   r = x W_r^T;  p_t = Softmax(r_t);
 *        I_t = TopK(p_t, K);  alpha_{t,e} = p_{t,e} / sum_{j in I_t} p_{t,j}.
 *   "MoE", section 3:  E_e(x) = W_down (SiLU(W_gate x) (.) W_up x), gate_up weights
 *        stored as one [2f, D] matrix whose first f rows are the gate and last f the up
 *        projection (the expert loop splits F.linear's output in two halves).
 *   "MoE", section 4:  y_t = sum_{e in I_t} alpha_{t,e} E_e(x_t)
 *                            + sigma(w_s^T x_t) E_s(x_t)   (shared expert, optional).
 *   "1.6 混合专家（MoE）" (llm.satori-ai.cn), section 2 worked example: the selected
 *        scores are renormalised among the selected experts only (0.90, 0.60 -> 0.60,
 *        0.40); the unselected experts never enter the forward pass.
 *
 * Readings where the pages are silent: the router logits are not rounded (fp32 or
 * better); top-K ties go to the lower expert index and the selected indices are listed
 * by descending probability; the renormalisation has no epsilon; the shared-expert gate
 * has no bias.  An optional per-expert logit bias b (added to r before the softmax)
 * expresses the synthetic routing regimes.
 *
 * Build: gcc -O2 -ffp-contract=off -fopenmp -shared -fPIC moe_oracle.c -lm
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

static double bf16_to_double(uint16_t bits) {
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static double dot_bf16(const uint16_t* a, const uint16_t* b, int n) {
    double s = 0.0;
    for (int i = 0; i < n; ++i) s += bf16_to_double(a[i]) * bf16_to_double(b[i]);
    return s;
}

static double sigmoid(double z) { return 1.0 / (1.0 + exp(-z)); }

static double silu(double z) { return z * sigmoid(z); }

/* bf16 rounding of a routing weight the way the reference casts it back to the model
 * dtype: the fp32 weight rounded to the nearest bf16, ties to even ("MoE", section 2:
 * the renormalised fp32 scores are converted to the model's bf16). */
static double round_to_bf16(double v) {
    float f = (float)v;
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    u = (u + 0x7FFFu + ((u >> 16) & 1u)) & 0xFFFF0000u;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/*
 * Router ("MoE", section 2; "1.6 混合专家（MoE）", section 2 top-k gating and section 3
 * bias method).  For each token t:
 *   r_t[e]  = x_t . W_r[e]  (+ bias[e])
 *   p_t     = softmax(r_t)          score_mode 0 (max-subtracted, double), or
 *   p_t[e]  = sigma(r_t[e])         score_mode 1 (per-expert sigmoid affinity)
 *   key[e]  = p_t[e] + select_bias[e]   (selection-only bias; 0 when NULL)
 *   I_t     = the K largest keys; ties -> lower e; listed by descending key
 *   alpha   = p_t[I_t] / sum p_t[I_t]   (the raw scores, never the bias)
 *             rounded to bf16 when bf16_weights != 0
 *   gap[t]  = key_(K) - key_(K+1)  (+inf if K == E)
 *   sgate[t]= sigma(w_s . x_t)      (shared-expert scalar gate, "MoE" section 4)
 * Outputs idx [T*K], alpha [T*K]; probs [T*E] (the scores p), gap [T], sgate [T] are
 * optional (NULL).  Returns 0, or -1 on bad arguments.
 */
int oracle_route_ex(const uint16_t* x, const uint16_t* w_r, const double* bias,
                    const uint16_t* w_sg, int T, int D, int E, int K, int score_mode,
                    const double* select_bias, int bf16_weights,
                    int32_t* idx, double* alpha, double* probs, double* gap, double* sgate) {
    if (T < 0 || D <= 0 || E <= 0 || K <= 0 || K > E || score_mode < 0 || score_mode > 1)
        return -1;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int t = 0; t < T; ++t) {
        double* p = (double*)malloc(sizeof(double) * (size_t)E);
        double* key = (double*)malloc(sizeof(double) * (size_t)E);
        char* taken = (char*)calloc((size_t)E, 1);
        if (!p || !key || !taken) { bad = 1; free(p); free(key); free(taken); continue; }
        const uint16_t* xt = x + (size_t)t * D;
        double m = -INFINITY;
        for (int e = 0; e < E; ++e) {
            p[e] = dot_bf16(xt, w_r + (size_t)e * D, D) + (bias ? bias[e] : 0.0);
            if (p[e] > m) m = p[e];
        }
        if (score_mode == 0) {
            double z = 0.0;
            for (int e = 0; e < E; ++e) { p[e] = exp(p[e] - m); z += p[e]; }
            for (int e = 0; e < E; ++e) p[e] /= z;
        } else {
            for (int e = 0; e < E; ++e) p[e] = sigmoid(p[e]);
        }
        for (int e = 0; e < E; ++e) key[e] = p[e] + (select_bias ? select_bias[e] : 0.0);
        if (probs) memcpy(probs + (size_t)t * E, p, sizeof(double) * (size_t)E);

        /* TopK by repeated selection of the largest remaining key. */
        double sel_sum = 0.0;
        for (int k = 0; k < K; ++k) {
            int best = -1;
            for (int e = 0; e < E; ++e)
                if (!taken[e] && (best < 0 || key[e] > key[best])) best = e;
            taken[best] = 1;
            idx[(size_t)t * K + k] = best;
            sel_sum += p[best];
        }
        for (int k = 0; k < K; ++k) {
            double a = p[idx[(size_t)t * K + k]] / sel_sum;
            alpha[(size_t)t * K + k] = bf16_weights ? round_to_bf16(a) : a;
        }
        if (gap) {
            double next = -INFINITY;
            for (int e = 0; e < E; ++e)
                if (!taken[e] && key[e] > next) next = key[e];
            gap[t] = (K == E) ? INFINITY : key[idx[(size_t)t * K + K - 1]] - next;
        }
        if (sgate) sgate[t] = w_sg ? sigmoid(dot_bf16(xt, w_sg, D)) : 0.0;
        free(p);
        free(key);
        free(taken);
    }
    return bad ? -1 : 0;
}

/* The softmax router without selection bias and with fp32 weights (the layer's default). */
int oracle_route(const uint16_t* x, const uint16_t* w_r, const double* bias,
                 const uint16_t* w_sg, int T, int D, int E, int K,
                 int32_t* idx, double* alpha, double* probs, double* gap, double* sgate) {
    return oracle_route_ex(x, w_r, bias, w_sg, T, D, E, K, 0, NULL, 0, idx, alpha, probs, gap,
                           sgate);
}

/*
 * One SwiGLU expert applied to one token ("MoE", section 3), accumulated with a weight:
 *   acc += a * W_down (SiLU(W_gate x) (.) W_up x)
 * w_gu is the expert's [2f, D] gate_up matrix (gate rows first), w_d its [D, f] down
 * matrix.  h is caller scratch of f doubles.
 */
static void expert_accumulate(const uint16_t* xt, const uint16_t* w_gu, const uint16_t* w_d,
                              int D, int f, double a, double* h, double* acc) {
    for (int n = 0; n < f; ++n) {
        double g = dot_bf16(xt, w_gu + (size_t)n * D, D);
        double u = dot_bf16(xt, w_gu + (size_t)(f + n) * D, D);
        h[n] = silu(g) * u;
    }
    for (int d = 0; d < D; ++d) {
        const uint16_t* row = w_d + (size_t)d * f;
        double s = 0.0;
        for (int n = 0; n < f; ++n) s += bf16_to_double(row[n]) * h[n];
        acc[d] += a * s;
    }
}

/*
 * Sparse layer output ("MoE", section 4) for the listed tokens:
 *   y[i] = sum_k alpha[t,k] E_{idx[t,k]}(x_t)  (+ sgate[t] E_s(x_t) when w_s_gu != NULL)
 * with t = tokens[i] (or t = i when tokens == NULL).  Expert e's weights are
 * w_gu + e*2f*D and w_d + e*D*f, so callers may pass a compacted weight set with idx
 * renumbered into it.  Output y is [ntok, D] double.
 */
int oracle_experts(const uint16_t* x, const int32_t* idx, const double* alpha,
                   const uint16_t* w_gu, const uint16_t* w_d,
                   const uint16_t* w_s_gu, const uint16_t* w_s_d, const double* sgate,
                   int D, int E, int K, int f, int f_s,
                   const int32_t* tokens, int ntok, double* y) {
    if (D <= 0 || E <= 0 || K <= 0 || f <= 0 || ntok < 0) return -1;
    if (w_s_gu && (!w_s_d || !sgate || f_s <= 0)) return -1;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int i = 0; i < ntok; ++i) {
        int t = tokens ? tokens[i] : i;
        int hn = (w_s_gu && f_s > f) ? f_s : f;
        double* h = (double*)malloc(sizeof(double) * (size_t)hn);
        if (!h) { bad = 1; continue; }
        double* acc = y + (size_t)i * D;
        for (int d = 0; d < D; ++d) acc[d] = 0.0;
        const uint16_t* xt = x + (size_t)t * D;
        for (int k = 0; k < K; ++k) {
            int e = idx[(size_t)t * K + k];
            if (e < 0 || e >= E) { bad = 1; continue; }
            expert_accumulate(xt, w_gu + (size_t)e * 2 * f * D, w_d + (size_t)e * D * f,
                              D, f, alpha[(size_t)t * K + k], h, acc);
        }
        if (w_s_gu) expert_accumulate(xt, w_s_gu, w_s_d, D, f_s, sgate[t], h, acc);
        free(h);
    }
    return bad ? -1 : 0;
}

/*
 * Dense-masked layer output, the brute-force form of the same sum: every one of the E
 * experts is evaluated on every token and weighted by dense_alpha[t,e] (zero for the
 * experts outside I_t).  Unselected experts contribute exactly nothing, so this equals
 * oracle_experts when dense_alpha scatters the sparse alpha ("1.6 混合专家（MoE）",
 * section 2: the weighting acts on each expert's output vector).  y is [T, D] double.
 */
int oracle_dense_masked(const uint16_t* x, const double* dense_alpha,
                        const uint16_t* w_gu, const uint16_t* w_d,
                        const uint16_t* w_s_gu, const uint16_t* w_s_d, const double* sgate,
                        int T, int D, int E, int f, int f_s, double* y) {
    if (T < 0 || D <= 0 || E <= 0 || f <= 0) return -1;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int t = 0; t < T; ++t) {
        int hn = (w_s_gu && f_s > f) ? f_s : f;
        double* h = (double*)malloc(sizeof(double) * (size_t)hn);
        if (!h) { bad = 1; continue; }
        double* acc = y + (size_t)t * D;
        for (int d = 0; d < D; ++d) acc[d] = 0.0;
        const uint16_t* xt = x + (size_t)t * D;
        for (int e = 0; e < E; ++e)
            expert_accumulate(xt, w_gu + (size_t)e * 2 * f * D, w_d + (size_t)e * D * f,
                              D, f, dense_alpha[(size_t)t * E + e], h, acc);
        if (w_s_gu) expert_accumulate(xt, w_s_gu, w_s_d, D, f_s, sgate[t], h, acc);
        free(h);
    }
    return bad ? -1 : 0;
}

/*
 * Token permutation: group the T*K (token, slot) pairs by expert ("MoE", section 3.2:
 * each routed expert gathers the tokens routed to it; "1.6 混合专家（MoE）", section 2:
 * tokens are first grouped by their routes).  Plain definition: walk the experts in
 * order, and for each expert walk the tokens in ascending order and their slots.
 *   counts[e]          rows of expert e
 *   offsets[e]         first row of expert e (offsets[E] = T*K)
 *   sorted_token[row]  token of that row
 *   sorted_slot[row]   t*K + k of that row
 *   slot_to_row[t*K+k] row of that pair (the inverse map)
 */
int oracle_permute(const int32_t* idx, int T, int E, int K, int32_t* counts, int32_t* offsets,
                   int32_t* sorted_token, int32_t* sorted_slot, int32_t* slot_to_row) {
    if (T < 0 || E <= 0 || K <= 0) return -1;
    int32_t row = 0;
    for (int e = 0; e < E; ++e) {
        offsets[e] = row;
        for (int t = 0; t < T; ++t)
            for (int k = 0; k < K; ++k)
                if (idx[(size_t)t * K + k] == e) {
                    sorted_token[row] = t;
                    sorted_slot[row] = t * K + k;
                    slot_to_row[(size_t)t * K + k] = row;
                    ++row;
                }
        counts[e] = row - offsets[e];
    }
    offsets[E] = row;
    return row == T * K ? 0 : -1;
}

/*
 * Expert capacity and token dropping ("1.6 混合专家（MoE）", section "专家容量与 token
 * 丢弃"; the zskr.cn training configuration's capacity_factor / min_capacity keys): every
 * expert processes at most C of the (token, expert) assignments routed to it; the ones
 * past capacity are dropped -- they skip the expert, so the token keeps only its other
 * experts' terms (nothing at all when every assignment is dropped: the layer's output is
 * then zero and the token passes on through the residual).
 *   C = max(min_capacity, ceil(capacity_factor * T * K / E))
 * Readings: the capacity counts assignments (T*K of them spread over E experts; counting
 * tokens alone, T/E, would drop most assignments at K = 8); an expert keeps its first C
 * assignments in ascending token order; the surviving weights are not renormalised again.
 */
long long oracle_expert_capacity(int T, int K, int E, double capacity_factor, int min_capacity) {
    if (T < 0 || K <= 0 || E <= 0 || capacity_factor <= 0.0) return -1;
    const double c = ceil(capacity_factor * (double)T * (double)K / (double)E);
    long long cap = (long long)c;
    if (cap < min_capacity) cap = min_capacity;
    return cap;
}

/* keep[t*K+k] = 1 when assignment (t, k) is among the first C of its expert in ascending
 * token order, else 0.  Walks the tokens in order with one running count per expert. */
int oracle_capacity_keep(const int32_t* idx, int T, int K, int E, long long C, uint8_t* keep) {
    if (T < 0 || K <= 0 || E <= 0 || C < 0) return -1;
    long long* seen = (long long*)calloc((size_t)E, sizeof(long long));
    if (!seen) return -1;
    int bad = 0;
    for (int t = 0; t < T; ++t)
        for (int k = 0; k < K; ++k) {
            const int e = idx[(size_t)t * K + k];
            if (e < 0 || e >= E) { bad = 1; keep[(size_t)t * K + k] = 0; continue; }
            keep[(size_t)t * K + k] = seen[e] < C ? 1 : 0;
            ++seen[e];
        }
    free(seen);
    return bad ? -1 : 0;
}

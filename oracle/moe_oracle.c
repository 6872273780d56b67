/*
 * oracle/moe_oracle.c -- fp64 reference ("oracle") for the sparsely-gated
 * Mixture-of-Experts FFN layer.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is plain, slow, obviously-correct C.
 * Only tests/, the smoke check in __graft_entry__.py and the CPU-baseline leg
 * of bench.py may build, load or call it.  The product (the CUDA library under
 * sparse_mixture_experts_10_b200/ and its Python binding) shares no code with
 * it and never calls it.
 *
 * Every quantity is computed in double precision with plain loops in the
 * order the pages state; there is no blocking, fusion or reordering.  Inputs
 * arrive as fp32 or as bf16 bit patterns and are widened exactly to double.
 *
 * Sources, cited per function by page title and section:
 *   "MoE(Mixture of Experts)"  (sharin-2a1.pages.dev/parts/moe), sections
 *        (1) parameter accounting, (2) routing "choose the top k and softmax
 *        again", (3) load balancing "prevent collapse with a loss".
 *   "Outrageously Large Neural Networks" explained (qiita, Shazeer et al.
 *        2017), sections "Sparsely-Gated MoE layer formula", "gating: Noisy
 *        Top-k Softmax" and "load-balancing losses".
 *   "Extending Raschka's GPT-2: an MoE trained from scratch on an RTX 3090"
 *        (techfeed summary), sections "how MoE works" (GPT-2 FFN) and
 *        "making the router trainable" (worked router example).
 *   Transformers-v5 MoE article (smart-guide.co.kr), section 1 "Weight
 *        Loading Refactor" (packed gate_up_proj: experts on dim 0, gate then
 *        up on dim 1) and section 2 "Expert Backend".
 *
 * Readings where the pages are silent:
 *   - Load(X) of the Shazeer article is a smooth estimator that needs the
 *     training noise; it is not printed.  The oracle uses the hard per-expert
 *     count instead.  The smooth estimator itself is not implemented:
 *     parity unpinned, out of scope.
 *   - CV^2 uses the population variance and is 0 when the mean is 0.
 *   - GELU is the exact erf form.
 *   - The router bias b_g is an input of the skewed synthetic workloads; the
 *     pages' router has none, so it is optional (NULL = absent).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_F32 0
#define ORC_BF16 1
#define ORC_ACT_GELU 0
#define ORC_ACT_SWIGLU 1

/* Element i of a tensor stored as fp32 or as bf16 bits, widened exactly. */
static double orc_get(const void *p, int dtype, int64_t i) {
    if (dtype == ORC_F32) return (double)((const float *)p)[i];
    uint32_t bits = (uint32_t)((const uint16_t *)p)[i] << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/* Widen one token row (D elements) to double. */
void orc_load_row(int64_t D, const void *x, int dtype, int64_t t, double *row) {
    for (int64_t i = 0; i < D; ++i) row[i] = orc_get(x, dtype, t * D + i);
}

/* ------------------------------------------------------------------------
 * Router scores.  Shazeer article, gating section: the gate's scores are
 * H(x) = x W_g with W_g of shape [DModel, NExperts], i.e. the matrix-vector
 * product s_e = sum_i x_i W_g[i, e] (summed here in ascending i).  b_g
 * (optional) is added after the sum.
 * ---------------------------------------------------------------------- */
void orc_router_scores(int64_t D, int64_t N, const double *x_row,
                       const void *Wg, int w_dtype, const float *bg,
                       double *scores) {
    for (int64_t e = 0; e < N; ++e) {
        double s = 0.0;
        for (int64_t i = 0; i < D; ++i) s += x_row[i] * orc_get(Wg, w_dtype, i * N + e);
        if (bg) s += (double)bg[e];
        scores[e] = s;
    }
}

/* ------------------------------------------------------------------------
 * Ranking of the experts.  Shazeer article, gating section: KeepTopK(v, k)
 * keeps the k largest entries of the score vector v.  Which of several equal
 * scores count as "largest" is the reading that the lower expert index comes
 * first (the chapter "MoE(Mixture of Experts)", section (2), gets the same
 * order from a stable sort of the indices by descending score).  So the rank
 * of expert e is the number of experts placed before it: those with a
 * strictly larger score, and those with an equal score and a lower index.
 * Ranks are a permutation of 0..N-1.
 * ---------------------------------------------------------------------- */
int64_t orc_expert_rank(int64_t N, const double *scores, int64_t e) {
    int64_t r = 0;
    for (int64_t j = 0; j < N; ++j) {
        if (scores[j] > scores[e]) r += 1;
        else if (scores[j] == scores[e] && j < e) r += 1;
    }
    return r;
}

/* All experts by rank: order[rank(e)] = e. */
void orc_rank_experts(int64_t N, const double *scores, int32_t *order) {
    for (int64_t e = 0; e < N; ++e) order[orc_expert_rank(N, scores, e)] = (int32_t)e;
}

/* The set KeepTopK keeps: the experts of rank below K, listed best first
 * (slot j holds the expert of rank j). */
void orc_select_topk(int64_t N, int64_t K, const double *scores, int32_t *sel) {
    for (int64_t e = 0; e < N; ++e) {
        int64_t r = orc_expert_rank(N, scores, e);
        if (r < K) sel[r] = (int32_t)e;
    }
}

/* softmax(v)_i = exp(v_i) / sum_m exp(v_m) over n entries, an entry of -inf
 * giving exp(-inf) = 0.  Evaluated as exp(v_i - M) / sum_m exp(v_m - M) with M
 * the largest entry (the softmax does not change when every entry is
 * shifted by the same amount). */
void orc_softmax(int64_t n, const double *v, double *p) {
    double M = -INFINITY;
    for (int64_t i = 0; i < n; ++i)
        if (v[i] > M) M = v[i];
    double z = 0.0;
    for (int64_t i = 0; i < n; ++i) {
        p[i] = v[i] == -INFINITY ? 0.0 : exp(v[i] - M);
        z += p[i];
    }
    for (int64_t i = 0; i < n; ++i) p[i] = p[i] / z;
}

/* ------------------------------------------------------------------------
 * Gate weights.  Shazeer article, gating section, inference form (no noise
 * term): G(x) = softmax(KeepTopK(H(x), k)) with H(x) = x W_g and
 * KeepTopK(v, k)_e = v_e for a kept expert, -inf for every other one.  The
 * kept set is given as sel (K experts, normally orc_select_topk of these same
 * scores); G is dense over the N experts and zero outside the kept set.  The
 * weight of slot j is G at expert sel_j.
 * ---------------------------------------------------------------------- */
void orc_gate_weights(int64_t N, int64_t K, const double *scores, const int32_t *sel, double *w) {
    double *v = (double *)malloc(sizeof(double) * (size_t)N);
    double *G = (double *)malloc(sizeof(double) * (size_t)N);
    for (int64_t e = 0; e < N; ++e) v[e] = -INFINITY;
    for (int64_t j = 0; j < K; ++j) v[sel[j]] = scores[sel[j]];
    orc_softmax(N, v, G);
    for (int64_t j = 0; j < K; ++j) w[j] = G[sel[j]];
    free(v);
    free(G);
}

/* Exact-erf GELU: gelu(v) = v * Phi(v) = 0.5 v (1 + erf(v / sqrt 2)). */
double orc_gelu(double v) { return 0.5 * v * (1.0 + erf(v / sqrt(2.0))); }

/* SiLU: silu(g) = g * sigmoid(g) = g / (1 + exp(-g)). */
double orc_silu(double g) { return g / (1.0 + exp(-g)); }

/* ------------------------------------------------------------------------
 * GPT-2 FFN expert.  "Extending Raschka's GPT-2 ...", section on how MoE
 * works: Linear D -> 4D, GELU, Linear 4D -> D.  Weights are stored out x in:
 * W1e [H, D], b1e [H], W2e [D, H], b2e [D]; biases optional (NULL).
 *   hid[n] = gelu(sum_i W1e[n, i] x[i] + b1e[n])
 *   out[c] = sum_n W2e[c, n] hid[n] + b2e[c]
 * ---------------------------------------------------------------------- */
void orc_expert_gelu(int64_t D, int64_t H, const double *x_row,
                     const void *W1e, const float *b1e,
                     const void *W2e, const float *b2e, int dtype,
                     double *hid, double *out) {
    for (int64_t n = 0; n < H; ++n) {
        double a = 0.0;
        for (int64_t i = 0; i < D; ++i) a += orc_get(W1e, dtype, n * D + i) * x_row[i];
        if (b1e) a += (double)b1e[n];
        hid[n] = orc_gelu(a);
    }
    for (int64_t c = 0; c < D; ++c) {
        double a = 0.0;
        for (int64_t n = 0; n < H; ++n) a += orc_get(W2e, dtype, c * H + n) * hid[n];
        if (b2e) a += (double)b2e[c];
        out[c] = a;
    }
}

/* ------------------------------------------------------------------------
 * SwiGLU expert with the packed gate_up weight.  Transformers-v5 article,
 * section 1: per-expert gate (w1) and up (w3) projections are concatenated on
 * dim 1, gate first, so W_gu[e] is [2H, D] with gate rows 0..H-1 and up rows
 * H..2H-1; "MoE(Mixture of Experts)" notes real experts are SwiGLU FFNs.
 *   g[n] = sum_i Wgu[n, i] x[i],  u[n] = sum_i Wgu[H + n, i] x[i]
 *   hid[n] = silu(g[n]) * u[n],   out[c] = sum_n Wdown[c, n] hid[n]
 * ---------------------------------------------------------------------- */
void orc_expert_swiglu(int64_t D, int64_t H, const double *x_row,
                       const void *Wgue, const void *Wdowne, int dtype,
                       double *hid, double *out) {
    for (int64_t n = 0; n < H; ++n) {
        double g = 0.0, u = 0.0;
        for (int64_t i = 0; i < D; ++i) g += orc_get(Wgue, dtype, n * D + i) * x_row[i];
        for (int64_t i = 0; i < D; ++i) u += orc_get(Wgue, dtype, (H + n) * D + i) * x_row[i];
        hid[n] = orc_silu(g) * u;
    }
    for (int64_t c = 0; c < D; ++c) {
        double a = 0.0;
        for (int64_t n = 0; n < H; ++n) a += orc_get(Wdowne, dtype, c * H + n) * hid[n];
        out[c] = a;
    }
}

/* ------------------------------------------------------------------------
 * Combine.  Shazeer article: y = sum_i G(x)_i E_i(x) with unselected experts
 * skipped; "MoE(Mixture of Experts)" section (2), Forward: out starts at 0 and
 * out = out + w * y is applied for each assignment in selection order.
 * E holds the K expert outputs of one token, [K, D], slot order.
 * ---------------------------------------------------------------------- */
void orc_combine(int64_t K, int64_t D, const double *w, const double *E, double *y) {
    for (int64_t c = 0; c < D; ++c) y[c] = 0.0;
    for (int64_t j = 0; j < K; ++j)
        for (int64_t c = 0; c < D; ++c) y[c] = y[c] + w[j] * E[j * D + c];
}

/* One layer description; all pointers are host memory. */
typedef struct {
    int64_t D, H, N, K;
    int32_t act;      /* ORC_ACT_GELU / ORC_ACT_SWIGLU */
    int32_t dtype;    /* ORC_F32 / ORC_BF16 for x and all weight matrices */
    const void *x;    /* [T, D] */
    const void *Wg;   /* [D, N] */
    const float *bg;  /* [N] or NULL */
    const void *W1;   /* GELU [N, H, D] ; SwiGLU [N, 2H, D] */
    const float *b1;  /* [N, H] or NULL (GELU only) */
    const void *W2;   /* [N, D, H] */
    const float *b2;  /* [N, D] or NULL (GELU only) */
    const float *bsel; /* [N] or NULL: selection-only bias (see orc_moe_layer_rows) */
    const void *S1;   /* shared expert or NULL: GELU [H, D] ; SwiGLU [2H, D] */
    const float *sb1; /* [H] or NULL (GELU only) */
    const void *S2;   /* shared expert [D, H] */
    const float *sb2; /* [D] or NULL (GELU only) */
} orc_layer;

/* Byte size of one element of the layer's dtype. */
static int64_t orc_elem(const orc_layer *L) { return L->dtype == ORC_F32 ? 4 : 2; }

/* One expert's output for one token row: dispatch on the activation. */
void orc_expert(const orc_layer *L, int64_t e, const double *x_row, double *hid, double *out) {
    int64_t D = L->D, H = L->H, es = orc_elem(L);
    if (L->act == ORC_ACT_GELU) {
        const char *W1e = (const char *)L->W1 + e * H * D * es;
        const char *W2e = (const char *)L->W2 + e * D * H * es;
        orc_expert_gelu(D, H, x_row, W1e, L->b1 ? L->b1 + e * H : NULL, W2e,
                        L->b2 ? L->b2 + e * D : NULL, L->dtype, hid, out);
    } else {
        const char *Wgue = (const char *)L->W1 + e * 2 * H * D * es;
        const char *Wde = (const char *)L->W2 + e * D * H * es;
        orc_expert_swiglu(D, H, x_row, Wgue, Wde, L->dtype, hid, out);
    }
}

/* ------------------------------------------------------------------------
 * Capacity.  "MoE(Mixture of Experts)", design notes (capacity factor): real
 * layers give each expert an upper limit on the tokens it accepts; what
 * overflows is dropped or passed to the next candidate.  Readings: the limit
 * is C = ceil(cf * T * K / N) (the expected number of assignments per expert
 * times the capacity factor cf; computed in double); cf <= 0 means no limit.
 * ---------------------------------------------------------------------- */
int64_t orc_capacity(double cf, int64_t T, int64_t K, int64_t N) {
    if (cf <= 0.0) return INT64_MAX;
    return (int64_t)ceil(cf * (double)T * (double)K / (double)N);
}

/* Drop: the rows are served in order (the chapter's Forward visits rows
 * r = 0, 1, ...) and each of a row's K assignments is accepted when its expert
 * has accepted fewer than C so far; keep[t*K + j] = 1 for an accepted
 * assignment, 0 for a dropped one.  A dropped assignment contributes nothing
 * to y (the kept weights are not renormalised). */
void orc_capacity_keep(int64_t T, int64_t N, int64_t K, const int32_t *sel, int64_t C, uint8_t *keep) {
    int64_t *load = (int64_t *)calloc((size_t)N, sizeof(int64_t));
    for (int64_t t = 0; t < T; ++t) {
        for (int64_t j = 0; j < K; ++j) {
            const int32_t e = sel[t * K + j];
            if (load[e] < C) {
                load[e] += 1;
                keep[t * K + j] = 1;
            } else {
                keep[t * K + j] = 0;
            }
        }
    }
    free(load);
}

/* ------------------------------------------------------------------------
 * Shared expert.  "MoE(Mixture of Experts)", design notes (merits and
 * examples): the fine-grained MoE of DeepSeek-V3 adds to the many small routed
 * experts a shared part that every token passes through.  Read here as one
 * FFN of the same form and sizes as a routed expert (GELU or SwiGLU), not
 * gated: its output is added with weight 1 after the routed experts' sum.
 * ---------------------------------------------------------------------- */
void orc_shared_expert(const orc_layer *L, const double *x_row, double *hid, double *out) {
    if (L->act == ORC_ACT_GELU)
        orc_expert_gelu(L->D, L->H, x_row, L->S1, L->sb1, L->S2, L->sb2, L->dtype, hid, out);
    else
        orc_expert_swiglu(L->D, L->H, x_row, L->S1, L->S2, L->dtype, hid, out);
}

/* y = y + s, element by element. */
void orc_add_shared(int64_t D, const double *s, double *y) {
    for (int64_t c = 0; c < D; ++c) y[c] = y[c] + s[c];
}

/* ------------------------------------------------------------------------
 * The whole layer for tokens t0..t1-1 ("MoE(Mixture of Experts)" section (2),
 * Forward: route each row, evaluate only the selected experts, mix in order).
 *   bsel (optional, in the layer): a per-expert bias that changes which
 *       experts are kept and nothing else -- the auxiliary-loss-free load
 *       balancing of DeepSeek-V3 named in the chapter's design notes (a bias
 *       adjusted during training).  Read here as: KeepTopK is taken on
 *       s_e + bsel_e, and the gate weights are softmax(KeepTopK) of the raw
 *       scores s over that kept set; the statistics use the raw scores.
 *   S1/S2 (optional): the shared expert, added after the routed sum.
 *   keep [T, K] (optional): capacity decisions (orc_capacity_keep); a slot
 *       with keep 0 is not evaluated and adds nothing.
 *   scores_out [T, N]: fp64 router scores.
 *   sel_scores [T, N] (optional): if given, the expert selection is made on
 *       these scores instead of the fp64 s + bsel (used to apply the oracle's
 *       ranking to the device's fp32 logits, with any selection bias already
 *       added in fp32); the gate weights always use the fp64 scores.
 *   sel_out [T, K], w_out [T, K], y_out [T, D].
 * Rows outside [t0, t1) are not touched, so disjoint ranges may run on
 * separate threads.
 * ---------------------------------------------------------------------- */
void orc_moe_layer_rows(const orc_layer *L, int64_t t0, int64_t t1,
                        const float *sel_scores, const uint8_t *keep, double *scores_out,
                        int32_t *sel_out, double *w_out, double *y_out) {
    int64_t D = L->D, H = L->H, N = L->N, K = L->K;
    double *x_row = (double *)malloc(sizeof(double) * (size_t)D);
    double *hid = (double *)malloc(sizeof(double) * (size_t)H);
    double *E = (double *)malloc(sizeof(double) * (size_t)(K * D));
    double *tmp = (double *)malloc(sizeof(double) * (size_t)N);
    double *sh = (double *)malloc(sizeof(double) * (size_t)D);
    for (int64_t t = t0; t < t1; ++t) {
        double *s = scores_out + t * N;
        int32_t *sel = sel_out + t * K;
        double *w = w_out + t * K;
        orc_load_row(D, L->x, L->dtype, t, x_row);
        orc_router_scores(D, N, x_row, L->Wg, L->dtype, L->bg, s);
        if (sel_scores) {
            for (int64_t e = 0; e < N; ++e) tmp[e] = (double)sel_scores[t * N + e];
        } else {
            for (int64_t e = 0; e < N; ++e) tmp[e] = s[e] + (L->bsel ? (double)L->bsel[e] : 0.0);
        }
        orc_select_topk(N, K, tmp, sel);
        orc_gate_weights(N, K, s, sel, w);
        for (int64_t j = 0; j < K; ++j) {
            if (keep && !keep[t * K + j]) {
                for (int64_t c = 0; c < D; ++c) E[j * D + c] = 0.0;   /* dropped: no contribution */
                continue;
            }
            orc_expert(L, sel[j], x_row, hid, E + j * D);
        }
        orc_combine(K, D, w, E, y_out + t * D);
        if (L->S1) {
            orc_shared_expert(L, x_row, hid, sh);
            orc_add_shared(D, sh, y_out + t * D);
        }
    }
    free(x_row);
    free(hid);
    free(E);
    free(tmp);
    free(sh);
}

/* ------------------------------------------------------------------------
 * Coefficient of variation squared.  Shazeer article, load-balancing
 * losses: L = w * CV(v)^2.  Population variance; 0 when the mean is 0.
 * ---------------------------------------------------------------------- */
double orc_cv_squared(int64_t n, const double *v) {
    double mean = 0.0;
    for (int64_t i = 0; i < n; ++i) mean += v[i];
    mean /= (double)n;
    if (mean == 0.0) return 0.0;
    double var = 0.0;
    for (int64_t i = 0; i < n; ++i) var += (v[i] - mean) * (v[i] - mean);
    var /= (double)n;
    return var / (mean * mean);
}

/* ------------------------------------------------------------------------
 * "MoE(Mixture of Experts)" section (3), LoadBalanceLoss: with f_e the share
 * of the routed tokens that went to expert e (n_e over the total), the loss is
 * N * sum_e f_e^2, and 0 when nothing was routed.
 * ---------------------------------------------------------------------- */
double orc_simple_balance_loss(int64_t N, const double *counts) {
    double total = 0.0;
    for (int64_t e = 0; e < N; ++e) total += counts[e];
    if (total == 0.0) return 0.0;
    double sum = 0.0;
    for (int64_t e = 0; e < N; ++e) {
        double f = counts[e] / total;
        sum += f * f;
    }
    return (double)N * sum;
}

/* ------------------------------------------------------------------------
 * Per-batch statistics and auxiliary losses for T tokens.
 *   counts[e]      tokens routed to e ("MoE(Mixture of Experts)" section (2),
 *                  Stats.TokensPerExpert, one per (token, selected expert)).
 *   importance[e]  Shazeer article: Importance(X)_e = sum_x G(x)_e.
 *   p_mean[e]      (1/T) sum_t softmax(scores_t)_e, the full N-way softmax
 *                  gate of the Shazeer article, before KeepTopK.
 *   scalars[0]     Switch-style N * sum_e f_e P_e, f_e = counts[e] / (T K),
 *                  P_e = p_mean[e] ("Extending Raschka's GPT-2", auxiliary
 *                  loss section: Switch-Transformers approach).
 *   scalars[1]     N * sum_e f_e^2 (section (3) LoadBalanceLoss).
 *   scalars[2]     CV(importance)^2,  scalars[3] CV(counts)^2 (hard Load).
 * All zero when T == 0.
 * ---------------------------------------------------------------------- */
void orc_aux_stats(int64_t T, int64_t N, int64_t K, const double *scores,
                   const int32_t *sel, const double *w, double *counts,
                   double *importance, double *p_mean, double *scalars) {
    for (int64_t e = 0; e < N; ++e) counts[e] = importance[e] = p_mean[e] = 0.0;
    for (int i = 0; i < 4; ++i) scalars[i] = 0.0;
    if (T == 0) return;
    double *p = (double *)malloc(sizeof(double) * (size_t)N);
    for (int64_t t = 0; t < T; ++t) {
        for (int64_t j = 0; j < K; ++j) {
            counts[sel[t * K + j]] += 1.0;
            importance[sel[t * K + j]] += w[t * K + j];
        }
        const double *s = scores + t * N;
        double smax = s[0];
        for (int64_t e = 1; e < N; ++e)
            if (s[e] > smax) smax = s[e];
        double z = 0.0;
        for (int64_t e = 0; e < N; ++e) {
            p[e] = exp(s[e] - smax);
            z += p[e];
        }
        for (int64_t e = 0; e < N; ++e) p_mean[e] += p[e] / z;
    }
    for (int64_t e = 0; e < N; ++e) p_mean[e] /= (double)T;
    double fP = 0.0;
    for (int64_t e = 0; e < N; ++e) fP += (counts[e] / (double)(T * K)) * p_mean[e];
    scalars[0] = (double)N * fP;
    scalars[1] = orc_simple_balance_loss(N, counts);
    scalars[2] = orc_cv_squared(N, importance);
    scalars[3] = orc_cv_squared(N, counts);
    free(p);
}

/* ------------------------------------------------------------------------
 * Parameter accounting.  "MoE(Mixture of Experts)" section (1): the router
 * holds DModel*NExperts weights and each GELU expert 2*DModel*DHidden; the
 * total counts all NExperts experts, the active count only TopK of them.
 * Extended, as stated here, to expert biases (H + D more per GELU expert) and
 * to SwiGLU experts (gate, up and down: 3*D*H, no biases).
 * ---------------------------------------------------------------------- */
int64_t orc_expert_params(int64_t D, int64_t H, int32_t act, int32_t has_bias) {
    if (act == ORC_ACT_SWIGLU) return 3 * D * H;
    return 2 * D * H + (has_bias ? H + D : 0);
}

int64_t orc_total_params(int64_t D, int64_t H, int64_t N, int64_t K, int32_t act, int32_t has_bias) {
    (void)K;
    return D * N + N * orc_expert_params(D, H, act, has_bias);
}

int64_t orc_active_params(int64_t D, int64_t H, int64_t N, int64_t K, int32_t act, int32_t has_bias) {
    return D * N + K * orc_expert_params(D, H, act, has_bias);
}

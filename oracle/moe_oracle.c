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

/* The values the experts are ranked on for selection: the device's fp32
 * selection scores when given (sel_row), else the fp64 score plus the
 * selection-only bias (if any). */
static void orc_selection_row(int64_t N, const double *s, const float *bsel, const float *sel_row, double *v) {
    for (int64_t e = 0; e < N; ++e)
        v[e] = sel_row ? (double)sel_row[e] : s[e] + (bsel ? (double)bsel[e] : 0.0);
}

/* Reroute: the other overflow policy of the chapter's design notes -- an
 * assignment that does not fit goes to the next candidate instead of being
 * dropped.  Rows are served in order, as for the drop.  Row t first offers each
 * of its K selected experts its slot (accepted while the expert holds fewer
 * than C); each refused slot, in slot order, then goes to the best-ranked
 * expert (larger selection value first, ties to the lower index) that is not
 * already one of row t's experts and still holds fewer than C.  If no such
 * expert is left the slot is dropped (assign -1).  The slot keeps its gate
 * weight: the router's weights are not recomputed, as for the drop.
 *   v [T, N]: the selection values (orc_selection_row); sel [T, K];
 *   assign [T, K] out: the expert that serves each slot, or -1. */
void orc_capacity_reroute(int64_t T, int64_t N, int64_t K, const double *v, const int32_t *sel, int64_t C,
                          int32_t *assign) {
    int64_t *load = (int64_t *)calloc((size_t)N, sizeof(int64_t));
    uint8_t *held = (uint8_t *)malloc((size_t)N);
    for (int64_t t = 0; t < T; ++t) {
        const double *vt = v + t * N;
        memset(held, 0, (size_t)N);
        for (int64_t j = 0; j < K; ++j) held[sel[t * K + j]] = 1;
        for (int64_t j = 0; j < K; ++j) {
            const int32_t e = sel[t * K + j];
            if (load[e] < C) {
                load[e] += 1;
                assign[t * K + j] = e;
            } else {
                assign[t * K + j] = -1;   /* refused: rerouted below */
            }
        }
        for (int64_t j = 0; j < K; ++j) {
            if (assign[t * K + j] >= 0) continue;
            int64_t best = -1;
            for (int64_t e = 0; e < N; ++e) {
                if (held[e] || load[e] >= C) continue;
                if (best < 0 || vt[e] > vt[best]) best = e;   /* ascending e: ties keep the lower index */
            }
            if (best >= 0) {
                load[best] += 1;
                held[best] = 1;
                assign[t * K + j] = (int32_t)best;
            }
        }
    }
    free(load);
    free(held);
}

/* The selection values of rows t0..t1-1 (fp64 scores plus bias, or the given
 * fp32 selection scores), for orc_capacity_reroute. */
void orc_selection_values(const orc_layer *L, int64_t t0, int64_t t1, const double *scores, const float *sel_scores,
                          double *v) {
    for (int64_t t = t0; t < t1; ++t)
        orc_selection_row(L->N, scores + t * L->N, L->bsel, sel_scores ? sel_scores + t * L->N : NULL, v + t * L->N);
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
 *   assign [T, K] (optional): the expert serving each slot after a reroute
 *       (orc_capacity_reroute), -1 for none; the slot's gate weight is kept.
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
                        const float *sel_scores, const uint8_t *keep, const int32_t *assign,
                        double *scores_out, int32_t *sel_out, double *w_out, double *y_out) {
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
        orc_selection_row(N, s, L->bsel, sel_scores ? sel_scores + t * N : NULL, tmp);
        orc_select_topk(N, K, tmp, sel);
        orc_gate_weights(N, K, s, sel, w);
        for (int64_t j = 0; j < K; ++j) {
            const int32_t e = assign ? assign[t * K + j] : sel[j];
            if ((keep && !keep[t * K + j]) || e < 0) {
                for (int64_t c = 0; c < D; ++c) E[j * D + c] = 0.0;   /* dropped: no contribution */
                continue;
            }
            orc_expert(L, e, x_row, hid, E + j * D);
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
 * Backward pass.  "Extending Raschka's GPT-2 ...", section on making the
 * router trainable: the router learns through the gate weights it produces
 * (the softmax over the kept scores) and through the auxiliary loss; the
 * experts learn through the outputs they are weighted into.  Everything below
 * is the chain rule applied to the forward definitions above, in fp64:
 *   y = sum_j w_j o_j,  o_j = E_{sel_j}(x),  w = softmax over the kept scores
 *   dL/dw_j = <dy, o_j>,  dL/do_j = w_j dy
 *   softmax over the kept set: ds_kept_j = w_j (dw_j - sum_m w_m dw_m), 0 for
 *   the others; scores s = x W_g + b_g: dW_g += x ds, db_g += ds, dx += W_g ds
 * plus, with weights alpha_switch and alpha_importance, the gradients of the
 * Switch-style loss N sum_e f_e P_e (f_e counts, constant almost everywhere;
 * P_e the mean full softmax) and of CV(importance)^2 (importance = sum of the
 * gate weights per expert).  The count-based terms (N sum f^2, CV(load)^2)
 * are piecewise constant and carry no gradient.
 * ---------------------------------------------------------------------- */

/* GELU'(v) = Phi(v) + v phi(v) for the exact-erf GELU. */
double orc_gelu_grad(double v) {
    return 0.5 * (1.0 + erf(v / sqrt(2.0))) + v * exp(-0.5 * v * v) / sqrt(2.0 * 3.14159265358979323846);
}

/* silu'(g) = s (1 + g (1 - s)) with s = 1 / (1 + exp(-g)). */
double orc_silu_grad(double g) {
    double sg = 1.0 / (1.0 + exp(-g));
    return sg * (1.0 + g * (1.0 - sg));
}

/* One expert's backward for one token row: upstream gradient go [D] of its
 * output; accumulates into dW1e ([H, D] or [2H, D]), db1e [H], dW2e [D, H],
 * db2e [D] (bias pointers NULL for SwiGLU) and adds the input gradient to
 * dx_row [D].  pre [2H], hid [H], dh [H] are scratch. */
void orc_expert_backward(const orc_layer *L, int64_t e, const double *x_row, const double *go, double *dx_row,
                         double *dW1e, double *db1e, double *dW2e, double *db2e, double *pre, double *hid,
                         double *dh) {
    int64_t D = L->D, H = L->H, es = orc_elem(L);
    int swiglu = L->act == ORC_ACT_SWIGLU;
    const char *W1e = (const char *)L->W1 + e * (swiglu ? 2 : 1) * H * D * es;
    const char *W2e = (const char *)L->W2 + e * D * H * es;
    /* forward of the expert again: pre-activations and hidden values */
    for (int64_t n = 0; n < (swiglu ? 2 * H : H); ++n) {
        double a = 0.0;
        for (int64_t i = 0; i < D; ++i) a += orc_get(W1e, L->dtype, n * D + i) * x_row[i];
        if (!swiglu && L->b1) a += (double)L->b1[e * H + n];
        pre[n] = a;
    }
    for (int64_t n = 0; n < H; ++n) hid[n] = swiglu ? orc_silu(pre[n]) * pre[H + n] : orc_gelu(pre[n]);
    /* second linear: dW2 += go hid^T, db2 += go, dh = W2^T go */
    for (int64_t c = 0; c < D; ++c) {
        for (int64_t n = 0; n < H; ++n) dW2e[c * H + n] += go[c] * hid[n];
        if (db2e) db2e[c] += go[c];
    }
    for (int64_t n = 0; n < H; ++n) {
        double a = 0.0;
        for (int64_t c = 0; c < D; ++c) a += orc_get(W2e, L->dtype, c * H + n) * go[c];
        dh[n] = a;
    }
    /* activation, then first linear: dW1 += da x^T, db1 += da, dx += W1^T da */
    for (int64_t n = 0; n < H; ++n) {
        if (swiglu) {
            double dg = dh[n] * pre[H + n] * orc_silu_grad(pre[n]);
            double du = dh[n] * orc_silu(pre[n]);
            for (int64_t i = 0; i < D; ++i) {
                dW1e[n * D + i] += dg * x_row[i];
                dW1e[(H + n) * D + i] += du * x_row[i];
                dx_row[i] += orc_get(W1e, L->dtype, n * D + i) * dg + orc_get(W1e, L->dtype, (H + n) * D + i) * du;
            }
        } else {
            double da = dh[n] * orc_gelu_grad(pre[n]);
            if (db1e) db1e[n] += da;
            for (int64_t i = 0; i < D; ++i) {
                dW1e[n * D + i] += da * x_row[i];
                dx_row[i] += orc_get(W1e, L->dtype, n * D + i) * da;
            }
        }
    }
}

/* The layer's backward for T tokens (single thread; the kept sets are chosen
 * as in the forward: on sel_scores when given, else on the fp64 scores plus
 * bsel).  dy [T, D]; outputs (zeroed here): dx [T, D], dWg [D, N], dbg [N],
 * dW1 like W1, db1 [N, H] (GELU, else may be NULL), dW2 [N, D, H], db2
 * [N, D] (GELU, else may be NULL). */
void orc_moe_layer_backward(const orc_layer *L, int64_t T, const float *sel_scores, const double *dy,
                            double alpha_switch, double alpha_importance, double *dx, double *dWg, double *dbg,
                            double *dW1, double *db1, double *dW2, double *db2) {
    int64_t D = L->D, H = L->H, N = L->N, K = L->K;
    int swiglu = L->act == ORC_ACT_SWIGLU;
    int64_t rows1 = swiglu ? 2 * H : H;
    for (int64_t i = 0; i < T * D; ++i) dx[i] = 0.0;
    for (int64_t i = 0; i < D * N; ++i) dWg[i] = 0.0;
    for (int64_t e = 0; e < N; ++e) dbg[e] = 0.0;
    for (int64_t i = 0; i < N * rows1 * D; ++i) dW1[i] = 0.0;
    for (int64_t i = 0; i < N * D * H; ++i) dW2[i] = 0.0;
    if (db1) for (int64_t i = 0; i < N * H; ++i) db1[i] = 0.0;
    if (db2) for (int64_t i = 0; i < N * D; ++i) db2[i] = 0.0;
    if (T == 0) return;
    double *scores = (double *)malloc(sizeof(double) * (size_t)(T * N));
    int32_t *sel = (int32_t *)malloc(sizeof(int32_t) * (size_t)(T * K));
    double *w = (double *)malloc(sizeof(double) * (size_t)(T * K));
    double *y = (double *)malloc(sizeof(double) * (size_t)(T * D));
    orc_moe_layer_rows(L, 0, T, sel_scores, NULL, NULL, scores, sel, w, y);
    /* batch quantities of the auxiliary losses: f_e and the importance */
    double *f = (double *)calloc((size_t)N, sizeof(double));
    double *imp = (double *)calloc((size_t)N, sizeof(double));
    for (int64_t t = 0; t < T; ++t)
        for (int64_t j = 0; j < K; ++j) {
            f[sel[t * K + j]] += 1.0 / (double)(T * K);
            imp[sel[t * K + j]] += w[t * K + j];
        }
    /* dCV^2/dimp_e = 2 (imp_e - m) / (N m^2) - 2 var / (N m^3), population variance */
    double m = 0.0, var = 0.0;
    for (int64_t e = 0; e < N; ++e) m += imp[e];
    m /= (double)N;
    for (int64_t e = 0; e < N; ++e) var += (imp[e] - m) * (imp[e] - m);
    var /= (double)N;
    double *dimp = (double *)calloc((size_t)N, sizeof(double));
    if (m != 0.0)
        for (int64_t e = 0; e < N; ++e)
            dimp[e] = 2.0 * (imp[e] - m) / ((double)N * m * m) - 2.0 * var / ((double)N * m * m * m);
    double *x_row = (double *)malloc(sizeof(double) * (size_t)D);
    double *o = (double *)malloc(sizeof(double) * (size_t)D);
    double *go = (double *)malloc(sizeof(double) * (size_t)D);
    double *pre = (double *)malloc(sizeof(double) * (size_t)(2 * H));
    double *hid = (double *)malloc(sizeof(double) * (size_t)H);
    double *dh = (double *)malloc(sizeof(double) * (size_t)H);
    double *dw = (double *)malloc(sizeof(double) * (size_t)K);
    double *ds = (double *)malloc(sizeof(double) * (size_t)N);
    double *p = (double *)malloc(sizeof(double) * (size_t)N);
    int64_t es = orc_elem(L);
    for (int64_t t = 0; t < T; ++t) {
        orc_load_row(D, L->x, L->dtype, t, x_row);
        double *dxr = dx + t * D;
        const double *dyr = dy + t * D;
        for (int64_t j = 0; j < K; ++j) {
            int32_t e = sel[t * K + j];
            orc_expert(L, e, x_row, hid, o);
            double a = 0.0;
            for (int64_t c = 0; c < D; ++c) a += dyr[c] * o[c];
            dw[j] = a + alpha_importance * dimp[e];
            for (int64_t c = 0; c < D; ++c) go[c] = w[t * K + j] * dyr[c];
            orc_expert_backward(L, e, x_row, go, dxr, dW1 + e * rows1 * D, db1 ? db1 + e * H : NULL,
                                dW2 + e * D * H, db2 ? db2 + e * D : NULL, pre, hid, dh);
        }
        /* the softmax over the kept scores, then the Switch-style loss on the full softmax */
        for (int64_t e = 0; e < N; ++e) ds[e] = 0.0;
        double wdw = 0.0;
        for (int64_t j = 0; j < K; ++j) wdw += w[t * K + j] * dw[j];
        for (int64_t j = 0; j < K; ++j) ds[sel[t * K + j]] += w[t * K + j] * (dw[j] - wdw);
        if (alpha_switch != 0.0) {
            orc_softmax(N, scores + t * N, p);
            double fp = 0.0;
            for (int64_t e = 0; e < N; ++e) fp += f[e] * p[e];
            for (int64_t e = 0; e < N; ++e) ds[e] += alpha_switch * ((double)N / (double)T) * p[e] * (f[e] - fp);
        }
        for (int64_t e = 0; e < N; ++e) {
            dbg[e] += ds[e];
            for (int64_t i = 0; i < D; ++i) {
                dWg[i * N + e] += x_row[i] * ds[e];
                dxr[i] += orc_get(L->Wg, L->dtype, i * N + e) * ds[e];
            }
        }
    }
    (void)es;
    free(scores); free(sel); free(w); free(y); free(f); free(imp); free(dimp);
    free(x_row); free(o); free(go); free(pre); free(hid); free(dh); free(dw); free(ds); free(p);
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

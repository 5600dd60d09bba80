/*
 * ckv_oracle.c -- plain, slow CPU oracle for ClusterKV-style semantic cluster
 * recall. TEST INFRASTRUCTURE ONLY: it is what the CUDA path is checked
 * against, and only the tests, the package's smoke check and the benchmark's
 * CPU-baseline leg may load it. It shares no code with the CUDA path.
 *
 * Source of the method: "ClusterKV: Manipulating LLM KV Cache in Semantic
 * Space for Recallable Compression" (Liu, Li, Zhao, Zhang, Guo;
 * arXiv 2412.03213v2), as summarised section by section on its paperlayer.ai
 * page. Section names below are that page's headings.
 *
 * Arithmetic: every dot product, mean, norm and softmax accumulates in double,
 * in index order, with no blocking or reordering. The one exception is the
 * cluster score used to rank clusters (ckvo_score): a floating-point value
 * that decides an integer result (which clusters are recalled), so it is
 * computed in fp32 in one fixed order that the GPU kernel also follows (see
 * ckvo_score). Build with -O2 -ffp-contract=off -fno-fast-math.
 *
 * Conventions (one problem = one (layer, batch, KV head); d = head dim):
 *   keys      float [n][d]  the clustered rows, exact values of the stored
 *                           bf16 or fp32 keys (bf16 -> float is exact)
 *   mu        double [C][d] centroids: the mean of the raw assigned keys
 *   muhat     double [C][d] the assignment copy mu/||mu||, rounded to the
 *                           storage format (bf16 or fp32) or left in double
 *   labels    int32 [n]     cluster of each clustered token, in [0, C)
 *   offsets   int32 [C+1]   perm_base + number of tokens in clusters < c
 *   perm      int32 [n]     absolute token positions grouped by cluster,
 *                           ascending within each cluster
 *
 * Parity unpinned: nothing. Every function is pinned by the not-gpu tests
 * (brute force, invariants, closed forms, special cases, library routines).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define CKVO_ROUND_NONE 0 /* keep double */
#define CKVO_ROUND_F32 1  /* round to fp32 (round to nearest even) */
#define CKVO_ROUND_BF16 2 /* round to bf16 (round to nearest even) */

/* ---- number formats ---------------------------------------------------- */

/* Round a double to the nearest bf16 value (ties to even), returned as the
 * 16-bit pattern. bf16 keeps fp32's exponent range and 8 significant bits. */
uint16_t ckvo_bf16_bits(double x) {
    uint16_t sign = signbit(x) ? 0x8000u : 0u;
    double a = fabs(x);
    if (isnan(x)) return 0x7FC0u;
    if (a == 0.0) return sign;
    /* quantum of the bf16 grid at |x|: 2^(e-8) for a = m*2^e, m in [0.5,1),
     * never finer than the smallest subnormal step 2^-133 */
    int e;
    frexp(a, &e);
    int qexp = e - 8;
    if (qexp < -133) qexp = -133;
    double scaled = ldexp(a, -qexp);     /* exact: power-of-two scaling */
    double r = nearbyint(scaled);        /* default mode: ties to even */
    double v = ldexp(r, qexp);
    if (v >= ldexp(1.0, 128)) return (uint16_t)(sign | 0x7F80u); /* inf */
    /* encode v (a bf16 value) exactly */
    float f = (float)v; /* exact: v has <= 8 significant bits in fp32 range */
    uint32_t u;
    memcpy(&u, &f, 4);
    return (uint16_t)(sign | ((u >> 16) & 0x7FFFu));
}

double ckvo_bf16_value(uint16_t h) {
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

static double round_to(double x, int mode) {
    if (mode == CKVO_ROUND_F32) return (double)(float)x;
    if (mode == CKVO_ROUND_BF16) return ckvo_bf16_value(ckvo_bf16_bits(x));
    return x;
}

static double dot_d(const float *a, const double *b, int d) {
    double s = 0.0;
    for (int t = 0; t < d; ++t) s += (double)a[t] * b[t];
    return s;
}

/* muhat = round(mu / ||mu||); a zero vector stays zero. */
static void normalise_row(const double *mu, int d, int mode, double *muhat) {
    double ss = 0.0;
    for (int t = 0; t < d; ++t) ss += mu[t] * mu[t];
    double nrm = sqrt(ss);
    for (int t = 0; t < d; ++t) muhat[t] = nrm > 0.0 ? round_to(mu[t] / nrm, mode) : 0.0;
}

/* ---- clustering: "III.B Clustering in the Semantic Space" --------------- */

/* Similarity: cosine (the method), with L2 and inner product as the paper's
 * ablation of the clustering distance. */

#define CKVO_METRIC_COSINE 0
#define CKVO_METRIC_INNER 1
#define CKVO_METRIC_L2 2

/* The copy of a centroid that assignment compares keys with: mu/||mu|| for
 * cosine, mu itself for inner product and L2, rounded to the storage format. */
static void assign_copy(const double *mu, int d, int mode, int metric, double *out) {
    if (metric == CKVO_METRIC_COSINE) {
        normalise_row(mu, d, mode, out);
        return;
    }
    for (int t = 0; t < d; ++t) out[t] = round_to(mu[t], mode);
}

/* Similarity of key k to assignment copy m; larger is closer. L2 uses the
 * plain definition, minus half the squared distance. */
static double similarity(const float *k, const double *m, int d, int metric) {
    if (metric != CKVO_METRIC_L2) return dot_d(k, m, d);
    double s = 0.0;
    for (int t = 0; t < d; ++t) {
        double e = (double)k[t] - m[t];
        s += e * e;
    }
    return -0.5 * s;
}

/* Initial centroids. The paper does not say how k-means is seeded; this
 * build seeds deterministically by stride: centroid c starts at the key of
 * clustered offset c * floor(n / C). */
void ckvo_init_m(const float *keys, int n, int d, int C, int mode, int metric, double *mu,
                 double *mhat) {
    int stride = n / C;
    for (int c = 0; c < C; ++c) {
        const float *k = keys + (size_t)c * stride * d;
        for (int t = 0; t < d; ++t) mu[(size_t)c * d + t] = (double)k[t];
        assign_copy(mu + (size_t)c * d, d, mode, metric, mhat + (size_t)c * d);
    }
}

/* Assignment: each key joins the centroid of highest similarity; an exact
 * tie goes to the lowest c. Under cosine the key's own norm does not change
 * which centroid wins, so the score is k_i . muhat_c. gap (optional)
 * receives (best - second best) / ||k_i||, the top-2 margin in cosine units
 * under cosine. */
void ckvo_assign_m(const float *keys, int n, int d, const double *mhat, int C, int metric,
                   int32_t *labels, double *gap) {
    for (int i = 0; i < n; ++i) {
        const float *k = keys + (size_t)i * d;
        double best = -INFINITY, second = -INFINITY;
        int arg = 0;
        for (int c = 0; c < C; ++c) {
            double s = similarity(k, mhat + (size_t)c * d, d, metric);
            if (s > best) {
                second = best;
                best = s;
                arg = c;
            } else if (s > second) {
                second = s;
            }
        }
        labels[i] = arg;
        if (gap) {
            double kk = 0.0;
            for (int t = 0; t < d; ++t) kk += (double)k[t] * (double)k[t];
            double kn = sqrt(kk);
            if (C == 1) gap[i] = INFINITY;
            else gap[i] = kn > 0.0 ? (best - second) / kn : 0.0;
        }
    }
}

/* Update: each centroid becomes the mean of the raw keys assigned to it. A
 * cluster with no keys keeps its previous mu and assignment copy; under
 * cosine so does one whose mean is the zero vector (it has no direction).
 * sizes receives the member counts. */
void ckvo_update_m(const float *keys, int n, int d, const int32_t *labels, int C, int mode,
                   int metric, double *mu, double *mhat, int32_t *sizes) {
    double *sum = (double *)calloc((size_t)C * d, sizeof(double));
    int32_t *cnt = (int32_t *)calloc((size_t)C, sizeof(int32_t));
    for (int i = 0; i < n; ++i) {
        int c = labels[i];
        cnt[c] += 1;
        for (int t = 0; t < d; ++t) sum[(size_t)c * d + t] += (double)keys[(size_t)i * d + t];
    }
    for (int c = 0; c < C; ++c) {
        sizes[c] = cnt[c];
        if (cnt[c] == 0) continue;
        double ss = 0.0;
        for (int t = 0; t < d; ++t) {
            double m = sum[(size_t)c * d + t] / (double)cnt[c];
            ss += m * m;
        }
        if (metric == CKVO_METRIC_COSINE && ss == 0.0) continue;
        for (int t = 0; t < d; ++t) mu[(size_t)c * d + t] = sum[(size_t)c * d + t] / (double)cnt[c];
        assign_copy(mu + (size_t)c * d, d, mode, metric, mhat + (size_t)c * d);
    }
    free(sum);
    free(cnt);
}

/* Cluster metadata, "IV.C Selection and Indexing": sizes, their prefix sums
 * and the token indices sorted by cluster. Within a cluster, tokens keep
 * ascending position (a stable bucket sort). offsets and perm are absolute:
 * offsets[c] counts from perm_base, perm holds positions tok_begin + i. */
void ckvo_index(const int32_t *labels, int n, int C, int tok_begin, int perm_base,
                int32_t *offsets, int32_t *perm) {
    int32_t *cnt = (int32_t *)calloc((size_t)C + 1, sizeof(int32_t));
    for (int i = 0; i < n; ++i) cnt[labels[i]] += 1;
    offsets[0] = perm_base;
    for (int c = 0; c < C; ++c) offsets[c + 1] = offsets[c] + cnt[c];
    int32_t *next = (int32_t *)malloc(((size_t)C + 1) * sizeof(int32_t));
    for (int c = 0; c < C; ++c) next[c] = offsets[c] - perm_base;
    for (int i = 0; i < n; ++i) perm[next[labels[i]]++] = tok_begin + i;
    free(next);
    free(cnt);
}

/* The whole clustering of one problem: strided init, then T rounds of
 * (assign, update) under the given similarity, then the index of the final
 * labels. Optional histories: labels_hist [T][n] (labels of round t),
 * mhat_hist [T+1][C][d] (the assignment copy each round used, plus the final
 * one), gap_hist [T][n]. T >= 1. */
void ckvo_kmeans_m(const float *keys, int n, int d, int C, int T, int mode, int metric,
                   int tok_begin, int perm_base, double *mu, double *mhat, int32_t *labels,
                   int32_t *sizes, int32_t *offsets, int32_t *perm, int32_t *labels_hist,
                   double *mhat_hist, double *gap_hist) {
    ckvo_init_m(keys, n, d, C, mode, metric, mu, mhat);
    for (int t = 0; t < T; ++t) {
        if (mhat_hist) memcpy(mhat_hist + (size_t)t * C * d, mhat, sizeof(double) * (size_t)C * d);
        ckvo_assign_m(keys, n, d, mhat, C, metric, labels,
                      gap_hist ? gap_hist + (size_t)t * n : NULL);
        if (labels_hist) memcpy(labels_hist + (size_t)t * n, labels, sizeof(int32_t) * (size_t)n);
        ckvo_update_m(keys, n, d, labels, C, mode, metric, mu, mhat, sizes);
    }
    if (mhat_hist) memcpy(mhat_hist + (size_t)T * C * d, mhat, sizeof(double) * (size_t)C * d);
    ckvo_index(labels, n, C, tok_begin, perm_base, offsets, perm);
}

/* The method's clustering (cosine similarity). */
void ckvo_init(const float *keys, int n, int d, int C, int mode, double *mu, double *muhat) {
    ckvo_init_m(keys, n, d, C, mode, CKVO_METRIC_COSINE, mu, muhat);
}

void ckvo_assign(const float *keys, int n, int d, const double *muhat, int C,
                 int32_t *labels, double *gap) {
    ckvo_assign_m(keys, n, d, muhat, C, CKVO_METRIC_COSINE, labels, gap);
}

void ckvo_update(const float *keys, int n, int d, const int32_t *labels, int C, int mode,
                 double *mu, double *muhat, int32_t *sizes) {
    ckvo_update_m(keys, n, d, labels, C, mode, CKVO_METRIC_COSINE, mu, muhat, sizes);
}

void ckvo_kmeans(const float *keys, int n, int d, int C, int T, int mode, int tok_begin,
                 int perm_base, double *mu, double *muhat, int32_t *labels, int32_t *sizes,
                 int32_t *offsets, int32_t *perm, int32_t *labels_hist, double *muhat_hist,
                 double *gap_hist) {
    ckvo_kmeans_m(keys, n, d, C, T, mode, CKVO_METRIC_COSINE, tok_begin, perm_base, mu, muhat,
                  labels, sizes, offsets, perm, labels_hist, muhat_hist, gap_hist);
}

/* The copy of the centroids used for scoring: mu rounded to the storage
 * format. */
void ckvo_round(const double *x, size_t count, int mode, double *out) {
    for (size_t j = 0; j < count; ++j) out[j] = round_to(x[j], mode);
}

/* ---- selection: "III.C Selection at the Granularity of Semantic Clusters",
 * "IV.C Selection and Indexing" ----------------------------------------- */

/* Cluster score: the attention logit of the query against the centroid,
 * summed over the G query heads that share the KV head. Softmax is monotone,
 * so ranking by logits ranks by attention weight; the 1/sqrt(d) factor is
 * dropped. Fixed fp32 order: channels are split into 32 consecutive groups of
 * ceil(d/32); group l accumulates fmaf(q[t], mu[t], acc) from 0 in channel
 * order; the 32 group sums are combined pairwise by the butterfly
 * v[l] = v[l] + v[l ^ o] for o = 16, 8, 4, 2, 1 (v[0] is the head's score);
 * head scores are added in head order: ((s0 + s1) + s2) + ... */
static float score_one_head(const float *q, const float *m, int d) {
    float v[32];
    int per = (d + 31) / 32;
    for (int l = 0; l < 32; ++l) {
        float acc = 0.0f;
        for (int j = 0; j < per; ++j) {
            int t = l * per + j;
            if (t < d) acc = fmaf(q[t], m[t], acc);
        }
        v[l] = acc;
    }
    for (int o = 16; o >= 1; o >>= 1) {
        float w[32];
        for (int l = 0; l < 32; ++l) w[l] = v[l] + v[l ^ o];
        memcpy(v, w, sizeof(v));
    }
    return v[0];
}

void ckvo_score(const float *q, int G, int d, const float *mu_lp, int C, float *s) {
    for (int c = 0; c < C; ++c) {
        float tot = 0.0f;
        for (int g = 0; g < G; ++g) {
            float h = score_one_head(q + (size_t)g * d, mu_lp + (size_t)c * d, d);
            tot = (g == 0) ? h : tot + h;
        }
        s[c] = tot;
    }
}

typedef struct {
    float s;
    int32_t c;
} ranked_t;

/* higher score first; equal scores: lower cluster id first */
static int rank_cmp(const void *a, const void *b) {
    const ranked_t *x = (const ranked_t *)a, *y = (const ranked_t *)b;
    if (x->s > y->s) return -1;
    if (x->s < y->s) return 1;
    return (x->c > y->c) - (x->c < y->c);
}

/* Budgeted recall: walk clusters from the highest score down; a cluster that
 * fits in what is left of the budget is taken whole; the first one that does
 * not fit is trimmed to its first (lowest-position) tokens so that exactly the
 * budget is used, and the walk stops there. Empty clusters take nothing.
 * sel_idx receives positions in rank order, then perm order; returns the
 * number selected, min(budget, total clustered tokens). */
int ckvo_select(const float *s, int C, const int32_t *offsets, const int32_t *perm,
                int perm_base, int budget, int32_t *sel_idx) {
    ranked_t *r = (ranked_t *)malloc(sizeof(ranked_t) * (size_t)(C > 0 ? C : 1));
    for (int c = 0; c < C; ++c) {
        r[c].s = s[c];
        r[c].c = c;
    }
    qsort(r, (size_t)C, sizeof(ranked_t), rank_cmp);
    int taken = 0;
    for (int j = 0; j < C && taken < budget; ++j) {
        int c = r[j].c;
        int n_c = offsets[c + 1] - offsets[c];
        int take = n_c <= budget - taken ? n_c : budget - taken;
        for (int k = 0; k < take; ++k) sel_idx[taken + k] = perm[offsets[c] - perm_base + k];
        taken += take;
    }
    free(r);
    return taken;
}

/* ---- caching the KV of selected clusters: "D. Caching KV of Selected
 * Tokens" ---------------------------------------------------------------- */

/* The clusters one selection recalls, in rank order: non-empty clusters
 * walked from the highest score until the budget is met, as in ckvo_select.
 * taken[j] receives how many tokens of clusters[j] are recalled (all of them
 * except in a trimmed last cluster). Returns the number of clusters. */
int ckvo_selected_clusters(const float *s, int C, const int32_t *offsets, int budget,
                           int32_t *clusters, int32_t *taken) {
    ranked_t *r = (ranked_t *)malloc(sizeof(ranked_t) * (size_t)(C > 0 ? C : 1));
    for (int c = 0; c < C; ++c) {
        r[c].s = s[c];
        r[c].c = c;
    }
    qsort(r, (size_t)C, sizeof(ranked_t), rank_cmp);
    int total = 0, m = 0;
    for (int j = 0; j < C && total < budget; ++j) {
        int c = r[j].c;
        int n_c = offsets[c + 1] - offsets[c];
        if (n_c == 0) continue;
        int take = n_c <= budget - total ? n_c : budget - total;
        clusters[m] = c;
        taken[m] = take;
        ++m;
        total += take;
    }
    free(r);
    return m;
}

/* One decoding step of a cache that keeps the clusters selected in the last R
 * steps: cluster c is cached at `step` when it was selected at one of steps
 * step - R .. step - 1 (last[c] holds the last step that selected it; a
 * never-selected cluster holds a value far below any step). Counts the hits
 * among this step's clusters and the recalled tokens of those hits, lists the
 * misses (the clusters to load) in rank order, then records this step's
 * selection in last. Returns the number of hits. */
int ckvo_cache_step(const int32_t *clusters, const int32_t *taken, int n, int step, int R,
                    int32_t *last, int32_t *misses, int32_t *hit_tokens) {
    int hits = 0, nm = 0, ht = 0;
    for (int j = 0; j < n; ++j) {
        int c = clusters[j];
        int cached = R > 0 && last[c] < step && last[c] >= step - R;
        if (cached) {
            hits += 1;
            ht += taken[j];
        } else {
            misses[nm++] = c;
        }
    }
    for (int j = 0; j < n; ++j) last[clusters[j]] = step;
    *hit_tokens = ht;
    return hits;
}

/* ---- attention: "II.A LLM Inference and KV Cache" ---------------------- */

/* out[g] = sum_j softmax_j(scale * q_g . k_j) v_j over the rows listed in
 * rows (positions into K and V, [L][d]), summed in the order given. */
void ckvo_attend(const float *q, int G, int d, const float *K, const float *V,
                 const int32_t *rows, int n_rows, double scale, double *out) {
    double *logit = (double *)malloc(sizeof(double) * (size_t)(n_rows > 0 ? n_rows : 1));
    for (int g = 0; g < G; ++g) {
        const float *qg = q + (size_t)g * d;
        double m = -INFINITY;
        for (int j = 0; j < n_rows; ++j) {
            const float *k = K + (size_t)rows[j] * d;
            double s = 0.0;
            for (int t = 0; t < d; ++t) s += (double)qg[t] * (double)k[t];
            logit[j] = scale * s;
            if (logit[j] > m) m = logit[j];
        }
        double z = 0.0;
        double *o = out + (size_t)g * d;
        for (int t = 0; t < d; ++t) o[t] = 0.0;
        for (int j = 0; j < n_rows; ++j) {
            double w = exp(logit[j] - m);
            z += w;
            const float *v = V + (size_t)rows[j] * d;
            for (int t = 0; t < d; ++t) o[t] += w * (double)v[t];
        }
        for (int t = 0; t < d; ++t) o[t] = n_rows > 0 ? o[t] / z : 0.0;
    }
    free(logit);
}

/* The attended set of one decode step, sorted by position: the sink tokens
 * [0, sink), the recalled tokens sel_idx[0..sel_cnt), and the recent tokens
 * [tail_begin, tail_end). Returns its size. */
int ckvo_attended_rows(int sink, const int32_t *sel_idx, int sel_cnt, int tail_begin,
                       int tail_end, int32_t *rows) {
    int n = 0;
    for (int j = 0; j < sink; ++j) rows[n++] = j;
    int first_sel = n;
    for (int j = 0; j < sel_cnt; ++j) rows[n++] = sel_idx[j];
    /* insertion sort of the recalled positions (they lie in [sink, tail_begin)) */
    for (int a = first_sel + 1; a < n; ++a) {
        int32_t x = rows[a];
        int b = a - 1;
        while (b >= first_sel && rows[b] > x) {
            rows[b + 1] = rows[b];
            --b;
        }
        rows[b + 1] = x;
    }
    for (int j = tail_begin; j < tail_end; ++j) rows[n++] = j;
    return n;
}

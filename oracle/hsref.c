/*
 * hsref.c -- fp64 CPU oracle for the HySparse hybrid block.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file: it is used by the tests, by the package's smoke check and by
 * the benchmark's CPU-baseline leg.  It shares no code, header, table or
 * constant with the CUDA library.
 *
 * What it computes (every step is the plain definition, in fp64, one query
 * row at a time, with no blocking, fusion or reordering):
 *
 *   pos(i) = Lkv - Lq + i            bottom-right-aligned causal position
 *   G      = Hq / Hkv                query head h reads KV head h / G
 *
 *   Full layer ("the full attention layer is the oracle of token importance":
 *   HySparse abstract; intelliparadigm write-up section 2.1):
 *     s_hj   = scale * <q_h, k_j>                     j = 0 .. pos(i)
 *     P_hj   = exp(s_hj - m_h) / l_h,  m_h = max_j s_hj,  l_h = sum_j exp(s_hj - m_h)
 *     O_h    = sum_j P_hj v_j,         LSE_h = m_h + ln l_h
 *   Importance score, per query row and KV head g (the sum over the group's
 *   query heads of the softmax probabilities; the write-up's section 3.1 says
 *   only that the full layer's importance scores are reused):
 *     S_gj   = sum_{h in group g} P_hj
 *   Top-k (write-up section 2.2, global branch over the full layer's TopK
 *   indices; baidu article "Top-K selection"): the k keys that come first in
 *   the order (-S_gj, j), i.e. the largest scores with ties going to the lower
 *   key index; a row with pos+1 <= k takes all its keys; the set is written
 *   in ascending key order and padded with -1.
 *   Sparse layer (write-up section 2.2, dual-branch sparse attention):
 *     Og_h   = softmax attention of q'_h over { k_j : j in idx_g }
 *     Ol_h   = softmax attention of q'_h over { k_j : pos-w+1 <= j <= pos }
 *     out_h  = sigma(gl_h) * Og_h + (1 - sigma(gl_h)) * Ol_h,
 *              sigma(x) = 1 / (1 + exp(-x))
 *   An empty global set (only possible with a caller-made index list of -1)
 *   gives Og = 0.
 *   Own-window variant (the same section: the global branch computes "on the
 *   shared KV cache", while the local branch "maintains a 128-token sliding
 *   window"; read as: each sparse layer keeps its own K/V for its window):
 *     Ol_h   = softmax attention of q'_h over { kw_j : pos-w+1 <= j <= pos }
 *   with kw, vw the layer's own keys and values, stored for the last Lwin
 *   positions of the sequence: buffer row r holds position Lkv - Lwin + r.
 *
 * Layouts (all row-major, C order):
 *   q_rows  [nrows][Hq][d]     float   the listed rows' queries
 *   k, v    [B][Lkv][Hkv][d]   float   the shared KV cache
 *   kw, vw  [B][Lwin][Hkv][d]  float   a sparse layer's own window K/V (positions Lkv-Lwin ..)
 *   out     [nrows][Hq][d]     double
 *   lse     [nrows][Hq]        double
 *   scores  [nrows][Hkv][Lkv]  double  (entries j > pos are set to 0)
 *   idx     [nrows][Hkv][topk] int32
 *   gate    [nrows][Hq]        float   gate logits
 *
 * Return values: 0 on success, -1 on a bad argument, -2 on an index list
 * that is not strictly ascending valid keys followed by -1 padding, -3 on an
 * allocation failure.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static double dot_fd(const float *a, const float *b, int d) {
    double acc = 0.0;
    for (int t = 0; t < d; ++t) acc += (double)a[t] * (double)b[t];
    return acc;
}

static const float *kv_row(const float *base, int b, int j, int g, int Lkv, int Hkv, int d) {
    return base + (((size_t)b * Lkv + j) * Hkv + g) * (size_t)d;
}

/* softmax attention of one query over an explicit key list; out[d] (may be
 * NULL), returns the log-sum-exp; adds P_j to acc_p[t] when acc_p != NULL.  An
 * empty list writes zeros and returns -INFINITY. */
static double attend_list(const float *q, const float *k, const float *v, int b, int g,
                          int Lkv, int Hkv, int d, double scale, const int *keys, int nkeys,
                          double *s, double *out, double *acc_p) {
    if (out) memset(out, 0, sizeof(double) * (size_t)d);
    if (nkeys <= 0) return -INFINITY;
    double m = -INFINITY;
    for (int t = 0; t < nkeys; ++t) {
        s[t] = scale * dot_fd(q, kv_row(k, b, keys[t], g, Lkv, Hkv, d), d);
        if (s[t] > m) m = s[t];
    }
    double l = 0.0;
    for (int t = 0; t < nkeys; ++t) l += exp(s[t] - m);
    for (int t = 0; t < nkeys; ++t) {
        double p = exp(s[t] - m) / l;
        if (acc_p) acc_p[t] += p;
        if (out) {
            const float *vr = kv_row(v, b, keys[t], g, Lkv, Hkv, d);
            for (int c = 0; c < d; ++c) out[c] += p * (double)vr[c];
        }
    }
    return m + log(l);
}

static int check_shape(int B, int Lq, int Lkv, int Hq, int Hkv, int d) {
    if (B < 1 || Lq < 1 || Lkv < 1 || Hq < 1 || Hkv < 1 || d < 1) return -1;
    if (Lq > Lkv || Hq % Hkv != 0) return -1;
    return 0;
}

/* Full layer for the listed rows: O, LSE and the group-summed importance. */
int hsref_full_rows(int B, int Lq, int Lkv, int Hq, int Hkv, int d, double scale,
                    const float *q_rows, const float *k, const float *v,
                    const int *row_b, const int *row_i, int nrows,
                    double *out, double *lse, double *scores) {
    if (check_shape(B, Lq, Lkv, Hq, Hkv, d) || nrows < 0) return -1;
    for (int r = 0; r < nrows; ++r)
        if (row_b[r] < 0 || row_b[r] >= B || row_i[r] < 0 || row_i[r] >= Lq) return -1;
    const int G = Hq / Hkv;
    int err = 0;
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int r = 0; r < nrows; ++r) {
        for (int g = 0; g < Hkv; ++g) {
            const int b = row_b[r];
            const int pos = Lkv - Lq + row_i[r];
            const int n = pos + 1;
            int *keys = (int *)malloc(sizeof(int) * (size_t)n);
            double *s = (double *)malloc(sizeof(double) * (size_t)n);
            double *acc = (double *)calloc((size_t)n, sizeof(double));
            double *o = (double *)malloc(sizeof(double) * (size_t)d);
            if (!keys || !s || !acc || !o) {
#pragma omp atomic write
                err = -3;
            } else {
                for (int j = 0; j < n; ++j) keys[j] = j;
                for (int hh = 0; hh < G; ++hh) {
                    const int h = g * G + hh;
                    const float *q = q_rows + ((size_t)r * Hq + h) * (size_t)d;
                    double l = attend_list(q, k, v, b, g, Lkv, Hkv, d, scale, keys, n, s, o, acc);
                    if (out) memcpy(out + ((size_t)r * Hq + h) * (size_t)d, o, sizeof(double) * (size_t)d);
                    if (lse) lse[(size_t)r * Hq + h] = l;
                }
                if (scores) {
                    double *row = scores + ((size_t)r * Hkv + g) * (size_t)Lkv;
                    memcpy(row, acc, sizeof(double) * (size_t)n);
                    for (int j = n; j < Lkv; ++j) row[j] = 0.0;
                }
            }
            free(keys); free(s); free(acc); free(o);
        }
    }
    return err;
}

typedef struct { double s; int j; } keyed;

/* order (-S, j): larger score first, equal scores by the lower key index */
static int cmp_rank(const void *a, const void *b) {
    const keyed *x = (const keyed *)a, *y = (const keyed *)b;
    if (x->s > y->s) return -1;
    if (x->s < y->s) return 1;
    return (x->j > y->j) - (x->j < y->j);
}

static int cmp_int(const void *a, const void *b) {
    int x = *(const int *)a, y = *(const int *)b;
    return (x > y) - (x < y);
}

/* Top-k of one score row over its first n entries into idx[topk]. */
static void topk_one(const double *s, int n, int topk, int *idx, keyed *tmp) {
    for (int j = 0; j < n; ++j) { tmp[j].s = s[j]; tmp[j].j = j; }
    qsort(tmp, (size_t)n, sizeof(keyed), cmp_rank);
    int take = n < topk ? n : topk;
    for (int t = 0; t < take; ++t) idx[t] = tmp[t].j;
    qsort(idx, (size_t)take, sizeof(int), cmp_int);
    for (int t = take; t < topk; ++t) idx[t] = -1;
}

/* Top-k for nrows score rows.  Row r has n_valid[r] candidate keys
 * (pos+1) and starts at scores + r*ld. */
int hsref_topk_rows(const double *scores, long long ld, const int *n_valid, int nrows,
                    int topk, int *idx) {
    if (nrows < 0 || topk < 1 || ld < 1) return -1;
    for (int r = 0; r < nrows; ++r)
        if (n_valid[r] < 0 || n_valid[r] > ld) return -1;
    int err = 0;
#pragma omp parallel for schedule(dynamic, 4)
    for (int r = 0; r < nrows; ++r) {
        int n = n_valid[r];
        keyed *tmp = (keyed *)malloc(sizeof(keyed) * (size_t)(n > 0 ? n : 1));
        if (!tmp) {
#pragma omp atomic write
            err = -3;
            continue;
        }
        topk_one(scores + (size_t)r * (size_t)ld, n, topk, idx + (size_t)r * topk, tmp);
        free(tmp);
    }
    return err;
}

/* Valid keys of an index list: strictly ascending keys in [0, pos] followed
 * only by -1.  Returns the count, or -2 when the list breaks that form. */
static int index_list_keys(const int *lst, int topk, int pos) {
    int n = 0, prev = -1, padded = 0;
    for (int t = 0; t < topk; ++t) {
        int j = lst[t];
        if (j == -1) { padded = 1; continue; }
        if (padded || j < 0 || j > pos || j <= prev) return -2;
        prev = j;
        ++n;
    }
    return n;
}

static double sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }

/* Sparse layer for the listed rows; the window branch reads kw / vw (Lwin
 * rows per batch element, positions Lkv - Lwin ..) when kw != NULL, else the
 * shared cache.  out_g / out_l may be NULL. */
static int sparse_rows_impl(int B, int Lq, int Lkv, int Hq, int Hkv, int d, double scale,
                            const float *q_rows, const float *k, const float *v,
                            const float *kw, const float *vw, int Lwin,
                            const int *row_b, const int *row_i, int nrows,
                            const int *idx, int topk, const float *gate, int window,
                            double *out, double *out_g, double *out_l) {
    if (check_shape(B, Lq, Lkv, Hq, Hkv, d) || nrows < 0 || topk < 1 || window < 1) return -1;
    for (int r = 0; r < nrows; ++r)
        if (row_b[r] < 0 || row_b[r] >= B || row_i[r] < 0 || row_i[r] >= Lq) return -1;
    const int woff = kw ? Lkv - Lwin : 0;   /* position of window-buffer row 0 */
    if (kw) {
        if (!vw || Lwin < 1 || Lwin > Lkv) return -1;
        for (int r = 0; r < nrows; ++r) {
            const int pos = Lkv - Lq + row_i[r];
            const int lo = pos - window + 1 < 0 ? 0 : pos - window + 1;
            if (lo < woff) return -1;        /* the window reaches below the buffer */
        }
    }
    const int G = Hq / Hkv;
    int err = 0;
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int r = 0; r < nrows; ++r) {
        for (int g = 0; g < Hkv; ++g) {
            const int b = row_b[r];
            const int pos = Lkv - Lq + row_i[r];
            const int *lst = idx + ((size_t)r * Hkv + g) * (size_t)topk;
            int ng = index_list_keys(lst, topk, pos);
            if (ng < 0) {
#pragma omp atomic write
                err = -2;
                continue;
            }
            int lo = pos - window + 1;
            if (lo < 0) lo = 0;
            int nl = pos - lo + 1;
            int cap = (ng > nl ? ng : nl);
            int *keys_g = (int *)malloc(sizeof(int) * (size_t)(ng > 0 ? ng : 1));
            int *keys_l = (int *)malloc(sizeof(int) * (size_t)nl);
            double *s = (double *)malloc(sizeof(double) * (size_t)cap);
            double *og = (double *)malloc(sizeof(double) * (size_t)d);
            double *ol = (double *)malloc(sizeof(double) * (size_t)d);
            if (!keys_g || !keys_l || !s || !og || !ol) {
#pragma omp atomic write
                err = -3;
            } else {
                int n = 0;
                for (int t = 0; t < topk; ++t)
                    if (lst[t] != -1) keys_g[n++] = lst[t];
                for (int t = 0; t < nl; ++t) keys_l[t] = lo + t - woff;   /* rows of the window's buffer */
                for (int hh = 0; hh < G; ++hh) {
                    const int h = g * G + hh;
                    const size_t o = ((size_t)r * Hq + h) * (size_t)d;
                    const float *q = q_rows + o;
                    attend_list(q, k, v, b, g, Lkv, Hkv, d, scale, keys_g, ng, s, og, NULL);
                    if (kw)
                        attend_list(q, kw, vw, b, g, Lwin, Hkv, d, scale, keys_l, nl, s, ol, NULL);
                    else
                        attend_list(q, k, v, b, g, Lkv, Hkv, d, scale, keys_l, nl, s, ol, NULL);
                    double gs = sigmoid((double)gate[(size_t)r * Hq + h]);
                    for (int c = 0; c < d; ++c) {
                        if (out) out[o + c] = gs * og[c] + (1.0 - gs) * ol[c];
                        if (out_g) out_g[o + c] = og[c];
                        if (out_l) out_l[o + c] = ol[c];
                    }
                }
            }
            free(keys_g); free(keys_l); free(s); free(og); free(ol);
        }
    }
    return err;
}

int hsref_sparse_rows(int B, int Lq, int Lkv, int Hq, int Hkv, int d, double scale,
                      const float *q_rows, const float *k, const float *v,
                      const int *row_b, const int *row_i, int nrows,
                      const int *idx, int topk, const float *gate, int window,
                      double *out, double *out_g, double *out_l) {
    return sparse_rows_impl(B, Lq, Lkv, Hq, Hkv, d, scale, q_rows, k, v, NULL, NULL, 0, row_b, row_i, nrows,
                            idx, topk, gate, window, out, out_g, out_l);
}

/* The sparse layer with its own window K/V (kw, vw: [B][Lwin][Hkv][d],
 * positions Lkv - Lwin .. Lkv - 1); every listed row's window must lie in it. */
int hsref_sparse_rows_own_window(int B, int Lq, int Lkv, int Hq, int Hkv, int d, double scale,
                                 const float *q_rows, const float *k, const float *v,
                                 const float *kw, const float *vw, int Lwin,
                                 const int *row_b, const int *row_i, int nrows,
                                 const int *idx, int topk, const float *gate, int window,
                                 double *out, double *out_g, double *out_l) {
    if (!kw) return -1;
    return sparse_rows_impl(B, Lq, Lkv, Hq, Hkv, d, scale, q_rows, k, v, kw, vw, Lwin, row_b, row_i, nrows,
                            idx, topk, gate, window, out, out_g, out_l);
}

/* A whole hybrid block for the listed rows: the full layer, its top-k, then
 * n_sparse sparse layers that reuse the same index lists and KV cache.
 *   q_sparse_rows [n_sparse][nrows][Hq][d], gate_rows [n_sparse][nrows][Hq]
 *   out_full [nrows][Hq][d], idx [nrows][Hkv][topk],
 *   out_sparse [n_sparse][nrows][Hq][d]
 * Holds the listed rows' scores, nrows*Hkv*Lkv doubles, while it runs. */
int hsref_block_rows(int B, int Lq, int Lkv, int Hq, int Hkv, int d, double scale,
                     const float *q_rows, const float *k, const float *v,
                     const int *row_b, const int *row_i, int nrows,
                     int n_sparse, const float *q_sparse_rows, const float *gate_rows,
                     int topk, int window,
                     double *out_full, int *idx, double *out_sparse) {
    if (check_shape(B, Lq, Lkv, Hq, Hkv, d) || nrows < 0 || topk < 1 || window < 1 ||
        n_sparse < 0)
        return -1;
    for (int r = 0; r < nrows; ++r)
        if (row_b[r] < 0 || row_b[r] >= B || row_i[r] < 0 || row_i[r] >= Lq) return -1;
    double *sc = (double *)malloc(sizeof(double) * (size_t)nrows * Hkv * (size_t)Lkv);
    int *nv = (int *)malloc(sizeof(int) * (size_t)nrows * Hkv + 1);
    if (!sc || !nv) { free(sc); free(nv); return -3; }
    int rc = hsref_full_rows(B, Lq, Lkv, Hq, Hkv, d, scale, q_rows, k, v, row_b, row_i, nrows,
                             out_full, NULL, sc);
    for (int r = 0; r < nrows; ++r)
        for (int g = 0; g < Hkv; ++g) nv[(size_t)r * Hkv + g] = Lkv - Lq + row_i[r] + 1;
    if (rc == 0) rc = hsref_topk_rows(sc, Lkv, nv, nrows * Hkv, topk, idx);
    for (int s = 0; s < n_sparse && rc == 0; ++s) {
        const size_t qo = (size_t)s * nrows * Hq * (size_t)d;
        rc = hsref_sparse_rows(B, Lq, Lkv, Hq, Hkv, d, scale, q_sparse_rows + qo, k, v,
                               row_b, row_i, nrows, idx, topk,
                               gate_rows + (size_t)s * nrows * Hq, window,
                               out_sparse + qo, NULL, NULL);
    }
    free(sc); free(nv);
    return rc;
}

int hsref_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void hsref_set_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

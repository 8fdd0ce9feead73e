/*
 * oracle.c -- plain, slow CPU restatement of content-adaptive block-sparse
 * video attention, in fp64.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or call
 * this file; only the tests, the package smoke check and the benchmark's CPU
 * baseline do.  It shares no code, header, table or helper with the CUDA path.
 *
 * Sources (the web pages this method is described on):
 *   NABLA: Neighborhood Adaptive Block-Level Attention (gist.science summary of
 *     arXiv 2507.13546), "Methodology" items 1 (token reordering / fractal
 *     flattening), 2 (block pooling, reduced attention, CDF threshold,
 *     expansion) and 3 (hybrid with Sliding Tile Attention, M = M_nabla OR M_STA).
 *   Sparse VideoGen2 (gist.science summary of arXiv 2505.18875), section 2B
 *     (top-p: clusters sorted by estimated score, taken until the cumulative
 *     score reaches p) and section 2A (permuted attention equals dense
 *     attention).
 *
 * Readings where the pages are silent (kept identical on both sides):
 *   - a block is one P x P spatial patch of one frame (P = 8 -> 64 tokens);
 *   - flattening is one level: frame, then patch row, patch column, then the
 *     token's row and column inside the patch, all row-major;
 *   - pooled scores are scaled by 1/sqrt(d); the CDF rule keeps the smallest
 *     prefix of the descending-sorted row whose mass reaches 1 - thr, equal
 *     probabilities going to the lower block index; thr = 0 keeps every block;
 *   - the STA window keeps key blocks within a Chebyshev radius (rt, rh, rw)
 *     in (frame, patch row, patch column), clipped at the grid edges;
 *   - attention is bidirectional; LSE is the natural log of the softmax
 *     denominator including the scale.
 *
 * Build: gcc -O2 -fopenmp -fPIC -shared oracle.c -o liboracle.so -lm
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* bf16 -> double is exact: a bf16 is the top half of an IEEE float. */
static double bf16_value(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * O1. Fractal flattening order (NABLA, Methodology item 1): tokens of each
 * P x P spatial patch are grouped into one contiguous run, the time axis keeps
 * its order.  order[k] = raster index (t*H + y)*W + x of the token that sits at
 * flattened position k.  Built by enumerating the tokens in flattened order.
 */
void oracle_fractal_order(int T, int H, int W, int P, int64_t *order)
{
    int64_t k = 0;
    for (int t = 0; t < T; ++t)
        for (int py = 0; py < H / P; ++py)
            for (int px = 0; px < W / P; ++px)
                for (int iy = 0; iy < P; ++iy)
                    for (int ix = 0; ix < P; ++ix) {
                        int y = py * P + iy;
                        int x = px * P + ix;
                        order[k++] = ((int64_t)t * H + y) * W + x;
                    }
}

/* y[bh, k, :] = x[bh, order[k], :] for every (batch, head) slice. */
void oracle_flatten(const uint16_t *x, uint16_t *y, int64_t BH, int T, int H,
                    int W, int P, int d)
{
    int64_t N = (int64_t)T * H * W;
    int64_t *order = (int64_t *)malloc(sizeof(int64_t) * N);
    oracle_fractal_order(T, H, W, P, order);
    for (int64_t bh = 0; bh < BH; ++bh)
        for (int64_t k = 0; k < N; ++k)
            memcpy(y + (bh * N + k) * d, x + (bh * N + order[k]) * d,
                   sizeof(uint16_t) * d);
    free(order);
}

/* Inverse of oracle_flatten: x[bh, order[k], :] = y[bh, k, :]. */
void oracle_unflatten_f64(const double *y, double *x, int64_t BH, int T, int H,
                          int W, int P, int d)
{
    int64_t N = (int64_t)T * H * W;
    int64_t *order = (int64_t *)malloc(sizeof(int64_t) * N);
    oracle_fractal_order(T, H, W, P, order);
    for (int64_t bh = 0; bh < BH; ++bh)
        for (int64_t k = 0; k < N; ++k)
            memcpy(x + (bh * N + order[k]) * d, y + (bh * N + k) * d,
                   sizeof(double) * d);
    free(order);
}

void oracle_unflatten(const uint16_t *y, uint16_t *x, int64_t BH, int T, int H,
                      int W, int P, int d)
{
    int64_t N = (int64_t)T * H * W;
    int64_t *order = (int64_t *)malloc(sizeof(int64_t) * N);
    oracle_fractal_order(T, H, W, P, order);
    for (int64_t bh = 0; bh < BH; ++bh)
        for (int64_t k = 0; k < N; ++k)
            memcpy(x + (bh * N + order[k]) * d, y + (bh * N + k) * d,
                   sizeof(uint16_t) * d);
    free(order);
}

/*
 * O2. Block mean pooling (NABLA, Methodology item 2, "downsampling"): every
 * run of S consecutive flattened tokens is one block; its pooled vector is the
 * arithmetic mean of the S token vectors.  xp has shape [BH, N/S, d].
 */
void oracle_pool(const uint16_t *xf, double *xp, int64_t BH, int64_t N, int d,
                 int S)
{
    int64_t Nb = N / S;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < BH * Nb; ++r) {
        for (int j = 0; j < d; ++j) {
            double sum = 0.0;
            for (int i = 0; i < S; ++i)
                sum += bf16_value(xf[(r * S + i) * d + j]);
            xp[r * d + j] = sum / S;
        }
    }
}

/*
 * O3. Reduced attention (NABLA, Methodology item 2, "reduced attention"): the
 * full attention map over pooled blocks, A[r, :] = softmax(qp_r . kp_c / sqrt d)
 * over all key blocks c of the same head.  `rows` lists global block-row ids
 * bh*Nb + r (NULL = all rows); a_out receives one row of Nb per listed row.
 */
static void reduced_row(const double *qp, const double *kp, int64_t row, int Nb,
                        int d, double *a)
{
    int64_t bh = row / Nb;
    const double *q = qp + row * d;
    double scale = 1.0 / sqrt((double)d);
    double m = -INFINITY;
    for (int c = 0; c < Nb; ++c) {
        const double *k = kp + (bh * Nb + c) * d;
        double s = 0.0;
        for (int j = 0; j < d; ++j)
            s += q[j] * k[j];
        a[c] = s * scale;
        if (a[c] > m)
            m = a[c];
    }
    double z = 0.0;
    for (int c = 0; c < Nb; ++c) {
        a[c] = exp(a[c] - m);
        z += a[c];
    }
    for (int c = 0; c < Nb; ++c)
        a[c] /= z;
}

void oracle_reduced_attention(const double *qp, const double *kp, int64_t BH,
                              int Nb, int d, const int64_t *rows, int64_t nrows,
                              double *a_out)
{
    if (!rows)
        nrows = BH * Nb;
#pragma omp parallel for schedule(dynamic, 16)
    for (int64_t i = 0; i < nrows; ++i)
        reduced_row(qp, kp, rows ? rows[i] : i, Nb, d, a_out + i * Nb);
}

/*
 * O4a. CDF / top-p selection of one row (NABLA, Methodology item 2, "CDF
 * threshold"; Sparse VideoGen2 section 2B).  Blocks are visited in descending
 * probability (equal probabilities: lower index first) and kept while the
 * mass of the blocks kept before them is still below 1 - thr, which keeps the
 * smallest prefix whose mass reaches 1 - thr.  thr = 0 keeps every block; if
 * the sums never reach 1 - thr every block is kept as well.
 *
 * diag (5 doubles, may be NULL) describes the cut: [0] mass of the kept prefix,
 * [1] mass of the prefix without its last block, [2] probability of the last
 * kept block, [3] probability of the first dropped block (-1 if none),
 * [4] number of kept blocks.
 */
typedef struct {
    double p;
    int idx;
} ranked;

static int ranked_cmp(const void *a, const void *b)
{
    const ranked *x = (const ranked *)a, *y = (const ranked *)b;
    if (x->p > y->p) return -1;
    if (x->p < y->p) return 1;
    return (x->idx > y->idx) - (x->idx < y->idx);
}

void oracle_select_row(const double *a, int n, double thr, uint8_t *keep,
                       double *diag)
{
    if (n <= 0)
        return;
    ranked *r = (ranked *)malloc(sizeof(ranked) * (size_t)n);
    for (int c = 0; c < n; ++c) {
        r[c].p = a[c];
        r[c].idx = c;
    }
    qsort(r, (size_t)n, sizeof(ranked), ranked_cmp);
    memset(keep, 0, (size_t)n);
    double before = 0.0, mass = 0.0;
    int kept = 0;
    for (int i = 0; i < n; ++i) {
        if (thr > 0.0 && mass >= 1.0 - thr)
            break;
        before = mass;
        mass += r[i].p;
        keep[r[i].idx] = 1;
        ++kept;
    }
    if (diag) {
        diag[0] = mass;
        diag[1] = before;
        diag[2] = kept > 0 ? r[kept - 1].p : -1.0;
        diag[3] = kept < n ? r[kept].p : -1.0;
        diag[4] = (double)kept;
    }
    free(r);
}

/*
 * O4b. Sliding-tile window (NABLA, Methodology item 3; STA in the problem
 * statement): query block r keeps key block c when their (frame, patch row,
 * patch column) coordinates differ by at most (rt, rh, rw); block index
 * = (t*Hb + py)*Wb + px in flattened order.
 */
int oracle_sta_keep(int64_t r, int64_t c, int Hb, int Wb, int rt, int rh, int rw)
{
    int64_t tr = r / ((int64_t)Hb * Wb), yr = (r / Wb) % Hb, xr = r % Wb;
    int64_t tc = c / ((int64_t)Hb * Wb), yc = (c / Wb) % Hb, xc = c % Wb;
    return llabs(tr - tc) <= rt && llabs(yr - yc) <= rh && llabs(xr - xc) <= rw;
}

/*
 * O4. Block mask: reduced attention row, CDF selection, then the union with
 * the STA window (M = M_nabla OR M_STA).  keep_out: nrows x Nb flags;
 * diag_out: nrows x 5 (see oracle_select_row), may be NULL.
 */
void oracle_block_mask(const double *qp, const double *kp, int64_t BH, int Nb,
                       int d, int Hb, int Wb, double thr, int use_sta, int rt,
                       int rh, int rw, const int64_t *rows, int64_t nrows,
                       uint8_t *keep_out, double *diag_out)
{
    if (!rows)
        nrows = BH * Nb;
#pragma omp parallel
    {
        double *a = (double *)malloc(sizeof(double) * (size_t)Nb);
#pragma omp for schedule(dynamic, 16)
        for (int64_t i = 0; i < nrows; ++i) {
            int64_t row = rows ? rows[i] : i;
            int64_t r = row % Nb;
            uint8_t *keep = keep_out + i * Nb;
            reduced_row(qp, kp, row, Nb, d, a);
            oracle_select_row(a, Nb, thr, keep, diag_out ? diag_out + i * 5 : NULL);
            if (use_sta)
                for (int c = 0; c < Nb; ++c)
                    if (oracle_sta_keep(r, c, Hb, Wb, rt, rh, rw))
                        keep[c] = 1;
        }
        free(a);
    }
}

/*
 * Static-ratio selection (DynamicRad summary, section 2, "Dual-Mode
 * Strategy", Static-Ratio mode: every row keeps a fixed share of its
 * blocks).  The page does not say which blocks; reading taken: the k blocks of
 * highest reduced-attention probability, ordered exactly as in the top-p rule
 * (probability descending, equal probabilities to the lower block index);
 * k >= n keeps the whole row, k <= 0 keeps nothing.  diag[0] is the last kept
 * probability, diag[1] the first dropped one (-1 where there is none).
 */
void oracle_select_topk_row(const double *a, int n, int k, uint8_t *keep,
                            double *diag)
{
    if (n <= 0)
        return;
    ranked *r = (ranked *)malloc(sizeof(ranked) * (size_t)n);
    for (int c = 0; c < n; ++c) {
        r[c].p = a[c];
        r[c].idx = c;
    }
    qsort(r, (size_t)n, sizeof(ranked), ranked_cmp);
    memset(keep, 0, (size_t)n);
    int kept = k < 0 ? 0 : (k < n ? k : n);
    for (int i = 0; i < kept; ++i)
        keep[r[i].idx] = 1;
    if (diag) {
        diag[0] = kept > 0 ? r[kept - 1].p : -1.0;
        diag[1] = kept < n ? r[kept].p : -1.0;
    }
    free(r);
}

/* The static-ratio mask for the listed rows (all rows when rows is NULL),
 * with the STA union as in oracle_block_mask.  diag: 2 values per row. */
void oracle_block_mask_topk(const double *qp, const double *kp, int64_t BH,
                            int Nb, int d, int Hb, int Wb, int k, int use_sta,
                            int rt, int rh, int rw, const int64_t *rows,
                            int64_t nrows, uint8_t *keep_out, double *diag_out)
{
    if (!rows)
        nrows = BH * Nb;
#pragma omp parallel
    {
        double *a = (double *)malloc(sizeof(double) * (size_t)Nb);
#pragma omp for schedule(dynamic, 16)
        for (int64_t i = 0; i < nrows; ++i) {
            int64_t row = rows ? rows[i] : i;
            int64_t r = row % Nb;
            uint8_t *keep = keep_out + i * Nb;
            reduced_row(qp, kp, row, Nb, d, a);
            oracle_select_topk_row(a, Nb, k, keep, diag_out ? diag_out + i * 2 : NULL);
            if (use_sta)
                for (int c = 0; c < Nb; ++c)
                    if (oracle_sta_keep(r, c, Hb, Wb, rt, rh, rw))
                        keep[c] = 1;
        }
        free(a);
    }
}

/*
 * Semantic-aware permutation (Sparse VideoGen2 summary, section 2A; k-means
 * on Q and on K, independently, tokens of one cluster made contiguous) and
 * centroid top-p (section 2B).  Readings where the page is silent: Lloyd's
 * iterations from the tokens at positions floor(j*N/C) (or from cached
 * centroids, section 2C), squared Euclidean distance, ties to the lower
 * cluster, the assignment decided with the centroids rounded to bf16 (the
 * precision the kernel's tensor-core contraction uses), an empty cluster
 * keeping its centroid; the estimated attention of query cluster i on key
 * cluster j proportional to |K_j| exp(c_qi . c_kj / sqrt(d)).
 */

/* bf16 rounding (round to nearest even) of a float, as the kernel's operand */
static double bf16_round(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7F800000u) != 0x7F800000u)
        u = (u + 0x7FFFu + ((u >> 16) & 1u)) & 0xFFFF0000u;
    float r;
    memcpy(&r, &u, 4);
    return (double)r;
}

/* Assignment step for one (batch, head): x bf16 [N][d], centroids fp32
 * [C][d].  label[t] = argmin_j ||x_t - c~_j||^2 with c~ = bf16(c), computed as
 * ||c~_j||^2 - 2 x_t . c~_j in fp64.  diag[t] = (best, second best). */
void oracle_kmeans_assign(const uint16_t *x, const float *cent, int64_t N, int d, int C,
                          int32_t *label, double *diag)
{
    double *ct = (double *)malloc(sizeof(double) * (size_t)C * d);
    double *cn = (double *)malloc(sizeof(double) * (size_t)C);
    for (int j = 0; j < C; ++j) {
        double s = 0.0;
        for (int i = 0; i < d; ++i) {
            double v = bf16_round(cent[(size_t)j * d + i]);
            ct[(size_t)j * d + i] = v;
            s += v * v;
        }
        cn[j] = s;
    }
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < N; ++t) {
        double best = INFINITY, second = INFINITY;
        int arg = 0;
        for (int j = 0; j < C; ++j) {
            double dot = 0.0;
            for (int i = 0; i < d; ++i)
                dot += bf16_value(x[t * d + i]) * ct[(size_t)j * d + i];
            double dist = cn[j] - 2.0 * dot;
            if (dist < best) {
                second = best;
                best = dist;
                arg = j;
            } else if (dist < second) {
                second = dist;
            }
        }
        label[t] = arg;
        if (diag) {
            diag[2 * t] = best;
            diag[2 * t + 1] = second;
        }
    }
    free(ct);
    free(cn);
}

/* Update step: the centroid of each non-empty cluster becomes the mean of
 * its members (fp64 sum in token order, stored as fp32); an empty cluster
 * keeps its centroid.  count[j] receives the cluster sizes. */
void oracle_kmeans_update(const uint16_t *x, const int32_t *label, int64_t N, int d, int C,
                          float *cent, int32_t *count)
{
    double *sum = (double *)calloc((size_t)C * d, sizeof(double));
    memset(count, 0, sizeof(int32_t) * (size_t)C);
    for (int64_t t = 0; t < N; ++t) {
        int j = label[t];
        ++count[j];
        for (int i = 0; i < d; ++i)
            sum[(size_t)j * d + i] += bf16_value(x[t * d + i]);
    }
    for (int j = 0; j < C; ++j)
        if (count[j] > 0)
            for (int i = 0; i < d; ++i)
                cent[(size_t)j * d + i] = (float)(sum[(size_t)j * d + i] / count[j]);
    free(sum);
}

/* The permutation: tokens in order of cluster, and in token order within a
 * cluster (a stable sort by label).  order[p] = token at position p;
 * start[j] = first position of cluster j (start[C] = N). */
void oracle_cluster_order(const int32_t *label, int64_t N, int C, int64_t *order,
                          int64_t *start)
{
    int64_t *cnt = (int64_t *)calloc((size_t)C + 1, sizeof(int64_t));
    for (int64_t t = 0; t < N; ++t)
        ++cnt[label[t] + 1];
    for (int j = 0; j < C; ++j)
        cnt[j + 1] += cnt[j];
    for (int j = 0; j <= C; ++j)
        start[j] = cnt[j];
    for (int64_t t = 0; t < N; ++t)
        order[cnt[label[t]]++] = t;
    free(cnt);
}

/* Centroid top-p for one (batch, head): for query cluster i the estimated
 * attention over key clusters a_ij = n_j exp(s_ij) / sum, s_ij = c_qi.c_kj /
 * sqrt(d) (fp64, fp32 centroids as stored); the kept key clusters are the
 * smallest prefix of (a desc, index asc) whose mass reaches p (the top-p rule
 * of oracle_select_row with thr = 1 - p).  keep [Cq][Ck]; diag [Cq][5] as in
 * oracle_select_row.  Empty key clusters have a = 0. */
void oracle_centroid_topp(const float *cq, const float *ck, const int32_t *nk, int Cq,
                          int Ck, int d, double p, uint8_t *keep, double *diag)
{
#pragma omp parallel
    {
        double *a = (double *)malloc(sizeof(double) * (size_t)Ck);
#pragma omp for schedule(static)
        for (int i = 0; i < Cq; ++i) {
            double m = -INFINITY;
            for (int j = 0; j < Ck; ++j) {
                double s = 0.0;
                for (int e = 0; e < d; ++e)
                    s += (double)cq[(size_t)i * d + e] * (double)ck[(size_t)j * d + e];
                a[j] = nk[j] > 0 ? s / sqrt((double)d) : -INFINITY;
                if (a[j] > m)
                    m = a[j];
            }
            double z = 0.0;
            for (int j = 0; j < Ck; ++j) {
                a[j] = nk[j] > 0 ? (double)nk[j] * exp(a[j] - m) : 0.0;
                z += a[j];
            }
            for (int j = 0; j < Ck; ++j)
                a[j] /= z;
            oracle_select_row(a, Ck, 1.0 - p, keep + (size_t)i * Ck,
                              diag ? diag + (size_t)i * 5 : NULL);
        }
        free(a);
    }
}

/* Attention of the listed query tokens of one (batch, head) over the key
 * tokens whose key cluster is kept for the query token's cluster, in the
 * original token order (the permutation changes no result, SVG2 section 2A).
 * q, k, v bf16 [N][d]; lq, lk labels; keep [Cq][Ck]; o [nq][d], lse [nq]. */
void oracle_cluster_attention(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                              int64_t N, int d, const int32_t *lq, const int32_t *lk,
                              const uint8_t *keep, int Ck, double scale,
                              const int64_t *qtok, int64_t nq, double *o, double *lse)
{
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)N);
#pragma omp for schedule(dynamic, 4)
        for (int64_t a = 0; a < nq; ++a) {
            int64_t t = qtok[a];
            const uint8_t *kr = keep + (size_t)lq[t] * Ck;
            double m = -INFINITY;
            for (int64_t u = 0; u < N; ++u) {
                if (!kr[lk[u]]) {
                    s[u] = -INFINITY;
                    continue;
                }
                double dot = 0.0;
                for (int e = 0; e < d; ++e)
                    dot += bf16_value(q[t * d + e]) * bf16_value(k[u * d + e]);
                s[u] = dot * scale;
                if (s[u] > m)
                    m = s[u];
            }
            double z = 0.0;
            for (int e = 0; e < d; ++e)
                o[a * d + e] = 0.0;
            if (m == -INFINITY) {
                lse[a] = -INFINITY;
                continue;
            }
            for (int64_t u = 0; u < N; ++u) {
                if (s[u] == -INFINITY)
                    continue;
                double w = exp(s[u] - m);
                z += w;
                for (int e = 0; e < d; ++e)
                    o[a * d + e] += w * bf16_value(v[u * d + e]);
            }
            for (int e = 0; e < d; ++e)
                o[a * d + e] /= z;
            lse[a] = m + log(z);
        }
        free(s);
    }
}

/*
 * The STA window on its own (NABLA summary, "Methodology" item 3, the
 * sliding-tile component M_STA of M = M_nabla OR M_STA, used without the
 * content-adaptive part): keep[r][c] = 1 exactly when key block c lies within
 * the Chebyshev radii of query block r.  One head's Nb x Nb grid; every head
 * has the same mask.
 */
void oracle_sta_mask(int Nb, int Hb, int Wb, int rt, int rh, int rw, uint8_t *keep)
{
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < Nb; ++r)
        for (int64_t c = 0; c < Nb; ++c)
            keep[r * Nb + c] = (uint8_t)oracle_sta_keep(r, c, Hb, Wb, rt, rh, rw);
}

/*
 * O5. Block-sparse attention (NABLA, Methodology item 2, "expansion": the
 * block mask decides which 64 x 64 tiles are computed).  For every query token
 * of query block r, softmax attention over the keys of the kept key blocks
 * col_idx[row_ptr[g] .. row_ptr[g+1]) with g = bh*Nb + r:
 *   s_j = scale * q . k_j,  O = sum_j exp(s_j - m) v_j / l,  l = sum_j exp(s_j - m),
 *   LSE = m + ln l.
 * An empty block list gives O = 0 and LSE = -inf.  qblocks lists global
 * query-block ids (NULL = all); outputs are nq x 64 x d and nq x 64.
 */
void oracle_sparse_attention(const uint16_t *qf, const uint16_t *kf,
                             const uint16_t *vf, int64_t BH, int64_t N, int d,
                             const int64_t *row_ptr, const int32_t *col_idx,
                             double scale, const int64_t *qblocks, int64_t nq,
                             double *o_out, double *lse_out)
{
    const int S = 64;
    int64_t Nb = N / S;
    if (!qblocks)
        nq = BH * Nb;
#pragma omp parallel
    {
        double *q = (double *)malloc(sizeof(double) * d);
        double *acc = (double *)malloc(sizeof(double) * d);
        double *s = (double *)malloc(sizeof(double) * (size_t)Nb * S);
#pragma omp for schedule(dynamic, 1)
        for (int64_t i = 0; i < nq * S; ++i) {
            int64_t g = qblocks ? qblocks[i / S] : i / S;
            int64_t bh = g / Nb, r = g % Nb;
            int64_t tok = r * S + i % S;
            for (int j = 0; j < d; ++j)
                q[j] = bf16_value(qf[(bh * N + tok) * d + j]);
            int64_t nk = 0;
            double m = -INFINITY;
            for (int64_t e = row_ptr[g]; e < row_ptr[g + 1]; ++e)
                for (int kk = 0; kk < S; ++kk) {
                    int64_t key = (int64_t)col_idx[e] * S + kk;
                    const uint16_t *k = kf + (bh * N + key) * d;
                    double dot = 0.0;
                    for (int j = 0; j < d; ++j)
                        dot += q[j] * bf16_value(k[j]);
                    s[nk] = scale * dot;
                    if (s[nk] > m)
                        m = s[nk];
                    ++nk;
                }
            double *o = o_out + i * d;
            if (nk == 0) {
                for (int j = 0; j < d; ++j)
                    o[j] = 0.0;
                lse_out[i] = -INFINITY;
                continue;
            }
            double l = 0.0;
            for (int j = 0; j < d; ++j)
                acc[j] = 0.0;
            nk = 0;
            for (int64_t e = row_ptr[g]; e < row_ptr[g + 1]; ++e)
                for (int kk = 0; kk < S; ++kk) {
                    int64_t key = (int64_t)col_idx[e] * S + kk;
                    const uint16_t *v = vf + (bh * N + key) * d;
                    double p = exp(s[nk++] - m);
                    l += p;
                    for (int j = 0; j < d; ++j)
                        acc[j] += p * bf16_value(v[j]);
                }
            for (int j = 0; j < d; ++j)
                o[j] = acc[j] / l;
            lse_out[i] = m + log(l);
        }
        free(q);
        free(acc);
        free(s);
    }
}

/*
 * vsa_oracle.c -- plain, slow, fp64 CPU oracle for block-sparse video
 * self-attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg use this file.  It shares no code, header,
 * table or helper with the CUDA library; each function restates one step as
 * the source pages define it, with no blocking, fusion or reordering beyond
 * that definition.  Inputs are float arrays that carry the exact bf16 / fp32
 * input values; all arithmetic is in double.
 *
 * Sources (page title, section):
 *  [ADR]  "ADR-0001: Sparse-attention roadmap for video DiTs", Conventions
 *         (T-major token order) and step 1 / step 2 / step 6 (video masks,
 *         head profile, permutation).
 *  [SVG]  "SVG implementation for LTX 2", overview (heads profiled on query
 *         tokens, spatial or temporal pattern per head).
 *  [WIN]  "fastvideo/mlx_runtime/windowed_attention.py", module docstring
 *         ("Window policy"), _default_scale, _key_ranges_for_block,
 *         windowed_attention.
 *  [SPADE] "Adaptive tiling (SPADE)", "The idea" steps 1-4, the function
 *         table (block_self_similarity O(block*D), select_tiling,
 *         minmax_block_scores, top_k_block_mask), the Recipe
 *         (argsort of tile labels, floor budget, inverse permutation) and the
 *         recipe note (OR static sink / diagonal blocks into the mask; drop
 *         skipped blocks).
 *
 * Parity pins live in tests/test_oracle_pins.py.  Every function below is
 * pinned there; none is "parity unpinned".
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ----------------------------------------------------------------------- */
/* Tile labels and the tile-contiguous permutation  [ADR step 6; SPADE Recipe] */
/* ----------------------------------------------------------------------- */

/* label of token (t,h,w) = row-major index of its tile in the tile grid.  */
void orc_tile_labels(int T, int H, int W, int tt, int th, int tw, int64_t *label)
{
    int nth = H / th, ntw = W / tw;
    for (int t = 0; t < T; ++t)
        for (int h = 0; h < H; ++h)
            for (int w = 0; w < W; ++w) {
                int64_t i = ((int64_t)t * H + h) * W + w;
                label[i] = ((int64_t)(t / tt) * nth + h / th) * ntw + w / tw;
            }
}

typedef struct { int64_t label; int64_t index; } orc_pair;

static int orc_cmp_pair(const void *a, const void *b)
{
    const orc_pair *x = (const orc_pair *)a, *y = (const orc_pair *)b;
    if (x->label != y->label) return x->label < y->label ? -1 : 1;
    if (x->index != y->index) return x->index < y->index ? -1 : 1;
    return 0;
}

/* perm = stable argsort of the tile labels: tiles become contiguous, tokens
 * inside a tile keep their T-major order.  perm[p] is the T-major index of
 * the token that lands at permuted position p.                            */
void orc_tile_permutation(int T, int H, int W, int tt, int th, int tw, int64_t *perm)
{
    int64_t S = (int64_t)T * H * W;
    int64_t *label = (int64_t *)malloc(sizeof(int64_t) * S);
    orc_pair *pairs = (orc_pair *)malloc(sizeof(orc_pair) * S);
    orc_tile_labels(T, H, W, tt, th, tw, label);
    for (int64_t i = 0; i < S; ++i) { pairs[i].label = label[i]; pairs[i].index = i; }
    qsort(pairs, (size_t)S, sizeof(orc_pair), orc_cmp_pair);
    for (int64_t p = 0; p < S; ++p) perm[p] = pairs[p].index;
    free(pairs);
    free(label);
}

/* y[p] = x[perm[p]]  (rows of D values)                                    */
void orc_permute_rows(const float *x, int64_t S, int D, const int64_t *perm, float *y)
{
    for (int64_t p = 0; p < S; ++p)
        memcpy(y + p * D, x + perm[p] * D, sizeof(float) * (size_t)D);
}

/* x[perm[p]] = y[p]  -- the inverse permutation                           */
void orc_unpermute_rows(const float *y, int64_t S, int D, const int64_t *perm, float *x)
{
    for (int64_t p = 0; p < S; ++p)
        memcpy(x + perm[p] * D, y + p * D, sizeof(float) * (size_t)D);
}

/* ----------------------------------------------------------------------- */
/* Grids the tiles do not divide  [SPADE "Deviations and notes": pad the     */
/* grid to a multiple of the tiles with zero tokens, excluded from the       */
/* cohesion, and mask the padded keys]                                      */
/* ----------------------------------------------------------------------- */

/* y = x zero-padded from the T-major grid (T, H, W) to (Tp, Hp, Wp): token
 * (t, h, w) keeps its coordinates, every token outside (T, H, W) is zero.  */
void orc_pad_grid(const float *x, int T, int H, int W, int D, int Tp, int Hp, int Wp, float *y)
{
    memset(y, 0, sizeof(float) * (size_t)((int64_t)Tp * Hp * Wp * D));
    for (int t = 0; t < T; ++t)
        for (int h = 0; h < H; ++h)
            for (int w = 0; w < W; ++w)
                memcpy(y + (((int64_t)t * Hp + h) * Wp + w) * D, x + (((int64_t)t * H + h) * W + w) * D,
                       sizeof(float) * (size_t)D);
}

/* ----------------------------------------------------------------------- */
/* Query cohesion (SICS) and the per-head tiling choice  [SPADE step 1;     */
/* function table: block_self_similarity, select_tiling; "Deviations"]      */
/* ----------------------------------------------------------------------- */

/* For every tile of one candidate tiling: the mean cosine similarity over
 * the distinct pairs of its non-zero-norm queries.  With unit vectors n_i and
 * m of them, sum_{i != j} n_i . n_j = |sum_i n_i|^2 - m, so the mean over the
 * m(m-1) ordered pairs is (|sum n_i|^2 - m) / (m(m-1)); this is the O(block*D)
 * form the page gives.  Zero-norm queries are left out; a tile with fewer
 * than two queries scores 0.                                              */
void orc_tile_sics(const float *q, int T, int H, int W, int D,
                   int tt, int th, int tw, double *tile_sics)
{
    int64_t S = (int64_t)T * H * W;
    int64_t n_tiles = S / ((int64_t)tt * th * tw);
    int64_t *label = (int64_t *)malloc(sizeof(int64_t) * S);
    double *sum = (double *)calloc((size_t)(n_tiles * D), sizeof(double));
    int64_t *m = (int64_t *)calloc((size_t)n_tiles, sizeof(int64_t));
    orc_tile_labels(T, H, W, tt, th, tw, label);
    for (int64_t i = 0; i < S; ++i) {
        double ss = 0.0;
        for (int d = 0; d < D; ++d) ss += (double)q[i * D + d] * (double)q[i * D + d];
        if (ss == 0.0) continue;
        double nrm = sqrt(ss);
        double *acc = sum + label[i] * D;
        for (int d = 0; d < D; ++d) acc[d] += (double)q[i * D + d] / nrm;
        m[label[i]] += 1;
    }
    for (int64_t c = 0; c < n_tiles; ++c) {
        double s2 = 0.0;
        for (int d = 0; d < D; ++d) s2 += sum[c * D + d] * sum[c * D + d];
        double mm = (double)m[c];
        tile_sics[c] = m[c] >= 2 ? (s2 - mm) / (mm * (mm - 1.0)) : 0.0;
    }
    free(m);
    free(sum);
    free(label);
}

/* Number of non-zero-norm queries in every tile of one tiling.            */
void orc_tile_counts(const float *q, int T, int H, int W, int D,
                     int tt, int th, int tw, int64_t *m)
{
    int64_t S = (int64_t)T * H * W;
    int64_t n_tiles = S / ((int64_t)tt * th * tw);
    int64_t *label = (int64_t *)malloc(sizeof(int64_t) * S);
    orc_tile_labels(T, H, W, tt, th, tw, label);
    for (int64_t c = 0; c < n_tiles; ++c) m[c] = 0;
    for (int64_t i = 0; i < S; ++i) {
        int nz = 0;
        for (int d = 0; d < D && !nz; ++d) nz = q[i * D + d] != 0.0f;
        if (nz) m[label[i]] += 1;
    }
    free(label);
}

/* Cohesion of a tiling = mean of its tiles' SICS, over the tiles that hold
 * at least one non-zero-norm query (a tile made only of zero padding is not
 * a tile of the video; with no zero tokens every tile counts).  The choice
 * is the candidate with the largest cohesion; equal cohesion goes to the
 * lower candidate index.  scores[c] receives each candidate's cohesion.   */
int orc_select_tiling(const float *q, int T, int H, int W, int D,
                      const int *tiles, int n_tiles, double *scores)
{
    int best = 0;
    for (int c = 0; c < n_tiles; ++c) {
        int tt = tiles[3 * c], th = tiles[3 * c + 1], tw = tiles[3 * c + 2];
        int64_t n = ((int64_t)T * H * W) / ((int64_t)tt * th * tw);
        double *ts = (double *)malloc(sizeof(double) * (size_t)n);
        int64_t *m = (int64_t *)malloc(sizeof(int64_t) * (size_t)n);
        orc_tile_sics(q, T, H, W, D, tt, th, tw, ts);
        orc_tile_counts(q, T, H, W, D, tt, th, tw, m);
        double acc = 0.0;
        int64_t used = 0;
        for (int64_t i = 0; i < n; ++i)
            if (m[i] >= 1) { acc += ts[i]; ++used; }
        scores[c] = used > 0 ? acc / (double)used : 0.0;
        free(m);
        free(ts);
        if (scores[c] > scores[best]) best = c;
    }
    return best;
}

/* ----------------------------------------------------------------------- */
/* Block summaries and block scores  [SPADE step 3; minmax_block_scores]    */
/* ----------------------------------------------------------------------- */

/* Element-wise (per channel) max and min over the tokens of each block of
 * `block` consecutive (permuted) tokens.                                  */
void orc_block_minmax(const float *xp, int64_t S, int D, int block,
                      double *xmax, double *xmin)
{
    int64_t nb = S / block;
    for (int64_t b = 0; b < nb; ++b)
        for (int d = 0; d < D; ++d) {
            double mx = -INFINITY, mn = INFINITY;
            for (int r = 0; r < block; ++r) {
                double x = (double)xp[(b * block + r) * D + d];
                if (x > mx) mx = x;
                if (x < mn) mn = x;
            }
            xmax[b * D + d] = mx;
            xmin[b * D + d] = mn;
        }
}

/* score(i, j) = max((q_max_i + q_min_i) . k_max_j, (q_max_i + q_min_i) . k_min_j),
 * unscaled.                                                                */
void orc_block_scores(const double *qmax, const double *qmin,
                      const double *kmax, const double *kmin,
                      int64_t nb, int D, double *score)
{
    double *a = (double *)malloc(sizeof(double) * (size_t)D);
    for (int64_t i = 0; i < nb; ++i) {
        for (int d = 0; d < D; ++d) a[d] = qmax[i * D + d] + qmin[i * D + d];
        for (int64_t j = 0; j < nb; ++j) {
            double s1 = 0.0, s2 = 0.0;
            for (int d = 0; d < D; ++d) {
                s1 += a[d] * kmax[j * D + d];
                s2 += a[d] * kmin[j * D + d];
            }
            score[i * nb + j] = s1 > s2 ? s1 : s2;
        }
    }
    free(a);
}

/* ----------------------------------------------------------------------- */
/* Top-k key blocks plus static sink and diagonal blocks  [SPADE step 4;    */
/* top_k_block_mask; Recipe (floor budget); recipe note (OR the sink and    */
/* diagonal blocks into the mask)]                                          */
/* ----------------------------------------------------------------------- */

typedef struct { double score; int64_t j; } orc_scored;

static int orc_cmp_scored(const void *a, const void *b)
{
    const orc_scored *x = (const orc_scored *)a, *y = (const orc_scored *)b;
    if (x->score != y->score) return x->score > y->score ? -1 : 1; /* larger first */
    if (x->j != y->j) return x->j < y->j ? -1 : 1;                 /* lower index first */
    return 0;
}

/* Row i keeps the k highest-scoring key blocks (equal scores: lower block
 * index first), then ORs in the sink blocks j < n_sink and the diagonal band
 * |j - i| <= diag_halfwidth.  The kept blocks are written in ascending order
 * to idx[i*cap ...], unused slots get -1, cnt[i] the number kept.
 * Returns 0, or -1 if a row needs more than cap slots.                    */
int orc_topk_block_list(const double *score, int64_t nb, int k, int n_sink,
                        int diag_halfwidth, int cap, int32_t *idx, int32_t *cnt)
{
    orc_scored *row = (orc_scored *)malloc(sizeof(orc_scored) * (size_t)nb);
    unsigned char *keep = (unsigned char *)malloc((size_t)nb);
    int rc = 0;
    for (int64_t i = 0; i < nb; ++i) {
        for (int64_t j = 0; j < nb; ++j) { row[j].score = score[i * nb + j]; row[j].j = j; }
        qsort(row, (size_t)nb, sizeof(orc_scored), orc_cmp_scored);
        memset(keep, 0, (size_t)nb);
        for (int r = 0; r < k && r < nb; ++r) keep[row[r].j] = 1;
        for (int64_t j = 0; j < nb; ++j) {
            if (j < n_sink) keep[j] = 1;
            if (llabs(j - i) <= diag_halfwidth) keep[j] = 1;
        }
        int c = 0;
        for (int64_t j = 0; j < nb; ++j)
            if (keep[j]) {
                if (c < cap) idx[i * cap + c] = (int32_t)j;
                ++c;
            }
        if (c > cap) rc = -1;
        for (int s = c; s < cap; ++s) idx[i * cap + s] = -1;
        cnt[i] = c;
    }
    free(keep);
    free(row);
    return rc;
}

/* Top-p (mass budget) block list  ["Adaptive tiling (SPADE)", function
 * table: top_p_block_mask is named as one of the functions the recipe
 * composes with, with no definition.  Reading: a row's probabilities are
 * softmax(scale * s) over its key blocks; the kept blocks are the shortest
 * prefix of the row in descending score order (equal scores: lower index
 * first) whose probabilities sum to at least p, and the sink and diagonal
 * blocks are ORed in as for top-k.]  Same output layout as
 * orc_topk_block_list.  Returns 0, or -1 if a row needs more than cap slots. */
int orc_topp_block_list(const double *score, int64_t nb, double p, double scale, int n_sink,
                        int diag_halfwidth, int cap, int32_t *idx, int32_t *cnt)
{
    orc_scored *row = (orc_scored *)malloc(sizeof(orc_scored) * (size_t)nb);
    unsigned char *keep = (unsigned char *)malloc((size_t)nb);
    int rc = 0;
    for (int64_t i = 0; i < nb; ++i) {
        double m = -INFINITY;
        for (int64_t j = 0; j < nb; ++j) {
            row[j].score = score[i * nb + j];
            row[j].j = j;
            if (row[j].score > m) m = row[j].score;
        }
        double z = 0.0;
        for (int64_t j = 0; j < nb; ++j) z += exp(scale * (score[i * nb + j] - m));
        qsort(row, (size_t)nb, sizeof(orc_scored), orc_cmp_scored);
        memset(keep, 0, (size_t)nb);
        double acc = 0.0;
        for (int64_t r = 0; r < nb; ++r) {
            keep[row[r].j] = 1;
            acc += exp(scale * (row[r].score - m));
            if (acc >= p * z) break;
        }
        for (int64_t j = 0; j < nb; ++j) {
            if (j < n_sink) keep[j] = 1;
            if (llabs(j - i) <= diag_halfwidth) keep[j] = 1;
        }
        int c = 0;
        for (int64_t j = 0; j < nb; ++j)
            if (keep[j]) {
                if (c < cap) idx[i * cap + c] = (int32_t)j;
                ++c;
            }
        if (c > cap) rc = -1;
        for (int s2 = c; s2 < cap; ++s2) idx[i * cap + s2] = -1;
        cnt[i] = c;
    }
    free(keep);
    free(row);
    return rc;
}

/* ----------------------------------------------------------------------- */
/* Structured masks as block lists  [ADR step 1: spatial_only_mask,         */
/* temporal_only_mask, sliding_tile_block_mask, sliding_tile_centered_mask]  */
/* ----------------------------------------------------------------------- */

/* Tile-neighbourhood mask: query token i sees key token j iff their tiles'
 * coordinates differ by at most (rt, rh, rw) along (t, h, w), with no
 * wrap-around or shift at the grid border.  spatial_only is tile (1,H,W)
 * radius 0 (same frame), temporal_only is tile (T,1,1) radius 0 (same (h,w)),
 * the sliding-tile mask is a tile with radius 1.
 *
 * The centred form (sliding_tile_centered_mask) keeps the window's size
 * fixed instead: along an axis of n tiles a query tile c sees the
 * w = min(2r + 1, n) consecutive tiles starting at c - r, the start moved
 * into [0, n - w] when the window would cross the border.  Away from the
 * border the two forms agree.
 *
 * In the tile-contiguous order, with blocks of `block` tokens:
 *   - if a tile is a whole number of blocks, query block i lists every block
 *     of every neighbouring tile (ascending), group size 0;
 *   - if a block is a whole number of tiles and the radius is 0, query block
 *     i lists only itself and a key is visible iff it shares the query's
 *     group of tile-volume tokens (group size = tile volume).
 * Returns 0, -1 for an unsupported combination, -2 if cap is too small.   */

/* The key tiles [*lo, *hi] a query tile c sees along one axis of n tiles. */
static void orc_axis_window(int c, int r, int n, int centered, int *lo, int *hi)
{
    if (!centered) {
        *lo = c - r;
        *hi = c + r;
        if (*lo < 0) *lo = 0;
        if (*hi > n - 1) *hi = n - 1;
        return;
    }
    int w = 2 * r + 1;
    if (w > n) w = n;
    int start = c - r;
    if (start > n - w) start = n - w;
    if (start < 0) start = 0;
    *lo = start;
    *hi = start + w - 1;
}

static int orc_neighbourhood(int T, int H, int W, int tt, int th, int tw,
                             int rt, int rh, int rw, int centered, int block,
                             int cap, int32_t *idx, int32_t *cnt,
                             int *group_size)
{
    int64_t S = (int64_t)T * H * W;
    int64_t vol = (int64_t)tt * th * tw;
    int64_t nb = S / block;
    int ntt = T / tt, nth = H / th, ntw = W / tw;
    if (vol % block == 0) {
        int64_t bpt = vol / block; /* blocks per tile */
        *group_size = 0;
        for (int64_t i = 0; i < nb; ++i) {
            int64_t tile = i / bpt;
            int ct = (int)(tile / ((int64_t)nth * ntw));
            int ch = (int)((tile / ntw) % nth);
            int cw = (int)(tile % ntw);
            int t0, t1, h0, h1, w0, w1;
            orc_axis_window(ct, rt, ntt, centered, &t0, &t1);
            orc_axis_window(ch, rh, nth, centered, &h0, &h1);
            orc_axis_window(cw, rw, ntw, centered, &w0, &w1);
            int c = 0;
            for (int at = t0; at <= t1; ++at)
                for (int ah = h0; ah <= h1; ++ah)
                    for (int aw = w0; aw <= w1; ++aw) {
                        int64_t nt = ((int64_t)at * nth + ah) * ntw + aw;
                        for (int64_t q = 0; q < bpt; ++q) {
                            if (c >= cap) return -2;
                            idx[i * cap + c++] = (int32_t)(nt * bpt + q);
                        }
                    }
            for (int s = c; s < cap; ++s) idx[i * cap + s] = -1;
            cnt[i] = c;
        }
        return 0;
    }
    if (block % vol == 0 && rt == 0 && rh == 0 && rw == 0) {
        if (cap < 1) return -2;
        *group_size = (int)vol;
        for (int64_t i = 0; i < nb; ++i) {
            idx[i * cap] = (int32_t)i;
            for (int s = 1; s < cap; ++s) idx[i * cap + s] = -1;
            cnt[i] = 1;
        }
        return 0;
    }
    return -1;
}

int orc_tile_neighbourhood_list(int T, int H, int W, int tt, int th, int tw,
                                int rt, int rh, int rw, int block, int cap,
                                int32_t *idx, int32_t *cnt, int *group_size)
{
    return orc_neighbourhood(T, H, W, tt, th, tw, rt, rh, rw, 0, block, cap,
                             idx, cnt, group_size);
}

int orc_centered_tile_neighbourhood_list(int T, int H, int W, int tt, int th,
                                         int tw, int rt, int rh, int rw,
                                         int block, int cap, int32_t *idx,
                                         int32_t *cnt, int *group_size)
{
    return orc_neighbourhood(T, H, W, tt, th, tw, rt, rh, rw, 1, block, cap,
                             idx, cnt, group_size);
}

/* ----------------------------------------------------------------------- */
/* Head profile  [ADR step 2: classify_heads_from_qk, classify_heads_from_  */
/* probs, classify; SVG overview: each head is profiled on sampled query    */
/* tokens and given the spatial or the temporal pattern]                    */
/* ----------------------------------------------------------------------- */

/* Attention probabilities of the sampled query rows over every key of one
 * head: probs[r][j] = softmax_j(scale * q[rows[r]] . k[j]).  T-major q, k
 * of S = T*H*W rows.                                                        */
void orc_sampled_probs(const float *q, const float *k, int64_t S, int D,
                       const int32_t *rows, int R, double scale, double *probs)
{
    #pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < R; ++r) {
        const float *qi = q + (int64_t)rows[r] * D;
        double *p = probs + (int64_t)r * S;
        double mx = -INFINITY;
        for (int64_t j = 0; j < S; ++j) {
            double s = 0.0;
            for (int d = 0; d < D; ++d) s += (double)qi[d] * (double)k[j * D + d];
            p[j] = scale * s;
            if (p[j] > mx) mx = p[j];
        }
        double sum = 0.0;
        for (int64_t j = 0; j < S; ++j) {
            p[j] = exp(p[j] - mx);
            sum += p[j];
        }
        for (int64_t j = 0; j < S; ++j) p[j] /= sum;
    }
}

/* The probability mass each sampled row puts inside the two structured
 * patterns: mass[r][0] on the keys of its own frame (spatial_only_mask),
 * mass[r][1] on the keys at its own (h, w) (temporal_only_mask).           */
void orc_pattern_masses(const double *probs, int T, int H, int W,
                        const int32_t *rows, int R, double *mass)
{
    int64_t S = (int64_t)T * H * W, HW = (int64_t)H * W;
    for (int r = 0; r < R; ++r) {
        int64_t i = rows[r];
        int64_t ti = i / HW, pi = i % HW;
        double sp = 0.0, tp = 0.0;
        for (int64_t j = 0; j < S; ++j) {
            if (j / HW == ti) sp += probs[(int64_t)r * S + j];
            if (j % HW == pi) tp += probs[(int64_t)r * S + j];
        }
        mass[2 * r] = sp;
        mass[2 * r + 1] = tp;
    }
}

/* ----------------------------------------------------------------------- */
/* Attention  [WIN: full_attention, windowed_attention; SPADE recipe note:   */
/* skipped blocks are dropped]                                              */
/* ----------------------------------------------------------------------- */

/* out = sum_j w_j v_j / sum_j w_j over the visible keys j of query row i,
 * w_j = exp(scale * q_i . k_j - max_j'(scale * q_i . k_j')), all in double. */
static void orc_softmax_row(const float *q, const float *k, const float *v,
                            int64_t i, int D, double scale,
                            const unsigned char *visible, int64_t S,
                            double *logit, double *out)
{
    double mx = -INFINITY;
    for (int64_t j = 0; j < S; ++j) {
        if (!visible[j]) continue;
        double s = 0.0;
        for (int d = 0; d < D; ++d) s += (double)q[i * D + d] * (double)k[j * D + d];
        logit[j] = scale * s;
        if (logit[j] > mx) mx = logit[j];
    }
    double den = 0.0;
    for (int d = 0; d < D; ++d) out[d] = 0.0;
    for (int64_t j = 0; j < S; ++j) {
        if (!visible[j]) continue;
        double w = exp(logit[j] - mx);
        den += w;
        for (int d = 0; d < D; ++d) out[d] += w * (double)v[j * D + d];
    }
    for (int d = 0; d < D; ++d) out[d] = den > 0.0 ? out[d] / den : NAN;
}

/* Windowed attention for one head, rows[0..n_rows) of the output.  Key j is
 * visible to query i iff j < sink or |i - j| <= window / 2; a window of at
 * least S makes every key visible (the page returns dense attention then).
 * dense != 0 forces every key visible (full_attention).                   */
void orc_window_attention(const float *q, const float *k, const float *v,
                          int64_t S, int D, int window, int sink, double scale,
                          int dense, const int64_t *rows, int64_t n_rows,
                          double *out)
{
    int64_t half = window / 2;
    int all = dense || (int64_t)window >= S;
    #pragma omp parallel
    {
        unsigned char *vis = (unsigned char *)malloc((size_t)S);
        double *logit = (double *)malloc(sizeof(double) * (size_t)S);
        #pragma omp for schedule(dynamic, 4)
        for (int64_t r = 0; r < n_rows; ++r) {
            int64_t i = rows[r];
            for (int64_t j = 0; j < S; ++j)
                vis[j] = (unsigned char)(all || j < sink || llabs(i - j) <= half);
            orc_softmax_row(q, k, v, i, D, scale, vis, S, logit, out + r * D);
        }
        free(logit);
        free(vis);
    }
}

/* Block-sparse attention for one head in the permuted order: query row p of
 * query block i = p / block sees every key of every block listed for i
 * (idx[i*cap .. i*cap+cnt[i])), restricted to keys of the same group of
 * group_size tokens when group_size > 0, and to keys with key_ok[t] != 0
 * when key_ok is given (padded keys are masked).  rows[] selects output rows. */
void orc_block_sparse_attention(const float *q, const float *k, const float *v,
                                int64_t S, int D, int block,
                                const int32_t *idx, const int32_t *cnt, int cap,
                                int group_size, double scale, const unsigned char *key_ok,
                                const int64_t *rows, int64_t n_rows, double *out)
{
    #pragma omp parallel
    {
        unsigned char *vis = (unsigned char *)malloc((size_t)S);
        double *logit = (double *)malloc(sizeof(double) * (size_t)S);
        #pragma omp for schedule(dynamic, 4)
        for (int64_t r = 0; r < n_rows; ++r) {
            int64_t p = rows[r];
            int64_t i = p / block;
            memset(vis, 0, (size_t)S);
            for (int c = 0; c < cnt[i]; ++c) {
                int64_t j = idx[i * cap + c];
                for (int64_t t = j * block; t < (j + 1) * block; ++t)
                    if ((group_size <= 0 || t / group_size == p / group_size) && (!key_ok || key_ok[t])) vis[t] = 1;
            }
            orc_softmax_row(q, k, v, p, D, scale, vis, S, logit, out + r * D);
        }
        free(logit);
        free(vis);
    }
}

/* centroid_compensated_attention [SPADE Recipe: the attention call with
 * q_labels, k_labels and the block mask; "compensate skipped blocks instead
 * of dropping them"].  The pages give the call and its arguments only.  The
 * reading: query i (block a = q_labels[i]) attends exactly to every key t
 * whose block k_labels[t] is kept (block_mask[a][k_labels[t]] != 0); each
 * skipped key block b with n_b > 0 keys takes part as one centroid key
 * kbar_b (the mean of its keys) with value vbar_b (the mean of its values)
 * and weight n_b:
 *   o_i = (sum_kept e^{s(q_i, k_t)} v_t + sum_skipped n_b e^{s(q_i, kbar_b)} vbar_b)
 *       / (sum_kept e^{s(q_i, k_t)}     + sum_skipped n_b e^{s(q_i, kbar_b)}),
 * s(q, k) = scale q . k.  A skipped block whose keys are all equal then
 * contributes exactly what it would have if kept.  All in double.          */
void orc_centroid_compensated_attention(const float *q, const float *k, const float *v,
                                        int64_t S, int D, const int32_t *q_labels,
                                        const int32_t *k_labels, int n_qb, int n_kb,
                                        const unsigned char *block_mask, double scale,
                                        const int64_t *rows, int64_t n_rows, double *out)
{
    /* the centroids */
    double *kbar = (double *)calloc((size_t)n_kb * D, sizeof(double));
    double *vbar = (double *)calloc((size_t)n_kb * D, sizeof(double));
    int64_t *nb = (int64_t *)calloc((size_t)n_kb, sizeof(int64_t));
    for (int64_t t = 0; t < S; ++t) {
        int b = k_labels[t];
        nb[b] += 1;
        for (int d = 0; d < D; ++d) {
            kbar[(int64_t)b * D + d] += (double)k[t * D + d];
            vbar[(int64_t)b * D + d] += (double)v[t * D + d];
        }
    }
    for (int b = 0; b < n_kb; ++b)
        if (nb[b] > 0)
            for (int d = 0; d < D; ++d) {
                kbar[(int64_t)b * D + d] /= (double)nb[b];
                vbar[(int64_t)b * D + d] /= (double)nb[b];
            }
    #pragma omp parallel
    {
        /* logits of the S keys, then of the n_kb centroids */
        double *logit = (double *)malloc(sizeof(double) * (size_t)(S + n_kb));
        #pragma omp for schedule(dynamic, 4)
        for (int64_t r = 0; r < n_rows; ++r) {
            int64_t i = rows[r];
            const unsigned char *keep = block_mask + (int64_t)q_labels[i] * n_kb;
            double mx = -INFINITY;
            for (int64_t t = 0; t < S; ++t) {
                if (!keep[k_labels[t]]) continue;
                double s = 0.0;
                for (int d = 0; d < D; ++d) s += (double)q[i * D + d] * (double)k[t * D + d];
                logit[t] = scale * s;
                if (logit[t] > mx) mx = logit[t];
            }
            for (int b = 0; b < n_kb; ++b) {
                if (keep[b] || nb[b] == 0) continue;
                double s = 0.0;
                for (int d = 0; d < D; ++d) s += (double)q[i * D + d] * kbar[(int64_t)b * D + d];
                logit[S + b] = scale * s;
                if (logit[S + b] > mx) mx = logit[S + b];
            }
            double den = 0.0;
            double *o = out + r * D;
            for (int d = 0; d < D; ++d) o[d] = 0.0;
            for (int64_t t = 0; t < S; ++t) {
                if (!keep[k_labels[t]]) continue;
                double w = exp(logit[t] - mx);
                den += w;
                for (int d = 0; d < D; ++d) o[d] += w * (double)v[t * D + d];
            }
            for (int b = 0; b < n_kb; ++b) {
                if (keep[b] || nb[b] == 0) continue;
                double w = (double)nb[b] * exp(logit[S + b] - mx);
                den += w;
                for (int d = 0; d < D; ++d) o[d] += w * vbar[(int64_t)b * D + d];
            }
            for (int d = 0; d < D; ++d) o[d] /= den;
        }
        free(logit);
    }
    free(nb);
    free(vbar);
    free(kbar);
}

/* _key_ranges_for_block: ordered, non-overlapping key ranges [start, end)
 * that query rows [qs, qe) need: the local window over every row, plus the
 * sinks [0, sink), merged into one range when they touch.  Writes up to two
 * (start, end) pairs and returns how many.                                 */
int orc_window_key_ranges(int64_t qs, int64_t qe, int64_t S, int64_t half,
                          int64_t sink, int64_t *ranges)
{
    int64_t lo = qs - half > 0 ? qs - half : 0;
    int64_t hi = qe + half < S ? qe + half : S;
    if (lo >= hi) {
        if (sink > 0) { ranges[0] = 0; ranges[1] = sink < S ? sink : S; return 1; }
        return 0;
    }
    if (sink <= 0) { ranges[0] = lo; ranges[1] = hi; return 1; }
    int64_t se = sink < S ? sink : S;
    if (lo <= se) { ranges[0] = 0; ranges[1] = hi > se ? hi : se; return 1; }
    ranges[0] = 0; ranges[1] = se; ranges[2] = lo; ranges[3] = hi;
    return 2;
}

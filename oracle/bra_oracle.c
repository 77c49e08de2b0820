/*
 * bra_oracle.c -- CPU oracle for the forward pass of Bi-Level Routing Attention (BRA).
 *
 * TEST INFRASTRUCTURE. Only the test suite, the package smoke check and the benchmark's
 * CPU-baseline / reference legs load this library; the product path never does, and this
 * file shares no code, header, table or helper with the CUDA library.
 *
 * Everything here is a plain, slow, double-precision restatement of what the pages define,
 * step by step in the pages' order:
 *
 *   1. region partition: the H x W map is cut into n_win x n_win non-overlapping windows
 *      ("从零构建BiFormer", §1 region_partition; "手把手带你读懂BiFormer源码", §1.1
 *      RegionPartition; "医学图像分割模块：BiFormer / 双层路由注意力", §七: H % n_win == 0);
 *   2. region-mean descriptors q_r, k_r = mean of the region's tokens
 *      ("手把手带你读懂BiFormer源码", §1.2 step 1);
 *   3. region affinity A_r = Q_r K_r^T, here with the scale C^-1/2
 *      ("手把手带你读懂BiFormer源码", §1.2 step 2; "从静态到动态", §2.1 TopkRouting);
 *   4. top-k routing index I_r: the k largest affinities of each row
 *      ("手把手带你读懂BiFormer源码", §1.2 step 3);
 *   5. gather of the routed regions' key/value tokens and token-to-token softmax attention
 *      of each region's queries over them, per head, scale head_dim^-1/2
 *      ("从零构建BiFormer", §2.2 TokenAttention; "医学图像分割模块", §五 steps ⑤-⑦).
 *
 * Readings taken where the pages are silent or disagree:
 *   - routing is shared by all heads and uses the full-C region means;
 *   - idx rows are ordered by affinity descending, equal affinities by lower region index
 *     first, and NaN ranks below every number (including -inf);
 *   - regions are numbered row-major over the window grid, tokens row-major inside a region;
 *   - no routing weight, no LePE, no projection: the output is the attention output itself.
 *
 * Layout: q, k, v, out are [B, H, W, C] (channels innermost), head j owns channels
 * [j*hd, (j+1)*hd) ("医学图像分割模块", §五 step ①: reshape(B, N, 3, heads, hd)).
 * Means are [B, R, C], affinities [B, R, R], idx int32 [B, R, topk].
 *
 * Beyond the forward pass the pages describe, and restated the same way:
 *   - per-head routing ("医学图像分割模块", §五 steps ③④): region means and affinities per head
 *     over its head_dim channels, scale head_dim^-1/2, topk clamped to R, idx [B, heads, R, k],
 *     and attention in which head h gathers the regions of its own index rows;
 *   - LePE ("医学图像分割模块", §五 step ⑧): the attention output viewed as a [C, H, W] image
 *     plus its 5 x 5 depthwise convolution (padding 2, zeros outside, one 5 x 5 filter and a
 *     bias per channel), y = x + lepe(x);
 *   - the backward pass of step 5 with the routing index held fixed (the pages train the model,
 *     "从静态到动态", §3.2, "BiFormer用双层路由注意力重塑视觉Transformer效率极限", §3.2, but print
 *     no backward): the gradients of sum(dout * out) with respect to q, k and v;
 *   - auto_pad ("从静态到动态", §4.2; "从零构建BiFormer", §1: a padding layer in front when the
 *     size is not a multiple of the region grid): q, k and v padded with zeros at the bottom
 *     and the right to multiples of n_win, BRA on the padded map, the output cropped back.
 *
 * Every entry point returns 0 on success, 1 on a bad argument and 2 on an index outside
 * [0, R).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_OK 0
#define ORC_BAD_ARG 1
#define ORC_BAD_INDEX 2

int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

static int geometry_ok(int B, int H, int W, int C, int n_win)
{
    if (B < 0 || H <= 0 || W <= 0 || C <= 0 || n_win <= 0) return 0;
    if (H % n_win != 0 || W % n_win != 0) return 0;
    return 1;
}

/* Flat offset of channel 0 of token (y, x) of image b in a [B, H, W, C] array. */
static int64_t token_offset(int b, int y, int x, int H, int W, int C)
{
    return (((int64_t)b * H + y) * W + x) * C;
}

/* Step 2: xm[b, r, c] = (1 / rs) * sum over the rs tokens of region r of x[b, token, c]. */
int oracle_region_means(const double *x, int B, int H, int W, int C, int n_win, double *xm)
{
    if (!geometry_ok(B, H, W, C, n_win)) return ORC_BAD_ARG;
    const int hr = H / n_win, wr = W / n_win, rs = hr * wr, R = n_win * n_win;
    for (int b = 0; b < B; ++b)
        for (int ry = 0; ry < n_win; ++ry)
            for (int rx = 0; rx < n_win; ++rx) {
                const int r = ry * n_win + rx;
                for (int c = 0; c < C; ++c) {
                    double sum = 0.0;
                    for (int yy = 0; yy < hr; ++yy)
                        for (int xx = 0; xx < wr; ++xx)
                            sum += x[token_offset(b, ry * hr + yy, rx * wr + xx, H, W, C) + c];
                    xm[((int64_t)b * R + r) * C + c] = sum / rs;
                }
            }
    return ORC_OK;
}

/* Step 3: A[b, r, s] = (C^-1/2 * qm[b, r, :]) . km[b, s, :]. */
int oracle_affinity(const double *qm, const double *km, int B, int R, int C, double *A)
{
    if (B < 0 || R <= 0 || C <= 0) return ORC_BAD_ARG;
    const double scale = 1.0 / sqrt((double)C);
    for (int b = 0; b < B; ++b)
        for (int r = 0; r < R; ++r)
            for (int s = 0; s < R; ++s) {
                double dot = 0.0;
                for (int c = 0; c < C; ++c)
                    dot += (scale * qm[((int64_t)b * R + r) * C + c]) * km[((int64_t)b * R + s) * C + c];
                A[((int64_t)b * R + r) * R + s] = dot;
            }
    return ORC_OK;
}

/* One candidate region of a routing row. */
typedef struct {
    double value;
    int region;
} candidate;

/* Ranking order of step 4: larger affinity first; equal affinities by lower region index;
   NaN after every number. Region indices in a row are distinct, so the order is total. */
static int candidate_order(const void *pa, const void *pb)
{
    const candidate *a = (const candidate *)pa, *b = (const candidate *)pb;
    const int a_nan = isnan(a->value), b_nan = isnan(b->value);
    if (a_nan != b_nan) return a_nan ? 1 : -1;
    if (!a_nan) {
        if (a->value > b->value) return -1;
        if (a->value < b->value) return 1;
    }
    return (a->region < b->region) ? -1 : (a->region > b->region ? 1 : 0);
}

/* Step 4: idx[b, r, :] = the first topk regions of row A[b, r, :] in the ranking order. */
int oracle_topk(const double *A, int B, int R, int topk, int32_t *idx)
{
    if (B < 0 || R <= 0 || topk <= 0 || topk > R) return ORC_BAD_ARG;
    candidate *row = (candidate *)malloc(sizeof(candidate) * (size_t)R);
    if (!row) return ORC_BAD_ARG;
    for (int b = 0; b < B; ++b)
        for (int r = 0; r < R; ++r) {
            for (int s = 0; s < R; ++s) {
                row[s].value = A[((int64_t)b * R + r) * R + s];
                row[s].region = s;
            }
            qsort(row, (size_t)R, sizeof(candidate), candidate_order);
            for (int j = 0; j < topk; ++j) idx[((int64_t)b * R + r) * topk + j] = row[j].region;
        }
    free(row);
    return ORC_OK;
}

/* Step 5 for one query token (b, y, x): for every head, softmax over the tokens of the
   routed regions idx[b, r, 0..topk-1] (in that order, row-major inside each region) of the
   scaled dot products, then the weighted sum of their values. `logits` has room for
   topk * rs entries. Writes C outputs to out_row. */
static int attend_one_token(const double *q, const double *k, const double *v, const int32_t *idx,
                            int idx_heads, int b, int y, int x, int H, int W, int C, int heads, int n_win,
                            int topk, double *logits, double *out_row)
{
    const int hr = H / n_win, wr = W / n_win, rs = hr * wr, R = n_win * n_win;
    const int hd = C / heads;
    const double scale = 1.0 / sqrt((double)hd);
    const int r = (y / hr) * n_win + (x / wr);
    const double *qt = q + token_offset(b, y, x, H, W, C);

    for (int h = 0; h < heads; ++h) {
        const int c0 = h * hd;
        /* the index row of this query's region: shared by all heads, or this head's own */
        const int32_t *routed = idx + (((int64_t)b * idx_heads + (idx_heads > 1 ? h : 0)) * R + r) * topk;
        for (int j = 0; j < topk; ++j)
            if (routed[j] < 0 || routed[j] >= R) return ORC_BAD_INDEX;
        /* logits over the gathered keys */
        int n = 0;
        double max_logit = -INFINITY;
        for (int j = 0; j < topk; ++j) {
            const int sy = routed[j] / n_win, sx = routed[j] % n_win;
            for (int yy = 0; yy < hr; ++yy)
                for (int xx = 0; xx < wr; ++xx) {
                    const double *kt = k + token_offset(b, sy * hr + yy, sx * wr + xx, H, W, C);
                    double dot = 0.0;
                    for (int c = 0; c < hd; ++c) dot += qt[c0 + c] * kt[c0 + c];
                    logits[n] = scale * dot;
                    if (logits[n] > max_logit) max_logit = logits[n];
                    ++n;
                }
        }
        /* softmax weights (max-subtracted) and their sum */
        double denom = 0.0;
        for (int i = 0; i < n; ++i) {
            logits[i] = exp(logits[i] - max_logit);
            denom += logits[i];
        }
        /* weighted sum of the gathered values, in the same key order */
        for (int c = 0; c < hd; ++c) out_row[c0 + c] = 0.0;
        n = 0;
        for (int j = 0; j < topk; ++j) {
            const int sy = routed[j] / n_win, sx = routed[j] % n_win;
            for (int yy = 0; yy < hr; ++yy)
                for (int xx = 0; xx < wr; ++xx) {
                    const double *vt = v + token_offset(b, sy * hr + yy, sx * wr + xx, H, W, C);
                    const double p = logits[n] / denom;
                    for (int c = 0; c < hd; ++c) out_row[c0 + c] += p * vt[c0 + c];
                    ++n;
                }
        }
    }
    return ORC_OK;
}

static int attend_args_ok(int B, int H, int W, int C, int heads, int n_win, int topk)
{
    if (!geometry_ok(B, H, W, C, n_win)) return 0;
    if (heads <= 0 || C % heads != 0) return 0;
    if (topk <= 0 || topk > n_win * n_win) return 0;
    return 1;
}

/* Step 5 for every token of every image; idx holds idx_heads index rows per region (1: shared
   by all heads, [B, R, topk]; heads: one per head, [B, heads, R, topk]). */
static int attend_all(const double *q, const double *k, const double *v, const int32_t *idx, int idx_heads,
                      int B, int H, int W, int C, int heads, int n_win, int topk, double *out)
{
    if (!attend_args_ok(B, H, W, C, heads, n_win, topk)) return ORC_BAD_ARG;
    const int rs = (H / n_win) * (W / n_win);
    int status = ORC_OK;
#pragma omp parallel
    {
        double *logits = (double *)malloc(sizeof(double) * (size_t)topk * (size_t)rs);
#pragma omp for collapse(2) schedule(dynamic)
        for (int b = 0; b < B; ++b)
            for (int y = 0; y < H; ++y)
                for (int x = 0; x < W; ++x) {
                    int st = attend_one_token(q, k, v, idx, idx_heads, b, y, x, H, W, C, heads, n_win, topk,
                                              logits, out + token_offset(b, y, x, H, W, C));
                    if (st != ORC_OK) {
#pragma omp atomic write
                        status = st;
                    }
                }
        free(logits);
    }
    return status;
}

/* Step 5 for every token of every image, one index row per region shared by all heads. */
int oracle_attend(const double *q, const double *k, const double *v, const int32_t *idx, int B, int H,
                  int W, int C, int heads, int n_win, int topk, double *out)
{
    return attend_all(q, k, v, idx, 1, B, H, W, C, heads, n_win, topk, out);
}

/* Step 5 with per-head routing ("医学图像分割模块", §五 steps ⑤-⑦): head h of a query in region r
   attends over the regions idx[b, h, r, 0..topk-1]. */
int oracle_attend_heads(const double *q, const double *k, const double *v, const int32_t *idx, int B,
                        int H, int W, int C, int heads, int n_win, int topk, double *out)
{
    return attend_all(q, k, v, idx, heads, B, H, W, C, heads, n_win, topk, out);
}

/* Step 5 for a list of tokens only: tokens[i] = b * H * W + y * W + x; out_rows is
   [ntokens, C]. Used to check sampled outputs of full-size workloads. */
int oracle_attend_tokens(const double *q, const double *k, const double *v, const int32_t *idx, int B,
                         int H, int W, int C, int heads, int n_win, int topk, const int64_t *tokens,
                         int64_t ntokens, double *out_rows)
{
    if (!attend_args_ok(B, H, W, C, heads, n_win, topk) || ntokens < 0) return ORC_BAD_ARG;
    const int rs = (H / n_win) * (W / n_win);
    for (int64_t i = 0; i < ntokens; ++i)
        if (tokens[i] < 0 || tokens[i] >= (int64_t)B * H * W) return ORC_BAD_ARG;
    int status = ORC_OK;
#pragma omp parallel
    {
        double *logits = (double *)malloc(sizeof(double) * (size_t)topk * (size_t)rs);
#pragma omp for schedule(dynamic)
        for (int64_t i = 0; i < ntokens; ++i) {
            const int64_t t = tokens[i];
            const int b = (int)(t / ((int64_t)H * W));
            const int y = (int)((t / W) % H), x = (int)(t % W);
            int st = attend_one_token(q, k, v, idx, 1, b, y, x, H, W, C, heads, n_win, topk, logits,
                                      out_rows + i * C);
            if (st != ORC_OK) {
#pragma omp atomic write
                status = st;
            }
        }
        free(logits);
    }
    return status;
}

/* Steps 2-4: routing index of every region. A (optional, may be NULL) receives the
   affinities [B, R, R]. */
int oracle_route(const double *q, const double *k, int B, int H, int W, int C, int n_win, int topk,
                 int32_t *idx, double *A)
{
    if (!geometry_ok(B, H, W, C, n_win)) return ORC_BAD_ARG;
    const int R = n_win * n_win;
    if (topk <= 0 || topk > R) return ORC_BAD_ARG;
    double *qm = (double *)malloc(sizeof(double) * (size_t)B * R * C + 1);
    double *km = (double *)malloc(sizeof(double) * (size_t)B * R * C + 1);
    double *aff = A ? A : (double *)malloc(sizeof(double) * (size_t)B * R * R + 1);
    int st = (qm && km && aff) ? ORC_OK : ORC_BAD_ARG;
    if (st == ORC_OK) st = oracle_region_means(q, B, H, W, C, n_win, qm);
    if (st == ORC_OK) st = oracle_region_means(k, B, H, W, C, n_win, km);
    if (st == ORC_OK) st = oracle_affinity(qm, km, B, R, C, aff);
    if (st == ORC_OK) st = oracle_topk(aff, B, R, topk, idx);
    free(qm);
    free(km);
    if (!A) free(aff);
    return st;
}

/* The whole forward pass: steps 2-5. */
int oracle_forward(const double *q, const double *k, const double *v, int B, int H, int W, int C,
                   int heads, int n_win, int topk, int32_t *idx, double *out)
{
    int st = oracle_route(q, k, B, H, W, C, n_win, topk, idx, NULL);
    if (st == ORC_OK) st = oracle_attend(q, k, v, idx, B, H, W, C, heads, n_win, topk, out);
    return st;
}

/* Per-head routing ("医学图像分割模块", §五 steps ③④): the region means of head h are its
   head_dim channels of the region-mean descriptors, the affinity of head h is
   A[b, h, r, s] = (hd^-1/2 qm[b, r, head h]) . km[b, s, head h], and each row keeps its
   min(topk, R) largest entries (the pages clamp topk to the number of regions) in the ranking
   order of step 4. idx: [B, heads, R, min(topk, R)]; A (optional): [B, heads, R, R]. */
int oracle_route_heads(const double *q, const double *k, int B, int H, int W, int C, int heads, int n_win,
                       int topk, int32_t *idx, double *A)
{
    if (!geometry_ok(B, H, W, C, n_win) || heads <= 0 || C % heads != 0 || topk <= 0) return ORC_BAD_ARG;
    const int R = n_win * n_win, hd = C / heads;
    const int k_eff = topk < R ? topk : R;
    const double head_scale = 1.0 / sqrt((double)hd);
    double *qm = (double *)malloc(sizeof(double) * (size_t)B * R * C + 1);
    double *km = (double *)malloc(sizeof(double) * (size_t)B * R * C + 1);
    double *aff = A ? A : (double *)malloc(sizeof(double) * (size_t)B * heads * R * R + 1);
    int st = (qm && km && aff) ? ORC_OK : ORC_BAD_ARG;
    if (st == ORC_OK) st = oracle_region_means(q, B, H, W, C, n_win, qm);
    if (st == ORC_OK) st = oracle_region_means(k, B, H, W, C, n_win, km);
    if (st == ORC_OK) {
        for (int b = 0; b < B; ++b)
            for (int h = 0; h < heads; ++h)
                for (int r = 0; r < R; ++r)
                    for (int s2 = 0; s2 < R; ++s2) {
                        double dot = 0.0;
                        for (int d = 0; d < hd; ++d)
                            dot += (head_scale * qm[((int64_t)b * R + r) * C + h * hd + d]) *
                                   km[((int64_t)b * R + s2) * C + h * hd + d];
                        aff[(((int64_t)b * heads + h) * R + r) * R + s2] = dot;
                    }
        st = oracle_topk(aff, B * heads, R, k_eff, idx);
    }
    free(qm);
    free(km);
    if (!A) free(aff);
    return st;
}

/* LePE ("医学图像分割模块", §五 step ⑧): the attention output x, viewed as a [C, H, W] image, plus
   its 5 x 5 depthwise convolution with zero padding 2 (nn.Conv2d(C, C, 5, padding=2, groups=C):
   one filter w[c, 0..4, 0..4] and one bias per channel, cross-correlation):
   y[b, i, j, c] = x[b, i, j, c] + bias[c] + sum_{di, dj} w[c, di, dj] x[b, i + di - 2, j + dj - 2, c].
   x, y: [B, H, W, C]; w: [C, 5, 5]; bias: [C]. */
int oracle_lepe(const double *x, const double *w, const double *bias, int B, int H, int W, int C, double *y)
{
    if (B < 0 || H <= 0 || W <= 0 || C <= 0) return ORC_BAD_ARG;
#pragma omp parallel for collapse(2) schedule(static)
    for (int b = 0; b < B; ++b)
        for (int i = 0; i < H; ++i)
            for (int j = 0; j < W; ++j)
                for (int c = 0; c < C; ++c) {
                    double conv = bias[c];
                    for (int di = 0; di < 5; ++di)
                        for (int dj = 0; dj < 5; ++dj) {
                            const int ii = i + di - 2, jj = j + dj - 2;
                            if (ii < 0 || ii >= H || jj < 0 || jj >= W) continue;
                            conv += w[(int64_t)c * 25 + di * 5 + dj] * x[token_offset(b, ii, jj, H, W, C) + c];
                        }
                    y[token_offset(b, i, j, H, W, C) + c] = x[token_offset(b, i, j, H, W, C) + c] + conv;
                }
    return ORC_OK;
}

/* Backward of step 5 with the index fixed: given dout = dL/dout, the gradients of
   L = sum(dout * out) with respect to q, k and v. Per query token and head, with the logits
   l_i = hd^-1/2 q . k_i over the gathered keys i, p = softmax(l) and out = sum_i p_i v_i:
     dv_i += p_i dout,   dp_i = dout . v_i,   ds_i = p_i (dp_i - sum_j p_j dp_j),
     dq = hd^-1/2 sum_i ds_i k_i,   dk_i += hd^-1/2 ds_i q.
   A key gathered twice receives both contributions. dq, dk, dv: [B, H, W, C], overwritten. */
int oracle_attend_backward(const double *q, const double *k, const double *v, const int32_t *idx,
                           const double *dout, int B, int H, int W, int C, int heads, int n_win, int topk,
                           double *dq, double *dk, double *dv)
{
    if (!attend_args_ok(B, H, W, C, heads, n_win, topk)) return ORC_BAD_ARG;
    const int hr = H / n_win, wr = W / n_win, rs = hr * wr, R = n_win * n_win;
    const int hd = C / heads;
    const double inv_sqrt_hd = 1.0 / sqrt((double)hd);
    const int64_t total = (int64_t)B * H * W * C;
    for (int64_t i = 0; i < total; ++i) dq[i] = dk[i] = dv[i] = 0.0;
    for (int64_t i = 0; i < (int64_t)B * R * topk; ++i)
        if (idx[i] < 0 || idx[i] >= R) return ORC_BAD_INDEX;
    int status = ORC_OK;
    /* images are independent: each image's dk and dv only receive its own queries' terms */
#pragma omp parallel
    {
        const int n_keys = topk * rs;
        double *p = (double *)malloc(sizeof(double) * (size_t)n_keys);
        double *dp = (double *)malloc(sizeof(double) * (size_t)n_keys);
        int64_t *key = (int64_t *)malloc(sizeof(int64_t) * (size_t)n_keys);
        if (!p || !dp || !key) {
#pragma omp atomic write
            status = ORC_BAD_ARG;
        }
#pragma omp for schedule(dynamic)
        for (int b = 0; b < B; ++b) {
            if (!p || !dp || !key) continue;
            for (int y = 0; y < H; ++y)
                for (int x = 0; x < W; ++x) {
                    const int qr = (y / hr) * n_win + (x / wr);
                    const int32_t *routed = idx + ((int64_t)b * R + qr) * topk;
                    const int64_t qo = token_offset(b, y, x, H, W, C);
                    /* the gathered keys, in idx order, row-major inside each region */
                    int n = 0;
                    for (int j = 0; j < topk; ++j) {
                        const int ky = routed[j] / n_win, kx = routed[j] % n_win;
                        for (int yy = 0; yy < hr; ++yy)
                            for (int xx = 0; xx < wr; ++xx) key[n++] = token_offset(b, ky * hr + yy, kx * wr + xx, H, W, C);
                    }
                    for (int h = 0; h < heads; ++h) {
                        const int c0 = h * hd;
                        double mx = -INFINITY, denom = 0.0, pdp = 0.0;
                        for (int i = 0; i < n; ++i) {
                            double dot = 0.0;
                            for (int c = 0; c < hd; ++c) dot += q[qo + c0 + c] * k[key[i] + c0 + c];
                            p[i] = inv_sqrt_hd * dot;
                            if (p[i] > mx) mx = p[i];
                        }
                        for (int i = 0; i < n; ++i) {
                            p[i] = exp(p[i] - mx);
                            denom += p[i];
                        }
                        for (int i = 0; i < n; ++i) {
                            p[i] /= denom;
                            double d = 0.0;
                            for (int c = 0; c < hd; ++c) d += dout[qo + c0 + c] * v[key[i] + c0 + c];
                            dp[i] = d;
                            pdp += p[i] * d;
                        }
                        for (int i = 0; i < n; ++i) {
                            const double ds = p[i] * (dp[i] - pdp);
                            for (int c = 0; c < hd; ++c) {
                                dv[key[i] + c0 + c] += p[i] * dout[qo + c0 + c];
                                dq[qo + c0 + c] += inv_sqrt_hd * ds * k[key[i] + c0 + c];
                                dk[key[i] + c0 + c] += inv_sqrt_hd * ds * q[qo + c0 + c];
                            }
                        }
                    }
                }
        }
        free(p);
        free(dp);
        free(key);
    }
    return status;
}

/* The padded size of auto_pad: the next multiple of n_win. */
static int padded(int n, int n_win) { return (n + n_win - 1) / n_win * n_win; }

/* x [B, H, W, C] copied into the top-left of a zeroed [B, Hp, Wp, C] array. */
static double *pad_map(const double *x, int B, int H, int W, int C, int Hp, int Wp)
{
    double *xp = (double *)calloc((size_t)B * Hp * Wp * C + 1, sizeof(double));
    if (!xp) return NULL;
    for (int b = 0; b < B; ++b)
        for (int i = 0; i < H; ++i)
            for (int j = 0; j < W; ++j)
                for (int c = 0; c < C; ++c)
                    xp[token_offset(b, i, j, Hp, Wp, C) + c] = x[token_offset(b, i, j, H, W, C) + c];
    return xp;
}

/* auto_pad ("从静态到动态", §4.2; "从零构建BiFormer", §1): q, k, v padded with zeros at the bottom
   and the right to Hp x Wp, multiples of n_win; steps 2-5 on the padded map (the padded tokens
   are zeros: they count in the region means and take part as keys); out cropped back to
   [B, H, W, C]. idx: [B, R, topk] of the padded map. With given_idx set, idx is read instead of
   routed (step 5 only). */
static int auto_pad_run(const double *q, const double *k, const double *v, int B, int H, int W, int C,
                        int heads, int n_win, int topk, int32_t *idx, int given_idx, double *out)
{
    if (B < 0 || H <= 0 || W <= 0 || C <= 0 || n_win <= 0 || heads <= 0 || C % heads != 0) return ORC_BAD_ARG;
    const int Hp = padded(H, n_win), Wp = padded(W, n_win);
    double *qp = pad_map(q, B, H, W, C, Hp, Wp), *kp = pad_map(k, B, H, W, C, Hp, Wp);
    double *vp = pad_map(v, B, H, W, C, Hp, Wp);
    double *op = (double *)malloc(sizeof(double) * (size_t)B * Hp * Wp * C + 1);
    int st = (qp && kp && vp && op) ? ORC_OK : ORC_BAD_ARG;
    if (st == ORC_OK)
        st = given_idx ? oracle_attend(qp, kp, vp, idx, B, Hp, Wp, C, heads, n_win, topk, op)
                       : oracle_forward(qp, kp, vp, B, Hp, Wp, C, heads, n_win, topk, idx, op);
    if (st == ORC_OK)
        for (int b = 0; b < B; ++b)
            for (int i = 0; i < H; ++i)
                for (int j = 0; j < W; ++j)
                    for (int c = 0; c < C; ++c)
                        out[token_offset(b, i, j, H, W, C) + c] = op[token_offset(b, i, j, Hp, Wp, C) + c];
    free(qp);
    free(kp);
    free(vp);
    free(op);
    return st;
}

int oracle_forward_auto_pad(const double *q, const double *k, const double *v, int B, int H, int W, int C,
                            int heads, int n_win, int topk, int32_t *idx, double *out)
{
    return auto_pad_run(q, k, v, B, H, W, C, heads, n_win, topk, idx, 0, out);
}

int oracle_attend_auto_pad(const double *q, const double *k, const double *v, const int32_t *idx, int B, int H,
                           int W, int C, int heads, int n_win, int topk, double *out)
{
    return auto_pad_run(q, k, v, B, H, W, C, heads, n_win, topk, (int32_t *)idx, 1, out);
}

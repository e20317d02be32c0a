/*
 * FP64 CPU oracle for the fine stage of Video Sparse Attention (VSA).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may load or call
 * this file: it is used by tests/, by the smoke check in __graft_entry__.py
 * and by the CPU-baseline leg of bench.py.  It shares no code, header,
 * table or helper with the CUDA library in video_block_sparse_b200/csrc.
 *
 * It is plain and slow on purpose: every result is the textbook definition
 * written out in double precision, one element at a time, so that a reader
 * can hold it against the pages by eye.
 *
 * Sources (titles of the pages this restates):
 *  - "baseten-admin/wan2.2_production_values" (dataset card), sections
 *    "Shapes" and "Operator contract": cube-major 4x4x4 tiling, 64-token
 *    cubes, S_padded = 64 * Nq, out = softmax(q k_sel^T / sqrt(D)) v_sel,
 *    topk_idx names the selected KV cubes per (batch, head, query cube),
 *    vbs[c] keeps only the first vbs[c] of the 64 tokens of cube c.
 *  - "align VisualGen VSA with block-sparse FMHA" (TensorRT-LLM PR #7),
 *    review excerpts: cube means are sums over the valid tokens divided by
 *    the valid count and cast back to the tiled dtype; untiling is an index
 *    gather.
 *  - "Video Sparse Attention Runner" (TensorRT-Edge-LLM API docs): block
 *    means of K rounded to bf16 before they are used for routing, query
 *    blocks routed by a centroid score.
 *
 * Readings where the pages leave a step open (the design notes list each):
 *  - inside a cube the real tokens come first, in local (t,h,w) row-major
 *    order over the cube's real extent, then zero pads up to 64;
 *  - routing scores are the dot products of bf16 cube means (sequential
 *    FP64 sum, IEEE divide, RNE to bf16), accumulated sequentially in FP64
 *    over d; top-k ordered by score descending, index ascending, NaN as -inf;
 *  - a row whose selected tokens are all masked gives out = 0, lse = -inf;
 *  - lse is the natural-log log-sum-exp of the scaled logits.
 *
 * Parity pins for every function live in tests/test_oracle_pins.py.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <float.h>

#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_ERR_ARG -1
#define ORACLE_ERR_NOMEM -2

/* ---- bf16 <-> double -------------------------------------------------- */

/* A bf16 value is the upper half of an IEEE binary32 word. Widening is exact. */
static double bf16_bits_to_f64(uint16_t h)
{
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Round a double to the nearest bf16 value, ties to even, in one step
 * (no intermediate rounding to binary32).  bf16 keeps 8 significant bits
 * and the binary32 exponent range (normal from 2^-126, subnormal step
 * 2^-133, largest finite (2 - 2^-7) * 2^127). */
static uint16_t f64_to_bf16_bits(double x)
{
    if (isnan(x)) return (uint16_t)0x7FC0;
    if (isinf(x)) return (uint16_t)(x > 0 ? 0x7F80 : 0xFF80);
    if (x == 0.0) return (uint16_t)(signbit(x) ? 0x8000 : 0x0000);
    double ax = fabs(x);
    int e;
    (void)frexp(ax, &e); /* ax = f * 2^e, f in [0.5, 1) -> leading bit weight 2^(e-1) */
    int ulp_exp = (e - 1) - 7; /* 8 significant bits */
    if (ulp_exp < -133) ulp_exp = -133; /* subnormal spacing */
    double scaled = ldexp(ax, -ulp_exp); /* exact: power-of-two scaling */
    double r = nearbyint(scaled); /* current rounding mode: to nearest, ties to even */
    double y = ldexp(r, ulp_exp);
    const double bf16_max = ldexp(255.0, 127 - 7); /* (2 - 2^-7) * 2^127 */
    uint16_t sign = signbit(x) ? 0x8000 : 0x0000;
    if (y > bf16_max) return (uint16_t)(sign | 0x7F80);
    float f = (float)y; /* exact: y has at most 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(sign | ((u >> 16) & 0x7FFF));
}

int oracle_f64_to_bf16(const double *x, uint16_t *y, int64_t n)
{
    if (n < 0 || (n > 0 && (!x || !y))) return ORACLE_ERR_ARG;
    for (int64_t i = 0; i < n; ++i) y[i] = f64_to_bf16_bits(x[i]);
    return ORACLE_OK;
}

int oracle_bf16_to_f64(const uint16_t *x, double *y, int64_t n)
{
    if (n < 0 || (n > 0 && (!x || !y))) return ORACLE_ERR_ARG;
    for (int64_t i = 0; i < n; ++i) y[i] = bf16_bits_to_f64(x[i]);
    return ORACLE_OK;
}

/* ---- cube-major layout -------------------------------------------------
 * Dataset card, "Shapes": Nq = ceil(T/4) * ceil(H/4) * ceil(W/4) cubes of
 * 64 slots; cube c keeps vbs[c] real tokens. */

static int ceil4(int n) { return (n + 3) / 4; }

int oracle_cube_counts(int T, int Hh, int W, int32_t *vbs, int *nq_out)
{
    if (T <= 0 || Hh <= 0 || W <= 0) return ORACLE_ERR_ARG;
    int nct = ceil4(T), nch = ceil4(Hh), ncw = ceil4(W);
    if (nq_out) *nq_out = nct * nch * ncw;
    if (!vbs) return ORACLE_OK;
    for (int ct = 0; ct < nct; ++ct)
        for (int ch = 0; ch < nch; ++ch)
            for (int cw = 0; cw < ncw; ++cw) {
                int et = (T - 4 * ct < 4) ? T - 4 * ct : 4;
                int eh = (Hh - 4 * ch < 4) ? Hh - 4 * ch : 4;
                int ew = (W - 4 * cw < 4) ? W - 4 * cw : 4;
                vbs[(ct * nch + ch) * ncw + cw] = et * eh * ew;
            }
    return ORACLE_OK;
}

/* Slot (0..S-1) in the tiled sequence of raster token (t, h, w). */
static int64_t tiled_slot(int t, int h, int w, int Hh, int W)
{
    int nch = ceil4(Hh), ncw = ceil4(W);
    int ct = t / 4, ch = h / 4, cw = w / 4;
    int eh = (Hh - 4 * ch < 4) ? Hh - 4 * ch : 4;
    int ew = (W - 4 * cw < 4) ? W - 4 * cw : 4;
    int lt = t - 4 * ct, lh = h - 4 * ch, lw = w - 4 * cw;
    int64_t cube = ((int64_t)ct * nch + ch) * ncw + cw;
    return cube * 64 + ((int64_t)lt * eh + lh) * ew + lw;
}

/* x_grid [B, T*Hh*W, H, D] raster order -> x_tiled [B, 64*Nq, H, D]; pads = 0. */
int oracle_tile(const uint16_t *x_grid, uint16_t *x_tiled, int B, int T, int Hh, int W, int H, int D)
{
    int nq;
    if (B <= 0 || H <= 0 || D <= 0 || oracle_cube_counts(T, Hh, W, NULL, &nq)) return ORACLE_ERR_ARG;
    int64_t S = 64LL * nq, L = (int64_t)T * Hh * W, row = (int64_t)H * D;
    memset(x_tiled, 0, (size_t)(B * S * row) * sizeof(uint16_t));
    for (int b = 0; b < B; ++b)
        for (int t = 0; t < T; ++t)
            for (int h = 0; h < Hh; ++h)
                for (int w = 0; w < W; ++w) {
                    int64_t src = ((int64_t)t * Hh + h) * W + w;
                    int64_t dst = tiled_slot(t, h, w, Hh, W);
                    memcpy(x_tiled + ((int64_t)b * S + dst) * row,
                           x_grid + ((int64_t)b * L + src) * row, (size_t)row * sizeof(uint16_t));
                }
    return ORACLE_OK;
}

/* Inverse of oracle_tile: keep the real slots, drop pads. */
int oracle_untile(const uint16_t *x_tiled, uint16_t *x_grid, int B, int T, int Hh, int W, int H, int D)
{
    int nq;
    if (B <= 0 || H <= 0 || D <= 0 || oracle_cube_counts(T, Hh, W, NULL, &nq)) return ORACLE_ERR_ARG;
    int64_t S = 64LL * nq, L = (int64_t)T * Hh * W, row = (int64_t)H * D;
    for (int b = 0; b < B; ++b)
        for (int t = 0; t < T; ++t)
            for (int h = 0; h < Hh; ++h)
                for (int w = 0; w < W; ++w) {
                    int64_t dst = ((int64_t)t * Hh + h) * W + w;
                    int64_t src = tiled_slot(t, h, w, Hh, W);
                    memcpy(x_grid + ((int64_t)b * L + dst) * row,
                           x_tiled + ((int64_t)b * S + src) * row, (size_t)row * sizeof(uint16_t));
                }
    return ORACLE_OK;
}

/* ---- routing ----------------------------------------------------------- */

/* Cube means over valid tokens (TensorRT-LLM PR #7 review excerpt: sum over
 * valid tokens / valid count, cast back to the tiled dtype).
 * x [B, S, H, D] bf16 -> xc [B, H, Nq, D] bf16.  A cube with vbs = 0 has mean 0. */
int oracle_cube_means(const uint16_t *x, const int32_t *vbs, uint16_t *xc,
                      int B, int S, int H, int D, int Nq)
{
    if (B <= 0 || H <= 0 || D <= 0 || Nq <= 0 || S != 64 * Nq) return ORACLE_ERR_ARG;
    for (int c = 0; c < Nq; ++c)
        if (vbs[c] < 0 || vbs[c] > 64) return ORACLE_ERR_ARG;
#pragma omp parallel for collapse(2) schedule(static)
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h)
            for (int c = 0; c < Nq; ++c)
                for (int d = 0; d < D; ++d) {
                    double sum = 0.0;
                    for (int u = 0; u < vbs[c]; ++u)
                        sum += bf16_bits_to_f64(x[(((int64_t)b * S + 64LL * c + u) * H + h) * D + d]);
                    double mean = vbs[c] > 0 ? sum / (double)vbs[c] : 0.0;
                    xc[(((int64_t)b * H + h) * Nq + c) * D + d] = f64_to_bf16_bits(mean);
                }
    return ORACLE_OK;
}

typedef struct {
    double score;
    int32_t idx;
} scored_t;

/* Order: larger score first; NaN counts as -inf; equal scores -> lower index first. */
static int cmp_scored(const void *pa, const void *pb)
{
    const scored_t *a = (const scored_t *)pa, *b = (const scored_t *)pb;
    double sa = isnan(a->score) ? -INFINITY : a->score;
    double sb = isnan(b->score) ? -INFINITY : b->score;
    if (sa > sb) return -1;
    if (sa < sb) return 1;
    return (a->idx > b->idx) - (a->idx < b->idx);
}

/* Cube-mean q.k routing: for every (b, h, query cube i) pick the topk KV cubes
 * with the largest score sc[i][j] = sum_d qc[i][d] * kc[j][d] (sequential FP64).
 * scores (optional) receives sc as [B, H, Nq, Nq]. */
int oracle_route(const uint16_t *q, const uint16_t *k, const int32_t *vbs, int32_t *topk_idx,
                 int B, int S, int H, int D, int Nq, int topk, double *scores)
{
    if (topk < 1 || topk > Nq) return ORACLE_ERR_ARG;
    int64_t nmean = (int64_t)B * H * Nq * D;
    uint16_t *qc = (uint16_t *)malloc((size_t)nmean * sizeof(uint16_t));
    uint16_t *kc = (uint16_t *)malloc((size_t)nmean * sizeof(uint16_t));
    if (!qc || !kc) { free(qc); free(kc); return ORACLE_ERR_NOMEM; }
    int rc = oracle_cube_means(q, vbs, qc, B, S, H, D, Nq);
    if (!rc) rc = oracle_cube_means(k, vbs, kc, B, S, H, D, Nq);
    if (rc) { free(qc); free(kc); return rc; }
    int failed = 0;
#pragma omp parallel
    {
        scored_t *row = (scored_t *)malloc((size_t)Nq * sizeof(scored_t));
        if (!row) {
#pragma omp atomic write
            failed = 1;
        }
#pragma omp for collapse(3) schedule(static)
        for (int b = 0; b < B; ++b)
            for (int h = 0; h < H; ++h)
                for (int i = 0; i < Nq; ++i) {
                    if (!row) continue;
                    const uint16_t *qi = qc + (((int64_t)b * H + h) * Nq + i) * D;
                    for (int j = 0; j < Nq; ++j) {
                        const uint16_t *kj = kc + (((int64_t)b * H + h) * Nq + j) * D;
                        double acc = 0.0;
                        for (int d = 0; d < D; ++d)
                            acc += bf16_bits_to_f64(qi[d]) * bf16_bits_to_f64(kj[d]);
                        row[j].score = acc;
                        row[j].idx = j;
                        if (scores) scores[(((int64_t)b * H + h) * Nq + i) * Nq + j] = acc;
                    }
                    qsort(row, (size_t)Nq, sizeof(scored_t), cmp_scored);
                    int32_t *dst = topk_idx + (((int64_t)b * H + h) * Nq + i) * topk;
                    for (int t = 0; t < topk; ++t) dst[t] = row[t].idx;
                }
        free(row);
    }
    free(qc);
    free(kc);
    return failed ? ORACLE_ERR_NOMEM : ORACLE_OK;
}

/* ---- fine forward --------------------------------------------------------
 * Dataset card, "Operator contract": for query row s of cube i, head h,
 * batch b, the keys are the first vbs[j] tokens of every selected cube j
 * (a cube listed twice counts twice); x_u = sigma * q_s . k_u;
 * out_s = sum_u softmax(x)_u v_u; lse_s = log sum_u exp(x_u).
 * Work is given as a list of (b, h, i) items; results are item-major:
 * out [n_items, 64, D], lse [n_items, 64].  If wabs is not NULL it receives,
 * per output element, sum_u softmax(x)_u |v_u[d]| (same layout as out): the
 * scale of the error that rounding each weight to a short format can cause. */
int oracle_fwd_items_ex(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                        const int32_t *topk_idx, const int32_t *vbs,
                        int B, int S, int H, int D, int Nq, int topk, double sigma,
                        const int32_t *items, int64_t n_items, double *out, double *lse, double *wabs)
{
    if (B <= 0 || H <= 0 || D <= 0 || Nq <= 0 || S != 64 * Nq || topk < 1) return ORACLE_ERR_ARG;
    for (int c = 0; c < Nq; ++c)
        if (vbs[c] < 0 || vbs[c] > 64) return ORACLE_ERR_ARG;
    for (int64_t it = 0; it < n_items; ++it) {
        int b = items[3 * it], h = items[3 * it + 1], i = items[3 * it + 2];
        if (b < 0 || b >= B || h < 0 || h >= H || i < 0 || i >= Nq) return ORACLE_ERR_ARG;
        const int32_t *sel = topk_idx + (((int64_t)b * H + h) * Nq + i) * topk;
        for (int t = 0; t < topk; ++t)
            if (sel[t] < 0 || sel[t] >= Nq) return ORACLE_ERR_ARG;
    }
    int failed = 0;
#pragma omp parallel
    {
        int64_t *keys = (int64_t *)malloc((size_t)topk * 64 * sizeof(int64_t));
        double *x = (double *)malloc((size_t)topk * 64 * sizeof(double));
        if (!keys || !x) {
#pragma omp atomic write
            failed = 1;
        }
#pragma omp for schedule(dynamic, 1)
        for (int64_t it = 0; it < n_items; ++it) {
            if (!keys || !x) continue;
            int b = items[3 * it], h = items[3 * it + 1], i = items[3 * it + 2];
            const int32_t *sel = topk_idx + (((int64_t)b * H + h) * Nq + i) * topk;
            /* the selected token set, multiplicity kept */
            int64_t nkeys = 0;
            for (int t = 0; t < topk; ++t)
                for (int u = 0; u < vbs[sel[t]]; ++u) keys[nkeys++] = 64LL * sel[t] + u;
            for (int r = 0; r < 64; ++r) {
                int64_t s = 64LL * i + r;
                const uint16_t *qs = q + (((int64_t)b * S + s) * H + h) * D;
                double *o = out + (it * 64 + r) * D;
                if (nkeys == 0) {
                    for (int d = 0; d < D; ++d) o[d] = 0.0;
                    if (wabs != NULL)
                        for (int d = 0; d < D; ++d) wabs[(it * 64 + r) * D + d] = 0.0;
                    lse[it * 64 + r] = -INFINITY;
                    continue;
                }
                double m = -INFINITY;
                for (int64_t n = 0; n < nkeys; ++n) {
                    const uint16_t *ku = k + (((int64_t)b * S + keys[n]) * H + h) * D;
                    double dot = 0.0;
                    for (int d = 0; d < D; ++d) dot += bf16_bits_to_f64(qs[d]) * bf16_bits_to_f64(ku[d]);
                    x[n] = sigma * dot;
                    if (x[n] > m) m = x[n];
                }
                double l = 0.0;
                for (int d = 0; d < D; ++d) o[d] = 0.0;
                for (int64_t n = 0; n < nkeys; ++n) {
                    double p = exp(x[n] - m);
                    const uint16_t *vu = v + (((int64_t)b * S + keys[n]) * H + h) * D;
                    l += p;
                    for (int d = 0; d < D; ++d) o[d] += p * bf16_bits_to_f64(vu[d]);
                }
                for (int d = 0; d < D; ++d) o[d] /= l;
                lse[it * 64 + r] = m + log(l);
                if (wabs != NULL) {
                    /* the softmax-weighted mean of |v|: sum_u (p_u / l) |v_u[d]| */
                    double *a = wabs + (it * 64 + r) * D;
                    for (int d = 0; d < D; ++d) a[d] = 0.0;
                    for (int64_t n = 0; n < nkeys; ++n) {
                        double w = exp(x[n] - m) / l;
                        const uint16_t *vu = v + (((int64_t)b * S + keys[n]) * H + h) * D;
                        for (int d = 0; d < D; ++d) a[d] += w * fabs(bf16_bits_to_f64(vu[d]));
                    }
                }
            }
        }
        free(keys);
        free(x);
    }
    return failed ? ORACLE_ERR_NOMEM : ORACLE_OK;
}

/* ------------------------------------------------------------------ proxy compensation
 *
 * TensorRT-LLM PR #7 (the embedded FlashInfer PR "support proxy-compensated
 * block-sparse attention"): selected blocks stay exact; every omitted KV block
 * contributes through one arithmetic-mean K summary and one summed-V summary;
 * a block already covered by an exact route is not counted again by its proxy
 * (score-keep); the softmax denominator is corrected by the token mass the
 * proxy represents, the true length of a partial block included.
 * TensorRT-Edge-LLM "Video Sparse Attention Runner": KC and VC are BF16 block
 * means of K and block sums of V; every block not attended exactly contributes
 * through its mean key and summed value.
 *
 * For query row s of cube i, with E the selected tokens (multiplicity kept)
 * and O the cubes j with vbs[j] > 0 that i does not select:
 *   x_u  = sigma * q_s . k_u                 (u in E)
 *   y_j  = sigma * q_s . kc_j                (j in O)
 *   out  = (sum_u e^{x_u} v_u + sum_j e^{y_j} vc_j) / (sum_u e^{x_u} + sum_j vbs[j] e^{y_j})
 *   lse  = log of that denominator
 * Rows with E and O both empty: out = 0, lse = -inf. */

/* vc[b, h, c, :] = bf16_rne(sequential FP64 sum of x over the first vbs[c] tokens of cube c) */
int oracle_cube_sums(const uint16_t *x, const int32_t *vbs, uint16_t *xs, int B, int S, int H, int D, int Nq)
{
    if (B <= 0 || H <= 0 || D <= 0 || Nq <= 0 || S != 64 * Nq) return ORACLE_ERR_ARG;
    for (int c = 0; c < Nq; ++c)
        if (vbs[c] < 0 || vbs[c] > 64) return ORACLE_ERR_ARG;
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h)
            for (int c = 0; c < Nq; ++c)
                for (int d = 0; d < D; ++d) {
                    double acc = 0.0;
                    for (int u = 0; u < vbs[c]; ++u)
                        acc += bf16_bits_to_f64(x[(((int64_t)b * S + 64LL * c + u) * H + h) * D + d]);
                    xs[(((int64_t)b * H + h) * Nq + c) * D + d] = f64_to_bf16_bits(acc);
                }
    return ORACLE_OK;
}

int oracle_fwd_proxy_items(const uint16_t *q, const uint16_t *k, const uint16_t *v, const uint16_t *kc,
                           const uint16_t *vc, const int32_t *topk_idx, const int32_t *vbs, int B, int S, int H,
                           int D, int Nq, int topk, double sigma, const int32_t *items, int64_t n_items,
                           double *out, double *lse)
{
    if (B <= 0 || H <= 0 || D <= 0 || Nq <= 0 || S != 64 * Nq || topk < 1) return ORACLE_ERR_ARG;
    for (int c = 0; c < Nq; ++c)
        if (vbs[c] < 0 || vbs[c] > 64) return ORACLE_ERR_ARG;
    for (int64_t it = 0; it < n_items; ++it) {
        int b = items[3 * it], h = items[3 * it + 1], i = items[3 * it + 2];
        if (b < 0 || b >= B || h < 0 || h >= H || i < 0 || i >= Nq) return ORACLE_ERR_ARG;
        const int32_t *sel = topk_idx + (((int64_t)b * H + h) * Nq + i) * topk;
        for (int t = 0; t < topk; ++t)
            if (sel[t] < 0 || sel[t] >= Nq) return ORACLE_ERR_ARG;
    }
    int failed = 0;
#pragma omp parallel
    {
        int64_t *keys = (int64_t *)malloc((size_t)topk * 64 * sizeof(int64_t));
        int32_t *omitted = (int32_t *)malloc((size_t)Nq * sizeof(int32_t));
        char *chosen = (char *)malloc((size_t)Nq);
        double *x = (double *)malloc((size_t)(topk * 64 + Nq) * sizeof(double));
        if (!keys || !omitted || !chosen || !x) {
#pragma omp atomic write
            failed = 1;
        }
#pragma omp for schedule(dynamic, 1)
        for (int64_t it = 0; it < n_items; ++it) {
            if (!keys || !omitted || !chosen || !x) continue;
            int b = items[3 * it], h = items[3 * it + 1], i = items[3 * it + 2];
            const int32_t *sel = topk_idx + (((int64_t)b * H + h) * Nq + i) * topk;
            /* exact tokens (multiplicity kept) and the omitted cubes (score-keep: a selected cube has no proxy) */
            int64_t nkeys = 0;
            for (int c = 0; c < Nq; ++c) chosen[c] = 0;
            for (int t = 0; t < topk; ++t) {
                chosen[sel[t]] = 1;
                for (int u = 0; u < vbs[sel[t]]; ++u) keys[nkeys++] = 64LL * sel[t] + u;
            }
            int nom = 0;
            for (int c = 0; c < Nq; ++c)
                if (!chosen[c] && vbs[c] > 0) omitted[nom++] = c;
            for (int r = 0; r < 64; ++r) {
                int64_t s = 64LL * i + r;
                const uint16_t *qs = q + (((int64_t)b * S + s) * H + h) * D;
                double *o = out + (it * 64 + r) * D;
                if (nkeys == 0 && nom == 0) {
                    for (int d = 0; d < D; ++d) o[d] = 0.0;
                    lse[it * 64 + r] = -INFINITY;
                    continue;
                }
                double m = -INFINITY;
                for (int64_t n = 0; n < nkeys; ++n) {
                    const uint16_t *ku = k + (((int64_t)b * S + keys[n]) * H + h) * D;
                    double dot = 0.0;
                    for (int d = 0; d < D; ++d) dot += bf16_bits_to_f64(qs[d]) * bf16_bits_to_f64(ku[d]);
                    x[n] = sigma * dot;
                    if (x[n] > m) m = x[n];
                }
                for (int n = 0; n < nom; ++n) {
                    const uint16_t *kj = kc + (((int64_t)b * H + h) * Nq + omitted[n]) * D;
                    double dot = 0.0;
                    for (int d = 0; d < D; ++d) dot += bf16_bits_to_f64(qs[d]) * bf16_bits_to_f64(kj[d]);
                    x[nkeys + n] = sigma * dot;
                    if (x[nkeys + n] > m) m = x[nkeys + n];
                }
                double l = 0.0;
                for (int d = 0; d < D; ++d) o[d] = 0.0;
                for (int64_t n = 0; n < nkeys; ++n) {
                    double p = exp(x[n] - m);
                    const uint16_t *vu = v + (((int64_t)b * S + keys[n]) * H + h) * D;
                    l += p;
                    for (int d = 0; d < D; ++d) o[d] += p * bf16_bits_to_f64(vu[d]);
                }
                for (int n = 0; n < nom; ++n) {
                    double p = exp(x[nkeys + n] - m);
                    const uint16_t *vj = vc + (((int64_t)b * H + h) * Nq + omitted[n]) * D;
                    l += (double)vbs[omitted[n]] * p; /* the token mass the proxy stands for */
                    for (int d = 0; d < D; ++d) o[d] += p * bf16_bits_to_f64(vj[d]);
                }
                for (int d = 0; d < D; ++d) o[d] /= l;
                lse[it * 64 + r] = m + log(l);
            }
        }
        free(keys);
        free(omitted);
        free(chosen);
        free(x);
    }
    return failed ? ORACLE_ERR_NOMEM : ORACLE_OK;
}

/* ------------------------------------------------------------------ BSR rows
 *
 * TensorRT-LLM PR #7 (the embedded FlashInfer PR "support proxy-compensated
 * block-sparse attention", "Bitmask format"): exact-block selections as
 * canonical BSR rows (block_indptr / block_indices) or packed UInt32 bitmaps
 * per (batch, KV head, Q block); both describe the same selection, and a
 * bitmap is first written out as BSR rows (oracle/__init__.py).  Here a row is
 * r = (b*H + h)*Nq + i and lists the cubes indices[indptr[r] .. indptr[r+1])
 * of query cube i, any number of them, multiplicity kept.  Without kc and vc
 * (both NULL) the result is the fine forward over the listed cubes' valid
 * tokens; with them, every cube with vbs > 0 that the row does not list adds
 * its proxy as in oracle_fwd_proxy_items.  wabs (plain mode, may be NULL): the
 * softmax-weighted mean of |v|. */
int oracle_fwd_bsr_items(const uint16_t *q, const uint16_t *k, const uint16_t *v, const uint16_t *kc,
                         const uint16_t *vc, const int32_t *indptr, const int32_t *indices, int64_t nnz,
                         const int32_t *vbs, int B, int S, int H, int D, int Nq, double sigma,
                         const int32_t *items, int64_t n_items, double *out, double *lse, double *wabs)
{
    if (B <= 0 || H <= 0 || D <= 0 || Nq <= 0 || S != 64 * Nq || nnz < 0) return ORACLE_ERR_ARG;
    if ((kc == NULL) != (vc == NULL) || (kc != NULL && wabs != NULL)) return ORACLE_ERR_ARG;
    for (int c = 0; c < Nq; ++c)
        if (vbs[c] < 0 || vbs[c] > 64) return ORACLE_ERR_ARG;
    int64_t maxlen = 0;
    for (int64_t it = 0; it < n_items; ++it) {
        int b = items[3 * it], h = items[3 * it + 1], i = items[3 * it + 2];
        if (b < 0 || b >= B || h < 0 || h >= H || i < 0 || i >= Nq) return ORACLE_ERR_ARG;
        int64_t r = ((int64_t)b * H + h) * Nq + i;
        if (indptr[r] < 0 || indptr[r + 1] < indptr[r] || indptr[r + 1] > nnz) return ORACLE_ERR_ARG;
        for (int64_t t = indptr[r]; t < indptr[r + 1]; ++t)
            if (indices[t] < 0 || indices[t] >= Nq) return ORACLE_ERR_ARG;
        if (indptr[r + 1] - indptr[r] > maxlen) maxlen = indptr[r + 1] - indptr[r];
    }
    int failed = 0;
#pragma omp parallel
    {
        int64_t *keys = (int64_t *)malloc((size_t)(maxlen * 64 + 1) * sizeof(int64_t));
        int32_t *omitted = (int32_t *)malloc((size_t)Nq * sizeof(int32_t));
        char *chosen = (char *)malloc((size_t)Nq);
        double *x = (double *)malloc((size_t)(maxlen * 64 + Nq + 1) * sizeof(double));
        if (!keys || !omitted || !chosen || !x) {
#pragma omp atomic write
            failed = 1;
        }
#pragma omp for schedule(dynamic, 1)
        for (int64_t it = 0; it < n_items; ++it) {
            if (!keys || !omitted || !chosen || !x) continue;
            int b = items[3 * it], h = items[3 * it + 1], i = items[3 * it + 2];
            int64_t r = ((int64_t)b * H + h) * Nq + i;
            /* the listed cubes' tokens (multiplicity kept) and, with proxies, the cubes not listed */
            int64_t nkeys = 0;
            for (int c = 0; c < Nq; ++c) chosen[c] = 0;
            for (int64_t t = indptr[r]; t < indptr[r + 1]; ++t) {
                int j = indices[t];
                chosen[j] = 1;
                for (int u = 0; u < vbs[j]; ++u) keys[nkeys++] = 64LL * j + u;
            }
            int nom = 0;
            if (kc != NULL)
                for (int c = 0; c < Nq; ++c)
                    if (!chosen[c] && vbs[c] > 0) omitted[nom++] = c;
            for (int rr = 0; rr < 64; ++rr) {
                int64_t s = 64LL * i + rr;
                const uint16_t *qs = q + (((int64_t)b * S + s) * H + h) * D;
                double *o = out + (it * 64 + rr) * D;
                if (nkeys == 0 && nom == 0) {
                    for (int d = 0; d < D; ++d) o[d] = 0.0;
                    if (wabs != NULL)
                        for (int d = 0; d < D; ++d) wabs[(it * 64 + rr) * D + d] = 0.0;
                    lse[it * 64 + rr] = -INFINITY;
                    continue;
                }
                double m = -INFINITY;
                for (int64_t n = 0; n < nkeys; ++n) {
                    const uint16_t *ku = k + (((int64_t)b * S + keys[n]) * H + h) * D;
                    double dot = 0.0;
                    for (int d = 0; d < D; ++d) dot += bf16_bits_to_f64(qs[d]) * bf16_bits_to_f64(ku[d]);
                    x[n] = sigma * dot;
                    if (x[n] > m) m = x[n];
                }
                for (int n = 0; n < nom; ++n) {
                    const uint16_t *kj = kc + (((int64_t)b * H + h) * Nq + omitted[n]) * D;
                    double dot = 0.0;
                    for (int d = 0; d < D; ++d) dot += bf16_bits_to_f64(qs[d]) * bf16_bits_to_f64(kj[d]);
                    x[nkeys + n] = sigma * dot;
                    if (x[nkeys + n] > m) m = x[nkeys + n];
                }
                double l = 0.0;
                for (int d = 0; d < D; ++d) o[d] = 0.0;
                for (int64_t n = 0; n < nkeys; ++n) {
                    double p = exp(x[n] - m);
                    const uint16_t *vu = v + (((int64_t)b * S + keys[n]) * H + h) * D;
                    l += p;
                    for (int d = 0; d < D; ++d) o[d] += p * bf16_bits_to_f64(vu[d]);
                }
                for (int n = 0; n < nom; ++n) {
                    double p = exp(x[nkeys + n] - m);
                    const uint16_t *vj = vc + (((int64_t)b * H + h) * Nq + omitted[n]) * D;
                    l += (double)vbs[omitted[n]] * p; /* the token mass the proxy stands for */
                    for (int d = 0; d < D; ++d) o[d] += p * bf16_bits_to_f64(vj[d]);
                }
                for (int d = 0; d < D; ++d) o[d] /= l;
                lse[it * 64 + rr] = m + log(l);
                if (wabs != NULL) {
                    double *a = wabs + (it * 64 + rr) * D;
                    for (int d = 0; d < D; ++d) a[d] = 0.0;
                    for (int64_t n = 0; n < nkeys; ++n) {
                        double w = exp(x[n] - m) / l;
                        const uint16_t *vu = v + (((int64_t)b * S + keys[n]) * H + h) * D;
                        for (int d = 0; d < D; ++d) a[d] += w * fabs(bf16_bits_to_f64(vu[d]));
                    }
                }
            }
        }
        free(keys);
        free(omitted);
        free(chosen);
        free(x);
    }
    return failed ? ORACLE_ERR_NOMEM : ORACLE_OK;
}

/* ------------------------------------------------------------------ short-KV cross-attention
 *
 * maxdiffusion PR #509 (a fused short-KV cross-attention kernel for Wan's 512-token
 * text KV): every query row attends to every key of a separate, short key/value
 * sequence with one exact softmax (no mask).  q: [B, S, H, D], k and v: [B, S_kv,
 * H, D]; items (b, h, i) are query blocks of 64 rows (S = 64 * number of blocks):
 *   out[b, s, h] = sum_u e^{x_u} v_u / sum_u e^{x_u},  x_u = sigma q_s . k_u
 *   lse          = log sum_u e^{x_u}  (u over all S_kv keys).
 * wabs (may be NULL): the softmax-weighted mean of |v|. */
int oracle_cross_items(const uint16_t *q, const uint16_t *k, const uint16_t *v, int B, int S, int S_kv, int H,
                       int D, double sigma, const int32_t *items, int64_t n_items, double *out, double *lse,
                       double *wabs)
{
    if (B <= 0 || H <= 0 || D <= 0 || S <= 0 || S % 64 != 0 || S_kv <= 0) return ORACLE_ERR_ARG;
    for (int64_t it = 0; it < n_items; ++it) {
        int b = items[3 * it], h = items[3 * it + 1], i = items[3 * it + 2];
        if (b < 0 || b >= B || h < 0 || h >= H || i < 0 || i >= S / 64) return ORACLE_ERR_ARG;
    }
    int failed = 0;
#pragma omp parallel
    {
        double *x = (double *)malloc((size_t)S_kv * sizeof(double));
        if (!x) {
#pragma omp atomic write
            failed = 1;
        }
#pragma omp for schedule(dynamic, 1)
        for (int64_t it = 0; it < n_items; ++it) {
            if (!x) continue;
            int b = items[3 * it], h = items[3 * it + 1], i = items[3 * it + 2];
            for (int r = 0; r < 64; ++r) {
                int64_t s = 64LL * i + r;
                const uint16_t *qs = q + (((int64_t)b * S + s) * H + h) * D;
                double *o = out + (it * 64 + r) * D;
                double m = -INFINITY;
                for (int u = 0; u < S_kv; ++u) {
                    const uint16_t *ku = k + (((int64_t)b * S_kv + u) * H + h) * D;
                    double dot = 0.0;
                    for (int d = 0; d < D; ++d) dot += bf16_bits_to_f64(qs[d]) * bf16_bits_to_f64(ku[d]);
                    x[u] = sigma * dot;
                    if (x[u] > m) m = x[u];
                }
                double l = 0.0;
                for (int d = 0; d < D; ++d) o[d] = 0.0;
                for (int u = 0; u < S_kv; ++u) {
                    double p = exp(x[u] - m);
                    const uint16_t *vu = v + (((int64_t)b * S_kv + u) * H + h) * D;
                    l += p;
                    for (int d = 0; d < D; ++d) o[d] += p * bf16_bits_to_f64(vu[d]);
                }
                for (int d = 0; d < D; ++d) o[d] /= l;
                lse[it * 64 + r] = m + log(l);
                if (wabs != NULL) {
                    double *a = wabs + (it * 64 + r) * D;
                    for (int d = 0; d < D; ++d) a[d] = 0.0;
                    for (int u = 0; u < S_kv; ++u) {
                        double w = exp(x[u] - m) / l;
                        const uint16_t *vu = v + (((int64_t)b * S_kv + u) * H + h) * D;
                        for (int d = 0; d < D; ++d) a[d] += w * fabs(bf16_bits_to_f64(vu[d]));
                    }
                }
            }
        }
        free(x);
    }
    return failed ? ORACLE_ERR_NOMEM : ORACLE_OK;
}

int oracle_fwd_items(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                     const int32_t *topk_idx, const int32_t *vbs,
                     int B, int S, int H, int D, int Nq, int topk, double sigma,
                     const int32_t *items, int64_t n_items, double *out, double *lse)
{
    return oracle_fwd_items_ex(q, k, v, topk_idx, vbs, B, S, H, D, Nq, topk, sigma, items, n_items, out, lse,
                               NULL);
}

/* ---- tile plan -----------------------------------------------------------
 * Not from the pages: the pairing schedule of the paired forward kernel,
 * restated as plainly as possible so the GPU planner can be checked bit for
 * bit.  For each (b, h): overlap(i, j) = number of distinct cubes that both
 * lists name; each cube's candidates are the 8 cubes j != i with the largest
 * overlap (ties: smaller j); rounds: each unpaired cube proposes to its first
 * unpaired candidate, mutual proposals pair, until a round pairs none (at
 * most 64 rounds).  Refills: while two or more cubes are unpaired, each
 * unpaired cube's candidates become the 8 unpaired cubes j != i with the
 * largest overlap (same ties) and the rounds run again; stop when a refill
 * pairs none (at most 64 refills).  Leftovers pair in index order; tiles
 * are listed by smaller index as (smaller, larger) or (i, -1).
 * plan is [B*H][ceil(Nq/2)][2]. */
int oracle_plan(const int32_t *topk_idx, int B, int H, int Nq, int topk, int32_t *plan)
{
    if (B <= 0 || H <= 0 || Nq <= 0 || topk < 1) return ORACLE_ERR_ARG;
    const int NC = 8;
    unsigned char *member = (unsigned char *)malloc((size_t)Nq * Nq);
    int *cand = (int *)malloc((size_t)Nq * NC * sizeof(int));
    int *partner = (int *)malloc((size_t)Nq * sizeof(int));
    int *prop = (int *)malloc((size_t)Nq * sizeof(int));
    int *dist = (int *)malloc((size_t)Nq * (topk < Nq ? topk : Nq) * sizeof(int));
    int *ndist = (int *)malloc((size_t)Nq * sizeof(int));
    if (!member || !cand || !partner || !prop || !dist || !ndist) {
        free(member); free(cand); free(partner); free(prop); free(dist); free(ndist);
        return ORACLE_ERR_NOMEM;
    }
    const int tiles = (Nq + 1) / 2;
    for (int bh = 0; bh < B * H; ++bh) {
        memset(member, 0, (size_t)Nq * Nq);
        for (int i = 0; i < Nq; ++i)
            for (int t = 0; t < topk; ++t) {
                int j = topk_idx[((int64_t)bh * Nq + i) * topk + t];
                if (j >= 0 && j < Nq) member[(size_t)i * Nq + j] = 1;
            }
        /* the distinct cubes of each list, ascending */
        int ndist_max = topk < Nq ? topk : Nq;
        for (int j = 0; j < Nq; ++j) {
            int n = 0;
            for (int c = 0; c < Nq; ++c)
                if (member[(size_t)j * Nq + c]) dist[(size_t)j * ndist_max + n++] = c;
            ndist[j] = n;
        }
        for (int i = 0; i < Nq; ++i) partner[i] = -1;
        /* refill 0 computes every cube's candidates among all cubes; refill r > 0
           recomputes those of the unpaired cubes among the unpaired cubes */
        for (int refill = 0; refill <= 64; ++refill) {
            int unpaired = 0;
            for (int i = 0; i < Nq; ++i) unpaired += partner[i] < 0;
            if (refill > 0 && unpaired < 2) break;
            for (int i = 0; i < Nq; ++i) {
                if (partner[i] >= 0) continue;
                int best_ov[8], best_j[8];
                for (int c = 0; c < NC; ++c) { best_ov[c] = -1; best_j[c] = -1; }
                for (int j = 0; j < Nq; ++j) {
                    if (j == i || partner[j] >= 0) continue;
                    int ov = 0;
                    for (int e = 0; e < ndist[j]; ++e) ov += member[(size_t)i * Nq + dist[(size_t)j * ndist_max + e]];
                    /* j ascends, so a later j with an equal overlap never displaces an earlier one */
                    int pos = NC;
                    while (pos > 0 && ov > best_ov[pos - 1]) --pos;
                    if (pos < NC) {
                        for (int c = NC - 1; c > pos; --c) { best_ov[c] = best_ov[c - 1]; best_j[c] = best_j[c - 1]; }
                        best_ov[pos] = ov;
                        best_j[pos] = j;
                    }
                }
                for (int c = 0; c < NC; ++c) cand[i * NC + c] = best_j[c];
            }
            int paired_any = 0;
            for (int round = 0; round < 64; ++round) {
                for (int i = 0; i < Nq; ++i) {
                    prop[i] = -1;
                    if (partner[i] >= 0) continue;
                    for (int c = 0; c < NC; ++c) {
                        int j = cand[i * NC + c];
                        if (j >= 0 && partner[j] < 0) { prop[i] = j; break; }
                    }
                }
                int changed = 0;
                for (int i = 0; i < Nq; ++i) {
                    int j = prop[i];
                    if (j >= 0 && prop[j] == i) { partner[i] = j; changed = 1; }
                }
                if (!changed) break;
                paired_any = 1;
            }
            if (!paired_any) break;
        }
        int pending = -1, odd = -1;
        for (int i = 0; i < Nq; ++i) {
            if (partner[i] >= 0) continue;
            if (pending < 0) pending = i;
            else { partner[pending] = i; partner[i] = pending; pending = -1; }
        }
        odd = pending;
        int p = 0;
        for (int i = 0; i < Nq; ++i) {
            if (partner[i] > i || i == odd) {
                plan[((int64_t)bh * tiles + p) * 2] = i;
                plan[((int64_t)bh * tiles + p) * 2 + 1] = i == odd ? -1 : partner[i];
                ++p;
            }
        }
    }
    free(member); free(cand); free(partner); free(prop); free(dist); free(ndist);
    return ORACLE_OK;
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

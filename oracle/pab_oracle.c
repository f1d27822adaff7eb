/*
 * pab_oracle.c -- plain, slow, fp64 CPU oracle for the Pyramid Attention
 * Broadcast (PAB) attention stack.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path (the CUDA library
 * under step_reuse_b200/) links, loads or calls this file; only the tests,
 * the smoke check and the benchmark's CPU-baseline leg do.  It shares no
 * code, header, table or constant with the CUDA path.
 *
 * Sources (the PAB pages):
 *  - "Real-Time Video Generation with Pyramid Attention Broadcast"
 *    (chatpaper.ai abstract): attention outputs are broadcast to later
 *    diffusion steps in a pyramid style, a different strategy per attention.
 *  - m.sbmmt.com PAB report, section "Implementation" and Fig. 2: the three
 *    attention kinds (spatial, temporal, cross); the U-shaped attention
 *    difference (first and last 15% of steps change a lot, the middle 70% is
 *    stable); in the middle segment one step's attention output is broadcast
 *    to the next few steps, with a wider range for kinds that change less.
 *  - same report, Fig. 1: the difference between the attention outputs of
 *    consecutive diffusion steps is quantified by MSE.
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *  - attention is the textbook softmax(Q K^T / sqrt(d)) V per head, no mask,
 *    no bias, no output projection; head h owns channels [h*d, (h+1)*d);
 *  - the 15% edge is rounded up: e = ceil(edge_pct * steps / 100);
 *  - in the middle [e, steps - e) a compute serves itself plus the next
 *    (range - 1) steps; windows are anchored at the first middle step and the
 *    last one is cut at the end of the middle segment;
 *  - MSE is the mean over all elements of (a - b)^2.
 *
 * Every function works in double precision.  The attention inputs are the
 * bf16 values the GPU consumes, widened to double by the caller.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------------ */
/* Attention: one query row against Lk keys (the textbook definition).       */
/*   s_j = (q . k_j) / sqrt(d);  m = max_j s_j;  p_j = exp(s_j - m);         */
/*   o   = sum_j p_j v_j / sum_j p_j                                         */
/* k_j starts at kbase + j*kstride (d contiguous doubles), likewise v_j.     */
/* ------------------------------------------------------------------------ */
static void attend_one_query(const double *q, const double *kbase, long kstride,
                             const double *vbase, long vstride, int Lk, int d,
                             double *o, double *p /* Lk scratch */)
{
    const double scale = 1.0 / sqrt((double)d);
    double m = -INFINITY;
    for (int j = 0; j < Lk; ++j) {
        const double *kj = kbase + (long)j * kstride;
        double s = 0.0;
        for (int c = 0; c < d; ++c)
            s += q[c] * kj[c];
        s *= scale;
        p[j] = s;
        if (s > m)
            m = s;
    }
    double denom = 0.0;
    for (int j = 0; j < Lk; ++j) {
        p[j] = exp(p[j] - m);
        denom += p[j];
    }
    for (int c = 0; c < d; ++c) {
        double acc = 0.0;
        for (int j = 0; j < Lk; ++j)
            acc += p[j] * vbase[(long)j * vstride + c];
        o[c] = acc / denom;
    }
}

/* Spatial attention (attention within a frame).
 * q, k, v, o: [T][N][C] with C = heads*d.  For every frame t and head h the
 * N tokens of frame t attend to each other. */
int oracle_spatial_attention(const double *q, const double *k, const double *v,
                             double *o, int T, int N, int heads, int d)
{
    if (T < 0 || N < 0 || heads <= 0 || d <= 0)
        return -1;
    const long C = (long)heads * d;
    int bad = 0;
#pragma omp parallel
    {
        double *p = (double *)malloc(sizeof(double) * (N > 0 ? N : 1));
        if (!p) {
#pragma omp atomic write
            bad = 1;
        } else {
#pragma omp for collapse(2) schedule(dynamic)
            for (int t = 0; t < T; ++t)
                for (int h = 0; h < heads; ++h) {
                    const long frame = (long)t * N * C;
                    for (int n = 0; n < N; ++n)
                        attend_one_query(q + frame + (long)n * C + (long)h * d,
                                         k + frame + (long)h * d, C,
                                         v + frame + (long)h * d, C, N, d,
                                         o + frame + (long)n * C + (long)h * d, p);
                }
            free(p);
        }
    }
    return bad ? -2 : 0;
}

/* Temporal attention (attention across frames at one spatial position).
 * q, k, v, o: [N][T][C].  For every position n and head h the T frames at
 * position n attend to each other. */
int oracle_temporal_attention(const double *q, const double *k, const double *v,
                              double *o, int N, int T, int heads, int d)
{
    if (T < 0 || N < 0 || heads <= 0 || d <= 0)
        return -1;
    const long C = (long)heads * d;
    int bad = 0;
#pragma omp parallel
    {
        double *p = (double *)malloc(sizeof(double) * (T > 0 ? T : 1));
        if (!p) {
#pragma omp atomic write
            bad = 1;
        } else {
#pragma omp for collapse(2) schedule(dynamic, 64)
            for (int n = 0; n < N; ++n)
                for (int h = 0; h < heads; ++h) {
                    const long pos = (long)n * T * C;
                    for (int t = 0; t < T; ++t)
                        attend_one_query(q + pos + (long)t * C + (long)h * d,
                                         k + pos + (long)h * d, C,
                                         v + pos + (long)h * d, C, T, d,
                                         o + pos + (long)t * C + (long)h * d, p);
                }
            free(p);
        }
    }
    return bad ? -2 : 0;
}

/* Cross attention (video tokens attend to text tokens).
 * q, o: [R][C] (R video tokens, any order); kt, vt: [Lt][C] text tokens. */
int oracle_cross_attention(const double *q, const double *kt, const double *vt,
                           double *o, long R, int Lt, int heads, int d)
{
    if (R < 0 || Lt < 0 || heads <= 0 || d <= 0)
        return -1;
    const long C = (long)heads * d;
    int bad = 0;
#pragma omp parallel
    {
        double *p = (double *)malloc(sizeof(double) * (Lt > 0 ? Lt : 1));
        if (!p) {
#pragma omp atomic write
            bad = 1;
        } else {
#pragma omp for schedule(dynamic, 256)
            for (long r = 0; r < R; ++r)
                for (int h = 0; h < heads; ++h)
                    attend_one_query(q + r * C + (long)h * d, kt + (long)h * d, C,
                                     vt + (long)h * d, C, Lt, d,
                                     o + r * C + (long)h * d, p);
            free(p);
        }
    }
    return bad ? -2 : 0;
}

/* Sliding tile attention (STA) as the spatial kind: sgqg.cn summary of
 * "Fast Video Generation with Sliding Tile Attention", section "Sliding Tile
 * Attention (STA)" -- a frame is cut into non-overlapping tiles, every query
 * of a tile attends to the keys of the tiles inside a window around its own
 * tile, and frame and window sizes are whole numbers of tiles, so the tile
 * fits the window exactly.  2-D reading (PAB's spatial attention is per
 * frame): tiles of tile x tile tokens on the H x W token grid (token n = y*W
 * + x, the [T][N][C] layout), a window of win_h x win_w tokens = an odd
 * number of tiles in each direction centred on the query's tile, cut off at
 * the frame edge (no shift).  Per (frame, head, query tile) the window's keys
 * and values are gathered into scratch in row-major token order and every
 * query of the tile attends to them with the textbook definition above.
 * Returns -1 on arguments that break these rules. */
int oracle_sta_attention(const double *q, const double *k, const double *v,
                         double *o, int T, int H, int W, int heads, int d,
                         int tile, int win_h, int win_w)
{
    if (T < 0 || H < 0 || W < 0 || heads <= 0 || d <= 0 || tile <= 0)
        return -1;
    if (H % tile || W % tile || win_h <= 0 || win_w <= 0 || win_h % tile || win_w % tile)
        return -1;
    if ((win_h / tile) % 2 == 0 || (win_w / tile) % 2 == 0)
        return -1;
    const long C = (long)heads * d;
    const long N = (long)H * W;
    const int th = H / tile, tw = W / tile;
    const int rh = (win_h / tile - 1) / 2, rw = (win_w / tile - 1) / 2;
    const long maxkeys = (long)(2 * rh + 1) * tile * (2 * rw + 1) * tile;
    int bad = 0;
#pragma omp parallel
    {
        double *p = (double *)malloc(sizeof(double) * (maxkeys > 0 ? maxkeys : 1));
        double *kw = (double *)malloc(sizeof(double) * (size_t)(maxkeys > 0 ? maxkeys : 1) * d);
        double *vw = (double *)malloc(sizeof(double) * (size_t)(maxkeys > 0 ? maxkeys : 1) * d);
        if (!p || !kw || !vw) {
#pragma omp atomic write
            bad = 1;
        } else {
#pragma omp for collapse(3) schedule(dynamic)
            for (int t = 0; t < T; ++t)
                for (int h = 0; h < heads; ++h)
                    for (int qt = 0; qt < th * tw; ++qt) {
                        const int ty = qt / tw, tx = qt % tw;
                        const int y0 = (ty - rh < 0 ? 0 : ty - rh) * tile;
                        const int y1 = (ty + rh >= th ? th : ty + rh + 1) * tile;
                        const int x0 = (tx - rw < 0 ? 0 : tx - rw) * tile;
                        const int x1 = (tx + rw >= tw ? tw : tx + rw + 1) * tile;
                        const long frame = (long)t * N * C + (long)h * d;
                        int nk = 0;
                        for (int y = y0; y < y1; ++y)
                            for (int x = x0; x < x1; ++x, ++nk) {
                                const long src = frame + ((long)y * W + x) * C;
                                memcpy(kw + (long)nk * d, k + src, sizeof(double) * d);
                                memcpy(vw + (long)nk * d, v + src, sizeof(double) * d);
                            }
                        for (int y = ty * tile; y < (ty + 1) * tile; ++y)
                            for (int x = tx * tile; x < (tx + 1) * tile; ++x) {
                                const long at = frame + ((long)y * W + x) * C;
                                attend_one_query(q + at, kw, d, vw, d, nk, d, o + at, p);
                            }
                    }
        }
        free(p);
        free(kw);
        free(vw);
    }
    return bad ? -2 : 0;
}

/* Draft attention as the spatial kind: crisp3r.com article on "Draft
 * Attention" (low-resolution attention guidance), its steps 1-4 -- the
 * latent frame is average-pooled into a low-resolution sketch of the queries
 * and keys, the draft attention map of the sketch ranks regions, the
 * best-scoring regions form a structured sparse mask for the full-resolution
 * attention, and tokens are grouped so the kept blocks are contiguous.
 * Readings: regions of `region` x `region` tokens per frame; the sketch of a
 * region is the mean of its tokens' q (and k) per head; the draft score of
 * query region i and key region j is qbar_i . kbar_j / sqrt(d) (the draft
 * softmax is monotone along a row, so ranking scores ranks the map); every
 * query region keeps its `keep` best key regions, ties to the lower region
 * index; the selection is listed in ascending region index.
 * sel: [T][heads][R][keep] with R = (H/region) * (W/region). */
int oracle_draft_select(const double *q, const double *k, int T, int H, int W, int heads, int d,
                        int region, int keep, int *sel)
{
    if (T < 0 || H < 0 || W < 0 || heads <= 0 || d <= 0 || region <= 0)
        return -1;
    if (H % region || W % region)
        return -1;
    const int rw = W / region, R = (H / region) * rw;
    if (keep < 1 || keep > R)
        return -1;
    const long C = (long)heads * d;
    const long N = (long)H * W;
    const double scale = 1.0 / sqrt((double)d);
    int bad = 0;
#pragma omp parallel
    {
        double *qb = (double *)malloc(sizeof(double) * (size_t)R * d);
        double *kb = (double *)malloc(sizeof(double) * (size_t)R * d);
        double *sc = (double *)malloc(sizeof(double) * (size_t)R);
        char *taken = (char *)malloc((size_t)R);
        if (!qb || !kb || !sc || !taken) {
#pragma omp atomic write
            bad = 1;
        } else {
#pragma omp for collapse(2) schedule(dynamic)
            for (int t = 0; t < T; ++t)
                for (int h = 0; h < heads; ++h) {
                    /* step 1: the sketch -- per region, the mean of q and of k */
                    for (int r = 0; r < R; ++r) {
                        const int y0 = (r / rw) * region, x0 = (r % rw) * region;
                        for (int c = 0; c < d; ++c) {
                            double sq = 0.0, sk = 0.0;
                            for (int y = y0; y < y0 + region; ++y)
                                for (int x = x0; x < x0 + region; ++x) {
                                    const long at = (long)t * N * C + ((long)y * W + x) * C + (long)h * d + c;
                                    sq += q[at];
                                    sk += k[at];
                                }
                            qb[(long)r * d + c] = sq / ((double)region * region);
                            kb[(long)r * d + c] = sk / ((double)region * region);
                        }
                    }
                    /* steps 2-3: draft scores of each query region, keep the best */
                    for (int i = 0; i < R; ++i) {
                        for (int j = 0; j < R; ++j) {
                            double s = 0.0;
                            for (int c = 0; c < d; ++c)
                                s += qb[(long)i * d + c] * kb[(long)j * d + c];
                            sc[j] = s * scale;
                            taken[j] = 0;
                        }
                        for (int n = 0; n < keep; ++n) {
                            int best = -1;
                            for (int j = 0; j < R; ++j)
                                if (!taken[j] && (best < 0 || sc[j] > sc[best]))
                                    best = j;
                            taken[best] = 1;
                        }
                        int *row = sel + (((long)t * heads + h) * R + i) * keep;
                        int n = 0;
                        for (int j = 0; j < R; ++j)
                            if (taken[j])
                                row[n++] = j;
                    }
                }
        }
        free(qb);
        free(kb);
        free(sc);
        free(taken);
    }
    return bad ? -2 : 0;
}

/* Full-resolution attention under a region selection (step 3's sparse
 * mask): every query of region i attends to the tokens of the key regions
 * sel[t][h][i][0..keep), gathered in list order then row-major within a
 * region, with the textbook definition. */
int oracle_region_sparse_attention(const double *q, const double *k, const double *v, double *o,
                                   int T, int H, int W, int heads, int d, int region, int keep,
                                   const int *sel)
{
    if (T < 0 || H < 0 || W < 0 || heads <= 0 || d <= 0 || region <= 0)
        return -1;
    if (H % region || W % region)
        return -1;
    const int rw = W / region, R = (H / region) * rw;
    if (keep < 1 || keep > R)
        return -1;
    for (long i = 0; i < (long)T * heads * R * keep; ++i)
        if (sel[i] < 0 || sel[i] >= R)
            return -1;
    const long C = (long)heads * d;
    const long N = (long)H * W;
    const long maxkeys = (long)keep * region * region;
    int bad = 0;
#pragma omp parallel
    {
        double *p = (double *)malloc(sizeof(double) * maxkeys);
        double *kw = (double *)malloc(sizeof(double) * (size_t)maxkeys * d);
        double *vw = (double *)malloc(sizeof(double) * (size_t)maxkeys * d);
        if (!p || !kw || !vw) {
#pragma omp atomic write
            bad = 1;
        } else {
#pragma omp for collapse(3) schedule(dynamic)
            for (int t = 0; t < T; ++t)
                for (int h = 0; h < heads; ++h)
                    for (int i = 0; i < R; ++i) {
                        const int *row = sel + (((long)t * heads + h) * R + i) * keep;
                        const long frame = (long)t * N * C + (long)h * d;
                        int nk = 0;
                        for (int n = 0; n < keep; ++n) {
                            const int y0 = (row[n] / rw) * region, x0 = (row[n] % rw) * region;
                            for (int y = y0; y < y0 + region; ++y)
                                for (int x = x0; x < x0 + region; ++x, ++nk) {
                                    const long src = frame + ((long)y * W + x) * C;
                                    memcpy(kw + (long)nk * d, k + src, sizeof(double) * d);
                                    memcpy(vw + (long)nk * d, v + src, sizeof(double) * d);
                                }
                        }
                        const int y0 = (i / rw) * region, x0 = (i % rw) * region;
                        for (int y = y0; y < y0 + region; ++y)
                            for (int x = x0; x < x0 + region; ++x) {
                                const long at = frame + ((long)y * W + x) * C;
                                attend_one_query(q + at, kw, d, vw, d, nk, d, o + at, p);
                            }
                    }
        }
        free(p);
        free(kw);
        free(vw);
    }
    return bad ? -2 : 0;
}

/* ------------------------------------------------------------------------ */
/* PAB schedule, walked step by step in execution order (noisiest first).    */
/*   edge steps (first and last edge_pct%): always compute;                  */
/*   middle steps: a compute makes its output servable for the next          */
/*   (range - 1) steps; while that budget lasts the step is a broadcast hit  */
/*   (served from the cache), else it computes.                              */
/* Outputs, per step i: is_compute[i] in {0,1} and source[i] = the step      */
/* whose computed output step i uses (i itself when it computes).            */
/* ------------------------------------------------------------------------ */
int oracle_pab_edge_steps(int steps, int edge_pct)
{
    if (steps < 0 || edge_pct < 0 || edge_pct > 50)
        return -1;
    return (edge_pct * steps + 99) / 100; /* ceil(edge_pct% of steps) */
}

int oracle_pab_schedule(int steps, int edge_pct, int range, int *is_compute, int *source)
{
    if (steps < 0 || range < 1)
        return -1;
    const int e = oracle_pab_edge_steps(steps, edge_pct);
    if (e < 0)
        return -1;
    const int lo = e, hi = steps - e;
    int budget = 0;  /* further steps the cached output may still serve */
    int cached = -1; /* step whose output is in the cache */
    for (int i = 0; i < steps; ++i) {
        const int middle = (i >= lo && i < hi);
        if (middle && budget > 0 && cached >= 0) {
            is_compute[i] = 0;
            source[i] = cached;
            budget -= 1;
        } else {
            is_compute[i] = 1;
            source[i] = i;
            cached = i;
            budget = middle ? range - 1 : 0;
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Attention-difference diagnostic: mean over all n elements of (a - b)^2.   */
/* ------------------------------------------------------------------------ */
double oracle_mse(const double *a, const double *b, long n)
{
    if (n <= 0)
        return 0.0;
    double acc = 0.0;
    for (long i = 0; i < n; ++i) {
        const double diff = a[i] - b[i];
        acc += diff * diff;
    }
    return acc / (double)n;
}

/* ------------------------------------------------------------------------ */
/* Layout change between the spatial view [T][N][C] and the temporal view    */
/* [N][T][C]; elements are moved as opaque elem_size-byte units.             */
/* ------------------------------------------------------------------------ */
int oracle_layout(int to_temporal, const void *src, void *dst, int T, int N, int C,
                  int elem_size)
{
    if (T < 0 || N < 0 || C < 0 || elem_size <= 0)
        return -1;
    const char *s = (const char *)src;
    char *o = (char *)dst;
    const size_t row = (size_t)C * elem_size;
    for (int t = 0; t < T; ++t)
        for (int n = 0; n < N; ++n) {
            const size_t spatial_off = ((size_t)t * N + n) * row;
            const size_t temporal_off = ((size_t)n * T + t) * row;
            if (to_temporal)
                memcpy(o + temporal_off, s + spatial_off, row);
            else
                memcpy(o + spatial_off, s + temporal_off, row);
        }
    return 0;
}

/* Sequence-parallel packing (PAB report, "Parallel", Fig. 3: dynamic sequence
 * parallel moves each rank's frames of every position chunk to the rank
 * that owns the chunk, and back): swap the two outer dimensions of
 * [P][Q][block][C] -> [Q][P][block][C]; blocks of `block` rows of C
 * elements move unchanged. */
int oracle_permute_blocks(const void *src, void *dst, int P, int Q, long block, int C, int elem_size)
{
    if (P < 0 || Q < 0 || block < 0 || C < 0 || elem_size <= 0)
        return -1;
    const char *s = (const char *)src;
    char *o = (char *)dst;
    const size_t blk = (size_t)block * C * elem_size;
    for (int p = 0; p < P; ++p)
        for (int q = 0; q < Q; ++q)
            memcpy(o + ((size_t)q * P + p) * blk, s + ((size_t)p * Q + q) * blk, blk);
    return 0;
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

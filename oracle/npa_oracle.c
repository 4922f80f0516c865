/*
 * CPU oracle for patch-restricted self-attention, float64.
 *
 * TEST INFRASTRUCTURE ONLY. The tests, the package's smoke check and the
 * benchmark's CPU-baseline leg may call this code; the library's compute path
 * never does, and nothing here is shared with the CUDA sources.
 *
 * What it computes. For every requested query token t of every (batch, head)
 * the oracle
 *   1. builds the index set S(t) of the keys t may attend to, straight from
 *      the definition of the geometry (below);
 *   2. gathers K[S] and V[S], widening the bfloat16 inputs to double (exact);
 *   3. forms z_j = (q_t . k_j) / sqrt(d), m = max_j z_j, w_j = exp(z_j - m),
 *      l = sum_j w_j and o_t = sum_j (w_j / l) v_j, all in double;
 *   4. checks that the normalised weights sum to 1 within 1e-12.
 * The order of S is immaterial: softmax attention is invariant under any
 * permutation of its keys.
 *
 * Geometries.
 *  - Neighborhood Patch Attention (NPA). ScaleDiff: Higher-Resolution Image
 *    Synthesis via Efficient and Model-Agnostic Diffusion (atlas.scime.ai
 *    summary), "Approach" and the opening summary: the query grid is cut
 *    into non-overlapping patches and each patch attends to an overlapping
 *    key/value neighbourhood. Reading taken here: square patches of side P
 *    (ceil(H/P) x ceil(W/P) patches, the last row/column of patches smaller
 *    when P does not divide the grid); the neighbourhood is the patch grown
 *    by m tokens on each side and clipped to the grid (not shifted inward).
 *  - Partially conditioned attention (PCPP). Partially Conditioned Patch
 *    Parallelism for Accelerated Diffusion Model Inference (pith.science
 *    review), "What carries the argument" and "Core claim": a patch attends to
 *    itself plus the p-fraction of each neighbouring patch's height that lies
 *    next to it (the bottom rows of the patch above, the top rows of the
 *    patch below). Reading taken here: patches are n horizontal strips of
 *    s = H/n rows spanning the full width; the neighbour row count is
 *    r = ceil(p*s), evaluated in double with a 1e-9 allowance so that
 *    products that are whole numbers up to rounding stay whole, and limited
 *    to s; edge strips have one neighbour.
 *  - Both geometries may append G global tokens (separate K/V tensors) to
 *    every key set, once each.
 *
 * The same steps serve the later forms, each defined where it is written:
 * PCPP with the borrowed rows read from the previous step's keys/values, the
 * global tokens as queries over all keys, and the overlapping-window
 * (MultiDiffusion-style) attention NPA is compared with.
 *
 * Layout: q, k, v, out are [B, heads, H*W, d] with token t = row*W + col;
 * global k/v are [B, heads, G, d]. Inputs are bfloat16 bit patterns
 * (uint16); the output is double.
 *
 * Return codes: 0 success, -1 bad argument, -2 weights failed to sum to 1,
 * -3 out of memory.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_BAD_ARG (-1)
#define ORACLE_SUM_CHECK (-2)
#define ORACLE_NOMEM (-3)

static double bf16_to_double(uint16_t bits) {
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static int imin(int a, int b) { return a < b ? a : b; }
static int imax(int a, int b) { return a > b ? a : b; }

/* ------------------------------------------------------------------ */
/* Geometry: the key set of one query token.                           */
/* ------------------------------------------------------------------ */

/* Rows (or columns) of the window of the patch that holds coordinate x,
 * along an axis of length L cut into patches of side P and grown by m. */
static void npa_axis_window(int L, int P, int m, int x, int *lo, int *hi) {
    int pi = x / P;                       /* which patch along this axis   */
    int p0 = pi * P;                      /* first coordinate of the patch */
    int p1 = imin(L, p0 + P);             /* one past its last coordinate  */
    *lo = imax(0, p0 - m);                /* grown by m, clipped to grid   */
    *hi = imin(L, p1 + m);
}

/* Neighbour rows r = ceil(p*s), limited to [0, s]. */
int oracle_pcpp_neighbor_rows(int s, double p) {
    if (s < 1 || !(p >= 0.0) || !(p <= 1.0)) return -1;
    double x = p * (double)s;
    int r = (int)ceil(x - 1e-9);
    if (r < 0) r = 0;
    if (r > s) r = s;
    return r;
}

/* NPA key set of token t (image tokens only), written in ascending order.
 * Returns its size, or -1 on bad arguments. */
int oracle_npa_key_set(int H, int W, int P, int m, int t, int32_t *out) {
    if (H < 1 || W < 1 || P < 1 || m < 0 || t < 0 || t >= H * W) return -1;
    int row = t / W, col = t % W;
    int r_lo, r_hi, c_lo, c_hi;
    npa_axis_window(H, P, m, row, &r_lo, &r_hi);
    npa_axis_window(W, P, m, col, &c_lo, &c_hi);
    int n = 0;
    for (int r = r_lo; r < r_hi; ++r)
        for (int c = c_lo; c < c_hi; ++c)
            out[n++] = r * W + c;
    return n;
}

/* PCPP key set of token t: its own strip's rows, then the r rows of each
 * adjacent strip that touch it. Ascending order. Returns size or -1. */
int oracle_pcpp_key_set(int H, int W, int n_strips, double p, int t, int32_t *out) {
    if (H < 1 || W < 1 || n_strips < 1 || H % n_strips != 0 || t < 0 || t >= H * W) return -1;
    int s = H / n_strips;
    int r = oracle_pcpp_neighbor_rows(s, p);
    if (r < 0) return -1;
    int i = (t / W) / s;                 /* strip index of the query */
    int own_lo = i * s, own_hi = own_lo + s;
    int n = 0;
    /* bottom r rows of the strip above (if any) */
    if (i > 0)
        for (int row = own_lo - r; row < own_lo; ++row)
            for (int c = 0; c < W; ++c) out[n++] = row * W + c;
    /* the strip itself */
    for (int row = own_lo; row < own_hi; ++row)
        for (int c = 0; c < W; ++c) out[n++] = row * W + c;
    /* top r rows of the strip below (if any) */
    if (i < n_strips - 1)
        for (int row = own_hi; row < own_hi + r; ++row)
            for (int c = 0; c < W; ++c) out[n++] = row * W + c;
    return n;
}

/* ------------------------------------------------------------------ */
/* Attention over an explicit key set.                                 */
/* ------------------------------------------------------------------ */

/* One query row. keys: n_img image token ids into k/v (rows of d), then all
 * G global rows. When stale[j] is set, image key j is read from ks/vs instead
 * of k/v. Scratch z must hold n_img + G doubles. */
static int attend_one(const uint16_t *q_row, const uint16_t *k_bh, const uint16_t *v_bh,
                      const uint16_t *ks_bh, const uint16_t *vs_bh, const unsigned char *stale,
                      const uint16_t *gk_bh, const uint16_t *gv_bh, int G, int d,
                      const int32_t *keys, int n_img, double *z, double *o_row) {
    const double scale = 1.0 / sqrt((double)d);
    int n = n_img + G;
    double m = -INFINITY;
    for (int j = 0; j < n; ++j) {
        const uint16_t *kr = j >= n_img ? gk_bh + (size_t)(j - n_img) * d
                           : (stale && stale[j] ? ks_bh : k_bh) + (size_t)keys[j] * d;
        double dot = 0.0;
        for (int c = 0; c < d; ++c) dot += bf16_to_double(q_row[c]) * bf16_to_double(kr[c]);
        z[j] = dot * scale;
        if (z[j] > m) m = z[j];
    }
    double l = 0.0;
    for (int j = 0; j < n; ++j) {
        z[j] = exp(z[j] - m);
        l += z[j];
    }
    for (int c = 0; c < d; ++c) o_row[c] = 0.0;
    double wsum = 0.0;
    for (int j = 0; j < n; ++j) {
        double w = z[j] / l;
        wsum += w;
        const uint16_t *vr = j >= n_img ? gv_bh + (size_t)(j - n_img) * d
                           : (stale && stale[j] ? vs_bh : v_bh) + (size_t)keys[j] * d;
        for (int c = 0; c < d; ++c) o_row[c] += w * bf16_to_double(vr[c]);
    }
    if (fabs(wsum - 1.0) > 1e-12) return ORACLE_SUM_CHECK;
    return ORACLE_OK;
}

/* geometry id: 0 = NPA(a=P, b=m), 1 = PCPP(a=n_strips, p) */
static int key_set(int geom, int H, int W, int a, int b, double p, int t, int32_t *out) {
    return geom == 0 ? oracle_npa_key_set(H, W, a, b, t, out)
                     : oracle_pcpp_key_set(H, W, a, p, t, out);
}

/* Runs attention for a list of queries. queries holds n_queries triples
 * (b, h, t); out_rows receives n_queries rows of d doubles, in list order.
 * When queries is NULL, every (b, h, t) is computed and out_rows is the full
 * [B, heads, H*W, d] tensor. For PCPP with ks/vs given, the keys of a query's
 * own strip come from k/v and the neighbour rows from ks/vs. */
static int run(int geom, const uint16_t *q, const uint16_t *k, const uint16_t *v,
               const uint16_t *ks, const uint16_t *vs,
               const uint16_t *gk, const uint16_t *gv, double *out_rows,
               int B, int heads, int H, int W, int d, int a, int b, double p, int G,
               const int32_t *queries, long n_queries) {
    if (B < 1 || heads < 1 || H < 1 || W < 1 || d < 1 || G < 0) return ORACLE_BAD_ARG;
    if (G > 0 && (!gk || !gv)) return ORACLE_BAD_ARG;
    if ((ks != NULL) != (vs != NULL) || (ks && geom != 1)) return ORACLE_BAD_ARG;
    const long N = (long)H * W;
    const long total = queries ? n_queries : (long)B * heads * N;
    int status = ORACLE_OK;
    /* a probe call validates the geometry arguments once */
    {
        int32_t *tmp = (int32_t *)malloc(sizeof(int32_t) * (size_t)N);
        if (!tmp) return ORACLE_NOMEM;
        int rc = key_set(geom, H, W, a, b, p, 0, tmp);
        free(tmp);
        if (rc < 0) return ORACLE_BAD_ARG;
    }
#pragma omp parallel
    {
        int32_t *keys = (int32_t *)malloc(sizeof(int32_t) * (size_t)N);
        double *z = (double *)malloc(sizeof(double) * (size_t)(N + G));
        unsigned char *stale = ks ? (unsigned char *)malloc((size_t)N) : NULL;
        if (!keys || !z || (ks && !stale)) {
#pragma omp critical
            status = ORACLE_NOMEM;
        } else {
#pragma omp for schedule(dynamic, 64)
            for (long i = 0; i < total; ++i) {
                long bb, hh, t;
                if (queries) {
                    bb = queries[3 * i]; hh = queries[3 * i + 1]; t = queries[3 * i + 2];
                    if (bb < 0 || bb >= B || hh < 0 || hh >= heads || t < 0 || t >= N) {
#pragma omp critical
                        status = ORACLE_BAD_ARG;
                        continue;
                    }
                } else {
                    t = i % N; hh = (i / N) % heads; bb = i / (N * heads);
                }
                size_t bh = (size_t)bb * heads + hh;
                const uint16_t *k_bh = k + bh * N * d, *v_bh = v + bh * N * d;
                const uint16_t *gk_bh = G ? gk + bh * (size_t)G * d : NULL;
                const uint16_t *gv_bh = G ? gv + bh * (size_t)G * d : NULL;
                int n_img = key_set(geom, H, W, a, b, p, (int)t, keys);
                const uint16_t *ks_bh = ks ? ks + bh * N * d : NULL, *vs_bh = vs ? vs + bh * N * d : NULL;
                if (stale) {
                    /* a key is stale when its row lies outside the query's own strip */
                    int s_rows = H / a, own = (int)(t / W) / s_rows;
                    for (int j = 0; j < n_img; ++j) stale[j] = (unsigned char)((keys[j] / W) / s_rows != own);
                }
                int rc = attend_one(q + (bh * N + t) * d, k_bh, v_bh, ks_bh, vs_bh, stale, gk_bh, gv_bh, G, d, keys,
                                    n_img, z, out_rows + (size_t)i * d);
                if (rc != ORACLE_OK) {
#pragma omp critical
                    status = rc;
                }
            }
        }
        free(keys);
        free(z);
        free(stale);
    }
    return status;
}

int oracle_npa_attention(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                         const uint16_t *gk, const uint16_t *gv, double *out,
                         int B, int heads, int H, int W, int d, int P, int m, int G,
                         const int32_t *queries, long n_queries) {
    return run(0, q, k, v, NULL, NULL, gk, gv, out, B, heads, H, W, d, P, m, 0.0, G, queries, n_queries);
}

int oracle_pcpp_attention(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                          const uint16_t *gk, const uint16_t *gv, double *out,
                          int B, int heads, int H, int W, int d, int n_strips, double p, int G,
                          const int32_t *queries, long n_queries) {
    return run(1, q, k, v, NULL, NULL, gk, gv, out, B, heads, H, W, d, n_strips, 0, p, G, queries, n_queries);
}

/* PCPP with stale neighbour rows (PCPP review, "Core claim": a patch is
 * updated from its own activation plus the top or bottom p-fraction of the
 * neighbouring patches *from the previous step*): keys of the query's own
 * strip from k/v, the neighbour rows from ks/vs (same layout). */
int oracle_pcpp_attention_stale(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                                const uint16_t *ks, const uint16_t *vs,
                                const uint16_t *gk, const uint16_t *gv, double *out,
                                int B, int heads, int H, int W, int d, int n_strips, double p, int G,
                                const int32_t *queries, long n_queries) {
    if (!ks || !vs) return ORACLE_BAD_ARG;
    return run(1, q, k, v, ks, vs, gk, gv, out, B, heads, H, W, d, n_strips, 0, p, G, queries, n_queries);
}

/* Text-query half of joint attention: the G global tokens as queries, each
 * attending to every image token and every global token (full attention;
 * the pages leave the text tokens unrestricted - ScaleDiff summary: NPA
 * restricts the image-token queries of self-attention). gq, out: [B, heads,
 * G, d]; queries: optional (b, h, g) triples. */
int oracle_global_query_attention(const uint16_t *gq, const uint16_t *k, const uint16_t *v,
                                  const uint16_t *gk, const uint16_t *gv, double *out,
                                  int B, int heads, int H, int W, int d, int G,
                                  const int32_t *queries, long n_queries) {
    if (B < 1 || heads < 1 || H < 1 || W < 1 || d < 1 || G < 1 || !gq || !k || !v || !gk || !gv)
        return ORACLE_BAD_ARG;
    const long N = (long)H * W;
    const long total = queries ? n_queries : (long)B * heads * G;
    int status = ORACLE_OK;
#pragma omp parallel
    {
        int32_t *keys = (int32_t *)malloc(sizeof(int32_t) * (size_t)N);
        double *z = (double *)malloc(sizeof(double) * (size_t)(N + G));
        if (!keys || !z) {
#pragma omp critical
            status = ORACLE_NOMEM;
        } else {
            for (long j = 0; j < N; ++j) keys[j] = (int32_t)j;   /* every image token */
#pragma omp for schedule(dynamic, 16)
            for (long i = 0; i < total; ++i) {
                long bb, hh, g;
                if (queries) {
                    bb = queries[3 * i]; hh = queries[3 * i + 1]; g = queries[3 * i + 2];
                    if (bb < 0 || bb >= B || hh < 0 || hh >= heads || g < 0 || g >= G) {
#pragma omp critical
                        status = ORACLE_BAD_ARG;
                        continue;
                    }
                } else {
                    g = i % G; hh = (i / G) % heads; bb = i / ((long)G * heads);
                }
                size_t bh = (size_t)bb * heads + hh;
                int rc = attend_one(gq + (bh * G + g) * d, k + bh * N * d, v + bh * N * d, NULL, NULL, NULL,
                                    gk + bh * (size_t)G * d, gv + bh * (size_t)G * d, G, d, keys, (int)N, z,
                                    out + (size_t)i * d);
                if (rc != ORACLE_OK) {
#pragma omp critical
                    status = rc;
                }
            }
        }
        free(keys);
        free(z);
    }
    return status;
}

/* ------------------------------------------------------------------ */
/* MultiDiffusion-style overlapping-window attention (comparator).      */
/* ------------------------------------------------------------------ */
/* ScaleDiff summary, "Approach" and "Problem": MultiDiffusion covers the
 * latent with overlapping patches, processes each patch on its own and
 * averages the overlaps; NPA instead keeps the query patches disjoint and
 * lets each attend to an overlapping neighbourhood. Reading taken here, at
 * the level of one attention layer and with the NPA windows as the
 * overlapping patches: window (pi, pj) is NPA patch (pi, pj) grown by m and
 * clipped; inside each window every token attends to every token of that
 * window (plus the G global tokens); a token's output is the mean, over the
 * windows that contain it, of its attention output in each. */

/* Window (pi, pj) as row range [r0, r1) x column range [c0, c1). */
static void md_window(int H, int W, int P, int m, int pi, int pj, int *r0, int *r1, int *c0, int *c1) {
    *r0 = imax(0, pi * P - m);
    *r1 = imin(H, (pi + 1) * P + m);
    *c0 = imax(0, pj * P - m);
    *c1 = imin(W, (pj + 1) * P + m);
}

/* Tokens of window (pi, pj), ascending. Returns the count or -1. */
int oracle_md_window_keys(int H, int W, int P, int m, int pi, int pj, int32_t *out) {
    if (H < 1 || W < 1 || P < 1 || m < 0) return -1;
    int nph = (H + P - 1) / P, npw = (W + P - 1) / P;
    if (pi < 0 || pi >= nph || pj < 0 || pj >= npw) return -1;
    int r0, r1, c0, c1, n = 0;
    md_window(H, W, P, m, pi, pj, &r0, &r1, &c0, &c1);
    for (int r = r0; r < r1; ++r)
        for (int c = c0; c < c1; ++c) out[n++] = r * W + c;
    return n;
}

/* Number of windows that contain token t, by testing every window. */
int oracle_md_window_count(int H, int W, int P, int m, int t) {
    if (H < 1 || W < 1 || P < 1 || m < 0 || t < 0 || t >= H * W) return -1;
    int r = t / W, c = t % W, n = 0;
    for (int pi = 0; pi < (H + P - 1) / P; ++pi)
        for (int pj = 0; pj < (W + P - 1) / P; ++pj) {
            int r0, r1, c0, c1;
            md_window(H, W, P, m, pi, pj, &r0, &r1, &c0, &c1);
            n += (r >= r0 && r < r1 && c >= c0 && c < c1);
        }
    return n;
}

/* (query, key) pairs of one (b, h): sum over windows of |W| (|W| + G). */
long long oracle_md_pair_count(int H, int W, int P, int m, int G) {
    if (H < 1 || W < 1 || P < 1 || m < 0 || G < 0) return -1;
    long long total = 0;
    for (int pi = 0; pi < (H + P - 1) / P; ++pi)
        for (int pj = 0; pj < (W + P - 1) / P; ++pj) {
            int r0, r1, c0, c1;
            md_window(H, W, P, m, pi, pj, &r0, &r1, &c0, &c1);
            long long n = (long long)(r1 - r0) * (c1 - c0);
            total += n * (n + G);
        }
    return total;
}

/* Overlapping-window attention for a list of (b, h, t) queries (NULL: all,
 * out is then [B, heads, H*W, d]). */
int oracle_multidiffusion_attention(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                                    const uint16_t *gk, const uint16_t *gv, double *out,
                                    int B, int heads, int H, int W, int d, int P, int m, int G,
                                    const int32_t *queries, long n_queries) {
    if (B < 1 || heads < 1 || H < 1 || W < 1 || d < 1 || P < 1 || m < 0 || G < 0) return ORACLE_BAD_ARG;
    if (G > 0 && (!gk || !gv)) return ORACLE_BAD_ARG;
    const long N = (long)H * W;
    const long total = queries ? n_queries : (long)B * heads * N;
    const int nph = (H + P - 1) / P, npw = (W + P - 1) / P;
    int status = ORACLE_OK;
#pragma omp parallel
    {
        int32_t *keys = (int32_t *)malloc(sizeof(int32_t) * (size_t)N);
        double *z = (double *)malloc(sizeof(double) * (size_t)(N + G));
        double *o_w = (double *)malloc(sizeof(double) * (size_t)d);
        if (!keys || !z || !o_w) {
#pragma omp critical
            status = ORACLE_NOMEM;
        } else {
#pragma omp for schedule(dynamic, 16)
            for (long i = 0; i < total; ++i) {
                long bb, hh, t;
                if (queries) {
                    bb = queries[3 * i]; hh = queries[3 * i + 1]; t = queries[3 * i + 2];
                    if (bb < 0 || bb >= B || hh < 0 || hh >= heads || t < 0 || t >= N) {
#pragma omp critical
                        status = ORACLE_BAD_ARG;
                        continue;
                    }
                } else {
                    t = i % N; hh = (i / N) % heads; bb = i / (N * heads);
                }
                size_t bh = (size_t)bb * heads + hh;
                double *o = out + (size_t)i * d;
                for (int c = 0; c < d; ++c) o[c] = 0.0;
                int count = 0, r = (int)(t / W), col = (int)(t % W);
                for (int pi = 0; pi < nph; ++pi)
                    for (int pj = 0; pj < npw; ++pj) {
                        int r0, r1, c0, c1;
                        md_window(H, W, P, m, pi, pj, &r0, &r1, &c0, &c1);
                        if (r < r0 || r >= r1 || col < c0 || col >= c1) continue;
                        int n_img = oracle_md_window_keys(H, W, P, m, pi, pj, keys);
                        int rc = attend_one(q + (bh * N + t) * d, k + bh * N * d, v + bh * N * d, NULL, NULL, NULL,
                                            G ? gk + bh * (size_t)G * d : NULL, G ? gv + bh * (size_t)G * d : NULL,
                                            G, d, keys, n_img, z, o_w);
                        if (rc != ORACLE_OK) {
#pragma omp critical
                            status = rc;
                        }
                        for (int c = 0; c < d; ++c) o[c] += o_w[c];
                        ++count;
                    }
                for (int c = 0; c < d; ++c) o[c] /= (double)count;
            }
        }
        free(keys);
        free(z);
        free(o_w);
    }
    return status;
}

/* Number of (query, key) pairs, summed over all queries of one (b, h),
 * counting image keys and global keys. Brute force over every token. */
long long oracle_pair_count(int geom, int H, int W, int a, int b, double p, int G) {
    long N = (long)H * W;
    int32_t *tmp = (int32_t *)malloc(sizeof(int32_t) * (size_t)N);
    if (!tmp) return -1;
    long long total = 0;
    for (long t = 0; t < N; ++t) {
        int n = key_set(geom, H, W, a, b, p, (int)t, tmp);
        if (n < 0) { free(tmp); return -1; }
        total += n + G;
    }
    free(tmp);
    return total;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}

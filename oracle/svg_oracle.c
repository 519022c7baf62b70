/*
 * svg_oracle.c -- plain, slow, fp64 CPU oracle for block-sparse spatio-temporal attention.
 *
 * TEST INFRASTRUCTURE ONLY. Only the test-suite, the smoke check and the bench's CPU
 * baseline call this code; the product (the CUDA library) never links, loads or runs it,
 * and it shares no code, header or table with the CUDA path.
 *
 * What it computes, and where it comes from ("Accelerating Spatio-Temporal Attention for
 * Video Diffusion on TPUs", Google Developers Blog case study, as summarised by the three
 * pages on the subject):
 *   - Spatial heads attend to keys in the same or nearby frames; temporal heads attend to
 *     keys in a narrow spatial region across all frames ("Sparse Attention Patterns").
 *     Read here as: spatial keep(i,j) <=> |t(i)-t(j)| <= k, temporal keep(i,j) <=>
 *     |s(i)-s(j)| <= b, where t = frame and s = flattened patch index of a token.
 *   - Both masks keep full attention to the first frame as a sink ("Interesting facts").
 *     Read here as: keep(i,j) also holds whenever t(j) < F0 (F0 = sink frames, 1 by default).
 *   - Temporal heads use a different token order ("Interesting facts"); read here as the
 *     position map pi below (frame-0 prefix, then space-major), or fully space-major.
 *   - Tiles are "full" (only retained pairs), "boundary" (both), or skipped when empty
 *     ("Efficient Kernel Implementation", tile-aware masking; summary of the case study).
 *   - The tile-aligned ("rounded") variant snaps the mask to tile boundaries (summary,
 *     "What changed"). The pages give no rule; the reading used here keeps a whole tile
 *     iff at least half of its in-range pairs are retained (2*count >= area), else drops it.
 *   - Attention itself is exact softmax attention restricted to kept pairs.
 *
 * Every routine evaluates those definitions directly: the tile classifier visits every
 * element of every requested tile, attention visits every key of every requested row.
 * Floating point is fp64 throughout; inputs arrive as raw bf16 bit patterns and are
 * widened exactly (bits << 16 is the fp32 value, which fp64 represents exactly).
 * OpenMP only splits independent rows/tiles across threads; each result is computed by
 * one thread in a fixed order.
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <math.h>

#define OR_ROUTE_SPATIAL 0
#define OR_ROUTE_TEMPORAL 1
#define OR_LAYOUT_SINK_PREFIX 0
#define OR_LAYOUT_FULL_SPACE_MAJOR 1

/* bf16 bit pattern -> double, exactly. */
static double bf16_to_f64(uint16_t h) {
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Frame and flattened patch index of ORIGINAL token i (frame-major order, i = t*S + s). */
static void token_ts(int64_t i, int64_t S, int64_t *t, int64_t *s) {
    *t = i / S;
    *s = i % S;
}

/*
 * Position of original token (t, s) in the order a head of the given route uses.
 * Spatial heads keep the frame-major order. Temporal heads are reordered so that tokens
 * sharing a patch index sit next to each other (space-major), which is what turns the
 * temporal band into contiguous key ranges:
 *   SINK_PREFIX:      frames [0, F0) first, frame-major; then the remaining frames
 *                     space-major: pos = F0*S + s*(T-F0) + (t-F0).
 *   FULL_SPACE_MAJOR: pos = s*T + t for every frame.
 */
int64_t or_position(int route, int layout, int64_t T, int64_t S, int64_t F0, int64_t t, int64_t s) {
    if (route == OR_ROUTE_SPATIAL) return t * S + s;
    if (layout == OR_LAYOUT_FULL_SPACE_MAJOR) return s * T + t;
    if (t < F0) return t * S + s;
    return F0 * S + s * (T - F0) + (t - F0);
}

/* pi[i] = position of original token i. */
void or_perm_table(int route, int layout, int64_t T, int64_t S, int64_t F0, int64_t *pi) {
    int64_t N = T * S;
    for (int64_t i = 0; i < N; ++i) {
        int64_t t, s;
        token_ts(i, S, &t, &s);
        pi[i] = or_position(route, layout, T, S, F0, t, s);
    }
}

/* inv[p] = original token at position p (the inverse of pi, by scattering pi). */
void or_inverse_table(int route, int layout, int64_t T, int64_t S, int64_t F0, int64_t *inv) {
    int64_t N = T * S;
    for (int64_t i = 0; i < N; ++i) {
        int64_t t, s;
        token_ts(i, S, &t, &s);
        inv[or_position(route, layout, T, S, F0, t, s)] = i;
    }
}

/* The mask on original token identities (see header). */
int or_keep(int route, int64_t S, int64_t k, int64_t b, int64_t F0, int64_t i, int64_t j) {
    int64_t ti, si, tj, sj;
    token_ts(i, S, &ti, &si);
    token_ts(j, S, &tj, &sj);
    if (tj < F0) return 1;                       /* first-frame sink */
    if (route == OR_ROUTE_SPATIAL) return llabs(ti - tj) <= k;
    return llabs(si - sj) <= b;
}

/*
 * Brute-force tile classifier for one route class.
 * Tiles are [qt*bq, min(N,(qt+1)*bq)) x [kt*bk, min(N,(kt+1)*bk)) in POSITION space; each
 * in-range element (r, c) is mapped back to original tokens through inv and tested.
 * Only the q-tile rows listed in qts (n_qts of them) are evaluated; for each, every k-tile.
 * Outputs, row-major over (listed q-tile, kt):
 *   count[.] = retained pairs in the tile; cls[.] = 0 empty, 1 full, 2 boundary.
 */
void or_tile_counts(int route, int layout, int64_t T, int64_t S, int64_t k, int64_t b, int64_t F0,
                    int64_t bq, int64_t bk, const int64_t *qts, int64_t n_qts,
                    uint32_t *count, uint8_t *cls) {
    int64_t N = T * S;
    int64_t nk = (N + bk - 1) / bk;
    int64_t *inv = (int64_t *)malloc(sizeof(int64_t) * (size_t)N);
    or_inverse_table(route, layout, T, S, F0, inv);
    #pragma omp parallel for schedule(dynamic, 1)
    for (int64_t e = 0; e < n_qts * nk; ++e) {
        int64_t qt = qts[e / nk], kt = e % nk;
        int64_t r0 = qt * bq, r1 = r0 + bq < N ? r0 + bq : N;
        int64_t c0 = kt * bk, c1 = c0 + bk < N ? c0 + bk : N;
        uint64_t kept = 0, area = 0;
        for (int64_t r = r0; r < r1; ++r)
            for (int64_t c = c0; c < c1; ++c) {
                kept += (uint64_t)or_keep(route, S, k, b, F0, inv[r], inv[c]);
                ++area;
            }
        count[e] = (uint32_t)kept;
        cls[e] = kept == 0 ? 0 : (kept == area ? 1 : 2);
    }
    free(inv);
}

/*
 * Rounded ("tile-aligned") class of one tile from its exact retained count: the whole tile
 * is kept (class 1) iff 2*count >= in-range area, otherwise dropped (class 0).
 */
uint8_t or_rounded_class(uint32_t count, int64_t area) {
    return (2 * (uint64_t)count >= (uint64_t)area) ? 1 : 0;
}

/* Retained pairs of one head under the exact mask: every (i, j) pair is tested. */
uint64_t or_retained_pairs(int route, int64_t T, int64_t S, int64_t k, int64_t b, int64_t F0) {
    int64_t N = T * S;
    uint64_t total = 0;
    #pragma omp parallel for reduction(+:total) schedule(static)
    for (int64_t i = 0; i < N; ++i) {
        uint64_t row = 0;
        for (int64_t j = 0; j < N; ++j) row += (uint64_t)or_keep(route, S, k, b, F0, i, j);
        total += row;
    }
    return total;
}

/*
 * Masked softmax attention for listed query rows of one head, fp64.
 *   q, k, v: bf16 bit patterns, [N, d] row-major, ORIGINAL token order.
 *   rows:    n_rows original query indices.
 *   mask_kind: 0 exact mask (or_keep), 1 rounded tile mask (needs rcls), 2 every pair kept.
 *   rcls:    rounded classes [nq*nk] of this head's route (POSITION-space tiles bq x bk),
 *            used only for mask_kind 1: keep(i,j) <=> rcls[qt(pi(i))*nk + kt(pi(j))] == 1.
 *   out:     [n_rows, d] fp64, O = sum_j p_j v_j / sum_j p_j with p_j = exp(scale*q.k_j - m)
 *            over kept j, m = max over kept j of scale*q.k_j.
 *   lse:     [n_rows] fp64, m + log(sum_j p_j); rows with no kept key get O = 0, lse = -inf.
 */
void or_attention_rows(const uint16_t *q, const uint16_t *kk, const uint16_t *v,
                       int64_t N, int64_t d, double scale,
                       int route, int layout, int64_t T, int64_t S, int64_t k, int64_t b, int64_t F0,
                       int mask_kind, const uint8_t *rcls, int64_t bq, int64_t bk,
                       const int64_t *rows, int64_t n_rows, double *out, double *lse) {
    int64_t nk = (N + bk - 1) / bk;
    int64_t *pi = NULL;
    /* widen K and V once (exact), so the row loops below read doubles */
    double *kd = (double *)malloc(sizeof(double) * (size_t)(N * d));
    double *vd = (double *)malloc(sizeof(double) * (size_t)(N * d));
    for (int64_t x = 0; x < N * d; ++x) {
        kd[x] = bf16_to_f64(kk[x]);
        vd[x] = bf16_to_f64(v[x]);
    }
    if (mask_kind == 1) {
        pi = (int64_t *)malloc(sizeof(int64_t) * (size_t)N);
        or_perm_table(route, layout, T, S, F0, pi);
    }
    #pragma omp parallel
    {
        double *qrow = (double *)malloc(sizeof(double) * (size_t)d);
        double *sc = (double *)malloc(sizeof(double) * (size_t)N);
        unsigned char *kp = (unsigned char *)malloc((size_t)N);
        double *acc = (double *)malloc(sizeof(double) * (size_t)d);
        #pragma omp for schedule(dynamic, 1)
        for (int64_t r = 0; r < n_rows; ++r) {
            int64_t i = rows[r];
            for (int64_t x = 0; x < d; ++x) qrow[x] = bf16_to_f64(q[i * d + x]);
            double m = -INFINITY;
            for (int64_t j = 0; j < N; ++j) {
                int keep;
                if (mask_kind == 0) keep = or_keep(route, S, k, b, F0, i, j);
                else if (mask_kind == 1) keep = rcls[(pi[i] / bq) * nk + pi[j] / bk] == 1;
                else keep = 1;
                kp[j] = (unsigned char)keep;
                if (!keep) continue;
                double dot = 0.0;
                for (int64_t x = 0; x < d; ++x) dot += qrow[x] * kd[j * d + x];
                sc[j] = scale * dot;
                if (sc[j] > m) m = sc[j];
            }
            for (int64_t x = 0; x < d; ++x) acc[x] = 0.0;
            double l = 0.0;
            if (m != -INFINITY) {
                for (int64_t j = 0; j < N; ++j) {
                    if (!kp[j]) continue;
                    double p = exp(sc[j] - m);
                    l += p;
                    for (int64_t x = 0; x < d; ++x) acc[x] += p * vd[j * d + x];
                }
            }
            for (int64_t x = 0; x < d; ++x) out[r * d + x] = l > 0.0 ? acc[x] / l : 0.0;
            lse[r] = l > 0.0 ? m + log(l) : -INFINITY;
        }
        free(qrow); free(sc); free(kp); free(acc);
    }
    free(pi); free(kd); free(vd);
}

/*
 * Head routing by sampled rows (Sparse VideoGen's inference-time profiling, read as: attend the
 * sampled rows under the dense, spatial and temporal masks and compare with dense):
 *   out[0] = sum_rows |O_spatial - O_dense|^2, out[1] = sum_rows |O_temporal - O_dense|^2,
 *   out[2] = sum_rows |O_dense|^2  (fp64; exact masks on original identities).
 * The route is spatial iff out[0] <= out[1].
 */
void or_route_errors(const uint16_t *q, const uint16_t *kk, const uint16_t *v, int64_t N, int64_t d, double scale,
                     int64_t T, int64_t S, int64_t k, int64_t b, int64_t F0, const int64_t *rows, int64_t n_rows,
                     double *out) {
    double *od = (double *)malloc(sizeof(double) * (size_t)(n_rows * d));
    double *os = (double *)malloc(sizeof(double) * (size_t)(n_rows * d));
    double *ot = (double *)malloc(sizeof(double) * (size_t)(n_rows * d));
    double *lse = (double *)malloc(sizeof(double) * (size_t)n_rows);
    or_attention_rows(q, kk, v, N, d, scale, OR_ROUTE_SPATIAL, 0, T, S, k, b, F0, 2, NULL, 1, 1, rows, n_rows, od, lse);
    or_attention_rows(q, kk, v, N, d, scale, OR_ROUTE_SPATIAL, 0, T, S, k, b, F0, 0, NULL, 1, 1, rows, n_rows, os, lse);
    or_attention_rows(q, kk, v, N, d, scale, OR_ROUTE_TEMPORAL, 0, T, S, k, b, F0, 0, NULL, 1, 1, rows, n_rows, ot, lse);
    double es = 0.0, et = 0.0, ed = 0.0;
    for (int64_t x = 0; x < n_rows * d; ++x) {
        es += (os[x] - od[x]) * (os[x] - od[x]);
        et += (ot[x] - od[x]) * (ot[x] - od[x]);
        ed += od[x] * od[x];
    }
    out[0] = es;
    out[1] = et;
    out[2] = ed;
    free(od); free(os); free(ot); free(lse);
}

/* Threads the OpenMP runtime will use (reported next to oracle timings). */
int or_num_threads(void) {
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * Reference oracle for reciprocal nearest-neighbour matching.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the plain, slow, double-precision
 * statement of what the CUDA path computes.  Only the tests, the smoke check
 * and the CPU-baseline leg of the benchmark may load it.  It shares no code,
 * header, table or helper with the CUDA library.
 *
 * Sources (the page title, then the section):
 *  - cv-learn.com "MASt3R" note, section "Method and architecture", matching
 *    head: descriptors D1, D2 in R^{H x W x d}, one d-vector per pixel.
 *  - same note, paragraph "Fast reciprocal matching (FRM)": the reciprocal set
 *    M = {(i,j) | j = NN2(D1_i) and i = NN1(D2_j)}, and FRM: start from k
 *    pixels on a regular grid, iterate U^t -> V^t -> U^{t+1}, keep the
 *    correspondences that have converged.
 *  - staskaer.github.io blog on DUSt3R/MASt3R, section on MASt3R matching,
 *    the quoted function fast_reciprocal_NNs: the seed grid, the two
 *    half-steps with their convergence tests, the iteration cap and the
 *    de-duplicated, sorted output.
 *
 * Readings taken where the pages are silent (each is listed in the design
 * notes):
 *  - NN is the argmax of the dot product s(i,j) = sum_c D1[i][c] * D2[j][c];
 *    the descriptors are unit vectors, so this is the nearest neighbour in
 *    Euclidean distance as well.
 *  - Ties go to the lowest index: the scan is in increasing index order and
 *    only a strictly larger score replaces the best.
 *  - Pixel index p = y * W + x.
 *
 * Precision: every input value is an fp16 or bf16 number converted exactly to
 * double by the caller; scores are summed in double in channel order.
 *
 * Threads: independent queries are spread over OpenMP threads; the result
 * does not depend on the thread count.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <omp.h>

/* s(i,j): the dot product of two d-vectors, summed in channel order. */
static double score(const double *a, const double *b, int d)
{
    double s = 0.0;
    for (int c = 0; c < d; ++c)
        s += a[c] * b[c];
    return s;
}

/*
 * Metric of the nearest-neighbour query.  METRIC_DOT: the largest dot
 * product (the reading used throughout).  METRIC_L2: the smallest Euclidean
 * distance, which is what the quoted function's brute-force matcher computes
 * (it forms all the distances and keeps the smallest); it is scored here as the
 * negated squared distance so that "largest score" still means "nearest".
 */
enum { METRIC_DOT = 0, METRIC_L2 = 1 };

/* -||a - b||^2, summed in channel order. */
static double neg_sqdist(const double *a, const double *b, int d)
{
    double s = 0.0;
    for (int c = 0; c < d; ++c) {
        const double t = a[c] - b[c];
        s += t * t;
    }
    return -s;
}

static double score_metric(const double *a, const double *b, int d, int metric)
{
    return metric == METRIC_L2 ? neg_sqdist(a, b, d) : score(a, b, d);
}

/*
 * Nearest neighbour of query q among the n rows of X (row-major, d columns):
 * the lowest index attaining the largest score.  Also returns the best score
 * and the best score over every other index (-inf when n == 1).
 */
static int32_t nearest_m(const double *q, const double *X, int64_t n, int d, int metric,
                         double *best_out, double *second_out)
{
    double best = -INFINITY, second = -INFINITY;
    int32_t arg = -1;
    for (int64_t j = 0; j < n; ++j) {
        double s = score_metric(q, X + j * (int64_t)d, d, metric);
        if (s > best) {
            second = best;
            best = s;
            arg = (int32_t)j;
        } else if (s > second) {
            second = s;
        }
    }
    if (best_out) *best_out = best;
    if (second_out) *second_out = second;
    return arg;
}

static int32_t nearest(const double *q, const double *X, int64_t n, int d, double *best_out,
                       double *second_out)
{
    return nearest_m(q, X, n, d, METRIC_DOT, best_out, second_out);
}

static void set_threads(int nthreads)
{
    if (nthreads > 0) omp_set_num_threads(nthreads);
}

int oracle_max_threads(void) { return omp_get_max_threads(); }

/*
 * NN of every query row of Q (nq x d) among the rows of X (nx x d).
 * arg[q] = NN(q); best[q] = its score; second[q] = best score over the other
 * indices.  best/second may be NULL.
 */
void oracle_nn_metric(const double *Q, int64_t nq, const double *X, int64_t nx, int d,
                      int metric, int32_t *arg, double *best, double *second, int nthreads)
{
    set_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 16)
    for (int64_t i = 0; i < nq; ++i) {
        double b, s2;
        arg[i] = nearest_m(Q + i * (int64_t)d, X, nx, d, metric, &b, &s2);
        if (best) best[i] = b;
        if (second) second[i] = s2;
    }
}

void oracle_nn(const double *Q, int64_t nq, const double *X, int64_t nx, int d,
               int32_t *arg, double *best, double *second, int nthreads)
{
    oracle_nn_metric(Q, nq, X, nx, d, METRIC_DOT, arg, best, second, nthreads);
}

/*
 * Score of chosen pairs: out[t] = s(rows_a[t], rows_b[t]) between A and B.
 */
void oracle_pair_scores(const double *A, const double *B, int d, const int32_t *ia,
                        const int32_t *ib, int64_t n, double *out)
{
    for (int64_t t = 0; t < n; ++t)
        out[t] = score(A + (int64_t)ia[t] * d, B + (int64_t)ib[t] * d, d);
}

/*
 * The reciprocal (mutual) nearest-neighbour set
 *   M = {(i, j) : j = NN2(D1_i) and i = NN1(D2_j)}
 * listed in increasing i.  rowarg[i] = NN2(D1_i) and colarg[j] = NN1(D2_j)
 * are written too, with the best and second-best scores of every query when
 * the pointers are not NULL.  pairs holds room for min(n1, n2) (i, j) pairs.
 * Returns |M|.
 */
int64_t oracle_mnn_metric(const double *D1, int64_t n1, const double *D2, int64_t n2, int d,
                          int metric, int32_t *pairs, int32_t *rowarg, int32_t *colarg,
                          double *rowbest, double *rowsecond, double *colbest,
                          double *colsecond, int nthreads)
{
    oracle_nn_metric(D1, n1, D2, n2, d, metric, rowarg, rowbest, rowsecond, nthreads);
    oracle_nn_metric(D2, n2, D1, n1, d, metric, colarg, colbest, colsecond, nthreads);
    int64_t m = 0;
    for (int64_t i = 0; i < n1; ++i) {
        int32_t j = rowarg[i];
        if (colarg[j] == (int32_t)i) {
            pairs[2 * m] = (int32_t)i;
            pairs[2 * m + 1] = j;
            ++m;
        }
    }
    return m;
}

int64_t oracle_mnn(const double *D1, int64_t n1, const double *D2, int64_t n2, int d,
                   int32_t *pairs, int32_t *rowarg, int32_t *colarg,
                   double *rowbest, double *rowsecond, double *colbest, double *colsecond,
                   int nthreads)
{
    return oracle_mnn_metric(D1, n1, D2, n2, d, METRIC_DOT, pairs, rowarg, colarg, rowbest,
                             rowsecond, colbest, colsecond, nthreads);
}

/*
 * FRM seed grid on image 1: rows y = S//2, S//2 + S, ... < H and columns
 * x = S//2, S//2 + S, ... < W, as linear indices y*W + x.  The grid is
 * generated row by row, so the list is already unique and ascending (the
 * quoted function applies a unique() that sorts).  seeds may be NULL to only
 * count.  Returns the number of seeds.
 */
int64_t oracle_frm_seeds(int H, int W, int S, int32_t *seeds)
{
    int64_t k = 0;
    for (int y = S / 2; y < H; y += S)
        for (int x = S / 2; x < W; x += S) {
            if (seeds) seeds[k] = (int32_t)(y * (int64_t)W + x);
            ++k;
        }
    return k;
}

static int cmp_pair(const void *a, const void *b)
{
    const int32_t *p = (const int32_t *)a, *q = (const int32_t *)b;
    if (p[0] != q[0]) return p[0] < q[0] ? -1 : 1;
    if (p[1] != q[1]) return p[1] < q[1] ? -1 : 1;
    return 0;
}

/*
 * Fast reciprocal matching, following the quoted fast_reciprocal_NNs with a
 * stride (integer subsample) and no pixel tolerance, no basin output:
 *
 *   U = seeds, V = -1, U_old = U, V_old = V, all seeds active, t = 0
 *   while some seed is active:
 *     for active s: V[s] = NN2(D1[U[s]]);  active[s] = (V[s] != V_old[s])
 *     for active s: U[s] = NN1(D2[V[s]]);  active[s] = (U[s] != U_old[s])
 *     t = t + 1;  stop when t >= max_iter
 *     V_old = V;  U_old = U
 *   output the pairs (U[s], V[s]) of the seeds that are no longer active,
 *   de-duplicated and sorted by U (then V).
 *
 * Outputs:
 *   pairs      room for k pairs (k = number of seeds); returns the pair count.
 *   seed_u, seed_v   final U[s], V[s] of every seed (may be NULL).
 *   seed_queries     number of NN queries made for the seed (may be NULL).
 *   seed_converged   1 if the seed is not active at the end (may be NULL).
 *   seed_min_gap     smallest best-minus-second score gap over the seed's
 *                    queries (may be NULL).
 *   traj       (may be NULL) k x max_iter x 3: for every seed and iteration,
 *              (U queried in half-step 1, V found, U found in half-step 2);
 *              -1 where that query was not made.
 *   active_per_half  (may be NULL) 2*max_iter counts of queries issued in each
 *              half-step (0 after the loop ends).
 */
int64_t oracle_frm(const double *D1, int H1, int W1, const double *D2, int H2, int W2,
                   int d, int S, int max_iter, int32_t *pairs,
                   int32_t *seed_u, int32_t *seed_v, int32_t *seed_queries,
                   uint8_t *seed_converged, double *seed_min_gap, int32_t *traj,
                   int64_t *active_per_half, int nthreads)
{
    set_threads(nthreads);
    const int64_t n1 = (int64_t)H1 * W1, n2 = (int64_t)H2 * W2;
    const int64_t k = oracle_frm_seeds(H1, W1, S, NULL);
    if (active_per_half)
        for (int h = 0; h < 2 * max_iter; ++h) active_per_half[h] = 0;
    if (k == 0) return 0;

    int32_t *U = malloc(sizeof(int32_t) * k), *V = malloc(sizeof(int32_t) * k);
    int32_t *Uold = malloc(sizeof(int32_t) * k), *Vold = malloc(sizeof(int32_t) * k);
    int32_t *nq = calloc(k, sizeof(int32_t));
    uint8_t *active = malloc(k);
    double *gap = malloc(sizeof(double) * k);
    oracle_frm_seeds(H1, W1, S, U);
    for (int64_t s = 0; s < k; ++s) {
        V[s] = -1;
        Uold[s] = U[s];
        Vold[s] = V[s];
        active[s] = 1;
        gap[s] = INFINITY;
    }
    if (traj)
        for (int64_t e = 0; e < k * max_iter * 3; ++e) traj[e] = -1;

    int t = 0;
    for (;;) {
        int any = 0;
        for (int64_t s = 0; s < k; ++s) any |= active[s];
        if (!any) break;

        /* half-step 1: V = NN2(U) for the active seeds, then test V. */
        int64_t count = 0;
#pragma omp parallel for schedule(dynamic, 8) reduction(+ : count)
        for (int64_t s = 0; s < k; ++s) {
            if (!active[s]) continue;
            double b, s2;
            V[s] = nearest(D1 + (int64_t)U[s] * d, D2, n2, d, &b, &s2);
            if (b - s2 < gap[s]) gap[s] = b - s2;
            nq[s] += 1;
            count += 1;
        }
        if (active_per_half) active_per_half[2 * t] = count;
        for (int64_t s = 0; s < k; ++s)
            if (active[s] && traj) {
                traj[(s * max_iter + t) * 3] = U[s];
                traj[(s * max_iter + t) * 3 + 1] = V[s];
            }
        for (int64_t s = 0; s < k; ++s)
            if (active[s] && V[s] == Vold[s]) active[s] = 0;

        /* half-step 2: U = NN1(V) for the seeds still active, then test U. */
        count = 0;
#pragma omp parallel for schedule(dynamic, 8) reduction(+ : count)
        for (int64_t s = 0; s < k; ++s) {
            if (!active[s]) continue;
            double b, s2;
            U[s] = nearest(D2 + (int64_t)V[s] * d, D1, n1, d, &b, &s2);
            if (b - s2 < gap[s]) gap[s] = b - s2;
            nq[s] += 1;
            count += 1;
        }
        if (active_per_half) active_per_half[2 * t + 1] = count;
        for (int64_t s = 0; s < k; ++s)
            if (active[s] && traj) traj[(s * max_iter + t) * 3 + 2] = U[s];
        for (int64_t s = 0; s < k; ++s)
            if (active[s] && U[s] == Uold[s]) active[s] = 0;

        t += 1;
        if (t >= max_iter) break;
        for (int64_t s = 0; s < k; ++s) {
            Vold[s] = V[s];
            Uold[s] = U[s];
        }
    }

    int64_t m = 0;
    for (int64_t s = 0; s < k; ++s)
        if (!active[s]) {
            pairs[2 * m] = U[s];
            pairs[2 * m + 1] = V[s];
            ++m;
        }
    qsort(pairs, (size_t)m, 2 * sizeof(int32_t), cmp_pair);
    int64_t u = 0;
    for (int64_t r = 0; r < m; ++r)
        if (u == 0 || cmp_pair(pairs + 2 * r, pairs + 2 * (u - 1)) != 0) {
            pairs[2 * u] = pairs[2 * r];
            pairs[2 * u + 1] = pairs[2 * r + 1];
            ++u;
        }

    for (int64_t s = 0; s < k; ++s) {
        if (seed_u) seed_u[s] = U[s];
        if (seed_v) seed_v[s] = V[s];
        if (seed_queries) seed_queries[s] = nq[s];
        if (seed_converged) seed_converged[s] = (uint8_t)!active[s];
        if (seed_min_gap) seed_min_gap[s] = gap[s];
    }
    free(U); free(V); free(Uold); free(Vold); free(nq); free(active); free(gap);
    return u;
}

static int cmp_i32(const void *a, const void *b)
{
    const int32_t x = *(const int32_t *)a, y = *(const int32_t *)b;
    return x < y ? -1 : x > y;
}

/*
 * Fast reciprocal matching with the quoted function's other options:
 *
 *  - init, n_init: the start pixels are given (linear indices y*W1 + x) and
 *    are made unique and ascending, as the quoted function's unique() does;
 *    NULL means the grid of stride S.  (The quoted function then also fixes
 *    max_iter to 1; the caller passes max_iter.)
 *  - pixel_tol > 0: a seed has converged when its final U lies less than
 *    pixel_tol pixels (Euclidean distance between (row, column) positions)
 *    from U_old, the U it held at the start of the last iteration; with given
 *    start pixels the output pair is then (U_old, V), i.e. the start pixel
 *    and its match.  pixel_tol == 0: converged = no longer active, output
 *    (U, V).
 *  - basin_mode: the NN2 half-step does not deactivate anyone, and after
 *    the NN1 half-step basin[U_old] = U for every seed that was active in it
 *    (before its own test), so basin maps a visited pixel to the pixel its
 *    round trip returned to.  basin has H1*W1 + 1 entries, -1 where never
 *    written (the last entry is never written).
 *  - metric: METRIC_DOT or METRIC_L2 for every NN query.
 *
 * The loop is the one of oracle_frm:
 *   while some seed is active:
 *     V = NN2(U) for active seeds; [not basin_mode] deactivate V == V_old
 *     U = NN1(V) for active seeds; [basin_mode] basin[U_old] = U;
 *                                  deactivate U == U_old
 *     t += 1; stop when t >= max_iter; U_old = U, V_old = V
 *
 * pairs: room for pairs_cap pairs (the seed count suffices); returns the
 * number of unique pairs, sorted.  seed_* (each may be NULL) as in
 * oracle_frm, over the seeds in ascending order; n_seeds_out (may be NULL)
 * receives the seed count.
 */
int64_t oracle_frm_ex(const double *D1, int H1, int W1, const double *D2, int H2, int W2,
                      int d, const int32_t *init, int64_t n_init, int S, int max_iter,
                      double pixel_tol, int basin_mode, int metric, int32_t *pairs,
                      int64_t pairs_cap, int32_t *seed_u, int32_t *seed_v,
                      int32_t *seed_queries, uint8_t *seed_converged, int32_t *basin,
                      int64_t *n_seeds_out, int nthreads)
{
    set_threads(nthreads);
    const int64_t n1 = (int64_t)H1 * W1, n2 = (int64_t)H2 * W2;
    int64_t k;
    int32_t *U;
    if (init) {
        U = malloc(sizeof(int32_t) * (n_init > 0 ? n_init : 1));
        memcpy(U, init, sizeof(int32_t) * (size_t)n_init);
        qsort(U, (size_t)n_init, sizeof(int32_t), cmp_i32);
        k = 0;
        for (int64_t r = 0; r < n_init; ++r)
            if (k == 0 || U[r] != U[k - 1]) U[k++] = U[r];
    } else {
        k = oracle_frm_seeds(H1, W1, S, NULL);
        U = malloc(sizeof(int32_t) * (k > 0 ? k : 1));
        oracle_frm_seeds(H1, W1, S, U);
    }
    if (n_seeds_out) *n_seeds_out = k;
    if (basin)
        for (int64_t p = 0; p <= n1; ++p) basin[p] = -1;
    int32_t *V = malloc(sizeof(int32_t) * (k > 0 ? k : 1));
    int32_t *Uold = malloc(sizeof(int32_t) * (k > 0 ? k : 1));
    int32_t *Vold = malloc(sizeof(int32_t) * (k > 0 ? k : 1));
    int32_t *nq = calloc(k > 0 ? k : 1, sizeof(int32_t));
    uint8_t *active = malloc(k > 0 ? k : 1);
    for (int64_t s = 0; s < k; ++s) {
        V[s] = -1;
        Uold[s] = U[s];
        Vold[s] = -1;
        active[s] = 1;
    }

    int t = 0;
    while (k > 0) {
        int any = 0;
        for (int64_t s = 0; s < k; ++s) any |= active[s];
        if (!any) break;
#pragma omp parallel for schedule(dynamic, 8)
        for (int64_t s = 0; s < k; ++s) {
            if (!active[s]) continue;
            V[s] = nearest_m(D1 + (int64_t)U[s] * d, D2, n2, d, metric, NULL, NULL);
            nq[s] += 1;
        }
        if (!basin_mode)
            for (int64_t s = 0; s < k; ++s)
                if (active[s] && V[s] == Vold[s]) active[s] = 0;
#pragma omp parallel for schedule(dynamic, 8)
        for (int64_t s = 0; s < k; ++s) {
            if (!active[s]) continue;
            U[s] = nearest_m(D2 + (int64_t)V[s] * d, D1, n1, d, metric, NULL, NULL);
            nq[s] += 1;
        }
        if (basin_mode && basin)
            for (int64_t s = 0; s < k; ++s)
                if (active[s]) basin[Uold[s]] = U[s];
        for (int64_t s = 0; s < k; ++s)
            if (active[s] && U[s] == Uold[s]) active[s] = 0;
        t += 1;
        if (t >= max_iter) break;
        for (int64_t s = 0; s < k; ++s) {
            Vold[s] = V[s];
            Uold[s] = U[s];
        }
    }

    int64_t m = 0;
    for (int64_t s = 0; s < k; ++s) {
        int conv;
        int32_t u = U[s];
        if (pixel_tol > 0) {
            const double dy = (double)(Uold[s] / W1) - (double)(U[s] / W1);
            const double dx = (double)(Uold[s] % W1) - (double)(U[s] % W1);
            conv = sqrt(dy * dy + dx * dx) < pixel_tol;
            if (init) u = Uold[s];
        } else {
            conv = !active[s];
        }
        if (conv && m < pairs_cap) {
            pairs[2 * m] = u;
            pairs[2 * m + 1] = V[s];
            ++m;
        }
        if (seed_u) seed_u[s] = U[s];
        if (seed_v) seed_v[s] = V[s];
        if (seed_queries) seed_queries[s] = nq[s];
        if (seed_converged) seed_converged[s] = (uint8_t)conv;
    }
    qsort(pairs, (size_t)m, 2 * sizeof(int32_t), cmp_pair);
    int64_t un = 0;
    for (int64_t r = 0; r < m; ++r)
        if (un == 0 || cmp_pair(pairs + 2 * r, pairs + 2 * (un - 1)) != 0) {
            pairs[2 * un] = pairs[2 * r];
            pairs[2 * un + 1] = pairs[2 * r + 1];
            ++un;
        }
    free(U); free(V); free(Uold); free(Vold); free(nq); free(active);
    return un;
}

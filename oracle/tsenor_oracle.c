/*
 * CPU oracle for transposable N:M mask search (TSENOR).
 *
 * TEST INFRASTRUCTURE.  This file is a plain, slow, obviously-correct
 * restatement of the method, used only by the test suite, by the smoke check
 * and by the CPU-baseline leg of the benchmark.  The CUDA library shares no
 * code with it and never calls it.
 *
 * Source: "Pith review of TSENOR: Highly-Efficient Algorithm for Finding
 * Transposable N:M Sparse Masks" (pith.science/paper/2505.23949), sections
 * "What carries the argument", "Core claim", referee comments 1-3 and minor
 * comment 2, "Assumptions & free parameters".
 *
 * Problem (Core claim): split W into MxM blocks; per block maximise
 * sum_ij |W_ij| s_ij over 0/1 matrices s with every row sum and every column
 * sum equal to N.
 *
 * Method (What carries the argument): relax to 0 <= S <= 1 (a capacitated
 * transport problem), add an entropy term, solve it with Dykstra's
 * alternating KL projections (row normalisation, column normalisation, clip
 * at 1) in log space, then round: sort entries by S descending, take an entry
 * while its row and column budgets remain, then swap entries in with the
 * 2-in/1-out move scored (|W_ij'| + |W_i'j|) - |W_i'j'|.
 *
 * Readings taken where the pages leave a step open:
 *  - kernel: x0_ij = tau * a_ij / max(a over the block), x0 = 0 for an
 *    all-zero block; logQ0 = 0.
 *  - one iteration = row step, column step, clip; only the clip carries a
 *    Dykstra correction (the row and column sets are affine).
 *  - the plan is S = exp(x) after the clip of the last iteration; the sort
 *    key is that S rounded to fp32, ties broken by a descending, then by the
 *    flat index i*M + j ascending.
 *  - the greedy scans all M*M entries.
 *  - repair: while a row is short, take the lowest short row i and the lowest
 *    short column j and apply the 2-in/1-out move with the best score,
 *    whatever its sign (ties: lowest i'*M + j').  With the full greedy scan a
 *    candidate always exists; the block is reported as failed only if none
 *    does (never expected).  Why one exists: the greedy visits every entry,
 *    so when it ends every pair (short row i, short column j) is taken --
 *    entry (i,j) was visited while both still had budget.  A short row
 *    exists only if a short column does (rows and columns hold the same
 *    number of ones), and column j short means some row i' has s_i'j = 0;
 *    such a row is full (N ones), for otherwise (i',j) would be a short
 *    pair that is not taken.  Row i is short, so it has at least M-N+1
 *    zeros, and N + (M-N+1) > M: some column j' holds a one of row i' and a
 *    zero of row i, and (i,j'),(i',j) in, (i',j') out is a candidate.  A
 *    move takes a one only from a full row and adds ones to row i and
 *    column j, so "every short row x short column pair is taken" still holds
 *    after it, and the argument repeats until no row is short.
 *  - local search: one sweep visits anchor rows i = 0..M-1; for each anchor
 *    the best partner row i' is chosen by the net gain of freeing (i,j) and
 *    taking the 2-in/1-out move, and the move is applied only if that gain is
 *    positive.
 * Floating point: the Dykstra iteration is fp64 with libm exp/log; every
 * quantity that decides an integer (sort keys, repair scores, swap gains) is
 * fp32, the precision the CUDA kernels take the same decisions in.
 *
 * Parity pins: see tests/test_oracle_*.py (brute force, linear programming,
 * assignment, closed forms, an independent dual solve, hand-worked fixtures).
 */
#define _GNU_SOURCE
#include <float.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct {
    int64_t repairs;    /* 2-in/1-out repair moves applied */
    int64_t ls_swaps;   /* improving local-search swaps applied */
    int64_t failures;   /* blocks with non-finite input or no repair move */
    int64_t short_after_greedy; /* blocks left infeasible by the greedy */
} oracle_stats;

/* ------------------------------------------------------------------ */
/* Dykstra's algorithm in log space (What carries the argument; Core claim;
 * minor comment 2 on Algorithm 1).                                     */

static double row_lse(const double* x, int M, int i) {
    double m = -INFINITY;
    for (int j = 0; j < M; ++j) if (x[i * M + j] > m) m = x[i * M + j];
    double s = 0.0;
    for (int j = 0; j < M; ++j) s += exp(x[i * M + j] - m);
    return m + log(s);
}

static double col_lse(const double* x, int M, int j) {
    double m = -INFINITY;
    for (int i = 0; i < M; ++i) if (x[i * M + j] > m) m = x[i * M + j];
    double s = 0.0;
    for (int i = 0; i < M; ++i) s += exp(x[i * M + j] - m);
    return m + log(s);
}

/* a: M*M magnitudes (row-major).  S_out: M*M plan after `iters` iterations.
 * x and q are M*M scratch arrays. */
static void block_plan(const float* a, int N, int M, double tau, int iters,
                       double* x, double* q, double* S_out) {
    const int E = M * M;
    double mb = 0.0;
    for (int e = 0; e < E; ++e) if ((double)a[e] > mb) mb = (double)a[e];
    for (int e = 0; e < E; ++e) {
        x[e] = mb > 0.0 ? tau * ((double)a[e] / mb) : 0.0;
        q[e] = 0.0;
    }
    const double lnN = log((double)N);
    for (int t = 0; t < iters; ++t) {
        /* C1: every row of exp(x) sums to N. */
        for (int i = 0; i < M; ++i) {
            double lse = row_lse(x, M, i);
            for (int j = 0; j < M; ++j) x[i * M + j] = x[i * M + j] - lse + lnN;
        }
        /* C2: every column of exp(x) sums to N. */
        for (int j = 0; j < M; ++j) {
            double lse = col_lse(x, M, j);
            for (int i = 0; i < M; ++i) x[i * M + j] = x[i * M + j] - lse + lnN;
        }
        /* C3: exp(x) <= 1, with Dykstra's correction term logQ. */
        for (int e = 0; e < E; ++e) {
            double y = x[e] + q[e];
            x[e] = y < 0.0 ? y : 0.0;
            q[e] = y - x[e];
        }
    }
    for (int e = 0; e < E; ++e) S_out[e] = exp(x[e]);
}

/* Warm start and adaptive stopping of the Dykstra loop.  The review fixes T
 * and gives no convergence test ("Assumptions & free parameters"); these two
 * extensions rest on one identity.  The row and column steps add potentials
 * to x (r_i = ln N - LSE_i, c_j = ln N - LSE_j), and the clip only moves an
 * amount between x and the correction q, so after every clip
 *     x + q = y0 + U_i + V_j,   x = min(x + q, 0),   q = max(x + q, 0),
 * where U, V are the potentials accumulated so far and y0 = x0 - tau.  The
 * 2M numbers (U, V) are therefore the whole state of a block.
 *  - Cold start: U = V = 0, i.e. x = y0 (<= 0), q = 0.  That is the start x0
 *    of block_plan shifted by -tau in every row; the first row step removes
 *    any per-row shift, so every later iterate equals block_plan's.
 *  - Warm start: the caller's (U, V), e.g. the final potentials of an earlier
 *    call on a nearby W.
 *  - Stopping: after iteration t, with delta_t = the largest |r_i| and |c_j|
 *    of that iteration, stop when tol > 0 and delta_t <= tol (at most iters
 *    iterations).  tol = 0 runs all iters.
 * uv (2M doubles, U then V): read when warm, always overwritten with the
 * final potentials.  Returns the number of iterations run. */
static int block_plan_ext(const float* a, int N, int M, double tau, int iters, double tol, int warm,
                          double* uv, double* x, double* q, double* S_out) {
    const int E = M * M;
    double* U = uv;
    double* V = uv + M;
    if (!warm)
        for (int k = 0; k < 2 * M; ++k) uv[k] = 0.0;
    double mb = 0.0;
    for (int e = 0; e < E; ++e) if ((double)a[e] > mb) mb = (double)a[e];
    for (int i = 0; i < M; ++i)
        for (int j = 0; j < M; ++j) {
            const int e = i * M + j;
            const double x0 = mb > 0.0 ? tau * ((double)a[e] / mb) : 0.0;
            const double y = (x0 - tau) + U[i] + V[j];
            x[e] = y < 0.0 ? y : 0.0;
            q[e] = y - x[e];
        }
    const double lnN = log((double)N);
    int t = 0;
    while (t < iters) {
        double delta = 0.0;
        for (int i = 0; i < M; ++i) {
            const double r = lnN - row_lse(x, M, i);
            for (int j = 0; j < M; ++j) x[i * M + j] += r;
            U[i] += r;
            if (fabs(r) > delta) delta = fabs(r);
        }
        for (int j = 0; j < M; ++j) {
            const double c = lnN - col_lse(x, M, j);
            for (int i = 0; i < M; ++i) x[i * M + j] += c;
            V[j] += c;
            if (fabs(c) > delta) delta = fabs(c);
        }
        for (int e = 0; e < E; ++e) {
            double y = x[e] + q[e];
            x[e] = y < 0.0 ? y : 0.0;
            q[e] = y - x[e];
        }
        ++t;
        if (tol > 0.0 && delta <= tol) break;
    }
    for (int e = 0; e < E; ++e) S_out[e] = exp(x[e]);
    return t;
}

/* ------------------------------------------------------------------ */
/* Rounding (What carries the argument; Fig. 2 caption; referee comment 3). */

typedef struct { const float* key; const float* a; } sort_ctx;

/* Total order: key descending, then a descending, then flat index ascending. */
static int cmp_entries(const void* pa, const void* pb, void* pctx) {
    const sort_ctx* c = (const sort_ctx*)pctx;
    int e1 = *(const int*)pa, e2 = *(const int*)pb;
    if (c->key[e1] != c->key[e2]) return c->key[e1] > c->key[e2] ? -1 : 1;
    if (c->a[e1] != c->a[e2]) return c->a[e1] > c->a[e2] ? -1 : 1;
    return e1 < e2 ? -1 : (e1 > e2 ? 1 : 0);
}

static void greedy(const float* key, const float* a, int N, int M, uint8_t* s, int* order) {
    const int E = M * M;
    for (int e = 0; e < E; ++e) order[e] = e;
    sort_ctx ctx = {key, a};
    qsort_r(order, (size_t)E, sizeof(int), cmp_entries, &ctx);
    int r[64], c[64];
    for (int i = 0; i < M; ++i) { r[i] = 0; c[i] = 0; }
    memset(s, 0, (size_t)E);
    for (int k = 0; k < E; ++k) {
        int e = order[k], i = e / M, j = e % M;
        if (r[i] < N && c[j] < N) { s[e] = 1; r[i]++; c[j]++; }
    }
}

/* Returns 0 when every row and column holds N ones, -1 if a move was missing. */
static int repair(const float* a, int N, int M, uint8_t* s, int64_t* moves) {
    for (;;) {
        int i = -1, j = -1;
        for (int r = 0; r < M && i < 0; ++r) {
            int cnt = 0;
            for (int k = 0; k < M; ++k) cnt += s[r * M + k];
            if (cnt < N) i = r;
        }
        if (i < 0) return 0;
        for (int col = 0; col < M && j < 0; ++col) {
            int cnt = 0;
            for (int k = 0; k < M; ++k) cnt += s[k * M + col];
            if (cnt < N) j = col;
        }
        if (j < 0) return -1;
        float best = -INFINITY;
        int bi = -1, bj = -1;
        for (int ip = 0; ip < M; ++ip) {
            for (int jp = 0; jp < M; ++jp) {
                if (!s[ip * M + jp] || s[i * M + jp] || s[ip * M + j]) continue;
                float sigma = (a[i * M + jp] + a[ip * M + j]) - a[ip * M + jp];
                if (bi < 0 || sigma > best) { best = sigma; bi = ip; bj = jp; }
            }
        }
        if (bi < 0) return -1;
        s[i * M + bj] = 1;
        s[bi * M + j] = 1;
        s[bi * M + bj] = 0;
        (*moves)++;
    }
}

static void local_search(const float* a, int M, int sweeps, uint8_t* s, int64_t* swaps) {
    for (int sw = 0; sw < sweeps; ++sw) {
        for (int i = 0; i < M; ++i) {
            float best_g = -INFINITY;
            int bp = -1, bj = -1, bjp = -1;
            for (int ip = 0; ip < M; ++ip) {
                if (ip == i) continue;
                /* best entry of row i to hand over to row ip */
                float t1 = -INFINITY; int j1 = -1;
                for (int j = 0; j < M; ++j) {
                    if (s[i * M + j] && !s[ip * M + j]) {
                        float d = a[ip * M + j] - a[i * M + j];
                        if (j1 < 0 || d > t1) { t1 = d; j1 = j; }
                    }
                }
                if (j1 < 0) continue;        /* rows i and ip hold the same columns */
                /* best entry of row ip to hand over to row i */
                float t2 = -INFINITY; int j2 = -1;
                for (int j = 0; j < M; ++j) {
                    if (!s[i * M + j] && s[ip * M + j]) {
                        float d = a[i * M + j] - a[ip * M + j];
                        if (j2 < 0 || d > t2) { t2 = d; j2 = j; }
                    }
                }
                float g = t1 + t2;
                if (bp < 0 || g > best_g) { best_g = g; bp = ip; bj = j1; bjp = j2; }
            }
            if (bp >= 0 && best_g > 0.0f) {
                s[i * M + bj] = 0;
                s[bp * M + bjp] = 0;
                s[i * M + bjp] = 1;
                s[bp * M + bj] = 1;
                (*swaps)++;
            }
        }
    }
}

/* stage: 1 = greedy only, 2 = greedy + repair, 3 = greedy + repair + local search.
 * Returns 0, or -1 when the block could not be made feasible. */
static int block_round(const float* key, const float* a, int N, int M, int sweeps, int stage,
                       uint8_t* s, int* order, oracle_stats* st) {
    greedy(key, a, N, M, s, order);
    if (stage < 2) return 0;
    int short_rows = 0;
    for (int i = 0; i < M; ++i) {
        int cnt = 0;
        for (int k = 0; k < M; ++k) cnt += s[i * M + k];
        short_rows += cnt < N;
    }
    if (short_rows) st->short_after_greedy++;
    if (repair(a, N, M, s, &st->repairs) != 0) return -1;
    if (stage < 3) return 0;
    local_search(a, M, sweeps, s, &st->ls_swaps);
    return 0;
}

/* ------------------------------------------------------------------ */
/* Exact optimum: min-cost flow (successive shortest paths, Dijkstra with
 * potentials).  The LP relaxation is integral (Core claim: bipartite
 * matching polytope; Assumptions: "standard math"), so the flow optimum is
 * the block optimum.                                                   */

static double block_opt(const float* a, int N, int M, uint8_t* f) {
    /* nodes: 0 source, 1..M rows, M+1..2M columns, 2M+1 sink */
    const int V = 2 * M + 2, S = 0, T = 2 * M + 1;
    double pi[130], d[130];
    int prev[130], done[130], r[64], c[64];
    memset(f, 0, (size_t)M * M);
    for (int i = 0; i < M; ++i) { r[i] = 0; c[i] = 0; }
    pi[S] = 0.0;
    for (int i = 0; i < M; ++i) pi[1 + i] = 0.0;
    double pt = INFINITY;
    for (int j = 0; j < M; ++j) {
        double mx = -INFINITY;
        for (int i = 0; i < M; ++i) if ((double)a[i * M + j] > mx) mx = (double)a[i * M + j];
        pi[1 + M + j] = -mx;
        if (-mx < pt) pt = -mx;
    }
    pi[T] = pt;
    for (int unit = 0; unit < N * M; ++unit) {
        for (int v = 0; v < V; ++v) { d[v] = INFINITY; prev[v] = -1; done[v] = 0; }
        d[S] = 0.0;
        for (;;) {
            int u = -1;
            for (int v = 0; v < V; ++v)
                if (!done[v] && d[v] < INFINITY && (u < 0 || d[v] < d[u])) u = v;
            if (u < 0) break;
            done[u] = 1;
            if (u == T) break;
            if (u == S) {
                for (int i = 0; i < M; ++i) if (r[i] < N) {
                    int v = 1 + i;
                    double nd = d[u] + (0.0 + pi[u] - pi[v]);
                    if (nd < d[v]) { d[v] = nd; prev[v] = u; }
                }
            } else if (u <= M) {
                int i = u - 1;
                for (int j = 0; j < M; ++j) if (!f[i * M + j]) {
                    int v = 1 + M + j;
                    double nd = d[u] + (-(double)a[i * M + j] + pi[u] - pi[v]);
                    if (nd < d[v]) { d[v] = nd; prev[v] = u; }
                }
            } else {
                int j = u - 1 - M;
                for (int i = 0; i < M; ++i) if (f[i * M + j]) {
                    int v = 1 + i;
                    double nd = d[u] + ((double)a[i * M + j] + pi[u] - pi[v]);
                    if (nd < d[v]) { d[v] = nd; prev[v] = u; }
                }
                if (c[j] < N) {
                    double nd = d[u] + (0.0 + pi[u] - pi[T]);
                    if (nd < d[T]) { d[T] = nd; prev[T] = u; }
                }
            }
        }
        if (d[T] == INFINITY) return NAN;
        const double D = d[T];
        for (int v = 0; v < V; ++v) pi[v] += (d[v] < D ? d[v] : D);
        /* augment one unit along the path */
        int v = T;
        while (prev[v] != S) {
            int u = prev[v];
            if (v == T) { c[u - 1 - M]++; }
            else if (u >= 1 && u <= M && v > M) { f[(u - 1) * M + (v - 1 - M)] = 1; }
            else { f[(v - 1) * M + (u - 1 - M)] = 0; }   /* column -> row: undo */
            v = u;
        }
        r[v - 1]++;
    }
    double obj = 0.0;
    for (int e = 0; e < M * M; ++e) if (f[e]) obj += (double)a[e];
    return obj;
}

/* ------------------------------------------------------------------ */
/* Matrix-level entry points.                                          */

static void get_block(const float* W, int64_t cols, int M, int64_t br, int64_t bc, float* a) {
    for (int i = 0; i < M; ++i)
        for (int j = 0; j < M; ++j)
            a[i * M + j] = fabsf(W[(br * M + i) * cols + bc * M + j]);
}

static int block_finite(const float* a, int E) {
    for (int e = 0; e < E; ++e) if (!isfinite(a[e])) return 0;
    return 1;
}

/* Blocks are solved in parallel into a byte-per-entry matrix; words shared by
 * several blocks are only assembled afterwards, by one thread. */
static void put_bits(uint8_t* bits, int64_t cols, int M, int64_t br, int64_t bc, const uint8_t* s) {
    for (int i = 0; i < M; ++i)
        for (int j = 0; j < M; ++j)
            bits[(br * M + i) * cols + bc * M + j] = s[i * M + j];
}

static void pack_bits(const uint8_t* bits, int64_t rows, int64_t cols, uint32_t* mask) {
    const int64_t wpr = (cols + 31) / 32;
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t w = 0; w < wpr; ++w) {
            uint32_t word = 0;
            for (int k = 0; k < 32 && w * 32 + k < cols; ++k)
                if (bits[r * cols + w * 32 + k]) word |= (uint32_t)1 << k;
            mask[r * wpr + w] = word;
        }
    }
}

static int check_args(int64_t rows, int64_t cols, int N, int M) {
    if (rows < 0 || cols < 0 || M < 1 || M > 64 || N < 1 || N > M) return -1;
    if (rows % M || cols % M) return -2;
    return 0;
}

static void set_threads(int threads) {
#ifdef _OPENMP
    if (threads > 0) omp_set_num_threads(threads);
#else
    (void)threads;
#endif
}

int oracle_threads_used(int threads) {
#ifdef _OPENMP
    int n = 1;
    set_threads(threads);
#pragma omp parallel
    {
#pragma omp single
        n = omp_get_num_threads();
    }
    return n;
#else
    (void)threads;
    return 1;
#endif
}

/* Block-level entry points (used by the stage tests). */
int oracle_block_plan(const float* a, int N, int M, double tau, int iters, double* S_out) {
    if (check_args(M, M, N, M)) return -1;
    double* x = (double*)malloc(sizeof(double) * M * M);
    double* q = (double*)malloc(sizeof(double) * M * M);
    block_plan(a, N, M, tau, iters, x, q, S_out);
    free(x); free(q);
    return 0;
}

int oracle_block_round(const float* key, const float* a, int N, int M, int sweeps, int stage,
                       uint8_t* s, oracle_stats* st) {
    if (check_args(M, M, N, M)) return -1;
    int order[4096];
    oracle_stats local = {0, 0, 0, 0};
    int rc = block_round(key, a, N, M, sweeps, stage, s, order, &local);
    if (st) {
        st->repairs += local.repairs; st->ls_swaps += local.ls_swaps;
        st->short_after_greedy += local.short_after_greedy; st->failures += rc != 0;
    }
    return rc;
}

/* One block of block_plan_ext; returns the iterations run (or -1). */
int oracle_block_plan_ext(const float* a, int N, int M, double tau, int iters, double tol, int warm,
                          double* uv, double* S_out) {
    if (check_args(M, M, N, M) || !(tol >= 0.0)) return -1;
    double* x = (double*)malloc(sizeof(double) * M * M);
    double* q = (double*)malloc(sizeof(double) * M * M);
    int t = block_plan_ext(a, N, M, tau, iters, tol, warm, uv, x, q, S_out);
    free(x); free(q);
    return t;
}

double oracle_block_opt(const float* a, int N, int M, uint8_t* f) {
    if (check_args(M, M, N, M)) return NAN;
    return block_opt(a, N, M, f);
}

/* plan_out: rows*cols doubles, S of every block at its place in W. */
int oracle_plan(const float* W, int64_t rows, int64_t cols, int N, int M, double tau, int iters,
                double* plan_out, int threads) {
    int rc = check_args(rows, cols, N, M);
    if (rc) return rc;
    const int64_t nbr = rows / M, nbc = cols / M, nb = nbr * nbc;
    set_threads(threads);
#pragma omp parallel
    {
        float* a = (float*)malloc(sizeof(float) * M * M);
        double* x = (double*)malloc(sizeof(double) * M * M);
        double* q = (double*)malloc(sizeof(double) * M * M);
        double* S = (double*)malloc(sizeof(double) * M * M);
#pragma omp for schedule(dynamic, 8)
        for (int64_t b = 0; b < nb; ++b) {
            int64_t br = b / nbc, bc = b % nbc;
            get_block(W, cols, M, br, bc, a);
            block_plan(a, N, M, tau, iters, x, q, S);
            for (int i = 0; i < M; ++i)
                for (int j = 0; j < M; ++j)
                    plan_out[(br * M + i) * cols + bc * M + j] = S[i * M + j];
        }
        free(a); free(x); free(q); free(S);
    }
    return 0;
}

/* Rounding of a given fp32 plan (keys) for every block of W. */
int oracle_round(const float* key, const float* W, int64_t rows, int64_t cols, int N, int M,
                 int sweeps, uint32_t* mask, int threads, oracle_stats* st) {
    int rc = check_args(rows, cols, N, M);
    if (rc) return rc;
    const int64_t nbr = rows / M, nbc = cols / M, nb = nbr * nbc;
    int64_t rep = 0, sw = 0, fail = 0, shortg = 0;
    uint8_t* bits = (uint8_t*)malloc((size_t)(rows * cols > 0 ? rows * cols : 1));
    set_threads(threads);
#pragma omp parallel reduction(+:rep, sw, fail, shortg)
    {
        float* a = (float*)malloc(sizeof(float) * M * M);
        float* k = (float*)malloc(sizeof(float) * M * M);
        uint8_t* s = (uint8_t*)malloc((size_t)M * M);
        int* order = (int*)malloc(sizeof(int) * M * M);
#pragma omp for schedule(dynamic, 8)
        for (int64_t b = 0; b < nb; ++b) {
            int64_t br = b / nbc, bc = b % nbc;
            get_block(W, cols, M, br, bc, a);
            get_block(key, cols, M, br, bc, k);   /* keys are >= 0: fabsf is the identity */
            oracle_stats l = {0, 0, 0, 0};
            int ok = block_finite(a, M * M) && block_finite(k, M * M) &&
                     block_round(k, a, N, M, sweeps, 3, s, order, &l) == 0;
            if (!ok) { memset(s, 0, (size_t)M * M); fail++; }
            rep += l.repairs; sw += l.ls_swaps; shortg += l.short_after_greedy;
            put_bits(bits, cols, M, br, bc, s);
        }
        free(a); free(k); free(s); free(order);
    }
    pack_bits(bits, rows, cols, mask);
    free(bits);
    if (st) { st->repairs += rep; st->ls_swaps += sw; st->failures += fail; st->short_after_greedy += shortg; }
    return 0;
}

/* Full pipeline.  key_out (optional, rows*cols fp32) receives the sort keys. */
int oracle_mask(const float* W, int64_t rows, int64_t cols, int N, int M, double tau, int iters,
                int sweeps, uint32_t* mask, float* key_out, int threads, oracle_stats* st) {
    int rc = check_args(rows, cols, N, M);
    if (rc) return rc;
    const int64_t nbr = rows / M, nbc = cols / M, nb = nbr * nbc;
    int64_t rep = 0, sw = 0, fail = 0, shortg = 0;
    uint8_t* bits = (uint8_t*)malloc((size_t)(rows * cols > 0 ? rows * cols : 1));
    set_threads(threads);
#pragma omp parallel reduction(+:rep, sw, fail, shortg)
    {
        const int E = M * M;
        float* a = (float*)malloc(sizeof(float) * E);
        float* k = (float*)malloc(sizeof(float) * E);
        double* x = (double*)malloc(sizeof(double) * E);
        double* q = (double*)malloc(sizeof(double) * E);
        double* S = (double*)malloc(sizeof(double) * E);
        uint8_t* s = (uint8_t*)malloc((size_t)E);
        int* order = (int*)malloc(sizeof(int) * E);
#pragma omp for schedule(dynamic, 4)
        for (int64_t b = 0; b < nb; ++b) {
            int64_t br = b / nbc, bc = b % nbc;
            get_block(W, cols, M, br, bc, a);
            oracle_stats l = {0, 0, 0, 0};
            int ok = block_finite(a, E);
            if (ok) {
                block_plan(a, N, M, tau, iters, x, q, S);
                for (int e = 0; e < E; ++e) k[e] = (float)S[e];
                ok = block_round(k, a, N, M, sweeps, 3, s, order, &l) == 0;
            } else {
                for (int e = 0; e < E; ++e) k[e] = NAN;
            }
            if (!ok) { memset(s, 0, (size_t)E); fail++; }
            rep += l.repairs; sw += l.ls_swaps; shortg += l.short_after_greedy;
            put_bits(bits, cols, M, br, bc, s);
            if (key_out)
                for (int i = 0; i < M; ++i)
                    for (int j = 0; j < M; ++j)
                        key_out[(br * M + i) * cols + bc * M + j] = k[i * M + j];
        }
        free(a); free(k); free(x); free(q); free(S); free(s); free(order);
    }
    pack_bits(bits, rows, cols, mask);
    free(bits);
    if (st) { st->repairs += rep; st->ls_swaps += sw; st->failures += fail; st->short_after_greedy += shortg; }
    return 0;
}

/* Full pipeline with warm start and adaptive stopping (block_plan_ext).
 * uv: nb * 2M doubles, block b at 2M*b (U then V); read when warm, always
 * overwritten (NaN for a block with non-finite W).  used_out (optional): nb
 * ints, the iterations each block ran (0 for a non-finite block).
 * plan_out (optional): rows*cols doubles.  mask (optional): when NULL the
 * rounding is skipped. */
int oracle_solve_ext(const float* W, int64_t rows, int64_t cols, int N, int M, double tau, int iters,
                     int sweeps, double tol, int warm, double* uv, int* used_out, double* plan_out,
                     uint32_t* mask, int threads, oracle_stats* st) {
    int rc = check_args(rows, cols, N, M);
    if (rc) return rc;
    if (!(tol >= 0.0) || !uv) return -1;
    const int64_t nbr = rows / M, nbc = cols / M, nb = nbr * nbc;
    int64_t rep = 0, sw = 0, fail = 0, shortg = 0;
    uint8_t* bits = mask ? (uint8_t*)malloc((size_t)(rows * cols > 0 ? rows * cols : 1)) : NULL;
    set_threads(threads);
#pragma omp parallel reduction(+:rep, sw, fail, shortg)
    {
        const int E = M * M;
        float* a = (float*)malloc(sizeof(float) * E);
        float* k = (float*)malloc(sizeof(float) * E);
        double* x = (double*)malloc(sizeof(double) * E);
        double* q = (double*)malloc(sizeof(double) * E);
        double* S = (double*)malloc(sizeof(double) * E);
        uint8_t* s = (uint8_t*)malloc((size_t)E);
        int* order = (int*)malloc(sizeof(int) * E);
#pragma omp for schedule(dynamic, 4)
        for (int64_t b = 0; b < nb; ++b) {
            int64_t br = b / nbc, bc = b % nbc;
            double* buv = uv + 2 * M * b;
            get_block(W, cols, M, br, bc, a);
            oracle_stats l = {0, 0, 0, 0};
            int ok = block_finite(a, E);
            int used = 0;
            if (ok) {
                used = block_plan_ext(a, N, M, tau, iters, tol, warm, buv, x, q, S);
            } else {
                for (int e = 0; e < 2 * M; ++e) buv[e] = NAN;
                for (int e = 0; e < E; ++e) S[e] = NAN;
            }
            if (used_out) used_out[b] = used;
            if (plan_out)
                for (int i = 0; i < M; ++i)
                    for (int j = 0; j < M; ++j)
                        plan_out[(br * M + i) * cols + bc * M + j] = S[i * M + j];
            if (bits) {
                if (ok) {
                    for (int e = 0; e < E; ++e) k[e] = (float)S[e];
                    ok = block_round(k, a, N, M, sweeps, 3, s, order, &l) == 0;
                }
                if (!ok) { memset(s, 0, (size_t)E); fail++; }
                put_bits(bits, cols, M, br, bc, s);
            } else if (!ok) {
                fail++;
            }
            rep += l.repairs; sw += l.ls_swaps; shortg += l.short_after_greedy;
        }
        free(a); free(k); free(x); free(q); free(S); free(s); free(order);
    }
    if (bits) { pack_bits(bits, rows, cols, mask); free(bits); }
    if (st) { st->repairs += rep; st->ls_swaps += sw; st->failures += fail; st->short_after_greedy += shortg; }
    return 0;
}

/* Kept sum_ij |W_ij| s_ij per block in fp64; NaN when a row or column of the
 * block does not hold exactly N ones. */
int oracle_objective(const float* W, const uint32_t* mask, int64_t rows, int64_t cols, int N, int M,
                     double* out) {
    int rc = check_args(rows, cols, N, M);
    if (rc) return rc;
    const int64_t nbr = rows / M, nbc = cols / M, wpr = (cols + 31) / 32;
    for (int64_t br = 0; br < nbr; ++br) {
        for (int64_t bc = 0; bc < nbc; ++bc) {
            double obj = 0.0;
            int valid = 1;
            int cc[64];
            for (int j = 0; j < M; ++j) cc[j] = 0;
            for (int i = 0; i < M; ++i) {
                int rcnt = 0;
                for (int j = 0; j < M; ++j) {
                    int64_t row = br * M + i, col = bc * M + j;
                    if ((mask[row * wpr + col / 32] >> (col % 32)) & 1u) {
                        obj += (double)fabsf(W[row * cols + col]);
                        rcnt++; cc[j]++;
                    }
                }
                if (rcnt != N) valid = 0;
            }
            for (int j = 0; j < M; ++j) if (cc[j] != N) valid = 0;
            out[br * nbc + bc] = valid ? obj : NAN;
        }
    }
    return 0;
}

/* Exact per-block optimum.  mask_out (optional) receives an optimal mask. */
int oracle_opt(const float* W, int64_t rows, int64_t cols, int N, int M, double* opt_out,
               uint32_t* mask_out, int threads) {
    int rc = check_args(rows, cols, N, M);
    if (rc) return rc;
    const int64_t nbr = rows / M, nbc = cols / M, nb = nbr * nbc;
    uint8_t* bits = mask_out ? (uint8_t*)malloc((size_t)(rows * cols > 0 ? rows * cols : 1)) : NULL;
    set_threads(threads);
#pragma omp parallel
    {
        float* a = (float*)malloc(sizeof(float) * M * M);
        uint8_t* f = (uint8_t*)malloc((size_t)M * M);
#pragma omp for schedule(dynamic, 4)
        for (int64_t b = 0; b < nb; ++b) {
            int64_t br = b / nbc, bc = b % nbc;
            get_block(W, cols, M, br, bc, a);
            opt_out[b] = block_finite(a, M * M) ? block_opt(a, N, M, f) : NAN;
            if (bits) put_bits(bits, cols, M, br, bc, f);
        }
        free(a); free(f);
    }
    if (bits) { pack_bits(bits, rows, cols, mask_out); free(bits); }
    return 0;
}

/* ------------------------------------------------------------------ */
/* Monotonicity safeguard ("Assumptions & free parameters", Assumption 1 of
 * Theorem 1; referee comment 2): per block, keep the previous mask when it is
 * a valid N:M block whose kept mass exceeds the new mask's.  Kept mass is
 * summed in fp64 over the block in row-major order.  out may alias new_mask.
 * Returns the number of blocks that kept the previous mask. */
static double block_mass(const float* W, const uint32_t* mask, int64_t cols, int M, int64_t br, int64_t bc,
                         int N, int* valid) {
    const int64_t wpr = (cols + 31) / 32;
    double obj = 0.0;
    int cc[64];
    for (int j = 0; j < M; ++j) cc[j] = 0;
    *valid = 1;
    for (int i = 0; i < M; ++i) {
        int rcnt = 0;
        for (int j = 0; j < M; ++j) {
            const int64_t row = br * M + i, col = bc * M + j;
            if ((mask[row * wpr + col / 32] >> (col % 32)) & 1u) {
                obj += (double)fabsf(W[row * cols + col]);
                rcnt++; cc[j]++;
            }
        }
        if (rcnt != N) *valid = 0;
    }
    for (int j = 0; j < M; ++j) if (cc[j] != N) *valid = 0;
    return obj;
}

int64_t oracle_safeguard(const float* W, const uint32_t* prev_mask, const uint32_t* new_mask, int64_t rows,
                         int64_t cols, int N, int M, uint32_t* out) {
    if (check_args(rows, cols, N, M)) return -1;
    const int64_t nbr = rows / M, nbc = cols / M, wpr = (cols + 31) / 32;
    if (out != new_mask) memcpy(out, new_mask, sizeof(uint32_t) * (size_t)(rows * wpr));
    int64_t kept = 0;
    for (int64_t br = 0; br < nbr; ++br)
        for (int64_t bc = 0; bc < nbc; ++bc) {
            int vp = 0, vn = 0;
            const double op = block_mass(W, prev_mask, cols, M, br, bc, N, &vp);
            const double on = block_mass(W, new_mask, cols, M, br, bc, N, &vn);
            if (vp && op > on) {
                kept++;
                for (int i = 0; i < M; ++i)
                    for (int j = 0; j < M; ++j) {
                        const int64_t row = br * M + i, col = bc * M + j;
                        const uint32_t bit = 1u << (col % 32);
                        uint32_t* w = out + row * wpr + col / 32;
                        if ((prev_mask[row * wpr + col / 32] >> (col % 32)) & 1u) *w |= bit; else *w &= ~bit;
                    }
            }
        }
    return kept;
}

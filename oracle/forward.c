/*
 * Oracle: explicit edgewise evaluation of the equivariant message-passing
 * convolution in float64 (test infrastructure only; never on a product path).
 *
 * Follows e3j.core.Convolution (page "e3j.core.Convolution", class docstring:
 * the formula m_b = (1/N) sum_a (x_a (x) y_ab) . s_ab and the four plain
 * steps gather / tensor product / scalar mix / scatter-add, then the division
 * by avg_num_neighbors), with the channelwise ("uvu") tensor product of the
 * cuEquivariance-JAX notes (section "Dense polynomial: broadcasting, JIT, and
 * a gradient": per-channel product with weights first) and their advice to
 * check message passing against an explicit edgewise summation
 * (section "Dense polynomial", last paragraph).
 *
 * For every receiver b and every edge e with receivers[e] == b:
 *   out[b, ooff_p + k, u] += s[e, p, u] * CG_p[i, j, k]
 *                            * x[senders[e], xoff_p + i, u] * Y[e, yoff_p + j]
 * summed over paths p, channels u and the dense (i, j, k) box of every path
 * (zeros included: nothing depends on which coefficients are nonzero), and
 * finally out[b] *= inv_avg.  Loop order: edge -> path -> channel -> i, j, k.
 *
 * Returns 0, or -1 if a sender / receiver index is out of range.
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

int oracle_forward(int64_t num_nodes, int64_t num_edges, int C, int nx, int ny, int P, int nout,
                   const double* x, const double* Y, const double* s,
                   const int64_t* senders, const int64_t* receivers,
                   const int* l1, const int* xoff, const int* l2, const int* yoff,
                   const int* l3, const int* ooff, const double* cg, const int64_t* cg_off,
                   double inv_avg, double* out, int num_threads)
{
    for (int64_t e = 0; e < num_edges; ++e) {
        if (senders[e] < 0 || senders[e] >= num_nodes) return -1;
        if (receivers[e] < 0 || receivers[e] >= num_nodes) return -1;
    }
    /* edges of each receiver, in their original order (plain counting sort) */
    int64_t* start = (int64_t*)calloc((size_t)num_nodes + 1, sizeof(int64_t));
    int64_t* order = (int64_t*)malloc(sizeof(int64_t) * (size_t)(num_edges > 0 ? num_edges : 1));
    int64_t* fill = (int64_t*)malloc(sizeof(int64_t) * (size_t)(num_nodes > 0 ? num_nodes : 1));
    if (!start || !order || !fill) { free(start); free(order); free(fill); return -2; }
    for (int64_t e = 0; e < num_edges; ++e) start[receivers[e] + 1]++;
    for (int64_t b = 0; b < num_nodes; ++b) start[b + 1] += start[b];
    for (int64_t b = 0; b < num_nodes; ++b) fill[b] = start[b];
    for (int64_t e = 0; e < num_edges; ++e) order[fill[receivers[e]]++] = e;
    free(fill);

#ifdef _OPENMP
    if (num_threads > 0) omp_set_num_threads(num_threads);
#else
    (void)num_threads;
#endif

#pragma omp parallel for schedule(dynamic, 16)
    for (int64_t b = 0; b < num_nodes; ++b) {
        double* acc = out + (size_t)b * nout * C;
        memset(acc, 0, sizeof(double) * (size_t)nout * C);
        for (int64_t t = start[b]; t < start[b + 1]; ++t) {
            const int64_t e = order[t];
            const int64_t a = senders[e];
            for (int p = 0; p < P; ++p) {
                const int d1 = 2 * l1[p] + 1, d2 = 2 * l2[p] + 1, d3 = 2 * l3[p] + 1;
                const double* w = cg + cg_off[p];
                for (int u = 0; u < C; ++u) {
                    const double sv = s[((size_t)e * P + p) * C + u];
                    for (int i = 0; i < d1; ++i) {
                        const double xv = x[((size_t)a * nx + xoff[p] + i) * C + u];
                        for (int j = 0; j < d2; ++j) {
                            const double yv = Y[(size_t)e * ny + yoff[p] + j];
                            for (int k = 0; k < d3; ++k)
                                acc[(size_t)(ooff[p] + k) * C + u] +=
                                    sv * w[(i * d2 + j) * d3 + k] * xv * yv;
                        }
                    }
                }
            }
        }
        for (size_t q = 0; q < (size_t)nout * C; ++q) acc[q] *= inv_avg;
    }
    free(start);
    free(order);
    return 0;
}

int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * Oracle: explicit edgewise gradients of the equivariant message-passing
 * convolution in float64 (test infrastructure only; never on a product path).
 *
 * The forward (page "e3j.core.Convolution", class docstring) is
 *   out[b, ooff_p + k, u] = inv_avg * sum_{e: receivers[e] = b} sum_p sum_{i,j}
 *        s[e, p, u] * CG_p[i, j, k] * x[senders[e], xoff_p + i, u] * Y[e, yoff_p + j]
 * which is linear in each of x, Y and s.  For an upstream gradient g of out,
 * the chain rule gives, edge by edge, the same four-factor products with one
 * factor removed:
 *   gx[a, xoff_p + i, u] += inv_avg g[b, ooff_p + k, u] s[e,p,u] CG_p[i,j,k] Y[e, yoff_p + j]
 *   gY[e, yoff_p + j]    += inv_avg g[b, ooff_p + k, u] s[e,p,u] CG_p[i,j,k] x[a, xoff_p + i, u]
 *   gs[e, p, u]          += inv_avg g[b, ooff_p + k, u] CG_p[i,j,k] x[a, xoff_p + i, u] Y[e, yoff_p + j]
 * with a = senders[e], b = receivers[e], over all edges, paths, channels and
 * the dense (i, j, k) box (zeros included).  Loop order: edge -> path ->
 * channel -> i, j, k; single-threaded (the gx sums over senders are not
 * partitioned by receiver).
 *
 * Returns 0, or -1 if a sender / receiver index is out of range.
 */
#include <stdint.h>
#include <string.h>

int oracle_backward(int64_t num_nodes, int64_t num_edges, int C, int nx, int ny, int P, int nout,
                    const double* x, const double* Y, const double* s,
                    const int64_t* senders, const int64_t* receivers,
                    const int* l1, const int* xoff, const int* l2, const int* yoff,
                    const int* l3, const int* ooff, const double* cg, const int64_t* cg_off,
                    double inv_avg, const double* g, double* gx, double* gY, double* gs)
{
    for (int64_t e = 0; e < num_edges; ++e) {
        if (senders[e] < 0 || senders[e] >= num_nodes) return -1;
        if (receivers[e] < 0 || receivers[e] >= num_nodes) return -1;
    }
    memset(gx, 0, sizeof(double) * (size_t)num_nodes * nx * C);
    memset(gY, 0, sizeof(double) * (size_t)num_edges * ny);
    memset(gs, 0, sizeof(double) * (size_t)num_edges * P * C);
    for (int64_t e = 0; e < num_edges; ++e) {
        const int64_t a = senders[e], b = receivers[e];
        for (int p = 0; p < P; ++p) {
            const int d1 = 2 * l1[p] + 1, d2 = 2 * l2[p] + 1, d3 = 2 * l3[p] + 1;
            const double* w = cg + cg_off[p];
            for (int u = 0; u < C; ++u) {
                const double sv = s[((size_t)e * P + p) * C + u];
                for (int i = 0; i < d1; ++i) {
                    const double xv = x[((size_t)a * nx + xoff[p] + i) * C + u];
                    for (int j = 0; j < d2; ++j) {
                        const double yv = Y[(size_t)e * ny + yoff[p] + j];
                        for (int k = 0; k < d3; ++k) {
                            const double gv = inv_avg * g[((size_t)b * nout + ooff[p] + k) * C + u];
                            const double c = w[(i * d2 + j) * d3 + k];
                            gx[((size_t)a * nx + xoff[p] + i) * C + u] += gv * sv * c * yv;
                            gY[(size_t)e * ny + yoff[p] + j] += gv * sv * c * xv;
                            gs[((size_t)e * P + p) * C + u] += gv * c * xv * yv;
                        }
                    }
                }
            }
        }
    }
    return 0;
}

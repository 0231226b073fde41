/*
 * Plain-C loop oracle (O3) for the Mixtral top-2 sparse-MoE SwiGLU layer.
 *
 * TEST INFRASTRUCTURE ONLY: built by oracle/build_oracle.py and called from the
 * tests through ctypes.  It is not linked into, and shares nothing with, the CUDA
 * library.  Everything is evaluated per token with explicit loops in double
 * precision, with no sorting, grouping or permutation, so that it checks the
 * routed NumPy oracle by a different route.
 *
 * Per token t (crackai "Mixtral of Experts", "Top-2 Routing in Detail"; notion
 * notes "Mixtral of Experts", "Sparse gating" eq. G(x) and "Implementation" eq. y):
 *   l[e]  = sum_i x[t,i] * Wg[i,e]
 *   i1    = first index of the largest logit, i2 = first index of the largest
 *           of the rest (ties go to the lower index)
 *   w1    = 1 / (1 + exp(l[i2] - l[i1])),  w2 = 1 / (1 + exp(l[i1] - l[i2]))
 *   E_e   : a_j = sum_i W1[e,j,i] x[t,i],  b_j = sum_i W3[e,j,i] x[t,i],
 *           g_j = a_j / (1 + exp(-a_j)) * b_j,  out_c = sum_j W2[e,c,j] g_j
 *   y[t]  = w1 * E_{i1} + w2 * E_{i2}
 * Layouts: x[T,d], Wg[d,E], W1/W3[E,h,d], W2[E,d,h], all row-major doubles.
 * Returns 0, or -1 on a bad argument (E < 2, non-positive sizes).
 */
#include <math.h>
#include <stdlib.h>

int moe_oracle_loops(const double *x, const double *Wg, const double *W1,
                     const double *W3, const double *W2, int T, int d, int h,
                     int E, int *idx, double *w, double *y) {
    if (T < 0 || d <= 0 || h <= 0 || E < 2) return -1;
    double *l = (double *)malloc(sizeof(double) * (size_t)E);
    double *g = (double *)malloc(sizeof(double) * (size_t)h);
    if (!l || !g) { free(l); free(g); return -1; }
    for (int t = 0; t < T; ++t) {
        const double *xt = x + (size_t)t * d;
        for (int e = 0; e < E; ++e) {
            double s = 0.0;
            for (int i = 0; i < d; ++i) s += xt[i] * Wg[(size_t)i * E + e];
            l[e] = s;
        }
        int i1 = 0;
        for (int e = 1; e < E; ++e)
            if (l[e] > l[i1]) i1 = e;
        int i2 = (i1 == 0) ? 1 : 0;
        for (int e = 0; e < E; ++e)
            if (e != i1 && l[e] > l[i2]) i2 = e;
        double w1 = 1.0 / (1.0 + exp(l[i2] - l[i1]));
        double w2 = 1.0 / (1.0 + exp(l[i1] - l[i2]));
        idx[2 * t] = i1;
        idx[2 * t + 1] = i2;
        w[2 * t] = w1;
        w[2 * t + 1] = w2;
        double *yt = y + (size_t)t * d;
        for (int c = 0; c < d; ++c) yt[c] = 0.0;
        for (int s = 0; s < 2; ++s) {
            int e = (s == 0) ? i1 : i2;
            double we = (s == 0) ? w1 : w2;
            const double *w1e = W1 + (size_t)e * h * d;
            const double *w3e = W3 + (size_t)e * h * d;
            const double *w2e = W2 + (size_t)e * d * h;
            for (int j = 0; j < h; ++j) {
                double a = 0.0, b = 0.0;
                for (int i = 0; i < d; ++i) {
                    a += w1e[(size_t)j * d + i] * xt[i];
                    b += w3e[(size_t)j * d + i] * xt[i];
                }
                g[j] = a / (1.0 + exp(-a)) * b;
            }
            for (int c = 0; c < d; ++c) {
                double o = 0.0;
                for (int j = 0; j < h; ++j) o += w2e[(size_t)c * h + j] * g[j];
                yt[c] += we * o;
            }
        }
    }
    free(l);
    free(g);
    return 0;
}

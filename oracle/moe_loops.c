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

/*
 * Backward of the same layer (O3), per token with explicit loops, no grouping.
 * The pages print no gradient (crackai "Mixtral of Experts", "Key Takeaways", only
 * says the router is learned jointly with the experts); this is the exact
 * derivative of y with the top-2 choice held fixed, written from the chain rule:
 * for token t, slot s with expert e and weight w_s, and upstream gradient dy[t],
 *   Y_c   = sum_j W2[e,c,j] H_j,             H_j = silu(a_j) b_j
 *   dw_s  = sum_c dy_c Y_c                   (y = sum_s w_s Y^(s))
 *   dW2[e,c,j] += w_s dy_c H_j
 *   dH_j  = sum_c w_s dy_c W2[e,c,j]
 *   da_j  = dH_j b_j silu'(a_j),  silu'(a) = sig(a) (1 + a (1 - sig(a)))
 *   db_j  = dH_j silu(a_j)
 *   dW1[e,j,i] += da_j x_i,  dW3[e,j,i] += db_j x_i
 *   dx_i += sum_j (da_j W1[e,j,i] + db_j W3[e,j,i])
 * and for the gate, w1 = sig(l_i1 - l_i2), w2 = 1 - w1:
 *   g = (dw_1 - dw_2) w1 w2,  dlogit[i1] = g,  dlogit[i2] = -g
 *   dWg[i,e] += x_i dlogit[e],  dx_i += sum_e dlogit[e] Wg[i,e].
 * Outputs (dx[T,d], dWg[d,E], dW1/dW3[E,h,d], dW2[E,d,h]) are overwritten.
 * Returns 0, or -1 on a bad argument or a failed allocation.
 */
int moe_oracle_loops_backward(const double *x, const double *Wg, const double *W1,
                              const double *W3, const double *W2, const double *dy,
                              int T, int d, int h, int E, double *dx, double *dWg,
                              double *dW1, double *dW3, double *dW2) {
    if (T < 0 || d <= 0 || h <= 0 || E < 2) return -1;
    double *l = (double *)malloc(sizeof(double) * (size_t)E);
    double *a = (double *)malloc(sizeof(double) * (size_t)h);
    double *b = (double *)malloc(sizeof(double) * (size_t)h);
    double *hh = (double *)malloc(sizeof(double) * (size_t)h);
    double *dh = (double *)malloc(sizeof(double) * (size_t)h);
    if (!l || !a || !b || !hh || !dh) {
        free(l); free(a); free(b); free(hh); free(dh);
        return -1;
    }
    for (size_t i = 0; i < (size_t)T * d; ++i) dx[i] = 0.0;
    for (size_t i = 0; i < (size_t)d * E; ++i) dWg[i] = 0.0;
    for (size_t i = 0; i < (size_t)E * h * d; ++i) dW1[i] = dW3[i] = dW2[i] = 0.0;
    for (int t = 0; t < T; ++t) {
        const double *xt = x + (size_t)t * d;
        const double *gt = dy + (size_t)t * d;
        double *dxt = dx + (size_t)t * d;
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
        const double w1 = 1.0 / (1.0 + exp(l[i2] - l[i1]));
        const double w2 = 1.0 / (1.0 + exp(l[i1] - l[i2]));
        double dw[2];
        for (int s = 0; s < 2; ++s) {
            const int e = (s == 0) ? i1 : i2;
            const double ws = (s == 0) ? w1 : w2;
            const double *w1e = W1 + (size_t)e * h * d;
            const double *w3e = W3 + (size_t)e * h * d;
            const double *w2e = W2 + (size_t)e * d * h;
            for (int j = 0; j < h; ++j) {
                double aj = 0.0, bj = 0.0;
                for (int i = 0; i < d; ++i) {
                    aj += w1e[(size_t)j * d + i] * xt[i];
                    bj += w3e[(size_t)j * d + i] * xt[i];
                }
                a[j] = aj;
                b[j] = bj;
                hh[j] = aj / (1.0 + exp(-aj)) * bj;
                dh[j] = 0.0;
            }
            double dws = 0.0;
            for (int c = 0; c < d; ++c) {
                double yc = 0.0;
                for (int j = 0; j < h; ++j) yc += w2e[(size_t)c * h + j] * hh[j];
                dws += gt[c] * yc;
                const double dyc = ws * gt[c];
                double *dw2row = dW2 + ((size_t)e * d + c) * h;
                for (int j = 0; j < h; ++j) {
                    dw2row[j] += dyc * hh[j];
                    dh[j] += dyc * w2e[(size_t)c * h + j];
                }
            }
            dw[s] = dws;
            for (int j = 0; j < h; ++j) {
                const double sig = 1.0 / (1.0 + exp(-a[j]));
                const double da = dh[j] * b[j] * sig * (1.0 + a[j] * (1.0 - sig));
                const double db = dh[j] * a[j] * sig;
                double *dw1row = dW1 + ((size_t)e * h + j) * d;
                double *dw3row = dW3 + ((size_t)e * h + j) * d;
                for (int i = 0; i < d; ++i) {
                    dw1row[i] += da * xt[i];
                    dw3row[i] += db * xt[i];
                    dxt[i] += da * w1e[(size_t)j * d + i] + db * w3e[(size_t)j * d + i];
                }
            }
        }
        const double g = (dw[0] - dw[1]) * w1 * w2;
        for (int i = 0; i < d; ++i) {
            dWg[(size_t)i * E + i1] += xt[i] * g;
            dWg[(size_t)i * E + i2] -= xt[i] * g;
            dxt[i] += g * Wg[(size_t)i * E + i1] - g * Wg[(size_t)i * E + i2];
        }
    }
    free(l); free(a); free(b); free(hh); free(dh);
    return 0;
}

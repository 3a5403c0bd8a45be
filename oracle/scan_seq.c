/*
 * Plain sequential fp64 selective scan (oracle; test infrastructure only).
 *
 * Same computation as selective_scan() in mamba.py, as a C loop so that
 * sequences of 10^5 steps finish in seconds on the CPU:
 *   h[c][n] <- exp(dt[t][c] * A[c][n]) * h[c][n] + dt[t][c] * B[t][n] * x[t][c]
 *   y[t][c]  = (sum_n C[t][n] * h[c][n] + D[c] * x[t][c]) * (z ? SiLU(z[t][c]) : 1)
 * Layouts (row-major, float64): x, dt, z, y [batch][L][C]; B, Cm [batch][L][N];
 * A [C][N]; D [C]; h0, h_last [batch][C][N] (h0 may be NULL for zeros).
 * Batch rows are independent; everything else runs in natural order.
 */
#include <math.h>
#include <stddef.h>
#include <stdlib.h>
#include <string.h>

void oracle_selective_scan(const double *x, const double *dt, const double *A,
                           const double *B, const double *Cm, const double *D,
                           const double *z, const double *h0, double *y,
                           double *h_last, long nbatch, long L, long C, long N)
{
    double *h = (double *)malloc(sizeof(double) * (size_t)(C * N));
    for (long b = 0; b < nbatch; ++b) {
        if (h0)
            memcpy(h, h0 + b * C * N, sizeof(double) * (size_t)(C * N));
        else
            memset(h, 0, sizeof(double) * (size_t)(C * N));
        for (long t = 0; t < L; ++t) {
            const double *xt = x + (b * L + t) * C;
            const double *dtt = dt + (b * L + t) * C;
            const double *Bt = B + (b * L + t) * N;
            const double *Ct = Cm + (b * L + t) * N;
            double *yt = y + (b * L + t) * C;
            for (long c = 0; c < C; ++c) {
                double acc = 0.0;
                for (long n = 0; n < N; ++n) {
                    double *hc = h + c * N + n;
                    *hc = exp(dtt[c] * A[c * N + n]) * (*hc) + dtt[c] * Bt[n] * xt[c];
                    acc += Ct[n] * (*hc);
                }
                double out = acc + D[c] * xt[c];
                if (z) {
                    double zz = z[(b * L + t) * C + c];
                    out *= zz / (1.0 + exp(-zz));
                }
                yt[c] = out;
            }
        }
        memcpy(h_last + b * C * N, h, sizeof(double) * (size_t)(C * N));
    }
    free(h);
}

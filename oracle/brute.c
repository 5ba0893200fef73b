/* Brute-force exact attention in plain C -- TEST INFRASTRUCTURE ONLY.
 *
 * A second, independent oracle for tiny shapes: triple loops, long double
 * accumulation, no BLAS, no blocking.  It follows the definition on page
 * "attention 的显存线性化" §一 (O = softmax(Q K^T / sqrt(d_k)) V) with the
 * max-subtracted row softmax of page "注意力计算的计算与显存瓶颈" §1.1.8, and the
 * exact gradient of sum(O * dO) for the backward (the pages only say the
 * backward recomputes local blocks; the formulas are the chain rule).
 *
 * Layout: q, o, dO, dq are [B][Hq][N][d]; k, v, dk, dv are [B][Hkv][N][d];
 * lse is [B][Hq][N]; all double, row-major.  Causal: query i sees keys j <= i.
 * Local window (page "attn-efficient", sliding-window row of the family table):
 * query i sees keys j with i - wl <= j <= i + wr; wl or wr < 0 means no limit on
 * that side; intersected with the causal rule when causal != 0.
 * q-head h reads kv-head h / (Hq / Hkv).
 */
#include <math.h>
#include <stdlib.h>

static long double score(const double* qi, const double* kj, int d, long double scale) {
    long double s = 0.0L;
    for (int c = 0; c < d; ++c) s += (long double)qi[c] * (long double)kj[c];
    return scale * s;
}

static int sees(int i, int j, int causal, int wl, int wr) {
    if (causal && j > i) return 0;
    if (wl >= 0 && j < i - wl) return 0;
    if (wr >= 0 && j > i + wr) return 0;
    return 1;
}

/* Fills p[0..N) with the softmax row of query i (masked keys get 0); returns LSE. */
static long double prob_row(const double* q, const double* k, int N, int d, int i,
                            long double scale, int causal, int wl, int wr, long double* p) {
    long double m = -INFINITY;
    for (int j = 0; j < N; ++j) {
        if (!sees(i, j, causal, wl, wr)) continue;
        p[j] = score(q + (size_t)i * d, k + (size_t)j * d, d, scale);
        if (p[j] > m) m = p[j];
    }
    long double l = 0.0L;
    for (int j = 0; j < N; ++j) {
        if (!sees(i, j, causal, wl, wr)) continue;
        p[j] = expl(p[j] - m);
        l += p[j];
    }
    for (int j = 0; j < N; ++j) p[j] = sees(i, j, causal, wl, wr) ? p[j] / l : 0.0L;
    return m + logl(l);
}

int brute_fwd(const double* q, const double* k, const double* v, double* o, double* lse,
              int B, int Hq, int Hkv, int N, int d, double scale, int causal, int wl, int wr) {
    if (B < 1 || Hq < 1 || Hkv < 1 || N < 1 || d < 1 || Hq % Hkv) return -1;
    int G = Hq / Hkv;
    long double* p = (long double*)malloc(sizeof(long double) * (size_t)N);
    if (!p) return -2;
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < Hq; ++h) {
            size_t qoff = ((size_t)b * Hq + h) * N * d;
            size_t koff = ((size_t)b * Hkv + h / G) * N * d;
            for (int i = 0; i < N; ++i) {
                lse[((size_t)b * Hq + h) * N + i] =
                    (double)prob_row(q + qoff, k + koff, N, d, i, scale, causal, wl, wr, p);
                for (int c = 0; c < d; ++c) {
                    long double acc = 0.0L;
                    for (int j = 0; j < N; ++j) acc += p[j] * (long double)v[koff + (size_t)j * d + c];
                    o[qoff + (size_t)i * d + c] = (double)acc;
                }
            }
        }
    free(p);
    return 0;
}

int brute_bwd(const double* q, const double* k, const double* v, const double* dO,
              double* dq, double* dk, double* dv,
              int B, int Hq, int Hkv, int N, int d, double scale, int causal, int wl, int wr) {
    if (B < 1 || Hq < 1 || Hkv < 1 || N < 1 || d < 1 || Hq % Hkv) return -1;
    int G = Hq / Hkv;
    long double* p = (long double*)malloc(sizeof(long double) * (size_t)N);
    long double* ds = (long double*)malloc(sizeof(long double) * (size_t)N);
    long double* dka = (long double*)calloc((size_t)B * Hkv * N * d, sizeof(long double));
    long double* dva = (long double*)calloc((size_t)B * Hkv * N * d, sizeof(long double));
    if (!p || !ds || !dka || !dva) { free(p); free(ds); free(dka); free(dva); return -2; }
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < Hq; ++h) {
            size_t qoff = ((size_t)b * Hq + h) * N * d;
            size_t koff = ((size_t)b * Hkv + h / G) * N * d;
            for (int i = 0; i < N; ++i) {
                const double* doi = dO + qoff + (size_t)i * d;
                prob_row(q + qoff, k + koff, N, d, i, scale, causal, wl, wr, p);
                /* D_i = sum_c dO_ic O_ic with O_i = sum_j p_j V_j */
                long double D = 0.0L;
                for (int c = 0; c < d; ++c) {
                    long double oc = 0.0L;
                    for (int j = 0; j < N; ++j) oc += p[j] * (long double)v[koff + (size_t)j * d + c];
                    D += (long double)doi[c] * oc;
                }
                for (int j = 0; j < N; ++j) {
                    long double dp = 0.0L;   /* dP_ij = dO_i . V_j */
                    for (int c = 0; c < d; ++c) dp += (long double)doi[c] * (long double)v[koff + (size_t)j * d + c];
                    ds[j] = p[j] * (dp - D);
                }
                for (int c = 0; c < d; ++c) {
                    long double acc = 0.0L;
                    for (int j = 0; j < N; ++j) acc += ds[j] * (long double)k[koff + (size_t)j * d + c];
                    dq[qoff + (size_t)i * d + c] = (double)(scale * acc);
                }
                for (int j = 0; j < N; ++j)
                    for (int c = 0; c < d; ++c) {
                        dka[koff + (size_t)j * d + c] += scale * ds[j] * (long double)q[qoff + (size_t)i * d + c];
                        dva[koff + (size_t)j * d + c] += p[j] * (long double)doi[c];
                    }
            }
        }
    for (size_t x = 0; x < (size_t)B * Hkv * N * d; ++x) { dk[x] = (double)dka[x]; dv[x] = (double)dva[x]; }
    free(p); free(ds); free(dka); free(dva);
    return 0;
}

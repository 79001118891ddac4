/*
 * Mamba-3 SSM core: plain sequential fp64 CPU oracle.
 *
 * TEST INFRASTRUCTURE. Only the tests, the smoke check and the benchmark's CPU-baseline
 * leg may load this library. The product path never calls it.
 *
 * What it computes, per (batch b, head h) unit, one token at a time (no chunking,
 * no re-association):
 *
 *   Bn  = RMSNorm_N(B_raw) + bias_B[h]      (norm optional; bias added after the norm:
 *   Cn  = RMSNorm_N(C_raw) + bias_C[h]       "Mamba-3: Improved Sequence Modeling using
 *                                             State Space Principles", Sec. 3.4, BC norm
 *                                             and B,C bias)
 *   alpha = exp(dt*A), beta = (1-lam)*dt*alpha, gamma = lam*dt      (Sec. 3.1.1, Prop. 1)
 *   (zero-order hold instead, when asked: beta = 0, gamma = (alpha - 1)/A, lam unused:
 *    "Mamba-3：推理优先的状态空间模型", Sec. 1.2; the rotation is unchanged)
 *   Phi  += dt*theta                     cumulative angle of the rotations R_0..R_t
 *                                        (Sec. 3.2.1, Prop. 2: R_t = Block{R(dt_t*theta_t[i])})
 *   Bbar  = R(Phi)^T Bn, Cbar = R(Phi)^T Cn, Bpbar = R(Phi_prev)^T Bpn
 *                                        (Sec. 3.2.2, Prop. 4, the "RoPE trick")
 *   h     = alpha*h + beta * sum_r Bpbar[r] xp[r]^T + gamma * sum_r Bbar[r] x[r]^T
 *   y[r]  = h^T Cbar[r]                  (Prop. 4 for the three-term update; Appendix C
 *                                        for the rank-R MIMO state update H = aH + B X^T and
 *                                        output Y = H^T C; Remark 6 for combining the two)
 *   Bp = B_raw, xp = x                   (the previous token's inputs, kept raw)
 *
 * Pairing: the complex state of dimension N/2 is stored as [Re; Im] halves, so pair i is
 * (i, i + N/2) (Prop. 2: B = [B; B_hat]). R(phi)^T maps (u, v) to
 * (u cos phi + v sin phi, -u sin phi + v cos phi).
 *
 * The state is kept in the rotated frame h~ of Appendix B.3, together with the cumulative
 * angle Phi and the previous token's raw B and x, which the trapezoid's beta term needs.
 * A fresh sequence starts from an all-zero state: h_{-1} = 0 and x_{-1} = 0, so the first
 * step is h_0 = gamma_0 B_0 x_0 (Sec. 3.1.3).
 *
 * Layouts (row-major, contiguous):
 *   x      [b, L, H, R, P]     B, C  [b, L, G, R, N]    theta [b, L, H, N/2]
 *   dt, A, lam [b, L, H]       bias_B, bias_C [H, R, N] (NULL = 0)
 *   h [b, H, N, P]  phi [b, H, N/2]  prev_B [b, H, R, N]  prev_x [b, H, R, P]  (in/out)
 *   y [b, L, H, R, P]
 * Head h reads B/C group g = h / (H / G).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct {
    int64_t batch, seqlen, nheads, ngroups, headdim, dstate, rank;
    int32_t bc_norm;
    double norm_eps;
    int32_t zoh; /* nonzero: zero-order-hold weights */
} m3o_dims;

/* RMS normalisation over the N entries of v (no learnable weight), then add bias. */
static void norm_bias(const double* v, const double* bias, int64_t n, int norm, double eps,
                      double* out) {
    double scale = 1.0;
    if (norm) {
        double ss = 0.0;
        for (int64_t i = 0; i < n; ++i) ss += v[i] * v[i];
        scale = 1.0 / sqrt(ss / (double)n + eps);
    }
    for (int64_t i = 0; i < n; ++i) out[i] = v[i] * scale + (bias ? bias[i] : 0.0);
}

/* out = R(phi)^T v, pair i = (i, i + N/2). */
static void rotate_T(const double* v, const double* phi, int64_t n, double* out) {
    int64_t half = n / 2;
    for (int64_t i = 0; i < half; ++i) {
        double c = cos(phi[i]), s = sin(phi[i]);
        double u = v[i], w = v[i + half];
        out[i] = u * c + w * s;
        out[i + half] = -u * s + w * c;
    }
}

static void scan_unit(const m3o_dims* d, int64_t b, int64_t hh, const double* x,
                      const double* B, const double* C, const double* theta, const double* dt,
                      const double* A, const double* lam, const double* B_bias,
                      const double* C_bias, double* h, double* phi, double* prev_B,
                      double* prev_x, double* y) {
    const int64_t L = d->seqlen, H = d->nheads, G = d->ngroups, P = d->headdim,
                  N = d->dstate, R = d->rank, half = N / 2;
    const int64_t g = hh / (H / G);
    double* hs = h + (b * H + hh) * N * P;
    double* ph = phi + (b * H + hh) * half;
    double* Bp = prev_B + (b * H + hh) * R * N;
    double* xp = prev_x + (b * H + hh) * R * P;
    const double* biasB = B_bias ? B_bias + hh * R * N : NULL;
    const double* biasC = C_bias ? C_bias + hh * R * N : NULL;

    double* work = (double*)malloc(sizeof(double) * (size_t)(6 * R * N + half));
    double* Bbar = work;
    double* Cbar = Bbar + R * N;
    double* Bpbar = Cbar + R * N;
    double* tmp = Bpbar + R * N;
    double* phi_prev = tmp + R * N;

    for (int64_t t = 0; t < L; ++t) {
        const int64_t tok = b * L + t;
        const int64_t sc = tok * H + hh; /* index into dt, A, lam */
        const double a_dt = dt[sc] * A[sc];
        const double alpha = exp(a_dt);
        const double beta = d->zoh ? 0.0 : (1.0 - lam[sc]) * dt[sc] * alpha;
        const double gamma = d->zoh ? (a_dt != 0.0 ? expm1(a_dt) / A[sc] : dt[sc])
                                    : lam[sc] * dt[sc];

        memcpy(phi_prev, ph, sizeof(double) * (size_t)half);
        const double* th = theta + sc * half;
        for (int64_t i = 0; i < half; ++i) ph[i] += dt[sc] * th[i];

        for (int64_t r = 0; r < R; ++r) {
            const double* braw = B + ((tok * G + g) * R + r) * N;
            const double* craw = C + ((tok * G + g) * R + r) * N;
            norm_bias(braw, biasB ? biasB + r * N : NULL, N, d->bc_norm, d->norm_eps, tmp);
            rotate_T(tmp, ph, N, Bbar + r * N);
            norm_bias(craw, biasC ? biasC + r * N : NULL, N, d->bc_norm, d->norm_eps, tmp);
            rotate_T(tmp, ph, N, Cbar + r * N);
            norm_bias(Bp + r * N, biasB ? biasB + r * N : NULL, N, d->bc_norm, d->norm_eps,
                      tmp);
            rotate_T(tmp, phi_prev, N, Bpbar + r * N);
        }

        const double* xt = x + sc * R * P;
        for (int64_t n = 0; n < N; ++n) {
            for (int64_t p = 0; p < P; ++p) {
                double acc = alpha * hs[n * P + p];
                for (int64_t r = 0; r < R; ++r)
                    acc += beta * Bpbar[r * N + n] * xp[r * P + p] +
                           gamma * Bbar[r * N + n] * xt[r * P + p];
                hs[n * P + p] = acc;
            }
        }
        double* yt = y + sc * R * P;
        for (int64_t r = 0; r < R; ++r) {
            for (int64_t p = 0; p < P; ++p) {
                double acc = 0.0;
                for (int64_t n = 0; n < N; ++n) acc += hs[n * P + p] * Cbar[r * N + n];
                yt[r * P + p] = acc;
            }
        }
        for (int64_t r = 0; r < R; ++r)
            memcpy(Bp + r * N, B + ((tok * G + g) * R + r) * N, sizeof(double) * (size_t)N);
        memcpy(xp, xt, sizeof(double) * (size_t)(R * P));
    }
    free(work);
}

/* Runs the recurrence over all units. Returns 0 on success, -1 on a bad argument.
 * nthreads <= 0 means "whatever OpenMP picks"; 1 means strictly single-threaded. */
int m3o_scan(const m3o_dims* d, const double* x, const double* B, const double* C,
             const double* theta, const double* dt, const double* A, const double* lam,
             const double* B_bias, const double* C_bias, double* h, double* phi,
             double* prev_B, double* prev_x, double* y, int nthreads) {
    if (!d || d->batch < 0 || d->seqlen < 0 || d->nheads <= 0 || d->ngroups <= 0 ||
        d->nheads % d->ngroups != 0 || d->headdim <= 0 || d->dstate <= 0 ||
        d->dstate % 2 != 0 || d->rank <= 0)
        return -1;
    const int64_t units = d->batch * d->nheads;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
    for (int64_t u = 0; u < units; ++u)
        scan_unit(d, u / d->nheads, u % d->nheads, x, B, C, theta, dt, A, lam, B_bias,
                  C_bias, h, phi, prev_B, prev_x, y);
    (void)nthreads;
    return 0;
}

/* Number of threads an OpenMP region would use (1 without OpenMP). */
int m3o_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

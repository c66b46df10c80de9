/*
 * retention_oracle.c -- plain fp64 CPU oracle for multi-scale retention.
 *
 * TEST INFRASTRUCTURE ONLY.  This file exists so that the tests, the smoke
 * check and the CPU baseline of the benchmark have an independent, obviously
 * correct reference to compare the CUDA library against.  Nothing in the
 * product library links, includes or calls it, and it shares no code with
 * the CUDA path.  It is deliberately slow: straight loops in the order the
 * pages state the mathematics, fp64 throughout, no blocking and no fusion.
 * The only parallelism is an OpenMP loop over independent (batch, head)
 * slices, which does not change any arithmetic.
 *
 * Sources (page title, section / equation):
 *   [P1] "Hybrid Architectures: RetNet and the Three Computation Paradigms"
 *        (prathamp.com blog), sections 2-8.
 *   [P3] "Retentive Network: A Successor to Transformer for Large Language
 *        Models" paper summary, Eq. 5 (parallel), Eq. 6 (recurrent),
 *        Eq. 7 (chunkwise).
 *   [P4] "RetNet math" (aicassindra transformer-math notes), recurrent and
 *        chunkwise-recurrent sections.
 *
 * Layouts (row-major, last index fastest):
 *   q, k  [B, N, H, dk]     v, out [B, N, H, dv]
 *   state [B, H, dk, dv]    gammas [H]
 * Positions are 0-based: token n of a sequence sits at position n.
 */
#include <math.h>
#include <stddef.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

#define IDX4(a, b, c, d, B1, C1, D1) ((((size_t)(a) * (B1) + (b)) * (C1) + (c)) * (D1) + (d))

static void set_threads(int nthreads) {
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
}

int orc_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * gamma^e for an integer exponent e >= 0, with 0^0 = 1.
 * [P1] section 2.3 (decay table gamma^(n-m)); [P1] section 4.2 (D matrix,
 * diagonal entries gamma^0 = 1 even where gamma = 0).
 */
double orc_gamma_pow(double gamma, long long e) {
    if (e == 0) return 1.0;
    return pow(gamma, (double)e);
}

/*
 * xPos / rotary rotation, in place, on x [B, N, H, d] (d even).
 * [P1] section 6.6 (Q_n = q_n * e^{i n theta}), section 6.8 (real form: each
 * consecutive pair (2p, 2p+1) is turned by a 2x2 rotation through the angle
 * position * theta_p).  theta_p = theta_base^(-2p/d).
 * Both Q and K are turned by +position*theta_p; the K-side conjugate of the
 * complex form is the transpose in the real dot product, so q'.k' depends on
 * the position difference only ([P1] section 6.7).
 */
void orc_xpos_rotate(double *x, int B, int N, int H, int d, long long pos_offset,
                     double theta_base) {
    for (int b = 0; b < B; b++)
        for (int n = 0; n < N; n++)
            for (int h = 0; h < H; h++) {
                double *row = x + IDX4(b, n, h, 0, N, H, d);
                double pos = (double)(pos_offset + n);
                for (int p = 0; p < d / 2; p++) {
                    double theta = pow(theta_base, -2.0 * p / (double)d);
                    double ang = pos * theta;
                    double c = cos(ang), s = sin(ang);
                    double x0 = row[2 * p], x1 = row[2 * p + 1];
                    row[2 * p] = x0 * c - x1 * s;
                    row[2 * p + 1] = x0 * s + x1 * c;
                }
            }
}

/*
 * The definition: recurrent retention.
 * [P1] section 2.1:  S_n = gamma S_{n-1} + k_n v_n^T,  o_n = q_n^T S_n,  S_0 = 0.
 * [P3] Eq. 6 states the same recurrence.  The state is updated before the
 * read-out, so token n reads its own contribution.
 *
 * init_state (nullable) replaces S_0 = 0; this is how a decode step continues
 * a prefix ([P3] recurrent representation: S_n is a sufficient statistic of
 * the past).  final_state (nullable) receives S_N.
 */
void orc_retention_recurrent(const double *q, const double *k, const double *v,
                             const double *gammas, int B, int N, int H, int dk, int dv,
                             const double *init_state, double *out, double *final_state,
                             int nthreads) {
    set_threads(nthreads);
    int BH = B * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (int bh = 0; bh < BH; bh++) {
        int b = bh / H, h = bh % H;
        double gamma = gammas[h];
        double *S = (double *)calloc((size_t)dk * dv, sizeof(double));
        if (init_state) memcpy(S, init_state + (size_t)bh * dk * dv, (size_t)dk * dv * sizeof(double));
        for (int n = 0; n < N; n++) {
            const double *qn = q + IDX4(b, n, h, 0, N, H, dk);
            const double *kn = k + IDX4(b, n, h, 0, N, H, dk);
            const double *vn = v + IDX4(b, n, h, 0, N, H, dv);
            /* S_n = gamma S_{n-1} + k_n v_n^T */
            for (int i = 0; i < dk; i++)
                for (int j = 0; j < dv; j++)
                    S[(size_t)i * dv + j] = gamma * S[(size_t)i * dv + j] + kn[i] * vn[j];
            /* o_n = q_n^T S_n  (for each j the sum runs over i = 0..dk-1 in order) */
            double *on = out + IDX4(b, n, h, 0, N, H, dv);
            for (int j = 0; j < dv; j++) on[j] = 0.0;
            for (int i = 0; i < dk; i++)
                for (int j = 0; j < dv; j++) on[j] += qn[i] * S[(size_t)i * dv + j];
        }
        if (final_state) memcpy(final_state + (size_t)bh * dk * dv, S, (size_t)dk * dv * sizeof(double));
        free(S);
    }
}

/*
 * Brute-force parallel form, used only to check the definition above.
 * [P1] sections 4.2-4.3 and [P3] Eq. 5:  Retention = (Q K^T (.) D) V with
 * D_nm = gamma^(n-m) for n >= m and 0 above the diagonal.
 */
void orc_retention_parallel(const double *q, const double *k, const double *v,
                            const double *gammas, int B, int N, int H, int dk, int dv,
                            double *out, int nthreads) {
    set_threads(nthreads);
    int BH = B * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (int bh = 0; bh < BH; bh++) {
        int b = bh / H, h = bh % H;
        double gamma = gammas[h];
        for (int n = 0; n < N; n++) {
            double *on = out + IDX4(b, n, h, 0, N, H, dv);
            for (int j = 0; j < dv; j++) on[j] = 0.0;
            const double *qn = q + IDX4(b, n, h, 0, N, H, dk);
            for (int m = 0; m <= n; m++) {
                const double *km = k + IDX4(b, m, h, 0, N, H, dk);
                const double *vm = v + IDX4(b, m, h, 0, N, H, dv);
                double qk = 0.0; /* (Q K^T)_nm */
                for (int i = 0; i < dk; i++) qk += qn[i] * km[i];
                double w = qk * orc_gamma_pow(gamma, n - m); /* (Q K^T (.) D)_nm */
                for (int j = 0; j < dv; j++) on[j] += w * vm[j];
            }
        }
    }
}

/*
 * Chunkwise recurrent form, used only to check the definition above.
 * [P1] section 7.2, [P3] Eq. 7, [P4] chunkwise-recurrent section.  With chunk
 * length Bc and 0-based in-chunk row index j:
 *   inner_i = (Q_[i] K_[i]^T (.) D_chunk) V_[i]
 *   cross_i = (Q_[i] R_{i-1}) (.) xi,         xi_j   = gamma^(j+1)
 *   R_i     = gamma^Bc R_{i-1} + K_[i]^T (V_[i] (.) zeta),  zeta_j = gamma^(Bc-1-j)
 * The pages assume N is a multiple of the chunk; for a shorter last chunk of
 * length L the same formulas are used with Bc replaced by L (the plain
 * reading; it keeps R equal to the recurrent S at every chunk boundary).
 */
void orc_retention_chunkwise(const double *q, const double *k, const double *v,
                             const double *gammas, int B, int N, int H, int dk, int dv,
                             int chunk, double *out, double *final_state, int nthreads) {
    set_threads(nthreads);
    int BH = B * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (int bh = 0; bh < BH; bh++) {
        int b = bh / H, h = bh % H;
        double gamma = gammas[h];
        double *R = (double *)calloc((size_t)dk * dv, sizeof(double));
        double *dR = (double *)calloc((size_t)dk * dv, sizeof(double));
        for (int c0 = 0; c0 < N; c0 += chunk) {
            int L = (N - c0 < chunk) ? (N - c0) : chunk;
            for (int r = 0; r < L; r++) {
                int n = c0 + r;
                const double *qn = q + IDX4(b, n, h, 0, N, H, dk);
                double *on = out + IDX4(b, n, h, 0, N, H, dv);
                /* inner: sum over c <= r of (q_r . k_c) gamma^(r-c) v_c */
                for (int j = 0; j < dv; j++) on[j] = 0.0;
                for (int c = 0; c <= r; c++) {
                    const double *kc = k + IDX4(b, c0 + c, h, 0, N, H, dk);
                    const double *vc = v + IDX4(b, c0 + c, h, 0, N, H, dv);
                    double qk = 0.0;
                    for (int i = 0; i < dk; i++) qk += qn[i] * kc[i];
                    double w = qk * orc_gamma_pow(gamma, r - c);
                    for (int j = 0; j < dv; j++) on[j] += w * vc[j];
                }
                /* cross: (q_r^T R_{i-1}) * xi_r */
                double xi = orc_gamma_pow(gamma, r + 1);
                for (int j = 0; j < dv; j++) {
                    double acc = 0.0;
                    for (int i = 0; i < dk; i++) acc += qn[i] * R[(size_t)i * dv + j];
                    on[j] += acc * xi;
                }
            }
            /* R_i = gamma^L R_{i-1} + K^T (V (.) zeta) */
            memset(dR, 0, (size_t)dk * dv * sizeof(double));
            for (int r = 0; r < L; r++) {
                const double *kr = k + IDX4(b, c0 + r, h, 0, N, H, dk);
                const double *vr = v + IDX4(b, c0 + r, h, 0, N, H, dv);
                double zeta = orc_gamma_pow(gamma, L - 1 - r);
                for (int i = 0; i < dk; i++)
                    for (int j = 0; j < dv; j++) dR[(size_t)i * dv + j] += kr[i] * (vr[j] * zeta);
            }
            double gL = orc_gamma_pow(gamma, L);
            for (size_t e = 0; e < (size_t)dk * dv; e++) R[e] = gL * R[e] + dR[e];
        }
        if (final_state) memcpy(final_state + (size_t)bh * dk * dv, R, (size_t)dk * dv * sizeof(double));
        free(R);
        free(dR);
    }
}

/*
 * One recurrent decode step on a carried state, in place.
 * [P1] section 5.2 and [P3] recurrent representation / inference protocol:
 * S <- gamma S + k v^T, then o = q^T S.  q, k [B, H, dk], v [B, H, dv],
 * state [B, H, dk, dv], out [B, H, dv].
 */
void orc_decode_step(const double *q, const double *k, const double *v,
                     const double *gammas, int B, int H, int dk, int dv,
                     double *state, double *out, int nthreads) {
    set_threads(nthreads);
    int BH = B * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (int bh = 0; bh < BH; bh++) {
        int h = bh % H;
        double gamma = gammas[h];
        double *S = state + (size_t)bh * dk * dv;
        const double *qb = q + (size_t)bh * dk;
        const double *kb = k + (size_t)bh * dk;
        const double *vb = v + (size_t)bh * dv;
        for (int i = 0; i < dk; i++)
            for (int j = 0; j < dv; j++)
                S[(size_t)i * dv + j] = gamma * S[(size_t)i * dv + j] + kb[i] * vb[j];
        double *ob = out + (size_t)bh * dv;
        for (int j = 0; j < dv; j++) ob[j] = 0.0;
        for (int i = 0; i < dk; i++)
            for (int j = 0; j < dv; j++) ob[j] += qb[i] * S[(size_t)i * dv + j];
    }
}

/*
 * Gradients of the definition (the recurrent form above, [P1] section 2.1,
 * [P3] Eq. 6) with respect to q, k and v, for an upstream gradient dout of
 * the output.  The pages train through the chunkwise form ([P3] training
 * protocol) but print no backward pass; these are the derivatives of the
 * unrolled definition o_n = sum_{m<=n} gamma^(n-m) (q_n . k_m) v_m, summed
 * straight from it over every pair m <= n (brute force, O(N^2)):
 *     dq_n += gamma^(n-m) (dout_n . v_m) k_m
 *     dk_m += gamma^(n-m) (dout_n . v_m) q_n
 *     dv_m += gamma^(n-m) (q_n . k_m)   dout_n
 * q and k are the vectors the definition multiplies (rotated ones when the
 * caller rotates); dq, dk, dv are overwritten.
 */
void orc_retention_backward(const double *q, const double *k, const double *v, const double *dout,
                            const double *gammas, int B, int N, int H, int dk, int dv,
                            double *dq, double *dkk, double *dvv, int nthreads) {
    set_threads(nthreads);
    int BH = B * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (int bh = 0; bh < BH; bh++) {
        int b = bh / H, h = bh % H;
        double gamma = gammas[h];
        for (int n = 0; n < N; n++) {
            for (int i = 0; i < dk; i++) {
                dq[IDX4(b, n, h, i, N, H, dk)] = 0.0;
                dkk[IDX4(b, n, h, i, N, H, dk)] = 0.0;
            }
            for (int j = 0; j < dv; j++) dvv[IDX4(b, n, h, j, N, H, dv)] = 0.0;
        }
        for (int n = 0; n < N; n++) {
            const double *qn = q + IDX4(b, n, h, 0, N, H, dk);
            const double *gn = dout + IDX4(b, n, h, 0, N, H, dv);
            for (int m = 0; m <= n; m++) {
                const double *km = k + IDX4(b, m, h, 0, N, H, dk);
                const double *vm = v + IDX4(b, m, h, 0, N, H, dv);
                double w = orc_gamma_pow(gamma, n - m);
                double a = 0.0, g = 0.0;
                for (int i = 0; i < dk; i++) a += qn[i] * km[i];
                for (int j = 0; j < dv; j++) g += gn[j] * vm[j];
                for (int i = 0; i < dk; i++) {
                    dq[IDX4(b, n, h, i, N, H, dk)] += w * g * km[i];
                    dkk[IDX4(b, m, h, i, N, H, dk)] += w * g * qn[i];
                }
                for (int j = 0; j < dv; j++) dvv[IDX4(b, m, h, j, N, H, dv)] += w * a * gn[j];
            }
        }
    }
}

/*
 * Retention with the score normalizations 2 and 3, parallel form by brute
 * force.  [P1] section 8.5 and [P3] "Retention Score Normalization":
 *   2. the decay matrix row-normalized:  Dt_nm = D_nm / sqrt(sum_{i<=n} D_ni)
 *   3. the scores row-normalized:        Rt_nm = R_nm / max(|sum_{i<=n} R_ni|, 1)
 *      with R = (Q K^T) (.) Dt (the scores after normalization 2)
 * and out = Rt V.  Normalization 1 (the 1/sqrt(d) on Q K^T) is the caller's
 * scaling of q.  The row sums are taken as written: the absolute value of the
 * sum, not the sum of absolute values.  flags bit 0 turns on normalization
 * 2, bit 1 normalization 3; flags = 0 is orc_retention_parallel.
 */
void orc_retention_normalized(const double *q, const double *k, const double *v,
                              const double *gammas, int B, int N, int H, int dk, int dv,
                              int flags, double *out, int nthreads) {
    set_threads(nthreads);
    int BH = B * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (int bh = 0; bh < BH; bh++) {
        int b = bh / H, h = bh % H;
        double gamma = gammas[h];
        double *row = (double *)malloc(sizeof(double) * (size_t)(N > 0 ? N : 1)); /* R_n. */
        for (int n = 0; n < N; n++) {
            const double *qn = q + IDX4(b, n, h, 0, N, H, dk);
            /* sum_{i<=n} D_ni */
            double dsum = 0.0;
            for (int i = 0; i <= n; i++) dsum += orc_gamma_pow(gamma, n - i);
            double dscale = (flags & 1) ? 1.0 / sqrt(dsum) : 1.0;
            /* R_nm = (Q K^T)_nm Dt_nm */
            double rsum = 0.0;
            for (int m = 0; m <= n; m++) {
                const double *km = k + IDX4(b, m, h, 0, N, H, dk);
                double qk = 0.0;
                for (int i = 0; i < dk; i++) qk += qn[i] * km[i];
                row[m] = qk * orc_gamma_pow(gamma, n - m) * dscale;
                rsum += row[m];
            }
            double den = 1.0;
            if (flags & 2) den = fabs(rsum) > 1.0 ? fabs(rsum) : 1.0;
            double *on = out + IDX4(b, n, h, 0, N, H, dv);
            for (int j = 0; j < dv; j++) on[j] = 0.0;
            for (int m = 0; m <= n; m++) {
                const double *vm = v + IDX4(b, m, h, 0, N, H, dv);
                double w = row[m] / den;
                for (int j = 0; j < dv; j++) on[j] += w * vm[j];
            }
        }
        free(row);
    }
}

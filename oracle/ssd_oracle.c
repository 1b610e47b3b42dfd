/*
 * ssd_oracle.c -- plain, slow, fp64 CPU oracle for the Mamba-2 SSD hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the CPU-baseline
 * leg of the benchmark may load this library.  The product (the sm_100a kernels behind
 * include/ssd.h) never calls it, shares no code with it and has no CPU fallback.
 *
 * Source of every formula: "Compiler-First State Space Duality and Portable O(1)
 * Autoregressive Caching" (arXiv 2603.09555), cited below as [CF-SSD]:
 *   - SSM background: the continuous SSM (Eq. 1) discretised with step Delta (Eq. 2);
 *     Mamba-2 makes B, C, Delta input dependent and A a scalar per head.
 *   - the dual form over a chunk (Eq. 3) with the lower-triangular decay matrix obtained
 *     by exponentiating a segment-wise prefix sum of A*Delta, and the separate
 *     sequential recurrence over chunk summary states ("Chunked recurrence" property).
 *   - the O(1) cache section: a depthwise convolution over a window of k-1 cached inputs
 *     followed by one recurrence step h_t = Abar h_{t-1} + Bbar x_t; the state is
 *     h in R^{H x P x N}, the conv state has shape (B, D_conv, k-1).
 *
 * Readings where the pages are silent (the display equations were lost):
 *   R1  discretisation: Abar = exp(dt*A) (exact for a scalar A), Bbar = dt*B (the
 *       first-order input term used by Mamba-2); y_t = C_t . h_t + D * x_t.
 *   R2  the decay matrix is Lmat[i][j] = exp(cs_i - cs_j) for j <= i (0 above the
 *       diagonal) with cs the inclusive prefix sum of a = dt*A inside the chunk.
 *   R4  the state is P x N per head: h[p][n] += dt * x[p] * B[n].
 *   R5  head h reads group g = h / (H/G) of B and C.
 *   R6  conv channel order [x (H*P) | B (G*N) | C (G*N)]; activation SiLU or none.
 *
 * All arithmetic is double precision.  Inputs arrive as doubles that hold exactly the
 * values the GPU sees (bf16- or fp32-rounded by the caller).
 *
 * Layouts (row-major, last index contiguous):
 *   x  [b][T][H][P]   dt [b][T][H]   A [H]   D [H]   B, C [b][T][G][N]
 *   h0, h_final [b][H][P][N]   y [b][T][H][P]
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define IDX4(a, b, c, d, B_, C_, D_) ((((size_t)(a) * (B_) + (b)) * (C_) + (c)) * (D_) + (d))

static void set_threads(int nthreads) {
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
}

int oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * Token-by-token recurrence ([CF-SSD] Eq. 2 with readings R1, R4, R5).
 *   for t: alpha = exp(dt_t*A_h);  h[p][n] = alpha*h[p][n] + dt_t*x_t[p]*B_t[n]
 *          y_t[p] = sum_n C_t[n]*h[p][n] + D_h*x_t[p]
 * This is the definition every other form must reproduce.
 */
void oracle_ssd_recurrence(int b, int T, int H, int P, int N, int G,
                           const double* x, const double* dt, const double* A,
                           const double* B, const double* C, const double* D,
                           const double* h0, double* y, double* h_final, int nthreads) {
    set_threads(nthreads);
    const int hpg = H / G;
#pragma omp parallel for schedule(dynamic, 1)
    for (int bh = 0; bh < b * H; ++bh) {
        const int bi = bh / H, hi = bh % H, g = hi / hpg;
        double* st = (double*)malloc(sizeof(double) * (size_t)P * N);
        for (int i = 0; i < P * N; ++i)
            st[i] = h0 ? h0[IDX4(bi, hi, 0, 0, H, P, N) + i] : 0.0;
        for (int t = 0; t < T; ++t) {
            const double d = dt[((size_t)bi * T + t) * H + hi];
            const double alpha = exp(d * A[hi]);
            const double* xt = x + IDX4(bi, t, hi, 0, T, H, P);
            const double* Bt = B + IDX4(bi, t, g, 0, T, G, N);
            const double* Ct = C + IDX4(bi, t, g, 0, T, G, N);
            double* yt = y + IDX4(bi, t, hi, 0, T, H, P);
            for (int p = 0; p < P; ++p) {
                double acc = 0.0;
                for (int n = 0; n < N; ++n) {
                    double v = alpha * st[p * N + n] + d * xt[p] * Bt[n];
                    st[p * N + n] = v;
                    acc += Ct[n] * v;
                }
                yt[p] = acc + D[hi] * xt[p];
            }
        }
        if (h_final)
            for (int i = 0; i < P * N; ++i) h_final[IDX4(bi, hi, 0, 0, H, P, N) + i] = st[i];
        free(st);
    }
}

/*
 * Naive chunked dual form, written step by step as [CF-SSD] describes it:
 *   1. per chunk of L tokens, a = dt*A and its inclusive prefix sum cs (segment-wise);
 *   2. Lmat[i][j] = exp(cs_i - cs_j) for j <= i else 0 (R2);
 *   3. intra-chunk output  Y_diag = (C B^T o Lmat) (dt o X)            (Eq. 3);
 *   4. chunk summary state S_c[p][n] = sum_j exp(cs_last - cs_j) dt_j x_j[p] B_j[n];
 *   5. sequential recurrence over chunks: H_0 = h0, H_{c+1} = exp(cs_last(c)) H_c + S_c;
 *   6. state-to-output term Y_off[i][p] = exp(cs_i) sum_n C_i[n] H_c[p][n];
 *   7. y = Y_diag + Y_off + D x;  h_final = H_{n_c}.
 * No blocking beyond the chunk, no reordering.  L must divide T.
 */
void oracle_ssd_chunked(int b, int T, int H, int P, int N, int G, int L,
                        const double* x, const double* dt, const double* A,
                        const double* B, const double* C, const double* D,
                        const double* h0, double* y, double* h_final, int nthreads) {
    set_threads(nthreads);
    const int hpg = H / G, nc = T / L;
#pragma omp parallel for schedule(dynamic, 1)
    for (int bh = 0; bh < b * H; ++bh) {
        const int bi = bh / H, hi = bh % H, g = hi / hpg;
        double* cs = (double*)malloc(sizeof(double) * (size_t)L);
        double* Lm = (double*)malloc(sizeof(double) * (size_t)L * L);
        double* Hc = (double*)malloc(sizeof(double) * (size_t)P * N);
        double* S = (double*)malloc(sizeof(double) * (size_t)P * N);
        for (int i = 0; i < P * N; ++i) Hc[i] = h0 ? h0[IDX4(bi, hi, 0, 0, H, P, N) + i] : 0.0;
        for (int c = 0; c < nc; ++c) {
            const int t0 = c * L;
            /* step 1: segment-wise prefix sum of A*dt */
            double run = 0.0;
            for (int i = 0; i < L; ++i) {
                run += dt[((size_t)bi * T + t0 + i) * H + hi] * A[hi];
                cs[i] = run;
            }
            /* step 2: lower-triangular decay matrix */
            for (int i = 0; i < L; ++i)
                for (int j = 0; j < L; ++j) Lm[i * L + j] = (j <= i) ? exp(cs[i] - cs[j]) : 0.0;
            /* steps 3, 6, 7: outputs of this chunk (state term uses H_c, the state entering it) */
            for (int i = 0; i < L; ++i) {
                const double* Ci = C + IDX4(bi, t0 + i, g, 0, T, G, N);
                const double* xi = x + IDX4(bi, t0 + i, hi, 0, T, H, P);
                double* yi = y + IDX4(bi, t0 + i, hi, 0, T, H, P);
                for (int p = 0; p < P; ++p) yi[p] = 0.0;
                for (int j = 0; j <= i; ++j) {
                    const double* Bj = B + IDX4(bi, t0 + j, g, 0, T, G, N);
                    const double* xj = x + IDX4(bi, t0 + j, hi, 0, T, H, P);
                    const double dtj = dt[((size_t)bi * T + t0 + j) * H + hi];
                    double cb = 0.0;
                    for (int n = 0; n < N; ++n) cb += Ci[n] * Bj[n];
                    const double s = cb * Lm[i * L + j] * dtj;
                    for (int p = 0; p < P; ++p) yi[p] += s * xj[p];
                }
                const double ei = exp(cs[i]);
                for (int p = 0; p < P; ++p) {
                    double acc = 0.0;
                    for (int n = 0; n < N; ++n) acc += Ci[n] * Hc[p * N + n];
                    yi[p] += ei * acc + D[hi] * xi[p];
                }
            }
            /* step 4: chunk summary state */
            for (int i = 0; i < P * N; ++i) S[i] = 0.0;
            for (int j = 0; j < L; ++j) {
                const double* Bj = B + IDX4(bi, t0 + j, g, 0, T, G, N);
                const double* xj = x + IDX4(bi, t0 + j, hi, 0, T, H, P);
                const double w = exp(cs[L - 1] - cs[j]) * dt[((size_t)bi * T + t0 + j) * H + hi];
                for (int p = 0; p < P; ++p)
                    for (int n = 0; n < N; ++n) S[p * N + n] += w * xj[p] * Bj[n];
            }
            /* step 5: sequential inter-chunk recurrence */
            const double gam = exp(cs[L - 1]);
            for (int i = 0; i < P * N; ++i) Hc[i] = gam * Hc[i] + S[i];
        }
        if (h_final)
            for (int i = 0; i < P * N; ++i) h_final[IDX4(bi, hi, 0, 0, H, P, N) + i] = Hc[i];
        free(cs); free(Lm); free(Hc); free(S);
    }
}

/*
 * Whole-sequence quadratic form (the dual form of [CF-SSD] Eq. 3 with one chunk spanning
 * the sequence).  The decay between j and i is the exponential of the direct sum
 * sum_{k=j+1..i} a_k, not a difference of prefix sums, so it shares no rounding path
 * with the chunked form:
 *   y_i = sum_{j<=i} (C_i.B_j) exp(sum_{k=j+1..i} a_k) dt_j x_j
 *         + exp(sum_{k=0..i} a_k) C_i.h0 + D x_i
 *   h_final = exp(sum_all a) h0 + sum_j exp(sum_{k=j+1..T-1} a_k) dt_j x_j B_j^T
 */
void oracle_ssd_quadratic(int b, int T, int H, int P, int N, int G,
                          const double* x, const double* dt, const double* A,
                          const double* B, const double* C, const double* D,
                          const double* h0, double* y, double* h_final, int nthreads) {
    set_threads(nthreads);
    const int hpg = H / G;
#pragma omp parallel for schedule(dynamic, 1)
    for (int bh = 0; bh < b * H; ++bh) {
        const int bi = bh / H, hi = bh % H, g = hi / hpg;
        double* a = (double*)malloc(sizeof(double) * (size_t)T);
        for (int t = 0; t < T; ++t) a[t] = dt[((size_t)bi * T + t) * H + hi] * A[hi];
        const double* h0b = h0 ? h0 + IDX4(bi, hi, 0, 0, H, P, N) : NULL;
        for (int i = 0; i < T; ++i) {
            const double* Ci = C + IDX4(bi, i, g, 0, T, G, N);
            const double* xi = x + IDX4(bi, i, hi, 0, T, H, P);
            double* yi = y + IDX4(bi, i, hi, 0, T, H, P);
            for (int p = 0; p < P; ++p) yi[p] = D[hi] * xi[p];
            for (int j = 0; j <= i; ++j) {
                double seg = 0.0;
                for (int k = j + 1; k <= i; ++k) seg += a[k];
                const double* Bj = B + IDX4(bi, j, g, 0, T, G, N);
                const double* xj = x + IDX4(bi, j, hi, 0, T, H, P);
                double cb = 0.0;
                for (int n = 0; n < N; ++n) cb += Ci[n] * Bj[n];
                const double s = cb * exp(seg) * dt[((size_t)bi * T + j) * H + hi];
                for (int p = 0; p < P; ++p) yi[p] += s * xj[p];
            }
            if (h0b) {
                double seg = 0.0;
                for (int k = 0; k <= i; ++k) seg += a[k];
                const double e = exp(seg);
                for (int p = 0; p < P; ++p) {
                    double acc = 0.0;
                    for (int n = 0; n < N; ++n) acc += Ci[n] * h0b[p * N + n];
                    yi[p] += e * acc;
                }
            }
        }
        if (h_final) {
            double* hf = h_final + IDX4(bi, hi, 0, 0, H, P, N);
            double tot = 0.0;
            for (int k = 0; k < T; ++k) tot += a[k];
            for (int i = 0; i < P * N; ++i) hf[i] = h0b ? exp(tot) * h0b[i] : 0.0;
            for (int j = 0; j < T; ++j) {
                double seg = 0.0;
                for (int k = j + 1; k < T; ++k) seg += a[k];
                const double w = exp(seg) * dt[((size_t)bi * T + j) * H + hi];
                const double* Bj = B + IDX4(bi, j, g, 0, T, G, N);
                const double* xj = x + IDX4(bi, j, hi, 0, T, H, P);
                for (int p = 0; p < P; ++p)
                    for (int n = 0; n < N; ++n) hf[p * N + n] += w * xj[p] * Bj[n];
            }
        }
        free(a);
    }
}

/*
 * One cached decode step over every layer ([CF-SSD] O(1) cache section, readings R1,
 * R4, R5, R6).  Per (layer l, batch row r):
 *   window   = [conv_state[c][0..k-2], xbc[c]]               (k taps, oldest first)
 *   u[c]     = act( sum_{i<k} w[l][c][i] * window[i] + bias[l][c] )
 *   conv_state[c] <- window[1..k-1]                            (drop the oldest input)
 *   x = u[0 : H*P],  Bv = u[H*P : H*P+G*N],  Cv = u[H*P+G*N : H*P+2*G*N]
 *   per head h (group g): alpha = exp(dt*A), h[p][n] = alpha*h[p][n] + dt*x[h][p]*Bv[g][n]
 *                         y[h][p] = sum_n Cv[g][n]*h[p][n] + D*x[h][p]
 * act: 0 = none, 1 = SiLU (u * sigmoid(u)).
 * Layouts: h [layers][b][H][P][N]  conv_state [layers][b][Dc][k-1]  xbc [layers][b][Dc]
 *          dt [layers][b][H]  A, D [layers][H]  conv_w [layers][Dc][k]  conv_b [layers][Dc]
 *          y [layers][b][H][P]      with Dc = H*P + 2*G*N.
 */
void oracle_decode_step(int layers, int b, int H, int P, int N, int G, int kconv, int act,
                        double* h, double* conv_state, const double* xbc, const double* dt,
                        const double* A, const double* D, const double* conv_w,
                        const double* conv_b, double* y, int nthreads) {
    set_threads(nthreads);
    const int Dc = H * P + 2 * G * N, hpg = H / G, km1 = kconv - 1;
#pragma omp parallel for schedule(dynamic, 1)
    for (int lb = 0; lb < layers * b; ++lb) {
        const int l = lb / b, r = lb % b;
        double* u = (double*)malloc(sizeof(double) * (size_t)Dc);
        double* cst = conv_state + ((size_t)l * b + r) * Dc * km1;
        const double* xin = xbc + ((size_t)l * b + r) * Dc;
        for (int c = 0; c < Dc; ++c) {
            double acc = conv_b[(size_t)l * Dc + c];
            const double* w = conv_w + ((size_t)l * Dc + c) * kconv;
            for (int i = 0; i < km1; ++i) acc += w[i] * cst[(size_t)c * km1 + i];
            acc += w[km1] * xin[c];
            if (act == 1) acc = acc / (1.0 + exp(-acc));
            u[c] = acc;
            for (int i = 0; i + 1 < km1; ++i) cst[(size_t)c * km1 + i] = cst[(size_t)c * km1 + i + 1];
            if (km1 > 0) cst[(size_t)c * km1 + km1 - 1] = xin[c];
        }
        for (int hi = 0; hi < H; ++hi) {
            const int g = hi / hpg;
            const double d = dt[((size_t)l * b + r) * H + hi];
            const double alpha = exp(d * A[(size_t)l * H + hi]);
            const double* xv = u + hi * P;
            const double* Bv = u + H * P + g * N;
            const double* Cv = u + H * P + G * N + g * N;
            double* st = h + ((((size_t)l * b + r) * H + hi) * P) * N;
            double* yo = y + (((size_t)l * b + r) * H + hi) * P;
            for (int p = 0; p < P; ++p) {
                double acc = 0.0;
                for (int n = 0; n < N; ++n) {
                    double v = alpha * st[p * N + n] + d * xv[p] * Bv[n];
                    st[p * N + n] = v;
                    acc += Cv[n] * v;
                }
                yo[p] = acc + D[(size_t)l * H + hi] * xv[p];
            }
        }
        free(u);
    }
}

/*
 * Step sizes from the raw projection output, as the Mamba-2 block forms them before the
 * SSD ([CF-SSD]: the elementwise chain -- bias add, softplus, clamp -- ahead of the scan,
 * which the paper fuses into the surrounding computation):
 *   dt[i] = min(max(softplus(raw[i] + bias[i % H]), lo), hi),  softplus(z) = log(1 + e^z).
 * The softplus is evaluated as max(z, 0) + log1p(exp(-|z|)), which equals log(1 + e^z)
 * for every z and never overflows.  bias may be NULL (no bias); hi may be +inf.
 * n = b * T * H entries in [b][T][H] order.
 */
void oracle_dt_from_raw(size_t n, int H, const double* raw, const double* bias, double lo, double hi,
                        double* dt) {
    for (size_t i = 0; i < n; ++i) {
        const double z = raw[i] + (bias ? bias[i % (size_t)H] : 0.0);
        double sp = (z > 0.0 ? z : 0.0) + log1p(exp(-fabs(z)));
        if (sp < lo) sp = lo;
        if (sp > hi) sp = hi;
        dt[i] = sp;
    }
}

/*
 * Term magnitudes of one decode step, for per-element error bounds.  Every output of the
 * step is a sum of products; an fp32 evaluation of it carries a rounding error of a few
 * ulps of the SUM OF THE ABSOLUTE VALUES of those products, not of the output itself
 * (which may cancel to near zero).  This function walks the same step as
 * oracle_decode_step with each sum taken over absolute values:
 *   window   = [conv_state[c][0..k-2], xbc[c]]      (read only: call before the value step)
 *   m[c]     = sum_i |w[l][c][i] * window[i]| + |bias[l][c]|         the conv's terms
 *   M[c]     = m[c] with no activation; |silu(v[c])| + m[c] with SiLU (its slope lies in
 *              [-0.1, 1.1], so an error in the conv sum v moves the output by about as much)
 *   hm[p][n] <- alpha*hm[p][n] + dt*Mx[p]*MB[n]    (hm starts from |h| and is updated in place)
 *   ym[h][p] = sum_n MC[n]*hm[p][n] + |D|*Mx[p]
 * Mx, MB, MC are the M of the x, B and C channels of the head's group.  Every magnitude
 * bounds the absolute value of its output (triangle inequality), with equality when all
 * inputs, weights and states are non-negative and no activation is applied.
 */
void oracle_decode_step_mag(int layers, int b, int H, int P, int N, int G, int kconv, int act,
                            double* hm, const double* conv_state, const double* xbc, const double* dt,
                            const double* A, const double* D, const double* conv_w,
                            const double* conv_b, double* ym, int nthreads) {
    set_threads(nthreads);
    const int Dc = H * P + 2 * G * N, hpg = H / G, km1 = kconv - 1;
#pragma omp parallel for schedule(dynamic, 1)
    for (int lb = 0; lb < layers * b; ++lb) {
        const int l = lb / b, r = lb % b;
        double* M = (double*)malloc(sizeof(double) * (size_t)Dc);
        const double* cst = conv_state + ((size_t)l * b + r) * Dc * km1;
        const double* xin = xbc + ((size_t)l * b + r) * Dc;
        for (int c = 0; c < Dc; ++c) {
            const double bias = conv_b[(size_t)l * Dc + c];
            const double* w = conv_w + ((size_t)l * Dc + c) * kconv;
            double v = bias, m = fabs(bias);
            for (int i = 0; i < km1; ++i) {
                v += w[i] * cst[(size_t)c * km1 + i];
                m += fabs(w[i] * cst[(size_t)c * km1 + i]);
            }
            v += w[km1] * xin[c];
            m += fabs(w[km1] * xin[c]);
            M[c] = act == 1 ? fabs(v / (1.0 + exp(-v))) + m : m;
        }
        for (int hi = 0; hi < H; ++hi) {
            const int g = hi / hpg;
            const double d = dt[((size_t)l * b + r) * H + hi];
            const double alpha = exp(d * A[(size_t)l * H + hi]);
            const double* Mx = M + hi * P;
            const double* MB = M + H * P + g * N;
            const double* MC = M + H * P + G * N + g * N;
            double* st = hm + ((((size_t)l * b + r) * H + hi) * P) * N;
            double* yo = ym + (((size_t)l * b + r) * H + hi) * P;
            for (int p = 0; p < P; ++p) {
                double acc = 0.0;
                for (int n = 0; n < N; ++n) {
                    const double v = alpha * st[p * N + n] + d * Mx[p] * MB[n];
                    st[p * N + n] = v;
                    acc += MC[n] * v;
                }
                yo[p] = acc + fabs(D[(size_t)l * H + hi]) * Mx[p];
            }
        }
        free(M);
    }
}

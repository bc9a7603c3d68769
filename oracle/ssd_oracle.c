/*
 * fp64 CPU oracle for the scalar-decay selective state-space layer (SSD).
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path may call, link or
 * load this file: only the tests, the package smoke check and the benchmark's
 * CPU-baseline leg use it. It shares no code, header or constant with the
 * CUDA library.
 *
 * Every function is the plain definition, written for a reader to check by
 * eye against the pages:
 *
 *   [M2-matrix]   "Mamba-2 — 注意力的远亲" (docsaid.org), section
 *                 "把 SSM 写成一个矩阵": h_t = A_t h_{t-1} + B_t x_t,
 *                 y_t = C_t^T h_t, and the unrolled sum / matrix form
 *                 y_j = sum_{i<=j} C_j^T A_j...A_{i+1} B_i x_i.
 *   [M2-scalar]   same page, section "把 A 简化成一个数": A_t = a_t I, so
 *                 M = L o (C B^T) with L_ji = a_j x ... x a_{i+1} (j >= i).
 *   [M2-example]  same page, section "跟着四个 token 算一次": the state is
 *                 updated first (h = a h + B x) and then read (y = C h).
 *   [M2-chunks]   same page, section "两条路各走一半", and "Mamba-2 模型解读"
 *                 (139.9.1.231), sections 6.1 / 6.2: split the sequence into
 *                 blocks; diagonal blocks in quadratic form; off-diagonal
 *                 blocks through input->state, state->state, state->output;
 *                 only the block-end state passes between blocks; the
 *                 function returns Y and the final state.
 *   [Mamba-disc]  "精读笔记 #12：Mamba" (llm-papers-study), section 2.2:
 *                 the decay is A_bar = exp(Delta A); under the zero-order
 *                 hold rule the input matrix is
 *                 B_bar = (Delta A)^-1 (exp(Delta A) - I) Delta B.
 *   [Mamba-scan]  same page, sections 2.2 and 3: the selective scan with a
 *                 diagonal A per channel (oracle_selective_scan).
 *   [Mamba-sel]   same page, section 3 (the selection mechanism, algorithm
 *                 2): Delta = softplus(Linear(x)), a positive step made from
 *                 a raw projection; and section 3.5, theorem 1: with N = 1,
 *                 A = -1, B = 1 the recurrence is the gate
 *                 h_t = (1 - g_t) h_{t-1} + g_t x_t, g_t = sigmoid(.).
 *
 * The layer computed here (the scalar-decay SSD layer with Euler input
 * weight and a skip term):
 *
 *   for each batch b, head h (group g = h / (H/G)):
 *     h = h0[b,h]                                (P x N; zeros if NULL)
 *     for t = 0 .. L-1:
 *       a = exp(ell[b,t,h])                      ell = dt*A in the layer
 *       h[p][n] = a*h[p][n] + w[b,t,h]*x[b,t,h,p]*B[b,t,g,n]   (w = dt)
 *       y[b,t,h,p] = sum_n C[b,t,g,n]*h[p][n] + D[h]*x[b,t,h,p]
 *     h_final[b,h] = h
 *
 * Layouts (row-major, last index fastest):
 *   x, y   (batch, L, H, P)      ell, w, dt  (batch, L, H)
 *   B, C   (batch, L, G, N)      A, D        (H)
 *   h0, h_final, h   (batch, H, P, N)
 *
 * All arithmetic is IEEE fp64 in the order written; build without
 * -ffast-math. OpenMP runs independent (b,h) lanes on separate threads,
 * which does not change any lane's arithmetic.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_BAD_ARG 1
#define ORACLE_NO_MEMORY 2

static int dims_ok(int64_t batch, int64_t L, int64_t H, int64_t P, int64_t N,
                   int64_t G)
{
    if (batch < 0 || L < 0 || H < 1 || P < 1 || N < 1 || G < 1) return 0;
    if (H % G != 0) return 0;
    return 1;
}

static void set_threads(int nthreads)
{
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
}

/* Number of threads an OpenMP region of this library would use. */
int oracle_max_threads(int nthreads)
{
#ifdef _OPENMP
    if (nthreads > 0) return nthreads;
    return omp_get_max_threads();
#else
    (void)nthreads;
    return 1;
#endif
}

/*
 * One (b,h) lane of the recurrence [M2-matrix], [M2-scalar], [M2-example].
 * `hs` is P*N scratch. Strides are in elements, for the time axis.
 */
static void scan_lane(int64_t L, int64_t P, int64_t N,
                      const double *x, int64_t sx,        /* x[t*sx + p]   */
                      const double *ell, const double *w, int64_t sa,
                      const double *Bg, const double *Cg, int64_t sb,
                      double Dh, const double *h0,         /* P*N or NULL */
                      double *y, int64_t sy, double *hf, double *hs)
{
    if (h0) memcpy(hs, h0, (size_t)(P * N) * sizeof(double));
    else memset(hs, 0, (size_t)(P * N) * sizeof(double));
    for (int64_t t = 0; t < L; ++t) {
        const double a = exp(ell[t * sa]);
        const double wt = w[t * sa];
        const double *xt = x + t * sx;
        const double *Bt = Bg + t * sb;
        const double *Ct = Cg + t * sb;
        for (int64_t p = 0; p < P; ++p) {
            double *hp = hs + p * N;
            const double wx = wt * xt[p];
            double acc = 0.0;
            for (int64_t n = 0; n < N; ++n) {
                hp[n] = a * hp[n] + wx * Bt[n];
                acc += Ct[n] * hp[n];
            }
            y[t * sy + p] = acc + Dh * xt[p];
        }
    }
    if (hf) memcpy(hf, hs, (size_t)(P * N) * sizeof(double));
}

/*
 * General recurrence with the per-step log-decay ell (a_t = exp(ell_t)) and
 * input weight w given directly. The worked four-token example of
 * [M2-example] is this function with ell = log(a), w = 1, D = 0, h0 = 0.
 * D may be NULL (no skip term); h0 and h_final may be NULL.
 */
int oracle_scan(int64_t batch, int64_t L, int64_t H, int64_t P, int64_t N,
                int64_t G, const double *x, const double *ell,
                const double *w, const double *B, const double *C,
                const double *D, const double *h0, double *y,
                double *h_final, int nthreads)
{
    if (!dims_ok(batch, L, H, P, N, G)) return ORACLE_BAD_ARG;
    if ((L > 0 && (!x || !ell || !w || !B || !C || !y))) return ORACLE_BAD_ARG;
    const int64_t hpg = H / G;
    int err = ORACLE_OK;
    set_threads(nthreads);
#pragma omp parallel
    {
        double *hs = (double *)malloc((size_t)(P * N) * sizeof(double));
        if (!hs) {
#pragma omp atomic write
            err = ORACLE_NO_MEMORY;
        }
#pragma omp for schedule(dynamic, 1)
        for (int64_t lane = 0; lane < batch * H; ++lane) {
            if (!hs) continue;
            const int64_t b = lane / H, h = lane % H, g = h / hpg;
            scan_lane(L, P, N,
                      x + (b * L * H + h) * P, H * P,
                      ell + b * L * H + h, w + b * L * H + h, H,
                      B + (b * L * G + g) * N, C + (b * L * G + g) * N, G * N,
                      D ? D[h] : 0.0,
                      h0 ? h0 + (b * H + h) * P * N : NULL,
                      y + (b * L * H + h) * P, H * P,
                      h_final ? h_final + (b * H + h) * P * N : NULL, hs);
        }
        free(hs);
    }
    return err;
}

/*
 * The layer's forward pass: the recurrence with a_t = exp(dt_t * A_h)
 * ([Mamba-disc]: A_bar = exp(Delta A)) and input weight w_t = dt_t.
 * dt is taken as given (already positive; no bias or softplus applied here).
 */
int oracle_ssd_forward(int64_t batch, int64_t L, int64_t H, int64_t P,
                       int64_t N, int64_t G, const double *x, const double *dt,
                       const double *A, const double *B, const double *C,
                       const double *D, const double *h0, double *y,
                       double *h_final, int nthreads)
{
    if (!dims_ok(batch, L, H, P, N, G) || !A) return ORACLE_BAD_ARG;
    if (L > 0 && !dt) return ORACLE_BAD_ARG;
    const int64_t n_ell = batch * L * H;
    double *ell = (double *)malloc((size_t)(n_ell > 0 ? n_ell : 1) * sizeof(double));
    if (!ell) return ORACLE_NO_MEMORY;
    for (int64_t i = 0; i < n_ell; ++i) ell[i] = dt[i] * A[i % H];
    int rc = oracle_scan(batch, L, H, P, N, G, x, ell, dt, B, C, D, h0, y,
                         h_final, nthreads);
    free(ell);
    return rc;
}

/*
 * Step preparation of the layer's options, element by element over a
 * (batch, L, H) array of raw steps:
 *   dt  = raw + bias[h]                       (bias NULL: none)
 *   dt  = softplus(dt) = log(1 + exp(dt))     when `softplus` ([Mamba-sel])
 *   dt  = min(max(dt, dt_min), dt_max)        when dt_max > 0
 *   ell = dt * A[h]                           (a_t = exp(ell), [Mamba-disc])
 *   w   = dt                                  Euler input weight, or with
 *   w   = (exp(dt A) - 1) / A                 `zoh`: the zero-order hold
 *                                             B_bar = (dt A)^-1 (exp(dt A) - 1) dt B
 *                                             for a scalar A ([Mamba-disc]);
 *                                             w = dt when A = 0 (its limit).
 * softplus is evaluated as max(v, 0) + log1p(exp(-|v|)), the same function
 * written so that exp cannot overflow; expm1 gives exp(dt A) - 1 without
 * cancellation.
 */
int oracle_dt_prepare(int64_t batch, int64_t L, int64_t H, const double *raw,
                      const double *A, const double *bias, int softplus,
                      double dt_min, double dt_max, int zoh, double *dt_out,
                      double *ell, double *w)
{
    if (batch < 0 || L < 0 || H < 1 || !A) return ORACLE_BAD_ARG;
    const int64_t n = batch * L * H;
    if (n > 0 && (!raw || !ell || !w)) return ORACLE_BAD_ARG;
    for (int64_t i = 0; i < n; ++i) {
        const int64_t h = i % H;
        double dt = raw[i] + (bias ? bias[h] : 0.0);
        if (softplus) dt = fmax(dt, 0.0) + log1p(exp(-fabs(dt)));
        if (dt_max > 0.0) dt = fmin(fmax(dt, dt_min), dt_max);
        if (dt_out) dt_out[i] = dt;
        ell[i] = dt * A[h];
        w[i] = (zoh && A[h] != 0.0) ? expm1(dt * A[h]) / A[h] : dt;
    }
    return ORACLE_OK;
}

/*
 * The layer's forward pass with the step options of oracle_dt_prepare:
 * the recurrence on the prepared ell and w. With no bias, no softplus, no
 * clamp and Euler weights this is oracle_ssd_forward.
 */
int oracle_ssd_forward_ex(int64_t batch, int64_t L, int64_t H, int64_t P,
                          int64_t N, int64_t G, const double *x,
                          const double *dt_raw, const double *A,
                          const double *B, const double *C, const double *D,
                          const double *h0, const double *bias, int softplus,
                          double dt_min, double dt_max, int zoh, double *y,
                          double *h_final, int nthreads)
{
    if (!dims_ok(batch, L, H, P, N, G) || !A) return ORACLE_BAD_ARG;
    if (L > 0 && !dt_raw) return ORACLE_BAD_ARG;
    const int64_t n = batch * L * H;
    double *ell = (double *)malloc((size_t)(n > 0 ? n : 1) * sizeof(double));
    double *w = (double *)malloc((size_t)(n > 0 ? n : 1) * sizeof(double));
    int rc = ORACLE_NO_MEMORY;
    if (ell && w) {
        rc = oracle_dt_prepare(batch, L, H, dt_raw, A, bias, softplus, dt_min,
                               dt_max, zoh, NULL, ell, w);
        if (rc == ORACLE_OK)
            rc = oracle_scan(batch, L, H, P, N, G, x, ell, w, B, C, D, h0, y,
                             h_final, nthreads);
    }
    free(ell);
    free(w);
    return rc;
}

/*
 * One decode step: exactly one iteration of the loop body above, applied to
 * the state h in place. x (batch,H,P), dt (batch,H), B/C (batch,G,N),
 * y (batch,H,P), h (batch,H,P,N).
 */
int oracle_ssd_step(int64_t batch, int64_t H, int64_t P, int64_t N, int64_t G,
                    double *h, const double *x, const double *dt,
                    const double *A, const double *B, const double *C,
                    const double *D, double *y, int nthreads)
{
    if (!dims_ok(batch, 1, H, P, N, G) || !h || !A) return ORACLE_BAD_ARG;
    const int64_t hpg = H / G;
    set_threads(nthreads);
#pragma omp parallel for schedule(static)
    for (int64_t lane = 0; lane < batch * H; ++lane) {
        const int64_t b = lane / H, hh = lane % H, g = hh / hpg;
        const double a = exp(dt[lane] * A[hh]);
        const double wt = dt[lane];
        const double *Bt = B + (b * G + g) * N;
        const double *Ct = C + (b * G + g) * N;
        double *hl = h + lane * P * N;
        for (int64_t p = 0; p < P; ++p) {
            const double xp = x[lane * P + p];
            double *hp = hl + p * N;
            double acc = 0.0;
            for (int64_t n = 0; n < N; ++n) {
                hp[n] = a * hp[n] + wt * xp * Bt[n];
                acc += Ct[n] * hp[n];
            }
            y[lane * P + p] = acc + (D ? D[hh] : 0.0) * xp;
        }
    }
    return ORACLE_OK;
}

/*
 * One decode step with the step options of oracle_dt_prepare: the loop body
 * of the recurrence with a = exp(ell), input weight w, applied to h in place.
 */
int oracle_ssd_step_ex(int64_t batch, int64_t H, int64_t P, int64_t N,
                       int64_t G, double *h, const double *x,
                       const double *dt_raw, const double *A, const double *B,
                       const double *C, const double *D, const double *bias,
                       int softplus, double dt_min, double dt_max, int zoh,
                       double *y, int nthreads)
{
    if (!dims_ok(batch, 1, H, P, N, G) || !h || !A || !dt_raw) return ORACLE_BAD_ARG;
    const int64_t hpg = H / G;
    double *ell = (double *)malloc((size_t)(batch * H) * sizeof(double));
    double *w = (double *)malloc((size_t)(batch * H) * sizeof(double));
    int rc = ORACLE_NO_MEMORY;
    if (ell && w)
        rc = oracle_dt_prepare(batch, 1, H, dt_raw, A, bias, softplus, dt_min,
                               dt_max, zoh, NULL, ell, w);
    if (rc == ORACLE_OK) {
        set_threads(nthreads);
#pragma omp parallel for schedule(static)
        for (int64_t lane = 0; lane < batch * H; ++lane) {
            const int64_t b = lane / H, hh = lane % H, g = hh / hpg;
            const double a = exp(ell[lane]);
            const double wt = w[lane];
            const double *Bt = B + (b * G + g) * N;
            const double *Ct = C + (b * G + g) * N;
            double *hl = h + lane * P * N;
            for (int64_t p = 0; p < P; ++p) {
                const double xp = x[lane * P + p];
                double *hp = hl + p * N;
                double acc = 0.0;
                for (int64_t n = 0; n < N; ++n) {
                    hp[n] = a * hp[n] + wt * xp * Bt[n];
                    acc += Ct[n] * hp[n];
                }
                y[lane * P + p] = acc + (D ? D[hh] : 0.0) * xp;
            }
        }
    }
    free(ell);
    free(w);
    return rc;
}

/*
 * segsum of a lane's log-decays: sum_{k=s+1..t} ell_k for t >= s. The decay
 * mask entry L_ts = a_t x ... x a_{s+1} = exp(segsum(t, s)) ([M2-scalar]);
 * L_tt = 1.
 */
static double segsum(const double *ell, int64_t sa, int64_t t, int64_t s)
{
    double acc = 0.0;
    for (int64_t k = s + 1; k <= t; ++k) acc += ell[k * sa];
    return acc;
}

/*
 * The sequence-transformation matrix of one (b,h) lane ([M2-matrix],
 * [M2-scalar]): M_ts = L_ts * (C_t . B_s) * w_s for s <= t, 0 above the
 * diagonal. M is L x L, row-major. ell, w have time stride `sa`; B, C have
 * time stride `sb` and point at the lane's group.
 */
static void lane_matrix(int64_t L, int64_t N, const double *ell,
                        const double *w, int64_t sa, const double *Bg,
                        const double *Cg, int64_t sb, double *M)
{
    for (int64_t t = 0; t < L; ++t) {
        for (int64_t s = 0; s < L; ++s) {
            if (s > t) { M[t * L + s] = 0.0; continue; }
            double cb = 0.0;
            for (int64_t n = 0; n < N; ++n) cb += Cg[t * sb + n] * Bg[s * sb + n];
            M[t * L + s] = exp(segsum(ell, sa, t, s)) * cb * w[s * sa];
        }
    }
}

/* Public: M for lane (b,h) of the general (ell, w) problem. */
int oracle_matrix(int64_t batch, int64_t L, int64_t H, int64_t N, int64_t G,
                  int64_t b, int64_t h, const double *ell, const double *w,
                  const double *B, const double *C, double *M)
{
    if (!dims_ok(batch, L, H, 1, N, G) || b < 0 || b >= batch || h < 0 || h >= H)
        return ORACLE_BAD_ARG;
    const int64_t g = h / (H / G);
    lane_matrix(L, N, ell + b * L * H + h, w + b * L * H + h, H,
                B + (b * L * G + g) * N, C + (b * L * G + g) * N, G * N, M);
    return ORACLE_OK;
}

/*
 * Brute-force quadratic ("attention") form, an independent second route to
 * the same result ([M2-scalar], [M2-example] second half): y = M x per lane
 * and head-dim column, plus the initial state's contribution, which reaches
 * token t through a_t ... a_0 = exp(sum_{k<=t} ell_k), plus the skip term:
 *
 *   y_t[p] = sum_{s<=t} M_ts x_s[p]
 *          + exp(sum_{k=0..t} ell_k) * sum_n C_t[n] h0[p][n]
 *          + D x_t[p]
 *   h_final[p][n] = exp(sum_{k=0..L-1} ell_k) h0[p][n]
 *          + sum_s exp(segsum(L-1, s)) w_s x_s[p] B_s[n]
 *
 * Materialises L x L per lane: tiny inputs only.
 */
int oracle_quadratic(int64_t batch, int64_t L, int64_t H, int64_t P, int64_t N,
                     int64_t G, const double *x, const double *ell,
                     const double *w, const double *B, const double *C,
                     const double *D, const double *h0, double *y,
                     double *h_final, int nthreads)
{
    if (!dims_ok(batch, L, H, P, N, G)) return ORACLE_BAD_ARG;
    const int64_t hpg = H / G;
    int err = ORACLE_OK;
    set_threads(nthreads);
#pragma omp parallel
    {
        double *M = (double *)malloc((size_t)(L * L > 0 ? L * L : 1) * sizeof(double));
        if (!M) {
#pragma omp atomic write
            err = ORACLE_NO_MEMORY;
        }
#pragma omp for schedule(dynamic, 1)
        for (int64_t lane = 0; lane < batch * H; ++lane) {
            if (!M) continue;
            const int64_t b = lane / H, h = lane % H, g = h / hpg;
            const double *el = ell + b * L * H + h;
            const double *wl = w + b * L * H + h;
            const double *Bg = B + (b * L * G + g) * N;
            const double *Cg = C + (b * L * G + g) * N;
            const double *xl = x + (b * L * H + h) * P;
            const double *h0l = h0 ? h0 + lane * P * N : NULL;
            double *yl = y + (b * L * H + h) * P;
            lane_matrix(L, N, el, wl, H, Bg, Cg, G * N, M);
            for (int64_t t = 0; t < L; ++t) {
                const double carry = exp(segsum(el, H, t, -1));
                for (int64_t p = 0; p < P; ++p) {
                    double acc = 0.0;
                    for (int64_t s = 0; s <= t; ++s) acc += M[t * L + s] * xl[s * H * P + p];
                    if (h0l) {
                        double ch = 0.0;
                        for (int64_t n = 0; n < N; ++n) ch += Cg[t * G * N + n] * h0l[p * N + n];
                        acc += carry * ch;
                    }
                    yl[t * H * P + p] = acc + (D ? D[h] : 0.0) * xl[t * H * P + p];
                }
            }
            if (h_final) {
                double *hf = h_final + lane * P * N;
                const double carry = exp(segsum(el, H, L - 1, -1));
                for (int64_t p = 0; p < P; ++p)
                    for (int64_t n = 0; n < N; ++n) {
                        double acc = h0l ? carry * h0l[p * N + n] : 0.0;
                        for (int64_t s = 0; s < L; ++s)
                            acc += exp(segsum(el, H, L - 1, s)) * wl[s * H] *
                                   xl[s * H * P + p] * Bg[s * G * N + n];
                        hf[p * N + n] = acc;
                    }
            }
        }
        free(M);
    }
    return err;
}

/*
 * Chunked (block-decomposed) form [M2-chunks], in the pages' four steps, fp64:
 *
 *  chunk c covers tokens [cQ, min(cQ+Q, L)); the last chunk may be short.
 *  (1) diagonal block:  Ydiag_t = sum_{s in c, s<=t} exp(segsum(t,s)) (C_t.B_s) w_s x_s
 *  (2) chunk state (input->state):
 *        S_c = sum_{s in c} exp(segsum(end_c, s)) w_s x_s (x) B_s
 *  (3) state passing (state->state), only block-end states cross blocks:
 *        H_0 = h0;  H_{c+1} = exp(sum_{k in c} ell_k) H_c + S_c;  h_final = H_nc
 *  (4) state->output:
 *        Yoff_t = exp(sum_{k=start_c..t} ell_k) C_t . H_c
 *  y = Ydiag + Yoff + D x.
 *
 * Optional per-stage outputs for debugging kernels (NULL to skip):
 *   S_out (batch,H,nc,P,N): S_c;  Hs_out (batch,H,nc,P,N): H_c (state entering c).
 */
int oracle_chunked(int64_t batch, int64_t L, int64_t H, int64_t P, int64_t N,
                   int64_t G, int64_t Q, const double *x, const double *ell,
                   const double *w, const double *B, const double *C,
                   const double *D, const double *h0, double *y,
                   double *h_final, double *S_out, double *Hs_out,
                   int nthreads)
{
    if (!dims_ok(batch, L, H, P, N, G) || Q < 1) return ORACLE_BAD_ARG;
    const int64_t hpg = H / G;
    const int64_t nc = (L + Q - 1) / Q;
    int err = ORACLE_OK;
    set_threads(nthreads);
#pragma omp parallel
    {
        double *Hc = (double *)malloc((size_t)(P * N) * sizeof(double));
        double *Sc = (double *)malloc((size_t)(P * N) * sizeof(double));
        if (!Hc || !Sc) {
#pragma omp atomic write
            err = ORACLE_NO_MEMORY;
        }
#pragma omp for schedule(dynamic, 1)
        for (int64_t lane = 0; lane < batch * H; ++lane) {
            if (!Hc || !Sc) continue;
            const int64_t b = lane / H, h = lane % H, g = h / hpg;
            const double *el = ell + b * L * H + h;
            const double *wl = w + b * L * H + h;
            const double *Bg = B + (b * L * G + g) * N;
            const double *Cg = C + (b * L * G + g) * N;
            const double *xl = x + (b * L * H + h) * P;
            double *yl = y + (b * L * H + h) * P;
            const int64_t sa = H, sb = G * N, sx = H * P;
            if (h0) memcpy(Hc, h0 + lane * P * N, (size_t)(P * N) * sizeof(double));
            else memset(Hc, 0, (size_t)(P * N) * sizeof(double));
            for (int64_t c = 0; c < nc; ++c) {
                const int64_t t0 = c * Q;
                const int64_t t1 = (t0 + Q < L) ? t0 + Q : L;
                if (Hs_out) memcpy(Hs_out + (lane * nc + c) * P * N, Hc,
                                   (size_t)(P * N) * sizeof(double));
                /* (1) diagonal block and (4) state->output */
                for (int64_t t = t0; t < t1; ++t) {
                    const double into = exp(segsum(el, sa, t, t0 - 1));
                    for (int64_t p = 0; p < P; ++p) {
                        double yd = 0.0;
                        for (int64_t s = t0; s <= t; ++s) {
                            double cb = 0.0;
                            for (int64_t n = 0; n < N; ++n) cb += Cg[t * sb + n] * Bg[s * sb + n];
                            yd += exp(segsum(el, sa, t, s)) * cb * wl[s * sa] * xl[s * sx + p];
                        }
                        double yo = 0.0;
                        for (int64_t n = 0; n < N; ++n) yo += Cg[t * sb + n] * Hc[p * N + n];
                        yl[t * sx + p] = yd + into * yo + (D ? D[h] : 0.0) * xl[t * sx + p];
                    }
                }
                /* (2) chunk state */
                for (int64_t p = 0; p < P; ++p)
                    for (int64_t n = 0; n < N; ++n) {
                        double acc = 0.0;
                        for (int64_t s = t0; s < t1; ++s)
                            acc += exp(segsum(el, sa, t1 - 1, s)) * wl[s * sa] *
                                   xl[s * sx + p] * Bg[s * sb + n];
                        Sc[p * N + n] = acc;
                    }
                if (S_out) memcpy(S_out + (lane * nc + c) * P * N, Sc,
                                  (size_t)(P * N) * sizeof(double));
                /* (3) state passing */
                const double total = exp(segsum(el, sa, t1 - 1, t0 - 1));
                for (int64_t i = 0; i < P * N; ++i) Hc[i] = total * Hc[i] + Sc[i];
            }
            if (h_final) memcpy(h_final + lane * P * N, Hc, (size_t)(P * N) * sizeof(double));
        }
        free(Hc);
        free(Sc);
    }
    return err;
}

/*
 * The selective scan of "精读笔记 #12：Mamba" (llm-papers-study), sections 2.2
 * and 3 (algorithm 2), the prior art the Mamba-2 pages compare SSD with:
 * every channel d (of D) carries its own N-vector state with a DIAGONAL
 * A[d][n]; the step dt is per (token, channel), B and C per token (shared by
 * the D/G channels of a group). Steps are prepared as in oracle_dt_prepare
 * (bias per channel, softplus, clamp); the decay of state n is
 * exp(dt A[d][n]) and its input weight dt (Euler) or, with `zoh`, the
 * zero-order hold (exp(dt A[d][n]) - 1) / A[d][n] (dt where A = 0):
 *
 *   h[n] = exp(dt A[d][n]) h[n] + w[n] x[t][d] B[t][g][n]
 *   y[t][d] = sum_n C[t][g][n] h[n] + Dskip[d] x[t][d]
 *
 * x, dt, y (batch, L, D); A (D, N); B, C (batch, L, G, N); Dskip (D) or NULL;
 * h0, h_final (batch, D, N) or NULL; bias (D) or NULL.
 */
int oracle_selective_scan(int64_t batch, int64_t L, int64_t D, int64_t N,
                          int64_t G, const double *x, const double *dt_raw,
                          const double *A, const double *B, const double *C,
                          const double *Dskip, const double *h0,
                          const double *bias, int softplus, double dt_min,
                          double dt_max, int zoh, double *y, double *h_final,
                          int nthreads)
{
    if (batch < 0 || L < 0 || D < 1 || N < 1 || G < 1 || D % G != 0 || !A)
        return ORACLE_BAD_ARG;
    if (L > 0 && (!x || !dt_raw || !B || !C || !y)) return ORACLE_BAD_ARG;
    const int64_t dpg = D / G;
    int err = ORACLE_OK;
    set_threads(nthreads);
#pragma omp parallel
    {
        double *h = (double *)malloc((size_t)N * sizeof(double));
        if (!h) {
#pragma omp atomic write
            err = ORACLE_NO_MEMORY;
        }
#pragma omp for schedule(dynamic, 4)
        for (int64_t lane = 0; lane < batch * D; ++lane) {
            if (!h) continue;
            const int64_t b = lane / D, d = lane % D, g = d / dpg;
            for (int64_t n = 0; n < N; ++n) h[n] = h0 ? h0[lane * N + n] : 0.0;
            for (int64_t t = 0; t < L; ++t) {
                const int64_t i = (b * L + t) * D + d;
                double v = dt_raw[i] + (bias ? bias[d] : 0.0);
                if (softplus) v = fmax(v, 0.0) + log1p(exp(-fabs(v)));
                if (dt_max > 0.0) v = fmin(fmax(v, dt_min), dt_max);
                const double *Bt = B + ((b * L + t) * G + g) * N;
                const double *Ct = C + ((b * L + t) * G + g) * N;
                double acc = 0.0;
                for (int64_t n = 0; n < N; ++n) {
                    const double Adn = A[d * N + n];
                    const double a = exp(v * Adn);
                    const double w = (zoh && Adn != 0.0) ? expm1(v * Adn) / Adn : v;
                    h[n] = a * h[n] + w * x[i] * Bt[n];
                    acc += Ct[n] * h[n];
                }
                y[i] = acc + (Dskip ? Dskip[d] : 0.0) * x[i];
            }
            if (h_final)
                for (int64_t n = 0; n < N; ++n) h_final[lane * N + n] = h[n];
        }
        free(h);
    }
    return err;
}

/*
 * Backward pass of the layer (the plain forward: a_t = exp(dt_t A_h), input
 * weight dt_t), by the exact adjoint of the recurrence, token by token in
 * reverse ("精读笔记 #12：Mamba", section 3.3: the intermediate states are
 * recomputed for the backward pass rather than stored by the forward; here
 * they are recomputed by a forward sweep of each lane). For the scalar loss
 * sum_t dy_t . y_t + sum dh_final . h_final it returns
 *   dx, ddt (batch, L, H), dA (H), dB, dC (batch, L, G, N), dD (H), dh0.
 * Per lane, with g the gradient with respect to the current state:
 *   g = dh_final; for t = L-1 .. 0:
 *     g += dy_t (x) C_t                       (y_t = C_t . h_t)
 *     dC_t += dy_t^T h_t;  dD += dy_t . x_t;  dx_t = D dy_t + dt_t g B_t
 *     dB_t += dt_t g^T x_t
 *     ddt_t = sum g o (x_t (x) B_t + A a_t h_{t-1});  dA += dt_t sum g o a_t h_{t-1}
 *     g = a_t g
 *   dh0 = g
 * dB, dC, dA, dD are sums over the lanes that share them. Any of the
 * outputs may be NULL; dh_final and h0 may be NULL (zeros).
 */
int oracle_ssd_backward(int64_t batch, int64_t L, int64_t H, int64_t P, int64_t N,
                        int64_t G, const double *x, const double *dt,
                        const double *A, const double *B, const double *C,
                        const double *D, const double *h0, const double *dy,
                        const double *dh_final, double *dx, double *ddt,
                        double *dA, double *dB, double *dC, double *dD,
                        double *dh0)
{
    if (!dims_ok(batch, L, H, P, N, G) || !A) return ORACLE_BAD_ARG;
    if (L > 0 && (!x || !dt || !B || !C || !dy)) return ORACLE_BAD_ARG;
    const int64_t hpg = H / G, PN = P * N;
    double *hs = (double *)malloc((size_t)((L + 1) * PN) * sizeof(double));
    double *g = (double *)malloc((size_t)PN * sizeof(double));
    if (!hs || !g) {
        free(hs);
        free(g);
        return ORACLE_NO_MEMORY;
    }
    if (dB) memset(dB, 0, (size_t)(batch * L * G * N) * sizeof(double));
    if (dC) memset(dC, 0, (size_t)(batch * L * G * N) * sizeof(double));
    if (dA) memset(dA, 0, (size_t)H * sizeof(double));
    if (dD) memset(dD, 0, (size_t)H * sizeof(double));
    for (int64_t b = 0; b < batch; ++b) {
        for (int64_t h = 0; h < H; ++h) {
            const int64_t gr = h / hpg;
            const double Ah = A[h], Dh = D ? D[h] : 0.0;
            /* forward sweep: hs[t + 1] = state after token t, hs[0] = h0 */
            for (int64_t i = 0; i < PN; ++i) hs[i] = h0 ? h0[(b * H + h) * PN + i] : 0.0;
            for (int64_t t = 0; t < L; ++t) {
                const double dtt = dt[(b * L + t) * H + h];
                const double a = exp(dtt * Ah);
                const double *xt = x + ((b * L + t) * H + h) * P;
                const double *Bt = B + ((b * L + t) * G + gr) * N;
                for (int64_t p = 0; p < P; ++p)
                    for (int64_t n = 0; n < N; ++n)
                        hs[(t + 1) * PN + p * N + n] =
                            a * hs[t * PN + p * N + n] + dtt * xt[p] * Bt[n];
            }
            for (int64_t i = 0; i < PN; ++i) g[i] = dh_final ? dh_final[(b * H + h) * PN + i] : 0.0;
            for (int64_t t = L - 1; t >= 0; --t) {
                const double dtt = dt[(b * L + t) * H + h];
                const double a = exp(dtt * Ah);
                const double *xt = x + ((b * L + t) * H + h) * P;
                const double *yt = dy + ((b * L + t) * H + h) * P;
                const double *Bt = B + ((b * L + t) * G + gr) * N;
                const double *Ct = C + ((b * L + t) * G + gr) * N;
                const double *ht = hs + (t + 1) * PN, *hp = hs + t * PN;
                for (int64_t p = 0; p < P; ++p)
                    for (int64_t n = 0; n < N; ++n) g[p * N + n] += yt[p] * Ct[n];
                if (dC)
                    for (int64_t n = 0; n < N; ++n) {
                        double acc = 0.0;
                        for (int64_t p = 0; p < P; ++p) acc += yt[p] * ht[p * N + n];
                        dC[((b * L + t) * G + gr) * N + n] += acc;
                    }
                if (dD)
                    for (int64_t p = 0; p < P; ++p) dD[h] += yt[p] * xt[p];
                if (dx)
                    for (int64_t p = 0; p < P; ++p) {
                        double acc = 0.0;
                        for (int64_t n = 0; n < N; ++n) acc += g[p * N + n] * Bt[n];
                        dx[((b * L + t) * H + h) * P + p] = Dh * yt[p] + dtt * acc;
                    }
                if (dB)
                    for (int64_t n = 0; n < N; ++n) {
                        double acc = 0.0;
                        for (int64_t p = 0; p < P; ++p) acc += g[p * N + n] * xt[p];
                        dB[((b * L + t) * G + gr) * N + n] += dtt * acc;
                    }
                double s_in = 0.0, s_dec = 0.0;
                for (int64_t p = 0; p < P; ++p)
                    for (int64_t n = 0; n < N; ++n) {
                        s_in += g[p * N + n] * xt[p] * Bt[n];
                        s_dec += g[p * N + n] * a * hp[p * N + n];
                    }
                if (ddt) ddt[(b * L + t) * H + h] = s_in + Ah * s_dec;
                if (dA) dA[h] += dtt * s_dec;
                for (int64_t i = 0; i < PN; ++i) g[i] *= a;
            }
            if (dh0)
                for (int64_t i = 0; i < PN; ++i) dh0[(b * H + h) * PN + i] = g[i];
        }
    }
    free(hs);
    free(g);
    return ORACLE_OK;
}

/*
 * m3_oracle.c -- plain, slow, fp64 CPU oracle of the Mamba-3 SSM layer scan.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and
 * bench.py's cpu_baseline / reference leg may load this library.  The product
 * path (selective_state_space_m3_b200) never links, imports or calls it, and
 * this file shares no code, header, table or constant with the CUDA sources.
 *
 * What it computes (all in double precision, token by token, no chunking,
 * no reordering beyond the loops written below):
 *
 *   For every batch b and head h (group g = h / (H/G)):
 *     alpha_t = exp(dt_t * A_h)
 *     beta_t  = (1 - lambda_t) * dt_t * exp(dt_t * A_h)
 *     gamma_t = lambda_t * dt_t
 *       -- "Mamba-3" summary (b-lab.team), section 1 "Exponential-Trapezoidal
 *          Discretization": the recurrence and the definitions of alpha, beta,
 *          gamma.
 *     R_t = blockdiag_i R(dt_t * theta_t[i]),  R(phi) = [[cos,-sin],[sin,cos]]
 *       -- same page, section 2 "Complex-Valued State Space Model"
 *          (Proposition 2), the 2x2 rotation blocks.
 *     h_t = R_t (alpha_t h_{t-1} + beta_t B_{t-1} X_{t-1}^T) + gamma_t B_t X_t^T
 *     y_t = C_t^T h_t                          (R x P per head: MIMO, section 3)
 *
 *   Reading (the pages never print the trapezoid and the rotation together):
 *   the rotation R_t multiplies the whole t-1 -> t transition, i.e. both the
 *   carried state and the beta term, because beta carries exp(dt A), which
 *   for the complex SSM is exp(dt (A + i theta)).  This is the reading under
 *   which Proposition 3 (data-dependent RoPE on B and C) holds with every B_s
 *   rotated by its own cumulative phase.
 *
 * Two transition variants follow the main scan further down:
 * oracle_scan_damped (damping regimes: the rotation block of every pair
 * replaced by the critically damped shear or the overdamped hyperbolic
 * block, same input rule) and oracle_scan_reflect (a rank-one Householder
 * reflection added to the diagonal part of the transition).  Their readings
 * are stated above each.
 *
 * Layouts (row-major, innermost last):
 *   x      [b][t][h][r][p]        y      [b][t][h][r][p]
 *   B, C   [b][t][g][r][n]        theta  [b][t][g][N/2]
 *   dt,lam [b][t][h]              A      [h]
 *   carry: h [b][h][n][p], prev_B [b][h][r][n], prev_x [b][h][r][p]
 *   Rotary pair i occupies state rows (2i, 2i+1).
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    int batch, seqlen, nheads, ngroups, headdim, dstate, rank;
} oracle_dims;

static int dims_ok(const oracle_dims* d)
{
    if (!d) return 0;
    if (d->batch < 0 || d->seqlen < 0 || d->nheads <= 0 || d->ngroups <= 0) return 0;
    if (d->headdim <= 0 || d->dstate <= 0 || d->rank <= 0) return 0;
    if (d->dstate % 2 != 0) return 0;
    if (d->nheads % d->ngroups != 0) return 0;
    return 1;
}

/* One token of the recurrence for one (b, h), in the original frame.
 * H: N*P state, PB: R*N previous B (stored [r][n]), PX: R*P previous x.
 * xt: R*P, Bt/Ct: R*N, th: N/2, yt: R*P (output). */
static void step_bh(int N, int P, int R,
                    double* H, double* PB, double* PX,
                    const double* xt, const double* Bt, const double* Ct,
                    double d, double a, double lam, const double* th,
                    double* yt)
{
    const double alpha = exp(d * a);
    const double beta = (1.0 - lam) * d * exp(d * a);
    const double gamma = lam * d;

    /* carried part: alpha h + beta * B_{t-1} X_{t-1}^T */
    for (int n = 0; n < N; ++n)
        for (int p = 0; p < P; ++p) {
            double bx = 0.0;
            for (int r = 0; r < R; ++r) bx += PB[r * N + n] * PX[r * P + p];
            H[n * P + p] = alpha * H[n * P + p] + beta * bx;
        }

    /* rotation R_t on every pair (2i, 2i+1), every column p */
    for (int i = 0; i < N / 2; ++i) {
        const double phi = d * th[i];
        const double c = cos(phi), s = sin(phi);
        for (int p = 0; p < P; ++p) {
            const double u0 = H[(2 * i) * P + p];
            const double u1 = H[(2 * i + 1) * P + p];
            H[(2 * i) * P + p] = c * u0 - s * u1;
            H[(2 * i + 1) * P + p] = s * u0 + c * u1;
        }
    }

    /* current input: + gamma * B_t X_t^T */
    for (int n = 0; n < N; ++n)
        for (int p = 0; p < P; ++p) {
            double bx = 0.0;
            for (int r = 0; r < R; ++r) bx += Bt[r * N + n] * xt[r * P + p];
            H[n * P + p] += gamma * bx;
        }

    /* readout y_t = C_t^T h_t : [r][p] */
    for (int r = 0; r < R; ++r)
        for (int p = 0; p < P; ++p) {
            double acc = 0.0;
            for (int n = 0; n < N; ++n) acc += Ct[r * N + n] * H[n * P + p];
            yt[r * P + p] = acc;
        }

    /* the next step's beta term needs this step's (B, x) */
    memcpy(PB, Bt, sizeof(double) * (size_t)R * N);
    memcpy(PX, xt, sizeof(double) * (size_t)R * P);
}

/* Full sequence.  init_h / init_pB / init_pX may be NULL (zeros).
 * y must hold batch*seqlen*H*R*P doubles.  out_h / out_pB / out_pX may be NULL.
 * Returns 0 on success, -1 on bad arguments. */
int oracle_scan(const oracle_dims* d,
                const double* x, const double* B, const double* C,
                const double* dt, const double* A, const double* lam,
                const double* theta,
                const double* init_h, const double* init_pB, const double* init_pX,
                double* y, double* out_h, double* out_pB, double* out_pX)
{
    if (!dims_ok(d) || !x || !B || !C || !dt || !A || !lam || !theta || !y) return -1;
    const int Bn = d->batch, L = d->seqlen, H = d->nheads, G = d->ngroups;
    const int P = d->headdim, N = d->dstate, R = d->rank;
    const int hpg = H / G;

#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int b = 0; b < Bn; ++b)
        for (int h = 0; h < H; ++h) {
            const int g = h / hpg;
            double* Hs = (double*)calloc((size_t)N * P, sizeof(double));
            double* PB = (double*)calloc((size_t)R * N, sizeof(double));
            double* PX = (double*)calloc((size_t)R * P, sizeof(double));
            const size_t bh = (size_t)b * H + h;
            if (init_h) memcpy(Hs, init_h + bh * N * P, sizeof(double) * (size_t)N * P);
            if (init_pB) memcpy(PB, init_pB + bh * R * N, sizeof(double) * (size_t)R * N);
            if (init_pX) memcpy(PX, init_pX + bh * R * P, sizeof(double) * (size_t)R * P);
            for (int t = 0; t < L; ++t) {
                const size_t bt = (size_t)b * L + t;
                const double* xt = x + ((bt * H + h) * R) * P;
                const double* Bt = B + ((bt * G + g) * R) * N;
                const double* Ct = C + ((bt * G + g) * R) * N;
                const double* th = theta + (bt * G + g) * (N / 2);
                double* yt = y + ((bt * H + h) * R) * P;
                step_bh(N, P, R, Hs, PB, PX, xt, Bt, Ct,
                        dt[bt * H + h], A[h], lam[bt * H + h], th, yt);
            }
            if (out_h) memcpy(out_h + bh * N * P, Hs, sizeof(double) * (size_t)N * P);
            if (out_pB) memcpy(out_pB + bh * R * N, PB, sizeof(double) * (size_t)R * N);
            if (out_pX) memcpy(out_pX + bh * R * P, PX, sizeof(double) * (size_t)R * P);
            free(Hs); free(PB); free(PX);
        }
    return 0;
}

/* One decode token for every (b, h): the carry (h, prev_B, prev_x) is updated
 * in place.  Per-token layouts: x [b][h][r][p], B/C [b][g][r][n],
 * theta [b][g][N/2], dt/lam [b][h], y [b][h][r][p].  d->seqlen is ignored. */
int oracle_step(const oracle_dims* d,
                double* h_state, double* prev_B, double* prev_x,
                const double* x, const double* B, const double* C,
                const double* dt, const double* A, const double* lam,
                const double* theta, double* y)
{
    if (!dims_ok(d) || !h_state || !prev_B || !prev_x || !x || !B || !C ||
        !dt || !A || !lam || !theta || !y) return -1;
    const int Bn = d->batch, H = d->nheads, G = d->ngroups;
    const int P = d->headdim, N = d->dstate, R = d->rank;
    const int hpg = H / G;

#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int b = 0; b < Bn; ++b)
        for (int h = 0; h < H; ++h) {
            const int g = h / hpg;
            const size_t bh = (size_t)b * H + h;
            const size_t bg = (size_t)b * G + g;
            step_bh(N, P, R, h_state + bh * N * P, prev_B + bh * R * N, prev_x + bh * R * P,
                    x + bh * R * P, B + bg * R * N, C + bg * R * N,
                    dt[bh], A[h], lam[bh], theta + bg * (N / 2), y + bh * R * P);
        }
    return 0;
}

/* Cumulative phase and rotated B, C (the "RoPE trick", Proposition 3 of the
 * same page):  Phi_t[i] = sum_{s<=t} dt_s theta_s[i]  (per head, since dt is),
 *   (Bt_{2i}, Bt_{2i+1}) = R(Phi_t[i])^T (B_{2i}, B_{2i+1})
 *                        = ( cos*B_{2i} + sin*B_{2i+1}, -sin*B_{2i} + cos*B_{2i+1} ).
 * Outputs: B_rot, C_rot [b][t][h][r][n]; phase [b][t][h][N/2] (unreduced,
 * may be NULL). */
int oracle_rope_bc(const oracle_dims* d,
                   const double* B, const double* C, const double* dt,
                   const double* theta, double* B_rot, double* C_rot, double* phase)
{
    if (!dims_ok(d) || !B || !C || !dt || !theta || !B_rot || !C_rot) return -1;
    const int Bn = d->batch, L = d->seqlen, H = d->nheads, G = d->ngroups;
    const int N = d->dstate, R = d->rank, hpg = H / G;

#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int b = 0; b < Bn; ++b)
        for (int h = 0; h < H; ++h) {
            const int g = h / hpg;
            double* Phi = (double*)calloc((size_t)N / 2, sizeof(double));
            for (int t = 0; t < L; ++t) {
                const size_t bt = (size_t)b * L + t;
                const double dd = dt[bt * H + h];
                const double* th = theta + (bt * G + g) * (N / 2);
                for (int i = 0; i < N / 2; ++i) Phi[i] += dd * th[i];
                if (phase)
                    memcpy(phase + (bt * H + h) * (N / 2), Phi, sizeof(double) * (size_t)N / 2);
                for (int r = 0; r < R; ++r) {
                    const double* Bs = B + ((bt * G + g) * R + r) * N;
                    const double* Cs = C + ((bt * G + g) * R + r) * N;
                    double* Bo = B_rot + ((bt * H + h) * R + r) * N;
                    double* Co = C_rot + ((bt * H + h) * R + r) * N;
                    for (int i = 0; i < N / 2; ++i) {
                        const double c = cos(Phi[i]), s = sin(Phi[i]);
                        Bo[2 * i] = c * Bs[2 * i] + s * Bs[2 * i + 1];
                        Bo[2 * i + 1] = -s * Bs[2 * i] + c * Bs[2 * i + 1];
                        Co[2 * i] = c * Cs[2 * i] + s * Cs[2 * i + 1];
                        Co[2 * i + 1] = -s * Cs[2 * i] + c * Cs[2 * i + 1];
                    }
                }
            }
            free(Phi);
        }
    return 0;
}

/* Reverse-mode gradient of oracle_scan (the backward pass of the layer scan).
 *
 * Loss  J = sum_t <dy_t, y_t> + <dh, h_{L-1}> + <dpB, B_{L-1}> + <dpX, x_{L-1}>
 * (dh, dpB, dpX: gradients arriving at the final carry; any may be NULL).
 * Written out from the recurrence above by the chain rule, token by token in
 * reverse.  With g_t = dJ/dh_t (the total adjoint of the state after token t),
 * v_t = alpha_t h_{t-1} + beta_t B_{t-1} x_{t-1}^T (the state before R_t) and
 * h_t = R_t v_t + gamma_t B_t x_t^T:
 *   g_t      = C_t dy_t + alpha_{t+1} R_{t+1}^T g_{t+1}        (g_{L-1} starts at dh)
 *   dC_t     = h_t dy_t^T
 *   D_t      = gamma_t g_t + beta_{t+1} R_{t+1}^T g_{t+1}       (= dJ/d(B_t x_t^T))
 *   dB_t     = D_t x_t,   dx_t = D_t^T B_t
 *   dgamma_t = <g_t, B_t x_t^T>,  dalpha_t = <R_t^T g_t, h_{t-1}>,
 *   dbeta_t  = <R_t^T g_t, B_{t-1} x_{t-1}^T>,
 *   dphi_t[i] = sum_p g_t[pair i]^T R'(phi) v_t[pair i],  R' = dR/dphi,
 * and, with alpha = e^{dt A}, beta = (1 - lam) dt alpha, gamma = lam dt,
 * phi_i = dt theta_i:
 *   ddt  = dalpha A alpha + dbeta (1 - lam)(alpha + dt A alpha) + dgamma lam + sum_i dphi_i theta_i
 *   dA  += dalpha dt alpha + dbeta (1 - lam) dt^2 alpha
 *   dlam = -dbeta dt alpha + dgamma dt,     dtheta_i = dphi_i dt.
 * The carry-in gradients are g_{-1} = alpha_0 R_0^T g_0 (d init_h) and
 * D_{-1} = beta_0 R_0^T g_0 (d init_pB = D_{-1} init_pX, d init_pX = D_{-1}^T init_pB).
 *
 * Outputs (overwritten; B, C and theta gradients are summed over the heads of
 * a group, dA over batch and tokens): dx [b][t][h][r][p], dB, dC
 * [b][t][g][r][n], ddt, dlam [b][t][h], dA [h], dtheta [b][t][g][N/2],
 * d_init_h [b][h][n][p], d_init_pB [b][h][r][n], d_init_pX [b][h][r][p]
 * (the d_init_* may be NULL).  Returns 0, or -1 on bad arguments. */
int oracle_scan_bwd(const oracle_dims* d,
                    const double* x, const double* B, const double* C,
                    const double* dt, const double* A, const double* lam,
                    const double* theta,
                    const double* init_h, const double* init_pB, const double* init_pX,
                    const double* dy, const double* dh, const double* dpB, const double* dpX,
                    double* dx, double* dB, double* dC, double* ddt, double* dA,
                    double* dlam, double* dtheta,
                    double* d_init_h, double* d_init_pB, double* d_init_pX)
{
    if (!dims_ok(d) || !x || !B || !C || !dt || !A || !lam || !theta || !dy) return -1;
    if (!dx || !dB || !dC || !ddt || !dA || !dlam || !dtheta) return -1;
    const int Bn = d->batch, L = d->seqlen, H = d->nheads, G = d->ngroups;
    const int P = d->headdim, N = d->dstate, R = d->rank;
    const int hpg = H / G, NP = N * P;

    /* per-head partial results, reduced over the heads of a group below */
    double* dBh = (double*)calloc((size_t)Bn * L * H * R * N + 1, sizeof(double));
    double* dCh = (double*)calloc((size_t)Bn * L * H * R * N + 1, sizeof(double));
    double* dTh = (double*)calloc((size_t)Bn * L * H * (N / 2) + 1, sizeof(double));
    double* dAh = (double*)calloc((size_t)Bn * H + 1, sizeof(double));
    if (!dBh || !dCh || !dTh || !dAh) { free(dBh); free(dCh); free(dTh); free(dAh); return -1; }

#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int b = 0; b < Bn; ++b)
        for (int h = 0; h < H; ++h) {
            const int g = h / hpg;
            const size_t bh = (size_t)b * H + h;
            const double a = A[h];
            /* forward: every state h_{t-1} .. h_{L-1}; hs[t + 1] = h_t, hs[0] = h_{-1} */
            double* hs = (double*)calloc((size_t)(L + 1) * NP, sizeof(double));
            double* PB0 = (double*)calloc((size_t)R * N, sizeof(double));
            double* PX0 = (double*)calloc((size_t)R * P, sizeof(double));
            double* PB = (double*)calloc((size_t)R * N, sizeof(double));
            double* PX = (double*)calloc((size_t)R * P, sizeof(double));
            double* yscratch = (double*)calloc((size_t)R * P, sizeof(double));
            double* gk = (double*)calloc((size_t)NP, sizeof(double));
            double* gv = (double*)calloc((size_t)NP, sizeof(double));
            double* Db = (double*)calloc((size_t)NP, sizeof(double));
            double* Dt = (double*)calloc((size_t)NP, sizeof(double));
            double* v = (double*)calloc((size_t)NP, sizeof(double));
            if (init_h) memcpy(hs, init_h + bh * NP, sizeof(double) * (size_t)NP);
            if (init_pB) memcpy(PB0, init_pB + bh * R * N, sizeof(double) * (size_t)R * N);
            if (init_pX) memcpy(PX0, init_pX + bh * R * P, sizeof(double) * (size_t)R * P);
            memcpy(PB, PB0, sizeof(double) * (size_t)R * N);
            memcpy(PX, PX0, sizeof(double) * (size_t)R * P);
            for (int t = 0; t < L; ++t) {
                const size_t bt = (size_t)b * L + t;
                memcpy(hs + (size_t)(t + 1) * NP, hs + (size_t)t * NP, sizeof(double) * (size_t)NP);
                step_bh(N, P, R, hs + (size_t)(t + 1) * NP, PB, PX,
                        x + ((bt * H + h) * R) * P, B + ((bt * G + g) * R) * N, C + ((bt * G + g) * R) * N,
                        dt[bt * H + h], a, lam[bt * H + h], theta + (bt * G + g) * (N / 2), yscratch);
            }
            /* reverse */
            if (dh) memcpy(gk, dh + bh * NP, sizeof(double) * (size_t)NP);
            for (int t = L - 1; t >= 0; --t) {
                const size_t bt = (size_t)b * L + t;
                const double* xt = x + ((bt * H + h) * R) * P;
                const double* Bt = B + ((bt * G + g) * R) * N;
                const double* Ct = C + ((bt * G + g) * R) * N;
                const double* th = theta + (bt * G + g) * (N / 2);
                const double* dyt = dy + ((bt * H + h) * R) * P;
                const double* ht = hs + (size_t)(t + 1) * NP;
                const double* hp = hs + (size_t)t * NP;
                const double* pBt = t > 0 ? B + (((bt - 1) * G + g) * R) * N : PB0;
                const double* pXt = t > 0 ? x + (((bt - 1) * H + h) * R) * P : PX0;
                const double dd = dt[bt * H + h], lm = lam[bt * H + h];
                const double al = exp(dd * a), be = (1.0 - lm) * dd * al, ga = lm * dd;
                double* dxt = dx + ((bt * H + h) * R) * P;
                double* dBt = dBh + ((bt * H + h) * R) * N;
                double* dCt = dCh + ((bt * H + h) * R) * N;
                double* dTt = dTh + (bt * H + h) * (N / 2);
                memset(dxt, 0, sizeof(double) * (size_t)R * P);

                /* readout: g_t += C_t dy_t,  dC_t = h_t dy_t^T */
                for (int n = 0; n < N; ++n)
                    for (int p = 0; p < P; ++p) {
                        double acc = 0.0;
                        for (int r = 0; r < R; ++r) acc += Ct[r * N + n] * dyt[r * P + p];
                        gk[n * P + p] += acc;
                    }
                for (int r = 0; r < R; ++r)
                    for (int n = 0; n < N; ++n) {
                        double acc = 0.0;
                        for (int p = 0; p < P; ++p) acc += ht[n * P + p] * dyt[r * P + p];
                        dCt[r * N + n] = acc;
                    }
                /* the input term gamma_t B_t x_t^T and the beta term of token t+1 */
                double dga = 0.0;
                for (int n = 0; n < N; ++n)
                    for (int p = 0; p < P; ++p) {
                        double bx = 0.0;
                        for (int r = 0; r < R; ++r) bx += Bt[r * N + n] * xt[r * P + p];
                        dga += gk[n * P + p] * bx;
                        Dt[n * P + p] = ga * gk[n * P + p] + Db[n * P + p];
                    }
                if (t == L - 1) {
                    /* gradients arriving at the final (B, x) copies */
                    if (dpB) for (int e = 0; e < R * N; ++e) dBt[e] += dpB[bh * R * N + e];
                    if (dpX) for (int e = 0; e < R * P; ++e) dxt[e] += dpX[bh * R * P + e];
                }
                for (int r = 0; r < R; ++r) {
                    for (int n = 0; n < N; ++n) {
                        double acc = 0.0;
                        for (int p = 0; p < P; ++p) acc += Dt[n * P + p] * xt[r * P + p];
                        dBt[r * N + n] += acc;
                    }
                    for (int p = 0; p < P; ++p) {
                        double acc = 0.0;
                        for (int n = 0; n < N; ++n) acc += Dt[n * P + p] * Bt[r * N + n];
                        dxt[r * P + p] += acc;
                    }
                }
                /* v_t (the state before the rotation) */
                for (int n = 0; n < N; ++n)
                    for (int p = 0; p < P; ++p) {
                        double bx = 0.0;
                        for (int r = 0; r < R; ++r) bx += pBt[r * N + n] * pXt[r * P + p];
                        v[n * P + p] = al * hp[n * P + p] + be * bx;
                    }
                /* rotation: dphi, and gv = R_t^T g_t */
                double dphi_th = 0.0;
                for (int i = 0; i < N / 2; ++i) {
                    const double phi = dd * th[i];
                    const double c = cos(phi), s = sin(phi);
                    double dphi = 0.0;
                    for (int p = 0; p < P; ++p) {
                        const double g0 = gk[(2 * i) * P + p], g1 = gk[(2 * i + 1) * P + p];
                        const double v0 = v[(2 * i) * P + p], v1 = v[(2 * i + 1) * P + p];
                        dphi += g0 * (-s * v0 - c * v1) + g1 * (c * v0 - s * v1);
                        gv[(2 * i) * P + p] = c * g0 + s * g1;
                        gv[(2 * i + 1) * P + p] = -s * g0 + c * g1;
                    }
                    dTt[i] = dphi * dd;
                    dphi_th += dphi * th[i];
                }
                double dal = 0.0, dbe = 0.0;
                for (int n = 0; n < N; ++n)
                    for (int p = 0; p < P; ++p) {
                        double bx = 0.0;
                        for (int r = 0; r < R; ++r) bx += pBt[r * N + n] * pXt[r * P + p];
                        dal += gv[n * P + p] * hp[n * P + p];
                        dbe += gv[n * P + p] * bx;
                        Db[n * P + p] = be * gv[n * P + p];
                        gk[n * P + p] = al * gv[n * P + p];
                    }
                ddt[bt * H + h] = dal * a * al + dbe * (1.0 - lm) * (al + dd * a * al) + dga * lm + dphi_th;
                dAh[bh] += dal * dd * al + dbe * (1.0 - lm) * dd * dd * al;
                dlam[bt * H + h] = -dbe * dd * al + dga * dd;
            }
            if (d_init_h) memcpy(d_init_h + bh * NP, gk, sizeof(double) * (size_t)NP);
            if (d_init_pB)
                for (int r = 0; r < R; ++r)
                    for (int n = 0; n < N; ++n) {
                        double acc = 0.0;
                        for (int p = 0; p < P; ++p) acc += Db[n * P + p] * PX0[r * P + p];
                        d_init_pB[bh * R * N + r * N + n] = acc;
                    }
            if (d_init_pX)
                for (int r = 0; r < R; ++r)
                    for (int p = 0; p < P; ++p) {
                        double acc = 0.0;
                        for (int n = 0; n < N; ++n) acc += Db[n * P + p] * PB0[r * N + n];
                        d_init_pX[bh * R * P + r * P + p] = acc;
                    }
            free(hs); free(PB0); free(PX0); free(PB); free(PX); free(yscratch);
            free(gk); free(gv); free(Db); free(Dt); free(v);
        }
    /* sum over the heads of each group (B, C, theta) and over the batch (A) */
    for (int b = 0; b < Bn; ++b)
        for (int t = 0; t < L; ++t)
            for (int gi = 0; gi < G; ++gi) {
                const size_t bg = ((size_t)b * L + t) * G + gi;
                for (int e = 0; e < R * N; ++e) {
                    double sb = 0.0, sc = 0.0;
                    for (int k = 0; k < hpg; ++k) {
                        const size_t bh = ((size_t)b * L + t) * H + gi * hpg + k;
                        sb += dBh[bh * R * N + e];
                        sc += dCh[bh * R * N + e];
                    }
                    dB[bg * R * N + e] = sb;
                    dC[bg * R * N + e] = sc;
                }
                for (int i = 0; i < N / 2; ++i) {
                    double st = 0.0;
                    for (int k = 0; k < hpg; ++k) {
                        const size_t bh = ((size_t)b * L + t) * H + gi * hpg + k;
                        st += dTh[bh * (N / 2) + i];
                    }
                    dtheta[bg * (N / 2) + i] = st;
                }
            }
    for (int h = 0; h < H; ++h) {
        double s = 0.0;
        for (int b = 0; b < Bn; ++b) s += dAh[(size_t)b * H + h];
        dA[h] = s;
    }
    free(dBh); free(dCh); free(dTh); free(dAh);
    return 0;
}

/* ------------------------------------------------------------------------
 * Damping-regime variants ("Understanding Mamba-3 Through Oscillatory
 * Dynamics", section 2.2 and Table 1 (the three regimes of a damped
 * second-order system), section 4.1 (variants with the same coupled 2-D
 * state, input-update rule and state dimension, the damping parameter
 * selecting the regime around a shared spectral centre), section 4.2 and
 * appendix C.2 (mode persistence)).
 *
 * Reading: rotary pair i of token t evolves, over its interval, under the
 * generator dt_t (A_h I + theta_t[i] K_s) with K_s = [[0, -1], [s, 0]]:
 *   s = +1  underdamped  (eigenvalues A +- i theta: Mamba-3's decay-rotation),
 *   s =  0  critically damped (double eigenvalue A, one eigenvector),
 *   s = -1  overdamped   (real eigenvalues A +- theta),
 * so the centre A of the eigenvalue pair is the same in every regime.  Since
 * K_s^2 = -s I, exp(phi K_s) = c(phi) I + sn(phi) K_s with
 *   (c, sn) = (cos, sin) for s = +1, (1, phi) for s = 0, (cosh, sinh) for
 *   s = -1,
 * i.e. the 2x2 block T = [[c, -sn], [s sn, c]], phi = dt_t theta_t[i].  The
 * input-update rule is Mamba-3's exponential-trapezoidal one with T_t in
 * place of R_t:
 *   h_t = T_t (alpha_t h_{t-1} + beta_t B_{t-1} X_{t-1}^T) + gamma_t B_t X_t^T,
 *   y_t = C_t^T h_t.
 * regime: 0 = underdamped, 1 = critically damped, 2 = overdamped.
 * Written on its own (not through step_bh), so that the underdamped regime
 * checks the general 2x2 block against step_bh's rotation.
 * ---------------------------------------------------------------------- */
static void pair_block(int regime, double phi, double* c, double* sn, double* sg)
{
    if (regime == 0) { *c = cos(phi); *sn = sin(phi); *sg = 1.0; }
    else if (regime == 1) { *c = 1.0; *sn = phi; *sg = 0.0; }
    else { *c = cosh(phi); *sn = sinh(phi); *sg = -1.0; }
}

/* One token of either variant for one (b, h).  regime selects the pair block
 * (damped variants); u (length N, may be NULL) is the reflection direction
 * of the reflection variant, which then uses the underdamped block. */
static void step_bh_general(int N, int P, int R, int regime, const double* u,
                            double* H, double* PB, double* PX,
                            const double* xt, const double* Bt, const double* Ct,
                            double d, double a, double lam, const double* th,
                            double* yt)
{
    const double alpha = exp(d * a);
    const double beta = (1.0 - lam) * d * alpha;
    const double gamma = lam * d;

    /* v = alpha h + beta B_{t-1} X_{t-1}^T */
    for (int n = 0; n < N; ++n)
        for (int p = 0; p < P; ++p) {
            double pend = 0.0;
            for (int r = 0; r < R; ++r) pend += PX[r * P + p] * PB[r * N + n];
            H[n * P + p] = alpha * H[n * P + p] + beta * pend;
        }

    /* reflection v <- (I - 2 u u^T / u^T u) v, column by column (u = 0: none) */
    if (u) {
        double uu = 0.0;
        for (int n = 0; n < N; ++n) uu += u[n] * u[n];
        if (uu > 0.0) {
            for (int p = 0; p < P; ++p) {
                double dot = 0.0;
                for (int n = 0; n < N; ++n) dot += u[n] * H[n * P + p];
                const double f = 2.0 * dot / uu;
                for (int n = 0; n < N; ++n) H[n * P + p] -= f * u[n];
            }
        }
    }

    /* pair blocks T (regime) on rows (2i, 2i+1) */
    for (int i = 0; i < N / 2; ++i) {
        double c, sn, sg;
        pair_block(regime, d * th[i], &c, &sn, &sg);
        for (int p = 0; p < P; ++p) {
            const double u0 = H[(2 * i) * P + p];
            const double u1 = H[(2 * i + 1) * P + p];
            H[(2 * i) * P + p] = c * u0 - sn * u1;
            H[(2 * i + 1) * P + p] = sg * sn * u0 + c * u1;
        }
    }

    /* + gamma B_t X_t^T */
    for (int n = 0; n < N; ++n)
        for (int p = 0; p < P; ++p) {
            double cur = 0.0;
            for (int r = 0; r < R; ++r) cur += xt[r * P + p] * Bt[r * N + n];
            H[n * P + p] += gamma * cur;
        }

    for (int r = 0; r < R; ++r)
        for (int p = 0; p < P; ++p) {
            double out = 0.0;
            for (int n = 0; n < N; ++n) out += H[n * P + p] * Ct[r * N + n];
            yt[r * P + p] = out;
        }

    memcpy(PB, Bt, (size_t)R * N * sizeof(double));
    memcpy(PX, xt, (size_t)R * P * sizeof(double));
}

static int scan_general(const oracle_dims* d, int regime, const double* u,
                        const double* x, const double* B, const double* C,
                        const double* dt, const double* A, const double* lam,
                        const double* theta,
                        const double* init_h, const double* init_pB, const double* init_pX,
                        double* y, double* out_h, double* out_pB, double* out_pX)
{
    if (!dims_ok(d) || !x || !B || !C || !dt || !A || !lam || !theta || !y) return -1;
    if (regime < 0 || regime > 2) return -1;
    const int Bn = d->batch, L = d->seqlen, H = d->nheads, G = d->ngroups;
    const int P = d->headdim, N = d->dstate, R = d->rank;
    const int hpg = H / G;

#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int b = 0; b < Bn; ++b)
        for (int h = 0; h < H; ++h) {
            const int g = h / hpg;
            double* Hs = (double*)calloc((size_t)N * P, sizeof(double));
            double* PB = (double*)calloc((size_t)R * N, sizeof(double));
            double* PX = (double*)calloc((size_t)R * P, sizeof(double));
            const size_t bh = (size_t)b * H + h;
            if (init_h) memcpy(Hs, init_h + bh * N * P, sizeof(double) * (size_t)N * P);
            if (init_pB) memcpy(PB, init_pB + bh * R * N, sizeof(double) * (size_t)R * N);
            if (init_pX) memcpy(PX, init_pX + bh * R * P, sizeof(double) * (size_t)R * P);
            for (int t = 0; t < L; ++t) {
                const size_t bt = (size_t)b * L + t;
                step_bh_general(N, P, R, regime, u ? u + (bt * G + g) * N : NULL, Hs, PB, PX,
                                x + ((bt * H + h) * R) * P, B + ((bt * G + g) * R) * N,
                                C + ((bt * G + g) * R) * N, dt[bt * H + h], A[h], lam[bt * H + h],
                                theta + (bt * G + g) * (N / 2), y + ((bt * H + h) * R) * P);
            }
            if (out_h) memcpy(out_h + bh * N * P, Hs, sizeof(double) * (size_t)N * P);
            if (out_pB) memcpy(out_pB + bh * R * N, PB, sizeof(double) * (size_t)R * N);
            if (out_pX) memcpy(out_pX + bh * R * P, PX, sizeof(double) * (size_t)R * P);
            free(Hs); free(PB); free(PX);
        }
    return 0;
}

/* Damping-regime variant of oracle_scan (regime 0, 1, 2 as above); same
 * arguments and layouts otherwise. */
int oracle_scan_damped(const oracle_dims* d, int regime,
                       const double* x, const double* B, const double* C,
                       const double* dt, const double* A, const double* lam,
                       const double* theta,
                       const double* init_h, const double* init_pB, const double* init_pX,
                       double* y, double* out_h, double* out_pB, double* out_pX)
{
    return scan_general(d, regime, NULL, x, B, C, dt, A, lam, theta, init_h, init_pB, init_pX,
                        y, out_h, out_pB, out_pX);
}

/* Low-rank reflection extension (abstract of the extension of Mamba-3's
 * diagonal transition with an input-dependent rank-one reflection term,
 * listed on "Understanding Mamba-3 Through Oscillatory Dynamics"; two
 * reflections compose to a rotation, appendix C.4 of that paper).
 * Reading: the diagonal part alpha_t I of the transition becomes
 * alpha_t (I - 2 u_t u_t^T / u_t^T u_t), a Householder reflection along the
 * input-dependent direction u_t (per token and group, like B), and the
 * exponential-trapezoidal rule, the rotation R_t and the readout stay:
 *   h_t = R_t H_t (alpha_t h_{t-1} + beta_t B_{t-1} X_{t-1}^T) + gamma_t B_t X_t^T,
 *   H_t = I - 2 u_t u_t^T / (u_t^T u_t)   (H_t = I where u_t = 0).
 * u: [b][t][g][N]. */
int oracle_scan_reflect(const oracle_dims* d, const double* u,
                        const double* x, const double* B, const double* C,
                        const double* dt, const double* A, const double* lam,
                        const double* theta,
                        const double* init_h, const double* init_pB, const double* init_pX,
                        double* y, double* out_h, double* out_pB, double* out_pX)
{
    if (!u) return -1;
    return scan_general(d, 0, u, x, B, C, dt, A, lam, theta, init_h, init_pB, init_pX,
                        y, out_h, out_pB, out_pX);
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Sets the OpenMP thread count of later calls (n >= 1); timing only, the
 * results do not depend on it (each (b, h) is computed by one thread). */
void oracle_set_num_threads(int n)
{
#ifdef _OPENMP
    extern void omp_set_num_threads(int);
    if (n >= 1) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

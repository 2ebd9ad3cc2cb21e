/*
 * Plain fp64 CPU oracle for the Newton-solved diag-mix sLSTM.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, includes
 * or calls this file; only the tests, the smoke check and the benchmark's
 * CPU-baseline leg use it.  It shares no code, header, table or constant with
 * the CUDA path.
 *
 * Everything here is written for clarity, not speed: one lane (a (batch,
 * feature) pair) at a time, one time step at a time, fp64 throughout, libm
 * transcendentals.
 *
 * Data layout used by every function (lane-major, contiguous):
 *   P  [lanes][T][4]   pre-activations, gate order (z, i, f, o)
 *   R  [lanes][4]      channelwise recurrent weights, gate order (z, i, f, o)
 *   s0 [lanes][4]      initial state, slot order (c, n, m, h)
 *   S  [lanes][T][4]   state trajectory, slot order (c, n, m, h)
 * The Python wrapper in oracle/__init__.py converts to and from the
 * (B, T, 4, d_h) tensors of the library boundary.
 *
 * Sources (page titles and sections):
 *   [xlstm-edu]  "xLSTM - a from-scratch, educational reimplementation",
 *                section "Exponential gating + the stabilizer (the crux)".
 *   [xlstm-sum]  "xLSTM: Extended Long Short-Term Memory" (paper summary),
 *                section "Method", the sLSTM step pseudocode and the
 *                stabilizer equation of section 2.2.
 *   [pararnn]    "sLSTM in this library" (pararnn-torch docs), sections
 *                "Cell", "Backward", "Packed sequences".
 *   [structure]  "pararnn-torch structure", sections "Current surface" and
 *                "Naming".
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_FORGET_SIGMOID 0
#define ORACLE_FORGET_EXP 1

static double sigm(double x) { return 1.0 / (1.0 + exp(-x)); }

/* log(sigmoid(x)) written so that neither branch overflows. */
static double log_sigm(double x)
{
    if (x >= 0.0) return -log1p(exp(-x));
    return x - log1p(exp(x));
}

/*
 * One stabilised sLSTM step for one feature ([xlstm-edu]; [xlstm-sum] sLSTM
 * step pseudocode; stabilizer m_t = max(log f_t + m_{t-1}, log i_t) from
 * [xlstm-sum] section 2.2).  Diag mixing ([pararnn] "Cell", mix='diag'):
 * the recurrent contribution to gate g is r_g * h_{t-1}.
 *
 *   a_g = p_g + r_g h_{t-1}           g in (z, i, f, o)
 *   z = tanh a_z,  o = sigmoid a_o,  log i = a_i
 *   log f = log sigmoid a_f  (sigmoid forget)  or  a_f  (exp forget)
 *   m = max(log f + m_{t-1}, a_i)
 *   i' = exp(a_i - m),  f' = exp(log f + m_{t-1} - m)
 *   c = f' c_{t-1} + i' z,  n = f' n_{t-1} + i',  h = o c / n
 *
 * Read-out is the paper's h = o * c / n ([xlstm-sum] sLSTM step pseudocode).
 * The max breaks ties toward the forget branch (beta = 1 when equal).
 *
 * If J is not NULL it receives d s_t / d s_{t-1} (4x4 row-major, rows and
 * columns in slot order (c, n, m, h)); if G is not NULL it receives
 * d s_t / d a_t (4x4 row-major, rows in slot order, columns in gate order).
 * Both are the hand derivation below, written out term by term.
 */
void oracle_step(const double sp[4], const double p[4], const double r[4],
                 int forget, double out[4], double *J, double *G)
{
    const double c0 = sp[0], n0 = sp[1], m0 = sp[2], h0 = sp[3];
    const double az = p[0] + r[0] * h0;
    const double ai = p[1] + r[1] * h0;
    const double af = p[2] + r[2] * h0;
    const double ao = p[3] + r[3] * h0;

    const double z = tanh(az);
    const double o = sigm(ao);
    double lf, dlf; /* log f and d(log f)/d a_f */
    if (forget == ORACLE_FORGET_EXP) {
        lf = af;
        dlf = 1.0;
    } else {
        lf = log_sigm(af);
        dlf = sigm(-af);
    }
    const double u = lf + m0;
    const double m = (u >= ai) ? u : ai;
    const double beta = (u >= ai) ? 1.0 : 0.0;
    const double ip = exp(ai - m);
    const double fp = exp(u - m);
    const double c = fp * c0 + ip * z;
    const double n = fp * n0 + ip;
    const double h = o * c / n;
    out[0] = c;
    out[1] = n;
    out[2] = m;
    out[3] = h;

    if (J == NULL && G == NULL) return;

    /* Partial derivatives of m, log i', log f' with respect to m_{t-1}
     * and h_{t-1} (through a_i and a_f). */
    const double dm_dm0 = beta;
    const double dm_dh0 = beta * dlf * r[2] + (1.0 - beta) * r[1];
    const double dli_dm0 = -dm_dm0;               /* log i' = a_i - m        */
    const double dli_dh0 = r[1] - dm_dh0;
    const double dlf_dm0 = 1.0 - dm_dm0;          /* log f' = lf + m0 - m    */
    const double dlf_dh0 = dlf * r[2] - dm_dh0;
    const double dz_dh0 = (1.0 - z * z) * r[0];
    const double do_dh0 = o * (1.0 - o) * r[3];
    const double y = c / n;

    if (J != NULL) {
        /* row c */
        J[0] = fp;
        J[1] = 0.0;
        J[2] = fp * c0 * dlf_dm0 + ip * z * dli_dm0;
        J[3] = fp * c0 * dlf_dh0 + ip * z * dli_dh0 + ip * dz_dh0;
        /* row n */
        J[4] = 0.0;
        J[5] = fp;
        J[6] = fp * n0 * dlf_dm0 + ip * dli_dm0;
        J[7] = fp * n0 * dlf_dh0 + ip * dli_dh0;
        /* row m */
        J[8] = 0.0;
        J[9] = 0.0;
        J[10] = dm_dm0;
        J[11] = dm_dh0;
        /* row h: h = o c / n  ->  dh = (o/n)(dc - y dn) + y do */
        for (int k = 0; k < 4; ++k)
            J[12 + k] = (o / n) * (J[k] - y * J[4 + k]);
        J[15] += y * do_dh0;
    }
    if (G != NULL) {
        /* derivatives with respect to a_i and a_f of m, log i', log f' */
        const double dm_dai = 1.0 - beta, dm_daf = beta * dlf;
        const double dli_dai = 1.0 - dm_dai, dli_daf = -dm_daf;
        const double dlf_dai = -dm_dai, dlf_daf = dlf - dm_daf;
        /* columns: a_z, a_i, a_f, a_o */
        G[0] = ip * (1.0 - z * z);
        G[1] = fp * c0 * dlf_dai + ip * z * dli_dai;
        G[2] = fp * c0 * dlf_daf + ip * z * dli_daf;
        G[3] = 0.0;
        G[4] = 0.0;
        G[5] = fp * n0 * dlf_dai + ip * dli_dai;
        G[6] = fp * n0 * dlf_daf + ip * dli_daf;
        G[7] = 0.0;
        G[8] = 0.0;
        G[9] = dm_dai;
        G[10] = dm_daf;
        G[11] = 0.0;
        for (int k = 0; k < 4; ++k)
            G[12 + k] = (o / n) * (G[k] - y * G[4 + k]);
        G[15] += y * o * (1.0 - o);
    }
}

/*
 * Sequential (time-stepping) solve of the recurrence: S_t = f(S_{t-1}, P_t)
 * from s0.  This is the plain definition the Newton solve must reproduce
 * ([pararnn] "API notes": the sequential path of ParaRNN).
 */
void oracle_sequential(int lanes, int T, const double *P, const double *R,
                       const double *s0, int forget, double *S)
{
    for (int l = 0; l < lanes; ++l) {
        double prev[4];
        memcpy(prev, s0 + 4 * l, sizeof prev);
        for (int t = 0; t < T; ++t) {
            double *out = S + ((size_t)l * T + t) * 4;
            oracle_step(prev, P + ((size_t)l * T + t) * 4, R + 4 * l, forget,
                        out, NULL, NULL);
            memcpy(prev, out, sizeof prev);
        }
    }
}

/*
 * Unstabilised recurrence ([xlstm-sum] "Method" item 1: stabilised and
 * unstabilised forms give identical outputs):
 *   i = exp(a_i),  f = sigmoid(a_f) or exp(a_f)
 *   c_u = f c_u + i z,  n_u = f n_u + i,  h = o c_u / n_u
 * Initial values c_u = c0 exp(m0), n_u = n0 exp(m0).  Outputs the raw c_u,
 * n_u and h, each [lanes][T].  Overflows for long exp-forget sequences; the
 * caller keeps T small.
 */
void oracle_sequential_unstabilised(int lanes, int T, const double *P,
                                    const double *R, const double *s0,
                                    int forget, double *cu, double *nu,
                                    double *h)
{
    for (int l = 0; l < lanes; ++l) {
        const double *r = R + 4 * l;
        double c = s0[4 * l + 0] * exp(s0[4 * l + 2]);
        double n = s0[4 * l + 1] * exp(s0[4 * l + 2]);
        double hp = s0[4 * l + 3];
        for (int t = 0; t < T; ++t) {
            const double *p = P + ((size_t)l * T + t) * 4;
            const double z = tanh(p[0] + r[0] * hp);
            const double ig = exp(p[1] + r[1] * hp);
            const double af = p[2] + r[2] * hp;
            const double fg = (forget == ORACLE_FORGET_EXP) ? exp(af) : sigm(af);
            const double o = sigm(p[3] + r[3] * hp);
            c = fg * c + ig * z;
            n = fg * n + ig;
            hp = o * c / n;
            cu[(size_t)l * T + t] = c;
            nu[(size_t)l * T + t] = n;
            h[(size_t)l * T + t] = hp;
        }
    }
}

/* Residual F_t = S_t - f(S_{t-1}, P_t) and Jacobian J_t at a guess S. */
static void residual_and_jacobian(int T, const double *P, const double *r,
                                  const double *s0, int forget, const double *S,
                                  double *F, double *J)
{
    for (int t = 0; t < T; ++t) {
        const double *prev = (t == 0) ? s0 : S + (size_t)(t - 1) * 4;
        double fval[4];
        oracle_step(prev, P + (size_t)t * 4, r, forget, fval,
                    J ? J + (size_t)t * 16 : NULL, NULL);
        for (int k = 0; k < 4; ++k) F[(size_t)t * 4 + k] = S[(size_t)t * 4 + k] - fval[k];
    }
}

/*
 * Sequential solve of an affine recurrence of 4-vectors, one lane at a time
 * ([pararnn] "Packed sequences": the Newton inner solve is a scan on the
 * (J, r) monoid; [structure] "Naming": scan_block4 for (B,T,4,4,d)).
 *   forward  (reverse = 0):  y_t = A_t y_{t-1} + b_t,   y_{-1} = y0
 *   reverse  (reverse = 1):  y_t = A_t^T y_{t+1} + b_t, y_T  = y0
 * A is [lanes][T][4][4] row-major, b and y are [lanes][T][4], y0 is
 * [lanes][4] or NULL for zero.
 */
void oracle_affine_solve(int lanes, int T, const double *A, const double *b,
                         const double *y0, int reverse, double *y)
{
    for (int l = 0; l < lanes; ++l) {
        double carry[4] = {0, 0, 0, 0};
        if (y0) memcpy(carry, y0 + 4 * l, sizeof carry);
        for (int step = 0; step < T; ++step) {
            const int t = reverse ? T - 1 - step : step;
            const double *At = A + ((size_t)l * T + t) * 16;
            const double *bt = b + ((size_t)l * T + t) * 4;
            double nxt[4];
            for (int i = 0; i < 4; ++i) {
                double acc = bt[i];
                for (int k = 0; k < 4; ++k)
                    acc += (reverse ? At[k * 4 + i] : At[i * 4 + k]) * carry[k];
                nxt[i] = acc;
            }
            memcpy(y + ((size_t)l * T + t) * 4, nxt, sizeof nxt);
            memcpy(carry, nxt, sizeof carry);
        }
    }
}

/*
 * The decoupled trajectory: the cell run with the recurrent weights set to
 * zero, so that no gate sees h_{t-1} while c, n and m still recur exactly.
 * It is one of the initial guesses of oracle_newton below.  The pages give
 * no initial guess beyond prepending h0 ([structure] "Current surface"); this
 * is the reading taken for the default one.
 */
static void decoupled_trajectory(int T, const double *P, const double *s0, int forget, double *S)
{
    const double zero[4] = {0.0, 0.0, 0.0, 0.0};
    const double *prev = s0;
    for (int t = 0; t < T; ++t) {
        oracle_step(prev, P + (size_t)t * 4, zero, forget, S + (size_t)t * 4, NULL, NULL);
        prev = S + (size_t)t * 4;
    }
}

/*
 * One refinement sweep of the decoupled guess: the gates of step t see the
 * previous guess's h_{t-1} (Sold), while c, n and m recur exactly from the
 * new sweep's own previous state, as in decoupled_trajectory:
 *   a_t = P_t + r h^old_{t-1}  (h^old_{-1} = s0's h),  Snew_t = step(Snew_{t-1}, a_t) with r = 0.
 * It is a fixed-point (Picard) sweep of the recurrence on h: the solution is
 * its fixed point, and after k sweeps the first k steps are exact.  Reading
 * taken for the guess's refinement: the pages give no initial guess.
 */
static void guess_sweep(int T, const double *P, const double *r, const double *s0, int forget,
                        const double *Sold, double *Snew)
{
    const double zero[4] = {0.0, 0.0, 0.0, 0.0};
    const double *prev = s0;
    for (int t = 0; t < T; ++t) {
        const double h_old = (t == 0) ? s0[3] : Sold[(size_t)(t - 1) * 4 + 3];
        double a[4];
        for (int g = 0; g < 4; ++g) a[g] = P[(size_t)t * 4 + g] + r[g] * h_old;
        oracle_step(prev, a, zero, forget, Snew + (size_t)t * 4, NULL, NULL);
        prev = Snew + (size_t)t * 4;
    }
}

/* Raw and scaled maxima of the residual of every lane at S; returns 1 when
 * some residual or state entry is not finite. */
static int residual_maxima(int lanes, int T, const double *P, const double *R, const double *s0,
                           int forget, const double *S, double *F, double *raw, double *scaled)
{
    const size_t n4 = (size_t)T * 4;
    int bad = 0;
    *raw = 0.0;
    *scaled = 0.0;
    for (int l = 0; l < lanes; ++l) {
        const double *Sl = S + (size_t)l * n4;
        residual_and_jacobian(T, P + (size_t)l * n4, R + 4 * l, s0 + 4 * l, forget, Sl, F, NULL);
        for (size_t q = 0; q < n4; ++q) {
            const double a = fabs(F[q]);
            if (!isfinite(a) || !isfinite(Sl[q])) bad = 1;
            if (a > *raw) *raw = a;
            const double sc = a / (1.0 + fabs(Sl[q]));
            if (sc > *scaled) *scaled = sc;
        }
    }
    if (bad) {
        *raw = INFINITY;
        *scaled = INFINITY;
    }
    return bad;
}

/*
 * Newton solve of the whole trajectory (ParaRNN Newton, as described in
 * [pararnn] "Cell" and [structure] "Current surface"):
 *   initial guess (s0 is fixed and enters as the step before t = 0):
 *     init 0: the decoupled trajectory (decoupled_trajectory above), then
 *             `sweeps` refinement sweeps (guess_sweep above);
 *     init 1: S = 0 for every t;
 *     init 2: S as given on entry;
 *   the residual of the initial guess is recorded in init_res (raw, scaled)
 *   when init is 0, the mode is tolerance and max_iters >= 1, else init_res
 *   holds -1; it does not stop the solve: the test starts with iteration 1;
 *   max_iters = 0 returns the initial guess itself (iters 0, neither
 *   converged nor diverged);
 *   repeat k = 1..max_iters:
 *     F_t = S_t - f(S_{t-1}, P_t),  J_t = d f / d s_{t-1} at the guess
 *     solve delta_t = J_t delta_{t-1} - F_t,  delta_{-1} = 0
 *     S <- S + delta
 *     Fn = residual at the new S; record max|Fn| and max |Fn|/(1+|S|)
 *     stop when (not fixed) and the test holds: max |Fn|/(1+|S|) <= tol
 *     (residual_mode 0) or max|Fn| <= tol (residual_mode 1)
 *   diverged when not converged and (max|Fn| > 1 or non-finite) after the
 *   last iteration ([structure] "Current surface": NewtonDivergenceError if
 *   max|F| > 1 after K).  In fixed mode "converged" reports whether the final
 *   residual meets the test.
 * All lanes iterate together and stop together (the residual is a max over
 * every lane, step and slot).
 * hist_raw / hist_scaled receive one value per iteration (max_iters long);
 * init_res (2 values, may be NULL) the raw and scaled residual of the initial
 * guess, or -1 when it is not evaluated.
 */
void oracle_newton(int lanes, int T, const double *P, const double *R,
                   const double *s0, int forget, int max_iters, int fixed,
                   double tol, int init, int sweeps, int residual_mode, double *S,
                   double *hist_raw, double *hist_scaled, double *init_res,
                   int *iters, int *converged, int *diverged)
{
    const size_t n4 = (size_t)T * 4;
    double *F = malloc(sizeof(double) * n4);
    double *J = malloc(sizeof(double) * n4 * 4);
    double *negF = malloc(sizeof(double) * n4);
    double *delta = malloc(sizeof(double) * n4);
    if (init == 0) {
        for (int l = 0; l < lanes; ++l) {
            double *Sl = S + (size_t)l * n4;
            decoupled_trajectory(T, P + (size_t)l * n4, s0 + 4 * l, forget, Sl);
            for (int k = 0; k < sweeps; ++k) {
                guess_sweep(T, P + (size_t)l * n4, R + 4 * l, s0 + 4 * l, forget, Sl, delta);
                memcpy(Sl, delta, sizeof(double) * n4);
            }
        }
    } else if (init == 1) {
        memset(S, 0, sizeof(double) * n4 * lanes);
    }
    *iters = 0;
    *converged = 0;
    *diverged = 0;
    if (init_res) init_res[0] = init_res[1] = -1.0;
    double raw = INFINITY, scaled = INFINITY;
    if (init == 0 && !fixed && max_iters >= 1 && init_res)
        (void)residual_maxima(lanes, T, P, R, s0, forget, S, F, &init_res[0], &init_res[1]);
    for (int k = 1; k <= max_iters; ++k) {
        for (int l = 0; l < lanes; ++l) {
            double *Sl = S + (size_t)l * n4;
            residual_and_jacobian(T, P + (size_t)l * n4, R + 4 * l, s0 + 4 * l,
                                  forget, Sl, F, J);
            for (size_t q = 0; q < n4; ++q) negF[q] = -F[q];
            oracle_affine_solve(1, T, J, negF, NULL, 0, delta);
            for (size_t q = 0; q < n4; ++q) Sl[q] += delta[q];
        }
        const int bad = residual_maxima(lanes, T, P, R, s0, forget, S, F, &raw, &scaled);
        hist_raw[k - 1] = raw;
        hist_scaled[k - 1] = scaled;
        *iters = k;
        if (bad) break;
        const double test = residual_mode ? raw : scaled;
        if (!fixed && test <= tol) {
            *converged = 1;
            break;
        }
    }
    if (fixed && max_iters >= 1 && (residual_mode ? raw : scaled) <= tol) *converged = 1;
    if (*iters > 0 && !*converged && !(raw <= 1.0)) *diverged = 1;
    free(F);
    free(J);
    free(negF);
    free(delta);
}

/*
 * Backpropagation through time for L = sum_t dH_t * h_t ([pararnn]
 * "Backward": one reverse scan of J^T, then the cell VJP).
 *   lambda_t = e_h dH_t + J_{t+1}^T lambda_{t+1},   lambda past the end = 0
 *   dP_t     = G_t^T lambda_t          (a_t = P_t + R h_{t-1}, so dL/dP = dL/da)
 *   dR_g     = sum_t dP_t[g] h_{t-1}   (h_{-1} = s0.h)
 *   db_g     = sum_t dP_t[g]
 *   ds0      = J_0^T lambda_0
 * S is the trajectory the gradient is taken at (the solution).  dH is
 * [lanes][T]; dP [lanes][T][4]; dR, db, ds0 [lanes][4].
 */
void oracle_bptt(int lanes, int T, const double *P, const double *R,
                 const double *s0, const double *S, const double *dH, int forget,
                 double *dP, double *dR, double *db, double *ds0)
{
    for (int l = 0; l < lanes; ++l) {
        const double *Pl = P + (size_t)l * T * 4;
        const double *Sl = S + (size_t)l * T * 4;
        const double *r = R + 4 * l;
        double lam_next[4] = {0, 0, 0, 0}; /* lambda_{t+1} */
        double Jnext[16];                  /* J_{t+1} */
        int have_next = 0;
        double dr[4] = {0, 0, 0, 0}, dbl[4] = {0, 0, 0, 0};
        for (int t = T - 1; t >= 0; --t) {
            const double *prev = (t == 0) ? s0 + 4 * l : Sl + (size_t)(t - 1) * 4;
            double fval[4], Jt[16], Gt[16];
            oracle_step(prev, Pl + (size_t)t * 4, r, forget, fval, Jt, Gt);
            double lam[4] = {0, 0, 0, dH[(size_t)l * T + t]};
            if (have_next)
                for (int i = 0; i < 4; ++i)
                    for (int k = 0; k < 4; ++k) lam[i] += Jnext[k * 4 + i] * lam_next[k];
            double *dp = dP + ((size_t)l * T + t) * 4;
            for (int g = 0; g < 4; ++g) {
                double acc = 0.0;
                for (int k = 0; k < 4; ++k) acc += Gt[k * 4 + g] * lam[k];
                dp[g] = acc;
                dr[g] += acc * prev[3];
                dbl[g] += acc;
            }
            memcpy(lam_next, lam, sizeof lam);
            memcpy(Jnext, Jt, sizeof Jt);
            have_next = 1;
        }
        for (int i = 0; i < 4; ++i) {
            double acc = 0.0;
            if (have_next)
                for (int k = 0; k < 4; ++k) acc += Jnext[k * 4 + i] * lam_next[k];
            ds0[4 * l + i] = acc;
            dR[4 * l + i] = dr[i];
            db[4 * l + i] = dbl[i];
        }
    }
}

/*
 * Plain GEMM, C[m][n] = sum_k A(m,k) B(k,n) (+ bias[n] when bias != NULL),
 * fp64 accumulation.  ta / tb select the storage of A and B:
 *   ta = 0: A stored [M][K];  ta = 1: A stored [K][M]
 *   tb = 0: B stored [K][N];  tb = 1: B stored [N][K]
 * Used for the input projection P = x W_x^T + b ([xlstm-sum] sLSTM step
 * pseudocode, W_* @ x + b_*) and the gradients dx = dP W_x, dW_x = dP^T x
 * ([pararnn] "Backward", the packed VJP for the W_x gradient).
 */
void oracle_gemm(int M, int N, int K, const double *A, int ta, const double *B,
                 int tb, const double *bias, double *C)
{
    for (int m = 0; m < M; ++m)
        for (int n = 0; n < N; ++n) {
            double acc = bias ? bias[n] : 0.0;
            for (int k = 0; k < K; ++k) {
                const double a = ta ? A[(size_t)k * M + m] : A[(size_t)m * K + k];
                const double bb = tb ? B[(size_t)n * K + k] : B[(size_t)k * N + n];
                acc += a * bb;
            }
            C[(size_t)m * N + n] = acc;
        }
}

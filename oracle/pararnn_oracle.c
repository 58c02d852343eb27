/*
 * pararnn_oracle.c -- plain fp64 CPU oracle for the ParaRNN hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  The test suite, the smoke check and the CPU
 * baseline leg of the benchmark call this code; the CUDA library never does,
 * and this file includes nothing from it.
 *
 * What it computes (all in double precision, one channel at a time, with no
 * scan, no blocking and no fusion):
 *
 *   - the sequential unroll s_t = f(s_{t-1}, x_t), s_{-1} = h0
 *     ("sequential_apply" / ".eval() keeps the one-step recurrence",
 *      pararnn-torch PyPI page, Quickstart and API overview sections);
 *   - K Newton iterations on the whole-trajectory system
 *     F(H)_t = h_t - f(h_{t-1}, x_t) = 0 (pararnn-torch PyPI page, Method
 *     section; ParaRNN thread, tweet [3/8]), starting from the warm start
 *     h_t^(0) = f(0, x_t) (Method section, "paper App. A"), each linear
 *     system J delta = -F solved by a plain forward substitution in time;
 *   - optionally P Picard (fixed-point) sweeps before the Newton iterations,
 *     h_t^(p+1) = f(h_{t-1}^(p), x_t) with h_{-1}^(p) = h0, which warm the
 *     first guess further (API overview, "Solver": picard_iters; Method
 *     section: zero-hidden start plus Picard);
 *   - the adjoint of the recurrence at a given trajectory H: the reverse
 *     recursion lambda_t = g_t + A_{t+1}^T lambda_{t+1} and the parameter
 *     gradients it implies (Method section, "Backward follows paper eq. 2.6";
 *     the equation itself is not printed, so this is the plain adjoint of the
 *     triangular system F(H) = 0).
 *
 * Cells (state width S, gate count G, pre-activations p_g, diagonal
 * recurrent weights a_g, one channel):
 *   0 linear   S=1 G=2  f = p_a * h + p_b                     (no weights)
 *   1 diag GRU S=1 G=3  z = sig(p_z + a_z h), r = sig(p_r + a_r h),
 *                       c = tanh(p_c + a_c r h), f = (1 - z) h + z c
 *   2 diag LSTM S=2 G=4 state (c, h), gates (i, f, o, c):
 *                       i = sig(p_i + a_i h), f = sig(p_f + a_f h + 1),
 *                       o = sig(p_o + a_o h), g = tanh(p_c + a_c h),
 *                       c' = f c + i g, h' = o tanh(c')
 * GRU and LSTM are the diagonal (per-channel) forms of the ParaGRU / ParaLSTM
 * cells listed on the pararnn-torch page (Models, Usage); the linear cell is
 * the affine recurrence that the News section says needs no Newton iteration
 * beyond one exact scan.
 *
 * Layouts (row-major, D fastest): px (B,T,G,D), w (G,D), h0 (B,S,D),
 * H / dL_dH (B,T,S,D), dL_dpx (B,T,G,D), dL_da (G,D), dL_dh0 (B,S,D).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define MAXS 2
#define MAXG 4

static int ncell_gates(int cell) { return cell == 0 ? 2 : cell == 1 ? 3 : cell == 2 ? 4 : -1; }
static int ncell_state(int cell) { return cell == 0 ? 1 : cell == 1 ? 1 : cell == 2 ? 2 : -1; }

int oracle_num_gates(int cell) { return ncell_gates(cell); }
int oracle_state_width(int cell) { return ncell_state(cell); }

static double sig(double x) { return 1.0 / (1.0 + exp(-x)); }

/* max that lets a NaN through, so that a non-finite residual is visible */
static double nanmax(double a, double b) {
    if (a != a) return a;
    if (b != b) return b;
    return a > b ? a : b;
}

/* ---- one cell application and its derivatives ------------------------- */

/* s' = f(s, p) for one channel.  p: G pre-activations, w: G weights (may be
 * NULL for the linear cell), s: S state values. */
void oracle_cell_step(int cell, const double* p, const double* w, const double* s, double* out) {
    if (cell == 0) {
        out[0] = p[0] * s[0] + p[1];
    } else if (cell == 1) {
        double h = s[0];
        double z = sig(p[0] + w[0] * h);
        double r = sig(p[1] + w[1] * h);
        double c = tanh(p[2] + w[2] * r * h);
        out[0] = (1.0 - z) * h + z * c;
    } else {
        double c = s[0], h = s[1];
        double ig = sig(p[0] + w[0] * h);
        double fg = sig(p[1] + w[1] * h + 1.0);
        double og = sig(p[2] + w[2] * h);
        double gg = tanh(p[3] + w[3] * h);
        double cn = fg * c + ig * gg;
        out[0] = cn;
        out[1] = og * tanh(cn);
    }
}

/* A = d f / d s at (s, p), S x S row-major: A[i*S + j] = d s'_i / d s_j. */
void oracle_cell_jacobian(int cell, const double* p, const double* w, const double* s, double* A) {
    if (cell == 0) {
        A[0] = p[0];
    } else if (cell == 1) {
        double h = s[0];
        double z = sig(p[0] + w[0] * h);
        double r = sig(p[1] + w[1] * h);
        double c = tanh(p[2] + w[2] * r * h);
        /* d f/d p_z, d f/d p_c, d f/d p_r by the chain rule */
        double Gz = (c - h) * z * (1.0 - z);
        double Gc = z * (1.0 - c * c);
        double Gr = Gc * w[2] * h * r * (1.0 - r);
        /* h enters directly through (1 - z) h, and through each gate's
         * pre-activation: a_z h, a_r h and a_c r h (d(r h)/dh = r + h dr/dh) */
        A[0] = (1.0 - z) + w[0] * Gz + w[1] * Gr + w[2] * r * Gc;
    } else {
        double c = s[0], h = s[1];
        double ig = sig(p[0] + w[0] * h);
        double fg = sig(p[1] + w[1] * h + 1.0);
        double og = sig(p[2] + w[2] * h);
        double gg = tanh(p[3] + w[3] * h);
        double cn = fg * c + ig * gg;
        double tn = tanh(cn);
        double dcn_dh = c * fg * (1.0 - fg) * w[1] + gg * ig * (1.0 - ig) * w[0] + ig * (1.0 - gg * gg) * w[3];
        A[0] = fg;                                   /* dc'/dc */
        A[1] = dcn_dh;                               /* dc'/dh */
        A[2] = og * (1.0 - tn * tn) * fg;            /* dh'/dc */
        A[3] = og * (1.0 - og) * w[2] * tn + og * (1.0 - tn * tn) * dcn_dh; /* dh'/dh */
    }
}

/* dp[i*G + g] = d s'_i / d p_g and da[i*G + g] = d s'_i / d a_g at (s, p). */
void oracle_cell_param_grads(int cell, const double* p, const double* w, const double* s, double* dp, double* da) {
    if (cell == 0) {
        dp[0] = s[0];
        dp[1] = 1.0;
        da[0] = 0.0;
        da[1] = 0.0;
    } else if (cell == 1) {
        double h = s[0];
        double z = sig(p[0] + w[0] * h);
        double r = sig(p[1] + w[1] * h);
        double c = tanh(p[2] + w[2] * r * h);
        double Gz = (c - h) * z * (1.0 - z);
        double Gc = z * (1.0 - c * c);
        double Gr = Gc * w[2] * h * r * (1.0 - r);
        dp[0] = Gz;
        dp[1] = Gr;
        dp[2] = Gc;
        da[0] = Gz * h;
        da[1] = Gr * h;
        da[2] = Gc * r * h;
    } else {
        double c = s[0], h = s[1];
        double ig = sig(p[0] + w[0] * h);
        double fg = sig(p[1] + w[1] * h + 1.0);
        double og = sig(p[2] + w[2] * h);
        double gg = tanh(p[3] + w[3] * h);
        double cn = fg * c + ig * gg;
        double tn = tanh(cn);
        double dc[4], dh[4];
        dc[0] = gg * ig * (1.0 - ig);     /* dc'/dp_i */
        dc[1] = c * fg * (1.0 - fg);      /* dc'/dp_f */
        dc[2] = 0.0;                      /* dc'/dp_o */
        dc[3] = ig * (1.0 - gg * gg);     /* dc'/dp_c */
        for (int g = 0; g < 4; ++g) dh[g] = og * (1.0 - tn * tn) * dc[g];
        dh[2] = og * (1.0 - og) * tn;     /* dh'/dp_o */
        for (int g = 0; g < 4; ++g) {
            dp[0 * 4 + g] = dc[g];
            dp[1 * 4 + g] = dh[g];
            /* every gate's pre-activation carries a_g * h */
            da[0 * 4 + g] = dc[g] * h;
            da[1 * 4 + g] = dh[g] * h;
        }
    }
}

/* ---- per-channel drivers ----------------------------------------------- */

typedef struct {
    int cell, S, G;
    int64_t B, T, D;
    int K;
    int P;                /* Picard sweeps before the Newton iterations */
    const double* px;
    const double* w;
    const double* h0;
    const double* H_in;   /* adjoint: trajectory to linearise at */
    const double* dLdH;
    double* H;            /* unroll / newton output */
    double* dLdpx;
    double* dLda_b;       /* adjoint: per-batch partial (B,G,D) */
    double* dLdh0;
    int mode;             /* 0 unroll, 1 newton, 2 adjoint, 3 residual */
    int nthreads;
    int tid;
    double resid[64];     /* per-thread residual history (K+1 <= 64) */
} job_t;

static void load_p(const job_t* j, int64_t b, int64_t t, int64_t d, double* p) {
    for (int g = 0; g < j->G; ++g) p[g] = j->px[((b * j->T + t) * j->G + g) * j->D + d];
}
static void load_w(const job_t* j, int64_t d, double* w) {
    for (int g = 0; g < j->G; ++g) w[g] = j->w ? j->w[g * j->D + d] : 0.0;
}
static void load_h0(const job_t* j, int64_t b, int64_t d, double* s) {
    for (int i = 0; i < j->S; ++i) s[i] = j->h0 ? j->h0[(b * j->S + i) * j->D + d] : 0.0;
}
static double* Hat(double* H, const job_t* j, int64_t b, int64_t t, int i, int64_t d) {
    return &H[((b * j->T + t) * j->S + i) * j->D + d];
}
static double Hget(const double* H, const job_t* j, int64_t b, int64_t t, int i, int64_t d) {
    return H[((b * j->T + t) * j->S + i) * j->D + d];
}

static void channel_unroll(job_t* j, int64_t b, int64_t d) {
    double w[MAXG], p[MAXG], s[MAXS], sn[MAXS];
    load_w(j, d, w);
    load_h0(j, b, d, s);
    for (int64_t t = 0; t < j->T; ++t) {
        load_p(j, b, t, d, p);
        oracle_cell_step(j->cell, p, w, s, sn);
        for (int i = 0; i < j->S; ++i) {
            s[i] = sn[i];
            *Hat(j->H, j, b, t, i, d) = s[i];
        }
    }
}

/* max_t |h_t - f(h_{t-1}, x_t)| of the trajectory currently stored in H */
static double channel_residual(job_t* j, int64_t b, int64_t d) {
    double w[MAXG], p[MAXG], prev[MAXS], cur[MAXS], fv[MAXS];
    double r = 0.0;
    load_w(j, d, w);
    load_h0(j, b, d, prev);
    for (int64_t t = 0; t < j->T; ++t) {
        load_p(j, b, t, d, p);
        oracle_cell_step(j->cell, p, w, prev, fv);
        for (int i = 0; i < j->S; ++i) {
            cur[i] = Hget(j->H, j, b, t, i, d);
            r = nanmax(r, fabs(cur[i] - fv[i]));
        }
        for (int i = 0; i < j->S; ++i) prev[i] = cur[i];
    }
    return r;
}

static void channel_newton(job_t* j, int64_t b, int64_t d) {
    const int S = j->S;
    double w[MAXG], p[MAXG], zero[MAXS] = {0.0, 0.0}, fv[MAXS];
    load_w(j, d, w);
    /* warm start: h_t^(0) = f(0, x_t) */
    for (int64_t t = 0; t < j->T; ++t) {
        load_p(j, b, t, d, p);
        oracle_cell_step(j->cell, p, w, zero, fv);
        for (int i = 0; i < S; ++i) *Hat(j->H, j, b, t, i, d) = fv[i];
    }
    /* Picard sweeps: h_t^(p+1) = f(h_{t-1}^(p), x_t), h_{-1}^(p) = h0.  The
     * rows are rewritten from the last one back, so that row t-1 still holds
     * sweep p's value when row t is formed. */
    for (int sweep = 0; sweep < j->P; ++sweep) {
        double prev[MAXS];
        for (int64_t t = j->T - 1; t >= 0; --t) {
            load_p(j, b, t, d, p);
            if (t > 0)
                for (int i = 0; i < S; ++i) prev[i] = Hget(j->H, j, b, t - 1, i, d);
            else
                load_h0(j, b, d, prev);
            oracle_cell_step(j->cell, p, w, prev, fv);
            for (int i = 0; i < S; ++i) *Hat(j->H, j, b, t, i, d) = fv[i];
        }
    }
    for (int k = 0; k < j->K; ++k) {
        /* Newton step: J(H) delta = -F(H).  J is lower block-bidiagonal with
         * identity on the diagonal and -A_t below it, so the solve is the
         * forward substitution delta_t = A_t delta_{t-1} - F_t, delta_{-1} = 0. */
        double prev_old[MAXS], cur_old[MAXS], delta[MAXS] = {0.0, 0.0}, nd[MAXS], A[MAXS * MAXS];
        double rk = 0.0;
        load_h0(j, b, d, prev_old);
        for (int64_t t = 0; t < j->T; ++t) {
            load_p(j, b, t, d, p);
            for (int i = 0; i < S; ++i) cur_old[i] = Hget(j->H, j, b, t, i, d);
            oracle_cell_step(j->cell, p, w, prev_old, fv);
            oracle_cell_jacobian(j->cell, p, w, prev_old, A);
            for (int i = 0; i < S; ++i) {
                double F = cur_old[i] - fv[i];
                rk = nanmax(rk, fabs(F));
                double acc = -F;
                for (int m = 0; m < S; ++m) acc += A[i * S + m] * delta[m];
                nd[i] = acc;
            }
            for (int i = 0; i < S; ++i) {
                delta[i] = nd[i];
                *Hat(j->H, j, b, t, i, d) = cur_old[i] + delta[i];
                prev_old[i] = cur_old[i];
            }
        }
        j->resid[k] = nanmax(j->resid[k], rk);
    }
    j->resid[j->K] = nanmax(j->resid[j->K], channel_residual(j, b, d));
}

static void channel_adjoint(job_t* j, int64_t b, int64_t d) {
    const int S = j->S, G = j->G;
    double w[MAXG], p[MAXG], pn[MAXG], s[MAXS], sp[MAXS], A[MAXS * MAXS];
    double dp[MAXS * MAXG], da[MAXS * MAXG];
    double lam[MAXS] = {0.0, 0.0}, acc_a[MAXG] = {0.0, 0.0, 0.0, 0.0};
    load_w(j, d, w);
    for (int64_t t = j->T - 1; t >= 0; --t) {
        /* lambda_t = g_t + A_{t+1}^T lambda_{t+1}, A_{t+1} = df/ds at (h_t, x_{t+1}) */
        double nl[MAXS];
        for (int i = 0; i < S; ++i) nl[i] = j->dLdH[((b * j->T + t) * S + i) * j->D + d];
        if (t + 1 < j->T) {
            load_p(j, b, t + 1, d, pn);
            for (int i = 0; i < S; ++i) s[i] = Hget(j->H_in, j, b, t, i, d);
            oracle_cell_jacobian(j->cell, pn, w, s, A);
            for (int i = 0; i < S; ++i)
                for (int m = 0; m < S; ++m) nl[i] += A[m * S + i] * lam[m];
        }
        for (int i = 0; i < S; ++i) lam[i] = nl[i];
        /* parameter gradients of row t, linearised at (h_{t-1}, x_t) */
        load_p(j, b, t, d, p);
        if (t > 0)
            for (int i = 0; i < S; ++i) sp[i] = Hget(j->H_in, j, b, t - 1, i, d);
        else
            load_h0(j, b, d, sp);
        oracle_cell_param_grads(j->cell, p, w, sp, dp, da);
        for (int g = 0; g < G; ++g) {
            double gp = 0.0, ga = 0.0;
            for (int i = 0; i < S; ++i) {
                gp += lam[i] * dp[i * G + g];
                ga += lam[i] * da[i * G + g];
            }
            j->dLdpx[((b * j->T + t) * G + g) * j->D + d] = gp;
            acc_a[g] += ga;
        }
    }
    for (int g = 0; g < G; ++g) j->dLda_b[(b * G + g) * j->D + d] = acc_a[g];
    if (j->dLdh0) {
        /* dL/dh0 = A_0^T lambda_0 with A_0 = df/ds at (h0, x_0) */
        load_p(j, b, 0, d, p);
        load_h0(j, b, d, sp);
        oracle_cell_jacobian(j->cell, p, w, sp, A);
        for (int i = 0; i < S; ++i) {
            double acc = 0.0;
            for (int m = 0; m < S; ++m) acc += A[m * S + i] * lam[m];
            j->dLdh0[(b * S + i) * j->D + d] = acc;
        }
    }
}

static void* worker(void* arg) {
    job_t* j = (job_t*)arg;
    int64_t nch = j->B * j->D;
    int64_t per = (nch + j->nthreads - 1) / j->nthreads;
    int64_t lo = (int64_t)j->tid * per, hi = lo + per < nch ? lo + per : nch;
    for (int64_t c = lo; c < hi; ++c) {
        int64_t b = c / j->D, d = c % j->D;
        if (j->mode == 0) channel_unroll(j, b, d);
        else if (j->mode == 1) channel_newton(j, b, d);
        else if (j->mode == 2) channel_adjoint(j, b, d);
        else j->resid[0] = nanmax(j->resid[0], channel_residual(j, b, d));
    }
    return NULL;
}

static int run(job_t* proto, int nthreads) {
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    job_t* jobs = (job_t*)calloc((size_t)nthreads, sizeof(job_t));
    pthread_t* th = (pthread_t*)calloc((size_t)nthreads, sizeof(pthread_t));
    if (!jobs || !th) { free(jobs); free(th); return -2; }
    for (int i = 0; i < nthreads; ++i) {
        jobs[i] = *proto;
        jobs[i].nthreads = nthreads;
        jobs[i].tid = i;
        for (int k = 0; k < 64; ++k) jobs[i].resid[k] = 0.0;
    }
    for (int i = 1; i < nthreads; ++i) pthread_create(&th[i], NULL, worker, &jobs[i]);
    worker(&jobs[0]);
    for (int i = 1; i < nthreads; ++i) pthread_join(th[i], NULL);
    for (int k = 0; k < 64; ++k) {
        double r = 0.0;
        for (int i = 0; i < nthreads; ++i) r = nanmax(r, jobs[i].resid[k]);
        proto->resid[k] = r;
    }
    free(jobs);
    free(th);
    return 0;
}

static int check(int cell, int64_t B, int64_t T, int64_t D, const double* px) {
    if (ncell_gates(cell) < 0 || B < 0 || T < 0 || D < 0 || (B * T * D > 0 && !px)) return -1;
    return 0;
}

/* Sequential unroll.  Returns 0 on success, negative on bad arguments. */
int oracle_unroll(int cell, int64_t B, int64_t T, int64_t D, const double* px, const double* w,
                  const double* h0, double* H, int nthreads) {
    if (check(cell, B, T, D, px) || (cell != 0 && !w)) return -1;
    job_t j;
    memset(&j, 0, sizeof j);
    j.cell = cell; j.S = ncell_state(cell); j.G = ncell_gates(cell);
    j.B = B; j.T = T; j.D = D; j.px = px; j.w = w; j.h0 = h0; j.H = H; j.mode = 0;
    return run(&j, nthreads);
}

/* P Picard sweeps from the warm start, then K Newton iterations.  resid
 * (K+1 doubles, may be NULL) receives max |F(H^(k))| over the whole batch for
 * k = 0..K, H^(0) being the guess after the sweeps. */
int oracle_newton_picard(int cell, int64_t B, int64_t T, int64_t D, const double* px, const double* w,
                         const double* h0, int P, int K, double* H, double* resid, int nthreads) {
    if (check(cell, B, T, D, px) || (cell != 0 && !w) || K < 0 || K > 62 || P < 0) return -1;
    job_t j;
    memset(&j, 0, sizeof j);
    j.cell = cell; j.S = ncell_state(cell); j.G = ncell_gates(cell);
    j.B = B; j.T = T; j.D = D; j.K = K; j.P = P; j.px = px; j.w = w; j.h0 = h0; j.H = H; j.mode = 1;
    int rc = run(&j, nthreads);
    if (rc == 0 && resid)
        for (int k = 0; k <= K; ++k) resid[k] = j.resid[k];
    return rc;
}

/* K Newton iterations from the warm start (no Picard sweep). */
int oracle_newton(int cell, int64_t B, int64_t T, int64_t D, const double* px, const double* w,
                  const double* h0, int K, double* H, double* resid, int nthreads) {
    return oracle_newton_picard(cell, B, T, D, px, w, h0, 0, K, H, resid, nthreads);
}

/* max |F(H)| = max_{b,t,s,d} |H_t - f(H_{t-1}, x_t)| (H_{-1} = h0) of a given
 * trajectory H, the quantity the residual history records; channels are
 * shared among nthreads threads.  Returns a negative value on bad arguments. */
double oracle_residual(int cell, int64_t B, int64_t T, int64_t D, const double* px, const double* w,
                       const double* h0, const double* H, int nthreads) {
    if (check(cell, B, T, D, px) || (cell != 0 && !w) || (B * T * D > 0 && !H)) return -1.0;
    job_t j;
    memset(&j, 0, sizeof j);
    j.cell = cell; j.S = ncell_state(cell); j.G = ncell_gates(cell);
    j.B = B; j.T = T; j.D = D; j.px = px; j.w = w; j.h0 = h0; j.H = (double*)H; j.mode = 3;
    if (run(&j, nthreads)) return -2.0;
    return j.resid[0];
}

/* Adjoint at trajectory H: dL_dpx (B,T,G,D), dL_da (G,D) summed over b then
 * t in natural order (may be NULL), dL_dh0 (B,S,D, may be NULL). */
int oracle_adjoint(int cell, int64_t B, int64_t T, int64_t D, const double* px, const double* w,
                   const double* h0, const double* H, const double* dLdH, double* dLdpx, double* dLda,
                   double* dLdh0, int nthreads) {
    if (check(cell, B, T, D, px) || (cell != 0 && !w) || !H || !dLdH || !dLdpx) return -1;
    int G = ncell_gates(cell);
    double* part = (double*)calloc((size_t)(B * G * D > 0 ? B * G * D : 1), sizeof(double));
    if (!part) return -2;
    job_t j;
    memset(&j, 0, sizeof j);
    j.cell = cell; j.S = ncell_state(cell); j.G = G;
    j.B = B; j.T = T; j.D = D; j.px = px; j.w = w; j.h0 = h0; j.H_in = H; j.dLdH = dLdH;
    j.dLdpx = dLdpx; j.dLda_b = part; j.dLdh0 = dLdh0; j.mode = 2;
    int rc = run(&j, nthreads);
    if (rc == 0 && dLda) {
        for (int g = 0; g < G; ++g)
            for (int64_t d = 0; d < D; ++d) {
                double acc = 0.0;
                for (int64_t b = 0; b < B; ++b) acc += part[(b * G + g) * D + d];
                dLda[g * D + d] = acc;
            }
    }
    free(part);
    return rc;
}

/* ==== head-wise GRU (block-diagonal recurrent weights) ====================
 *
 * The ParaGRU(mix='head', n_heads) variant of the pararnn-torch page
 * (Models / Usage, "Dreamer-style block GRU": block-diagonal A, one dense
 * block per head).  The page prints no equations; the reading here is the
 * GRU of torch.nn.GRUCell with its recurrent weight restricted to
 * block-diagonal form, written with this file's gate convention.  For one
 * head of width d, state s (d values), pre-activations p = (p_z, p_r, p_c)
 * (3 x d) and recurrent weights U_z, U_r, U_c (d x d each):
 *     z = sig(p_z + U_z s),  r = sig(p_r + U_r s),  n = U_c s,
 *     c = tanh(p_c + r * n), f = (1 - z) * s + z * c        (elementwise *)
 * which is the diagonal GRU above when the U_g are diagonal.  Its Jacobian
 * with respect to s is the dense d x d block
 *     A = diag(1 - z) + diag(alpha) U_z + diag(beta) U_r + diag(gamma) U_c,
 *     alpha = (c - s) z (1 - z),  beta = z (1 - c^2) n r (1 - r),
 *     gamma = z (1 - c^2) r.
 * Layouts (row-major): px (B,T,3,D) with D = n_heads * d and head h owning
 * channels h*d .. h*d+d-1; U (3, n_heads, d, d) with U[g][h][i][j] the
 * weight of state j in gate pre-activation i; h0 (B,D); H (B,T,D).
 */

/* one head, one step: out = f(s, p); p holds p_z[0..d), p_r[0..d), p_c[0..d);
 * U holds U_z, U_r, U_c of the head, each d x d */
void oracle_head_gru_step(int d, const double* p, const double* U, const double* s, double* out) {
    const double* Uz = U;
    const double* Ur = U + (size_t)d * d;
    const double* Uc = U + 2 * (size_t)d * d;
    for (int i = 0; i < d; ++i) {
        double az = p[i], ar = p[d + i], n = 0.0;
        for (int j = 0; j < d; ++j) {
            az += Uz[(size_t)i * d + j] * s[j];
            ar += Ur[(size_t)i * d + j] * s[j];
            n += Uc[(size_t)i * d + j] * s[j];
        }
        double z = sig(az), r = sig(ar), c = tanh(p[2 * d + i] + r * n);
        out[i] = (1.0 - z) * s[i] + z * c;
    }
}

/* A[i*d + j] = d f_i / d s_j at (s, p) */
void oracle_head_gru_jacobian(int d, const double* p, const double* U, const double* s, double* A) {
    const double* Uz = U;
    const double* Ur = U + (size_t)d * d;
    const double* Uc = U + 2 * (size_t)d * d;
    for (int i = 0; i < d; ++i) {
        double az = p[i], ar = p[d + i], n = 0.0;
        for (int j = 0; j < d; ++j) {
            az += Uz[(size_t)i * d + j] * s[j];
            ar += Ur[(size_t)i * d + j] * s[j];
            n += Uc[(size_t)i * d + j] * s[j];
        }
        double z = sig(az), r = sig(ar), c = tanh(p[2 * d + i] + r * n);
        double alpha = (c - s[i]) * z * (1.0 - z);
        double beta = z * (1.0 - c * c) * n * r * (1.0 - r);
        double gamma = z * (1.0 - c * c) * r;
        for (int j = 0; j < d; ++j)
            A[(size_t)i * d + j] = (i == j ? 1.0 - z : 0.0) + alpha * Uz[(size_t)i * d + j] +
                                   beta * Ur[(size_t)i * d + j] + gamma * Uc[(size_t)i * d + j];
    }
}

typedef struct {
    int64_t B, T, D;
    int nh, d, K, mode, nthreads, tid;
    const double *px, *U, *h0;
    double* H;
    double resid[64];
} hjob_t;

/* pre-activations of head h at (b, t), gathered as p_z, p_r, p_c */
static void head_p(const hjob_t* j, int64_t b, int64_t t, int h, double* p) {
    for (int g = 0; g < 3; ++g)
        for (int i = 0; i < j->d; ++i) p[g * j->d + i] = j->px[((b * j->T + t) * 3 + g) * j->D + (int64_t)h * j->d + i];
}

static const double* head_U(const hjob_t* j, int h, double* buf) {
    /* U_z, U_r, U_c of head h gathered contiguously */
    size_t dd = (size_t)j->d * j->d;
    for (int g = 0; g < 3; ++g) memcpy(buf + g * dd, j->U + ((size_t)g * j->nh + h) * dd, dd * sizeof(double));
    return buf;
}

static void head_h0(const hjob_t* j, int64_t b, int h, double* s) {
    for (int i = 0; i < j->d; ++i) s[i] = j->h0 ? j->h0[b * j->D + (int64_t)h * j->d + i] : 0.0;
}

static void head_seq(hjob_t* j, int64_t b, int h) {
    const int d = j->d;
    const int64_t T = j->T;
    size_t dd = (size_t)d * d;
    double* Ubuf = (double*)malloc(3 * dd * sizeof(double));
    double* s = (double*)malloc((size_t)(T > 0 ? T : 1) * d * sizeof(double));   /* iterate, (T, d) */
    double* del = (double*)malloc((size_t)d * sizeof(double));
    double* F = (double*)malloc((size_t)d * sizeof(double));
    double* A = (double*)malloc(dd * sizeof(double));
    double* p = (double*)malloc(3 * (size_t)d * sizeof(double));
    double* prev = (double*)malloc((size_t)d * sizeof(double));
    double* fv = (double*)malloc((size_t)d * sizeof(double));
    double* tmp = (double*)malloc((size_t)d * sizeof(double));
    const double* U = head_U(j, h, Ubuf);
    if (j->mode == 0) {
        /* sequential unroll */
        head_h0(j, b, h, prev);
        for (int64_t t = 0; t < T; ++t) {
            head_p(j, b, t, h, p);
            oracle_head_gru_step(d, p, U, prev, s + t * d);
            memcpy(prev, s + t * d, d * sizeof(double));
        }
    } else {
        /* warm start s^(0)_t = f(0, x_t) */
        for (int i = 0; i < d; ++i) tmp[i] = 0.0;
        for (int64_t t = 0; t < T; ++t) {
            head_p(j, b, t, h, p);
            oracle_head_gru_step(d, p, U, tmp, s + t * d);
        }
        for (int k = 0; k <= j->K; ++k) {
            /* residual F(s^(k)), then (k < K) the Newton step: A_t at s_{t-1},
             * delta_t = A_t delta_{t-1} - F_t by forward substitution */
            double rk = 0.0;
            for (int i = 0; i < d; ++i) del[i] = 0.0;
            head_h0(j, b, h, prev);
            for (int64_t t = 0; t < T; ++t) {
                head_p(j, b, t, h, p);
                oracle_head_gru_step(d, p, U, prev, fv);
                for (int i = 0; i < d; ++i) {
                    F[i] = s[t * d + i] - fv[i];
                    rk = nanmax(rk, fabs(F[i]));
                }
                if (k < j->K) {
                    oracle_head_gru_jacobian(d, p, U, prev, A);
                    for (int i = 0; i < d; ++i) {
                        double acc = -F[i];
                        for (int m = 0; m < d; ++m) acc += A[(size_t)i * d + m] * del[m];
                        tmp[i] = acc;
                    }
                    memcpy(del, tmp, d * sizeof(double));
                }
                memcpy(prev, s + t * d, d * sizeof(double));   /* s^(k)_t, the next row's s_{t-1} */
                if (k < j->K)
                    for (int i = 0; i < d; ++i) s[t * d + i] += del[i];
            }
            j->resid[k] = nanmax(j->resid[k], rk);
        }
    }
    for (int64_t t = 0; t < T; ++t)
        for (int i = 0; i < d; ++i) j->H[(b * T + t) * j->D + (int64_t)h * d + i] = s[t * d + i];
    free(Ubuf); free(s); free(del); free(F); free(A); free(p); free(prev); free(fv); free(tmp);
}

static void* head_worker(void* arg) {
    hjob_t* j = (hjob_t*)arg;
    int64_t nseq = j->B * j->nh;
    int64_t per = (nseq + j->nthreads - 1) / j->nthreads;
    int64_t lo = (int64_t)j->tid * per, hi = lo + per < nseq ? lo + per : nseq;
    for (int64_t q = lo; q < hi; ++q) head_seq(j, q / j->nh, (int)(q % j->nh));
    return NULL;
}

static int head_run(hjob_t* proto, int nthreads) {
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    hjob_t* jobs = (hjob_t*)calloc((size_t)nthreads, sizeof(hjob_t));
    pthread_t* th = (pthread_t*)calloc((size_t)nthreads, sizeof(pthread_t));
    if (!jobs || !th) { free(jobs); free(th); return -2; }
    for (int i = 0; i < nthreads; ++i) {
        jobs[i] = *proto;
        jobs[i].nthreads = nthreads;
        jobs[i].tid = i;
        for (int k = 0; k < 64; ++k) jobs[i].resid[k] = 0.0;
    }
    for (int i = 1; i < nthreads; ++i) pthread_create(&th[i], NULL, head_worker, &jobs[i]);
    head_worker(&jobs[0]);
    for (int i = 1; i < nthreads; ++i) pthread_join(th[i], NULL);
    for (int k = 0; k < 64; ++k) {
        double r = 0.0;
        for (int i = 0; i < nthreads; ++i) r = nanmax(r, jobs[i].resid[k]);
        proto->resid[k] = r;
    }
    free(jobs);
    free(th);
    return 0;
}

static int head_check(int64_t B, int64_t T, int64_t D, int nh, const double* px, const double* U) {
    if (B < 0 || T < 0 || D < 0 || nh < 1 || D % nh != 0 || (B * T * D > 0 && (!px || !U))) return -1;
    return 0;
}

/* Sequential unroll of the head-wise GRU. */
int oracle_head_gru_unroll(int64_t B, int64_t T, int64_t D, int nh, const double* px, const double* U,
                           const double* h0, double* H, int nthreads) {
    if (head_check(B, T, D, nh, px, U)) return -1;
    hjob_t j;
    memset(&j, 0, sizeof j);
    j.B = B; j.T = T; j.D = D; j.nh = nh; j.d = (int)(D / nh); j.px = px; j.U = U; j.h0 = h0; j.H = H; j.mode = 0;
    return head_run(&j, nthreads);
}

/* K Newton iterations of the head-wise GRU from the warm start; resid (K+1
 * doubles, may be NULL) receives max |F(H^(k))| for k = 0..K. */
int oracle_head_gru_newton(int64_t B, int64_t T, int64_t D, int nh, const double* px, const double* U,
                           const double* h0, int K, double* H, double* resid, int nthreads) {
    if (head_check(B, T, D, nh, px, U) || K < 0 || K > 62) return -1;
    hjob_t j;
    memset(&j, 0, sizeof j);
    j.B = B; j.T = T; j.D = D; j.nh = nh; j.d = (int)(D / nh); j.K = K; j.px = px; j.U = U; j.h0 = h0; j.H = H;
    j.mode = 1;
    int rc = head_run(&j, nthreads);
    if (rc == 0 && resid)
        for (int k = 0; k <= K; ++k) resid[k] = j.resid[k];
    return rc;
}

/* ---- head-wise GRU: the adjoint ------------------------------------------
 * At a trajectory H (the forward's output), g_t = dL/dH_t, per head:
 *     lambda_t = g_t + A_{t+1}^T lambda_{t+1},  lambda_{T-1} = g_{T-1},
 * with A_{t+1} the Jacobian at (h_t, x_{t+1}); then, with the gate factors
 * at (h_{t-1}, x_t) (h_{-1} = h0):
 *     dL/dp_z = lambda * alpha,  dL/dp_r = lambda * beta,
 *     dL/dp_c = lambda * z (1 - c^2),
 *     dL/dU_z[i][j] = sum_{b,t} lambda_i alpha_i h_{t-1,j}   (likewise U_r with
 *     beta, U_c with gamma), summed over b then t in natural order,
 *     dL/dh0 = A_0^T lambda_0.
 * Layouts: dL_dH (B,T,D), dL_dpx (B,T,3,D), dL_dU (3, n_heads, d, d),
 * dL_dh0 (B,D). */

typedef struct {
    int64_t B, T, D;
    int nh, d, nthreads, tid;
    const double *px, *U, *h0, *H, *g;
    double *dpx, *dU_b, *dh0;  /* dU_b: per batch row partials [B][3][nh][d][d] */
} ajob_t;

/* the gate factors of head h at (s, x_t): alpha, beta, z (1 - c^2), gamma */
static void head_factors(int d, const double* p, const double* U, const double* s, double* al, double* be, double* zc,
                         double* ga) {
    const double* Uz = U;
    const double* Ur = U + (size_t)d * d;
    const double* Uc = U + 2 * (size_t)d * d;
    for (int i = 0; i < d; ++i) {
        double az = p[i], ar = p[d + i], n = 0.0;
        for (int j = 0; j < d; ++j) {
            az += Uz[(size_t)i * d + j] * s[j];
            ar += Ur[(size_t)i * d + j] * s[j];
            n += Uc[(size_t)i * d + j] * s[j];
        }
        double z = sig(az), r = sig(ar), c = tanh(p[2 * d + i] + r * n);
        al[i] = (c - s[i]) * z * (1.0 - z);
        be[i] = z * (1.0 - c * c) * n * r * (1.0 - r);
        zc[i] = z * (1.0 - c * c);
        ga[i] = z * (1.0 - c * c) * r;
    }
}

static void head_adjoint_seq(ajob_t* j, int64_t b, int h) {
    const int d = j->d;
    const int64_t T = j->T;
    size_t dd = (size_t)d * d;
    hjob_t hj;  /* only for the gather helpers */
    memset(&hj, 0, sizeof hj);
    hj.B = j->B; hj.T = j->T; hj.D = j->D; hj.nh = j->nh; hj.d = d; hj.px = j->px; hj.U = j->U; hj.h0 = j->h0;
    double* Ubuf = (double*)malloc(3 * dd * sizeof(double));
    double* lam = (double*)malloc((size_t)d * sizeof(double));
    double* nl = (double*)malloc((size_t)d * sizeof(double));
    double* A = (double*)malloc(dd * sizeof(double));
    double* p = (double*)malloc(3 * (size_t)d * sizeof(double));
    double* prev = (double*)malloc((size_t)d * sizeof(double));
    double* cur = (double*)malloc((size_t)d * sizeof(double));
    double* al = (double*)malloc((size_t)d * sizeof(double));
    double* be = (double*)malloc((size_t)d * sizeof(double));
    double* zc = (double*)malloc((size_t)d * sizeof(double));
    double* ga = (double*)malloc((size_t)d * sizeof(double));
    const double* U = head_U(&hj, h, Ubuf);
    double* dU = j->dU_b + (size_t)b * 3 * j->nh * dd;
    for (int64_t t = T - 1; t >= 0; --t) {
        /* lambda_t = g_t + A_{t+1}^T lambda_{t+1} */
        for (int i = 0; i < d; ++i) lam[i] = j->g[(b * T + t) * j->D + (int64_t)h * d + i] + (t + 1 < T ? nl[i] : 0.0);
        /* state before row t */
        if (t == 0) head_h0(&hj, b, h, prev);
        else
            for (int i = 0; i < d; ++i) prev[i] = j->H[(b * T + t - 1) * j->D + (int64_t)h * d + i];
        head_p(&hj, b, t, h, p);
        head_factors(d, p, U, prev, al, be, zc, ga);
        for (int i = 0; i < d; ++i) {
            const int64_t o = ((b * T + t) * 3) * j->D + (int64_t)h * d + i;
            j->dpx[o] = lam[i] * al[i];
            j->dpx[o + j->D] = lam[i] * be[i];
            j->dpx[o + 2 * j->D] = lam[i] * zc[i];
            for (int m = 0; m < d; ++m) {
                dU[((size_t)0 * j->nh + h) * dd + (size_t)i * d + m] += lam[i] * al[i] * prev[m];
                dU[((size_t)1 * j->nh + h) * dd + (size_t)i * d + m] += lam[i] * be[i] * prev[m];
                dU[((size_t)2 * j->nh + h) * dd + (size_t)i * d + m] += lam[i] * ga[i] * prev[m];
            }
        }
        /* A_t^T lambda_t: the next (earlier) row's propagated term, and dL/dh0 at t = 0 */
        oracle_head_gru_jacobian(d, p, U, prev, A);
        for (int m = 0; m < d; ++m) {
            double acc = 0.0;
            for (int i = 0; i < d; ++i) acc += A[(size_t)i * d + m] * lam[i];
            cur[m] = acc;
        }
        memcpy(nl, cur, d * sizeof(double));
        if (t == 0 && j->dh0)
            for (int m = 0; m < d; ++m) j->dh0[b * j->D + (int64_t)h * d + m] = cur[m];
    }
    free(Ubuf); free(lam); free(nl); free(A); free(p); free(prev); free(cur); free(al); free(be); free(zc); free(ga);
}

static void* head_adjoint_worker(void* arg) {
    ajob_t* j = (ajob_t*)arg;
    int64_t nseq = j->B * j->nh;
    int64_t per = (nseq + j->nthreads - 1) / j->nthreads;
    int64_t lo = (int64_t)j->tid * per, hi = lo + per < nseq ? lo + per : nseq;
    for (int64_t q = lo; q < hi; ++q) head_adjoint_seq(j, q / j->nh, (int)(q % j->nh));
    return NULL;
}

/* The head-wise GRU adjoint at trajectory H.  dL_dU (may be NULL) is summed
 * over b in natural order (each b's sum over t is in reverse time order, as
 * the recursion runs); dL_dh0 may be NULL. */
int oracle_head_gru_adjoint(int64_t B, int64_t T, int64_t D, int nh, const double* px, const double* U,
                            const double* h0, const double* H, const double* dLdH, double* dLdpx, double* dLdU,
                            double* dLdh0, int nthreads) {
    if (head_check(B, T, D, nh, px, U) || !H || !dLdH || !dLdpx) return -1;
    const int d = (int)(D / nh);
    const size_t per_b = (size_t)3 * nh * d * d;
    double* part = (double*)calloc(B * per_b > 0 ? B * per_b : 1, sizeof(double));
    if (!part) return -2;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    ajob_t proto;
    memset(&proto, 0, sizeof proto);
    proto.B = B; proto.T = T; proto.D = D; proto.nh = nh; proto.d = d; proto.px = px; proto.U = U; proto.h0 = h0;
    proto.H = H; proto.g = dLdH; proto.dpx = dLdpx; proto.dU_b = part; proto.dh0 = dLdh0;
    ajob_t* jobs = (ajob_t*)calloc((size_t)nthreads, sizeof(ajob_t));
    pthread_t* th = (pthread_t*)calloc((size_t)nthreads, sizeof(pthread_t));
    if (!jobs || !th) { free(jobs); free(th); free(part); return -2; }
    for (int i = 0; i < nthreads; ++i) {
        jobs[i] = proto;
        jobs[i].nthreads = nthreads;
        jobs[i].tid = i;
    }
    for (int i = 1; i < nthreads; ++i) pthread_create(&th[i], NULL, head_adjoint_worker, &jobs[i]);
    head_adjoint_worker(&jobs[0]);
    for (int i = 1; i < nthreads; ++i) pthread_join(th[i], NULL);
    if (dLdU)
        for (size_t k = 0; k < per_b; ++k) {
            double acc = 0.0;
            for (int64_t b = 0; b < B; ++b) acc += part[(size_t)b * per_b + k];
            dLdU[k] = acc;
        }
    free(jobs);
    free(th);
    free(part);
    return 0;
}

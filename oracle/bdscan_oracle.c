/*
 * bdscan_oracle.c -- fp64 CPU oracle for the block-diffusion bidirectional
 * Mamba-2 scan.  TEST INFRASTRUCTURE ONLY: it is loaded by the test suite,
 * by the package's smoke check and by the benchmark's CPU-baseline leg, and
 * by nothing on the product path.  It shares no code, header or constant
 * with the CUDA library.
 *
 * What it computes (plain sequential definition, no chunking, no reordering):
 *
 *   Selective state-space update, "Training Hybrid Block Diffusion Language
 *   Models with Partial Bidirectionality" eq. (1), in the Mamba-2 form with a
 *   scalar decay per head (same page, Mamba-2 paragraph):
 *       a_t  = exp(dt_t * A_h)
 *       h_t  = a_t * h_{t-1} + dt_t * x_t B_t^T          (h_t is P x N)
 *       y_t  = h_t C_t + D_h * x_t                         (y_t is P)
 *   optionally gated: y_t <- y_t * silu(z_t).
 *
 *   Forward boundary state over the clean prefix, same page eq. (10):
 *       states[k] = h after the last token of block k   (k = 0 .. L/T-1)
 *   Forward continuation of a block from the cached state, eq. (11).
 *   Reverse scan confined to the block, eq. (12): the same recurrence run
 *   from the block's last token to its first, from a zero state, with the
 *   reverse direction's own parameters.
 *   Combination, eq. (13) (and "Breaking the Bottleneck with DiffuApriel",
 *   section 3.2 eq. (6)): y = y_fwd + y_rev.
 *
 *   All-block objective (first page, eq. (14) and the all-block paragraph
 *   after eq. (5)): every block of the noisy stream is scanned forward from
 *   the clean stream's boundary state before it (h0 for block 0) and gets its
 *   own block-local reverse scan.
 *
 *   The short convolution (+SiLU) in front of the scan, causal for the
 *   forward direction and anti-causal inside the block for the reverse one,
 *   with the conv state of the cache (see the section before
 *   oracle_max_threads for its definition and citations).
 *
 *   The gated RMSNorm of the summed output (same place).
 *
 * Layouts (row-major, innermost last):
 *   x, z, y  [B][L][H][P]    dt [B][L][H]    Bm, Cm [B][L][G][N]
 *   A, D     [H]             state [B][H][P][N]   states [B][K][H][P][N]
 *   head h uses group g = h / (H / G).
 *
 * Everything is double precision; inputs are the exact values the device
 * path consumes, widened to double by the caller.  exp() is libm's.
 * Parallelised with OpenMP over (batch, head): every (b, h) pair is an
 * independent recurrence, so the result does not depend on the thread count.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct {
    int64_t batch, seqlen, nheads, headdim, dstate, ngroups, block_len;
} oracle_shape_t;

typedef struct {
    const double *x, *dt, *Bm, *Cm, *z; /* z may be NULL (no gate) */
    const double *A, *D;                /* [H] */
} oracle_dir_t;

enum { ORACLE_OK = 0, ORACLE_EINVAL = -1, ORACLE_ENOMEM = -2 };

static int check_shape(const oracle_shape_t *s) {
    if (!s) return ORACLE_EINVAL;
    if (s->batch < 0 || s->seqlen < 0 || s->nheads < 1 || s->headdim < 1 ||
        s->dstate < 1 || s->ngroups < 1 || s->block_len < 1)
        return ORACLE_EINVAL;
    if (s->nheads % s->ngroups) return ORACLE_EINVAL;
    if (s->seqlen % s->block_len) return ORACLE_EINVAL;
    return ORACLE_OK;
}

static int check_dir(const oracle_dir_t *d) {
    if (!d || !d->x || !d->dt || !d->Bm || !d->Cm || !d->A || !d->D) return ORACLE_EINVAL;
    return ORACLE_OK;
}

static double silu(double v) { return v / (1.0 + exp(-v)); }

/* One step of eq. (1) for token t of (b, h): update hs in place and write the
 * direction's output y_t into ydir (length P). */
static void ssm_step(const oracle_shape_t *s, const oracle_dir_t *d, int64_t b, int64_t h,
                     int64_t t, double *hs, double *ydir) {
    const int64_t L = s->seqlen, H = s->nheads, P = s->headdim, N = s->dstate, G = s->ngroups;
    const int64_t g = h / (H / G);
    const double dt = d->dt[(b * L + t) * H + h];
    const double a = exp(dt * d->A[h]);
    const double *x = d->x + ((b * L + t) * H + h) * P;
    const double *Bt = d->Bm + ((b * L + t) * G + g) * N;
    const double *Ct = d->Cm + ((b * L + t) * G + g) * N;
    for (int64_t p = 0; p < P; ++p) {
        double acc = 0.0;
        double *row = hs + p * N;
        for (int64_t n = 0; n < N; ++n) {
            row[n] = a * row[n] + dt * x[p] * Bt[n];
            acc += Ct[n] * row[n];
        }
        double yp = acc + d->D[h] * x[p];
        if (d->z) yp *= silu(d->z[((b * L + t) * H + h) * P + p]);
        ydir[p] = yp;
    }
}

/* Forward scan of tokens [t0, t1) of (b, h) from the state in hs (modified).
 * The outputs are ADDED into y (so a forward and a reverse pass sum, eq. (13)).
 * If states != NULL, the state after the last token of every block is stored
 * at states[b][k][h] (boundary-state index rule: k = t / T for t = (k+1)T - 1). */
static void scan_forward(const oracle_shape_t *s, const oracle_dir_t *d, int64_t b, int64_t h,
                         int64_t t0, int64_t t1, double *hs, double *y, double *states,
                         double *ydir) {
    const int64_t L = s->seqlen, H = s->nheads, P = s->headdim, N = s->dstate, T = s->block_len;
    const int64_t K = L / T;
    for (int64_t t = t0; t < t1; ++t) {
        ssm_step(s, d, b, h, t, hs, ydir);
        double *yo = y + ((b * L + t) * H + h) * P;
        for (int64_t p = 0; p < P; ++p) yo[p] += ydir[p];
        if (states && (t + 1) % T == 0) {
            const int64_t k = t / T;
            memcpy(states + ((b * K + k) * H + h) * P * N, hs, sizeof(double) * P * N);
        }
    }
}

/* Block-local reverse scan, eq. (12): tokens t1-1 down to t0 from a zero
 * state; outputs added into y. */
static void scan_reverse(const oracle_shape_t *s, const oracle_dir_t *d, int64_t b, int64_t h,
                         int64_t t0, int64_t t1, double *hs, double *y, double *ydir) {
    const int64_t L = s->seqlen, H = s->nheads, P = s->headdim, N = s->dstate;
    memset(hs, 0, sizeof(double) * P * N);
    for (int64_t t = t1 - 1; t >= t0; --t) {
        ssm_step(s, d, b, h, t, hs, ydir);
        double *yo = y + ((b * L + t) * H + h) * P;
        for (int64_t p = 0; p < P; ++p) yo[p] += ydir[p];
    }
}

static void load_state(double *hs, const double *src, int64_t b, int64_t h, int64_t H,
                       int64_t PN) {
    if (src)
        memcpy(hs, src + (b * H + h) * PN, sizeof(double) * PN);
    else
        memset(hs, 0, sizeof(double) * PN);
}

/* Clean-stream pass used by prefix and allblock: forward scan over the whole
 * sequence from h0 with boundary states, then (if rev) a block-local reverse
 * scan of every block.  y must be zeroed by the caller. */
static void clean_pass(const oracle_shape_t *s, const oracle_dir_t *fwd, const oracle_dir_t *rev,
                       const double *h0, double *y, double *states, double *final_state,
                       int64_t b, int64_t h, double *hs, double *ydir) {
    const int64_t L = s->seqlen, H = s->nheads, PN = s->headdim * s->dstate, T = s->block_len;
    load_state(hs, h0, b, h, H, PN);
    scan_forward(s, fwd, b, h, 0, L, hs, y, states, ydir);
    if (final_state) memcpy(final_state + (b * H + h) * PN, hs, sizeof(double) * PN);
    if (rev)
        for (int64_t t0 = 0; t0 < L; t0 += T) scan_reverse(s, rev, b, h, t0, t0 + T, hs, y, ydir);
}

int oracle_prefix(const oracle_shape_t *s, const oracle_dir_t *fwd, const oracle_dir_t *rev,
                  const double *h0, double *y, double *states, double *final_state) {
    int rc = check_shape(s);
    if (rc || (rc = check_dir(fwd))) return rc;
    if (rev && (rc = check_dir(rev))) return rc;
    if (!y) return ORACLE_EINVAL;
    const int64_t B = s->batch, L = s->seqlen, H = s->nheads, P = s->headdim, N = s->dstate;
    memset(y, 0, sizeof(double) * B * L * H * P);
    int failed = 0;
#pragma omp parallel
    {
        double *hs = (double *)malloc(sizeof(double) * P * N);
        double *ydir = (double *)malloc(sizeof(double) * P);
        if (!hs || !ydir) {
#pragma omp atomic write
            failed = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t bh = 0; bh < B * H; ++bh)
                clean_pass(s, fwd, rev, h0, y, states, final_state, bh / H, bh % H, hs, ydir);
        }
        free(hs);
        free(ydir);
    }
    return failed ? ORACLE_ENOMEM : ORACLE_OK;
}

/* One denoising step on a single block (seqlen == block_len): forward from
 * state_in (eq. (11)), block-local reverse (eq. (12)), sum (eq. (13)).  If
 * state_out != NULL it receives the forward state after the block (the
 * commit that appends the block to the cache). */
int oracle_block_step(const oracle_shape_t *s, const oracle_dir_t *fwd, const oracle_dir_t *rev,
                      const double *state_in, double *y, double *state_out) {
    int rc = check_shape(s);
    if (rc || (rc = check_dir(fwd))) return rc;
    if (rev && (rc = check_dir(rev))) return rc;
    if (!y || s->seqlen != s->block_len) return ORACLE_EINVAL;
    oracle_shape_t one = *s;
    return oracle_prefix(&one, fwd, rev, state_in, y, NULL, state_out);
}

/* All-block pass: clean stream as in prefix (outputs y_clean, states); then
 * every noisy block k scanned forward from (k == 0 ? h0 : states[k-1]) plus
 * its block-local reverse, into y_noisy.  y_clean may be NULL. */
int oracle_allblock(const oracle_shape_t *s, const oracle_dir_t *cf, const oracle_dir_t *cr,
                    const oracle_dir_t *nf, const oracle_dir_t *nr, const double *h0,
                    double *y_clean, double *y_noisy, double *states) {
    int rc = check_shape(s);
    if (rc || (rc = check_dir(cf)) || (rc = check_dir(nf))) return rc;
    if (cr && (rc = check_dir(cr))) return rc;
    if (nr && (rc = check_dir(nr))) return rc;
    if (!y_noisy || !states) return ORACLE_EINVAL;
    const int64_t B = s->batch, L = s->seqlen, H = s->nheads, P = s->headdim, N = s->dstate;
    const int64_t T = s->block_len, K = L / T, PN = P * N;
    double *yc = y_clean;
    double *yc_own = NULL;
    if (!yc) {
        yc_own = (double *)malloc(sizeof(double) * (B * L * H * P > 0 ? B * L * H * P : 1));
        if (!yc_own) return ORACLE_ENOMEM;
        yc = yc_own;
    }
    memset(yc, 0, sizeof(double) * B * L * H * P);
    memset(y_noisy, 0, sizeof(double) * B * L * H * P);
    int failed = 0;
#pragma omp parallel
    {
        double *hs = (double *)malloc(sizeof(double) * PN);
        double *ydir = (double *)malloc(sizeof(double) * P);
        if (!hs || !ydir) {
#pragma omp atomic write
            failed = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t bh = 0; bh < B * H; ++bh) {
                const int64_t b = bh / H, h = bh % H;
                clean_pass(s, cf, cr, h0, yc, states, NULL, b, h, hs, ydir);
                for (int64_t k = 0; k < K; ++k) {
                    if (k == 0)
                        load_state(hs, h0, b, h, H, PN);
                    else
                        memcpy(hs, states + ((b * K + k - 1) * H + h) * PN, sizeof(double) * PN);
                    scan_forward(s, nf, b, h, k * T, (k + 1) * T, hs, y_noisy, NULL, ydir);
                    if (nr) scan_reverse(s, nr, b, h, k * T, (k + 1) * T, hs, y_noisy, ydir);
                }
            }
        }
        free(hs);
        free(ydir);
    }
    free(yc_own);
    return failed ? ORACLE_ENOMEM : ORACLE_OK;
}

/* ------------------------------------------------------------------ backward
 *
 * Reverse-mode derivative of oracle_allblock (ungated), for the training pass
 * that the all-block objective implies: gradients of a loss
 * L(y_clean, y_noisy, states) reach every input, and through the boundary
 * states the noisy blocks' losses reach the clean prefix scan ("Training
 * Hybrid Block Diffusion Language Models with Partial Bidirectionality",
 * all-block paragraph after eq. (5) and eq. (14)).
 *
 * Plain adjoint of the recurrence of eq. (1), token by token in reverse
 * processing order, with the forward states of each pass recomputed and
 * stored (no chunking).  For a token t with a_t = exp(dt_t A):
 *     G        <- G + dy_t C_t^T                 (dL/dh_t, P x N)
 *     dC_t     += dy_t^T h_t          dx_t += D dy_t + dt_t G B_t
 *     dB_t     += dt_t G^T x_t        dD   += dy_t . x_t
 *     ddt_t    += sum G o (A a_t h_prev + x_t B_t^T)
 *     dA       += sum G o (dt_t a_t h_prev)
 *     G        <- a_t G                          (dL/dh_prev)
 * dB and dC of a group sum over its heads; dA and dD sum over batch and
 * tokens.  Sums are taken in a fixed order (per (b, h) partials, then a
 * serial reduction), so the result does not depend on the thread count. */
typedef struct {
    double *dx, *ddt, *dB, *dC, *dA, *dD; /* any may be NULL (not wanted) */
} oracle_grad_t;

typedef struct {
    double *dx, *ddt; /* [L][P], [L] of this (b, h) */
    double *dB, *dC;  /* [L][N] of this (b, h) (group sums taken later) */
    double dA, dD;
} bwd_acc_t;

/* Backward through the pass that processed tokens order[0..n-1] (in that
 * order) from the state h_start.  G holds dL/d(state after the last processed
 * token) on entry and dL/dh_start on return.  dstate_at(i) (may be NULL)
 * adds the incoming gradient on the state after processed token i.
 * hist: scratch of n * P * N doubles. */
static void pass_backward(const oracle_shape_t *s, const oracle_dir_t *d, int64_t b, int64_t h,
                          const int64_t *order, int64_t n, const double *h_start, const double *dy,
                          const double *const *dstate_at, double *G, double *hist, bwd_acc_t *acc) {
    const int64_t L = s->seqlen, H = s->nheads, P = s->headdim, N = s->dstate, Gn = s->ngroups;
    const int64_t g = h / (H / Gn), PN = P * N;
    /* forward recompute */
    for (int64_t i = 0; i < n; ++i) {
        const int64_t t = order[i];
        const double dt = d->dt[(b * L + t) * H + h];
        const double a = exp(d->A[h] * dt); /* (same decay as the forward pass) */
        const double *x = d->x + ((b * L + t) * H + h) * P;
        const double *Bt = d->Bm + ((b * L + t) * Gn + g) * N;
        const double *prev = i ? hist + (i - 1) * PN : h_start;
        double *cur = hist + i * PN;
        for (int64_t p = 0; p < P; ++p)
            for (int64_t q = 0; q < N; ++q)
                cur[p * N + q] = a * (prev ? prev[p * N + q] : 0.0) + dt * x[p] * Bt[q];
    }
    /* adjoint, reverse processing order */
    for (int64_t i = n - 1; i >= 0; --i) {
        const int64_t t = order[i];
        const double dt = d->dt[(b * L + t) * H + h];
        const double A = d->A[h];
        const double a = exp(dt * A);
        const double *x = d->x + ((b * L + t) * H + h) * P;
        const double *Bt = d->Bm + ((b * L + t) * Gn + g) * N;
        const double *Ct = d->Cm + ((b * L + t) * Gn + g) * N;
        const double *dyt = dy ? dy + ((b * L + t) * H + h) * P : NULL;
        const double *ht = hist + i * PN;
        const double *prev = i ? hist + (i - 1) * PN : h_start;
        if (dstate_at && dstate_at[i])
            for (int64_t e = 0; e < PN; ++e) G[e] += dstate_at[i][e];
        if (dyt)
            for (int64_t p = 0; p < P; ++p)
                for (int64_t q = 0; q < N; ++q) G[p * N + q] += dyt[p] * Ct[q];
        double ddt = 0.0, dA = 0.0;
        for (int64_t p = 0; p < P; ++p) {
            double gb = 0.0;
            for (int64_t q = 0; q < N; ++q) {
                const double Gv = G[p * N + q];
                const double hp = prev ? prev[p * N + q] : 0.0;
                gb += Gv * Bt[q];
                ddt += Gv * (A * a * hp + x[p] * Bt[q]);
                dA += Gv * dt * a * hp;
            }
            acc->dx[t * P + p] += dt * gb + (dyt ? d->D[h] * dyt[p] : 0.0);
        }
        for (int64_t q = 0; q < N; ++q) {
            double sb = 0.0, sc = 0.0;
            for (int64_t p = 0; p < P; ++p) {
                sb += G[p * N + q] * x[p];
                if (dyt) sc += dyt[p] * ht[p * N + q];
            }
            acc->dB[t * N + q] += dt * sb;
            acc->dC[t * N + q] += sc;
        }
        if (dyt)
            for (int64_t p = 0; p < P; ++p) acc->dD += dyt[p] * x[p];
        acc->ddt[t] += ddt;
        acc->dA += dA;
        for (int64_t e = 0; e < PN; ++e) G[e] *= a;
    }
}

int oracle_allblock_backward(const oracle_shape_t *s, const oracle_dir_t *cf, const oracle_dir_t *cr,
                             const oracle_dir_t *nf, const oracle_dir_t *nr, const double *h0,
                             const double *dy_clean, const double *dy_noisy, const double *dstates,
                             oracle_grad_t *gcf, oracle_grad_t *gcr, oracle_grad_t *gnf, oracle_grad_t *gnr,
                             double *dh0) {
    int rc = check_shape(s);
    if (rc || (rc = check_dir(cf)) || (rc = check_dir(nf))) return rc;
    if (cr && (rc = check_dir(cr))) return rc;
    if (nr && (rc = check_dir(nr))) return rc;
    if (cf->z || nf->z || (cr && cr->z) || (nr && nr->z)) return ORACLE_EINVAL; /* ungated only */
    if (!gcf || !gnf || (cr && !gcr) || (nr && !gnr)) return ORACLE_EINVAL;
    const int64_t B = s->batch, L = s->seqlen, H = s->nheads, P = s->headdim, N = s->dstate;
    const int64_t Gn = s->ngroups, T = s->block_len, K = L / T, PN = P * N;
    const oracle_dir_t *dirs[4] = {cf, cr, nf, nr};
    oracle_grad_t *grads[4] = {gcf, gcr, gnf, gnr};
    /* forward states of the clean stream (the checkpoints of the pass) */
    double *states = (double *)malloc(sizeof(double) * (B * K * H * PN > 0 ? B * K * H * PN : 1));
    double *ytmp = (double *)malloc(sizeof(double) * (B * L * H * P > 0 ? B * L * H * P : 1));
    /* per (direction, b, h) partials */
    const size_t nbh = (size_t)(B * H);
    bwd_acc_t *acc = (bwd_acc_t *)calloc(4 * (nbh ? nbh : 1), sizeof(bwd_acc_t));
    double *pool = (double *)calloc(4 * (nbh ? nbh : 1) * (size_t)(L * P + L + 2 * L * N), sizeof(double));
    if (!states || !ytmp || !acc || !pool) {
        free(states); free(ytmp); free(acc); free(pool);
        return ORACLE_ENOMEM;
    }
    for (size_t i = 0; i < 4 * nbh; ++i) {
        double *base = pool + i * (size_t)(L * P + L + 2 * L * N);
        acc[i].dx = base;
        acc[i].ddt = base + L * P;
        acc[i].dB = base + L * P + L;
        acc[i].dC = base + L * P + L + L * N;
    }
    rc = oracle_allblock(s, cf, cr, nf, nr, h0, NULL, ytmp, states);
    free(ytmp);
    if (rc) { free(states); free(acc); free(pool); return rc; }
    int failed = 0;
#pragma omp parallel
    {
        double *G = (double *)malloc(sizeof(double) * PN);
        double *hist = (double *)malloc(sizeof(double) * (L > 0 ? L : 1) * PN);
        int64_t *order = (int64_t *)malloc(sizeof(int64_t) * (L > 0 ? L : 1));
        const double **dat = (const double **)calloc(L > 0 ? L : 1, sizeof(double *));
        double *dsn = (double *)malloc(sizeof(double) * (K > 0 ? K : 1) * PN); /* dL/d states[k] from noisy block k+1 */
        if (!G || !hist || !order || !dat || !dsn) {
#pragma omp atomic write
            failed = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t bh = 0; bh < B * H; ++bh) {
                const int64_t b = bh / H, h = bh % H;
                memset(dsn, 0, sizeof(double) * K * PN);
                double *dh0_bh = dh0 ? dh0 + (b * H + h) * PN : NULL;
                if (dh0_bh) memset(dh0_bh, 0, sizeof(double) * PN);
                /* noisy blocks: forward from the clean boundary state before it */
                for (int64_t k = 0; k < K; ++k) {
                    const double *hs0 = k ? states + ((b * K + k - 1) * H + h) * PN
                                          : (h0 ? h0 + (b * H + h) * PN : NULL);
                    for (int64_t i = 0; i < T; ++i) order[i] = k * T + i;
                    memset(G, 0, sizeof(double) * PN);
                    pass_backward(s, nf, b, h, order, T, hs0, dy_noisy, NULL, G, hist, &acc[2 * nbh + bh]);
                    if (k) {
                        for (int64_t e = 0; e < PN; ++e) dsn[(k - 1) * PN + e] += G[e];
                    } else if (dh0_bh) {
                        for (int64_t e = 0; e < PN; ++e) dh0_bh[e] += G[e];
                    }
                    if (nr) {
                        for (int64_t i = 0; i < T; ++i) order[i] = (k + 1) * T - 1 - i;
                        memset(G, 0, sizeof(double) * PN);
                        pass_backward(s, nr, b, h, order, T, NULL, dy_noisy, NULL, G, hist, &acc[3 * nbh + bh]);
                    }
                    if (cr) {
                        for (int64_t i = 0; i < T; ++i) order[i] = (k + 1) * T - 1 - i;
                        memset(G, 0, sizeof(double) * PN);
                        pass_backward(s, cr, b, h, order, T, NULL, dy_clean, NULL, G, hist, &acc[1 * nbh + bh]);
                    }
                }
                /* clean forward over the whole sequence; incoming gradients on
                 * states[k] (given, and from noisy block k + 1) after token (k+1)T-1 */
                if (dstates)
                    for (int64_t k = 0; k < K; ++k)
                        for (int64_t e = 0; e < PN; ++e)
                            dsn[k * PN + e] += dstates[((b * K + k) * H + h) * PN + e];
                for (int64_t i = 0; i < L; ++i) {
                    order[i] = i;
                    dat[i] = ((i + 1) % T == 0) ? dsn + (i / T) * PN : NULL;
                }
                memset(G, 0, sizeof(double) * PN);
                pass_backward(s, cf, b, h, order, L, h0 ? h0 + (b * H + h) * PN : NULL, dy_clean, dat, G,
                              hist, &acc[0 * nbh + bh]);
                if (dh0_bh)
                    for (int64_t e = 0; e < PN; ++e) dh0_bh[e] += G[e];
            }
        }
        free(G); free(hist); free(order); free((void *)dat); free(dsn);
    }
    if (!failed) {
        /* fixed-order reductions */
        for (int di = 0; di < 4; ++di) {
            if (!dirs[di]) continue;
            oracle_grad_t *gr = grads[di];
            if (gr->dB) memset(gr->dB, 0, sizeof(double) * B * L * Gn * N);
            if (gr->dC) memset(gr->dC, 0, sizeof(double) * B * L * Gn * N);
            if (gr->dA) memset(gr->dA, 0, sizeof(double) * H);
            if (gr->dD) memset(gr->dD, 0, sizeof(double) * H);
            for (int64_t b = 0; b < B; ++b)
                for (int64_t h = 0; h < H; ++h) {
                    const bwd_acc_t *a = &acc[di * nbh + b * H + h];
                    const int64_t g = h / (H / Gn);
                    for (int64_t t = 0; t < L; ++t) {
                        if (gr->dx)
                            memcpy(gr->dx + ((b * L + t) * H + h) * P, a->dx + t * P, sizeof(double) * P);
                        if (gr->ddt) gr->ddt[(b * L + t) * H + h] = a->ddt[t];
                        for (int64_t q = 0; q < N; ++q) {
                            if (gr->dB) gr->dB[((b * L + t) * Gn + g) * N + q] += a->dB[t * N + q];
                            if (gr->dC) gr->dC[((b * L + t) * Gn + g) * N + q] += a->dC[t * N + q];
                        }
                    }
                    if (gr->dA) gr->dA[h] += a->dA;
                    if (gr->dD) gr->dD[h] += a->dD;
                }
        }
    }
    free(states); free(acc); free(pool);
    return failed ? ORACLE_ENOMEM : ORACLE_OK;
}

/* ---- Short convolution in front of the scan ---------------------------------
 *
 * In a Mamba-2 layer every x, B and C channel goes through a depthwise
 * convolution of `width` taps over time, then a SiLU, before the scan.  A Mamba
 * layer's cache holds this convolution's state (the last width-1 input rows)
 * beside the scan state ("Training Hybrid Block Diffusion Language Models with
 * Partial Bidirectionality", the paragraph after eq. (14)).  The reverse
 * direction's convolution is anti-causal ("Breaking the Bottleneck with
 * DiffuApriel", section 3.2, after eq. (5)) and, like the reverse scan, stays
 * inside its block (first page, eq. (12)).
 *
 * Rows are flat: u[b][t][c] with c < channels (the caller packs x | B | C).
 * The conv state is [b][width-1][channels], oldest row first.
 *   causal:       v[t] = act(bias + sum_{j < W} w[j] * u[t - (W-1) + j])
 *   anti-causal:  v[t] = act(bias + sum_{j < W} w[j] * u[t + (W-1) - j]),
 *                 u taken as 0 past the end of t's block
 * act is silu when asked for, else the identity. */
typedef struct {
    int64_t batch, seqlen, channels, width, block_len;
    int64_t silu;
} oracle_conv_shape_t;

typedef struct {
    const double *u;    /* [B][L][channels] pre-convolution rows */
    const double *w;    /* [channels][width] taps */
    const double *bias; /* [channels] or NULL (zeros) */
    double *v;          /* [B][L][channels] output */
} oracle_conv_dir_t;

/* Pre-convolution value of channel c at token tp of batch row b as a causal
 * convolution sees it: the direction's own rows from token own_from on, the
 * rows of `halo` (another stream, same layout) between token 0 and own_from,
 * the conv state before token 0, and zeros before the state (or without one). */
static double conv_input(const oracle_conv_shape_t *s, const double *own, int64_t own_from,
                         const double *halo, const double *state, int64_t b, int64_t tp, int64_t c) {
    const int64_t L = s->seqlen, Cx = s->channels, W = s->width;
    if (tp >= own_from) return own[(b * L + tp) * Cx + c];
    if (tp >= 0) return halo[(b * L + tp) * Cx + c];
    if (state && tp >= -(W - 1)) return state[(b * (W - 1) + (W - 1 + tp)) * Cx + c];
    return 0.0;
}

static double conv_act(const oracle_conv_shape_t *s, const oracle_conv_dir_t *d, int64_t c, double acc) {
    const double v = acc + (d->bias ? d->bias[c] : 0.0);
    return s->silu ? silu(v) : v;
}

/* Causal convolution of one direction.  halo == NULL: over the whole stream;
 * otherwise every block continues from `halo`'s rows before it. */
static void conv_causal(const oracle_conv_shape_t *s, const oracle_conv_dir_t *d, const double *halo,
                        const double *state) {
    const int64_t L = s->seqlen, Cx = s->channels, W = s->width, T = s->block_len;
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t b = 0; b < s->batch; ++b)
        for (int64_t t = 0; t < L; ++t) {
            const int64_t own_from = halo ? (t / T) * T : 0;
            for (int64_t c = 0; c < Cx; ++c) {
                double acc = 0.0;
                for (int64_t j = 0; j < W; ++j)
                    acc += d->w[c * W + j] * conv_input(s, d->u, own_from, halo, state, b, t - (W - 1) + j, c);
                d->v[(b * L + t) * Cx + c] = conv_act(s, d, c, acc);
            }
        }
}

/* Anti-causal convolution confined to each block, from zeros past its end. */
static void conv_anticausal(const oracle_conv_shape_t *s, const oracle_conv_dir_t *d) {
    const int64_t L = s->seqlen, Cx = s->channels, W = s->width, T = s->block_len;
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t b = 0; b < s->batch; ++b)
        for (int64_t t = 0; t < L; ++t) {
            const int64_t block_end = (t / T + 1) * T;
            for (int64_t c = 0; c < Cx; ++c) {
                double acc = 0.0;
                for (int64_t j = 0; j < W; ++j) {
                    const int64_t tp = t + (W - 1) - j;
                    acc += d->w[c * W + j] * (tp < block_end ? d->u[(b * L + tp) * Cx + c] : 0.0);
                }
                d->v[(b * L + t) * Cx + c] = conv_act(s, d, c, acc);
            }
        }
}

static int conv_check(const oracle_conv_shape_t *s, const oracle_conv_dir_t *d) {
    if (!s || s->batch < 0 || s->seqlen < 0 || s->channels < 1 || s->width < 1 || s->block_len < 1 ||
        s->seqlen % s->block_len)
        return ORACLE_EINVAL;
    if (d && (!d->u || !d->w || !d->v)) return ORACLE_EINVAL;
    return ORACLE_OK;
}

/* Convolution of one sequence (prefill, commit or a denoising step): the
 * forward direction causal from state_in (NULL: zeros), the reverse one
 * anti-causal inside each block; state_out (or NULL) receives the last W-1
 * rows of the forward stream, state_in's rows included when L < W-1. */
int oracle_conv_prefix(const oracle_conv_shape_t *s, const oracle_conv_dir_t *fwd,
                       const oracle_conv_dir_t *rev, const double *state_in, double *state_out) {
    if (conv_check(s, fwd) || !fwd || conv_check(s, rev)) return ORACLE_EINVAL;
    conv_causal(s, fwd, NULL, state_in);
    if (rev) conv_anticausal(s, rev);
    if (state_out) {
        const int64_t W = s->width, Cx = s->channels;
        for (int64_t b = 0; b < s->batch; ++b)
            for (int64_t r = 0; r < W - 1; ++r)
                for (int64_t c = 0; c < Cx; ++c)
                    state_out[(b * (W - 1) + r) * Cx + c] =
                        conv_input(s, fwd->u, 0, NULL, state_in, b, s->seqlen - (W - 1) + r, c);
    }
    return ORACLE_OK;
}

/* Convolution of the all-block pass: the clean stream as by oracle_conv_prefix;
 * noisy block k's forward convolution reads the clean rows before the block
 * (state_in before token 0), the noisy reverse stays inside the block. */
int oracle_conv_allblock(const oracle_conv_shape_t *s, const oracle_conv_dir_t *cf,
                         const oracle_conv_dir_t *cr, const oracle_conv_dir_t *nf,
                         const oracle_conv_dir_t *nr, const double *state_in) {
    if (conv_check(s, cf) || !cf || conv_check(s, cr) || conv_check(s, nf) || !nf || conv_check(s, nr))
        return ORACLE_EINVAL;
    conv_causal(s, cf, NULL, state_in);
    if (cr) conv_anticausal(s, cr);
    conv_causal(s, nf, cf->u, state_in);
    if (nr) conv_anticausal(s, nr);
    return ORACLE_OK;
}

/* ---- Gated RMSNorm after the directional sum ----------------------------------
 *
 * "Breaking the Bottleneck with DiffuApriel", section 3.2 (after eq. (6)): the
 * summed hidden sequence y = y_fwd + y_rev is normalised before the layer's
 * projection.  Read as the Mamba-2 layer's gated RMSNorm with the gate applied
 * before the norm: per token row, v_c = y_c * silu(z_c) (v = y without z); the
 * channels are cut into `groups` consecutive groups of gs = C / groups; per
 * group, r = 1 / sqrt(mean_{c in group} v_c^2 + eps); out_c = v_c * r * w_c.
 * Rows: y, z, out [rows][C] (C = H * P), w [C]. */
int oracle_gated_rmsnorm(int64_t rows, int64_t channels, int64_t groups, double eps, const double *y,
                         const double *z, const double *w, double *out) {
    if (rows < 0 || channels < 1 || groups < 1 || channels % groups || !w || !out || (rows && !y))
        return ORACLE_EINVAL;
    const int64_t gs = channels / groups;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t g = 0; g < groups; ++g) {
            double ss = 0.0;
            for (int64_t c = g * gs; c < (g + 1) * gs; ++c) {
                const double v = y[r * channels + c] * (z ? silu(z[r * channels + c]) : 1.0);
                ss += v * v;
            }
            const double rstd = 1.0 / sqrt(ss / (double)gs + eps);
            for (int64_t c = g * gs; c < (g + 1) * gs; ++c) {
                const double v = y[r * channels + c] * (z ? silu(z[r * channels + c]) : 1.0);
                out[r * channels + c] = v * rstd * w[c];
            }
        }
    }
    return ORACLE_OK;
}

int oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

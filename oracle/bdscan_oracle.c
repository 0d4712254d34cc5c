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

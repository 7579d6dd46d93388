/*
 * Plain fp64 CPU oracle of the SketchSSM "write-full, read-sketch" decode path.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the bench's CPU
 * baseline leg load this file's library; the CUDA path shares no code with it.
 *
 * Sources (SketchSSM: Write to the Full State, Read from a Compact Sketch):
 *   [ABS]  paper abstract (newx.sg page "Abstract"; mlsanity page "Abstract (arXiv)"):
 *          state updates are buffered (ReplaySSM); at every state update the full
 *          state is read once to precompute the outputs for fixed offline basis
 *          vectors (the sketch); each later decode step combines the sketch with
 *          query-dependent coefficients instead of reading the full state.
 *   [SUM]  newx.sg page "AI Summary": sketches precomputed at update time, outputs
 *          rebuilt from coefficients at decode time.
 *   [PYPI] sketchssm 0.1.0 PyPI page, calibration stages "basis" (one shared basis
 *          per head group) and "allocate" (a rank or a dense fallback per head).
 *   [CARD] Nemotron Nano 9B v2 calibration card, "Contents": K=128, V=80, W=16,
 *          8 basis groups, basis omega stored as (layers, groups, 79, 128) rows.
 *   Recurrences: Mamba-2 scalar decay ("Transformers are SSMs"), Gated DeltaNet
 *   ("Gated Delta Networks: Improving Mamba2 with Delta Rule"), both in the
 *   mlsanity index's "Builds on" list; KDA = per-key-channel decay with the delta
 *   rule, applied as diag(a)(I - beta k k^T).
 *
 * Conventions (all arrays C-contiguous, fp64; inputs are the fp32 draws upcast):
 *   S [B][H][K][V], omega [G][Rb][K] (row m = basis vector m of the group),
 *   Y [B][Rtot][V] (head h owns rows off[h] .. off[h]+rank[h]-1),
 *   q, k [B][Hqk][K], v [B][H][V], a [B][H] (KDA [B][H][K]), beta [B][H],
 *   kbuf [B][Hqk][W][K], vbuf [B][H][W][V], abuf [B][H][W] (KDA [B][H][W][K]),
 *   bbuf [B][H][W], y [B][H][V].
 *   Head h uses basis group h*G/H and q/k head h*Hqk/H (integer division).
 *   rank[h] = -1 marks a dense-fallback head.
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_DENSE (-1)
enum { ORACLE_MAMBA2 = 0, ORACLE_GDN = 1, ORACLE_KDA = 2 };

typedef struct {
    int32_t kind, B, H, Hqk, K, V, W, G, Rb;
} oracle_dims;

/* ------------------------------------------------------------------ layout
 * Packed sketch layout of one layer [PYPI stage "allocate"; ABS, the sketch]:
 * off[h] = sum of the ranks of the sketch heads before h (dense heads own no rows),
 * off[H] = Rtot; rmax[g] = largest sketch rank in group g (0 if none).
 * Returns Rtot, or -1 if a rank is neither DENSE nor >= 1. */
int64_t oracle_layout(int32_t H, int32_t G, const int32_t *rank, int32_t *off, int32_t *rmax)
{
    for (int32_t g = 0; g < G; ++g) rmax[g] = 0;
    int64_t acc = 0;
    for (int32_t h = 0; h < H; ++h) {
        off[h] = (int32_t)acc;
        if (rank[h] == ORACLE_DENSE) continue;
        if (rank[h] < 1) return -1;
        acc += rank[h];
        int32_t g = (int32_t)(((int64_t)h * G) / H);
        if (rank[h] > rmax[g]) rmax[g] = rank[h];
    }
    off[H] = (int32_t)acc;
    return acc;
}

static double a_scalar(const oracle_dims *d, const double *abuf, int64_t bh, int i)
{
    return abuf[bh * d->W + i];
}

/* ------------------------------------------------------------------ flush
 * Write-full step [ABS: every update reaches the full state]: for every (b, h) apply the n
 * buffered tokens in order, S <- M_i S + beta_i k_i v_i^T with
 *   Mamba-2: M_i = a_i I, beta_i = 1
 *   GDN:     M_i = a_i (I - beta_i k_i k_i^T)
 *   KDA:     M_i = diag(a_i) (I - beta_i k_i k_i^T)
 * then read the new state once to form the sketch of every sketch head
 * [ABS: the one read of the state, at the update, yields the basis outputs]:
 *   Y[off[h] + m][:] = sum_k omega[g][m][k] S[k][:]   for m < rank[h].
 * Dense heads keep no sketch. */
void oracle_flush(const oracle_dims *d, const int32_t *rank, const int32_t *off, int64_t rtot,
                  double *S, const double *omega, const double *kbuf, const double *vbuf,
                  const double *abuf, const double *bbuf, int32_t n, double *Y)
{
    const int64_t K = d->K, V = d->V, W = d->W;
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t b = 0; b < d->B; ++b) {
        for (int64_t h = 0; h < d->H; ++h) {
            const int64_t bh = b * d->H + h;
            const int64_t qh = (h * d->Hqk) / d->H;
            double *Sh = S + bh * K * V;
            double *dv = (double *)malloc(sizeof(double) * V);
            for (int i = 0; i < n; ++i) {
                const double *ki = kbuf + ((b * d->Hqk + qh) * W + i) * K;
                const double *vi = vbuf + (bh * W + i) * V;
                const double beta = (d->kind == ORACLE_MAMBA2) ? 1.0 : bbuf[bh * W + i];
                if (d->kind == ORACLE_MAMBA2) {
                    const double a = a_scalar(d, abuf, bh, i);
                    for (int64_t kk = 0; kk < K; ++kk)
                        for (int64_t j = 0; j < V; ++j)
                            Sh[kk * V + j] = a * Sh[kk * V + j] + ki[kk] * vi[j];
                } else {
                    /* d = S^T k_i (the erase term needs k_i^T S before the update) */
                    for (int64_t j = 0; j < V; ++j) {
                        double s = 0.0;
                        for (int64_t kk = 0; kk < K; ++kk) s += ki[kk] * Sh[kk * V + j];
                        dv[j] = s;
                    }
                    for (int64_t kk = 0; kk < K; ++kk) {
                        const double a = (d->kind == ORACLE_KDA) ? abuf[(bh * W + i) * K + kk]
                                                                 : a_scalar(d, abuf, bh, i);
                        for (int64_t j = 0; j < V; ++j)
                            Sh[kk * V + j] = a * (Sh[kk * V + j] - beta * ki[kk] * dv[j])
                                             + beta * ki[kk] * vi[j];
                    }
                }
            }
            free(dv);
            if (rank[h] == ORACLE_DENSE) continue;
            const int64_t g = (h * d->G) / d->H;
            for (int64_t m = 0; m < rank[h]; ++m) {
                const double *om = omega + (g * d->Rb + m) * K;
                double *Yr = Y + (b * rtot + off[h] + m) * V;
                for (int64_t j = 0; j < V; ++j) {
                    double s = 0.0;
                    for (int64_t kk = 0; kk < K; ++kk) s += om[kk] * Sh[kk * V + j];
                    Yr[j] = s;
                }
            }
        }
    }
}

/* ------------------------------------------------------------------ decode
 * One decode step at buffer slot pos (pos tokens already buffered since the last
 * flush).  The step's token is appended at slot pos, then with n = pos + 1:
 *
 * Buffer replay [ABS "ReplaySSM amortizes state updates by buffering keys and
 * values"]: the output must equal S_t^T q with S_t = M_n ... M_1 S_f + (buffered
 * terms).  Walking the tokens newest first with x = q:
 *   y_rep += beta_i (k_i . x) v_i;   x <- M_i^T x
 * where M_i^T x = a_i x (Mamba-2), a_i (x - beta_i k_i (k_i . x)) (GDN),
 * a_i o x - beta_i k_i (k_i . (a_i o x)) (KDA).  After the walk x = q0 is the query
 * seen by the flushed state S_f.
 *
 * State read: dense head (or dense_all) -> S_f^T q0 exactly [PYPI "dense fallback"];
 * sketch head [ABS: sketch rows mixed with coefficients that depend on the query]:
 *   c_m = omega[g][m] . q0 (m < rank),  y_state = sum_m c_m Y[off + m][:].
 * y = y_state + y_rep. */
void oracle_decode(const oracle_dims *d, const int32_t *rank, const int32_t *off, int64_t rtot,
                   int32_t pos, const double *q, const double *k, const double *v,
                   const double *a, const double *beta, double *kbuf, double *vbuf,
                   double *abuf, double *bbuf, const double *Y, const double *omega,
                   const double *S, int32_t dense_all, double *y)
{
    const int64_t K = d->K, V = d->V, W = d->W;
    const int64_t da = (d->kind == ORACLE_KDA) ? K : 1;
    /* append the step's token at slot pos */
    for (int64_t b = 0; b < d->B; ++b) {
        for (int64_t qh = 0; qh < d->Hqk; ++qh)
            memcpy(kbuf + ((b * d->Hqk + qh) * W + pos) * K, k + (b * d->Hqk + qh) * K,
                   sizeof(double) * K);
        for (int64_t h = 0; h < d->H; ++h) {
            const int64_t bh = b * d->H + h;
            memcpy(vbuf + (bh * W + pos) * V, v + bh * V, sizeof(double) * V);
            memcpy(abuf + (bh * W + pos) * da, a + bh * da, sizeof(double) * da);
            if (d->kind != ORACLE_MAMBA2) bbuf[bh * W + pos] = beta[bh];
        }
    }
    const int32_t n = pos + 1;
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t b = 0; b < d->B; ++b) {
        for (int64_t h = 0; h < d->H; ++h) {
            const int64_t bh = b * d->H + h;
            const int64_t qh = (h * d->Hqk) / d->H;
            double *x = (double *)malloc(sizeof(double) * K);
            double *xa = (double *)malloc(sizeof(double) * K);
            double *yo = y + bh * V;
            memcpy(x, q + (b * d->Hqk + qh) * K, sizeof(double) * K);
            for (int64_t j = 0; j < V; ++j) yo[j] = 0.0;
            for (int i = n - 1; i >= 0; --i) {
                const double *ki = kbuf + ((b * d->Hqk + qh) * W + i) * K;
                const double *vi = vbuf + (bh * W + i) * V;
                const double bi = (d->kind == ORACLE_MAMBA2) ? 1.0 : bbuf[bh * W + i];
                double s = 0.0;
                for (int64_t kk = 0; kk < K; ++kk) s += ki[kk] * x[kk];
                for (int64_t j = 0; j < V; ++j) yo[j] += bi * s * vi[j];
                if (d->kind == ORACLE_MAMBA2) {
                    const double ai = abuf[bh * W + i];
                    for (int64_t kk = 0; kk < K; ++kk) x[kk] = ai * x[kk];
                } else if (d->kind == ORACLE_GDN) {
                    const double ai = abuf[bh * W + i];
                    for (int64_t kk = 0; kk < K; ++kk) x[kk] = ai * (x[kk] - bi * ki[kk] * s);
                } else {
                    const double *ai = abuf + (bh * W + i) * K;
                    double s2 = 0.0;
                    for (int64_t kk = 0; kk < K; ++kk) {
                        xa[kk] = ai[kk] * x[kk];
                        s2 += ki[kk] * xa[kk];
                    }
                    for (int64_t kk = 0; kk < K; ++kk) x[kk] = xa[kk] - bi * ki[kk] * s2;
                }
            }
            if (dense_all || rank[h] == ORACLE_DENSE) {
                const double *Sh = S + bh * K * V;
                for (int64_t j = 0; j < V; ++j) {
                    double s = 0.0;
                    for (int64_t kk = 0; kk < K; ++kk) s += Sh[kk * V + j] * x[kk];
                    yo[j] += s;
                }
            } else {
                const int64_t g = (h * d->G) / d->H;
                for (int64_t m = 0; m < rank[h]; ++m) {
                    const double *om = omega + (g * d->Rb + m) * K;
                    double c = 0.0;
                    for (int64_t kk = 0; kk < K; ++kk) c += om[kk] * x[kk];
                    const double *Yr = Y + (b * rtot + off[h] + m) * V;
                    for (int64_t j = 0; j < V; ++j) yo[j] += c * Yr[j];
                }
            }
            free(x);
            free(xa);
        }
    }
}

/* ------------------------------------------------------------------ standard step
 * The per-step recurrent decode the paper measures its speedup against [ABS: standard
 * decoding reads and updates the full state for every token]: for every (b, h), apply
 * the step's token to the state, S <- M S + beta k v^T (the transition table above;
 * Mamba-2 beta = 1), then read it, y = S^T q (read after the update, as in the
 * decode).  No buffer, no sketch.  Inputs of one step: q, k [B][Hqk][K],
 * v [B][H][V], a [B][H] (KDA [B][H][K]), beta [B][H] (unused for Mamba-2). */
void oracle_step(const oracle_dims *d, double *S, const double *q, const double *k, const double *v,
                 const double *a, const double *beta, double *y)
{
    const int64_t K = d->K, V = d->V;
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t b = 0; b < d->B; ++b) {
        for (int64_t h = 0; h < d->H; ++h) {
            const int64_t bh = b * d->H + h;
            const int64_t qh = (h * d->Hqk) / d->H;
            double *Sh = S + bh * K * V;
            const double *kt = k + (b * d->Hqk + qh) * K;
            const double *qt = q + (b * d->Hqk + qh) * K;
            const double *vt = v + bh * V;
            if (d->kind == ORACLE_MAMBA2) {
                const double at = a[bh];
                for (int64_t kk = 0; kk < K; ++kk)
                    for (int64_t j = 0; j < V; ++j) Sh[kk * V + j] = at * Sh[kk * V + j] + kt[kk] * vt[j];
            } else {
                const double bt = beta[bh];
                for (int64_t j = 0; j < V; ++j) {
                    double e = 0.0; /* (k^T S)_j, taken before the update */
                    for (int64_t kk = 0; kk < K; ++kk) e += kt[kk] * Sh[kk * V + j];
                    for (int64_t kk = 0; kk < K; ++kk) {
                        const double at = (d->kind == ORACLE_KDA) ? a[bh * K + kk] : a[bh];
                        Sh[kk * V + j] = at * (Sh[kk * V + j] - bt * kt[kk] * e) + bt * kt[kk] * vt[j];
                    }
                }
            }
            double *yo = y + bh * V;
            for (int64_t j = 0; j < V; ++j) {
                double s = 0.0;
                for (int64_t kk = 0; kk < K; ++kk) s += Sh[kk * V + j] * qt[kk];
                yo[j] = s;
            }
        }
    }
}

/* ------------------------------------------------------------------ prefill
 * Prefill handoff, the step before decoding.  The pages say only that every update
 * reaches the full state [ABS, write-full]; how a prompt is taken in is left to the
 * model's own kernels, so the plain reading is used: the prompt's T tokens are applied
 * to the state one after another, t = 0 .. T-1, with the transition table above,
 * S <- M_t S + beta_t k_t v_t^T.  The caller then forms the sketch with
 * oracle_flush(n = 0); the window buffer is not touched and decoding starts at
 * pos = 0.  Prompt layout (token-major): pk [B][T][Hqk][K], pv [B][T][H][V],
 * pa [B][T][H] (KDA [B][T][H][K]), pb [B][T][H] (unused for Mamba-2). */
void oracle_prefill(const oracle_dims *d, int32_t T, double *S, const double *pk, const double *pv,
                    const double *pa, const double *pb)
{
    const int64_t K = d->K, V = d->V, H = d->H;
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t b = 0; b < d->B; ++b) {
        for (int64_t h = 0; h < H; ++h) {
            const int64_t qh = (h * d->Hqk) / H;
            double *St = S + (b * H + h) * K * V;
            double *ev = (double *)malloc(sizeof(double) * V);
            for (int64_t t = 0; t < T; ++t) {
                const int64_t bth = (b * T + t) * H + h; /* token t of row b, head h */
                const double *kp = pk + ((b * T + t) * d->Hqk + qh) * K;
                const double *vp = pv + bth * V;
                if (d->kind == ORACLE_MAMBA2) {
                    const double ap = pa[bth];
                    for (int64_t r = 0; r < K; ++r)
                        for (int64_t c = 0; c < V; ++c) St[r * V + c] = ap * St[r * V + c] + kp[r] * vp[c];
                    continue;
                }
                const double bp = pb[bth];
                for (int64_t c = 0; c < V; ++c) { /* (k_t^T S)_c before the update */
                    double acc = 0.0;
                    for (int64_t r = 0; r < K; ++r) acc += kp[r] * St[r * V + c];
                    ev[c] = acc;
                }
                for (int64_t r = 0; r < K; ++r) {
                    const double ap = (d->kind == ORACLE_KDA) ? pa[bth * K + r] : pa[bth];
                    for (int64_t c = 0; c < V; ++c)
                        St[r * V + c] = ap * (St[r * V + c] - bp * kp[r] * ev[c]) + bp * kp[r] * vp[c];
                }
            }
            free(ev);
        }
    }
}

/* Host threads the loops above use from now on (a single-thread baseline sets 1). */
void oracle_set_num_threads(int n)
{
#ifdef _OPENMP
    extern void omp_set_num_threads(int);
    omp_set_num_threads(n < 1 ? 1 : n);
#else
    (void)n;
#endif
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

/*
 * oracle.c -- plain float64 CPU oracle of the ZGCM-1 attention core.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
 * baseline leg of the benchmark may load this library.  The product path
 * (the CUDA library) shares no code, header, table or helper with it.
 *
 * What it computes, with the passage each step follows:
 *
 *   ZGCM-1, §2.1 Model overview (papers.lianghsun.dev translation of the
 *   paper; the same facts restated on the e-cogni.com.br summary, "Como
 *   funciona"): decoder with GQA, 32 query / 8 key-value heads of dim 128;
 *   27 of 32 layers use gated sliding-window attention over a 128-token
 *   window, 5 layers (6, 12, 18, 24, 30) use global causal attention; QK
 *   normalisation is an RMSNorm; partial RoPE with rotary fraction 0.33.
 *
 *   ZGCM-1, §2.1 Figure 3 caption: the q/k branches receive RMS
 *   normalisation and partial RoPE; with A_SWA the 128-token sliding-window
 *   GQA output, GatedSWA(h) = o_proj(A_SWA(q,k,v) ⊙ σ(g_proj(h))); the
 *   sigmoid gate acts elementwise before the output projection; global
 *   layers drop the gate and attend over the whole context.
 *
 *   ZGCM-1, §2.3 KV-cache analysis: SWA layers keep a fixed 128-token
 *   window in the cache, global layers keep the whole sequence; per-token KV
 *   of 128 KiB (all global) vs 20 KiB (hybrid).
 *
 *   ZGCM-1, §3.2 Mid-training: RoPE base 10M for the 256K stage.
 *
 * Readings where the pages are silent (each one is a choice, stated here):
 *   - window: key j is visible to query i iff i-W < j <= i (W keys, self
 *     included); the look-ahead direction of the paperglide.net toy example
 *     ("ZGCM-1 Architecture" walkthrough) contradicts "causal" on the other
 *     pages and is rejected;
 *   - RMSNorm per (token, head) over the head dim, eps inside the root, one
 *     weight vector of length D for q and one for k, applied before RoPE;
 *   - RoPE rotates the first R dims (R = 42 for D = 128) as R/2 pairs
 *     (p, p + R/2), angle pos * base^(-2p/R), pos = 0-based token index;
 *   - softmax scale 1/sqrt(D) (passed in); query head h reads KV head
 *     h / (Hq/Hkv);
 *   - the gate is elementwise per (token, head, dim); global layers are
 *     ungated but use the same norm and RoPE;
 *   - caches hold the normed+rotated key and the raw value.
 *
 * Everything is computed in float64 from bf16 inputs widened exactly (or from
 * float64 inputs, for the finite-difference checks).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_EINVAL (-1)
#define ORACLE_ENOMEM (-2)

/* bf16 -> float64, exact: a bf16 is the top half of an IEEE float32. */
static double bf(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static double sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }

/*
 * An input tensor: either bf16 bit patterns (the normal case) or float64
 * (used by the finite-difference checks, which need perturbations far below
 * bf16 resolution).  Every read widens to float64.
 */
typedef struct {
    const void *p;
    int f64;
} in_t;

static double ld(in_t a, int64_t i)
{
    return a.f64 ? ((const double *)a.p)[i] : bf(((const uint16_t *)a.p)[i]);
}

static in_t mk(const void *p, int f64)
{
    in_t a = {p, f64};
    return a;
}

/* Rotary angle of pair p at position pos: pos * base^(-2p/R). */
static double rope_angle(int64_t pos, int p, int R, double base)
{
    return (double)pos * pow(base, -2.0 * (double)p / (double)R);
}

/*
 * QK-RMSNorm followed by partial RoPE of one head vector (§2.1 Figure 3:
 * RMS normalisation and partial RoPE act on the query/key branches).
 *   r   = (mean_d x_d^2 + eps)^(-1/2)
 *   n_d = x_d * r
 *   u_d = w_d * n_d                      (normed, not yet rotated)
 *   out = u with the first R dims rotated pairwise by the position angle.
 * x is read at element offset off of the input; n and r are returned for
 * the backward pass when the pointers are non-null.
 */
static void prep_row(in_t x, int64_t off, const double *w, int D, int R, double base,
                     double eps, int64_t pos, double *out, double *n_out, double *r_out)
{
    double ss = 0.0;
    for (int d = 0; d < D; ++d) {
        double xv = ld(x, off + d);
        ss += xv * xv;
    }
    double r = 1.0 / sqrt(ss / (double)D + eps);
    for (int d = 0; d < D; ++d) {
        double n = ld(x, off + d) * r;
        if (n_out) n_out[d] = n;
        out[d] = w[d] * n;
    }
    if (r_out) *r_out = r;
    int half = R / 2;
    for (int p = 0; p < half; ++p) {
        double phi = rope_angle(pos, p, R, base);
        double c = cos(phi), s = sin(phi);
        double a = out[p], b = out[p + half];
        out[p] = a * c - b * s;
        out[p + half] = b * c + a * s;
    }
}

/* Transpose of the rotation above: maps d(out) to d(u). */
static void rope_transpose(double *du, int R, double base, int64_t pos)
{
    int half = R / 2;
    for (int p = 0; p < half; ++p) {
        double phi = rope_angle(pos, p, R, base);
        double c = cos(phi), s = sin(phi);
        double a = du[p], b = du[p + half];
        du[p] = a * c + b * s;
        du[p + half] = b * c - a * s;
    }
}

/*
 * Backward of u = w ⊙ (x r):  given du, n, r, w:
 *   dn = w ⊙ du
 *   dx = r (dn - n * mean_d(dn ⊙ n))
 *   dw += du ⊙ n
 */
static void rmsnorm_backward(const double *du, const double *n, double r, const double *w,
                             int D, double *dx, double *dw_acc)
{
    double m = 0.0;
    for (int d = 0; d < D; ++d) m += w[d] * du[d] * n[d];
    m /= (double)D;
    for (int d = 0; d < D; ++d) {
        dx[d] = r * (w[d] * du[d] - n[d] * m);
        dw_acc[d] += du[d] * n[d];
    }
}

/* Visible key range of query i is [first_visible(i), i]; window <= 0 means
 * full causal (§2.1: global layers attend over the whole context). */
static int64_t first_visible(int64_t i, int window)
{
    if (window <= 0) return 0;
    int64_t lo = i - window + 1;
    return lo < 0 ? 0 : lo;
}

static int check_shape(int B, int64_t T, int Hq, int Hkv, int D, int R)
{
    if (B < 0 || T < 0 || Hq <= 0 || Hkv <= 0 || D <= 0) return ORACLE_EINVAL;
    if (Hq % Hkv != 0) return ORACLE_EINVAL;
    if (R < 0 || R > D || (R & 1)) return ORACLE_EINVAL;
    return ORACLE_OK;
}

static double *widen(in_t w, int D)
{
    double *out = malloc(sizeof(double) * D);
    if (out)
        for (int d = 0; d < D; ++d) out[d] = ld(w, d);
    return out;
}

/*
 * Prepared (normed + rotated) heads: x [B, T, H, D] -> out [B, T, H, D] f64,
 * position of token t = pos0 + t.
 */
int oracle_qk_prep(int in_f64, int B, int64_t T, int H, int D, int R, double base, double eps,
                   int64_t pos0, const void *x, const void *w_in, double *out)
{
    if (check_shape(B, T, H, H, D, R)) return ORACLE_EINVAL;
    double *w = widen(mk(w_in, in_f64), D);
    if (!w) return ORACLE_ENOMEM;
    int64_t rows = (int64_t)B * T * H;
#pragma omp parallel for schedule(static)
    for (int64_t row = 0; row < rows; ++row) {
        int64_t t = (row / H) % T;
        prep_row(mk(x, in_f64), row * D, w, D, R, base, eps, pos0 + t, out + row * D, NULL,
                 NULL);
    }
    free(w);
    return ORACLE_OK;
}

/*
 * Forward of the attention core at a set of query positions.
 *
 *   s_ij = scale <q~_i, k~_j>  for i-W < j <= i  (full causal: j <= i)
 *   p_ij = exp(s_ij - lse_i),  lse_i = log sum_j exp(s_ij)
 *   A_i  = sum_j p_ij v_j
 *   y_i  = A_i ⊙ σ(g_i)   (gated SWA layers)   or   A_i   (global layers)
 *
 * q, g: [B, T, Hq, D]; k, v: [B, T, Hkv, D]; w_q, w_k: [D]; element type
 * bf16 (in_f64 = 0) or float64 (in_f64 = 1).
 * rows: nrows query positions (NULL: all T, nrows must equal T).
 * y: [B, nrows, Hq, D] f64; lse: [B, Hq, nrows] f64 (nullable).
 */
int oracle_attn_fwd(int in_f64, int B, int64_t T, int Hq, int Hkv, int D, int window,
                    int gated, int R, double base, double eps, double scale, const void *q_in,
                    const void *k_in, const void *v_in, const void *g_in, const void *wq_in,
                    const void *wk_in, int64_t nrows, const int64_t *rows, double *y,
                    double *lse)
{
    if (check_shape(B, T, Hq, Hkv, D, R)) return ORACLE_EINVAL;
    if (!rows && nrows != T) return ORACLE_EINVAL;
    if (gated && !g_in) return ORACLE_EINVAL;
    for (int64_t r = 0; rows && r < nrows; ++r)
        if (rows[r] < 0 || rows[r] >= T) return ORACLE_EINVAL;
    const in_t q = mk(q_in, in_f64), k = mk(k_in, in_f64), v = mk(v_in, in_f64),
               g = mk(g_in, in_f64);
    const int G = Hq / Hkv;
    double *wq = widen(mk(wq_in, in_f64), D), *wk = widen(mk(wk_in, in_f64), D);
    double *kp = malloc(sizeof(double) * (size_t)(T > 0 ? T : 1) * D);
    if (!wq || !wk || !kp) { free(wq); free(wk); free(kp); return ORACLE_ENOMEM; }
    int status = ORACLE_OK;

    for (int b = 0; b < B; ++b) {
        for (int kh = 0; kh < Hkv; ++kh) {
            /* Prepared keys of this (sequence, kv head). */
#pragma omp parallel for schedule(static)
            for (int64_t j = 0; j < T; ++j)
                prep_row(k, (((int64_t)b * T + j) * Hkv + kh) * D, wk, D, R, base, eps, j,
                         kp + j * D, NULL, NULL);

#pragma omp parallel for collapse(2) schedule(dynamic, 4)
            for (int hh = 0; hh < G; ++hh) {
                for (int64_t ri = 0; ri < nrows; ++ri) {
                    int h = kh * G + hh; /* query head h reads kv head h / G */
                    int64_t i = rows ? rows[ri] : ri;
                    int64_t lo = first_visible(i, window);
                    int64_t n = i - lo + 1;
                    double *qt = malloc(sizeof(double) * D);
                    double *s = malloc(sizeof(double) * n);
                    double *acc = calloc(D, sizeof(double));
                    if (!qt || !s || !acc) {
                        free(qt); free(s); free(acc);
#pragma omp atomic write
                        status = ORACLE_ENOMEM;
                        continue;
                    }
                    int64_t qrow = ((int64_t)b * T + i) * Hq + h;
                    prep_row(q, qrow * D, wq, D, R, base, eps, i, qt, NULL, NULL);
                    double mx = -INFINITY;
                    for (int64_t j = lo; j <= i; ++j) {
                        double dot = 0.0;
                        for (int d = 0; d < D; ++d) dot += qt[d] * kp[j * D + d];
                        s[j - lo] = scale * dot;
                        if (s[j - lo] > mx) mx = s[j - lo];
                    }
                    double l = 0.0;
                    for (int64_t j = 0; j < n; ++j) {
                        s[j] = exp(s[j] - mx);
                        l += s[j];
                    }
                    for (int64_t j = lo; j <= i; ++j) {
                        double p = s[j - lo] / l;
                        int64_t vrow = ((int64_t)b * T + j) * Hkv + kh;
                        for (int d = 0; d < D; ++d) acc[d] += p * ld(v, vrow * D + d);
                    }
                    double *yo = y + (((int64_t)b * nrows + ri) * Hq + h) * D;
                    for (int d = 0; d < D; ++d)
                        yo[d] = gated ? acc[d] * sigmoid(ld(g, qrow * D + d)) : acc[d];
                    if (lse) lse[((int64_t)b * Hq + h) * nrows + ri] = mx + log(l);
                    free(qt); free(s); free(acc);
                }
            }
        }
    }
    free(wq); free(wk); free(kp);
    return status;
}

/*
 * Backward of the attention core (chain rule through every step above).
 * Given dy [B, T, Hq, D], returns
 *   dq [B,T,Hq,D], dk, dv [B,T,Hkv,D], dg [B,T,Hq,D] (gated only, nullable),
 *   dwq, dwk [D]; all f64, overwritten.
 * Per query row i of head h (kv head c = h / G):
 *   σ = σ(g_i);  dA = dy ⊙ σ;  dg = dy ⊙ A ⊙ σ (1 - σ)     (ungated: dA = dy)
 *   dp_ij = <dA, v_j>;  dv_j += p_ij dA
 *   ds_ij = p_ij (dp_ij - sum_j' p_ij' dp_ij')
 *   dq~_i += scale sum_j ds_ij k~_j;  dk~_j += scale ds_ij q~_i
 * then each dq~, dk~ goes back through the rotation and the RMSNorm.
 */
int oracle_attn_bwd(int in_f64, int B, int64_t T, int Hq, int Hkv, int D, int window,
                    int gated, int R, double base, double eps, double scale, const void *q_in,
                    const void *k_in, const void *v_in, const void *g_in, const void *wq_in,
                    const void *wk_in, const void *dy_in, double *dq, double *dk, double *dv,
                    double *dg, double *dwq, double *dwk)
{
    if (check_shape(B, T, Hq, Hkv, D, R)) return ORACLE_EINVAL;
    if (gated && (!g_in || !dg)) return ORACLE_EINVAL;
    const in_t q = mk(q_in, in_f64), k = mk(k_in, in_f64), v = mk(v_in, in_f64),
               g = mk(g_in, in_f64), dy = mk(dy_in, in_f64);
    const int G = Hq / Hkv;
    double *wq = widen(mk(wq_in, in_f64), D), *wk = widen(mk(wk_in, in_f64), D);
    if (!wq || !wk) { free(wq); free(wk); return ORACLE_ENOMEM; }
    memset(dwq, 0, sizeof(double) * D);
    memset(dwk, 0, sizeof(double) * D);
    int status = ORACLE_OK;
    const size_t TD = (size_t)(T > 0 ? T : 1) * D;
    const size_t T1 = (size_t)(T > 0 ? T : 1);

#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int b = 0; b < B; ++b) {
        for (int kh = 0; kh < Hkv; ++kh) {
            /* Per-group buffers: prepared keys, their norm state, key grads. */
            double *kt = malloc(sizeof(double) * TD), *kn = malloc(sizeof(double) * TD);
            double *kr = malloc(sizeof(double) * T1);
            double *dkt = calloc(TD, sizeof(double)), *dvv = calloc(TD, sizeof(double));
            double *qt = malloc(sizeof(double) * D), *qn = malloc(sizeof(double) * D);
            double *dqt = malloc(sizeof(double) * D), *acc = malloc(sizeof(double) * D);
            double *dA = malloc(sizeof(double) * D), *tmp = malloc(sizeof(double) * D);
            double *pw = malloc(sizeof(double) * T1), *dp = malloc(sizeof(double) * T1);
            double *dwq_l = calloc(D, sizeof(double)), *dwk_l = calloc(D, sizeof(double));
            if (!kt || !kn || !kr || !dkt || !dvv || !qt || !qn || !dqt || !acc || !dA || !tmp ||
                !pw || !dp || !dwq_l || !dwk_l) {
#pragma omp atomic write
                status = ORACLE_ENOMEM;
                goto cleanup;
            }
            for (int64_t j = 0; j < T; ++j)
                prep_row(k, (((int64_t)b * T + j) * Hkv + kh) * D, wk, D, R, base, eps, j,
                         kt + j * D, kn + j * D, kr + j);

            for (int hh = 0; hh < G; ++hh) {
                int h = kh * G + hh;
                for (int64_t i = 0; i < T; ++i) {
                    int64_t row = ((int64_t)b * T + i) * Hq + h;
                    double qr;
                    prep_row(q, row * D, wq, D, R, base, eps, i, qt, qn, &qr);
                    int64_t lo = first_visible(i, window);
                    /* forward of this row */
                    double mx = -INFINITY;
                    for (int64_t j = lo; j <= i; ++j) {
                        double dot = 0.0;
                        for (int d = 0; d < D; ++d) dot += qt[d] * kt[j * D + d];
                        pw[j - lo] = scale * dot;
                        if (pw[j - lo] > mx) mx = pw[j - lo];
                    }
                    double l = 0.0;
                    for (int64_t j = lo; j <= i; ++j) {
                        pw[j - lo] = exp(pw[j - lo] - mx);
                        l += pw[j - lo];
                    }
                    for (int d = 0; d < D; ++d) acc[d] = 0.0;
                    for (int64_t j = lo; j <= i; ++j) {
                        pw[j - lo] /= l;
                        int64_t vrow = ((int64_t)b * T + j) * Hkv + kh;
                        for (int d = 0; d < D; ++d) acc[d] += pw[j - lo] * ld(v, vrow * D + d);
                    }
                    /* gate */
                    for (int d = 0; d < D; ++d) {
                        double dyd = ld(dy, row * D + d);
                        if (gated) {
                            double sg = sigmoid(ld(g, row * D + d));
                            dA[d] = dyd * sg;
                            dg[row * D + d] = dyd * acc[d] * sg * (1.0 - sg);
                        } else {
                            dA[d] = dyd;
                        }
                    }
                    /* softmax and the two products */
                    double Drow = 0.0;
                    for (int64_t j = lo; j <= i; ++j) {
                        int64_t vrow = ((int64_t)b * T + j) * Hkv + kh;
                        double s = 0.0;
                        for (int d = 0; d < D; ++d) s += dA[d] * ld(v, vrow * D + d);
                        dp[j - lo] = s;
                        Drow += pw[j - lo] * s;
                    }
                    for (int d = 0; d < D; ++d) dqt[d] = 0.0;
                    for (int64_t j = lo; j <= i; ++j) {
                        double p = pw[j - lo];
                        double ds = p * (dp[j - lo] - Drow);
                        for (int d = 0; d < D; ++d) {
                            dvv[j * D + d] += p * dA[d];
                            dqt[d] += scale * ds * kt[j * D + d];
                            dkt[j * D + d] += scale * ds * qt[d];
                        }
                    }
                    /* back through rotation and norm of q */
                    rope_transpose(dqt, R, base, i);
                    rmsnorm_backward(dqt, qn, qr, wq, D, dq + row * D, dwq_l);
                }
            }
            for (int64_t j = 0; j < T; ++j) {
                int64_t row = ((int64_t)b * T + j) * Hkv + kh;
                for (int d = 0; d < D; ++d) {
                    tmp[d] = dkt[j * D + d];
                    dv[row * D + d] = dvv[j * D + d];
                }
                rope_transpose(tmp, R, base, j);
                rmsnorm_backward(tmp, kn + j * D, kr[j], wk, D, dk + row * D, dwk_l);
            }
#pragma omp critical
            {
                for (int d = 0; d < D; ++d) {
                    dwq[d] += dwq_l[d];
                    dwk[d] += dwk_l[d];
                }
            }
        cleanup:
            free(kt); free(kn); free(kr); free(dkt); free(dvv); free(qt); free(qn);
            free(dqt); free(acc); free(dA); free(tmp); free(pw); free(dp);
            free(dwq_l); free(dwk_l);
        }
    }
    free(wq); free(wk);
    return status;
}

/*
 * One decode step (§2.3: SWA layers keep a fixed window of W tokens in the
 * cache, global layers keep every token).
 *
 * For each sequence b with position pos[b]:
 *   q~ = prep(q_new) at pos, k~_new = prep(k_new) at pos; the new token is
 *   part of its own window (it is written to the cache before attending);
 *   ring cache (window > 0): [B, Hkv, W, D], token position t lives in slot
 *   t mod W; the query sees positions max(0, pos-W+1) .. pos;
 *   linear cache (window <= 0): [B, Hkv, Tmax, D], position t in row t; the
 *   query sees positions 0 .. pos.
 *   y = softmax(scale q~ K~^T) V, times σ(g_new) when gated.
 * Cache entries other than the new token are read as stored (prepared K,
 * raw V).  k_new_prepared [B, Hkv, D] returns the key written for pos.
 */
int oracle_decode(int in_f64, int B, int Hq, int Hkv, int D, int window, int gated, int R,
                  double base, double eps, double scale, int64_t Tmax, const int64_t *pos,
                  const void *q_in, const void *k_in, const void *v_in, const void *g_in,
                  const void *wq_in, const void *wk_in, const void *kc_in, const void *vc_in,
                  double *y, double *k_new_prepared)
{
    if (check_shape(B, 1, Hq, Hkv, D, R)) return ORACLE_EINVAL;
    if (gated && !g_in) return ORACLE_EINVAL;
    const int64_t slots = window > 0 ? window : Tmax;
    for (int b = 0; b < B; ++b)
        if (pos[b] < 0 || (window <= 0 && pos[b] >= Tmax)) return ORACLE_EINVAL;
    const in_t q = mk(q_in, in_f64), k = mk(k_in, in_f64), v = mk(v_in, in_f64),
               g = mk(g_in, in_f64), kc = mk(kc_in, in_f64), vc = mk(vc_in, in_f64);
    const int G = Hq / Hkv;
    double *wq = widen(mk(wq_in, in_f64), D), *wk = widen(mk(wk_in, in_f64), D);
    if (!wq || !wk) { free(wq); free(wk); return ORACLE_ENOMEM; }
    int status = ORACLE_OK;

#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int b = 0; b < B; ++b) {
        for (int h = 0; h < Hq; ++h) {
            int kh = h / G;
            int64_t p = pos[b];
            int64_t lo = first_visible(p, window);
            int64_t n = p - lo + 1;
            double *qt = malloc(sizeof(double) * D), *kt = malloc(sizeof(double) * D);
            double *s = malloc(sizeof(double) * n), *acc = calloc(D, sizeof(double));
            if (!qt || !kt || !s || !acc) {
                free(qt); free(kt); free(s); free(acc);
#pragma omp atomic write
                status = ORACLE_ENOMEM;
                continue;
            }
            prep_row(q, ((int64_t)b * Hq + h) * D, wq, D, R, base, eps, p, qt, NULL, NULL);
            prep_row(k, ((int64_t)b * Hkv + kh) * D, wk, D, R, base, eps, p, kt, NULL, NULL);
            if (k_new_prepared && h % G == 0)
                for (int d = 0; d < D; ++d) k_new_prepared[((int64_t)b * Hkv + kh) * D + d] = kt[d];
            const int64_t cbase = ((int64_t)b * Hkv + kh) * slots * D;
            double mx = -INFINITY;
            for (int64_t t = lo; t <= p; ++t) {
                double dot = 0.0;
                if (t == p) {
                    for (int d = 0; d < D; ++d) dot += qt[d] * kt[d];
                } else {
                    int64_t slot = window > 0 ? t % window : t;
                    for (int d = 0; d < D; ++d) dot += qt[d] * ld(kc, cbase + slot * D + d);
                }
                s[t - lo] = scale * dot;
                if (s[t - lo] > mx) mx = s[t - lo];
            }
            double l = 0.0;
            for (int64_t t = 0; t < n; ++t) {
                s[t] = exp(s[t] - mx);
                l += s[t];
            }
            for (int64_t t = lo; t <= p; ++t) {
                double pr = s[t - lo] / l;
                if (t == p) {
                    int64_t vb = ((int64_t)b * Hkv + kh) * D;
                    for (int d = 0; d < D; ++d) acc[d] += pr * ld(v, vb + d);
                } else {
                    int64_t slot = window > 0 ? t % window : t;
                    for (int d = 0; d < D; ++d) acc[d] += pr * ld(vc, cbase + slot * D + d);
                }
            }
            double *yo = y + ((int64_t)b * Hq + h) * D;
            for (int d = 0; d < D; ++d)
                yo[d] = gated ? acc[d] * sigmoid(ld(g, ((int64_t)b * Hq + h) * D + d)) : acc[d];
            free(qt); free(kt); free(s); free(acc);
        }
    }
    free(wq); free(wk);
    return status;
}

/*
 * KV-cache bytes at context length T (§2.3): a layer stores K and V of Hkv
 * heads of dim D per cached token; a global layer caches all T tokens, a
 * sliding-window layer at most W.
 */
int64_t oracle_kv_bytes(int n_global, int n_window, int window, int Hkv, int D,
                        int bytes_per_elem, int64_t T)
{
    int64_t per_token = 2LL * Hkv * D * bytes_per_elem;
    int64_t swa_tokens = T < window ? T : window;
    return per_token * ((int64_t)n_global * T + (int64_t)n_window * swa_tokens);
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * oracle.c -- plain, slow, step-by-step fp64 reference of the DiG token mixer.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test-suite, the smoke check and the CPU
 * baseline leg of the benchmark may load this library.  It shares no code,
 * header, table or constant with the CUDA path in gated_linear_attention_fwd_b200/.
 *
 * Sources ("DiG: Scalable and Efficient Diffusion Models with Gated Linear
 * Attention", the docswell study-group slides, page 2 of the reference set):
 *   - GLA recurrence: slide "Gated Linear Attention Transformer (GLA) の導入",
 *     eq. (5)-(8).  The gate is read as alpha_t = sigmoid(z_t)^(1/tau) with the
 *     value gate beta fixed to 1, the state is S_t = diag(alpha_t) S_{t-1} + k_t^T v_t
 *     and the output is the row-vector product o_t = q_t S_t (S includes token t).
 *   - Output gate and norm: same slide, eq. (9)-(10), with the norm read as
 *     RMSNorm over d_v (Fig. 4 labels it "RMS Norm").
 *   - SREM: slide "SREM (Spatial Reorient & Enhancement Module) の導入": a 3x3
 *     depthwise conv on the 2-D token grid followed by a transpose / flip of the
 *     scan order.
 *
 * Layouts (all fp64, row-major, tokens in grid row-major order g = row*Wg + col):
 *   q, k        [B][L][H][dk]
 *   v, o, dO    [B][L][H][dv]
 *   z, dlogalpha [B][L][Hz][dk]   (Hz = gate_heads, 1 or H)
 *   x (conv in) [B][Hg][Wg][C];  conv out y [B][L][C] in scan order
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Scan order: grid index visited at scan position t (DiG scanning directions;
 * the four modes are row-major forward / reversed and column-major forward /
 * reversed).  Returns -1 for a bad mode. */
long oracle_scan_index(int mode, long Hg, long Wg, long t)
{
    long L = Hg * Wg;
    switch (mode) {
    case 0: return t;                                   /* row-major, forward   */
    case 1: return L - 1 - t;                           /* row-major, reversed  */
    case 2: return (t % Hg) * Wg + t / Hg;              /* column-major forward */
    case 3: { long u = L - 1 - t; return (u % Hg) * Wg + u / Hg; } /* col, reversed */
    default: return -1;
    }
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_num_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* log(sigmoid(x)) evaluated without overflow. */
static double log_sigmoid(double x)
{
    return (x < 0.0 ? x : 0.0) - log1p(exp(-fabs(x)));
}

static int check_shape(long B, long H, long L, long dk, long dv, long Hg, long Wg,
                       int mode, int gate_heads)
{
    if (B < 0 || H <= 0 || L < 0 || dk <= 0 || dv <= 0) return 1;
    if (Hg * Wg != L) return 1;
    if (mode < 0 || mode > 3) return 1;
    if (gate_heads != 1 && gate_heads != H) return 1;
    return 0;
}

/* Forward recurrence, one token at a time in scan order. */
int oracle_gla_fwd(const double *q, const double *k, const double *v, const double *z,
                   int gate_heads, double inv_tau, double *o,
                   long B, long H, long L, long dk, long dv, long Hg, long Wg, int mode)
{
    if (check_shape(B, H, L, dk, dv, Hg, Wg, mode, gate_heads)) return 1;
    long n = B * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (long bh = 0; bh < n; ++bh) {
        long b = bh / H, h = bh % H, hz = (gate_heads == 1) ? 0 : h;
        double *S = (double *)calloc((size_t)(dk * dv), sizeof(double));
        double *alpha = (double *)malloc((size_t)dk * sizeof(double));
        for (long t = 0; t < L; ++t) {
            long g = oracle_scan_index(mode, Hg, Wg, t);
            const double *qt = q + ((b * L + g) * H + h) * dk;
            const double *kt = k + ((b * L + g) * H + h) * dk;
            const double *vt = v + ((b * L + g) * H + h) * dv;
            const double *zt = z + ((b * L + g) * gate_heads + hz) * dk;
            double *ot = o + ((b * L + g) * H + h) * dv;
            for (long c = 0; c < dk; ++c) alpha[c] = exp(inv_tau * log_sigmoid(zt[c]));
            /* S_t = diag(alpha_t) S_{t-1} + k_t^T v_t */
            for (long c = 0; c < dk; ++c)
                for (long j = 0; j < dv; ++j)
                    S[c * dv + j] = alpha[c] * S[c * dv + j] + kt[c] * vt[j];
            /* o_t = q_t S_t */
            for (long j = 0; j < dv; ++j) {
                double acc = 0.0;
                for (long c = 0; c < dk; ++c) acc += qt[c] * S[c * dv + j];
                ot[j] = acc;
            }
        }
        free(S);
        free(alpha);
    }
    return 0;
}

/* The recurrence with the general gate and state I/O ([Slides] eq. (5)-(8) before
 * the value gate is fixed to 1):
 *   G_t = alpha_t^T beta_t (d_k x d_v),  S_t = G_t (*) S_{t-1} + k_t^T v_t,  o_t = q_t S_t
 * with beta_t = sigmoid(zb_t)^(1/tau) from value-gate logits zb [B][L][Hz][dv]
 * (NULL: beta = 1), S_0 from S0 [B*H][dk][dv] (NULL: 0), and the state after the
 * last scan position written to S_final [B*H][dk][dv] (NULL: not written). */
int oracle_gla_fwd_ext(const double *q, const double *k, const double *v, const double *z,
                       const double *zb, int gate_heads, double inv_tau, const double *S0,
                       double *o, double *S_final,
                       long B, long H, long L, long dk, long dv, long Hg, long Wg, int mode)
{
    if (check_shape(B, H, L, dk, dv, Hg, Wg, mode, gate_heads)) return 1;
    long n = B * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (long bh = 0; bh < n; ++bh) {
        long b = bh / H, h = bh % H, hz = (gate_heads == 1) ? 0 : h;
        double *S = (double *)calloc((size_t)(dk * dv), sizeof(double));
        double *alpha = (double *)malloc((size_t)dk * sizeof(double));
        double *beta = (double *)malloc((size_t)dv * sizeof(double));
        if (S0)
            for (long e = 0; e < dk * dv; ++e) S[e] = S0[bh * dk * dv + e];
        for (long t = 0; t < L; ++t) {
            long g = oracle_scan_index(mode, Hg, Wg, t);
            const double *qt = q + ((b * L + g) * H + h) * dk;
            const double *kt = k + ((b * L + g) * H + h) * dk;
            const double *vt = v + ((b * L + g) * H + h) * dv;
            const double *zt = z + ((b * L + g) * gate_heads + hz) * dk;
            double *ot = o + ((b * L + g) * H + h) * dv;
            for (long c = 0; c < dk; ++c) alpha[c] = exp(inv_tau * log_sigmoid(zt[c]));
            for (long j = 0; j < dv; ++j)
                beta[j] = zb ? exp(inv_tau * log_sigmoid(zb[((b * L + g) * gate_heads + hz) * dv + j])) : 1.0;
            /* S_t = (alpha_t^T beta_t) (*) S_{t-1} + k_t^T v_t */
            for (long c = 0; c < dk; ++c)
                for (long j = 0; j < dv; ++j)
                    S[c * dv + j] = alpha[c] * beta[j] * S[c * dv + j] + kt[c] * vt[j];
            for (long j = 0; j < dv; ++j) {
                double acc = 0.0;
                for (long c = 0; c < dk; ++c) acc += qt[c] * S[c * dv + j];
                ot[j] = acc;
            }
        }
        if (S_final)
            for (long e = 0; e < dk * dv; ++e) S_final[bh * dk * dv + e] = S[e];
        free(S);
        free(alpha);
        free(beta);
    }
    return 0;
}

/* Backward of the recurrence: a reverse sweep over the scan order carrying
 * dS = dLoss/dS_t.  The forward states are rebuilt from checkpoints taken every
 * CK steps.  dlogalpha is the gradient with respect to log(alpha_t); with one
 * shared gate (gate_heads == 1) it is summed over heads. */
#define CK 64
int oracle_gla_bwd(const double *q, const double *k, const double *v, const double *z,
                   int gate_heads, double inv_tau, const double *dO,
                   double *dq, double *dk_out, double *dv_out, double *dlogalpha,
                   long B, long H, long L, long dk, long dv, long Hg, long Wg, int mode)
{
    if (check_shape(B, H, L, dk, dv, Hg, Wg, mode, gate_heads)) return 1;
    long n = B * H;
    long nblk = (L + CK - 1) / CK;
    /* per-head dlogalpha, reduced over heads afterwards in a fixed order */
    double *dla_h = (double *)calloc((size_t)(B * H * L * dk) + 1, sizeof(double));
    if (!dla_h) return 2;
#pragma omp parallel for schedule(dynamic, 1)
    for (long bh = 0; bh < n; ++bh) {
        long b = bh / H, h = bh % H, hz = (gate_heads == 1) ? 0 : h;
        size_t ssz = (size_t)(dk * dv);
        double *ckpt = (double *)calloc(ssz * (size_t)(nblk + 1), sizeof(double));
        double *blk = (double *)malloc(ssz * CK * sizeof(double));
        double *S = (double *)calloc(ssz, sizeof(double));
        double *dS = (double *)calloc(ssz, sizeof(double));
        double *alpha = (double *)malloc((size_t)dk * sizeof(double));
        /* forward sweep: ckpt[m] = state before the first token of block m */
        for (long t = 0; t < L; ++t) {
            if (t % CK == 0) memcpy(ckpt + (size_t)(t / CK) * ssz, S, ssz * sizeof(double));
            long g = oracle_scan_index(mode, Hg, Wg, t);
            const double *kt = k + ((b * L + g) * H + h) * dk;
            const double *vt = v + ((b * L + g) * H + h) * dv;
            const double *zt = z + ((b * L + g) * gate_heads + hz) * dk;
            for (long c = 0; c < dk; ++c) {
                double a = exp(inv_tau * log_sigmoid(zt[c]));
                for (long j = 0; j < dv; ++j) S[c * dv + j] = a * S[c * dv + j] + kt[c] * vt[j];
            }
        }
        /* reverse sweep */
        for (long m = nblk - 1; m >= 0; --m) {
            long t0 = m * CK, t1 = (t0 + CK < L) ? t0 + CK : L;
            /* rebuild S_t for t in [t0, t1) */
            memcpy(S, ckpt + (size_t)m * ssz, ssz * sizeof(double));
            for (long t = t0; t < t1; ++t) {
                long g = oracle_scan_index(mode, Hg, Wg, t);
                const double *kt = k + ((b * L + g) * H + h) * dk;
                const double *vt = v + ((b * L + g) * H + h) * dv;
                const double *zt = z + ((b * L + g) * gate_heads + hz) * dk;
                for (long c = 0; c < dk; ++c) {
                    double a = exp(inv_tau * log_sigmoid(zt[c]));
                    for (long j = 0; j < dv; ++j) S[c * dv + j] = a * S[c * dv + j] + kt[c] * vt[j];
                }
                memcpy(blk + (size_t)(t - t0) * ssz, S, ssz * sizeof(double));
            }
            for (long t = t1 - 1; t >= t0; --t) {
                long g = oracle_scan_index(mode, Hg, Wg, t);
                const double *qt = q + ((b * L + g) * H + h) * dk;
                const double *kt = k + ((b * L + g) * H + h) * dk;
                const double *vt = v + ((b * L + g) * H + h) * dv;
                const double *zt = z + ((b * L + g) * gate_heads + hz) * dk;
                const double *dot = dO + ((b * L + g) * H + h) * dv;
                const double *St = blk + (size_t)(t - t0) * ssz;
                const double *Sp = (t > t0) ? blk + (size_t)(t - 1 - t0) * ssz
                                            : ckpt + (size_t)m * ssz;
                double *dqt = dq + ((b * L + g) * H + h) * dk;
                double *dkt = dk_out + ((b * L + g) * H + h) * dk;
                double *dvt = dv_out + ((b * L + g) * H + h) * dv;
                double *dlat = dla_h + ((b * H + h) * L + g) * dk;
                for (long c = 0; c < dk; ++c) alpha[c] = exp(inv_tau * log_sigmoid(zt[c]));
                /* dS_t = q_t^T dO_t + (carried gradient from S_{t+1}) */
                for (long c = 0; c < dk; ++c)
                    for (long j = 0; j < dv; ++j) dS[c * dv + j] += qt[c] * dot[j];
                /* dq_t = dO_t S_t^T */
                for (long c = 0; c < dk; ++c) {
                    double acc = 0.0;
                    for (long j = 0; j < dv; ++j) acc += dot[j] * St[c * dv + j];
                    dqt[c] = acc;
                }
                /* dk_t = v_t dS_t^T,  dv_t = k_t dS_t */
                for (long c = 0; c < dk; ++c) {
                    double acc = 0.0;
                    for (long j = 0; j < dv; ++j) acc += dS[c * dv + j] * vt[j];
                    dkt[c] = acc;
                }
                for (long j = 0; j < dv; ++j) {
                    double acc = 0.0;
                    for (long c = 0; c < dk; ++c) acc += kt[c] * dS[c * dv + j];
                    dvt[j] = acc;
                }
                /* dLoss/dlog(alpha_t)[c] = alpha_t[c] * sum_j dS_t[c,j] S_{t-1}[c,j] */
                for (long c = 0; c < dk; ++c) {
                    double acc = 0.0;
                    for (long j = 0; j < dv; ++j) acc += dS[c * dv + j] * Sp[c * dv + j];
                    dlat[c] = alpha[c] * acc;
                }
                /* gradient carried to S_{t-1} */
                for (long c = 0; c < dk; ++c)
                    for (long j = 0; j < dv; ++j) dS[c * dv + j] *= alpha[c];
            }
        }
        free(ckpt); free(blk); free(S); free(dS); free(alpha);
    }
    /* scatter / reduce per-head values into the gate layout */
    for (long b = 0; b < B; ++b)
        for (long g = 0; g < L; ++g) {
            if (gate_heads == 1) {
                double *dst = dlogalpha + (b * L + g) * dk;
                for (long c = 0; c < dk; ++c) {
                    double acc = 0.0;
                    for (long h = 0; h < H; ++h) acc += dla_h[((b * H + h) * L + g) * dk + c];
                    dst[c] = acc;
                }
            } else {
                for (long h = 0; h < H; ++h)
                    memcpy(dlogalpha + ((b * L + g) * H + h) * dk,
                           dla_h + ((b * H + h) * L + g) * dk, (size_t)dk * sizeof(double));
            }
        }
    free(dla_h);
    return 0;
}

/* y = Swish(r) * RMSNorm(o) * gamma, the norm taken over the d_v features of
 * one (token, head) row (slide eq. (9)-(10)).  gamma may be NULL (all ones). */
int oracle_epilogue(const double *o, const double *r, const double *gamma, double eps,
                    double *y, long rows, long dv)
{
    if (rows < 0 || dv <= 0) return 1;
#pragma omp parallel for schedule(static)
    for (long i = 0; i < rows; ++i) {
        const double *oi = o + i * dv, *ri = r + i * dv;
        double ms = 0.0;
        for (long j = 0; j < dv; ++j) ms += oi[j] * oi[j];
        double inv = 1.0 / sqrt(ms / (double)dv + eps);
        for (long j = 0; j < dv; ++j) {
            double sw = ri[j] / (1.0 + exp(-ri[j]));
            y[i * dv + j] = sw * oi[j] * inv * (gamma ? gamma[j] : 1.0);
        }
    }
    return 0;
}

/* Backward of the epilogue above (same slide, eq. (9)-(10)), by the chain rule.
 * Per row, with s_j = Swish(r_j) = r_j sigmoid(r_j), inv = 1/sqrt(mean(o^2) + eps)
 * and y_j = s_j o_j inv gamma_j:
 *   dy_j/do_m    = s_j gamma_j (delta_jm inv + o_j dinv/do_m),  dinv/do_m = -inv^3 o_m / dv
 *   dy_j/dr_j    = o_j inv gamma_j Swish'(r_j),  Swish'(x) = sigmoid(x) (1 + x (1 - sigmoid(x)))
 *   dy_j/dgamma_j = s_j o_j inv
 * d_o, d_r are per row; d_gamma sums over rows (NULL skips it). */
int oracle_epilogue_bwd(const double *o, const double *r, const double *gamma, double eps,
                        const double *dy, double *d_o, double *d_r, double *d_gamma,
                        long rows, long dv)
{
    if (rows < 0 || dv <= 0) return 1;
#pragma omp parallel for schedule(static)
    for (long i = 0; i < rows; ++i) {
        const double *oi = o + i * dv, *ri = r + i * dv, *gi = dy + i * dv;
        double ms = 0.0;
        for (long j = 0; j < dv; ++j) ms += oi[j] * oi[j];
        double inv = 1.0 / sqrt(ms / (double)dv + eps);
        double dinv_sum = 0.0;  /* sum_j dy_j s_j gamma_j o_j: the weight of dinv/do_m */
        for (long j = 0; j < dv; ++j) {
            double sig = 1.0 / (1.0 + exp(-ri[j]));
            double gm = gamma ? gamma[j] : 1.0;
            dinv_sum += gi[j] * ri[j] * sig * gm * oi[j];
        }
        for (long m = 0; m < dv; ++m) {
            double sig = 1.0 / (1.0 + exp(-ri[m]));
            double gm = gamma ? gamma[m] : 1.0;
            double direct = gi[m] * ri[m] * sig * gm * inv;
            double through_inv = dinv_sum * (-inv * inv * inv * oi[m] / (double)dv);
            d_o[i * dv + m] = direct + through_inv;
            d_r[i * dv + m] = gi[m] * oi[m] * inv * gm * sig * (1.0 + ri[m] * (1.0 - sig));
        }
    }
    if (d_gamma) {
        for (long j = 0; j < dv; ++j) d_gamma[j] = 0.0;
        for (long i = 0; i < rows; ++i) {
            const double *oi = o + i * dv, *ri = r + i * dv, *gi = dy + i * dv;
            double ms = 0.0;
            for (long j = 0; j < dv; ++j) ms += oi[j] * oi[j];
            double inv = 1.0 / sqrt(ms / (double)dv + eps);
            for (long j = 0; j < dv; ++j)
                d_gamma[j] += gi[j] * ri[j] / (1.0 + exp(-ri[j])) * oi[j] * inv;
        }
    }
    return 0;
}

/* SREM: 3x3 depthwise cross-correlation with zero "same" padding on the grid,
 * result written in scan order: y[b][t][ch] = conv(x)[b][grid(t)][ch]. */
int oracle_srem_dwconv(const double *x, const double *w, const double *bias, double *y,
                       long B, long Hg, long Wg, long C, int mode)
{
    if (B < 0 || Hg < 0 || Wg < 0 || C <= 0 || mode < 0 || mode > 3) return 1;
    long L = Hg * Wg;
#pragma omp parallel for schedule(static)
    for (long bt = 0; bt < B * L; ++bt) {
        long b = bt / L, t = bt % L;
        long g = oracle_scan_index(mode, Hg, Wg, t);
        long r0 = g / Wg, c0 = g % Wg;
        for (long ch = 0; ch < C; ++ch) {
            double acc = bias ? bias[ch] : 0.0;
            for (long di = -1; di <= 1; ++di)
                for (long dj = -1; dj <= 1; ++dj) {
                    long rr = r0 + di, cc = c0 + dj;
                    if (rr < 0 || rr >= Hg || cc < 0 || cc >= Wg) continue;
                    acc += w[ch * 9 + (di + 1) * 3 + (dj + 1)] * x[((b * Hg + rr) * Wg + cc) * C + ch];
                }
            y[(b * L + t) * C + ch] = acc;
        }
    }
    return 0;
}

/* Backward of the SREM conv above: gradients of sum_t dy[b][t][ch] y[b][t][ch].
 * The scan-order gradient is first put back on the grid (dyg[b][pi(t)] = dy[b][t]);
 * then, from y_g = bias + sum_{di,dj} w[di,dj] x[g + (di,dj)],
 *   dx[g]       = sum_{di,dj} w[di,dj] dyg[g - (di,dj)]   (terms inside the grid)
 *   dw[di,dj]   = sum_{b,g} dyg[g] x[g + (di,dj)]            (zero outside the grid)
 *   dbias       = sum_{b,g} dyg[g]
 * dx is in grid order [B][Hg][Wg][C]; dw [C][3][3]; dbias [C] (NULL skips it). */
int oracle_srem_dwconv_bwd(const double *x, const double *w, const double *dy,
                           double *dx, double *dw, double *dbias,
                           long B, long Hg, long Wg, long C, int mode)
{
    if (B < 0 || Hg < 0 || Wg < 0 || C <= 0 || mode < 0 || mode > 3) return 1;
    long L = Hg * Wg;
    double *dyg = (double *)malloc(sizeof(double) * (size_t)(B * L * C > 0 ? B * L * C : 1));
    if (!dyg) return 2;
    for (long b = 0; b < B; ++b)
        for (long t = 0; t < L; ++t) {
            long g = oracle_scan_index(mode, Hg, Wg, t);
            for (long ch = 0; ch < C; ++ch) dyg[(b * L + g) * C + ch] = dy[(b * L + t) * C + ch];
        }
#pragma omp parallel for schedule(static)
    for (long bg = 0; bg < B * L; ++bg) {
        long b = bg / L, g = bg % L, r0 = g / Wg, c0 = g % Wg;
        for (long ch = 0; ch < C; ++ch) {
            double acc = 0.0;
            for (long di = -1; di <= 1; ++di)
                for (long dj = -1; dj <= 1; ++dj) {
                    long rr = r0 - di, cc = c0 - dj;  /* output pixel that read x[g] through tap (di,dj) */
                    if (rr < 0 || rr >= Hg || cc < 0 || cc >= Wg) continue;
                    acc += w[ch * 9 + (di + 1) * 3 + (dj + 1)] * dyg[((b * Hg + rr) * Wg + cc) * C + ch];
                }
            dx[bg * C + ch] = acc;
        }
    }
#pragma omp parallel for schedule(static)
    for (long ch = 0; ch < C; ++ch) {
        for (long tap = 0; tap < 9; ++tap) {
            long di = tap / 3 - 1, dj = tap % 3 - 1;
            double acc = 0.0;
            for (long b = 0; b < B; ++b)
                for (long rr = 0; rr < Hg; ++rr)
                    for (long cc = 0; cc < Wg; ++cc) {
                        long xr = rr + di, xc = cc + dj;
                        if (xr < 0 || xr >= Hg || xc < 0 || xc >= Wg) continue;
                        acc += dyg[((b * Hg + rr) * Wg + cc) * C + ch] * x[((b * Hg + xr) * Wg + xc) * C + ch];
                    }
            dw[ch * 9 + tap] = acc;
        }
        if (dbias) {
            double acc = 0.0;
            for (long bg = 0; bg < B * L; ++bg) acc += dyg[bg * C + ch];
            dbias[ch] = acc;
        }
    }
    free(dyg);
    return 0;
}

/* Gate projection (slide "Gated Linear Attention Transformer (GLA) の導入", eq. (5):
 * the gate logits come from the block input through a low-rank projection):
 *   u = x W1   [rows][R],   z = u W2 + b   [rows][dk]
 * x [rows][D], W1 [D][R], W2 [R][dk], b [dk] (NULL = 0).  u may be NULL. */
int oracle_gate_proj_fwd(const double *x, const double *W1, const double *W2, const double *b,
                         double *z, double *u, long rows, long D, long R, long dk)
{
    if (rows < 0 || D <= 0 || R <= 0 || dk <= 0) return 1;
#pragma omp parallel for schedule(static)
    for (long t = 0; t < rows; ++t) {
        double ut[64];
        if (R > 64) continue;
        for (long r = 0; r < R; ++r) {
            double acc = 0.0;
            for (long d = 0; d < D; ++d) acc += x[t * D + d] * W1[d * R + r];
            ut[r] = acc;
            if (u) u[t * R + r] = acc;
        }
        for (long k = 0; k < dk; ++k) {
            double acc = b ? b[k] : 0.0;
            for (long r = 0; r < R; ++r) acc += ut[r] * W2[r * dk + k];
            z[t * dk + k] = acc;
        }
    }
    return R > 64 ? 1 : 0;
}

/* Its backward from the GLA backward's d log(alpha): log(alpha) = inv_tau * logsigmoid(z),
 * so dz = dlog_alpha * inv_tau * sigmoid(-z); then, by the chain rule through z = (x W1) W2 + b,
 *   du = dz W2^T,  dx = du W1^T,  dW1 = x^T du,  dW2 = u^T dz (u = x W1),  db = sum_t dz. */
int oracle_gate_proj_bwd(const double *x, const double *W1, const double *W2, const double *z,
                         const double *dla, double inv_tau, double *dx, double *dW1, double *dW2,
                         double *db, long rows, long D, long R, long dk)
{
    if (rows < 0 || D <= 0 || R <= 0 || dk <= 0 || R > 64) return 1;
    double *u = (double *)malloc(sizeof(double) * (size_t)(rows * R > 0 ? rows * R : 1));
    double *du = (double *)malloc(sizeof(double) * (size_t)(rows * R > 0 ? rows * R : 1));
    double *dz = (double *)malloc(sizeof(double) * (size_t)(rows * dk > 0 ? rows * dk : 1));
    if (!u || !du || !dz) { free(u); free(du); free(dz); return 2; }
#pragma omp parallel for schedule(static)
    for (long t = 0; t < rows; ++t) {
        for (long k = 0; k < dk; ++k)
            dz[t * dk + k] = dla[t * dk + k] * inv_tau / (1.0 + exp(z[t * dk + k]));
        for (long r = 0; r < R; ++r) {
            double a = 0.0, g = 0.0;
            for (long d = 0; d < D; ++d) a += x[t * D + d] * W1[d * R + r];
            for (long k = 0; k < dk; ++k) g += dz[t * dk + k] * W2[r * dk + k];
            u[t * R + r] = a;
            du[t * R + r] = g;
        }
        for (long d = 0; d < D; ++d) {
            double acc = 0.0;
            for (long r = 0; r < R; ++r) acc += du[t * R + r] * W1[d * R + r];
            dx[t * D + d] = acc;
        }
    }
#pragma omp parallel for schedule(static)
    for (long d = 0; d < D; ++d)
        for (long r = 0; r < R; ++r) {
            double acc = 0.0;
            for (long t = 0; t < rows; ++t) acc += x[t * D + d] * du[t * R + r];
            dW1[d * R + r] = acc;
        }
    for (long r = 0; r < R; ++r)
        for (long k = 0; k < dk; ++k) {
            double acc = 0.0;
            for (long t = 0; t < rows; ++t) acc += u[t * R + r] * dz[t * dk + k];
            dW2[r * dk + k] = acc;
        }
    if (db)
        for (long k = 0; k < dk; ++k) {
            double acc = 0.0;
            for (long t = 0; t < rows; ++t) acc += dz[t * dk + k];
            db[k] = acc;
        }
    free(u); free(du); free(dz);
    return 0;
}

/* Backward of oracle_gla_fwd_ext: gradients of sum_t o_t . dO_t + sum S_final (*) dSf
 * (dSf [B*H][dk][dv], NULL = 0).  Reverse sweep carrying dS = dLoss/dS_t:
 *   dS += q_t^T dO_t;  dq_t = dO_t S_t^T;  dk_t = v_t dS^T;  dv_t = k_t dS;
 *   dlog(alpha_t)[c] = sum_j dS[c][j] G_t[c][j] S_{t-1}[c][j],
 *   dlog(beta_t)[j]  = sum_c dS[c][j] G_t[c][j] S_{t-1}[c][j],
 *   dS <- G_t (*) dS  (the gradient of S_{t-1});  after t = 0 it is dS0.
 * Forward states are rebuilt from checkpoints every CK steps.  dlogalpha
 * [B][L][Hz][dk] and dlogbeta [B][L][Hz][dv] (NULL: not formed) are summed over
 * heads for a shared gate; dS0 [B*H][dk][dv] may be NULL. */
int oracle_gla_bwd_ext(const double *q, const double *k, const double *v, const double *z,
                       const double *zb, int gate_heads, double inv_tau, const double *S0,
                       const double *dO, const double *dSf,
                       double *dq, double *dk_out, double *dv_out, double *dlogalpha,
                       double *dlogbeta, double *dS0,
                       long B, long H, long L, long dk, long dv, long Hg, long Wg, int mode)
{
    if (check_shape(B, H, L, dk, dv, Hg, Wg, mode, gate_heads)) return 1;
    long n = B * H;
    long nblk = (L + CK - 1) / CK;
    double *dla_h = (double *)calloc((size_t)(B * H * L * dk) + 1, sizeof(double));
    double *dlb_h = (double *)calloc((size_t)(B * H * L * dv) + 1, sizeof(double));
    if (!dla_h || !dlb_h) { free(dla_h); free(dlb_h); return 2; }
#pragma omp parallel for schedule(dynamic, 1)
    for (long bh = 0; bh < n; ++bh) {
        long b = bh / H, h = bh % H, hz = (gate_heads == 1) ? 0 : h;
        size_t ssz = (size_t)(dk * dv);
        double *ckpt = (double *)calloc(ssz * (size_t)(nblk + 1), sizeof(double));
        double *blk = (double *)malloc(ssz * CK * sizeof(double));
        double *S = (double *)calloc(ssz, sizeof(double));
        double *dS = (double *)calloc(ssz, sizeof(double));
        double *G = (double *)malloc(ssz * sizeof(double));
        /* the gate of token g: G[c][j] = alpha[c] beta[j] */
        #define EXT_GATE(g_)                                                                        \
            for (long c = 0; c < dk; ++c) {                                                         \
                double a_ = exp(inv_tau * log_sigmoid(z[((b * L + (g_)) * gate_heads + hz) * dk + c])); \
                for (long j = 0; j < dv; ++j)                                                       \
                    G[c * dv + j] = a_ * (zb ? exp(inv_tau * log_sigmoid(                           \
                                                   zb[((b * L + (g_)) * gate_heads + hz) * dv + j])) \
                                             : 1.0);                                                \
            }
        if (S0) memcpy(S, S0 + bh * ssz, ssz * sizeof(double));
        for (long t = 0; t < L; ++t) {
            if (t % CK == 0) memcpy(ckpt + (size_t)(t / CK) * ssz, S, ssz * sizeof(double));
            long g = oracle_scan_index(mode, Hg, Wg, t);
            const double *kt = k + ((b * L + g) * H + h) * dk;
            const double *vt = v + ((b * L + g) * H + h) * dv;
            EXT_GATE(g)
            for (long c = 0; c < dk; ++c)
                for (long j = 0; j < dv; ++j) S[c * dv + j] = G[c * dv + j] * S[c * dv + j] + kt[c] * vt[j];
        }
        if (dSf) memcpy(dS, dSf + bh * ssz, ssz * sizeof(double));
        for (long m = nblk - 1; m >= 0; --m) {
            long t0 = m * CK, t1 = (t0 + CK < L) ? t0 + CK : L;
            memcpy(S, ckpt + (size_t)m * ssz, ssz * sizeof(double));
            for (long t = t0; t < t1; ++t) {
                long g = oracle_scan_index(mode, Hg, Wg, t);
                const double *kt = k + ((b * L + g) * H + h) * dk;
                const double *vt = v + ((b * L + g) * H + h) * dv;
                EXT_GATE(g)
                for (long c = 0; c < dk; ++c)
                    for (long j = 0; j < dv; ++j) S[c * dv + j] = G[c * dv + j] * S[c * dv + j] + kt[c] * vt[j];
                memcpy(blk + (size_t)(t - t0) * ssz, S, ssz * sizeof(double));
            }
            for (long t = t1 - 1; t >= t0; --t) {
                long g = oracle_scan_index(mode, Hg, Wg, t);
                const double *qt = q + ((b * L + g) * H + h) * dk;
                const double *kt = k + ((b * L + g) * H + h) * dk;
                const double *vt = v + ((b * L + g) * H + h) * dv;
                const double *dot = dO + ((b * L + g) * H + h) * dv;
                const double *St = blk + (size_t)(t - t0) * ssz;
                const double *Sp = (t > t0) ? blk + (size_t)(t - 1 - t0) * ssz : ckpt + (size_t)m * ssz;
                double *dqt = dq + ((b * L + g) * H + h) * dk;
                double *dkt = dk_out + ((b * L + g) * H + h) * dk;
                double *dvt = dv_out + ((b * L + g) * H + h) * dv;
                double *dlat = dla_h + ((b * H + h) * L + g) * dk;
                double *dlbt = dlb_h + ((b * H + h) * L + g) * dv;
                EXT_GATE(g)
                for (long c = 0; c < dk; ++c)
                    for (long j = 0; j < dv; ++j) dS[c * dv + j] += qt[c] * dot[j];
                for (long c = 0; c < dk; ++c) {
                    double acc = 0.0;
                    for (long j = 0; j < dv; ++j) acc += dot[j] * St[c * dv + j];
                    dqt[c] = acc;
                }
                for (long c = 0; c < dk; ++c) {
                    double acc = 0.0;
                    for (long j = 0; j < dv; ++j) acc += dS[c * dv + j] * vt[j];
                    dkt[c] = acc;
                }
                for (long j = 0; j < dv; ++j) {
                    double acc = 0.0;
                    for (long c = 0; c < dk; ++c) acc += kt[c] * dS[c * dv + j];
                    dvt[j] = acc;
                }
                for (long c = 0; c < dk; ++c) dlat[c] = 0.0;
                for (long j = 0; j < dv; ++j) dlbt[j] = 0.0;
                for (long c = 0; c < dk; ++c)
                    for (long j = 0; j < dv; ++j) {
                        double w = dS[c * dv + j] * G[c * dv + j] * Sp[c * dv + j];
                        dlat[c] += w;
                        dlbt[j] += w;
                    }
                for (long e = 0; e < (long)ssz; ++e) dS[e] *= G[e];
            }
        }
        if (dS0) memcpy(dS0 + bh * ssz, dS, ssz * sizeof(double));
        #undef EXT_GATE
        free(ckpt); free(blk); free(S); free(dS); free(G);
    }
    long Hz = gate_heads;
    if (dlogalpha)
        for (long b = 0; b < B; ++b)
            for (long g = 0; g < L; ++g)
                for (long hz = 0; hz < Hz; ++hz)
                    for (long c = 0; c < dk; ++c) {
                        double acc = 0.0;
                        for (long h = 0; h < H; ++h)
                            if (Hz == 1 || h == hz) acc += dla_h[((b * H + h) * L + g) * dk + c];
                        dlogalpha[((b * L + g) * Hz + hz) * dk + c] = acc;
                    }
    if (dlogbeta)
        for (long b = 0; b < B; ++b)
            for (long g = 0; g < L; ++g)
                for (long hz = 0; hz < Hz; ++hz)
                    for (long j = 0; j < dv; ++j) {
                        double acc = 0.0;
                        for (long h = 0; h < H; ++h)
                            if (Hz == 1 || h == hz) acc += dlb_h[((b * H + h) * L + g) * dv + j];
                        dlogbeta[((b * L + g) * Hz + hz) * dv + j] = acc;
                    }
    free(dla_h);
    free(dlb_h);
    return 0;
}

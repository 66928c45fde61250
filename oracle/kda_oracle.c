/*
 * kda_oracle.c -- plain, slow CPU oracle for the Kimi Delta Attention (KDA)
 * chunk-prefill forward.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file; only the test suite, the smoke check and the CPU-baseline
 * leg of the benchmark use it.  It shares no code, header, table or helper
 * with the CUDA library.
 *
 * What it follows ("KDA Chunk Prefill on Ascend A3", section "Mathematical
 * definition"):
 *   - Q/K are L2-normalised row by row in float32 in the stated rounding
 *     order: widen bf16 -> f32, sum of squares in f32, add 1e-6 inside the
 *     square root, divide, round the quotient to bf16.
 *   - The normalised bf16 values are widened (here to float64) and the
 *     token-by-token recurrence is run for every (sequence, value head):
 *         Sdecay = exp(g_t)[:,None] * S
 *         r_t    = v_t - k_t^T Sdecay
 *         S      = Sdecay + beta_t k_t r_t^T
 *         o_t    = (K^-0.5 q_t)^T S
 *     The page states that the chunk form is an equivalent construction of
 *     this recurrence, so the recurrence is the definition the oracle uses.
 *   - Value head h reads Q/K head h // (HV/H) (section "Function and tensor
 *     contract").
 *
 * Readings where the page is silent (each is listed with its basis in the
 * design notes): the sum of squares is taken left to right; bf16 rounding is
 * round-to-nearest-even; the 1e-6 constant is the float32 literal; g is a
 * natural-log gate with one value per (token, value head, key channel); beta
 * has one value per (token, value head); a packed varlen batch is split by
 * int32 cu_seqlens with B == 1 and each sequence starts from its own state.
 *
 * Build: gcc -O2 -fopenmp -ffp-contract=off -shared -fPIC (no fast-math, so
 * that every float operation rounds exactly once as written).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ---- bf16 helpers -------------------------------------------------------- */

static float bf16_bits_to_f32(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* Round a float32 to the nearest bf16, ties to even; NaN stays NaN. */
static uint16_t f32_to_bf16_rne(float f)
{
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu) != 0u)
        return (uint16_t)((u >> 16) | 0x0040u);
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7fffu + lsb;
    return (uint16_t)(u >> 16);
}

/* Value of a finite bf16 magnitude pattern (sign bit clear). */
static double bf16_mag_value(uint32_t m)
{
    return (double)bf16_bits_to_f32((uint16_t)m);
}

/* Round a float64 straight to the nearest bf16 (ties to even), without an
 * intermediate float32 rounding.  Candidates are the bf16 magnitudes around
 * the truncated float32 pattern; the nearest one wins. */
static uint16_t f64_to_bf16_rne(double x)
{
    if (isnan(x)) return 0x7fc0u;
    uint16_t sign = signbit(x) ? 0x8000u : 0u;
    double a = fabs(x);
    if (a >= 3.3961775292304957e38) return (uint16_t)(sign | 0x7f80u); /* past the last tie */
    float af = (float)a;
    uint32_t u;
    memcpy(&u, &af, sizeof u);
    uint32_t base = u >> 16;
    uint32_t best = base;
    double best_err = fabs(bf16_mag_value(base) - a);
    for (int dlt = -1; dlt <= 1; dlt += 2) {
        int64_t c = (int64_t)base + dlt;
        if (c < 0 || c > 0x7f7f) continue;
        double err = fabs(bf16_mag_value((uint32_t)c) - a);
        if (err < best_err || (err == best_err && (c & 1) == 0)) {
            best = (uint32_t)c;
            best_err = err;
        }
    }
    return (uint16_t)(sign | best);
}

/* ---- normalisation ------------------------------------------------------- */

/* One row of K elements: xf = f32(x); xn = bf16(xf / sqrt(sum(xf*xf) + 1e-6)). */
static void l2norm_row(const uint16_t *x, int K, uint16_t *out)
{
    float ss = 0.0f;
    for (int d = 0; d < K; ++d) {
        float xf = bf16_bits_to_f32(x[d]);
        float sq = xf * xf;
        ss = ss + sq;
    }
    float den = sqrtf(ss + 1e-6f);
    for (int d = 0; d < K; ++d) {
        float xf = bf16_bits_to_f32(x[d]);
        out[d] = f32_to_bf16_rne(xf / den);
    }
}

void kda_oracle_l2norm_bf16(const uint16_t *x, int64_t rows, int K, uint16_t *out)
{
    for (int64_t r = 0; r < rows; ++r)
        l2norm_row(x + r * K, K, out + r * K);
}

/* ---- recurrence ---------------------------------------------------------- */

int kda_oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Token range of sequence n. */
static void seq_range(const int32_t *cu, int n, int T, int64_t *b, int64_t *t0, int64_t *t1)
{
    if (cu) {
        *b = 0;
        *t0 = cu[n];
        *t1 = cu[n + 1];
    } else {
        *b = n;
        *t0 = 0;
        *t1 = T;
    }
}

/*
 * Token-by-token recurrence in float64 on already-normalised inputs.
 *   q, k : [B,T,H,K]    v : [B,T,HV,V]    g : [B,T,HV,K]    beta : [B,T,HV]
 *   s0   : [N,HV,K,V] or NULL (zeros)     cu : [N+1] or NULL (then N == B)
 *   o    : [B,T,HV,V] (rows of tokens outside every sequence are left alone)
 *   sN   : [N,HV,K,V]
 * Units (sequence, value head) run in parallel; each one is sequential.
 * Returns 0, or -1 on a shape error.
 */
int kda_oracle_recurrence_f64(const double *q, const double *k, const double *v,
                              const double *g, const double *beta, const double *s0,
                              const int32_t *cu, int N, int B, int T, int H, int HV,
                              int K, int V, double *o, double *sN)
{
    if (N <= 0 || B <= 0 || T < 0 || H <= 0 || HV <= 0 || K <= 0 || V <= 0) return -1;
    if (HV % H != 0) return -1;
    if (cu && B != 1) return -1;
    if (!cu && N != B) return -1;
    const int group = HV / H;
    const double scale = 1.0 / sqrt((double)K);
    const int64_t units = (int64_t)N * HV;
    int bad = 0;

#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int64_t u = 0; u < units; ++u) {
        const int n = (int)(u / HV);
        const int h = (int)(u % HV);
        const int hq = h / group;
        int64_t b, t0, t1;
        seq_range(cu, n, T, &b, &t0, &t1);
        if (t0 < 0 || t1 < t0 || t1 > T) { bad |= 1; continue; }

        double *S = (double *)malloc(sizeof(double) * (size_t)K * V);
        double *r = (double *)malloc(sizeof(double) * (size_t)V);
        if (!S || !r) { free(S); free(r); bad |= 1; continue; }
        if (s0) memcpy(S, s0 + u * (int64_t)K * V, sizeof(double) * (size_t)K * V);
        else memset(S, 0, sizeof(double) * (size_t)K * V);

        for (int64_t t = t0; t < t1; ++t) {
            const int64_t row = b * T + t;
            const double *qt = q + (row * H + hq) * K;
            const double *kt = k + (row * H + hq) * K;
            const double *vt = v + (row * HV + h) * V;
            const double *gt = g + (row * HV + h) * K;
            const double bt = beta[row * HV + h];
            double *ot = o + (row * HV + h) * V;

            /* Sdecay = exp(g_t)[:,None] * S */
            for (int d = 0; d < K; ++d) {
                const double e = exp(gt[d]);
                for (int c = 0; c < V; ++c) S[(int64_t)d * V + c] *= e;
            }
            /* r = v_t - k_t^T Sdecay */
            for (int c = 0; c < V; ++c) {
                double acc = 0.0;
                for (int d = 0; d < K; ++d) acc += kt[d] * S[(int64_t)d * V + c];
                r[c] = vt[c] - acc;
            }
            /* S = Sdecay + beta_t k_t r^T */
            for (int d = 0; d < K; ++d) {
                const double bk = bt * kt[d];
                for (int c = 0; c < V; ++c) S[(int64_t)d * V + c] += bk * r[c];
            }
            /* o_t = (K^-0.5 q_t)^T S */
            for (int c = 0; c < V; ++c) {
                double acc = 0.0;
                for (int d = 0; d < K; ++d) acc += (scale * qt[d]) * S[(int64_t)d * V + c];
                ot[c] = acc;
            }
        }
        memcpy(sN + u * (int64_t)K * V, S, sizeof(double) * (size_t)K * V);
        free(S);
        free(r);
    }
    return bad ? -1 : 0;
}

/*
 * Whole forward from the raw inputs the library takes:
 *   q, k : bf16 bits [B,T,H,K] (unnormalised)   v : bf16 bits [B,T,HV,V]
 *   g : f32 [B,T,HV,K]   beta : f32 [B,T,HV]    s0 : f32 [N,HV,K,V] or NULL
 * Outputs: o64 [B,T,HV,V] float64, o16 the same rounded to bf16 (RNE),
 *          sN [N,HV,K,V] float64.  Optional qn/kn receive the normalised
 *          bf16 Q/K (pass NULL to skip).
 */
int kda_oracle_forward(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                       const float *g, const float *beta, const float *s0,
                       const int32_t *cu, int N, int B, int T, int H, int HV, int K, int V,
                       double *o64, uint16_t *o16, double *sN, uint16_t *qn, uint16_t *kn)
{
    const int64_t nqk = (int64_t)B * T * H * K;
    const int64_t nv = (int64_t)B * T * HV * V;
    const int64_t ng = (int64_t)B * T * HV * K;
    const int64_t nb = (int64_t)B * T * HV;
    const int64_t ns = (int64_t)N * HV * K * V;
    if (N <= 0 || B <= 0 || T < 0 || H <= 0 || HV <= 0 || K <= 0 || V <= 0) return -1;

    uint16_t *qn16 = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)(nqk ? nqk : 1));
    uint16_t *kn16 = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)(nqk ? nqk : 1));
    double *qd = (double *)malloc(sizeof(double) * (size_t)(nqk ? nqk : 1));
    double *kd = (double *)malloc(sizeof(double) * (size_t)(nqk ? nqk : 1));
    double *vd = (double *)malloc(sizeof(double) * (size_t)(nv ? nv : 1));
    double *gd = (double *)malloc(sizeof(double) * (size_t)(ng ? ng : 1));
    double *bd = (double *)malloc(sizeof(double) * (size_t)(nb ? nb : 1));
    double *sd = s0 ? (double *)malloc(sizeof(double) * (size_t)ns) : NULL;
    int rc = -1;
    if (!qn16 || !kn16 || !qd || !kd || !vd || !gd || !bd || (s0 && !sd)) goto done;

#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < (int64_t)B * T * H; ++r) {
        l2norm_row(q + r * K, K, qn16 + r * K);
        l2norm_row(k + r * K, K, kn16 + r * K);
    }
    for (int64_t i = 0; i < nqk; ++i) {
        qd[i] = (double)bf16_bits_to_f32(qn16[i]);
        kd[i] = (double)bf16_bits_to_f32(kn16[i]);
    }
    for (int64_t i = 0; i < nv; ++i) vd[i] = (double)bf16_bits_to_f32(v[i]);
    for (int64_t i = 0; i < ng; ++i) gd[i] = (double)g[i];
    for (int64_t i = 0; i < nb; ++i) bd[i] = (double)beta[i];
    if (s0)
        for (int64_t i = 0; i < ns; ++i) sd[i] = (double)s0[i];

    for (int64_t i = 0; i < nv; ++i) o64[i] = 0.0;
    rc = kda_oracle_recurrence_f64(qd, kd, vd, gd, bd, sd, cu, N, B, T, H, HV, K, V, o64, sN);
    if (rc == 0 && o16)
        for (int64_t i = 0; i < nv; ++i) o16[i] = f64_to_bf16_rne(o64[i]);
    if (rc == 0 && qn) memcpy(qn, qn16, sizeof(uint16_t) * (size_t)nqk);
    if (rc == 0 && kn) memcpy(kn, kn16, sizeof(uint16_t) * (size_t)nqk);

done:
    free(qn16); free(kn16); free(qd); free(kd); free(vd); free(gd); free(bd); free(sd);
    return rc;
}

/* Exposed for tests of the rounding helper itself. */
uint16_t kda_oracle_f64_to_bf16(double x) { return f64_to_bf16_rne(x); }

/*
 * Reverse mode of the float64 recurrence above, for the backward the page
 * "KDA Chunk Prefill on Ascend A3" leaves optional (section "Timing and
 * required submission"): the loss is sum(o * do) + sum(final_state * dht),
 * and the gradients are those of q, k, v, g, beta and the initial state.
 * This function differentiates the recurrence on the normalised inputs it is
 * given; the L2 normalisation's own derivative is applied by the caller.
 *
 * Inputs as kda_oracle_recurrence_f64, plus do_ [B,T,HV,V] and dht
 * [N,HV,K,V] (NULL = zero).  Outputs (all float64):
 *   dq, dk [B,T,HV,K]  gradient with respect to the normalised q/k row that
 *                      value head h read (the caller sums a Q/K head's group)
 *   dv [B,T,HV,V], dg [B,T,HV,K], dbeta [B,T,HV], ds0 [N,HV,K,V]
 * Rows outside every sequence (varlen) are left untouched.
 *
 * For a token t with S' = diag(exp g_t) S_{t-1}, r = v_t - S'^T k_t,
 * S_t = S' + beta_t k_t r^T and o_t = K^-0.5 S_t^T q_t, the adjoints, with dS
 * the gradient arriving at S_t, are taken in this order:
 *   dS  += K^-0.5 q_t do_t^T          dq_t  = K^-0.5 S_t do_t
 *   dr   = beta_t dS^T k_t             dbeta = k_t^T dS r
 *   dk_t = beta_t dS r - S' dr         dv_t  = dr
 *   dS'  = dS - k_t dr^T               dg_t  = rowsum(S' * dS')
 *   dS_{t-1} = diag(exp g_t) dS'
 * The states S_t are recomputed forward from checkpoints every 32 tokens.
 */
int kda_oracle_backward_f64(const double *q, const double *k, const double *v, const double *g,
                            const double *beta, const double *s0, const int32_t *cu, int N, int B, int T,
                            int H, int HV, int K, int V, const double *do_, const double *dht, double *dq,
                            double *dk, double *dv, double *dg, double *dbeta, double *ds0)
{
    if (N <= 0 || B <= 0 || T < 0 || H <= 0 || HV <= 0 || K <= 0 || V <= 0) return -1;
    if (HV % H != 0) return -1;
    if (cu && B != 1) return -1;
    if (!cu && N != B) return -1;
    const int group = HV / H;
    const double scale = 1.0 / sqrt((double)K);
    const int64_t units = (int64_t)N * HV;
    const int CK = 32;
    const size_t KV = (size_t)K * V;
    int bad = 0;

#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int64_t u = 0; u < units; ++u) {
        const int n = (int)(u / HV);
        const int h = (int)(u % HV);
        const int hq = h / group;
        int64_t b, t0, t1;
        seq_range(cu, n, T, &b, &t0, &t1);
        if (t0 < 0 || t1 < t0 || t1 > T) { bad |= 1; continue; }
        const int64_t len = t1 - t0, nblk = (len + CK - 1) / CK;
        /* ckpt[m] = state before token t0 + m*CK; blk[j] = state after token j of the current block */
        double *ckpt = (double *)malloc(sizeof(double) * KV * (size_t)(nblk > 0 ? nblk : 1));
        double *blk = (double *)malloc(sizeof(double) * KV * (size_t)(CK + 1));
        double *dS = (double *)malloc(sizeof(double) * KV);
        double *Sd = (double *)malloc(sizeof(double) * KV);
        double *r = (double *)malloc(sizeof(double) * V);
        double *dr = (double *)malloc(sizeof(double) * V);
        if (!ckpt || !blk || !dS || !Sd || !r || !dr) {
            free(ckpt); free(blk); free(dS); free(Sd); free(r); free(dr);
            bad |= 1;
            continue;
        }
        double *S = blk; /* running state during the checkpoint pass */
        if (s0) memcpy(S, s0 + u * (int64_t)KV, sizeof(double) * KV);
        else memset(S, 0, sizeof(double) * KV);

        /* one token forward: S_in -> S_out (may alias); fills Sd = S' and r */
#define KDA_STEP(t, S_in, S_out)                                                                   \
    do {                                                                                           \
        const int64_t row_ = b * T + (t);                                                          \
        const double *kt_ = k + (row_ * H + hq) * K;                                               \
        const double *vt_ = v + (row_ * HV + h) * V;                                               \
        const double *gt_ = g + (row_ * HV + h) * K;                                               \
        const double bt_ = beta[row_ * HV + h];                                                    \
        for (int d = 0; d < K; ++d) {                                                              \
            const double e_ = exp(gt_[d]);                                                         \
            for (int c = 0; c < V; ++c) Sd[(int64_t)d * V + c] = (S_in)[(int64_t)d * V + c] * e_; \
        }                                                                                          \
        for (int c = 0; c < V; ++c) {                                                              \
            double acc_ = 0.0;                                                                     \
            for (int d = 0; d < K; ++d) acc_ += kt_[d] * Sd[(int64_t)d * V + c];                   \
            r[c] = vt_[c] - acc_;                                                                  \
        }                                                                                          \
        for (int d = 0; d < K; ++d) {                                                              \
            const double bk_ = bt_ * kt_[d];                                                       \
            for (int c = 0; c < V; ++c) (S_out)[(int64_t)d * V + c] = Sd[(int64_t)d * V + c] + bk_ * r[c]; \
        }                                                                                          \
    } while (0)

        for (int64_t m = 0; m < nblk; ++m) {
            memcpy(ckpt + (size_t)m * KV, S, sizeof(double) * KV);
            const int64_t te = t0 + (m + 1) * CK < t1 ? t0 + (m + 1) * CK : t1;
            for (int64_t t = t0 + m * CK; t < te; ++t) KDA_STEP(t, S, S);
        }
        /* S now holds the final state: the gradient arriving there is dht */
        if (dht) memcpy(dS, dht + u * (int64_t)KV, sizeof(double) * KV);
        else memset(dS, 0, sizeof(double) * KV);

        for (int64_t m = nblk - 1; m >= 0; --m) {
            const int64_t tb = t0 + m * CK;
            const int64_t te = tb + CK < t1 ? tb + CK : t1;
            const int cnt = (int)(te - tb);
            memcpy(blk, ckpt + (size_t)m * KV, sizeof(double) * KV);
            for (int j = 0; j < cnt; ++j) KDA_STEP(tb + j, blk + (size_t)j * KV, blk + (size_t)(j + 1) * KV);
            for (int j = cnt - 1; j >= 0; --j) {
                const int64_t t = tb + j;
                const int64_t row = b * T + t;
                const double *qt = q + (row * H + hq) * K;
                const double *kt = k + (row * H + hq) * K;
                const double *gt = g + (row * HV + h) * K;
                const double bt = beta[row * HV + h];
                const double *dot = do_ + (row * HV + h) * V;
                const double *Sp = blk + (size_t)j * KV, *St = blk + (size_t)(j + 1) * KV;
                double *dqt = dq + (row * HV + h) * K, *dkt = dk + (row * HV + h) * K;
                double *dvt = dv + (row * HV + h) * V, *dgt = dg + (row * HV + h) * K;
                /* S' and r of this token again (from S_{t-1}) */
                for (int d = 0; d < K; ++d) {
                    const double e = exp(gt[d]);
                    for (int c = 0; c < V; ++c) Sd[(int64_t)d * V + c] = Sp[(int64_t)d * V + c] * e;
                }
                const double *vt = v + (row * HV + h) * V;
                for (int c = 0; c < V; ++c) {
                    double acc = 0.0;
                    for (int d = 0; d < K; ++d) acc += kt[d] * Sd[(int64_t)d * V + c];
                    r[c] = vt[c] - acc;
                }
                /* output: dq_t = K^-0.5 S_t do_t, dS += K^-0.5 q_t do_t^T */
                for (int d = 0; d < K; ++d) {
                    double acc = 0.0;
                    for (int c = 0; c < V; ++c) acc += St[(int64_t)d * V + c] * dot[c];
                    dqt[d] = scale * acc;
                    const double sq = scale * qt[d];
                    for (int c = 0; c < V; ++c) dS[(int64_t)d * V + c] += sq * dot[c];
                }
                /* dr = beta dS^T k, dbeta = k^T dS r */
                double db = 0.0;
                for (int c = 0; c < V; ++c) {
                    double acc = 0.0;
                    for (int d = 0; d < K; ++d) acc += kt[d] * dS[(int64_t)d * V + c];
                    dr[c] = bt * acc;
                    db += acc * r[c];
                }
                dbeta[row * HV + h] = db;
                /* dk = beta dS r - S' dr; dv = dr */
                for (int d = 0; d < K; ++d) {
                    double a1 = 0.0, a2 = 0.0;
                    for (int c = 0; c < V; ++c) {
                        a1 += dS[(int64_t)d * V + c] * r[c];
                        a2 += Sd[(int64_t)d * V + c] * dr[c];
                    }
                    dkt[d] = bt * a1 - a2;
                }
                for (int c = 0; c < V; ++c) dvt[c] = dr[c];
                /* dS' = dS - k dr^T; dg = rowsum(S' * dS'); dS_{t-1} = diag(exp g) dS' */
                for (int d = 0; d < K; ++d) {
                    const double e = exp(gt[d]);
                    double acc = 0.0;
                    for (int c = 0; c < V; ++c) {
                        const double x = dS[(int64_t)d * V + c] - kt[d] * dr[c];
                        acc += Sd[(int64_t)d * V + c] * x;
                        dS[(int64_t)d * V + c] = e * x;
                    }
                    dgt[d] = acc;
                }
            }
        }
#undef KDA_STEP
        if (ds0) memcpy(ds0 + u * (int64_t)KV, dS, sizeof(double) * KV);
        free(ckpt); free(blk); free(dS); free(Sd); free(r); free(dr);
    }
    return bad ? -1 : 0;
}

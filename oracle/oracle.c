/*
 * Reference oracle for the activation-sparsified linear layer y = prune(x) W^T.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file; only the tests, the smoke check and the benchmark's CPU
 * baseline leg use it.  It shares no code with the CUDA library.
 *
 * Plain, slow, obviously correct: every quantity is computed from its
 * definition, statistics and contractions in float64, with no blocking,
 * fusion or reordering.  The only float32 arithmetic is the channel score,
 * because the selection decision is taken in float32 on both sides (one
 * float32 subtraction for the mean shift, one float32 multiply for the
 * score).  Build with -ffp-contract=off and without fast-math.
 *
 * Sources (page title, section):
 *   [OVW]  "激活稀疏化技术：提升LLM推理效率的动态剪枝方法"
 *          (activation-sparsity overview): section 2.1 N:M patterns,
 *          2.2.1 magnitude pruning, 2.2.3 CLACT score, 3.1 D-PTS,
 *          3.2 VAR variance correction, 2.2.2 Amber-Pruner channel importance,
 *          3.3 R-Sparse low-rank compensation.
 *   [WIS]  "大模型推理优化：WiSparse激活稀疏化技术解析": section 2.1, eq. (4),
 *          weight-aware score s_i = |x_i| * ||W[:,i]||_2^alpha; section 2.2
 *          per-layer keep fraction (top-k).
 *   [SQR]  "利用2:4稀疏性与Squared-ReLU加速Transformer训练与推理": section 2.1
 *          2:4 pattern, 2.3 dropping the smallest of a 3-nonzero block,
 *          3.3 compressed layout with the kept values stored contiguously,
 *          3.2-3.3 sparse/dense feature split and the sparsity-driven mode,
 *          3.1 fused Squared-ReLU + 2:4 + FP8 producer and the FP8
 *          row-scaled 2:4 GEMM, 5.3 sparsify before quantising.
 *
 * Readings where the pages are silent or disagree (all listed in the design
 * notes): exactly N per M-block (or exactly k per token), equal float32
 * scores broken towards the lower channel index; blocks are [jM, jM+M);
 * the weight norm runs over the output rows of input column i; the CLACT
 * row factor is constant within a token and so the ranking uses |x_ij| * c_j;
 * D-PTS adds eta back to every channel, i.e. y = (xhat*m) W^T + eta*rowsum(W);
 * VAR: unbiased variances, running variance initialised to the first batch's
 * dense variance and updated with momentum before the scale is formed, scale
 * = sqrt(running / (Var[x*m] + eps)), applied to the whole output row.
 * Amber-Pruner: a percentile is the order statistic of ascending rank
 * floor(q (N-1)) of all N weights; weights outside [lo, hi] (inclusive ends)
 * are dropped and contribute nothing; z uses the population mean and standard
 * deviation of the kept weights; the exponent alpha of [WIS] eq. (4) also
 * applies (alpha = 1 gives the plain norm).
 * FP8 ([SQR] 3.1 names FP8 and row scaling but no format or scale rule):
 * E4M3 with round-to-nearest-even and saturation at 448; one float32 scale
 * per row (token row of the activation, output row of the weight),
 * scale = fl32(amax / 448) over the row's kept values, and the codes are
 * E4M3(fl32(v * inv)) with the reciprocal scale inv = fl32(448 / amax)
 * (scale = inv = 1 for an all-zero row); the activation is sparsified first ([SQR]
 * 5.3), so its amax runs over the kept values only.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

void or_select_nm(const float *s, int T, int k, int n, int m, uint8_t *mask);

/* ---------------------------------------------------------------------------
 * Weight preparation.  [WIS] section 2.1, eq. (4): g_i = (||W[:,i]||_2)^alpha,
 * the norm taken over the n_out output rows of input column i; precomputed
 * once per layer.  [OVW] section 3.1: rowsum_o = sum_i W[o,i], the term that
 * restores the shifted-out mean (y = (x_sparse + eta) W^T).
 * W is [n_out, k] row-major (PyTorch Linear layout).
 * ------------------------------------------------------------------------- */
void or_weight_prep(const float *W, int n_out, int k, double alpha,
                    double *g, double *rowsum)
{
    if (g) {
        #pragma omp parallel for schedule(static)
        for (int i = 0; i < k; i++) {
            double ss = 0.0;
            for (int o = 0; o < n_out; o++) {
                double w = (double)W[(size_t)o * k + i];
                ss += w * w;
            }
            g[i] = pow(sqrt(ss), alpha);
        }
    }
    if (rowsum) {
        #pragma omp parallel for schedule(static)
        for (int o = 0; o < n_out; o++) {
            double s = 0.0;
            for (int i = 0; i < k; i++) s += (double)W[(size_t)o * k + i];
            rowsum[o] = s;
        }
    }
}

/* ---------------------------------------------------------------------------
 * FP8 E4M3 (the OCP 8-bit float, "fn" variant): sign, 4 exponent bits with
 * bias 7, 3 mantissa bits; no infinities; exponent field 15 with mantissa 7
 * is NaN, so the largest finite value is 1.75 * 2^8 = 448; subnormals are
 * m * 2^-9, m = 1..7.  Encoding rounds to the nearest representable value,
 * ties to an even mantissa, and clamps finite magnitudes above 448 to 448.
 * ------------------------------------------------------------------------- */
uint8_t or_e4m3_encode(double v)
{
    if (isnan(v)) return 0x7F;
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    double a = fabs(v);
    if (a >= 448.0) return sign | 0x7E;
    if (a < ldexp(1.0, -6)) {                    /* subnormal range: step 2^-9 */
        double m = nearbyint(a / ldexp(1.0, -9)); /* ties to even */
        return sign | (uint8_t)m;                /* m == 8 is 2^-6: field 1, mantissa 0 */
    }
    int E;
    frexp(a, &E);                                /* a = f 2^E, f in [0.5, 1) */
    int e = E - 1;                               /* 2^e <= a < 2^(e+1) */
    double m = nearbyint(a / ldexp(1.0, e - 3)); /* 8 <= m <= 16 */
    if (m == 16.0) { m = 8.0; e += 1; }
    return sign | (uint8_t)((e + 7) << 3) | (uint8_t)(m - 8.0);
}

double or_e4m3_decode(uint8_t c)
{
    int ef = (c >> 3) & 15, mf = c & 7;
    double s = (c & 0x80) ? -1.0 : 1.0;
    if (ef == 15 && mf == 7) return NAN;
    if (ef == 0) return s * ldexp((double)mf, -9);
    return s * ldexp((double)(8 + mf), ef - 10);
}

/* One row of float32 values to E4M3 codes with its float32 scale. */
static float quant_row(const float *v, const uint8_t *keep, int n, uint8_t *codes)
{
    float amax = 0.0f;
    for (int i = 0; i < n; i++)
        if (!keep || keep[i]) {
            float a = fabsf(v[i]);
            if (a > amax) amax = a;
        }
    float scale = amax > 0.0f ? amax / 448.0f : 1.0f;
    float inv = amax > 0.0f ? 448.0f / amax : 1.0f;
    for (int i = 0; i < n; i++) {
        float q = v[i] * inv;
        codes[i] = (!keep || keep[i]) ? or_e4m3_encode((double)q) : 0;
    }
    return scale;
}

/* Weight side of the FP8 GEMM: W [n_out, k] float32 -> codes [n_out, k] and
 * one scale per output row. */
void or_quant_rows_fp8(const float *W, int n_out, int k, uint8_t *codes, float *scale)
{
    for (int o = 0; o < n_out; o++)
        scale[o] = quant_row(W + (size_t)o * k, NULL, k, codes + (size_t)o * k);
}

/* [SQR] 3.1 fused producer for one layer input, from the pre-activation z
 * (bfloat16 bit patterns, [T, k]):
 *   x = r * r with r = max(0, z) in float32 (one rounding),
 *   2:4 selection on |x| = x (exactly two per block of four, ties to the
 *   lower index), then the kept values to E4M3 with the row scale.
 * Outputs: mask [T, k], codes of the kept values [T, k/2] in channel order,
 * their positions in the block [T, k/2], scale [T], and x itself [T, k]. */
void or_sqrelu24_fp8(const uint16_t *z, int T, int k, uint8_t *mask, uint8_t *codes,
                     uint8_t *pos, float *scale, float *x)
{
    size_t kc = (size_t)k / 2;
    for (int t = 0; t < T; t++) {
        float *xt = x + (size_t)t * k;
        for (int i = 0; i < k; i++) {
            uint32_t bits = (uint32_t)z[(size_t)t * k + i] << 16;
            float zf;
            memcpy(&zf, &bits, 4);
            float r = zf > 0.0f ? zf : 0.0f;
            xt[i] = r * r;
        }
    }
    or_select_nm(x, T, k, 2, 4, mask);
    uint8_t *row_codes = (uint8_t *)malloc((size_t)k);
    for (int t = 0; t < T; t++) {
        const float *xt = x + (size_t)t * k;
        const uint8_t *mt = mask + (size_t)t * k;
        scale[t] = quant_row(xt, mt, k, row_codes);
        size_t w = 0;
        for (int b = 0; b < k; b += 4)
            for (int i = b; i < b + 4; i++)
                if (mt[i]) {
                    codes[(size_t)t * kc + w] = row_codes[i];
                    pos[(size_t)t * kc + w] = (uint8_t)(i - b);
                    w++;
                }
    }
    free(row_codes);
}

/* ---------------------------------------------------------------------------
 * Amber-Pruner channel importance.  [OVW] section 2.2.2: remove the weights
 * beyond the lo/hi percentiles (0.5 and 99.5 on the page), z-score the rest,
 * and score each input channel by the l2 norm of its standardised weights:
 *   v_lo, v_hi  = sorted(W)[floor(q (N-1))], q = lo_pct/100, hi_pct/100
 *   kept        = { W[o,i] : v_lo <= W[o,i] <= v_hi }
 *   mu, sigma   = mean and population standard deviation of the kept weights
 *   z[o,i]      = (W[o,i] - mu) / sigma for kept weights, 0 for dropped ones
 *   g_i         = (sqrt(sum_o z[o,i]^2))^alpha
 * sigma == 0 (all kept weights equal) gives z = 0 everywhere.
 * ------------------------------------------------------------------------- */
static int cmp_float(const void *a, const void *b)
{
    float x = *(const float *)a, y = *(const float *)b;
    return (x > y) - (x < y);
}

void or_amber(const float *W, int n_out, int k, double alpha, double lo_pct, double hi_pct,
              double *g, double *v_lo_out, double *v_hi_out)
{
    size_t N = (size_t)n_out * k;
    float *sorted = (float *)malloc(N * sizeof(float));
    memcpy(sorted, W, N * sizeof(float));
    qsort(sorted, N, sizeof(float), cmp_float);
    float v_lo = sorted[(size_t)floor(lo_pct / 100.0 * (double)(N - 1))];
    float v_hi = sorted[(size_t)floor(hi_pct / 100.0 * (double)(N - 1))];
    free(sorted);

    double count = 0.0, sum = 0.0;
    for (size_t j = 0; j < N; j++)
        if (W[j] >= v_lo && W[j] <= v_hi) {
            count += 1.0;
            sum += (double)W[j];
        }
    double mu = count > 0.0 ? sum / count : 0.0;
    double ss = 0.0;
    for (size_t j = 0; j < N; j++)
        if (W[j] >= v_lo && W[j] <= v_hi) ss += ((double)W[j] - mu) * ((double)W[j] - mu);
    double sigma = count > 0.0 ? sqrt(ss / count) : 0.0;

    for (int i = 0; i < k; i++) {
        double zz = 0.0;
        for (int o = 0; o < n_out; o++) {
            float w = W[(size_t)o * k + i];
            if (w >= v_lo && w <= v_hi && sigma > 0.0) {
                double z = ((double)w - mu) / sigma;
                zz += z * z;
            }
        }
        g[i] = pow(sqrt(zz), alpha);
    }
    if (v_lo_out) *v_lo_out = (double)v_lo;
    if (v_hi_out) *v_hi_out = (double)v_hi;
}

/* [OVW] section 3.1: eta_t = mean over the channels of token t. */
void or_token_mean(const float *x, int T, int k, double *eta)
{
    for (int t = 0; t < T; t++) {
        double s = 0.0;
        for (int i = 0; i < k; i++) s += (double)x[(size_t)t * k + i];
        eta[t] = s / (double)k;
    }
}

/* Unbiased variance of each token's k channels (two-pass, float64). */
void or_token_var(const float *x, int T, int k, double *var)
{
    for (int t = 0; t < T; t++) {
        double mean = 0.0;
        for (int i = 0; i < k; i++) mean += (double)x[(size_t)t * k + i];
        mean /= (double)k;
        double ss = 0.0;
        for (int i = 0; i < k; i++) {
            double d = (double)x[(size_t)t * k + i] - mean;
            ss += d * d;
        }
        var[t] = ss / (double)(k - 1);
    }
}

/* [OVW] section 2.2.3: column energy c_j = sqrt(sum_p x_pj^2) over the T
 * tokens of the call. */
void or_channel_energy(const float *x, int T, int k, double *c)
{
    for (int j = 0; j < k; j++) {
        double s = 0.0;
        for (int p = 0; p < T; p++) {
            double v = (double)x[(size_t)p * k + j];
            s += v * v;
        }
        c[j] = sqrt(s);
    }
}

/* [OVW] section 2.2.3, full CLACT score in float64:
 * S_ij = |x_ij| / sqrt(sum_k x_ik^2) * sqrt(sum_p x_pj^2). */
void or_clact_full(const float *x, int T, int k, double *S)
{
    double *c = (double *)malloc(sizeof(double) * (size_t)k);
    or_channel_energy(x, T, k, c);
    for (int t = 0; t < T; t++) {
        double r = 0.0;
        for (int i = 0; i < k; i++) {
            double v = (double)x[(size_t)t * k + i];
            r += v * v;
        }
        r = sqrt(r);
        for (int j = 0; j < k; j++)
            S[(size_t)t * k + j] = fabs((double)x[(size_t)t * k + j]) / r * c[j];
    }
    free(c);
}

/* ---------------------------------------------------------------------------
 * Channel score in float32, the precision the selection decision is taken in.
 *   xhat = fl32(x - eta_t)         when eta is given (D-PTS, [OVW] 3.1),
 *          x                        otherwise;
 *   s    = fl32(|xhat| * f_i)       f = g ([WIS] eq. 4), c (CLACT, [OVW]
 *                                   2.2.3, row factor dropped), or 1 when
 *                                   f is NULL (magnitude, [OVW] 2.2.1).
 * ------------------------------------------------------------------------- */
void or_score(const float *x, int T, int k, const float *eta, const float *f,
              float *s)
{
    for (int t = 0; t < T; t++) {
        for (int i = 0; i < k; i++) {
            float xh = x[(size_t)t * k + i];
            if (eta) xh = xh - eta[t];
            float a = fabsf(xh);
            s[(size_t)t * k + i] = f ? a * f[i] : a;
        }
    }
}

/* Strict ranking order: higher score first, equal scores by lower index. */
static int ahead(float sj, int j, float si, int i)
{
    return (sj > si) || (sj == si && j < i);
}

/* [OVW] section 2.1 / 2.2.1: in every block of m consecutive channels
 * [jm, jm+m) keep the n with the largest score (exactly n; ties to the lower
 * index).  mask is [T, k] of 0/1. */
void or_select_nm(const float *s, int T, int k, int n, int m, uint8_t *mask)
{
    #pragma omp parallel for schedule(static)
    for (int t = 0; t < T; t++) {
        const float *st = s + (size_t)t * k;
        for (int b = 0; b < k; b += m) {
            for (int i = b; i < b + m; i++) {
                int rank = 0;
                for (int j = b; j < b + m; j++)
                    if (j != i && ahead(st[j], j, st[i], i)) rank++;
                mask[(size_t)t * k + i] = (uint8_t)(rank < n);
            }
        }
    }
}

/* Threshold selection (WiSparse page section 3.1 builds on TEAL's sparse
 * operator; section 5 tunes its threshold tau): keep every channel whose
 * score is above tau. */
void or_select_thresh(const float *s, int T, int k, float tau, uint8_t *mask)
{
    #pragma omp parallel for schedule(static)
    for (int t = 0; t < T; t++)
        for (int i = 0; i < k; i++) mask[(size_t)t * k + i] = (uint8_t)(s[(size_t)t * k + i] > tau);
}

typedef struct { float s; int i; } keyed;

static int cmp_keyed(const void *a, const void *b)
{
    const keyed *p = (const keyed *)a, *q = (const keyed *)b;
    if (p->s > q->s) return -1;
    if (p->s < q->s) return 1;
    return (p->i < q->i) ? -1 : (p->i > q->i);
}

/* [WIS] section 2.2: per-layer keep fraction, i.e. keep the kk channels of
 * largest score per token (exactly kk; ties to the lower index). */
void or_select_topk(const float *s, int T, int k, int kk, uint8_t *mask)
{
    #pragma omp parallel for schedule(static)
    for (int t = 0; t < T; t++) {
        keyed *v = (keyed *)malloc(sizeof(keyed) * (size_t)k);
        for (int i = 0; i < k; i++) { v[i].s = s[(size_t)t * k + i]; v[i].i = i; }
        qsort(v, (size_t)k, sizeof(keyed), cmp_keyed);
        memset(mask + (size_t)t * k, 0, (size_t)k);
        for (int r = 0; r < kk; r++) mask[(size_t)t * k + v[r].i] = 1;
        free(v);
    }
}

/* ---------------------------------------------------------------------------
 * [OVW] section 3.2, variance correction:
 *   var_dense_t = Var[x_t]            (unbiased)
 *   var_kept_t  = Var[x_t * m_t]      (zeros included, unbiased)
 *   running_t   = var_dense_t                         on the first batch,
 *                 mom*running_in_t + (1-mom)*var_dense_t  afterwards
 *   nu_t        = sqrt(running_t / (var_kept_t + eps))
 * ------------------------------------------------------------------------- */
void or_var_scale(const float *x, const uint8_t *mask, int T, int k,
                  const double *running_in, double momentum, double eps,
                  double *var_dense, double *var_kept, double *running_out,
                  double *nu)
{
    #pragma omp parallel for schedule(static)
    for (int t = 0; t < T; t++) {
        double *xm = (double *)malloc(sizeof(double) * (size_t)k);
        double mean = 0.0, mk = 0.0;
        for (int i = 0; i < k; i++) {
            double v = (double)x[(size_t)t * k + i];
            xm[i] = mask[(size_t)t * k + i] ? v : 0.0;
            mean += v;
            mk += xm[i];
        }
        mean /= (double)k;
        mk /= (double)k;
        double sd = 0.0, sk = 0.0;
        for (int i = 0; i < k; i++) {
            double d = (double)x[(size_t)t * k + i] - mean;
            double e = xm[i] - mk;
            sd += d * d;
            sk += e * e;
        }
        double vd = sd / (double)(k - 1), vk = sk / (double)(k - 1);
        double run = running_in ? momentum * running_in[t] + (1.0 - momentum) * vd : vd;
        if (var_dense) var_dense[t] = vd;
        if (var_kept) var_kept[t] = vk;
        if (running_out) running_out[t] = run;
        if (nu) nu[t] = sqrt(run / (vk + eps));
        free(xm);
    }
}

/* ---------------------------------------------------------------------------
 * Contraction over the kept channels, float64:
 *   y[r,o] = nu_t * ( sum_i xhat_ti * m_ti * W[o,i]  +  eta_t * rowsum_o )
 * with t = rows[r] (all tokens when rows is NULL), xhat = x - eta when eta is
 * given (D-PTS, [OVW] 3.1: y = (x_sparse + eta) W^T, the eta added back to
 * every channel) else x, the rowsum term only with eta, and nu only when
 * given (VAR, [OVW] 3.2: y = scale * (x_sparse W^T)).
 * ------------------------------------------------------------------------- */
void or_linear(const float *x, const uint8_t *mask, int T, int k,
               const double *eta, const float *W, int n_out,
               const double *rowsum, const double *nu, const int *rows,
               int n_rows, double *y)
{
    (void)T;
    #pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < n_rows; r++) {
        double *xv = (double *)malloc(sizeof(double) * (size_t)k);
        int t = rows ? rows[r] : r;
        for (int i = 0; i < k; i++) {
            double v = (double)x[(size_t)t * k + i];
            if (eta) v -= eta[t];
            xv[i] = mask[(size_t)t * k + i] ? v : 0.0;
        }
        for (int o = 0; o < n_out; o++) {
            const float *wr = W + (size_t)o * k;
            double acc = 0.0;
            for (int i = 0; i < k; i++) acc += xv[i] * (double)wr[i];
            if (eta) acc += eta[t] * rowsum[o];
            if (nu) acc *= nu[t];
            y[(size_t)r * n_out + o] = acc;
        }
        free(xv);
    }
}

/* ---------------------------------------------------------------------------
 * R-Sparse low-rank compensation ([OVW] section 3.3): W ~ W_sparse + A_r B_r^T
 * with A_r = U_r diag(S_r) [n_out, r] and B_r = V_r [k, r] from a truncated
 * SVD of W.  Reading: the kept channels go through W itself and the dropped
 * ones through the rank-r factors, so the layer adds
 *   comp[t,o] = sum_j ( sum_i xhat_ti (1 - m_ti) B[i,j] ) A[o,j]
 * to y (xhat = x - eta with D-PTS, else x).  Computed in float64 in the
 * order written: first u = xhat_dropped B_r, then u A_r^T.
 * ------------------------------------------------------------------------- */
void or_rsparse(const float *x, const uint8_t *mask, int T, int k, const double *eta,
                const float *B, const float *A, int n_out, int r, double *comp)
{
    double *u = (double *)malloc(sizeof(double) * (size_t)(r > 0 ? r : 1));
    for (int t = 0; t < T; t++) {
        for (int j = 0; j < r; j++) u[j] = 0.0;
        for (int i = 0; i < k; i++) {
            if (mask[(size_t)t * k + i]) continue;
            double v = (double)x[(size_t)t * k + i];
            if (eta) v -= eta[t];
            for (int j = 0; j < r; j++) u[j] += v * (double)B[(size_t)i * r + j];
        }
        for (int o = 0; o < n_out; o++) {
            double acc = 0.0;
            for (int j = 0; j < r; j++) acc += u[j] * (double)A[(size_t)o * r + j];
            comp[(size_t)t * n_out + o] = acc;
        }
    }
    free(u);
}

/* ---------------------------------------------------------------------------
 * Hybrid 2:4 for inference ([SQR] sections 3.2 and 3.3): the layer's measured
 * sparsity picks the mode (above 95 %: pure 2:4; 90-95 %: split; below
 * 90 %: dense), and the split computes the densest features densely and
 * the rest with 2:4.  Readings: features are taken in 4-channel blocks so
 * the 2:4 part stays block-aligned; the dense set is the n_dense blocks
 * with the most nonzeros over the T tokens (ties to the lower block index);
 * the result is the masked product with mask = 1 on the dense blocks and
 * the 2:4 magnitude selection elsewhere.
 * nnz[b] = number of nonzero x[t, 4b..4b+3] over all t; total returned.
 * ------------------------------------------------------------------------- */
long long or_block_nnz(const float *x, int T, int k, int *nnz)
{
    long long total = 0;
    for (int b = 0; b < k / 4; b++) nnz[b] = 0;
    for (int t = 0; t < T; t++)
        for (int i = 0; i < k; i++)
            if (x[(size_t)t * k + i] != 0.0f) {
                nnz[i / 4]++;
                total++;
            }
    return total;
}

/* The n_dense blocks ranked first by (more nonzeros, then lower index),
 * returned in ascending block order. */
void or_pick_dense(const int *nnz, int nblocks, int n_dense, int *idx)
{
    uint8_t *taken = (uint8_t *)calloc((size_t)nblocks, 1);
    for (int b = 0; b < nblocks; b++) {
        int rank = 0;
        for (int c = 0; c < nblocks; c++)
            if (nnz[c] > nnz[b] || (nnz[c] == nnz[b] && c < b)) rank++;
        taken[b] = (uint8_t)(rank < n_dense);
    }
    int w = 0;
    for (int b = 0; b < nblocks; b++)
        if (taken[b]) idx[w++] = b;
    free(taken);
}

/* [SQR] section 3.3: compressed N:M layout, the kept values of every block
 * stored contiguously in ascending channel order, with their positions
 * inside the block.  values/pos are [T, k/m*n].  The mask must hold exactly n
 * per block. */
void or_compress_nm(const float *v, const uint8_t *mask, int T, int k, int n,
                    int m, float *values, uint8_t *pos)
{
    size_t kc = (size_t)k / (size_t)m * (size_t)n;
    for (int t = 0; t < T; t++) {
        size_t w = 0;
        for (int b = 0; b < k; b += m)
            for (int i = b; i < b + m; i++)
                if (mask[(size_t)t * k + i]) {
                    values[(size_t)t * kc + w] = v[(size_t)t * k + i];
                    pos[(size_t)t * kc + w] = (uint8_t)(i - b);
                    w++;
                }
    }
}

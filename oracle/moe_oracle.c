/*
 * moe_oracle.c -- plain fp64 CPU reference of the quantized MoE expert block.
 *
 * TEST INFRASTRUCTURE. Only the tests, the smoke check and the benchmark's CPU-baseline leg
 * load this file's library. It shares no code with the CUDA library (no headers, helpers or
 * tables) and is written to be checked by eye, not to be fast: every weight is unpacked bit
 * by bit and dequantised on the fly, every dot product is a sequential fp64 loop.
 *
 * What it computes (for each token t of x [T x H]):
 *   1. router logits     l_e = sum_h x_h * W_r[e,h] (+ bias_e)            (fp64)
 *   2. top-k             the k experts ordered by (l desc, expert index asc)
 *   3. renormalisation   w_i = exp(l_i - l_max) / sum_{j in top-k} exp(l_j - l_max)
 *   4. dequantisation    W[r,c] = (q[r,c] - z[r,c/64]) * s[r,c/64]  (q: b-bit integer code,
 *                        s, z: fp16 scale and zero of the 64-wide group along the input dim)
 *   5. expert FFN        g = Wg x, u = Wu x, h_r = g_r / (1 + exp(-g_r)) * u_r, y = Wd h
 *   6. combine           out = sum_i w_i y_{e_i}
 * This follows the method as stated for the MoE expert block on the pages "Krasis update"
 * (4/6/8-bit HQQ-style affine group quantisation), "--moe-direct-io" and "Qwen-tin"
 * (512 experts, top-10 routing) and "Raon-1-mini ... RTX 5070 Ti" (table, row "MoE
 * megakernel": one kernel for the whole expert block of a layer). The pages print no formula
 * for the block; steps 1-6 are the plain reading of gate/up, SiLU-GLU, down and a
 * routing-weighted combine with softmax renormalisation over the selected experts.
 *
 * Canonical storage read here: x bf16 bits [T x H]; W_r fp32 [E x H]; per expert and matrix
 * m (0 gate [I x H], 1 up [I x H], 2 down [H x I]) codes as rows x (cols*b/8) bytes where group
 * g of a row is a block of 8*b bytes and code j of the group occupies bits [j*b, (j+1)*b) of
 * the block read as a little-endian bit string; scale and zero fp16 bits [rows x cols/64].
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_GROUP 64

typedef struct {
    const uint8_t *codes[3];
    const uint16_t *scale[3];
    const uint16_t *zero[3];
    int32_t bits;
} oracle_expert_t;

/* bf16 bit pattern -> double (exact) */
static double bf16_to_f64(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* IEEE binary16 bit pattern -> double (exact), written from the format's definition */
static double f16_to_f64(uint16_t h) {
    int sign = (h >> 15) & 1;
    int ex = (h >> 10) & 31;
    int man = h & 1023;
    double v;
    if (ex == 0)
        v = ldexp((double)man, -24);                  /* subnormal: man * 2^-24 */
    else if (ex == 31)
        v = man ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + man), ex - 25);     /* (1 + man/1024) * 2^(ex-15) */
    return sign ? -v : v;
}

/* code c of a row (canonical layout), assembled bit by bit */
static unsigned code_at(const uint8_t *row, int bits, int c) {
    const uint8_t *grp = row + (size_t)(c / ORACLE_GROUP) * 8 * bits;
    unsigned first = (unsigned)(c % ORACLE_GROUP) * (unsigned)bits;
    unsigned v = 0;
    for (int i = 0; i < bits; i++) {
        unsigned pos = first + (unsigned)i;
        v |= (unsigned)((grp[pos >> 3] >> (pos & 7)) & 1u) << i;
    }
    return v;
}

/* dequantised weight W_m[r,c] of one expert */
double oracle_weight(const oracle_expert_t *ex, int m, int rows, int cols, int r, int c) {
    (void)rows;
    int bits = ex->bits;
    const uint8_t *row = ex->codes[m] + (size_t)r * ((size_t)cols * bits / 8);
    double q = (double)code_at(row, bits, c);
    size_t gi = (size_t)r * (cols / ORACLE_GROUP) + (size_t)(c / ORACLE_GROUP);
    double s = f16_to_f64(ex->scale[m][gi]);
    double z = f16_to_f64(ex->zero[m][gi]);
    return (q - z) * s;
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

/* step 1: logits [T x E] */
void oracle_router_logits(const uint16_t *x, const float *wr, const float *bias,
                          int T, int H, int E, double *logits) {
#pragma omp parallel for collapse(2) schedule(static)
    for (int t = 0; t < T; t++) {
        for (int e = 0; e < E; e++) {
            double acc = 0.0;
            for (int h = 0; h < H; h++)
                acc += bf16_to_f64(x[(size_t)t * H + h]) * (double)wr[(size_t)e * H + h];
            if (bias) acc += (double)bias[e];
            logits[(size_t)t * E + e] = acc;
        }
    }
}

/* steps 2-3: top-k by repeated arg-max (ties -> lower index), then softmax over the k */
void oracle_topk(const double *logits, int T, int E, int k, int32_t *idx, double *w) {
    for (int t = 0; t < T; t++) {
        const double *l = logits + (size_t)t * E;
        int32_t *it = idx + (size_t)t * k;
        double *wt = w + (size_t)t * k;
        for (int i = 0; i < k; i++) {
            int best = -1;
            for (int e = 0; e < E; e++) {
                int taken = 0;
                for (int j = 0; j < i; j++)
                    if (it[j] == e) taken = 1;
                if (taken) continue;
                if (best < 0 || l[e] > l[best]) best = e;   /* strict '>' keeps the lower index */
            }
            it[i] = best;
        }
        double lmax = l[it[0]];
        double den = 0.0;
        for (int i = 0; i < k; i++) den += exp(l[it[i]] - lmax);
        for (int i = 0; i < k; i++) wt[i] = exp(l[it[i]] - lmax) / den;
    }
}

/* step 5 for one token and one expert; g, u, h (length I) may be NULL; y has length H */
void oracle_expert_ffn(const uint16_t *x_tok, const oracle_expert_t *ex, int H, int I,
                       double *g_out, double *u_out, double *h_out, double *y) {
    double *h = (double *)malloc(sizeof(double) * (size_t)I);
#pragma omp parallel for schedule(static)
    for (int r = 0; r < I; r++) {
        double g = 0.0, u = 0.0;
        for (int c = 0; c < H; c++) {
            double xv = bf16_to_f64(x_tok[c]);
            g += oracle_weight(ex, 0, I, H, r, c) * xv;
            u += oracle_weight(ex, 1, I, H, r, c) * xv;
        }
        double silu = g / (1.0 + exp(-g));
        h[r] = silu * u;
        if (g_out) g_out[r] = g;
        if (u_out) u_out[r] = u;
    }
    if (h_out) memcpy(h_out, h, sizeof(double) * (size_t)I);
#pragma omp parallel for schedule(static)
    for (int r = 0; r < H; r++) {
        double acc = 0.0;
        for (int c = 0; c < I; c++) acc += oracle_weight(ex, 2, H, I, r, c) * h[c];
        y[r] = acc;
    }
    free(h);
}

/* step 6 for given selections: out [T x H] = sum_i w[t,i] * y_{idx[t,i]}(x_t) */
void oracle_combine(const uint16_t *x, const oracle_expert_t *experts, int T, int H, int I,
                    int E, int k, const int32_t *idx, const double *w, double *out) {
    (void)E;
    double *y = (double *)malloc(sizeof(double) * (size_t)H);
    for (int t = 0; t < T; t++) {
        double *o = out + (size_t)t * H;
        for (int r = 0; r < H; r++) o[r] = 0.0;
        for (int i = 0; i < k; i++) {
            int e = idx[(size_t)t * k + i];
            oracle_expert_ffn(x + (size_t)t * H, &experts[e], H, I, NULL, NULL, NULL, y);
            double wi = w[(size_t)t * k + i];
            for (int r = 0; r < H; r++) o[r] += wi * y[r];
        }
    }
    free(y);
}

/* steps 1-6 */
void oracle_moe_forward(const uint16_t *x, const float *wr, const float *bias,
                        const oracle_expert_t *experts, int T, int H, int I, int E, int k,
                        double *out, int32_t *idx, double *w, double *logits) {
    double *l = logits ? logits : (double *)malloc(sizeof(double) * (size_t)T * E);
    oracle_router_logits(x, wr, bias, T, H, E, l);
    oracle_topk(l, T, E, k, idx, w);
    oracle_combine(x, experts, T, H, I, E, k, idx, w, out);
    if (!logits) free(l);
}

/* ============================================================================= quantiser
 *
 * HQQ-style group quantiser: bf16 weights -> the canonical (codes, fp16 scale, fp16 zero)
 * format read above. The page "Krasis update" (list of the v1.0 results, the item on 4/6/8-bit
 * sensitivity-aware HQQ) names Half-Quadratic Quantization at 4, 6 and 8 bits, built from the
 * weights alone with no calibration run, but prints no steps. The steps below restate the published method
 * (H. Badri and A. Shaji, "Half-Quadratic Quantization of Large Machine Learning Models",
 * 2023): the min-max scale of each group is kept, and only the zero point is optimised. It
 * minimises an l_p norm (p < 1) of the reconstruction error by half-quadratic splitting, which
 * alternates a closed-form shrinkage of the error with a closed-form least-squares zero.
 *
 * One group w_0..w_63 (fp64, exact from bf16), Q = 2^b - 1, all arithmetic in fp64:
 *   1. lo = min w, hi = max w; a constant group c is widened to [min(c, 0), max(c, 0)], and
 *      an all-zero group to [0, Q].
 *      s = fp16((hi - lo) / Q), at least the smallest positive fp16 and at most 65504;
 *      z_0 = -lo / s (s is the stored fp16 value from here on).
 *   2. For i = 0 .. iters-1, with beta_0 = beta and beta_{i+1} = kappa * beta_i:
 *        q_j = clamp(rint(w_j / s + z_i), 0, Q),   r_j = (q_j - z_i) * s
 *        err_i = sum_j |w_j - r_j|; if err_i is not below (1 - 2^-40) times the best so far,
 *               stop; otherwise z_i becomes the best zero
 *        e_j = shrink_p(w_j - r_j, beta_i)
 *        z_{i+1} = (1/64) * sum_j (q_j - (w_j - e_j) / s)
 *      with the generalised soft threshold
 *      shrink_p(x, beta) = sign(x) * max(|x| - |x|^(p-1) / beta, 0), and shrink_p(0) = 0.
 *      For p = 1 this is the proximal map of |x| / beta (the soft threshold).
 *   3. z = fp16(best zero), clamped to +-65504; q_j = clamp(rint(w_j / s + z), 0, Q) with the
 *      stored fp16 s and z. These are the nearest points of the stored grid.
 * The readings this takes where the published text leaves room: the stop rule and the best
 * zero are per group (the objective is a sum of independent group terms); the codes are
 * recomputed from the stored fp16 scale and zero; iters = 0 is plain min-max rounding; and
 * the stop test is the one exact arithmetic takes. Near its optimum the L1 error is flat in
 * the zero (the residual signs balance), so successive iterates often have equal error, and a
 * strict comparison of two rounded 64-term sums would decide those ties by rounding. A fall
 * counts only if it exceeds 2^-40 of the error; the rounding of such a sum, in any order, is
 * below 2^-46 of it.
 */

#define HQQ_FALL (1.0 - 0x1p-40)   /* an error must fall below HQQ_FALL * best to count */

/* double -> IEEE binary16 bits, round to nearest, ties to even (from the format's definition:
 * 11 significant bits for normal values, a fixed quantum of 2^-24 below 2^-14, and infinity
 * from 65520 = 65504 + half a unit in the last place up) */
uint16_t oracle_f64_to_f16(double v) {
    uint16_t sign = signbit(v) ? 0x8000 : 0;
    double a = fabs(v);
    if (isnan(v)) return 0x7E00;
    if (a >= 65520.0) return (uint16_t)(sign | 0x7C00);
    int e;
    (void)frexp(a, &e);                       /* a in [2^(e-1), 2^e) */
    int qe = e - 11;                          /* quantum of an 11-bit significand */
    if (qe < -24) qe = -24;                   /* subnormal spacing */
    double n = rint(ldexp(a, -qe));           /* exact power-of-two scaling, then RNE */
    double r = ldexp(n, qe);
    if (r == 0.0) return sign;
    if (r < ldexp(1.0, -14)) return (uint16_t)(sign | (uint16_t)n);
    int re;
    double m = frexp(r, &re);                 /* r = m * 2^re, m in [0.5, 1) */
    uint16_t ex = (uint16_t)(re - 1 + 15);
    uint16_t man = (uint16_t)((2.0 * m - 1.0) * 1024.0);
    return (uint16_t)(sign | (uint16_t)(ex << 10) | man);
}

double oracle_hqq_shrink(double x, double beta, double p) {
    if (x == 0.0) return 0.0;
    double a = fabs(x);
    double t = a - pow(a, p - 1.0) / beta;
    return t > 0.0 ? copysign(t, x) : 0.0;
}

static double hqq_code(double w, double s, double z, double qmax) {
    double q = rint(w / s + z);
    return fmin(fmax(q, 0.0), qmax);
}

/* One group of ORACLE_GROUP weights. Outputs the stored scale/zero bits and the codes; the
 * optional traces receive z_i and err_i of every iteration that ran (at most iters entries),
 * *n_iter how many ran. */
void oracle_hqq_group(const double *w, int bits, double p, double beta, double kappa,
                      int iters, uint16_t *s16, uint16_t *z16, uint8_t *q_out,
                      double *z_trace, double *err_trace, int *n_iter) {
    const int n = ORACLE_GROUP;
    double qmax = (double)((1 << bits) - 1);
    double lo = w[0], hi = w[0];
    for (int j = 1; j < n; j++) {
        if (w[j] < lo) lo = w[j];
        if (w[j] > hi) hi = w[j];
    }
    if (lo == hi) {
        if (lo == 0.0) {
            hi = qmax;
        } else {
            lo = fmin(lo, 0.0);
            hi = fmax(hi, 0.0);
        }
    }
    uint16_t sb = oracle_f64_to_f16(fmin((hi - lo) / qmax, 65504.0));
    if (sb == 0) sb = 1;
    double s = f16_to_f64(sb);
    double z = -lo / s;
    double zbest = z, best = INFINITY;
    double q[ORACLE_GROUP], r[ORACLE_GROUP];
    int ran = 0;
    for (int i = 0; i < iters; i++) {
        double err = 0.0;
        for (int j = 0; j < n; j++) {
            q[j] = hqq_code(w[j], s, z, qmax);
            r[j] = (q[j] - z) * s;
            err += fabs(w[j] - r[j]);
        }
        if (z_trace) z_trace[i] = z;
        if (err_trace) err_trace[i] = err;
        ran = i + 1;
        if (!(err < best * HQQ_FALL)) break;
        best = err;
        zbest = z;
        double acc = 0.0;
        for (int j = 0; j < n; j++) {
            double e = oracle_hqq_shrink(w[j] - r[j], beta, p);
            acc += q[j] - (w[j] - e) / s;
        }
        z = acc / (double)n;
        beta *= kappa;
    }
    uint16_t zb = oracle_f64_to_f16(fmin(fmax(zbest, -65504.0), 65504.0));
    double zs = f16_to_f64(zb);
    for (int j = 0; j < n; j++) q_out[j] = (uint8_t)hqq_code(w[j], s, zs, qmax);
    *s16 = sb;
    *z16 = zb;
    if (n_iter) *n_iter = ran;
}

/* A bf16 matrix [rows x cols] (cols a multiple of 64), one group per 64 columns of a row:
 * codes q [rows x cols] (one byte each, unpacked), scale and zero bits [rows x cols/64],
 * iterations run per group (nullable). */
void oracle_hqq_quantize(const uint16_t *w_bf16, int rows, int cols, int bits, double p,
                         double beta, double kappa, int iters, uint8_t *q, uint16_t *s16,
                         uint16_t *z16, int32_t *iters_used) {
    int gpr = cols / ORACLE_GROUP;
#pragma omp parallel for schedule(static)
    for (long g = 0; g < (long)rows * gpr; g++) {
        long r = g / gpr, c0 = (g % gpr) * ORACLE_GROUP;
        double w[ORACLE_GROUP];
        for (int j = 0; j < ORACLE_GROUP; j++) w[j] = bf16_to_f64(w_bf16[r * cols + c0 + j]);
        int ran = 0;
        oracle_hqq_group(w, bits, p, beta, kappa, iters, &s16[g], &z16[g], &q[r * cols + c0],
                         NULL, NULL, &ran);
        if (iters_used) iters_used[g] = ran;
    }
}

/* Step 3 alone: the nearest codes of bf16 weights for given fp16 scale and zero bits. */
void oracle_hqq_codes(const uint16_t *w_bf16, int rows, int cols, int bits,
                      const uint16_t *s16, const uint16_t *z16, uint8_t *q) {
    int gpr = cols / ORACLE_GROUP;
    double qmax = (double)((1 << bits) - 1);
    for (long r = 0; r < rows; r++)
        for (long c = 0; c < cols; c++) {
            long g = r * gpr + c / ORACLE_GROUP;
            q[r * cols + c] = (uint8_t)hqq_code(bf16_to_f64(w_bf16[r * cols + c]),
                                                f16_to_f64(s16[g]), f16_to_f64(z16[g]), qmax);
        }
}

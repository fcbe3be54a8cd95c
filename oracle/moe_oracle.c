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

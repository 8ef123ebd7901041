/*
 * bfmoe_oracle.c -- plain, slow fp64 CPU oracle of the ButterflyMoE expert
 * layer forward.
 *
 * TEST INFRASTRUCTURE, NOT THE PRODUCT.  Only the tests, the package's smoke
 * check and the CPU-baseline leg of the benchmark may load this library.  It
 * shares no code, header, table or constant with the CUDA path.
 *
 * What it computes, and where the method is defined:
 *
 *  - Expert i is the map  W_i = B(phi_i) . W_base . B(theta_i)^T  with one
 *    shared ternary matrix W_base (entries in {-1,0,+1}) and orthogonal
 *    butterfly matrices B(.) made of layers of Givens rotations, O(d log d)
 *    angles each.  Source: "ButterflyMoE: Sub-Linear Ternary Experts via
 *    Structured Butterfly Orbits" summaries (gist.science, paper 2601.13563),
 *    section 2 "Methodology" / 2.1 "Mathematical formulation" / 2.2 "Key
 *    components" (layered Givens rotations).  The ButterflyViT summary
 *    (paper 2603.06746), section 2, restates the same factorisation.
 *  - Inference never materialises W_i: input rotation, then ternary product,
 *    then output rotation, in sequence (same pages, section 2 / 2.1).
 *  - A standard top-k gate picks the active experts (ButterflyMoE summary,
 *    Dutch page, section 2 "Three phases", gated routing).
 *  - A scale alpha multiplies the ternary product; the pages have none, the
 *    library's packed-base format carries one (reading A2 of the design).
 *
 * Conventions fixed by the library (the pages leave them open):
 *  - Butterfly stage s (0 <= s < L = log2 d) rotates the pairs (j, j + 2^s)
 *    for every j whose bit s is clear.  The pair's angle is angles[s][p] with
 *    p = (j >> (s+1)) * 2^s + (j & (2^s - 1)), a row-major [L][d/2] table.
 *    The rotation is  y_j = c x_j - s x_{j+h},  y_{j+h} = s x_j + c x_{j+h}
 *    with h = 2^s, c = cos(angle), s = sin(angle).
 *  - B = stage_{L-1} ... stage_0 (stage 0 acts first).  B^T applies the
 *    stages from L-1 down to 0 with negated angles.
 *  - Top-k order is (larger logit first, then lower expert index); -0 and +0
 *    tie; +-inf are ordinary values; any NaN logit is an error.
 *  - Gate g_j = softmax over the k selected logits (its limit when a
 *    selected logit is infinite: equal shares of the +inf entries, or 1/k
 *    when all selected logits are -inf).
 *  - Bucketing: rows (t, j) are sorted by (expert, t); perm[pos] = t*k + j;
 *    offsets[e] is the first position of expert e and offsets[N] = T*k.
 *  - Packed base: 16-byte header {u32 magic 0x32574642 ("BFW2"), u32 d,
 *    f32 alpha, u32 version 1}, then d*d/16 little-endian u32 words, row
 *    major; word w of row r holds columns 16w..16w+15, column c in bits
 *    2(c mod 16)..2(c mod 16)+1; codes 00 = 0, 01 = +1, 11 = -1, 10 unused.
 *
 * Every function works one vector at a time with plain loops, in fp64.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_ERR_INVALID_ARG 1
#define ORACLE_ERR_NONFINITE 4

static int ilog2_exact(int d)
{
    int L = 0;
    if (d < 2) return -1;
    while ((1 << L) < d) L++;
    return ((1 << L) == d) ? L : -1;
}

/* One butterfly stage on y (in place).  sign = +1 for B, -1 for B^T. */
static void stage_apply(double *y, int d, int s, const float *angles_s, double sign)
{
    int h = 1 << s;
    for (int j = 0; j < d; j++) {
        if (j & h) continue;
        int p = (j >> (s + 1)) * h + (j & (h - 1));
        double a = sign * (double)angles_s[p];
        double c = cos(a), sn = sin(a);
        double xa = y[j], xb = y[j + h];
        y[j] = c * xa - sn * xb;
        y[j + h] = sn * xa + c * xb;
    }
}

/* y = B(angles) x  (transpose == 0)  or  y = B(angles)^T x  (transpose != 0).
 * angles: [L][d/2] fp32.  x and y may alias. */
int oracle_butterfly_vec(int d, const float *angles, int transpose, const double *x, double *y)
{
    int L = ilog2_exact(d);
    if (L < 1) return ORACLE_ERR_INVALID_ARG;
    if (x != y) memcpy(y, x, sizeof(double) * (size_t)d);
    if (!transpose) {
        for (int s = 0; s < L; s++) stage_apply(y, d, s, angles + (size_t)s * (d / 2), 1.0);
    } else {
        for (int s = L - 1; s >= 0; s--) stage_apply(y, d, s, angles + (size_t)s * (d / 2), -1.0);
    }
    return ORACLE_OK;
}

/* Row-wise butterfly: y[r] = B(angles[e_r]) x[r] or its transpose, where
 * e_r = expert_of_row[r] (0 when expert_of_row is NULL).
 * x, y: [rows][d] fp64; angles: [N][L][d/2] fp32. */
int oracle_butterfly_rows(int rows, int d, int N, const float *angles, const int32_t *expert_of_row,
                          int transpose, const double *x, double *y)
{
    int L = ilog2_exact(d);
    if (L < 1 || rows < 0 || N < 1) return ORACLE_ERR_INVALID_ARG;
    for (int r = 0; r < rows; r++) {
        int e = expert_of_row ? expert_of_row[r] : 0;
        if (e < 0 || e >= N) return ORACLE_ERR_INVALID_ARG;
        oracle_butterfly_vec(d, angles + (size_t)e * L * (d / 2), transpose, x + (size_t)r * d,
                             y + (size_t)r * d);
    }
    return ORACLE_OK;
}

/* ---------------------------------------------------------------- routing */

/* Does expert a come before expert b?  Larger logit first, then lower index. */
static int ranks_before(double la, int a, double lb, int b)
{
    if (la > lb) return 1;
    if (la < lb) return 0;
    return a < b;
}

/* Top-k of one token's logits by a full insertion sort of the N experts. */
static void topk_one(const float *l, int N, int k, int32_t *idx_out, int *order_scratch)
{
    for (int e = 0; e < N; e++) order_scratch[e] = e;
    for (int i = 1; i < N; i++) {
        int e = order_scratch[i];
        int q = i - 1;
        while (q >= 0 && ranks_before((double)l[e], e, (double)l[order_scratch[q]], order_scratch[q])) {
            order_scratch[q + 1] = order_scratch[q];
            q--;
        }
        order_scratch[q + 1] = e;
    }
    for (int j = 0; j < k; j++) idx_out[j] = order_scratch[j];
}

/* Softmax over the k selected logits v[0..k-1] (v[0] is the largest), with
 * the limits for infinite entries described in the file header. */
static void gates_one(const double *v, int k, double *g)
{
    double m = v[0];
    if (isinf(m) && m > 0) {
        int c = 0;
        for (int j = 0; j < k; j++) c += (isinf(v[j]) && v[j] > 0);
        for (int j = 0; j < k; j++) g[j] = (isinf(v[j]) && v[j] > 0) ? 1.0 / c : 0.0;
        return;
    }
    if (isinf(m) && m < 0) {
        for (int j = 0; j < k; j++) g[j] = 1.0 / k;
        return;
    }
    double z = 0.0;
    for (int j = 0; j < k; j++) z += exp(v[j] - m);
    for (int j = 0; j < k; j++) g[j] = exp(v[j] - m) / z;
}

/* Route T tokens: top-k indices [T][k], gates [T][k] (fp64), and the
 * bucketing perm [T*k] / offsets [N+1] (either may be NULL).
 * Returns ORACLE_ERR_NONFINITE if any logit is NaN (outputs then undefined). */
int oracle_route(const float *logits, int T, int N, int k, int32_t *topk_idx, double *gates,
                 int32_t *perm, int32_t *offsets)
{
    if (T < 0 || N < 1 || k < 1 || k > N) return ORACLE_ERR_INVALID_ARG;
    for (size_t i = 0; i < (size_t)T * N; i++)
        if (isnan(logits[i])) return ORACLE_ERR_NONFINITE;
    int *order = (int *)malloc(sizeof(int) * (size_t)N);
    double *v = (double *)malloc(sizeof(double) * (size_t)k);
    for (int t = 0; t < T; t++) {
        const float *l = logits + (size_t)t * N;
        topk_one(l, N, k, topk_idx + (size_t)t * k, order);
        for (int j = 0; j < k; j++) v[j] = (double)l[topk_idx[(size_t)t * k + j]];
        if (gates) gates_one(v, k, gates + (size_t)t * k);
    }
    free(v);
    free(order);
    if (perm || offsets) {
        /* Stable counting sort of rows i = t*k + j by expert. */
        int32_t *count = (int32_t *)calloc((size_t)N + 1, sizeof(int32_t));
        int32_t *start = (int32_t *)calloc((size_t)N + 1, sizeof(int32_t));
        int R = T * k;
        for (int i = 0; i < R; i++) count[topk_idx[i]]++;
        start[0] = 0;
        for (int e = 0; e < N; e++) start[e + 1] = start[e] + count[e];
        if (offsets)
            for (int e = 0; e <= N; e++) offsets[e] = start[e];
        if (perm) {
            for (int i = 0; i < R; i++) perm[start[topk_idx[i]]++] = i;
        }
        free(count);
        free(start);
    }
    return ORACLE_OK;
}

/* ---------------------------------------------------------------- packing */

static uint32_t code_of(int8_t v)
{
    return v == 1 ? 1u : (v == -1 ? 3u : 0u);
}

size_t oracle_packed_base_bytes(int d)
{
    return 16 + (size_t)d * (size_t)d / 4;
}

static void put_u32(uint8_t *p, uint32_t v)
{
    p[0] = (uint8_t)(v & 0xff);
    p[1] = (uint8_t)((v >> 8) & 0xff);
    p[2] = (uint8_t)((v >> 16) & 0xff);
    p[3] = (uint8_t)((v >> 24) & 0xff);
}

/* Pack a ternary d x d matrix (int8, row major) into the 2-bit format. */
int oracle_pack_base(const int8_t *w, int d, float alpha, uint8_t *out)
{
    if (d < 16 || d % 16) return ORACLE_ERR_INVALID_ARG;
    for (size_t i = 0; i < (size_t)d * d; i++)
        if (w[i] < -1 || w[i] > 1) return ORACLE_ERR_INVALID_ARG;
    uint32_t abits;
    memcpy(&abits, &alpha, 4);
    put_u32(out + 0, 0x32574642u);
    put_u32(out + 4, (uint32_t)d);
    put_u32(out + 8, abits);
    put_u32(out + 12, 1u);
    for (int r = 0; r < d; r++) {
        for (int wd = 0; wd < d / 16; wd++) {
            uint32_t word = 0;
            for (int i = 0; i < 16; i++) word |= code_of(w[(size_t)r * d + 16 * wd + i]) << (2 * i);
            put_u32(out + 16 + 4 * ((size_t)r * (d / 16) + wd), word);
        }
    }
    return ORACLE_OK;
}

/* Inverse of oracle_pack_base: returns d via *d_out and alpha via *alpha_out;
 * w must hold d*d bytes (pass NULL to only read the header). */
int oracle_unpack_base(const uint8_t *in, int d_cap, int8_t *w, int *d_out, float *alpha_out)
{
    uint32_t magic = in[0] | (in[1] << 8) | (in[2] << 16) | ((uint32_t)in[3] << 24);
    uint32_t d = in[4] | (in[5] << 8) | (in[6] << 16) | ((uint32_t)in[7] << 24);
    uint32_t abits = in[8] | (in[9] << 8) | (in[10] << 16) | ((uint32_t)in[11] << 24);
    if (magic != 0x32574642u) return ORACLE_ERR_INVALID_ARG;
    if (d_out) *d_out = (int)d;
    if (alpha_out) memcpy(alpha_out, &abits, 4);
    if (!w) return ORACLE_OK;
    if ((int)d > d_cap) return ORACLE_ERR_INVALID_ARG;
    for (uint32_t r = 0; r < d; r++) {
        for (uint32_t c = 0; c < d; c++) {
            size_t off = 16 + 4 * ((size_t)r * (d / 16) + c / 16);
            uint32_t word = in[off] | (in[off + 1] << 8) | (in[off + 2] << 16) | ((uint32_t)in[off + 3] << 24);
            uint32_t code = (word >> (2 * (c % 16))) & 3u;
            w[(size_t)r * d + c] = code == 1 ? 1 : (code == 3 ? -1 : 0);
        }
    }
    return ORACLE_OK;
}

/* ---------------------------------------------------------------- forward */

/* z = W x for a ternary W: additions and subtractions only (the ternary
 * substrate "needs only additions", ButterflyMoE summaries, section 3). */
static void ternary_matvec(const int8_t *w, int d, const double *x, double *z)
{
    for (int r = 0; r < d; r++) {
        double acc = 0.0;
        const int8_t *row = w + (size_t)r * d;
        for (int c = 0; c < d; c++) {
            if (row[c] == 1) acc += x[c];
            else if (row[c] == -1) acc -= x[c];
        }
        z[r] = acc;
    }
}

/* Expert output for one input vector: u = alpha * B(phi) W B(theta)^T x. */
int oracle_expert_apply(int d, const int8_t *w, float alpha, const float *theta_e, const float *phi_e,
                        const double *x, double *u)
{
    int L = ilog2_exact(d);
    if (L < 1) return ORACLE_ERR_INVALID_ARG;
    double *xr = (double *)malloc(sizeof(double) * (size_t)d);
    double *z = (double *)malloc(sizeof(double) * (size_t)d);
    oracle_butterfly_vec(d, theta_e, 1, x, xr);   /* input rotation B(theta)^T */
    ternary_matvec(w, d, xr, z);                 /* shared ternary substrate */
    oracle_butterfly_vec(d, phi_e, 0, z, u);     /* output rotation B(phi) */
    for (int i = 0; i < d; i++) u[i] *= (double)alpha;
    free(xr);
    free(z);
    return ORACLE_OK;
}

/* The layer: y_t = sum_j g_{t,j} * alpha * B(phi_e) W B(theta_e)^T x_t over
 * the token's top-k experts e = e_{t,j}.
 * x: [T][d] fp32 values (bf16 inputs are passed widened); logits [T][N];
 * w: [d][d] int8; theta, phi: [N][L][d/2]; y: [T][d] fp64 out.
 * nthreads <= 0 uses the OpenMP default.  Returns a status code. */
int oracle_forward(const float *x, int T, int d, const float *logits, int N, int k, const int8_t *w,
                   float alpha, const float *theta, const float *phi, double *y, int nthreads)
{
    int L = ilog2_exact(d);
    if (L < 1 || T < 0 || N < 1 || k < 1 || k > N) return ORACLE_ERR_INVALID_ARG;
    int32_t *idx = (int32_t *)malloc(sizeof(int32_t) * ((size_t)T * k + 1));
    double *g = (double *)malloc(sizeof(double) * ((size_t)T * k + 1));
    int st = oracle_route(logits, T, N, k, idx, g, NULL, NULL);
    if (st != ORACLE_OK) {
        free(idx);
        free(g);
        return st;
    }
    size_t tab = (size_t)L * (d / 2);
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel
#endif
    {
        double *xt = (double *)malloc(sizeof(double) * (size_t)d);
        double *u = (double *)malloc(sizeof(double) * (size_t)d);
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 4)
#endif
        for (int t = 0; t < T; t++) {
            double *yt = y + (size_t)t * d;
            for (int i = 0; i < d; i++) xt[i] = (double)x[(size_t)t * d + i];
            for (int i = 0; i < d; i++) yt[i] = 0.0;
            for (int j = 0; j < k; j++) {
                int e = idx[(size_t)t * k + j];
                oracle_expert_apply(d, w, alpha, theta + (size_t)e * tab, phi + (size_t)e * tab, xt, u);
                for (int i = 0; i < d; i++) yt[i] += g[(size_t)t * k + j] * u[i];
            }
        }
        free(xt);
        free(u);
    }
    free(idx);
    free(g);
    return ORACLE_OK;
}

/* Threads the OpenMP runtime would use (1 without OpenMP). */
int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ---------------------------------------------------------------- memory model */

/* Butterfly angle count per butterfly: (d/2) * log2 d (O(d log d), the
 * ButterflyMoE summaries, section 2). */
long long oracle_angles_per_butterfly(int d)
{
    int L = ilog2_exact(d);
    if (L < 1) return -1;
    return (long long)(d / 2) * L;
}

/* Bytes of one ButterflyMoE layer as this library stores it: the packed
 * ternary base (header + 2 bits per weight) plus two fp32 angle tables per
 * expert.  This is the O(d^2 + N d log d) memory of the ButterflyMoE
 * summaries, section 2. */
long long oracle_layer_bytes(int d, int N)
{
    long long a = oracle_angles_per_butterfly(d);
    if (a < 0 || N < 1) return -1;
    return (long long)oracle_packed_base_bytes(d) + (long long)N * 2 * a * 4;
}

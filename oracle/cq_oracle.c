/*
 * cq_oracle.c -- plain, slow, obviously-correct CPU oracle for the CodeQuant /
 * CodeQuant2 low-precision MoE linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the CPU
 * baseline leg of the benchmark may load this library.  The product path (the
 * CUDA library) never calls it and shares no code with it.
 *
 * Arithmetic: fp64 and int64, plain loops, no blocking, no fusion.  Built with
 * -O2 and without -ffast-math.  OpenMP pragmas only split independent output
 * rows across host threads; they never change an operation's order.
 *
 * What is computed (notation: M tokens, K input dim, N output dim):
 *   rotation      x_rot = x . (I_{K/b} (x) H_b), H_b[i][j] = (-1)^popcount(i&j)
 *                 (Sylvester order, unnormalised, contiguous blocks of b).
 *                 CodeQuant abstract: activation outliers are smoothed by a
 *                 rotation; CodeQuant2 page, Figure 1: rotation and scaling
 *                 fused into the model.  The block Walsh-Hadamard form is the
 *                 online rotation of the QuaRot / QuIP# line both build on.
 *   quantization  per-token symmetric absmax to int4 (A4W4) or int8 (A8W4):
 *                 q = round_half_even(qmax * x_rot / max|x_rot|), exact, and
 *                 s_x = (max|x_rot| / sqrt(b)) / qmax  (CodeQuant2 page,
 *                 Tables 1, 2 and 9: the A4W4 / A8W4 settings).
 *   LUT product   y[m,n] = s_x[m] * sum_k C[n, I[n,k]] * q[m,k]; I are 4-bit
 *                 indices into a per-row codebook C of 16 fp16 centroids
 *                 (CodeQuant2 page, Figure 3: centroid matrix and per-row
 *                 assignment matrices; Figure 4: the LUT kernel).
 *                 S[m,n,c] = sum_{k : I[n,k] = c} q[m,k] is the same product
 *                 grouped by centroid (Figure 3's binary assignment matrices).
 *   routing       top-k experts per token (ties to the lower id), softmax
 *                 weights, per-expert counts, offsets and a stable permutation
 *                 of the token slots (the router of the MoE model the
 *                 CodeQuant podcast page describes).
 *   expert FFN    h = fp16(silu(g) * u); y = down(h); out = sum_j w_j y_j
 *                 (+ always-on shared experts with weight 1).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_OK 0
#define ORC_EINVAL 1

/* ------------------------------------------------------------------------ */
/* IEEE binary16 <-> binary64, from the format's definition                  */

double orc_f16_to_f64(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 31;
    int m = h & 1023;
    double v;
    if (e == 0)
        v = ldexp((double)m, -24);              /* subnormal: m * 2^-24 */
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + m), e - 25);  /* (1 + m/1024) * 2^(e-15) */
    return sign ? -v : v;
}

/* Round to nearest binary16, ties to even. */
uint16_t orc_f64_to_f16(double v)
{
    uint16_t sign = signbit(v) ? 0x8000 : 0;
    double a = fabs(v);
    if (isnan(v))
        return 0x7e00;
    if (a == 0.0)
        return sign;
    int ex;
    frexp(a, &ex);                 /* a = f * 2^ex, f in [0.5, 1) */
    int E = ex - 1;                /* floor(log2 a) */
    if (E < -14)
        E = -14;                   /* subnormal range shares the 2^-24 quantum */
    double quantum = ldexp(1.0, E - 10);
    double n = a / quantum;        /* exact: power-of-two scaling */
    double fl = floor(n);
    double frac = n - fl;          /* exact */
    if (frac > 0.5 || (frac == 0.5 && fmod(fl, 2.0) != 0.0))
        fl += 1.0;
    double r = fl * quantum;       /* exact */
    if (r >= 65536.0)
        return sign | 0x7c00;      /* overflow to infinity */
    if (r < ldexp(1.0, -14))
        return sign | (uint16_t)(r / ldexp(1.0, -24));   /* subnormal */
    frexp(r, &ex);
    int e16 = ex - 1 + 15;
    double mant = r / ldexp(1.0, ex - 1) - 1.0;          /* in [0, 1) */
    return sign | (uint16_t)(e16 << 10) | (uint16_t)(mant * 1024.0);
}

/* ------------------------------------------------------------------------ */
/* Hadamard                                                                  */

static int popcount64(uint64_t v)
{
    int c = 0;
    while (v) {
        c += (int)(v & 1u);
        v >>= 1;
    }
    return c;
}

/* H_b[i][j] = (-1)^popcount(i & j): Sylvester construction, natural order. */
int orc_hadamard_entry(int64_t i, int64_t j)
{
    return (popcount64((uint64_t)(i & j)) & 1) ? -1 : 1;
}

static int is_pow2(int64_t b)
{
    return b > 0 && (b & (b - 1)) == 0;
}

/* Dense H_b as a b x b fp64 matrix (row-major). */
int orc_hadamard_matrix(int64_t b, double *H)
{
    if (!is_pow2(b))
        return ORC_EINVAL;
    for (int64_t i = 0; i < b; i++)
        for (int64_t j = 0; j < b; j++)
            H[i * b + j] = (double)orc_hadamard_entry(i, j);
    return ORC_OK;
}

/*
 * x_rot[m, blk*b + j] = sum_i x[m, blk*b + i] * H_b[i][j], with the dense
 * matrix written out.  Exact in fp64: fp16 inputs are multiples of 2^-24 and
 * every partial sum is bounded by 65504 * b < 2^29 for b <= 8192, so each
 * partial sum is an integer multiple of 2^-24 below 2^53 units.
 * x: fp16 bits [M, K]; out: fp64 [M, K].
 */
int orc_rotate(const uint16_t *x, int64_t M, int64_t K, int64_t b, double *out)
{
    if (!is_pow2(b) || b > 8192 || K % b != 0)
        return ORC_EINVAL;
    double *H = (double *)malloc(sizeof(double) * (size_t)(b * b));
    if (!H)
        return ORC_EINVAL;
    orc_hadamard_matrix(b, H);
#pragma omp parallel for schedule(dynamic)
    for (int64_t m = 0; m < M; m++) {
        for (int64_t blk = 0; blk < K / b; blk++) {
            const uint16_t *xb = x + m * K + blk * b;
            double *ob = out + m * K + blk * b;
            for (int64_t j = 0; j < b; j++) {
                double s = 0.0;
                for (int64_t i = 0; i < b; i++)
                    s += orc_f16_to_f64(xb[i]) * H[i * b + j];
                ob[j] = s;
            }
        }
    }
    free(H);
    return ORC_OK;
}

/*
 * Per-token symmetric absmax quantization of rotated rows.
 *   A    = max_k |x_rot[m,k]|
 *   q    = round_half_even(qmax * x_rot / A), computed as an exact rational:
 *          v = x_rot * 2^24 and A' = A * 2^24 are integers (< 2^53), so
 *          num = qmax*|v| fits int64 and the quotient / remainder are exact.
 *   s_x  = (float)((A / sqrt(b)) / qmax)   (each step an IEEE fp64 op)
 * The 1/sqrt(b) normalisation of the rotation is folded into s_x; q is the
 * same whether or not the rotation is normalised.  A zero row gives q = 0,
 * s_x = 0.  qmax = 2^(bits-1) - 1, so -8 / -128 never occur.
 * xr: fp64 [M, K]; q: int8 [M, K] (unpacked); s: fp32 [M].
 */
int orc_quantize(const double *xr, int64_t M, int64_t K, int64_t b, int bits,
                 int8_t *q, float *s)
{
    if (bits != 4 && bits != 8)
        return ORC_EINVAL;
    if (!is_pow2(b))
        return ORC_EINVAL;
    const int64_t qmax = (1 << (bits - 1)) - 1;
    const double two24 = 16777216.0;
    for (int64_t m = 0; m < M; m++) {
        const double *row = xr + m * K;
        double A = 0.0;
        for (int64_t k = 0; k < K; k++)
            if (fabs(row[k]) > A)
                A = fabs(row[k]);
        if (A == 0.0) {
            for (int64_t k = 0; k < K; k++)
                q[m * K + k] = 0;
            s[m] = 0.0f;
            continue;
        }
        int64_t Ai = (int64_t)(A * two24);
        for (int64_t k = 0; k < K; k++) {
            int64_t v = (int64_t)(row[k] * two24);
            int64_t av = v < 0 ? -v : v;
            int64_t num = qmax * av;
            int64_t q0 = num / Ai;
            int64_t r = num - q0 * Ai;
            if (2 * r > Ai || (2 * r == Ai && (q0 & 1)))
                q0 += 1;
            q[m * K + k] = (int8_t)(v < 0 ? -q0 : q0);
        }
        s[m] = (float)((A / sqrt((double)b)) / (double)qmax);
    }
    return ORC_OK;
}

/*
 * Online smoothing scale and channel grouping ahead of the rotation.
 * CodeQuant2 page, Figure 1: rotation and scaling are fused into the model
 * (Table 5's base setting uses SmoothQuant scaling); CodeQuant podcast page,
 * "Summary": the channels are reordered before clustering so that outliers
 * are spread over different groups.  Both are applied to the layer input:
 *   out[m, j] = rne16( x[m, p(j)] * s(p(j)) )
 * with p = perm (the identity if perm is NULL) and s = scale (1 if NULL).
 * The product of two fp16 numbers is exact in fp64 (11 + 11 significant
 * bits), so out is the fp16 rounding, ties to even, of the exact product.
 * x, scale, out: fp16 bits.  Returns ORC_EINVAL unless perm is a permutation
 * of 0 .. K-1.
 */
int orc_scale_permute(const uint16_t *x, int64_t M, int64_t K, const uint16_t *scale,
                      const int32_t *perm, uint16_t *out)
{
    if (perm) {
        unsigned char *seen = (unsigned char *)calloc((size_t)K, 1);
        if (!seen)
            return ORC_EINVAL;
        for (int64_t j = 0; j < K; j++) {
            if (perm[j] < 0 || perm[j] >= K || seen[perm[j]]) {
                free(seen);
                return ORC_EINVAL;
            }
            seen[perm[j]] = 1;
        }
        free(seen);
    }
    for (int64_t m = 0; m < M; m++)
        for (int64_t j = 0; j < K; j++) {
            const int64_t c = perm ? perm[j] : j;
            const double v = orc_f16_to_f64(x[m * K + c]);
            const double sc = scale ? orc_f16_to_f64(scale[c]) : 1.0;
            out[m * K + j] = orc_f64_to_f16(v * sc);
        }
    return ORC_OK;
}

/* rotate then quantize; x fp16 bits [M, K]. */
int orc_rotate_quantize(const uint16_t *x, int64_t M, int64_t K, int64_t b, int bits,
                        int8_t *q, float *s)
{
    double *xr = (double *)malloc(sizeof(double) * (size_t)(M * K));
    if (!xr)
        return ORC_EINVAL;
    int rc = orc_rotate(x, M, K, b, xr);
    if (rc == ORC_OK)
        rc = orc_quantize(xr, M, K, b, bits, q, s);
    free(xr);
    return rc;
}

/* ------------------------------------------------------------------------ */
/* packed formats: element 2j in the low nibble of byte j, 2j+1 in the high  */

/* int4 two's-complement activation codes [M, K/2] -> int8 [M, K] */
void orc_unpack_int4(const uint8_t *p, int64_t M, int64_t K, int8_t *q)
{
    for (int64_t m = 0; m < M; m++)
        for (int64_t k = 0; k < K; k++) {
            uint8_t byte = p[m * (K / 2) + k / 2];
            int nib = (k & 1) ? (byte >> 4) : (byte & 15);
            q[m * K + k] = (int8_t)(nib >= 8 ? nib - 16 : nib);
        }
}

void orc_pack_int4(const int8_t *q, int64_t M, int64_t K, uint8_t *p)
{
    for (int64_t m = 0; m < M; m++)
        for (int64_t j = 0; j < K / 2; j++) {
            int lo = q[m * K + 2 * j] & 15, hi = q[m * K + 2 * j + 1] & 15;
            p[m * (K / 2) + j] = (uint8_t)(lo | (hi << 4));
        }
}

/* unsigned 4-bit weight indices [N, K/2] -> uint8 [N, K] in 0..15 */
void orc_unpack_idx(const uint8_t *p, int64_t N, int64_t K, uint8_t *idx)
{
    for (int64_t n = 0; n < N; n++)
        for (int64_t k = 0; k < K; k++) {
            uint8_t byte = p[n * (K / 2) + k / 2];
            idx[n * K + k] = (uint8_t)((k & 1) ? (byte >> 4) : (byte & 15));
        }
}

/*
 * Adaptive codebook size (CodeQuant2 page, abstract: codebook sizes adapted
 * to each layer's quantization difficulty; Figure 3: adaptive cluster
 * allocation): a layer's rows use 2^b centroids, b in {3, 4, 5}, and its
 * indices are b-bit fields, least significant bit first: index k of row n
 * occupies bits [b*k, b*k + b) of the row's byte string (bit i of byte j is
 * bit 8j + i).  b = 4 is the nibble format above.
 * p: uint8 [N, K*b/8]; idx: uint8 [N, K].
 */
void orc_unpack_idx_bits(const uint8_t *p, int64_t N, int64_t K, int b, uint8_t *idx)
{
    const int64_t rowbytes = K * b / 8;
    for (int64_t n = 0; n < N; n++)
        for (int64_t k = 0; k < K; k++) {
            int v = 0;
            for (int i = 0; i < b; i++) {
                const int64_t bit = k * b + i;
                v |= ((p[n * rowbytes + bit / 8] >> (bit % 8)) & 1) << i;
            }
            idx[n * K + k] = (uint8_t)v;
        }
}

/* ------------------------------------------------------------------------ */
/* LUT product                                                               */

/*
 * y[m,n]   = s[m] * sum_k C[n, idx[n,k]] * q[m,k]           (fp64)
 * mag[m,n] = |s[m]| * sum_k |C[n, idx[n,k]] * q[m,k]|        (error scale)
 * S[m,n,c] = sum_{k : idx[n,k] = c} q[m,k]                  (int32; optional)
 * q: int8 [M, K]; s: fp32 [M]; idx: uint8 [N, K] (0..15); cb: fp16 bits [N, 16].
 */
int orc_lut_gemm(const int8_t *q, const float *s, int64_t M, int64_t K,
                 const uint8_t *idx, const uint16_t *cb, int64_t N,
                 double *y, double *mag, int32_t *S)
{
#pragma omp parallel for schedule(dynamic)
    for (int64_t n = 0; n < N; n++) {
        double C[16];
        for (int c = 0; c < 16; c++)
            C[c] = orc_f16_to_f64(cb[n * 16 + c]);
        for (int64_t m = 0; m < M; m++) {
            double acc = 0.0, am = 0.0;
            int64_t sums[16] = {0};
            for (int64_t k = 0; k < K; k++) {
                int c = idx[n * K + k] & 15;
                double t = C[c] * (double)q[m * K + k];
                acc += t;
                am += fabs(t);
                sums[c] += q[m * K + k];
            }
            y[m * N + n] = (double)s[m] * acc;
            if (mag)
                mag[m * N + n] = fabs((double)s[m]) * am;
            if (S)
                for (int c = 0; c < 16; c++)
                    S[(m * N + n) * 16 + c] = (int32_t)sums[c];
        }
    }
    return ORC_OK;
}

/*
 * The LUT product with per-row codebooks of nc centroids (nc = 2^b):
 *   y[m,n]   = s[m] * sum_k C[n, idx[n,k]] * q[m,k]      (fp64)
 *   mag[m,n] = |s[m]| * sum_k |C[n, idx[n,k]] * q[m,k]|
 * q: int8 [M, K]; s: fp32 [M]; idx: uint8 [N, K] (0..nc-1); cb: fp16 bits [N, nc].
 */
int orc_lut_gemm_nc(const int8_t *q, const float *s, int64_t M, int64_t K,
                    const uint8_t *idx, const uint16_t *cb, int nc, int64_t N,
                    double *y, double *mag)
{
    if (nc < 1 || nc > 256)
        return ORC_EINVAL;
#pragma omp parallel for schedule(dynamic)
    for (int64_t n = 0; n < N; n++) {
        double C[256];
        for (int c = 0; c < nc; c++)
            C[c] = orc_f16_to_f64(cb[n * nc + c]);
        for (int64_t m = 0; m < M; m++) {
            double acc = 0.0, am = 0.0;
            for (int64_t k = 0; k < K; k++) {
                const double w = C[idx[n * K + k] % nc];
                const double t = w * (double)q[m * K + k];
                acc += t;
                am += fabs(t);
            }
            y[m * N + n] = (double)s[m] * acc;
            mag[m * N + n] = fabs((double)s[m]) * am;
        }
    }
    return ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* routing                                                                   */

/*
 * Per token t: the k largest logits, in descending order, ties to the lower
 * expert id.  Weights: renorm != 0 -> softmax over the k selected logits;
 * renorm == 0 -> softmax over all E logits, read at the selected experts.
 * counts[e] = number of slots routed to e; offsets = exclusive scan (E+1);
 * perm lists the flat slots t*k + j grouped by expert, each group in
 * increasing slot order (a stable counting sort).
 */
int orc_route(const float *logits, int64_t T, int64_t E, int64_t k, int renorm,
              int32_t *ids, double *w, int32_t *counts, int32_t *offsets, int32_t *perm)
{
    if (k < 1 || k > E)
        return ORC_EINVAL;
    char *taken = (char *)malloc((size_t)E);
    if (!taken)
        return ORC_EINVAL;
    for (int64_t t = 0; t < T; t++) {
        const float *l = logits + t * E;
        memset(taken, 0, (size_t)E);
        for (int64_t j = 0; j < k; j++) {
            int64_t best = -1;
            for (int64_t e = 0; e < E; e++)
                if (!taken[e] && (best < 0 || l[e] > l[best]))
                    best = e;
            taken[best] = 1;
            ids[t * k + j] = (int32_t)best;
        }
        if (renorm) {
            double lmax = (double)l[ids[t * k]];
            double den = 0.0;
            for (int64_t j = 0; j < k; j++)
                den += exp((double)l[ids[t * k + j]] - lmax);
            for (int64_t j = 0; j < k; j++)
                w[t * k + j] = exp((double)l[ids[t * k + j]] - lmax) / den;
        } else {
            double lmax = (double)l[0];
            for (int64_t e = 1; e < E; e++)
                if ((double)l[e] > lmax)
                    lmax = (double)l[e];
            double den = 0.0;
            for (int64_t e = 0; e < E; e++)
                den += exp((double)l[e] - lmax);
            for (int64_t j = 0; j < k; j++)
                w[t * k + j] = exp((double)l[ids[t * k + j]] - lmax) / den;
        }
    }
    free(taken);
    for (int64_t e = 0; e < E; e++)
        counts[e] = 0;
    for (int64_t sl = 0; sl < T * k; sl++)
        counts[ids[sl]]++;
    offsets[0] = 0;
    for (int64_t e = 0; e < E; e++)
        offsets[e + 1] = offsets[e] + counts[e];
    int32_t *cursor = (int32_t *)malloc(sizeof(int32_t) * (size_t)E);
    if (!cursor)
        return ORC_EINVAL;
    for (int64_t e = 0; e < E; e++)
        cursor[e] = offsets[e];
    for (int64_t sl = 0; sl < T * k; sl++)
        perm[cursor[ids[sl]]++] = (int32_t)sl;
    free(cursor);
    return ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* expert FFN pieces                                                         */

/* h = fp16_rne(silu(g) * u), silu(a) = a / (1 + exp(-a)), fp64. */
void orc_swiglu(const double *g, const double *u, int64_t n, uint16_t *h)
{
    for (int64_t i = 0; i < n; i++) {
        double a = g[i];
        h[i] = orc_f64_to_f16(a / (1.0 + exp(-a)) * u[i]);
    }
}

/*
 * out[t, :] = sum_{j<k} w[t,j] * y_slot[t*k + j, :]  (j in order)
 *             + sum_{s<n_shared} y_shared[s, t, :]    (weight 1)
 * y_slot: fp64 [T*k, H] (slot order); y_shared: fp64 [n_shared, T, H] or NULL.
 */
void orc_combine(const double *y_slot, const double *w, int64_t T, int64_t k, int64_t H,
                 const double *y_shared, int64_t n_shared, double *out)
{
    for (int64_t t = 0; t < T; t++)
        for (int64_t h = 0; h < H; h++) {
            double acc = 0.0;
            for (int64_t j = 0; j < k; j++)
                acc += w[t * k + j] * y_slot[(t * k + j) * H + h];
            for (int64_t s = 0; s < n_shared; s++)
                acc += y_shared[(s * T + t) * H + h];
            out[t * H + h] = acc;
        }
}

/* Host threads the loops above may use (timing only; results do not depend on it). */
void orc_set_threads(int n)
{
#ifdef _OPENMP
    omp_set_num_threads(n > 0 ? n : 1);
#else
    (void)n;
#endif
}

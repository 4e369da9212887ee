/*
 * kvq_oracle.c -- plain, slow CPU oracle for centroid-residual low-bit
 * KV-cache compression.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file; only the test suite, the smoke check and the benchmark's
 * CPU-baseline leg do.  It shares no code with the CUDA library.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math -fopenmp -shared -fPIC
 * (strict IEEE binary32/binary64, no fused multiply-add, x86-64 SSE math).
 *
 * What it computes, and where the pages define it:
 *
 *  - nearest-centroid assignment of every key/value token of a head:
 *    QuantWM: Temporally Consistent 2-Bit KV Cache Quantization for Video
 *    World Models, Sec. 4.1 (QVG applies k-means to assign each key token to
 *    its nearest centroid, then quantises the residual); TempoKV, Sec. 1
 *    (QVG groups similar tokens and subtracts the group centroid).
 *  - per-head k-means fitted online per cache block, separately for K and V:
 *    CORAL-KV, Sec. 2 (QVG fits per-head centroid codebooks online for each
 *    cache block); NanoKV page, Table 4 (QVG: 256 centres each for K/V, two
 *    k-means iterations, BF16 centres) and Table 5 (centres fitted separately
 *    for K and V).
 *  - residual form X^ = X~ + D(Q(X - X~)) with the centroid as prediction:
 *    TempoKV, Sec. 3.3, Eq. 2.
 *  - asymmetric b-bit affine quantisation s = (max - min)/(2^b - 1),
 *    z = round(-min/s), Q = round(X/s) + z, X^ = (Q - z) s: TempoKV, Sec. 3.1,
 *    Eq. 1, applied per contiguous channel group (QuantWM Sec. 4.1: group
 *    range R_g and step R_g/(2^b - 1)).
 *  - packed INT2/INT4 storage: NanoKV page, Table 4 (packed INT2/INT4);
 *    QuantWM, Fig. 9 (packed storage, on-demand reconstruction).
 *  - joint head-channel linear encoder/decoder with INT4 coefficients, centres
 *    added back after decoding: NanoKV page, abstract and Fig. 4(a,b).
 *  - query-sensitive centre selection (QSAC): QuantWM, Sec. 4.1 -- per-head
 *    channel weights w_c from the historical queries' second moments (the
 *    diagonal of M_h), a query-weighted distance that picks top-M candidate
 *    centres, then the candidate whose residual groups minimise the expected
 *    squared logit error sum_g (sum_{c in g} w_c) R_g^2 (the Widrow
 *    approximation with its common factor 1 / (12 (2^b - 1)^2) dropped);
 *    M = 4 (QuantWM, Table 11); w = 1 before any query has been seen
 *    (QuantWM, the appendix paragraph on the cold start).
 *
 * Readings taken where the pages are silent (each mirrored by the CUDA
 * library and listed in the design notes):
 *  - distance = squared Euclidean, evaluated as: widen to binary32; for
 *    c = 0..d-1 in order, e = x_c - mu_c, acc = acc + e*e, each operation
 *    rounded separately (no FMA); ties go to the lowest centroid index;
 *  - k-means seeds = the first C tokens (rounded to bf16); each iteration
 *    assigns, then sets mu_j = bf16(float(sum_fp64 / n_j)); empty clusters
 *    keep their centre; a fixed iteration count, no convergence test;
 *  - Eq. 1's round-to-nearest is round-half-to-even; X/s is evaluated as
 *    X * inv with inv = 1/s (one IEEE division per group); codes are clamped
 *    to [0, 2^b - 1];
 *  - a group whose range is zero, or whose scale s underflows below the
 *    smallest normal binary32, is "degenerate": s = |min|, z = -sign(min),
 *    codes 0, which decodes to exactly min (and to 0 when min == 0);
 *  - decode: x^_c = mu_c + (q_c - z) * s with the subtraction, multiply and
 *    add each rounded to binary32;
 *  - second residual stage (QVG's progressive residual quantisation, named
 *    by TempoKV, Sec. 2, without its steps; NanoKV page, Table 4 evaluates
 *    QVG with one stage): stage 2 quantises what stage 1 leaves,
 *    e_c = r_c - (q1_c - z1) s1 (binary32), with Eq. 1 on the same groups and
 *    bit width; decode x^_c = (mu_c + (q1_c - z1) s1) + (q2_c - z2) s2, each
 *    operation rounded to binary32;
 *  - compact {s, z} (16-bit scale and zero per group, the b + 1 bits per value
 *    of TempoKV, Table 1, at G = 32): s is formed as above, then rounded to
 *    binary16 (nearest, ties to even, magnitudes past the largest finite
 *    binary16 saturating to it); inv = 1/s16 and z = rint(-min * inv) use the
 *    rounded scale, z is rounded to binary16 in the same way, and the codes
 *    are q = clamp(rint(r * inv) + z16, 0, 2^b - 1), so that encode and decode
 *    use the stored values.  A degenerate group, or one whose scale rounds to
 *    zero in binary16, stores s16 = binary16(|min|), z16 = -sign(min) and
 *    codes 0 (decoding to min rounded to binary16);
 *  - QSAC arithmetic in binary32, channel order, no FMA: weighted distance
 *    acc += w_c * (e_c * e_c); group weight W_g = sum of w_c in channel order;
 *    R_g = max - min of the group's residuals; score += W_g * (R_g * R_g) over
 *    groups in order; candidates ranked by (distance, index); the final
 *    choice is the lowest score, ties to the better-ranked candidate.
 */

#include <float.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define KVQO_OK 0
#define KVQO_EINVAL 1
#define KVQO_ENOMEM 2

/* ------------------------------------------------------------------------ */
/* bf16 storage conversions                                                  */
/* ------------------------------------------------------------------------ */

static float bf16_widen(uint16_t h)
{
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* binary32 -> bf16, round to nearest, ties to even (NaN kept quiet). */
static uint16_t bf16_round(float f)
{
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu) != 0u)
        return (uint16_t)((u >> 16) | 0x0040u);
    uint32_t keep_lsb = (u >> 16) & 1u;
    u += 0x7fffu + keep_lsb;
    return (uint16_t)(u >> 16);
}

uint16_t kvqo_bf16_round(float f) { return bf16_round(f); }

/* ------------------------------------------------------------------------ */
/* binary16 storage conversions (compact {s, z})                             */
/* ------------------------------------------------------------------------ */

/*
 * binary32 -> binary16 by the IEEE 754 definition: round to nearest, ties to
 * even, gradual underflow to subnormals; a magnitude that would round to
 * infinity (>= 65520) saturates to the largest finite value 65504; NaN gives
 * the quiet NaN 0x7e00 with the sign kept.
 */
uint16_t kvqo_f16_round(float f)
{
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    const uint32_t sign = (u >> 16) & 0x8000u;
    const uint32_t a = u & 0x7fffffffu;
    if (a > 0x7f800000u)
        return (uint16_t)(sign | 0x7e00u);
    if (a >= 0x477ff000u) /* 65520 and above, infinity included */
        return (uint16_t)(sign | 0x7bffu);
    if (a >= 0x38800000u) { /* 2^-14 and above: a normal binary16 */
        const uint32_t exp = (a >> 23) - 112u, mant = a & 0x7fffffu;
        uint32_t h = (exp << 10) | (mant >> 13);
        const uint32_t rem = mant & 0x1fffu; /* the 13 bits dropped */
        if (rem > 0x1000u || (rem == 0x1000u && (h & 1u)))
            h += 1u; /* a carry into the exponent is the correct result */
        return (uint16_t)(sign | h);
    }
    /* subnormal or zero: a multiple of 2^-24; |f| 2^24 is exact in binary32 */
    float t;
    memcpy(&t, &a, sizeof t);
    t = rintf(t * 16777216.0f); /* ties to even (the default rounding mode) */
    return (uint16_t)(sign | (uint32_t)t);
}

/* binary16 -> binary32 (exact). */
float kvqo_f16_widen(uint16_t h)
{
    const uint32_t sign = ((uint32_t)h & 0x8000u) << 16;
    const uint32_t e = (h >> 10) & 0x1fu, m = h & 0x3ffu;
    float f;
    if (e == 0) {
        f = (float)m * (1.0f / 16777216.0f); /* m 2^-24, exact */
        uint32_t v;
        memcpy(&v, &f, sizeof v);
        v |= sign;
        memcpy(&f, &v, sizeof f);
        return f;
    }
    uint32_t v = sign | (e == 31 ? (0xffu << 23) | (m << 13) : ((e + 112u) << 23) | (m << 13));
    memcpy(&f, &v, sizeof f);
    return f;
}

/* x is either binary32 ([n]) or bf16 bit patterns ([n]); returns binary32. */
static float load_x(const void *x, int x_is_bf16, int64_t i)
{
    if (x_is_bf16)
        return bf16_widen(((const uint16_t *)x)[i]);
    return ((const float *)x)[i];
}

/* ------------------------------------------------------------------------ */
/* distance and assignment                                                   */
/* ------------------------------------------------------------------------ */

/* The specified squared distance: sequential over channels, no FMA. */
float kvqo_distance(const float *x, const float *mu, int d)
{
    float acc = 0.0f;
    for (int c = 0; c < d; ++c) {
        float e = x[c] - mu[c];
        float sq = e * e;
        acc = acc + sq;
    }
    return acc;
}

/* Brute-force nearest centre of one vector; strict '<' keeps the lowest index
 * among equal distances.  mu is [C][d] binary32. */
static int nearest(const float *x, const float *mu, int C, int d, float *best_out)
{
    int best = 0;
    float bd = kvqo_distance(x, mu, d);
    for (int j = 1; j < C; ++j) {
        float dj = kvqo_distance(x, mu + (int64_t)j * d, d);
        if (dj < bd) {
            bd = dj;
            best = j;
        }
    }
    if (best_out)
        *best_out = bd;
    return best;
}

/* Widen one head's centres [C][d] (bf16) to binary32. */
static void widen_centres(const uint16_t *cent_h, int C, int d, float *out)
{
    for (int64_t i = 0; i < (int64_t)C * d; ++i)
        out[i] = bf16_widen(cent_h[i]);
}

/* Gather token t of head h ([T][H][d] input) as binary32. */
static void gather_token(const void *x, int x_is_bf16, int H, int d, int64_t t, int h, float *out)
{
    int64_t base = (t * H + h) * (int64_t)d;
    for (int c = 0; c < d; ++c)
        out[c] = load_x(x, x_is_bf16, base + c);
}

/*
 * idx[h][t] = argmin_j D(x_{t,h}, mu_{h,j}).
 * x: [T][H][d] (binary32 or bf16), cent: [H][C][d] bf16, idx: [H][T] uint16.
 * dist_out (optional): [H][T] binary32 distance of the chosen centre.
 */
int kvqo_assign(const void *x, int x_is_bf16, int64_t T, int H, int d,
                const uint16_t *cent, int C, uint16_t *idx, float *dist_out)
{
    if (T < 0 || H <= 0 || d <= 0 || C <= 0 || C > 65536)
        return KVQO_EINVAL;
    int rc = KVQO_OK;
#pragma omp parallel for schedule(dynamic, 1)
    for (int h = 0; h < H; ++h) {
        float *mu = (float *)malloc(sizeof(float) * (size_t)C * d);
        float *xv = (float *)malloc(sizeof(float) * (size_t)d);
        if (!mu || !xv) {
            rc = KVQO_ENOMEM;
        } else {
            widen_centres(cent + (int64_t)h * C * d, C, d, mu);
            for (int64_t t = 0; t < T; ++t) {
                gather_token(x, x_is_bf16, H, d, t, h, xv);
                float bd;
                int j = nearest(xv, mu, C, d, &bd);
                idx[(int64_t)h * T + t] = (uint16_t)j;
                if (dist_out)
                    dist_out[(int64_t)h * T + t] = bd;
            }
        }
        free(mu);
        free(xv);
    }
    return rc;
}

/* ------------------------------------------------------------------------ */
/* k-means fitting                                                           */
/* ------------------------------------------------------------------------ */

/*
 * Per head: seed mu_j = bf16(x_j) for the first C tokens; then `iters` times:
 * assign every token, mu_j = bf16(float(sum_{t in j} x_t / n_j)) with the sum
 * in binary64 in token order; a centre with no tokens keeps its value.
 * inertia_out (optional): [H][iters + 1] binary64 sum of exact squared
 * distances of every token to its assigned centre, measured with the centres
 * in force before each iteration's update (index 0..iters-1) and with the
 * final centres (index iters).
 */
int kvqo_fit(const void *x, int x_is_bf16, int64_t T, int H, int d, int C, int iters,
             uint16_t *cent_out, double *inertia_out)
{
    if (T < C || H <= 0 || d <= 0 || C <= 0 || C > 65536 || iters < 0)
        return KVQO_EINVAL;
    int rc = KVQO_OK;
#pragma omp parallel for schedule(dynamic, 1)
    for (int h = 0; h < H; ++h) {
        uint16_t *cent_h = cent_out + (int64_t)h * C * d;
        float *mu = (float *)malloc(sizeof(float) * (size_t)C * d);
        float *xv = (float *)malloc(sizeof(float) * (size_t)d);
        double *sums = (double *)malloc(sizeof(double) * (size_t)C * d);
        int64_t *counts = (int64_t *)malloc(sizeof(int64_t) * (size_t)C);
        if (!mu || !xv || !sums || !counts) {
            rc = KVQO_ENOMEM;
            goto done;
        }
        for (int j = 0; j < C; ++j) {
            gather_token(x, x_is_bf16, H, d, j, h, xv);
            for (int c = 0; c < d; ++c)
                cent_h[(int64_t)j * d + c] = bf16_round(xv[c]);
        }
        for (int it = 0; it <= iters; ++it) {
            widen_centres(cent_h, C, d, mu);
            memset(sums, 0, sizeof(double) * (size_t)C * d);
            memset(counts, 0, sizeof(int64_t) * (size_t)C);
            double inertia = 0.0;
            for (int64_t t = 0; t < T; ++t) {
                gather_token(x, x_is_bf16, H, d, t, h, xv);
                int j = nearest(xv, mu, C, d, NULL);
                counts[j] += 1;
                for (int c = 0; c < d; ++c) {
                    sums[(int64_t)j * d + c] += (double)xv[c];
                    double e = (double)xv[c] - (double)mu[(int64_t)j * d + c];
                    inertia += e * e;
                }
            }
            if (inertia_out)
                inertia_out[(int64_t)h * (iters + 1) + it] = inertia;
            if (it == iters)
                break;
            for (int j = 0; j < C; ++j) {
                if (counts[j] == 0)
                    continue;
                for (int c = 0; c < d; ++c) {
                    double mean = sums[(int64_t)j * d + c] / (double)counts[j];
                    cent_h[(int64_t)j * d + c] = bf16_round((float)mean);
                }
            }
        }
    done:
        free(mu);
        free(xv);
        free(sums);
        free(counts);
    }
    return rc;
}

/* ------------------------------------------------------------------------ */
/* Eq. 1 quantisation of one group                                           */
/* ------------------------------------------------------------------------ */

/*
 * r: G residuals.  Writes scale s, zero z and G codes in [0, 2^bits - 1].
 */
void kvqo_quant_group(const float *r, int G, int bits, float *s_out, float *z_out, uint8_t *q)
{
    float mn = r[0], mx = r[0];
    for (int c = 1; c < G; ++c) {
        if (r[c] < mn)
            mn = r[c];
        if (r[c] > mx)
            mx = r[c];
    }
    const float qmax = (float)((1 << bits) - 1);
    float s = 0.0f;
    if (mx != mn)
        s = (mx - mn) / qmax;
    if (mx == mn || !(s >= FLT_MIN)) {
        /* degenerate group: decodes to exactly mn */
        if (mn == 0.0f) {
            *s_out = 0.0f;
            *z_out = 0.0f;
        } else {
            *s_out = fabsf(mn);
            *z_out = (mn > 0.0f) ? -1.0f : 1.0f;
        }
        for (int c = 0; c < G; ++c)
            q[c] = 0;
        return;
    }
    float inv = 1.0f / s;
    float z = rintf(-mn * inv);
    for (int c = 0; c < G; ++c) {
        float v = rintf(r[c] * inv) + z;
        if (v < 0.0f)
            v = 0.0f;
        if (v > qmax)
            v = qmax;
        q[c] = (uint8_t)v;
    }
    *s_out = s;
    *z_out = z;
}

/*
 * Eq. 1 with 16-bit {s, z} (the compact reading in the header): writes the
 * binary16 bits of s and z and G codes computed with the stored values.
 */
void kvqo_quant_group16(const float *r, int G, int bits, uint16_t *s_out, uint16_t *z_out, uint8_t *q)
{
    float mn = r[0], mx = r[0];
    for (int c = 1; c < G; ++c) {
        if (r[c] < mn)
            mn = r[c];
        if (r[c] > mx)
            mx = r[c];
    }
    const float qmax = (float)((1 << bits) - 1);
    float s = 0.0f;
    if (mx != mn)
        s = (mx - mn) / qmax;
    const uint16_t s16 = kvqo_f16_round(s);
    if (mx == mn || !(s >= FLT_MIN) || (s16 & 0x7fffu) == 0u) {
        if (mn == 0.0f) {
            *s_out = 0u;
            *z_out = 0u;
        } else {
            *s_out = kvqo_f16_round(fabsf(mn));
            *z_out = (mn > 0.0f) ? 0xbc00u /* -1 */ : 0x3c00u /* +1 */;
        }
        for (int c = 0; c < G; ++c)
            q[c] = 0;
        return;
    }
    const float sf = kvqo_f16_widen(s16);
    const float inv = 1.0f / sf;
    const uint16_t z16 = kvqo_f16_round(rintf(-mn * inv));
    const float zf = kvqo_f16_widen(z16);
    for (int c = 0; c < G; ++c) {
        float v = rintf(r[c] * inv) + zf;
        if (v < 0.0f)
            v = 0.0f;
        if (v > qmax)
            v = qmax;
        q[c] = (uint8_t)v;
    }
    *s_out = s16;
    *z_out = z16;
}

/* x^ = (q - z) * s, each step rounded to binary32. */
float kvqo_dequant(uint8_t q, float s, float z)
{
    float t = (float)q - z;
    return t * s;
}

/* ------------------------------------------------------------------------ */
/* packing                                                                   */
/* ------------------------------------------------------------------------ */

/* n codes of `bits` (2 or 4) into n*bits/8 bytes, least significant first. */
void kvqo_pack(const uint8_t *q, int n, int bits, uint8_t *out)
{
    int per = 8 / bits;
    for (int k = 0; k < n / per; ++k) {
        unsigned byte = 0;
        for (int i = 0; i < per; ++i)
            byte |= ((unsigned)q[k * per + i] & ((1u << bits) - 1u)) << (i * bits);
        out[k] = (uint8_t)byte;
    }
}

void kvqo_unpack(const uint8_t *in, int n, int bits, uint8_t *q)
{
    int per = 8 / bits;
    for (int c = 0; c < n; ++c)
        q[c] = (uint8_t)((in[c / per] >> ((c % per) * bits)) & ((1u << bits) - 1u));
}

/* ------------------------------------------------------------------------ */
/* per-head encode / decode                                                  */
/* ------------------------------------------------------------------------ */

static int check_codec(int H, int d, int C, int bits, int G)
{
    if (H <= 0 || d <= 0 || C <= 0 || C > 65536)
        return 0;
    if (bits != 2 && bits != 4)
        return 0;
    if (G <= 0 || d % G != 0 || (d * bits) % 8 != 0 || G > 256)
        return 0;
    return 1;
}

/*
 * Encode one K or V history.
 *   x     [T][H][d]  binary32 or bf16
 *   cent  [H][C][d]  bf16
 *   idx   [H][T]     uint16 (out)
 *   codes [H][T][d*bits/8]  packed (out)
 *   meta  [H][T][d/G][2]    {s, z} binary32 (out)
 */
int kvqo_encode(const void *x, int x_is_bf16, int64_t T, int H, int d, const uint16_t *cent, int C,
                int bits, int G, uint16_t *idx, uint8_t *codes, float *meta)
{
    if (T < 0 || !check_codec(H, d, C, bits, G))
        return KVQO_EINVAL;
    const int cb = d * bits / 8, ng = d / G;
    int rc = KVQO_OK;
#pragma omp parallel for schedule(dynamic, 1)
    for (int h = 0; h < H; ++h) {
        float *mu = (float *)malloc(sizeof(float) * (size_t)C * d);
        float *xv = (float *)malloc(sizeof(float) * (size_t)d);
        float *r = (float *)malloc(sizeof(float) * (size_t)d);
        uint8_t *q = (uint8_t *)malloc((size_t)d);
        if (!mu || !xv || !r || !q) {
            rc = KVQO_ENOMEM;
        } else {
            widen_centres(cent + (int64_t)h * C * d, C, d, mu);
            for (int64_t t = 0; t < T; ++t) {
                int64_t th = (int64_t)h * T + t;
                gather_token(x, x_is_bf16, H, d, t, h, xv);
                int j = nearest(xv, mu, C, d, NULL);
                idx[th] = (uint16_t)j;
                for (int c = 0; c < d; ++c)
                    r[c] = xv[c] - mu[(int64_t)j * d + c];
                for (int g = 0; g < ng; ++g) {
                    float s, z;
                    kvqo_quant_group(r + g * G, G, bits, &s, &z, q + g * G);
                    meta[(th * ng + g) * 2 + 0] = s;
                    meta[(th * ng + g) * 2 + 1] = z;
                }
                kvqo_pack(q, d, bits, codes + th * cb);
            }
        }
        free(mu);
        free(xv);
        free(r);
        free(q);
    }
    return rc;
}

/* Reconstruct [T][H][d] binary32 from the encoded form. */
int kvqo_decode(const uint16_t *idx, const uint8_t *codes, const float *meta, const uint16_t *cent,
                int64_t T, int H, int d, int C, int bits, int G, float *out)
{
    if (T < 0 || !check_codec(H, d, C, bits, G))
        return KVQO_EINVAL;
    const int cb = d * bits / 8, ng = d / G;
    int rc = KVQO_OK;
#pragma omp parallel for schedule(dynamic, 1)
    for (int h = 0; h < H; ++h) {
        uint8_t *q = (uint8_t *)malloc((size_t)d);
        if (!q) {
            rc = KVQO_ENOMEM;
            continue;
        }
        for (int64_t t = 0; t < T; ++t) {
            int64_t th = (int64_t)h * T + t;
            int j = idx[th];
            if (j >= C) {
                rc = KVQO_EINVAL;
                break;
            }
            kvqo_unpack(codes + th * cb, d, bits, q);
            for (int c = 0; c < d; ++c) {
                int g = c / G;
                float s = meta[(th * ng + g) * 2 + 0];
                float z = meta[(th * ng + g) * 2 + 1];
                float mu = bf16_widen(cent[((int64_t)h * C + j) * d + c]);
                out[(t * H + h) * (int64_t)d + c] = mu + kvqo_dequant(q[c], s, z);
            }
        }
        free(q);
    }
    return rc;
}

/*
 * kvqo_encode with 16-bit {s, z}: meta16 [H][T][d/G][2] binary16 bits
 * {s, z}; everything else as kvqo_encode.
 */
int kvqo_encode16(const void *x, int x_is_bf16, int64_t T, int H, int d, const uint16_t *cent, int C, int bits,
                  int G, uint16_t *idx, uint8_t *codes, uint16_t *meta16)
{
    if (T < 0 || !check_codec(H, d, C, bits, G))
        return KVQO_EINVAL;
    const int cb = d * bits / 8, ng = d / G;
    int rc = KVQO_OK;
#pragma omp parallel for schedule(dynamic, 1)
    for (int h = 0; h < H; ++h) {
        float *mu = (float *)malloc(sizeof(float) * (size_t)C * d);
        float *xv = (float *)malloc(sizeof(float) * (size_t)d);
        float *r = (float *)malloc(sizeof(float) * (size_t)d);
        uint8_t *q = (uint8_t *)malloc((size_t)d);
        if (!mu || !xv || !r || !q) {
            rc = KVQO_ENOMEM;
        } else {
            widen_centres(cent + (int64_t)h * C * d, C, d, mu);
            for (int64_t t = 0; t < T; ++t) {
                int64_t th = (int64_t)h * T + t;
                gather_token(x, x_is_bf16, H, d, t, h, xv);
                int j = nearest(xv, mu, C, d, NULL);
                idx[th] = (uint16_t)j;
                for (int c = 0; c < d; ++c)
                    r[c] = xv[c] - mu[(int64_t)j * d + c];
                for (int g = 0; g < ng; ++g)
                    kvqo_quant_group16(r + g * G, G, bits, &meta16[(th * ng + g) * 2 + 0],
                                       &meta16[(th * ng + g) * 2 + 1], q + g * G);
                kvqo_pack(q, d, bits, codes + th * cb);
            }
        }
        free(mu);
        free(xv);
        free(r);
        free(q);
    }
    return rc;
}

/* kvqo_decode for 16-bit {s, z}: x^ = mu + (q - z16) * s16 in binary32. */
int kvqo_decode16(const uint16_t *idx, const uint8_t *codes, const uint16_t *meta16, const uint16_t *cent,
                  int64_t T, int H, int d, int C, int bits, int G, float *out)
{
    if (T < 0 || !check_codec(H, d, C, bits, G))
        return KVQO_EINVAL;
    const int cb = d * bits / 8, ng = d / G;
    int rc = KVQO_OK;
#pragma omp parallel for schedule(dynamic, 1)
    for (int h = 0; h < H; ++h) {
        uint8_t *q = (uint8_t *)malloc((size_t)d);
        if (!q) {
            rc = KVQO_ENOMEM;
            continue;
        }
        for (int64_t t = 0; t < T; ++t) {
            int64_t th = (int64_t)h * T + t;
            int j = idx[th];
            if (j >= C) {
                rc = KVQO_EINVAL;
                break;
            }
            kvqo_unpack(codes + th * cb, d, bits, q);
            for (int c = 0; c < d; ++c) {
                int g = c / G;
                float s = kvqo_f16_widen(meta16[(th * ng + g) * 2 + 0]);
                float z = kvqo_f16_widen(meta16[(th * ng + g) * 2 + 1]);
                float mu = bf16_widen(cent[((int64_t)h * C + j) * d + c]);
                out[(t * H + h) * (int64_t)d + c] = mu + kvqo_dequant(q[c], s, z);
            }
        }
        free(q);
    }
    return rc;
}

/* ------------------------------------------------------------------------ */
/* second residual stage                                                     */
/* ------------------------------------------------------------------------ */

/*
 * kvqo_encode followed by a second stage: idx, codes and meta exactly as
 * kvqo_encode writes them; then, per group, the stage-1 error
 * e = r - (q1 - z1) s1 and its Eq. 1 form in codes2 [H][T][d*bits/8] and
 * meta2 [H][T][d/G][2].
 */
int kvqo_encode2(const void *x, int x_is_bf16, int64_t T, int H, int d, const uint16_t *cent, int C, int bits,
                 int G, uint16_t *idx, uint8_t *codes, float *meta, uint8_t *codes2, float *meta2)
{
    if (T < 0 || !check_codec(H, d, C, bits, G))
        return KVQO_EINVAL;
    const int cb = d * bits / 8, ng = d / G;
    int rc = KVQO_OK;
#pragma omp parallel for schedule(dynamic, 1)
    for (int h = 0; h < H; ++h) {
        float *mu = (float *)malloc(sizeof(float) * (size_t)C * d);
        float *xv = (float *)malloc(sizeof(float) * (size_t)d);
        float *r = (float *)malloc(sizeof(float) * (size_t)d);
        float *e = (float *)malloc(sizeof(float) * (size_t)d);
        uint8_t *q = (uint8_t *)malloc((size_t)d);
        if (!mu || !xv || !r || !e || !q) {
            rc = KVQO_ENOMEM;
        } else {
            widen_centres(cent + (int64_t)h * C * d, C, d, mu);
            for (int64_t t = 0; t < T; ++t) {
                int64_t th = (int64_t)h * T + t;
                gather_token(x, x_is_bf16, H, d, t, h, xv);
                int j = nearest(xv, mu, C, d, NULL);
                idx[th] = (uint16_t)j;
                for (int c = 0; c < d; ++c)
                    r[c] = xv[c] - mu[(int64_t)j * d + c];
                /* stage 1 */
                for (int g = 0; g < ng; ++g) {
                    float s1, z1;
                    kvqo_quant_group(r + g * G, G, bits, &s1, &z1, q + g * G);
                    meta[(th * ng + g) * 2 + 0] = s1;
                    meta[(th * ng + g) * 2 + 1] = z1;
                    for (int c = g * G; c < (g + 1) * G; ++c)
                        e[c] = r[c] - kvqo_dequant(q[c], s1, z1);
                }
                kvqo_pack(q, d, bits, codes + th * cb);
                /* stage 2: the error stage 1 leaves */
                for (int g = 0; g < ng; ++g) {
                    float s2, z2;
                    kvqo_quant_group(e + g * G, G, bits, &s2, &z2, q + g * G);
                    meta2[(th * ng + g) * 2 + 0] = s2;
                    meta2[(th * ng + g) * 2 + 1] = z2;
                }
                kvqo_pack(q, d, bits, codes2 + th * cb);
            }
        }
        free(mu);
        free(xv);
        free(r);
        free(e);
        free(q);
    }
    return rc;
}

/* Reconstruction from both stages: (mu + (q1 - z1) s1) + (q2 - z2) s2. */
int kvqo_decode2(const uint16_t *idx, const uint8_t *codes, const float *meta, const uint8_t *codes2,
                 const float *meta2, const uint16_t *cent, int64_t T, int H, int d, int C, int bits, int G,
                 float *out)
{
    if (T < 0 || !check_codec(H, d, C, bits, G))
        return KVQO_EINVAL;
    const int cb = d * bits / 8, ng = d / G;
    int rc = KVQO_OK;
#pragma omp parallel for schedule(dynamic, 1)
    for (int h = 0; h < H; ++h) {
        uint8_t *q1 = (uint8_t *)malloc((size_t)d);
        uint8_t *q2 = (uint8_t *)malloc((size_t)d);
        if (!q1 || !q2) {
            rc = KVQO_ENOMEM;
            free(q1);
            free(q2);
            continue;
        }
        for (int64_t t = 0; t < T; ++t) {
            int64_t th = (int64_t)h * T + t;
            int j = idx[th];
            if (j >= C) {
                rc = KVQO_EINVAL;
                break;
            }
            kvqo_unpack(codes + th * cb, d, bits, q1);
            kvqo_unpack(codes2 + th * cb, d, bits, q2);
            for (int c = 0; c < d; ++c) {
                int g = c / G;
                float mu = bf16_widen(cent[((int64_t)h * C + j) * d + c]);
                float stage1 = mu + kvqo_dequant(q1[c], meta[(th * ng + g) * 2], meta[(th * ng + g) * 2 + 1]);
                out[(t * H + h) * (int64_t)d + c] =
                    stage1 + kvqo_dequant(q2[c], meta2[(th * ng + g) * 2], meta2[(th * ng + g) * 2 + 1]);
            }
        }
        free(q1);
        free(q2);
    }
    return rc;
}

/* ------------------------------------------------------------------------ */
/* query-sensitive centre selection (QSAC)                                   */
/* ------------------------------------------------------------------------ */

/* Query-weighted squared distance sum_c w_c (x_c - mu_c)^2, binary32. */
float kvqo_weighted_distance(const float *x, const float *mu, const float *w, int d)
{
    float total = 0.0f;
    for (int c = 0; c < d; ++c) {
        const float diff = x[c] - mu[c];
        const float diff2 = diff * diff;
        const float term = w[c] * diff2;
        total = total + term;
    }
    return total;
}

/* QSAC score of one residual: sum over groups of W_g * R_g^2, binary32. */
float kvqo_qsac_score(const float *r, const float *w, int d, int G)
{
    float score = 0.0f;
    for (int g = 0; g < d / G; ++g) {
        float lo = r[g * G], hi = r[g * G], wg = 0.0f;
        for (int c = g * G; c < (g + 1) * G; ++c) {
            if (r[c] < lo)
                lo = r[c];
            if (r[c] > hi)
                hi = r[c];
            wg = wg + w[c];
        }
        const float range = hi - lo;
        const float range2 = range * range;
        const float term = wg * range2;
        score = score + term;
    }
    return score;
}

/* Centre chosen by QSAC for one vector.  mu [C][d] binary32, w [d].  cand
 * (M entries) receives the candidates in rank order. */
static int qsac_choose(const float *x, const float *mu, const float *w, int C, int d, int G, int M, int *cand,
                       float *cand_dist, float *r)
{
    int m = M < C ? M : C;
    /* top-m by (distance, index): insertion into a sorted list */
    int n = 0;
    for (int j = 0; j < C; ++j) {
        const float dj = kvqo_weighted_distance(x, mu + (int64_t)j * d, w, d);
        int pos = n;
        while (pos > 0 && dj < cand_dist[pos - 1])
            --pos;
        if (pos >= m)
            continue;
        int last = n < m ? n : m - 1;
        for (int k = last; k > pos; --k) {
            cand[k] = cand[k - 1];
            cand_dist[k] = cand_dist[k - 1];
        }
        cand[pos] = j;
        cand_dist[pos] = dj;
        if (n < m)
            ++n;
    }
    int choice = cand[0];
    float best = 0.0f;
    for (int k = 0; k < m; ++k) {
        const float *mj = mu + (int64_t)cand[k] * d;
        for (int c = 0; c < d; ++c)
            r[c] = x[c] - mj[c];
        const float sc = kvqo_qsac_score(r, w, d, G);
        if (k == 0 || sc < best) {
            best = sc;
            choice = cand[k];
        }
    }
    return choice;
}

/*
 * QSAC assignment of one K history.  w: [H][d] binary32 channel weights.
 * idx [H][T] (out); cand (optional) [H][T][M] the ranked candidates (-1 where
 * C < M).
 */
int kvqo_qsac_assign(const void *x, int x_is_bf16, int64_t T, int H, int d, const uint16_t *cent, int C,
                     const float *w, int G, int M, uint16_t *idx, int32_t *cand_out)
{
    if (T < 0 || H <= 0 || d <= 0 || C <= 0 || C > 65536 || M <= 0 || G <= 0 || d % G != 0)
        return KVQO_EINVAL;
    int rc = KVQO_OK;
#pragma omp parallel for schedule(dynamic, 1)
    for (int h = 0; h < H; ++h) {
        float *mu = (float *)malloc(sizeof(float) * (size_t)C * d);
        float *xv = (float *)malloc(sizeof(float) * (size_t)d);
        float *r = (float *)malloc(sizeof(float) * (size_t)d);
        int *cand = (int *)malloc(sizeof(int) * (size_t)M);
        float *cdist = (float *)malloc(sizeof(float) * (size_t)M);
        if (!mu || !xv || !r || !cand || !cdist) {
            rc = KVQO_ENOMEM;
        } else {
            widen_centres(cent + (int64_t)h * C * d, C, d, mu);
            for (int64_t t = 0; t < T; ++t) {
                gather_token(x, x_is_bf16, H, d, t, h, xv);
                for (int k = 0; k < M; ++k)
                    cand[k] = -1;
                const int j = qsac_choose(xv, mu, w + (int64_t)h * d, C, d, G, M, cand, cdist, r);
                idx[(int64_t)h * T + t] = (uint16_t)j;
                if (cand_out)
                    for (int k = 0; k < M; ++k)
                        cand_out[((int64_t)h * T + t) * M + k] = cand[k];
            }
        }
        free(mu);
        free(xv);
        free(r);
        free(cand);
        free(cdist);
    }
    return rc;
}

/*
 * Residual quantisation against GIVEN centre indices (the QSAC choice):
 * codes and {s, z} exactly as kvqo_encode writes them for that index.
 */
int kvqo_encode_given(const void *x, int x_is_bf16, int64_t T, int H, int d, const uint16_t *cent, int C,
                      int bits, int G, const uint16_t *idx, uint8_t *codes, float *meta)
{
    if (T < 0 || !check_codec(H, d, C, bits, G))
        return KVQO_EINVAL;
    const int cb = d * bits / 8, ng = d / G;
    int rc = KVQO_OK;
#pragma omp parallel for schedule(dynamic, 1)
    for (int h = 0; h < H; ++h) {
        float *xv = (float *)malloc(sizeof(float) * (size_t)d);
        float *res = (float *)malloc(sizeof(float) * (size_t)d);
        uint8_t *q = (uint8_t *)malloc((size_t)d);
        if (!xv || !res || !q) {
            rc = KVQO_ENOMEM;
        } else {
            for (int64_t t = 0; t < T; ++t) {
                const int64_t th = (int64_t)h * T + t;
                const int j = idx[th];
                if (j >= C) {
                    rc = KVQO_EINVAL;
                    break;
                }
                gather_token(x, x_is_bf16, H, d, t, h, xv);
                for (int c = 0; c < d; ++c)
                    res[c] = xv[c] - bf16_widen(cent[((int64_t)h * C + j) * d + c]);
                for (int g = 0; g < ng; ++g) {
                    float sg, zg;
                    kvqo_quant_group(res + g * G, G, bits, &sg, &zg, q + g * G);
                    meta[(th * ng + g) * 2 + 0] = sg;
                    meta[(th * ng + g) * 2 + 1] = zg;
                }
                kvqo_pack(q, d, bits, codes + th * cb);
            }
        }
        free(xv);
        free(res);
        free(q);
    }
    return rc;
}

/* ------------------------------------------------------------------------ */
/* joint head-channel path                                                   */
/* ------------------------------------------------------------------------ */

/*
 * Quantise a [T][r] binary32 coefficient matrix with Eq. 1 per contiguous
 * group of G coefficients: codes [T][r*bits/8], meta [T][r/G][2].
 */
int kvqo_quant_rows(const float *coef, int64_t T, int r, int bits, int G, uint8_t *codes, float *meta)
{
    if (T < 0 || r <= 0 || (bits != 2 && bits != 4) || G <= 0 || r % G != 0 || (r * bits) % 8 != 0)
        return KVQO_EINVAL;
    const int cb = r * bits / 8, ng = r / G;
    int rc = KVQO_OK;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        uint8_t *q = (uint8_t *)malloc((size_t)r);
        if (!q) {
            rc = KVQO_ENOMEM;
            continue;
        }
        for (int g = 0; g < ng; ++g) {
            float s, z;
            kvqo_quant_group(coef + t * r + g * G, G, bits, &s, &z, q + g * G);
            meta[(t * ng + g) * 2 + 0] = s;
            meta[(t * ng + g) * 2 + 1] = z;
        }
        kvqo_pack(q, r, bits, codes + t * cb);
        free(q);
    }
    return rc;
}

/*
 * Joint encoder.  Per token: assign each head to its nearest centre (as the
 * per-head codec), form the residual over all H*d channels, round it to bf16,
 * project with W_enc ([H*d][r] bf16) in binary64, round to binary32, and
 * quantise the r coefficients per group of G.
 *   idx [H][T], codes [T][r*bits/8], meta [T][r/G][2]; coef_out (optional)
 *   [T][r] binary32 coefficients before quantisation.
 */
int kvqo_joint_encode(const void *x, int x_is_bf16, int64_t T, int H, int d, const uint16_t *cent, int C,
                      const uint16_t *w_enc, int r, int bits, int G,
                      uint16_t *idx, uint8_t *codes, float *meta, float *coef_out)
{
    if (T < 0 || H <= 0 || d <= 0 || C <= 0 || C > 65536 || r <= 0)
        return KVQO_EINVAL;
    if ((bits != 2 && bits != 4) || G <= 0 || r % G != 0 || (r * bits) % 8 != 0)
        return KVQO_EINVAL;
    const int64_t n = (int64_t)H * d;
    float *coef = (float *)malloc(sizeof(float) * (size_t)(T > 0 ? T : 1) * r);
    float *w = (float *)malloc(sizeof(float) * (size_t)n * r);
    float *mu = (float *)malloc(sizeof(float) * (size_t)H * C * d);
    if (!coef || !w || !mu) {
        free(coef);
        free(w);
        free(mu);
        return KVQO_ENOMEM;
    }
    for (int64_t i = 0; i < n * r; ++i)
        w[i] = bf16_widen(w_enc[i]);
    for (int64_t i = 0; i < (int64_t)H * C * d; ++i)
        mu[i] = bf16_widen(cent[i]);
    int rc = KVQO_OK;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        float *xv = (float *)malloc(sizeof(float) * (size_t)d);
        float *res = (float *)malloc(sizeof(float) * (size_t)n);
        if (!xv || !res) {
            rc = KVQO_ENOMEM;
            free(xv);
            free(res);
            continue;
        }
        for (int h = 0; h < H; ++h) {
            const float *mu_h = mu + (int64_t)h * C * d;
            gather_token(x, x_is_bf16, H, d, t, h, xv);
            int j = nearest(xv, mu_h, C, d, NULL);
            idx[(int64_t)h * T + t] = (uint16_t)j;
            for (int c = 0; c < d; ++c) {
                float e = xv[c] - mu_h[(int64_t)j * d + c];
                res[h * d + c] = bf16_widen(bf16_round(e));
            }
        }
        for (int k = 0; k < r; ++k) {
            double acc = 0.0;
            for (int64_t i = 0; i < n; ++i)
                acc += (double)res[i] * (double)w[i * r + k];
            coef[t * r + k] = (float)acc;
        }
        free(xv);
        free(res);
    }
    if (rc == KVQO_OK)
        rc = kvqo_quant_rows(coef, T, r, bits, G, codes, meta);
    if (coef_out && rc == KVQO_OK)
        memcpy(coef_out, coef, sizeof(float) * (size_t)T * r);
    free(coef);
    free(w);
    free(mu);
    return rc;
}

/*
 * Joint decoder: c^ = (q - z) s per coefficient (binary32), R^ = c^ W_dec in
 * binary64 with W_dec [r][H*d] bf16, rounded to binary32, then
 * x^_{t,h,c} = mu_{h, idx}[c] + R^[h*d + c] in binary32.  out [T][H][d].
 */
int kvqo_joint_decode(const uint16_t *idx, const uint8_t *codes, const float *meta, const uint16_t *cent,
                      const uint16_t *w_dec, int64_t T, int H, int d, int C, int r, int bits, int G,
                      float *out)
{
    if (T < 0 || H <= 0 || d <= 0 || C <= 0 || r <= 0 || (bits != 2 && bits != 4) || G <= 0 || r % G != 0)
        return KVQO_EINVAL;
    const int64_t n = (int64_t)H * d;
    const int cb = r * bits / 8, ng = r / G;
    float *w = (float *)malloc(sizeof(float) * (size_t)n * r);
    if (!w)
        return KVQO_ENOMEM;
    for (int64_t i = 0; i < n * r; ++i)
        w[i] = bf16_widen(w_dec[i]);
    int rc = KVQO_OK;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        uint8_t *q = (uint8_t *)malloc((size_t)r);
        float *ch = (float *)malloc(sizeof(float) * (size_t)r);
        if (!q || !ch) {
            rc = KVQO_ENOMEM;
            free(q);
            free(ch);
            continue;
        }
        kvqo_unpack(codes + t * cb, r, bits, q);
        for (int k = 0; k < r; ++k) {
            int g = k / G;
            ch[k] = kvqo_dequant(q[k], meta[(t * ng + g) * 2 + 0], meta[(t * ng + g) * 2 + 1]);
        }
        for (int h = 0; h < H; ++h) {
            int j = idx[(int64_t)h * T + t];
            for (int c = 0; c < d; ++c) {
                double acc = 0.0;
                for (int k = 0; k < r; ++k)
                    acc += (double)ch[k] * (double)w[(int64_t)k * n + h * d + c];
                float mu = bf16_widen(cent[((int64_t)h * C + j) * d + c]);
                out[(t * H + h) * (int64_t)d + c] = mu + (float)acc;
            }
        }
        free(q);
        free(ch);
    }
    free(w);
    return rc;
}

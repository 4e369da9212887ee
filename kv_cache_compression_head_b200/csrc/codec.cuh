// codec.cuh -- per-head centroid-residual codec: assignment, Eq. 1 group
// quantisation, packing, reconstruction and k-means fitting.
//
// Method: QuantWM: Temporally Consistent 2-Bit KV Cache Quantization for
// Video World Models, Sec. 4.1 (nearest-centroid assignment, residual
// quantisation); TempoKV, Sec. 3.1 Eq. 1 (asymmetric affine quantiser) and
// Sec. 3.3 Eq. 2 (residual form); CORAL-KV, Sec. 2 (per-head codebooks fitted
// online per cache block); NanoKV page, Table 4 (two k-means iterations, BF16
// centres, packed INT2 residuals).
//
// Arithmetic contract (bit-exact with the independent CPU oracle):
//  - distance: binary32, channel 0 first, e = x - mu, acc = acc + e*e, every
//    operation separately rounded (__fsub_rn/__fmul_rn/__fadd_rn, no FMA);
//    strict '<' over increasing centroid index, so ties keep the lowest index;
//  - group min/max by strict comparisons in channel order; s = (mx-mn)/(2^b-1),
//    inv = 1/s, z = rint(-mn*inv), q = clamp(rint(r*inv) + z, 0, 2^b-1);
//    zero-range or underflowing (s < FLT_MIN) groups: s = |mn|, z = -sign(mn),
//    q = 0;
//  - reconstruction x^ = mu + (q - z)*s, three separately rounded operations.
#pragma once

#include <float.h>
#include <limits.h>

#include "common.cuh"

namespace kvq {

struct GroupQ {
    float s, z, inv;
    bool degenerate;
};

// Eq. 1 parameters of one group given its exact min and max.
__device__ __forceinline__ GroupQ group_params(float mn, float mx, int bits)
{
    const float qmax = (float)((1 << bits) - 1);
    GroupQ g;
    g.degenerate = true;
    g.inv = 0.0f;
    float s = 0.0f;
    if (mx != mn)
        s = __fdiv_rn(__fsub_rn(mx, mn), qmax);
    if (mx == mn || !(s >= FLT_MIN)) {
        if (mn == 0.0f) {
            g.s = 0.0f;
            g.z = 0.0f;
        } else {
            g.s = fabsf(mn);
            g.z = (mn > 0.0f) ? -1.0f : 1.0f;
        }
        return g;
    }
    g.degenerate = false;
    g.s = s;
    g.inv = __fdiv_rn(1.0f, s);
    g.z = rintf(__fmul_rn(-mn, g.inv));
    return g;
}

__device__ __forceinline__ uint32_t quant_code(float r, const GroupQ &g, int bits)
{
    if (g.degenerate)
        return 0u;
    const float qmax = (float)((1 << bits) - 1);
    float v = __fadd_rn(rintf(__fmul_rn(r, g.inv)), g.z);
    if (v < 0.0f)
        v = 0.0f;
    if (v > qmax)
        v = qmax;
    return (uint32_t)v;
}

// binary32 -> binary16 bits: round to nearest, ties to even, saturating at
// the largest finite value (cvt .satfinite); and back (exact).
__device__ __forceinline__ uint16_t f16_round_sat(float f)
{
    uint32_t r;
    asm("cvt.rn.satfinite.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(0.0f), "f"(f));
    return (uint16_t)(r & 0xffffu);
}

__device__ __forceinline__ float f16_widen(uint32_t h)
{
    float f;
    asm("{\n\t.reg .b16 t;\n\tcvt.u16.u32 t, %1;\n\tcvt.f32.f16 %0, t;\n\t}" : "=f"(f) : "r"(h & 0xffffu));
    return f;
}

// Eq. 1 parameters with compact 16-bit {s, z}: s rounded to binary16, 1/s and
// z formed from the rounded scale, z rounded to binary16; the returned s and
// z are the stored values widened, and *packed = s16 | z16 << 16.  A group
// whose scale rounds to zero is stored as degenerate.
__device__ __forceinline__ GroupQ group_params16(float mn, float mx, int bits, uint32_t *packed)
{
    const float qmax = (float)((1 << bits) - 1);
    GroupQ g;
    g.degenerate = true;
    g.inv = 0.0f;
    float s = 0.0f;
    if (mx != mn)
        s = __fdiv_rn(__fsub_rn(mx, mn), qmax);
    const uint16_t sh = f16_round_sat(s);
    if (mx == mn || !(s >= FLT_MIN) || (sh & 0x7fffu) == 0u) {
        if (mn == 0.0f) {
            g.s = 0.0f;
            g.z = 0.0f;
            *packed = 0u;
        } else {
            const uint16_t ah = f16_round_sat(fabsf(mn));
            const uint16_t zh = (mn > 0.0f) ? 0xbc00u : 0x3c00u;
            g.s = f16_widen(ah);
            g.z = (mn > 0.0f) ? -1.0f : 1.0f;
            *packed = (uint32_t)ah | ((uint32_t)zh << 16);
        }
        return g;
    }
    g.degenerate = false;
    g.s = f16_widen(sh);
    g.inv = __fdiv_rn(1.0f, g.s);
    const uint16_t zh = f16_round_sat(rintf(__fmul_rn(-mn, g.inv)));
    g.z = f16_widen(zh);
    *packed = (uint32_t)sh | ((uint32_t)zh << 16);
    return g;
}

// Eq. 1 parameters of a group in the storage format (meta16: compact
// 16-bit {s, z}), stored at group index g of this token-head's meta row.
__device__ __forceinline__ GroupQ group_params_store(float mn, float mx, int bits, bool meta16, void *meta_row, int g)
{
    if (meta16) {
        uint32_t packed;
        const GroupQ gq = group_params16(mn, mx, bits, &packed);
        static_cast<uint32_t *>(meta_row)[g] = packed;
        return gq;
    }
    const GroupQ gq = group_params(mn, mx, bits);
    static_cast<float2 *>(meta_row)[g] = make_float2(gq.s, gq.z);
    return gq;
}

// {s, z} of group g of a meta row in either storage format, as binary32.
__device__ __forceinline__ float2 load_sz(const void *meta_row, int g, bool meta16)
{
    if (meta16) {
        const uint32_t w = static_cast<const uint32_t *>(meta_row)[g];
        return make_float2(f16_widen(w), f16_widen(w >> 16));
    }
    return static_cast<const float2 *>(meta_row)[g];
}

// Eq. 1 codes of a group whose every |r * inv| is below 2^22 (checked once
// per group), without the conversion unit: t + 1.5 2^23 rounds t to the
// nearest integer, ties to even -- rint(t) -- in the low significand bits, so
// rint(t) + z is an integer add on those bits.  Equal to quant_code.
struct GroupFast {
    float inv;
    int zoff;  // z - bits(1.5 2^23)
    bool fast;
};

__device__ __forceinline__ GroupFast group_fast(const GroupQ &g, float mn, float mx)
{
    GroupFast f;
    f.inv = g.inv;
    f.fast = !g.degenerate && __fmul_rn(fmaxf(fabsf(mn), fabsf(mx)), g.inv) < 4194304.0f;
    f.zoff = f.fast ? (int)g.z - 0x4B400000 : 0;
    return f;
}

template <int BITS>
__device__ __forceinline__ uint32_t quant_code_fast(float r, const GroupFast &f)
{
    const int v = __float_as_int(__fadd_rn(__fmul_rn(r, f.inv), 12582912.0f)) + f.zoff;
    return (uint32_t)min(max(v, 0), (1 << BITS) - 1);
}

// Codes of the G values r[0..G) of one group, added (the bit fields are
// disjoint) into words at channel offset c0 (low bits first).
template <int G, int BITS>
__device__ __forceinline__ void quant_group_into(const float *r, const GroupQ &g, float mn, float mx, uint32_t *words,
                                                 int c0)
{
    constexpr int kPerWord = 32 / BITS;
    const GroupFast f = group_fast(g, mn, mx);
    if (f.fast) {
#pragma unroll
        for (int c = 0; c < G; ++c)
            words[(c0 + c) / kPerWord] += quant_code_fast<BITS>(r[c], f) << (((c0 + c) % kPerWord) * BITS);
    } else {
#pragma unroll
        for (int c = 0; c < G; ++c)
            words[(c0 + c) / kPerWord] += quant_code(r[c], g, BITS) << (((c0 + c) % kPerWord) * BITS);
    }
}

__device__ __forceinline__ float dequant_spec(uint32_t q, float s, float z, float mu)
{
    return __fadd_rn(mu, __fmul_rn(__fsub_rn((float)q, z), s));
}

// Load 8 consecutive history values (one 16-byte bf16 unit or two float4s).
__device__ __forceinline__ void load_x8(const void *x, bool x_bf16, int64_t elem, float *out)
{
    if (x_bf16) {
        const uint4 w = __ldg(reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(x) + elem));
        out[0] = bf16_lo(w.x); out[1] = bf16_hi(w.x);
        out[2] = bf16_lo(w.y); out[3] = bf16_hi(w.y);
        out[4] = bf16_lo(w.z); out[5] = bf16_hi(w.z);
        out[6] = bf16_lo(w.w); out[7] = bf16_hi(w.w);
    } else {
        const float4 a = __ldg(reinterpret_cast<const float4 *>(static_cast<const float *>(x) + elem));
        const float4 b = __ldg(reinterpret_cast<const float4 *>(static_cast<const float *>(x) + elem + 4));
        out[0] = a.x; out[1] = a.y; out[2] = a.z; out[3] = a.w;
        out[4] = b.x; out[5] = b.y; out[6] = b.z; out[7] = b.w;
    }
}

__device__ __forceinline__ void load_bf16x8(const uint16_t *p, float *out)
{
    const uint4 w = __ldg(reinterpret_cast<const uint4 *>(p));
    out[0] = bf16_lo(w.x); out[1] = bf16_hi(w.x);
    out[2] = bf16_lo(w.y); out[3] = bf16_hi(w.y);
    out[4] = bf16_lo(w.z); out[5] = bf16_hi(w.z);
    out[6] = bf16_lo(w.w); out[7] = bf16_hi(w.w);
}

// Quantise a residual row of D channels held in registers: per group of G
// channels the Eq. 1 parameters, then packed codes (low bits first) and the
// {s, z} pairs.  codes_row must be 16-byte aligned (D*BITS/8 is 16, 32 or 64).
// ERR: also replace every r_c by the error this stage leaves,
// r_c - (q_c - z) s (binary32; the input of a second residual stage).
template <int D, int BITS, int G, bool ERR = false>
__device__ __forceinline__ void encode_residual_row(float *r, uint8_t *codes_row, void *meta_row, bool meta16)
{
    constexpr int kWords = D * BITS / 32;
    uint32_t words[kWords];
#pragma unroll
    for (int w = 0; w < kWords; ++w)
        words[w] = 0u;
#pragma unroll
    for (int g = 0; g < D / G; ++g) {
        float mn = r[g * G], mx = r[g * G];
#pragma unroll
        for (int c = g * G + 1; c < (g + 1) * G; ++c) {
            if (r[c] < mn) mn = r[c];
            if (r[c] > mx) mx = r[c];
        }
        const GroupQ gq = group_params_store(mn, mx, BITS, meta16, meta_row, g);
        quant_group_into<G, BITS>(r + g * G, gq, mn, mx, words, g * G);
        if constexpr (ERR) {
#pragma unroll
            for (int c = g * G; c < (g + 1) * G; ++c)
                r[c] = __fsub_rn(r[c], __fmul_rn(__fsub_rn((float)quant_code(r[c], gq, BITS), gq.z), gq.s));
        }
    }
    uint4 *dst = reinterpret_cast<uint4 *>(codes_row);
#pragma unroll
    for (int v = 0; v < kWords / 4; ++v)
        dst[v] = make_uint4(words[4 * v], words[4 * v + 1], words[4 * v + 2], words[4 * v + 3]);
}

// ---------------------------------------------------------------------------
// Exact assignment + residual quantisation on CUDA cores.
// One thread per token; a block covers 128 tokens of one head and streams
// the head's centres through shared memory (binary32) in chunks.
// ---------------------------------------------------------------------------
constexpr int kDirectTokens = 128;
constexpr int kDirectChunk = 64;  // centres per shared-memory chunk

struct EncodeArgs {
    const void *x;
    int x_bf16;
    int64_t T;
    int H;
    int C;
    int bits;
    int G;
    const uint16_t *cent;  // [H][C][D] bf16
    uint16_t *idx;         // [H][T]
    uint8_t *codes;        // [H][T][D*bits/8] (may be null when assign_only)
    void *meta;            // [H][T][D/G][2] float, or binary16 when meta16
    int assign_only;
    int meta16;
    uint8_t *codes2;       // second residual stage: as codes,
    float *meta2;          // and as meta (binary32); NULL: one stage
};

template <int D, int BITS, int G>
__global__ void __launch_bounds__(kDirectTokens) encode_direct_kernel(EncodeArgs a)
{
    __shared__ __align__(16) float s_mu[kDirectChunk * D];
    const int h = blockIdx.y;
    const int64_t t = (int64_t)blockIdx.x * kDirectTokens + threadIdx.x;
    const bool active = t < a.T;

    float xr[D];
    if (active) {
#pragma unroll
        for (int c = 0; c < D; c += 8)
            load_x8(a.x, a.x_bf16, (t * a.H + h) * D + c, xr + c);
    } else {
#pragma unroll
        for (int c = 0; c < D; ++c)
            xr[c] = 0.0f;
    }

    const uint16_t *cent_h = a.cent + (int64_t)h * a.C * D;
    float best = 0.0f;
    int best_j = 0;
    for (int j0 = 0; j0 < a.C; j0 += kDirectChunk) {
        const int nj = min(kDirectChunk, a.C - j0);
        __syncthreads();
        for (int e = threadIdx.x * 8; e < nj * D; e += kDirectTokens * 8)
            load_bf16x8(cent_h + (int64_t)j0 * D + e, s_mu + e);
        __syncthreads();
        if (active) {
            // four centres at a time: four independent sequential sums keep
            // the adders busy (each sum alone is one dependent chain of D adds)
            for (int jq = 0; jq < nj; jq += 4) {
                float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
                for (int c4 = 0; c4 < D / 4; ++c4) {
                    const float2 x01 = make_float2(xr[4 * c4], xr[4 * c4 + 1]);
                    const float2 x23 = make_float2(xr[4 * c4 + 2], xr[4 * c4 + 3]);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        // rows past nj hold stale centres of the chunk buffer; their sums are dropped
                        const float4 m = reinterpret_cast<const float4 *>(s_mu + (jq + q) * D)[c4];
                        // e_c e_c of two channels at a time (packed binary32
                        // operations round each lane as the scalar ones do),
                        // summed in channel order
                        const float2 e01 = sub2(x01, make_float2(m.x, m.y));
                        const float2 e23 = sub2(x23, make_float2(m.z, m.w));
                        const float2 q01 = mul2(e01, e01), q23 = mul2(e23, e23);
                        acc[q] = __fadd_rn(acc[q], q01.x);
                        acc[q] = __fadd_rn(acc[q], q01.y);
                        acc[q] = __fadd_rn(acc[q], q23.x);
                        acc[q] = __fadd_rn(acc[q], q23.y);
                    }
                }
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int j = j0 + jq + q;
                    if (jq + q < nj && (j == 0 || acc[q] < best)) {
                        best = acc[q];
                        best_j = j;
                    }
                }
            }
        }
    }
    if (!active)
        return;
    a.idx[(int64_t)h * a.T + t] = (uint16_t)best_j;
    if (a.assign_only)
        return;

    // residual r = x - mu[best] (binary32), overwriting xr
    const uint16_t *mu_row = cent_h + (int64_t)best_j * D;
#pragma unroll
    for (int c = 0; c < D; c += 8) {
        float m8[8];
        load_bf16x8(mu_row + c, m8);
#pragma unroll
        for (int k = 0; k < 8; ++k)
            xr[c + k] = __fsub_rn(xr[c + k], m8[k]);
    }
    const int64_t th = (int64_t)h * a.T + t;
    if (a.codes2) {
        // two residual stages: the error stage 1 leaves, quantised again
        encode_residual_row<D, BITS, G, true>(xr, a.codes + th * (D * BITS / 8),
                                              static_cast<uint8_t *>(a.meta) + th * (D / G) * 8, false);
        encode_residual_row<D, BITS, G>(xr, a.codes2 + th * (D * BITS / 8), a.meta2 + th * (D / G) * 2, false);
    } else {
        encode_residual_row<D, BITS, G>(xr, a.codes + th * (D * BITS / 8),
                                        static_cast<uint8_t *>(a.meta) + th * (D / G) * (a.meta16 ? 4 : 8),
                                        a.meta16 != 0);
    }
}

// ---------------------------------------------------------------------------
// QSAC (QuantWM, Sec. 4.1): query-sensitive centre selection, exact on CUDA
// cores.  One thread per token; a block covers 128 tokens of one head and
// streams the head's centres through shared memory (binary32) in chunks.
//  - weighted distance sum_c w_c ((x_c - mu_c)^2), every operation rounded
//    separately in channel order; the M smallest by (distance, index) are
//    kept (strict comparisons while scanning centres in index order);
//  - score of each candidate: sum over groups of W_g R_g^2, W_g the sum of
//    the group's w_c in channel order, R_g = max - min of the group's
//    residual (strict scans); the lowest score wins, ties to the better-
//    ranked candidate (QuantWM, Table 11: M = 4; the Widrow factor
//    1 / (12 (2^b - 1)^2) is common to all candidates and dropped);
//  - the chosen centre's residual is quantised exactly as the plain encode.
// ---------------------------------------------------------------------------
constexpr int kQsacMaxM = 8;

struct QsacArgs {
    EncodeArgs e;     // history, centres, outputs (assign_only unused)
    const float *w;   // [H][D] channel weights, binary32
    int M;            // candidates, 1 .. kQsacMaxM
};

template <int D, int BITS, int G>
__global__ void __launch_bounds__(kDirectTokens) qsac_encode_kernel(QsacArgs q)
{
    const EncodeArgs &a = q.e;
    __shared__ __align__(16) float s_mu[kDirectChunk * D];
    __shared__ __align__(16) float s_w[D];
    const int h = blockIdx.y;
    const int64_t t = (int64_t)blockIdx.x * kDirectTokens + threadIdx.x;
    const bool active = t < a.T;
    for (int c = threadIdx.x; c < D; c += kDirectTokens)
        s_w[c] = q.w[(int64_t)h * D + c];

    float xr[D];
    if (active) {
#pragma unroll
        for (int c = 0; c < D; c += 8)
            load_x8(a.x, a.x_bf16, (t * a.H + h) * D + c, xr + c);
    } else {
#pragma unroll
        for (int c = 0; c < D; ++c)
            xr[c] = 0.0f;
    }
    const int m = q.M < a.C ? q.M : a.C;
    float cd[kQsacMaxM];
    int cand[kQsacMaxM];
#pragma unroll
    for (int k = 0; k < kQsacMaxM; ++k) {
        cd[k] = INFINITY;
        cand[k] = -1;
    }
    const uint16_t *cent_h = a.cent + (int64_t)h * a.C * D;
    for (int j0 = 0; j0 < a.C; j0 += kDirectChunk) {
        const int nj = min(kDirectChunk, a.C - j0);
        __syncthreads();
        for (int e = threadIdx.x * 8; e < nj * D; e += kDirectTokens * 8)
            load_bf16x8(cent_h + (int64_t)j0 * D + e, s_mu + e);
        __syncthreads();
        if (active) {
            for (int jj = 0; jj < nj; ++jj) {
                const float4 *mu4 = reinterpret_cast<const float4 *>(s_mu + jj * D);
                const float4 *w4 = reinterpret_cast<const float4 *>(s_w);
                // the terms w_c (e_c e_c) of two channels at a time (packed
                // binary32 operations round each lane as the scalar ones do),
                // summed one by one in channel order
                float acc = 0.0f;
#pragma unroll
                for (int c4 = 0; c4 < D / 4; ++c4) {
                    const float4 mv = mu4[c4], wv = w4[c4];
                    const float2 e01 = sub2(make_float2(xr[4 * c4], xr[4 * c4 + 1]), make_float2(mv.x, mv.y));
                    const float2 e23 = sub2(make_float2(xr[4 * c4 + 2], xr[4 * c4 + 3]), make_float2(mv.z, mv.w));
                    const float2 t01 = mul2(make_float2(wv.x, wv.y), mul2(e01, e01));
                    const float2 t23 = mul2(make_float2(wv.z, wv.w), mul2(e23, e23));
                    acc = __fadd_rn(acc, t01.x);
                    acc = __fadd_rn(acc, t01.y);
                    acc = __fadd_rn(acc, t23.x);
                    acc = __fadd_rn(acc, t23.y);
                }
                const int j = j0 + jj;
                // insert (acc, j) into the ascending lists (an empty slot
                // takes any value, infinite ones included); equal distances
                // keep the earlier (lower-index) entry first
#pragma unroll
                for (int k = kQsacMaxM - 1; k >= 1; --k) {
                    if (k < m) {
                        if (acc < cd[k - 1]) {
                            cd[k] = cd[k - 1];
                            cand[k] = cand[k - 1];
                        } else if (cand[k - 1] >= 0 && (cand[k] < 0 || acc < cd[k])) {
                            cd[k] = acc;
                            cand[k] = j;
                        }
                    }
                }
                if (cand[0] < 0 || acc < cd[0]) {
                    cd[0] = acc;
                    cand[0] = j;
                }
            }
        }
    }
    if (!active)
        return;
    // scores of the candidates; the group weights do not depend on the centre
    float wg[D / G];
#pragma unroll
    for (int g = 0; g < D / G; ++g) {
        float acc = 0.0f;
#pragma unroll
        for (int c = g * G; c < (g + 1) * G; ++c)
            acc = __fadd_rn(acc, s_w[c]);
        wg[g] = acc;
    }
    int choice = cand[0] < 0 ? 0 : cand[0];
    float best = 0.0f;
#pragma unroll
    for (int k = 0; k < kQsacMaxM; ++k) {
        if (k < m && cand[k] >= 0) {
            const uint16_t *mu_row = cent_h + (int64_t)cand[k] * D;
            float score = 0.0f;
#pragma unroll
            for (int g = 0; g < D / G; ++g) {
                float lo = 0.0f, hi = 0.0f;
#pragma unroll
                for (int c = g * G; c < (g + 1) * G; c += 8) {
                    float m8[8];
                    load_bf16x8(mu_row + c, m8);
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        const float r = __fsub_rn(xr[c + kk], m8[kk]);
                        if (c + kk == g * G) {
                            lo = r;
                            hi = r;
                        } else {
                            if (r < lo) lo = r;
                            if (r > hi) hi = r;
                        }
                    }
                }
                const float range = __fsub_rn(hi, lo);
                score = __fadd_rn(score, __fmul_rn(wg[g], __fmul_rn(range, range)));
            }
            if (k == 0 || score < best) {
                best = score;
                choice = cand[k];
            }
        }
    }
    a.idx[(int64_t)h * a.T + t] = (uint16_t)choice;
    // residual against the chosen centre, quantised as the plain encode does
    const uint16_t *mu_row = cent_h + (int64_t)choice * D;
#pragma unroll
    for (int c = 0; c < D; c += 8) {
        float m8[8];
        load_bf16x8(mu_row + c, m8);
#pragma unroll
        for (int k = 0; k < 8; ++k)
            xr[c + k] = __fsub_rn(xr[c + k], m8[k]);
    }
    const int64_t th = (int64_t)h * a.T + t;
    encode_residual_row<D, BITS, G>(xr, a.codes + th * (D * BITS / 8),
                                    static_cast<uint8_t *>(a.meta) + th * (D / G) * (a.meta16 ? 4 : 8), a.meta16 != 0);
}

// ---------------------------------------------------------------------------
// Per-head reconstruction: one thread per 8 channels of a token-head.
// ---------------------------------------------------------------------------
struct DecodeArgs {
    const uint16_t *cent;
    const uint16_t *idx;
    const uint8_t *codes;
    const void *meta;
    int64_t T;
    int H;
    int D;
    int C;
    int bits;
    int G;
    void *out;
    int out_bf16;
    int meta16;
    const uint8_t *codes2;  // second residual stage (binary32 {s, z} only); NULL: one stage
    const float *meta2;
};

// One block per (tile of 256 / (D/8) tokens, head); thread = 8 channels of
// one token: the encoded rows of the head are read contiguously and every
// token-head's output row is one contiguous run of D values.
template <int D>
__global__ void __launch_bounds__(256) decode_kernel(DecodeArgs a)
{
    constexpr int kUnits = D / 8;
    constexpr int kTokens = 256 / kUnits;
    const int u = threadIdx.x % kUnits;
    const int64_t t = (int64_t)blockIdx.x * kTokens + threadIdx.x / kUnits;
    const int h = blockIdx.y;
    if (t >= a.T)
        return;
    const int64_t th = (int64_t)h * a.T + t;  // encoded-row index
    int j = a.idx[th];
    if (j >= a.C) {
        raise_status(DEVSTAT_BAD_INDEX);
        j = 0;
    }
    const int c0 = u * 8;
    const float2 sz = load_sz(static_cast<const uint8_t *>(a.meta) + th * (D / a.G) * (a.meta16 ? 4 : 8), c0 / a.G,
                              a.meta16 != 0);
    uint32_t cw;
    if (a.bits == 2)
        cw = *reinterpret_cast<const uint16_t *>(a.codes + th * (D / 4) + c0 / 4);
    else
        cw = *reinterpret_cast<const uint32_t *>(a.codes + th * (D / 2) + c0 / 2);
    float mu[8];
    load_bf16x8(a.cent + ((int64_t)h * a.C + j) * D + c0, mu);
    const uint32_t mask = (1u << a.bits) - 1u;
    float v[8];
    if (fabsf(sz.y) < 4194304.0f) {
        // q - z = (2^23 + q) - (2^23 + z), both terms and the difference exact:
        // the same value dequant_spec forms, without the int -> float convert
        const float zz = __fadd_rn(8388608.0f, sz.y);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const float d = __fsub_rn(__uint_as_float(0x4B000000u | ((cw >> (k * a.bits)) & mask)), zz);
            v[k] = __fadd_rn(mu[k], __fmul_rn(d, sz.x));
        }
    } else {
#pragma unroll
        for (int k = 0; k < 8; ++k)
            v[k] = dequant_spec((cw >> (k * a.bits)) & mask, sz.x, sz.y, mu[k]);
    }
    if (a.codes2) {  // + (q2 - z2) s2
        const float2 sz2 = reinterpret_cast<const float2 *>(a.meta2)[th * (D / a.G) + c0 / a.G];
        const uint32_t cw2 = a.bits == 2 ? *reinterpret_cast<const uint16_t *>(a.codes2 + th * (D / 4) + c0 / 4)
                                         : *reinterpret_cast<const uint32_t *>(a.codes2 + th * (D / 2) + c0 / 2);
#pragma unroll
        for (int k = 0; k < 8; ++k)
            v[k] = __fadd_rn(v[k], __fmul_rn(__fsub_rn((float)((cw2 >> (k * a.bits)) & mask), sz2.y), sz2.x));
    }
    const int64_t o = (t * a.H + h) * D + c0;
    if (a.out_bf16) {
        uint4 w = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                             pack_bf16x2(v[6], v[7]));
        *reinterpret_cast<uint4 *>(static_cast<uint16_t *>(a.out) + o) = w;
    } else {
        float *dst = static_cast<float *>(a.out) + o;
        *reinterpret_cast<float4 *>(dst) = make_float4(v[0], v[1], v[2], v[3]);
        *reinterpret_cast<float4 *>(dst + 4) = make_float4(v[4], v[5], v[6], v[7]);
    }
}

// ---------------------------------------------------------------------------
// PSAC coefficients (QuantWM, Sec. 4.2: principal query-subspace attention
// correction): C[t][h] = (x - x^)[t][h] U_h, the part of the key's
// reconstruction error along the r = 8 leading eigenvectors of the head's
// query second-moment matrix.  One thread per token-head; x^ is formed as
// decode_kernel forms it (binary32), e = x - x^ in binary32, the r dot
// products accumulate in binary32 FMAs in channel order.
// ---------------------------------------------------------------------------
constexpr int kPsacRank = 8;

struct PsacCoefArgs {
    DecodeArgs d;     // the compressed K history (out / out_bf16 unused)
    const void *x;    // original keys [T][H][D], float or bf16
    int x_bf16;
    const float *U;   // [H][D][8]
    float *coef;      // [H][T][8]
};

template <int D>
__global__ void __launch_bounds__(128) psac_coef_kernel(PsacCoefArgs p)
{
    const DecodeArgs &a = p.d;
    __shared__ __align__(16) float sU[D * kPsacRank];
    const int h = blockIdx.y;
    for (int e = threadIdx.x; e < D * kPsacRank; e += 128)
        sU[e] = p.U[(int64_t)h * D * kPsacRank + e];
    __syncthreads();
    const int64_t t = (int64_t)blockIdx.x * 128 + threadIdx.x;
    if (t >= a.T)
        return;
    const int64_t th = (int64_t)h * a.T + t;
    int j = a.idx[th];
    if (j >= a.C) {
        raise_status(DEVSTAT_BAD_INDEX);
        j = 0;
    }
    const uint8_t *meta_row = static_cast<const uint8_t *>(a.meta) + th * (D / a.G) * (a.meta16 ? 4 : 8);
    const uint32_t mask = (1u << a.bits) - 1u;
    float acc[kPsacRank];
#pragma unroll
    for (int r = 0; r < kPsacRank; ++r)
        acc[r] = 0.0f;
#pragma unroll 1
    for (int c0 = 0; c0 < D; c0 += 8) {
        const float2 sz = load_sz(meta_row, c0 / a.G, a.meta16 != 0);
        uint32_t cw;
        if (a.bits == 2)
            cw = *reinterpret_cast<const uint16_t *>(a.codes + th * (D / 4) + c0 / 4);
        else
            cw = *reinterpret_cast<const uint32_t *>(a.codes + th * (D / 2) + c0 / 2);
        float mu[8], xv[8];
        load_bf16x8(a.cent + ((int64_t)h * a.C + j) * D + c0, mu);
        load_x8(p.x, p.x_bf16, (t * a.H + h) * D + c0, xv);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const float xh = dequant_spec((cw >> (k * a.bits)) & mask, sz.x, sz.y, mu[k]);
            const float e = __fsub_rn(xv[k], xh);
            const float4 u0 = *reinterpret_cast<const float4 *>(sU + (c0 + k) * kPsacRank);
            const float4 u1 = *reinterpret_cast<const float4 *>(sU + (c0 + k) * kPsacRank + 4);
            acc[0] = fmaf(e, u0.x, acc[0]);
            acc[1] = fmaf(e, u0.y, acc[1]);
            acc[2] = fmaf(e, u0.z, acc[2]);
            acc[3] = fmaf(e, u0.w, acc[3]);
            acc[4] = fmaf(e, u1.x, acc[4]);
            acc[5] = fmaf(e, u1.y, acc[5]);
            acc[6] = fmaf(e, u1.z, acc[6]);
            acc[7] = fmaf(e, u1.w, acc[7]);
        }
    }
    float4 *dst = reinterpret_cast<float4 *>(p.coef + th * kPsacRank);
    dst[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
    dst[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
}

// ---------------------------------------------------------------------------
// k-means fitting: seeding, binary64 accumulation, update
// ---------------------------------------------------------------------------
struct FitArgs {
    const void *x;
    int x_bf16;
    int64_t T;
    int H;
    int D;
    int C;
    uint16_t *cent;  // [H][C][D]
};

// ---------------------------------------------------------------------------
// Deterministic centre update.  The specification sums every centre's tokens
// sequentially in token order in binary64.  That sum is exact -- and then
// equal to the sum in any order -- whenever every value is a multiple of 2^L
// and every partial sum stays below 2^(53 + L) in magnitude: all partial sums
// are then integers times 2^L representable in 53 bits.  With A the largest
// |x| of the head and n the centre's token count, n A <= 2^(52 + L) suffices;
// L is bounded below by the exponent of the smallest nonzero |x| of the head
// less 134 (bf16 values: 8 significant bits) or 150 (binary32).  So:
//   fit_hist:    per (head, token chunk) centre counts            [H][C][nch]
//   fit_scan:    per (head, centre), per-chunk bases and totals    [H][C][nch], [H][C]
//   fit_starts:  per head, bucket starts (prefix of the totals)    [H][C+1]
//   fit_scatter: per (head, chunk), stable placement of token ids  order[H][T]
//                and of their centres                               order_j[H][T]
//   fit_segsum:  one warp per 64 consecutive slots of the sorted order: per
//                run of one centre, binary64 sums per channel, added to the
//                centre's totals with atomics (exact sums are order
//                independent); in the first round also the head's largest
//                and smallest nonzero |x|
//   fit_finalize: one warp per (head, centre): if n A <= 2^(52 + L) the sums
//                are exact: mean in binary64, binary32, then bf16 (empty:
//                keep); otherwise the centre is marked for
//   fit_bucket_update: the sequential token-order sum (marked centres only).
// ---------------------------------------------------------------------------
constexpr int kFitChunk = 256;
constexpr int kFitSegSlots = 64;

struct FitSortArgs {
    const void *x;
    int x_bf16;
    int64_t T;
    int H;
    int D;
    int C;
    int nchunks;
    uint16_t *cent;          // [H][C][D]
    const uint16_t *idx;     // [H][T]
    int *chunk_counts;       // [H][C][nchunks] (counts, then bases)
    int *bucket_start;       // [H][C + 1]
    int *order;              // [H][T]
    uint16_t *order_j;       // [H][T] centre of each slot of order
    double *sums;            // [H][C][D]
    unsigned *abs_max;       // [H] bits of the largest |x|
    unsigned *abs_min;       // [H] bits of the smallest nonzero |x| (+inf: none)
    int *redo;               // [H][C]
    int track;               // segsum also updates abs_max / abs_min
    unsigned *bkt_max;       // [H][C] bits of the largest |x| of the round's bucket
    unsigned *bkt_minv;      // [H][C] ~bits of its smallest nonzero |x| (0: none)
};

// mu_j = bf16(x_j) for the first C tokens; the update totals start cleared.
__global__ void __launch_bounds__(256) fit_seed_kernel(FitArgs a, FitSortArgs fs)
{
    const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t total = (int64_t)a.H * a.C * a.D;
    if (gid >= total)
        return;
    const int c = (int)(gid % a.D);
    const int64_t hj = gid / a.D;
    const int j = (int)(hj % a.C);
    const int h = (int)(hj / a.C);
    const int64_t e = ((int64_t)j * a.H + h) * a.D + c;
    float v = a.x_bf16 ? __uint_as_float((uint32_t)static_cast<const uint16_t *>(a.x)[e] << 16)
                       : static_cast<const float *>(a.x)[e];
    const __nv_bfloat16 b = __float2bfloat16_rn(v);
    a.cent[gid] = *reinterpret_cast<const uint16_t *>(&b);
    fs.sums[gid] = 0.0;
    if (c == 0) {
        fs.redo[hj] = 0;
        fs.bkt_max[hj] = 0u;
        fs.bkt_minv[hj] = 0u;
    }
    if (c == 0 && j == 0) {
        fs.abs_max[h] = 0u;
        fs.abs_min[h] = 0x7f800000u;
    }
}

__global__ void __launch_bounds__(256) fit_hist_kernel(FitSortArgs a)
{
    extern __shared__ int s_cnt[];  // [C]
    const int h = blockIdx.y, ch = blockIdx.x;
    for (int j = threadIdx.x; j < a.C; j += blockDim.x)
        s_cnt[j] = 0;
    __syncthreads();
    const int64_t t0 = (int64_t)ch * kFitChunk;
    const int64_t t1 = min(a.T, t0 + kFitChunk);
    for (int64_t t = t0 + threadIdx.x; t < t1; t += blockDim.x)
        atomicAdd(&s_cnt[a.idx[(int64_t)h * a.T + t]], 1);
    __syncthreads();
    int *dst = a.chunk_counts + (int64_t)h * a.C * a.nchunks + ch;
    for (int j = threadIdx.x; j < a.C; j += blockDim.x)
        dst[(int64_t)j * a.nchunks] = s_cnt[j];
}

// One warp per (head, centre): the centre's chunk counts become chunk bases
// (prefix over chunks) and its total goes to bucket_start[h][j] (turned into
// bucket starts by fit_starts_kernel).
__global__ void __launch_bounds__(256) fit_scan_kernel(FitSortArgs a)
{
    const int lane = threadIdx.x & 31;
    const int j = blockIdx.x * 8 + (threadIdx.x >> 5), h = blockIdx.y;
    if (j >= a.C)
        return;
    int *row = a.chunk_counts + ((int64_t)h * a.C + j) * a.nchunks;
    int run = 0;
    for (int c0 = 0; c0 < a.nchunks; c0 += 32) {
        const int c = c0 + lane;
        const int v = c < a.nchunks ? row[c] : 0;
        int incl = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o)
                incl += n;
        }
        if (c < a.nchunks)
            row[c] = run + incl - v;
        run += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0)
        a.bucket_start[(int64_t)h * (a.C + 1) + j] = run;
}

// One block (1024 threads) per head: exclusive prefix of the centre totals
// in bucket_start[h][0..C) in place, total in bucket_start[h][C].
__global__ void __launch_bounds__(1024) fit_starts_kernel(FitSortArgs a)
{
    __shared__ int s_warp[32];
    const int h = blockIdx.x, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int *bs = a.bucket_start + (int64_t)h * (a.C + 1);
    // thread k owns entries [k per, (k + 1) per)
    const int per = (a.C + 1023) / 1024;
    const int j0 = threadIdx.x * per, j1 = min(a.C, j0 + per);
    int local = 0;
    for (int j = j0; j < j1; ++j)
        local += bs[j];
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o)
            incl += n;
    }
    if (lane == 31)
        s_warp[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int v = s_warp[lane];
        int wi = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o)
                wi += n;
        }
        s_warp[lane] = wi - v;
    }
    __syncthreads();
    int run = s_warp[warp] + incl - local;
    for (int j = j0; j < j1; ++j) {
        const int t = bs[j];
        bs[j] = run;
        run += t;
    }
    if (threadIdx.x == 1023)
        bs[a.C] = run;
}

// One warp per (head, chunk): tokens in order, 32 at a time; lanes holding the
// same centre get consecutive slots in lane order, so every bucket lists its
// tokens in increasing token order.
__global__ void __launch_bounds__(32) fit_scatter_kernel(FitSortArgs a)
{
    extern __shared__ int s_cur[];  // [C] running offset of each centre in this chunk
    const int h = blockIdx.y, ch = blockIdx.x, lane = threadIdx.x;
    const int *base = a.chunk_counts + (int64_t)h * a.C * a.nchunks + ch;
    const int *bs = a.bucket_start + (int64_t)h * (a.C + 1);
    for (int j = lane; j < a.C; j += 32)
        s_cur[j] = bs[j] + base[(int64_t)j * a.nchunks];
    __syncwarp();
    const int64_t t0 = (int64_t)ch * kFitChunk;
    const int64_t t1 = min(a.T, t0 + kFitChunk);
    for (int64_t tb = t0; tb < t1; tb += 32) {
        const int64_t t = tb + lane;
        const bool on = t < t1;
        const int j = on ? (int)a.idx[(int64_t)h * a.T + t] : -1;
        const unsigned peers = __match_any_sync(0xffffffffu, j);
        const int rank = __popc(peers & ((1u << lane) - 1u));
        const int leader = __ffs(peers) - 1;
        int slot = 0;
        if (on)
            slot = s_cur[j] + rank;
        __syncwarp();
        if (on && lane == leader)
            s_cur[j] += __popc(peers);
        __syncwarp();
        if (on) {
            a.order[(int64_t)h * a.T + slot] = (int)t;
            a.order_j[(int64_t)h * a.T + slot] = (uint16_t)j;
        }
    }
}

// Lane l owns channels kPer l .. kPer l + kPer - 1 of token t.
template <int D>
__device__ __forceinline__ void fit_load_row(const FitSortArgs &a, int h, int64_t t, int lane, float *v)
{
    constexpr int kPer = D / 32;
    const int64_t e = (t * a.H + h) * D + lane * kPer;
    if (a.x_bf16) {
        if constexpr (kPer == 4) {
            const uint2 w = __ldg(reinterpret_cast<const uint2 *>(static_cast<const uint16_t *>(a.x) + e));
            v[0] = bf16_lo(w.x);
            v[1] = bf16_hi(w.x);
            v[2] = bf16_lo(w.y);
            v[3] = bf16_hi(w.y);
        } else {
            const uint32_t w = __ldg(reinterpret_cast<const uint32_t *>(static_cast<const uint16_t *>(a.x) + e));
            v[0] = bf16_lo(w);
            v[1] = bf16_hi(w);
        }
    } else {
#pragma unroll
        for (int k = 0; k < kPer; ++k)
            v[k] = __ldg(static_cast<const float *>(a.x) + e + k);
    }
}

// Raw words of lane l's kPer channels of token t (bf16: kPer / 2 words,
// binary32: kPer words), loaded as one vector.
template <int D, bool BF16>
struct FitRow {
    static constexpr int kPer = D / 32;
    static constexpr int kWords = BF16 ? kPer / 2 : kPer;
    uint32_t w[kWords];

    __device__ __forceinline__ void load(const FitSortArgs &a, int h, int64_t t, int lane)
    {
        const int64_t e = (t * a.H + h) * D + lane * kPer;
        const uint32_t *p = BF16 ? reinterpret_cast<const uint32_t *>(static_cast<const uint16_t *>(a.x) + e)
                                 : reinterpret_cast<const uint32_t *>(static_cast<const float *>(a.x) + e);
        if constexpr (kWords == 4) {
            const uint4 v = __ldg(reinterpret_cast<const uint4 *>(p));
            w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
        } else if constexpr (kWords == 2) {
            const uint2 v = __ldg(reinterpret_cast<const uint2 *>(p));
            w[0] = v.x; w[1] = v.y;
        } else {
            w[0] = __ldg(p);
        }
    }
    __device__ __forceinline__ float value(int k) const
    {
        if constexpr (BF16)
            return (k & 1) ? bf16_hi(w[k >> 1]) : bf16_lo(w[k >> 1]);
        else
            return __uint_as_float(w[k]);
    }
};

// One warp per kFitSegSlots consecutive slots of the sorted order.  The
// slots' token ids and centres are read coalesced up front (lane l holds
// slots l and 32 + l), so no load waits on another; rows are then gathered
// kBatch at a time, kept as raw words until used, and summed in slot order.
// 64 registers (4 blocks of 256 per SM) keep more gathers in flight per SM
// than a larger batch at lower occupancy.
template <int D, bool BF16>
__global__ void __launch_bounds__(256, 4) fit_segsum_kernel(FitSortArgs a)
{
    static_assert(kFitSegSlots == 64, "two slots per lane");
    constexpr int kPer = D / 32;
    constexpr int kBatch = 8;
    const int lane = threadIdx.x & 31;
    const int64_t segs = (a.T + kFitSegSlots - 1) / kFitSegSlots;
    const int64_t gw = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (gw >= segs * a.H)
        return;
    const int h = (int)(gw / segs);
    const int64_t i0 = (gw % segs) * kFitSegSlots;
    const int nb = (int)min((int64_t)kFitSegSlots, a.T - i0);
    const int *ord = a.order + (int64_t)h * a.T + i0;
    const uint16_t *oj = a.order_j + (int64_t)h * a.T + i0;
    const int tA = lane < nb ? ord[lane] : 0, tB = 32 + lane < nb ? ord[32 + lane] : 0;
    const int jA = lane < nb ? (int)oj[lane] : -1, jB = 32 + lane < nb ? (int)oj[32 + lane] : -1;

    double acc[kPer];
    unsigned amax = 0u, amin = 0x7f800000u;
    unsigned rmax = 0u, rmin = 0x7f800000u;  // |x| bounds of the current run (bucket)
    int cur = -1;
#pragma unroll
    for (int k = 0; k < kPer; ++k)
        acc[k] = 0.0;
    auto flush = [&]() {
        double *dst = a.sums + ((int64_t)h * a.C + cur) * D + lane * kPer;
#pragma unroll
        for (int k = 0; k < kPer; ++k) {
            atomicAdd(dst + k, acc[k]);
            acc[k] = 0.0;
        }
        // the run's bounds join the bucket's (the run is the whole warp's)
        const unsigned bmax = __reduce_max_sync(0xffffffffu, rmax);
        const unsigned bmin = __reduce_min_sync(0xffffffffu, rmin);
        if (lane == 0) {
            atomicMax(a.bkt_max + (int64_t)h * a.C + cur, bmax);
            atomicMax(a.bkt_minv + (int64_t)h * a.C + cur, ~bmin);
        }
        rmax = 0u;
        rmin = 0x7f800000u;
    };
#pragma unroll 1
    for (int b0 = 0; b0 < nb; b0 += kBatch) {
        // a batch lies within one half (kBatch divides 32)
        const int t_src = b0 < 32 ? tA : tB, j_src = b0 < 32 ? jA : jB;
        FitRow<D, BF16> rows[kBatch];
#pragma unroll
        for (int b = 0; b < kBatch; ++b) {
            const int t = __shfl_sync(0xffffffffu, t_src, (b0 + b) & 31);
            if (b0 + b < nb)
                rows[b].load(a, h, t, lane);
        }
#pragma unroll
        for (int b = 0; b < kBatch; ++b) {
            const int j = __shfl_sync(0xffffffffu, j_src, (b0 + b) & 31);
            if (b0 + b >= nb)
                break;
            if (j != cur) {
                if (cur >= 0)
                    flush();
                cur = j;
            }
#pragma unroll
            for (int k = 0; k < kPer; ++k) {
                const float v = rows[b].value(k);
                acc[k] = __dadd_rn(acc[k], (double)v);
                const unsigned u = __float_as_uint(v) & 0x7fffffffu;
                rmax = max(rmax, u);
                rmin = min(rmin, u ? u : 0x7f800000u);
                if (a.track) {
                    amax = max(amax, u);
                    amin = min(amin, u ? u : 0x7f800000u);
                }
            }
        }
    }
    if (cur >= 0)
        flush();
    if (a.track) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            amax = max(amax, __shfl_xor_sync(0xffffffffu, amax, o));
            amin = min(amin, __shfl_xor_sync(0xffffffffu, amin, o));
        }
        if (lane == 0) {
            atomicMax(a.abs_max + h, amax);
            atomicMin(a.abs_min + h, amin);
        }
    }
}

// One warp per (head, centre): exact totals -> new centre; otherwise mark the
// centre for the sequential pass.  Clears the totals for the next round.
template <int D>
__global__ void __launch_bounds__(256) fit_finalize_kernel(FitSortArgs a)
{
    constexpr int kPer = D / 32;
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
    if (warp >= a.H * a.C)
        return;
    const int h = warp / a.C, j = warp % a.C;
    const int64_t hj = (int64_t)h * a.C + j;
    const int *bs = a.bucket_start + (int64_t)h * (a.C + 1);
    const int n = bs[j + 1] - bs[j];
    // every partial sum is a multiple of 2^L below 2^(53 + L) in magnitude,
    // L from the head's smallest nonzero |x| or from the bucket's own (every
    // value is a multiple of its own ulp, hence of that of the smallest)
    const unsigned amin = a.abs_min[h];
    const int L = (int)(amin >> 23) - (a.x_bf16 ? 134 : 150);
    const unsigned bmin = ~a.bkt_minv[hj];
    const int Lb = (int)(bmin >> 23) - (a.x_bf16 ? 134 : 150);
    const bool exact =
        amin >= 0x7f800000u || (double)n * (double)__uint_as_float(a.abs_max[h]) <= ldexp(1.0, 52 + L) ||
        bmin >= 0x7f800000u || (double)n * (double)__uint_as_float(a.bkt_max[hj]) <= ldexp(1.0, 52 + Lb);
    double *sum = a.sums + hj * D + lane * kPer;
    if (n > 0 && exact) {
        uint16_t *dst = a.cent + hj * D + lane * kPer;
#pragma unroll
        for (int k = 0; k < kPer; ++k) {
            const __nv_bfloat16 b = __float2bfloat16_rn(__double2float_rn(__ddiv_rn(sum[k], (double)n)));
            dst[k] = *reinterpret_cast<const uint16_t *>(&b);
        }
    }
#pragma unroll
    for (int k = 0; k < kPer; ++k)
        sum[k] = 0.0;
    __syncwarp();  // every lane has read the bucket's bounds
    if (lane == 0) {
        a.redo[hj] = (n > 0 && !exact) ? 1 : 0;
        a.bkt_max[hj] = 0u;
        a.bkt_minv[hj] = 0u;
    }
}

// One warp per (head, centre) marked by fit_finalize; lane l owns channels
// kPer l .. kPer l + kPer - 1.  Sums in binary64 in token order.
template <int D>
__global__ void __launch_bounds__(256) fit_bucket_update_kernel(FitSortArgs a)
{
    constexpr int kPer = D / 32;
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
    if (warp >= a.H * a.C)
        return;
    const int h = warp / a.C, j = warp % a.C;
    if (!a.redo[(int64_t)h * a.C + j])
        return;
    const int *bs = a.bucket_start + (int64_t)h * (a.C + 1);
    const int b0 = bs[j], b1 = bs[j + 1];
    if (b1 == b0)
        return;  // empty: the centre keeps its value
    const int *ord = a.order + (int64_t)h * a.T;
    double acc[kPer];
#pragma unroll
    for (int k = 0; k < kPer; ++k)
        acc[k] = 0.0;
    // tokens in batches of 8: loads of a batch are issued together, the adds
    // then run in token order
    constexpr int kBatch = 8;
    for (int i0 = b0; i0 < b1; i0 += kBatch) {
        float v[kBatch][kPer];
#pragma unroll
        for (int b = 0; b < kBatch; ++b) {
            const int i = i0 + b;
#pragma unroll
            for (int k = 0; k < kPer; ++k)
                v[b][k] = 0.0f;
            if (i < b1)
                fit_load_row<D>(a, h, ord[i], lane, v[b]);
        }
#pragma unroll
        for (int b = 0; b < kBatch; ++b) {
            if (i0 + b >= b1)
                break;
#pragma unroll
            for (int k = 0; k < kPer; ++k)
                acc[k] = __dadd_rn(acc[k], (double)v[b][k]);
        }
    }
    const double n = (double)(b1 - b0);
    uint16_t *dst = a.cent + ((int64_t)h * a.C + j) * D + lane * kPer;
#pragma unroll
    for (int k = 0; k < kPer; ++k) {
        const __nv_bfloat16 b = __float2bfloat16_rn(__double2float_rn(__ddiv_rn(acc[k], n)));
        dst[k] = *reinterpret_cast<const uint16_t *>(&b);
    }
}

}  // namespace kvq

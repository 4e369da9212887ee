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
template <int D, int BITS, int G>
__device__ __forceinline__ void encode_residual_row(const float *r, uint8_t *codes_row, float2 *meta_row)
{
    constexpr int kWords = D * BITS / 32;
    constexpr int kPerWord = 32 / BITS;
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
        const GroupQ gq = group_params(mn, mx, BITS);
        meta_row[g] = make_float2(gq.s, gq.z);
#pragma unroll
        for (int c = g * G; c < (g + 1) * G; ++c)
            words[c / kPerWord] |= quant_code(r[c], gq, BITS) << ((c % kPerWord) * BITS);
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
    float *meta;           // [H][T][D/G][2]
    int assign_only;
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
            for (int jj = 0; jj < nj; ++jj) {
                const float4 *mu4 = reinterpret_cast<const float4 *>(s_mu + jj * D);
                float acc = 0.0f;
#pragma unroll
                for (int c4 = 0; c4 < D / 4; ++c4) {
                    const float4 m = mu4[c4];
                    float e;
                    e = __fsub_rn(xr[4 * c4 + 0], m.x); acc = __fadd_rn(acc, __fmul_rn(e, e));
                    e = __fsub_rn(xr[4 * c4 + 1], m.y); acc = __fadd_rn(acc, __fmul_rn(e, e));
                    e = __fsub_rn(xr[4 * c4 + 2], m.z); acc = __fadd_rn(acc, __fmul_rn(e, e));
                    e = __fsub_rn(xr[4 * c4 + 3], m.w); acc = __fadd_rn(acc, __fmul_rn(e, e));
                }
                const int j = j0 + jj;
                if (j == 0 || acc < best) {
                    best = acc;
                    best_j = j;
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
    encode_residual_row<D, BITS, G>(xr, a.codes + th * (D * BITS / 8),
                                    reinterpret_cast<float2 *>(a.meta) + th * (D / G));
}

// ---------------------------------------------------------------------------
// Per-head reconstruction: one thread per 8 channels of a token-head.
// ---------------------------------------------------------------------------
struct DecodeArgs {
    const uint16_t *cent;
    const uint16_t *idx;
    const uint8_t *codes;
    const float *meta;
    int64_t T;
    int H;
    int D;
    int C;
    int bits;
    int G;
    void *out;
    int out_bf16;
};

__global__ void __launch_bounds__(256) decode_kernel(DecodeArgs a)
{
    const int units = a.D / 8;
    const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t total = a.T * a.H * units;
    if (gid >= total)
        return;
    const int u = (int)(gid % units);
    const int64_t th_out = gid / units;       // t * H + h
    const int h = (int)(th_out % a.H);
    const int64_t t = th_out / a.H;
    const int64_t th = (int64_t)h * a.T + t;  // encoded-row index
    int j = a.idx[th];
    if (j >= a.C) {
        raise_status(DEVSTAT_BAD_INDEX);
        j = 0;
    }
    const int c0 = u * 8;
    const int g = c0 / a.G;
    const float2 sz = reinterpret_cast<const float2 *>(a.meta)[th * (a.D / a.G) + g];
    uint32_t cw;
    if (a.bits == 2)
        cw = *reinterpret_cast<const uint16_t *>(a.codes + th * (a.D / 4) + c0 / 4);
    else
        cw = *reinterpret_cast<const uint32_t *>(a.codes + th * (a.D / 2) + c0 / 2);
    float mu[8];
    load_bf16x8(a.cent + ((int64_t)h * a.C + j) * a.D + c0, mu);
    const uint32_t mask = (1u << a.bits) - 1u;
    float v[8];
#pragma unroll
    for (int k = 0; k < 8; ++k)
        v[k] = dequant_spec((cw >> (k * a.bits)) & mask, sz.x, sz.y, mu[k]);
    const int64_t o = th_out * a.D + c0;
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
// k-means fitting: seeding, binary64 accumulation, update
// ---------------------------------------------------------------------------
struct FitArgs {
    const void *x;
    int x_bf16;
    int64_t T;
    int H;
    int D;
    int C;
    uint16_t *cent;          // [H][C][D]
    const uint16_t *idx;     // [H][T]
    double *sums;            // [H][C][D]
    unsigned int *counts;    // [H][C]
};

// mu_j = bf16(x_j) for the first C tokens.
__global__ void __launch_bounds__(256) fit_seed_kernel(FitArgs a)
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
}

// sums[h][idx][c] += x (binary64), counts[h][idx] += 1; one thread per
// 8 channels of a token-head.
__global__ void __launch_bounds__(256) fit_accumulate_kernel(FitArgs a)
{
    const int units = a.D / 8;
    const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t total = a.T * a.H * units;
    if (gid >= total)
        return;
    const int u = (int)(gid % units);
    const int64_t th_in = gid / units;  // t * H + h
    const int h = (int)(th_in % a.H);
    const int64_t t = th_in / a.H;
    const int j = a.idx[(int64_t)h * a.T + t];
    float xv[8];
    load_x8(a.x, a.x_bf16, th_in * a.D + u * 8, xv);
    double *dst = a.sums + ((int64_t)h * a.C + j) * a.D + u * 8;
#pragma unroll
    for (int k = 0; k < 8; ++k)
        atomicAdd(dst + k, (double)xv[k]);
    if (u == 0)
        atomicAdd(a.counts + (int64_t)h * a.C + j, 1u);
}

// Same sums with far fewer global atomics: a block owns one head, one slice
// of W channels and a contiguous token range; it accumulates into binary64
// shared-memory sums [C][W] and adds them to the global sums once at the end.
// Token counts are added by the slice-0 blocks.
template <int W>
__global__ void __launch_bounds__(256) fit_accumulate_smem_kernel(FitArgs a, int64_t tokens_per_block)
{
    extern __shared__ double s_sum[];  // [C][W]
    const int h = blockIdx.y, slice = blockIdx.z;
    const int64_t t_lo = (int64_t)blockIdx.x * tokens_per_block;
    const int64_t t_hi = min(a.T, t_lo + tokens_per_block);
    for (int e = threadIdx.x; e < a.C * W; e += blockDim.x)
        s_sum[e] = 0.0;
    __syncthreads();
    // a group of W lanes handles one token; lane c adds channel slice*W + c.
    // Tokens go in batches of 8 so that their loads are in flight together.
    constexpr int kGroups = 256 / W, kBatch = 8;
    const int grp = threadIdx.x / W, c = threadIdx.x % W;
    for (int64_t t0 = t_lo + grp; t0 < t_hi; t0 += (int64_t)kGroups * kBatch) {
        int j[kBatch];
        float v[kBatch];
#pragma unroll
        for (int b = 0; b < kBatch; ++b) {
            const int64_t t = t0 + (int64_t)b * kGroups;
            j[b] = t < t_hi ? __ldg(a.idx + (int64_t)h * a.T + t) : -1;
        }
#pragma unroll
        for (int b = 0; b < kBatch; ++b) {
            const int64_t t = t0 + (int64_t)b * kGroups;
            const int64_t e = (t * a.H + h) * a.D + slice * W + c;
            v[b] = 0.0f;
            if (j[b] >= 0)
                v[b] = a.x_bf16 ? __uint_as_float((uint32_t)__ldg(static_cast<const uint16_t *>(a.x) + e) << 16)
                                : __ldg(static_cast<const float *>(a.x) + e);
        }
#pragma unroll
        for (int b = 0; b < kBatch; ++b) {
            if (j[b] < 0)
                continue;
            atomicAdd(&s_sum[j[b] * W + c], (double)v[b]);
            if (slice == 0 && c == 0)
                atomicAdd(a.counts + (int64_t)h * a.C + j[b], 1u);
        }
    }
    __syncthreads();
    for (int e = threadIdx.x; e < a.C * W; e += blockDim.x) {
        const double v = s_sum[e];
        if (v != 0.0)
            atomicAdd(a.sums + ((int64_t)h * a.C + e / W) * a.D + slice * W + e % W, v);
    }
}

// mu_j = bf16(float(sum_j / n_j)) where n_j > 0; empty centres keep mu_j.
__global__ void __launch_bounds__(256) fit_update_kernel(FitArgs a)
{
    const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t total = (int64_t)a.H * a.C * a.D;
    if (gid >= total)
        return;
    const unsigned n = a.counts[gid / a.D];
    if (n == 0)
        return;
    const double mean = __ddiv_rn(a.sums[gid], (double)n);
    const __nv_bfloat16 b = __float2bfloat16_rn(__double2float_rn(mean));
    a.cent[gid] = *reinterpret_cast<const uint16_t *>(&b);
}

}  // namespace kvq

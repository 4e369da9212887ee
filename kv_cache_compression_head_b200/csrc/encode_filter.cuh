// encode_filter.cuh -- nearest-centroid assignment + residual quantisation with
// a tensor-core distance filter (bf16 history, C <= 512 centres per head).
//
// Method: QuantWM: Temporally Consistent 2-Bit KV Cache Quantization for
// Video World Models, Sec. 4.1 (nearest centroid, then residual
// quantisation); TempoKV, Sec. 3.1 Eq. 1 (quantiser).  The result is
// bit-identical to the exact kernel in codec.cuh: the tensor cores only narrow
// the search, the decision is taken by the specified binary32 distance.
//
// For a tile of 128 tokens of head h:
//   1. TMA loads the tile X [128][d] (bf16, 128-byte swizzle) from [T][H][d];
//   2. one thread issues P = X mu^T (M=128, N=C, K=d, fp32 in TMEM); the
//      centres of the head stay resident in shared memory for every tile the
//      CTA processes;
//   3. two threads per token (one per half of the TMEM columns and of the
//      channels) compute v_j = |mu_j|^2 - 2 p_j, the row minimum m and the
//      candidate window  v_j <= m + kappa (|x| + max_j |mu_j|)^2,  which
//      provably contains the specified argmin: kappa covers the tensor-core
//      accumulation error, the rounding of |mu_j|^2 and of v_j, the rounding
//      of the specified distance and the index bits carried in v.  When the
//      second smallest v lies outside the window the smallest is the answer;
//      when only the two smallest lie inside it, the two threads of the token
//      each score one of them with the specified distance; otherwise the
//      whole window is re-scored (lowest index wins ties everywhere);
//   4. the residual against the chosen centre is quantised (Eq. 1) per group
//      and packed, each thread covering its half of the channels.
#pragma once

#include <cuda.h>

#include "codec.cuh"
#include "common.cuh"

namespace kvq {

constexpr int kFltRows = 128;
constexpr int kFltThreads = 256;
constexpr int kFltMaxC = 512;

struct FilterArgs {
    int64_t T;
    int H;
    int C;
    int Cpad;          // C rounded up to a multiple of 32
    int tmem_cols;     // power of two >= max(32, Cpad)
    const uint16_t *cent;
    uint16_t *idx;
    uint8_t *codes;
    float *meta;
    int assign_only;
    float kappa;       // window = kappa * (|x| + M)^2
};

constexpr uint32_t kFltPairBytes = 7168u;  // pair exchange: float4 [2][128] | int [2][128] | float4 [128]

__host__ __device__ constexpr uint32_t flt_smem_bytes(int D, int Cpad)
{
    // X tile | centres | norms | pair exchange | 2 barriers + slots
    return (uint32_t)(D * 2 * kFltRows) + (uint32_t)(Cpad * D * 2) + (uint32_t)(Cpad * 4) + kFltPairBytes + 64u;
}

// Insert (v, c) into the ascending list (b1, c1) <= (b2, c2) <= (b3, c3);
// on equal values the entry already present stays first.
__device__ __forceinline__ void top3_insert(float v, int c, float &b1, int &c1, float &b2, int &c2, float &b3,
                                            int &c3)
{
    if (v < b3) {
        if (v < b2) {
            b3 = b2;
            c3 = c2;
            if (v < b1) {
                b2 = b1;
                c2 = c1;
                b1 = v;
                c1 = c;
            } else {
                b2 = v;
                c2 = c;
            }
        } else {
            b3 = v;
            c3 = c;
        }
    }
}

// Specified binary32 distance of row `row` of the X tile to centre j of the
// resident centre tile (both 128-byte swizzled bf16).
template <int D>
__device__ __forceinline__ float spec_distance_smem(const uint8_t *sX, const uint8_t *sMu, int Cpad, int row, int j)
{
    float acc = 0.0f;
#pragma unroll 2
    for (int u = 0; u < D / 8; ++u) {
        const uint4 xw = *reinterpret_cast<const uint4 *>(sX + sw128_unit_offset(row, u, kFltRows));
        const uint4 mw = *reinterpret_cast<const uint4 *>(sMu + sw128_unit_offset(j, u, Cpad));
        const uint32_t xa[4] = {xw.x, xw.y, xw.z, xw.w}, ma[4] = {mw.x, mw.y, mw.z, mw.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            float e = __fsub_rn(bf16_lo(xa[k]), bf16_lo(ma[k]));
            acc = __fadd_rn(acc, __fmul_rn(e, e));
            e = __fsub_rn(bf16_hi(xa[k]), bf16_hi(ma[k]));
            acc = __fadd_rn(acc, __fmul_rn(e, e));
        }
    }
    return acc;
}

// Residual r = x - mu[best] of channels [half*CH, half*CH + CH) of one token,
// read from the swizzled tiles, quantised per group (Eq. 1) and packed.  Two
// passes over shared memory (min/max, then codes) keep r out of registers.
// Group min/max use strict comparisons in channel order, as specified.
template <int CH, int BITS, int G>
__device__ __forceinline__ void encode_residual_smem(const uint8_t *sX, const uint8_t *sMu, int Cpad, int row,
                                                     int best, int half, uint8_t *codes_dst, float2 *meta_dst)
{
    constexpr int kPerWord = 32 / BITS;
    constexpr int kWords = CH * BITS / 32;
    uint32_t words[kWords];
#pragma unroll
    for (int w = 0; w < kWords; ++w)
        words[w] = 0u;
#pragma unroll
    for (int g = 0; g < CH / G; ++g) {
        if constexpr (G <= 32) {
            // the group's residuals stay in registers
            float r[G];
#pragma unroll
            for (int uu = 0; uu < G / 8; ++uu) {
                const int u = half * (CH / 8) + g * (G / 8) + uu;
                const uint4 xw = *reinterpret_cast<const uint4 *>(sX + sw128_unit_offset(row, u, kFltRows));
                const uint4 mw = *reinterpret_cast<const uint4 *>(sMu + sw128_unit_offset(best, u, Cpad));
                const uint32_t xa[4] = {xw.x, xw.y, xw.z, xw.w}, ma[4] = {mw.x, mw.y, mw.z, mw.w};
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const float2 d = sub2(make_float2(bf16_lo(xa[k]), bf16_hi(xa[k])),
                                          make_float2(bf16_lo(ma[k]), bf16_hi(ma[k])));
                    r[uu * 8 + 2 * k] = d.x;
                    r[uu * 8 + 2 * k + 1] = d.y;
                }
            }
            float mn = fminf(r[0], r[1]), mx = fmaxf(r[0], r[1]);
#pragma unroll
            for (int c = 2; c < G; c += 2) {
                mn = fmin3(mn, r[c], r[c + 1]);
                mx = fmax3(mx, r[c], r[c + 1]);
            }
            if (mn == 0.0f || mx == 0.0f) {
                // a zero extreme: take its sign exactly as the ordered strict scan does
                mn = r[0];
                mx = r[0];
#pragma unroll
                for (int c = 1; c < G; ++c) {
                    if (r[c] < mn) mn = r[c];
                    if (r[c] > mx) mx = r[c];
                }
            }
            const GroupQ gq = group_params(mn, mx, BITS);
            meta_dst[g] = make_float2(gq.s, gq.z);
            quant_group_into<G, BITS>(r, gq, mn, mx, words, g * G);
            continue;
        }
        float mn = 0.0f, mx = 0.0f;
#pragma unroll
        for (int uu = 0; uu < G / 8; ++uu) {
            const int u = half * (CH / 8) + g * (G / 8) + uu;
            const uint4 xw = *reinterpret_cast<const uint4 *>(sX + sw128_unit_offset(row, u, kFltRows));
            const uint4 mw = *reinterpret_cast<const uint4 *>(sMu + sw128_unit_offset(best, u, Cpad));
            const uint32_t xa[4] = {xw.x, xw.y, xw.z, xw.w}, ma[4] = {mw.x, mw.y, mw.z, mw.w};
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const float r = __fsub_rn((k & 1) ? bf16_hi(xa[k >> 1]) : bf16_lo(xa[k >> 1]),
                                          (k & 1) ? bf16_hi(ma[k >> 1]) : bf16_lo(ma[k >> 1]));
                if (uu == 0 && k == 0) {
                    mn = r;
                    mx = r;
                } else {
                    if (r < mn) mn = r;
                    if (r > mx) mx = r;
                }
            }
        }
        const GroupQ gq = group_params(mn, mx, BITS);
        meta_dst[g] = make_float2(gq.s, gq.z);
        const GroupFast gf = group_fast(gq, mn, mx);
#pragma unroll
        for (int uu = 0; uu < G / 8; ++uu) {
            const int u = half * (CH / 8) + g * (G / 8) + uu;
            const uint4 xw = *reinterpret_cast<const uint4 *>(sX + sw128_unit_offset(row, u, kFltRows));
            const uint4 mw = *reinterpret_cast<const uint4 *>(sMu + sw128_unit_offset(best, u, Cpad));
            const uint32_t xa[4] = {xw.x, xw.y, xw.z, xw.w}, ma[4] = {mw.x, mw.y, mw.z, mw.w};
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const float r = __fsub_rn((k & 1) ? bf16_hi(xa[k >> 1]) : bf16_lo(xa[k >> 1]),
                                          (k & 1) ? bf16_hi(ma[k >> 1]) : bf16_lo(ma[k >> 1]));
                const int c = g * G + uu * 8 + k;
                words[c / kPerWord] += (gf.fast ? quant_code_fast<BITS>(r, gf) : quant_code(r, gq, BITS))
                                       << ((c % kPerWord) * BITS);
            }
        }
    }
    if constexpr (kWords >= 4) {
        uint4 *dst = reinterpret_cast<uint4 *>(codes_dst);
#pragma unroll
        for (int v = 0; v < kWords / 4; ++v)
            dst[v] = make_uint4(words[4 * v], words[4 * v + 1], words[4 * v + 2], words[4 * v + 3]);
    } else {
        uint32_t *dst = reinterpret_cast<uint32_t *>(codes_dst);
#pragma unroll
        for (int v = 0; v < kWords; ++v)
            dst[v] = words[v];
    }
}

template <int D, int BITS, int G>
__global__ void __launch_bounds__(kFltThreads, 2)
    encode_filter_kernel(const __grid_constant__ CUtensorMap tmap_x, FilterArgs a)
{
    static_assert(G <= D / 2, "a group must lie inside one half of the channels");
    constexpr int CH = D / 2;             // channels per thread
    constexpr int kMaxChunks = kFltMaxC / 32 / 2;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int Cpad = a.Cpad;
    uint8_t *sX = smem;
    uint8_t *sMu = smem + D * 2 * kFltRows;
    float *sNrm = reinterpret_cast<float *>(sMu + Cpad * D * 2);
    float4 *sPair = reinterpret_cast<float4 *>(sNrm + Cpad);               // [2][128] {|x|^2 part, top 3}
    int *sPairC = reinterpret_cast<int *>(sPair + 2 * 128);                  // [2][128] top-3 chunk ids
    float4 *sWin = reinterpret_cast<float4 *>(sPairC + 2 * 128);             // [128] exact winners / distances
    uint64_t *bars = reinterpret_cast<uint64_t *>(reinterpret_cast<uint8_t *>(sPair) + kFltPairBytes);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 2);
    uint32_t *sMaxNrm = tmem_slot + 1;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int half = warp >> 2;
    const int row = (warp & 3) * 32 + lane;
    const int h = blockIdx.y;
    const uint32_t bar_x = smem_u32(bars), bar_m = smem_u32(bars + 1);

    if (warp == 0)
        tmem_alloc(smem_u32(tmem_slot), a.tmem_cols);
    if (tid == 0) {
        mbar_init(bar_x, 1);
        mbar_init(bar_m, 1);
        fence_mbar_init();
        *sMaxNrm = 0u;
    }
    __syncthreads();

    // centres of head h -> swizzled K-major tile [D/64][Cpad][128 B]; norms
    const uint16_t *cent_h = a.cent + (int64_t)h * a.C * D;
    for (int e = tid; e < Cpad * (D / 8); e += kFltThreads) {
        const int j = e / (D / 8), u = e % (D / 8);
        const uint4 w = j < a.C ? __ldg(reinterpret_cast<const uint4 *>(cent_h + (int64_t)j * D) + u)
                                : make_uint4(0, 0, 0, 0);
        *reinterpret_cast<uint4 *>(sMu + sw128_unit_offset(j, u, Cpad)) = w;
    }
    for (int j = tid; j < Cpad; j += kFltThreads) {
        float nrm = INFINITY;
        if (j < a.C) {
            nrm = 0.0f;
            for (int u = 0; u < D / 8; ++u) {
                float m8[8];
                load_bf16x8(cent_h + (int64_t)j * D + u * 8, m8);
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    nrm = fmaf(m8[k], m8[k], nrm);
            }
            atomicMax(sMaxNrm, __float_as_uint(nrm));
        }
        sNrm[j] = nrm;
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const float Mnorm = sqrtf(__uint_as_float(*sMaxNrm));
    const uint32_t lane_off = ((uint32_t)(warp & 3) * 32u) << 16;
    const uint32_t aX = smem_u32(sX), aMu = smem_u32(sMu);

    // this thread's 32-column chunks of the TMEM row
    const int nchunks = Cpad / 32;
    const int c_lo = half == 0 ? 0 : (nchunks + 1) / 2;
    const int c_hi = half == 0 ? (nchunks + 1) / 2 : nchunks;

    const int64_t ntiles = (a.T + kFltRows - 1) / kFltRows;
    uint32_t ph_x = 0, ph_m = 0;
    bool ok = true;
    for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
        const int64_t t0 = tile * kFltRows;
        if (tid == 0) {
            mbar_arrive_expect_tx(bar_x, D * 2 * kFltRows);
#pragma unroll
            for (int ch = 0; ch < D / 64; ++ch)
                tma_load_3d(aX + ch * (kFltRows * 128), &tmap_x, bar_x, ch * 64, h, (int)t0);
        }
        ok = mbar_wait(bar_x, ph_x) && ok;
        ph_x ^= 1u;
        if (tid == 0) {
            tc_fence_after();
            for (int n0 = 0; n0 < Cpad; n0 += 256) {
                const int N = min(256, Cpad - n0);
                const uint32_t idesc = idesc_f32acc(128, N, true, false, false);
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks) {
                    const uint32_t aoff = (uint32_t)(ks >> 2) * (kFltRows * 128u) + (uint32_t)(ks & 3) * 32u;
                    const uint32_t boff =
                        (uint32_t)(ks >> 2) * (uint32_t)(Cpad * 128) + (uint32_t)n0 * 128u + (uint32_t)(ks & 3) * 32u;
                    umma_ss(tmem + (uint32_t)n0, sdesc_sw128(aX + aoff, 16, 1024), sdesc_sw128(aMu + boff, 16, 1024),
                            idesc, ks > 0 ? 1u : 0u);
                }
            }
            umma_commit(bar_m);
        }
        ok = mbar_wait(bar_m, ph_m) && ok;
        ph_m ^= 1u;
        tc_fence_after();

        // (1) |x|^2 over this thread's channel half
        float xx = 0.0f;
#pragma unroll
        for (int u = half * (CH / 8); u < (half + 1) * (CH / 8); ++u) {
            const uint4 w = *reinterpret_cast<const uint4 *>(sX + sw128_unit_offset(row, u, kFltRows));
            const uint32_t wa[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                xx = fmaf(bf16_lo(wa[k]), bf16_lo(wa[k]), xx);
                xx = fmaf(bf16_hi(wa[k]), bf16_hi(wa[k]), xx);
            }
        }
        // (2) v_j = |mu_j|^2 - 2 p_j over this thread's chunks.  The chunk-local
        // column index rides in the low 5 mantissa bits of v, so one pass keeps
        // the three smallest values (the window below absorbs the <= 31 ulp
        // this perturbs v); chunk ids are kept beside them.
        float b1 = INFINITY, b2 = INFINITY, b3 = INFINITY;
        int k1 = 0, k2 = 0, k3 = 0;
#pragma unroll
        for (int k = 0; k < kMaxChunks; ++k) {
            const int c = c_lo + k;
            if (c < c_hi) {
                float p[32];
                tmem_ld32(tmem + lane_off + (uint32_t)(c * 32), p);
                // two independent chains (pairs 4q and 4q + 2 / 4q + 1 and 4q + 3
                // of the chunk) so consecutive updates do not wait on each other
                float a1 = INFINITY, a2 = INFINITY, a3 = INFINITY;
                float c1 = INFINITY, c2 = INFINITY, c3 = INFINITY;
                const float4 *nrm4 = reinterpret_cast<const float4 *>(sNrm + c * 32);
                auto pair_into = [](float pa, float pb, float &m1, float &m2, float &m3) {
                    // sort the pair, then merge it into the three smallest
                    // (k-th smallest of two sorted lists = min over i + j = k
                    // of max(a_i, b_j))
                    const float lo = fminf(pa, pb), hi = fmaxf(pa, pb);
                    const float n3 = fmin3(m3, fmaxf(m2, lo), fmaxf(m1, hi));
                    const float n2 = fmin3(fmaxf(m1, lo), m2, hi);
                    m1 = fminf(m1, lo);
                    m2 = n2;
                    m3 = n3;
                };
#pragma unroll
                for (int i4 = 0; i4 < 8; ++i4) {
                    const float4 n4 = nrm4[i4];
                    const float nn[4] = {n4.x, n4.y, n4.z, n4.w};
                    float pk[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int i = i4 * 4 + e;
                        const float v = fmaf(-2.0f, p[i], nn[e]);
                        pk[e] = __uint_as_float((__float_as_uint(v) & ~31u) | (uint32_t)i);
                    }
                    pair_into(pk[0], pk[1], a1, a2, a3);
                    pair_into(pk[2], pk[3], c1, c2, c3);
                }
                // merge the two chains' three smallest
                const float m1 = fminf(a1, c1);
                const float m2 = fmin3(a2, fmaxf(a1, c1), c2);
                const float m3 = fminf(fmin3(a3, fmaxf(a2, c1), fmaxf(a1, c2)), c3);
                top3_insert(m1, c, b1, k1, b2, k2, b3, k3);
                top3_insert(m2, c, b1, k1, b2, k2, b3, k3);
                top3_insert(m3, c, b1, k1, b2, k2, b3, k3);
            }
        }
        // (3) exchange with the partner thread of this row (warps w and w+4);
        // both threads then hold the row's three smallest values, half-0
        // entries first on equal values
        sPair[half * 128 + row] = make_float4(xx, b1, b2, b3);
        sPairC[half * 128 + row] = k1 | (k2 << 8) | (k3 << 16);
        named_barrier_sync_q(warp & 3, 64);
        const float4 other = sPair[(half ^ 1) * 128 + row];
        const int oc = sPairC[(half ^ 1) * 128 + row];
        float g1, g2, g3;
        int h1, h2, h3;
        {
            // list of half 0, then insert half 1's entries
            const bool h0 = half == 0;
            g1 = h0 ? b1 : other.y;
            g2 = h0 ? b2 : other.z;
            g3 = h0 ? b3 : other.w;
            const int cc = h0 ? (k1 | (k2 << 8) | (k3 << 16)) : oc;
            h1 = cc & 0xff;
            h2 = (cc >> 8) & 0xff;
            h3 = (cc >> 16) & 0xff;
            const int dc = h0 ? oc : (k1 | (k2 << 8) | (k3 << 16));
            top3_insert(h0 ? other.y : b1, dc & 0xff, g1, h1, g2, h2, g3, h3);
            top3_insert(h0 ? other.z : b2, (dc >> 8) & 0xff, g1, h1, g2, h2, g3, h3);
            top3_insert(h0 ? other.w : b3, (dc >> 16) & 0xff, g1, h1, g2, h2, g3, h3);
        }
        const float xn = sqrtf(xx + other.x);
        const float thr = g1 + a.kappa * (xn + Mnorm) * (xn + Mnorm);
        int best = h1 * 32 + (int)(__float_as_uint(g1) & 31u);
        const bool finite = thr < INFINITY;
        const bool pair_case = finite && !(g2 > thr) && g3 > thr;    // two candidates
        const bool wide_case = !finite || (!(g2 > thr) && !(g3 > thr));  // three or more
        // two candidates: each thread of the pair scores one with the specified
        // distance; the smaller wins, the lower index on a tie
        if (__any_sync(0xffffffffu, pair_case)) {
            const int j1 = best, j2 = h2 * 32 + (int)(__float_as_uint(g2) & 31u);
            float dmine = 0.0f;
            if (pair_case)
                dmine = spec_distance_smem<D>(sX, sMu, Cpad, row, half == 0 ? j1 : j2);
            if (pair_case) {
                if (half == 0)
                    sWin[row].x = dmine;
            }
            named_barrier_sync_q(warp & 3, 64);
            if (pair_case) {
                const float d1 = half == 0 ? dmine : sWin[row].x;
                const float d2 = half == 0 ? 0.0f : dmine;
                if (half == 1) {
                    const int lo = j1 < j2 ? j1 : j2;
                    const int hi = j1 < j2 ? j2 : j1;
                    const float dlo = j1 < j2 ? d1 : d2, dhi = j1 < j2 ? d2 : d1;
                    sWin[row].y = __int_as_float(dhi < dlo ? hi : lo);
                }
            }
            named_barrier_sync_q(warp & 3, 64);
            if (pair_case)
                best = __float_as_int(sWin[row].y);
        }
        // three or more candidates (rare): re-score the window (or every centre
        // when the window is not finite) with the specified distance.  Each
        // thread of the pair scans its own half of the columns in increasing
        // index order; the lower half wins ties.  Both warps of the pair see
        // the same flags, so they take the branch together.
        if (__any_sync(0xffffffffu, wide_case)) {
            float bd = INFINITY;
            int bj = -1;
            for (int c = c_lo; c < c_hi; ++c) {
                float p[32];
                tmem_ld32(tmem + lane_off + (uint32_t)(c * 32), p);
                uint32_t cand = 0u;
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int j = c * 32 + i;
                    const float v = fmaf(-2.0f, p[i], sNrm[j]);
                    if (wide_case && j < a.C && (!finite || v <= thr))
                        cand |= 1u << i;
                }
                while (cand) {  // increasing index order
                    const int i = __ffs(cand) - 1;
                    cand &= cand - 1u;
                    const int j = c * 32 + i;
                    const float dj = spec_distance_smem<D>(sX, sMu, Cpad, row, j);
                    if (bj < 0 || dj < bd) {
                        bd = dj;
                        bj = j;
                    }
                }
            }
            reinterpret_cast<float2 *>(sWin + row)[half] = make_float2(bd, __int_as_float(bj));
            named_barrier_sync_q(warp & 3, 64);
            if (wide_case) {
                const float4 w = sWin[row];
                const int j0 = __float_as_int(w.y), j1 = __float_as_int(w.w);
                best = (j0 < 0 || (j1 >= 0 && w.z < w.x)) ? j1 : j0;
            }
        }
        if (best < 0 || best >= a.C)
            best = 0;  // unreachable for finite inputs

        // (4) residual + Eq. 1 + packing for this thread's channel half
        const int64_t t = t0 + row;
        if (t < a.T) {
            const int64_t th = (int64_t)h * a.T + t;
            if (half == 0)
                a.idx[th] = (uint16_t)best;
            if (!a.assign_only)
                encode_residual_smem<CH, BITS, G>(sX, sMu, Cpad, row, best, half,
                                                  a.codes + th * (D * BITS / 8) + half * (CH * BITS / 8),
                                                  reinterpret_cast<float2 *>(a.meta) + th * (D / G) + half * (CH / G));
        }
        tc_fence_before();
        ok = __syncthreads_and(ok) != 0;
        if (!ok)
            break;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0)
        tmem_dealloc(tmem, a.tmem_cols);
}

}  // namespace kvq

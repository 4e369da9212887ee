// encode_filter.cuh -- nearest-centroid assignment + residual quantisation with
// a tensor-core distance filter (bf16 history, C <= 512 centres per head).
//
// Method: QuantWM: Temporally Consistent 2-Bit KV Cache Quantization for
// Video World Models, Sec. 4.1 (nearest centroid, then residual
// quantisation); TempoKV, Sec. 3.1 Eq. 1 (quantiser).  The result is
// bit-identical to the exact kernel in codec.cuh: the tensor cores only narrow
// the search, the decision is taken by the specified binary32 distance.
//
// Certified candidate set.  With R_j = |x| + |mu_j|, the tensor-core value
// v~_j = |mu_j|^2 - 2 x.mu_j (binary32 norms, fp32 MMA accumulation, one
// rounded FMA) is within tau R_j^2 of the exact |x - mu_j|^2 - |x|^2, and the
// specified binary32 distance D_j is within gamma_{d+2} R_j^2 of the exact
// squared distance.  Hence the specified argmin j* satisfies, for every j,
//   L_j* <= U_j,   L_j = v~_j - k R_j^2,   U_j = v~_j + k R_j^2,
// k = tau + gamma_{d+2} (plus margins for the rounding of L and the index
// bits carried in v).  The scan ranks centres by L (three smallest kept) and
// takes U of the first as the threshold: every centre with L <= U(first) is a
// candidate, a superset of {j : L_j <= min U}.  The bound is per centre, so a
// far-off centre with a large norm does not widen anyone's window.
//
// Persistent, warp-specialised kernel.  The (head, 128-token tile) units of
// the whole call are split into equal contiguous ranges, one per CTA (one CTA
// per SM), so a CTA changes head at most a few times; at each change the
// CTA reloads that head's centres into shared memory.  Roles:
//   warp 17 (TMA): loads X tiles [128][d] (bf16, 128-byte swizzle) from
//     [T][H][d] into a ring of stages, as far ahead as the ring allows;
//   warp 16 (MMA): one thread issues P = X mu^T (M = 128, K = d, fp32 in
//     TMEM) in sub-units of up to 256 centre columns; tiles alternate between
//     two epilogue groups, each with its own 256-column TMEM accumulator, so
//     the tensor core fills one group's accumulator while the other reads;
//   warps 0-7 and 8-15 (two epilogue groups, even and odd tiles): two threads
//     per token (one per half of the TMEM columns and of the channels) compute
//     L_j, keep the three smallest, release the accumulator, and decide: one
//     candidate: done; two: the two threads of the token score one each with
//     the specified distance; three or more: the warp pair scores every
//     centre of the head with the specified distance (rare).  Lowest index
//     wins ties everywhere.  Then the residual against the chosen centre is
//     quantised (Eq. 1) per group and packed, each thread covering its half
//     of the channels, and the X stage is released.
#pragma once

#include <cuda.h>

#include "codec.cuh"
#include "common.cuh"

namespace kvq {

constexpr int kFltRows = 128;
constexpr int kFltGroupThreads = 256;            // one epilogue group: 8 warps
constexpr int kFltMmaWarp = 16, kFltTmaWarp = 17;
constexpr int kFltThreads = 576;
constexpr int kFltMaxC = 512;
constexpr int kFltAccCols = 256;                 // columns of one group's TMEM accumulator
constexpr int kFltMaxStages = 4;

struct FilterArgs {
    int64_t T;
    int H;
    int C;
    int Cpad;          // C rounded up to a multiple of 32
    int stages;        // X tiles in the ring (2 .. kFltMaxStages)
    int64_t ntiles;    // 128-token tiles per head
    const uint16_t *cent;
    uint16_t *idx;
    uint8_t *codes;
    void *meta;        // [H][T][d/G][2] float, or binary16 when meta16
    int assign_only;
    int meta16;
    float kappa;       // k of the certified bound (see above)
    uint8_t *codes2;   // second residual stage (kernel instantiated with TWO):
    float *meta2;      // as codes, and as meta in binary32
};

// pair exchange of one epilogue group, two slots by tile parity:
// float4 [2][2][128] | int [2][2][128] | float4 [128]
constexpr uint32_t kFltPairBytes = 12288u;

__host__ __device__ constexpr uint32_t flt_tile_bytes(int D) { return (uint32_t)(D * 2 * kFltRows); }

__host__ __device__ constexpr uint32_t flt_smem_bytes(int D, int Cpad, int stages)
{
    // X ring | centres | A_j, |mu_j| | pair exchange x 2 groups | barriers + slots
    return (uint32_t)stages * flt_tile_bytes(D) + (uint32_t)(Cpad * D * 2) + (uint32_t)(Cpad * 8) +
           2u * kFltPairBytes + 256u;
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

// One residual stage of channels [half*CH, half*CH + CH) of one token: the
// values come from val(uu, v8) (the 8 channels of unit uu of the half; group
// g holds units g G/8 .. (g + 1) G/8 - 1), are quantised per group (Eq. 1)
// and packed.  Three phases over all of the thread's groups at once, so that
// the groups' chains (min/max, the two IEEE divisions of Eq. 1, the codes)
// run side by side: (1) min and max of every group, (2) Eq. 1 parameters of
// every group, (3) codes, asking val again.  Group min/max are those of a
// strict scan in channel order; the two differ only in the sign of a zero
// extreme, for which the group is rescanned in order.  The groups'
// parameters are copied to gq_out / gf_out unless these are null.
template <int CH, int BITS, int G, class Val>
__device__ __forceinline__ void quantise_half(const Val &val, uint8_t *codes_dst, void *meta_dst, bool meta16,
                                              GroupQ *gq_out, GroupFast *gf_out)
{
    constexpr int kPerWord = 32 / BITS;
    constexpr int kWords = CH * BITS / 32;
    constexpr int NG = CH / G;
    // (1) min / max of every group
    float mn[NG], mx[NG];
#pragma unroll
    for (int g = 0; g < NG; ++g) {
        float r8[8];
        val(g * (G / 8), r8);
        float a = fminf(r8[0], r8[1]), b = fmaxf(r8[0], r8[1]);
#pragma unroll
        for (int c = 2; c < 8; c += 2) {
            a = fmin3(a, r8[c], r8[c + 1]);
            b = fmax3(b, r8[c], r8[c + 1]);
        }
#pragma unroll
        for (int uu = 1; uu < G / 8; ++uu) {
            val(g * (G / 8) + uu, r8);
#pragma unroll
            for (int c = 0; c < 8; c += 2) {
                a = fmin3(a, r8[c], r8[c + 1]);
                b = fmax3(b, r8[c], r8[c + 1]);
            }
        }
        mn[g] = a;
        mx[g] = b;
    }
#pragma unroll
    for (int g = 0; g < NG; ++g) {
        if (mn[g] == 0.0f || mx[g] == 0.0f) {
            // a zero extreme: take its sign exactly as the ordered strict scan does
            float a = 0.0f, b = 0.0f;
            for (int uu = 0; uu < G / 8; ++uu) {
                float r8[8];
                val(g * (G / 8) + uu, r8);
                for (int c = 0; c < 8; ++c) {
                    if (uu == 0 && c == 0) {
                        a = r8[0];
                        b = r8[0];
                    } else {
                        if (r8[c] < a) a = r8[c];
                        if (r8[c] > b) b = r8[c];
                    }
                }
            }
            mn[g] = a;
            mx[g] = b;
        }
    }
    // (2) Eq. 1 parameters of every group
    GroupQ gq[NG];
    GroupFast gf[NG];
#pragma unroll
    for (int g = 0; g < NG; ++g)
        gq[g] = group_params_store(mn[g], mx[g], BITS, meta16, meta_dst, g);
#pragma unroll
    for (int g = 0; g < NG; ++g)
        gf[g] = group_fast(gq[g], mn[g], mx[g]);
    // (3) codes
    uint32_t words[kWords];
#pragma unroll
    for (int w = 0; w < kWords; ++w)
        words[w] = 0u;
#pragma unroll
    for (int g = 0; g < NG; ++g) {
        if (gf[g].fast) {  // one branch per group, not per value
#pragma unroll
            for (int uu = 0; uu < G / 8; ++uu) {
                float r8[8];
                val(g * (G / 8) + uu, r8);
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const int c = g * G + uu * 8 + k;
                    words[c / kPerWord] += quant_code_fast<BITS>(r8[k], gf[g]) << ((c % kPerWord) * BITS);
                }
            }
        } else {
#pragma unroll
            for (int uu = 0; uu < G / 8; ++uu) {
                float r8[8];
                val(g * (G / 8) + uu, r8);
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const int c = g * G + uu * 8 + k;
                    words[c / kPerWord] += quant_code(r8[k], gq[g], BITS) << ((c % kPerWord) * BITS);
                }
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
    if (gq_out) {
#pragma unroll
        for (int g = 0; g < NG; ++g) {
            gq_out[g] = gq[g];
            gf_out[g] = gf[g];
        }
    }
}

// Residual r = x - mu[best] of channels [half*CH, half*CH + CH) of one token,
// read from the swizzled tiles, quantised per group (Eq. 1) and packed.  With
// TWO, a second residual stage follows: the error e = r - (q - z) s the first
// stage leaves (each operation rounded in binary32) is quantised on the same
// groups with the same code width into codes2_dst / meta2_dst (binary32
// {s, z}).
template <int CH, int BITS, int G, bool TWO>
__device__ __forceinline__ void encode_residual_smem(const uint8_t *sX, const uint8_t *sMu, int Cpad, int row,
                                                     int best, int half, uint8_t *codes_dst, void *meta_dst,
                                                     bool meta16, uint8_t *codes2_dst, float *meta2_dst)
{
    constexpr int NG = CH / G;
    // residual of the 8 channels of unit uu of this thread's half
    auto residual = [&](int uu, float *r8) {
        const int u = half * (CH / 8) + uu;
        const uint4 xw = *reinterpret_cast<const uint4 *>(sX + sw128_unit_offset(row, u, kFltRows));
        const uint4 mw = *reinterpret_cast<const uint4 *>(sMu + sw128_unit_offset(best, u, Cpad));
        const uint32_t xa[4] = {xw.x, xw.y, xw.z, xw.w}, ma[4] = {mw.x, mw.y, mw.z, mw.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float2 d = sub2(make_float2(bf16_lo(xa[k]), bf16_hi(xa[k])), make_float2(bf16_lo(ma[k]), bf16_hi(ma[k])));
            r8[2 * k] = d.x;
            r8[2 * k + 1] = d.y;
        }
    };
    GroupQ gq[NG];
    GroupFast gf[NG];
    quantise_half<CH, BITS, G>(residual, codes_dst, meta_dst, meta16, TWO ? gq : nullptr, TWO ? gf : nullptr);
    if constexpr (TWO) {
        // error of the first stage: the code again (quant_code_fast equals
        // quant_code), then r - (q - z) s
        auto error = [&](int uu, float *e8) {
            const int g = uu / (G / 8);
            residual(uu, e8);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const uint32_t q = gf[g].fast ? quant_code_fast<BITS>(e8[k], gf[g]) : quant_code(e8[k], gq[g], BITS);
                e8[k] = __fsub_rn(e8[k], __fmul_rn(__fsub_rn((float)q, gq[g].z), gq[g].s));
            }
        };
        quantise_half<CH, BITS, G>(error, codes2_dst, meta2_dst, false, nullptr, nullptr);
    }
}

// Bounded mbarrier wait that also gives up at once when another role of the
// CTA has given up (abort flag in shared memory); on its own expiry it raises
// the device status and sets the flag.
__device__ __forceinline__ bool flt_wait(uint32_t bar, uint32_t parity, volatile int *abort)
{
    const uint32_t limit = c_wait_limit;
    for (uint32_t i = 0; i < limit; ++i) {
        if (mbar_try_wait(bar, parity))
            return true;
        if ((i & 255u) == 255u && *abort)
            return false;
    }
    raise_status(DEVSTAT_TIMEOUT);
    *abort = 1;
    return false;
}

// Specified binary32 distances of row `row` of the X tile to the centres
// j = j0 + 64 m (m = 0, 1, ...) below C, two chains at a time; returns the
// smallest (distance, index), lowest index on ties.
template <int D>
__device__ __forceinline__ void flt_bruteforce_part(const uint8_t *sX, const uint8_t *sMu, int Cpad, int C, int row,
                                                    int j0, float &bd, int &bj)
{
    bd = INFINITY;
    bj = -1;
    for (int j = j0; j < C; j += 128) {
        const int j2 = j + 64;
        const float da = spec_distance_smem<D>(sX, sMu, Cpad, row, j);
        const float db = j2 < C ? spec_distance_smem<D>(sX, sMu, Cpad, row, j2) : INFINITY;
        if (bj < 0 || da < bd) {
            bd = da;
            bj = j;
        }
        if (j2 < C && db < bd) {
            bd = db;
            bj = j2;
        }
    }
}

// Named barrier 1 + 4 g + q over the 64 threads of one row group (warps w and
// w + 4 of epilogue group g).
__device__ __forceinline__ void flt_pair_sync(int g, int q)
{
    switch ((g << 2) | (q & 3)) {
    case 0: named_barrier_sync<1>(64); break;
    case 1: named_barrier_sync<2>(64); break;
    case 2: named_barrier_sync<3>(64); break;
    case 3: named_barrier_sync<4>(64); break;
    case 4: named_barrier_sync<5>(64); break;
    case 5: named_barrier_sync<6>(64); break;
    case 6: named_barrier_sync<7>(64); break;
    default: named_barrier_sync<8>(64); break;
    }
}

// L'_j of 32 columns (L_j + k |x|^2, the same shift for every j of the row),
// with the chunk-local index in the low 5 mantissa bits, merged into the three
// smallest of two independent chains.
__device__ __forceinline__ void flt_scan_chunk(const float *p, const float *sA, const float *sM, float nB, float &a1,
                                               float &a2, float &a3, float &e1, float &e2, float &e3)
{
    auto pair_into = [](float pa, float pb, float &m1, float &m2, float &m3) {
        // sort the pair, then merge it into the three smallest (k-th smallest
        // of two sorted lists = min over i + j = k of max(a_i, b_j))
        const float lo = fminf(pa, pb), hi = fmaxf(pa, pb);
        const float n3 = fmin3(m3, fmaxf(m2, lo), fmaxf(m1, hi));
        const float n2 = fmin3(fmaxf(m1, lo), m2, hi);
        m1 = fminf(m1, lo);
        m2 = n2;
        m3 = n3;
    };
    const float4 *A4 = reinterpret_cast<const float4 *>(sA);
    const float4 *M4 = reinterpret_cast<const float4 *>(sM);
#pragma unroll
    for (int i4 = 0; i4 < 8; ++i4) {
        const float4 av = A4[i4], mv = M4[i4];
        // L' = (A_j - 2 p_j) - 2 k |x| |mu_j|, pairs of columns at a time
        const float2 t01 = fma2(make_float2(-2.0f, -2.0f), make_float2(p[4 * i4], p[4 * i4 + 1]),
                                make_float2(av.x, av.y));
        const float2 t23 = fma2(make_float2(-2.0f, -2.0f), make_float2(p[4 * i4 + 2], p[4 * i4 + 3]),
                                make_float2(av.z, av.w));
        const float2 l01 = fma2(make_float2(nB, nB), make_float2(mv.x, mv.y), t01);
        const float2 l23 = fma2(make_float2(nB, nB), make_float2(mv.z, mv.w), t23);
        const uint32_t i = (uint32_t)(i4 * 4);
        const float pk0 = __uint_as_float((__float_as_uint(l01.x) & ~31u) | i);
        const float pk1 = __uint_as_float((__float_as_uint(l01.y) & ~31u) | (i + 1));
        const float pk2 = __uint_as_float((__float_as_uint(l23.x) & ~31u) | (i + 2));
        const float pk3 = __uint_as_float((__float_as_uint(l23.y) & ~31u) | (i + 3));
        pair_into(pk0, pk1, a1, a2, a3);
        pair_into(pk2, pk3, e1, e2, e3);
    }
}


template <int D, int BITS, int G, bool TWO>
__global__ void __launch_bounds__(kFltThreads, 1)
    encode_filter_kernel(const __grid_constant__ CUtensorMap tmap_x, FilterArgs a)
{
    static_assert(G <= D / 2, "a group must lie inside one half of the channels");
    constexpr int CH = D / 2;             // channels per epilogue thread
    constexpr int kSubChunks = kFltAccCols / 32;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int Cpad = a.Cpad, S = a.stages;
    const uint32_t tile_bytes = flt_tile_bytes(D);
    uint8_t *sXring = smem;
    uint8_t *sMu = smem + S * tile_bytes;
    float *sA = reinterpret_cast<float *>(sMu + Cpad * D * 2);  // A_j = N_j - k |mu_j|^2 (inf past C)
    float *sM = sA + Cpad;                                      // |mu_j| (0 past C)
    uint8_t *sPairBase = reinterpret_cast<uint8_t *>(sM + Cpad);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sPairBase + 2 * kFltPairBytes);
    // bars: xfull[4] xempty[4] afull[2] aempty[2] drain
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 13);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 2);
    auto xfull = [&](int st) { return smem_u32(bars + st); };
    auto xempty = [&](int st) { return smem_u32(bars + kFltMaxStages + st); };
    auto afull = [&](int g) { return smem_u32(bars + 2 * kFltMaxStages + g); };
    auto aempty = [&](int g) { return smem_u32(bars + 2 * kFltMaxStages + 2 + g); };
    const uint32_t bar_drain = smem_u32(bars + 2 * kFltMaxStages + 4);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    if (warp == 0)
        tmem_alloc(smem_u32(tmem_slot), 2 * kFltAccCols);
    if (tid == 0) {
        for (int st = 0; st < kFltMaxStages; ++st) {
            mbar_init(xfull(st), 1);
            mbar_init(xempty(st), kFltGroupThreads / 32);
        }
        for (int g = 0; g < 2; ++g) {
            mbar_init(afull(g), 1);
            mbar_init(aempty(g), kFltGroupThreads / 32);
        }
        mbar_init(bar_drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t aMu = smem_u32(sMu);

    const int nsub = (Cpad + kFltAccCols - 1) / kFltAccCols;
    const int64_t units = (int64_t)a.H * a.ntiles;
    const int64_t u_begin = (int64_t)blockIdx.x * units / gridDim.x;
    const int64_t u_end = (int64_t)(blockIdx.x + 1) * units / gridDim.x;

    // epilogue thread geometry: group, row (TMEM lane) and half of columns /
    // channels
    const int grp = warp >> 3, w8 = warp & 7;
    const int half = w8 >> 2;
    const int row = (w8 & 3) * 32 + lane;
    const uint32_t lane_off = ((uint32_t)(w8 & 3) * 32u) << 16;
    float4 *sPair2 = reinterpret_cast<float4 *>(sPairBase + grp * kFltPairBytes);  // [2][2][128]
    int *sPairC2 = reinterpret_cast<int *>(sPair2 + 2 * 2 * 128);                   // [2][2][128]
    float4 *sWin = reinterpret_cast<float4 *>(sPairC2 + 2 * 2 * 128);               // [128]

    int64_t tile_seq = 0;  // tiles this CTA has handled (X ring position, group = parity)
    uint32_t mma_issued = 0;
    int64_t tma_last = -1;  // TMA lane: the last tile whose X load it issued
    for (int64_t u = u_begin; u < u_end;) {
        const int h = (int)(u / a.ntiles);
        const int64_t seg_end = min(u_end, (int64_t)(h + 1) * a.ntiles);
        const int64_t tile0 = u - (int64_t)h * a.ntiles;
        const int n = (int)(seg_end - u);

        // ---- centres of head h -> swizzled K-major tile [D/64][Cpad][128 B];
        // A_j and |mu_j|
        __syncthreads();  // the previous segment is fully consumed
        const uint16_t *cent_h = a.cent + (int64_t)h * a.C * D;
        for (int e = tid; e < Cpad * (D / 8); e += kFltThreads) {
            const int j = e / (D / 8), uu = e % (D / 8);
            const uint4 w = j < a.C ? __ldg(reinterpret_cast<const uint4 *>(cent_h + (int64_t)j * D) + uu)
                                    : make_uint4(0, 0, 0, 0);
            *reinterpret_cast<uint4 *>(sMu + sw128_unit_offset(j, uu, Cpad)) = w;
        }
        for (int j = tid; j < Cpad; j += kFltThreads) {
            float A = INFINITY, m = 0.0f;
            if (j < a.C) {
                float nrm = 0.0f;
                for (int uu = 0; uu < D / 8; ++uu) {
                    float m8[8];
                    load_bf16x8(cent_h + (int64_t)j * D + uu * 8, m8);
#pragma unroll
                    for (int k = 0; k < 8; ++k)
                        nrm = fmaf(m8[k], m8[k], nrm);
                }
                m = sqrtf(nrm);
                A = fmaf(-a.kappa, nrm, nrm);
            }
            sA[j] = A;
            sM[j] = m;
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();

        if (warp == kFltTmaWarp) {
            // ------------------------------------------------------------ TMA
            if (lane == 0) {
                for (int k = 0; k < n && !*abort_flag; ++k) {
                    const int64_t seq = tile_seq + k;
                    const int st = (int)(seq % S);
                    if (seq >= S && !flt_wait(xempty(st), (uint32_t)(((seq / S) - 1) & 1), abort_flag))
                        break;
                    const uint32_t dst = smem_u32(sXring + st * tile_bytes);
                    mbar_arrive_expect_tx(xfull(st), tile_bytes);
                    const int t0 = (int)((tile0 + k) * kFltRows);
#pragma unroll
                    for (int ch = 0; ch < D / 64; ++ch)
                        tma_load_3d(dst + ch * (kFltRows * 128), &tmap_x, xfull(st), ch * 64, h, t0);
                    tma_last = seq;
                }
            }
        } else if (warp == kFltMmaWarp) {
            // ------------------------------------------------------------ MMA
            // issue order: for each pair of consecutive tiles (one per group),
            // sub-unit 0 of both, then sub-unit 1 of both, ... so neither
            // group's accumulator release holds up the other's MMAs
            if (lane == 0) {
                bool ok = true;
                for (int kb = 0; ok && kb < n; kb += 2) {
                    for (int sub = 0; ok && sub < nsub; ++sub) {
                        for (int kk = kb; ok && kk < kb + 2 && kk < n; ++kk) {
                            const int64_t seq = tile_seq + kk;
                            const int st = (int)(seq % S);
                            const int g = (int)(seq & 1);
                            if (sub == 0 && !(ok = flt_wait(xfull(st), (uint32_t)((seq / S) & 1), abort_flag)))
                                break;
                            const int64_t gsub = (seq >> 1) * nsub + sub;  // group g's sub-unit count
                            if (gsub >= 1 && !(ok = flt_wait(aempty(g), (uint32_t)((gsub - 1) & 1), abort_flag)))
                                break;
                            tc_fence_after();
                            const uint32_t aX = smem_u32(sXring + st * tile_bytes);
                            const int n0 = sub * kFltAccCols;
                            const int N = min(kFltAccCols, Cpad - n0);
                            const uint32_t idesc = idesc_f32acc(128, N, true, false, false);
#pragma unroll
                            for (int ks = 0; ks < D / 16; ++ks) {
                                const uint32_t aoff =
                                    (uint32_t)(ks >> 2) * (kFltRows * 128u) + (uint32_t)(ks & 3) * 32u;
                                const uint32_t boff = (uint32_t)(ks >> 2) * (uint32_t)(Cpad * 128) +
                                                      (uint32_t)n0 * 128u + (uint32_t)(ks & 3) * 32u;
                                umma_ss(tmem + (uint32_t)(g * kFltAccCols), sdesc_sw128(aX + aoff, 16, 1024),
                                        sdesc_sw128(aMu + boff, 16, 1024), idesc, ks > 0 ? 1u : 0u);
                            }
                            umma_commit(afull(g));
                            ++mma_issued;
                        }
                    }
                }
            }
        } else {
            // ------------------------------------------------------------ epilogue group grp
            bool ok = true;
            for (int k = 0; k < n; ++k) {
                const int64_t seq = tile_seq + k;
                if ((int)(seq & 1) != grp)
                    continue;
                const int st = (int)(seq % S);
                const uint8_t *sX = sXring + st * tile_bytes;
                float4 *sPair = sPair2 + ((seq >> 1) & 1) * 256;
                int *sPairC = sPairC2 + ((seq >> 1) & 1) * 256;
                ok = ok && __all_sync(0xffffffffu, flt_wait(xfull(st), (uint32_t)((seq / S) & 1), abort_flag));
                // (1) |x|^2 over this thread's channel half
                float xx = 0.0f;
                if (ok) {
#pragma unroll
                    for (int uu = half * (CH / 8); uu < (half + 1) * (CH / 8); ++uu) {
                        const uint4 w = *reinterpret_cast<const uint4 *>(sX + sw128_unit_offset(row, uu, kFltRows));
                        const uint32_t wa[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            xx = fmaf(bf16_lo(wa[q]), bf16_lo(wa[q]), xx);
                            xx = fmaf(bf16_hi(wa[q]), bf16_hi(wa[q]), xx);
                        }
                    }
                }
                // both threads of the row need |x|: exchange the halves
                sPair[half * 128 + row].x = xx;
                flt_pair_sync(grp, w8 & 3);
                const float xn = sqrtf(xx + sPair[(half ^ 1) * 128 + row].x);
                const float nB = -2.0f * a.kappa * xn;
                // (2) L'_j over this thread's chunks of every sub-unit; the
                // chunk-local column index rides in the low 5 mantissa bits,
                // so one pass keeps the three smallest values (the margin in k
                // absorbs the <= 31 ulp this perturbs them); global chunk ids
                // are kept beside them
                float b1 = INFINITY, b2 = INFINITY, b3 = INFINITY;
                int k1 = 0, k2 = 0, k3 = 0;
                for (int sub = 0; sub < nsub; ++sub) {
                    const int64_t gsub = (seq >> 1) * nsub + sub;
                    ok = ok && __all_sync(0xffffffffu, flt_wait(afull(grp), (uint32_t)(gsub & 1), abort_flag));
                    if (!ok)
                        break;
                    tc_fence_after();
                    const int n0 = sub * kFltAccCols;
                    const int nch = min(kSubChunks, (Cpad - n0) / 32);
                    const int c_lo = half == 0 ? 0 : (nch + 1) / 2;
                    const int c_hi = half == 0 ? (nch + 1) / 2 : nch;
                    const uint32_t tbase = tmem + lane_off + (uint32_t)(grp * kFltAccCols);
#pragma unroll
                    for (int kk = 0; kk < kSubChunks / 2; ++kk) {
                        const int c = c_lo + kk;
                        if (c < c_hi) {
                            uint32_t pw[32];
                            tmem_ld32_nowait(tbase + (uint32_t)(c * 32), pw);
                            tmem_ld_wait();
                            float a1 = INFINITY, a2 = INFINITY, a3 = INFINITY;
                            float e1 = INFINITY, e2 = INFINITY, e3 = INFINITY;
                            flt_scan_chunk(reinterpret_cast<const float *>(pw), sA + n0 + c * 32, sM + n0 + c * 32, nB,
                                           a1, a2, a3, e1, e2, e3);
                            const int gc = sub * kSubChunks + c;
                            top3_insert(fminf(a1, e1), gc, b1, k1, b2, k2, b3, k3);
                            top3_insert(fmin3(a2, fmaxf(a1, e1), e2), gc, b1, k1, b2, k2, b3, k3);
                            top3_insert(fminf(fmin3(a3, fmaxf(a2, e1), fmaxf(a1, e2)), e3), gc, b1, k1, b2, k2, b3, k3);
                        }
                    }
                    // accumulator read: the MMA may overwrite it
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0)
                        mbar_arrive(aempty(grp));
                }
                // (3) exchange with the partner thread of this row (warps w and
                // w+4 of the group); both then hold the row's three smallest
                // values, half-0 entries first on equal values.  Both warps
                // always meet here and carry their status (bit 31) along, so
                // every later named barrier is taken by both or by neither.
                sPair[half * 128 + row] = make_float4(xx, b1, b2, b3);
                sPairC[half * 128 + row] = (k1 | (k2 << 8) | (k3 << 16)) | (ok ? 0 : (int)0x80000000u);
                flt_pair_sync(grp, w8 & 3);
                const int oc_raw = sPairC[(half ^ 1) * 128 + row];
                ok = ok && oc_raw >= 0;
                if (ok) {
                    const float4 other = sPair[(half ^ 1) * 128 + row];
                    const int oc = oc_raw;
                    float g1, g2, g3;
                    int h1, h2, h3;
                    {
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
                    int best = h1 * 32 + (int)(__float_as_uint(g1) & 31u);
                    // threshold: U'(best) = L'(best) + 2 k (|x| + |mu_best|)^2
                    const float r1 = xn + sM[min(best, Cpad - 1)];
                    const float thr = g1 + 2.0f * a.kappa * r1 * r1;
                    const bool finite = thr < INFINITY;
                    const bool pair_case = finite && !(g2 > thr) && g3 > thr;        // two candidates
                    const bool wide_case = !finite || (!(g2 > thr) && !(g3 > thr));  // three or more
                    // two candidates: each thread of the pair scores one with the
                    // specified distance; the smaller wins, the lower index on a tie
                    if (__any_sync(0xffffffffu, pair_case)) {
                        const int j1 = best, j2 = h2 * 32 + (int)(__float_as_uint(g2) & 31u);
                        float dmine = 0.0f;
                        if (pair_case) {
                            dmine = spec_distance_smem<D>(sX, sMu, Cpad, row, half == 0 ? j1 : j2);
                            if (half == 0)
                                sWin[row].x = dmine;
                        }
                        flt_pair_sync(grp, w8 & 3);
                        if (pair_case && half == 1) {
                            const float d1 = sWin[row].x, d2 = dmine;
                            const int lo = j1 < j2 ? j1 : j2;
                            const int hi = j1 < j2 ? j2 : j1;
                            const float dlo = j1 < j2 ? d1 : d2, dhi = j1 < j2 ? d2 : d1;
                            sWin[row].y = __int_as_float(dhi < dlo ? hi : lo);
                        }
                        flt_pair_sync(grp, w8 & 3);
                        if (pair_case)
                            best = __float_as_int(sWin[row].y);
                    }
                    // three or more candidates (rare): the two warps of this row
                    // group score every centre of the head for each such row,
                    // lane-parallel over the centres, and take the smallest
                    // (distance, index).  Both warps see the same flags.
                    uint32_t wide = __ballot_sync(0xffffffffu, wide_case);
                    while (wide) {
                        const int wl = __ffs(wide) - 1;
                        wide &= wide - 1u;
                        const int wrow = (w8 & 3) * 32 + wl;
                        float bd;
                        int bj;
                        flt_bruteforce_part<D>(sX, sMu, Cpad, a.C, wrow, half * 32 + lane, bd, bj);
#pragma unroll
                        for (int off = 16; off > 0; off >>= 1) {
                            const float od = __shfl_xor_sync(0xffffffffu, bd, off);
                            const int oj = __shfl_xor_sync(0xffffffffu, bj, off);
                            if (oj >= 0 && (bj < 0 || od < bd || (od == bd && oj < bj))) {
                                bd = od;
                                bj = oj;
                            }
                        }
                        if (lane == 0)
                            reinterpret_cast<float2 *>(sWin + wrow)[half] = make_float2(bd, __int_as_float(bj));
                        flt_pair_sync(grp, w8 & 3);
                        if (lane == wl) {
                            const float4 wv = sWin[wrow];
                            const int j0 = __float_as_int(wv.y), jj1 = __float_as_int(wv.w);
                            best = (j0 < 0 || (jj1 >= 0 && (wv.z < wv.x || (wv.z == wv.x && jj1 < j0)))) ? jj1 : j0;
                        }
                        flt_pair_sync(grp, w8 & 3);
                    }
                    if (best < 0 || best >= a.C)
                        best = 0;  // unreachable for finite inputs

                    // (4) residual + Eq. 1 + packing for this thread's channel half
                    const int64_t t = (tile0 + k) * kFltRows + row;
                    if (t < a.T) {
                        const int64_t th = (int64_t)h * a.T + t;
                        if (half == 0)
                            a.idx[th] = (uint16_t)best;
                        if (!a.assign_only)
                            encode_residual_smem<CH, BITS, G, TWO>(
                                sX, sMu, Cpad, row, best, half, a.codes + th * (D * BITS / 8) + half * (CH * BITS / 8),
                                static_cast<uint8_t *>(a.meta) + (th * (D / G) + half * (CH / G)) * (a.meta16 ? 4 : 8),
                                a.meta16 != 0,
                                TWO ? a.codes2 + th * (D * BITS / 8) + half * (CH * BITS / 8) : nullptr,
                                TWO ? a.meta2 + (th * (D / G) + half * (CH / G)) * 2 : nullptr);
                    }
                }
                // X stage read: the TMA may refill it
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(xempty(st));
            }
        }
        tile_seq += n;
        u = seg_end;
    }
    // drain: the X loads of the last tiles issued have landed (after a
    // give-up nobody else waits for them) before the CTA may exit ...
    if (warp == kFltTmaWarp && lane == 0) {
        for (int64_t seq = tma_last - S + 1 < 0 ? 0 : tma_last - S + 1; seq <= tma_last; ++seq) {
            uint32_t spins = 0;
            while (!mbar_try_wait(xfull((int)(seq % S)), (uint32_t)((seq / S) & 1)) && ++spins < kSpinLimit) {
            }
        }
    }
    // ... and every MMA issued has completed before TMEM is freed
    if (warp == kFltMmaWarp && lane == 0 && mma_issued > 0) {
        umma_commit(bar_drain);
        uint32_t spins = 0;
        while (!mbar_try_wait(bar_drain, 0) && ++spins < kSpinLimit) {
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0)
        tmem_dealloc(tmem, 2 * kFltAccCols);
}

}  // namespace kvq

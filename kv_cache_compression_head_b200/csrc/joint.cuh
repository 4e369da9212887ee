// joint.cuh -- joint head-channel linear encoder / decoder of the residual
// (NanoKV page, abstract and Fig. 4(a,b): joint head-channel residuals are
// encoded into low-bit (INT4) coefficients; the decoder reconstructs them and
// adds back the centres).
//
// Encoder, per 128-token tile (one CTA):
//   R[t][i] = bf16( x[t][h][c] - mu_h[idx[h][t]][c] ),  i = h d + c
//   Coef[t][n] = sum_i R[t][i] W_enc[i][n]    (tcgen05, M = 128, N = r, K = H d,
//                bf16 operands, binary32 accumulation in TMEM)
//   per row, Eq. 1 on each group of G coefficients -> packed codes, {s, z}
// The A operand (R) is built in shared memory by the CTA's threads, 64
// channels per K-block; W_enc [H d][r] (r contiguous) is the MN-major B
// operand.  A ring of four stages: TMA brings K-blocks up to three ahead while
// the threads rebuild block k in place and the MMAs of earlier blocks run.
//
// Decoder, per 128-token tile and 128 output channels (one head):
//   c^[t][n] = (q - z) s                       (binary32, the quantiser's grid)
//   R^[t][i] = sum_n c^[t][n] W_dec[n][i]      (tcgen05, c^ as bf16 hi + lo
//                parts against bf16 W_dec, binary32 accumulation)
//   x^[t][h][c] = mu_h[idx[h][t]][c] + R^[t][h d + c]
#pragma once

#include "codec.cuh"
#include "common.cuh"

namespace kvq {

constexpr int kJRows = 128;      // tokens per CTA
constexpr int kJThreads = 128;   // decoder helpers: one thread per token row (TMEM lane)
constexpr int kJEThreads = 256;  // encoder: two threads per token row
constexpr int kJKBlock = 64;     // channels per K-block

struct JointEncArgs {
    const uint16_t *x;     // [T][H][D] bf16
    const uint16_t *cent;  // [H][C][D]
    const uint16_t *idx;   // [H][T]
    const uint16_t *w;     // [H*D][r] bf16
    int64_t T;
    int H, D, C, r, bits, G;
    uint8_t *codes;        // [T][r*bits/8]
    float *meta;           // [T][r/G][2]
    float *coef_out;       // [T][r] or null
};

// shared memory: kJEStages stages of {A: 128 x 64 bf16 (16 KB), B: 64 x r bf16}
constexpr int kJEStages = 4;
__host__ __device__ constexpr uint32_t joint_enc_stage_bytes(int r) { return 16384u + 64u * (uint32_t)r * 2u; }
__host__ __device__ constexpr uint32_t joint_enc_smem_bytes(int r)
{
    return (uint32_t)kJEStages * joint_enc_stage_bytes(r) + 128u;
}

__host__ __device__ constexpr uint32_t pow2_cols(int n)
{
    uint32_t c = 32;
    while (c < (uint32_t)n)
        c <<= 1;
    return c;
}

// Quantise groups g0, g0 + gstep, ... of one row's r coefficients held in
// TMEM (columns [0, r) of this thread's lane) with Eq. 1 per group of G, and
// store codes / {s, z} (and the binary32 coefficients themselves when
// coef_row is set).
template <int G, int BITS>
__device__ __forceinline__ void joint_quant_row(uint32_t trow, int r, uint8_t *codes_row, float2 *meta_row,
                                                float *coef_row, int g0, int gstep)
{
    static_assert(G % 16 == 0 && G <= 64, "group of 16, 32 or 64 coefficients");
    constexpr int kWords = G * BITS / 32;
    for (int g = g0; g < r / G; g += gstep) {
        float v[G];
#pragma unroll
        for (int c = 0; c < G; c += 16) {
            uint32_t w16[16];
            asm volatile(
                "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, "
                "[%16];"
                : "=r"(w16[0]), "=r"(w16[1]), "=r"(w16[2]), "=r"(w16[3]), "=r"(w16[4]), "=r"(w16[5]), "=r"(w16[6]),
                  "=r"(w16[7]), "=r"(w16[8]), "=r"(w16[9]), "=r"(w16[10]), "=r"(w16[11]), "=r"(w16[12]),
                  "=r"(w16[13]), "=r"(w16[14]), "=r"(w16[15])
                : "r"(trow + (uint32_t)(g * G + c)));
            asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
            for (int k = 0; k < 16; ++k)
                v[c + k] = __uint_as_float(w16[k]);
        }
        if (coef_row) {
#pragma unroll
            for (int c = 0; c < G; c += 4)
                *reinterpret_cast<float4 *>(coef_row + g * G + c) = make_float4(v[c], v[c + 1], v[c + 2], v[c + 3]);
        }
        if (!codes_row)
            continue;
        float mn = v[0], mx = v[0];
#pragma unroll
        for (int c = 1; c < G; ++c) {
            if (v[c] < mn) mn = v[c];
            if (v[c] > mx) mx = v[c];
        }
        const GroupQ gq = group_params(mn, mx, BITS);
        meta_row[g] = make_float2(gq.s, gq.z);
        uint32_t wv[kWords];
#pragma unroll
        for (int w = 0; w < kWords; ++w)
            wv[w] = 0u;
        quant_group_into<G, BITS>(v, gq, mn, mx, wv, 0);
        uint32_t *words = reinterpret_cast<uint32_t *>(codes_row) + g * kWords;
#pragma unroll
        for (int w = 0; w < kWords; ++w)
            words[w] = wv[w];
    }
}

// One CTA per 128-token tile, K-blocks of 64 channels in a ring of kJEStages
// stages.  Thread 0 loads each block's x tile (3-D map over [T][H][D], 128-byte
// swizzle: already the K-major A layout) and W_enc rows (2-D map, MN-major B)
// with TMA three blocks ahead and issues the MMAs.  All 256 threads (two per
// token row, 32 channels each) rewrite their units of the x tile in place as
// A = bf16(x - mu[idx]), the centre units fetched one block ahead.  In the
// epilogue the two threads of a row (warps w and w + 4 share the TMEM lanes)
// quantise alternate groups.
template <int G, int BITS>
__global__ void __launch_bounds__(kJEThreads, 1)
    joint_encode_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
                        JointEncArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t stage_bytes = joint_enc_stage_bytes(a.r);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kJEStages * stage_bytes);  // full[4], done[4]
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 2 * kJEStages);
    auto full = [&](int st) { return smem_u32(bars + st); };
    auto done = [&](int st) { return smem_u32(bars + kJEStages + st); };
    const int tid = threadIdx.x, warp = tid >> 5;
    const int row = tid & 127, half = tid >> 7;
    const int64_t t0 = (int64_t)blockIdx.x * kJRows;
    const int64_t t = t0 + row;
    const bool valid = t < a.T;
    const uint32_t ncols = pow2_cols(a.r);
    const int nk = a.H * a.D / kJKBlock;
    const uint32_t tx_bytes = stage_bytes;

    if (warp == 0)
        tmem_alloc(smem_u32(tmem_slot), ncols);
    if (tid == 0) {
        for (int st = 0; st < kJEStages; ++st) {
            mbar_init(full(st), 1);
            mbar_init(done(st), 1);
        }
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t idesc = idesc_f32acc(128, a.r, true, false, true);  // bf16, B MN-major
    auto issue_loads = [&](int kb) {  // thread 0: TMA of block kb into its stage
        const int st = kb % kJEStages;
        uint8_t *sA = smem + (uint32_t)st * stage_bytes;
        const int i0 = kb * kJKBlock;
        mbar_arrive_expect_tx(full(st), tx_bytes);
        tma_load_3d(smem_u32(sA), &tmap_x, full(st), i0 % a.D, i0 / a.D, (int)t0);
        for (int c = 0; c < a.r / 64; ++c)
            tma_load_2d(smem_u32(sA + 16384u + (uint32_t)c * 8192u), &tmap_w, full(st), c * 64, i0);
    };
    if (tid == 0)
        for (int kb = 0; kb < kJEStages - 1 && kb < nk; ++kb)
            issue_loads(kb);

    // centre units of this thread's 32 channels of block kb (one block ahead)
    int jh = -1, j = 0;
    auto fetch_mu = [&](int kb, uint4 *mu) {
        const int i0 = kb * kJKBlock, h = i0 / a.D, c0 = i0 % a.D;
        if (!valid)
            return;
        if (h != jh) {
            jh = h;
            j = a.idx[(int64_t)h * a.T + t];
            if (j >= a.C) {
                raise_status(DEVSTAT_BAD_INDEX);
                j = 0;
            }
        }
        const uint4 *src = reinterpret_cast<const uint4 *>(a.cent + ((int64_t)h * a.C + j) * a.D + c0) + 4 * half;
#pragma unroll
        for (int u = 0; u < 4; ++u)
            mu[u] = __ldg(src + u);
    };
    uint4 mu_next[4];
    fetch_mu(0, mu_next);
    bool ok = true;

    for (int kb = 0; kb < nk; ++kb) {
        const int s = kb % kJEStages;
        uint8_t *sA = smem + (uint32_t)s * stage_bytes;
        uint4 mu[4];
#pragma unroll
        for (int u = 0; u < 4; ++u)
            mu[u] = mu_next[u];
        if (kb + 1 < nk)
            fetch_mu(kb + 1, mu_next);
        ok = mbar_wait(full(s), (uint32_t)((kb / kJEStages) & 1)) && ok;
        // A in place: this thread's 4 units of its row
#pragma unroll
        for (int uu = 0; uu < 4; ++uu) {
            const int u = 4 * half + uu;
            uint4 *p = reinterpret_cast<uint4 *>(sA + sw128_unit_offset(row, u, kJRows));
            uint4 w = make_uint4(0, 0, 0, 0);
            if (valid) {
                const uint4 xw = *p;
                const uint32_t xa[4] = {xw.x, xw.y, xw.z, xw.w}, ma[4] = {mu[uu].x, mu[uu].y, mu[uu].z, mu[uu].w};
                uint32_t o[4];
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    o[k] = pack_bf16x2(__fsub_rn(bf16_lo(xa[k]), bf16_lo(ma[k])),
                                       __fsub_rn(bf16_hi(xa[k]), bf16_hi(ma[k])));
                w = make_uint4(o[0], o[1], o[2], o[3]);
            }
            *p = w;
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
            const uint32_t aA = smem_u32(sA), aB = smem_u32(sA + 16384u);
#pragma unroll
            for (int ks = 0; ks < kJKBlock / 16; ++ks)
                umma_ss(tmem, sdesc_sw128(aA + (uint32_t)ks * 32u, 16, 1024),
                        sdesc_sw128(aB + (uint32_t)ks * 2048u, kJKBlock * 128u, 1024), idesc,
                        (kb > 0 || ks > 0) ? 1u : 0u);
            umma_commit(done(s));
            // block kb + 3 goes into the stage of block kb - 1 once its MMAs are done
            const int kn = kb + kJEStages - 1;
            if (kn < nk) {
                if (kb >= 1)
                    ok = mbar_wait(done((kb - 1) % kJEStages), (uint32_t)(((kb - 1) / kJEStages) & 1)) && ok;
                issue_loads(kn);
            }
        }
    }
    // the last block's MMAs complete after all earlier ones: wait for them
    ok = mbar_wait(done((nk - 1) % kJEStages), (uint32_t)(((nk - 1) / kJEStages) & 1)) && ok;
    tc_fence_after();
    const uint32_t trow = tmem + (((uint32_t)(warp & 3) * 32u) << 16);
    ok = __all_sync(0xffffffffu, ok);  // tcgen05.ld below is warp-collective
    if (ok) {
        uint8_t *codes_row = (valid && a.codes) ? a.codes + t * (a.r * a.bits / 8) : nullptr;
        float2 *meta_row = (valid && a.meta) ? reinterpret_cast<float2 *>(a.meta) + t * (a.r / G) : nullptr;
        float *coef_row = (valid && a.coef_out) ? a.coef_out + t * a.r : nullptr;
        joint_quant_row<G, BITS>(trow, a.r, codes_row, meta_row, coef_row, half, 2);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0)
        tmem_dealloc(tmem, ncols);
}

struct JointDecArgs {
    const uint16_t *cent;  // [H][C][D]
    const uint16_t *idx;   // [H][T]
    const uint8_t *codes;  // [T][r*bits/8]
    const float *meta;     // [T][r/G][2]
    int64_t T;
    int H, D, C, r, bits, G;
    void *out;             // [T][H][D]
    int out_bf16;
};

// Decoder roles (288 threads): warps 0-3 and 4-7 are two epilogue groups
// (even and odd heads; each thread one token row = TMEM lane), warp 8 lane 0
// loads W_dec slices with TMA and issues the MMAs.  All 256 epilogue threads
// first build c^ (two threads per token, half the coefficients each).
constexpr int kJDThreads = 288;

constexpr uint32_t kJDSmemLimit = 227u * 1024u - 1024u;  // less the alignment slack

constexpr uint32_t kJDStageRow = 80;                 // staged output row: 32 bf16 + 16 B pad
constexpr uint32_t kJDStageWarp = 32u * kJDStageRow;  // per epilogue warp

struct JDLayout {
    uint32_t a_bytes;  // one of A hi / A lo: [r/64][128][128 B]
    uint32_t w_bytes;  // one W stage: [D/64][r][128 B]
    int nst;           // W stages: 2 where they fit, else 1
    uint32_t off_lo, off_w, off_bar, off_stg, total;
    __host__ __device__ JDLayout(int r, int D)
    {
        a_bytes = 128u * (uint32_t)r * 2u;
        w_bytes = (uint32_t)(D / 64) * (uint32_t)r * 128u;
        const uint32_t fixed = 2u * a_bytes + 128u + 8u * kJDStageWarp;
        nst = (fixed + 2u * w_bytes <= kJDSmemLimit) ? 2 : 1;
        off_lo = a_bytes;
        off_w = 2u * a_bytes;
        off_bar = off_w + (uint32_t)nst * w_bytes;
        off_stg = off_bar + 128u;
        total = off_stg + 8u * kJDStageWarp;
    }
};

enum { JD_WFULL0 = 0, JD_WFULL1, JD_DONE0, JD_FREE0 = JD_DONE0 + 4, JD_DRAIN = JD_FREE0 + 4, JD_COUNT };

// One CTA per 128-token tile; head h: TMEM buffer h & 3 (D columns) and
// W stage h & 1.  The MMA of head h overlaps the epilogue of head h - 1.
__global__ void __launch_bounds__(kJDThreads, 1)
    joint_decode_kernel(const __grid_constant__ CUtensorMap tmap_w, JointDecArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const JDLayout L(a.r, a.D);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L.off_bar);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + JD_COUNT);
    auto bar = [&](int i) { return smem_u32(bars + i); };
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t t0 = (int64_t)blockIdx.x * kJRows;
    const uint32_t tcols = (uint32_t)(a.D == 128 ? 512 : 256);

    if (warp == 0)
        tmem_alloc(smem_u32(tmem_slot), tcols);
    if (tid == 0) {
        mbar_init(bar(JD_WFULL0), 1);
        mbar_init(bar(JD_WFULL1), 1);
        for (int b = 0; b < 4; ++b) {
            mbar_init(bar(JD_DONE0 + b), 1);
            mbar_init(bar(JD_FREE0 + b), 4);  // the 4 warps of one epilogue group
        }
        mbar_init(bar(JD_DRAIN), 1);
        fence_mbar_init();
    }
    __syncthreads();  // barriers initialised before any TMA names them
    if (warp == 8 && lane == 0) {
        // W slices of the first heads while c^ is being built
        for (int h = 0; h < L.nst && h < a.H; ++h) {
            mbar_arrive_expect_tx(bar(JD_WFULL0 + h), L.w_bytes);
            for (int c = 0; c < a.D / 64; ++c)
                tma_load_2d(smem_u32(smem + L.off_w + (uint32_t)h * L.w_bytes + (uint32_t)c * (uint32_t)a.r * 128u),
                            &tmap_w, bar(JD_WFULL0 + h), h * a.D + c * 64, 0);
        }
    }
    if (warp < 8) {
        // A: c^ = (q - z) s, split into bf16 hi (truncated) + lo (rounded
        // remainder), K-major [r/64][128][128 B]
        const int row = tid & 127, half = tid >> 7;
        const int64_t t = t0 + row;
        const bool valid = t < a.T;
        const int ng = a.r / a.G;
        const uint32_t mask = (1u << a.bits) - 1u;
        for (int u = half * (a.r / 16); u < (half + 1) * (a.r / 16); ++u) {
            uint4 wh = make_uint4(0, 0, 0, 0), wl = make_uint4(0, 0, 0, 0);
            if (valid) {
                const int c0 = u * 8;
                const float2 sz = __ldg(reinterpret_cast<const float2 *>(a.meta) + t * ng + c0 / a.G);
                uint32_t cw;
                if (a.bits == 4)
                    cw = __ldg(reinterpret_cast<const uint32_t *>(a.codes + t * (a.r / 2) + c0 / 2));
                else
                    cw = __ldg(reinterpret_cast<const uint16_t *>(a.codes + t * (a.r / 4) + c0 / 4));
                uint32_t hi[4], lo[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const float v0 = __fmul_rn(__fsub_rn((float)((cw >> (2 * k * a.bits)) & mask), sz.y), sz.x);
                    const float v1 = __fmul_rn(__fsub_rn((float)((cw >> ((2 * k + 1) * a.bits)) & mask), sz.y), sz.x);
                    const uint32_t a0 = __float_as_uint(v0) & 0xffff0000u, a1 = __float_as_uint(v1) & 0xffff0000u;
                    hi[k] = __byte_perm(a0, a1, 0x7632);
                    lo[k] = pack_bf16x2(v0 - __uint_as_float(a0), v1 - __uint_as_float(a1));
                }
                wh = make_uint4(hi[0], hi[1], hi[2], hi[3]);
                wl = make_uint4(lo[0], lo[1], lo[2], lo[3]);
            }
            const uint32_t off = sw128_unit_offset(row, u, kJRows);
            *reinterpret_cast<uint4 *>(smem + off) = wh;
            *reinterpret_cast<uint4 *>(smem + L.off_lo + off) = wl;
        }
        fence_proxy_async_smem();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    bool ok = true;

    if (warp == 8) {
        // ------------------------------------------------ W loads + MMAs
        if (lane == 0) {
            const uint32_t idesc = idesc_f32acc(128, a.D, true, false, true);
            const uint32_t aAh = smem_u32(smem), aAl = smem_u32(smem + L.off_lo);
            const int nks = a.r / 16;
            const int nst = L.nst;
            int h = 0;
            for (; ok && h < a.H; ++h) {
                const int s = h % nst, b = h & 3;
                ok = mbar_wait(bar(JD_WFULL0 + s), (uint32_t)((h / nst) & 1));
                if (ok && h >= 4)
                    ok = mbar_wait(bar(JD_FREE0 + b), (uint32_t)(((h - 4) >> 2) & 1));
                if (!ok)
                    break;
                tc_fence_after();
                const uint32_t aB = smem_u32(smem + L.off_w + (uint32_t)s * L.w_bytes);
                for (int part = 0; part < 2; ++part)
                    for (int ks = 0; ks < nks; ++ks) {
                        const uint32_t aoff = (uint32_t)(ks >> 2) * (128u * 128u) + (uint32_t)(ks & 3) * 32u;
                        umma_ss(tmem + (uint32_t)(b * a.D), sdesc_sw128((part ? aAl : aAh) + aoff, 16, 1024),
                                sdesc_sw128(aB + (uint32_t)ks * 2048u, (uint32_t)a.r * 128u, 1024), idesc,
                                (part || ks) ? 1u : 0u);
                    }
                umma_commit(bar(JD_DONE0 + b));
                if (h + nst < a.H) {
                    // stage s is free once this head's MMAs are done
                    ok = mbar_wait(bar(JD_DONE0 + b), (uint32_t)((h >> 2) & 1));
                    if (!ok)
                        break;
                    mbar_arrive_expect_tx(bar(JD_WFULL0 + s), L.w_bytes);
                    for (int c = 0; c < a.D / 64; ++c)
                        tma_load_2d(smem_u32(smem + L.off_w + (uint32_t)s * L.w_bytes +
                                             (uint32_t)c * (uint32_t)a.r * 128u),
                                    &tmap_w, bar(JD_WFULL0 + s), (h + nst) * a.D + c * 64, 0);
                }
            }
            // wait for every MMA issued before teardown; after a give-up also
            // for the W loads already issued (heads h .. h + nst - 1)
            umma_commit(bar(JD_DRAIN));
            mbar_wait(bar(JD_DRAIN), 0);
            if (!ok)
                for (int hh = h; hh < a.H && hh < h + nst; ++hh)
                    mbar_wait(bar(JD_WFULL0 + hh % nst), (uint32_t)((hh / nst) & 1));
        }
        __syncwarp();
    } else {
        // ------------------------------------------------ epilogue
        const int g = warp >> 2;
        const int row = (warp & 3) * 32 + lane;
        const int64_t t = t0 + row;
        const bool valid = t < a.T;
        const uint32_t lane_off = ((uint32_t)(warp & 3) * 32u) << 16;
        // the centre row of the next head is fetched before its MMAs are awaited
        auto centre_row = [&](int h, uint4 *mw) {
            if (!valid || h >= a.H)
                return;
            int j = __ldg(a.idx + (int64_t)h * a.T + t);
            if (j >= a.C) {
                raise_status(DEVSTAT_BAD_INDEX);
                j = 0;
            }
            const uint4 *mu = reinterpret_cast<const uint4 *>(a.cent + ((int64_t)h * a.C + j) * a.D);
#pragma unroll
            for (int u = 0; u < 16; ++u)
                if (u < a.D / 8)
                    mw[u] = __ldg(mu + u);
        };
        uint4 mw[16];
        centre_row(g, mw);
        for (int h = g; h < a.H; h += 2) {
            const int b = h & 3;
            ok = __all_sync(0xffffffffu, ok && mbar_wait(bar(JD_DONE0 + b), (uint32_t)((h >> 2) & 1)));
            if (!ok)
                break;
            tc_fence_after();
#pragma unroll
            for (int cb = 0; cb < 4; ++cb) {
                if (cb >= a.D / 32)
                    break;
                float v[32];
                tmem_ld32(tmem + lane_off + (uint32_t)(b * a.D + cb * 32), v);
                if (valid) {
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const uint4 m4 = mw[cb * 4 + u];
                        const uint32_t m[4] = {m4.x, m4.y, m4.z, m4.w};
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            v[u * 8 + 2 * k] = __fadd_rn(bf16_lo(m[k]), v[u * 8 + 2 * k]);
                            v[u * 8 + 2 * k + 1] = __fadd_rn(bf16_hi(m[k]), v[u * 8 + 2 * k + 1]);
                        }
                    }
                }
                if (a.out_bf16) {
                    // through the warp's staging rows, so the stores of a warp
                    // cover whole 64-byte row pieces of 8 rows at a time
                    uint8_t *stg = smem + L.off_stg + (uint32_t)warp * kJDStageWarp;
                    if (valid) {
#pragma unroll
                        for (int u = 0; u < 4; ++u)
                            *reinterpret_cast<uint4 *>(stg + (uint32_t)lane * kJDStageRow + 16u * (uint32_t)u) =
                                make_uint4(pack_bf16x2(v[8 * u], v[8 * u + 1]),
                                           pack_bf16x2(v[8 * u + 2], v[8 * u + 3]),
                                           pack_bf16x2(v[8 * u + 4], v[8 * u + 5]),
                                           pack_bf16x2(v[8 * u + 6], v[8 * u + 7]));
                    }
                    __syncwarp();
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int rr = 8 * i + (lane >> 2), uu = lane & 3;
                        const int64_t tr = t0 + 32 * (warp & 3) + rr;
                        if (tr < a.T)
                            *reinterpret_cast<uint4 *>(static_cast<uint16_t *>(a.out) + (tr * a.H + h) * a.D +
                                                       cb * 32 + 8 * uu) =
                                *reinterpret_cast<const uint4 *>(stg + (uint32_t)rr * kJDStageRow + 16u * (uint32_t)uu);
                    }
                    __syncwarp();
                } else if (valid) {
                    const int64_t o = (t * a.H + h) * a.D + cb * 32;
                    float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(a.out) + o);
#pragma unroll
                    for (int u = 0; u < 8; ++u)
                        dst[u] = make_float4(v[4 * u], v[4 * u + 1], v[4 * u + 2], v[4 * u + 3]);
                }
            }
            centre_row(h + 2, mw);
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(bar(JD_FREE0 + b));
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0)
        tmem_dealloc(tmem, tcols);
}

}  // namespace kvq

// attention.cuh -- attention of the current chunk's queries over a compressed
// K/V history, reconstruction fused into the kernel, tcgen05 tensor cores.
//
// Method: NanoKV page, Fig. 4(a) (history read through the decoder:
// centres added back to the dequantised residual) and Fig. 4(d) (partial
// results carry their log-sum-exp for merging); QuantWM, Fig. 9 (packed
// storage with on-demand reconstruction during attention).
//
// One CTA owns 128 query rows of one head (one TMEM lane per row, one thread
// per row).  For every 128-token history tile it
//   1. rebuilds k^ = mu[idx] + (q - z) s and v^ likewise from codes, {s, z},
//      idx and the bf16 centres (binary32, the decoder's arithmetic) and
//      writes them into shared memory in the 128-byte-swizzled operand layout:
//      k^ as two bf16 tiles, hi = bf16(k^) and lo = bf16(k^ - hi), so that the
//      logits keep ~16 mantissa bits; v^ as one fp16 tile;
//   2. issues S = Q K_hi^T + Q K_lo^T (M=128, N=128, K=d each, bf16) on the
//      tensor cores into TMEM;
//   3. runs the online softmax on its TMEM row (exp2 domain), writes P (fp16)
//      into the freed K_hi buffer;
//   4. issues O_tile = P V^ (M=128, N=d, K=128, fp16, V^ as an MN-major
//      operand) into TMEM and folds it into the register accumulator with
//      the running-max correction.
// The split logits and fp16 P/V^ keep the result within the accuracy the
// tests demand on heavy-tailed outlier channels (|k|, |v| ~ 100), where bf16
// operands alone lose up to ~4e-2 in the log-sum-exp.
// Every mbarrier wait is bounded; on expiry the CTA records a timeout in the
// device status word, drains its MMAs with a second bounded wait, frees its
// TMEM and returns.
#pragma once

#include "codec.cuh"
#include "common.cuh"

namespace kvq {

struct CodecView {
    const uint16_t *cent;  // [H][C][D] bf16
    const uint16_t *idx;   // [H][T]
    const uint8_t *codes;  // [H][T][D*bits/8]
    const float *meta;     // [H][T][D/G][2]
    int64_t T;
    int C;
    int bits;
    int G;
};

struct AttnArgs {
    const uint16_t *q;  // [Tq][H][D] bf16
    int64_t Tq;
    int H;
    CodecView k, v;
    int64_t t_begin, t_end;
    float scale_log2;  // softmax scale * log2(e)
    void *o_out;
    int o_bf16;
    float *lse_out;  // [H][Tq]
    int nsplit;      // > 1: blockIdx.z selects a sub-range; o_out / lse_out
                     // then hold nsplit float partials [z][Tq][H][D], [z][H][Tq]
};

constexpr int kAttnRows = 128;     // query rows per CTA
constexpr int kAttnTile = 128;     // history tokens per tile
constexpr int kAttnThreads = 128;
constexpr uint32_t kAttnTmemCols = 256;

template <int D>
struct AttnSmem {
    static constexpr uint32_t kQ = D * 2 * kAttnRows;                     // Q tile bytes
    static constexpr uint32_t kK = D * 2 * kAttnTile;                     // one k^ / v^ tile
    static constexpr uint32_t kP = 2 * kAttnTile * kAttnRows;             // P tile
    static constexpr uint32_t kKP = kK > kP ? kK : kP;                    // K_hi, later P
    static constexpr uint32_t offQ = 0, offKP = kQ, offKL = kQ + kKP, offV = offKL + kK, offBar = offV + kK;
    static constexpr uint32_t kBytes = offBar + 64;
    static constexpr uint32_t kLaunchBytes = kBytes + 1024;  // slack for 1024-byte alignment
};

// Rebuild one history row (D channels) of a compressed K or V into swizzled
// operand tiles, 16 bytes (8 channels) at a time.  SPLIT: two bf16 tiles
// (hi, lo); otherwise one fp16 tile (tile_lo unused).
template <int D, bool SPLIT>
__device__ __forceinline__ void dequant_row_to_smem(const CodecView &cv, int h, int64_t tok, bool valid,
                                                    uint8_t *tile, uint8_t *tile_lo, uint32_t row)
{
    if (!valid) {
#pragma unroll
        for (int u = 0; u < D / 8; ++u) {
            *reinterpret_cast<uint4 *>(tile + sw128_unit_offset(row, u, kAttnTile)) = make_uint4(0, 0, 0, 0);
            if (SPLIT)
                *reinterpret_cast<uint4 *>(tile_lo + sw128_unit_offset(row, u, kAttnTile)) = make_uint4(0, 0, 0, 0);
        }
        return;
    }
    const int64_t th = (int64_t)h * cv.T + tok;
    int j = cv.idx[th];
    if (j >= cv.C) {
        raise_status(DEVSTAT_BAD_INDEX);
        j = 0;
    }
    const uint16_t *mu_row = cv.cent + ((int64_t)h * cv.C + j) * D;
    const float2 *meta_row = reinterpret_cast<const float2 *>(cv.meta) + th * (D / cv.G);
    const uint32_t mask = (1u << cv.bits) - 1u;
    const uint8_t *code_row = cv.codes + th * (D * cv.bits / 8);
#pragma unroll 4
    for (int u = 0; u < D / 8; ++u) {
        const int c0 = u * 8;
        const float2 sz = __ldg(meta_row + c0 / cv.G);
        uint32_t cw;
        if (cv.bits == 2)
            cw = __ldg(reinterpret_cast<const uint16_t *>(code_row) + u);
        else
            cw = __ldg(reinterpret_cast<const uint32_t *>(code_row) + u);
        float mu[8];
        load_bf16x8(mu_row + c0, mu);
        float val[8];
#pragma unroll
        for (int k = 0; k < 8; ++k)
            val[k] = dequant_spec((cw >> (k * cv.bits)) & mask, sz.x, sz.y, mu[k]);
        const uint32_t off = sw128_unit_offset(row, u, kAttnTile);
        if (SPLIT) {
            uint32_t hi[4], lo[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                hi[k] = pack_bf16x2(val[2 * k], val[2 * k + 1]);
                lo[k] = pack_bf16x2(val[2 * k] - bf16_lo(hi[k]), val[2 * k + 1] - bf16_hi(hi[k]));
            }
            *reinterpret_cast<uint4 *>(tile + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
            *reinterpret_cast<uint4 *>(tile_lo + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
        } else {
            *reinterpret_cast<uint4 *>(tile + off) =
                make_uint4(pack_f16x2_sat(val[0], val[1]), pack_f16x2_sat(val[2], val[3]),
                           pack_f16x2_sat(val[4], val[5]), pack_f16x2_sat(val[6], val[7]));
        }
    }
}

template <int D>
__global__ void __launch_bounds__(kAttnThreads, 1) attention_lse_kernel(AttnArgs a)
{
    using L = AttnSmem<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sQ = smem + L::offQ;
    uint8_t *sKP = smem + L::offKP;
    uint8_t *sKL = smem + L::offKL;
    uint8_t *sV = smem + L::offV;
    uint64_t *bar = reinterpret_cast<uint64_t *>(smem + L::offBar);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::offBar + 16);

    const uint32_t tid = threadIdx.x, warp = tid >> 5;
    const int h = blockIdx.y;
    const int64_t q0 = (int64_t)blockIdx.x * kAttnRows;
    const uint32_t bar_a = smem_u32(bar);

    if (warp == 0)
        tmem_alloc(smem_u32(tmem_slot), kAttnTmemCols);
    if (tid == 0) {
        mbar_init(bar_a, 1);
        fence_mbar_init();
    }

    // Q rows -> swizzled K-major tile (zero rows past the end)
    {
        const int64_t qr = q0 + tid;
        const bool valid = qr < a.Tq;
        const uint16_t *src = a.q + (qr * a.H + h) * D;
#pragma unroll
        for (int u = 0; u < D / 8; ++u) {
            uint4 w = valid ? __ldg(reinterpret_cast<const uint4 *>(src) + u) : make_uint4(0, 0, 0, 0);
            *reinterpret_cast<uint4 *>(sQ + sw128_unit_offset(tid, u, kAttnRows)) = w;
        }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tS = tmem, tO = tmem + 128;
    const uint32_t lane_off = (warp * 32u) << 16;

    constexpr uint32_t idescS = idesc_f32acc(128, 128, true, false, false);   // bf16
    constexpr uint32_t idescO = idesc_f32acc(128, D, false, false, true);     // fp16, V MN-major
    const uint32_t aQ = smem_u32(sQ), aKP = smem_u32(sKP), aKL = smem_u32(sKL), aV = smem_u32(sV);

    float o[D];
#pragma unroll
    for (int c = 0; c < D; ++c)
        o[c] = 0.0f;
    float m_run = -INFINITY, l_run = 0.0f;
    uint32_t phase = 0;
    bool ok = true;

    for (int64_t t0 = a.t_begin; t0 < a.t_end; t0 += kAttnTile) {
        const int64_t tok = t0 + tid;
        const bool tv = tok < a.t_end;
        dequant_row_to_smem<D, true>(a.k, h, tok, tv, sKP, sKL, tid);
        dequant_row_to_smem<D, false>(a.v, h, tok, tv, sV, nullptr, tid);
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();

        // S = Q K_hi^T + Q K_lo^T : K-major A (queries) and B (history rows)
        if (tid == 0) {
#pragma unroll
            for (int part = 0; part < 2; ++part) {
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks) {
                    const uint32_t koff = (uint32_t)(ks >> 2) * (kAttnRows * 128u) + (uint32_t)(ks & 3) * 32u;
                    const uint32_t kkoff = (uint32_t)(ks >> 2) * (kAttnTile * 128u) + (uint32_t)(ks & 3) * 32u;
                    umma_ss(tS, sdesc_sw128(aQ + koff, 16, 1024),
                            sdesc_sw128((part ? aKL : aKP) + kkoff, 16, 1024), idescS, (part | ks) ? 1u : 0u);
                }
            }
            umma_commit(bar_a);
        }
        ok = mbar_wait(bar_a, phase) && ok;
        phase ^= 1u;
        tc_fence_after();

        // online softmax on this thread's row of S
        float tile_max = -INFINITY;
#pragma unroll 1
        for (int cb = 0; cb < kAttnTile / 32; ++cb) {
            float sv[32];
            tmem_ld32(tS + lane_off + cb * 32, sv);
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const bool valid = t0 + cb * 32 + i < a.t_end;
                tile_max = fmaxf(tile_max, valid ? sv[i] * a.scale_log2 : -INFINITY);
            }
        }
        const float m_new = fmaxf(m_run, tile_max);
        const float alpha = (m_run == -INFINITY) ? 0.0f : ex2_approx(m_run - m_new);
        float l_tile = 0.0f;
#pragma unroll 1
        for (int cb = 0; cb < kAttnTile / 32; ++cb) {
            float sv[32];
            tmem_ld32(tS + lane_off + cb * 32, sv);
            float p[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const bool valid = t0 + cb * 32 + i < a.t_end;
                p[i] = valid ? ex2_approx(sv[i] * a.scale_log2 - m_new) : 0.0f;
                l_tile += p[i];
            }
            // P row (query row tid, tokens cb*32 .. +31) -> K-major fp16 A tile
#pragma unroll
            for (int uu = 0; uu < 4; ++uu) {
                const int u = cb * 4 + uu;
                *reinterpret_cast<uint4 *>(sKP + sw128_unit_offset(tid, u, kAttnRows)) = make_uint4(
                    pack_f16x2_sat(p[8 * uu + 0], p[8 * uu + 1]), pack_f16x2_sat(p[8 * uu + 2], p[8 * uu + 3]),
                    pack_f16x2_sat(p[8 * uu + 4], p[8 * uu + 5]), pack_f16x2_sat(p[8 * uu + 6], p[8 * uu + 7]));
            }
        }
        l_run = l_run * alpha + l_tile;
        m_run = m_new;
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();

        // O_tile = P V (fp16): K-major A (P), MN-major B (V rows are K, channels N)
        if (tid == 0) {
#pragma unroll
            for (int ks = 0; ks < kAttnTile / 16; ++ks) {
                const uint32_t poff = (uint32_t)(ks >> 2) * (kAttnRows * 128u) + (uint32_t)(ks & 3) * 32u;
                const uint32_t voff = (uint32_t)ks * (16u * 128u);
                umma_ss(tO, sdesc_sw128(aKP + poff, 16, 1024), sdesc_sw128(aV + voff, kAttnTile * 128u, 1024),
                        idescO, ks > 0 ? 1u : 0u);
            }
            umma_commit(bar_a);
        }
        ok = mbar_wait(bar_a, phase) && ok;
        phase ^= 1u;
        tc_fence_after();
#pragma unroll
        for (int cb = 0; cb < D / 32; ++cb) {
            float ov[32];
            tmem_ld32(tO + lane_off + cb * 32, ov);
#pragma unroll
            for (int i = 0; i < 32; ++i)
                o[cb * 32 + i] = fmaf(o[cb * 32 + i], alpha, ov[i]);
        }
        tc_fence_before();
        ok = __syncthreads_and(ok) != 0;
        if (!ok)
            break;
    }

    // epilogue: normalise and store this row
    const int64_t qr = q0 + tid;
    if (qr < a.Tq) {
        const bool empty = !(l_run > 0.0f);
        const float inv_l = empty ? 0.0f : 1.0f / l_run;
        if (a.o_bf16) {
            uint4 *dst = reinterpret_cast<uint4 *>(static_cast<uint16_t *>(a.o_out) + (qr * a.H + h) * D);
#pragma unroll
            for (int u = 0; u < D / 8; ++u)
                dst[u] = make_uint4(pack_bf16x2(o[8 * u] * inv_l, o[8 * u + 1] * inv_l),
                                    pack_bf16x2(o[8 * u + 2] * inv_l, o[8 * u + 3] * inv_l),
                                    pack_bf16x2(o[8 * u + 4] * inv_l, o[8 * u + 5] * inv_l),
                                    pack_bf16x2(o[8 * u + 6] * inv_l, o[8 * u + 7] * inv_l));
        } else {
            float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(a.o_out) + (qr * a.H + h) * D);
#pragma unroll
            for (int u = 0; u < D / 4; ++u)
                dst[u] = make_float4(o[4 * u] * inv_l, o[4 * u + 1] * inv_l, o[4 * u + 2] * inv_l,
                                     o[4 * u + 3] * inv_l);
        }
        a.lse_out[(int64_t)h * a.Tq + qr] = empty ? -INFINITY : (m_run + log2f(l_run)) * 0.69314718055994531f;
    }

    if (!ok && tid == 0) {
        // drain: wait (bounded) for any MMA still in flight before TMEM is freed
        umma_commit(bar_a);
        mbar_wait(bar_a, phase);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0)
        tmem_dealloc(tmem, kAttnTmemCols);
}

}  // namespace kvq

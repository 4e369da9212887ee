// attention_tma.cuh -- attention over a compressed K/V history on CTA pairs
// (thread-block clusters of 2 on two SMs, tcgen05 cta_group::2), d = 128,
// with every byte of the compressed history staged by TMA.
//
// Method: NanoKV page, Fig. 4(a,d) (history read through the decoder: centres
// added back to the dequantised residual; partial results carry their
// log-sum-exp); QuantWM, Fig. 9 (on-demand reconstruction during attention).
//
// Work split, MMAs and softmax are those of attention_pair.cuh: a pair owns
// 512 query rows of one head (CTA v: rows [256 v, 256 v + 256) as two 128-row
// tiles); per 128-token history tile CTA v rebuilds history rows
// [64 v, 64 v + 64) of K^ (all 128 channels, bf16 hi + lo) and channels
// [64 v, 64 v + 64) of V^ (all 128 rows, fp16); the leader issues M = 256
// MMAs (S = Q K_hi^T + Q K_lo^T, O += P V) in ping-pong order across the two
// query tiles; two softmax warpgroups per CTA keep the online softmax.
//
// Staging.  One loader warp per CTA fills a stage of the three-stage ring for
// each tile, as soon as the MMAs of the tile three back have released it:
//  - tiled TMA loads of the tile's packed codes and {s, z} pairs into the
//    stage's K lo slot (the CTA's 64 K rows whole; the CTA's channel half of
//    all 128 V rows), from 2-D views [H T][row bytes] of the codec arrays;
//    compact binary16 {s, z} rows (8 to 32 bytes, too narrow for a tiled
//    copy at G = 64) are read by the loader lanes instead and stored before
//    the fill barrier's arrival, which releases them to the producers;
//  - TMA gathers (tile::gather4) of the centre rows mu_h[idx] straight into
//    their 128-byte-swizzled operand rows: both 64-channel halves of the 64 K
//    rows into K hi, this CTA's channel half of the 128 V rows into V, four
//    rows per gather, the row numbers h C + idx read by the loader lanes;
// all completing on the stage's fill barrier.  The producers (8 warps) wait
// on that barrier, copy their code words and {s, z} to registers, meet at a
// named barrier (the K lo writes overwrite the staged words), rebuild their
// units of K and V in place and publish both behind one proxy fence.  They have no copies of
// their own in flight, so the fence does not wait on memory.
//
// PSAC (QuantWM, Sec. 4.2; rank 8, Table 9): with a basis U_h [d][8] and
// per-key coefficients C [H][T][8], the logits are those of the corrected
// keys k^ + U_h C; the loader stages each tile's coefficient rows with a
// tiled load beside the codes, and the producers add U_h C (binary32, U_h
// resident in shared memory) to every rebuilt K value before the hi/lo split.
//
// Barriers (parity = use count & 1): those of attention_pair.cuh plus
// fill[s] (1 arrival with the stage's byte count, completed by the TMA
// traffic; local to each CTA).  The loader waits kfree[s] and vfree[s] (the
// leader's multicast commits) before reusing a stage.  Waits are bounded and
// poll a per-CTA abort flag; before TMEM is freed the leader drains its MMAs,
// the loaders wait for their last copies, and both CTAs meet at a cluster
// barrier.
#pragma once

#include <cuda.h>

#include "attention.cuh"
#include "attention2.cuh"
#include "attention_pair.cuh"
#include "codec.cuh"
#include "common.cuh"

namespace kvq {

constexpr int kATThreads = 576;  // 8 producer, 1 MMA, 8 softmax, 1 loader warps
constexpr int kATLoaderWarp = 17;

// Tensor maps of one compressed K/V history (host-encoded per call).
struct AttnMaps {
    CUtensorMap kc;     // K codes   [H T][128 bK/8] u8,     box {row, 64}
    CUtensorMap km;     // K {s, z}  [H T][2 128/G_K] f32,   box {row, 64}
    CUtensorMap vc;     // V codes   [H T][128 bV/8] u8,     box {half row, 128}
    CUtensorMap vm;     // V {s, z}  [H T][2 128/G_V] f32,   box {half row (>= 16 B), 128}
    CUtensorMap kcent;  // K centres [H C_K][128] bf16,      box {64, 1}, 128-byte swizzle
    CUtensorMap vcent;  // V centres [H C_V][128] bf16,      box {64, 1}, 128-byte swizzle
    CUtensorMap kpc;    // PSAC coefficients [H T][8] f32,   box {8, 64} (when used)
};

// Offsets of the staged words inside a stage's K lo slot (16 KB).
constexpr uint32_t kATStKc = 0, kATStKm = 4096, kATStVc = 8192, kATStVm = 12288;

// Shared memory beyond the pair kernel's layout: the PSAC basis of the head
// [128][8] binary32 and one coefficient tile [64][8] per stage.
struct ATSmem {
    static constexpr uint32_t offU = APSmem::kBytes;
    static constexpr uint32_t offC = offU + 128 * 8 * 4;
    static constexpr uint32_t kBytes = offC + kAPStages * 64 * 8 * 4;
    static constexpr uint32_t kLaunchBytes = kBytes + 1024;
};

enum { AT_FILL0 = P_COUNT, AT_COUNT = AT_FILL0 + kAPStages };

// Bytes of V {s, z} staged per row: the CTA's half of the groups, or the
// whole row when that half is under 16 bytes (G = 64).
__host__ __device__ constexpr int at_vm_row_bytes(int G) { return G == 64 ? 16 : (64 / G) * 8; }

// Loader (one warp): stage every tile of [t_begin, t_end).
template <int BK, int BV>
__device__ __forceinline__ void at_load(const AttnArgs &a, const AttnMaps &m, int h, uint32_t rank, int lane,
                                        int ntiles, uint8_t *smem, uint64_t *bars, volatile int *abort_flag)
{
    using L = APSmem;
    auto bar = [&](int i) { return smem_u32(bars + i); };
    auto khi = [&](int s) { return smem_u32(smem + L::offK + (uint32_t)(2 * s) * L::kKh); };
    auto klo = [&](int s) { return smem_u32(smem + L::offK + (uint32_t)(2 * s + 1) * L::kKh); };
    auto vst = [&](int s) { return smem_u32(smem + L::offV + (uint32_t)s * L::kV); };
    const int Gk = a.k.G, Gv = a.v.G;
    const bool k16 = a.k.meta16 != 0, v16 = a.v.meta16 != 0;
    const bool psac = a.psac_coef != nullptr;
    const uint32_t bytes = 16384u + 16384u + 64u * 16u * BK + (k16 ? 0u : 64u * (uint32_t)(128 / Gk) * 8u) +
                           128u * 8u * BV + (v16 ? 0u : 128u * (uint32_t)at_vm_row_bytes(Gv)) + (psac ? 2048u : 0u);
    // compact {s, z}: whole rows of 4 (128/G) bytes, in 8-byte words
    const int kw_row = (128 / Gk) / 2, vw_row = (128 / Gv) / 2;  // words per row
    const int kw_lane = 64 * kw_row / 32, vw_lane = 128 * vw_row / 32;
    const int vc_x = (int)rank * 8 * BV;
    const int vm_x = Gv == 64 ? 0 : (int)rank * (64 / Gv) * 2;
    const int64_t rowK = (int64_t)h * a.k.T, rowV = (int64_t)h * a.v.T;
    const int centK = h * a.k.C, centV = h * a.v.C;
    bool ok = true;
    int issued = 0;
    for (int i = 0; ok && i < ntiles; ++i) {
        const int s = i % kAPStages;
        const int64_t t0 = a.t_begin + (int64_t)i * 128;
        // centre rows of this lane's gathers: K rows 4 (lane & 15) .. + 3 of
        // this CTA's 64, V rows 4 lane .. + 3
        int kr[4], vr[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int64_t tk = t0 + 64 * rank + 4 * (lane & 15) + q;
            const int64_t tv = t0 + 4 * lane + q;
            int ik = tk < a.t_end ? (int)__ldg(a.k.idx + rowK + tk) : 0;
            int iv = tv < a.t_end ? (int)__ldg(a.v.idx + rowV + tv) : 0;
            if (ik >= a.k.C || iv >= a.v.C) {
                raise_status(DEVSTAT_BAD_INDEX);
                ik = ik >= a.k.C ? 0 : ik;
                iv = iv >= a.v.C ? 0 : iv;
            }
            kr[q] = centK + ik;
            vr[q] = centV + iv;
        }
        uint2 km16[8], vm16[16];
        if (k16) {
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const int w = lane + 32 * q;
                km16[q] = make_uint2(0u, 0u);
                if (q < kw_lane) {
                    const int64_t t = t0 + 64 * rank + w / kw_row;
                    if (t < a.k.T)
                        km16[q] = __ldg(static_cast<const uint2 *>(a.k.meta) + (rowK + t) * kw_row + w % kw_row);
                }
            }
        }
        if (v16) {
#pragma unroll
            for (int q = 0; q < 16; ++q) {
                const int w = lane + 32 * q;
                vm16[q] = make_uint2(0u, 0u);
                if (q < vw_lane) {
                    const int64_t t = t0 + w / vw_row;
                    if (t < a.v.T)
                        vm16[q] = __ldg(static_cast<const uint2 *>(a.v.meta) + (rowV + t) * vw_row + w % vw_row);
                }
            }
        }
        if (i >= kAPStages) {
            const uint32_t par = (uint32_t)(((i / kAPStages) - 1) & 1);
            ok = __all_sync(0xffffffffu, ap_wait(bar(P_KFREE0 + s), par, abort_flag) &&
                                             ap_wait(bar(P_VFREE0 + s), par, abort_flag));
            if (!ok)
                break;
        }
        {
            uint8_t *lo_p = smem + L::offK + (uint32_t)(2 * s + 1) * L::kKh;
            if (k16) {
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    if (q < kw_lane)
                        reinterpret_cast<uint2 *>(lo_p + kATStKm)[lane + 32 * q] = km16[q];
            }
            if (v16) {
#pragma unroll
                for (int q = 0; q < 16; ++q)
                    if (q < vw_lane)
                        reinterpret_cast<uint2 *>(lo_p + kATStVm)[lane + 32 * q] = vm16[q];
            }
            __syncwarp();  // the lanes' stores precede lane 0's arrival (release)
        }
        if (lane == 0)
            mbar_arrive_expect_tx(bar(AT_FILL0 + s), bytes);
        __syncwarp();
        const uint32_t fill = bar(AT_FILL0 + s);
        if (lane == 0) {
            const int rk = (int)(rowK + t0 + 64 * rank), rv = (int)(rowV + t0);
            tma_load_2d(klo(s) + kATStKc, &m.kc, fill, 0, rk);
            if (!k16)
                tma_load_2d(klo(s) + kATStKm, &m.km, fill, 0, rk);
            tma_load_2d(klo(s) + kATStVc, &m.vc, fill, vc_x, rv);
            if (!v16)
                tma_load_2d(klo(s) + kATStVm, &m.vm, fill, vm_x, rv);
            if (psac)
                tma_load_2d(smem_u32(smem + ATSmem::offC + (uint32_t)s * 2048u), &m.kpc, fill, 0, rk);
        }
        tma_gather4(khi(s) + (uint32_t)(lane >> 4) * 8192u + (uint32_t)(lane & 15) * 512u, &m.kcent, fill,
                    (lane >> 4) * 64, kr[0], kr[1], kr[2], kr[3]);
        tma_gather4(vst(s) + (uint32_t)lane * 512u, &m.vcent, fill, 64 * (int)rank, vr[0], vr[1], vr[2], vr[3]);
        issued = i + 1;
    }
    // the copies of the last tiles issued have landed before the CTA may exit
    for (int i = issued - kAPStages < 0 ? 0 : issued - kAPStages; i < issued; ++i) {
        uint32_t spins = 0;
        while (!mbar_try_wait(bar(AT_FILL0 + i % kAPStages), (uint32_t)((i / kAPStages) & 1)) && ++spins < kSpinLimit) {
        }
    }
}

// Code words and per-unit {s, z} of 4 units from the staging slots: binary32
// pairs (as ap_read_stage) or, with compact metadata, binary16 pairs widened.
template <int BITS>
__device__ __forceinline__ void at_read_stage(const uint8_t *stage_cw, const uint8_t *stage_sz, int G, bool meta16,
                                              uint32_t *cw, float2 *sz)
{
    if (!meta16) {
        ap_read_stage<BITS>(stage_cw, stage_sz, G, cw, sz);
        return;
    }
    if (BITS == 2) {
        const uint2 w = *reinterpret_cast<const uint2 *>(stage_cw);
        cw[0] = w.x & 0xffffu;
        cw[1] = w.x >> 16;
        cw[2] = w.y & 0xffffu;
        cw[3] = w.y >> 16;
    } else {
        const uint4 w = *reinterpret_cast<const uint4 *>(stage_cw);
        cw[0] = w.x;
        cw[1] = w.y;
        cw[2] = w.z;
        cw[3] = w.w;
    }
    if (G == 16) {
        const uint2 m = *reinterpret_cast<const uint2 *>(stage_sz);
        sz[0] = sz[1] = make_float2(f16_widen(m.x), f16_widen(m.x >> 16));
        sz[2] = sz[3] = make_float2(f16_widen(m.y), f16_widen(m.y >> 16));
    } else {
        const uint32_t m = *reinterpret_cast<const uint32_t *>(stage_sz);
        sz[0] = sz[1] = sz[2] = sz[3] = make_float2(f16_widen(m), f16_widen(m >> 16));
    }
}

// K rebuild with the PSAC correction: as ap_rebuild<BITS, true>, with
// sum_r U[c][r] C[r] added to each value (binary32) before the hi/lo split.
// Units uu cover channels ch0 + 8 uu .. + 7.
template <int BITS>
__device__ __forceinline__ void at_rebuild_k_psac(uint8_t *tile, uint8_t *lo, const uint32_t *off, const uint32_t *cw,
                                                  const float2 *sz, bool valid, const float *sU, const float *Crow,
                                                  int ch0)
{
    constexpr float kTwoB = (float)(1 << BITS);
    const float4 c0 = reinterpret_cast<const float4 *>(Crow)[0], c1 = reinterpret_cast<const float4 *>(Crow)[1];
#pragma unroll
    for (int uu = 0; uu < 4; ++uu) {
        uint4 *dst = reinterpret_cast<uint4 *>(tile + off[uu]);
        if (!valid) {
            *dst = make_uint4(0, 0, 0, 0);
            *reinterpret_cast<uint4 *>(lo + off[uu]) = make_uint4(0, 0, 0, 0);
            continue;
        }
        const uint4 mw = *dst;
        const float sc = kTwoB * sz[uu].x;
        const float nb = -__fmul_rn(kTwoB + sz[uu].y, sz[uu].x);
        const uint32_t ma[4] = {mw.x, mw.y, mw.z, mw.w};
        uint32_t hi[4], lw[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float2 f = make_float2(code_as_unit_float<BITS>(cw[uu], 2 * k),
                                         code_as_unit_float<BITS>(cw[uu], 2 * k + 1));
            const float2 b = add2(make_float2(bf16_lo(ma[k]), bf16_hi(ma[k])), make_float2(nb, nb));
            float2 val = fma2(f, make_float2(sc, sc), b);
            float corr[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const float *u = sU + (ch0 + 8 * uu + 2 * k + e) * 8;
                const float4 u0 = reinterpret_cast<const float4 *>(u)[0], u1 = reinterpret_cast<const float4 *>(u)[1];
                float acc = u0.x * c0.x;
                acc = fmaf(u0.y, c0.y, acc);
                acc = fmaf(u0.z, c0.z, acc);
                acc = fmaf(u0.w, c0.w, acc);
                acc = fmaf(u1.x, c1.x, acc);
                acc = fmaf(u1.y, c1.y, acc);
                acc = fmaf(u1.z, c1.z, acc);
                corr[e] = fmaf(u1.w, c1.w, acc);
            }
            val = add2(val, make_float2(corr[0], corr[1]));
            const uint32_t a0 = __float_as_uint(val.x) & 0xffff0000u;
            const uint32_t a1 = __float_as_uint(val.y) & 0xffff0000u;
            hi[k] = __byte_perm(a0, a1, 0x7632);
            const float2 d = sub2(val, make_float2(__uint_as_float(a0), __uint_as_float(a1)));
            lw[k] = pack_bf16x2(d.x, d.y);
        }
        *dst = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        *reinterpret_cast<uint4 *>(lo + off[uu]) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
    }
}

// Producers (8 warps): rebuild the staged tiles in place.
template <int BK, int BV>
__device__ __forceinline__ void at_produce(const AttnArgs &a, uint32_t rank, int tid, int ntiles, uint8_t *smem,
                                           uint64_t *bars, volatile int *abort_flag)
{
    using L = APSmem;
    auto bar = [&](int i) { return smem_u32(bars + i); };
    auto lead = [&](int i) { return mapa_shared(bar(i), 0); };
    auto khi = [&](int s) { return smem + L::offK + (uint32_t)(2 * s) * L::kKh; };
    auto klo = [&](int s) { return smem + L::offK + (uint32_t)(2 * s + 1) * L::kKh; };
    auto vst = [&](int s) { return smem + L::offV + (uint32_t)s * L::kV; };
    const int Gk = a.k.G, Gv = a.v.G;
    // K: history row krow of the CTA's 64, units 4 kq .. 4 kq + 3 (channels
    // 32 kq .. + 31); V: row vrow, units 4 vh .. + 3 of the CTA's channel half
    const uint32_t krow = (uint32_t)(tid & 63);
    const int kq = tid >> 6;
    const uint32_t vrow = (uint32_t)(tid & 127);
    const int vh = tid >> 7;
    uint32_t koff[4], voff[4];
#pragma unroll
    for (int uu = 0; uu < 4; ++uu) {
        koff[uu] = sw128_unit_offset(krow, 4 * kq + uu, 64);
        voff[uu] = sw128_unit_offset(vrow, 4 * vh + uu, 128);
    }
    const bool k16 = a.k.meta16 != 0, v16 = a.v.meta16 != 0;
    const uint32_t kcw_off = kATStKc + krow * 16u * BK + (uint32_t)kq * 4u * BK;
    const uint32_t vcw_off = kATStVc + vrow * 8u * BV + (uint32_t)vh * 4u * BV;
    uint32_t ksz_off, vsz_off;
    if (k16)  // whole binary16 rows of 4 (128/G) bytes; this thread's groups
        ksz_off = kATStKm + krow * (uint32_t)(4 * (128 / Gk)) + (uint32_t)(4 * ((32 * kq) / Gk));
    else
        ksz_off = kATStKm + krow * (uint32_t)(128 / Gk) * 8u +
                  (uint32_t)(Gk == 16 ? 16 * kq : Gk == 32 ? 8 * kq : 8 * (kq >> 1));
    if (v16)  // whole rows; the groups of channels 64 rank + 32 vh ..
        vsz_off = kATStVm + vrow * (uint32_t)(4 * (128 / Gv)) +
                  (uint32_t)(4 * ((64 * (int)rank + 32 * vh) / Gv));
    else
        vsz_off = kATStVm + vrow * (uint32_t)at_vm_row_bytes(Gv) +
                  (uint32_t)(Gv == 16 ? 16 * vh : Gv == 32 ? 8 * vh : 8 * (int)rank);
    for (int i = 0; i < ntiles; ++i) {
        const int s = i % kAPStages;
        const bool filled = ap_wait(bar(AT_FILL0 + s), (uint32_t)((i / kAPStages) & 1), abort_flag);
        const int64_t t0 = a.t_begin + (int64_t)i * 128;
        uint32_t kcw[4], vcw[4];
        float2 ksz[4], vsz[4];
        const uint8_t *lo = klo(s);
        if (filled) {
            at_read_stage<BK>(lo + kcw_off, lo + ksz_off, Gk, k16, kcw, ksz);
            at_read_stage<BV>(lo + vcw_off, lo + vsz_off, Gv, v16, vcw, vsz);
        }
        const float *crow = reinterpret_cast<const float *>(smem + ATSmem::offC + (uint32_t)s * 2048u) + krow * 8;
        // every staged word is in registers (the K lo writes below overwrite
        // them); all producers arrive, and all leave if any wait gave up
        if (!named_barrier_and<5>(kAPProducers, filled))
            return;
        if (a.psac_coef)
            at_rebuild_k_psac<BK>(khi(s), klo(s), koff, kcw, ksz, t0 + 64 * rank + krow < a.t_end,
                                  reinterpret_cast<const float *>(smem + ATSmem::offU), crow, 32 * kq);
        else
            ap_rebuild<BK, true>(khi(s), klo(s), koff, kcw, ksz, t0 + 64 * rank + krow < a.t_end);
        ap_rebuild<BV, false>(vst(s), nullptr, voff, vcw, vsz, t0 + vrow < a.t_end);
        // one proxy fence for both tiles (a fence costs more than a rebuild)
        fence_proxy_async_smem();
        __syncwarp();
        if ((threadIdx.x & 31) == 0) {
            mbar_arrive_cluster(lead(P_KFULL0 + s));
            mbar_arrive_cluster(lead(P_VFULL0 + s));
        }
    }
}

// Largest of 64 S values (TMEM columns taddr .. taddr + 63 of this thread's
// lane; columns at or past nvalid - cbase left out): two loads, one wait.
template <bool MASKED>
__device__ __forceinline__ float at_max64(uint32_t taddr, int cbase, int nvalid)
{
    uint32_t r0[32], r1[32];
    tmem_ld32_nowait(taddr, r0);
    tmem_ld32_nowait(taddr + 32, r1);
    tmem_ld_wait();
    float m = -INFINITY;
#pragma unroll
    for (int i = 0; i < 32; i += 2) {
        float a0 = __uint_as_float(r0[i]), a1 = __uint_as_float(r0[i + 1]);
        float b0 = __uint_as_float(r1[i]), b1 = __uint_as_float(r1[i + 1]);
        if (MASKED) {
            a0 = cbase + i < nvalid ? a0 : -INFINITY;
            a1 = cbase + i + 1 < nvalid ? a1 : -INFINITY;
            b0 = cbase + 32 + i < nvalid ? b0 : -INFINITY;
            b1 = cbase + 33 + i < nvalid ? b1 : -INFINITY;
        }
        m = fmax3(m, a0, a1);
        m = fmax3(m, b0, b1);
    }
    return m;
}

// One 32-column chunk of P = exp2(s * scale - m), packed fp16 pairs, stored
// (without waiting) as 16 columns of the A operand of P V at tp; the chunk's
// unrounded p are added, pairwise, into acc.
template <bool MASKED>
__device__ __forceinline__ float2 at_exp_chunk(const uint32_t *sv, float scale, float m, int cbase, int nvalid,
                                               uint32_t tp, float2 acc)
{
    uint32_t pk[16];
#pragma unroll
    for (int i = 0; i < 32; i += 2) {
        const float2 x =
            fma2(make_float2(__uint_as_float(sv[i]), __uint_as_float(sv[i + 1])), make_float2(scale, scale),
                 make_float2(-m, -m));
        float p0 = ex2_approx(x.x), p1 = ex2_approx(x.y);
        if (MASKED) {
            p0 = (cbase + i < nvalid) ? p0 : 0.0f;
            p1 = (cbase + i + 1 < nvalid) ? p1 : 0.0f;
        }
        acc = add2(acc, make_float2(p0, p1));
        pk[i / 2] = pack_f16x2_sat(p0, p1);
    }
    tmem_st16(tp, pk);
    return acc;
}

// P of one 128-key tile from S in TMEM (this thread's lane), loads one chunk
// ahead of the arithmetic; returns the tile's sum of p.  P chunk c goes to
// columns 16 c .. 16 c + 15, which hold S values already read.
template <bool MASKED>
__device__ __forceinline__ float at_exp_tile(uint32_t tS, float scale, float m, int nvalid)
{
    uint32_t ra[32], rb[32];
    float2 acc = make_float2(0.0f, 0.0f);
    tmem_ld32_nowait(tS, ra);
    tmem_ld_wait();
    tmem_ld32_nowait(tS + 32, rb);
    acc = at_exp_chunk<MASKED>(ra, scale, m, 0, nvalid, tS, acc);
    tmem_ld_wait();
    tmem_ld32_nowait(tS + 64, ra);
    acc = at_exp_chunk<MASKED>(rb, scale, m, 32, nvalid, tS + 16, acc);
    tmem_ld_wait();
    tmem_ld32_nowait(tS + 96, rb);
    acc = at_exp_chunk<MASKED>(ra, scale, m, 64, nvalid, tS + 32, acc);
    tmem_ld_wait();
    acc = at_exp_chunk<MASKED>(rb, scale, m, 96, nvalid, tS + 48, acc);
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
    return acc.x + acc.y;
}

template <int BK, int BV>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kATThreads, 1)
    attention_tma_kernel(const __grid_constant__ AttnMaps maps, AttnArgs a)
{
    constexpr int D = 128;
    using L = APSmem;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::offBar);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + AT_COUNT);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    auto bar = [&](int i) { return smem_u32(bars + i); };
    auto ksl = [&](int st, int part) { return smem + L::offK + (uint32_t)(2 * st + part) * L::kKh; };
    auto vsl = [&](int st) { return smem + L::offV + (uint32_t)st * L::kV; };

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t rank = cluster_ctarank();
    const int h = blockIdx.y;
    const int64_t q0 = (int64_t)(blockIdx.x >> 1) * kAPRowsPerPair + (int64_t)rank * kAPRowsPerCta;
    if (a.nsplit > 1) {
        const int64_t tiles_all = (a.t_end - a.t_begin + 127) / 128;
        const int z = blockIdx.z;
        const int64_t b0 = a.t_begin + (tiles_all * z / a.nsplit) * 128;
        const int64_t b1 = a.t_begin + (tiles_all * (z + 1) / a.nsplit) * 128;
        a.t_end = b1 < a.t_end ? b1 : a.t_end;
        a.t_begin = b0 < a.t_end ? b0 : a.t_end;
        a.o_out = static_cast<float *>(a.o_out) + (int64_t)z * a.Tq * a.H * D;
        a.lse_out += (int64_t)z * a.H * a.Tq;
        a.o_bf16 = 0;
    }
    const int64_t span = a.t_end - a.t_begin;
    const int ntiles = (int)((span + 127) / 128);

    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(512)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
    if (tid == 0) {
        constexpr uint32_t kProdWarps = 2 * kAPProducers / 32;  // both CTAs
        mbar_init(bar(P_QREADY), kProdWarps);
        for (int st = 0; st < kAPStages; ++st) {
            mbar_init(bar(P_KFULL0 + st), kProdWarps);
            mbar_init(bar(P_VFULL0 + st), kProdWarps);
            mbar_init(bar(P_KFREE0 + st), 1);
            mbar_init(bar(P_VFREE0 + st), 1);
            mbar_init(bar(AT_FILL0 + st), 1);
        }
        mbar_init(bar(P_SFULL0), 1);
        mbar_init(bar(P_SFULL1), 1);
        mbar_init(bar(P_PFULL0), 8);  // 4 softmax warps per CTA and query tile
        mbar_init(bar(P_PFULL1), 8);
        mbar_init(bar(P_OFULL), 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    tc_fence_before();
    cluster_barrier();  // barriers of both CTAs initialised, TMEM allocated
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    auto lead = [&](int i) { return mapa_shared(bar(i), 0); };

    if (warp < kAPProducers / 32) {
        // ------------------------------------------------------------ producer
        {
            const int qt = tid >> 7;
            const uint32_t r = (uint32_t)(tid & 127);
            const int64_t qr = q0 + qt * 128 + r;
            const bool valid = qr < a.Tq;
            const uint16_t *src = a.q + (qr * a.H + h) * D;
            uint8_t *dst = smem + L::offQ + (uint32_t)qt * L::kQ;
#pragma unroll
            for (int u = 0; u < D / 8; ++u) {
                const uint4 w = valid ? __ldg(reinterpret_cast<const uint4 *>(src) + u) : make_uint4(0, 0, 0, 0);
                *reinterpret_cast<uint4 *>(dst + sw128_unit_offset(r, u, 128)) = w;
            }
        }
        if (a.psac_u) {  // the head's PSAC basis; read by producers after their first named barrier
            const float4 *src = reinterpret_cast<const float4 *>(a.psac_u + (int64_t)h * D * 8);
            float4 *dst = reinterpret_cast<float4 *>(smem + ATSmem::offU);
            dst[tid] = __ldg(src + tid);
        }
        ap_publish(lead(P_QREADY));
        if (ntiles > 0)
            at_produce<BK, BV>(a, rank, tid, ntiles, smem, bars, abort_flag);
    } else if (warp == kATLoaderWarp) {
        // ------------------------------------------------------------ loader
        if (ntiles > 0)
            at_load<BK, BV>(a, maps, h, rank, lane, ntiles, smem, bars, abort_flag);
    } else if (warp == kAPProducers / 32) {
        // ------------------------------------------------------------ MMA issuer (leader)
        if (rank == 0 && lane == 0 && ntiles > 0) {
            constexpr uint32_t idescS = idesc_f32acc(256, 128, true, false, false);
            constexpr uint32_t idescO = idesc_f32acc(256, D, false, false, true);
            const uint32_t aQ[2] = {smem_u32(smem + L::offQ), smem_u32(smem + L::offQ + L::kQ)};
            const uint32_t tS[2] = {tmem, tmem + 128}, tO[2] = {tmem + 256, tmem + 384};
            // S(j, qt) = Q_qt (K_j hi + K_j lo)^T into tS[qt]
            auto issue_s = [&](int j, int qt) {
                const int ks_ = j % kAPStages;
                const uint32_t aK[2] = {smem_u32(ksl(ks_, 0)), smem_u32(ksl(ks_, 1))};
#pragma unroll
                for (int part = 0; part < 2; ++part) {
#pragma unroll
                    for (int ks = 0; ks < D / 16; ++ks) {
                        const uint32_t offa = (uint32_t)(ks >> 2) * (128u * 128u) + (uint32_t)(ks & 3) * 32u;
                        const uint32_t offb = (uint32_t)(ks >> 2) * (64u * 128u) + (uint32_t)(ks & 3) * 32u;
                        umma2_ss(tS[qt], sdesc_sw128(aQ[qt] + offa, 16, 1024), sdesc_sw128(aK[part] + offb, 16, 1024),
                                 idescS, (part | ks) ? 1u : 0u);
                    }
                }
                umma2_commit_both(bar(qt ? P_SFULL1 : P_SFULL0));
                if (qt == 1)
                    umma2_commit_both(bar(P_KFREE0 + ks_));
            };
            bool ok = ap_wait(bar(P_QREADY), 0, abort_flag) && ap_wait(bar(P_KFULL0), 0, abort_flag);
            if (ok) {
                tc_fence_after();
                issue_s(0, 0);
                issue_s(0, 1);
            }
            for (int j = 0; ok && j < ntiles; ++j) {
                const int s = j % kAPStages;
                ok = ap_wait(bar(P_VFULL0 + s), (uint32_t)((j / kAPStages) & 1), abort_flag);
                const uint32_t aV = smem_u32(vsl(s));
                for (int qt = 0; ok && qt < 2; ++qt) {
                    ok = ap_wait(bar(qt ? P_PFULL1 : P_PFULL0), (uint32_t)(j & 1), abort_flag);
                    if (!ok)
                        break;
                    tc_fence_after();
#pragma unroll
                    for (int ks = 0; ks < 128 / 16; ++ks)
                        umma2_ts(tO[qt], tS[qt] + (uint32_t)ks * 8u, sdesc_sw128(aV + (uint32_t)ks * 2048u, 16384, 1024),
                                 idescO, (j > 0 || ks > 0) ? 1u : 0u);
                    if (qt == 1)
                        umma2_commit_both(bar(P_VFREE0 + s));
                    if (j + 1 < ntiles) {
                        if (qt == 0) {
                            const int s1 = (j + 1) % kAPStages;
                            ok = ap_wait(bar(P_KFULL0 + s1), (uint32_t)(((j + 1) / kAPStages) & 1), abort_flag);
                            if (!ok)
                                break;
                            tc_fence_after();
                        }
                        issue_s(j + 1, qt);
                    }
                }
            }
            // success: signals the epilogues; failure: drains every MMA issued
            umma2_commit_both(bar(P_OFULL));
            if (!ok) {
                uint32_t spins = 0;
                while (!mbar_try_wait_cluster(bar(P_OFULL), 0) && ++spins < kSpinLimit) {
                }
            }
        }
    } else {
        // ------------------------------------------------------------ softmax
        const int grp = (warp - kAPProducers / 32 - 1) >> 2;
        const uint32_t quarter = (uint32_t)(warp & 3);
        const uint32_t r = quarter * 32u + (uint32_t)lane;
        const uint32_t lane_off = (quarter * 32u) << 16;
        const uint32_t tS = tmem + (grp ? 128u : 0u), tO = tmem + 256u + (grp ? 128u : 0u);
        const uint32_t pfull = lead(grp ? P_PFULL1 : P_PFULL0);
        float m_used = -INFINITY, l = 0.0f;
        bool ok = true;
        for (int j = 0; j < ntiles; ++j) {
            ok = __all_sync(0xffffffffu, ap_wait(bar(grp ? P_SFULL1 : P_SFULL0), (uint32_t)(j & 1), abort_flag));
            if (!ok)
                break;
            tc_fence_after();
            const int64_t t0 = a.t_begin + (int64_t)j * 128;
            const int64_t rem = a.t_end - t0;
            const int nvalid = rem < 128 ? (int)rem : 128;
            const float tmax = nvalid == 128 ? fmaxf(at_max64<false>(tS + lane_off, 0, nvalid),
                                                     at_max64<false>(tS + lane_off + 64u, 64, nvalid))
                                             : fmaxf(at_max64<true>(tS + lane_off, 0, nvalid),
                                                     at_max64<true>(tS + lane_off + 64u, 64, nvalid));
            const float m_tile = tmax * a.scale_log2;
            const bool grow = m_tile > m_used + 8.0f;
            if (__any_sync(0xffffffffu, grow)) {
                const float m_new = grow ? fmaxf(m_tile, m_used) : m_used;
                const float alpha = (m_used == -INFINITY) ? 0.0f : ex2_approx(m_used - m_new);
                if (j > 0) {
#pragma unroll 1
                    for (int cb = 0; cb < D / 32; ++cb) {
                        float ov[32];
                        tmem_ld32(tO + lane_off + (uint32_t)(cb * 32), ov);
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            ov[i] *= alpha;
                        tmem_st32(tO + lane_off + (uint32_t)(cb * 32), ov);
                    }
                }
                l *= alpha;
                m_used = m_new;
            }
            const float lt = nvalid == 128 ? at_exp_tile<false>(tS + lane_off, a.scale_log2, m_used, nvalid)
                                           : at_exp_tile<true>(tS + lane_off, a.scale_log2, m_used, nvalid);
            l += lt;
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive_cluster(pfull);
        }
        const int64_t qr = q0 + grp * 128 + r;
        const bool have =
            __all_sync(0xffffffffu, ntiles > 0 && ok && ap_wait(bar(P_OFULL), 0, abort_flag));
        if (have)
            tc_fence_after();
        else if (ntiles > 0)
            ap_drain_ofull(bar(P_OFULL));  // the leader's last commit lands before this CTA exits
        const bool empty = !(l > 0.0f);
        const float inv_l = empty ? 0.0f : 1.0f / l;
#pragma unroll 1
        for (int cb = 0; cb < D / 32; ++cb) {
            float ov[32];
            if (have)
                tmem_ld32(tO + lane_off + (uint32_t)(cb * 32), ov);
            if (qr < a.Tq) {
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    ov[i] = have ? ov[i] * inv_l : 0.0f;
                if (a.o_bf16) {
                    uint4 *dst =
                        reinterpret_cast<uint4 *>(static_cast<uint16_t *>(a.o_out) + (qr * a.H + h) * D + cb * 32);
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        dst[u] = make_uint4(pack_bf16x2(ov[8 * u], ov[8 * u + 1]), pack_bf16x2(ov[8 * u + 2], ov[8 * u + 3]),
                                            pack_bf16x2(ov[8 * u + 4], ov[8 * u + 5]),
                                            pack_bf16x2(ov[8 * u + 6], ov[8 * u + 7]));
                } else {
                    float4 *dst =
                        reinterpret_cast<float4 *>(static_cast<float *>(a.o_out) + (qr * a.H + h) * D + cb * 32);
#pragma unroll
                    for (int u = 0; u < 8; ++u)
                        dst[u] = make_float4(ov[4 * u], ov[4 * u + 1], ov[4 * u + 2], ov[4 * u + 3]);
                }
            }
        }
        if (qr < a.Tq)
            a.lse_out[(int64_t)h * a.Tq + qr] =
                (empty || !have) ? -INFINITY : (m_used + log2f(l)) * 0.69314718055994531f;
    }

    __syncwarp();  // the MMA lane rejoins its warp before the aligned barrier
    tc_fence_before();
    cluster_barrier();  // all MMAs into either CTA's TMEM are done and read
    tc_fence_after();
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512) : "memory");
}

}  // namespace kvq

// attention_pair.cuh -- attention over a compressed K/V history on CTA pairs
// (thread-block clusters of 2 on two SMs, tcgen05 cta_group::2), d = 128.
//
// Method: NanoKV page, Fig. 4(a,d) (history read through the decoder: centres
// added back to the dequantised residual; partial results carry their
// log-sum-exp); QuantWM, Fig. 9 (on-demand reconstruction during attention).
//
// A pair owns 512 query rows of one head: CTA v holds rows [256 v, 256 v + 256)
// as two 128-row tiles.  For every 128-token history tile the pair's MMAs are
// M = 256 (128 rows from each CTA) and the B operand is split along N:
//   S = Q K_hi^T + Q K_lo^T : CTA v rebuilds the 64 history rows
//       [64 v, 64 v + 64) of the tile (all 128 channels, bf16 hi + lo);
//   O += P V              : CTA v rebuilds channels [64 v, 64 v + 64) of all
//       128 history rows (fp16, MN-major); P comes from each CTA's TMEM.
// So each SM rebuilds half of every tile and every rebuilt element feeds 512
// query rows.  The MMAs are issued by one thread of CTA 0 (the leader).
//
// Roles per CTA (544 threads): warps 0-7 producer (Q tiles, then the CTA's
// halves of k^ and v^), warp 8 MMA issuer (leader only), warps 9-12 / 13-16
// online softmax for query tile 0 / 1 (one thread per row = TMEM lane, lazy
// rescaling of O in TMEM, P written back over S as fp16 pairs).
//
// Barriers (parity = use count & 1).  Counted on the leader, arrived on from
// both CTAs (release.cluster): qready (512), kfull[s], vfull[s] (512 each:
// the producers of both CTAs), pfull[i] (256: the softmax threads of both
// CTAs).  Signalled by multicast tcgen05.commit into both CTAs: sfull[i]
// (S_i ready), kfree[s] (QK of the tile in K stage s done), vfree[s] (P V of
// the tile in V stage s done), ofull (last P V done).  No waiter can fall two
// phases behind: every barrier's next completion needs an action of the
// waiting role.  Waits are bounded and poll a per-CTA abort flag; before TMEM
// is freed the leader drains its MMAs and both CTAs meet at a cluster barrier.
#pragma once

#include "attention.cuh"
#include "attention2.cuh"
#include "codec.cuh"
#include "common.cuh"

namespace kvq {

constexpr int kAPThreads = 544;
constexpr int kAPProducers = 256;
constexpr int kAPRowsPerCta = 256;
constexpr int kAPRowsPerPair = 512;

struct APSmem {
    static constexpr uint32_t kQ = 128 * 2 * 128;     // one 128-row Q tile (d = 128)
    static constexpr uint32_t kKh = 64 * 2 * 128;     // 64 history rows x 128 channels, bf16
    static constexpr uint32_t kV = 128 * 2 * 64;      // 128 history rows x 64 channels, fp16
    static constexpr uint32_t offQ = 0;               // Q tile t at offQ + t kQ
    static constexpr uint32_t offK = 2 * kQ;          // K stage s part p at offK + (2 s + p) kKh
    static constexpr uint32_t offV = offK + 4 * kKh;  // V stage s at offV + s kV
    static constexpr uint32_t offBar = offV + 2 * kV;
    static constexpr uint32_t kBytes = offBar + 256;
    static constexpr uint32_t kLaunchBytes = kBytes + 1024;
};

enum {
    P_QREADY = 0, P_KFULL0, P_KFULL1, P_VFULL0, P_VFULL1, P_SFULL0, P_SFULL1, P_PFULL0, P_PFULL1,
    P_KFREE0, P_KFREE1, P_VFREE0, P_VFREE1, P_OFULL, P_COUNT
};

__device__ __forceinline__ uint32_t cluster_ctarank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ void cluster_barrier()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank)
{
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}

__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr)
{
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ bool ap_wait(uint32_t bar, uint32_t parity, volatile int *abort)
{
    for (uint32_t i = 0; i < kSpinLimit; ++i) {
        if (mbar_try_wait_cluster(bar, parity))
            return true;
        if ((i & 255u) == 255u && *abort)
            return false;
    }
    raise_status(DEVSTAT_TIMEOUT);
    *abort = 1;
    return false;
}

__device__ __forceinline__ void umma2_ss(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t acc)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc)
        : "memory");
}

__device__ __forceinline__ void umma2_ts(uint32_t d, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc, uint32_t acc)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(acc)
        : "memory");
}

// Arrive on the barrier at `bar` in both CTAs of the pair once all tcgen05
// operations issued so far by this thread are complete.
__device__ __forceinline__ void umma2_commit_both(uint32_t bar)
{
    asm volatile(
        "{\n\t.reg .b16 m;\n\tmov.b16 m, 3;\n\t"
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], m;\n\t}" ::"r"(
            bar)
        : "memory");
}

// Rebuild 8-channel units [u0, u0 + n) of history row `tok` (K: bf16 hi + lo
// split; V: fp16) into `tile` at swizzled row `row` of a tile with `rows`
// rows.  Unit u of the row lands at unit (u - ubase) of the tile row.
template <int BITS, bool SPLIT, int NU>
__device__ __forceinline__ void ap_dequant_units(const CodecView &cv, int h, int64_t tok, bool valid, int u0,
                                                 int ubase, uint8_t *tile, uint8_t *tile_lo, uint32_t row,
                                                 uint32_t rows)
{
    constexpr int D = 128;
    if (!valid) {
#pragma unroll
        for (int uu = 0; uu < NU; ++uu) {
            const uint32_t off = sw128_unit_offset(row, u0 + uu - ubase, rows);
            *reinterpret_cast<uint4 *>(tile + off) = make_uint4(0, 0, 0, 0);
            if (SPLIT)
                *reinterpret_cast<uint4 *>(tile_lo + off) = make_uint4(0, 0, 0, 0);
        }
        return;
    }
    const int64_t th = (int64_t)h * cv.T + tok;
    int j = __ldg(cv.idx + th);
    if (j >= cv.C) {
        raise_status(DEVSTAT_BAD_INDEX);
        j = 0;
    }
    const uint4 *mu_row = reinterpret_cast<const uint4 *>(cv.cent + ((int64_t)h * cv.C + j) * D) + u0;
    uint4 mw[NU];
#pragma unroll
    for (int uu = 0; uu < NU; ++uu)
        mw[uu] = __ldg(mu_row + uu);
    uint32_t cws[NU];
    if (BITS == 2) {
        const uint16_t *cr = reinterpret_cast<const uint16_t *>(cv.codes + th * (D / 4)) + u0;
#pragma unroll
        for (int uu = 0; uu < NU; ++uu)
            cws[uu] = __ldg(cr + uu);
    } else {
        const uint32_t *cr = reinterpret_cast<const uint32_t *>(cv.codes + th * (D / 2)) + u0;
#pragma unroll
        for (int uu = 0; uu < NU; ++uu)
            cws[uu] = __ldg(cr + uu);
    }
    const float2 *meta_row = reinterpret_cast<const float2 *>(cv.meta) + th * (D / cv.G);
    constexpr float kTwoB = (float)(1 << BITS);
#pragma unroll
    for (int uu = 0; uu < NU; ++uu) {
        const int c0 = (u0 + uu) * 8;
        const float2 sz = __ldg(meta_row + c0 / cv.G);
        const float sc = kTwoB * sz.x;
        const float nb = -__fmul_rn(kTwoB + sz.y, sz.x);
        const uint32_t ma[4] = {mw[uu].x, mw[uu].y, mw[uu].z, mw[uu].w};
        float2 val[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float2 f = make_float2(code_as_unit_float<BITS>(cws[uu], 2 * k),
                                         code_as_unit_float<BITS>(cws[uu], 2 * k + 1));
            const float2 b = add2(make_float2(bf16_lo(ma[k]), bf16_hi(ma[k])), make_float2(nb, nb));
            val[k] = fma2(f, make_float2(sc, sc), b);
        }
        const uint32_t off = sw128_unit_offset(row, u0 + uu - ubase, rows);
        if (SPLIT) {
            uint32_t hi[4], lo[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint32_t a0 = __float_as_uint(val[k].x) & 0xffff0000u;
                const uint32_t a1 = __float_as_uint(val[k].y) & 0xffff0000u;
                hi[k] = __byte_perm(a0, a1, 0x7632);
                const float2 r = sub2(val[k], make_float2(__uint_as_float(a0), __uint_as_float(a1)));
                lo[k] = pack_bf16x2(r.x, r.y);
            }
            *reinterpret_cast<uint4 *>(tile + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
            *reinterpret_cast<uint4 *>(tile_lo + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
        } else {
            *reinterpret_cast<uint4 *>(tile + off) =
                make_uint4(pack_f16x2_sat(val[0].x, val[0].y), pack_f16x2_sat(val[1].x, val[1].y),
                           pack_f16x2_sat(val[2].x, val[2].y), pack_f16x2_sat(val[3].x, val[3].y));
        }
    }
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kAPThreads, 1) attention_pair_kernel(AttnArgs a)
{
    constexpr int D = 128;
    using L = APSmem;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::offBar);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + P_COUNT);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    auto bar = [&](int i) { return smem_u32(bars + i); };
    auto ksl = [&](int s, int part) { return smem + L::offK + (uint32_t)(2 * s + part) * L::kKh; };
    auto vsl = [&](int s) { return smem + L::offV + (uint32_t)s * L::kV; };

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
        mbar_init(bar(P_QREADY), 2 * kAPProducers);
        mbar_init(bar(P_KFULL0), 2 * kAPProducers);
        mbar_init(bar(P_KFULL1), 2 * kAPProducers);
        mbar_init(bar(P_VFULL0), 2 * kAPProducers);
        mbar_init(bar(P_VFULL1), 2 * kAPProducers);
        mbar_init(bar(P_SFULL0), 1);
        mbar_init(bar(P_SFULL1), 1);
        mbar_init(bar(P_PFULL0), 256);
        mbar_init(bar(P_PFULL1), 256);
        mbar_init(bar(P_KFREE0), 1);
        mbar_init(bar(P_KFREE1), 1);
        mbar_init(bar(P_VFREE0), 1);
        mbar_init(bar(P_VFREE1), 1);
        mbar_init(bar(P_OFULL), 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    tc_fence_before();
    cluster_barrier();  // barriers of both CTAs initialised, TMEM allocated
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // the leader's copy of a barrier, as a cluster address (for arrivals)
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
        fence_proxy_async_smem();
        mbar_arrive_cluster(lead(P_QREADY));
        // K half: history rows [64 rank, 64 rank + 64) of the tile; thread ->
        // (row p & 63, channel quarter p >> 6: units 4q .. 4q+3)
        const uint32_t krow = (uint32_t)(tid & 63);
        const int kq = tid >> 6;
        // V half: channels [64 rank, 64 rank + 64); thread -> (row p & 127,
        // units 8 rank + 4 hh .. + 3, hh = p >> 7)
        const uint32_t vrow = (uint32_t)(tid & 127);
        const int vu0 = 8 * (int)rank + 4 * (tid >> 7);
        auto make_k = [&](int jt, int s) {
            const int64_t tok = a.t_begin + (int64_t)jt * 128 + 64 * rank + krow;
            if (a.k.bits == 2)
                ap_dequant_units<2, true, 4>(a.k, h, tok, tok < a.t_end, 4 * kq, 0, ksl(s, 0), ksl(s, 1), krow, 64);
            else
                ap_dequant_units<4, true, 4>(a.k, h, tok, tok < a.t_end, 4 * kq, 0, ksl(s, 0), ksl(s, 1), krow, 64);
            fence_proxy_async_smem();
            mbar_arrive_cluster(lead(s ? P_KFULL1 : P_KFULL0));
        };
        auto make_v = [&](int jt, int s) {
            const int64_t tok = a.t_begin + (int64_t)jt * 128 + vrow;
            if (a.v.bits == 2)
                ap_dequant_units<2, false, 4>(a.v, h, tok, tok < a.t_end, vu0, 8 * (int)rank, vsl(s), nullptr, vrow,
                                              128);
            else
                ap_dequant_units<4, false, 4>(a.v, h, tok, tok < a.t_end, vu0, 8 * (int)rank, vsl(s), nullptr, vrow,
                                              128);
            fence_proxy_async_smem();
            mbar_arrive_cluster(lead(s ? P_VFULL1 : P_VFULL0));
        };
        if (ntiles > 0) {
            make_k(0, 0);
            make_v(0, 0);
            if (ntiles > 1)
                make_k(1, 1);
            for (int j = 0; j < ntiles; ++j) {
                if (j + 1 < ntiles) {
                    const int s = (j + 1) & 1;
                    if (j >= 1 && !ap_wait(bar(s ? P_VFREE1 : P_VFREE0), (uint32_t)(((j - 1) >> 1) & 1), abort_flag))
                        break;
                    make_v(j + 1, s);
                }
                if (j + 2 < ntiles) {
                    const int s = j & 1;
                    if (!ap_wait(bar(s ? P_KFREE1 : P_KFREE0), (uint32_t)((j >> 1) & 1), abort_flag))
                        break;
                    make_k(j + 2, s);
                }
            }
        }
    } else if (warp == kAPProducers / 32) {
        // ------------------------------------------------------------ MMA issuer (leader)
        if (rank == 0 && lane == 0 && ntiles > 0) {
            constexpr uint32_t idescS = idesc_f32acc(256, 128, true, false, false);
            constexpr uint32_t idescO = idesc_f32acc(256, D, false, false, true);
            const uint32_t aQ[2] = {smem_u32(smem + L::offQ), smem_u32(smem + L::offQ + L::kQ)};
            const uint32_t tS[2] = {tmem, tmem + 128}, tO[2] = {tmem + 256, tmem + 384};
            bool ok = ap_wait(bar(P_QREADY), 0, abort_flag);
            for (int j = 0; ok && j < ntiles; ++j) {
                const int s = j & 1;
                ok = ap_wait(bar(s ? P_KFULL1 : P_KFULL0), (uint32_t)((j >> 1) & 1), abort_flag);
                if (!ok)
                    break;
                tc_fence_after();
                const uint32_t aK[2] = {smem_u32(ksl(s, 0)), smem_u32(ksl(s, 1))};
#pragma unroll
                for (int part = 0; part < 2; ++part) {
#pragma unroll
                    for (int qt = 0; qt < 2; ++qt) {
#pragma unroll
                        for (int ks = 0; ks < D / 16; ++ks) {
                            const uint32_t offa = (uint32_t)(ks >> 2) * (128u * 128u) + (uint32_t)(ks & 3) * 32u;
                            const uint32_t offb = (uint32_t)(ks >> 2) * (64u * 128u) + (uint32_t)(ks & 3) * 32u;
                            umma2_ss(tS[qt], sdesc_sw128(aQ[qt] + offa, 16, 1024),
                                     sdesc_sw128(aK[part] + offb, 16, 1024), idescS, (part | ks) ? 1u : 0u);
                        }
                        if (part == 1)
                            umma2_commit_both(bar(qt ? P_SFULL1 : P_SFULL0));
                    }
                }
                umma2_commit_both(bar(s ? P_KFREE1 : P_KFREE0));
                ok = ap_wait(bar(s ? P_VFULL1 : P_VFULL0), (uint32_t)((j >> 1) & 1), abort_flag);
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
                }
                if (!ok)
                    break;
                umma2_commit_both(bar(s ? P_VFREE1 : P_VFREE0));
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
            float tmax = -INFINITY;
#pragma unroll
            for (int cb = 0; cb < 4; ++cb) {
                float sv[32];
                tmem_ld32(tS + lane_off + (uint32_t)(cb * 32), sv);
                if (nvalid == 128) {
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        tmax = fmaxf(tmax, sv[i]);
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        if (cb * 32 + i < nvalid)
                            tmax = fmaxf(tmax, sv[i]);
                }
            }
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
            float lt = 0.0f;
#pragma unroll
            for (int cb = 0; cb < 4; ++cb) {
                float sv[32];
                tmem_ld32(tS + lane_off + (uint32_t)(cb * 32), sv);
                const uint32_t tp = tS + lane_off + (uint32_t)(cb * 16);
                if (nvalid == 128)
                    lt += a2_softmax_chunk<false>(sv, a.scale_log2, m_used, cb * 32, nvalid, tp);
                else
                    lt += a2_softmax_chunk<true>(sv, a.scale_log2, m_used, cb * 32, nvalid, tp);
            }
            asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
            l += lt;
            tc_fence_before();
            mbar_arrive_cluster(pfull);
        }
        const int64_t qr = q0 + grp * 128 + r;
        const bool have =
            __all_sync(0xffffffffu, ntiles > 0 && ok && ap_wait(bar(P_OFULL), 0, abort_flag));
        if (have)
            tc_fence_after();
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

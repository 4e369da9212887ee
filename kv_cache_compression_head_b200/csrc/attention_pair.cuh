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
// MMA issue order (the two query tiles run half a tile apart, so that the
// softmax of one overlaps the tensor-core work of the other):
//   S(0,0) S(0,1) | P V(0,0) S(1,0) P V(0,1) S(1,1) | P V(1,0) S(2,0) ...
// where S(j,i) = Q_i K_j^T (hi and lo) and P V(j,i) needs the softmax of
// S(j,i).  tcgen05 MMAs of one issuer run in order, so S(j+1,i) overwrites
// P(j,i) in TMEM only after P V(j,i) has read it.
//
// Producers: each thread rebuilds 4 units (32 channels) of one K row and of
// one V row per tile.  The global loads of the next item (its centre row,
// codes and {s, z}) are issued before the current item is rebuilt, and the
// centre index two items ahead, so the gather latency overlaps arithmetic.
//
// Barriers (parity = use count & 1).  Counted on the leader, arrived on once
// per warp from both CTAs (release.cluster, after each lane's proxy fence and
// a warp barrier): qready, kfull[s], vfull[s] (16 each: the producer warps of
// both CTAs), pfull[i] (8: the softmax warps of both CTAs).  Signalled by
// multicast tcgen05.commit into both CTAs: sfull[i] (S_i ready), kfree[s] (QK
// of the tile in K stage s done), vfree[s] (P V of the tile in V stage s
// done), ofull (last P V done).  No waiter can fall two phases behind: every
// barrier's next completion needs an action of the waiting role.  Waits are
// bounded and poll a per-CTA abort flag; before TMEM is freed the leader
// drains its MMAs and both CTAs meet at a cluster barrier.
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

// One thread's share of one history row: 4 units (8 channels each) of the
// centre row, their code words and their groups' {s, z}.
struct APRow {
    uint4 mu[4];
    uint32_t cw[4];
    float2 sz[4];
};

// Centre index of history row `tok` (0 for rows past the range).
__device__ __forceinline__ int ap_index(const CodecView &cv, int h, int64_t tok, bool valid)
{
    return valid ? (int)__ldg(cv.idx + (int64_t)h * cv.T + tok) : 0;
}

// Issue the loads of units [u0, u0 + 4) of row `tok` (centre j).
template <int BITS>
__device__ __forceinline__ void ap_load(const CodecView &cv, int h, int64_t tok, bool valid, int j, int u0,
                                        APRow &r)
{
    constexpr int D = 128;
    if (!valid)
        return;
    if (j >= cv.C) {
        raise_status(DEVSTAT_BAD_INDEX);
        j = 0;
    }
    const int64_t th = (int64_t)h * cv.T + tok;
    const uint4 *mu_row = reinterpret_cast<const uint4 *>(cv.cent + ((int64_t)h * cv.C + j) * D) + u0;
#pragma unroll
    for (int uu = 0; uu < 4; ++uu)
        r.mu[uu] = __ldg(mu_row + uu);
    if (BITS == 2) {
        const uint16_t *cr = reinterpret_cast<const uint16_t *>(cv.codes + th * (D / 4)) + u0;
#pragma unroll
        for (int uu = 0; uu < 4; ++uu)
            r.cw[uu] = __ldg(cr + uu);
    } else {
        const uint32_t *cr = reinterpret_cast<const uint32_t *>(cv.codes + th * (D / 2)) + u0;
#pragma unroll
        for (int uu = 0; uu < 4; ++uu)
            r.cw[uu] = __ldg(cr + uu);
    }
    const float2 *meta_row = reinterpret_cast<const float2 *>(cv.meta) + th * (D / cv.G);
#pragma unroll
    for (int uu = 0; uu < 4; ++uu)
        r.sz[uu] = __ldg(meta_row + (u0 + uu) * 8 / cv.G);
}

// Rebuild the loaded units into `tile` at swizzled row `row` of a tile with
// `rows` rows (unit u0 + uu lands at unit u0 + uu - ubase):
//   x^ = fma(f, 2^b s, mu - (2^b + z) s),  f = 1 + q 2^-b
// which is the decoder's mu + (q - z) s up to one rounding.  K (SPLIT): bf16
// hi (truncated) + lo (the rounded remainder) tiles; V: one fp16 tile.
template <int BITS, bool SPLIT>
__device__ __forceinline__ void ap_store(const APRow &r, bool valid, int u0, int ubase, uint8_t *tile,
                                         uint8_t *tile_lo, uint32_t row, uint32_t rows)
{
    constexpr float kTwoB = (float)(1 << BITS);
#pragma unroll
    for (int uu = 0; uu < 4; ++uu) {
        const uint32_t off = sw128_unit_offset(row, u0 + uu - ubase, rows);
        if (!valid) {
            *reinterpret_cast<uint4 *>(tile + off) = make_uint4(0, 0, 0, 0);
            if (SPLIT)
                *reinterpret_cast<uint4 *>(tile_lo + off) = make_uint4(0, 0, 0, 0);
            continue;
        }
        const float2 sz = r.sz[uu];
        const float sc = kTwoB * sz.x;
        const float nb = -__fmul_rn(kTwoB + sz.y, sz.x);
        const uint32_t ma[4] = {r.mu[uu].x, r.mu[uu].y, r.mu[uu].z, r.mu[uu].w};
        float2 val[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float2 f = make_float2(code_as_unit_float<BITS>(r.cw[uu], 2 * k),
                                         code_as_unit_float<BITS>(r.cw[uu], 2 * k + 1));
            const float2 b = add2(make_float2(bf16_lo(ma[k]), bf16_hi(ma[k])), make_float2(nb, nb));
            val[k] = fma2(f, make_float2(sc, sc), b);
        }
        if (SPLIT) {
            uint32_t hi[4], lo[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint32_t a0 = __float_as_uint(val[k].x) & 0xffff0000u;
                const uint32_t a1 = __float_as_uint(val[k].y) & 0xffff0000u;
                hi[k] = __byte_perm(a0, a1, 0x7632);
                const float2 d = sub2(val[k], make_float2(__uint_as_float(a0), __uint_as_float(a1)));
                lo[k] = pack_bf16x2(d.x, d.y);
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

// Make the warp's generic-proxy writes visible to the tensor core, then one
// lane arrives on the leader's barrier (cluster address).
__device__ __forceinline__ void ap_publish(uint32_t lead_bar)
{
    fence_proxy_async_smem();
    __syncwarp();
    if ((threadIdx.x & 31) == 0)
        mbar_arrive_cluster(lead_bar);
}

// Producer loop: items K(0), V(0), K(1), V(1), ...; K(i) and V(i) reuse the
// stage of tile i - 2 once its MMAs are done.
template <int BK, int BV>
__device__ __forceinline__ void ap_produce(const AttnArgs &a, int h, uint32_t rank, int tid, int ntiles,
                                           uint8_t *smem, uint64_t *bars, volatile int *abort_flag)
{
    using L = APSmem;
    auto bar = [&](int i) { return smem_u32(bars + i); };
    auto lead = [&](int i) { return mapa_shared(bar(i), 0); };
    // K: history rows [64 rank, 64 rank + 64) of the tile; thread -> (row
    // tid & 63, channel quarter tid >> 6: units 4q .. 4q + 3)
    const uint32_t krow = (uint32_t)(tid & 63);
    const int ku0 = 4 * (tid >> 6);
    // V: channels [64 rank, 64 rank + 64); thread -> (row tid & 127, units
    // 8 rank + 4 (tid >> 7) .. + 3)
    const uint32_t vrow = (uint32_t)(tid & 127);
    const int vu0 = 8 * (int)rank + 4 * (tid >> 7);
    auto ktok = [&](int i) { return a.t_begin + (int64_t)i * 128 + 64 * rank + krow; };
    auto vtok = [&](int i) { return a.t_begin + (int64_t)i * 128 + vrow; };

    APRow rk, rv;
    int jk = ap_index(a.k, h, ktok(0), ktok(0) < a.t_end);
    int jv = ap_index(a.v, h, vtok(0), vtok(0) < a.t_end);
    ap_load<BK>(a.k, h, ktok(0), ktok(0) < a.t_end, jk, ku0, rk);
    jk = (ntiles > 1) ? ap_index(a.k, h, ktok(1), ktok(1) < a.t_end) : 0;
    for (int i = 0; i < ntiles; ++i) {
        const int s = i & 1;
        const uint32_t par = (uint32_t)(((i - 2) >> 1) & 1);
        ap_load<BV>(a.v, h, vtok(i), vtok(i) < a.t_end, jv, vu0, rv);
        jv = (i + 1 < ntiles) ? ap_index(a.v, h, vtok(i + 1), vtok(i + 1) < a.t_end) : 0;
        if (i >= 2 && !__all_sync(0xffffffffu, ap_wait(bar(s ? P_KFREE1 : P_KFREE0), par, abort_flag)))
            return;
        ap_store<BK, true>(rk, ktok(i) < a.t_end, ku0, 0, smem + L::offK + (uint32_t)(2 * s) * L::kKh,
                           smem + L::offK + (uint32_t)(2 * s + 1) * L::kKh, krow, 64);
        ap_publish(lead(s ? P_KFULL1 : P_KFULL0));
        if (i + 1 < ntiles) {
            ap_load<BK>(a.k, h, ktok(i + 1), ktok(i + 1) < a.t_end, jk, ku0, rk);
            jk = (i + 2 < ntiles) ? ap_index(a.k, h, ktok(i + 2), ktok(i + 2) < a.t_end) : 0;
        }
        if (i >= 2 && !__all_sync(0xffffffffu, ap_wait(bar(s ? P_VFREE1 : P_VFREE0), par, abort_flag)))
            return;
        ap_store<BV, false>(rv, vtok(i) < a.t_end, vu0, 8 * (int)rank, smem + L::offV + (uint32_t)s * L::kV,
                            nullptr, vrow, 128);
        ap_publish(lead(s ? P_VFULL1 : P_VFULL0));
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
        constexpr uint32_t kProdWarps = 2 * kAPProducers / 32;  // both CTAs
        mbar_init(bar(P_QREADY), kProdWarps);
        mbar_init(bar(P_KFULL0), kProdWarps);
        mbar_init(bar(P_KFULL1), kProdWarps);
        mbar_init(bar(P_VFULL0), kProdWarps);
        mbar_init(bar(P_VFULL1), kProdWarps);
        mbar_init(bar(P_SFULL0), 1);
        mbar_init(bar(P_SFULL1), 1);
        mbar_init(bar(P_PFULL0), 8);  // 4 softmax warps per CTA and query tile
        mbar_init(bar(P_PFULL1), 8);
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
        ap_publish(lead(P_QREADY));
        if (ntiles > 0) {
            if (a.k.bits == 2 && a.v.bits == 2)
                ap_produce<2, 2>(a, h, rank, tid, ntiles, smem, bars, abort_flag);
            else if (a.k.bits == 2)
                ap_produce<2, 4>(a, h, rank, tid, ntiles, smem, bars, abort_flag);
            else if (a.v.bits == 2)
                ap_produce<4, 2>(a, h, rank, tid, ntiles, smem, bars, abort_flag);
            else
                ap_produce<4, 4>(a, h, rank, tid, ntiles, smem, bars, abort_flag);
        }
    } else if (warp == kAPProducers / 32) {
        // ------------------------------------------------------------ MMA issuer (leader)
        if (rank == 0 && lane == 0 && ntiles > 0) {
            constexpr uint32_t idescS = idesc_f32acc(256, 128, true, false, false);
            constexpr uint32_t idescO = idesc_f32acc(256, D, false, false, true);
            const uint32_t aQ[2] = {smem_u32(smem + L::offQ), smem_u32(smem + L::offQ + L::kQ)};
            const uint32_t tS[2] = {tmem, tmem + 128}, tO[2] = {tmem + 256, tmem + 384};
            // S(j, qt) = Q_qt (K_j hi + K_j lo)^T into tS[qt]
            auto issue_s = [&](int j, int qt) {
                const int ks_ = j & 1;
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
                    umma2_commit_both(bar(ks_ ? P_KFREE1 : P_KFREE0));
            };
            bool ok = ap_wait(bar(P_QREADY), 0, abort_flag) && ap_wait(bar(P_KFULL0), 0, abort_flag);
            if (ok) {
                tc_fence_after();
                issue_s(0, 0);
                issue_s(0, 1);
            }
            for (int j = 0; ok && j < ntiles; ++j) {
                const int s = j & 1;
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
                    if (qt == 1)
                        umma2_commit_both(bar(s ? P_VFREE1 : P_VFREE0));
                    if (j + 1 < ntiles) {
                        if (qt == 0) {
                            const int s1 = (j + 1) & 1;
                            ok = ap_wait(bar(s1 ? P_KFULL1 : P_KFULL0), (uint32_t)(((j + 1) >> 1) & 1), abort_flag);
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
            __syncwarp();
            if (lane == 0)
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

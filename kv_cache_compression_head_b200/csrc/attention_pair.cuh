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
// Dense mode (uncompressed bf16 K and V, e.g. the current chunk): the same
// pipeline with the staged rows copied straight into their slots; S takes
// the K hi MMAs only and V is widened in place from bf16 to fp16 (exact in
// fp16's normal range).
//
// Producers: each thread rebuilds 4 units (32 channels) of one K row and of
// one V row per tile.  Two tiles ahead it stages, with per-thread
// asynchronous copies, the centre rows of its units directly into their
// swizzled slots of the operand tiles (K hi, V) and its code words and
// {s, z} into its own slots of the K lo tile; when the tile's turn comes it
// rebuilds the values in place.  Three stages of K and V tiles.
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

constexpr int kAPStages = 3;

struct APSmem {
    static constexpr uint32_t kQ = 128 * 2 * 128;     // one 128-row Q tile (d = 128)
    static constexpr uint32_t kKh = 64 * 2 * 128;     // 64 history rows x 128 channels, bf16
    static constexpr uint32_t kV = 128 * 2 * 64;      // 128 history rows x 64 channels, fp16
    static constexpr uint32_t offQ = 0;               // Q tile t at offQ + t kQ
    static constexpr uint32_t offK = 2 * kQ;          // K stage s part p at offK + (2 s + p) kKh
    static constexpr uint32_t offV = offK + 2 * kAPStages * kKh;  // V stage s at offV + s kV
    static constexpr uint32_t offBar = offV + kAPStages * kV;
    static constexpr uint32_t kBytes = offBar + 256;
    static constexpr uint32_t kLaunchBytes = kBytes + 1024;
};

enum {
    P_QREADY = 0, P_KFULL0, P_VFULL0 = P_KFULL0 + kAPStages, P_SFULL0 = P_VFULL0 + kAPStages, P_SFULL1,
    P_PFULL0, P_PFULL1, P_KFREE0, P_VFREE0 = P_KFREE0 + kAPStages, P_OFULL = P_VFREE0 + kAPStages, P_COUNT
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
    const uint32_t limit = c_wait_limit;
    for (uint32_t i = 0; i < limit; ++i) {
        if (mbar_try_wait_cluster(bar, parity))
            return true;
        if ((i & 255u) == 255u && *abort)
            return false;
    }
    raise_status(DEVSTAT_TIMEOUT);
    *abort = 1;
    return false;
}

// After a give-up: wait (bounded, ignoring the abort flag) for the leader's
// final commit, which it issues on every path once the CTA pair has work.
__device__ __forceinline__ void ap_drain_ofull(uint32_t bar)
{
    uint32_t spins = 0;
    while (!mbar_try_wait_cluster(bar, 0) && ++spins < kSpinLimit) {
    }
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

// Rebuild 4 units of one row in place: the centre units were staged at
// `tile + off[uu]`; codes `cw` and each unit's {s, z} come from the staging
// slots.  x^ = fma(f, 2^b s, mu - (2^b + z) s),  f = 1 + q 2^-b, which is the
// decoder's mu + (q - z) s up to one rounding.  K (SPLIT): bf16 hi
// (truncated) in place + lo (the rounded remainder) at `lo + off[uu]`; V: fp16.
template <int BITS, bool SPLIT>
__device__ __forceinline__ void ap_rebuild(uint8_t *tile, uint8_t *lo, const uint32_t *off, const uint32_t *cw,
                                           const float2 *sz, bool valid)
{
    constexpr float kTwoB = (float)(1 << BITS);
#pragma unroll
    for (int uu = 0; uu < 4; ++uu) {
        uint4 *dst = reinterpret_cast<uint4 *>(tile + off[uu]);
        if (!valid) {
            *dst = make_uint4(0, 0, 0, 0);
            if (SPLIT)
                *reinterpret_cast<uint4 *>(lo + off[uu]) = make_uint4(0, 0, 0, 0);
            continue;
        }
        const uint4 mw = *dst;
        const float sc = kTwoB * sz[uu].x;
        const float nb = -__fmul_rn(kTwoB + sz[uu].y, sz[uu].x);
        const uint32_t ma[4] = {mw.x, mw.y, mw.z, mw.w};
        float2 val[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float2 f = make_float2(code_as_unit_float<BITS>(cw[uu], 2 * k),
                                         code_as_unit_float<BITS>(cw[uu], 2 * k + 1));
            const float2 b = add2(make_float2(bf16_lo(ma[k]), bf16_hi(ma[k])), make_float2(nb, nb));
            val[k] = fma2(f, make_float2(sc, sc), b);
        }
        if (SPLIT) {
            uint32_t hi[4], lw[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint32_t a0 = __float_as_uint(val[k].x) & 0xffff0000u;
                const uint32_t a1 = __float_as_uint(val[k].y) & 0xffff0000u;
                hi[k] = __byte_perm(a0, a1, 0x7632);
                const float2 d = sub2(val[k], make_float2(__uint_as_float(a0), __uint_as_float(a1)));
                lw[k] = pack_bf16x2(d.x, d.y);
            }
            *dst = make_uint4(hi[0], hi[1], hi[2], hi[3]);
            *reinterpret_cast<uint4 *>(lo + off[uu]) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
        } else {
            *dst = make_uint4(pack_f16x2_sat(val[0].x, val[0].y), pack_f16x2_sat(val[1].x, val[1].y),
                              pack_f16x2_sat(val[2].x, val[2].y), pack_f16x2_sat(val[3].x, val[3].y));
        }
    }
}

// Stage units [u0, u0 + 4) of history row `tok` (centre j) of one codec: the
// centre units into `tile + off[uu]`, the code words (8 or 16 B) into
// `stage_cw` and the {s, z} of their groups (8 or 16 B) into `stage_sz`.
template <int BITS>
__device__ __forceinline__ void ap_stage(const CodecView &cv, int h, int64_t tok, int j, int u0, uint32_t tile,
                                         const uint32_t *off, uint32_t stage_cw, uint32_t stage_sz)
{
    constexpr int D = 128;
    if (j >= cv.C) {
        raise_status(DEVSTAT_BAD_INDEX);
        j = 0;
    }
    const int64_t th = (int64_t)h * cv.T + tok;
    const uint16_t *mu = cv.cent + ((int64_t)h * cv.C + j) * D + u0 * 8;
#pragma unroll
    for (int uu = 0; uu < 4; ++uu)
        cp_async16(tile + off[uu], mu + uu * 8);
    if (BITS == 2)
        cp_async8(stage_cw, cv.codes + th * (D / 4) + u0 * 2);
    else
        cp_async16(stage_cw, cv.codes + th * (D / 2) + u0 * 4);
    const float *meta = static_cast<const float *>(cv.meta) + (th * (D / cv.G) + (u0 * 8) / cv.G) * 2;  // binary32 {s, z}
    if (cv.G == 16)
        cp_async16(stage_sz, meta);
    else
        cp_async8(stage_sz, meta);
}

// Code words and per-unit {s, z} of 4 units from the staging slots.
template <int BITS>
__device__ __forceinline__ void ap_read_stage(const uint8_t *stage_cw, const uint8_t *stage_sz, int G, uint32_t *cw,
                                              float2 *sz)
{
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
        const float4 m = *reinterpret_cast<const float4 *>(stage_sz);
        sz[0] = sz[1] = make_float2(m.x, m.y);
        sz[2] = sz[3] = make_float2(m.z, m.w);
    } else {
        const float2 m = *reinterpret_cast<const float2 *>(stage_sz);
        sz[0] = sz[1] = sz[2] = sz[3] = m;
    }
}

// Dense mode: stage units [u0, u0 + 4) of row `tok` of a bf16 [Tk][H][128]
// key or value array straight into their swizzled slots.
__device__ __forceinline__ void ap_stage_dense(const uint16_t *x, int H, int h, int64_t tok, int u0, uint32_t tile,
                                               const uint32_t *off)
{
    const uint16_t *src = x + (tok * H + h) * 128 + u0 * 8;
#pragma unroll
    for (int uu = 0; uu < 4; ++uu)
        cp_async16(tile + off[uu], src + uu * 8);
}

// Dense mode, once the staged copies have landed: rows past the end become
// zeros; V units (VALUE) are widened in place from bf16 to fp16.
template <bool VALUE>
__device__ __forceinline__ void ap_finish_dense(uint8_t *tile, const uint32_t *off, bool valid)
{
#pragma unroll
    for (int uu = 0; uu < 4; ++uu) {
        uint4 *dst = reinterpret_cast<uint4 *>(tile + off[uu]);
        if (!valid) {
            *dst = make_uint4(0, 0, 0, 0);
        } else if (VALUE) {
            const uint4 w = *dst;
            *dst = make_uint4(pack_f16x2_sat(bf16_lo(w.x), bf16_hi(w.x)), pack_f16x2_sat(bf16_lo(w.y), bf16_hi(w.y)),
                              pack_f16x2_sat(bf16_lo(w.z), bf16_hi(w.z)), pack_f16x2_sat(bf16_lo(w.w), bf16_hi(w.w)));
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

// Producer loop over tiles i: rebuild K(i) and V(i), then stage K(i + 2)
// once the QK of tile i - 1 has freed its stage and V(i + 2) once its P V
// has.  One commit group per staging step (empty past the end), so "all but
// the newest two groups" is always the pair K(i), V(i).  DENSE: bf16 K and V
// rows instead of codes (BK, BV unused).
template <int BK, int BV, bool DENSE>
__device__ __forceinline__ void ap_produce(const AttnArgs &a, int h, uint32_t rank, int tid, int ntiles,
                                           uint8_t *smem, uint64_t *bars, volatile int *abort_flag)
{
    using L = APSmem;
    auto bar = [&](int i) { return smem_u32(bars + i); };
    auto lead = [&](int i) { return mapa_shared(bar(i), 0); };
    auto khi = [&](int s) { return smem + L::offK + (uint32_t)(2 * s) * L::kKh; };
    auto klo = [&](int s) { return smem + L::offK + (uint32_t)(2 * s + 1) * L::kKh; };
    auto vst = [&](int s) { return smem + L::offV + (uint32_t)s * L::kV; };
    // K: history rows [64 rank, 64 rank + 64) of the tile; thread -> (row
    // tid & 63, channel quarter tid >> 6: units 4q .. 4q + 3).  Its 4 K lo
    // slots double as staging: K codes, K {s, z}, V codes, V {s, z}.
    const uint32_t krow = (uint32_t)(tid & 63);
    const int ku0 = 4 * (tid >> 6);
    // V: channels [64 rank, 64 rank + 64); thread -> (row tid & 127, units
    // 8 rank + 4 (tid >> 7) .. + 3)
    const uint32_t vrow = (uint32_t)(tid & 127);
    const int vu0 = 8 * (int)rank + 4 * (tid >> 7);
    uint32_t koff[4], voff[4];
#pragma unroll
    for (int uu = 0; uu < 4; ++uu) {
        koff[uu] = sw128_unit_offset(krow, ku0 + uu, 64);
        voff[uu] = sw128_unit_offset(vrow, vu0 - 8 * (int)rank + uu, 128);
    }
    auto ktok = [&](int i) { return a.t_begin + (int64_t)i * 128 + 64 * rank + krow; };
    auto vtok = [&](int i) { return a.t_begin + (int64_t)i * 128 + vrow; };
    auto kidx = [&](int i) {
        if constexpr (DENSE) {
            return 0;
        } else {
            const int64_t t = ktok(i);
            return (i < ntiles && t < a.t_end) ? (int)__ldg(a.k.idx + (int64_t)h * a.k.T + t) : 0;
        }
    };
    auto vidx = [&](int i) {
        if constexpr (DENSE) {
            return 0;
        } else {
            const int64_t t = vtok(i);
            return (i < ntiles && t < a.t_end) ? (int)__ldg(a.v.idx + (int64_t)h * a.v.T + t) : 0;
        }
    };
    auto stage_k = [&](int i, int j) {
        const int s = i % kAPStages;
        if (ktok(i) < a.t_end) {
            if constexpr (DENSE)
                ap_stage_dense(a.k_dense, a.H, h, ktok(i), ku0, smem_u32(khi(s)), koff);
            else
                ap_stage<BK>(a.k, h, ktok(i), j, ku0, smem_u32(khi(s)), koff, smem_u32(klo(s) + koff[0]),
                             smem_u32(klo(s) + koff[1]));
        }
    };
    auto stage_v = [&](int i, int j) {
        const int s = i % kAPStages;
        if (vtok(i) < a.t_end) {
            if constexpr (DENSE)
                ap_stage_dense(a.v_dense, a.H, h, vtok(i), vu0, smem_u32(vst(s)), voff);
            else
                ap_stage<BV>(a.v, h, vtok(i), j, vu0, smem_u32(vst(s)), voff, smem_u32(klo(s) + koff[2]),
                             smem_u32(klo(s) + koff[3]));
        }
    };

    // prologue: tiles 0 and 1
    {
        const int jk0 = kidx(0), jv0 = vidx(0), jk1 = kidx(1), jv1 = vidx(1);
        stage_k(0, jk0);
        cp_async_commit();
        stage_v(0, jv0);
        cp_async_commit();
        if (ntiles > 1)
            stage_k(1, jk1);
        cp_async_commit();
        if (ntiles > 1)
            stage_v(1, jv1);
        cp_async_commit();
    }
    int jk = kidx(2), jv = vidx(2);
    for (int i = 0; i < ntiles; ++i) {
        const int s = i % kAPStages;
        // (1) rebuild K(i) and V(i) from their staged data (all but the newest
        // two commit groups); V's staged words are read first: K lo is
        // overwritten by the K rebuild
        cp_async_wait<2>();
        if constexpr (DENSE) {
            ap_finish_dense<false>(khi(s), koff, ktok(i) < a.t_end);
            ap_publish(lead(P_KFULL0 + s));
            ap_finish_dense<true>(vst(s), voff, vtok(i) < a.t_end);
            ap_publish(lead(P_VFULL0 + s));
        } else {
            uint32_t kcw[4], vcw[4];
            float2 ksz[4], vsz[4];
            ap_read_stage<BK>(klo(s) + koff[0], klo(s) + koff[1], a.k.G, kcw, ksz);
            ap_read_stage<BV>(klo(s) + koff[2], klo(s) + koff[3], a.v.G, vcw, vsz);
            ap_rebuild<BK, true>(khi(s), klo(s), koff, kcw, ksz, ktok(i) < a.t_end);
            ap_publish(lead(P_KFULL0 + s));
            ap_rebuild<BV, false>(vst(s), nullptr, voff, vcw, vsz, vtok(i) < a.t_end);
            ap_publish(lead(P_VFULL0 + s));
        }
        // (2) stage tile i + 2 into the stage of tile i - 1 once its QK (K) and
        // its P V (V) are done.  Issued after the publications above, whose
        // proxy fences then need not wait for these copies.
        const int sp = (i + 2) % kAPStages;
        const uint32_t par_prev = (uint32_t)(((i - 1) / kAPStages) & 1);
        if (i + 2 < ntiles) {
            if (i >= 1 && !__all_sync(0xffffffffu, ap_wait(bar(P_KFREE0 + sp), par_prev, abort_flag))) {
                cp_async_wait<0>();
                return;
            }
            stage_k(i + 2, jk);
            jk = kidx(i + 3);
        }
        cp_async_commit();
        if (i + 2 < ntiles) {
            if (i >= 1 && !__all_sync(0xffffffffu, ap_wait(bar(P_VFREE0 + sp), par_prev, abort_flag))) {
                cp_async_wait<0>();
                return;
            }
            stage_v(i + 2, jv);
            jv = vidx(i + 3);
        }
        cp_async_commit();
    }
    cp_async_wait<0>();
}

// One instantiation per (K bits, V bits) of a compressed history, and one for
// dense keys and values (BK = BV = 0), so that each carries only its producer.
template <int BK, int BV, bool DENSE>
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
        if (ntiles > 0)
            ap_produce<BK, BV, DENSE>(a, h, rank, tid, ntiles, smem, bars, abort_flag);
    } else if (warp == kAPProducers / 32) {
        // ------------------------------------------------------------ MMA issuer (leader)
        if (rank == 0 && lane == 0 && ntiles > 0) {
            constexpr uint32_t idescS = idesc_f32acc(256, 128, true, false, false);
            constexpr uint32_t idescO = idesc_f32acc(256, D, false, false, true);
            const uint32_t aQ[2] = {smem_u32(smem + L::offQ), smem_u32(smem + L::offQ + L::kQ)};
            const uint32_t tS[2] = {tmem, tmem + 128}, tO[2] = {tmem + 256, tmem + 384};
            constexpr int nparts = DENSE ? 1 : 2;  // dense keys have no lo part
            // S(j, qt) = Q_qt (K_j hi + K_j lo)^T into tS[qt]
            auto issue_s = [&](int j, int qt) {
                const int ks_ = j % kAPStages;
                const uint32_t aK[2] = {smem_u32(ksl(ks_, 0)), smem_u32(ksl(ks_, 1))};
#pragma unroll
                for (int part = 0; part < nparts; ++part) {
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

// attention2.cuh -- warp-specialised attention over a compressed K/V history
// (tcgen05 / TMEM), two 128-row query tiles per CTA.
//
// Method: NanoKV page, Fig. 4(a,d) (history read through the decoder: centres
// added back to the dequantised residual; partial results carry their
// log-sum-exp); QuantWM, Fig. 9 (on-demand reconstruction during attention).
//
// Roles (544 threads):
//   warps 0-7   producer: load the two Q tiles, then for every 128-token
//               history tile rebuild k^ (bf16 hi + lo tiles) and v^ (fp16
//               tile) from codes, {s, z}, idx and the bf16 centres straight
//               into the 128-byte-swizzled operand layout; two threads per
//               history row, one per half of the channels.  Dense mode
//               (uncompressed bf16 K and V): the rows are copied instead, K
//               has no lo tile and V is widened to fp16.
//   warp 8      MMA issuer (one thread): S_i = Q_i K_hi^T + Q_i K_lo^T into
//               TMEM for both query tiles, then O_i += P_i V^ (fp16) once the
//               softmax has published P_i.
//   warps 9-12  softmax for query tile 0, warps 13-16 for query tile 1: one
//               thread per query row (its TMEM lane); online softmax in the
//               exp2 domain with lazy rescaling (O in TMEM is rescaled only
//               when the running maximum grows by more than 2^8); P (fp16
//               pairs) is written back over the S tile it came from and read
//               by the P V MMA straight from TMEM.
// Shared memory: Q tiles 2 x 32 KB, two K stages of 2 x 32 KB (K_hi, K_lo),
// one V tile of 32 KB (d = 128).  TMEM: S_0, S_1 (128 columns each; P_i in the
// first 64 columns of S_i) and O_0, O_1 (d columns each).
//
// Ordering (mbarriers; parity = use count & 1):
//   kfull[s]  producer -> MMA   K stage s holds tile j (j = s mod 2)
//   vfull     producer -> MMA   V tile j written
//   sfull[i]  MMA -> softmax    S_i(j) complete (QK MMAs run hi(0), hi(1),
//             lo(0), lo(1))
//   pfull[i]  softmax -> MMA    P_i(j) in TMEM, O_i rescaled.  The next
//             QK_i overwrites S_i only after P V_i(j), issued before it, has
//             read P_i (tcgen05 MMAs of one thread execute in order)
//   pvdone    MMA -> producer   PV_0(j), PV_1(j) complete: V and K stage j free
//   ofull     MMA -> softmax    last PV complete
// Every wait is bounded and also polls a shared abort flag, so that one
// role giving up releases the others; the MMA thread drains its tcgen05 work
// before TMEM is freed.
#pragma once

#include "attention.cuh"
#include "codec.cuh"
#include "common.cuh"

namespace kvq {

constexpr int kA2Threads = 544;
constexpr int kA2Producers = 256;
constexpr int kA2Rows = 256;  // query rows per CTA (two tiles)

template <int D>
struct A2Smem {
    static constexpr uint32_t kQ = D * 2 * 128;
    static constexpr uint32_t kKt = D * 2 * 128;           // one K_hi / K_lo tile
    static constexpr uint32_t kSlot = kKt;
    static constexpr uint32_t offQ0 = 0, offQ1 = kQ;
    static constexpr uint32_t offStage = 2 * kQ;          // stage s slot t at offStage + (2s + t) kSlot
    static constexpr uint32_t offV = offStage + 4 * kSlot;
    static constexpr uint32_t offBar = offV + kKt;
    static constexpr uint32_t kBytes = offBar + 128;
    static constexpr uint32_t kLaunchBytes = kBytes + 1024;
};

enum { B_QREADY = 0, B_KFULL0, B_KFULL1, B_VFULL, B_SFULL0, B_SFULL1, B_PFULL0, B_PFULL1, B_PVDONE, B_OFULL, B_COUNT };

// Bounded wait that also gives up when another role has raised `abort`.
__device__ __forceinline__ bool a2_wait(uint32_t bar, uint32_t parity, volatile int *abort)
{
    for (uint32_t i = 0; i < kSpinLimit; ++i) {
        if (mbar_try_wait(bar, parity))
            return true;
        if ((i & 255u) == 255u && *abort)
            return false;
    }
    raise_status(DEVSTAT_TIMEOUT);
    *abort = 1;
    return false;
}

// f = 1 + q 2^-b for the code of channel k (0..7) of a unit: the code bits are
// moved into the top of the mantissa of 1.0f.
template <int BITS>
__device__ __forceinline__ float code_as_unit_float(uint32_t cw, int k)
{
    constexpr int kShift = 23 - BITS;
    constexpr uint32_t kMask = ((1u << BITS) - 1u) << kShift;
    const int sh = kShift - k * BITS;
    const uint32_t qb = (sh >= 0 ? (cw << sh) : (cw >> -sh)) & kMask;
    return __uint_as_float(0x3F800000u | qb);
}

// Rebuild channels [d/2 half, d/2 half + d/2) of history row `tok` of a
// compressed K (SPLIT: bf16 hi + lo tiles) or V (fp16 tile) into the swizzled
// tiles:  x^ = fma(f, 2^b s, mu - (2^b + z) s),  f = 1 + q 2^-b,  which is the
// decoder's mu + (q - z) s up to one rounding.  The loads of the half row are
// issued together before any arithmetic.
template <int D, int BITS, bool SPLIT>
__device__ __forceinline__ void a2_dequant_half(const CodecView &cv, int h, int64_t tok, bool valid, int half,
                                                uint8_t *tile, uint8_t *tile_lo, uint32_t row)
{
    constexpr int kUnits = D / 16;  // 8-channel units in a half row
    const int u0 = half * kUnits;
    if (!valid) {
#pragma unroll
        for (int uu = 0; uu < kUnits; ++uu) {
            const uint32_t off = sw128_unit_offset(row, u0 + uu, 128);
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
    uint4 mw[kUnits];
#pragma unroll
    for (int uu = 0; uu < kUnits; ++uu)
        mw[uu] = __ldg(mu_row + uu);
    uint32_t cws[kUnits];
    if (BITS == 2) {
        const uint16_t *cr = reinterpret_cast<const uint16_t *>(cv.codes + th * (D / 4)) + u0;
#pragma unroll
        for (int uu = 0; uu < kUnits; ++uu)
            cws[uu] = __ldg(cr + uu);
    } else {
        const uint32_t *cr = reinterpret_cast<const uint32_t *>(cv.codes + th * (D / 2)) + u0;
#pragma unroll
        for (int uu = 0; uu < kUnits; ++uu)
            cws[uu] = __ldg(cr + uu);
    }
    const float2 *meta_row = static_cast<const float2 *>(cv.meta) + th * (D / cv.G);  // binary32 {s, z} only
    constexpr float kTwoB = (float)(1 << BITS);
#pragma unroll
    for (int uu = 0; uu < kUnits; ++uu) {
        const int c0 = (u0 + uu) * 8;
        const float2 sz = __ldg(meta_row + c0 / cv.G);
        const float sc = kTwoB * sz.x;                  // 2^b s (exact)
        const float nb = -__fmul_rn(kTwoB + sz.y, sz.x); // -(2^b + z) s
        const uint32_t ma[4] = {mw[uu].x, mw[uu].y, mw[uu].z, mw[uu].w};
        float2 val[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float2 f = make_float2(code_as_unit_float<BITS>(cws[uu], 2 * k),
                                         code_as_unit_float<BITS>(cws[uu], 2 * k + 1));
            const float2 b = add2(make_float2(bf16_lo(ma[k]), bf16_hi(ma[k])), make_float2(nb, nb));
            val[k] = fma2(f, make_float2(sc, sc), b);
        }
        const uint32_t off = sw128_unit_offset(row, u0 + uu, 128);
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

template <int D, bool SPLIT>
__device__ __forceinline__ void a2_dequant(const CodecView &cv, int h, int64_t tok, bool valid, int half, uint8_t *tile,
                                           uint8_t *tile_lo, uint32_t row)
{
    if (cv.bits == 2)
        a2_dequant_half<D, 2, SPLIT>(cv, h, tok, valid, half, tile, tile_lo, row);
    else
        a2_dequant_half<D, 4, SPLIT>(cv, h, tok, valid, half, tile, tile_lo, row);
}

// Dense mode: channels [d/2 half, d/2 half + d/2) of row `tok` of an
// uncompressed bf16 [Tk][H][D] array into the swizzled tile -- keys as they
// are (the K hi tile; no lo part), values (VALUE) widened to fp16.
template <int D, bool VALUE>
__device__ __forceinline__ void a2_dense_half(const uint16_t *x, int H, int h, int64_t tok, bool valid, int half,
                                              uint8_t *tile, uint32_t row)
{
    constexpr int kUnits = D / 16;
    const int u0 = half * kUnits;
    uint4 w[kUnits];
    const uint4 *src = reinterpret_cast<const uint4 *>(x + (tok * H + h) * D) + u0;
#pragma unroll
    for (int uu = 0; uu < kUnits; ++uu)
        w[uu] = valid ? __ldg(src + uu) : make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int uu = 0; uu < kUnits; ++uu) {
        if (VALUE)
            w[uu] = make_uint4(pack_f16x2_sat(bf16_lo(w[uu].x), bf16_hi(w[uu].x)),
                               pack_f16x2_sat(bf16_lo(w[uu].y), bf16_hi(w[uu].y)),
                               pack_f16x2_sat(bf16_lo(w[uu].z), bf16_hi(w[uu].z)),
                               pack_f16x2_sat(bf16_lo(w[uu].w), bf16_hi(w[uu].w)));
        *reinterpret_cast<uint4 *>(tile + sw128_unit_offset(row, u0 + uu, 128)) = w[uu];
    }
}

// One history row's half of the K operand (hi, lo) or of the V operand,
// rebuilt from the compressed view or copied in dense mode.
template <int D>
__device__ __forceinline__ void a2_fill_k(const AttnArgs &a, int h, int64_t tok, int half, uint8_t *hi, uint8_t *lo,
                                          uint32_t row)
{
    if (a.dense)
        a2_dense_half<D, false>(a.k_dense, a.H, h, tok, tok < a.t_end, half, hi, row);
    else
        a2_dequant<D, true>(a.k, h, tok, tok < a.t_end, half, hi, lo, row);
}

template <int D>
__device__ __forceinline__ void a2_fill_v(const AttnArgs &a, int h, int64_t tok, int half, uint8_t *tile, uint32_t row)
{
    if (a.dense)
        a2_dense_half<D, true>(a.v_dense, a.H, h, tok, tok < a.t_end, half, tile, row);
    else
        a2_dequant<D, false>(a.v, h, tok, tok < a.t_end, half, tile, nullptr, row);
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float *v)
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
        "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
        "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
        "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
        "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
        "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
        "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
        "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
        "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
        "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
        "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
        : "memory");
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// 16 consecutive 32-bit TMEM columns of this thread's lane.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t *v)
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
        "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
        : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]; A is M rows (lanes) x K 16-bit elements, two
// per 32-bit column (even element in the low half).
__device__ __forceinline__ void umma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                        uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// One 32-column chunk of P = exp2(s * scale - m), packed fp16 pairs, written
// back into TMEM as 16 columns of the A operand of P V (columns 16 cb ..
// 16 cb + 15 of the S tile, which this thread has already read); returns the
// chunk's sum of the (unrounded) p.
template <bool MASKED>
__device__ __forceinline__ float a2_softmax_chunk(const float *sv, float scale, float m, int cbase, int nvalid,
                                                  uint32_t tp)
{
    float lt = 0.0f;
    uint32_t pk[16];
#pragma unroll
    for (int i = 0; i < 32; i += 2) {
        float p0 = ex2_approx(fmaf(sv[i], scale, -m));
        float p1 = ex2_approx(fmaf(sv[i + 1], scale, -m));
        if (MASKED) {
            p0 = (cbase + i < nvalid) ? p0 : 0.0f;
            p1 = (cbase + i + 1 < nvalid) ? p1 : 0.0f;
        }
        lt += p0 + p1;
        pk[i / 2] = pack_f16x2_sat(p0, p1);
    }
    tmem_st16(tp, pk);
    return lt;
}

template <int D>
__global__ void __launch_bounds__(kA2Threads, 1) attention2_kernel(AttnArgs a)
{
    using L = A2Smem<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::offBar);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + B_COUNT);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    auto bar = [&](int i) { return smem_u32(bars + i); };
    auto slot = [&](int s, int t) { return smem + L::offStage + (uint32_t)(2 * s + t) * L::kSlot; };

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int h = blockIdx.y;
    const int64_t q0 = (int64_t)blockIdx.x * kA2Rows;
    if (a.nsplit > 1) {
        // sub-range z of the history, split at 128-token tile boundaries; the
        // partial result (binary32) goes to slice z of the partial buffers
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

    if (warp == 0)
        tmem_alloc(smem_u32(tmem_slot), 512);
    if (tid == 0) {
        mbar_init(bar(B_QREADY), kA2Producers);
        mbar_init(bar(B_KFULL0), kA2Producers);
        mbar_init(bar(B_KFULL1), kA2Producers);
        mbar_init(bar(B_VFULL), kA2Producers);
        mbar_init(bar(B_SFULL0), 1);
        mbar_init(bar(B_SFULL1), 1);
        mbar_init(bar(B_PFULL0), 128);
        mbar_init(bar(B_PFULL1), 128);
        mbar_init(bar(B_PVDONE), 1);
        mbar_init(bar(B_OFULL), 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp < kA2Producers / 32) {
        // ------------------------------------------------------------ producer
        {
            const int qt = tid >> 7;
            const uint32_t r = (uint32_t)(tid & 127);
            const int64_t qr = q0 + qt * 128 + r;
            const bool valid = qr < a.Tq;
            const uint16_t *src = a.q + (qr * a.H + h) * D;
            uint8_t *dst = smem + (qt ? L::offQ1 : L::offQ0);
#pragma unroll
            for (int u = 0; u < D / 8; ++u) {
                const uint4 w = valid ? __ldg(reinterpret_cast<const uint4 *>(src) + u) : make_uint4(0, 0, 0, 0);
                *reinterpret_cast<uint4 *>(dst + sw128_unit_offset(r, u, 128)) = w;
            }
        }
        fence_proxy_async_smem();
        mbar_arrive(bar(B_QREADY));
        const uint32_t r = (uint32_t)(tid & 127);
        const int half = tid >> 7;
        if (ntiles > 0) {
            {
                const int64_t tok = a.t_begin + r;
                a2_fill_k<D>(a, h, tok, half, slot(0, 0), slot(0, 1), r);
                fence_proxy_async_smem();
                mbar_arrive(bar(B_KFULL0));
            }
            for (int j = 0; j < ntiles; ++j) {
                if (j >= 1 && !a2_wait(bar(B_PVDONE), (uint32_t)((j - 1) & 1), abort_flag))
                    break;
                const int64_t tok = a.t_begin + (int64_t)j * 128 + r;
                a2_fill_v<D>(a, h, tok, half, smem + L::offV, r);
                fence_proxy_async_smem();
                mbar_arrive(bar(B_VFULL));
                if (j + 1 < ntiles) {
                    const int s = (j + 1) & 1;
                    const int64_t tk = tok + 128;
                    a2_fill_k<D>(a, h, tk, half, slot(s, 0), slot(s, 1), r);
                    fence_proxy_async_smem();
                    mbar_arrive(bar(s ? B_KFULL1 : B_KFULL0));
                }
            }
        }
    } else if (warp == kA2Producers / 32) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0 && ntiles > 0) {
            constexpr uint32_t idescS = idesc_f32acc(128, 128, true, false, false);
            constexpr uint32_t idescO = idesc_f32acc(128, D, false, false, true);
            const uint32_t aQ[2] = {smem_u32(smem + L::offQ0), smem_u32(smem + L::offQ1)};
            const uint32_t aV = smem_u32(smem + L::offV);
            const uint32_t tS[2] = {tmem, tmem + 128}, tO[2] = {tmem + 256, tmem + 256 + D};
            const int last_part = a.dense ? 0 : 1;  // dense keys have no lo part
            bool ok = a2_wait(bar(B_QREADY), 0, abort_flag);
            for (int j = 0; ok && j < ntiles; ++j) {
                const int s = j & 1;
                ok = a2_wait(bar(s ? B_KFULL1 : B_KFULL0), (uint32_t)((j >> 1) & 1), abort_flag);
                if (!ok)
                    break;
                tc_fence_after();
                const uint32_t aKh = smem_u32(slot(s, 0)), aKl = smem_u32(slot(s, 1));
                // order hi(0), hi(1), lo(0), lo(1): when S_0 completes, K_hi is no
                // longer read and can take P_0; S_1 completes last (K_lo -> P_1)
#pragma unroll
                for (int part = 0; part < 2; ++part) {
                    if (part > last_part)
                        break;
#pragma unroll
                    for (int qt = 0; qt < 2; ++qt) {
#pragma unroll
                        for (int ks = 0; ks < D / 16; ++ks) {
                            const uint32_t off = (uint32_t)(ks >> 2) * (128u * 128u) + (uint32_t)(ks & 3) * 32u;
                            umma_ss(tS[qt], sdesc_sw128(aQ[qt] + off, 16, 1024),
                                    sdesc_sw128((part ? aKl : aKh) + off, 16, 1024), idescS, (part | ks) ? 1u : 0u);
                        }
                        if (part == last_part)
                            umma_commit(bar(qt ? B_SFULL1 : B_SFULL0));
                    }
                }
                ok = a2_wait(bar(B_VFULL), (uint32_t)(j & 1), abort_flag);
                for (int qt = 0; ok && qt < 2; ++qt) {
                    ok = a2_wait(bar(qt ? B_PFULL1 : B_PFULL0), (uint32_t)(j & 1), abort_flag);
                    if (!ok)
                        break;
                    tc_fence_after();
#pragma unroll
                    for (int ks = 0; ks < 128 / 16; ++ks)
                        umma_ts(tO[qt], tS[qt] + (uint32_t)ks * 8u,
                                sdesc_sw128(aV + (uint32_t)ks * 2048u, 128u * 128u, 1024), idescO,
                                (j > 0 || ks > 0) ? 1u : 0u);
                }
                if (!ok)
                    break;
                umma_commit(bar(B_PVDONE));
            }
            // on success this signals the epilogue; on failure it drains every
            // MMA issued so far before TMEM is freed
            umma_commit(bar(B_OFULL));
            if (!ok) {
                uint32_t spins = 0;
                while (!mbar_try_wait(bar(B_OFULL), 0) && ++spins < kSpinLimit) {
                }
            }
        }
    } else {
        // ------------------------------------------------------------ softmax
        const int grp = (warp - kA2Producers / 32 - 1) >> 2;  // query tile 0 or 1
        const uint32_t quarter = (uint32_t)(warp & 3);
        const uint32_t r = quarter * 32u + (uint32_t)lane;    // row in the tile == TMEM lane
        const uint32_t lane_off = (quarter * 32u) << 16;
        const uint32_t tS = tmem + (grp ? 128u : 0u), tO = tmem + 256u + (grp ? (uint32_t)D : 0u);
        float m_used = -INFINITY, l = 0.0f;
        bool ok = true;
        for (int j = 0; j < ntiles; ++j) {
            ok = __all_sync(0xffffffffu, a2_wait(bar(grp ? B_SFULL1 : B_SFULL0), (uint32_t)(j & 1), abort_flag));
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
            // lazy rescale: keep the stale maximum while exp2 stays below 2^8
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
            // P = exp2(s * scale - m_used), fp16 pairs, back into the first 64
            // columns of S_i: the A operand of P V, read from TMEM
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
            mbar_arrive(bar(grp ? B_PFULL1 : B_PFULL0));
        }
        // epilogue
        const int64_t qr = q0 + grp * 128 + r;
        const bool have =
            __all_sync(0xffffffffu, ntiles > 0 && ok && a2_wait(bar(B_OFULL), 0, abort_flag));
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

    __syncwarp();  // the MMA lane rejoins its warp before the block barrier
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0)
        tmem_dealloc(tmem, 512);
}

}  // namespace kvq

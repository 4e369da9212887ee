// fast.cuh -- NanoKV-Fast's query reduction and output restoration around the
// low-dimensional history attention (NanoKV page, Fig. 4(d): the queries are
// reduced into a head's low space, attention runs there over keys and values
// decoded straight into that space, and the outputs are restored to the head
// dimension before the LSE merge; per-head low dims, Table 6).
//
// Both maps are small per-head matrices applied to every query row: the
// reduction q_low = q_h P_h ([d] x [d][d_low]) and the restoration
// o_h = o_low R_h ([d_low] x [d_low][d]).  Each is d d_low MACs per row, under
// 1% of the attention's 2 T d_low per row, so they run on CUDA cores: one
// thread per query row of one head, the map resident in shared memory as
// binary32 (read by every thread at the same address: broadcasts), the row
// streamed from global memory in 16-byte pieces.
//
// The reduced query is rounded to bf16 once from the exact sum: every
// bf16 x bf16 product is exact in binary64 and the sum of d of them stays
// exact there unless their magnitudes span more than about 2^30, so the
// reduction accumulates in binary64 (32 outputs per pass) and converts by
// round-to-odd to binary32 followed by round-to-nearest-even to bf16, which
// is the correctly rounded result (the binary32 step keeps 16 extra bits;
// Boldo and Melquiond, "Emulation of FMA and correctly rounded sums: proved
// algorithms using rounding to odd", IEEE Trans. Computers 57(4), 2008).  An
// FMA chain in binary32 would flip the bf16 rounding of a fair share of
// values near a rounding boundary.  The restoration keeps binary32 (64
// outputs per pass, FMA chains in input-channel order).
#pragma once

#include "common.cuh"

namespace kvq {

constexpr int kFastThreads = 128;

struct FastMapArgs {
    const void *in;   // [Tq][H][DIN]: bf16 (reduction) or float (restoration)
    const uint16_t *map;  // [H][DIN][DOUT] bf16
    void *out;        // [Tq][H][DOUT]: bf16 (reduction), float or bf16 (restoration)
    int64_t Tq;
    int H;
    int out_bf16;
};

// Eight input values of a row from 16 (bf16) or 32 (float) bytes.
template <bool IN_BF16>
__device__ __forceinline__ void fast_load8(const void *row, int c, float *v)
{
    if (IN_BF16) {
        const uint4 w = __ldg(reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(row) + c));
        const uint32_t a[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            v[2 * k] = __uint_as_float(a[k] << 16);
            v[2 * k + 1] = __uint_as_float(a[k] & 0xffff0000u);
        }
    } else {
        const float4 *p = reinterpret_cast<const float4 *>(static_cast<const float *>(row) + c);
        const float4 x = __ldg(p), y = __ldg(p + 1);
        v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
        v[4] = y.x; v[5] = y.y; v[6] = y.z; v[7] = y.w;
    }
}

// binary64 -> bf16, correctly rounded: round-to-odd into binary32, then
// round-to-nearest-even.
__device__ __forceinline__ float round_odd_f32(double v)
{
    const float f = __double2float_rz(v);
    return ((double)f == v) ? f : __uint_as_float(__float_as_uint(f) | 1u);
}

// out[t][h][:] = in[t][h][:] M_h for one block of 128 rows of head blockIdx.y.
// Dynamic shared memory: M_h as binary32 [DIN][DOUT].  IN_BF16 selects the
// reduction (bf16 rows, binary64 sums, bf16 out), else the restoration.
template <int DIN, int DOUT, bool IN_BF16>
__global__ void __launch_bounds__(kFastThreads) fast_map_kernel(FastMapArgs a)
{
    extern __shared__ __align__(16) float sM[];
    const int h = blockIdx.y;
    const uint16_t *m = a.map + (int64_t)h * DIN * DOUT;
    for (int e = threadIdx.x * 8; e < DIN * DOUT; e += kFastThreads * 8) {
        const uint4 w = __ldg(reinterpret_cast<const uint4 *>(m + e));
        const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            sM[e + 2 * k] = __uint_as_float(u[k] << 16);
            sM[e + 2 * k + 1] = __uint_as_float(u[k] & 0xffff0000u);
        }
    }
    __syncthreads();
    const int64_t t = (int64_t)blockIdx.x * kFastThreads + threadIdx.x;
    if (t >= a.Tq)
        return;
    const int64_t row = t * a.H + h;
    const void *in_row = IN_BF16 ? static_cast<const void *>(static_cast<const uint16_t *>(a.in) + row * DIN)
                                 : static_cast<const void *>(static_cast<const float *>(a.in) + row * DIN);
    if constexpr (IN_BF16) {
#pragma unroll 1
        for (int o0 = 0; o0 < DOUT; o0 += 32) {
            double acc[32];
#pragma unroll
            for (int j = 0; j < 32; ++j)
                acc[j] = 0.0;
#pragma unroll 1
            for (int c = 0; c < DIN; c += 8) {
                float x[8];
                fast_load8<true>(in_row, c, x);
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const float4 *mr = reinterpret_cast<const float4 *>(sM + (c + k) * DOUT + o0);
                    const double xk = (double)x[k];
#pragma unroll
                    for (int j4 = 0; j4 < 8; ++j4) {
                        const float4 mv = mr[j4];
                        acc[4 * j4 + 0] = fma(xk, (double)mv.x, acc[4 * j4 + 0]);
                        acc[4 * j4 + 1] = fma(xk, (double)mv.y, acc[4 * j4 + 1]);
                        acc[4 * j4 + 2] = fma(xk, (double)mv.z, acc[4 * j4 + 2]);
                        acc[4 * j4 + 3] = fma(xk, (double)mv.w, acc[4 * j4 + 3]);
                    }
                }
            }
            uint4 *dst = reinterpret_cast<uint4 *>(static_cast<uint16_t *>(a.out) + row * DOUT + o0);
#pragma unroll
            for (int j8 = 0; j8 < 4; ++j8)
                dst[j8] = make_uint4(pack_bf16x2(round_odd_f32(acc[8 * j8 + 0]), round_odd_f32(acc[8 * j8 + 1])),
                                     pack_bf16x2(round_odd_f32(acc[8 * j8 + 2]), round_odd_f32(acc[8 * j8 + 3])),
                                     pack_bf16x2(round_odd_f32(acc[8 * j8 + 4]), round_odd_f32(acc[8 * j8 + 5])),
                                     pack_bf16x2(round_odd_f32(acc[8 * j8 + 6]), round_odd_f32(acc[8 * j8 + 7])));
        }
    } else {
#pragma unroll 1
    for (int o0 = 0; o0 < DOUT; o0 += 64) {
        float acc[64];
#pragma unroll
        for (int j = 0; j < 64; ++j)
            acc[j] = 0.0f;
#pragma unroll 1
        for (int c = 0; c < DIN; c += 8) {
            float x[8];
            fast_load8<false>(in_row, c, x);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const float4 *mr = reinterpret_cast<const float4 *>(sM + (c + k) * DOUT + o0);
#pragma unroll
                for (int j4 = 0; j4 < 16; ++j4) {
                    const float4 mv = mr[j4];
                    acc[4 * j4 + 0] = fmaf(x[k], mv.x, acc[4 * j4 + 0]);
                    acc[4 * j4 + 1] = fmaf(x[k], mv.y, acc[4 * j4 + 1]);
                    acc[4 * j4 + 2] = fmaf(x[k], mv.z, acc[4 * j4 + 2]);
                    acc[4 * j4 + 3] = fmaf(x[k], mv.w, acc[4 * j4 + 3]);
                }
            }
        }
        if (a.out_bf16) {
            uint4 *dst = reinterpret_cast<uint4 *>(static_cast<uint16_t *>(a.out) + row * DOUT + o0);
#pragma unroll
            for (int j8 = 0; j8 < 8; ++j8)
                dst[j8] = make_uint4(pack_bf16x2(acc[8 * j8 + 0], acc[8 * j8 + 1]),
                                     pack_bf16x2(acc[8 * j8 + 2], acc[8 * j8 + 3]),
                                     pack_bf16x2(acc[8 * j8 + 4], acc[8 * j8 + 5]),
                                     pack_bf16x2(acc[8 * j8 + 6], acc[8 * j8 + 7]));
        } else {
            float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(a.out) + row * DOUT + o0);
#pragma unroll
            for (int j4 = 0; j4 < 16; ++j4)
                dst[j4] = make_float4(acc[4 * j4], acc[4 * j4 + 1], acc[4 * j4 + 2], acc[4 * j4 + 3]);
        }
    }
    }
}

}  // namespace kvq

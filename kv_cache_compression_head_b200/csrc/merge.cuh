// merge.cuh -- log-sum-exp merging of partial attention results over
// disjoint history parts (NanoKV page, Fig. 4(d): output dimensions are
// restored before the LSE merge of the history parts).
//
//   m = max_b lse_b;  lse = m + ln sum_b exp(lse_b - m);
//   o = sum_b exp(lse_b - lse) * o_b;  parts with lse_b = -inf weigh 0.
#pragma once

#include "common.cuh"

namespace kvq {

constexpr int kMaxMergeParts = 64;

struct MergeArgs {
    const float *o[kMaxMergeParts];
    const float *lse[kMaxMergeParts];
    int n;
    int64_t Tq;
    int H;
    int D;
    void *o_out;
    int o_bf16;
    float *lse_out;
};

// One block per (tile of 256 / (D/4) queries, head); thread = 4 channels of
// one (query, head) row.  Every thread of a row recomputes the row's weights
// (n exps), which keeps the kernel a single pass over the o_b reads and the
// output write.
template <int D>
__global__ void __launch_bounds__(256) lse_merge_kernel(MergeArgs a)
{
    constexpr int kUnits = D / 4;
    constexpr int kRows = 256 / kUnits;
    const int u = threadIdx.x % kUnits;
    const int64_t t = (int64_t)blockIdx.x * kRows + threadIdx.x / kUnits;
    const int h = blockIdx.y;
    if (t >= a.Tq)
        return;
    const int64_t row = t * a.H + h;
    const int64_t li = (int64_t)h * a.Tq + t;

    float m = -INFINITY;
    for (int b = 0; b < a.n; ++b)
        m = fmaxf(m, a.lse[b][li]);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float lse = -INFINITY;
    if (m != -INFINITY) {
        float tot = 0.0f;
        for (int b = 0; b < a.n; ++b) {
            const float l = a.lse[b][li];
            if (l != -INFINITY)
                tot += expf(l - m);
        }
        lse = m + logf(tot);
        for (int b = 0; b < a.n; ++b) {
            const float l = a.lse[b][li];
            if (l == -INFINITY)
                continue;
            const float w = expf(l - lse);
            const float4 v = *reinterpret_cast<const float4 *>(a.o[b] + row * D + u * 4);
            acc.x = fmaf(w, v.x, acc.x);
            acc.y = fmaf(w, v.y, acc.y);
            acc.z = fmaf(w, v.z, acc.z);
            acc.w = fmaf(w, v.w, acc.w);
        }
    }
    if (a.o_bf16) {
        uint2 w = make_uint2(pack_bf16x2(acc.x, acc.y), pack_bf16x2(acc.z, acc.w));
        *reinterpret_cast<uint2 *>(static_cast<uint16_t *>(a.o_out) + row * D + u * 4) = w;
    } else {
        *reinterpret_cast<float4 *>(static_cast<float *>(a.o_out) + row * D + u * 4) = acc;
    }
    if (u == 0)
        a.lse_out[li] = lse;
}

}  // namespace kvq

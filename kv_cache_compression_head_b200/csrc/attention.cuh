// attention.cuh -- argument structures shared by the attention kernels
// (attention2.cuh: single-CTA, attention_pair.cuh: CTA pairs).
//
// A compressed K or V history is read through CodecView: idx, packed codes,
// {s, z} pairs and the bf16 centres, from which the kernels rebuild
// k^ = mu[idx] + (q - z) s on the fly (NanoKV page, Fig. 4(a,b); QuantWM,
// Fig. 9: on-demand reconstruction).  In dense mode the same kernels read
// uncompressed bf16 keys and values instead: the current chunk and the raw
// protected tokens (sinks, recent window) whose partial result is merged with
// the compressed history's by LSE (NanoKV page, Fig. 4(d) and Table 4).
#pragma once

#include "codec.cuh"
#include "common.cuh"

namespace kvq {

struct CodecView {
    const uint16_t *cent;  // [H][C][D] bf16
    const uint16_t *idx;   // [H][T]
    const uint8_t *codes;  // [H][T][D*bits/8]
    const void *meta;      // [H][T][D/G][2] float, or binary16 when meta16
    int64_t T;
    int C;
    int bits;
    int G;
    int meta16;
};

struct AttnArgs {
    const uint16_t *q;  // [Tq][H][D] bf16
    int64_t Tq;
    int H;
    CodecView k, v;
    const uint16_t *k_dense;  // dense mode: keys [Tk][H][D] bf16 (k, v unused)
    const uint16_t *v_dense;  // dense mode: values [Tk][H][D] bf16
    int dense;
    int64_t t_begin, t_end;
    float scale_log2;  // softmax scale * log2(e)
    void *o_out;
    int o_bf16;
    float *lse_out;  // [H][Tq]
    int nsplit;      // > 1: blockIdx.z selects a sub-range; o_out / lse_out
                     // then hold nsplit float partials [z][Tq][H][D], [z][H][Tq]
    const float *psac_u;     // PSAC: basis [H][D][8] (NULL: no correction)
    const float *psac_coef;  // PSAC: coefficients [H][T][8] of the K history
};

}  // namespace kvq

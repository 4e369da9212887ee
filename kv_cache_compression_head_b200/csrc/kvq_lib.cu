// kvq_lib.cu -- the C ABI of libkvq (declared in include/kvq.h): argument
// validation, workspace accounting and kernel launches.  Built as a single
// translation unit for sm_100a.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <math.h>

#include <atomic>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "attention.cuh"
#include "attention2.cuh"
#include "attention_pair.cuh"
#include "attention_tma.cuh"
#include "codec.cuh"
#include "common.cuh"
#include "encode_filter.cuh"
#include "fast.cuh"
#include "joint.cuh"
#include "merge.cuh"

using namespace kvq;

namespace {

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

bool supported_dim(int d) { return d == 64 || d == 128; }

// Shared checks of a per-head codec description.
kvq_status check_desc(const kvq_codec_desc *d, bool allow_joint)
{
    if (!d)
        return KVQ_ERR_INVALID_ARG;
    if (d->num_heads < 1 || d->num_centroids < 1 || d->num_centroids > 65536)
        return KVQ_ERR_INVALID_ARG;
    if (!supported_dim(d->head_dim))
        return KVQ_ERR_UNSUPPORTED;
    if (d->bits != 2 && d->bits != 4)
        return KVQ_ERR_UNSUPPORTED;
    if (d->joint_rank < 0)
        return KVQ_ERR_INVALID_ARG;
    if (d->joint_rank > 0 && !allow_joint)
        return KVQ_ERR_UNSUPPORTED;
    if (d->meta_format != KVQ_META_F32 && d->meta_format != KVQ_META_F16)
        return KVQ_ERR_INVALID_ARG;
    if (d->meta_format == KVQ_META_F16 && d->joint_rank > 0)
        return KVQ_ERR_UNSUPPORTED;  // compact {s, z} is a per-head codec format
    if (d->residual_stages < 0)
        return KVQ_ERR_INVALID_ARG;
    if (d->residual_stages > 2 ||
        (d->residual_stages == 2 && (d->joint_rank > 0 || d->meta_format != KVQ_META_F32)))
        return KVQ_ERR_UNSUPPORTED;
    const int span = d->joint_rank > 0 ? d->joint_rank : d->head_dim;
    if (d->group_size < 8 || d->group_size % 8 != 0 || span % d->group_size != 0)
        return KVQ_ERR_INVALID_ARG;
    if (d->group_size != 16 && d->group_size != 32 && d->group_size != 64)
        return KVQ_ERR_UNSUPPORTED;
    // joint code: rank a multiple of 64 up to 256 (one MMA N extent)
    if (d->joint_rank > 0 && (d->joint_rank % 64 != 0 || d->joint_rank > 256))
        return KVQ_ERR_UNSUPPORTED;
    return KVQ_OK;
}

// A failed launch is reported as KVQ_ERR_CUDA; with KVQ_DEBUG set in the
// environment the CUDA error string is also printed to stderr.
kvq_status launch_status()
{
    const cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess)
        return KVQ_OK;
    if (getenv("KVQ_DEBUG"))
        fprintf(stderr, "libkvq: CUDA error %d: %s\n", (int)e, cudaGetErrorString(e));
    return KVQ_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// per-head encode dispatch
// ---------------------------------------------------------------------------
template <int D, int BITS>
kvq_status launch_encode_direct_g(const EncodeArgs &a, cudaStream_t s)
{
    const dim3 grid((unsigned)ceil_div(a.T, kDirectTokens), (unsigned)a.H);
    switch (a.G) {
    case 16: encode_direct_kernel<D, BITS, 16><<<grid, kDirectTokens, 0, s>>>(a); break;
    case 32: encode_direct_kernel<D, BITS, 32><<<grid, kDirectTokens, 0, s>>>(a); break;
    case 64: encode_direct_kernel<D, BITS, 64><<<grid, kDirectTokens, 0, s>>>(a); break;
    default: return KVQ_ERR_UNSUPPORTED;
    }
    return launch_status();
}

kvq_status launch_encode_direct(int D, const EncodeArgs &a, cudaStream_t s)
{
    if (a.T == 0)
        return KVQ_OK;
    if (D == 128)
        return a.bits == 2 ? launch_encode_direct_g<128, 2>(a, s) : launch_encode_direct_g<128, 4>(a, s);
    return a.bits == 2 ? launch_encode_direct_g<64, 2>(a, s) : launch_encode_direct_g<64, 4>(a, s);
}

// ---------------------------------------------------------------------------
// tensor-core filtered encode (bf16 history, C <= 512, G <= d/2)
// ---------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// 3-D map of a [T][H][D] bf16 history: box = 64 channels x 1 head x 128 tokens,
// 128-byte swizzle (the K-major operand layout), zero fill past T.
bool make_history_map(CUtensorMap *m, const void *x, int64_t T, int H, int D)
{
    PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (!enc)
        return false;
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)T};
    cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2};
    cuuint32_t box[3] = {64, 1, (cuuint32_t)kFltRows};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(x), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int sm_count()
{
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n;
}

bool filter_applies(int D, int C, int G, bool x_bf16)
{
    return x_bf16 && C <= kFltMaxC && G <= D / 2 && (D == 64 || D == 128);
}

// X stages that fit beside the centres (2 .. kFltMaxStages).
int filter_stages(int D, int Cpad)
{
    const uint32_t budget = 227u * 1024u - 1024u;
    const uint32_t fixed = flt_smem_bytes(D, Cpad, 0);
    const int fit = fixed < budget ? (int)((budget - fixed) / flt_tile_bytes(D)) : 0;
    return fit < 2 ? 2 : (fit > kFltMaxStages ? kFltMaxStages : fit);
}

template <int D, int BITS, int G, bool TWO>
kvq_status launch_filter_t(const CUtensorMap &m, const FilterArgs &a, cudaStream_t s)
{
    const uint32_t smem = flt_smem_bytes(D, a.Cpad, a.stages) + 1024;
    static std::atomic<bool> configured[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return KVQ_ERR_CUDA;
    if (!configured[dev].load()) {
        if (cudaFuncSetAttribute(encode_filter_kernel<D, BITS, G, TWO>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 227 * 1024) != cudaSuccess)
            return KVQ_ERR_CUDA;
        configured[dev].store(true);
    }
    // persistent: one CTA per SM (the two 256-column accumulators take all of
    // TMEM), each with an equal contiguous share of the (head, tile) units
    const int64_t units = (int64_t)a.H * a.ntiles;
    const int64_t sms = sm_count();
    const unsigned grid = (unsigned)(units < sms ? units : sms);
    encode_filter_kernel<D, BITS, G, TWO><<<grid, kFltThreads, smem, s>>>(m, a);
    return launch_status();
}

template <int D, int BITS>
kvq_status launch_filter_g(int G, const CUtensorMap &m, const FilterArgs &a, cudaStream_t s)
{
    switch (G) {
    case 16: return a.codes2 ? launch_filter_t<D, BITS, 16, true>(m, a, s) : launch_filter_t<D, BITS, 16, false>(m, a, s);
    case 32: return a.codes2 ? launch_filter_t<D, BITS, 32, true>(m, a, s) : launch_filter_t<D, BITS, 32, false>(m, a, s);
    case 64:
        if constexpr (D >= 128)
            return a.codes2 ? launch_filter_t<D, BITS, 64, true>(m, a, s) : launch_filter_t<D, BITS, 64, false>(m, a, s);
        return KVQ_ERR_UNSUPPORTED;
    default: return KVQ_ERR_UNSUPPORTED;
    }
}

// k of the certified candidate set (see encode_filter.cuh), with R_j =
// |x| + |mu_j| and u = 2^-24:
//  - every computed L'_j is within rho R_j^2 of its exact value, rho =
//    gamma_d (the binary32 centre norm) + eps_tc / 2 (the tensor-core dot
//    product, eps_tc = d 2^-21 relative to sum |x_c mu_c| <= |x||mu_j| <=
//    R_j^2 / 4, taken twice) + 129 u (the roundings of A_j, of the two FMAs
//    and of |x|, and the <= 31 ulp of the column index carried in L');
//  - the specified distance is within gamma_{d+3} R_j^2 of the exact one.
// k >= rho + gamma_{d+3} suffices; the factor 1.25 and 2^-20 cover the
// relative error of the threshold's own (|x| + |mu|)^2.
float filter_kappa(int D)
{
    const double u = ldexp(1.0, -24);
    const double eps_tc = D * ldexp(1.0, -21);
    auto gamma = [&](int n) { return n * u / (1.0 - n * u); };
    const double rho = gamma(D) + eps_tc / 2.0 + 129.0 * u;
    return (float)(1.25 * (rho + gamma(D + 3)) + ldexp(1.0, -20));
}

kvq_status launch_encode_filter(int D, int bits, int G, const void *x, const EncodeArgs &e, cudaStream_t s)
{
    CUtensorMap m;
    if (!make_history_map(&m, x, e.T, e.H, D))
        return KVQ_ERR_CUDA;
    FilterArgs a;
    a.T = e.T;
    a.H = e.H;
    a.C = e.C;
    a.Cpad = (e.C + 31) / 32 * 32;
    a.stages = filter_stages(D, a.Cpad);
    a.ntiles = (e.T + kFltRows - 1) / kFltRows;
    a.cent = e.cent;
    a.idx = e.idx;
    a.codes = e.codes;
    a.meta = e.meta;
    a.assign_only = e.assign_only;
    a.meta16 = e.meta16;
    a.kappa = filter_kappa(D);
    a.codes2 = e.codes2;
    a.meta2 = e.meta2;
    if (D == 128)
        return bits == 2 ? launch_filter_g<128, 2>(G, m, a, s) : launch_filter_g<128, 4>(G, m, a, s);
    return bits == 2 ? launch_filter_g<64, 2>(G, m, a, s) : launch_filter_g<64, 4>(G, m, a, s);
}

// Assignment (+ residual quantisation unless assign_only): the filtered
// tensor-core kernel where it applies, else the exact CUDA-core kernel.  Both
// produce identical results.
kvq_status launch_encode(int D, const EncodeArgs &e, cudaStream_t s)
{
    if (e.T == 0)
        return KVQ_OK;
    if (filter_applies(D, e.C, e.G, e.x_bf16 != 0))
        return launch_encode_filter(D, e.bits, e.G, e.x, e, s);
    return launch_encode_direct(D, e, s);
}

// ---------------------------------------------------------------------------
// joint head-channel code
// ---------------------------------------------------------------------------
template <int G, int BITS>
kvq_status launch_joint_encode_t(const JointEncArgs &a, cudaStream_t s)
{
    const uint32_t smem = joint_enc_smem_bytes(a.r) + 1024;
    static bool configured[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return KVQ_ERR_CUDA;
    if (!configured[dev]) {
        if (cudaFuncSetAttribute(joint_encode_kernel<G, BITS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)(joint_enc_smem_bytes(256) + 1024)) != cudaSuccess)
            return KVQ_ERR_CUDA;
        configured[dev] = true;
    }
    CUtensorMap mx, mw;
    if (!make_history_map(&mx, a.x, a.T, a.H, a.D))
        return KVQ_ERR_CUDA;
    PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (!enc)
        return KVQ_ERR_CUDA;
    // W_enc [H d][r] bf16: box = 64 coefficients x 64 rows, 128-byte swizzle
    // (the MN-major B layout of the encoder's MMA)
    cuuint64_t dims[2] = {(cuuint64_t)a.r, (cuuint64_t)a.H * a.D};
    cuuint64_t strides[1] = {(cuuint64_t)a.r * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)kJKBlock};
    cuuint32_t estr[2] = {1, 1};
    if (enc(&mw, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t *>(a.w), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return KVQ_ERR_CUDA;
    joint_encode_kernel<G, BITS><<<(unsigned)ceil_div(a.T, kJRows), kJEThreads, smem, s>>>(mx, mw, a);
    return launch_status();
}

kvq_status launch_joint_encode(const JointEncArgs &a, cudaStream_t s)
{
    if (a.T == 0)
        return KVQ_OK;
    switch (a.G * 8 + a.bits) {
    case 16 * 8 + 2: return launch_joint_encode_t<16, 2>(a, s);
    case 16 * 8 + 4: return launch_joint_encode_t<16, 4>(a, s);
    case 32 * 8 + 2: return launch_joint_encode_t<32, 2>(a, s);
    case 32 * 8 + 4: return launch_joint_encode_t<32, 4>(a, s);
    case 64 * 8 + 2: return launch_joint_encode_t<64, 2>(a, s);
    case 64 * 8 + 4: return launch_joint_encode_t<64, 4>(a, s);
    default: return KVQ_ERR_UNSUPPORTED;
    }
}

// 2-D map of W_dec [r][H*D] bf16: box = 64 output channels x r rows,
// 128-byte swizzle (the MN-major B layout of the decoder's MMA).
bool make_wdec_map(CUtensorMap *m, const void *w, int r, int HD)
{
    PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (!enc)
        return false;
    cuuint64_t dims[2] = {(cuuint64_t)HD, (cuuint64_t)r};
    cuuint64_t strides[1] = {(cuuint64_t)HD * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)r};
    cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(w), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

kvq_status launch_joint_decode(const JointDecArgs &a, const void *w_dec, cudaStream_t s)
{
    if (a.T == 0)
        return KVQ_OK;
    static bool configured[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return KVQ_ERR_CUDA;
    if (!configured[dev]) {
        if (cudaFuncSetAttribute(joint_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)(kJDSmemLimit + 1024)) != cudaSuccess)
            return KVQ_ERR_CUDA;
        configured[dev] = true;
    }
    CUtensorMap m;
    if (!make_wdec_map(&m, w_dec, a.r, a.H * a.D))
        return KVQ_ERR_CUDA;
    const JDLayout L(a.r, a.D);
    joint_decode_kernel<<<(unsigned)ceil_div(a.T, kJRows), kJDThreads, L.total + 1024, s>>>(m, a);
    return launch_status();
}

// Validates and runs the joint encoder: per-head assignment into idx, then the
// projection + quantisation (codes/meta) and/or the binary32 coefficients.
kvq_status joint_encode_call(const kvq_codec_desc *desc, const void *x, kvq_dtype x_dtype, int64_t T,
                             const void *centroids, const void *w_enc, uint16_t *idx, uint8_t *codes, void *meta,
                             float *coef_out, cudaStream_t s)
{
    if (x_dtype != KVQ_BF16)
        return KVQ_ERR_UNSUPPORTED;  // the joint residual is formed from a bf16 history
    if (T < 0)
        return KVQ_ERR_INVALID_ARG;
    if (T == 0)
        return KVQ_OK;
    if (!x || !centroids || !w_enc || !idx || (!coef_out && (!codes || !meta)))
        return KVQ_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(centroids) || !aligned16(w_enc) || (codes && !aligned16(codes)) ||
        (meta && !aligned16(meta)) || (coef_out && !aligned16(coef_out)) || (reinterpret_cast<uintptr_t>(idx) & 1u))
        return KVQ_ERR_ALIGNMENT;
    EncodeArgs e;
    memset(&e, 0, sizeof e);
    e.x = x;
    e.x_bf16 = 1;
    e.T = T;
    e.H = desc->num_heads;
    e.C = desc->num_centroids;
    e.bits = 2;
    e.G = 16;
    e.cent = static_cast<const uint16_t *>(centroids);
    e.idx = idx;
    e.assign_only = 1;
    kvq_status st = launch_encode(desc->head_dim, e, s);
    if (st != KVQ_OK)
        return st;
    JointEncArgs a;
    a.x = static_cast<const uint16_t *>(x);
    a.cent = e.cent;
    a.idx = idx;
    a.w = static_cast<const uint16_t *>(w_enc);
    a.T = T;
    a.H = desc->num_heads;
    a.D = desc->head_dim;
    a.C = desc->num_centroids;
    a.r = desc->joint_rank;
    a.bits = desc->bits;
    a.G = desc->group_size;
    a.codes = codes;
    a.meta = static_cast<float *>(meta);
    a.coef_out = coef_out;
    return launch_joint_encode(a, s);
}

// Fit workspace: idx [H][T] u16 | per-chunk centre counts [H][nch][C] i32 |
// bucket starts [H][C+1] i32 | token order [H][T] i32.
struct FitLayout {
    size_t idx, counts, starts, order, order_j, sums, bounds, redo, bkt, total;
    int nchunks;
};

FitLayout fit_layout(const kvq_codec_desc *d, int64_t T)
{
    FitLayout L;
    const size_t H = (size_t)d->num_heads, C = (size_t)d->num_centroids;
    L.nchunks = (int)((T + kFitChunk - 1) / kFitChunk);
    if (L.nchunks < 1)
        L.nchunks = 1;
    L.idx = 0;
    L.counts = round_up(H * (size_t)T * 2, 256);
    L.starts = L.counts + round_up(H * (size_t)L.nchunks * C * 4, 256);
    L.order = L.starts + round_up(H * (C + 1) * 4, 256);
    L.order_j = L.order + round_up(H * (size_t)T * 4, 256);
    L.sums = L.order_j + round_up(H * (size_t)T * 2, 256);
    L.bounds = L.sums + round_up(H * C * (size_t)d->head_dim * 8, 256);
    L.redo = L.bounds + round_up(H * 8, 256);
    L.bkt = L.redo + round_up(H * C * 4, 256);
    L.total = L.bkt + H * C * 8;
    return L;
}

size_t fit_workspace(const kvq_codec_desc *d, int64_t T) { return fit_layout(d, T).total; }

// Largest centre count the fit's shared-memory histograms take.
constexpr int kFitMaxC = 32768;

template <typename K>
kvq_status smem_opt_in(K kernel, size_t bytes)
{
    if (bytes <= 48 * 1024)
        return KVQ_OK;
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) == cudaSuccess
               ? KVQ_OK
               : KVQ_ERR_CUDA;
}

kvq_status check_view(const kvq_compressed_view *v)
{
    if (!v)
        return KVQ_ERR_INVALID_ARG;
    kvq_status st = check_desc(&v->desc, true);
    if (st != KVQ_OK)
        return st;
    if (v->num_tokens < 0)
        return KVQ_ERR_INVALID_ARG;
    if (v->num_tokens > 0 && (!v->centroids || !v->idx || !v->codes || !v->meta))
        return KVQ_ERR_INVALID_ARG;
    if (!aligned16(v->centroids) || !aligned16(v->codes) || !aligned16(v->meta) ||
        (reinterpret_cast<uintptr_t>(v->idx) & 1u))
        return KVQ_ERR_ALIGNMENT;
    return KVQ_OK;
}

CodecView to_codec_view(const kvq_compressed_view *v)
{
    CodecView cv;
    cv.cent = static_cast<const uint16_t *>(v->centroids);
    cv.idx = v->idx;
    cv.codes = v->codes;
    cv.meta = v->meta;
    cv.meta16 = v->desc.meta_format == KVQ_META_F16;
    cv.T = v->num_tokens;
    cv.C = v->desc.num_centroids;
    cv.bits = v->desc.bits;
    cv.G = v->desc.group_size;
    return cv;
}

constexpr int kMaxAttnSplit = 4;

// Partial-result buffers for `slots` binary32 partials: O slices
// [slot][Tq][H][d], then (256-byte aligned) lse slices [slot][H][Tq].
size_t partials_bytes(int slots, int H, int d, int64_t Tq)
{
    const size_t o = (size_t)slots * (size_t)Tq * H * d * 4;
    return round_up(o, 256) + (size_t)slots * H * (size_t)Tq * 4;
}

size_t attention_workspace(const kvq_codec_desc *d, int64_t Tq)
{
    return partials_bytes(kMaxAttnSplit, d->num_heads, d->head_dim, Tq);
}

// Full-layer attention: up to kMaxAttnSplit partials for the compressed
// history and as many for the dense keys.
size_t layer_workspace(const kvq_codec_desc *d, int64_t Tq)
{
    return partials_bytes(2 * kMaxAttnSplit, d->num_heads, d->head_dim, Tq);
}

// Number of history sub-ranges for one attention call: the CTA count
// (query-tile pairs x heads x splits) should fill whole waves of one CTA per
// SM, and every sub-range should keep at least 8 history tiles.
int attention_splits(int64_t Tq, int H, int64_t span, size_t ws_bytes, size_t ws_need, int rows_per_unit,
                     int ctas_per_unit)
{
    if (ws_bytes < ws_need)
        return 1;
    const int64_t base = ((Tq + rows_per_unit - 1) / rows_per_unit) * ctas_per_unit * H;
    const int64_t sms = sm_count();
    const int64_t tiles = (span + 127) / 128;
    int best = 1;
    double best_eff = (double)base / (double)(((base + sms - 1) / sms) * sms);
    for (int k = 2; k <= kMaxAttnSplit; ++k) {
        if (tiles / k < 8)
            break;
        const int64_t n = base * k;
        const double eff = (double)n / (double)(((n + sms - 1) / sms) * sms);
        if (eff > best_eff + 0.02) {
            best = k;
            best_eff = eff;
        }
    }
    return best;
}

void launch_merge(const MergeArgs &m, cudaStream_t s)
{
    if (m.D == 128)
        lse_merge_kernel<128><<<dim3((unsigned)ceil_div(m.Tq, 256 / 32), (unsigned)m.H), 256, 0, s>>>(m);
    else
        lse_merge_kernel<64><<<dim3((unsigned)ceil_div(m.Tq, 256 / 16), (unsigned)m.H), 256, 0, s>>>(m);
}

template <int BK, int BV, bool DENSE>
kvq_status launch_attention_pair_t(const AttnArgs &a, cudaStream_t s)
{
    static bool configured[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return KVQ_ERR_CUDA;
    if (!configured[dev]) {
        if (cudaFuncSetAttribute(attention_pair_kernel<BK, BV, DENSE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)APSmem::kLaunchBytes) != cudaSuccess)
            return KVQ_ERR_CUDA;
        configured[dev] = true;
    }
    const dim3 grid((unsigned)(2 * ceil_div(a.Tq, kAPRowsPerPair)), (unsigned)a.H,
                    (unsigned)(a.nsplit > 1 ? a.nsplit : 1));
    attention_pair_kernel<BK, BV, DENSE><<<grid, kAPThreads, APSmem::kLaunchBytes, s>>>(a);
    return launch_status();
}

// 2-D tensor map over rows of `row_bytes` bytes (dims innermost first).
bool encode_2d(CUtensorMap *m, CUtensorMapDataType dt, const void *base, uint64_t inner, uint64_t rows,
               uint64_t row_bytes, uint32_t box_inner, uint32_t box_rows, CUtensorMapSwizzle sw)
{
    PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (!enc || !base)
        return false;
    cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
    cuuint32_t box[2] = {box_inner, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return enc(m, dt, 2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
               CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Tensor maps of a compressed K/V history for attention_tma_kernel (d = 128).
bool make_attn_maps(AttnMaps *m, const AttnArgs &a)
{
    const uint64_t rows = (uint64_t)a.H * (uint64_t)a.k.T;
    const CodecView &k = a.k, &v = a.v;
    const uint32_t vm_box = v.G == 64 ? 4u : (uint32_t)(64 / v.G) * 2u;
    // compact binary16 {s, z} is read by the loader lanes: no map
    memset(&m->km, 0, sizeof m->km);
    memset(&m->vm, 0, sizeof m->vm);
    memset(&m->kpc, 0, sizeof m->kpc);
    return encode_2d(&m->kc, CU_TENSOR_MAP_DATA_TYPE_UINT8, k.codes, 16u * k.bits, rows, 16u * k.bits,
                     16u * k.bits, 64, CU_TENSOR_MAP_SWIZZLE_NONE) &&
           (k.meta16 || encode_2d(&m->km, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, k.meta, 2u * (128 / k.G), rows,
                                  8u * (128 / k.G), 2u * (128 / k.G), 64, CU_TENSOR_MAP_SWIZZLE_NONE)) &&
           encode_2d(&m->vc, CU_TENSOR_MAP_DATA_TYPE_UINT8, v.codes, 16u * v.bits, rows, 16u * v.bits,
                     8u * v.bits, 128, CU_TENSOR_MAP_SWIZZLE_NONE) &&
           (v.meta16 || encode_2d(&m->vm, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, v.meta, 2u * (128 / v.G), rows,
                                  8u * (128 / v.G), vm_box, 128, CU_TENSOR_MAP_SWIZZLE_NONE)) &&
           encode_2d(&m->kcent, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, k.cent, 128, (uint64_t)a.H * k.C, 256, 64, 1,
                     CU_TENSOR_MAP_SWIZZLE_128B) &&
           encode_2d(&m->vcent, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, v.cent, 128, (uint64_t)a.H * v.C, 256, 64, 1,
                     CU_TENSOR_MAP_SWIZZLE_128B) &&
           (!a.psac_coef || encode_2d(&m->kpc, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, a.psac_coef, 8, rows, 32, 8, 64,
                                      CU_TENSOR_MAP_SWIZZLE_NONE));
}

template <int BK, int BV>
kvq_status launch_attention_tma_t(const AttnArgs &a, cudaStream_t s)
{
    static std::atomic<bool> configured[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return KVQ_ERR_CUDA;
    if (!configured[dev].load()) {
        if (cudaFuncSetAttribute(attention_tma_kernel<BK, BV>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)ATSmem::kLaunchBytes) != cudaSuccess)
            return KVQ_ERR_CUDA;
        configured[dev].store(true);
    }
    AttnMaps maps;
    if (!make_attn_maps(&maps, a))
        return KVQ_ERR_CUDA;
    const dim3 grid((unsigned)(2 * ceil_div(a.Tq, kAPRowsPerPair)), (unsigned)a.H,
                    (unsigned)(a.nsplit > 1 ? a.nsplit : 1));
    attention_tma_kernel<BK, BV><<<grid, kATThreads, ATSmem::kLaunchBytes, s>>>(maps, a);
    return launch_status();
}

// The compressed d = 128 history goes to the TMA-staged kernel when its row
// coordinates fit the 32-bit tensor-map coordinates and the range is not empty.
bool uses_tma_attention(const AttnArgs &a, int D)
{
    return D == 128 && !a.dense && a.t_end > a.t_begin && (int64_t)a.H * a.k.T < (int64_t)INT32_MAX &&
           (int64_t)a.H * (a.k.C > a.v.C ? a.k.C : a.v.C) < (int64_t)INT32_MAX;
}

kvq_status launch_attention_pair(const AttnArgs &a, cudaStream_t s)
{
    if (a.dense)
        return launch_attention_pair_t<0, 0, true>(a, s);
    // compressed history with keys to read: every byte staged by TMA (row
    // coordinates are 32-bit); an empty range needs no staging
    if (uses_tma_attention(a, 128)) {
        if (a.k.bits == 2)
            return a.v.bits == 2 ? launch_attention_tma_t<2, 2>(a, s) : launch_attention_tma_t<2, 4>(a, s);
        return a.v.bits == 2 ? launch_attention_tma_t<4, 2>(a, s) : launch_attention_tma_t<4, 4>(a, s);
    }
    if ((a.k.meta16 || a.v.meta16 || a.psac_coef) && a.t_end > a.t_begin)
        return KVQ_ERR_UNSUPPORTED;  // only the TMA-staged kernel reads compact {s, z} and PSAC terms
    if (a.k.bits == 2)
        return a.v.bits == 2 ? launch_attention_pair_t<2, 2, false>(a, s) : launch_attention_pair_t<2, 4, false>(a, s);
    return a.v.bits == 2 ? launch_attention_pair_t<4, 2, false>(a, s) : launch_attention_pair_t<4, 4, false>(a, s);
}

template <int D>
kvq_status launch_attention2(const AttnArgs &a, cudaStream_t s)
{
    using L = A2Smem<D>;
    static bool configured[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return KVQ_ERR_CUDA;
    if (!configured[dev]) {
        if (cudaFuncSetAttribute(attention2_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)L::kLaunchBytes) != cudaSuccess)
            return KVQ_ERR_CUDA;
        configured[dev] = true;
    }
    const dim3 grid((unsigned)ceil_div(a.Tq, kA2Rows), (unsigned)a.H, (unsigned)(a.nsplit > 1 ? a.nsplit : 1));
    attention2_kernel<D><<<grid, kA2Threads, L::kLaunchBytes, s>>>(a);
    return launch_status();
}


// d = 128 runs on CTA pairs (512 query rows per pair), d = 64 on single CTAs.
kvq_status launch_attention(const AttnArgs &a, int D, cudaStream_t s)
{
    return D == 128 ? launch_attention_pair(a, s) : launch_attention2<64>(a, s);
}

// Sub-ranges for one attention whose partials may go to a workspace.
int attention_split_for(const AttnArgs &a, int D, int64_t span)
{
    const bool pair = D == 128;
    return attention_splits(a.Tq, a.H, span, 1, 0, pair ? kAPRowsPerPair : kA2Rows, pair ? 2 : 1);
}

// Launch one attention with its key range split into `nsplit` sub-ranges,
// writing binary32 partials: O to o_part[z] = o_part + z Tq H D and lse to
// l_part + z H Tq, z < nsplit.
kvq_status launch_attention_partials(AttnArgs a, int D, int nsplit, float *o_part, float *l_part, cudaStream_t s)
{
    a.o_out = o_part;
    a.lse_out = l_part;
    a.o_bf16 = 0;
    a.nsplit = nsplit;
    return launch_attention(a, D, s);
}

// One attention call into o_out / lse_out: unsplit, or split into partials
// in the workspace and merged by LSE when that fills the GPU better.
kvq_status attention_call(const AttnArgs &a, int D, void *workspace, size_t workspace_bytes, cudaStream_t s)
{
    const size_t need = partials_bytes(kMaxAttnSplit, a.H, D, a.Tq);
    const int nsplit = (workspace && aligned16(workspace) && workspace_bytes >= need)
                           ? attention_split_for(a, D, a.t_end - a.t_begin)
                           : 1;
    if (nsplit == 1)
        return launch_attention(a, D, s);
    float *o_part = static_cast<float *>(workspace);
    float *l_part = reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) +
                                              round_up((size_t)kMaxAttnSplit * (size_t)a.Tq * a.H * D * 4, 256));
    kvq_status st = launch_attention_partials(a, D, nsplit, o_part, l_part, s);
    if (st != KVQ_OK)
        return st;
    MergeArgs m;
    memset(&m, 0, sizeof m);
    for (int z = 0; z < nsplit; ++z) {
        m.o[z] = o_part + (int64_t)z * a.Tq * a.H * D;
        m.lse[z] = l_part + (int64_t)z * a.H * a.Tq;
    }
    m.n = nsplit;
    m.Tq = a.Tq;
    m.H = a.H;
    m.D = D;
    m.o_out = a.o_out;
    m.o_bf16 = a.o_bf16;
    m.lse_out = a.lse_out;
    launch_merge(m, s);
    return launch_status();
}

// Checks shared by the compressed-history attention calls: two per-head
// views with the same H, d and length, and [t_begin, t_end) inside them.
kvq_status check_history_pair(const kvq_compressed_view *k, const kvq_compressed_view *v, int64_t t_begin,
                              int64_t t_end)
{
    kvq_status st;
    if ((st = check_view(k)) != KVQ_OK || (st = check_view(v)) != KVQ_OK)
        return st;
    if (k->desc.joint_rank > 0 || v->desc.joint_rank > 0)
        return KVQ_ERR_UNSUPPORTED;
    if (k->desc.residual_stages == 2 || v->desc.residual_stages == 2)
        return KVQ_ERR_UNSUPPORTED;  // two-stage histories: decode, then dense attention
    if (k->desc.num_heads != v->desc.num_heads || k->desc.head_dim != v->desc.head_dim ||
        k->num_tokens != v->num_tokens)
        return KVQ_ERR_INVALID_ARG;
    if (t_begin < 0 || t_end < t_begin || t_end > k->num_tokens)
        return KVQ_ERR_INVALID_ARG;
    if (k->desc.num_heads > 65535)
        return KVQ_ERR_UNSUPPORTED;
    if (k->desc.head_dim != 128 && (k->desc.meta_format == KVQ_META_F16 || v->desc.meta_format == KVQ_META_F16))
        return KVQ_ERR_UNSUPPORTED;  // compact {s, z} is read by the d = 128 kernel only
    return KVQ_OK;
}

AttnArgs attn_args(const void *q, int64_t Tq, int H, int D, int64_t t_begin, int64_t t_end, float softmax_scale,
                   void *o_out, kvq_dtype o_dtype, float *lse_out)
{
    AttnArgs a;
    memset(&a, 0, sizeof a);
    a.q = static_cast<const uint16_t *>(q);
    a.Tq = Tq;
    a.H = H;
    a.t_begin = t_begin;
    a.t_end = t_end;
    const float scale = softmax_scale > 0.0f ? softmax_scale : 1.0f / sqrtf((float)D);
    a.scale_log2 = scale * 1.4426950408889634f;
    a.o_out = o_out;
    a.o_bf16 = o_dtype == KVQ_BF16;
    a.lse_out = lse_out;
    a.nsplit = 1;
    return a;
}
}  // namespace

extern "C" {

const char *kvq_status_string(kvq_status s)
{
    switch (s) {
    case KVQ_OK: return "KVQ_OK";
    case KVQ_ERR_INVALID_ARG: return "KVQ_ERR_INVALID_ARG";
    case KVQ_ERR_UNSUPPORTED: return "KVQ_ERR_UNSUPPORTED";
    case KVQ_ERR_ALIGNMENT: return "KVQ_ERR_ALIGNMENT";
    case KVQ_ERR_WORKSPACE: return "KVQ_ERR_WORKSPACE";
    case KVQ_ERR_CUDA: return "KVQ_ERR_CUDA";
    case KVQ_ERR_DEVICE_TIMEOUT: return "KVQ_ERR_DEVICE_TIMEOUT";
    }
    return "KVQ_ERR_UNKNOWN";
}

kvq_status kvq_encoded_sizes(const kvq_codec_desc *desc, int64_t T, size_t *idx_bytes, size_t *code_bytes,
                             size_t *meta_bytes)
{
    kvq_status st = check_desc(desc, true);
    if (st != KVQ_OK)
        return st;
    if (T < 0)
        return KVQ_ERR_INVALID_ARG;
    const size_t H = (size_t)desc->num_heads, d = (size_t)desc->head_dim;
    size_t ib = H * (size_t)T * 2, cb, mb;
    if (desc->joint_rank > 0) {
        const size_t r = (size_t)desc->joint_rank;
        cb = (size_t)T * r * desc->bits / 8;
        mb = (size_t)T * (r / desc->group_size) * 8;
    } else {
        cb = H * (size_t)T * d * desc->bits / 8;
        mb = H * (size_t)T * (d / desc->group_size) * (desc->meta_format == KVQ_META_F16 ? 4 : 8);
    }
    if (idx_bytes) *idx_bytes = ib;
    if (code_bytes) *code_bytes = cb;
    if (meta_bytes) *meta_bytes = mb;
    return KVQ_OK;
}

kvq_status kvq_workspace_size(kvq_op op, const kvq_codec_desc *desc, int64_t T, int64_t Tq, size_t *bytes)
{
    if (!bytes)
        return KVQ_ERR_INVALID_ARG;
    kvq_status st = check_desc(desc, true);
    if (st != KVQ_OK)
        return st;
    if (T < 0 || Tq < 0)
        return KVQ_ERR_INVALID_ARG;
    switch (op) {
    case KVQ_OP_FIT: *bytes = fit_workspace(desc, T); return KVQ_OK;
    case KVQ_OP_ENCODE:
    case KVQ_OP_DECODE: *bytes = 0; return KVQ_OK;
    case KVQ_OP_ATTENTION: *bytes = attention_workspace(desc, Tq); return KVQ_OK;
    case KVQ_OP_LAYER_ATTENTION: *bytes = layer_workspace(desc, Tq); return KVQ_OK;
    }
    return KVQ_ERR_INVALID_ARG;
}

kvq_status kvq_fit_centroids(const kvq_codec_desc *desc, const void *x, kvq_dtype x_dtype, int64_t T, int32_t iters,
                             void *centroids_out, void *workspace, size_t workspace_bytes, kvq_stream_t stream)
{
    kvq_status st = check_desc(desc, true);
    if (st != KVQ_OK)
        return st;
    if (desc->joint_rank > 0)
        return KVQ_ERR_INVALID_ARG;  // centres are per head; fit with joint_rank = 0
    if (!x || !centroids_out || iters < 0 || T < desc->num_centroids || (x_dtype != KVQ_F32 && x_dtype != KVQ_BF16))
        return KVQ_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(centroids_out) || !aligned16(workspace))
        return KVQ_ERR_ALIGNMENT;
    if (desc->num_centroids > kFitMaxC)
        return KVQ_ERR_UNSUPPORTED;
    const FitLayout Lw = fit_layout(desc, T);
    if (!workspace || workspace_bytes < Lw.total)
        return KVQ_ERR_WORKSPACE;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int H = desc->num_heads, D = desc->head_dim, C = desc->num_centroids;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    FitArgs f;
    f.x = x;
    f.x_bf16 = x_dtype == KVQ_BF16;
    f.T = T;
    f.H = H;
    f.D = D;
    f.C = C;
    f.cent = static_cast<uint16_t *>(centroids_out);
    FitSortArgs fs;
    fs.x = x;
    fs.x_bf16 = f.x_bf16;
    fs.T = T;
    fs.H = H;
    fs.D = D;
    fs.C = C;
    fs.nchunks = Lw.nchunks;
    fs.cent = f.cent;
    fs.idx = reinterpret_cast<const uint16_t *>(ws + Lw.idx);
    fs.chunk_counts = reinterpret_cast<int *>(ws + Lw.counts);
    fs.bucket_start = reinterpret_cast<int *>(ws + Lw.starts);
    fs.order = reinterpret_cast<int *>(ws + Lw.order);
    fs.order_j = reinterpret_cast<uint16_t *>(ws + Lw.order_j);
    fs.sums = reinterpret_cast<double *>(ws + Lw.sums);
    fs.abs_max = reinterpret_cast<unsigned *>(ws + Lw.bounds);
    fs.abs_min = fs.abs_max + H;
    fs.track = 1;
    fs.redo = reinterpret_cast<int *>(ws + Lw.redo);
    fs.bkt_max = reinterpret_cast<unsigned *>(ws + Lw.bkt);
    fs.bkt_minv = fs.bkt_max + (size_t)H * C;

    const int64_t n_cent = (int64_t)H * C * D;
    fit_seed_kernel<<<(unsigned)ceil_div(n_cent, 256), 256, 0, s>>>(f, fs);
    if ((st = launch_status()) != KVQ_OK)
        return st;
    const size_t cbytes = (size_t)C * 4;
    if ((st = smem_opt_in(fit_hist_kernel, cbytes)) != KVQ_OK ||
        (st = smem_opt_in(fit_scatter_kernel, cbytes)) != KVQ_OK)
        return st;
    EncodeArgs e;
    memset(&e, 0, sizeof e);
    e.x = x;
    e.x_bf16 = f.x_bf16;
    e.T = T;
    e.H = H;
    e.C = C;
    e.bits = 2;
    e.G = 16;
    e.cent = f.cent;
    e.idx = reinterpret_cast<uint16_t *>(ws + Lw.idx);
    e.assign_only = 1;
    const dim3 chunks((unsigned)Lw.nchunks, (unsigned)H);
    for (int it = 0; it < iters; ++it) {
        if ((st = launch_encode(D, e, s)) != KVQ_OK)
            return st;
        fit_hist_kernel<<<chunks, 256, cbytes, s>>>(fs);
        fit_scan_kernel<<<dim3((unsigned)ceil_div(C, 8), (unsigned)H), 256, 0, s>>>(fs);
        fit_starts_kernel<<<(unsigned)H, 1024, 0, s>>>(fs);
        fit_scatter_kernel<<<chunks, 32, cbytes, s>>>(fs);
        const int64_t warps = (int64_t)H * C;
        const unsigned seg_blocks = (unsigned)ceil_div((int64_t)H * ceil_div(T, kFitSegSlots) * 32, 256);
        const unsigned cent_blocks = (unsigned)ceil_div(warps * 32, 256);
        fs.track = it == 0 ? 1 : 0;  // the head bounds need one pass over x
        if (D == 128) {
            if (fs.x_bf16)
                fit_segsum_kernel<128, true><<<seg_blocks, 256, 0, s>>>(fs);
            else
                fit_segsum_kernel<128, false><<<seg_blocks, 256, 0, s>>>(fs);
            fit_finalize_kernel<128><<<cent_blocks, 256, 0, s>>>(fs);
            fit_bucket_update_kernel<128><<<cent_blocks, 256, 0, s>>>(fs);
        } else {
            if (fs.x_bf16)
                fit_segsum_kernel<64, true><<<seg_blocks, 256, 0, s>>>(fs);
            else
                fit_segsum_kernel<64, false><<<seg_blocks, 256, 0, s>>>(fs);
            fit_finalize_kernel<64><<<cent_blocks, 256, 0, s>>>(fs);
            fit_bucket_update_kernel<64><<<cent_blocks, 256, 0, s>>>(fs);
        }
        if ((st = launch_status()) != KVQ_OK)
            return st;
    }
    return KVQ_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Fit with a fixed device scratch array instead of a caller workspace.
// Host code only ever uses the array's device address, looked up once per
// device with that device current; the symbol itself is a host-side stand-in.
// ---------------------------------------------------------------------------
static __device__ __align__(256) unsigned char g_fit_static_scratch[KVQ_FIT_STATIC_SCRATCH_BYTES];

namespace {

// The address is cached per device.  Two host threads making their first call
// at the same time both look it up and store the same value; the atomics make
// that well defined.  The cache is not refreshed after cudaDeviceReset, so the
// library must not be used across a device reset in one process.
void *fit_static_scratch(kvq_status *st)
{
    static std::atomic<void *> by_device[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        *st = KVQ_ERR_CUDA;
        return nullptr;
    }
    void *p = by_device[dev].load(std::memory_order_acquire);
    if (!p) {
        if (cudaGetSymbolAddress(&p, g_fit_static_scratch) != cudaSuccess || !p) {
            *st = KVQ_ERR_CUDA;
            return nullptr;
        }
        by_device[dev].store(p, std::memory_order_release);
    }
    return p;
}

}  // namespace

extern "C" {

kvq_status kvq_fit_centroids_static(const kvq_codec_desc *desc, const void *x, kvq_dtype x_dtype, int64_t T,
                                    int32_t iters, void *centroids_out, kvq_stream_t stream)
{
    kvq_status st = check_desc(desc, true);
    if (st != KVQ_OK)
        return st;
    if (desc->joint_rank > 0 || T < 0)
        return KVQ_ERR_INVALID_ARG;
    if (fit_workspace(desc, T) > (size_t)KVQ_FIT_STATIC_SCRATCH_BYTES)
        return KVQ_ERR_WORKSPACE;
    void *scratch = fit_static_scratch(&st);
    if (!scratch)
        return st;
    return kvq_fit_centroids(desc, x, x_dtype, T, iters, centroids_out, scratch, KVQ_FIT_STATIC_SCRATCH_BYTES,
                             stream);
}

kvq_status kvq_encode(const kvq_codec_desc *desc, const void *x, kvq_dtype x_dtype, int64_t T,
                      const void *centroids, const void *w_enc, uint16_t *idx, uint8_t *codes, void *meta,
                      void *workspace, size_t workspace_bytes, kvq_stream_t stream)
{
    (void)workspace;
    (void)workspace_bytes;
    kvq_status st = check_desc(desc, true);
    if (st != KVQ_OK)
        return st;
    if (desc->joint_rank > 0 || w_enc) {
        if (desc->joint_rank == 0 || !w_enc)
            return KVQ_ERR_INVALID_ARG;  // w_enc is given exactly for the joint code
        if (x_dtype != KVQ_F32 && x_dtype != KVQ_BF16)
            return KVQ_ERR_INVALID_ARG;
        return joint_encode_call(desc, x, x_dtype, T, centroids, w_enc, idx, codes, meta, nullptr,
                                 reinterpret_cast<cudaStream_t>(stream));
    }
    if (T < 0 || (x_dtype != KVQ_F32 && x_dtype != KVQ_BF16))
        return KVQ_ERR_INVALID_ARG;
    if (T == 0)
        return KVQ_OK;
    if (!x || !centroids || !idx || !codes || !meta)
        return KVQ_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(centroids) || !aligned16(codes) || !aligned16(meta) ||
        (reinterpret_cast<uintptr_t>(idx) & 1u))
        return KVQ_ERR_ALIGNMENT;
    if (desc->residual_stages == 2)
        return KVQ_ERR_INVALID_ARG;  // two stages write two code sets: kvq_encode_stages
    EncodeArgs e;
    memset(&e, 0, sizeof e);
    e.x = x;
    e.x_bf16 = x_dtype == KVQ_BF16;
    e.T = T;
    e.H = desc->num_heads;
    e.C = desc->num_centroids;
    e.bits = desc->bits;
    e.G = desc->group_size;
    e.cent = static_cast<const uint16_t *>(centroids);
    e.idx = idx;
    e.codes = codes;
    e.meta = meta;
    e.assign_only = 0;
    e.meta16 = desc->meta_format == KVQ_META_F16;
    return launch_encode(desc->head_dim, e, reinterpret_cast<cudaStream_t>(stream));
}

kvq_status kvq_encode_stages(const kvq_codec_desc *desc, const void *x, kvq_dtype x_dtype, int64_t T,
                             const void *centroids, uint16_t *idx, uint8_t *codes, float *meta, uint8_t *codes2,
                             float *meta2, kvq_stream_t stream)
{
    kvq_status st = check_desc(desc, false);
    if (st != KVQ_OK)
        return st;
    if (desc->residual_stages != 2)
        return KVQ_ERR_INVALID_ARG;
    if (T < 0 || (x_dtype != KVQ_F32 && x_dtype != KVQ_BF16))
        return KVQ_ERR_INVALID_ARG;
    if (desc->num_heads > 65535)
        return KVQ_ERR_UNSUPPORTED;
    if (T == 0)
        return KVQ_OK;
    if (!x || !centroids || !idx || !codes || !meta || !codes2 || !meta2)
        return KVQ_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(centroids) || !aligned16(codes) || !aligned16(meta) || !aligned16(codes2) ||
        !aligned16(meta2) || (reinterpret_cast<uintptr_t>(idx) & 1u))
        return KVQ_ERR_ALIGNMENT;
    EncodeArgs e;
    memset(&e, 0, sizeof e);
    e.x = x;
    e.x_bf16 = x_dtype == KVQ_BF16;
    e.T = T;
    e.H = desc->num_heads;
    e.C = desc->num_centroids;
    e.bits = desc->bits;
    e.G = desc->group_size;
    e.cent = static_cast<const uint16_t *>(centroids);
    e.idx = idx;
    e.codes = codes;
    e.meta = meta;
    e.codes2 = codes2;
    e.meta2 = meta2;
    return launch_encode(desc->head_dim, e, reinterpret_cast<cudaStream_t>(stream));
}

kvq_status kvq_encode_qsac(const kvq_codec_desc *desc, const void *x, kvq_dtype x_dtype, int64_t T,
                           const void *centroids, const float *w, int32_t M, uint16_t *idx, uint8_t *codes,
                           void *meta, kvq_stream_t stream)
{
    kvq_status st = check_desc(desc, false);
    if (st != KVQ_OK)
        return st;
    if (T < 0 || (x_dtype != KVQ_F32 && x_dtype != KVQ_BF16) || M < 1 || M > kQsacMaxM)
        return KVQ_ERR_INVALID_ARG;
    if (desc->meta_format != KVQ_META_F32 || desc->residual_stages == 2 || desc->num_heads > 65535)
        return KVQ_ERR_UNSUPPORTED;
    if (T == 0)
        return KVQ_OK;
    if (!x || !centroids || !w || !idx || !codes || !meta)
        return KVQ_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(centroids) || !aligned16(w) || !aligned16(codes) || !aligned16(meta) ||
        (reinterpret_cast<uintptr_t>(idx) & 1u))
        return KVQ_ERR_ALIGNMENT;
    QsacArgs q;
    memset(&q, 0, sizeof q);
    q.e.x = x;
    q.e.x_bf16 = x_dtype == KVQ_BF16;
    q.e.T = T;
    q.e.H = desc->num_heads;
    q.e.C = desc->num_centroids;
    q.e.bits = desc->bits;
    q.e.G = desc->group_size;
    q.e.cent = static_cast<const uint16_t *>(centroids);
    q.e.idx = idx;
    q.e.codes = codes;
    q.e.meta = meta;
    q.w = w;
    q.M = M;
    const dim3 grid((unsigned)ceil_div(T, kDirectTokens), (unsigned)desc->num_heads);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int D = desc->head_dim, B = desc->bits, G = desc->group_size;
#define KVQ_QSAC(DD, BB, GG)                                                          \
    if (D == DD && B == BB && G == GG) {                                              \
        qsac_encode_kernel<DD, BB, GG><<<grid, kDirectTokens, 0, s>>>(q);             \
        return launch_status();                                                       \
    }
    KVQ_QSAC(128, 2, 16) KVQ_QSAC(128, 2, 32) KVQ_QSAC(128, 2, 64)
    KVQ_QSAC(128, 4, 16) KVQ_QSAC(128, 4, 32) KVQ_QSAC(128, 4, 64)
    KVQ_QSAC(64, 2, 16) KVQ_QSAC(64, 2, 32) KVQ_QSAC(64, 2, 64)
    KVQ_QSAC(64, 4, 16) KVQ_QSAC(64, 4, 32) KVQ_QSAC(64, 4, 64)
#undef KVQ_QSAC
    return KVQ_ERR_UNSUPPORTED;
}

kvq_status kvq_joint_coefficients(const kvq_codec_desc *desc, const void *x, kvq_dtype x_dtype, int64_t T,
                                  const void *centroids, const void *w_enc, uint16_t *idx, float *coef_out,
                                  void *workspace, size_t workspace_bytes, kvq_stream_t stream)
{
    (void)workspace;
    (void)workspace_bytes;
    kvq_status st = check_desc(desc, true);
    if (st != KVQ_OK)
        return st;
    if (desc->joint_rank == 0 || !w_enc)
        return KVQ_ERR_INVALID_ARG;
    if (x_dtype != KVQ_F32 && x_dtype != KVQ_BF16)
        return KVQ_ERR_INVALID_ARG;
    if (T > 0 && !coef_out)
        return KVQ_ERR_INVALID_ARG;
    return joint_encode_call(desc, x, x_dtype, T, centroids, w_enc, idx, nullptr, nullptr, coef_out,
                             reinterpret_cast<cudaStream_t>(stream));
}

kvq_status kvq_decode(const kvq_compressed_view *view, void *x_out, kvq_dtype out_dtype, void *workspace,
                      size_t workspace_bytes, kvq_stream_t stream)
{
    (void)workspace;
    (void)workspace_bytes;
    kvq_status st = check_view(view);
    if (st != KVQ_OK)
        return st;
    if (out_dtype != KVQ_F32 && out_dtype != KVQ_BF16)
        return KVQ_ERR_INVALID_ARG;
    if (view->num_tokens == 0)
        return KVQ_OK;
    if (!x_out)
        return KVQ_ERR_INVALID_ARG;
    if (!aligned16(x_out))
        return KVQ_ERR_ALIGNMENT;
    if (view->desc.joint_rank > 0) {
        if (!view->w_dec)
            return KVQ_ERR_INVALID_ARG;
        if (!aligned16(view->w_dec))
            return KVQ_ERR_ALIGNMENT;
        JointDecArgs j;
        j.cent = static_cast<const uint16_t *>(view->centroids);
        j.idx = view->idx;
        j.codes = view->codes;
        j.meta = static_cast<const float *>(view->meta);
        j.T = view->num_tokens;
        j.H = view->desc.num_heads;
        j.D = view->desc.head_dim;
        j.C = view->desc.num_centroids;
        j.r = view->desc.joint_rank;
        j.bits = view->desc.bits;
        j.G = view->desc.group_size;
        j.out = x_out;
        j.out_bf16 = out_dtype == KVQ_BF16;
        return launch_joint_decode(j, view->w_dec, reinterpret_cast<cudaStream_t>(stream));
    }
    DecodeArgs a;
    memset(&a, 0, sizeof a);
    if (view->desc.residual_stages == 2) {
        if (!view->codes2 || !view->meta2)
            return KVQ_ERR_INVALID_ARG;
        if (!aligned16(view->codes2) || !aligned16(view->meta2))
            return KVQ_ERR_ALIGNMENT;
        a.codes2 = view->codes2;
        a.meta2 = view->meta2;
    }
    a.cent = static_cast<const uint16_t *>(view->centroids);
    a.idx = view->idx;
    a.codes = view->codes;
    a.meta = view->meta;
    a.T = view->num_tokens;
    a.H = view->desc.num_heads;
    a.D = view->desc.head_dim;
    a.C = view->desc.num_centroids;
    a.bits = view->desc.bits;
    a.G = view->desc.group_size;
    a.out = x_out;
    a.out_bf16 = out_dtype == KVQ_BF16;
    a.meta16 = view->desc.meta_format == KVQ_META_F16;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (a.D == 128)
        decode_kernel<128><<<dim3((unsigned)ceil_div(a.T, 256 / 16), (unsigned)a.H), 256, 0, s>>>(a);
    else
        decode_kernel<64><<<dim3((unsigned)ceil_div(a.T, 256 / 8), (unsigned)a.H), 256, 0, s>>>(a);
    return launch_status();
}

kvq_status kvq_attention_lse(const void *q, int64_t Tq, const kvq_compressed_view *k, const kvq_compressed_view *v,
                             int64_t t_begin, int64_t t_end, float softmax_scale, void *o_out, kvq_dtype o_dtype,
                             float *lse_out, void *workspace, size_t workspace_bytes, kvq_stream_t stream)
{
    kvq_status st = check_history_pair(k, v, t_begin, t_end);
    if (st != KVQ_OK)
        return st;
    if (Tq < 0 || (o_dtype != KVQ_F32 && o_dtype != KVQ_BF16))
        return KVQ_ERR_INVALID_ARG;
    if (Tq == 0)
        return KVQ_OK;
    if (!q || !o_out || !lse_out)
        return KVQ_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(o_out) || !aligned16(lse_out))
        return KVQ_ERR_ALIGNMENT;
    const int D = k->desc.head_dim;
    AttnArgs a = attn_args(q, Tq, k->desc.num_heads, D, t_begin, t_end, softmax_scale, o_out, o_dtype, lse_out);
    a.k = to_codec_view(k);
    a.v = to_codec_view(v);
    return attention_call(a, D, workspace, workspace_bytes, reinterpret_cast<cudaStream_t>(stream));
}

kvq_status kvq_attention_psac_lse(const void *q, int64_t Tq, const kvq_compressed_view *k,
                                  const kvq_compressed_view *v, const float *U, const float *coef, int32_t rank,
                                  int64_t t_begin, int64_t t_end, float softmax_scale, void *o_out, kvq_dtype o_dtype,
                                  float *lse_out, void *workspace, size_t workspace_bytes, kvq_stream_t stream)
{
    kvq_status st = check_history_pair(k, v, t_begin, t_end);
    if (st != KVQ_OK)
        return st;
    if (Tq < 0 || (o_dtype != KVQ_F32 && o_dtype != KVQ_BF16))
        return KVQ_ERR_INVALID_ARG;
    if (rank != kPsacRank || k->desc.head_dim != 128)
        return KVQ_ERR_UNSUPPORTED;
    const int H = k->desc.num_heads;
    const int Cmax = k->desc.num_centroids > v->desc.num_centroids ? k->desc.num_centroids : v->desc.num_centroids;
    if ((int64_t)H * k->num_tokens >= (int64_t)INT32_MAX || (int64_t)H * Cmax >= (int64_t)INT32_MAX)
        return KVQ_ERR_UNSUPPORTED;
    if (Tq == 0)
        return KVQ_OK;
    if (!q || !o_out || !lse_out || !U || !coef)
        return KVQ_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(o_out) || !aligned16(lse_out) || !aligned16(U) || !aligned16(coef))
        return KVQ_ERR_ALIGNMENT;
    AttnArgs a = attn_args(q, Tq, H, 128, t_begin, t_end, softmax_scale, o_out, o_dtype, lse_out);
    a.k = to_codec_view(k);
    a.v = to_codec_view(v);
    a.psac_u = U;
    a.psac_coef = coef;
    return attention_call(a, 128, workspace, workspace_bytes, reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"

namespace {

// NanoKV-Fast workspace: q_low bf16 [Tq][H][d_low] and o_low float
// [Tq][H][d_low] (each 256-byte aligned), then optional split partials.
size_t fast_base_bytes(int H, int dl, int64_t Tq)
{
    return round_up((size_t)Tq * H * dl * 2, 256) + round_up((size_t)Tq * H * dl * 4, 256);
}

template <int DIN, int DOUT, bool IN_BF16>
kvq_status launch_fast_map(const FastMapArgs &f, cudaStream_t s)
{
    constexpr int kSmem = DIN * DOUT * 4;
    static std::atomic<bool> configured[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return KVQ_ERR_CUDA;
    if (!configured[dev].load()) {
        if (cudaFuncSetAttribute(fast_map_kernel<DIN, DOUT, IN_BF16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kSmem) != cudaSuccess)
            return KVQ_ERR_CUDA;
        configured[dev].store(true);
    }
    const dim3 grid((unsigned)ceil_div(f.Tq, kFastThreads), (unsigned)f.H);
    fast_map_kernel<DIN, DOUT, IN_BF16><<<grid, kFastThreads, kSmem, s>>>(f);
    return launch_status();
}

kvq_status launch_fast_reduce(const FastMapArgs &f, int d, int dl, cudaStream_t s)
{
    if (d == 128)
        return dl == 128 ? launch_fast_map<128, 128, true>(f, s) : launch_fast_map<128, 64, true>(f, s);
    return launch_fast_map<64, 64, true>(f, s);
}

kvq_status launch_fast_restore(const FastMapArgs &f, int d, int dl, cudaStream_t s)
{
    if (d == 128)
        return dl == 128 ? launch_fast_map<128, 128, false>(f, s) : launch_fast_map<64, 128, false>(f, s);
    return launch_fast_map<64, 64, false>(f, s);
}

bool fast_dims_ok(int d, int dl) { return supported_dim(d) && supported_dim(dl) && dl <= d; }

}  // namespace

extern "C" {

kvq_status kvq_set_wait_limit(uint32_t polls)
{
    if (cudaMemcpyToSymbol(c_wait_limit, &polls, sizeof polls) != cudaSuccess)
        return KVQ_ERR_CUDA;
    return KVQ_OK;
}

kvq_status kvq_fast_attention_workspace_size(int32_t H, int32_t d, int32_t d_low, int64_t Tq, size_t *bytes)
{
    if (!bytes || H < 1 || Tq < 0)
        return KVQ_ERR_INVALID_ARG;
    if (!fast_dims_ok(d, d_low) || H > 65535)
        return KVQ_ERR_UNSUPPORTED;
    *bytes = fast_base_bytes(H, d_low, Tq) + partials_bytes(kMaxAttnSplit, H, d_low, Tq);
    return KVQ_OK;
}

kvq_status kvq_fast_attention_lse(const void *q, int64_t Tq, const void *k_low, const void *v_low, int64_t num_keys,
                                  int32_t H, int32_t d, int32_t d_low, const void *P, const void *R, int64_t t_begin,
                                  int64_t t_end, float softmax_scale, void *o_out, kvq_dtype o_dtype, float *lse_out,
                                  void *workspace, size_t workspace_bytes, kvq_stream_t stream)
{
    if (H < 1 || Tq < 0 || num_keys < 0 || t_begin < 0 || t_end < t_begin || t_end > num_keys)
        return KVQ_ERR_INVALID_ARG;
    if (!fast_dims_ok(d, d_low) || H > 65535)
        return KVQ_ERR_UNSUPPORTED;
    if (o_dtype != KVQ_F32 && o_dtype != KVQ_BF16)
        return KVQ_ERR_INVALID_ARG;
    if (Tq == 0)
        return KVQ_OK;
    if (!q || !P || !R || !o_out || !lse_out || (t_end > t_begin && (!k_low || !v_low)))
        return KVQ_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(P) || !aligned16(R) || !aligned16(o_out) || !aligned16(lse_out) ||
        !aligned16(k_low) || !aligned16(v_low) || !aligned16(workspace))
        return KVQ_ERR_ALIGNMENT;
    const size_t base = fast_base_bytes(H, d_low, Tq);
    if (!workspace || workspace_bytes < base)
        return KVQ_ERR_WORKSPACE;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    uint16_t *q_low = reinterpret_cast<uint16_t *>(ws);
    float *o_low = reinterpret_cast<float *>(ws + round_up((size_t)Tq * H * d_low * 2, 256));
    // (1) queries into the low space, rounded to bf16
    FastMapArgs f;
    f.in = q;
    f.map = static_cast<const uint16_t *>(P);
    f.out = q_low;
    f.Tq = Tq;
    f.H = H;
    f.out_bf16 = 1;
    kvq_status st = launch_fast_reduce(f, d, d_low, s);
    if (st != KVQ_OK)
        return st;
    // (2) attention in the low space with the full head dimension's scale
    const float scale = softmax_scale > 0.0f ? softmax_scale : 1.0f / sqrtf((float)d);
    AttnArgs a = attn_args(q_low, Tq, H, d_low, t_begin, t_end, scale, o_low, KVQ_F32, lse_out);
    a.dense = 1;
    a.k_dense = static_cast<const uint16_t *>(k_low);
    a.v_dense = static_cast<const uint16_t *>(v_low);
    if ((st = attention_call(a, d_low, ws + base, workspace_bytes - base, s)) != KVQ_OK)
        return st;
    // (3) outputs restored to the head dimension
    f.in = o_low;
    f.map = static_cast<const uint16_t *>(R);
    f.out = o_out;
    f.out_bf16 = o_dtype == KVQ_BF16;
    return launch_fast_restore(f, d, d_low, s);
}

kvq_status kvq_psac_coefficients(const kvq_compressed_view *k, const void *x, kvq_dtype x_dtype, const float *U,
                                 int32_t rank, float *coef_out, kvq_stream_t stream)
{
    kvq_status st = check_view(k);
    if (st != KVQ_OK)
        return st;
    if (k->desc.joint_rank > 0 || k->desc.residual_stages == 2 || rank != kPsacRank)
        return KVQ_ERR_UNSUPPORTED;
    if (x_dtype != KVQ_F32 && x_dtype != KVQ_BF16)
        return KVQ_ERR_INVALID_ARG;
    if (k->num_tokens == 0)
        return KVQ_OK;
    if (!x || !U || !coef_out)
        return KVQ_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(U) || !aligned16(coef_out))
        return KVQ_ERR_ALIGNMENT;
    if (k->desc.num_heads > 65535)
        return KVQ_ERR_UNSUPPORTED;
    PsacCoefArgs p;
    DecodeArgs &a = p.d;
    memset(&p, 0, sizeof p);
    a.cent = static_cast<const uint16_t *>(k->centroids);
    a.idx = k->idx;
    a.codes = k->codes;
    a.meta = k->meta;
    a.T = k->num_tokens;
    a.H = k->desc.num_heads;
    a.D = k->desc.head_dim;
    a.C = k->desc.num_centroids;
    a.bits = k->desc.bits;
    a.G = k->desc.group_size;
    a.meta16 = k->desc.meta_format == KVQ_META_F16;
    p.x = x;
    p.x_bf16 = x_dtype == KVQ_BF16;
    p.U = U;
    p.coef = coef_out;
    const dim3 grid((unsigned)ceil_div(a.T, 128), (unsigned)a.H);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (a.D == 128)
        psac_coef_kernel<128><<<grid, 128, 0, s>>>(p);
    else
        psac_coef_kernel<64><<<grid, 128, 0, s>>>(p);
    return launch_status();
}

kvq_status kvq_attention_dense_lse(const void *q, int64_t Tq, const void *k, const void *v, int64_t num_keys,
                                   int32_t H, int32_t d, int64_t t_begin, int64_t t_end, float softmax_scale,
                                   void *o_out, kvq_dtype o_dtype, float *lse_out, void *workspace,
                                   size_t workspace_bytes, kvq_stream_t stream)
{
    if (H < 1 || Tq < 0 || num_keys < 0 || t_begin < 0 || t_end < t_begin || t_end > num_keys)
        return KVQ_ERR_INVALID_ARG;
    if (!supported_dim(d) || H > 65535)
        return KVQ_ERR_UNSUPPORTED;
    if (o_dtype != KVQ_F32 && o_dtype != KVQ_BF16)
        return KVQ_ERR_INVALID_ARG;
    if (Tq == 0)
        return KVQ_OK;
    if (!q || !o_out || !lse_out || (t_end > t_begin && (!k || !v)))
        return KVQ_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(o_out) || !aligned16(lse_out) || !aligned16(k) || !aligned16(v))
        return KVQ_ERR_ALIGNMENT;
    AttnArgs a = attn_args(q, Tq, H, d, t_begin, t_end, softmax_scale, o_out, o_dtype, lse_out);
    a.dense = 1;
    a.k_dense = static_cast<const uint16_t *>(k);
    a.v_dense = static_cast<const uint16_t *>(v);
    return attention_call(a, d, workspace, workspace_bytes, reinterpret_cast<cudaStream_t>(stream));
}

kvq_status kvq_layer_attention(const void *q, int64_t Tq, const kvq_compressed_view *k_hist,
                               const kvq_compressed_view *v_hist, int64_t t_begin, int64_t t_end, const void *k_cur,
                               const void *v_cur, int64_t num_cur, float softmax_scale, void *o_out,
                               kvq_dtype o_dtype, float *lse_out, void *workspace, size_t workspace_bytes,
                               kvq_stream_t stream)
{
    kvq_status st = check_history_pair(k_hist, v_hist, t_begin, t_end);
    if (st != KVQ_OK)
        return st;
    if (Tq < 0 || num_cur < 0 || (o_dtype != KVQ_F32 && o_dtype != KVQ_BF16))
        return KVQ_ERR_INVALID_ARG;
    if (Tq == 0)
        return KVQ_OK;
    if (!q || !o_out || !lse_out || (num_cur > 0 && (!k_cur || !v_cur)))
        return KVQ_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(o_out) || !aligned16(lse_out) || !aligned16(k_cur) || !aligned16(v_cur) ||
        !aligned16(workspace))
        return KVQ_ERR_ALIGNMENT;
    const int H = k_hist->desc.num_heads, D = k_hist->desc.head_dim;
    if (!workspace || workspace_bytes < layer_workspace(&k_hist->desc, Tq))
        return KVQ_ERR_WORKSPACE;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    AttnArgs hist = attn_args(q, Tq, H, D, t_begin, t_end, softmax_scale, o_out, o_dtype, lse_out);
    hist.k = to_codec_view(k_hist);
    hist.v = to_codec_view(v_hist);
    AttnArgs cur = attn_args(q, Tq, H, D, 0, num_cur, softmax_scale, o_out, o_dtype, lse_out);
    cur.dense = 1;
    cur.k_dense = static_cast<const uint16_t *>(k_cur);
    cur.v_dense = static_cast<const uint16_t *>(v_cur);
    // partials: history in slots [0, nh), dense keys in [nh, nh + nc)
    const int nh = attention_split_for(hist, D, t_end - t_begin);
    const int nc = attention_split_for(cur, D, num_cur);
    const int64_t slice = Tq * (int64_t)H * D;
    float *o_part = static_cast<float *>(workspace);
    float *l_part = reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) +
                                              round_up((size_t)(2 * kMaxAttnSplit) * (size_t)slice * 4, 256));
    if ((st = launch_attention_partials(hist, D, nh, o_part, l_part, s)) != KVQ_OK)
        return st;
    if ((st = launch_attention_partials(cur, D, nc, o_part + nh * slice, l_part + (int64_t)nh * H * Tq, s)) !=
        KVQ_OK)
        return st;
    MergeArgs m;
    memset(&m, 0, sizeof m);
    for (int z = 0; z < nh + nc; ++z) {
        m.o[z] = o_part + z * slice;
        m.lse[z] = l_part + (int64_t)z * H * Tq;
    }
    m.n = nh + nc;
    m.Tq = Tq;
    m.H = H;
    m.D = D;
    m.o_out = o_out;
    m.o_bf16 = o_dtype == KVQ_BF16;
    m.lse_out = lse_out;
    launch_merge(m, s);
    return launch_status();
}

kvq_status kvq_lse_merge(int32_t n_parts, const float *const *o_parts, const float *const *lse_parts, int64_t Tq,
                         int32_t H, int32_t d, void *o_out, kvq_dtype o_dtype, float *lse_out, kvq_stream_t stream)
{
    if (n_parts < 1 || n_parts > kMaxMergeParts || !o_parts || !lse_parts || Tq < 0 || H < 1)
        return KVQ_ERR_INVALID_ARG;
    if (!supported_dim(d))
        return KVQ_ERR_UNSUPPORTED;
    if (o_dtype != KVQ_F32 && o_dtype != KVQ_BF16)
        return KVQ_ERR_INVALID_ARG;
    if (Tq == 0)
        return KVQ_OK;
    if (!o_out || !lse_out)
        return KVQ_ERR_INVALID_ARG;
    MergeArgs a;
    memset(&a, 0, sizeof a);
    for (int b = 0; b < n_parts; ++b) {
        if (!o_parts[b] || !lse_parts[b])
            return KVQ_ERR_INVALID_ARG;
        if (!aligned16(o_parts[b]) || (reinterpret_cast<uintptr_t>(lse_parts[b]) & 3u))
            return KVQ_ERR_ALIGNMENT;
        a.o[b] = o_parts[b];
        a.lse[b] = lse_parts[b];
    }
    if (!aligned16(o_out) || (reinterpret_cast<uintptr_t>(lse_out) & 3u))
        return KVQ_ERR_ALIGNMENT;
    a.n = n_parts;
    a.Tq = Tq;
    a.H = H;
    a.D = d;
    a.o_out = o_out;
    a.o_bf16 = o_dtype == KVQ_BF16;
    a.lse_out = lse_out;
    launch_merge(a, reinterpret_cast<cudaStream_t>(stream));
    return launch_status();
}

kvq_status kvq_last_device_status(kvq_stream_t stream)
{
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess)
        return KVQ_ERR_CUDA;
    unsigned int word = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&word, g_device_status, sizeof word) != cudaSuccess)
        return KVQ_ERR_CUDA;
    if (word != 0 && cudaMemcpyToSymbol(g_device_status, &zero, sizeof zero) != cudaSuccess)
        return KVQ_ERR_CUDA;
    if (word & DEVSTAT_TIMEOUT)
        return KVQ_ERR_DEVICE_TIMEOUT;
    if (word & DEVSTAT_BAD_INDEX)
        return KVQ_ERR_INVALID_ARG;
    return KVQ_OK;
}

}  // extern "C"

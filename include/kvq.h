/*
 * kvq.h -- C ABI of libkvq: centroid-residual low-bit compression of an
 * autoregressive video model's historical KV cache, and attention of the
 * current chunk's queries over that compressed history (NVIDIA B200, sm_100a).
 *
 * The method, as the pages state it:
 *  - QVG-style codec: every key/value token of a head is assigned to its
 *    nearest centroid (k-means fitted online per head, per cache block,
 *    separately for K and V) and only the residual is quantised to low bit
 *    width (QuantWM: Temporally Consistent 2-Bit KV Cache Quantization for
 *    Video World Models, Sec. 4.1; CORAL-KV, Sec. 2; TempoKV, Sec. 1 and
 *    Sec. 3.3 Eq. 2; NanoKV page, Table 4).
 *  - asymmetric affine b-bit quantisation per channel group (TempoKV, Sec. 3.1,
 *    Eq. 1), packed storage (NanoKV page, Table 4; QuantWM, Fig. 9).
 *  - optional joint head-channel linear encoder/decoder of the residual with
 *    INT4 coefficients, centres added back after decoding (NanoKV page,
 *    abstract, Fig. 4(a,b)).
 *  - attention over the compressed history with the reconstruction done on
 *    demand, and log-sum-exp merging of partial results (NanoKV page,
 *    Fig. 4(a,d); QuantWM, Fig. 9).
 *  - the current chunk's full attention: the compressed history together
 *    with uncompressed keys (the chunk itself, raw protected tokens; NanoKV
 *    page, Table 4) under one softmax, by the same LSE merging.
 *
 * Conventions for every call:
 *  - All tensor pointers are DEVICE pointers owned by the caller; the library
 *    allocates no device memory and keeps no state across calls apart from a
 *    per-device status word (see kvq_last_device_status).  Pointers must be
 *    16-byte aligned unless stated otherwise (KVQ_ERR_ALIGNMENT).
 *  - Calls are asynchronous on `stream` (NULL = the legacy default stream).
 *  - Arguments are validated on the host before anything is launched; a
 *    rejected call launches nothing and returns the error.  No call aborts
 *    or throws.  Launch failures return KVQ_ERR_CUDA.
 *  - bf16 values are stored as raw 16-bit patterns (same bits as
 *    __nv_bfloat16); float is IEEE binary32.
 *  - Layouts (T = history tokens, H = heads, d = head dim, C = centroids,
 *    b = bits, G = group size, r = joint rank, Tq = query tokens):
 *      history   x      [T][H][d]        (token t = frame * S + position)
 *      centroids        [H][C][d]        bf16
 *      idx              [H][T]           uint16
 *      codes (per-head) [H][T][d*b/8]    uint8, code of channel c of a byte
 *                                         holds bits (c % (8/b)) * b ..; low
 *                                         bits first
 *      meta  (per-head) [H][T][d/G][2]   {scale s, zero z}: float, or
 *                                         binary16 bits (meta_format)
 *      codes (joint)    [T][r*b/8]       meta (joint) [T][r/G][2]
 *      queries q        [Tq][H][d]       bf16;  output o [Tq][H][d]
 *      lse              [H][Tq]          float, natural logarithm
 */
#ifndef KVQ_H_
#define KVQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define KVQ_API __attribute__((visibility("default")))
#else
#define KVQ_API
#endif

struct CUstream_st;
/* Same type as cudaStream_t. */
typedef struct CUstream_st *kvq_stream_t;

typedef enum {
    KVQ_OK = 0,
    KVQ_ERR_INVALID_ARG = 1,    /* null pointer, bad size or shape */
    KVQ_ERR_UNSUPPORTED = 2,    /* a valid request the library does not serve */
    KVQ_ERR_ALIGNMENT = 3,      /* a pointer is not 16-byte aligned */
    KVQ_ERR_WORKSPACE = 4,      /* workspace missing or smaller than required */
    KVQ_ERR_CUDA = 5,           /* a CUDA runtime call or launch failed */
    KVQ_ERR_DEVICE_TIMEOUT = 6  /* a kernel gave up a bounded wait (device status) */
} kvq_status;

typedef enum { KVQ_F32 = 0, KVQ_BF16 = 1 } kvq_dtype;

/* Storage of the per-group {scale, zero} pair (kvq_codec_desc.meta_format). */
typedef enum {
    KVQ_META_F32 = 0, /* binary32 {s, z}: 8 bytes per group */
    KVQ_META_F16 = 1  /* binary16 {s, z}: 4 bytes per group (see kvq_encode) */
} kvq_meta_format;

typedef enum {
    KVQ_OP_FIT = 0,
    KVQ_OP_ENCODE = 1,
    KVQ_OP_DECODE = 2,
    KVQ_OP_ATTENTION = 3,
    KVQ_OP_LAYER_ATTENTION = 4
} kvq_op;

/* Codec of one K or V branch.  K and V are described separately, which is
 * how mixed bit widths (k4v2 etc.; TempoKV, Sec. 4.2, Table 4) are set. */
typedef struct {
    int32_t num_heads;     /* H >= 1 */
    int32_t head_dim;      /* d: 64 or 128 */
    int32_t num_centroids; /* C: 1 .. 65536 */
    int32_t bits;          /* b: 2 or 4 */
    int32_t group_size;    /* G: multiple of 8 dividing d (per-head) or r (joint) */
    int32_t joint_rank;    /* 0: per-head codec; r > 0: joint head-channel code */
    int32_t meta_format;   /* kvq_meta_format; 0 (binary32) when zero-initialised */
    int32_t residual_stages; /* 0 or 1: one residual stage; 2: a second stage
                              * (kvq_encode_stages; per-head codec with binary32
                              * {s, z} only) */
} kvq_codec_desc;

/* A compressed K or V history as produced by kvq_encode (read-only view). */
typedef struct {
    kvq_codec_desc desc;
    int64_t num_tokens;     /* T */
    const void *centroids;  /* [H][C][d] bf16 */
    const uint16_t *idx;    /* [H][T] */
    const uint8_t *codes;   /* per-head [H][T][d*b/8]; joint [T][r*b/8] */
    const void *meta;       /* per-head [H][T][d/G][2]; joint [T][r/G][2] (meta_format) */
    const void *w_dec;      /* joint only: decoder [r][H*d] bf16; else NULL */
    const uint8_t *codes2;  /* residual_stages = 2: stage-2 codes, laid out as codes */
    const float *meta2;     /* residual_stages = 2: stage-2 {s, z}, laid out as meta */
} kvq_compressed_view;

/* Human-readable name of a status code (static string, never NULL). */
KVQ_API const char *kvq_status_string(kvq_status s);

/* Byte sizes of the three encoded arrays for T tokens of this codec (host
 * only; no device work).  Any output pointer may be NULL. */
KVQ_API kvq_status kvq_encoded_sizes(const kvq_codec_desc *desc, int64_t num_tokens, size_t *idx_bytes,
                             size_t *code_bytes, size_t *meta_bytes);

/* Device workspace (bytes) an operation needs for these sizes; 0 means the
 * call accepts workspace = NULL.  Tq is used by KVQ_OP_ATTENTION and
 * KVQ_OP_LAYER_ATTENTION only, and only H and d of desc matter for them.
 * KVQ_OP_ATTENTION also sizes kvq_attention_dense_lse's optional workspace
 * (pass a desc with the same H and d). */
KVQ_API kvq_status kvq_workspace_size(kvq_op op, const kvq_codec_desc *desc, int64_t num_tokens,
                              int64_t num_queries, size_t *bytes);

/*
 * Fit per-head centroids to one K or V history (k-means; CORAL-KV, Sec. 2:
 * per-head codebooks fitted online for each cache block; NanoKV page,
 * Table 4: QVG uses 256 centres and two k-means iterations, BF16 centres).
 *   x            [T][H][d] float or bf16 (x_dtype); T >= C
 *   iters        >= 0 rounds of {assign every token to its nearest centre;
 *                move each centre to the mean of its tokens}
 *   centroids_out [H][C][d] bf16.  Seeds are the first C tokens.  A centre
 *                 that receives no token keeps its value.  Means are summed
 *                 in binary64 and rounded to binary32, then to bf16.
 *   workspace    >= kvq_workspace_size(KVQ_OP_FIT, ...) bytes.
 */
KVQ_API kvq_status kvq_fit_centroids(const kvq_codec_desc *desc, const void *x, kvq_dtype x_dtype, int64_t num_tokens,
                             int32_t iters, void *centroids_out, void *workspace, size_t workspace_bytes,
                             kvq_stream_t stream);

/* Size of the fixed device scratch behind kvq_fit_centroids_static. */
#define KVQ_FIT_STATIC_SCRATCH_BYTES (16u << 20)

/*
 * kvq_fit_centroids without a caller-supplied workspace: the same fit, with
 * its scratch in a fixed device array inside the library.  No passage of the
 * pages corresponds to this call; it exists for callers that cannot
 * allocate device memory on demand -- for example a serving runtime that
 * reserves nearly all HBM up front for its KV cache and routes every
 * allocation through its own pool, or a plain C caller with no allocator
 * handle at the point of the call.  Such callers still pass x and
 * centroids_out; nothing is allocated, and no cudaMalloc / cudaFree or
 * allocating library routine is called.
 *
 *  - Limit: the scratch kvq_workspace_size(KVQ_OP_FIT, desc, T, ...) reports
 *    must not exceed KVQ_FIT_STATIC_SCRATCH_BYTES (16 MiB: e.g. 12 heads x
 *    32,760 tokens x 256 centres x 128 channels needs 7.9 MB); larger requests return
 *    KVQ_ERR_WORKSPACE before anything is launched.
 *  - The array is one per GPU that loads the library and is held until the
 *    process exits.  Every call on a device shares it: two calls whose work
 *    overlaps on that GPU (different streams, no ordering between them) race
 *    and corrupt each other's results.  Order them on one stream or with
 *    events.  Sums and counts are cleared at the start of every round, so
 *    no state carries over from an earlier call.
 *  - The first call on each device looks up the array's device address
 *    (cudaGetSymbolAddress with that device current) and caches it; make
 *    that first call before any stream capture.  The cache is not refreshed
 *    by a cudaDeviceReset: do not use this call across a device reset in one
 *    process.
 * Other arguments, validation and results are those of kvq_fit_centroids.
 */
KVQ_API kvq_status kvq_fit_centroids_static(const kvq_codec_desc *desc, const void *x, kvq_dtype x_dtype,
                                            int64_t num_tokens, int32_t iters, void *centroids_out,
                                            kvq_stream_t stream);

/*
 * Encode one K or V history against fitted centroids.
 * Per-head codec (desc->joint_rank == 0, w_enc == NULL):
 *   idx[h][t]  = nearest centre (squared Euclidean distance evaluated in
 *                binary32 channel by channel without FMA; ties go to the
 *                lowest index) -- QuantWM, Sec. 4.1;
 *   residual   r = x - mu[idx] (binary32; TempoKV, Sec. 3.3, Eq. 2);
 *   per group of G channels: s = (max - min)/(2^b - 1), z = rint(-min/s),
 *   q = clamp(rint(r/s) + z, 0, 2^b - 1) with 1/s formed once per group
 *   (TempoKV, Sec. 3.1, Eq. 1); a zero-range (or underflowing) group stores
 *   s = |min|, z = -sign(min), q = 0.  Codes packed low bits first.
 *   Compact {s, z} (meta_format = KVQ_META_F16; the b + 1 bits per value of
 *   TempoKV, Table 1, at G = 32): s is rounded to binary16 (nearest, ties to
 *   even, saturating at 65504), 1/s and z are formed from the rounded scale,
 *   z is rounded to binary16 likewise, and the codes use the stored values;
 *   a zero-range group, or one whose scale rounds to zero, stores
 *   s = binary16(|min|), z = -sign(min), q = 0.  Per-head codec only (the
 *   joint codec returns KVQ_ERR_UNSUPPORTED).
 * Joint codec (desc->joint_rank = r > 0, w_enc = [H*d][r] bf16):
 *   idx as above per head; the residual of all H*d channels of a token is
 *   rounded to bf16 and projected, c = R W_enc (tensor-core GEMM, binary32
 *   accumulation), and the r coefficients are quantised per group of G as
 *   above (NanoKV page, Fig. 4(b)).  Needs x in bf16 (KVQ_ERR_UNSUPPORTED
 *   otherwise), r a multiple of 64 up to 256 and G in {16, 32, 64}
 *   (KVQ_ERR_UNSUPPORTED otherwise); w_enc 16-byte aligned.  w_enc given
 *   without joint_rank, or joint_rank without w_enc, is KVQ_ERR_INVALID_ARG.
 * Outputs: idx [H][T], codes, meta as in the layout table.  Neither codec
 * needs workspace (kvq_workspace_size(KVQ_OP_ENCODE, ...) reports 0; the
 * arguments are accepted and ignored).
 */
KVQ_API kvq_status kvq_encode(const kvq_codec_desc *desc, const void *x, kvq_dtype x_dtype, int64_t num_tokens,
                      const void *centroids, const void *w_enc, uint16_t *idx, uint8_t *codes, void *meta,
                      void *workspace, size_t workspace_bytes, kvq_stream_t stream);

/*
 * Encode with two residual stages (desc->residual_stages = 2).  The reading
 * of QVG's progressive residual quantisation, which TempoKV (Sec. 2) names
 * without giving its steps (NanoKV page, Table 4 evaluates QVG with one
 * stage): idx, codes and meta exactly as kvq_encode writes them; then, per
 * group, the error stage 1 leaves, e_c = r_c - (q_c - z) s (binary32), is
 * quantised again with Eq. 1 on the same groups and bit width into codes2
 * and meta2 (the same sizes and layouts as codes and meta).  kvq_decode of a
 * view carrying codes2 / meta2 reconstructs (mu + (q1 - z1) s1) + (q2 - z2) s2,
 * each operation rounded to binary32.  Per-head codec with binary32 {s, z}
 * (KVQ_ERR_UNSUPPORTED otherwise); all arrays 16-byte aligned.  Runs where
 * kvq_encode does (the tensor-core filter for bf16 histories and the C it
 * takes, else the exact CUDA-core kernel), with identical results on both
 * paths.  The attention calls refuse
 * two-stage views (KVQ_ERR_UNSUPPORTED): decode them and use
 * kvq_attention_dense_lse.
 */
KVQ_API kvq_status kvq_encode_stages(const kvq_codec_desc *desc, const void *x, kvq_dtype x_dtype, int64_t num_tokens,
                                     const void *centroids, uint16_t *idx, uint8_t *codes, float *meta,
                                     uint8_t *codes2, float *meta2, kvq_stream_t stream);

/*
 * Encode one K history with QuantWM's query-sensitive centre selection
 * (QSAC; QuantWM: Temporally Consistent 2-Bit KV Cache Quantization for Video
 * World Models, Sec. 4.1).  Per token-head:
 *   d_j   = sum_c w_c (x_c - mu_jc)^2 in binary32, each operation rounded, in
 *           channel order; the M smallest by (d_j, j) are the candidates;
 *   score = sum over groups g of W_g R_g^2 (binary32, group order), W_g the
 *           sum of the group's w_c in channel order, R_g = max - min of the
 *           group's residual x - mu_j (the Widrow factor 1/(12 (2^b - 1)^2)
 *           is common to all candidates and dropped);
 *   idx   = the candidate with the lowest score, ties to the better-ranked;
 *   codes and {s, z} of x - mu[idx] exactly as kvq_encode writes them.
 *   w       [H][d] binary32 channel weights: the diagonal of the head's
 *           second-moment matrix of the queries seen so far (all ones
 *           before any query; QuantWM, cold start); device pointer, 16-byte
 *           aligned.  Computing them is the caller's (they come from the
 *           model's queries, not from this history).
 *   M       1 .. 8 candidates (QuantWM, Table 11: M = 4); M = 1 is the plain
 *           nearest centre under the weighted distance.
 * Per-head codec only (joint_rank = 0) with binary32 {s, z} (meta_format
 * KVQ_META_F32; KVQ_ERR_UNSUPPORTED otherwise), d in {64, 128}; x float or
 * bf16; outputs and other requirements as for kvq_encode.  Runs on CUDA cores with
 * the specified arithmetic, so idx, codes and {s, z} are bit-exact.
 */
KVQ_API kvq_status kvq_encode_qsac(const kvq_codec_desc *desc, const void *x, kvq_dtype x_dtype, int64_t num_tokens,
                                   const void *centroids, const float *w, int32_t M, uint16_t *idx, uint8_t *codes,
                                   void *meta, kvq_stream_t stream);

/*
 * Joint codec only: the binary32 coefficient matrix c = R W_enc [T][r] that
 * kvq_encode quantises, and idx [H][T].  Lets a caller quantise the same
 * coefficients independently: they are bit-identical to the ones kvq_encode
 * quantises for the same inputs.  coef_out 16-byte aligned; requirements and
 * workspace as for the joint kvq_encode.
 */
KVQ_API kvq_status kvq_joint_coefficients(const kvq_codec_desc *desc, const void *x, kvq_dtype x_dtype,
                                  int64_t num_tokens, const void *centroids, const void *w_enc, uint16_t *idx,
                                  float *coef_out, void *workspace, size_t workspace_bytes,
                                  kvq_stream_t stream);

/*
 * Reconstruct a history from its compressed view (NanoKV page, Fig. 4(b):
 * the decoder reconstructs the residual and adds back the centres).
 * Per-head: x^ = mu[idx] + (q - z) * s, each step rounded to binary32
 * (subtract, multiply, add; no FMA), then stored as float or bf16 (RNE);
 * with compact {s, z} the binary16 values are widened first.
 * Joint: c^ = (q - z) s (binary32); R^ = c^ W_dec (tensor-core GEMM: c^ is
 *   carried as a bf16 high part plus a bf16 remainder, about 16 significant
 *   bits, against bf16 W_dec with binary32 accumulation); x^ = mu[idx] + R^
 *   rounded to binary32.  view->w_dec [r][H*d] bf16, 16-byte aligned.
 *   x_out [T][H][d] in out_dtype.  No workspace is needed (the arguments are
 *   accepted and ignored).
 */
KVQ_API kvq_status kvq_decode(const kvq_compressed_view *view, void *x_out, kvq_dtype out_dtype, void *workspace,
                      size_t workspace_bytes, kvq_stream_t stream);

/*
 * Attention of the current chunk's queries over history tokens
 * [t_begin, t_end) of a compressed K and V (per-head codec), with the
 * reconstruction fused into the kernel (NanoKV page, Fig. 4(a); QuantWM,
 * Fig. 9: on-demand reconstruction):
 *   s_ij = softmax_scale * q_i . k^_j   (softmax_scale <= 0 selects 1/sqrt(d))
 *   o_i  = sum_j softmax(s_i)_j v^_j,  lse_i = ln sum_j exp(s_ij)
 * k^ and v^ are rounded to bf16 for the tensor cores; logits, softmax and the
 * output accumulate in binary32.  No mask: the history precedes the chunk.
 *   q     [Tq][H][d] bf16;  o_out [Tq][H][d] (o_dtype);  lse_out [H][Tq]
 * k and v must have the same H, d and num_tokens; their bits, group sizes,
 * centroid counts and meta formats may differ.  Compact {s, z} needs d = 128
 * (KVQ_ERR_UNSUPPORTED for d = 64).  An empty range gives o = 0,
 * lse = -inf.
 * Workspace (optional): with at least kvq_workspace_size(KVQ_OP_ATTENTION, k
 * desc, T, Tq) bytes (16-byte aligned), the call may split the history range
 * into up to 4 sub-ranges processed by separate CTAs when that fills the GPU
 * better, writing binary32 partial results to the workspace and merging them
 * by LSE as kvq_lse_merge does.  With NULL / 0 it runs unsplit.
 */
KVQ_API kvq_status kvq_attention_lse(const void *q, int64_t num_queries, const kvq_compressed_view *k,
                             const kvq_compressed_view *v, int64_t t_begin, int64_t t_end, float softmax_scale,
                             void *o_out, kvq_dtype o_dtype, float *lse_out, void *workspace,
                             size_t workspace_bytes, kvq_stream_t stream);

/*
 * PSAC coefficients of a compressed K history (QuantWM: Temporally Consistent
 * 2-Bit KV Cache Quantization for Video World Models, Sec. 4.2, principal
 * query-subspace attention correction; rank 8 as in its Table 9):
 *   C[h][t] = (k_t - k^_t) U_h   for every token t < num_tokens, head h,
 * k the original keys, k^ their reconstruction from `k` (the value
 * kvq_decode writes in binary32), U_h [d][8] the head's basis: the leading
 * eigenvectors of its query second-moment matrix, computed by the caller
 * from the model's queries.  Per token-head: e_c = k_c - k^_c in binary32,
 * each C_r accumulated by binary32 FMAs in channel order.
 *   k       per-head codec view (joint_rank = 0; KVQ_ERR_UNSUPPORTED
 *           otherwise), d in {64, 128}, either {s, z} format;
 *   x       [T][H][d] original keys, float or bf16 (x_dtype), 16-byte aligned;
 *   U       [H][d][8] float, 16-byte aligned;  rank must be 8
 *           (KVQ_ERR_UNSUPPORTED otherwise);
 *   coef_out [H][T][8] float, 16-byte aligned (caller-owned, 32 bytes per
 *           token-head: the stored cost of the correction).
 * An index past C sets KVQ_ERR_INVALID_ARG in the device status word (centre
 * 0 is used).  T = 0 returns KVQ_OK without touching memory.
 */
KVQ_API kvq_status kvq_psac_coefficients(const kvq_compressed_view *k, const void *x, kvq_dtype x_dtype,
                                         const float *U, int32_t rank, float *coef_out, kvq_stream_t stream);

/*
 * kvq_attention_lse with PSAC's corrected logits (QuantWM, Sec. 4.2):
 *   s_ij = scale (q_i . k^_j + (q_i U_h) . C_j) = scale q_i . (k^_j + U_h C_j),
 * evaluated as attention over the corrected keys: the kernel adds
 * sum_r U_h[c][r] C_j[r] (binary32) to every rebuilt key value before it
 * splits the key into its bf16 high and low parts; everything else is as in
 * kvq_attention_lse.  U [H][128][8] and coef [H][T][8] float (as written by
 * kvq_psac_coefficients for the same K history), both 16-byte aligned; rank
 * must be 8 and d 128 (KVQ_ERR_UNSUPPORTED otherwise, also when H T or H C
 * reaches 2^31).  Workspace as for kvq_attention_lse.
 */
KVQ_API kvq_status kvq_attention_psac_lse(const void *q, int64_t num_queries, const kvq_compressed_view *k,
                                          const kvq_compressed_view *v, const float *U, const float *coef,
                                          int32_t rank, int64_t t_begin, int64_t t_end, float softmax_scale,
                                          void *o_out, kvq_dtype o_dtype, float *lse_out, void *workspace,
                                          size_t workspace_bytes, kvq_stream_t stream);

/*
 * NanoKV-Fast low-dimensional history attention (NanoKV page, abstract,
 * Fig. 4(a,d); per-head attention dims, Table 6): for each head h with its
 * low dim d_low,
 *   q_low = bf16(q_h P_h)                  queries reduced into the low space
 *                                           (binary64 sums, correctly rounded
 *                                           to bf16: RNE of the exact sum);
 *   s_ij  = scale q_low,i . k_low,j         scale = softmax_scale if > 0, else
 *                                           1/sqrt(d): the FULL head dimension;
 *   o_low = softmax_j(s) v_low,  lse = ln sum_j exp(s_ij)  (as
 *           kvq_attention_dense_lse, binary32 partials);
 *   o_h   = o_low R_h                       restored to d channels (binary32).
 *   q      [Tq][H][d] bf16;
 *   k_low, v_low [num_keys][H][d_low] bf16: the history decoded straight into
 *           the low space -- kvq_decode of a joint view whose head_dim is
 *           d_low, whose centres are mu_h P_h and whose w_dec holds the folded
 *           decoder W_dec,h P_h (per branch; the V branch folds its own maps);
 *   P      [H][d][d_low] bf16 (query maps), R [H][d_low][d] bf16 (output maps);
 *   o_out  [Tq][H][d] (o_dtype);  lse_out [H][Tq] float (natural log).
 * d, d_low in {64, 128}, d_low <= d (KVQ_ERR_UNSUPPORTED otherwise; heads at
 * 32 or 96 dims run at 64 or 128 with zero-padded maps).  Keys
 * [t_begin, t_end) of the history; all pointers 16-byte aligned.
 * Workspace (required): at least the q_low and o_low buffers, 6 Tq H d_low
 * bytes rounded up; with kvq_fast_attention_workspace_size() bytes the
 * attention may also split the key range as kvq_attention_lse does.
 */
KVQ_API kvq_status kvq_fast_attention_lse(const void *q, int64_t num_queries, const void *k_low, const void *v_low,
                                          int64_t num_keys, int32_t num_heads, int32_t head_dim, int32_t d_low,
                                          const void *P, const void *R, int64_t t_begin, int64_t t_end,
                                          float softmax_scale, void *o_out, kvq_dtype o_dtype, float *lse_out,
                                          void *workspace, size_t workspace_bytes, kvq_stream_t stream);

/* Workspace bytes for kvq_fast_attention_lse with room to split. */
KVQ_API kvq_status kvq_fast_attention_workspace_size(int32_t num_heads, int32_t head_dim, int32_t d_low,
                                                     int64_t num_queries, size_t *bytes);

/*
 * Dense-mode attention: the same computation as kvq_attention_lse over keys
 * [t_begin, t_end) of UNCOMPRESSED bf16 keys and values -- the current
 * chunk's own keys, or raw protected history tokens such as attention sinks
 * and a recent window (NanoKV page, Table 4: protection keeps extra
 * historical tokens uncompressed) -- so that its partial result can be merged
 * with the compressed history's by LSE (NanoKV page, Fig. 4(d)).
 *   q [Tq][H][d] bf16;  k, v [num_keys][H][d] bf16 (may be NULL when the
 *   range is empty);  o_out [Tq][H][d] (o_dtype);  lse_out [H][Tq] float.
 * Logits are exact bf16 products accumulated in binary32 (no lo part); v is
 * widened to fp16 for the tensor cores (exact for |v| in [2^-14, 65504];
 * larger magnitudes saturate) and P is rounded to fp16, as in
 * kvq_attention_lse.  No mask: every query sees every key of the range.
 * d in {64, 128} (KVQ_ERR_UNSUPPORTED otherwise); all pointers 16-byte
 * aligned.  Workspace: optional, as for kvq_attention_lse, sized by
 * kvq_workspace_size(KVQ_OP_ATTENTION, desc with this H and d, 0, Tq).
 */
KVQ_API kvq_status kvq_attention_dense_lse(const void *q, int64_t num_queries, const void *k, const void *v,
                                           int64_t num_keys, int32_t num_heads, int32_t head_dim, int64_t t_begin,
                                           int64_t t_end, float softmax_scale, void *o_out, kvq_dtype o_dtype,
                                           float *lse_out, void *workspace, size_t workspace_bytes,
                                           kvq_stream_t stream);

/*
 * Full-layer attention of the current chunk: its queries attend to history
 * tokens [t_begin, t_end) of a compressed K and V (per-head codec, as in
 * kvq_attention_lse) AND to num_cur uncompressed bf16 keys and values (the
 * chunk itself, plus any raw protected tokens the caller places there), with
 * one softmax over all of them:
 *   o_i = sum_j softmax(s_i)_j v_j over both key sets, lse_i = ln sum_j exp(s_ij).
 * Computed as two partial attentions (compressed and dense) written as
 * binary32 partials to the workspace and merged by LSE (NanoKV page,
 * Fig. 4(a,d)).
 *   q [Tq][H][d] bf16; k_cur, v_cur [num_cur][H][d] bf16 (NULL allowed when
 *   num_cur = 0); o_out [Tq][H][d] (o_dtype); lse_out [H][Tq] float.
 * If both key sets are empty, o = 0 and lse = -inf.
 * Workspace (required, 16-byte aligned): at least
 * kvq_workspace_size(KVQ_OP_LAYER_ATTENTION, k_hist desc, T, Tq) bytes, else
 * KVQ_ERR_WORKSPACE.  Other requirements as for kvq_attention_lse.
 */
KVQ_API kvq_status kvq_layer_attention(const void *q, int64_t num_queries, const kvq_compressed_view *k_hist,
                                       const kvq_compressed_view *v_hist, int64_t t_begin, int64_t t_end,
                                       const void *k_cur, const void *v_cur, int64_t num_cur, float softmax_scale,
                                       void *o_out, kvq_dtype o_dtype, float *lse_out, void *workspace,
                                       size_t workspace_bytes, kvq_stream_t stream);

/*
 * Merge n partial attention results over disjoint history parts by their
 * log-sum-exp (NanoKV page, Fig. 4(d)):
 *   m = max_b lse_b;  lse = m + ln sum_b exp(lse_b - m);
 *   o = sum_b exp(lse_b - lse) o_b;  parts with lse_b = -inf weigh 0; if all
 *   parts are empty, o = 0 and lse = -inf.
 *   o_parts / lse_parts: HOST arrays of n (1..64) DEVICE pointers to
 *   o_b [Tq][H][d] float and lse_b [H][Tq] float.
 *   o_out [Tq][H][d] (o_dtype), lse_out [H][Tq] float.  The outputs must not
 *   overlap any part.
 */
KVQ_API kvq_status kvq_lse_merge(int32_t n_parts, const float *const *o_parts, const float *const *lse_parts,
                         int64_t num_queries, int32_t num_heads, int32_t head_dim, void *o_out,
                         kvq_dtype o_dtype, float *lse_out, kvq_stream_t stream);

/*
 * Test hook for the give-up path of the bounded waits.  Sets, for the current
 * device, how many times a waiting role of the encode filter (kvq_encode with
 * a bf16 history and C <= 512, the fit's assignment passes) and of the d = 128
 * attention kernels (kvq_attention_lse, kvq_attention_psac_lse, the dense and
 * full-layer attention) polls an mbarrier before it gives up, raising
 * KVQ_ERR_DEVICE_TIMEOUT in the status word and stopping the kernel's work
 * (its outputs are then undefined).  KVQ_WAIT_LIMIT_DEFAULT (the value at load
 * time, a wait of well under a few seconds) restores normal operation; 0 makes
 * every such wait give up at once.  Waits that drain the kernel's own copies
 * and tensor-core work before it exits are not affected.  Synchronous; applies
 * to kernels launched afterwards.
 */
#define KVQ_WAIT_LIMIT_DEFAULT 4194304u
KVQ_API kvq_status kvq_set_wait_limit(uint32_t polls);

/*
 * Synchronise `stream`, then read and clear this device's status word.
 * Returns KVQ_ERR_DEVICE_TIMEOUT if any kernel since the last read gave up a
 * bounded wait (its outputs are then undefined), KVQ_ERR_CUDA if the stream
 * reports an error, else KVQ_OK.
 */
KVQ_API kvq_status kvq_last_device_status(kvq_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* KVQ_H_ */

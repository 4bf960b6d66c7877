/*
 * sharq.h - C ABI of the SharQ per-linear-layer hot path for NVIDIA B200
 * (sm_100a).
 *
 * Method: "SharQ: Bridging Activation Sparsity and FP4 Quantization for LLM
 * Inference" (arXiv 2606.26587), Abstract. Each activation tensor goes
 * through one fused preparation operator: LayerNorm; a per-row N:M mask,
 * chosen from the data, that keeps a sparse backbone S of the large
 * (outlier) values; FP4 quantization of S; the dense residual
 * R = X_ln - deq(Q(S)), measured from the quantized backbone; and FP4
 * quantization of R. A sparse FP4 GEMM on Q(S) and a dense FP4 GEMM on Q(R)
 * use the same FP4 weight codes, each with a scale view of its own, and
 * their results are added.
 *
 * Formats: SHARQ_NVFP4 = E2M1 codes, one UE4M3 scale per 16 elements and one
 * fp32 tensor scale; SHARQ_MXFP4 = E2M1 codes and one E8M0 scale per 32
 * elements (OCP Microscaling Formats v1.0).
 *
 * Conventions for every entry point:
 *  - Pointers named *_dev are device pointers (cudaMalloc / torch CUDA
 *    memory) of the current device; pointers named *_host are host memory.
 *  - The caller owns all memory. The library never allocates device memory:
 *    size queries say how many bytes a buffer needs, and handles
 *    (sharq_wq, sharq_prep) are plain descriptors that point into the
 *    caller's buffers. They stay valid as long as those buffers do.
 *  - `stream` is a cudaStream_t (NULL = legacy default stream). All work is
 *    enqueued asynchronously on it; only the *_export calls and
 *    sharq_get_last_error synchronize it.
 *  - Arguments are validated on the host before anything is enqueued; a
 *    violation returns SHARQ_ERR_INVALID_ARG (or SHARQ_ERR_UNSUPPORTED) and
 *    enqueues nothing. Device buffers must be 256-byte aligned.
 *  - Inputs must be finite. Non-finite inputs are not detected and give
 *    unspecified (but memory-safe) results.
 *  - Kernels that wait on the hardware bound every wait; a wait that runs
 *    out records a status that sharq_get_last_error reports as
 *    SHARQ_ERR_TIMEOUT.
 *  - Host threads may call the library concurrently (each with its own
 *    buffers and streams): its per-device caches are filled once under a
 *    lock. sharq_last_launch_count and sharq_last_timeout_site report the
 *    most recent call of any thread; the device status word and the
 *    no-allocation entry point's array are shared by all callers.
 */
#ifndef SHARQ_H
#define SHARQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum sharq_fmt {
    SHARQ_NVFP4 = 0, /* E2M1 + UE4M3 scale per 16 + fp32 tensor scale */
    SHARQ_MXFP4 = 1  /* E2M1 + E8M0 scale per 32 */
} sharq_fmt;

typedef enum sharq_status {
    SHARQ_OK = 0,
    SHARQ_ERR_INVALID_ARG = 1, /* a precondition below does not hold */
    SHARQ_ERR_UNSUPPORTED = 2, /* valid request this build does not serve */
    SHARQ_ERR_CUDA = 3,        /* a CUDA runtime/driver call failed */
    SHARQ_ERR_TIMEOUT = 4      /* a bounded device-side wait ran out */
} sharq_status;

/* Shape limits. k must be a multiple of SHARQ_K_ALIGN (the GEMM's K tile)
 * and at most SHARQ_K_MAX; n_out must be a multiple of SHARQ_N_ALIGN. */
#define SHARQ_K_ALIGN 256
#define SHARQ_K_MAX 65536
#define SHARQ_N_ALIGN 32
/* Most segments of a fused weight (sharq_quantize_weight_fused). */
#define SHARQ_SEGMENTS_MAX 8

/*
 * Block-scale layout ("MMA scale view"). Scales of a [rows][k/blk] matrix
 * (blk = 16 for NVFP4, 32 for MXFP4) are stored in 512-byte atoms, each
 * holding 4 consecutive scales of 128 consecutive rows. The scale of row r,
 * block j is at byte
 *     ((r / 128) * (k / blk / 4) + j / 4) * 512
 *       + (r % 32) * 16 + ((r % 128) / 32) * 4 + (j % 4).
 * This is the order in which a 32-lane x 128-bit tensor-memory copy
 * delivers per-row scales to the block-scaled tcgen05 MMA. Rows are padded
 * to a multiple of 128 (activations) or 256 (weights) with zero scales.
 *
 * Code layout: E2M1 codes packed two per byte, row-major [rows][k/2];
 * element 2i in the low nibble, 2i+1 in the high nibble. Bit 3 of a code is
 * its sign, so -0 (code 8) is kept distinct from +0 (code 0).
 *
 * Mask metadata layout: per row, for each aligned group of m elements along
 * k, the n kept positions in ascending order, each ceil(log2 m) bits wide
 * (m = 2: 1 bit), concatenated LSB-first into a bit stream of
 * (k/m)*n*ceil(log2 m) bits; each row starts at a multiple of
 * meta_row_bytes = ceil(that / 8) bytes.
 */

/* Quantized weight: one E2M1 code payload that both GEMM paths read. The
 * backbone and the residual GEMM each see the scales through their own
 * scale view (scales + tensor_scale); both views hold the same values, as
 * the dequantized weight must be identical on both paths. */
typedef struct sharq_wq {
    int64_t n_out;       /* output features (rows of W) */
    int64_t k;           /* input features */
    int32_t fmt;         /* sharq_fmt */
    int32_t groups;      /* stacked weights (experts): 1 (0 reads as 1), or
                            n_groups from sharq_quantize_weight_grouped;
                            group g's payload is g * sharq_weight_bytes(n_out,
                            k, fmt) bytes after group 0's, which every pointer
                            refers to */
    int64_t sf_rows;     /* rows of the scale layout: n_out rounded up to 256 */
    void *codes;         /* device, [n_out][k/2] bytes */
    void *scales_backbone; /* device, MMA scale view for the backbone path */
    void *scales_residual; /* device, MMA scale view for the residual path */
    float *tensor_scale; /* device, 1 float: s_tW = amax(W)/2688 (NVFP4) or 1;
                            one float per segment for a fused weight */
    void *scratch;       /* device, library-internal words */
    int32_t segments;    /* fused weights: stacked segments along n_out, 1 (0
                            reads as 1) otherwise */
    int32_t seg_end[SHARQ_SEGMENTS_MAX]; /* exclusive end row of each segment */
    int32_t sparse;      /* 0: one scale per blk values; 1: the pair-wise
                            sparse mode's weight (sharq_quantize_weight_sparse):
                            one scale per 2 blk values */
} sharq_wq;

/* Prepared activation: outputs of the preparation operator. */
typedef struct sharq_prep {
    int64_t m_tok;       /* rows (tokens) */
    int64_t k;           /* input features */
    int32_t n, m;        /* N:M ratio of the mask */
    int32_t fmt;         /* sharq_fmt */
    int32_t groups;      /* 1 (0 reads as 1), or n_groups for the output of
                            sharq_gather_rows */
    int64_t sf_rows;     /* rows of the scale layouts: m_tok rounded up to 128 */
    int64_t meta_row_bytes;
    void *s_codes;       /* device, backbone Q(S) codes [m_tok][k/2] (zeros off the mask) */
    void *r_codes;       /* device, residual Q(R) codes [m_tok][k/2] */
    void *s_scales;      /* device, MMA scale view of Q(S) */
    void *r_scales;      /* device, MMA scale view of Q(R) */
    void *meta;          /* device, mask metadata [m_tok][meta_row_bytes] */
    float *tensor_scale; /* device, 1 float: s_t = amax(X_ln)/2688 (NVFP4) or 1 */
    void *scratch;       /* device, per-row statistics and reduction words */
    int32_t sparse;      /* 0: element-wise n:m mask, backbone codes stored
                            dense; 1: pair-wise 4:8 mode (sharq_prepare_sparse) */
} sharq_prep;

/* Bytes of the device buffer sharq_quantize_weight needs. 0 if the shape or
 * format is invalid. */
size_t sharq_weight_bytes(int64_t n_out, int64_t k, int fmt);

/* Bytes of the device buffer sharq_prepare needs. 0 if invalid. */
size_t sharq_prep_bytes(int64_t m_tok, int64_t k, int n, int m, int fmt);

/*
 * Weight quantization (offline). SharQ, Abstract: both GEMM paths read one
 * FP4 weight payload, each through a scale view of its own.
 *   w_dev    fp16 [n_out][k] row-major (K-major), so the layer computes X W^T.
 *   wq_dev   device buffer of at least sharq_weight_bytes(n_out, k, fmt).
 *   wq_out   host struct, filled with pointers into wq_dev.
 * NVFP4: s_tW = RN32(amax|W| / 2688) (1 if W == 0); each 16-element block
 * gets UE4M3 scale RN-satfinite(amax_blk / RN32(6 s_tW)) and codes
 * E2M1(RN32(w / RN32(scale * s_tW))). MXFP4: E8M0 exponent
 * floor(log2 amax_blk) - 2 per 32-element block and codes E2M1(w / 2^e).
 * Preconditions: n_out >= 1, n_out % SHARQ_N_ALIGN == 0, k % SHARQ_K_ALIGN
 * == 0, 0 < k <= SHARQ_K_MAX, fmt valid, pointers non-NULL and aligned.
 */
sharq_status sharq_quantize_weight(const void *w_dev, int64_t n_out, int64_t k, int fmt,
                                   void *wq_dev, size_t wq_bytes, sharq_wq *wq_out,
                                   void *stream);

/*
 * Fused preparation operator (per activation). SharQ, Abstract: LayerNorm,
 * mask generation and residual construction are done by one fused operator.
 *   x_dev     fp16 [m_tok][k] row-major activations.
 *   ln_w_dev  fp16 [k] LayerNorm gamma, or NULL (no multiply).
 *   ln_b_dev  fp16 [k] LayerNorm beta, or NULL (no add; -0 is preserved).
 *   eps       LayerNorm epsilon, finite and > 0.
 *   n, m      keep the n largest |X_ln| of every aligned group of m along k
 *             (equal magnitudes: lower index first); m in {2,4,8,16},
 *             1 <= n <= m.
 *   prep_dev  device buffer of at least sharq_prep_bytes(...).
 *   prep_out  host struct, filled with pointers into prep_dev.
 * Steps, each an IEEE binary32 operation rounded to nearest even:
 *   LayerNorm with statistics from exact integer sums: mu = RN32(S1/K),
 *   rstd = RN32(1/sqrt(var + eps)) in binary64 from D = K*S2 - S1^2;
 *   X_ln = RN32(RN32(RN32(x - mu) * rstd) * gamma) + beta;
 *   s_t = RN32(amax|X_ln| / 2688) (1 if zero; MXFP4: 1);
 *   S = X_ln on the mask, +0 elsewhere; Q(S) block-quantized as for weights;
 *   R = RN32(X_ln - deq(Q(S))), deq = RN32(E2M1 value * RN32(scale * s_t));
 *   Q(R) block-quantized with the same s_t.
 * m_tok == 0 is valid and enqueues nothing but the tensor scale (1).
 */
sharq_status sharq_prepare(const void *x_dev, int64_t m_tok, int64_t k,
                           const void *ln_w_dev, const void *ln_b_dev, float eps,
                           int n, int m, int fmt,
                           void *prep_dev, size_t prep_bytes, sharq_prep *prep_out,
                           void *stream);

/*
 * The preparation operator with RMSNorm in place of LayerNorm: the form the
 * evaluated model families (Llama, Qwen) normalize with. An interface
 * addition: the SharQ abstract names layer normalization only. Statistics
 * from the same exact integer sums, without centring:
 *   ms = RN64(S2) / (K 2^48), rstd = RN32(1/sqrt(ms + eps)) in binary64,
 *   X_n = RN32(RN32(x * rstd) * w)
 * then the mask, Q(S), R and Q(R) exactly as sharq_prepare. The exported
 * mu is 0.
 *   w_dev  fp16 [k] RMSNorm weight, or NULL (no multiply).
 * Everything else (arguments, buffer, preconditions) as sharq_prepare.
 */
sharq_status sharq_prepare_rms(const void *x_dev, int64_t m_tok, int64_t k, const void *w_dev, float eps,
                               int n, int m, int fmt, void *prep_dev, size_t prep_bytes, sharq_prep *prep_out,
                               void *stream);

/*
 * The preparation operator fused with the operation that produces its input.
 * SharQ, Abstract: one fused operator absorbs the layer normalization; in a
 * pre-norm transformer the normalization's input is the residual stream
 * right after the add x = h + d (h the residual stream, d the output of the
 * previous attention or MLP block). This call performs that add and takes
 * x's normalization statistics and tensor amax in the same pass, so that
 * the encode pass is the only other read of x (sharq_prepare on a stored x
 * reads it twice):
 *   x_out[i] = RN16(h[i] + d[i])   (binary16 addition, round to nearest even;
 *                                   a sum beyond 65504 gives +-inf, which the
 *                                   preparation's finiteness precondition
 *                                   then excludes)
 * then exactly what sharq_prepare (norm = 0) or sharq_prepare_rms (norm = 1,
 * ln_b NULL) computes on x_out, bit for bit.
 *   h_dev, d_dev  fp16 [m_tok][k], 16-byte aligned.
 *   x_out_dev     fp16 [m_tok][k]: may be h_dev itself (the residual stream
 *                 updated in place); must not otherwise overlap h or d.
 * Other arguments and preconditions as sharq_prepare; prep_bytes >=
 * sharq_prep_bytes(m_tok, k, n, m, fmt).
 */
sharq_status sharq_prepare_add(const void *h_dev, const void *d_dev, void *x_out_dev, int64_t m_tok, int64_t k,
                               const void *ln_w_dev, const void *ln_b_dev, float eps, int norm, int n, int m, int fmt,
                               void *prep_dev, size_t prep_bytes, sharq_prep *prep_out, void *stream);

/*
 * Preparation operator for callers that cannot allocate device memory.
 * (An interface addition: the SharQ paper has no counterpart.)
 *
 * sharq_prepare keeps its working memory (per-row LayerNorm statistics and
 * the word that collects the tensor's amax) inside the caller's prep buffer.
 * Some callers cannot provide that: a plugin or custom operator inside
 * another framework is handed its input and output tensors and owns no
 * allocator; code on a latency-critical path must not call cudaMalloc,
 * which waits for the device to go idle; and deployments that plan all
 * device memory ahead of time have no room for a per-call scratch region.
 * This entry point computes exactly what sharq_prepare computes (the same
 * results bit for bit; its statistics always come from the one-CTA-per-row
 * kernel, whose exact sums sharq_prepare's other statistics kernels equal)
 * but keeps that working memory in one
 * fixed array compiled into the library: 256 + 8 * SHARQ_NOALLOC_MAX_ROWS
 * bytes (about 128 KB) on every GPU that loads the library, held until the
 * process exits. It calls no allocator.
 *
 *   x_dev, m_tok, k, ln_w_dev, ln_b_dev, eps, n, m, fmt: as sharq_prepare.
 *   Outputs (device, 256-byte aligned, sizes in bytes; blk = 16 for NVFP4,
 *   32 for MXFP4; sf_rows = m_tok rounded up to 128, at least 128):
 *     s_codes_dev, r_codes_dev   m_tok * k / 2 each (code layout above)
 *     s_scales_dev, r_scales_dev sf_rows * k / blk each (MMA scale view)
 *     meta_dev                   m_tok * ceil((k/m) * n * ceil(log2 m) / 8)
 *     s_t_dev                    1 float (4-byte aligned)
 *   prep_out  host struct for sharq_linear / sharq_prep_export; its scratch
 *             pointer refers to the library's array.
 * Limits and sharing: m_tok <= SHARQ_NOALLOC_MAX_ROWS, else
 * SHARQ_ERR_UNSUPPORTED and nothing is enqueued. All calls share the one
 * array, which keeps the last call's contents (the statistics that
 * sharq_prep_export returns for prep_out are those of the latest call on the
 * device); the amax word is cleared at the start of every call. Calls whose
 * work overlaps on the GPU (different streams, no ordering between them)
 * race on the array and give wrong results. The first call on a device looks
 * up the array's device address with the device current; make that first
 * call before any stream capture.
 */
#define SHARQ_NOALLOC_MAX_ROWS 16384
sharq_status sharq_prepare_noalloc(const void *x_dev, int64_t m_tok, int64_t k,
                                   const void *ln_w_dev, const void *ln_b_dev, float eps,
                                   int n, int m, int fmt,
                                   void *s_codes_dev, void *r_codes_dev,
                                   void *s_scales_dev, void *r_scales_dev,
                                   void *meta_dev, float *s_t_dev,
                                   sharq_prep *prep_out, void *stream);

/*
 * Pair-wise 4:8 sparse-backbone mode. SharQ, Abstract: "A sparse FP4 GEMM
 * processes the backbone". The tensor cores' structured-sparse block-scaled
 * FP4 MMA (tcgen05.mma.sp, kind::mxf4nvf4 / kind::mxf4) accepts one
 * pattern: in every aligned group of 8 values along k, two of the four
 * adjacent pairs (2j, 2j+1) hold the non-zeros; and it applies one scale per
 * 32 logical values (NVFP4) or 64 (MXFP4) along k to both operands. This
 * opt-in mode makes the backbone match that pattern, so that the backbone
 * GEMM runs at the sparse tensor-core rate on half of K:
 *   mask   in every aligned group of 8, the two pairs with the largest
 *          max(|x_2j|, |x_2j+1|) of X_ln (equal: the lower pair);
 *   Q(S)   blocks of 32 (NVFP4) / 64 (MXFP4) values: the 16 / 32 kept
 *          values of a block quantized exactly like a block of the format;
 *   R, Q(R) as sharq_prepare (blocks of 16 / 32);
 *   W      one code payload with blocks of 32 / 64 (sharq_quantize_weight_
 *          sparse): the backbone path reads one scale per 32 / 64 values,
 *          the residual path the same scale for each half block, so deq(W)
 *          is the same on both paths.
 * The element-wise n:m mask of sharq_prepare is a different mask (it is not
 * pair-wise in general), so the two modes give different results.
 *
 * Layouts in the prep buffer (sparse = 1, n = 4, m = 8):
 *   s_codes  [m_tok][k/4] bytes: per group of 8, the four kept codes in
 *            order (first pair's two, then the second's), two per byte.
 *   s_scales MMA scale view with one scale per 32 (64) values.
 *   meta     [m_tok][k/16] bytes: per group g of a row, bits 4g .. 4g+3 hold
 *            first | second << 2 (the kept pairs' indices, ascending); the
 *            layout the sparse MMA reads.
 *   r_codes, r_scales as sharq_prepare.
 * sharq_prep_export returns the canonical forms: idx [m_tok][k/8][4] kept
 * positions, s_codes [m_tok][k] (+0 off the mask), s_scales
 * [m_tok][k/32] (NVFP4) or [m_tok][k/64] (MXFP4).
 */
size_t sharq_prep_bytes_sparse(int64_t m_tok, int64_t k, int fmt);

/*   norm  0: LayerNorm (ln_w, ln_b as sharq_prepare); 1: RMSNorm (ln_w as
 *         sharq_prepare_rms, ln_b must be NULL).
 * Other arguments, preconditions and the statistics as sharq_prepare;
 * prep_bytes >= sharq_prep_bytes_sparse(m_tok, k, fmt). */
sharq_status sharq_prepare_sparse(const void *x_dev, int64_t m_tok, int64_t k, const void *ln_w_dev,
                                  const void *ln_b_dev, float eps, int norm, int fmt, void *prep_dev,
                                  size_t prep_bytes, sharq_prep *prep_out, void *stream);

/* The weight of the pair-wise mode: as sharq_quantize_weight with blocks of
 * 32 (NVFP4) or 64 (MXFP4) values; wq_out->sparse = 1. sharq_weight_export
 * returns the backbone view as [n_out][k/32] ([n_out][k/64]) and the
 * residual view as [n_out][k/16] ([n_out][k/32]), every scale twice. */
size_t sharq_weight_bytes_sparse(int64_t n_out, int64_t k, int fmt);
sharq_status sharq_quantize_weight_sparse(const void *w_dev, int64_t n_out, int64_t k, int fmt, void *wq_dev,
                                          size_t wq_bytes, sharq_wq *wq_out, void *stream);

/*
 * Dual-path FP4 linear layer. SharQ, Abstract: the backbone goes through a
 * sparse FP4 GEMM, and a dense FP4 GEMM on the residual makes up both for
 * what the mask dropped and for the backbone's quantization error.
 *   out_dev  fp16 [m_tok][n_out] row-major:
 *     out = RN16( s_t * s_tW * sum_k (Q(S) + Q(R))[i,k] * Q(W)[j,k] )
 *   with the block-scaled code values; products are exact, accumulation is
 *   fp32 in tensor memory (both paths into one accumulator).
 * Preconditions: prep and wq from this library, prep->fmt == wq->fmt,
 * prep->k == wq->k, out_dev non-NULL (may be NULL only if m_tok == 0) and at
 * least 32-byte aligned (the epilogue writes whole 32-byte sectors).
 * A pair-wise-mode prep (sharq_prepare_sparse) needs a pair-wise-mode weight
 * (sharq_quantize_weight_sparse) and the reverse (SHARQ_ERR_INVALID_ARG
 * otherwise); its backbone then runs through the structured-sparse MMA on
 * the K-compacted codes. That mode takes no bias and no fused or grouped
 * weights (SHARQ_ERR_UNSUPPORTED).
 */
sharq_status sharq_linear(const sharq_prep *prep, const sharq_wq *wq, void *out_dev,
                          void *stream);

/*
 * Fused projections: weights that read the same prepared activation (q, k
 * and v of attention; gate and up of a gated MLP), stacked along n_out into
 * one payload so that one linear computes all of them. An interface
 * addition: the SharQ abstract describes one linear at a time. Each segment
 * is quantized on its own (its own tensor scale s_tW[g], block scales and
 * codes exactly as sharq_quantize_weight gives for that weight alone), so
 * every output column of the fused linear equals the column of the separate
 * linear bit for bit.
 *   w_dev     fp16 [sum seg_rows][k], the segments' rows one after another.
 *   seg_rows  host array of n_segs row counts, each >= 1 and a multiple of
 *             SHARQ_N_ALIGN; 1 <= n_segs <= SHARQ_SEGMENTS_MAX.
 *   wq_dev    device buffer of at least sharq_weight_bytes_fused(...) bytes
 *             (the same as sharq_weight_bytes of the stacked shape).
 * wq_out describes one weight of n_out = sum seg_rows rows with
 * segments = n_segs, seg_end[g] = rows of segments 0..g, and tensor_scale
 * pointing at n_segs floats.
 */
size_t sharq_weight_bytes_fused(const int64_t *seg_rows, int n_segs, int64_t k, int fmt);
sharq_status sharq_quantize_weight_fused(const void *w_dev, const int64_t *seg_rows, int n_segs, int64_t k,
                                         int fmt, void *wq_dev, size_t wq_bytes, sharq_wq *wq_out,
                                         void *stream);

/*
 * The dual-path linear with a bias (Qwen2.5's q, k and v projections have
 * one): column j of segment g is
 *     out = RN16( RN32( RN32(acc * RN32(s_t * s_tW[g])) + bias[j] ) )
 * with acc the fp32 accumulator of sharq_linear. bias_dev: fp16 [n_out],
 * 16-byte aligned, or NULL (then the result equals sharq_linear's).
 * sharq_linear accepts fused weights too (no bias). Preconditions as
 * sharq_linear.
 */
sharq_status sharq_linear_bias(const sharq_prep *prep, const sharq_wq *wq, const void *bias_dev, void *out_dev,
                               void *stream);

/* The tensor scales of a weight's segments (one float each) to the host.
 * Synchronizes `stream`. s_tw_host holds at least wq->segments floats. */
sharq_status sharq_weight_tensor_scales(const sharq_wq *wq, float *s_tw_host, void *stream);

/*
 * Mixture-of-experts grouped variant.
 *
 * The SharQ Abstract lists Qwen3-30B-A3B, a mixture-of-experts model, among
 * the evaluated models but does not say how expert layers are computed. The
 * reading taken here: each expert's linear is the dual-path linear above,
 * applied to the rows (tokens) routed to that expert; an activation tensor
 * is prepared ONCE over all its rows, so one tensor scale s_t covers every
 * row of every expert; each expert's weight is quantized on its own (its
 * own s_tW). Three calls:
 *   sharq_quantize_weight_grouped  the experts' weights, stacked
 *   sharq_gather_rows              prepared rows -> expert-grouped order
 *   sharq_linear_grouped           one launch over all experts' tiles
 *
 * Routing is given by device arrays, so that it can come from a router
 * kernel without a host round trip:
 *   offsets_dev  int32 [n_groups + 1]: offsets[0] = 0, nondecreasing,
 *                offsets[n_groups] = rows. Grouped rows offsets[g] ..
 *                offsets[g+1]-1 belong to group (expert) g.
 *   row_idx_dev  int32 [rows]: grouped row i is prepared row row_idx[i].
 * The kernels check these on the device. On a violation they write no
 * output, and sharq_get_last_error then reports SHARQ_ERR_INVALID_ARG.
 */
#define SHARQ_GROUPS_MAX 1024

/* Bytes of the buffer sharq_quantize_weight_grouped needs:
 * n_groups * sharq_weight_bytes(n_out, k, fmt). 0 if invalid. */
size_t sharq_weight_bytes_grouped(int64_t n_groups, int64_t n_out, int64_t k, int fmt);

/* Quantizes n_groups weights in one call, each exactly as
 * sharq_quantize_weight would (its own tensor scale and block scales).
 *   w_dev   fp16 [n_groups][n_out][k] row-major.
 *   wq_out  host struct describing group 0, with groups = n_groups.
 * Preconditions: 1 <= n_groups <= SHARQ_GROUPS_MAX, plus those of
 * sharq_quantize_weight. */
sharq_status sharq_quantize_weight_grouped(const void *w_dev, int64_t n_groups, int64_t n_out, int64_t k,
                                           int fmt, void *wq_dev, size_t wq_bytes, sharq_wq *wq_out,
                                           void *stream);

/* Rows of a grouped prep. Each group starts at a multiple of 128 rows, so
 * that no 128-row GEMM tile spans two groups: rows + 127 * n_groups, rounded
 * up to 128. -1 if invalid. */
int64_t sharq_grouped_rows(int64_t rows, int64_t n_groups);

/* Bytes of the buffer sharq_gather_rows needs:
 * sharq_prep_bytes(sharq_grouped_rows(rows, n_groups), k, n, m, fmt). */
size_t sharq_gather_bytes(int64_t rows, int64_t n_groups, int64_t k, int n, int m, int fmt);

/*
 * Copies prepared rows into expert-grouped order. No arithmetic: the codes,
 * block scales, mask metadata and LayerNorm statistics of each row move bit
 * for bit, and the tensor scale is copied.
 *   src          a prep from sharq_prepare.
 *   row_idx_dev  as above; NULL means row_idx[i] = i (src already in
 *                grouped order, as a down projection's input is).
 *   offsets_dev, n_groups, rows: as above; 1 <= n_groups <=
 *                SHARQ_GROUPS_MAX, 0 <= rows <= 2^30.
 *   dst_dev      buffer of at least sharq_gather_bytes(...) bytes.
 *   dst_out      host struct: m_tok = sharq_grouped_rows(rows, n_groups),
 *                groups = n_groups. Grouped row i of group g is stored at
 *                row 128 * T_g + (i - offsets[g]), where T_g counts the
 *                128-row tiles of groups 0 .. g-1 (ceil(size / 128) each).
 *                Every other row is zero (codes, scales, metadata and
 *                statistics).
 * Device-side checks: the offsets as above, and 0 <= row_idx[i] < src->m_tok.
 */
sharq_status sharq_gather_rows(const sharq_prep *src, const int32_t *row_idx_dev, const int32_t *offsets_dev,
                               int64_t n_groups, int64_t rows, void *dst_dev, size_t dst_bytes,
                               sharq_prep *dst_out, void *stream);

/*
 * Grouped dual-path FP4 linear: for every group g and grouped row i of g,
 *   out[i][j] = RN16( s_t * s_tW[g] * sum_k (Q(S) + Q(R))[i,k] * Q(W_g)[j,k] )
 * with the terms of sharq_linear. One persistent launch walks the 128 x 256
 * output tiles of all groups.
 *   prep     from sharq_gather_rows with the same offsets and n_groups.
 *   wq       from sharq_quantize_weight_grouped with groups == n_groups.
 *   out_dev  fp16 [rows][n_out] row-major, grouped order.
 * Preconditions: those of sharq_linear, plus prep->groups == wq->groups ==
 * n_groups and rows <= prep->m_tok. Device-side checks: the offsets, and
 * that the rows they pad to fit in prep->m_tok.
 */
/*
 * Preparation straight into the grouped layout, for an activation whose rows
 * are already in grouped order (the input of a mixture-of-experts down
 * projection: the output of the grouped gate/up linears and the activation
 * function). An interface addition. Equal, in codes, scales, mask metadata
 * and tensor scale, to sharq_gather_rows(prepare(x), NULL, offsets) bit for
 * bit, in one preparation pass instead of a preparation and a gather.
 *   x_dev        fp16 [rows][k], rows in grouped order (group g's rows are
 *                offsets[g] .. offsets[g+1] - 1).
 *   offsets_dev  int32 [n_groups + 1], device: offsets[0] = 0, ascending,
 *                offsets[n_groups] = rows; checked on the device (invalid
 *                offsets leave the output untouched and set the status that
 *                sharq_get_last_error reports).
 *   norm         0: LayerNorm (ln_w, ln_b as sharq_prepare); 1: RMSNorm
 *                (ln_w as sharq_prepare_rms, ln_b must be NULL).
 *   prep_dev     at least sharq_gather_bytes(rows, n_groups, k, n, m, fmt)
 *                bytes.
 * prep_out describes a grouped prep of sharq_grouped_rows(rows, n_groups)
 * rows (groups = n_groups) for sharq_linear_grouped; its per-row statistics
 * are indexed by source row. Other preconditions as sharq_prepare.
 */
sharq_status sharq_prepare_grouped(const void *x_dev, int64_t rows, int64_t k, const int32_t *offsets_dev,
                                   int64_t n_groups, const void *ln_w_dev, const void *ln_b_dev, float eps, int norm,
                                   int n, int m, int fmt, void *prep_dev, size_t prep_bytes, sharq_prep *prep_out,
                                   void *stream);

sharq_status sharq_linear_grouped(const sharq_prep *prep, const int32_t *offsets_dev, int64_t n_groups,
                                  int64_t rows, const sharq_wq *wq, void *out_dev, void *stream);

/*
 * Canonical host copies of a prepared activation, for inspection and tests.
 * Synchronizes `stream`. Every output may be NULL. One value per byte:
 *   idx_host      [m_tok][k/m][n] kept positions, ascending
 *   s_codes_host  [m_tok][k]      Q(S) codes (0..15)
 *   s_scales_host [m_tok][k/blk]  Q(S) scale codes
 *   r_codes_host, r_scales_host   same for Q(R)
 *   mu_host, rstd_host [m_tok]    LayerNorm statistics (float)
 *   s_t_host      1 float
 */
sharq_status sharq_prep_export(const sharq_prep *prep, uint8_t *idx_host,
                               uint8_t *s_codes_host, uint8_t *s_scales_host,
                               uint8_t *r_codes_host, uint8_t *r_scales_host,
                               float *mu_host, float *rstd_host, float *s_t_host,
                               void *stream);

/* Canonical host copies of a quantized weight. Synchronizes `stream`.
 *   codes_host [n_out][k], scales_host [n_out][k/blk] (backbone view),
 *   scales_residual_host [n_out][k/blk] (residual view), s_tw_host 1 float. */
sharq_status sharq_weight_export(const sharq_wq *wq, uint8_t *codes_host,
                                 uint8_t *scales_host, uint8_t *scales_residual_host,
                                 float *s_tw_host, void *stream);

/* Synchronizes `stream`, then reports (and clears) the device status word:
 * SHARQ_ERR_TIMEOUT if a bounded wait ran out since the last call,
 * SHARQ_ERR_INVALID_ARG if a device-side argument check failed (grouped
 * routing arrays), SHARQ_ERR_CUDA if the stream holds a CUDA error, else
 * SHARQ_OK. The first such event since the last call is the one reported. */
sharq_status sharq_get_last_error(void *stream);

/* Where the last SHARQ_ERR_TIMEOUT or device-side SHARQ_ERR_INVALID_ARG
 * came from (an internal site code; 0x2xx = argument checks), 0 if none.
 * Valid after sharq_get_last_error returned one of them. */
uint32_t sharq_last_timeout_site(void);

/* Test hook: the wait limit of the GEMM's bounded waits, in nanoseconds
 * (default 2e9). 0 restores the default. Returns the previous value. */
uint64_t sharq_set_wait_limit_ns(uint64_t ns);

/* Failure-detection self-test: enqueues one CTA whose single thread waits,
 * with the library's bounded wait, on a barrier that nothing ever arrives
 * at. After limit_ns (1 .. 1e10) the wait gives up and records site 0x1FF;
 * the kernel returns normally and the context stays usable. A following
 * sharq_get_last_error must report SHARQ_ERR_TIMEOUT. */
sharq_status sharq_selftest_wait(uint64_t limit_ns, void *stream);

/* Self-test of the quantizer's division: the encode kernels divide by a
 * block step d with a reciprocal and two fused multiply-add corrections
 * (Markstein's method), which must equal the correctly rounded quotient.
 * Runs `count` operand pairs drawn from `seed` (divisors in [2^-90, 2^90],
 * quotients of exponent -30 .. 30, many near the E2M1 rounding boundaries)
 * on the GPU and writes to *mismatches_host how many quotients of magnitude
 * >= 2^-4 differ from the hardware's correctly rounded division, plus how
 * many quotients of any size encode to a different E2M1 code (expected: 0). If examples_host is not NULL
 * it receives 16 x 4 floats: the first mismatching (dividend, divisor,
 * quotient, correctly rounded quotient) rows, zeros past the count.
 * Synchronizes `stream`. */
sharq_status sharq_selftest_division(uint64_t count, uint64_t seed, uint64_t *mismatches_host,
                                     float *examples_host, void *stream);

/* Human-readable status name (static string). */
const char *sharq_status_string(sharq_status s);

/* Number of kernel launches the last entry point enqueued (for launch
 * accounting in benchmarks). */
int sharq_last_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* SHARQ_H */

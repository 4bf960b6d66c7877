// Weight quantization (offline) of SharQ on sm_100a.
//
// "SharQ: Bridging Activation Sparsity and FP4 Quantization for LLM
// Inference", Abstract: both GEMM paths read the same FP4 weight codes, each
// through a scale view of its own. This kernel pair writes that payload: one
// E2M1 code matrix and one block-scale matrix in the tcgen05 MMA scale layout,
// which both paths' scale views point at (the same values, as the
// dequantized weight must be identical on both paths).
//   1. absmax_kernel: amax|W| over the whole matrix (NVFP4 tensor scale).
//   2. wq_encode_kernel: per 32-element chunk, block scales and E2M1 codes.
// A stack of weights (the experts of a mixture-of-experts layer) is
// quantized in the same two launches: blockIdx.y is the group, each group
// with its own tensor scale, its payload `gstride` bytes after the previous
// group's.
#include <cuda_fp16.h>

#include "sharq_dev.cuh"
#include "sq_internal.h"

namespace sq {

constexpr int kWThreads = 256;

// amax of |fp16| over `count` halves (count a multiple of 8): the absolute
// value of a finite fp16 orders like its low 15 bits.
__global__ void __launch_bounds__(kWThreads) absmax_kernel(const uint16_t *__restrict__ w, int64_t count,
                                                          unsigned *__restrict__ amax_word, int64_t gstride) {
    __shared__ unsigned red[kWThreads / 32];
    w += (int64_t)blockIdx.y * count;
    amax_word = reinterpret_cast<unsigned *>(reinterpret_cast<uint8_t *>(amax_word) + (int64_t)blockIdx.y * gstride);
    const uint4 *p = reinterpret_cast<const uint4 *>(w);
    const int64_t nvec = count / 8;
    unsigned m = 0;
    for (int64_t i = (int64_t)blockIdx.x * kWThreads + threadIdx.x; i < nvec; i += (int64_t)gridDim.x * kWThreads) {
        uint4 v = __ldg(p + i);
        const uint32_t ws[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            m = max(m, ws[q] & 0x7FFFu);
            m = max(m, (ws[q] >> 16) & 0x7FFFu);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    if (threadIdx.x % 32 == 0) red[threadIdx.x / 32] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        unsigned a = 0;
        for (int i = 0; i < kWThreads / 32; ++i) a = max(a, red[i]);
        atomicMax(amax_word, __float_as_uint(h2f((uint16_t)a)));
    }
}

// Rows [0, sf_rows) of one weight (rows >= n_out are scale-layout padding),
// written at rows row0 + r of the code and scale layouts (row0 > 0: a
// segment of a fused weight). BLK: the block length (the format's own, or
// twice it for the pair-wise sparse mode's weights); each thread takes a
// chunk of max(BLK, 32) values of a row.
template <int FMT, int BLK>
__global__ void __launch_bounds__(kWThreads)
wq_encode_kernel(const uint16_t *__restrict__ w, int64_t n_out, int64_t sf_rows, int64_t k,
                 const unsigned *__restrict__ amax_word, float *__restrict__ s_tw_out, uint8_t *__restrict__ codes,
                 uint8_t *__restrict__ sf, int64_t gstride, int64_t row0) {
    constexpr int CH = BLK > 32 ? BLK : 32;  // values per thread
    constexpr int NB = CH / BLK;             // blocks per chunk (1 or 2)
    {
        const int64_t gofs = (int64_t)blockIdx.y * gstride;
        w += (int64_t)blockIdx.y * n_out * k;
        amax_word = reinterpret_cast<const unsigned *>(reinterpret_cast<const uint8_t *>(amax_word) + gofs);
        s_tw_out = reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(s_tw_out) + gofs);
        codes += gofs;
        sf += gofs;
    }
    const float amax = __uint_as_float(*amax_word);
    const float s_t = (FMT == kFmtNV && amax != 0.0f) ? __fdiv_rn(amax, 2688.0f) : 1.0f;
    const float c6 = __fmul_rn(6.0f, s_t);
    if (blockIdx.x == 0 && threadIdx.x == 0) *s_tw_out = s_t;
    const int64_t cpr = k / CH, nblk = k / BLK, total = sf_rows * cpr;
    for (int64_t t = (int64_t)blockIdx.x * kWThreads + threadIdx.x; t < total; t += (int64_t)gridDim.x * kWThreads) {
        const int64_t row = t / cpr, c = t - row * cpr, orow = row0 + row;
        if (row >= n_out) {  // scale-layout padding rows
            if (NB == 2) *reinterpret_cast<uint16_t *>(sf + sf_offset(orow, 2 * c, nblk)) = 0;
            else sf[sf_offset(orow, c, nblk)] = 0;
            continue;
        }
        const uint4 *wp = reinterpret_cast<const uint4 *>(w + row * k + c * CH);
        float v[CH];
#pragma unroll
        for (int q = 0; q < CH / 8; ++q) {
            uint4 u = __ldcs(wp + q);
            const uint32_t ws[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int i = 0; i < 8; ++i) v[8 * q + i] = h2f((uint16_t)(ws[i / 2] >> (16 * (i % 2))));
        }
        uint32_t pk[CH / 8], sc[NB];
#pragma unroll
        for (int i = 0; i < CH / 8; ++i) pk[i] = 0;
#pragma unroll
        for (int bk = 0; bk < NB; ++bk) {
            float a = 0.0f;
#pragma unroll
            for (int i = bk * BLK; i < (bk + 1) * BLK; ++i) a = fmaxf(a, fabsf(v[i]));
            uint32_t code;
            const float d = block_step<FMT>(a, s_t, c6, code);
            sc[bk] = code;
            if (d != 0.0f) {
#pragma unroll
                for (int i = bk * BLK; i < (bk + 1) * BLK; i += 2)
                    pk[i / 8] |= e2m1x2(__fdiv_rn(v[i], d), __fdiv_rn(v[i + 1], d)) << (4 * (i % 8));
            }
        }
#pragma unroll
        for (int q = 0; q < CH / 32; ++q)
            *reinterpret_cast<uint4 *>(codes + orow * (k / 2) + c * (CH / 2) + 16 * q) =
                make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
        if (NB == 2) *reinterpret_cast<uint16_t *>(sf + sf_offset(orow, 2 * c, nblk)) = (uint16_t)(sc[0] | (sc[NB - 1] << 8));
        else sf[sf_offset(orow, c, nblk)] = (uint8_t)sc[0];
    }
}

// The encode launch of one weight payload's rows.
template <int FMT>
static void launch_wq_encode(dim3 grid, cudaStream_t stream, bool sparse, const uint16_t *w, int64_t n_out,
                             int64_t sf_rows, int64_t k, const unsigned *aw, float *s_tw, uint8_t *codes, uint8_t *sf,
                             int64_t gstride, int64_t row0) {
    if (sparse)
        wq_encode_kernel<FMT, FMT == kFmtNV ? 32 : 64><<<grid, kWThreads, 0, stream>>>(w, n_out, sf_rows, k, aw, s_tw,
                                                                                     codes, sf, gstride, row0);
    else
        wq_encode_kernel<FMT, FMT == kFmtNV ? 16 : 32><<<grid, kWThreads, 0, stream>>>(w, n_out, sf_rows, k, aw, s_tw,
                                                                                     codes, sf, gstride, row0);
}

sharq_status launch_quantize_weight(LaunchCtx &ctx, const sharq_wq &W, const void *w, int64_t groups,
                                   int64_t gstride) {
    unsigned *words = reinterpret_cast<unsigned *>(W.tensor_scale) - 1;  // [0] amax bits, [1] s_tW
    if (groups == 1) SQ_CUDA_TRY(cudaMemsetAsync(words, 0, sizeof(unsigned), ctx.stream));
    else SQ_CUDA_TRY(cudaMemset2DAsync(words, (size_t)gstride, 0, sizeof(unsigned), (size_t)groups, ctx.stream));
    // grid-stride loops: about 4 (absmax) and 8 (encode) CTAs per SM over all groups
    const int64_t per_group_cap = (int64_t)ctx.num_sms * 4 / groups > 0 ? (int64_t)ctx.num_sms * 4 / groups : 1;
    const int64_t count = W.n_out * W.k;
    int64_t blocks = (count / 8 + kWThreads - 1) / kWThreads;
    if (blocks > per_group_cap) blocks = per_group_cap;
    const dim3 ga((unsigned)blocks, (unsigned)groups);
    absmax_kernel<<<ga, kWThreads, 0, ctx.stream>>>((const uint16_t *)w, count, words, gstride);
    ctx.launches++;
    const bool sparse = W.sparse != 0;
    const int64_t ch = (sparse && W.fmt == kFmtMX) ? 64 : 32;  // values per encode thread
    const int64_t total = W.sf_rows * (W.k / ch);
    int64_t eb = (total + kWThreads - 1) / kWThreads;
    if (eb > 2 * per_group_cap) eb = 2 * per_group_cap;
    const dim3 ge((unsigned)eb, (unsigned)groups);
    if (W.fmt == kFmtNV)
        launch_wq_encode<kFmtNV>(ge, ctx.stream, sparse, (const uint16_t *)w, W.n_out, W.sf_rows, W.k, words,
                                 W.tensor_scale, (uint8_t *)W.codes, (uint8_t *)W.scales_backbone, gstride, 0);
    else
        launch_wq_encode<kFmtMX>(ge, ctx.stream, sparse, (const uint16_t *)w, W.n_out, W.sf_rows, W.k, words,
                                 W.tensor_scale, (uint8_t *)W.codes, (uint8_t *)W.scales_backbone, gstride, 0);
    ctx.launches++;
    SQ_CUDA_TRY(cudaGetLastError());
    return SHARQ_OK;
}

// Fused weight: segment g (rows seg_rows[g], after the earlier segments'
// rows) is quantized on its own, with its amax in word 0 (g = 0) or 8 + g of
// the weight's words and its tensor scale in tensor_scale[g] (words 1 + g);
// the last segment also zeroes the scale-layout padding rows.
sharq_status launch_quantize_weight_fused(LaunchCtx &ctx, const sharq_wq &W, const void *w, const int64_t *seg_rows,
                                         int n_segs) {
    unsigned *words = reinterpret_cast<unsigned *>(W.tensor_scale) - 1;
    SQ_CUDA_TRY(cudaMemsetAsync(words, 0, 16 * sizeof(unsigned), ctx.stream));
    int64_t off = 0;
    for (int g = 0; g < n_segs; ++g) {
        const int64_t rows = seg_rows[g];
        unsigned *aw = g == 0 ? words : words + 8 + g;
        const uint16_t *wg = (const uint16_t *)w + off * W.k;
        const int64_t count = rows * W.k;
        int64_t blocks = (count / 8 + kWThreads - 1) / kWThreads;
        if (blocks > (int64_t)ctx.num_sms * 4) blocks = (int64_t)ctx.num_sms * 4;
        absmax_kernel<<<(unsigned)blocks, kWThreads, 0, ctx.stream>>>(wg, count, aw, 0);
        ctx.launches++;
        const int64_t iter_rows = g + 1 == n_segs ? W.sf_rows - off : rows;
        int64_t eb = (iter_rows * (W.k / 32) + kWThreads - 1) / kWThreads;
        if (eb > (int64_t)ctx.num_sms * 8) eb = (int64_t)ctx.num_sms * 8;
        if (W.fmt == kFmtNV)
            launch_wq_encode<kFmtNV>(dim3((unsigned)eb), ctx.stream, false, wg, rows, iter_rows, W.k, aw,
                                     W.tensor_scale + g, (uint8_t *)W.codes, (uint8_t *)W.scales_backbone, 0, off);
        else
            launch_wq_encode<kFmtMX>(dim3((unsigned)eb), ctx.stream, false, wg, rows, iter_rows, W.k, aw,
                                     W.tensor_scale + g, (uint8_t *)W.codes, (uint8_t *)W.scales_backbone, 0, off);
        ctx.launches++;
        off += rows;
    }
    SQ_CUDA_TRY(cudaGetLastError());
    return SHARQ_OK;
}

}  // namespace sq

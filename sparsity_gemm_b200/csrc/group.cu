// Expert-grouped gather of prepared rows, for mixture-of-experts layers.
//
// "SharQ: Bridging Activation Sparsity and FP4 Quantization for LLM
// Inference", Abstract, lists Qwen3-30B-A3B (a mixture-of-experts model)
// without describing its expert layers. Reading: an activation tensor is
// prepared once over all its rows (one tensor scale for all experts), and
// each expert's linear reads the rows routed to it. This kernel moves those
// rows, bit for bit, into a prep whose groups start at multiples of 128
// rows, so that every 128-row GEMM tile, and with it every 512-byte scale
// atom (128 rows x 4 scales), belongs to one group.
//
// One CTA per 128-row destination tile. Warp 0 builds the groups' tile
// table from the device offsets (and checks them); the CTA then finds its
// group, reads the 128 source row indices, and copies codes (16-byte
// chunks over all threads), mask metadata, LayerNorm statistics and the
// scale atoms (4-byte words: one row's 4 scales of one atom are 4
// consecutive bytes in both layouts). Tile rows past the group's end are
// zero.
#include <cuda_runtime.h>

#include "sharq_dev.cuh"
#include "sq_internal.h"

namespace sq {

constexpr int kGatherThreads = 256;
constexpr int kCopyUnroll = 4;  // 16-byte code chunks per operand in flight per thread

// (row, column) of a flat index over rows of `width` items, stepped by a
// fixed stride without dividing again.
struct RowCol {
    int32_t r, c, width, step_r, step_c;
    __device__ RowCol(int32_t i, int32_t w, int32_t stride)
        : r(i / w), c(i % w), width(w), step_r(stride / w), step_c(stride % w) {}
    __device__ void advance() {
        r += step_r;
        c += step_c;
        if (c >= width) {
            c -= width;
            ++r;
        }
    }
};

struct GatherParams {
    const uint8_t *s_codes, *r_codes, *s_scales, *r_scales, *meta;
    const float2 *stats;
    const float *s_t;
    int64_t src_rows;
    uint8_t *d_s_codes, *d_r_codes, *d_s_scales, *d_r_scales, *d_meta;
    float2 *d_stats;
    float *d_words;          // [0] amax word (unused: 0), [1] s_t
    const int32_t *row_idx;  // NULL: identity
    const int32_t *offsets;
    int32_t groups;
    int64_t rows, cap_rows, k, meta_row;
    int32_t nblk;
    unsigned *status;
};

__global__ void __launch_bounds__(kGatherThreads) gather_kernel(const GatherParams p) {
    __shared__ int32_t tiles[kGroupsMax + 1];
    __shared__ int32_t src_row[128];
    __shared__ int table_ok;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    if (warp == 0) {
        const bool ok = build_tile_table(p.offsets, p.groups, p.rows, p.cap_rows, tiles);
        if (lane == 0) table_ok = ok ? 1 : 0;
    }
    __syncthreads();
    if (!table_ok) {
        if (blockIdx.x == 0 && threadIdx.x == 0) record_status(p.status, kSiteBadOffsets);
        return;
    }
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        p.d_words[0] = 0.0f;
        p.d_words[1] = *p.s_t;
    }
    const int32_t tile = (int32_t)blockIdx.x;
    if (tile >= tiles[p.groups]) return;
    const int g = group_of_tile(tiles, p.groups, tile);
    const int64_t i0 = (int64_t)p.offsets[g] + (int64_t)(tile - tiles[g]) * 128;  // first grouped row
    const int64_t count = min((int64_t)p.offsets[g + 1] - i0, (int64_t)128);
    if (threadIdx.x < 128) {
        int32_t src = -1;
        if (threadIdx.x < count) {
            const int64_t i = i0 + threadIdx.x;
            const int64_t t = p.row_idx ? (int64_t)p.row_idx[i] : i;
            if (t >= 0 && t < p.src_rows) src = (int32_t)t;
            else record_status(p.status, kSiteBadRowIndex);
        }
        src_row[threadIdx.x] = src;
    }
    __syncthreads();

    const int64_t d0 = (int64_t)tile * 128;  // first destination row
    const int64_t chunks = p.k / 32;  // 16-byte chunks per row (p.k / 2 bytes)
    // Codes: (row, chunk) pairs of the tile over all threads, consecutive
    // threads on consecutive chunks of a row; kCopyUnroll loads per operand
    // in flight before the stores (the copy is latency-bound).
    const int64_t items = 128 * chunks;  // < 2^18
    const uint4 zero4 = make_uint4(0, 0, 0, 0);
    RowCol rc(threadIdx.x, (int32_t)chunks, kGatherThreads);
    for (int64_t i0 = threadIdx.x; i0 < items; i0 += kCopyUnroll * kGatherThreads) {
        uint4 vs[kCopyUnroll], vr[kCopyUnroll];
        int64_t dst[kCopyUnroll];
#pragma unroll
        for (int j = 0; j < kCopyUnroll; ++j) {
            const int64_t i = i0 + (int64_t)j * kGatherThreads;
            vs[j] = zero4;
            vr[j] = zero4;
            dst[j] = -1;
            if (i < items) {
                const int64_t r = rc.r, c = rc.c;
                const int64_t src = src_row[r];
                dst[j] = (d0 + r) * chunks + c;
                if (src >= 0) {
                    vs[j] = __ldg(reinterpret_cast<const uint4 *>(p.s_codes) + src * chunks + c);
                    vr[j] = __ldg(reinterpret_cast<const uint4 *>(p.r_codes) + src * chunks + c);
                }
            }
            rc.advance();
        }
#pragma unroll
        for (int j = 0; j < kCopyUnroll; ++j)
            if (dst[j] >= 0) {
                reinterpret_cast<uint4 *>(p.d_s_codes)[dst[j]] = vs[j];
                reinterpret_cast<uint4 *>(p.d_r_codes)[dst[j]] = vr[j];
            }
    }
    // Metadata: 16-byte chunks when the rows allow (four loads in flight),
    // else 4-byte words, else bytes; then the statistics.
    if ((p.meta_row & 15) == 0) {
        const int64_t cpr = p.meta_row / 16, mitems = 128 * cpr;
        RowCol mc(threadIdx.x, (int32_t)cpr, kGatherThreads);
        for (int64_t i0 = threadIdx.x; i0 < mitems; i0 += 4 * kGatherThreads) {
            uint4 v[4];
            int64_t dst[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int64_t i = i0 + (int64_t)j * kGatherThreads;
                v[j] = zero4;
                dst[j] = -1;
                if (i < mitems) {
                    const int64_t src = src_row[mc.r];
                    dst[j] = (d0 + mc.r) * cpr + mc.c;
                    if (src >= 0) v[j] = __ldg(reinterpret_cast<const uint4 *>(p.meta) + src * cpr + mc.c);
                }
                mc.advance();
            }
#pragma unroll
            for (int j = 0; j < 4; ++j)
                if (dst[j] >= 0) reinterpret_cast<uint4 *>(p.d_meta)[dst[j]] = v[j];
        }
    } else if ((p.meta_row & 3) == 0) {
        const int64_t wpr = p.meta_row / 4, mitems = 128 * wpr;
        RowCol mc(threadIdx.x, (int32_t)wpr, kGatherThreads);
        for (int64_t i = threadIdx.x; i < mitems; i += kGatherThreads, mc.advance()) {
            const int64_t r = mc.r, c = mc.c;
            const int64_t src = src_row[r];
            reinterpret_cast<uint32_t *>(p.d_meta)[(d0 + r) * wpr + c] =
                src >= 0 ? reinterpret_cast<const uint32_t *>(p.meta)[src * wpr + c] : 0u;
        }
    } else {
        const int64_t mitems = 128 * p.meta_row;
        RowCol mc(threadIdx.x, (int32_t)p.meta_row, kGatherThreads);
        for (int64_t i = threadIdx.x; i < mitems; i += kGatherThreads, mc.advance()) {
            const int64_t r = mc.r, c = mc.c;
            const int64_t src = src_row[r];
            p.d_meta[(d0 + r) * p.meta_row + c] = src >= 0 ? p.meta[src * p.meta_row + c] : (uint8_t)0;
        }
    }
    if (threadIdx.x < 128) {
        const int64_t src = src_row[threadIdx.x];
        p.d_stats[d0 + threadIdx.x] = src >= 0 ? p.stats[src] : make_float2(0.0f, 0.0f);
    }

    // Scale atoms of this tile: (nblk / 4) atoms of 128 words per operand.
    // Word o of an atom holds row (o / 4) + 32 (o % 4).
    const int64_t atoms = p.nblk / 4, words = atoms * 128;
    const uint32_t *sws = reinterpret_cast<const uint32_t *>(p.s_scales);
    const uint32_t *swr = reinterpret_cast<const uint32_t *>(p.r_scales);
    uint32_t *dws = reinterpret_cast<uint32_t *>(p.d_s_scales) + (int64_t)tile * words;
    uint32_t *dwr = reinterpret_cast<uint32_t *>(p.d_r_scales) + (int64_t)tile * words;
    for (int64_t w0 = threadIdx.x; w0 < words; w0 += 4 * kGatherThreads) {  // four loads per operand in flight
        uint32_t vs[4], vr[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int64_t w = w0 + (int64_t)j * kGatherThreads;
            vs[j] = 0;
            vr[j] = 0;
            if (w < words) {
                const int64_t a = w >> 7, o = w & 127;
                const int64_t src = src_row[(o >> 2) + 32 * (o & 3)];
                if (src >= 0) {
                    const int64_t sw = ((src >> 7) * atoms + a) * 128 + (src & 31) * 4 + ((src >> 5) & 3);
                    vs[j] = __ldg(sws + sw);
                    vr[j] = __ldg(swr + sw);
                }
            }
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int64_t w = w0 + (int64_t)j * kGatherThreads;
            if (w < words) {
                dws[w] = vs[j];
                dwr[w] = vr[j];
            }
        }
    }
}

sharq_status launch_gather(LaunchCtx &ctx, const sharq_prep &S, const int32_t *row_idx, const int32_t *offsets,
                           int32_t groups, int64_t rows, const sharq_prep &D) {
    GatherParams p;
    p.s_codes = (const uint8_t *)S.s_codes;
    p.r_codes = (const uint8_t *)S.r_codes;
    p.s_scales = (const uint8_t *)S.s_scales;
    p.r_scales = (const uint8_t *)S.r_scales;
    p.meta = (const uint8_t *)S.meta;
    p.stats = (const float2 *)S.scratch;
    p.s_t = S.tensor_scale;
    p.src_rows = S.m_tok;
    p.d_s_codes = (uint8_t *)D.s_codes;
    p.d_r_codes = (uint8_t *)D.r_codes;
    p.d_s_scales = (uint8_t *)D.s_scales;
    p.d_r_scales = (uint8_t *)D.r_scales;
    p.d_meta = (uint8_t *)D.meta;
    p.d_stats = (float2 *)D.scratch;
    p.d_words = D.tensor_scale - 1;
    p.row_idx = row_idx;
    p.offsets = offsets;
    p.groups = groups;
    p.rows = rows;
    p.cap_rows = D.m_tok;
    p.k = D.k;
    p.meta_row = D.meta_row_bytes;
    p.nblk = (int32_t)(D.k / blk_of(D.fmt));
    p.status = ctx.status;
    const unsigned grid = (unsigned)(D.m_tok / 128);  // upper bound on the tiles; the rest exit at once
    gather_kernel<<<grid, kGatherThreads, 0, ctx.stream>>>(p);
    ctx.launches++;
    SQ_CUDA_TRY(cudaGetLastError());
    return SHARQ_OK;
}

}  // namespace sq

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
// chunks, one warp per row), mask metadata, LayerNorm statistics and the
// scale atoms (4-byte words: one row's 4 scales of one atom are 4
// consecutive bytes in both layouts). Tile rows past the group's end are
// zero.
#include <cuda_runtime.h>

#include "sharq_dev.cuh"
#include "sq_internal.h"

namespace sq {

constexpr int kGatherThreads = 256;

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
    const int64_t row_bytes = p.k / 2, chunks = p.k / 32;
    const uint4 zero4 = make_uint4(0, 0, 0, 0);
    for (int r = warp; r < 128; r += kGatherThreads / 32) {
        const int64_t src = src_row[r];
        const int64_t sp = src >= 0 ? src : 0;  // pointers stay inside the source for zero rows
        const int64_t dst = d0 + r;
        const uint4 *ss = reinterpret_cast<const uint4 *>(p.s_codes + sp * row_bytes);
        const uint4 *sr = reinterpret_cast<const uint4 *>(p.r_codes + sp * row_bytes);
        uint4 *ds = reinterpret_cast<uint4 *>(p.d_s_codes + dst * row_bytes);
        uint4 *dr = reinterpret_cast<uint4 *>(p.d_r_codes + dst * row_bytes);
        for (int64_t c = lane; c < chunks; c += 32) {
            ds[c] = src >= 0 ? __ldg(ss + c) : zero4;
            dr[c] = src >= 0 ? __ldg(sr + c) : zero4;
        }
        if ((p.meta_row & 3) == 0) {
            const uint32_t *sm = reinterpret_cast<const uint32_t *>(p.meta + sp * p.meta_row);
            uint32_t *dm = reinterpret_cast<uint32_t *>(p.d_meta + dst * p.meta_row);
            for (int64_t b = lane; b < p.meta_row / 4; b += 32) dm[b] = src >= 0 ? sm[b] : 0u;
        } else {
            const uint8_t *sm = p.meta + sp * p.meta_row;
            uint8_t *dm = p.d_meta + dst * p.meta_row;
            for (int64_t b = lane; b < p.meta_row; b += 32) dm[b] = src >= 0 ? sm[b] : (uint8_t)0;
        }
        if (lane == 0) p.d_stats[dst] = src >= 0 ? p.stats[src] : make_float2(0.0f, 0.0f);
    }

    // Scale atoms of this tile: (nblk / 4) atoms of 128 words per operand.
    // Word o of an atom holds row (o / 4) + 32 (o % 4).
    const int64_t atoms = p.nblk / 4, words = atoms * 128;
    const uint32_t *sws = reinterpret_cast<const uint32_t *>(p.s_scales);
    const uint32_t *swr = reinterpret_cast<const uint32_t *>(p.r_scales);
    uint32_t *dws = reinterpret_cast<uint32_t *>(p.d_s_scales) + (int64_t)tile * words;
    uint32_t *dwr = reinterpret_cast<uint32_t *>(p.d_r_scales) + (int64_t)tile * words;
    for (int64_t w = threadIdx.x; w < words; w += kGatherThreads) {
        const int64_t a = w >> 7, o = w & 127;
        const int64_t src = src_row[(o >> 2) + 32 * (o & 3)];
        uint32_t vs = 0, vr = 0;
        if (src >= 0) {
            const int64_t sw = ((src >> 7) * atoms + a) * 128 + (src & 31) * 4 + ((src >> 5) & 3);
            vs = __ldg(sws + sw);
            vr = __ldg(swr + sw);
        }
        dws[w] = vs;
        dwr[w] = vr;
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

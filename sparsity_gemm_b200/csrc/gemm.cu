// Dual-path FP4 GEMM of SharQ on sm_100a (tcgen05 block-scaled MMA).
//
// "SharQ: Bridging Activation Sparsity and FP4 Quantization for LLM
// Inference", Abstract: a sparse FP4 GEMM on the backbone and a dense FP4
// GEMM on the residual, both on the same FP4 weight codes (each path with a
// scale view of its own), added together. Here both paths issue into ONE tensor-memory
// accumulator, and every W tile (codes and scale view) is loaded once per
// K step and read by both paths' MMAs:
//     acc = sum_k Q(S)[i,k] W[j,k] + Q(R)[i,k] W[j,k]      (block-scaled)
//     out = RN16(acc * s_t * s_tW)
//
// The backbone runs as a dense FP4 MMA over the full K with zeros off the
// mask: the block-scaled FP4 sparse MMA kinds take pair-wise 4:8 metadata,
// which an element-wise top-n-of-m mask does not satisfy in general.
//
// Structure: persistent CTAs (one per SM), tile 128 x 256 (M x N) with a
// K step of 2 * SQ_GEMM_BKB FP4 values, a TMA pipeline as deep as shared
// memory allows, 10 warps:
//   warp 0      TMA producer (A_S, A_R, W tiles; scale atoms by bulk copy)
//   warp 1      tensor-memory allocation and the single-thread MMA issuer
//   warps 2..5  epilogue: tensor memory -> registers -> fp16 -> global
//   warps 6..9  scale writes: shared memory -> registers -> one of four
//               scale buffers in tensor memory, ahead of the MMAs
// Every mbarrier wait is bounded (global-timer limit); a wait that runs out
// records a site code in the status word and the CTA winds down cleanly.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_fp16.h>
#include <stdlib.h>
#include <string.h>

#include <mutex>

#include "sharq_dev.cuh"
#include "sq_internal.h"

namespace sq {

// K tile width in bytes per operand row (two FP4 values per byte). Measured
// on B200: 128-byte rows (3 stages) beat 64-byte rows (6 stages) by ~5%. 64 bytes
// (128 elements, 64-byte swizzle) gives 36 KB stages and a 6-deep pipeline;
// 128 bytes (256 elements, 128-byte swizzle) gives 72 KB stages, 3 deep.
#ifndef SQ_GEMM_BKB
#define SQ_GEMM_BKB 128
#endif
// Pause between the epilogue's 32-column store chunks, per K step of the
// main loop (the stores of a tile are spread over the next tile's loop).
#ifndef SQ_STORE_PAUSE_NS_PER_KSTEP
#define SQ_STORE_PAUSE_NS_PER_KSTEP 60
#endif
constexpr int kBM = 128, kBKBytes = SQ_GEMM_BKB;
constexpr int kABytes = kBM * kBKBytes;
constexpr int kSfaMax = 512 * (kBKBytes / 32);  // scale bytes of 128 rows per stage, NVFP4 (MXFP4 uses half)
constexpr int kOffAS = 0;
// Scale buffers in tensor memory after the accumulators: per buffer, the
// backbone A scales, the residual A scales and the W scales of one stage
// (NVFP4: kBKBytes / 32 atoms per 128 rows; MXFP4 uses half).
constexpr uint32_t kNvAtoms = kBKBytes / 32;
constexpr uint32_t kSfaS = 0, kSfaR = 4 * kNvAtoms, kSfb = 8 * kNvAtoms;
// Grouped launches: the tile table (kGroupsMax + 1 ints) and its valid flag.
constexpr int kTableBytes = 4 * (int)(kGroupsMax + 1) + 12;
constexpr int kMmaPerStage = kBKBytes / 32;                        // MMAs of K = 64 per path per stage
constexpr uint32_t kSwizzleLayout = kBKBytes == 128 ? 2u : 4u;     // descriptor layout: 128B / 64B swizzle
constexpr uint32_t kTmemCols = 512;
constexpr int kGemmThreads = 320;
constexpr int kMaxSplit = 8;
static_assert(kTableBytes % 4 == 0, "table alignment");

// Tile width N. 256: one accumulator (columns 0..255), four scale buffers
// after it. 128: two accumulators used in turn (columns 0..127 and
// 128..255), so that the next tile's MMAs run while the epilogue drains the
// previous tile, and a fourth pipeline stage in the smaller stage memory.
// Both widths give identical results. 256 is the default for dense and
// grouped launches alike: with two A operands (backbone and residual) per
// B tile, halving N raises the operand bytes per FLOP by half, which cost
// more than the hidden drain saved on the short-K expert GEMMs (Qwen3 MoE
// shapes, K = 2048 and 768: 22% slower at 128). SQ_GROUPED_BN=128 builds
// the other width for grouped launches.
// SP: the pair-wise 4:8 backbone (sharq_prepare_sparse): per stage the
// backbone tile holds the kept half of K (64-byte rows), its scales and the
// W view the sparse MMA reads hold one scale per 32 values (half the
// atoms), and the mask metadata rides with the scales (16 bytes per row).
// PAIR: a CTA pair computes a 256-row tile with cta_group::2 MMAs; each CTA
// stages its own 128 A rows and half of the tile's W rows (the W scale view
// for all of them), which leaves room for four stages.
template <int BN, bool SP = false, bool PAIR = false>
struct TileCfg {
    static constexpr int kBN = BN;
    static constexpr int kBlk = BN / 128;            // 128-row W blocks (scale atoms) per tile
    static constexpr int kNacc = BN == 256 ? 1 : 2;  // accumulators in tensor memory
    static constexpr int kASBytes = SP ? kABytes / 2 : kABytes;
    static constexpr int kOffAR = kASBytes, kOffB = kASBytes + kABytes;
    static constexpr int kBBytes = (PAIR ? BN / 2 : BN) * kBKBytes;
    static constexpr int kSfaSMax = SP ? kSfaMax / 2 : kSfaMax;  // backbone scale bytes per stage
    static constexpr int kSfbMax = kBlk * kSfaSMax;              // W scale view of the backbone path
    static constexpr int kMetaBytes = SP ? kBM * 16 : 0;
    static constexpr int kOffSFAS = kOffB + kBBytes, kOffSFAR = kOffSFAS + kSfaSMax, kOffSFB = kOffSFAR + kSfaMax;
    static constexpr int kOffMeta = kOffSFB + kSfbMax;
    static constexpr int kStageBytes = kOffMeta + kMetaBytes;  // a multiple of 1024
    static constexpr int kTableArea = PAIR ? 0 : kTableBytes;  // the grouped tile table (not in pair launches)
    static constexpr int kStages = (232448 - 2048) / kStageBytes;
    static constexpr int kBarOff = kStages * kStageBytes;
    static constexpr uint32_t kColSf0 = kNacc * BN;
    // Columns of one scale buffer. Dense: A_S, A_R, then kBlk W blocks.
    // SP (NVFP4 counts; MXFP4 uses half): backbone scales (2 atoms), the W
    // backbone view (2 atoms x kBlk), residual scales (4 atoms), the W
    // residual view (4 atoms x kBlk, written from the backbone view's values),
    // then the metadata (4 columns per MMA, two used).
    static constexpr uint32_t kSpS = 0, kSpWb = 8, kSpR = kSpWb + 8 * kBlk, kSpWr = kSpR + 16,
                              kSpMeta = kSpWr + 16 * kBlk;
    static constexpr uint32_t kSfBufCols = SP ? kSpMeta + 8 : (8 + 4 * kBlk) * kNvAtoms;
    static constexpr int kSfBufs = (int)((kTmemCols - kColSf0) / kSfBufCols) < 4 ? (int)((kTmemCols - kColSf0) / kSfBufCols) : 4;
    // mbarriers: full[s], empty[s], sf_loaded[s], acc_full[a], acc_empty[a],
    // drain, sf_full[b], sf_empty[b]; the tensor-memory slot follows.
    static constexpr int kBarBytes = 8 * (3 * kStages + 2 * kNacc + 1 + 2 * kSfBufs);
    static constexpr int kBarArea = (kBarBytes + 4 + 127) / 128 * 128;
    static constexpr int kTableOff = kBarOff + kBarArea;
    static constexpr int kSmemBytes = kTableOff + kTableArea + 1024;  // barriers, table, alignment slack
    // Split-K partial tile in the stage memory: 128 rows of BN fp32, rows
    // padded by 16 bytes so that a warp's 32 rows hit different banks.
    static constexpr uint32_t kPartStride = BN * 4 + 16;
    static_assert(BN == 128 || BN == 256, "tile width");
    static_assert(!SP || (BN == 256 && kBKBytes == 128), "the sparse mode uses the 256-column, 128-byte K tile");
    static_assert(!PAIR || (BN == 256 && !SP), "pair launches: dense mode, 256 columns");
    static_assert(kStageBytes % 1024 == 0, "stage buffers must stay 1024-byte aligned");
    static_assert(kSmemBytes <= 232448, "shared memory budget");
    static_assert(kBarBytes + 4 <= kBarArea, "barrier area");
    static_assert(kSfBufs >= 2, "scale buffers");
    static_assert(kColSf0 + kSfBufs * kSfBufCols <= kTmemCols, "tensor memory columns");
    static_assert(kBM * kPartStride <= (uint32_t)(kStages * kStageBytes), "split-K partial fits the stages");
};

#ifndef SQ_GROUPED_BN
#define SQ_GROUPED_BN 256
#endif
constexpr int kDenseBN = 256, kGroupedBN = SQ_GROUPED_BN;

enum : unsigned {
    kSiteProducer = 0x101,
    kSiteMmaAcc = 0x102,
    kSiteMmaFull = 0x103,
    kSiteEpilogue = 0x104,
    kSiteMmaScales = 0x105,
    kSiteScaleFull = 0x106,
    kSiteScaleEmpty = 0x107,
    kSiteProbe = 0x1FF,
};

// Exit drains (in-flight copies, outstanding MMAs) always get this long,
// whatever the configurable wait limit is.
constexpr uint64_t kDrainNs = 2000000000ull;

struct GemmParams {
    const uint8_t *sfa_s, *sfa_r, *sfb;
    const float *s_t, *s_tw;
    __half *out;
    int32_t m_tok, n_out, k;
    unsigned *status;
    uint64_t wait_ns;
    // grouped launches only
    const int32_t *offsets;  // [groups + 1], device
    int32_t groups;
    int64_t rows;            // grouped rows (= offsets[groups])
    int64_t w_gstride;       // bytes between two groups' weight payloads
    // split-K (dense launches only): `split` CTAs of one cluster share a
    // tile, each over a K range, and reduce through distributed shared
    // memory; 1 = no split.
    int32_t split;
    // dense launches only: fused weights (segs > 1: column j of segment g,
    // seg_end[g-1] <= j < seg_end[g], takes s_tw[g]; boundaries are
    // multiples of 32 columns) and an optional fp16 bias per column
    int32_t segs;
    int32_t seg_end[SHARQ_SEGMENTS_MAX];
    const __half *bias;
};

// alpha = RN32(s_t * s_tW[g]) of the segment holding column `col`.
__device__ __forceinline__ float alpha_of_col(const GemmParams &p, float s_t, float alpha0, int col) {
    if (p.segs <= 1) return alpha0;
    int g = 0;
#pragma unroll
    for (int i = 0; i + 1 < SHARQ_SEGMENTS_MAX; ++i)  // constant indices: no local copy of the parameters
        g += (i + 1 < p.segs && col >= p.seg_end[i]) ? 1 : 0;
    return __fmul_rn(s_t, p.s_tw[g]);
}

// Instruction descriptor of the block-scaled MMA (M = 128, N = BN, E2M1 x
// E2M1, K-major A and B): A/B format E2M1 at bits 7-9 / 10-12, N >> 3 at
// bits 17-22, scale format (0 = UE4M3, 1 = E8M0) at bit 23, M >> 4 at bits
// 24-28; scale-factor byte selectors at bits 29-30 (A) and 4-5 (B).
template <int FMT, int BN, int MM = kBM>
__device__ __forceinline__ uint32_t idesc_of(uint32_t sf_id) {
    return (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) | ((FMT == kFmtMX ? 1u : 0u) << 23) |
           ((uint32_t)(MM >> 4) << 24) | (sf_id << 29) | (sf_id << 4);
}

// K-major operand tile, rows of kBKBytes bytes swizzled in kBKBytes-wide
// atoms; 8-row groups are 8 * kBKBytes bytes apart.
__device__ __forceinline__ uint64_t desc_operand(uint32_t addr) {
    return smem_desc(addr, 16, 8 * kBKBytes, kSwizzleLayout);
}


// The sparse mode's compacted backbone tile: rows of kBKBytes / 2 bytes,
// 64-byte swizzle; 8-row groups 8 * kBKBytes / 2 bytes apart.
__device__ __forceinline__ uint64_t desc_operand_half(uint32_t addr) {
    return smem_desc(addr, 16, 8 * (kBKBytes / 2), 4u);
}

// Output tile of linear tile index `tile`. Dense launches walk the tiles in
// groups of kRasterRows 128-row blocks, M fastest inside a group: the CTAs
// running at one time share a few W tiles across many M blocks, and a W
// tile is streamed once per group instead of once per M block (the
// difference matters when W does not stay in L2 next to the outputs, as for
// a fused gate/up weight). Grouped launches keep N fastest (an expert's
// tiles stay together).
#ifndef SQ_RASTER_ROWS
#define SQ_RASTER_ROWS 16
#endif
constexpr int kRasterRows = SQ_RASTER_ROWS;
// Pair launches: groups of this many 256-row tiles (the same rows per group
// as kRasterRows single tiles).
#ifndef SQ_RASTER_PAIR_ROWS
#define SQ_RASTER_PAIR_ROWS 8
#endif
constexpr int kRasterPairRows = SQ_RASTER_PAIR_ROWS;

template <bool GROUPED, bool PAIR = false>
__device__ __forceinline__ void tile_coords(int tile, int m_tiles, int n_tiles, int &mb, int &nb) {
    constexpr int R = PAIR ? kRasterPairRows : kRasterRows;
    if (GROUPED || R <= 1) {
        mb = tile / n_tiles;
        nb = tile % n_tiles;
        return;
    }
    const int per_group = R * n_tiles;
    const int g = tile / per_group, in = tile - g * per_group;
    const int rows = min(R, m_tiles - g * R);  // the last group may be shorter
    nb = in / rows;
    mb = g * R + (in - nb * rows);
}

// Wait bounded only by time (used to drain in-flight copies on exit).
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
    uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity))
        if (globaltimer_ns() - t0 > limit_ns) break;
}

// GROUPED: the A rows are a grouped prep (groups start at multiples of 128
// rows; tile table in shared memory), W is a stack of `groups` weights read
// through a 3-D tensor map (K bytes, n_out, group), each group with its own
// tensor scale, and output rows are remapped to grouped-row order.
// EXT (dense only): fused-weight segments and/or a bias in the epilogue; the
// plain instantiation keeps the epilogue without them.
// SP (dense only): the pair-wise 4:8 backbone through tcgen05.mma.sp on a
// K-compacted tile (tm_as rows of k/4 bytes), its metadata tile tm_meta
// ([m_tok][k/16] bytes) moved to tensor memory by the scale writers.
// PAIR (dense only, default mode): clusters of two CTAs; the pair computes
// 256 x BN tiles with cta_group::2 MMAs issued by the even CTA (the leader).
// Each CTA loads its own 128 A rows (both paths), its half of the W rows
// (tm_b with 128-row boxes) and the W scales of all BN rows; the leader's
// full and scale barriers count both CTAs' bytes and scale writes, the MMA
// commits arrive on both CTAs' barriers, and the peer's epilogue releases
// the accumulator on the leader's barrier.
template <int FMT, bool GROUPED, bool EXT, int BN, bool SP = false, bool PAIR = false>
__global__ void __launch_bounds__(kGemmThreads, 1)
dual_gemm_kernel(const __grid_constant__ CUtensorMap tm_as, const __grid_constant__ CUtensorMap tm_ar,
                 const __grid_constant__ CUtensorMap tm_b, const __grid_constant__ CUtensorMap tm_meta,
                 const GemmParams p) {
    using C = TileCfg<BN, SP, PAIR>;
    static_assert(!SP || !GROUPED, "the sparse mode runs dense launches");
    static_assert(!PAIR || (!GROUPED && !SP), "pair launches: dense, default mode");
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_s = smem_u32(smem_raw);
    uint8_t *smem = smem_raw + (((raw_s + 1023u) & ~1023u) - raw_s);
    const uint32_t sbase = smem_u32(smem);
    // barriers: full[s] (operands), empty[s], sf_loaded[s] (scale atoms),
    // acc_full[a], acc_empty[a], drain, sf_full[b], sf_empty[b]
    const uint32_t bar0 = sbase + C::kBarOff;
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (C::kStages + s); };
    auto sf_loaded_bar = [&](int s) { return bar0 + 8u * (2 * C::kStages + s); };
    auto acc_full_bar = [&](int a) { return bar0 + 8u * (3 * C::kStages + a); };
    auto acc_empty_bar = [&](int a) { return bar0 + 8u * (3 * C::kStages + C::kNacc + a); };
    const uint32_t drain_bar = bar0 + 8u * (3 * C::kStages + 2 * C::kNacc);
    auto sf_full_bar = [&](int b) { return drain_bar + 8u + 8u * b; };
    auto sf_empty_bar = [&](int b) { return drain_bar + 8u + 8u * (C::kSfBufs + b); };
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::kBarOff + C::kBarBytes);
    int32_t *tiles = reinterpret_cast<int32_t *>(smem + C::kTableOff);
    int32_t *table_ok = tiles + (kGroupsMax + 1);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    // pair launches: this CTA's place in the pair (0: leader) and the
    // leader's address of a barrier
    const uint32_t prank = PAIR ? (cluster_ctarank() & 1u) : 0u;
    const bool leader = prank == 0;
    auto at_leader = [&](uint32_t bar) { return PAIR ? mapa_shared(bar, cluster_ctarank() & ~1u) : bar; };
    // Launched as a programmatic dependent (dense launches): the set-up
    // below (barriers, tensor memory) overlaps the previous kernel's tail,
    // and nothing reads or writes global memory before griddep_wait. The
    // grouped table reads device offsets, so grouped launches wait first.
    if constexpr (GROUPED) griddep_wait();
    if (GROUPED && warp == 2) {
        const bool ok = build_tile_table(p.offsets, p.groups, p.rows, p.m_tok, tiles);
        if (lane == 0) {
            *table_ok = ok ? 1 : 0;
            if (!ok && blockIdx.x == 0) record_status(p.status, kSiteBadOffsets);
        }
    }
    // 512-byte scale atoms (128 rows x 4 scales) per 128 rows per K tile
    constexpr int kAtomsPerTile = FMT == kFmtNV ? kBKBytes / 32 : kBKBytes / 64;
    constexpr uint32_t kSfBytes = 512u * kAtomsPerTile;
    // the backbone's (and the W backbone view's) atoms in the sparse mode
    constexpr int kAtomsS = SP ? kAtomsPerTile / 2 : kAtomsPerTile;
    constexpr uint32_t kSfBytesS = 512u * kAtomsS;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
            mbar_init(sf_loaded_bar(s), 1);
        }
        for (int a = 0; a < C::kNacc; ++a) {
            mbar_init(acc_full_bar(a), 1);
            mbar_init(acc_empty_bar(a), PAIR ? 256 : 128);  // pair: both CTAs' epilogue threads
        }
        mbar_init(drain_bar, 1);
        for (int b = 0; b < C::kSfBufs; ++b) {
            mbar_init(sf_full_bar(b), PAIR ? 256 : 128);  // pair: both CTAs' scale writers
            mbar_init(sf_empty_bar(b), 1);
        }
        mbar_fence_init();
        prefetch_tmap(&tm_as);
        prefetch_tmap(&tm_ar);
        prefetch_tmap(&tm_b);
        if (SP) prefetch_tmap(&tm_meta);
    }
    if (warp == 1) {
        if (PAIR) {
            tmem_alloc_pair(smem_u32(tmem_slot), kTmemCols);
            tmem_relinquish_pair();
        } else {
            tmem_alloc(smem_u32(tmem_slot), kTmemCols);
            tmem_relinquish();
        }
    }
    tc_fence_before();
    if (PAIR) cluster_sync();  // the peer's barriers exist before any remote arrival
    else __syncthreads();
    tc_fence_after();
    if constexpr (!GROUPED) griddep_wait();
    griddep_launch();  // the next kernel may start its own set-up
    const uint32_t tmem = *tmem_slot;
    // m tiles: 128-row tiles of the prep (grouped: of all groups; none if the
    // offsets are invalid)
    const int m_tiles = GROUPED ? (*table_ok ? tiles[p.groups] : 0)
                                : (p.m_tok + (PAIR ? 2 * kBM : kBM) - 1) / (PAIR ? 2 * kBM : kBM);
    const int n_tiles = (p.n_out + C::kBN - 1) / C::kBN;
    const int num_tiles = m_tiles * n_tiles, kt_count = p.k / (2 * kBKBytes);
    // Tiles of this CTA: tile_begin, tile_begin + tile_step, ...; K steps
    // kt_begin .. kt_end - 1 of each. Split-K: one tile per cluster, one K
    // range per CTA of the cluster.
    const bool split = !GROUPED && p.split > 1;
    int tile_begin = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x, tile_step = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;
    int kt_begin = 0, kt_end = kt_count, rank = 0;
    if (split) {
        rank = (int)cluster_ctarank();
        tile_begin = blockIdx.x / p.split;
        tile_step = num_tiles;
        kt_begin = rank * kt_count / p.split;
        kt_end = (rank + 1) * kt_count / p.split;
    }
    const int kt_n = kt_end - kt_begin;
    const int64_t atoms_per_row_blk = (int64_t)(p.k / (FMT == kFmtNV ? 16 : 32)) / 4;
    const int64_t atoms_per_row_blk_s = SP ? atoms_per_row_blk / 2 : atoms_per_row_blk;

    if (warp == 0) {
        if (lane == 0) {
            int32_t last[C::kStages];
            for (int s = 0; s < C::kStages; ++s) last[s] = -1;
            uint32_t it = 0;
            bool ok = true;
            for (int tile = tile_begin; ok && tile < num_tiles; tile += tile_step) {
                int nb, mb;
                tile_coords<GROUPED, PAIR>(tile, m_tiles, n_tiles, mb, nb);
                const int rb = PAIR ? 2 * mb + (int)prank : mb;  // this CTA's 128-row block
                // its scale atoms: a pair's second block past the last one (odd
                // block counts) is all padding (A zero-filled by the tile load);
                // it takes block 0's atoms, so that no copy reads past the scale
                // arrays, and its rows are never stored
                const int rb_sf = (PAIR && rb * kBM >= p.m_tok) ? 0 : rb;
                const int grp = GROUPED ? group_of_tile(tiles, p.groups, mb) : 0;
                const uint8_t *sfb = p.sfb + (GROUPED ? (int64_t)grp * p.w_gstride : 0);
                for (int kt = kt_begin; kt < kt_end; ++kt, ++it) {
                    const int s = (int)(it % C::kStages);
                    const uint32_t ph = (it / C::kStages) & 1u;
                    if (!mbar_wait(empty_bar(s), ph ^ 1u, p.status, kSiteProducer, p.wait_ns)) {
                        ok = false;
                        break;
                    }
                    const uint32_t fb = full_bar(s), lb = sf_loaded_bar(s);
                    const uint32_t st = sbase + (uint32_t)(s * C::kStageBytes);
                    // Scale atoms first, on their own barrier: the scale
                    // writers move them to tensor memory while the operand
                    // tiles are still in flight.
                    const int64_t a_off = ((int64_t)rb_sf * atoms_per_row_blk + (int64_t)kt * kAtomsPerTile) * 512;
                    const int64_t a_off_s = ((int64_t)rb_sf * atoms_per_row_blk_s + (int64_t)kt * kAtomsS) * 512;
                    const int64_t b0 =
                        ((int64_t)(C::kBlk * nb) * atoms_per_row_blk_s + (int64_t)kt * kAtomsS) * 512;
                    mbar_arrive_expect_tx(lb, (1 + C::kBlk) * kSfBytesS + kSfBytes + C::kMetaBytes);
                    bulk_load(st + C::kOffSFAS, p.sfa_s + a_off_s, kSfBytesS, lb);
                    bulk_load(st + C::kOffSFAR, p.sfa_r + a_off, kSfBytes, lb);
#pragma unroll
                    for (int bk = 0; bk < C::kBlk; ++bk)  // the tile's 128-row W blocks
                        bulk_load(st + C::kOffSFB + bk * kSfBytesS, sfb + b0 + bk * atoms_per_row_blk_s * 512,
                                  kSfBytesS, lb);
                    if (SP) tma_load_2d(st + C::kOffMeta, &tm_meta, kt * 16, mb * kBM, lb);
                    if constexpr (PAIR) {
                        // both CTAs' tiles complete on the leader's barrier
                        if (leader) mbar_arrive_expect_tx(fb, 2 * (C::kASBytes + kABytes + C::kBBytes));
                        const uint32_t lfb = at_leader(fb);
                        tma_load_2d_pair(st + kOffAS, &tm_as, kt * kBKBytes, rb * kBM, lfb);
                        tma_load_2d_pair(st + C::kOffAR, &tm_ar, kt * kBKBytes, rb * kBM, lfb);
                        tma_load_2d_pair(st + C::kOffB, &tm_b, kt * kBKBytes, nb * C::kBN + (int)prank * (C::kBN / 2), lfb);
                    } else {
                        mbar_arrive_expect_tx(fb, C::kASBytes + kABytes + C::kBBytes);
                        tma_load_2d(st + kOffAS, &tm_as, kt * (SP ? kBKBytes / 2 : kBKBytes), mb * kBM, fb);
                        tma_load_2d(st + C::kOffAR, &tm_ar, kt * kBKBytes, mb * kBM, fb);
                        if (GROUPED) tma_load_3d(st + C::kOffB, &tm_b, kt * kBKBytes, nb * C::kBN, grp, fb);
                        else tma_load_2d(st + C::kOffB, &tm_b, kt * kBKBytes, nb * C::kBN, fb);
                    }
                    last[s] = (int32_t)it;
                }
            }
            // Never leave the CTA with copies in flight.
            // (pair: the operand tiles of both CTAs complete on the leader's
            // barriers, which the leader drains before the final cluster barrier)
            for (int s = 0; s < C::kStages; ++s)
                if (last[s] >= 0) {
                    if (!PAIR || leader) drain_wait(full_bar(s), ((uint32_t)last[s] / C::kStages) & 1u, kDrainNs);
                    drain_wait(sf_loaded_bar(s), ((uint32_t)last[s] / C::kStages) & 1u, kDrainNs);
                }
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0 && (!PAIR || leader)) {  // pair: the leader issues for both CTAs
            uint32_t it = 0, tile_iter = 0;
            for (int tile = tile_begin; tile < num_tiles; tile += tile_step, ++tile_iter) {
                // accumulator of this tile (two in turn at BN = 128)
                const int ab = (int)(tile_iter % C::kNacc);
                const uint32_t acc_par = ((tile_iter / C::kNacc) & 1u) ^ 1u;
                if (!mbar_wait(acc_empty_bar(ab), acc_par, p.status, kSiteMmaAcc, p.wait_ns)) break;
                tc_fence_after();
                const uint32_t dacc = tmem + (uint32_t)(ab * BN);
                bool ok = true;
                for (int kt = kt_begin; kt < kt_end; ++kt, ++it) {
                    const int s = (int)(it % C::kStages);
                    const uint32_t ph = (it / C::kStages) & 1u;
                    if (!mbar_wait(full_bar(s), ph, p.status, kSiteMmaFull, p.wait_ns)) {
                        ok = false;
                        break;
                    }
                    const int sb = (int)(it % C::kSfBufs);  // scale buffer of this stage
                    if (!mbar_wait(sf_full_bar(sb), (it / C::kSfBufs) & 1u, p.status, kSiteMmaScales, p.wait_ns)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t st = sbase + (uint32_t)(s * C::kStageBytes);
                    const uint32_t sf = tmem + C::kColSf0 + C::kSfBufCols * (uint32_t)sb;
                    const uint64_t da_s = SP ? desc_operand_half(st + kOffAS) : desc_operand(st + kOffAS);
                    const uint64_t da_r = desc_operand(st + C::kOffAR);
                    const uint64_t db = desc_operand(st + C::kOffB);
                    if constexpr (SP) {
                        // backbone: two sparse MMAs of 128 logical K (32 bytes of
                        // the compacted tile, 64 of the W tile) each
#pragma unroll
                        for (int j = 0; j < 2; ++j) {
                            const uint32_t acc = (kt != kt_begin || j != 0) ? 1u : 0u;
                            const uint32_t e = sf + C::kSpMeta + 4 * j;
                            if (FMT == kFmtNV) {
                                tc_mma_sp_nvf4(dacc, da_s + 2 * j, db + 4 * j, idesc_of<FMT, BN>(0) | (1u << 2),
                                               sf + C::kSpS + 4 * j, sf + C::kSpWb + 4 * C::kBlk * j, e, acc);
                            } else {
                                const uint32_t sf_id = (uint32_t)j * 2u;  // 2 scales per row per MMA
                                tc_mma_sp_mxf4(dacc, da_s + 2 * j, db + 4 * j, idesc_of<FMT, BN>(sf_id) | (1u << 2),
                                               (sf + C::kSpS) | (sf_id << 30), (sf + C::kSpWb) | (sf_id << 30), e,
                                               acc);
                            }
                        }
                        // residual: the dense MMAs of K = 64 on the W residual view
#pragma unroll
                        for (int j = 0; j < kMmaPerStage; ++j) {
                            if (FMT == kFmtNV) {
                                tc_mma_nvf4(dacc, da_r + 2 * j, db + 2 * j, idesc_of<FMT, BN>(0), sf + C::kSpR + 4 * j,
                                            sf + C::kSpWr + 4 * C::kBlk * j, 1u);
                            } else {
                                const uint32_t sf_id = (uint32_t)(j & 1) * 2u;
                                const uint32_t a_col = 4 * (j >> 1), b_col = 4 * C::kBlk * (j >> 1);
                                tc_mma_mxf4(dacc, da_r + 2 * j, db + 2 * j, idesc_of<FMT, BN>(sf_id),
                                            (sf + C::kSpR + a_col) | (sf_id << 30),
                                            (sf + C::kSpWr + b_col) | (sf_id << 30), 1u);
                            }
                        }
                    }
                    if constexpr (PAIR) {
                        // M = 256 over the pair: each CTA's A rows and W half at
                        // the same shared-memory offsets, the W scales of all
                        // BN rows in each CTA's tensor memory
#pragma unroll
                        for (int j = 0; j < kMmaPerStage; ++j) {
                            const uint32_t acc = (kt != kt_begin || j != 0) ? 1u : 0u;
                            if (FMT == kFmtNV) {
                                const uint32_t idesc = idesc_of<FMT, BN, 2 * kBM>(0);
                                const uint32_t b_col = 4 * C::kBlk * j;
                                tc_mma_nvf4_pair(dacc, da_s + 2 * j, db + 2 * j, idesc, sf + kSfaS + 4 * j,
                                                 sf + kSfb + b_col, acc);
                                tc_mma_nvf4_pair(dacc, da_r + 2 * j, db + 2 * j, idesc, sf + kSfaR + 4 * j,
                                                 sf + kSfb + b_col, 1u);
                            } else {
                                const uint32_t sf_id = (uint32_t)(j & 1) * 2u;
                                const uint32_t idesc = idesc_of<FMT, BN, 2 * kBM>(sf_id);
                                const uint32_t a_col = 4 * (j >> 1), b_col = 4 * C::kBlk * (j >> 1);
                                tc_mma_mxf4_pair(dacc, da_s + 2 * j, db + 2 * j, idesc,
                                                 (sf + kSfaS + a_col) | (sf_id << 30), (sf + kSfb + b_col) | (sf_id << 30),
                                                 acc);
                                tc_mma_mxf4_pair(dacc, da_r + 2 * j, db + 2 * j, idesc,
                                                 (sf + kSfaR + a_col) | (sf_id << 30), (sf + kSfb + b_col) | (sf_id << 30),
                                                 1u);
                            }
                        }
                    }
#pragma unroll
                    for (int j = 0; j < ((SP || PAIR) ? 0 : kMmaPerStage); ++j) {  // MMAs of K = 64 (32 bytes) per K tile
                        const uint32_t acc = (kt != kt_begin || j != 0) ? 1u : 0u;
                        // W scales: 4 columns per 128-row block per atom, the
                        // tile's blocks side by side
                        if (FMT == kFmtNV) {
                            const uint32_t idesc = idesc_of<FMT, BN>(0);
                            const uint32_t b_col = 4 * C::kBlk * j;
                            tc_mma_nvf4(dacc, da_s + 2 * j, db + 2 * j, idesc, sf + kSfaS + 4 * j, sf + kSfb + b_col, acc);
                            tc_mma_nvf4(dacc, da_r + 2 * j, db + 2 * j, idesc, sf + kSfaR + 4 * j, sf + kSfb + b_col, 1u);
                        } else {
                            const uint32_t sf_id = (uint32_t)(j & 1) * 2u;  // 2 scales per row per MMA
                            const uint32_t idesc = idesc_of<FMT, BN>(sf_id);
                            const uint32_t a_col = 4 * (j >> 1), b_col = 4 * C::kBlk * (j >> 1);
                            tc_mma_mxf4(dacc, da_s + 2 * j, db + 2 * j, idesc, (sf + kSfaS + a_col) | (sf_id << 30),
                                        (sf + kSfb + b_col) | (sf_id << 30), acc);
                            tc_mma_mxf4(dacc, da_r + 2 * j, db + 2 * j, idesc, (sf + kSfaR + a_col) | (sf_id << 30),
                                        (sf + kSfb + b_col) | (sf_id << 30), 1u);
                        }
                    }
                    if (PAIR) {  // frees the stage and the scale buffer in both CTAs
                        tc_commit_pair(empty_bar(s), 0x3);
                        tc_commit_pair(sf_empty_bar(sb), 0x3);
                    } else {
                        tc_commit(empty_bar(s));      // frees the stage once these MMAs complete
                        tc_commit(sf_empty_bar(sb));  // and the scale buffer
                    }
                }
                if (!ok) break;
                if (PAIR) tc_commit_pair(acc_full_bar(ab), 0x3);
                else tc_commit(acc_full_bar(ab));
            }
            if (PAIR) tc_commit_pair(drain_bar, 0x1);
            else tc_commit(drain_bar);  // every MMA of this thread done before exit
            drain_wait(drain_bar, 0, kDrainNs);
        }
        __syncwarp();
    } else if (warp >= 6) {
        // Warps 6..9, one per tensor-memory lane quadrant q: scale writes.
        // Each stage's scale atoms go from shared memory into one of
        // kSfBufs scale buffers in tensor memory through registers
        // (tcgen05.st, which does not occupy the MMA pipe as tcgen05.cp
        // does). Every lane of quadrant q receives row (lane) of each atom:
        // the columns a 32x128b.warpx4 copy fills, with the same bytes.
        // Stage i waits for its scale atoms and for the MMAs of stage
        // i - kSfBufs to release its buffer, so these warps run up to
        // kSfBufs stages ahead of the MMAs, across tile boundaries; they
        // depend on nothing the epilogue does.
        const int q = warp & 3;
        const uint32_t lane_base = (uint32_t)(q * 32) << 16;
        const int my_tiles = tile_begin < num_tiles ? (num_tiles - 1 - tile_begin) / tile_step + 1 : 0;
        const uint32_t total_stages = (uint32_t)my_tiles * (uint32_t)kt_n;
        for (uint32_t it = 0; it < total_stages; ++it) {
            const int s = (int)(it % C::kStages);
            const int b = (int)(it % C::kSfBufs);
            const bool w1 = mbar_wait(sf_loaded_bar(s), (it / C::kStages) & 1u, p.status, kSiteScaleFull, p.wait_ns);
            const bool w2 = w1 && mbar_wait(sf_empty_bar(b), ((it / C::kSfBufs) & 1u) ^ 1u, p.status, kSiteScaleEmpty,
                                            p.wait_ns);
            if (!__all_sync(0xFFFFFFFFu, w2)) break;  // warp-uniform: tcgen05.st is .aligned
            tc_fence_after();
            const uint32_t st = sbase + (uint32_t)(s * C::kStageBytes) + (uint32_t)lane * 16u;
            const uint32_t sf = tmem + lane_base + C::kColSf0 + C::kSfBufCols * (uint32_t)b;
            if constexpr (SP) {
#pragma unroll
                for (int a = 0; a < kAtomsS; ++a) {
                    tmem_st4(sf + C::kSpS + 4 * a, lds128(st + C::kOffSFAS + 512 * a));
#pragma unroll
                    for (int bk = 0; bk < C::kBlk; ++bk) {
                        const uint4 w = lds128(st + C::kOffSFB + bk * kSfBytesS + 512 * a);
                        tmem_st4(sf + C::kSpWb + 4 * C::kBlk * a + 4 * bk, w);
                        // the residual view: each scale of a 32 (64) value block
                        // for both of its 16 (32) value halves
                        const uint4 lo = make_uint4(__byte_perm(w.x, 0u, 0x1100u), __byte_perm(w.y, 0u, 0x1100u),
                                                    __byte_perm(w.z, 0u, 0x1100u), __byte_perm(w.w, 0u, 0x1100u));
                        const uint4 hi = make_uint4(__byte_perm(w.x, 0u, 0x3322u), __byte_perm(w.y, 0u, 0x3322u),
                                                    __byte_perm(w.z, 0u, 0x3322u), __byte_perm(w.w, 0u, 0x3322u));
                        tmem_st4(sf + C::kSpWr + 4 * C::kBlk * (2 * a) + 4 * bk, lo);
                        tmem_st4(sf + C::kSpWr + 4 * C::kBlk * (2 * a + 1) + 4 * bk, hi);
                    }
                }
#pragma unroll
                for (int a = 0; a < kAtomsPerTile; ++a)
                    tmem_st4(sf + C::kSpR + 4 * a, lds128(st + C::kOffSFAR + 512 * a));
                // metadata of this lane's row (lane quadrant q holds rows 32q ..):
                // the first 64 bits for the first sparse MMA, the rest for the second
                const uint4 mt = lds128(sbase + (uint32_t)(s * C::kStageBytes) + C::kOffMeta +
                                        (uint32_t)(q * 32 + lane) * 16u);
                tmem_st2(sf + C::kSpMeta, mt.x, mt.y);
                tmem_st2(sf + C::kSpMeta + 4, mt.z, mt.w);
            }
#pragma unroll
            for (int a = 0; a < (SP ? 0 : kAtomsPerTile); ++a) {
                tmem_st4(sf + kSfaS + 4 * a, lds128(st + C::kOffSFAS + 512 * a));
                tmem_st4(sf + kSfaR + 4 * a, lds128(st + C::kOffSFAR + 512 * a));
#pragma unroll
                for (int bk = 0; bk < C::kBlk; ++bk)
                    tmem_st4(sf + kSfb + 4 * C::kBlk * a + 4 * bk, lds128(st + C::kOffSFB + bk * kSfBytes + 512 * a));
            }
            tmem_st_wait();
            tc_fence_before();
            if (PAIR) mbar_arrive_cluster(at_leader(sf_full_bar(b)));  // the leader's MMAs wait for both CTAs
            else mbar_arrive(sf_full_bar(b));
        }
    } else {
        // Warps 2..5, one per tensor-memory lane quadrant q: epilogue. The
        // accumulator is drained from tensor memory into registers (as
        // packed fp16) and handed back to the MMA warp, so that the next
        // tile's MMAs overlap with this tile's global stores.
        const int q = warp & 3;
        const uint32_t lane_base = (uint32_t)(q * 32) << 16;
        const float s_t = *p.s_t;
        float alpha = __fmul_rn(s_t, *p.s_tw);
        // (short loops, fewer than 8 K steps, store at once: the next drain
        // comes too soon for pacing to pay)
        const unsigned store_pause_ns = kt_n >= 8 ? (unsigned)min(SQ_STORE_PAUSE_NS_PER_KSTEP * kt_n, 1000) : 0u;
        uint32_t tile_iter = 0;
        for (int tile = tile_begin; tile < num_tiles; tile += tile_step, ++tile_iter) {
            int nb, mb;
            tile_coords<GROUPED, PAIR>(tile, m_tiles, n_tiles, mb, nb);
            if constexpr (GROUPED) {
                const int grp = group_of_tile(tiles, p.groups, mb);
                alpha = __fmul_rn(s_t, *reinterpret_cast<const float *>(
                                           reinterpret_cast<const uint8_t *>(p.s_tw) + (int64_t)grp * p.w_gstride));
            }
            const int ab = (int)(tile_iter % C::kNacc);  // the accumulator this tile used
            const bool got =
                mbar_wait(acc_full_bar(ab), (tile_iter / C::kNacc) & 1u, p.status, kSiteEpilogue, p.wait_ns);
            if (!__all_sync(0xFFFFFFFFu, got)) break;  // warp-uniform: tcgen05.ld is .aligned
            tc_fence_after();
            const uint32_t acc_base = tmem + lane_base + (uint32_t)(ab * BN);
            if (split) {
                // Split-K: the fp32 partial tile (rows below m_tok) goes to
                // this CTA's stage memory, which no copy or MMA uses any
                // more; the cluster reduces it at the end of the kernel.
                const int row_local = q * 32 + lane;
                const bool keep = (int64_t)mb * kBM + row_local < p.m_tok;
                const uint32_t dst = sbase + (uint32_t)row_local * C::kPartStride;
#pragma unroll
                for (int cc = 0; cc < C::kBN / 32; ++cc) {
                    uint32_t r[32];
                    tmem_ld32(acc_base + (uint32_t)(cc * 32), r);
                    tmem_ld_wait();
                    if (keep) {
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            sts128(dst + (uint32_t)(cc * 128 + 16 * i), r[4 * i], r[4 * i + 1], r[4 * i + 2], r[4 * i + 3]);
                    }
                }
                break;  // one tile per CTA
            }
            // out = RN16(RN32(acc * alpha)) (packed multiplies round each
            // product to fp32 before the conversion); with a bias,
            // RN16(RN32(RN32(acc * alpha) + bias)) in scalar operations, so
            // that no multiply is fused into the add. Fused weights: alpha
            // per 32-column chunk (a chunk never spans two segments).
            uint32_t h[C::kBN / 32][16];
#pragma unroll
            for (int cc = 0; cc < C::kBN / 32; ++cc) {
                const int col0 = nb * C::kBN + cc * 32;
                float a_cc = alpha;
                if constexpr (EXT) a_cc = alpha_of_col(p, s_t, alpha, col0);
                uint32_t r[32];
                tmem_ld32(acc_base + (uint32_t)(cc * 32), r);
                tmem_ld_wait();
                if (EXT && p.bias != nullptr && col0 < p.n_out) {
                    const uint4 *bp = reinterpret_cast<const uint4 *>(p.bias + col0);  // same for every lane
#pragma unroll
                    for (int v4 = 0; v4 < 4; ++v4) {
                        const uint4 bw = __ldg(bp + v4);
                        const uint32_t bb[4] = {bw.x, bw.y, bw.z, bw.w};
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const int i = 4 * v4 + j;
                            const float2 b = __half22float2(*reinterpret_cast<const __half2 *>(&bb[j]));
                            const float y0 = __fadd_rn(__fmul_rn(__uint_as_float(r[2 * i]), a_cc), b.x);
                            const float y1 = __fadd_rn(__fmul_rn(__uint_as_float(r[2 * i + 1]), a_cc), b.y);
                            __half2 v = __floats2half2_rn(y0, y1);
                            h[cc][i] = *reinterpret_cast<uint32_t *>(&v);
                        }
                    }
                } else {
                    const uint64_t alpha2 = pk2(a_cc, a_cc);
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const float2 f =
                            up2(mul2(pk2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1])), alpha2));
                        __half2 v = __floats2half2_rn(f.x, f.y);
                        h[cc][i] = *reinterpret_cast<uint32_t *>(&v);
                    }
                }
            }
            tc_fence_before();
            if (PAIR) mbar_arrive_cluster(at_leader(acc_empty_bar(ab)));
            else mbar_arrive(acc_empty_bar(ab));
            int64_t row, row_end;  // output row of this lane; end of the tile's valid rows
            if constexpr (GROUPED) {
                // looked up again rather than kept live across the drain (register pressure)
                const int g2 = group_of_tile(tiles, p.groups, mb);
                const int32_t first = p.offsets[g2], last = p.offsets[g2 + 1];
                row = (int64_t)first + (int64_t)(mb - tiles[g2]) * kBM + q * 32 + lane;
                row_end = last;
            } else {
                row = (PAIR ? 2 * mb + (int)prank : mb) * kBM + q * 32 + lane;
                row_end = p.m_tok;
            }
            const unsigned pause_ns = tile + tile_step < num_tiles ? store_pause_ns : 0u;
            // The stores are spread over the next tile's main loop: every SM
            // reaches its tile boundary at about the same time, and a burst
            // of all their stores delays the operand loads the next tile
            // starts with. The pause per 32-column chunk scales with the
            // main loop's length (about 60 ns per K step, at most 1 us); the
            // CTA's last tile stores at once.
#pragma unroll
            for (int cc = 0; cc < C::kBN / 32; ++cc) {
                const int col0 = nb * C::kBN + cc * 32;
                if (row < row_end && col0 < p.n_out) {
                    // two full 32-byte sectors (the output base is 32-byte aligned,
                    // rows are multiples of 64 bytes)
                    __half *dst = p.out + row * p.n_out + col0;
                    stg256(dst, h[cc][0], h[cc][1], h[cc][2], h[cc][3], h[cc][4], h[cc][5], h[cc][6], h[cc][7]);
                    stg256(dst + 16, h[cc][8], h[cc][9], h[cc][10], h[cc][11], h[cc][12], h[cc][13], h[cc][14],
                           h[cc][15]);
                }
                if (cc + 1 < C::kBN / 32 && pause_ns) __nanosleep(pause_ns);
            }
        }
    }

    if (split) {
        // Split-K reduction: CTA `rank` of the cluster sums column slice
        // rank of the tile over every CTA's partial, in rank order (a fixed
        // order, so results do not depend on timing), reading the peers'
        // shared memory; then scales, rounds to fp16 and stores. All
        // threads of all CTAs pass both cluster barriers.
        cluster_sync();  // every partial is in its CTA's shared memory
        if (warp >= 2 && warp <= 5 && tile_begin < num_tiles) {
            int mb, nb;
            tile_coords<GROUPED, PAIR>(tile_begin, m_tiles, n_tiles, mb, nb);
            const int S = p.split, cols = C::kBN / S, groups4 = cols / 4;
            const int valid = (int)min((int64_t)kBM, (int64_t)p.m_tok - (int64_t)mb * kBM);
            const float s_t = *p.s_t;
            const float alpha0 = __fmul_rn(s_t, *p.s_tw);
            for (int item = (warp - 2) * 32 + lane; item < valid * groups4; item += 128) {
                const int r = item / groups4, col = rank * cols + (item % groups4) * 4;
                if (nb * C::kBN + col >= p.n_out) continue;
                const float alpha = EXT ? alpha_of_col(p, s_t, alpha0, nb * C::kBN + col) : alpha0;
                const uint32_t off = sbase + (uint32_t)r * C::kPartStride + (uint32_t)col * 4u;
                // every CTA's values in flight at once, then the sums in rank order
                float4 v[kMaxSplit];
#pragma unroll
                for (int c = 0; c < kMaxSplit; ++c)
                    v[c] = c < S ? ld_cluster_f4(mapa_shared(off, (uint32_t)c)) : make_float4(0.f, 0.f, 0.f, 0.f);
                float4 acc = v[0];
#pragma unroll
                for (int c = 1; c < kMaxSplit; ++c)
                    if (c < S) {
                        acc.x = __fadd_rn(acc.x, v[c].x);
                        acc.y = __fadd_rn(acc.y, v[c].y);
                        acc.z = __fadd_rn(acc.z, v[c].z);
                        acc.w = __fadd_rn(acc.w, v[c].w);
                    }
                float4 y = make_float4(__fmul_rn(acc.x, alpha), __fmul_rn(acc.y, alpha), __fmul_rn(acc.z, alpha),
                                       __fmul_rn(acc.w, alpha));
                if (EXT && p.bias != nullptr) {
                    const uint2 bw = *reinterpret_cast<const uint2 *>(p.bias + nb * C::kBN + col);
                    const float2 b01 = __half22float2(*reinterpret_cast<const __half2 *>(&bw.x));
                    const float2 b23 = __half22float2(*reinterpret_cast<const __half2 *>(&bw.y));
                    y = make_float4(__fadd_rn(y.x, b01.x), __fadd_rn(y.y, b01.y), __fadd_rn(y.z, b23.x),
                                    __fadd_rn(y.w, b23.y));
                }
                __half2 h0 = __floats2half2_rn(y.x, y.y);
                __half2 h1 = __floats2half2_rn(y.z, y.w);
                *reinterpret_cast<uint2 *>(p.out + ((int64_t)mb * kBM + r) * p.n_out + nb * C::kBN + col) =
                    make_uint2(*reinterpret_cast<uint32_t *>(&h0), *reinterpret_cast<uint32_t *>(&h1));
            }
        }
        cluster_sync();  // no CTA leaves while its partial is being read
    }

    tc_fence_before();
    if (PAIR) cluster_sync();  // both CTAs done with the pair's tensor memory and barriers
    else __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        if (PAIR) tmem_dealloc_pair(tmem, kTmemCols);
        else tmem_dealloc(tmem, kTmemCols);
    }
}

// ---------------------------------------------------------------------------
// Decode GEMM (up to kDecTok tokens): the weight rows are the MMA's M side
// and the tokens its N side, out^T = W (Q(S) + Q(R))^T. The block-scaled
// MMA has M = 128 (or 256) rows; with the activation as A, a handful of
// tokens would pay for 128 rows of tensor work, whereas here the tensor work
// is 128 x 16 per K slice and the launch streams the weight. One CTA per
// (128-row weight tile, K range); K ranges of a tile go to the CTAs of a
// cluster, which reduce their fp32 partials through distributed shared
// memory as dual_gemm_kernel's split-K does. Two CTAs fit on an SM: one of
// this launch and one of the next, which does its set-up as a programmatic
// dependent while this one runs. Per stage: the W tile (A), the
// backbone and residual tiles of the tokens (B, 16 rows, zero-filled past
// m_tok), the W scale atoms (A scales) and the activations' first scale
// atoms (B scales: the block-scaled MMA reads B scales in the layout of a
// 128-row operand). 8 warps: warp 0 loads, warp 1 allocates tensor memory
// and issues the MMAs, warps 4..7 move each stage's scales to tensor memory
// and, after the K loop, drain the accumulator (lane = weight row, column =
// token).
constexpr int kDecTok = 16;                       // token rows of the B tiles (MMA N)
constexpr int kDecThreads = 256;
constexpr int kDecW = kBM * kBKBytes;             // W tile bytes (128 rows)
constexpr int kDecB = kDecTok * kBKBytes;         // one activation tile
constexpr int kDecSf = 512 * (kBKBytes / 32);     // scale bytes of one 128-row operand per stage (NVFP4)
constexpr int kDecOffS = kDecW, kDecOffR = kDecW + kDecB, kDecOffSfW = kDecW + 2 * kDecB;
constexpr int kDecOffSfS = kDecOffSfW + kDecSf, kDecOffSfR = kDecOffSfS + kDecSf;
constexpr int kDecStage = kDecOffSfR + kDecSf;    // 26 KB, a multiple of 1024
#ifndef SQ_DEC_STAGES
#define SQ_DEC_STAGES 4
#endif
constexpr int kDecStages = SQ_DEC_STAGES;         // 4: two CTAs fit on an SM (8 measured no faster)
constexpr int kDecBarOff = kDecStages * kDecStage;
constexpr int kDecSfBufs = 4;
constexpr int kDecSfCols = 3 * 4 * (kBKBytes / 32);  // W, S, R atoms per stage, 4 columns each
constexpr int kDecTmemCols = 256;                    // accumulator (16 columns) + scale buffers
constexpr int kDecSmem = kDecBarOff + 256 + 1024;
constexpr uint32_t kDecPartStride = kBM * 4 + 16;    // split-K partial: [token][column] fp32 rows
static_assert(kDecStage % 1024 == 0, "decode stage alignment");
static_assert(kDecTok + kDecSfBufs * kDecSfCols <= kDecTmemCols, "decode tensor memory");
static_assert(kDecSmem <= 232448, "decode shared memory");
static_assert(kDecTok * kDecPartStride <= (uint32_t)kDecBarOff, "decode split-K partial fits the stages");

template <int FMT, bool EXT>
__global__ void __launch_bounds__(kDecThreads, 2)
decode_gemm_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_s,
                   const __grid_constant__ CUtensorMap tm_r, const GemmParams p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_s = smem_u32(smem_raw);
    uint8_t *smem = smem_raw + (((raw_s + 1023u) & ~1023u) - raw_s);
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar0 = sbase + kDecBarOff;
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (kDecStages + s); };
    auto sf_loaded_bar = [&](int s) { return bar0 + 8u * (2 * kDecStages + s); };
    auto sf_full_bar = [&](int b) { return bar0 + 8u * (3 * kDecStages + b); };
    auto sf_empty_bar = [&](int b) { return bar0 + 8u * (3 * kDecStages + kDecSfBufs + b); };
    const uint32_t acc_bar = bar0 + 8u * (3 * kDecStages + 2 * kDecSfBufs);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + kDecBarOff + 8 * (3 * kDecStages + 2 * kDecSfBufs + 1));
    constexpr int kAtoms = FMT == kFmtNV ? kBKBytes / 32 : kBKBytes / 64;  // scale atoms per operand per stage
    constexpr uint32_t kSfBytes = 512u * kAtoms;
    // columns of a scale buffer: W atoms, then the backbone's, then the residual's
    constexpr uint32_t kColS = 4 * kAtoms, kColR = 8 * kAtoms;

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int kt_count = p.k / (2 * kBKBytes);
    const int S = p.split, rank = S > 1 ? (int)cluster_ctarank() : 0;
    const int nb = (int)blockIdx.x / S;  // weight tile (128 output columns)
    const int kt_begin = rank * kt_count / S, kt_end = (rank + 1) * kt_count / S, kt_n = kt_end - kt_begin;
    const int64_t apr = (int64_t)(p.k / (FMT == kFmtNV ? 16 : 32)) / 4;  // scale atoms per 128-row block
    if (threadIdx.x == 0) {
        for (int s = 0; s < kDecStages; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
            mbar_init(sf_loaded_bar(s), 1);
        }
        for (int b = 0; b < kDecSfBufs; ++b) {
            mbar_init(sf_full_bar(b), 128);
            mbar_init(sf_empty_bar(b), 1);
        }
        mbar_init(acc_bar, 1);
        mbar_fence_init();
        prefetch_tmap(&tm_w);
        prefetch_tmap(&tm_s);
        prefetch_tmap(&tm_r);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), kDecTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    griddep_wait();  // launched as a programmatic dependent: memory only from here
    griddep_launch();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            int32_t last[kDecStages];
            for (int s = 0; s < kDecStages; ++s) last[s] = -1;
            for (int i = 0; i < kt_n; ++i) {
                const int kt = kt_begin + i, s = i % kDecStages;
                if (!mbar_wait(empty_bar(s), ((i / kDecStages) & 1) ^ 1, p.status, kSiteProducer, p.wait_ns)) break;
                const uint32_t st = sbase + (uint32_t)(s * kDecStage);
                const uint32_t lb = sf_loaded_bar(s), fb = full_bar(s);
                mbar_arrive_expect_tx(lb, 3 * kSfBytes);
                bulk_load(st + kDecOffSfW, p.sfb + ((int64_t)nb * apr + (int64_t)kt * kAtoms) * 512, kSfBytes, lb);
                bulk_load(st + kDecOffSfS, p.sfa_s + (int64_t)kt * kAtoms * 512, kSfBytes, lb);
                bulk_load(st + kDecOffSfR, p.sfa_r + (int64_t)kt * kAtoms * 512, kSfBytes, lb);
                mbar_arrive_expect_tx(fb, kDecW + 2 * kDecB);
                tma_load_2d(st, &tm_w, kt * kBKBytes, nb * kBM, fb);
                tma_load_2d(st + kDecOffS, &tm_s, kt * kBKBytes, 0, fb);
                tma_load_2d(st + kDecOffR, &tm_r, kt * kBKBytes, 0, fb);
                last[s] = i;
            }
            for (int s = 0; s < kDecStages; ++s)
                if (last[s] >= 0) {
                    drain_wait(full_bar(s), ((uint32_t)last[s] / kDecStages) & 1u, kDrainNs);
                    drain_wait(sf_loaded_bar(s), ((uint32_t)last[s] / kDecStages) & 1u, kDrainNs);
                }
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) {
            bool ok = true;
            for (int i = 0; i < kt_n && ok; ++i) {
                const int s = i % kDecStages, sb = i % kDecSfBufs;
                if (!mbar_wait(full_bar(s), (i / kDecStages) & 1, p.status, kSiteMmaFull, p.wait_ns) ||
                    !mbar_wait(sf_full_bar(sb), (i / kDecSfBufs) & 1, p.status, kSiteMmaScales, p.wait_ns)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t st = sbase + (uint32_t)(s * kDecStage);
                const uint32_t sf = tmem + kDecTok + kDecSfCols * (uint32_t)sb;
                const uint64_t dw = desc_operand(st), ds = desc_operand(st + kDecOffS), dr = desc_operand(st + kDecOffR);
#pragma unroll
                for (int j = 0; j < kMmaPerStage; ++j) {
                    const uint32_t acc = (i != 0 || j != 0) ? 1u : 0u;
                    if (FMT == kFmtNV) {
                        // M = 128 weight rows, N = kDecTok tokens
                        const uint32_t idesc = idesc_of<FMT, kDecTok>(0);
                        tc_mma_nvf4(tmem, dw + 2 * j, ds + 2 * j, idesc, sf + 4 * j, sf + kColS + 4 * j, acc);
                        tc_mma_nvf4(tmem, dw + 2 * j, dr + 2 * j, idesc, sf + 4 * j, sf + kColR + 4 * j, 1u);
                    } else {
                        const uint32_t sf_id = (uint32_t)(j & 1) * 2u;
                        const uint32_t idesc = idesc_of<FMT, kDecTok>(sf_id);
                        const uint32_t col = 4 * (j >> 1);
                        tc_mma_mxf4(tmem, dw + 2 * j, ds + 2 * j, idesc, (sf + col) | (sf_id << 30),
                                    (sf + kColS + col) | (sf_id << 30), acc);
                        tc_mma_mxf4(tmem, dw + 2 * j, dr + 2 * j, idesc, (sf + col) | (sf_id << 30),
                                    (sf + kColR + col) | (sf_id << 30), 1u);
                    }
                }
                tc_commit(empty_bar(s));
                tc_commit(sf_empty_bar(sb));
            }
            tc_commit(acc_bar);  // also every MMA done before exit
            drain_wait(acc_bar, 0, kDrainNs);
        }
        __syncwarp();
    } else if (warp >= 4) {
        // Scale writes (lane quadrant q), then the accumulator drain.
        const int q = warp & 3;
        const uint32_t lane_base = (uint32_t)(q * 32) << 16;
        bool ok = true;
        for (int i = 0; i < kt_n; ++i) {
            const int s = i % kDecStages, b = i % kDecSfBufs;
            const bool w1 = mbar_wait(sf_loaded_bar(s), (i / kDecStages) & 1, p.status, kSiteScaleFull, p.wait_ns);
            const bool w2 = w1 && mbar_wait(sf_empty_bar(b), ((i / kDecSfBufs) & 1) ^ 1, p.status, kSiteScaleEmpty,
                                            p.wait_ns);
            if (!__all_sync(0xFFFFFFFFu, w2)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t st = sbase + (uint32_t)(s * kDecStage) + (uint32_t)lane * 16u;
            const uint32_t sf = tmem + lane_base + kDecTok + kDecSfCols * (uint32_t)b;
#pragma unroll
            for (int a = 0; a < kAtoms; ++a) {
                tmem_st4(sf + 4 * a, lds128(st + kDecOffSfW + 512 * a));
                tmem_st4(sf + kColS + 4 * a, lds128(st + kDecOffSfS + 512 * a));
                tmem_st4(sf + kColR + 4 * a, lds128(st + kDecOffSfR + 512 * a));
            }
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(sf_full_bar(b));
        }
        const bool got = ok && mbar_wait(acc_bar, 0, p.status, kSiteEpilogue, p.wait_ns);
        if (__all_sync(0xFFFFFFFFu, got)) {
            tc_fence_after();
            uint32_t r[16];
            tmem_ld16(tmem + lane_base, r);
            tmem_ld_wait();
            const int col_local = q * 32 + lane, col = nb * kBM + col_local;  // this lane's output column
            if (S > 1) {
                // fp32 partial [token][column] in the stage memory, reduced below
#pragma unroll
                for (int t = 0; t < kDecTok; ++t)
                    if (t < p.m_tok)
                        *reinterpret_cast<uint32_t *>(smem + (uint32_t)t * kDecPartStride + (uint32_t)col_local * 4u) = r[t];
            } else if (col < p.n_out) {
                const float s_t = *p.s_t;
                const float alpha = EXT ? alpha_of_col(p, s_t, __fmul_rn(s_t, *p.s_tw), col) : __fmul_rn(s_t, *p.s_tw);
                const float b = (EXT && p.bias != nullptr) ? __half2float(p.bias[col]) : 0.0f;
#pragma unroll
                for (int t = 0; t < kDecTok; ++t)
                    if (t < p.m_tok) {
                        float y = __fmul_rn(__uint_as_float(r[t]), alpha);
                        if (EXT && p.bias != nullptr) y = __fadd_rn(y, b);
                        p.out[(int64_t)t * p.n_out + col] = __float2half_rn(y);
                    }
            }
        }
    }
    if (S > 1) {
        // Split-K: CTA `rank` sums column slice `rank` of the tile over every
        // CTA's partial in rank order (fixed order: results do not depend on
        // timing), then scales, rounds and stores.
        cluster_sync();
        if (warp >= 4) {
            const int c0 = rank * kBM / S, cols = (rank + 1) * kBM / S - c0;  // this CTA's column slice
            const float s_t = *p.s_t;
            const float alpha0 = __fmul_rn(s_t, *p.s_tw);
            for (int item = (warp - 4) * 32 + lane; item < p.m_tok * cols; item += 128) {
                const int t = item / cols, cl = c0 + item % cols, col = nb * kBM + cl;
                if (col >= p.n_out) continue;
                const uint32_t off = sbase + (uint32_t)t * kDecPartStride + (uint32_t)cl * 4u;
                // every CTA's value in flight at once, then the sum in rank order
                float v[kMaxSplit];
#pragma unroll
                for (int c = 0; c < kMaxSplit; ++c)
                    v[c] = c < S ? __uint_as_float(ld_cluster_u32(mapa_shared(off, (uint32_t)c))) : 0.0f;
                float acc = v[0];
#pragma unroll
                for (int c = 1; c < kMaxSplit; ++c)
                    if (c < S) acc = __fadd_rn(acc, v[c]);
                float y = __fmul_rn(acc, EXT ? alpha_of_col(p, s_t, alpha0, col) : alpha0);
                if (EXT && p.bias != nullptr) y = __fadd_rn(y, __half2float(p.bias[col]));
                p.out[(int64_t)t * p.n_out + col] = __float2half_rn(y);
            }
        }
        cluster_sync();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kDecTmemCols);
    }
}

// Failure-detection probe: one thread waits, with the bounded wait the GEMM
// uses, on an mbarrier that nothing ever arrives at. The wait runs out and
// records kSiteProbe; the kernel then returns normally.
__global__ void wait_probe_kernel(unsigned *status, uint64_t limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    const uint32_t b = smem_u32(&bar);
    if (threadIdx.x == 0) {
        mbar_init(b, 1);
        mbar_fence_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait(b, 0, status, kSiteProbe, limit_ns);
}

sharq_status launch_wait_probe(LaunchCtx &ctx, uint64_t limit_ns) {
    wait_probe_kernel<<<1, 32, 0, ctx.stream>>>(ctx.status, limit_ns);
    ctx.launches++;
    SQ_CUDA_TRY(cudaGetLastError());
    return SHARQ_OK;
}

// ---------------------------------------------------------------------------
// Host side

static PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    // Initialised once (thread-safe static initialisation), also when host
    // threads make their first calls concurrently.
    static const PFN_cuTensorMapEncodeTiled_v12000 fn = []() -> PFN_cuTensorMapEncodeTiled_v12000 {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
        return nullptr;
    }();
    return fn;
}

// 2-D byte tensor [rows][row_bytes], box = box_bytes x box_rows (default: the
// K tile, swizzled in kBKBytes-wide atoms; 64 bytes: the sparse mode's
// compacted backbone, 64-byte swizzle; 16 bytes: its metadata, unswizzled).
static bool make_code_map(CUtensorMap *tm, const void *base, uint64_t row_bytes, uint64_t rows, uint32_t box_rows,
                          uint32_t box_bytes = kBKBytes) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    cuuint64_t dims[2] = {row_bytes, rows};
    cuuint64_t strides[1] = {row_bytes};
    cuuint32_t box[2] = {(cuuint32_t)box_bytes, box_rows};
    cuuint32_t estr[2] = {1, 1};
    const CUtensorMapSwizzle sw = box_bytes == 128  ? CU_TENSOR_MAP_SWIZZLE_128B
                                  : box_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                    : CU_TENSOR_MAP_SWIZZLE_NONE;
    CUresult r = enc(tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// 3-D byte tensor [groups][rows][row_bytes] with `group_stride` bytes
// between groups; box = kBKBytes x box_rows x 1, swizzled like make_code_map.
static bool make_grouped_code_map(CUtensorMap *tm, const void *base, uint64_t row_bytes, uint64_t rows,
                                  uint64_t groups, uint64_t group_stride, uint32_t box_rows) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    cuuint64_t dims[3] = {row_bytes, rows, groups};
    cuuint64_t strides[2] = {row_bytes, group_stride};
    cuuint32_t box[3] = {(cuuint32_t)kBKBytes, box_rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE,
                     kBKBytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <int FMT, bool GROUPED, bool EXT, int BN, bool SP = false, bool PAIR = false>
static sharq_status set_gemm_attrs() {
    static bool attr_done[64] = {};
    static std::mutex mu;  // one setter per device, also under concurrent first calls
    int dev = 0;
    SQ_CUDA_TRY(cudaGetDevice(&dev));
    if (dev < 0 || dev >= 64) return SHARQ_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(mu);
    if (!attr_done[dev]) {
        SQ_CUDA_TRY(cudaFuncSetAttribute(dual_gemm_kernel<FMT, GROUPED, EXT, BN, SP, PAIR>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, TileCfg<BN, SP, PAIR>::kSmemBytes));
        attr_done[dev] = true;
    }
    return SHARQ_OK;
}

template <int FMT, bool GROUPED, bool EXT, int BN, bool SP = false>
static sharq_status launch_gemm(LaunchCtx &ctx, const CUtensorMap &tm_as, const CUtensorMap &tm_ar,
                                const CUtensorMap &tm_b, const CUtensorMap &tm_meta, const GemmParams &gp,
                                int64_t max_tiles) {
    sharq_status st = set_gemm_attrs<FMT, GROUPED, EXT, BN, SP>();
    if (st != SHARQ_OK) return st;
    const unsigned grid = (unsigned)(max_tiles < ctx.num_sms ? max_tiles : ctx.num_sms);
    cudaLaunchConfig_t cfg;
    memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3(grid, 1, 1);
    cfg.blockDim = dim3(kGemmThreads, 1, 1);
    cfg.dynamicSmemBytes = TileCfg<BN, SP>::kSmemBytes;
    cfg.stream = ctx.stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = GROUPED ? 0 : 1;  // dense launches: a programmatic dependent of the previous kernel
    SQ_CUDA_TRY(cudaLaunchKernelEx(&cfg, dual_gemm_kernel<FMT, GROUPED, EXT, BN, SP>, tm_as, tm_ar, tm_b, tm_meta, gp));
    ctx.launches++;
    SQ_CUDA_TRY(cudaGetLastError());
    return SHARQ_OK;
}

// Pair launch: clusters of two CTAs, each pair walking 256-row tiles
// (`pair_tiles` of them) with the grid stride; as many pairs as can be
// resident at once.
template <int FMT, bool EXT>
static sharq_status launch_gemm_pair(LaunchCtx &ctx, const CUtensorMap &tm_as, const CUtensorMap &tm_ar,
                                     const CUtensorMap &tm_b, const GemmParams &gp, int64_t pair_tiles) {
    sharq_status st = set_gemm_attrs<FMT, false, EXT, kDenseBN, false, true>();
    if (st != SHARQ_OK) return st;
    static int cache[64] = {0};
    static std::mutex mu;
    int dev = 0;
    SQ_CUDA_TRY(cudaGetDevice(&dev));
    if (dev < 0 || dev >= 64) return SHARQ_ERR_UNSUPPORTED;
    cudaLaunchConfig_t cfg;
    memset(&cfg, 0, sizeof(cfg));
    cfg.blockDim = dim3(kGemmThreads, 1, 1);
    cfg.dynamicSmemBytes = TileCfg<kDenseBN, false, true>::kSmemBytes;
    cfg.stream = ctx.stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    int pairs = 0;
    {
        std::lock_guard<std::mutex> lock(mu);
        if (!cache[dev]) {
            cfg.gridDim = dim3(2, 1, 1);
            cfg.numAttrs = 1;
            int n = 0;
            if (cudaOccupancyMaxActiveClusters(&n, dual_gemm_kernel<FMT, false, EXT, kDenseBN, false, true>, &cfg) !=
                    cudaSuccess ||
                n < 1) {
                cudaGetLastError();
                n = ctx.num_sms / 2;
            }
            cache[dev] = n;
        }
        pairs = cache[dev];
    }
    if (pair_tiles < pairs) pairs = (int)pair_tiles;
    cfg.gridDim = dim3((unsigned)(2 * pairs), 1, 1);
    cfg.numAttrs = 2;
    SQ_CUDA_TRY(cudaLaunchKernelEx(&cfg, dual_gemm_kernel<FMT, false, EXT, kDenseBN, false, true>, tm_as, tm_ar, tm_b,
                                   tm_b, gp));
    ctx.launches++;
    SQ_CUDA_TRY(cudaGetLastError());
    return SHARQ_OK;
}

// Pair launches for the default mode's shapes of two or more 128-row tiles
// when SHARQ_GEMM_PAIR=1 is set in the environment (read once per process).
// Off by default: on B200 the pair kernel is correct but slower than the
// single-CTA kernel (down projection 8192 x 4096 x 14336: 0.43 ms against
// 0.30 ms), its tensor pipe idle half of the time between stages.
static bool pair_enabled() {
    static const bool on = []() {
        const char *e = getenv("SHARQ_GEMM_PAIR");
        return e && e[0] == '1';
    }();
    return on;
}

// Split-K launch: `tiles` clusters of gp.split CTAs, one tile per cluster.
template <int FMT, bool EXT, bool SP = false, int BN = kDenseBN>
static sharq_status launch_gemm_split(LaunchCtx &ctx, const CUtensorMap &tm_as, const CUtensorMap &tm_ar,
                                      const CUtensorMap &tm_b, const CUtensorMap &tm_meta, const GemmParams &gp,
                                      int64_t tiles) {
    sharq_status st = set_gemm_attrs<FMT, false, EXT, BN, SP>();
    if (st != SHARQ_OK) return st;
    cudaLaunchConfig_t cfg;
    memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3((unsigned)(tiles * gp.split), 1, 1);
    cfg.blockDim = dim3(kGemmThreads, 1, 1);
    cfg.dynamicSmemBytes = TileCfg<BN, SP>::kSmemBytes;
    cfg.stream = ctx.stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)gp.split;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    SQ_CUDA_TRY(cudaLaunchKernelEx(&cfg, dual_gemm_kernel<FMT, false, EXT, BN, SP>, tm_as, tm_ar, tm_b, tm_meta, gp));
    ctx.launches++;
    SQ_CUDA_TRY(cudaGetLastError());
    return SHARQ_OK;
}

// Clusters of `split` CTAs of this kernel that can be resident at once (0 if
// such a cluster does not fit), cached per device, format and size.
template <int FMT, int BN = kDenseBN>
static int active_clusters(int split) {
    static int cache[64][kMaxSplit + 1];
    static bool known[64][kMaxSplit + 1] = {};
    static std::mutex mu;  // set_gemm_attrs below takes its own lock (never this one)
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64 || split > kMaxSplit) return 0;
    std::lock_guard<std::mutex> lock(mu);
    if (!known[dev][split]) {
        if (set_gemm_attrs<FMT, false, false, BN>() != SHARQ_OK) return 0;
        cudaLaunchConfig_t cfg;
        memset(&cfg, 0, sizeof(cfg));
        cfg.gridDim = dim3((unsigned)split, 1, 1);
        cfg.blockDim = dim3(kGemmThreads, 1, 1);
        cfg.dynamicSmemBytes = TileCfg<BN>::kSmemBytes;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = (unsigned)split;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, dual_gemm_kernel<FMT, false, false, BN>, &cfg) != cudaSuccess) {
            cudaGetLastError();
            n = 0;
        }
        cache[dev][split] = n;
        known[dev][split] = true;
    }
    return cache[dev][split];
}

// Split-K factor for a dense launch: when the tiles fill less than half the
// SMs, the largest power of two <= 8 with tiles x split <= SMs, split <= K
// steps, and all the clusters resident at once; 1 otherwise.
template <int FMT, int BN = kDenseBN>
static int choose_split(LaunchCtx &ctx, int64_t tiles, int kt_count) {
    if (tiles * 2 > ctx.num_sms) return 1;
    int s = kMaxSplit;
    while (s > 1 && (tiles * s > ctx.num_sms || s > kt_count || active_clusters<FMT, BN>(s) < tiles)) s >>= 1;
    return s;
}

// Decode launches: clusters of gp.split CTAs per 128-row W tile.
template <int FMT, bool EXT>
static sharq_status set_decode_attrs() {
    static bool attr_done[64] = {};
    static std::mutex mu;
    int dev = 0;
    SQ_CUDA_TRY(cudaGetDevice(&dev));
    if (dev < 0 || dev >= 64) return SHARQ_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(mu);
    if (!attr_done[dev]) {
        SQ_CUDA_TRY(cudaFuncSetAttribute(decode_gemm_kernel<FMT, EXT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kDecSmem));
        attr_done[dev] = true;
    }
    return SHARQ_OK;
}

// Decode clusters of `split` CTAs that can be resident at once, cached per
// device and format.
template <int FMT>
static int decode_active_clusters(int split) {
    static int cache[64][kMaxSplit + 1];
    static bool known[64][kMaxSplit + 1] = {};
    static std::mutex mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64 || split > kMaxSplit) return 0;
    std::lock_guard<std::mutex> lock(mu);
    if (!known[dev][split]) {
        if (set_decode_attrs<FMT, false>() != SHARQ_OK) return 0;
        cudaLaunchConfig_t cfg;
        memset(&cfg, 0, sizeof(cfg));
        cfg.gridDim = dim3((unsigned)split, 1, 1);
        cfg.blockDim = dim3(kDecThreads, 1, 1);
        cfg.dynamicSmemBytes = kDecSmem;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = (unsigned)split;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, decode_gemm_kernel<FMT, false>, &cfg) != cudaSuccess) {
            cudaGetLastError();
            n = 0;
        }
        cache[dev][split] = n;
        known[dev][split] = true;
    }
    return cache[dev][split];
}

// Split-K factor of a decode launch: the largest split <= 8 (any integer)
// with tiles x split <= SQ_DECODE_WAVE CTAs per SM, split <= K steps and
// every cluster resident at once. One CTA per SM (the default) leaves each
// SM room for a CTA of the next launch, which then does its set-up while
// this one runs (a programmatic dependent). Measured on B200: the same time
// as two per SM (and an L2 prefetch of the weight before the dependency
// wait, by TMA or by plain prefetch instructions, made the layer set's
// decode GEMMs slower: it delays the running kernel's own loads).
#ifndef SQ_DECODE_WAVE
#define SQ_DECODE_WAVE 1
#endif
template <int FMT>
static int choose_decode_split(LaunchCtx &ctx, int64_t tiles, int kt_count) {
    int s = kMaxSplit;
    while (s > 1 && (tiles * s > SQ_DECODE_WAVE * (int64_t)ctx.num_sms || s > kt_count ||
                     decode_active_clusters<FMT>(s) < tiles))
        --s;
    return s;
}

template <int FMT, bool EXT>
static sharq_status launch_decode(LaunchCtx &ctx, const CUtensorMap &tm_w, const CUtensorMap &tm_s,
                                  const CUtensorMap &tm_r, const GemmParams &gp, int64_t tiles) {
    sharq_status st = set_decode_attrs<FMT, EXT>();
    if (st != SHARQ_OK) return st;
    cudaLaunchConfig_t cfg;
    memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3((unsigned)(tiles * gp.split), 1, 1);
    cfg.blockDim = dim3(kDecThreads, 1, 1);
    cfg.dynamicSmemBytes = kDecSmem;
    cfg.stream = ctx.stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = (unsigned)gp.split;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = gp.split > 1 ? 2 : 1;
    SQ_CUDA_TRY(cudaLaunchKernelEx(&cfg, decode_gemm_kernel<FMT, EXT>, tm_w, tm_s, tm_r, gp));
    ctx.launches++;
    SQ_CUDA_TRY(cudaGetLastError());
    return SHARQ_OK;
}

static GemmParams gemm_params(LaunchCtx &ctx, const sharq_prep &P, const sharq_wq &W, void *out) {
    GemmParams gp;
    memset(&gp, 0, sizeof(gp));
    gp.sfa_s = (const uint8_t *)P.s_scales;
    gp.sfa_r = (const uint8_t *)P.r_scales;
    gp.sfb = (const uint8_t *)W.scales_backbone;  // the residual view holds the same bytes
    gp.s_t = P.tensor_scale;
    gp.s_tw = W.tensor_scale;
    gp.out = (__half *)out;
    gp.m_tok = (int32_t)P.m_tok;
    gp.n_out = (int32_t)W.n_out;
    gp.k = (int32_t)P.k;
    gp.status = ctx.status;
    gp.wait_ns = ctx.wait_ns;
    gp.split = 1;
    gp.segs = W.segments > 1 ? W.segments : 1;
    for (int g = 0; g < gp.segs && g < SHARQ_SEGMENTS_MAX; ++g) gp.seg_end[g] = W.seg_end[g];
    gp.bias = nullptr;
    return gp;
}

sharq_status launch_linear(LaunchCtx &ctx, const sharq_prep &P, const sharq_wq &W, const void *bias, void *out) {
    if (P.m_tok == 0) return SHARQ_OK;
    const bool sp = P.sparse != 0;
    GemmParams gp = gemm_params(ctx, P, W, out);
    gp.bias = (const __half *)bias;
    const int kt_count = (int)(P.k / (2 * kBKBytes));
    // the extended epilogue (fused segments, bias) only where needed
    const bool ext = gp.bias != nullptr || gp.segs > 1;
    if (!sp && P.m_tok <= kDecTok) {
        // decode: W rows on the MMA's M side, the tokens on its N side
        CUtensorMap tm_w, tm_s, tm_r;
        if (!make_code_map(&tm_w, W.codes, (uint64_t)(W.k / 2), (uint64_t)W.n_out, kBM) ||
            !make_code_map(&tm_s, P.s_codes, (uint64_t)(P.k / 2), (uint64_t)P.m_tok, kDecTok) ||
            !make_code_map(&tm_r, P.r_codes, (uint64_t)(P.k / 2), (uint64_t)P.m_tok, kDecTok))
            return SHARQ_ERR_CUDA;
        const int64_t w_tiles = (W.n_out + kBM - 1) / kBM;
        gp.split = P.fmt == kFmtNV ? choose_decode_split<kFmtNV>(ctx, w_tiles, kt_count)
                                   : choose_decode_split<kFmtMX>(ctx, w_tiles, kt_count);
        if (ext)
            return P.fmt == kFmtNV ? launch_decode<kFmtNV, true>(ctx, tm_w, tm_s, tm_r, gp, w_tiles)
                                   : launch_decode<kFmtMX, true>(ctx, tm_w, tm_s, tm_r, gp, w_tiles);
        return P.fmt == kFmtNV ? launch_decode<kFmtNV, false>(ctx, tm_w, tm_s, tm_r, gp, w_tiles)
                               : launch_decode<kFmtMX, false>(ctx, tm_w, tm_s, tm_r, gp, w_tiles);
    }
    CUtensorMap tm_as, tm_ar, tm_b, tm_meta;
    if (!make_code_map(&tm_as, P.s_codes, (uint64_t)(P.k / (sp ? 4 : 2)), (uint64_t)P.m_tok, kBM,
                       sp ? kBKBytes / 2 : kBKBytes) ||
        !make_code_map(&tm_ar, P.r_codes, (uint64_t)(P.k / 2), (uint64_t)P.m_tok, kBM) ||
        !make_code_map(&tm_b, W.codes, (uint64_t)(W.k / 2), (uint64_t)W.n_out, kDenseBN))
        return SHARQ_ERR_CUDA;
    if (sp) {
        if (!make_code_map(&tm_meta, P.meta, (uint64_t)(P.k / 16), (uint64_t)P.m_tok, kBM, 16)) return SHARQ_ERR_CUDA;
    } else {
        tm_meta = tm_b;  // unused
    }
    const int64_t tiles = ((P.m_tok + kBM - 1) / kBM) * ((W.n_out + kDenseBN - 1) / kDenseBN);
    gp.split = P.fmt == kFmtNV ? choose_split<kFmtNV>(ctx, tiles, kt_count) : choose_split<kFmtMX>(ctx, tiles, kt_count);
    if (sp) {  // no bias or fused segments in this mode (checked by the caller)
        if (gp.split > 1)
            return P.fmt == kFmtNV ? launch_gemm_split<kFmtNV, false, true>(ctx, tm_as, tm_ar, tm_b, tm_meta, gp, tiles)
                                   : launch_gemm_split<kFmtMX, false, true>(ctx, tm_as, tm_ar, tm_b, tm_meta, gp, tiles);
        return P.fmt == kFmtNV
                   ? launch_gemm<kFmtNV, false, false, kDenseBN, true>(ctx, tm_as, tm_ar, tm_b, tm_meta, gp, tiles)
                   : launch_gemm<kFmtMX, false, false, kDenseBN, true>(ctx, tm_as, tm_ar, tm_b, tm_meta, gp, tiles);
    }
    const int64_t m_tiles = (P.m_tok + kBM - 1) / kBM;
    if (gp.split == 1 && m_tiles >= 2 && pair_enabled()) {
        // CTA pairs on 256-row tiles: W staged half per CTA
        CUtensorMap tm_bh;
        if (!make_code_map(&tm_bh, W.codes, (uint64_t)(W.k / 2), (uint64_t)W.n_out, kDenseBN / 2)) return SHARQ_ERR_CUDA;
        const int64_t pair_tiles = ((P.m_tok + 2 * kBM - 1) / (2 * kBM)) * ((W.n_out + kDenseBN - 1) / kDenseBN);
        if (ext)
            return P.fmt == kFmtNV ? launch_gemm_pair<kFmtNV, true>(ctx, tm_as, tm_ar, tm_bh, gp, pair_tiles)
                                   : launch_gemm_pair<kFmtMX, true>(ctx, tm_as, tm_ar, tm_bh, gp, pair_tiles);
        return P.fmt == kFmtNV ? launch_gemm_pair<kFmtNV, false>(ctx, tm_as, tm_ar, tm_bh, gp, pair_tiles)
                               : launch_gemm_pair<kFmtMX, false>(ctx, tm_as, tm_ar, tm_bh, gp, pair_tiles);
    }
    if (gp.split > 1) {
        if (ext)
            return P.fmt == kFmtNV ? launch_gemm_split<kFmtNV, true>(ctx, tm_as, tm_ar, tm_b, tm_meta, gp, tiles)
                                   : launch_gemm_split<kFmtMX, true>(ctx, tm_as, tm_ar, tm_b, tm_meta, gp, tiles);
        return P.fmt == kFmtNV ? launch_gemm_split<kFmtNV, false>(ctx, tm_as, tm_ar, tm_b, tm_meta, gp, tiles)
                               : launch_gemm_split<kFmtMX, false>(ctx, tm_as, tm_ar, tm_b, tm_meta, gp, tiles);
    }
    if (ext)
        return P.fmt == kFmtNV ? launch_gemm<kFmtNV, false, true, kDenseBN>(ctx, tm_as, tm_ar, tm_b, tm_meta, gp, tiles)
                               : launch_gemm<kFmtMX, false, true, kDenseBN>(ctx, tm_as, tm_ar, tm_b, tm_meta, gp, tiles);
    return P.fmt == kFmtNV ? launch_gemm<kFmtNV, false, false, kDenseBN>(ctx, tm_as, tm_ar, tm_b, tm_meta, gp, tiles)
                           : launch_gemm<kFmtMX, false, false, kDenseBN>(ctx, tm_as, tm_ar, tm_b, tm_meta, gp, tiles);
}

sharq_status launch_linear_grouped(LaunchCtx &ctx, const sharq_prep &P, const sharq_wq &W, const int32_t *offsets,
                                   int32_t groups, int64_t rows, int64_t w_gstride, void *out) {
    CUtensorMap tm_as, tm_ar, tm_b;
    if (!make_code_map(&tm_as, P.s_codes, (uint64_t)(P.k / 2), (uint64_t)P.m_tok, kBM) ||
        !make_code_map(&tm_ar, P.r_codes, (uint64_t)(P.k / 2), (uint64_t)P.m_tok, kBM) ||
        !make_grouped_code_map(&tm_b, W.codes, (uint64_t)(W.k / 2), (uint64_t)W.n_out, (uint64_t)groups,
                               (uint64_t)w_gstride, kGroupedBN))
        return SHARQ_ERR_CUDA;
    GemmParams gp = gemm_params(ctx, P, W, out);
    gp.segs = 1;  // stacked experts, never fused segments
    gp.offsets = offsets;
    gp.groups = groups;
    gp.rows = rows;
    gp.w_gstride = w_gstride;
    // at most P.m_tok / 128 m tiles (the device checks the offsets against it)
    const int64_t tiles = (P.m_tok / kBM) * ((W.n_out + kGroupedBN - 1) / kGroupedBN);
    if (tiles == 0) return SHARQ_OK;
    return P.fmt == kFmtNV ? launch_gemm<kFmtNV, true, false, kGroupedBN>(ctx, tm_as, tm_ar, tm_b, tm_b, gp, tiles)
                           : launch_gemm<kFmtMX, true, false, kGroupedBN>(ctx, tm_as, tm_ar, tm_b, tm_b, gp, tiles);
}

}  // namespace sq

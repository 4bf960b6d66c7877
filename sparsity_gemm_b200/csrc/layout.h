// Buffer layouts of the SharQ library (host and device). Not shared with the
// CPU oracle, which uses plain row-major arrays.
#pragma once
#include <stdint.h>

#ifdef __CUDACC__
#define SQ_HD __host__ __device__ __forceinline__
#else
#define SQ_HD static inline
#endif

namespace sq {

constexpr int kFmtNV = 0;
constexpr int kFmtMX = 1;
constexpr int64_t kAlign = 256;      // section alignment inside caller buffers
constexpr int64_t kActRowPad = 128;  // scale-layout rows: activations
constexpr int64_t kWRowPad = 256;    // scale-layout rows: weights (GEMM N tile)

SQ_HD int blk_of(int fmt) { return fmt == kFmtNV ? 16 : 32; }
SQ_HD int64_t round_up(int64_t v, int64_t a) { return (v + a - 1) / a * a; }
SQ_HD int idx_bits(int m) { return m <= 2 ? 1 : m <= 4 ? 2 : m <= 8 ? 3 : 4; }

// Byte offset of scale (row r, block j) in the MMA scale view of a matrix
// with `nblk` blocks per row: 512-byte atoms of 128 rows x 4 scales, row
// r = r0 + 32 r1 (r0 < 32, r1 < 4) at r0 * 16 + r1 * 4.
SQ_HD int64_t sf_offset(int64_t r, int64_t j, int64_t nblk) {
    return ((r >> 7) * (nblk >> 2) + (j >> 2)) * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4 + (j & 3);
}

// Mask-metadata bytes per row.
SQ_HD int64_t meta_row_bytes(int64_t k, int n, int m) {
    return ((k / m) * n * idx_bits(m) + 7) / 8;
}

// Rows of a grouped prep: every group starts at a multiple of 128 rows.
constexpr int64_t kGroupsMax = 1024;
SQ_HD int64_t grouped_rows(int64_t rows, int64_t groups) { return round_up(rows + 127 * groups, kActRowPad); }

// Sections of a prep buffer.
struct PrepLayout {
    int64_t s_codes, r_codes, s_scales, r_scales, meta, stats, words, total;
    int64_t sf_rows, sf_bytes, meta_row;
};

SQ_HD PrepLayout prep_layout(int64_t m_tok, int64_t k, int n, int m, int fmt) {
    PrepLayout L;
    int64_t codes = m_tok * (k / 2);
    L.sf_rows = round_up(m_tok > 0 ? m_tok : 1, kActRowPad);
    L.sf_bytes = L.sf_rows * (k / blk_of(fmt));
    L.meta_row = meta_row_bytes(k, n, m);
    int64_t off = 0;
    L.s_codes = off; off = round_up(off + codes, kAlign);
    L.r_codes = off; off = round_up(off + codes, kAlign);
    L.s_scales = off; off = round_up(off + L.sf_bytes, kAlign);
    L.r_scales = off; off = round_up(off + L.sf_bytes, kAlign);
    L.meta = off; off = round_up(off + m_tok * L.meta_row, kAlign);
    L.stats = off; off = round_up(off + m_tok * 8, kAlign);   // float2 (mu, rstd) per row
    L.words = off; off = round_up(off + 64, kAlign);          // [0] amax bits, [1] s_t
    L.total = off;
    return L;
}

// Sections of a prep buffer in the pair-wise 4:8 mode: backbone codes
// K-compacted to the kept half ([rows][k/4] bytes), backbone scales one per
// 2 blk values, metadata 4 bits per group of 8 ([rows][k/16] bytes, the
// layout the sparse MMA reads: group g of a row in bits 4g .. 4g+3, the
// lower kept pair's index in the low two bits); residual as in prep_layout.
SQ_HD PrepLayout prep_layout_sparse(int64_t m_tok, int64_t k, int fmt) {
    PrepLayout L;
    L.sf_rows = round_up(m_tok > 0 ? m_tok : 1, kActRowPad);
    L.sf_bytes = L.sf_rows * (k / blk_of(fmt));  // residual scales
    L.meta_row = k / 16;
    const int64_t s_sf = L.sf_rows * (k / (2 * blk_of(fmt)));
    int64_t off = 0;
    L.s_codes = off; off = round_up(off + m_tok * (k / 4), kAlign);
    L.r_codes = off; off = round_up(off + m_tok * (k / 2), kAlign);
    L.s_scales = off; off = round_up(off + s_sf, kAlign);
    L.r_scales = off; off = round_up(off + L.sf_bytes, kAlign);
    L.meta = off; off = round_up(off + m_tok * L.meta_row, kAlign);
    L.stats = off; off = round_up(off + m_tok * 8, kAlign);
    L.words = off; off = round_up(off + 64, kAlign);
    L.total = off;
    return L;
}

struct WLayout {
    int64_t codes, scales, words, total, sf_rows, sf_bytes;
};

// sparse: the pair-wise mode's weights, one scale per 2 blk values.
SQ_HD WLayout w_layout(int64_t n_out, int64_t k, int fmt, bool sparse = false) {
    WLayout L;
    L.sf_rows = round_up(n_out, kWRowPad);
    L.sf_bytes = L.sf_rows * (k / (blk_of(fmt) * (sparse ? 2 : 1)));
    int64_t off = 0;
    L.codes = off; off = round_up(off + n_out * (k / 2), kAlign);
    L.scales = off; off = round_up(off + L.sf_bytes, kAlign);
    L.words = off; off = round_up(off + 64, kAlign);          // [0] amax bits, [1] s_tW
    L.total = off;
    return L;
}

}  // namespace sq

// C ABI of the SharQ library: argument validation, buffer layout, the device
// status word and the canonical exports. All compute runs in the kernels of
// prep.cu, wquant.cu and gemm.cu.
#include <cuda_runtime.h>
#include <stdlib.h>
#include <string.h>

#include <atomic>
#include <mutex>
#include <vector>

#include "layout.h"
#include "sq_internal.h"

namespace {

__device__ unsigned g_status;  // first timeout site since the last sharq_get_last_error

// Process-wide settings and last-call diagnostics; atomics, so that callers on
// several host threads read and write them without a data race.
std::atomic<uint64_t> g_wait_ns{2000000000ull};
std::atomic<uint32_t> g_last_site{0};
std::atomic<int> g_last_launches{0};

}  // namespace

namespace sq {
// Last-call launch count for entry points outside this file.
void note_launches(int n) { g_last_launches = n; }
}  // namespace sq

namespace {

bool fmt_ok(int fmt) { return fmt == sq::kFmtNV || fmt == sq::kFmtMX; }
bool nm_ok(int n, int m) { return (m == 2 || m == 4 || m == 8 || m == 16) && n >= 1 && n <= m; }
bool k_ok(int64_t k) { return k > 0 && k <= SHARQ_K_MAX && k % SHARQ_K_ALIGN == 0; }
bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

sharq_status make_ctx(void *stream, sq::LaunchCtx &ctx) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return SHARQ_ERR_CUDA;
    static int sms[64] = {0};
    static unsigned *status_ptr[64] = {nullptr};
    static std::mutex mu;  // first calls from several host threads fill the caches once
    std::lock_guard<std::mutex> lock(mu);
    if (dev < 0 || dev >= 64) return SHARQ_ERR_UNSUPPORTED;
    if (!sms[dev] && cudaDeviceGetAttribute(&sms[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return SHARQ_ERR_CUDA;
    if (!status_ptr[dev] && cudaGetSymbolAddress((void **)&status_ptr[dev], g_status) != cudaSuccess)
        return SHARQ_ERR_CUDA;
    ctx.stream = reinterpret_cast<cudaStream_t>(stream);
    ctx.status = status_ptr[dev];
    ctx.wait_ns = g_wait_ns;
    ctx.num_sms = sms[dev];
    ctx.launches = 0;
    return SHARQ_OK;
}

void fill_prep(sharq_prep *P, void *buf, int64_t m_tok, int64_t k, int n, int m, int fmt) {
    sq::PrepLayout L = sq::prep_layout(m_tok, k, n, m, fmt);
    uint8_t *b = static_cast<uint8_t *>(buf);
    memset(P, 0, sizeof(*P));
    P->m_tok = m_tok;
    P->groups = 1;
    P->k = k;
    P->n = n;
    P->m = m;
    P->fmt = fmt;
    P->sf_rows = L.sf_rows;
    P->meta_row_bytes = L.meta_row;
    P->s_codes = b + L.s_codes;
    P->r_codes = b + L.r_codes;
    P->s_scales = b + L.s_scales;
    P->r_scales = b + L.r_scales;
    P->meta = b + L.meta;
    P->scratch = b + L.stats;
    P->tensor_scale = reinterpret_cast<float *>(b + L.words) + 1;
}

void fill_prep_sparse(sharq_prep *P, void *buf, int64_t m_tok, int64_t k, int fmt) {
    sq::PrepLayout L = sq::prep_layout_sparse(m_tok, k, fmt);
    uint8_t *b = static_cast<uint8_t *>(buf);
    memset(P, 0, sizeof(*P));
    P->m_tok = m_tok;
    P->groups = 1;
    P->k = k;
    P->n = 4;
    P->m = 8;
    P->fmt = fmt;
    P->sparse = 1;
    P->sf_rows = L.sf_rows;
    P->meta_row_bytes = L.meta_row;
    P->s_codes = b + L.s_codes;
    P->r_codes = b + L.r_codes;
    P->s_scales = b + L.s_scales;
    P->r_scales = b + L.r_scales;
    P->meta = b + L.meta;
    P->scratch = b + L.stats;
    P->tensor_scale = reinterpret_cast<float *>(b + L.words) + 1;
}

void fill_wq(sharq_wq *W, void *buf, int64_t n_out, int64_t k, int fmt, bool sparse = false) {
    sq::WLayout L = sq::w_layout(n_out, k, fmt, sparse);
    uint8_t *b = static_cast<uint8_t *>(buf);
    memset(W, 0, sizeof(*W));
    W->n_out = n_out;
    W->groups = 1;
    W->k = k;
    W->fmt = fmt;
    W->sparse = sparse ? 1 : 0;
    W->sf_rows = L.sf_rows;
    W->codes = b + L.codes;
    W->scales_backbone = b + L.scales;
    W->scales_residual = b + L.scales;  // same values in the same MMA layout
    W->scratch = b + L.words;
    W->tensor_scale = reinterpret_cast<float *>(b + L.words) + 1;
    W->segments = 1;
    W->seg_end[0] = (int32_t)n_out;
}

// Segments of a weight descriptor: 1..SHARQ_SEGMENTS_MAX, ends increasing,
// multiples of SHARQ_N_ALIGN, the last one n_out.
static bool segments_ok(const sharq_wq *wq) {
    const int s = wq->segments > 1 ? wq->segments : 1;
    if (s > SHARQ_SEGMENTS_MAX) return false;
    if (s == 1) return true;
    int64_t prev = 0;
    for (int g = 0; g < s; ++g) {
        const int64_t e = wq->seg_end[g];
        if (e <= prev || e % SHARQ_N_ALIGN != 0) return false;
        prev = e;
    }
    return prev == wq->n_out && wq->groups <= 1;
}

void unpack_codes(const std::vector<uint8_t> &packed, int64_t count, uint8_t *dst) {
    for (int64_t i = 0; i < count / 2; ++i) {
        dst[2 * i] = packed[i] & 0xF;
        dst[2 * i + 1] = packed[i] >> 4;
    }
}

void unpack_scales(const std::vector<uint8_t> &sf, int64_t rows, int64_t nblk, uint8_t *dst) {
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t j = 0; j < nblk; ++j) dst[r * nblk + j] = sf[sq::sf_offset(r, j, nblk)];
}

// Canonical export of a pair-wise-mode prep: kept positions [m_tok][k/8][4]
// (the two kept pairs' elements, ascending), backbone codes decompressed to
// [m_tok][k] (+0 off the mask), backbone scales [m_tok][k / (2 blk)].
sharq_status export_sparse(const sharq_prep *prep, uint8_t *idx_host, uint8_t *s_codes_host, uint8_t *s_scales_host,
                           uint8_t *r_codes_host, uint8_t *r_scales_host, float *mu_host, float *rstd_host,
                           float *s_t_host) {
    const int64_t m_tok = prep->m_tok, k = prep->k, blk = sq::blk_of(prep->fmt);
    const int64_t nblk_r = k / blk, nblk_s = k / (2 * blk);
    std::vector<uint8_t> buf, meta;
    auto fetch = [&](std::vector<uint8_t> &dst, const void *src, int64_t bytes) -> bool {
        dst.resize((size_t)(bytes > 0 ? bytes : 1));
        return bytes == 0 || cudaMemcpy(dst.data(), src, (size_t)bytes, cudaMemcpyDeviceToHost) == cudaSuccess;
    };
    if ((idx_host || s_codes_host) && !fetch(meta, prep->meta, m_tok * (k / 16))) return SHARQ_ERR_CUDA;
    auto pairs = [&](int64_t r, int64_t g, int &p0, int &p1) {
        const uint32_t f = (meta[(size_t)(r * (k / 16) + g / 2)] >> (4 * (g & 1))) & 0xFu;
        p0 = (int)(f & 3u);
        p1 = (int)(f >> 2);
    };
    if (idx_host)
        for (int64_t r = 0; r < m_tok; ++r)
            for (int64_t g = 0; g < k / 8; ++g) {
                int p0, p1;
                pairs(r, g, p0, p1);
                uint8_t *d = idx_host + (r * (k / 8) + g) * 4;
                d[0] = (uint8_t)(2 * p0), d[1] = (uint8_t)(2 * p0 + 1), d[2] = (uint8_t)(2 * p1), d[3] = (uint8_t)(2 * p1 + 1);
            }
    if (s_codes_host) {
        if (!fetch(buf, prep->s_codes, m_tok * (k / 4))) return SHARQ_ERR_CUDA;
        for (int64_t r = 0; r < m_tok; ++r)
            for (int64_t g = 0; g < k / 8; ++g) {
                int p0, p1;
                pairs(r, g, p0, p1);
                uint8_t *d = s_codes_host + r * k + g * 8;
                memset(d, 0, 8);
                const uint8_t b0 = buf[(size_t)(r * (k / 4) + g * 2)], b1 = buf[(size_t)(r * (k / 4) + g * 2 + 1)];
                d[2 * p0] = b0 & 0xF, d[2 * p0 + 1] = b0 >> 4, d[2 * p1] = b1 & 0xF, d[2 * p1 + 1] = b1 >> 4;
            }
    }
    if (r_codes_host) {
        if (!fetch(buf, prep->r_codes, m_tok * (k / 2))) return SHARQ_ERR_CUDA;
        unpack_codes(buf, m_tok * k, r_codes_host);
    }
    if (s_scales_host) {
        if (!fetch(buf, prep->s_scales, prep->sf_rows * nblk_s)) return SHARQ_ERR_CUDA;
        unpack_scales(buf, m_tok, nblk_s, s_scales_host);
    }
    if (r_scales_host) {
        if (!fetch(buf, prep->r_scales, prep->sf_rows * nblk_r)) return SHARQ_ERR_CUDA;
        unpack_scales(buf, m_tok, nblk_r, r_scales_host);
    }
    if (mu_host || rstd_host) {
        if (!fetch(buf, prep->scratch, m_tok * 8)) return SHARQ_ERR_CUDA;
        const float *st = reinterpret_cast<const float *>(buf.data());
        for (int64_t r = 0; r < m_tok; ++r) {
            if (mu_host) mu_host[r] = st[2 * r];
            if (rstd_host) rstd_host[r] = st[2 * r + 1];
        }
    }
    if (s_t_host && cudaMemcpy(s_t_host, prep->tensor_scale, sizeof(float), cudaMemcpyDeviceToHost) != cudaSuccess)
        return SHARQ_ERR_CUDA;
    return SHARQ_OK;
}

}  // namespace

extern "C" {

const char *sharq_status_string(sharq_status s) {
    switch (s) {
        case SHARQ_OK: return "SHARQ_OK";
        case SHARQ_ERR_INVALID_ARG: return "SHARQ_ERR_INVALID_ARG";
        case SHARQ_ERR_UNSUPPORTED: return "SHARQ_ERR_UNSUPPORTED";
        case SHARQ_ERR_CUDA: return "SHARQ_ERR_CUDA";
        case SHARQ_ERR_TIMEOUT: return "SHARQ_ERR_TIMEOUT";
    }
    return "SHARQ_ERR_UNKNOWN";
}

int sharq_last_launch_count(void) { return g_last_launches; }

uint64_t sharq_set_wait_limit_ns(uint64_t ns) {
    const uint64_t old = g_wait_ns.exchange(ns ? ns : 2000000000ull);
    return old;
}

uint32_t sharq_last_timeout_site(void) { return g_last_site; }

size_t sharq_weight_bytes(int64_t n_out, int64_t k, int fmt) {
    if (n_out < 1 || n_out % SHARQ_N_ALIGN != 0 || n_out > (1ll << 30) || !k_ok(k) || !fmt_ok(fmt)) return 0;
    return (size_t)sq::w_layout(n_out, k, fmt).total;
}

size_t sharq_prep_bytes(int64_t m_tok, int64_t k, int n, int m, int fmt) {
    if (m_tok < 0 || m_tok > (1ll << 30) || !k_ok(k) || !nm_ok(n, m) || !fmt_ok(fmt)) return 0;
    return (size_t)sq::prep_layout(m_tok, k, n, m, fmt).total;
}

sharq_status sharq_quantize_weight(const void *w_dev, int64_t n_out, int64_t k, int fmt, void *wq_dev,
                                   size_t wq_bytes, sharq_wq *wq_out, void *stream) {
    g_last_launches = 0;
    size_t need = sharq_weight_bytes(n_out, k, fmt);
    if (!need || !w_dev || !wq_dev || !wq_out || wq_bytes < need) return SHARQ_ERR_INVALID_ARG;
    if (!aligned(w_dev, 16) || !aligned(wq_dev, sq::kAlign)) return SHARQ_ERR_INVALID_ARG;
    sq::LaunchCtx ctx;
    sharq_status st = make_ctx(stream, ctx);
    if (st != SHARQ_OK) return st;
    fill_wq(wq_out, wq_dev, n_out, k, fmt);
    st = sq::launch_quantize_weight(ctx, *wq_out, w_dev, 1, (int64_t)need);
    g_last_launches = ctx.launches;
    return st;
}

static sharq_status prepare_norm(const void *x_dev, int64_t m_tok, int64_t k, const void *ln_w_dev,
                                 const void *ln_b_dev, float eps, int n, int m, int fmt, void *prep_dev,
                                 size_t prep_bytes, sharq_prep *prep_out, void *stream, int norm) {
    g_last_launches = 0;
    size_t need = sharq_prep_bytes(m_tok, k, n, m, fmt);
    if (!need || !prep_dev || !prep_out || prep_bytes < need) return SHARQ_ERR_INVALID_ARG;
    if (m_tok > 0 && !x_dev) return SHARQ_ERR_INVALID_ARG;
    if (!(eps > 0.0f) || eps != eps || eps > 3.0e38f) return SHARQ_ERR_INVALID_ARG;
    if ((x_dev && !aligned(x_dev, 16)) || !aligned(prep_dev, sq::kAlign) || (ln_w_dev && !aligned(ln_w_dev, 16)) ||
        (ln_b_dev && !aligned(ln_b_dev, 16)))
        return SHARQ_ERR_INVALID_ARG;
    sq::LaunchCtx ctx;
    sharq_status st = make_ctx(stream, ctx);
    if (st != SHARQ_OK) return st;
    fill_prep(prep_out, prep_dev, m_tok, k, n, m, fmt);
    st = sq::launch_prepare(ctx, *prep_out, x_dev, ln_w_dev, ln_b_dev, eps, norm);
    if (st == SHARQ_OK && cudaGetLastError() != cudaSuccess) st = SHARQ_ERR_CUDA;
    g_last_launches = ctx.launches;
    return st;
}

sharq_status sharq_prepare(const void *x_dev, int64_t m_tok, int64_t k, const void *ln_w_dev, const void *ln_b_dev,
                           float eps, int n, int m, int fmt, void *prep_dev, size_t prep_bytes, sharq_prep *prep_out,
                           void *stream) {
    return prepare_norm(x_dev, m_tok, k, ln_w_dev, ln_b_dev, eps, n, m, fmt, prep_dev, prep_bytes, prep_out, stream, 0);
}

sharq_status sharq_prepare_rms(const void *x_dev, int64_t m_tok, int64_t k, const void *w_dev, float eps, int n,
                               int m, int fmt, void *prep_dev, size_t prep_bytes, sharq_prep *prep_out, void *stream) {
    return prepare_norm(x_dev, m_tok, k, w_dev, nullptr, eps, n, m, fmt, prep_dev, prep_bytes, prep_out, stream, 1);
}

sharq_status sharq_prepare_add(const void *h_dev, const void *d_dev, void *x_out_dev, int64_t m_tok, int64_t k,
                               const void *ln_w_dev, const void *ln_b_dev, float eps, int norm, int n, int m, int fmt,
                               void *prep_dev, size_t prep_bytes, sharq_prep *prep_out, void *stream) {
    g_last_launches = 0;
    const size_t need = sharq_prep_bytes(m_tok, k, n, m, fmt);
    if (!need || !prep_dev || !prep_out || prep_bytes < need) return SHARQ_ERR_INVALID_ARG;
    if ((norm != 0 && norm != 1) || (norm == 1 && ln_b_dev)) return SHARQ_ERR_INVALID_ARG;
    if (m_tok > 0 && (!h_dev || !d_dev || !x_out_dev)) return SHARQ_ERR_INVALID_ARG;
    if (!(eps > 0.0f) || eps != eps || eps > 3.0e38f) return SHARQ_ERR_INVALID_ARG;
    if ((h_dev && !aligned(h_dev, 16)) || (d_dev && !aligned(d_dev, 16)) || (x_out_dev && !aligned(x_out_dev, 16)) ||
        !aligned(prep_dev, sq::kAlign) || (ln_w_dev && !aligned(ln_w_dev, 16)) || (ln_b_dev && !aligned(ln_b_dev, 16)))
        return SHARQ_ERR_INVALID_ARG;
    // x_out may be h itself (the residual stream updated in place), but must
    // not overlap d or h partly
    const uintptr_t bytes = (uintptr_t)(m_tok * k * 2);
    auto overlap = [bytes](const void *a, const void *b) {
        const uintptr_t pa = reinterpret_cast<uintptr_t>(a), pb = reinterpret_cast<uintptr_t>(b);
        return pa < pb + bytes && pb < pa + bytes;
    };
    if (m_tok > 0 && (overlap(x_out_dev, d_dev) || (x_out_dev != h_dev && overlap(x_out_dev, h_dev))))
        return SHARQ_ERR_INVALID_ARG;
    sq::LaunchCtx ctx;
    sharq_status st = make_ctx(stream, ctx);
    if (st != SHARQ_OK) return st;
    fill_prep(prep_out, prep_dev, m_tok, k, n, m, fmt);
    st = sq::launch_prepare_add(ctx, *prep_out, h_dev, d_dev, x_out_dev, ln_w_dev, ln_b_dev, eps, norm);
    if (st == SHARQ_OK && cudaGetLastError() != cudaSuccess) st = SHARQ_ERR_CUDA;
    g_last_launches = ctx.launches;
    return st;
}

size_t sharq_prep_bytes_sparse(int64_t m_tok, int64_t k, int fmt) {
    if (m_tok < 0 || m_tok > (1ll << 30) || !k_ok(k) || !fmt_ok(fmt)) return 0;
    return (size_t)sq::prep_layout_sparse(m_tok, k, fmt).total;
}

sharq_status sharq_prepare_sparse(const void *x_dev, int64_t m_tok, int64_t k, const void *ln_w_dev,
                                  const void *ln_b_dev, float eps, int norm, int fmt, void *prep_dev,
                                  size_t prep_bytes, sharq_prep *prep_out, void *stream) {
    g_last_launches = 0;
    const size_t need = sharq_prep_bytes_sparse(m_tok, k, fmt);
    if (!need || !prep_dev || !prep_out || prep_bytes < need) return SHARQ_ERR_INVALID_ARG;
    if ((norm != 0 && norm != 1) || (norm == 1 && ln_b_dev)) return SHARQ_ERR_INVALID_ARG;
    if (m_tok > 0 && !x_dev) return SHARQ_ERR_INVALID_ARG;
    if (!(eps > 0.0f) || eps != eps || eps > 3.0e38f) return SHARQ_ERR_INVALID_ARG;
    if ((x_dev && !aligned(x_dev, 16)) || !aligned(prep_dev, sq::kAlign) || (ln_w_dev && !aligned(ln_w_dev, 16)) ||
        (ln_b_dev && !aligned(ln_b_dev, 16)))
        return SHARQ_ERR_INVALID_ARG;
    sq::LaunchCtx ctx;
    sharq_status st = make_ctx(stream, ctx);
    if (st != SHARQ_OK) return st;
    fill_prep_sparse(prep_out, prep_dev, m_tok, k, fmt);
    st = sq::launch_prepare_sparse(ctx, *prep_out, x_dev, ln_w_dev, ln_b_dev, eps, norm);
    if (st == SHARQ_OK && cudaGetLastError() != cudaSuccess) st = SHARQ_ERR_CUDA;
    g_last_launches = ctx.launches;
    return st;
}

size_t sharq_weight_bytes_sparse(int64_t n_out, int64_t k, int fmt) {
    if (n_out < 1 || n_out % SHARQ_N_ALIGN != 0 || n_out > (1ll << 30) || !k_ok(k) || !fmt_ok(fmt)) return 0;
    return (size_t)sq::w_layout(n_out, k, fmt, true).total;
}

sharq_status sharq_quantize_weight_sparse(const void *w_dev, int64_t n_out, int64_t k, int fmt, void *wq_dev,
                                          size_t wq_bytes, sharq_wq *wq_out, void *stream) {
    g_last_launches = 0;
    const size_t need = sharq_weight_bytes_sparse(n_out, k, fmt);
    if (!need || !w_dev || !wq_dev || !wq_out || wq_bytes < need) return SHARQ_ERR_INVALID_ARG;
    if (!aligned(w_dev, 16) || !aligned(wq_dev, sq::kAlign)) return SHARQ_ERR_INVALID_ARG;
    sq::LaunchCtx ctx;
    sharq_status st = make_ctx(stream, ctx);
    if (st != SHARQ_OK) return st;
    fill_wq(wq_out, wq_dev, n_out, k, fmt, true);
    st = sq::launch_quantize_weight(ctx, *wq_out, w_dev, 1, (int64_t)need);
    g_last_launches = ctx.launches;
    return st;
}

sharq_status sharq_linear(const sharq_prep *prep, const sharq_wq *wq, void *out_dev, void *stream) {
    return sharq_linear_bias(prep, wq, nullptr, out_dev, stream);
}

sharq_status sharq_linear_bias(const sharq_prep *prep, const sharq_wq *wq, const void *bias_dev, void *out_dev,
                               void *stream) {
    g_last_launches = 0;
    if (!prep || !wq) return SHARQ_ERR_INVALID_ARG;
    if (!segments_ok(wq) || (bias_dev && !aligned(bias_dev, 16))) return SHARQ_ERR_INVALID_ARG;
    if (!fmt_ok(prep->fmt) || prep->fmt != wq->fmt || prep->k != wq->k || !k_ok(prep->k)) return SHARQ_ERR_INVALID_ARG;
    // the pair-wise mode's activation and weight go together (the weight's
    // scale blocks are the backbone's)
    if ((prep->sparse != 0) != (wq->sparse != 0)) return SHARQ_ERR_INVALID_ARG;
    if (prep->sparse && (bias_dev || wq->segments > 1 || wq->groups > 1)) return SHARQ_ERR_UNSUPPORTED;
    if (wq->n_out < 1 || wq->n_out % SHARQ_N_ALIGN != 0 || prep->m_tok < 0) return SHARQ_ERR_INVALID_ARG;
    if (wq->groups > 1) return SHARQ_ERR_INVALID_ARG;  // stacked weights: sharq_linear_grouped
    if (prep->sf_rows < prep->m_tok || wq->sf_rows < wq->n_out || wq->sf_rows % sq::kWRowPad != 0 ||
        prep->sf_rows % sq::kActRowPad != 0)
        return SHARQ_ERR_INVALID_ARG;
    if (prep->m_tok == 0) return SHARQ_OK;
    if (!out_dev || !aligned(out_dev, 32) || !prep->s_codes || !prep->r_codes || !wq->codes ||
        wq->scales_backbone != wq->scales_residual)
        return SHARQ_ERR_INVALID_ARG;
    if (prep->m_tok > (1ll << 31) - 256) return SHARQ_ERR_UNSUPPORTED;
    sq::LaunchCtx ctx;
    sharq_status st = make_ctx(stream, ctx);
    if (st != SHARQ_OK) return st;
    st = sq::launch_linear(ctx, *prep, *wq, bias_dev, out_dev);
    g_last_launches = ctx.launches;
    return st;
}

static int64_t fused_rows(const int64_t *seg_rows, int n_segs) {
    if (!seg_rows || n_segs < 1 || n_segs > SHARQ_SEGMENTS_MAX) return -1;
    int64_t total = 0;
    for (int g = 0; g < n_segs; ++g) {
        if (seg_rows[g] < 1 || seg_rows[g] % SHARQ_N_ALIGN != 0 || seg_rows[g] > (1ll << 30)) return -1;
        total += seg_rows[g];
    }
    return total <= (1ll << 30) ? total : -1;
}

size_t sharq_weight_bytes_fused(const int64_t *seg_rows, int n_segs, int64_t k, int fmt) {
    const int64_t total = fused_rows(seg_rows, n_segs);
    return total < 0 ? 0 : sharq_weight_bytes(total, k, fmt);
}

sharq_status sharq_quantize_weight_fused(const void *w_dev, const int64_t *seg_rows, int n_segs, int64_t k, int fmt,
                                         void *wq_dev, size_t wq_bytes, sharq_wq *wq_out, void *stream) {
    g_last_launches = 0;
    const size_t need = sharq_weight_bytes_fused(seg_rows, n_segs, k, fmt);
    if (!need || !w_dev || !wq_dev || !wq_out || wq_bytes < need) return SHARQ_ERR_INVALID_ARG;
    if (!aligned(w_dev, 16) || !aligned(wq_dev, sq::kAlign)) return SHARQ_ERR_INVALID_ARG;
    sq::LaunchCtx ctx;
    sharq_status st = make_ctx(stream, ctx);
    if (st != SHARQ_OK) return st;
    const int64_t total = fused_rows(seg_rows, n_segs);
    fill_wq(wq_out, wq_dev, total, k, fmt);
    wq_out->segments = n_segs;
    int64_t end = 0;
    for (int g = 0; g < n_segs; ++g) {
        end += seg_rows[g];
        wq_out->seg_end[g] = (int32_t)end;
    }
    st = sq::launch_quantize_weight_fused(ctx, *wq_out, w_dev, seg_rows, n_segs);
    g_last_launches = ctx.launches;
    return st;
}

sharq_status sharq_weight_tensor_scales(const sharq_wq *wq, float *s_tw_host, void *stream) {
    if (!wq || !s_tw_host || !wq->tensor_scale || !segments_ok(wq)) return SHARQ_ERR_INVALID_ARG;
    const int segs = wq->segments > 1 ? wq->segments : 1;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return SHARQ_ERR_CUDA;
    if (cudaMemcpy(s_tw_host, wq->tensor_scale, sizeof(float) * (size_t)segs, cudaMemcpyDeviceToHost) != cudaSuccess)
        return SHARQ_ERR_CUDA;
    return SHARQ_OK;
}

size_t sharq_weight_bytes_grouped(int64_t n_groups, int64_t n_out, int64_t k, int fmt) {
    const size_t one = sharq_weight_bytes(n_out, k, fmt);
    if (!one || n_groups < 1 || n_groups > sq::kGroupsMax) return 0;
    return one * (size_t)n_groups;
}

sharq_status sharq_quantize_weight_grouped(const void *w_dev, int64_t n_groups, int64_t n_out, int64_t k, int fmt,
                                           void *wq_dev, size_t wq_bytes, sharq_wq *wq_out, void *stream) {
    g_last_launches = 0;
    const size_t need = sharq_weight_bytes_grouped(n_groups, n_out, k, fmt);
    if (!need || !w_dev || !wq_dev || !wq_out || wq_bytes < need) return SHARQ_ERR_INVALID_ARG;
    if (!aligned(w_dev, 16) || !aligned(wq_dev, sq::kAlign)) return SHARQ_ERR_INVALID_ARG;
    sq::LaunchCtx ctx;
    sharq_status st = make_ctx(stream, ctx);
    if (st != SHARQ_OK) return st;
    fill_wq(wq_out, wq_dev, n_out, k, fmt);
    wq_out->groups = (int32_t)n_groups;
    st = sq::launch_quantize_weight(ctx, *wq_out, w_dev, n_groups, (int64_t)(need / (size_t)n_groups));
    g_last_launches = ctx.launches;
    return st;
}

int64_t sharq_grouped_rows(int64_t rows, int64_t n_groups) {
    if (rows < 0 || rows > (1ll << 30) || n_groups < 1 || n_groups > sq::kGroupsMax) return -1;
    return sq::grouped_rows(rows, n_groups);
}

size_t sharq_gather_bytes(int64_t rows, int64_t n_groups, int64_t k, int n, int m, int fmt) {
    const int64_t cap = sharq_grouped_rows(rows, n_groups);
    return cap < 0 ? 0 : sharq_prep_bytes(cap, k, n, m, fmt);
}

sharq_status sharq_gather_rows(const sharq_prep *src, const int32_t *row_idx_dev, const int32_t *offsets_dev,
                               int64_t n_groups, int64_t rows, void *dst_dev, size_t dst_bytes, sharq_prep *dst_out,
                               void *stream) {
    g_last_launches = 0;
    if (!src || !offsets_dev || !dst_dev || !dst_out) return SHARQ_ERR_INVALID_ARG;
    if (src->sparse) return SHARQ_ERR_UNSUPPORTED;  // grouped launches take the default mode
    if (!fmt_ok(src->fmt) || !nm_ok(src->n, src->m) || !k_ok(src->k) || src->m_tok < 0 || src->m_tok > (1ll << 30))
        return SHARQ_ERR_INVALID_ARG;
    if (src->meta_row_bytes != sq::meta_row_bytes(src->k, src->n, src->m) || src->sf_rows < src->m_tok ||
        src->sf_rows % sq::kActRowPad != 0)
        return SHARQ_ERR_INVALID_ARG;
    if (src->m_tok > 0 && (!src->s_codes || !src->r_codes || !src->s_scales || !src->r_scales || !src->meta ||
                           !src->scratch || !src->tensor_scale))
        return SHARQ_ERR_INVALID_ARG;
    if (!src->tensor_scale) return SHARQ_ERR_INVALID_ARG;
    const size_t need = sharq_gather_bytes(rows, n_groups, src->k, src->n, src->m, src->fmt);
    if (!need || dst_bytes < need || !aligned(dst_dev, sq::kAlign) || !aligned(offsets_dev, 4) ||
        (row_idx_dev && !aligned(row_idx_dev, 4)))
        return SHARQ_ERR_INVALID_ARG;
    if (rows > 0 && !row_idx_dev && rows > src->m_tok) return SHARQ_ERR_INVALID_ARG;
    sq::LaunchCtx ctx;
    sharq_status st = make_ctx(stream, ctx);
    if (st != SHARQ_OK) return st;
    fill_prep(dst_out, dst_dev, sq::grouped_rows(rows, n_groups), src->k, src->n, src->m, src->fmt);
    dst_out->groups = (int32_t)n_groups;
    st = sq::launch_gather(ctx, *src, row_idx_dev, offsets_dev, (int32_t)n_groups, rows, *dst_out);
    g_last_launches = ctx.launches;
    return st;
}

sharq_status sharq_prepare_grouped(const void *x_dev, int64_t rows, int64_t k, const int32_t *offsets_dev,
                                   int64_t n_groups, const void *ln_w_dev, const void *ln_b_dev, float eps, int norm,
                                   int n, int m, int fmt, void *prep_dev, size_t prep_bytes, sharq_prep *prep_out,
                                   void *stream) {
    g_last_launches = 0;
    if (!offsets_dev || !prep_dev || !prep_out || !aligned(offsets_dev, 4) || !aligned(prep_dev, sq::kAlign))
        return SHARQ_ERR_INVALID_ARG;
    if (!fmt_ok(fmt) || !nm_ok(n, m) || !k_ok(k) || rows < 0 || rows > (1ll << 30) || n_groups < 1 ||
        n_groups > sq::kGroupsMax)
        return SHARQ_ERR_INVALID_ARG;
    if ((norm != 0 && norm != 1) || (norm == 1 && ln_b_dev)) return SHARQ_ERR_INVALID_ARG;
    if (!(eps > 0.0f) || eps != eps || eps > 3.0e38f) return SHARQ_ERR_INVALID_ARG;
    if (rows > 0 && (!x_dev || !aligned(x_dev, 16))) return SHARQ_ERR_INVALID_ARG;
    if ((ln_w_dev && !aligned(ln_w_dev, 16)) || (ln_b_dev && !aligned(ln_b_dev, 16))) return SHARQ_ERR_INVALID_ARG;
    const size_t need = sharq_gather_bytes(rows, n_groups, k, n, m, fmt);
    if (!need || prep_bytes < need) return SHARQ_ERR_INVALID_ARG;
    sq::LaunchCtx ctx;
    sharq_status st = make_ctx(stream, ctx);
    if (st != SHARQ_OK) return st;
    fill_prep(prep_out, prep_dev, sq::grouped_rows(rows, n_groups), k, n, m, fmt);
    prep_out->groups = (int32_t)n_groups;
    st = sq::launch_prepare_grouped(ctx, *prep_out, x_dev, rows, offsets_dev, (int32_t)n_groups, ln_w_dev, ln_b_dev,
                                    eps, norm);
    if (st == SHARQ_OK && cudaGetLastError() != cudaSuccess) st = SHARQ_ERR_CUDA;
    g_last_launches = ctx.launches;
    return st;
}

sharq_status sharq_linear_grouped(const sharq_prep *prep, const int32_t *offsets_dev, int64_t n_groups, int64_t rows,
                                  const sharq_wq *wq, void *out_dev, void *stream) {
    g_last_launches = 0;
    if (!prep || !wq || !offsets_dev || !aligned(offsets_dev, 4)) return SHARQ_ERR_INVALID_ARG;
    if (!fmt_ok(prep->fmt) || prep->fmt != wq->fmt || prep->k != wq->k || !k_ok(prep->k)) return SHARQ_ERR_INVALID_ARG;
    if (prep->sparse || wq->sparse) return SHARQ_ERR_UNSUPPORTED;  // grouped launches take the default mode
    if (n_groups < 1 || n_groups > sq::kGroupsMax || prep->groups != n_groups || wq->groups != n_groups ||
        wq->segments > 1)
        return SHARQ_ERR_INVALID_ARG;
    if (wq->n_out < 1 || wq->n_out % SHARQ_N_ALIGN != 0 || rows < 0 || rows > prep->m_tok)
        return SHARQ_ERR_INVALID_ARG;
    if (prep->m_tok % sq::kActRowPad != 0 || prep->sf_rows != prep->m_tok || wq->sf_rows < wq->n_out ||
        wq->sf_rows % sq::kWRowPad != 0)
        return SHARQ_ERR_INVALID_ARG;
    if (!prep->s_codes || !prep->r_codes || !wq->codes || wq->scales_backbone != wq->scales_residual)
        return SHARQ_ERR_INVALID_ARG;
    if (rows > 0 && (!out_dev || !aligned(out_dev, 32))) return SHARQ_ERR_INVALID_ARG;
    if (prep->m_tok > (1ll << 31) - 256) return SHARQ_ERR_UNSUPPORTED;
    sq::LaunchCtx ctx;
    sharq_status st = make_ctx(stream, ctx);
    if (st != SHARQ_OK) return st;
    const int64_t gstride = (int64_t)sharq_weight_bytes(wq->n_out, wq->k, wq->fmt);
    st = sq::launch_linear_grouped(ctx, *prep, *wq, offsets_dev, (int32_t)n_groups, rows, gstride, out_dev);
    g_last_launches = ctx.launches;
    return st;
}

sharq_status sharq_prep_export(const sharq_prep *prep, uint8_t *idx_host, uint8_t *s_codes_host,
                               uint8_t *s_scales_host, uint8_t *r_codes_host, uint8_t *r_scales_host,
                               float *mu_host, float *rstd_host, float *s_t_host, void *stream) {
    if (!prep || !fmt_ok(prep->fmt) || !nm_ok(prep->n, prep->m) || prep->m_tok < 0) return SHARQ_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return SHARQ_ERR_CUDA;
    if (prep->sparse)
        return export_sparse(prep, idx_host, s_codes_host, s_scales_host, r_codes_host, r_scales_host, mu_host,
                             rstd_host, s_t_host);
    const int64_t m_tok = prep->m_tok, k = prep->k, nblk = k / sq::blk_of(prep->fmt);
    const int64_t codes = m_tok * (k / 2), sf = prep->sf_rows * nblk;
    std::vector<uint8_t> buf;
    auto fetch = [&](const void *src, int64_t bytes) -> bool {
        buf.resize((size_t)(bytes > 0 ? bytes : 1));
        return bytes == 0 || cudaMemcpy(buf.data(), src, (size_t)bytes, cudaMemcpyDeviceToHost) == cudaSuccess;
    };
    if (s_codes_host) {
        if (!fetch(prep->s_codes, codes)) return SHARQ_ERR_CUDA;
        unpack_codes(buf, m_tok * k, s_codes_host);
    }
    if (r_codes_host) {
        if (!fetch(prep->r_codes, codes)) return SHARQ_ERR_CUDA;
        unpack_codes(buf, m_tok * k, r_codes_host);
    }
    if (s_scales_host) {
        if (!fetch(prep->s_scales, sf)) return SHARQ_ERR_CUDA;
        unpack_scales(buf, m_tok, nblk, s_scales_host);
    }
    if (r_scales_host) {
        if (!fetch(prep->r_scales, sf)) return SHARQ_ERR_CUDA;
        unpack_scales(buf, m_tok, nblk, r_scales_host);
    }
    if (idx_host) {
        if (!fetch(prep->meta, m_tok * prep->meta_row_bytes)) return SHARQ_ERR_CUDA;
        const int ib = sq::idx_bits(prep->m), n = prep->n, groups = (int)(k / prep->m);
        for (int64_t r = 0; r < m_tok; ++r) {
            const uint8_t *row = buf.data() + r * prep->meta_row_bytes;
            for (int64_t f = 0; f < (int64_t)groups * n; ++f) {
                uint32_t v = 0;
                for (int b = 0; b < ib; ++b) {
                    int64_t bit = f * ib + b;
                    v |= (uint32_t)((row[bit >> 3] >> (bit & 7)) & 1u) << b;
                }
                idx_host[r * groups * n + f] = (uint8_t)v;
            }
        }
    }
    if (mu_host || rstd_host) {
        if (!fetch(prep->scratch, m_tok * 8)) return SHARQ_ERR_CUDA;
        const float *st = reinterpret_cast<const float *>(buf.data());
        for (int64_t r = 0; r < m_tok; ++r) {
            if (mu_host) mu_host[r] = st[2 * r];
            if (rstd_host) rstd_host[r] = st[2 * r + 1];
        }
    }
    if (s_t_host && cudaMemcpy(s_t_host, prep->tensor_scale, sizeof(float), cudaMemcpyDeviceToHost) != cudaSuccess)
        return SHARQ_ERR_CUDA;
    return SHARQ_OK;
}

sharq_status sharq_weight_export(const sharq_wq *wq, uint8_t *codes_host, uint8_t *scales_host,
                                 uint8_t *scales_residual_host, float *s_tw_host, void *stream) {
    if (!wq || !fmt_ok(wq->fmt)) return SHARQ_ERR_INVALID_ARG;
    if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return SHARQ_ERR_CUDA;
    // the pair-wise mode's weight: one scale per 2 blk values in the
    // backbone view; the residual view repeats each of them
    const int64_t nblk = wq->k / (sq::blk_of(wq->fmt) * (wq->sparse ? 2 : 1));
    std::vector<uint8_t> buf;
    if (codes_host) {
        buf.resize((size_t)(wq->n_out * (wq->k / 2)));
        if (cudaMemcpy(buf.data(), wq->codes, buf.size(), cudaMemcpyDeviceToHost) != cudaSuccess) return SHARQ_ERR_CUDA;
        unpack_codes(buf, wq->n_out * wq->k, codes_host);
    }
    const void *views[2] = {wq->scales_backbone, wq->scales_residual};
    uint8_t *dsts[2] = {scales_host, scales_residual_host};
    for (int v = 0; v < 2; ++v) {
        if (!dsts[v]) continue;
        buf.resize((size_t)(wq->sf_rows * nblk));
        if (cudaMemcpy(buf.data(), views[v], buf.size(), cudaMemcpyDeviceToHost) != cudaSuccess) return SHARQ_ERR_CUDA;
        if (wq->sparse && v == 1) {  // [n_out][k / blk]: every scale twice
            std::vector<uint8_t> once((size_t)(wq->n_out * nblk));
            unpack_scales(buf, wq->n_out, nblk, once.data());
            for (int64_t r = 0; r < wq->n_out; ++r)
                for (int64_t j = 0; j < 2 * nblk; ++j) dsts[v][r * 2 * nblk + j] = once[(size_t)(r * nblk + j / 2)];
        } else {
            unpack_scales(buf, wq->n_out, nblk, dsts[v]);
        }
    }
    if (s_tw_host && cudaMemcpy(s_tw_host, wq->tensor_scale, sizeof(float), cudaMemcpyDeviceToHost) != cudaSuccess)
        return SHARQ_ERR_CUDA;
    return SHARQ_OK;
}

sharq_status sharq_selftest_wait(uint64_t limit_ns, void *stream) {
    g_last_launches = 0;
    if (limit_ns == 0 || limit_ns > 10000000000ull) return SHARQ_ERR_INVALID_ARG;
    sq::LaunchCtx ctx;
    sharq_status st = make_ctx(stream, ctx);
    if (st != SHARQ_OK) return st;
    st = sq::launch_wait_probe(ctx, limit_ns);
    g_last_launches = ctx.launches;
    return st;
}

sharq_status sharq_selftest_division(uint64_t count, uint64_t seed, uint64_t *mismatches_host, float *examples_host,
                                     void *stream) {
    g_last_launches = 0;
    if (!mismatches_host || count == 0) return SHARQ_ERR_INVALID_ARG;
    sq::LaunchCtx ctx;
    sharq_status st = make_ctx(stream, ctx);
    if (st != SHARQ_OK) return st;
    st = sq::launch_div_check(ctx, count, seed, mismatches_host, examples_host);
    g_last_launches = ctx.launches;
    return st;
}

sharq_status sharq_get_last_error(void *stream) {
    if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return SHARQ_ERR_CUDA;
    if (cudaGetLastError() != cudaSuccess) return SHARQ_ERR_CUDA;
    unsigned v = 0;
    if (cudaMemcpyFromSymbol(&v, g_status, sizeof(v)) != cudaSuccess) return SHARQ_ERR_CUDA;
    if (v != 0) {
        g_last_site = v;
        unsigned zero = 0;
        if (cudaMemcpyToSymbol(g_status, &zero, sizeof(zero)) != cudaSuccess) return SHARQ_ERR_CUDA;
        return (v & 0xF00u) == 0x200u ? SHARQ_ERR_INVALID_ARG : SHARQ_ERR_TIMEOUT;
    }
    return SHARQ_OK;
}

}  // extern "C"

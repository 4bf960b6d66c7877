// Fused preparation operator of SharQ on sm_100a.
//
// "SharQ: Bridging Activation Sparsity and FP4 Quantization for LLM
// Inference", Abstract: a fused preparation kernel absorbs mask generation,
// residual construction and layer normalization into one operator; the
// residual is defined relative to the quantized sparse backbone.
//
// Two passes over the activations, because the NVFP4 tensor scale depends on
// amax(X_ln) over the whole tensor:
//   1. ln_stats_kernel (one CTA per row): exact LayerNorm statistics from
//      integer sums, then amax|X_ln| of the row (row cached in shared memory),
//      folded into one global word by an atomic max.
//   2. prep_encode_kernel (one thread per 32-element chunk): LayerNorm apply,
//      top-n-of-m selection, Q(S), R = X_ln - deq(Q(S)), Q(R), and packed
//      code / scale / metadata stores. The second read of x mostly hits L2.
#include <cuda_fp16.h>

#include "sharq_dev.cuh"
#include "sq_internal.h"

namespace sq {

constexpr int kStatsThreads = 256;
constexpr int kEncodeThreads = 256;

// ---------------------------------------------------------------------------
// Exact statistics. With a = x * 2^24 (an integer, |a| < 2^40), split
// |a| = hi * 2^20 + lo (hi, lo < 2^20). Then
//   S1 = sum(+-a),   S2 = sum a^2 = 2^40 sum hi^2 + 2^21 sum hi*lo + sum lo^2,
// where every partial sum fits a 64-bit integer for k <= 2^16.
struct ExactSums {
    int64_t s1;
    uint64_t hh, hl, ll;
};

__device__ __forceinline__ void accum_half(uint32_t h, ExactSums &e) {
    float t = __fmul_rn(fabsf(h2f((uint16_t)h)), 16.0f);                        // |x| * 2^4, exact
    float hf = floorf(t);
    uint32_t hi = (uint32_t)hf;                                                // < 2^20
    uint32_t lo = (uint32_t)__fmul_rn(__fsub_rn(t, hf), 1048576.0f);           // < 2^20, exact
    int64_t a = (int64_t)(((uint64_t)hi << 20) | lo);
    e.s1 += (h & 0x8000u) ? -a : a;
    e.hh += (uint64_t)hi * hi;
    e.hl += (uint64_t)hi * lo;
    e.ll += (uint64_t)lo * lo;
}

__device__ __forceinline__ void accum_word(uint32_t w, ExactSums &e) {
    accum_half(w & 0xFFFFu, e);
    accum_half(w >> 16, e);
}

// Round-to-nearest-even binary64 value of a non-negative 128-bit integer.
__device__ double u128_to_f64(unsigned __int128 v) {
    uint64_t hi = (uint64_t)(v >> 64), lo = (uint64_t)v;
    if (hi == 0 && lo < (1ull << 53)) return __ull2double_rn(lo);
    int top = hi ? 127 - __clzll((long long)hi) : 63 - __clzll((long long)lo);
    int drop = top - 52;
    unsigned __int128 q = v >> drop;
    unsigned __int128 rem = v - (q << drop);
    unsigned __int128 half = (unsigned __int128)1 << (drop - 1);
    if (rem > half || (rem == half && (q & 1))) q += 1;
    double scale = __longlong_as_double((long long)(1023 + drop) << 52);  // 2^drop, exact
    return __dmul_rn(__ull2double_rn((uint64_t)q), scale);
}

__global__ void __launch_bounds__(kStatsThreads)
ln_stats_kernel(const uint16_t *__restrict__ x, const uint16_t *__restrict__ gamma,
                const uint16_t *__restrict__ beta, float eps, int64_t k, float2 *__restrict__ stats,
                unsigned *__restrict__ amax_word) {
    extern __shared__ uint4 row_cache[];  // k / 8 vectors of 8 halves
    __shared__ int64_t red_s1[kStatsThreads / 32];
    __shared__ uint64_t red_hh[kStatsThreads / 32], red_hl[kStatsThreads / 32], red_ll[kStatsThreads / 32];
    __shared__ float red_max[kStatsThreads / 32];
    __shared__ float2 row_stat;

    const int64_t row = blockIdx.x;
    const int nvec = (int)(k / 8);
    const uint4 *xr = reinterpret_cast<const uint4 *>(x + row * k);
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

    ExactSums e = {0, 0, 0, 0};
    for (int c = threadIdx.x; c < nvec; c += kStatsThreads) {
        uint4 v = xr[c];  // default caching: the encode pass re-reads x from L2
        row_cache[c] = v;
        accum_word(v.x, e);
        accum_word(v.y, e);
        accum_word(v.z, e);
        accum_word(v.w, e);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        e.s1 += __shfl_xor_sync(0xFFFFFFFFu, e.s1, o);
        e.hh += __shfl_xor_sync(0xFFFFFFFFu, e.hh, o);
        e.hl += __shfl_xor_sync(0xFFFFFFFFu, e.hl, o);
        e.ll += __shfl_xor_sync(0xFFFFFFFFu, e.ll, o);
    }
    if (lane == 0) {
        red_s1[warp] = e.s1;
        red_hh[warp] = e.hh;
        red_hl[warp] = e.hl;
        red_ll[warp] = e.ll;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int64_t s1 = 0;
        uint64_t hh = 0, hl = 0, ll = 0;
        for (int w = 0; w < kStatsThreads / 32; ++w) {
            s1 += red_s1[w];
            hh += red_hh[w];
            hl += red_hl[w];
            ll += red_ll[w];
        }
        unsigned __int128 s2 = ((unsigned __int128)hh << 40) + ((unsigned __int128)hl << 21) + ll;
        __int128 d = (__int128)k * (__int128)s2 - (__int128)s1 * (__int128)s1;
        double kd = (double)k;
        double mean64 = __ddiv_rn(__ll2double_rn(s1), __dmul_rn(kd, 16777216.0));
        double var64 = __ddiv_rn(u128_to_f64((unsigned __int128)d), __dmul_rn(__dmul_rn(kd, kd), 281474976710656.0));
        float mu = __double2float_rn(mean64);
        float rstd = __double2float_rn(__ddiv_rn(1.0, __dsqrt_rn(__dadd_rn(var64, (double)eps))));
        row_stat = make_float2(mu, rstd);
        stats[row] = row_stat;
    }
    __syncthreads();
    const float mu = row_stat.x, rstd = row_stat.y;
    const bool has_g = gamma != nullptr, has_b = beta != nullptr;
    float amax = 0.0f;
    for (int c = threadIdx.x; c < nvec; c += kStatsThreads) {
        uint4 v = row_cache[c];
        uint4 g = has_g ? __ldg(reinterpret_cast<const uint4 *>(gamma) + c) : make_uint4(0, 0, 0, 0);
        uint4 b = has_b ? __ldg(reinterpret_cast<const uint4 *>(beta) + c) : make_uint4(0, 0, 0, 0);
        const uint32_t xv[4] = {v.x, v.y, v.z, v.w}, gv[4] = {g.x, g.y, g.z, g.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                float xl = ln_apply(h2f((uint16_t)(xv[q] >> (16 * h))), mu, rstd, has_g,
                                    h2f((uint16_t)(gv[q] >> (16 * h))), has_b, h2f((uint16_t)(bv[q] >> (16 * h))));
                amax = fmaxf(amax, fabsf(xl));
            }
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
    if (lane == 0) red_max[warp] = amax;
    __syncthreads();
    if (threadIdx.x == 0) {
        float a = 0.0f;
        for (int w = 0; w < kStatsThreads / 32; ++w) a = fmaxf(a, red_max[w]);
        atomicMax(amax_word, __float_as_uint(a));  // non-negative floats order like their bits
    }
}

// ---------------------------------------------------------------------------
// Encode pass.

// Store `nbytes` (<= 16) little-endian bytes of (hi:lo) at p, using the widest
// aligned stores the address allows.
__device__ __forceinline__ void store_bits(uint8_t *p, uint64_t lo, uint64_t hi, int nbytes) {
    int i = 0;
    while (i < nbytes) {
        uint64_t w = i < 8 ? (lo >> (8 * i)) | (i ? (hi << (64 - 8 * i)) : 0) : hi >> (8 * (i - 8));
        uintptr_t a = reinterpret_cast<uintptr_t>(p + i);
        if (nbytes - i >= 4 && (a & 3) == 0) {
            *reinterpret_cast<uint32_t *>(p + i) = (uint32_t)w;
            i += 4;
        } else if (nbytes - i >= 2 && (a & 1) == 0) {
            *reinterpret_cast<uint16_t *>(p + i) = (uint16_t)w;
            i += 2;
        } else {
            p[i] = (uint8_t)w;
            i += 1;
        }
    }
}

// Append a `bits`-wide field at bit position pos of a 128-bit stream.
__device__ __forceinline__ void put_bits(uint64_t &lo, uint64_t &hi, uint32_t val, int bits, int pos) {
    if (pos < 64) {
        lo |= (uint64_t)val << pos;
        if (pos + bits > 64) hi |= (uint64_t)val >> (64 - pos);
    } else {
        hi |= (uint64_t)val << (pos - 64);
    }
}

template <int FMT, int M>
__global__ void __launch_bounds__(kEncodeThreads)
prep_encode_kernel(const uint16_t *__restrict__ x, const uint16_t *__restrict__ gamma,
                   const uint16_t *__restrict__ beta, const float2 *__restrict__ stats,
                   const unsigned *__restrict__ amax_word, float *__restrict__ s_t_out, int64_t m_tok,
                   int64_t sf_rows, int64_t k, int n, uint8_t *__restrict__ s_codes, uint8_t *__restrict__ r_codes,
                   uint8_t *__restrict__ s_sf, uint8_t *__restrict__ r_sf, uint8_t *__restrict__ meta,
                   int64_t meta_row) {
    constexpr int BLK = FMT == kFmtNV ? 16 : 32;
    constexpr int NB = 32 / BLK;  // blocks per chunk
    constexpr int IB = M <= 2 ? 1 : M <= 4 ? 2 : M <= 8 ? 3 : 4;

    const float amax = __uint_as_float(*amax_word);
    const float s_t = (FMT == kFmtNV && amax != 0.0f) ? __fdiv_rn(amax, 2688.0f) : 1.0f;
    const float c6 = __fmul_rn(6.0f, s_t);
    if (blockIdx.x == 0 && threadIdx.x == 0) *s_t_out = s_t;

    const int64_t cpr = k / 32;
    const int64_t nblk = k / BLK;
    const int B = (32 / M) * n * IB;  // metadata bits per chunk
    const int64_t total = sf_rows * cpr;
    const int64_t stride = (int64_t)gridDim.x * kEncodeThreads;
    const bool has_g = gamma != nullptr, has_b = beta != nullptr;

    for (int64_t base = (int64_t)blockIdx.x * kEncodeThreads; base < total; base += stride) {
        const int64_t t = base + threadIdx.x;
        const bool active = t < total;
        const int64_t row = active ? t / cpr : 0;
        const int64_t c = active ? t - row * cpr : 0;
        const bool real = active && row < m_tok;
        uint64_t mlo = 0, mhi = 0;

        if (active && !real) {  // scale-layout padding rows: zero scales
            if (FMT == kFmtNV) {
                *reinterpret_cast<uint16_t *>(s_sf + sf_offset(row, 2 * c, nblk)) = 0;
                *reinterpret_cast<uint16_t *>(r_sf + sf_offset(row, 2 * c, nblk)) = 0;
            } else {
                s_sf[sf_offset(row, c, nblk)] = 0;
                r_sf[sf_offset(row, c, nblk)] = 0;
            }
        }
        if (real) {
            const uint4 *xp = reinterpret_cast<const uint4 *>(x + row * k + c * 32);
            const float2 st = stats[row];
            float v[32];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                uint4 xv = __ldcs(xp + q);
                uint4 gv = has_g ? __ldg(reinterpret_cast<const uint4 *>(gamma + c * 32) + q) : make_uint4(0, 0, 0, 0);
                uint4 bv = has_b ? __ldg(reinterpret_cast<const uint4 *>(beta + c * 32) + q) : make_uint4(0, 0, 0, 0);
                const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
                const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w};
                const uint32_t bw[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int wsel = i / 2, sh = 16 * (i % 2);
                    v[8 * q + i] = ln_apply(h2f((uint16_t)(xw[wsel] >> sh)), st.x, st.y, has_g,
                                            h2f((uint16_t)(gw[wsel] >> sh)), has_b, h2f((uint16_t)(bw[wsel] >> sh)));
                }
            }

            // Top-n of every group of M by magnitude; equal magnitudes go to
            // the lower index. rank_i = #{j < i: |v_j| >= |v_i|} + #{j > i: |v_j| > |v_i|}.
            uint32_t keep = 0;
#pragma unroll
            for (int g = 0; g < 32 / M; ++g) {
                uint32_t a[M];
                int rank[M];
#pragma unroll
                for (int i = 0; i < M; ++i) {
                    a[i] = __float_as_uint(v[g * M + i]) & 0x7FFFFFFFu;
                    rank[i] = 0;
                }
#pragma unroll
                for (int i = 0; i < M; ++i)
#pragma unroll
                    for (int j = i + 1; j < M; ++j) {
                        if (a[i] >= a[j]) ++rank[j];
                        else ++rank[i];
                    }
#pragma unroll
                for (int i = 0; i < M; ++i)
                    if (rank[i] < n) keep |= 1u << (g * M + i);
            }
            // Metadata: kept positions of every group, ascending, IB bits each.
            int pos = 0;
#pragma unroll
            for (int g = 0; g < 32 / M; ++g)
#pragma unroll
                for (int i = 0; i < M; ++i)
                    if ((keep >> (g * M + i)) & 1u) {
                        put_bits(mlo, mhi, (uint32_t)i, IB, pos);
                        pos += IB;
                    }

            // Backbone S = X_ln on the mask: block scales, codes, residual.
            float rr[32];
            uint32_t spk[4] = {0, 0, 0, 0}, rpk[4] = {0, 0, 0, 0};
            uint32_t s_sc[NB], r_sc[NB];
#pragma unroll
            for (int bk = 0; bk < NB; ++bk) {
                float a = 0.0f;
#pragma unroll
                for (int i = bk * BLK; i < (bk + 1) * BLK; ++i)
                    if ((keep >> i) & 1u) a = fmaxf(a, fabsf(v[i]));
                uint32_t code;
                const float d = block_step<FMT>(a, s_t, c6, code);
                s_sc[bk] = code;
#pragma unroll
                for (int i = bk * BLK; i < (bk + 1) * BLK; i += 2) {
                    const bool k0 = (keep >> i) & 1u, k1 = (keep >> (i + 1)) & 1u;
                    uint32_t byte = 0;
                    if (d != 0.0f) {
                        const float q0 = k0 ? __fdiv_rn(v[i], d) : 0.0f;
                        const float q1 = k1 ? __fdiv_rn(v[i + 1], d) : 0.0f;
                        byte = e2m1x2(q0, q1);
                    }
                    const float2 cv = e2m1x2_value(byte);
                    rr[i] = k0 ? __fsub_rn(v[i], __fmul_rn(cv.x, d)) : v[i];
                    rr[i + 1] = k1 ? __fsub_rn(v[i + 1], __fmul_rn(cv.y, d)) : v[i + 1];
                    spk[i / 8] |= byte << (4 * (i % 8));
                }
            }
            // Residual R: dense block quantization with the same tensor scale.
#pragma unroll
            for (int bk = 0; bk < NB; ++bk) {
                float a = 0.0f;
#pragma unroll
                for (int i = bk * BLK; i < (bk + 1) * BLK; ++i) a = fmaxf(a, fabsf(rr[i]));
                uint32_t code;
                const float d = block_step<FMT>(a, s_t, c6, code);
                r_sc[bk] = code;
                if (d != 0.0f) {
#pragma unroll
                    for (int i = bk * BLK; i < (bk + 1) * BLK; i += 2) {
                        const uint32_t byte = e2m1x2(__fdiv_rn(rr[i], d), __fdiv_rn(rr[i + 1], d));
                        rpk[i / 8] |= byte << (4 * (i % 8));
                    }
                }
            }
            *reinterpret_cast<uint4 *>(s_codes + row * (k / 2) + c * 16) = make_uint4(spk[0], spk[1], spk[2], spk[3]);
            *reinterpret_cast<uint4 *>(r_codes + row * (k / 2) + c * 16) = make_uint4(rpk[0], rpk[1], rpk[2], rpk[3]);
            if (FMT == kFmtNV) {
                *reinterpret_cast<uint16_t *>(s_sf + sf_offset(row, 2 * c, nblk)) = (uint16_t)(s_sc[0] | (s_sc[NB - 1] << 8));
                *reinterpret_cast<uint16_t *>(r_sf + sf_offset(row, 2 * c, nblk)) = (uint16_t)(r_sc[0] | (r_sc[NB - 1] << 8));
            } else {
                s_sf[sf_offset(row, c, nblk)] = (uint8_t)s_sc[0];
                r_sf[sf_offset(row, c, nblk)] = (uint8_t)r_sc[0];
            }
        }

        // Metadata store. B bits per chunk; when B is not a whole number of
        // bytes (m = 8 with odd n: B = 4 mod 8) the chunk pair (2i, 2i+1),
        // which sits in lanes (2i, 2i+1), shares one byte: the even lane
        // writes it with the odd lane's first nibble.
        if ((B & 7) == 0) {
            if (real) store_bits(meta + row * meta_row + c * (B / 8), mlo, mhi, B / 8);
        } else {
            const uint32_t first_nib = (uint32_t)(mlo & 0xF);
            const uint32_t partner = __shfl_down_sync(0xFFFFFFFFu, first_nib, 1);
            if (real) {
                const int full = B / 8;  // whole bytes before the shared nibble
                if ((c & 1) == 0) {
                    uint8_t *p = meta + row * meta_row + (c / 2) * (2 * B / 8);
                    store_bits(p, mlo, mhi, full);
                    const uint64_t last = full < 8 ? (mlo >> (8 * full)) | (full ? (mhi << (64 - 8 * full)) : 0)
                                                   : mhi >> (8 * (full - 8));
                    p[full] = (uint8_t)((last & 0xF) | (partner << 4));
                } else {
                    uint8_t *p = meta + row * meta_row + (c / 2) * (2 * B / 8) + full + 1;
                    const uint64_t lo4 = (mlo >> 4) | (mhi << 60), hi4 = mhi >> 4;
                    store_bits(p, lo4, hi4, (B - 4) / 8);
                }
            }
        }
    }
}

template <int FMT>
static void *encode_fn(int m) {
    switch (m) {
        case 2: return (void *)prep_encode_kernel<FMT, 2>;
        case 4: return (void *)prep_encode_kernel<FMT, 4>;
        case 8: return (void *)prep_encode_kernel<FMT, 8>;
        default: return (void *)prep_encode_kernel<FMT, 16>;
    }
}

sharq_status launch_prepare(LaunchCtx &ctx, const sharq_prep &P, const void *x, const void *gamma, const void *beta,
                            float eps) {
    static bool attr_done[64] = {false};
    int dev = 0;
    SQ_CUDA_TRY(cudaGetDevice(&dev));
    if (dev < 0 || dev >= 64) return SHARQ_ERR_UNSUPPORTED;
    if (!attr_done[dev]) {
        SQ_CUDA_TRY(cudaFuncSetAttribute(ln_stats_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)(2 * SHARQ_K_MAX)));
        attr_done[dev] = true;
    }
    unsigned *words = reinterpret_cast<unsigned *>(P.tensor_scale) - 1;  // [0] amax bits, [1] s_t
    SQ_CUDA_TRY(cudaMemsetAsync(words, 0, sizeof(unsigned), ctx.stream));
    float2 *stats = reinterpret_cast<float2 *>(P.scratch);
    if (P.m_tok > 0) {
        ln_stats_kernel<<<(unsigned)P.m_tok, kStatsThreads, (size_t)(2 * P.k), ctx.stream>>>(
            (const uint16_t *)x, (const uint16_t *)gamma, (const uint16_t *)beta, eps, P.k, stats, words);
        ctx.launches++;
    }
    const int64_t total = P.sf_rows * (P.k / 32);
    int64_t blocks = (total + kEncodeThreads - 1) / kEncodeThreads;
    const int64_t cap = (int64_t)ctx.num_sms * 8;
    if (blocks > cap) blocks = cap;
    void *fn = P.fmt == kFmtNV ? encode_fn<kFmtNV>(P.m) : encode_fn<kFmtMX>(P.m);
    const uint16_t *xx = (const uint16_t *)x, *gg = (const uint16_t *)gamma, *bb = (const uint16_t *)beta;
    const float2 *cst = stats;
    const unsigned *aw = words;
    float *st = P.tensor_scale;
    int64_t m_tok = P.m_tok, sf_rows = P.sf_rows, k = P.k, meta_row = P.meta_row_bytes;
    int n = P.n;
    uint8_t *sc = (uint8_t *)P.s_codes, *rc = (uint8_t *)P.r_codes, *ss = (uint8_t *)P.s_scales,
            *rs = (uint8_t *)P.r_scales, *mt = (uint8_t *)P.meta;
    void *args[] = {&xx, &gg, &bb, &cst, &aw, &st, &m_tok, &sf_rows, &k, &n, &sc, &rc, &ss, &rs, &mt, &meta_row};
    SQ_CUDA_TRY(cudaLaunchKernel(fn, dim3((unsigned)blocks), dim3(kEncodeThreads), args, 0, ctx.stream));
    ctx.launches++;
    return SHARQ_OK;
}

}  // namespace sq

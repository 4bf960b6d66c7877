// Fused preparation operator of SharQ on sm_100a.
//
// "SharQ: Bridging Activation Sparsity and FP4 Quantization for LLM
// Inference", Abstract: one fused operator does the LayerNorm, builds the
// mask and forms the residual, which is taken from the quantized backbone
// (not from the unquantized sparse values).
//
// Two passes over the activations, because the NVFP4 tensor scale depends on
// amax(X_ln) over the whole tensor:
//   1. ln_stats_kernel (one CTA per row; ln_stats_warp_kernel, one warp per
//      row, for short rows or many rows): exact LayerNorm statistics from
//      integer sums and the row's amax|X_ln|, folded into one global word by
//      an atomic max. Without gamma/beta, X_ln is a non-decreasing function of
//      x within a row, so amax|X_ln| comes from the row's min and max of x;
//      with gamma/beta the row is kept in shared memory and swept again.
//   2. prep_encode_kernel (one thread per 16 consecutive elements; an MXFP4
//      block of 32 spans a lane pair): LayerNorm apply, top-n-of-m selection,
//      Q(S), R = X_ln - deq(Q(S)), Q(R), and packed code / scale / metadata
//      stores. The second read of x hits L2 when x fits in it (126 MB).
#include <cuda_fp16.h>

#include <string.h>

#include <mutex>

#include "sharq_dev.cuh"
#include "sq_internal.h"

namespace sq {

// Resident encode CTAs per SM the register allocation must allow. Measured
// on B200 (K = 14336 / 3584 / 4096 preparations): 2 (80 registers) 202.8 /
// 36.9 / 69.6 us, 3 (71) 204.8 / 38.8 / 69.7, 4 (64, a few bytes spilled)
// 204.9 / 38.9 / 69.6: the encode is issue-bound, not short of warps.
#ifndef SQ_ENCODE_MIN_CTAS
#define SQ_ENCODE_MIN_CTAS 2
#endif
constexpr int kStatsThreads = 256;
constexpr int kEncodeThreads = 256;
constexpr int kUnit = 16;  // elements per encode thread

// ---------------------------------------------------------------------------
// Exact statistics. With a = x * 2^24 (an integer, |a| < 2^40), write
// x = hi * 2^-4 + lo * 2^-24 with hi = floor(x * 2^4) (|hi| <= 1048064,
// signed) and 0 <= lo < 2^20, so that a = hi * 2^20 + lo and
//   S1 = 2^20 sum hi + sum lo,
//   S2 = 2^40 sum hi^2 + 2^21 sum hi*lo + sum lo^2.
// hi and lo come out of the binary32 pipeline exactly: x + 1.5*2^19 rounded
// toward -inf lies in [2^19, 2^20), where the spacing of binary32 is 2^-4,
// so it is 1.5*2^19 + hi * 2^-4 and its bit pattern exceeds that of 1.5*2^19
// by hi; (x - hi * 2^-4) * 2^24 + 2^23 holds lo in its low mantissa bits
// (every step is exact).
struct ExactSums {
    int64_t hi, lo;  // sum hi, sum lo
    int64_t hh, hl;  // sum hi^2, sum hi*lo
    uint64_t ll;     // sum lo^2
};

// One lane's sums: hi and lo in 32 bits, the three products in binary64.
// A lane adds at most SHARQ_K_MAX / 32 values (one warp per row is the
// narrowest split of a row): 2048 * 1048064 < 2^31 and 2048 * (2^20 - 1) <
// 2^31; every product is an integer below 2^40, so each binary64 FMA adds
// an exact product to an integer sum below 2048 * 2^40 = 2^51 < 2^53 and
// rounds nothing. (On B200 the products on the FP64 pipe cost less than the
// 64-bit integer multiplies on the FMA pipe, which saturated it.)
struct LaneSums {
    int32_t hi, lo;
    double hh, hl, ll;
};
static_assert((int64_t)SHARQ_K_MAX / 32 * 1048064 < (1ll << 31), "lane sums of hi fit in 32 bits");
static_assert((int64_t)SHARQ_K_MAX / 32 * ((1 << 20) - 1) < (1ll << 31), "lane sums of lo fit in 32 bits");
static_assert((double)(SHARQ_K_MAX / 32) * 1099511627776.0 < 9007199254740992.0, "lane product sums exact in binary64");

__device__ __forceinline__ ExactSums widen(const LaneSums &l) {
    return ExactSums{l.hi, l.lo, __double2ll_rn(l.hh), __double2ll_rn(l.hl), (uint64_t)__double2ll_rn(l.ll)};
}

// Integer h (|h| < 2^31) as a binary64, exactly: the bit pattern of
// 1.5 * 2^52 plus h (sign-extended) is the value 1.5 * 2^52 + h.
__device__ __forceinline__ double i32_to_f64_exact(int32_t h) {
    return __dsub_rn(__hiloint2double(0x43380000 + (h >> 31), h), 6755399441055744.0);
}

__device__ __forceinline__ void accum_pair(uint32_t w, LaneSums &e) {
    const uint64_t f = h2_to_f2(w);                                    // x, exact
    const uint64_t hm = add2_rm(f, pk2(786432.0f, 786432.0f));         // 1.5*2^19 + hi * 2^-4
    const uint64_t hf = sub2(hm, pk2(786432.0f, 786432.0f));           // hi * 2^-4, exact
    const uint64_t lm = fma2(sub2(f, hf), pk2(16777216.0f, 16777216.0f),  // lo + 2^23, exact
                             pk2(8388608.0f, 8388608.0f));
    const float2 hmf = up2(hm), lmf = up2(lm);
    const int32_t h0 = (int32_t)__float_as_uint(hmf.x) - 0x49400000, h1 = (int32_t)__float_as_uint(hmf.y) - 0x49400000;
    const int32_t l0 = (int32_t)(__float_as_uint(lmf.x) & 0x7FFFFFu), l1 = (int32_t)(__float_as_uint(lmf.y) & 0x7FFFFFu);
    e.hi += h0 + h1;
    e.lo += l0 + l1;
    const double hd0 = i32_to_f64_exact(h0), hd1 = i32_to_f64_exact(h1);
    const double ld0 = i32_to_f64_exact(l0), ld1 = i32_to_f64_exact(l1);
    e.hh = __fma_rn(hd0, hd0, e.hh);
    e.hh = __fma_rn(hd1, hd1, e.hh);
    e.hl = __fma_rn(hd0, ld0, e.hl);
    e.hl = __fma_rn(hd1, ld1, e.hl);
    e.ll = __fma_rn(ld0, ld0, e.ll);
    e.ll = __fma_rn(ld1, ld1, e.ll);
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

// mu = RN32(RN64(S1) / (K 2^24)); rstd = RN32(1 / sqrt(RN64(D) / (K^2 2^48) + eps))
// from S1 = sum a and D = K S2 - S1^2 >= 0 (integers, a = x 2^24).
__device__ float2 finish_ld(int64_t s1, unsigned __int128 d, int64_t k, float eps) {
    const double kd = (double)k;
    const double mean64 = __ddiv_rn(__ll2double_rn((long long)s1), __dmul_rn(kd, 16777216.0));
    const double var64 = __ddiv_rn(u128_to_f64(d), __dmul_rn(__dmul_rn(kd, kd), 281474976710656.0));
    return make_float2(__double2float_rn(mean64),
                       __double2float_rn(__ddiv_rn(1.0, __dsqrt_rn(__dadd_rn(var64, (double)eps)))));
}

__device__ float2 finish_stats(const ExactSums &e, int64_t k, float eps) {
    const __int128 s1 = (__int128)e.hi * 1048576 + e.lo;
    const __int128 s2 = ((__int128)e.hh << 40) + ((__int128)e.hl << 21) + (__int128)e.ll;
    const __int128 d = (__int128)k * s2 - s1 * s1;
    return finish_ld((int64_t)s1, (unsigned __int128)d, k, eps);
}

// RMSNorm: ms = RN64(S2) / (K 2^48); rstd = RN32(1 / sqrt(ms + eps)); mu = 0.
__device__ float finish_rms_rstd(unsigned __int128 s2, int64_t k, float eps) {
    const double ms64 = __ddiv_rn(u128_to_f64(s2), __dmul_rn((double)k, 281474976710656.0));
    return __double2float_rn(__ddiv_rn(1.0, __dsqrt_rn(__dadd_rn(ms64, (double)eps))));
}

__device__ float2 finish_stats_rms(const ExactSums &e, int64_t k, float eps) {
    const __int128 s2 = ((__int128)e.hh << 40) + ((__int128)e.hl << 21) + (__int128)e.ll;
    return make_float2(0.0f, finish_rms_rstd((unsigned __int128)s2, k, eps));
}

// ---------------------------------------------------------------------------
// Certified statistics (long rows, one warp per row). Each lane sums x in
// binary64, exactly: every x is a multiple of 2^-24 below 2^16 and a lane
// adds at most SHARQ_K_MAX / 32 = 2048 of them, so every partial sum is a
// multiple of 2^-24 below 2^27 (52 significant bits). Each lane also sums
// x^2 in binary64 (each square exact, 22 significant bits) in two
// accumulators, one rounding per addition; with the join of the two and the
// five butterfly levels, no square passes through more than K/64 + 6
// roundings, so (Higham, Accuracy and Stability of Numerical Algorithms,
// 2nd ed., section 4.2, for non-negative terms) the computed sum s2 is
// within gamma_h S2 <= 2 h u s2 of S2 (h = K/64 + 6, u = 2^-53). The bound
// used below, (K/32 + 8) 2^-51 s2, is larger still. Every step from D (or
// S2, for RMSNorm) to rstd is a monotone rounding or a monotone function,
// so if rstd is the same binary32 value at both ends of the interval that
// holds the exact sum, it is the value at the exact sum: the statistics of
// the exact method, bit for bit. Otherwise the warp sums the row again with
// the exact integer method.
struct FastLane {
    double s1;        // sum x, exact
    double s2a, s2b;  // sum x^2 over alternate elements, rounded
};

__device__ __forceinline__ void fast_pair(uint32_t w, FastLane &f) {
    double d0, d1;
    asm("{\n\t.reg .f16 h0, h1;\n\tmov.b32 {h0, h1}, %2;\n\tcvt.f64.f16 %0, h0;\n\tcvt.f64.f16 %1, h1;\n\t}"
        : "=d"(d0), "=d"(d1) : "r"(w));
    f.s1 = __dadd_rn(f.s1, __dadd_rn(d0, d1));  // both sums exact (multiples of 2^-24 below 2^28)
    f.s2a = __fma_rn(d0, d0, f.s2a);
    f.s2b = __fma_rn(d1, d1, f.s2b);
}

// Floor (up = false) or ceiling (up = true) of a non-negative binary64 value
// below 2^127, as a 128-bit integer.
__device__ unsigned __int128 f64_to_u128(double v, bool up) {
    if (!(v > 0.0)) return 0;
    const uint64_t b = (uint64_t)__double_as_longlong(v);
    const int ex = (int)(b >> 52);
    if (ex == 0) return up ? 1 : 0;  // subnormal: 0 < v < 1
    const uint64_t m = (b & 0xFFFFFFFFFFFFFull) | (1ull << 52);
    const int e = ex - 1075;  // v = m 2^e
    if (e >= 0) return (unsigned __int128)m << e;
    if (e <= -53) return up ? 1 : 0;  // 0 < v < 1
    const uint64_t q = m >> -e;
    const bool frac = (m & ((1ull << -e) - 1ull)) != 0;
    return (unsigned __int128)(q + ((up && frac) ? 1ull : 0ull));
}

// Statistics from the warp's certified sums (s1 = sum a exactly, s2 the
// rounded sum of x^2), or false where the error bound leaves the binary32
// rstd undecided.
__device__ bool certified_stats(int64_t s1, double s2, int64_t k, float eps, bool rms, float2 &out) {
    const double err = __dmul_ru(s2, __dmul_ru((double)(k / 32 + 8), 0x1p-51));
    const unsigned __int128 lo = f64_to_u128(__dmul_rd(__dsub_rd(s2, err), 0x1p48), false);
    const unsigned __int128 hi = f64_to_u128(__dmul_ru(__dadd_ru(s2, err), 0x1p48), true);
    float r_lo, r_hi;
    if (rms) {
        out = make_float2(0.0f, finish_rms_rstd(lo, k, eps));
        r_lo = out.y;
        r_hi = finish_rms_rstd(hi, k, eps);
    } else {
        const __int128 sq = (__int128)s1 * s1;
        const __int128 dlo = (__int128)k * (__int128)lo - sq, dhi = (__int128)k * (__int128)hi - sq;
        out = finish_ld(s1, dlo < 0 ? (unsigned __int128)0 : (unsigned __int128)dlo, k, eps);
        r_lo = out.y;
        r_hi = finish_ld(s1, dhi < 0 ? (unsigned __int128)0 : (unsigned __int128)dhi, k, eps).y;
    }
    return __float_as_uint(r_lo) == __float_as_uint(r_hi);
}

// The exact statistics of one row, summed by a whole warp from global memory
// (every lane returns them).
template <bool RMS>
__device__ float2 exact_row_stats(const uint4 *xr, int nvec, int lane, int64_t k, float eps) {
    LaneSums l = {};
    for (int c = lane; c < nvec; c += 32) {
        const uint4 v = xr[c];
        accum_pair(v.x, l);
        accum_pair(v.y, l);
        accum_pair(v.z, l);
        accum_pair(v.w, l);
    }
    ExactSums e = widen(l);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        e.hi += __shfl_xor_sync(0xFFFFFFFFu, e.hi, o);
        e.lo += __shfl_xor_sync(0xFFFFFFFFu, e.lo, o);
        e.hh += __shfl_xor_sync(0xFFFFFFFFu, e.hh, o);
        e.hl += __shfl_xor_sync(0xFFFFFFFFu, e.hl, o);
        e.ll += __shfl_xor_sync(0xFFFFFFFFu, e.ll, o);
    }
    return RMS ? finish_stats_rms(e, k, eps) : finish_stats(e, k, eps);
}

// RMS: RMSNorm statistics (no centring) instead of LayerNorm's.
template <bool AFFINE, bool RMS>
__global__ void __launch_bounds__(kStatsThreads)
ln_stats_kernel(const uint16_t *__restrict__ x, const uint16_t *__restrict__ gamma,
                const uint16_t *__restrict__ beta, float eps, int64_t k, float2 *__restrict__ stats,
                unsigned *__restrict__ amax_word) {
    extern __shared__ uint4 row_cache[];  // AFFINE only: k / 8 vectors of 8 halves
    __shared__ ExactSums red[kStatsThreads / 32];
    __shared__ uint32_t red_mx[kStatsThreads / 32], red_mn[kStatsThreads / 32];
    __shared__ float red_max[kStatsThreads / 32];
    __shared__ float2 row_stat;

    const int64_t row = blockIdx.x;
    const int nvec = (int)(k / 8);
    const uint4 *xr = reinterpret_cast<const uint4 *>(x + row * k);
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

    LaneSums l = {0, 0, 0.0, 0.0, 0.0};
    uint32_t mx = 0xFC00FC00u, mn = 0x7C007C00u;  // (-inf, -inf), (+inf, +inf) as half2
    auto consume = [&](const uint4 &v, int c) {
        if (AFFINE) row_cache[c] = v;
        accum_pair(v.x, l);
        accum_pair(v.y, l);
        accum_pair(v.z, l);
        accum_pair(v.w, l);
        if (!AFFINE) {
            asm("max.f16x2 %0, %0, %1;" : "+r"(mx) : "r"(v.x));
            asm("max.f16x2 %0, %0, %1;" : "+r"(mx) : "r"(v.y));
            asm("max.f16x2 %0, %0, %1;" : "+r"(mx) : "r"(v.z));
            asm("max.f16x2 %0, %0, %1;" : "+r"(mx) : "r"(v.w));
            asm("min.f16x2 %0, %0, %1;" : "+r"(mn) : "r"(v.x));
            asm("min.f16x2 %0, %0, %1;" : "+r"(mn) : "r"(v.y));
            asm("min.f16x2 %0, %0, %1;" : "+r"(mn) : "r"(v.z));
            asm("min.f16x2 %0, %0, %1;" : "+r"(mn) : "r"(v.w));
        }
    };
    // Two loads in flight per thread (default caching: the encode pass
    // re-reads x from L2).
    int c = threadIdx.x;
    for (; c + kStatsThreads < nvec; c += 2 * kStatsThreads) {
        const uint4 v0 = xr[c], v1 = xr[c + kStatsThreads];
        consume(v0, c);
        consume(v1, c + kStatsThreads);
    }
    if (c < nvec) consume(xr[c], c);
    ExactSums e = widen(l);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        e.hi += __shfl_xor_sync(0xFFFFFFFFu, e.hi, o);
        e.lo += __shfl_xor_sync(0xFFFFFFFFu, e.lo, o);
        e.hh += __shfl_xor_sync(0xFFFFFFFFu, e.hh, o);
        e.hl += __shfl_xor_sync(0xFFFFFFFFu, e.hl, o);
        e.ll += __shfl_xor_sync(0xFFFFFFFFu, e.ll, o);
        if (!AFFINE) {
            const uint32_t omx = __shfl_xor_sync(0xFFFFFFFFu, mx, o), omn = __shfl_xor_sync(0xFFFFFFFFu, mn, o);
            asm("max.f16x2 %0, %0, %1;" : "+r"(mx) : "r"(omx));
            asm("min.f16x2 %0, %0, %1;" : "+r"(mn) : "r"(omn));
        }
    }
    if (lane == 0) {
        red[warp] = e;
        red_mx[warp] = mx;
        red_mn[warp] = mn;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        ExactSums t = red[0];
        uint32_t tmx = red_mx[0], tmn = red_mn[0];
        for (int w = 1; w < kStatsThreads / 32; ++w) {
            t.hi += red[w].hi;
            t.lo += red[w].lo;
            t.hh += red[w].hh;
            t.hl += red[w].hl;
            t.ll += red[w].ll;
            asm("max.f16x2 %0, %0, %1;" : "+r"(tmx) : "r"(red_mx[w]));
            asm("min.f16x2 %0, %0, %1;" : "+r"(tmn) : "r"(red_mn[w]));
        }
        const float2 st = RMS ? finish_stats_rms(t, k, eps) : finish_stats(t, k, eps);
        stats[row] = st;
        row_stat = st;
        if (!AFFINE) {
            // X_ln = RN(RN(x - mu) * rstd) is non-decreasing in x: the row's
            // amax|X_ln| is reached at its smallest or largest x.
            const float xmax = fmaxf(h2f((uint16_t)tmx), h2f((uint16_t)(tmx >> 16)));
            const float xmin = fminf(h2f((uint16_t)tmn), h2f((uint16_t)(tmn >> 16)));
            const float a = fmaxf(fabsf(__fmul_rn(__fsub_rn(xmax, st.x), st.y)),
                                  fabsf(__fmul_rn(__fsub_rn(xmin, st.x), st.y)));
            atomicMax(amax_word, __float_as_uint(a));  // non-negative floats order like their bits
        }
    }
    if (!AFFINE) return;
    __syncthreads();
    const float mu = row_stat.x, rstd = row_stat.y;
    const bool has_g = gamma != nullptr, has_b = beta != nullptr;
    float amax = 0.0f;
    for (int c = threadIdx.x; c < nvec; c += kStatsThreads) {
        const uint4 v = row_cache[c];
        const uint4 g = has_g ? __ldg(reinterpret_cast<const uint4 *>(gamma) + c) : make_uint4(0, 0, 0, 0);
        const uint4 b = has_b ? __ldg(reinterpret_cast<const uint4 *>(beta) + c) : make_uint4(0, 0, 0, 0);
        const uint32_t xv[4] = {v.x, v.y, v.z, v.w}, gv[4] = {g.x, g.y, g.z, g.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const float xl = ln_apply(h2f((uint16_t)(xv[q] >> (16 * h))), mu, rstd, has_g,
                                          h2f((uint16_t)(gv[q] >> (16 * h))), has_b, h2f((uint16_t)(bv[q] >> (16 * h))));
                amax = fmaxf(amax, fabsf(xl));
            }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
    if (lane == 0) red_max[warp] = amax;
    __syncthreads();
    if (threadIdx.x == 0) {
        float a = 0.0f;
        for (int w = 0; w < kStatsThreads / 32; ++w) a = fmaxf(a, red_max[w]);
        atomicMax(amax_word, __float_as_uint(a));
    }
}

// Warp per row (rows of at most kWarpRowMaxK elements, or any row length
// when the rows fill the GPU): eight warps per CTA, the statistics reduced
// with shuffles only, and one atomic per CTA for the tensor's amax (one CTA
// per row leaves most threads idle on short rows and puts one atomic per row
// on a single word). Same exact sums, so the results equal those of
// ln_stats_kernel bit for bit. The row streams through a ring of
// kStatsStages slots per lane (four 16-byte vectors each) filled by
// asynchronous copies issued two iterations ahead, so that loads stay in
// flight while the lane computes.
// Without gamma/beta, each warp takes `rpw` consecutive rows and leaves
// each row's reduced sums in shared memory; once all warps are done, one
// thread per row finishes the statistics (the binary64 divisions and the
// 128-bit products run on 8 * rpw threads at once instead of one lane per
// warp and row, which dominated on short rows). With gamma/beta (rpw = 1)
// lane 0 finishes each row at once and the warp reads the row a second time
// (from L2) for amax|X_ln|.
constexpr int64_t kWarpRowMaxK = 8192;
#ifndef SQ_STATS_AHEAD
#define SQ_STATS_AHEAD 2
#endif
// Iterations of copies in flight ahead of the one consumed. Measured on B200
// (K = 14336 / 4096 / 18944 preparations): 2 gives 203.8 / 69.7 / 145.2 us,
// 3 gives 204.8 / 70.7 / 141.8, 4 gives 204.7 / 71.7 / 141.3 (more ring
// leaves fewer CTAs resident).
constexpr int kStatsAhead = SQ_STATS_AHEAD;
constexpr int kStatsStages = kStatsAhead + 1;
constexpr int kStatsRingBytes = (kStatsThreads / 32) * kStatsStages * 4 * 32 * 16;  // 48 KB at depth 2
constexpr int kStatsMaxRpw = 4;  // rows per warp, short rows

// FAST: certified binary64 sums with the exact method as the fallback (rows
// longer than 2048 elements).
template <bool AFFINE, bool RMS, bool FAST>
__global__ void __launch_bounds__(kStatsThreads)
ln_stats_warp_kernel(const uint16_t *__restrict__ x, const uint16_t *__restrict__ gamma,
                     const uint16_t *__restrict__ beta, float eps, int64_t k, int64_t m_tok, int rpw,
                     float2 *__restrict__ stats, unsigned *__restrict__ amax_word) {
    constexpr int W = kStatsThreads / 32;
    constexpr int NS = (AFFINE || !FAST) ? 1 : W * kStatsMaxRpw;
    extern __shared__ uint4 ring[];  // [warp][stage][vector j][lane]
    __shared__ float red_max[W];
    __shared__ ExactSums rsum[(AFFINE || FAST) ? 1 : W * kStatsMaxRpw];
    __shared__ uint32_t rmx[AFFINE ? 1 : W * kStatsMaxRpw], rmn[AFFINE ? 1 : W * kStatsMaxRpw];
    __shared__ int64_t fs1[NS];
    __shared__ double fs2[NS];
    __shared__ int redo[NS];
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    if (AFFINE) rpw = 1;
    const int64_t cta_row0 = (int64_t)blockIdx.x * W * rpw;
    const int nvec = (int)(k / 8);
    const int nvl = nvec / 32;        // vectors per lane (k is a multiple of 256)
    const int iters = (nvl + 3) / 4;  // four vectors per lane per iteration
    uint4 *wring = ring + (size_t)warp * kStatsStages * 4 * 32;
    const uint32_t wbase = smem_u32(wring);
    float amax = 0.0f;
    for (int i = 0; i < rpw; ++i) {
        const int slot = warp * rpw + i;
        const int64_t row = cta_row0 + slot;
        if (row >= m_tok) break;  // warp-uniform
        const uint4 *xr = reinterpret_cast<const uint4 *>(x + row * k);
        auto issue = [&](int it) {
            if (it < iters) {
                const int st = it % kStatsStages;
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    if (4 * it + j < nvl)
                        cp_async16(wbase + (uint32_t)(((st * 4 + j) * 32 + lane) * 16), xr + lane + 32 * (4 * it + j));
            }
            cp_async_commit();  // possibly empty: one group per iteration keeps the count uniform
        };
        LaneSums l = {};
        FastLane f = {0.0, 0.0, 0.0};
        uint32_t mx = 0xFC00FC00u, mn = 0x7C007C00u;  // (-inf, -inf), (+inf, +inf) as half2
        auto consume = [&](const uint4 &v) {
            if (FAST) {
                fast_pair(v.x, f);
                fast_pair(v.y, f);
                fast_pair(v.z, f);
                fast_pair(v.w, f);
            } else {
                accum_pair(v.x, l);
                accum_pair(v.y, l);
                accum_pair(v.z, l);
                accum_pair(v.w, l);
            }
            if (!AFFINE) {
                const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    asm("max.f16x2 %0, %0, %1;" : "+r"(mx) : "r"(w4[q]));
                    asm("min.f16x2 %0, %0, %1;" : "+r"(mn) : "r"(w4[q]));
                }
            }
        };
#pragma unroll
        for (int a = 0; a < kStatsAhead; ++a) issue(a);
        for (int it = 0; it < iters; ++it) {
            cp_async_wait<kStatsAhead - 1>();  // this lane's copies of iteration `it` have landed
            const int st = it % kStatsStages;
            if (4 * it + 3 < nvl) {
                const uint4 v0 = wring[(st * 4 + 0) * 32 + lane], v1 = wring[(st * 4 + 1) * 32 + lane];
                const uint4 v2 = wring[(st * 4 + 2) * 32 + lane], v3 = wring[(st * 4 + 3) * 32 + lane];
                consume(v0);
                consume(v1);
                consume(v2);
                consume(v3);
            } else {
                for (int j = 0; 4 * it + j < nvl; ++j) consume(wring[(st * 4 + j) * 32 + lane]);
            }
            issue(it + kStatsAhead);  // refills the slot consumed in the previous iteration
        }
        cp_async_wait<0>();
        if (!AFFINE) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const uint32_t omx = __shfl_xor_sync(0xFFFFFFFFu, mx, o), omn = __shfl_xor_sync(0xFFFFFFFFu, mn, o);
                asm("max.f16x2 %0, %0, %1;" : "+r"(mx) : "r"(omx));
                asm("min.f16x2 %0, %0, %1;" : "+r"(mn) : "r"(omn));
            }
        }
        // Butterfly reductions: every lane ends with the same totals (each
        // step adds the same two operands on both lanes of a pair).
        ExactSums e = {};
        int64_t s1 = 0;
        double s2 = 0.0;
        if (FAST) {
            s1 = __double2ll_rn(__dmul_rn(f.s1, 16777216.0));  // sum a over the lane, an integer below 2^51
            s2 = __dadd_rn(f.s2a, f.s2b);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                s1 += __shfl_xor_sync(0xFFFFFFFFu, s1, o);
                s2 = __dadd_rn(s2, __shfl_xor_sync(0xFFFFFFFFu, s2, o));
            }
        } else {
            e = widen(l);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                e.hi += __shfl_xor_sync(0xFFFFFFFFu, e.hi, o);
                e.lo += __shfl_xor_sync(0xFFFFFFFFu, e.lo, o);
                e.hh += __shfl_xor_sync(0xFFFFFFFFu, e.hh, o);
                e.hl += __shfl_xor_sync(0xFFFFFFFFu, e.hl, o);
                e.ll += __shfl_xor_sync(0xFFFFFFFFu, e.ll, o);
            }
        }
        if (!AFFINE) {
            if (lane == 0) {
                if (FAST) {
                    fs1[slot] = s1;
                    fs2[slot] = s2;
                } else {
                    rsum[slot] = e;
                }
                rmx[slot] = mx;
                rmn[slot] = mn;
            }
            continue;
        }
        float2 st = make_float2(0.0f, 0.0f);
        if (FAST) {
            const bool ok = certified_stats(s1, s2, k, eps, RMS, st);  // the same on every lane
            if (!ok) st = exact_row_stats<RMS>(xr, nvec, lane, k, eps);
            if (lane == 0) stats[row] = st;
        } else {
            if (lane == 0) {
                st = RMS ? finish_stats_rms(e, k, eps) : finish_stats(e, k, eps);
                stats[row] = st;
            }
            st.x = __shfl_sync(0xFFFFFFFFu, st.x, 0);
            st.y = __shfl_sync(0xFFFFFFFFu, st.y, 0);
        }
        const bool has_g = gamma != nullptr, has_b = beta != nullptr;
        for (int cc = lane; cc < nvec; cc += 32) {
            const uint4 v = xr[cc];
            const uint4 g = has_g ? __ldg(reinterpret_cast<const uint4 *>(gamma) + cc) : make_uint4(0, 0, 0, 0);
            const uint4 bb = has_b ? __ldg(reinterpret_cast<const uint4 *>(beta) + cc) : make_uint4(0, 0, 0, 0);
            const uint32_t xv[4] = {v.x, v.y, v.z, v.w}, gv[4] = {g.x, g.y, g.z, g.w}, bv[4] = {bb.x, bb.y, bb.z, bb.w};
#pragma unroll
            for (int q = 0; q < 4; ++q)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const float xl = ln_apply(h2f((uint16_t)(xv[q] >> (16 * h))), st.x, st.y, has_g,
                                              h2f((uint16_t)(gv[q] >> (16 * h))), has_b,
                                              h2f((uint16_t)(bv[q] >> (16 * h))));
                    amax = fmaxf(amax, fabsf(xl));
                }
        }
    }
    if (!AFFINE) {
        // X_ln = RN(RN(x - mu) * rstd) is non-decreasing in x: the row's
        // amax|X_ln| is reached at its smallest or largest x.
        auto row_amax = [&](const float2 &st, int slot) {
            const uint32_t mx = rmx[slot], mn = rmn[slot];
            const float xmax = fmaxf(h2f((uint16_t)mx), h2f((uint16_t)(mx >> 16)));
            const float xmin = fminf(h2f((uint16_t)mn), h2f((uint16_t)(mn >> 16)));
            return fmaxf(fabsf(__fmul_rn(__fsub_rn(xmax, st.x), st.y)), fabsf(__fmul_rn(__fsub_rn(xmin, st.x), st.y)));
        };
        __syncthreads();  // every row's sums are in shared memory
        const int slot = threadIdx.x;
        const int64_t row = cta_row0 + slot;
        if (slot < W * rpw && row < m_tok) {
            float2 st;
            bool ok = true;
            if (FAST) {
                ok = certified_stats(fs1[slot], fs2[slot], k, eps, RMS, st);
                redo[slot] = ok ? 0 : 1;
            } else {
                st = RMS ? finish_stats_rms(rsum[slot], k, eps) : finish_stats(rsum[slot], k, eps);
            }
            if (ok) {
                stats[row] = st;
                amax = row_amax(st, slot);
            }
        }
        if (FAST) {
            __syncthreads();  // the undecided rows are marked
            for (int i = 0; i < rpw; ++i) {
                const int rs = warp * rpw + i;
                const int64_t rrow = cta_row0 + rs;
                if (rrow >= m_tok) break;  // warp-uniform
                if (!redo[rs]) continue;   // warp-uniform
                const float2 st = exact_row_stats<RMS>(reinterpret_cast<const uint4 *>(x + rrow * k), nvec, lane, k, eps);
                if (lane == 0) {
                    stats[rrow] = st;
                    amax = fmaxf(amax, row_amax(st, rs));
                }
            }
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
    if (lane == 0) red_max[warp] = amax;
    __syncthreads();
    if (threadIdx.x == 0) {
        float a = 0.0f;
        for (int w = 0; w < W; ++w) a = fmaxf(a, red_max[w]);
        atomicMax(amax_word, __float_as_uint(a));  // non-negative floats order like their bits
    }
}

// Statistics of rows longer than 2048 elements: one warp per row, the
// warps of a persistent grid (every CTA resident) taking rows in increasing
// order with the grid stride, so that no partial last wave is left. Certified
// binary64 sums as in ln_stats_warp_kernel's FAST form, each warp finishing
// its own rows (all lanes compute the same finish; undecided rows are summed
// again exactly). Without gamma/beta the row's amax|X_ln| comes from its
// min and max of x; with them the warp reads the row again (from L2). One
// amax atomic per CTA. The kernel lets the encode pass launch at once: its
// CTAs take an SM's slots only as this kernel's CTAs leave, and wait for
// this kernel's completion before reading anything it writes.
template <bool AFFINE, bool RMS>
__global__ void __launch_bounds__(kStatsThreads)
ln_stats_long_kernel(const uint16_t *__restrict__ x, const uint16_t *__restrict__ gamma,
                     const uint16_t *__restrict__ beta, float eps, int64_t k, int64_t m_tok,
                     float2 *__restrict__ stats, unsigned *__restrict__ amax_word) {
    constexpr int W = kStatsThreads / 32;
    extern __shared__ uint4 ring[];  // [warp][stage][vector j][lane]
    __shared__ float red_max[W];
    griddep_launch();
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int nvec = (int)(k / 8);
    const int nvl = nvec / 32;        // vectors per lane (k is a multiple of 256)
    const int iters = (nvl + 3) / 4;  // four vectors per lane per iteration
    uint4 *wring = ring + (size_t)warp * kStatsStages * 4 * 32;
    const uint32_t wbase = smem_u32(wring);
    const int64_t nwarps = (int64_t)gridDim.x * W;
    float amax = 0.0f;
    for (int64_t row = (int64_t)blockIdx.x * W + warp; row < m_tok; row += nwarps) {
        const uint4 *xr = reinterpret_cast<const uint4 *>(x + row * k);
        auto issue = [&](int it) {
            if (it < iters) {
                const int stg = it % kStatsStages;
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    if (4 * it + j < nvl)
                        cp_async16(wbase + (uint32_t)(((stg * 4 + j) * 32 + lane) * 16), xr + lane + 32 * (4 * it + j));
            }
            cp_async_commit();  // possibly empty: one group per iteration keeps the count uniform
        };
        FastLane f = {0.0, 0.0, 0.0};
        uint32_t mx = 0xFC00FC00u, mn = 0x7C007C00u;  // (-inf, -inf), (+inf, +inf) as half2
        auto consume = [&](const uint4 &v) {
            fast_pair(v.x, f);
            fast_pair(v.y, f);
            fast_pair(v.z, f);
            fast_pair(v.w, f);
            if (!AFFINE) {
                const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    asm("max.f16x2 %0, %0, %1;" : "+r"(mx) : "r"(w4[q]));
                    asm("min.f16x2 %0, %0, %1;" : "+r"(mn) : "r"(w4[q]));
                }
            }
        };
#pragma unroll
        for (int a = 0; a < kStatsAhead; ++a) issue(a);
        for (int it = 0; it < iters; ++it) {
            cp_async_wait<kStatsAhead - 1>();  // this lane's copies of iteration `it` have landed
            const int stg = it % kStatsStages;
            if (4 * it + 3 < nvl) {
                const uint4 v0 = wring[(stg * 4 + 0) * 32 + lane], v1 = wring[(stg * 4 + 1) * 32 + lane];
                const uint4 v2 = wring[(stg * 4 + 2) * 32 + lane], v3 = wring[(stg * 4 + 3) * 32 + lane];
                consume(v0);
                consume(v1);
                consume(v2);
                consume(v3);
            } else {
                for (int j = 0; 4 * it + j < nvl; ++j) consume(wring[(stg * 4 + j) * 32 + lane]);
            }
            issue(it + kStatsAhead);  // refills the slot consumed in the previous iteration
        }
        cp_async_wait<0>();
        // Butterfly reductions: every lane ends with the same totals.
        int64_t s1 = __double2ll_rn(__dmul_rn(f.s1, 16777216.0));  // sum a over the lane, an integer below 2^51
        double s2 = __dadd_rn(f.s2a, f.s2b);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            s1 += __shfl_xor_sync(0xFFFFFFFFu, s1, o);
            s2 = __dadd_rn(s2, __shfl_xor_sync(0xFFFFFFFFu, s2, o));
            if (!AFFINE) {
                const uint32_t omx = __shfl_xor_sync(0xFFFFFFFFu, mx, o), omn = __shfl_xor_sync(0xFFFFFFFFu, mn, o);
                asm("max.f16x2 %0, %0, %1;" : "+r"(mx) : "r"(omx));
                asm("min.f16x2 %0, %0, %1;" : "+r"(mn) : "r"(omn));
            }
        }
        float2 st;
        const bool ok = certified_stats(s1, s2, k, eps, RMS, st);  // the same on every lane
        if (!ok) st = exact_row_stats<RMS>(xr, nvec, lane, k, eps);
        if (lane == 0) stats[row] = st;
        if (!AFFINE) {
            // X_ln = RN(RN(x - mu) * rstd) is non-decreasing in x: the row's
            // amax|X_ln| is reached at its smallest or largest x.
            const float xmax = fmaxf(h2f((uint16_t)mx), h2f((uint16_t)(mx >> 16)));
            const float xmin = fminf(h2f((uint16_t)mn), h2f((uint16_t)(mn >> 16)));
            amax = fmaxf(amax, fmaxf(fabsf(__fmul_rn(__fsub_rn(xmax, st.x), st.y)),
                                     fabsf(__fmul_rn(__fsub_rn(xmin, st.x), st.y))));
        } else {
            const bool has_g = gamma != nullptr, has_b = beta != nullptr;
            for (int cc = lane; cc < nvec; cc += 32) {
                const uint4 v = xr[cc];
                const uint4 g = has_g ? __ldg(reinterpret_cast<const uint4 *>(gamma) + cc) : make_uint4(0, 0, 0, 0);
                const uint4 bb = has_b ? __ldg(reinterpret_cast<const uint4 *>(beta) + cc) : make_uint4(0, 0, 0, 0);
                const uint32_t xv[4] = {v.x, v.y, v.z, v.w}, gv[4] = {g.x, g.y, g.z, g.w},
                               bv[4] = {bb.x, bb.y, bb.z, bb.w};
#pragma unroll
                for (int q = 0; q < 4; ++q)
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const float xl = ln_apply(h2f((uint16_t)(xv[q] >> (16 * h))), st.x, st.y, has_g,
                                                  h2f((uint16_t)(gv[q] >> (16 * h))), has_b,
                                                  h2f((uint16_t)(bv[q] >> (16 * h))));
                        amax = fmaxf(amax, fabsf(xl));
                    }
            }
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
    if (lane == 0) red_max[warp] = amax;
    __syncthreads();
    if (threadIdx.x == 0) {
        float a = 0.0f;
        for (int w = 0; w < W; ++w) a = fmaxf(a, red_max[w]);
        atomicMax(amax_word, __float_as_uint(a));  // non-negative floats order like their bits
    }
}

// Residual add fused with the statistics pass: x = RN16(h + d) (binary16
// addition, the residual stream update of a pre-norm layer) is written out
// and, in the same pass, x's exact LayerNorm / RMSNorm statistics and the
// row's amax|X_ln| are taken as in ln_stats_long_kernel (FAST: certified
// binary64 sums with the exact fallback, for rows longer than 2048
// elements; otherwise the exact integer sums). One warp per row, the warps
// of a persistent grid taking rows with the grid stride; each lane adds and
// stores the 16-byte vectors lane, lane + 32, ... of its row, so the
// fallback and the affine amax sweep re-read only what the same lane wrote.
// The encode pass then reads x once more (the only other read of x).
template <bool AFFINE, bool RMS, bool FAST>
__global__ void __launch_bounds__(kStatsThreads)
add_stats_kernel(const uint16_t *h, const uint16_t *d, uint16_t *x_out,
                 const uint16_t *__restrict__ gamma, const uint16_t *__restrict__ beta, float eps, int64_t k,
                 int64_t m_tok, float2 *__restrict__ stats, unsigned *__restrict__ amax_word) {
    constexpr int W = kStatsThreads / 32;
    constexpr int V = 4;  // vectors per lane in flight
    __shared__ float red_max[W];
    griddep_launch();
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int nvec = (int)(k / 8);
    const int64_t nwarps = (int64_t)gridDim.x * W;
    float amax = 0.0f;
    for (int64_t row = (int64_t)blockIdx.x * W + warp; row < m_tok; row += nwarps) {
        const uint4 *hr = reinterpret_cast<const uint4 *>(h + row * k);
        const uint4 *dr = reinterpret_cast<const uint4 *>(d + row * k);
        uint4 *xr = reinterpret_cast<uint4 *>(x_out + row * k);
        LaneSums l = {};
        FastLane f = {0.0, 0.0, 0.0};
        uint32_t mx = 0xFC00FC00u, mn = 0x7C007C00u;  // (-inf, -inf), (+inf, +inf) as half2
        for (int c0 = lane; c0 < nvec; c0 += 32 * V) {
            uint4 hv[V], dv[V];
#pragma unroll
            for (int j = 0; j < V; ++j)
                if (c0 + 32 * j < nvec) {
                    hv[j] = __ldcs(hr + c0 + 32 * j);
                    dv[j] = __ldcs(dr + c0 + 32 * j);
                }
#pragma unroll
            for (int j = 0; j < V; ++j) {
                if (c0 + 32 * j >= nvec) break;
                uint4 xv;
                asm("add.rn.f16x2 %0, %1, %2;" : "=r"(xv.x) : "r"(hv[j].x), "r"(dv[j].x));
                asm("add.rn.f16x2 %0, %1, %2;" : "=r"(xv.y) : "r"(hv[j].y), "r"(dv[j].y));
                asm("add.rn.f16x2 %0, %1, %2;" : "=r"(xv.z) : "r"(hv[j].z), "r"(dv[j].z));
                asm("add.rn.f16x2 %0, %1, %2;" : "=r"(xv.w) : "r"(hv[j].w), "r"(dv[j].w));
                xr[c0 + 32 * j] = xv;
                const uint32_t w4[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    if (FAST) fast_pair(w4[q], f);
                    else accum_pair(w4[q], l);
                    if (!AFFINE) {
                        asm("max.f16x2 %0, %0, %1;" : "+r"(mx) : "r"(w4[q]));
                        asm("min.f16x2 %0, %0, %1;" : "+r"(mn) : "r"(w4[q]));
                    }
                }
            }
        }
        if (!AFFINE) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const uint32_t omx = __shfl_xor_sync(0xFFFFFFFFu, mx, o), omn = __shfl_xor_sync(0xFFFFFFFFu, mn, o);
                asm("max.f16x2 %0, %0, %1;" : "+r"(mx) : "r"(omx));
                asm("min.f16x2 %0, %0, %1;" : "+r"(mn) : "r"(omn));
            }
        }
        float2 st;
        if (FAST) {
            int64_t s1 = __double2ll_rn(__dmul_rn(f.s1, 16777216.0));
            double s2 = __dadd_rn(f.s2a, f.s2b);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                s1 += __shfl_xor_sync(0xFFFFFFFFu, s1, o);
                s2 = __dadd_rn(s2, __shfl_xor_sync(0xFFFFFFFFu, s2, o));
            }
            if (!certified_stats(s1, s2, k, eps, RMS, st))  // the same on every lane
                st = exact_row_stats<RMS>(xr, nvec, lane, k, eps);
        } else {
            ExactSums e = widen(l);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                e.hi += __shfl_xor_sync(0xFFFFFFFFu, e.hi, o);
                e.lo += __shfl_xor_sync(0xFFFFFFFFu, e.lo, o);
                e.hh += __shfl_xor_sync(0xFFFFFFFFu, e.hh, o);
                e.hl += __shfl_xor_sync(0xFFFFFFFFu, e.hl, o);
                e.ll += __shfl_xor_sync(0xFFFFFFFFu, e.ll, o);
            }
            st = RMS ? finish_stats_rms(e, k, eps) : finish_stats(e, k, eps);
        }
        if (lane == 0) stats[row] = st;
        if (!AFFINE) {
            const float xmax = fmaxf(h2f((uint16_t)mx), h2f((uint16_t)(mx >> 16)));
            const float xmin = fminf(h2f((uint16_t)mn), h2f((uint16_t)(mn >> 16)));
            amax = fmaxf(amax, fmaxf(fabsf(__fmul_rn(__fsub_rn(xmax, st.x), st.y)),
                                     fabsf(__fmul_rn(__fsub_rn(xmin, st.x), st.y))));
        } else {
            const bool has_g = gamma != nullptr, has_b = beta != nullptr;
            for (int cc = lane; cc < nvec; cc += 32) {
                const uint4 v = xr[cc];
                const uint4 g = has_g ? __ldg(reinterpret_cast<const uint4 *>(gamma) + cc) : make_uint4(0, 0, 0, 0);
                const uint4 bb = has_b ? __ldg(reinterpret_cast<const uint4 *>(beta) + cc) : make_uint4(0, 0, 0, 0);
                const uint32_t xv[4] = {v.x, v.y, v.z, v.w}, gv[4] = {g.x, g.y, g.z, g.w},
                               bv[4] = {bb.x, bb.y, bb.z, bb.w};
#pragma unroll
                for (int q = 0; q < 4; ++q)
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh)
                        amax = fmaxf(amax, fabsf(ln_apply(h2f((uint16_t)(xv[q] >> (16 * hh))), st.x, st.y, has_g,
                                                          h2f((uint16_t)(gv[q] >> (16 * hh))), has_b,
                                                          h2f((uint16_t)(bv[q] >> (16 * hh))))));
            }
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
    if (lane == 0) red_max[warp] = amax;
    __syncthreads();
    if (threadIdx.x == 0) {
        float a = 0.0f;
        for (int w = 0; w < W; ++w) a = fmaxf(a, red_max[w]);
        atomicMax(amax_word, __float_as_uint(a));
    }
}

// ---------------------------------------------------------------------------
// Encode pass.

// Store `nbytes` (<= 8) little-endian bytes of v at p, using the widest
// aligned stores the address allows.
__device__ __forceinline__ void store_bytes(uint8_t *p, uint64_t v, int nbytes) {
    int i = 0;
    while (i < nbytes) {
        const uintptr_t a = reinterpret_cast<uintptr_t>(p + i);
        const uint64_t w = v >> (8 * i);
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

// OR `bits` (<= 64) bits of v into the bit stream at bit position `pos` from
// a 4-byte-aligned base, with word atomics (neighbouring units share words).
__device__ __forceinline__ void or_bits(uint32_t *base, uint64_t pos, uint64_t v, int bits) {
    uint64_t w = pos >> 5;
    int sh = (int)(pos & 31);
    int done = 0;
    while (done < bits) {
        const uint32_t piece = (uint32_t)((v >> done) << sh);
        const int take = 32 - sh < bits - done ? 32 - sh : bits - done;
        const uint32_t mask = take >= 32 ? 0xFFFFFFFFu : (((1u << take) - 1u) << sh);
        if (piece & mask) atomicOr(base + w, piece & mask);
        done += take;
        sh = 0;
        ++w;
    }
}

// Keep mask of the 16 values of a unit: in every aligned group of M, the n
// largest magnitudes, equal magnitudes to the lower index. The rank of value
// i counts the values that beat it: larger, or equal at a lower index.
template <int M>
__device__ __forceinline__ uint32_t keep_mask(const float (&v)[kUnit], int n) {
    uint32_t keep = 0;
#pragma unroll
    for (int g = 0; g < kUnit / M; ++g) {
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
                const int c = a[i] >= a[j];  // i beats j
                rank[j] += c;
                rank[i] += 1 - c;
            }
#pragma unroll
        for (int i = 0; i < M; ++i) keep |= (uint32_t)(rank[i] < n) << (g * M + i);
    }
    return keep;
}

// Block quantization of one thread's 16 values (an NVFP4 block, or half of an
// MXFP4 block whose other half sits in the neighbouring lane). Produces the
// scale code, the step d and the 16 E2M1 codes (8 bytes).
// m = 4: the four ranks as the bytes of one word; each of the six pairs adds
// 1 to the byte of the element that loses the comparison. A rank byte r
// survives iff r < n: (0x80 + r - n) has bit 7 clear exactly then (no
// borrows cross bytes since r, n <= 4); a multiply gathers the four bits.
template <>
__device__ __forceinline__ uint32_t keep_mask<4>(const float (&v)[kUnit], int n) {
    const uint32_t nn = (uint32_t)n * 0x01010101u;
    uint32_t keep = 0;
#pragma unroll
    for (int g = 0; g < kUnit / 4; ++g) {
        const uint32_t a0 = __float_as_uint(v[4 * g]) & 0x7FFFFFFFu, a1 = __float_as_uint(v[4 * g + 1]) & 0x7FFFFFFFu;
        const uint32_t a2 = __float_as_uint(v[4 * g + 2]) & 0x7FFFFFFFu, a3 = __float_as_uint(v[4 * g + 3]) & 0x7FFFFFFFu;
        uint32_t r = (a0 >= a1 ? 0x00000100u : 0x00000001u) + (a0 >= a2 ? 0x00010000u : 0x00000001u) +
                     (a0 >= a3 ? 0x01000000u : 0x00000001u);
        r += (a1 >= a2 ? 0x00010000u : 0x00000100u) + (a1 >= a3 ? 0x01000000u : 0x00000100u) +
             (a2 >= a3 ? 0x01000000u : 0x00010000u);
        const uint32_t lost = ((r | 0x80808080u) - nn) & 0x80808080u;  // bit 7 of byte i: rank_i >= n
        const uint32_t kept = (~lost & 0x80808080u) >> 7;               // bits 0, 8, 16, 24
        keep |= ((kept * 0x00204081u) >> 21 & 0xFu) << (4 * g);
    }
    return keep;
}

// m = 2: keep both (n = 2) or the larger, the first on ties (n = 1).
template <>
__device__ __forceinline__ uint32_t keep_mask<2>(const float (&v)[kUnit], int n) {
    if (n >= 2) return 0xFFFFu;
    uint32_t keep = 0;
#pragma unroll
    for (int g = 0; g < kUnit / 2; ++g) {
        const uint32_t a0 = __float_as_uint(v[2 * g]) & 0x7FFFFFFFu, a1 = __float_as_uint(v[2 * g + 1]) & 0x7FFFFFFFu;
        keep |= (a0 >= a1 ? 1u : 2u) << (2 * g);
    }
    return keep;
}

// m = 4, n = 2 with n fixed at compile time: an element survives iff it
// beats at least two of the other three. For a before b in the group, the
// sign of RN(|a| - |b|) is set iff |a| < |b| (equal magnitudes give +0),
// i.e. iff b beats a; each verdict is a majority of three such signs, one
// three-input logic operation on the bit patterns. (Measured on B200: fewer
// instructions than comparisons into predicates and predicate logic.)
__device__ __forceinline__ uint32_t keep_mask_42(const float (&v)[kUnit]) {
    uint32_t keep = 0;
#pragma unroll
    for (int g = 0; g < kUnit / 4; ++g) {
        const float a0 = fabsf(v[4 * g]), a1 = fabsf(v[4 * g + 1]), a2 = fabsf(v[4 * g + 2]), a3 = fabsf(v[4 * g + 3]);
        const uint32_t s01 = __float_as_uint(__fsub_rn(a0, a1)), s02 = __float_as_uint(__fsub_rn(a0, a2));
        const uint32_t s03 = __float_as_uint(__fsub_rn(a0, a3)), s12 = __float_as_uint(__fsub_rn(a1, a2));
        const uint32_t s13 = __float_as_uint(__fsub_rn(a1, a3)), s23 = __float_as_uint(__fsub_rn(a2, a3));
        const uint32_t k0 = ~((s01 & s02) | (s01 & s03) | (s02 & s03));
        const uint32_t k1 = (s01 & ~s12) | (s01 & ~s13) | (~s12 & ~s13);
        const uint32_t k2 = (s02 & s12) | (s02 & ~s23) | (s12 & ~s23);
        const uint32_t k3 = (s03 & s13) | (s03 & s23) | (s13 & s23);
        keep |= ((k0 >> 31) | (k1 >> 31) << 1 | (k2 >> 31) << 2 | (k3 >> 31) << 3) << (4 * g);
    }
    return keep;
}

// m = 8, n = 4 with n fixed at compile time: the fourth largest magnitude t
// of a group comes from sorting each half with a four-input network and
// merging (for halves sorted descending, the four largest of the group are
// max(a_i, b_{3-i}), so t is the smallest of those); an element survives iff
// its magnitude is >= t. Where exactly four do, nothing ties at t and that
// is the top-4 set whatever the tie rule; otherwise (a tie at t) the
// rank-based selection decides the unit.
__device__ __forceinline__ uint32_t keep_mask_84(const float (&v)[kUnit]) {
    uint32_t keep = 0;
    bool exact = true;
#pragma unroll
    for (int g = 0; g < 2; ++g) {
        float a[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) a[i] = fabsf(v[8 * g + i]);
        float srt[2][4];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const float p = fmaxf(a[4 * h], a[4 * h + 1]), q = fminf(a[4 * h], a[4 * h + 1]);
            const float r = fmaxf(a[4 * h + 2], a[4 * h + 3]), s = fminf(a[4 * h + 2], a[4 * h + 3]);
            const float x = fminf(p, r), y = fmaxf(q, s);
            srt[h][0] = fmaxf(p, r);
            srt[h][1] = fmaxf(x, y);
            srt[h][2] = fminf(x, y);
            srt[h][3] = fminf(q, s);
        }
        const float t = fminf(fminf(fmaxf(srt[0][0], srt[1][3]), fmaxf(srt[0][1], srt[1][2])),
                              fminf(fmaxf(srt[0][2], srt[1][1]), fmaxf(srt[0][3], srt[1][0])));
        uint32_t kg = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) kg |= ((~__float_as_uint(__fsub_rn(a[i], t))) >> 31) << i;  // a_i >= t
        exact = exact && __popc(kg) == 4;
        keep |= kg << (8 * g);
    }
    return exact ? keep : keep_mask<8>(v, 4);
}

// Step d = RN32(value(code) s_t) and, for d in [2^-90, 2^90], y = RN(1/d)
// and the bracketing factors RN(y (1 -/+ 2^-21)) of e2m1x8_div (else all
// three 0) of every UE4M3 scale code: one table per CTA, so that a block's
// step and reciprocals are one shared-memory load instead of a conversion,
// a product and a correctly rounded reciprocal per block.
template <int FMT>
__device__ __forceinline__ void build_step_table(float4 *tab, float s_t) {
    if constexpr (FMT == kFmtNV)
        for (int c = threadIdx.x; c < 128; c += blockDim.x) {
            const float d = __fmul_rn(ue4m3_value((uint32_t)c), s_t);
            const float y = (d >= 0x1p-90f && d <= 0x1p90f) ? __frcp_rn(d) : 0.0f;
            tab[c] = make_float4(d, y, __fmul_rn(y, 1.0f - 0x1p-21f), __fmul_rn(y, 1.0f + 0x1p-21f));
        }
}

// Nibble mask of eight keep bits (bit i of k sets nibble i to 0xF): three
// spreading steps whose shifted copies never overlap, so each multiply is
// an OR of shifts.
__device__ __forceinline__ uint32_t nibble_mask8(uint32_t k) {
    uint32_t x = ((k & 0xFFu) * 0x1001u) & 0x000F000Fu;  // bits 0-3 at 0-3, bits 4-7 at 16-19
    x = (x * 0x41u) & 0x03030303u;                        // two bits per byte
    x = (x * 0x9u) & 0x11111111u;                         // one bit per nibble
    return x * 0xFu;
}

// Block quantization of one thread's 16 values given the amax `a` of the
// whole block they belong to (this unit's 16, or the 32 / 64 values of a
// lane pair / quad).
template <int FMT>
__device__ __forceinline__ float quantize16_amax(const float (&v)[kUnit], float a, float s_t, float c6, float y6,
                                                 const float4 *tab, uint32_t &scale_code, uint32_t &codes_lo,
                                                 uint32_t &codes_hi);

template <int FMT>
__device__ __forceinline__ float quantize16(const float (&v)[kUnit], float s_t, float c6, float y6, const float4 *tab,
                                            uint32_t &scale_code, uint32_t &codes_lo, uint32_t &codes_hi) {
    float a = 0.0f;
#pragma unroll
    for (int i = 0; i < kUnit; ++i) a = fmaxf(a, fabsf(v[i]));
    if (FMT == kFmtMX) a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, 1));
    return quantize16_amax<FMT>(v, a, s_t, c6, y6, tab, scale_code, codes_lo, codes_hi);
}

template <int FMT>
__device__ __forceinline__ float quantize16_amax(const float (&v)[kUnit], float a, float s_t, float c6, float y6,
                                                 const float4 *tab, uint32_t &scale_code, uint32_t &codes_lo,
                                                 uint32_t &codes_hi) {
    // Step d and scale code as block_step gives them. NVFP4: the division
    // a / c6 by the reciprocal method when y6 = RN(1/c6) != 0 (the caller
    // sets y6 = 0 unless c6 is in [2^-90, 2^90]), exact for quotients >=
    // 2^-11, and every smaller quotient has UE4M3 code 0 either way (the
    // code's smallest rounding boundary is 2^-10); d, y = RN(1/d) and the
    // bracketing factors from the step table.
    float d, y = 0.0f, ylo = 0.0f, yhi = 0.0f;
    if (FMT == kFmtNV) {
        const float u = y6 != 0.0f ? div1(a, c6, y6) : __fdiv_rn(a, c6);
        scale_code = ue4m3_code(u);
        const float4 dy = tab[scale_code];
        d = dy.x;
        y = dy.y;
        ylo = dy.z;
        yhi = dy.w;
    } else {
        d = block_step<FMT>(a, s_t, c6, scale_code);
    }
    codes_lo = 0u;
    codes_hi = 0u;
    if (d != 0.0f) {
        // Two halves of eight values each, so that only four quotient pairs
        // are live at a time.
        uint32_t c[2];
        if (FMT == kFmtMX) {
            const float inv = pow2f(-mx_exponent(a));  // division by 2^e is this exact product
            const uint64_t y2 = pk2(inv, inv);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                uint64_t q[4];
#pragma unroll
                for (int p = 0; p < 4; ++p) q[p] = mul2(pk2(v[8 * h + 2 * p], v[8 * h + 2 * p + 1]), y2);
                c[h] = e2m1x8(q, v + 8 * h);
            }
        } else if (y != 0.0f) {
            const uint64_t y2 = pk2(y, y), nd2 = pk2(-d, -d), d2 = pk2(d, d);
#pragma unroll
            for (int h = 0; h < 2; ++h) c[h] = e2m1x8_div(v + 8 * h, pk2(ylo, ylo), pk2(yhi, yhi), d2, nd2, y2);
        } else {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                uint64_t q[4];
#pragma unroll
                for (int p = 0; p < 4; ++p)
                    q[p] = pk2(__fdiv_rn(v[8 * h + 2 * p], d), __fdiv_rn(v[8 * h + 2 * p + 1], d));
                c[h] = e2m1x8(q, v + 8 * h);
            }
        }
        codes_lo = c[0];
        codes_hi = c[1];
    }
    return d;
}

// The encode arithmetic of one unit of 16 LayerNorm outputs v: mask, Q(S),
// R = X_ln - deq(Q(S)), Q(R) and the mask metadata bits of the unit's
// groups (n kept positions per group, ascending, LSB-first).
struct UnitCodes {
    uint32_t s_lo, s_hi, r_lo, r_hi;  // E2M1 codes of S and R, eight per word
    uint32_t s_scale, r_scale;        // block scale codes
    uint64_t mbits;                   // metadata bits of the unit
};

template <int FMT, int M, int NK>
__device__ __forceinline__ void encode_core(const float (&v)[kUnit], int n, const uint32_t *lut, const float4 *tab,
                                            float s_t, float c6, float y6, UnitCodes &o) {
    constexpr int IB = M <= 2 ? 1 : M <= 4 ? 2 : M <= 8 ? 3 : 4;
    constexpr int G = kUnit / M;  // mask groups per unit
    const int gbits = n * IB;     // metadata bits per group
    // Mask, and Q(S) for the backbone S = X_ln on the mask, +0 elsewhere.
    // Every group keeps its largest magnitude (n >= 1), so the block amax
    // of S is that of X_ln (over the lane pair too, for MXFP4) and so are
    // the step and the codes on the mask: Q(S) is the encoding of X_ln with
    // the dropped positions' nibbles cleared to the +0 code of S's zeros.
    uint32_t keep;
    if constexpr (M == 4 && NK == 2)
        keep = keep_mask_42(v);
    else if constexpr (M == 8 && NK == 4)
        keep = keep_mask_84(v);
    else
        keep = keep_mask<M>(v, n);
    const float ds = quantize16<FMT>(v, s_t, c6, y6, tab, o.s_scale, o.s_lo, o.s_hi);
    o.s_lo &= nibble_mask8(keep);
    o.s_hi &= nibble_mask8(keep >> 8);

    // Residual against the quantized backbone: R = RN32(X_ln - RN32(value * d)).
    // Scalar intrinsics: the product must be rounded before the subtraction.
    float r[kUnit];
#pragma unroll
    for (int i = 0; i < kUnit; i += 2) {
        const uint32_t byte = ((i < 8 ? o.s_lo : o.s_hi) >> (4 * (i % 8))) & 0xFFu;
        const float2 cv = e2m1x2_value(byte);
        r[i] = __fsub_rn(v[i], __fmul_rn(cv.x, ds));
        r[i + 1] = __fsub_rn(v[i + 1], __fmul_rn(cv.y, ds));
    }
    quantize16<FMT>(r, s_t, c6, y6, tab, o.r_scale, o.r_lo, o.r_hi);

    // Mask metadata: each group holds exactly n kept positions, so its
    // field sits at a fixed offset of the unit's bit range.
    uint64_t mbits = 0;
    if constexpr (M == 4 && NK == 2) {
        // 2:4: a group's keep nibble has two bits set, so nibble >> 1 is one
        // of 1..6 and selects the group's field (first | second << 2) from
        // a byte table; one byte permute does all four groups, then the
        // four fields are packed into 16 bits.
        const uint32_t sel = (keep >> 1) & 0x7777u;
        const uint32_t w = __byte_perm(0x09080400u, 0x000E0D0Cu, sel);  // table: -, 4, 8, 9, 12, 13, 14, -
        const uint32_t t = w | (w >> 4);                                  // bytes 0 and 2 hold two fields each
        mbits = __byte_perm(t, 0u, 0x4420u);
    } else if (M <= 8) {
#pragma unroll
        for (int g = 0; g < G; ++g)
            mbits |= (uint64_t)lut[(keep >> (g * M)) & ((1u << M) - 1u)] << (g * gbits);
    } else {
        int pos = 0;
#pragma unroll
        for (int i = 0; i < M; ++i)
            if ((keep >> i) & 1u) {
                mbits |= (uint64_t)i << pos;
                pos += IB;
            }
    }
    o.mbits = mbits;
}

// ---------------------------------------------------------------------------
// Pair-wise 4:8 sparse-backbone mode. In every aligned group of 8 values
// along K (four adjacent pairs) the two pairs with the largest pair
// magnitude max(|a|, |b|) are kept, equal magnitudes going to the lower
// pair; the backbone's blocks are 32 values (NVFP4, a lane pair of units) or
// 64 (MXFP4, a lane quad), the blocks the structured-sparse block-scaled MMA
// applies; its kept codes are stored K-compacted (2 bytes per group) beside
// 4 metadata bits per group (first kept pair | second << 2). The residual is
// as in the default mode.

// Bit j set: pair j is among the two largest keys (equal keys: lower pair
// first). The majority logic of keep_mask_42 on four non-negative keys.
__device__ __forceinline__ uint32_t keep_pairs(float a0, float a1, float a2, float a3) {
    const uint32_t s01 = __float_as_uint(__fsub_rn(a0, a1)), s02 = __float_as_uint(__fsub_rn(a0, a2));
    const uint32_t s03 = __float_as_uint(__fsub_rn(a0, a3)), s12 = __float_as_uint(__fsub_rn(a1, a2));
    const uint32_t s13 = __float_as_uint(__fsub_rn(a1, a3)), s23 = __float_as_uint(__fsub_rn(a2, a3));
    const uint32_t k0 = ~((s01 & s02) | (s01 & s03) | (s02 & s03));
    const uint32_t k1 = (s01 & ~s12) | (s01 & ~s13) | (~s12 & ~s13);
    const uint32_t k2 = (s02 & s12) | (s02 & ~s23) | (s12 & ~s23);
    const uint32_t k3 = (s03 & s13) | (s03 & s23) | (s13 & s23);
    return (k0 >> 31) | (k1 >> 31) << 1 | (k2 >> 31) << 2 | (k3 >> 31) << 3;
}

// 0xFF in byte j for every set bit j of a 4-bit mask (the four shifted
// copies never overlap).
__device__ __forceinline__ uint32_t pair_bytes(uint32_t n4) {
    return ((n4 * 0x00204081u) & 0x01010101u) * 0xFFu;
}

struct SparseUnitCodes {
    uint32_t s_comp;        // kept backbone codes, K-compacted (8 codes)
    uint32_t s_scale;       // backbone block scale code (of the lane pair / quad)
    uint32_t r_lo, r_hi;    // residual codes
    uint32_t r_scale;       // residual block scale code
    uint32_t meta;          // metadata byte: group 0 in bits 0-3, group 1 in bits 4-7
};

template <int FMT>
__device__ __forceinline__ void encode_core_sparse(const float (&v)[kUnit], const float4 *tab, float s_t, float c6,
                                                   float y6, SparseUnitCodes &o) {
    uint32_t pk = 0;  // kept pairs: 4 bits per group
#pragma unroll
    for (int g = 0; g < 2; ++g) {
        float key[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) key[j] = fmaxf(fabsf(v[8 * g + 2 * j]), fabsf(v[8 * g + 2 * j + 1]));
        pk |= keep_pairs(key[0], key[1], key[2], key[3]) << (4 * g);
    }
    // Every group keeps its largest magnitude, so the backbone block's amax
    // is that of X_ln over the block's units, and so are the step and the
    // kept codes: the codes of X_ln itself, the dropped pairs cleared.
    float a = 0.0f;
#pragma unroll
    for (int i = 0; i < kUnit; ++i) a = fmaxf(a, fabsf(v[i]));
    a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, 1));
    if (FMT == kFmtMX) a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, 2));
    uint32_t c0, c1;
    const float ds = quantize16_amax<FMT>(v, a, s_t, c6, y6, tab, o.s_scale, c0, c1);
    // A group's kept-pair nibble has two bits set, so nibble >> 1 (1..6)
    // indexes byte tables: the metadata field (first | second << 2) and the
    // byte selector (first | second << 4) of the group's kept code bytes.
    const uint32_t sel2 = (pk >> 1) & 0x77u;
    const uint32_t mt = __byte_perm(0x09080400u, 0x000E0D0Cu, sel2);  // -, 4, 8, 9, 12, 13, 14, -
    o.meta = (mt & 0xFu) | ((mt >> 4) & 0xF0u);
    const uint32_t ct = __byte_perm(0x21201000u, 0x00323130u, sel2);  // -, 10, 20, 21, 30, 31, 32, - (hex)
    o.s_comp = __byte_perm(c0, c1, ct + 0x4400u);                      // group 1's bytes are 4..7
    c0 &= pair_bytes(pk & 0xFu);
    c1 &= pair_bytes(pk >> 4);
    // Residual against the quantized backbone, as in the default mode.
    float r[kUnit];
#pragma unroll
    for (int i = 0; i < kUnit; i += 2) {
        const uint32_t byte = ((i < 8 ? c0 : c1) >> (4 * (i % 8))) & 0xFFu;
        const float2 cv = e2m1x2_value(byte);
        r[i] = __fsub_rn(v[i], __fmul_rn(cv.x, ds));
        r[i + 1] = __fsub_rn(v[i + 1], __fmul_rn(cv.y, ds));
    }
    quantize16<FMT>(r, s_t, c6, y6, tab, o.r_scale, o.r_lo, o.r_hi);
}

// Arguments of the encode step (one unit = 16 consecutive elements of a row).
struct EncodeArgs {
    const uint16_t *x, *gamma, *beta;
    const float2 *stats;
    int64_t m_tok, k, meta_row, nblk;
    int n;
    uint8_t *s_codes, *r_codes, *s_sf, *r_sf, *meta;
};

// Encode step of unit u of row `row`: LayerNorm apply, mask, Q(S), R, Q(R),
// stores. `active` lanes with row >= m_tok (or row < 0) are padding: zero
// scales, and with pad_codes also zero codes and metadata; inactive lanes
// only take part in the MXFP4 lane-pair exchanges. The outputs go to row
// `dst` (-1: the same row).
// NK > 0: n fixed at compile time (the 2:4 default takes its own mask).
template <int FMT, int M, int NK>
__device__ __forceinline__ void encode_unit(const EncodeArgs &a, const uint32_t *lut, const float4 *tab, int64_t row,
                                            int64_t u, bool active, float s_t, float c6, float y6, int64_t dst = -1,
                                            bool pad_codes = false) {
    constexpr int IB = M <= 2 ? 1 : M <= 4 ? 2 : M <= 8 ? 3 : 4;
    constexpr int G = kUnit / M;  // mask groups per unit
    const uint16_t *__restrict__ x = a.x;
    const uint16_t *__restrict__ gamma = a.gamma;
    const uint16_t *__restrict__ beta = a.beta;
    const float2 *__restrict__ stats = a.stats;
    const int64_t m_tok = a.m_tok, k = a.k, meta_row = a.meta_row, nblk = a.nblk;
    const int n = NK > 0 ? NK : a.n;
    uint8_t *__restrict__ s_codes = a.s_codes;
    uint8_t *__restrict__ r_codes = a.r_codes;
    uint8_t *__restrict__ s_sf = a.s_sf;
    uint8_t *__restrict__ r_sf = a.r_sf;
    uint8_t *__restrict__ meta = a.meta;
    const int gbits = n * IB;  // metadata bits per group
    const int B = G * gbits;   // metadata bits per unit
    const bool byte_aligned = (B & 7) == 0;
    const bool has_g = gamma != nullptr, has_b = beta != nullptr;
    const bool real = active && row >= 0 && row < m_tok;
    const int64_t orow = dst >= 0 ? dst : row;  // output row

    // LayerNorm apply on the unit's 16 values (zeros on idle lanes, which
    // still take part in the MXFP4 lane-pair exchanges).
    float v[kUnit];
    {
        uint4 xa = make_uint4(0, 0, 0, 0), xb = xa, ga = xa, gb = xa, ba = xa, bb = xa;
        float2 st = make_float2(0.0f, 1.0f);
        if (real) {
            const uint4 *xp = reinterpret_cast<const uint4 *>(x + row * k + u * kUnit);
            xa = __ldcs(xp);
            xb = __ldcs(xp + 1);
            st = stats[row];
            if (has_g) {
                ga = __ldg(reinterpret_cast<const uint4 *>(gamma + u * kUnit));
                gb = __ldg(reinterpret_cast<const uint4 *>(gamma + u * kUnit) + 1);
            }
            if (has_b) {
                ba = __ldg(reinterpret_cast<const uint4 *>(beta + u * kUnit));
                bb = __ldg(reinterpret_cast<const uint4 *>(beta + u * kUnit) + 1);
            }
        }
        const uint32_t xw[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
        const uint32_t gw[8] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w};
        const uint32_t bw[8] = {ba.x, ba.y, ba.z, ba.w, bb.x, bb.y, bb.z, bb.w};
        // (x - mu) * rstd in packed pairs (no multiply feeds an add here);
        // gamma and beta with scalar intrinsics, which the compiler never
        // fuses into a multiply-add (a packed multiply followed by a packed
        // add may be fused, which would skip the rounding of the product).
        const uint64_t mu2 = pk2(st.x, st.x), rs2 = pk2(st.y, st.y);
#pragma unroll
        for (int p = 0; p < 8; ++p) {
            float2 f = up2(mul2(sub2(h2_to_f2(xw[p]), mu2), rs2));
            if (has_g) {
                f.x = __fmul_rn(f.x, h2f((uint16_t)gw[p]));
                f.y = __fmul_rn(f.y, h2f((uint16_t)(gw[p] >> 16)));
            }
            if (has_b) {
                f.x = __fadd_rn(f.x, h2f((uint16_t)bw[p]));
                f.y = __fadd_rn(f.y, h2f((uint16_t)(bw[p] >> 16)));
            }
            v[2 * p] = f.x;
            v[2 * p + 1] = f.y;
        }
    }

    UnitCodes o;
    encode_core<FMT, M, NK>(v, n, lut, tab, s_t, c6, y6, o);
    const uint32_t s_lo = o.s_lo, s_hi = o.s_hi, r_lo = o.r_lo, r_hi = o.r_hi;
    const uint32_t s_scale = o.s_scale, r_scale = o.r_scale;
    const uint64_t mbits = o.mbits;

    if (real) {
        *reinterpret_cast<uint2 *>(s_codes + orow * (k / 2) + u * 8) = make_uint2(s_lo, s_hi);
        *reinterpret_cast<uint2 *>(r_codes + orow * (k / 2) + u * 8) = make_uint2(r_lo, r_hi);
        if (FMT == kFmtNV) {
            s_sf[sf_offset(orow, u, nblk)] = (uint8_t)s_scale;
            r_sf[sf_offset(orow, u, nblk)] = (uint8_t)r_scale;
        } else if ((u & 1) == 0) {
            s_sf[sf_offset(orow, u >> 1, nblk)] = (uint8_t)s_scale;
            r_sf[sf_offset(orow, u >> 1, nblk)] = (uint8_t)r_scale;
        }
        if (byte_aligned)
            store_bytes(meta + orow * meta_row + u * (B / 8), mbits, B / 8);
        else
            or_bits(reinterpret_cast<uint32_t *>(meta), (uint64_t)orow * meta_row * 8 + (uint64_t)u * B, mbits, B);
    } else if (active) {  // padding rows: zero scales (and codes and metadata where asked)
        if (FMT == kFmtNV) {
            s_sf[sf_offset(orow, u, nblk)] = 0;
            r_sf[sf_offset(orow, u, nblk)] = 0;
        } else if ((u & 1) == 0) {
            s_sf[sf_offset(orow, u >> 1, nblk)] = 0;
            r_sf[sf_offset(orow, u >> 1, nblk)] = 0;
        }
        if (pad_codes) {
            *reinterpret_cast<uint2 *>(s_codes + orow * (k / 2) + u * 8) = make_uint2(0u, 0u);
            *reinterpret_cast<uint2 *>(r_codes + orow * (k / 2) + u * 8) = make_uint2(0u, 0u);
            if (byte_aligned) store_bytes(meta + orow * meta_row + u * (B / 8), 0ull, B / 8);
            // (unaligned metadata fields are OR-ed into a stream zeroed beforehand)
        }
    }
}

template <int FMT, int M, int NK>
__global__ void __launch_bounds__(kEncodeThreads, SQ_ENCODE_MIN_CTAS)
prep_encode_kernel(const uint16_t *__restrict__ x, const uint16_t *__restrict__ gamma,
                   const uint16_t *__restrict__ beta, const float2 *__restrict__ stats,
                   const unsigned *__restrict__ amax_word, float *__restrict__ s_t_out, int64_t m_tok,
                   int64_t sf_rows, int64_t k, int n, uint8_t *__restrict__ s_codes, uint8_t *__restrict__ r_codes,
                   uint8_t *__restrict__ s_sf, uint8_t *__restrict__ r_sf, uint8_t *__restrict__ meta,
                   int64_t meta_row) {
    constexpr int IB = M <= 2 ? 1 : M <= 4 ? 2 : M <= 8 ? 3 : 4;
    __shared__ uint32_t lut[M <= 8 ? (1 << M) : 1];  // keep bits of a group -> kept positions, ascending
    if (M <= 8) {
        for (int msk = threadIdx.x; msk < (1 << M); msk += kEncodeThreads) {
            uint32_t packed = 0;
            int pos = 0;
            for (int i = 0; i < M; ++i)
                if ((msk >> i) & 1) {
                    packed |= (uint32_t)i << pos;
                    pos += IB;
                }
            lut[msk] = packed;
        }
        __syncthreads();
    }

    const float amax = __uint_as_float(*amax_word);
    const float s_t = (FMT == kFmtNV && amax != 0.0f) ? __fdiv_rn(amax, 2688.0f) : 1.0f;
    const float c6 = __fmul_rn(6.0f, s_t);
    const float y6 = (FMT == kFmtNV && c6 >= 0x1p-90f && c6 <= 0x1p90f) ? __frcp_rn(c6) : 0.0f;
    if (blockIdx.x == 0 && threadIdx.x == 0) *s_t_out = s_t;
    __shared__ float4 tab[128];  // NVFP4 steps and reciprocals by scale code
    build_step_table<FMT>(tab, s_t);
    __syncthreads();

    const int64_t upr = k / kUnit;                 // units per row
    const int64_t nblk = k / (FMT == kFmtNV ? 16 : 32);
    const int64_t total = sf_rows * upr;
    const int64_t stride = (int64_t)gridDim.x * kEncodeThreads;

    // (row, unit) of this thread's first unit, then stepped by the grid
    // stride without dividing again.
    const int64_t t0 = (int64_t)blockIdx.x * kEncodeThreads + threadIdx.x;
    int64_t row_i = t0 / upr, u_i = t0 - (t0 / upr) * upr;
    const int64_t step_rows = stride / upr, step_units = stride - (stride / upr) * upr;
    EncodeArgs ea{x, gamma, beta, stats, m_tok, k, meta_row, nblk, n, s_codes, r_codes, s_sf, r_sf, meta};
    for (int64_t base = (int64_t)blockIdx.x * kEncodeThreads; base < total; base += stride) {
        const int64_t t = base + threadIdx.x;
        const bool active = t < total;
        const int64_t row = row_i, u = u_i;
        row_i += step_rows;
        u_i += step_units;
        if (u_i >= upr) {
            u_i -= upr;
            ++row_i;
        }
        encode_unit<FMT, M, NK>(ea, lut, tab, row, u, active, s_t, c6, y6);
    }
}

// LayerNorm apply on one unit's 16 values (x as eight fp16 pairs): (x - mu)
// * rstd in packed pairs (no multiply feeds an add there), then gamma and
// beta (AFFINE; either may be NULL) with scalar intrinsics, which are never
// fused into a multiply-add.
template <bool AFFINE>
__device__ __forceinline__ void ln_apply16(const uint32_t (&xw)[8], float2 st, const uint16_t *gamma,
                                           const uint16_t *beta, int u, bool act, float (&v)[kUnit]) {
    const uint64_t mu2 = pk2(st.x, st.x), rs2 = pk2(st.y, st.y);
    uint4 ga = make_uint4(0, 0, 0, 0), gb = ga, ba = ga, bb = ga;
    if (AFFINE && act) {
        if (gamma) {
            ga = __ldg(reinterpret_cast<const uint4 *>(gamma + (int64_t)u * kUnit));
            gb = __ldg(reinterpret_cast<const uint4 *>(gamma + (int64_t)u * kUnit) + 1);
        }
        if (beta) {
            ba = __ldg(reinterpret_cast<const uint4 *>(beta + (int64_t)u * kUnit));
            bb = __ldg(reinterpret_cast<const uint4 *>(beta + (int64_t)u * kUnit) + 1);
        }
    }
    const uint32_t gw8[8] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w};
    const uint32_t bw8[8] = {ba.x, ba.y, ba.z, ba.w, bb.x, bb.y, bb.z, bb.w};
#pragma unroll
    for (int p = 0; p < 8; ++p) {
        float2 f = up2(mul2(sub2(h2_to_f2(xw[p]), mu2), rs2));
        if (AFFINE) {
            if (gamma) {
                f.x = __fmul_rn(f.x, h2f((uint16_t)gw8[p]));
                f.y = __fmul_rn(f.y, h2f((uint16_t)(gw8[p] >> 16)));
            }
            if (beta) {
                f.x = __fadd_rn(f.x, h2f((uint16_t)bw8[p]));
                f.y = __fadd_rn(f.y, h2f((uint16_t)(bw8[p] >> 16)));
            }
        }
        v[2 * p] = f.x;
        v[2 * p + 1] = f.y;
    }
}

// Encode pass over the rows of one activation: one warp per 512-element
// chunk of a row (a lane per 16-element unit), the chunks of the persistent
// grid's warps taken in reverse row order. The statistics pass reads the rows
// in increasing order, so the rows it read last (still in L2 when x is
// larger than L2) are the ones this pass reads first. Per chunk: one 32-byte
// load per lane, the row's statistics once, and addresses from per-row bases.
// The next chunk's loads are issued before the current chunk is encoded.
// Padding rows of the scale layouts (m_tok .. sf_rows - 1) are zeroed after
// the main loop. Launched with programmatic stream serialization: the look-up
// tables are built before griddep_wait, everything the statistics pass wrote
// is read after it.
template <int FMT, int M, int NK, bool AFFINE>
__global__ void __launch_bounds__(kEncodeThreads, SQ_ENCODE_MIN_CTAS)
prep_encode_rows_kernel(const EncodeArgs a, const unsigned *amax_word, float *__restrict__ s_t_out,
                        int64_t sf_rows) {
    constexpr int IB = M <= 2 ? 1 : M <= 4 ? 2 : M <= 8 ? 3 : 4;
    __shared__ uint32_t lut[M <= 8 ? (1 << M) : 1];  // keep bits of a group -> kept positions, ascending
    __shared__ float4 tab[128];                       // NVFP4 steps and reciprocals by scale code
    if (M <= 8)
        for (int msk = threadIdx.x; msk < (1 << M); msk += kEncodeThreads) {
            uint32_t packed = 0;
            int pos = 0;
            for (int i = 0; i < M; ++i)
                if ((msk >> i) & 1) {
                    packed |= (uint32_t)i << pos;
                    pos += IB;
                }
            lut[msk] = packed;
        }
    griddep_wait();  // the statistics and the amax word are complete
    griddep_launch();
    // What the statistics kernel wrote is read with L2 loads through pointers
    // without __restrict__, so that no load can move above the wait.
    const float amax = __uint_as_float(__ldcg(amax_word));
    const float s_t = (FMT == kFmtNV && amax != 0.0f) ? __fdiv_rn(amax, 2688.0f) : 1.0f;
    const float c6 = __fmul_rn(6.0f, s_t);
    const float y6 = (FMT == kFmtNV && c6 >= 0x1p-90f && c6 <= 0x1p90f) ? __frcp_rn(c6) : 0.0f;
    if (blockIdx.x == 0 && threadIdx.x == 0) *s_t_out = s_t;
    build_step_table<FMT>(tab, s_t);
    __syncthreads();

    const uint16_t *__restrict__ x = a.x;
    const float2 *stats = a.stats;
    uint8_t *__restrict__ s_codes = a.s_codes;
    uint8_t *__restrict__ r_codes = a.r_codes;
    uint8_t *__restrict__ s_sf = a.s_sf;
    uint8_t *__restrict__ r_sf = a.r_sf;
    uint8_t *__restrict__ meta = a.meta;
    const int64_t k = a.k, m_tok = a.m_tok, nblk = a.nblk, meta_row = a.meta_row;
    const int n = NK > 0 ? NK : a.n;
    const int B = (kUnit / M) * n * IB;  // metadata bits per unit
    const bool byte_aligned = (B & 7) == 0;
    const int lane = threadIdx.x & 31;
    const int upr = (int)(k / kUnit);         // units per row
    const int chunks = (upr + 31) >> 5;       // 32-unit chunks per row
    const int64_t nwarps = (int64_t)gridDim.x * (kEncodeThreads / 32);
    const int64_t gw = (int64_t)blockIdx.x * (kEncodeThreads / 32) + threadIdx.x / 32;
    const int64_t items = m_tok * chunks;
    const int64_t step_r = nwarps / chunks;
    const int step_c = (int)(nwarps - step_r * chunks);

    // Item `it` is chunk it % chunks of row m_tok - 1 - it / chunks.
    int64_t ri = gw / chunks;
    int ci = (int)(gw - ri * chunks);
    uint32_t xw[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    float2 st = make_float2(0.0f, 1.0f);
    // one 32-byte load where x is 32-byte aligned (every unit then is), else two
    const bool x32 = (reinterpret_cast<uintptr_t>(x) & 31u) == 0;
    auto fetch = [&](int64_t r, int c, uint32_t (&w)[8], float2 &sv) {
        const int u = c * 32 + lane;
        if (u < upr) {
            const uint16_t *p = x + r * k + (int64_t)u * kUnit;
            if (x32) {
                ldg256_cs(p, w);
            } else {
                const uint4 va = __ldcs(reinterpret_cast<const uint4 *>(p)), vb = __ldcs(reinterpret_cast<const uint4 *>(p) + 1);
                w[0] = va.x, w[1] = va.y, w[2] = va.z, w[3] = va.w, w[4] = vb.x, w[5] = vb.y, w[6] = vb.z, w[7] = vb.w;
            }
        }
        sv = __ldcg(stats + r);
    };
    if (gw < items) fetch(m_tok - 1 - ri, ci, xw, st);
    for (int64_t it = gw; it < items; it += nwarps) {
        const int64_t row = m_tok - 1 - ri;
        const int u = ci * 32 + lane;
        const bool act = u < upr;
        ri += step_r;
        ci += step_c;
        if (ci >= chunks) {
            ci -= chunks;
            ++ri;
        }
        // the next chunk's loads go out before this chunk is encoded
        uint32_t nw[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        float2 nst = make_float2(0.0f, 1.0f);
        if (it + nwarps < items) fetch(m_tok - 1 - ri, ci, nw, nst);

        float v[kUnit];
        ln_apply16<AFFINE>(xw, st, a.gamma, a.beta, u, act, v);
        UnitCodes o;
        encode_core<FMT, M, NK>(v, n, lut, tab, s_t, c6, y6, o);
        if (act) {
            const int64_t cofs = row * (k / 2) + (int64_t)u * 8;
            *reinterpret_cast<uint2 *>(s_codes + cofs) = make_uint2(o.s_lo, o.s_hi);
            *reinterpret_cast<uint2 *>(r_codes + cofs) = make_uint2(o.r_lo, o.r_hi);
            if (FMT == kFmtNV) {
                const int64_t so = sf_offset(row, u, nblk);
                s_sf[so] = (uint8_t)o.s_scale;
                r_sf[so] = (uint8_t)o.r_scale;
            } else if ((u & 1) == 0) {
                const int64_t so = sf_offset(row, u >> 1, nblk);
                s_sf[so] = (uint8_t)o.s_scale;
                r_sf[so] = (uint8_t)o.r_scale;
            }
            if constexpr (M == 4 && NK == 2)  // 16 bits per unit; rows are k / 8 bytes, so 2-byte aligned
                *reinterpret_cast<uint16_t *>(meta + row * meta_row + (int64_t)u * 2) = (uint16_t)o.mbits;
            else if (byte_aligned)
                store_bytes(meta + row * meta_row + (int64_t)u * (B / 8), o.mbits, B / 8);
            else
                or_bits(reinterpret_cast<uint32_t *>(meta), (uint64_t)row * meta_row * 8 + (uint64_t)u * B, o.mbits, B);
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) xw[i] = nw[i];
        st = nst;
    }
    // Zero scales of the padding rows of the last 128-row scale atoms.
    const int64_t pad = (sf_rows - m_tok) * nblk;
    const int64_t gthreads = (int64_t)gridDim.x * kEncodeThreads;
    for (int64_t i = (int64_t)blockIdx.x * kEncodeThreads + threadIdx.x; i < pad; i += gthreads) {
        const int64_t r = m_tok + i / nblk, j = i - (i / nblk) * nblk;
        s_sf[sf_offset(r, j, nblk)] = 0;
        r_sf[sf_offset(r, j, nblk)] = 0;
    }
}

// Encode pass of the pair-wise 4:8 mode: the walk of prep_encode_rows_kernel
// (a warp per 512-element row chunk, reverse row order, next chunk
// prefetched, launched as a programmatic dependent of the statistics pass),
// with the backbone stored K-compacted (4 bytes per unit), its block scale
// once per lane pair (NVFP4, 32 values) or quad (MXFP4, 64 values) and one
// metadata byte per unit.
template <int FMT, bool AFFINE>
__global__ void __launch_bounds__(kEncodeThreads, SQ_ENCODE_MIN_CTAS)
prep_encode_sparse_kernel(const EncodeArgs a, const unsigned *amax_word, float *__restrict__ s_t_out,
                          int64_t sf_rows) {
    __shared__ float4 tab[128];  // NVFP4 steps and reciprocals by scale code
    griddep_wait();  // the statistics and the amax word are complete
    griddep_launch();
    // (read with L2 loads through pointers without __restrict__, so that no
    // load can move above the wait)
    const float amax = __uint_as_float(__ldcg(amax_word));
    const float s_t = (FMT == kFmtNV && amax != 0.0f) ? __fdiv_rn(amax, 2688.0f) : 1.0f;
    const float c6 = __fmul_rn(6.0f, s_t);
    const float y6 = (FMT == kFmtNV && c6 >= 0x1p-90f && c6 <= 0x1p90f) ? __frcp_rn(c6) : 0.0f;
    if (blockIdx.x == 0 && threadIdx.x == 0) *s_t_out = s_t;
    build_step_table<FMT>(tab, s_t);
    __syncthreads();

    const uint16_t *__restrict__ x = a.x;
    const float2 *stats = a.stats;
    uint8_t *__restrict__ s_codes = a.s_codes;
    uint8_t *__restrict__ r_codes = a.r_codes;
    uint8_t *__restrict__ s_sf = a.s_sf;
    uint8_t *__restrict__ r_sf = a.r_sf;
    uint8_t *__restrict__ meta = a.meta;
    const int64_t k = a.k, m_tok = a.m_tok;
    const int64_t nblk_r = k / (FMT == kFmtNV ? 16 : 32), nblk_s = nblk_r / 2;
    const int lane = threadIdx.x & 31;
    const int upr = (int)(k / kUnit);
    const int chunks = (upr + 31) >> 5;
    const int64_t nwarps = (int64_t)gridDim.x * (kEncodeThreads / 32);
    const int64_t gw = (int64_t)blockIdx.x * (kEncodeThreads / 32) + threadIdx.x / 32;
    const int64_t items = m_tok * chunks;
    const int64_t step_r = nwarps / chunks;
    const int step_c = (int)(nwarps - step_r * chunks);
    int64_t ri = gw / chunks;
    int ci = (int)(gw - ri * chunks);
    uint32_t xw[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    float2 st = make_float2(0.0f, 1.0f);
    const bool x32 = (reinterpret_cast<uintptr_t>(x) & 31u) == 0;
    auto fetch = [&](int64_t r, int c, uint32_t (&w)[8], float2 &sv) {
        const int u = c * 32 + lane;
        if (u < upr) {
            const uint16_t *p = x + r * k + (int64_t)u * kUnit;
            if (x32) {
                ldg256_cs(p, w);
            } else {
                const uint4 va = __ldcs(reinterpret_cast<const uint4 *>(p)), vb = __ldcs(reinterpret_cast<const uint4 *>(p) + 1);
                w[0] = va.x, w[1] = va.y, w[2] = va.z, w[3] = va.w, w[4] = vb.x, w[5] = vb.y, w[6] = vb.z, w[7] = vb.w;
            }
        }
        sv = __ldcg(stats + r);
    };
    if (gw < items) fetch(m_tok - 1 - ri, ci, xw, st);
    for (int64_t it = gw; it < items; it += nwarps) {
        const int64_t row = m_tok - 1 - ri;
        const int u = ci * 32 + lane;
        const bool act = u < upr;
        ri += step_r;
        ci += step_c;
        if (ci >= chunks) {
            ci -= chunks;
            ++ri;
        }
        uint32_t nw[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        float2 nst = make_float2(0.0f, 1.0f);
        if (it + nwarps < items) fetch(m_tok - 1 - ri, ci, nw, nst);

        float v[kUnit];
        ln_apply16<AFFINE>(xw, st, a.gamma, a.beta, u, act, v);
        SparseUnitCodes o;
        encode_core_sparse<FMT>(v, tab, s_t, c6, y6, o);
        if (act) {
            *reinterpret_cast<uint32_t *>(s_codes + row * (k / 4) + (int64_t)u * 4) = o.s_comp;
            *reinterpret_cast<uint2 *>(r_codes + row * (k / 2) + (int64_t)u * 8) = make_uint2(o.r_lo, o.r_hi);
            meta[row * (k / 16) + u] = (uint8_t)o.meta;
            if (FMT == kFmtNV) {
                r_sf[sf_offset(row, u, nblk_r)] = (uint8_t)o.r_scale;
                if ((u & 1) == 0) s_sf[sf_offset(row, u >> 1, nblk_s)] = (uint8_t)o.s_scale;
            } else {
                if ((u & 1) == 0) r_sf[sf_offset(row, u >> 1, nblk_r)] = (uint8_t)o.r_scale;
                if ((u & 3) == 0) s_sf[sf_offset(row, u >> 2, nblk_s)] = (uint8_t)o.s_scale;
            }
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) xw[i] = nw[i];
        st = nst;
    }
    // Zero scales of the padding rows of the last 128-row scale atoms.
    const int64_t gthreads = (int64_t)gridDim.x * kEncodeThreads;
    const int64_t t0 = (int64_t)blockIdx.x * kEncodeThreads + threadIdx.x;
    for (int64_t i = t0; i < (sf_rows - m_tok) * nblk_r; i += gthreads)
        r_sf[sf_offset(m_tok + i / nblk_r, i % nblk_r, nblk_r)] = 0;
    for (int64_t i = t0; i < (sf_rows - m_tok) * nblk_s; i += gthreads)
        s_sf[sf_offset(m_tok + i / nblk_s, i % nblk_s, nblk_s)] = 0;
}

constexpr int kGroupedTileTable = 4096;  // tiles whose group the grouped encode tabulates in shared memory

// Encode pass straight into the expert-grouped layout (the layout of
// sharq_gather_rows): source rows in grouped order, group g's rows placed
// from row 128 T_g on (T_g: 128-row tiles of the groups before g), every
// other row zero. Warp 0 builds the groups' tile table from the device
// offsets; invalid offsets record the status and leave the outputs alone.
template <int FMT, int M, int NK>
__global__ void __launch_bounds__(kEncodeThreads, SQ_ENCODE_MIN_CTAS)
prep_encode_grouped_kernel(const EncodeArgs ea, const unsigned *__restrict__ amax_word, float *__restrict__ s_t_out,
                           int64_t cap_rows, const int32_t *__restrict__ offsets, int32_t groups, int64_t rows,
                           unsigned *status) {
    constexpr int IB = M <= 2 ? 1 : M <= 4 ? 2 : M <= 8 ? 3 : 4;
    __shared__ uint32_t lut[M <= 8 ? (1 << M) : 1];  // keep bits of a group -> kept positions, ascending
    __shared__ int32_t tiles[kGroupsMax + 1];
    __shared__ int16_t tile_group[kGroupedTileTable];  // group of each 128-row tile (small launches)
    __shared__ int table_ok;
    if (M <= 8) {
        for (int msk = threadIdx.x; msk < (1 << M); msk += kEncodeThreads) {
            uint32_t packed = 0;
            int pos = 0;
            for (int i = 0; i < M; ++i)
                if ((msk >> i) & 1) {
                    packed |= (uint32_t)i << pos;
                    pos += IB;
                }
            lut[msk] = packed;
        }
    }
    if (threadIdx.x / 32 == 0) {
        const bool ok = build_tile_table(offsets, groups, rows, cap_rows, tiles);
        if (threadIdx.x == 0) table_ok = ok ? 1 : 0;
    }
    __syncthreads();
    if (!table_ok) {
        if (blockIdx.x == 0 && threadIdx.x == 0) record_status(status, kSiteBadOffsets);
        return;
    }
    // Group of every used tile, once per CTA, when the tiles are few enough.
    const int32_t used_tiles = tiles[groups];
    const bool small_table = used_tiles <= kGroupedTileTable;
    if (small_table)
        for (int32_t t = threadIdx.x; t < used_tiles; t += kEncodeThreads)
            tile_group[t] = (int16_t)group_of_tile(tiles, groups, t);
    __syncthreads();
    const float amax = __uint_as_float(*amax_word);
    const float s_t = (FMT == kFmtNV && amax != 0.0f) ? __fdiv_rn(amax, 2688.0f) : 1.0f;
    const float c6 = __fmul_rn(6.0f, s_t);
    const float y6 = (FMT == kFmtNV && c6 >= 0x1p-90f && c6 <= 0x1p90f) ? __frcp_rn(c6) : 0.0f;
    if (blockIdx.x == 0 && threadIdx.x == 0) *s_t_out = s_t;
    __shared__ float4 tab[128];  // NVFP4 steps and reciprocals by scale code
    build_step_table<FMT>(tab, s_t);
    __syncthreads();
    constexpr int IBm = M <= 2 ? 1 : M <= 4 ? 2 : M <= 8 ? 3 : 4;
    const int unit_meta_bits = (kUnit / M) * ea.n * IBm;

    const int64_t upr = ea.k / kUnit;  // units per row
    const int64_t total = cap_rows * upr;
    const int64_t stride = (int64_t)gridDim.x * kEncodeThreads;
    const int64_t t0 = (int64_t)blockIdx.x * kEncodeThreads + threadIdx.x;
    int64_t row_i = t0 / upr, u_i = t0 - (t0 / upr) * upr;
    const int64_t step_rows = stride / upr, step_units = stride - (stride / upr) * upr;
    for (int64_t base = (int64_t)blockIdx.x * kEncodeThreads; base < total; base += stride) {
        const int64_t t = base + threadIdx.x;
        const bool active = t < total;
        const int64_t d = row_i, u = u_i;
        row_i += step_rows;
        u_i += step_units;
        if (u_i >= upr) {
            u_i -= upr;
            ++row_i;
        }
        int64_t src = -1;
        if (active) {
            const int32_t tile = (int32_t)(d >> 7);
            if (tile < used_tiles) {
                const int g = small_table ? (int)tile_group[tile] : group_of_tile(tiles, groups, tile);
                const int64_t local = d - 128 * (int64_t)tiles[g];
                if (local < (int64_t)offsets[g + 1] - offsets[g]) src = offsets[g] + local;
            }
        }
        if (FMT == kFmtNV && active && src < 0) {
            // A padding row: zeros, without the arithmetic (NVFP4 encodes
            // have no lane exchanges, so this lane may skip the unit).
            *reinterpret_cast<uint2 *>(ea.s_codes + d * (ea.k / 2) + u * 8) = make_uint2(0u, 0u);
            *reinterpret_cast<uint2 *>(ea.r_codes + d * (ea.k / 2) + u * 8) = make_uint2(0u, 0u);
            ea.s_sf[sf_offset(d, u, ea.nblk)] = 0;
            ea.r_sf[sf_offset(d, u, ea.nblk)] = 0;
            if ((unit_meta_bits & 7) == 0) store_bytes(ea.meta + d * ea.meta_row + u * (unit_meta_bits / 8), 0ull,
                                                       unit_meta_bits / 8);
            continue;
        }
        encode_unit<FMT, M, NK>(ea, lut, tab, src, u, active, s_t, c6, y6, d, true);
    }
}

// ---------------------------------------------------------------------------
// Few rows (decode): the whole preparation in one launch of one cluster.
// Phase 1: CTA r computes the exact statistics of rows r, r + kSmallCtas, ...
// (a whole CTA per row) and stores each row's amax|X_ln| into the shared
// memory of every CTA of the cluster, while the CTAs that own no row zero
// the scale layouts' padding rows (bytes no encode writes; where fields are
// OR-ed, every thread also zeroes the metadata). One cluster barrier makes
// the amaxes (and the zeroed metadata) visible everywhere; then every CTA
// derives the tensor scale from its own copy and encodes a share of the
// real rows' units. No CTA reads another's shared memory after the barrier, so none
// waits for the others at exit. No memset and no global atomic; the
// results equal the two-pass path bit for bit.
constexpr int kSmallCtas = 8, kSmallThreads = 512, kSmallMaxRows = 16, kSmallRows = 8;

template <int FMT, int M, bool RMS>
__global__ void __launch_bounds__(kSmallThreads)
prep_small_kernel(const EncodeArgs a, float eps, int64_t sf_rows, float *__restrict__ words, int meta_zero) {
    constexpr int IB = M <= 2 ? 1 : M <= 4 ? 2 : M <= 8 ? 3 : 4;
    constexpr int W = kSmallThreads / 32;
    __shared__ uint32_t lut[M <= 8 ? (1 << M) : 1];
    __shared__ float row_amax[kSmallMaxRows];
    __shared__ ExactSums red[W];
    __shared__ uint32_t red_mx[W], red_mn[W];
    __shared__ float red_max[W];
    __shared__ float2 row_stat;
    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
    const uint32_t rank = cluster_ctarank();
    cluster_arrive_relaxed();  // first half of the barrier before any remote store
    if (M <= 8)
        for (int msk = tid; msk < (1 << M); msk += kSmallThreads) {
            uint32_t packed = 0;
            int pos = 0;
            for (int i = 0; i < M; ++i)
                if ((msk >> i) & 1) {
                    packed |= (uint32_t)i << pos;
                    pos += IB;
                }
            lut[msk] = packed;
        }
    __syncthreads();
    // Launched as a programmatic dependent: everything above overlaps the
    // previous kernel's tail; global memory only after the wait.
    griddep_wait();
    griddep_launch();

    // Phase 1a: statistics (same sums, finish and amax rule as ln_stats_kernel).
    const int64_t k = a.k, m_tok = a.m_tok;
    const int nvec = (int)(k / 8);
    const bool affine = a.gamma != nullptr || a.beta != nullptr;
    for (int64_t row = rank; row < m_tok; row += kSmallCtas) {
        const uint4 *xr = reinterpret_cast<const uint4 *>(a.x + row * k);
        LaneSums l = {0, 0, 0.0, 0.0, 0.0};
        uint32_t mx = 0xFC00FC00u, mn = 0x7C007C00u;
        // Four loads in flight per thread before any is consumed: one
        // memory round trip per 4 x 512 vectors of the row.
        for (int c0 = tid; c0 < nvec; c0 += 4 * kSmallThreads) {
            uint4 v[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int c = c0 + j * kSmallThreads;
                v[j] = c < nvec ? xr[c] : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                if (c0 + j * kSmallThreads >= nvec) break;
                accum_pair(v[j].x, l);
                accum_pair(v[j].y, l);
                accum_pair(v[j].z, l);
                accum_pair(v[j].w, l);
                const uint32_t w4[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    asm("max.f16x2 %0, %0, %1;" : "+r"(mx) : "r"(w4[q]));
                    asm("min.f16x2 %0, %0, %1;" : "+r"(mn) : "r"(w4[q]));
                }
            }
        }
        ExactSums e = widen(l);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            e.hi += __shfl_xor_sync(0xFFFFFFFFu, e.hi, o);
            e.lo += __shfl_xor_sync(0xFFFFFFFFu, e.lo, o);
            e.hh += __shfl_xor_sync(0xFFFFFFFFu, e.hh, o);
            e.hl += __shfl_xor_sync(0xFFFFFFFFu, e.hl, o);
            e.ll += __shfl_xor_sync(0xFFFFFFFFu, e.ll, o);
            const uint32_t omx = __shfl_xor_sync(0xFFFFFFFFu, mx, o), omn = __shfl_xor_sync(0xFFFFFFFFu, mn, o);
            asm("max.f16x2 %0, %0, %1;" : "+r"(mx) : "r"(omx));
            asm("min.f16x2 %0, %0, %1;" : "+r"(mn) : "r"(omn));
        }
        if (lane == 0) {
            red[warp] = e;
            red_mx[warp] = mx;
            red_mn[warp] = mn;
        }
        __syncthreads();
        if (tid == 0) {
            ExactSums t = red[0];
            uint32_t tmx = red_mx[0], tmn = red_mn[0];
            for (int w = 1; w < W; ++w) {
                t.hi += red[w].hi;
                t.lo += red[w].lo;
                t.hh += red[w].hh;
                t.hl += red[w].hl;
                t.ll += red[w].ll;
                asm("max.f16x2 %0, %0, %1;" : "+r"(tmx) : "r"(red_mx[w]));
                asm("min.f16x2 %0, %0, %1;" : "+r"(tmn) : "r"(red_mn[w]));
            }
            const float2 st = RMS ? finish_stats_rms(t, k, eps) : finish_stats(t, k, eps);
            const_cast<float2 *>(a.stats)[row] = st;
            row_stat = st;
            if (!affine) {
                const float xmax = fmaxf(h2f((uint16_t)tmx), h2f((uint16_t)(tmx >> 16)));
                const float xmin = fminf(h2f((uint16_t)tmn), h2f((uint16_t)(tmn >> 16)));
                row_amax[row] = fmaxf(fabsf(__fmul_rn(__fsub_rn(xmax, st.x), st.y)),
                                      fabsf(__fmul_rn(__fsub_rn(xmin, st.x), st.y)));
            }
        }
        __syncthreads();
        if (affine) {
            const float mu = row_stat.x, rstd = row_stat.y;
            const bool has_g = a.gamma != nullptr, has_b = a.beta != nullptr;
            float amax = 0.0f;
            for (int c = tid; c < nvec; c += kSmallThreads) {
                const uint4 v = xr[c];
                const uint4 g = has_g ? __ldg(reinterpret_cast<const uint4 *>(a.gamma) + c) : make_uint4(0, 0, 0, 0);
                const uint4 bb = has_b ? __ldg(reinterpret_cast<const uint4 *>(a.beta) + c) : make_uint4(0, 0, 0, 0);
                const uint32_t xv[4] = {v.x, v.y, v.z, v.w}, gv[4] = {g.x, g.y, g.z, g.w}, bv[4] = {bb.x, bb.y, bb.z, bb.w};
#pragma unroll
                for (int q = 0; q < 4; ++q)
#pragma unroll
                    for (int h = 0; h < 2; ++h)
                        amax = fmaxf(amax, fabsf(ln_apply(h2f((uint16_t)(xv[q] >> (16 * h))), mu, rstd, has_g,
                                                          h2f((uint16_t)(gv[q] >> (16 * h))), has_b,
                                                          h2f((uint16_t)(bv[q] >> (16 * h))))));
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
            if (lane == 0) red_max[warp] = amax;
            __syncthreads();
            if (tid == 0) {
                float m = 0.0f;
                for (int w = 0; w < W; ++w) m = fmaxf(m, red_max[w]);
                row_amax[row] = m;
            }
        }
        __syncthreads();
    }

    // The scale layouts' padding rows (m_tok .. sf_rows - 1) read zero,
    // written by the CTAs that own no row where there are such (they would
    // otherwise wait at the barrier), else by all. Each 16-byte chunk holds
    // rows r0, r0 + 32, r0 + 64, r0 + 96 of a 128-row block (4 scales each);
    // only the padding rows' words are written, never bytes an encode writes.
    {
        const int64_t zctas = m_tok < kSmallCtas ? kSmallCtas - m_tok : kSmallCtas;
        const int64_t zrank = m_tok < kSmallCtas ? (int64_t)rank - m_tok : (int64_t)rank;
        const int64_t chunks = sf_rows * a.nblk / 16;
        if (zrank >= 0)
            for (int64_t c = zrank * kSmallThreads + tid; c < chunks; c += zctas * kSmallThreads) {
                const int64_t r0 = (c / (a.nblk / 4) / 32) * 128 + (c & 31);  // first row of the chunk
                if (r0 >= m_tok) {
                    reinterpret_cast<uint4 *>(a.s_sf)[c] = make_uint4(0, 0, 0, 0);
                    reinterpret_cast<uint4 *>(a.r_sf)[c] = make_uint4(0, 0, 0, 0);
                } else {
#pragma unroll
                    for (int q = 1; q < 4; ++q)
                        if (r0 + 32 * q >= m_tok) {
                            reinterpret_cast<uint32_t *>(a.s_sf)[4 * c + q] = 0u;
                            reinterpret_cast<uint32_t *>(a.r_sf)[4 * c + q] = 0u;
                        }
                }
            }
    }
    // Every CTA's copy of the owned rows' amax (remote stores, made visible
    // by the barrier below; the wait completes the barrier arrived at on
    // entry, so every CTA has started).
    cluster_wait();
    for (int i = tid; i < kSmallCtas * kSmallMaxRows; i += kSmallThreads) {
        const int c = i / kSmallMaxRows;
        const int64_t row = (int64_t)rank + (int64_t)(i % kSmallMaxRows) * kSmallCtas;  // an owned row
        if (row < m_tok)
            st_cluster_u32(mapa_shared(smem_u32(&row_amax[row]), (uint32_t)c), __float_as_uint(row_amax[row]));
    }
    const int64_t gtid = (int64_t)rank * kSmallThreads + tid, gstride = (int64_t)kSmallCtas * kSmallThreads;
    if (meta_zero)  // OR-ed fields: zeroed everywhere before any encode
        for (int64_t i = gtid; i < m_tok * a.meta_row; i += gstride) a.meta[i] = 0;
    cluster_sync();

    // Phase 2: the tensor scale from every row's amax, then the encode.
    float amax = 0.0f;
    for (int64_t row = 0; row < m_tok; ++row) amax = fmaxf(amax, row_amax[row]);
    const float s_t = (FMT == kFmtNV && amax != 0.0f) ? __fdiv_rn(amax, 2688.0f) : 1.0f;
    const float c6 = __fmul_rn(6.0f, s_t);
    const float y6 = (FMT == kFmtNV && c6 >= 0x1p-90f && c6 <= 0x1p90f) ? __frcp_rn(c6) : 0.0f;
    if (rank == 0 && tid == 0) {
        words[0] = amax;
        words[1] = s_t;
    }
    __shared__ float4 tab[128];  // NVFP4 steps and reciprocals by scale code
    build_step_table<FMT>(tab, s_t);
    __syncthreads();
    const int64_t upr = k / kUnit, total = m_tok * upr;
    for (int64_t base = (int64_t)rank * kSmallThreads; base < total; base += gstride) {
        const int64_t t = base + tid;
        const bool active = t < total;
        const int64_t row = active ? t / upr : m_tok, u = active ? t - (t / upr) * upr : 0;
        encode_unit<FMT, M, 0>(a, lut, tab, row, u, active, s_t, c6, y6);
    }
}

// ---------------------------------------------------------------------------
// Division self-test: the packed correction division (and its scalar form)
// against the correctly rounded hardware division, on operands drawn from a
// counter-based hash: random quotients in [2^-4, 2^4] and in [2^-11, 2^-4],
// quotients within a few ulps of the E2M1 and UE4M3 rounding boundaries, and
// quotients of exponent -30 .. 30; divisors span [2^-90, 2^90]. A mismatch
// is a quotient of magnitude >= 2^-11 whose bits differ, or any quotient
// whose E2M1 code (or UE4M3 code of its magnitude) differs, or a code of
// the bracketed eight-value encoding (e2m1x8_div) that differs from the
// code of the correctly rounded quotient. (Far below 2^-11
// the remainder of the method can leave the normal range; such quotients
// only ever give a zero code, whose sign comes from the dividend.)
__device__ unsigned long long g_div_mismatch;
__device__ float g_div_examples[16][4];  // first mismatches: v, d, quotient, reference

__device__ __forceinline__ uint64_t hash64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

__global__ void div_check_kernel(uint64_t count, uint64_t seed) {
    const float ties[7] = {0.25f, 0.75f, 1.25f, 1.75f, 2.5f, 3.5f, 5.0f};
    for (uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; i < count; i += (uint64_t)gridDim.x * blockDim.x) {
        const uint64_t h = hash64(seed + 0x9E3779B97F4A7C15ull * (i + 1)), g = hash64(h);
        const int de = (int)(h % 181) - 90;                       // divisor exponent in [-90, 90]
        const float d = __uint_as_float((uint32_t)(de + 127) << 23 | (uint32_t)(g & 0x7FFFFF));
        float v;
        const int kind = (int)((h >> 40) % 5);
        if (kind == 0) {  // near an E2M1 rounding boundary
            const float t = ties[(g >> 23) % 7];
            const int ulps = (int)((g >> 30) % 9) - 4;
            v = __fmul_rn(__uint_as_float(__float_as_uint(t) + ulps), d);
        } else if (kind == 1) {  // quotient exponent in [-30, 30]
            const int qe = (int)((g >> 24) % 61) - 30;
            v = __fmul_rn(__uint_as_float((uint32_t)(qe + 127) << 23 | (uint32_t)(h & 0x7FFFFF)), d);
        } else if (kind == 2) {  // quotient in [2^-4, 2^4]
            const int qe = (int)((g >> 24) % 9) - 4;
            v = __fmul_rn(__uint_as_float((uint32_t)(qe + 127) << 23 | (uint32_t)(h & 0x7FFFFF)), d);
        } else if (kind == 3) {  // quotient in [2^-11, 2^-4]
            const int qe = (int)((g >> 24) % 7) - 11;
            v = __fmul_rn(__uint_as_float((uint32_t)(qe + 127) << 23 | (uint32_t)(h & 0x7FFFFF)), d);
        } else {  // near a UE4M3 rounding boundary (the midpoint of two neighbouring codes)
            const uint32_t c = (uint32_t)((g >> 23) % 126);
            const float t = __fmul_rn(__fadd_rn(ue4m3_value(c), ue4m3_value(c + 1)), 0.5f);
            const int ulps = (int)((g >> 30) % 9) - 4;
            v = __fmul_rn(__uint_as_float(__float_as_uint(t) + ulps), d);
        }
        if ((g >> 63) & 1) v = -v;
        const float y = __frcp_rn(d);
        const float2 q = up2(div2(pk2(v, v), pk2(d, d), pk2(-d, -d), pk2(y, y)));
        const float ref = __fdiv_rn(v, d);
        const float q1 = div1(v, d, y);
        const uint32_t sv = __float_as_uint(v);
        const bool bits_differ = (__float_as_uint(q.x) & 0x7FFFFFFFu) != (__float_as_uint(ref) & 0x7FFFFFFFu) ||
                                 (__float_as_uint(q1) & 0x7FFFFFFFu) != (__float_as_uint(ref) & 0x7FFFFFFFu);
        const bool code_differs = (e2m1_pair(pk2(q.x, q.x), sv, sv) & 0xFu) != (e2m1_pair(pk2(ref, ref), sv, sv) & 0xFu) ||
                                  ue4m3_code(fabsf(q1)) != ue4m3_code(fabsf(ref));
        // The bracketed encoding of eight dividends around v (magnitudes
        // 20 ulps below to 15 ulps above |v|, signs alternating), so that
        // near a rounding boundary some quotients are decided by the
        // bracketing products and some by the fallback.
        float vs[8];
#pragma unroll
        for (int j = 0; j < 8; ++j)
            vs[j] = __uint_as_float(((sv & 0x7FFFFFFFu) + 5 * j - 20) | ((sv ^ (uint32_t)j << 31) & 0x80000000u));
        const uint32_t word = e2m1x8_div(vs, pk2(__fmul_rn(y, 1.0f - 0x1p-21f), __fmul_rn(y, 1.0f - 0x1p-21f)),
                                         pk2(__fmul_rn(y, 1.0f + 0x1p-21f), __fmul_rn(y, 1.0f + 0x1p-21f)), pk2(d, d),
                                         pk2(-d, -d), pk2(y, y));
        bool word_differs = false;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float rj = __fdiv_rn(vs[j], d);
            const uint32_t sj = __float_as_uint(vs[j]);
            word_differs |= ((word >> (4 * j)) & 0xFu) != (e2m1_pair(pk2(rj, rj), sj, sj) & 0xFu);
        }
        if (ref == ref && ((bits_differ && fabsf(ref) >= 0x1p-11f) || code_differs || word_differs)) {
            const unsigned long long slot = atomicAdd(&g_div_mismatch, 1ull);
            if (slot < 16) {
                g_div_examples[slot][0] = v;
                g_div_examples[slot][1] = d;
                g_div_examples[slot][2] = q.x;
                g_div_examples[slot][3] = ref;
            }
        }
    }
}

sharq_status launch_div_check(LaunchCtx &ctx, uint64_t count, uint64_t seed, uint64_t *mismatches, float *examples) {
    unsigned long long zero = 0;
    SQ_CUDA_TRY(cudaMemcpyToSymbolAsync(g_div_mismatch, &zero, sizeof(zero), 0, cudaMemcpyHostToDevice, ctx.stream));
    div_check_kernel<<<ctx.num_sms * 8, 256, 0, ctx.stream>>>(count, seed);
    ctx.launches++;
    SQ_CUDA_TRY(cudaGetLastError());
    unsigned long long host = 0;
    SQ_CUDA_TRY(cudaMemcpyFromSymbolAsync(&host, g_div_mismatch, sizeof(host), 0, cudaMemcpyDeviceToHost, ctx.stream));
    if (examples)
        SQ_CUDA_TRY(cudaMemcpyFromSymbolAsync(examples, g_div_examples, sizeof(g_div_examples), 0,
                                              cudaMemcpyDeviceToHost, ctx.stream));
    SQ_CUDA_TRY(cudaStreamSynchronize(ctx.stream));
    *mismatches = host;
    return SHARQ_OK;
}

// Encode grid: every CTA resident at once (SMs x resident CTAs per SM, as
// the occupancy calculator gives it for the kernel), each looping over units
// with the grid stride, so that no partial last wave is left.
static int64_t encode_grid(void *fn, int num_sms, int64_t total_units) {
    struct Entry {
        void *fn;
        int dev, occ;
    };
    static Entry cache[64];
    static int used = 0;
    static std::mutex mu;  // lookups and appends from concurrent host threads
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) dev = 0;
    std::lock_guard<std::mutex> lock(mu);
    int occ = 0;
    for (int i = 0; i < used; ++i)
        if (cache[i].fn == fn && cache[i].dev == dev) occ = cache[i].occ;
    if (occ == 0) {
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, fn, kEncodeThreads, 0) != cudaSuccess || occ < 1)
            occ = 1;
        if (used < 64) cache[used++] = Entry{fn, dev, occ};
    }
    const int64_t blocks = (total_units + kEncodeThreads - 1) / kEncodeThreads;
    const int64_t cap = (int64_t)num_sms * occ;
    return blocks < cap ? blocks : cap;
}

template <int FMT>
static void *encode_fn(int m, int n) {
    switch (m) {
        case 2: return (void *)prep_encode_kernel<FMT, 2, 0>;
        case 4: return n == 2 ? (void *)prep_encode_kernel<FMT, 4, 2> : (void *)prep_encode_kernel<FMT, 4, 0>;
        case 8: return (void *)prep_encode_kernel<FMT, 8, 0>;
        default: return (void *)prep_encode_kernel<FMT, 16, 0>;
    }
}

template <int FMT, bool AFFINE>
static void *encode_rows_fn(int m, int n) {
    switch (m) {
        case 2: return (void *)prep_encode_rows_kernel<FMT, 2, 0, AFFINE>;
        case 4: return n == 2 ? (void *)prep_encode_rows_kernel<FMT, 4, 2, AFFINE>
                              : (void *)prep_encode_rows_kernel<FMT, 4, 0, AFFINE>;
        case 8: return n == 4 ? (void *)prep_encode_rows_kernel<FMT, 8, 4, AFFINE>
                              : (void *)prep_encode_rows_kernel<FMT, 8, 0, AFFINE>;
        default: return (void *)prep_encode_rows_kernel<FMT, 16, 0, AFFINE>;
    }
}

// Grid of a persistent kernel: every CTA resident at once (SMs x resident
// CTAs per SM for `threads` threads and `smem` dynamic shared memory), at
// most `blocks`.
static int64_t resident_grid(void *fn, int num_sms, int threads, size_t smem, int64_t blocks) {
    struct Entry {
        void *fn;
        int dev, occ;
    };
    static Entry cache[64];
    static int used = 0;
    static std::mutex mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) dev = 0;
    std::lock_guard<std::mutex> lock(mu);
    int occ = 0;
    for (int i = 0; i < used; ++i)
        if (cache[i].fn == fn && cache[i].dev == dev) occ = cache[i].occ;
    if (occ == 0) {
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, fn, threads, smem) != cudaSuccess || occ < 1) {
            cudaGetLastError();
            occ = 1;
        }
        if (used < 64) cache[used++] = Entry{fn, dev, occ};
    }
    const int64_t cap = (int64_t)num_sms * occ;
    return blocks < cap ? blocks : cap;
}

template <int FMT>
static void *encode_grouped_fn(int m, int n) {
    switch (m) {
        case 2: return (void *)prep_encode_grouped_kernel<FMT, 2, 0>;
        case 4: return n == 2 ? (void *)prep_encode_grouped_kernel<FMT, 4, 2> : (void *)prep_encode_grouped_kernel<FMT, 4, 0>;
        case 8: return (void *)prep_encode_grouped_kernel<FMT, 8, 0>;
        default: return (void *)prep_encode_grouped_kernel<FMT, 16, 0>;
    }
}

template <int FMT, bool RMS>
static void *small_fn(int m) {
    switch (m) {
        case 2: return (void *)prep_small_kernel<FMT, 2, RMS>;
        case 4: return (void *)prep_small_kernel<FMT, 4, RMS>;
        case 8: return (void *)prep_small_kernel<FMT, 8, RMS>;
        default: return (void *)prep_small_kernel<FMT, 16, RMS>;
    }
}

// Few rows: the single-launch cluster kernel.
static sharq_status launch_prepare_small(LaunchCtx &ctx, const sharq_prep &P, const void *x, const void *gamma,
                                         const void *beta, float eps, int norm) {
    void *fn = P.fmt == kFmtNV ? (norm ? small_fn<kFmtNV, true>(P.m) : small_fn<kFmtNV, false>(P.m))
                               : (norm ? small_fn<kFmtMX, true>(P.m) : small_fn<kFmtMX, false>(P.m));
    EncodeArgs ea{(const uint16_t *)x, (const uint16_t *)gamma, (const uint16_t *)beta,
                  reinterpret_cast<const float2 *>(P.scratch), P.m_tok, P.k, P.meta_row_bytes,
                  P.k / (P.fmt == kFmtNV ? 16 : 32), P.n, (uint8_t *)P.s_codes, (uint8_t *)P.r_codes,
                  (uint8_t *)P.s_scales, (uint8_t *)P.r_scales, (uint8_t *)P.meta};
    int64_t sf_rows = P.sf_rows;
    float *words = P.tensor_scale - 1;
    int meta_zero = ((kUnit / P.m) * P.n * idx_bits(P.m)) % 8 != 0 ? 1 : 0;
    void *args[] = {&ea, &eps, &sf_rows, &words, &meta_zero};
    cudaLaunchConfig_t cfg;
    memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3(kSmallCtas, 1, 1);
    cfg.blockDim = dim3(kSmallThreads, 1, 1);
    cfg.stream = ctx.stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kSmallCtas;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    SQ_CUDA_TRY(cudaLaunchKernelExC(&cfg, fn, args));
    ctx.launches++;
    SQ_CUDA_TRY(cudaGetLastError());
    return SHARQ_OK;
}

// ---------------------------------------------------------------------------
// Preparation whose scratch lives in the library instead of the caller's
// buffer (sharq_prepare_noalloc). The statistics kernel's per-row (mu, rstd)
// and the tensor-amax word go into one fixed device array; every GPU that
// loads the library holds it until the process exits.

constexpr int64_t kStaticScratchRows = SHARQ_NOALLOC_MAX_ROWS;
constexpr size_t kStaticScratchBytes = 256 + 8 * (size_t)kStaticScratchRows;  // [0,4) amax word, [256,...) stats
static __device__ __align__(256) unsigned char g_prep_scratch[kStaticScratchBytes];

// Device address of g_prep_scratch on the current device, looked up once per
// device (in host code the array's name is only a stand-in for the symbol).
static sharq_status static_scratch(int dev, unsigned char **out) {
    static unsigned char *addr[64] = {nullptr};
    static std::mutex mu;
    if (dev < 0 || dev >= 64) return SHARQ_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        unsigned char *p = nullptr;
        if (cudaGetSymbolAddress((void **)&p, g_prep_scratch) != cudaSuccess || !p) return SHARQ_ERR_CUDA;
        addr[dev] = p;
    }
    *out = addr[dev];
    return SHARQ_OK;
}

static bool noalloc_aligned(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 255u) == 0; }

}  // namespace sq

extern "C" sharq_status sharq_prepare_noalloc(const void *x_dev, int64_t m_tok, int64_t k, const void *ln_w_dev,
                                              const void *ln_b_dev, float eps, int n, int m, int fmt,
                                              void *s_codes_dev, void *r_codes_dev, void *s_scales_dev,
                                              void *r_scales_dev, void *meta_dev, float *s_t_dev,
                                              sharq_prep *prep_out, void *stream) {
    using namespace sq;
    note_launches(0);
    const bool fmt_ok = fmt == kFmtNV || fmt == kFmtMX;
    const bool nm_ok = (m == 2 || m == 4 || m == 8 || m == 16) && n >= 1 && n <= m;
    if (!fmt_ok || !nm_ok || k <= 0 || k > SHARQ_K_MAX || k % SHARQ_K_ALIGN != 0 || m_tok < 0 || !prep_out ||
        !s_t_dev)
        return SHARQ_ERR_INVALID_ARG;
    if (!(eps > 0.0f) || eps > 3.0e38f) return SHARQ_ERR_INVALID_ARG;
    if (m_tok > kStaticScratchRows) return SHARQ_ERR_UNSUPPORTED;  // beyond the fixed scratch array
    if (!s_scales_dev || !r_scales_dev || !noalloc_aligned(s_scales_dev) || !noalloc_aligned(r_scales_dev) ||
        (reinterpret_cast<uintptr_t>(s_t_dev) & 3u))
        return SHARQ_ERR_INVALID_ARG;
    if (m_tok > 0 && (!x_dev || !s_codes_dev || !r_codes_dev || !meta_dev || !noalloc_aligned(s_codes_dev) ||
                      !noalloc_aligned(r_codes_dev) || !noalloc_aligned(meta_dev) ||
                      (reinterpret_cast<uintptr_t>(x_dev) & 15u)))
        return SHARQ_ERR_INVALID_ARG;
    if ((ln_w_dev && (reinterpret_cast<uintptr_t>(ln_w_dev) & 15u)) ||
        (ln_b_dev && (reinterpret_cast<uintptr_t>(ln_b_dev) & 15u)))
        return SHARQ_ERR_INVALID_ARG;

    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return SHARQ_ERR_CUDA;
    unsigned char *scratch = nullptr;
    sharq_status st = static_scratch(dev, &scratch);
    if (st != SHARQ_OK) return st;
    static int sms[64] = {0};
    static bool attr_done[64] = {false};
    {
        static std::mutex mu;
        std::lock_guard<std::mutex> lock(mu);
        if (!sms[dev] && cudaDeviceGetAttribute(&sms[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return SHARQ_ERR_CUDA;
        if (!attr_done[dev]) {
            if (cudaFuncSetAttribute(ln_stats_kernel<true, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)(2 * SHARQ_K_MAX)) != cudaSuccess)
                return SHARQ_ERR_CUDA;
            attr_done[dev] = true;
        }
    }

    const PrepLayout L = prep_layout(m_tok, k, n, m, fmt);
    sharq_prep P;
    memset(&P, 0, sizeof(P));
    P.m_tok = m_tok;
    P.k = k;
    P.n = n;
    P.m = m;
    P.fmt = fmt;
    P.sf_rows = L.sf_rows;
    P.meta_row_bytes = L.meta_row;
    P.s_codes = s_codes_dev;
    P.r_codes = r_codes_dev;
    P.s_scales = s_scales_dev;
    P.r_scales = r_scales_dev;
    P.meta = meta_dev;
    P.tensor_scale = s_t_dev;
    P.scratch = scratch + 256;  // per-row (mu, rstd)

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    unsigned *amax_word = reinterpret_cast<unsigned *>(scratch);
    float2 *stats = reinterpret_cast<float2 *>(scratch + 256);
    if (cudaMemsetAsync(amax_word, 0, sizeof(unsigned), s) != cudaSuccess) return SHARQ_ERR_CUDA;
    const bool meta_atomic = ((kUnit / m) * n * idx_bits(m)) % 8 != 0;
    if (meta_atomic && m_tok > 0 && cudaMemsetAsync(meta_dev, 0, (size_t)(m_tok * L.meta_row), s) != cudaSuccess)
        return SHARQ_ERR_CUDA;
    if (m_tok > 0) {
        if (ln_w_dev || ln_b_dev)
            ln_stats_kernel<true, false><<<(unsigned)m_tok, kStatsThreads, (size_t)(2 * k), s>>>(
                (const uint16_t *)x_dev, (const uint16_t *)ln_w_dev, (const uint16_t *)ln_b_dev, eps, k, stats,
                amax_word);
        else
            ln_stats_kernel<false, false><<<(unsigned)m_tok, kStatsThreads, 0, s>>>((const uint16_t *)x_dev, nullptr, nullptr,
                                                                           eps, k, stats, amax_word);
    }
    const int64_t total = P.sf_rows * (k / kUnit);
    void *fn = fmt == kFmtNV ? encode_fn<kFmtNV>(m, n) : encode_fn<kFmtMX>(m, n);
    const int64_t blocks = encode_grid(fn, sms[dev], total);
    const uint16_t *xx = (const uint16_t *)x_dev, *gg = (const uint16_t *)ln_w_dev, *bb = (const uint16_t *)ln_b_dev;
    const float2 *cst = stats;
    const unsigned *aw = amax_word;
    float *sto = s_t_dev;
    int64_t mt = m_tok, sfr = P.sf_rows, kk = k, mrow = L.meta_row;
    int nn = n;
    uint8_t *sc = (uint8_t *)s_codes_dev, *rc = (uint8_t *)r_codes_dev, *ss = (uint8_t *)s_scales_dev,
            *rs = (uint8_t *)r_scales_dev, *mt8 = (uint8_t *)meta_dev;
    void *args[] = {&xx, &gg, &bb, &cst, &aw, &sto, &mt, &sfr, &kk, &nn, &sc, &rc, &ss, &rs, &mt8, &mrow};
    if (cudaLaunchKernel(fn, dim3((unsigned)blocks), dim3(kEncodeThreads), args, 0, s) != cudaSuccess)
        return SHARQ_ERR_CUDA;
    if (cudaGetLastError() != cudaSuccess) return SHARQ_ERR_CUDA;
    note_launches(m_tok > 0 ? 2 : 1);  // statistics (rows only) and encode
    *prep_out = P;
    return SHARQ_OK;
}

namespace sq {

// Statistics pass: one warp per row when there are rows enough for a CTA of
// eight per SM (or the rows are short); one CTA per row keeps few-row
// (decode) launches short.
template <bool RMS>
static sharq_status launch_stats(LaunchCtx &ctx, const sharq_prep &P, const void *x, const void *gamma,
                                 const void *beta, float eps, float2 *stats, unsigned *words) {
    static bool attr_done[64] = {false};
    static std::mutex mu;
    int dev = 0;
    SQ_CUDA_TRY(cudaGetDevice(&dev));
    if (dev < 0 || dev >= 64) return SHARQ_ERR_UNSUPPORTED;
    {
        std::lock_guard<std::mutex> lock(mu);  // held for the attribute set-up only
        if (!attr_done[dev]) {
            SQ_CUDA_TRY(cudaFuncSetAttribute(ln_stats_kernel<true, RMS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)(2 * SHARQ_K_MAX)));
            SQ_CUDA_TRY(cudaFuncSetAttribute(ln_stats_warp_kernel<true, RMS, false>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, kStatsRingBytes));
            SQ_CUDA_TRY(cudaFuncSetAttribute(ln_stats_warp_kernel<false, RMS, false>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, kStatsRingBytes));
            SQ_CUDA_TRY(cudaFuncSetAttribute(ln_stats_warp_kernel<true, RMS, true>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, kStatsRingBytes));
            SQ_CUDA_TRY(cudaFuncSetAttribute(ln_stats_warp_kernel<false, RMS, true>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, kStatsRingBytes));
            SQ_CUDA_TRY(cudaFuncSetAttribute(ln_stats_long_kernel<true, RMS>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, kStatsRingBytes));
            SQ_CUDA_TRY(cudaFuncSetAttribute(ln_stats_long_kernel<false, RMS>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, kStatsRingBytes));
            attr_done[dev] = true;
        }
    }
    if (P.m_tok == 0) return SHARQ_OK;
    const bool warp_rows = P.m_tok >= (int64_t)ctx.num_sms * (kStatsThreads / 32) || P.k <= kWarpRowMaxK;
    const uint16_t *xx = (const uint16_t *)x, *gg = (const uint16_t *)gamma, *bb = (const uint16_t *)beta;
    if (warp_rows) {
        // Short rows and rows enough for 16 warps per SM: several rows per
        // warp, so that the per-row finish runs on many threads at once.
        int rpw = 1;
        if (!(gamma || beta) && P.k <= 2048) {
            const int64_t r = P.m_tok / ((int64_t)ctx.num_sms * 16);
            rpw = (int)(r < 1 ? 1 : (r > kStatsMaxRpw ? kStatsMaxRpw : r));
        }
        const int64_t per_cta = (int64_t)(kStatsThreads / 32) * rpw;
        const unsigned grid = (unsigned)((P.m_tok + per_cta - 1) / per_cta);
        // The certified sums (two finishes per row, the exact sums only where
        // they leave rstd undecided) for rows longer than 2048 elements, in
        // the persistent kernel, and for shorter rows when there are at least
        // 8 rows per SM, in this warp kernel's certified form. Measured on
        // B200: 32768 x 768 69.7 us against 75.9 with the exact integer sums,
        // 8192 x 2048 41.0 against 47.1; with few rows (256 x 768) the exact
        // sums are faster (12.3 against 14.3 us).
        const bool fast = P.k > 2048 || P.m_tok >= (int64_t)ctx.num_sms * 8;
        if (fast && P.k > 2048) {
            void *fn = (gamma || beta) ? (void *)ln_stats_long_kernel<true, RMS> : (void *)ln_stats_long_kernel<false, RMS>;
            const int64_t need = (P.m_tok + (kStatsThreads / 32) - 1) / (kStatsThreads / 32);
            const unsigned lgrid = (unsigned)resident_grid(fn, ctx.num_sms, kStatsThreads, kStatsRingBytes, need);
            float e = eps;
            int64_t kk = P.k, mt = P.m_tok;
            void *args[] = {&xx, &gg, &bb, &e, &kk, &mt, &stats, &words};
            SQ_CUDA_TRY(cudaLaunchKernel(fn, dim3(lgrid), dim3(kStatsThreads), args, kStatsRingBytes, ctx.stream));
        } else if (gamma || beta) {
            auto fn = fast ? ln_stats_warp_kernel<true, RMS, true> : ln_stats_warp_kernel<true, RMS, false>;
            fn<<<grid, kStatsThreads, kStatsRingBytes, ctx.stream>>>(xx, gg, bb, eps, P.k, P.m_tok, 1, stats, words);
        } else {
            auto fn = fast ? ln_stats_warp_kernel<false, RMS, true> : ln_stats_warp_kernel<false, RMS, false>;
            fn<<<grid, kStatsThreads, kStatsRingBytes, ctx.stream>>>(xx, nullptr, nullptr, eps, P.k, P.m_tok, rpw,
                                                                   stats, words);
        }
    } else {
        if (gamma || beta)
            ln_stats_kernel<true, RMS><<<(unsigned)P.m_tok, kStatsThreads, (size_t)(2 * P.k), ctx.stream>>>(
                xx, gg, bb, eps, P.k, stats, words);
        else
            ln_stats_kernel<false, RMS><<<(unsigned)P.m_tok, kStatsThreads, 0, ctx.stream>>>(xx, nullptr, nullptr,
                                                                                           eps, P.k, stats, words);
    }
    ctx.launches++;
    SQ_CUDA_TRY(cudaGetLastError());
    return SHARQ_OK;
}

sharq_status launch_prepare(LaunchCtx &ctx, const sharq_prep &P, const void *x, const void *gamma, const void *beta,
                            float eps, int norm) {
    // Up to 8 rows: the single-launch cluster kernel (measured on the
    // down-projection input: 13-16 us against 18 us for the two passes at
    // M = 1..8; at 16 rows its encode, on the cluster's 8 SMs only, is slower).
    if (P.m_tok >= 1 && P.m_tok <= kSmallRows) return launch_prepare_small(ctx, P, x, gamma, beta, eps, norm);
    unsigned *words = reinterpret_cast<unsigned *>(P.tensor_scale) - 1;  // [0] amax bits, [1] s_t
    SQ_CUDA_TRY(cudaMemsetAsync(words, 0, sizeof(unsigned), ctx.stream));
    const int ib = idx_bits(P.m);
    const bool meta_atomic = ((kUnit / P.m) * P.n * ib) % 8 != 0;
    if (meta_atomic && P.m_tok > 0)  // unaligned metadata fields are OR-ed into a zeroed stream
        SQ_CUDA_TRY(cudaMemsetAsync(P.meta, 0, (size_t)(P.m_tok * P.meta_row_bytes), ctx.stream));
    float2 *stats = reinterpret_cast<float2 *>(P.scratch);
    const sharq_status sst = norm ? launch_stats<true>(ctx, P, x, gamma, beta, eps, stats, words)
                                  : launch_stats<false>(ctx, P, x, gamma, beta, eps, stats, words);
    if (sst != SHARQ_OK) return sst;
    const bool affine = gamma != nullptr || beta != nullptr;
    void *fn = P.fmt == kFmtNV ? (affine ? encode_rows_fn<kFmtNV, true>(P.m, P.n) : encode_rows_fn<kFmtNV, false>(P.m, P.n))
                               : (affine ? encode_rows_fn<kFmtMX, true>(P.m, P.n) : encode_rows_fn<kFmtMX, false>(P.m, P.n));
    const int64_t chunks = (P.k / kUnit + 31) / 32;
    const int64_t warps = P.m_tok * chunks > 0 ? P.m_tok * chunks : 1;
    const int64_t blocks = encode_grid(fn, ctx.num_sms, warps * 32);
    EncodeArgs ea{(const uint16_t *)x, (const uint16_t *)gamma, (const uint16_t *)beta, stats, P.m_tok, P.k,
                  P.meta_row_bytes, P.k / (P.fmt == kFmtNV ? 16 : 32), P.n, (uint8_t *)P.s_codes,
                  (uint8_t *)P.r_codes, (uint8_t *)P.s_scales, (uint8_t *)P.r_scales, (uint8_t *)P.meta};
    const unsigned *aw = words;
    float *sto = P.tensor_scale;
    int64_t sf_rows = P.sf_rows;
    void *args[] = {&ea, &aw, &sto, &sf_rows};
    // Programmatic dependent launch: the encode may start while the
    // statistics kernel finishes (it waits for it before reading).
    cudaLaunchConfig_t cfg;
    memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3((unsigned)blocks, 1, 1);
    cfg.blockDim = dim3(kEncodeThreads, 1, 1);
    cfg.stream = ctx.stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = P.m_tok > 0 ? 1 : 0;  // no statistics kernel before it otherwise
    SQ_CUDA_TRY(cudaLaunchKernelExC(&cfg, fn, args));
    ctx.launches++;
    return SHARQ_OK;
}

// Pair-wise 4:8 mode: the statistics pass, then the sparse encode pass
// (a programmatic dependent of it).
sharq_status launch_prepare_sparse(LaunchCtx &ctx, const sharq_prep &P, const void *x, const void *gamma,
                                   const void *beta, float eps, int norm) {
    unsigned *words = reinterpret_cast<unsigned *>(P.tensor_scale) - 1;  // [0] amax bits, [1] s_t
    SQ_CUDA_TRY(cudaMemsetAsync(words, 0, sizeof(unsigned), ctx.stream));
    float2 *stats = reinterpret_cast<float2 *>(P.scratch);
    const sharq_status sst = norm ? launch_stats<true>(ctx, P, x, gamma, beta, eps, stats, words)
                                  : launch_stats<false>(ctx, P, x, gamma, beta, eps, stats, words);
    if (sst != SHARQ_OK) return sst;
    const bool affine = gamma != nullptr || beta != nullptr;
    void *fn = P.fmt == kFmtNV
                   ? (affine ? (void *)prep_encode_sparse_kernel<kFmtNV, true> : (void *)prep_encode_sparse_kernel<kFmtNV, false>)
                   : (affine ? (void *)prep_encode_sparse_kernel<kFmtMX, true> : (void *)prep_encode_sparse_kernel<kFmtMX, false>);
    const int64_t chunks = (P.k / kUnit + 31) / 32;
    const int64_t warps = P.m_tok * chunks > 0 ? P.m_tok * chunks : 1;
    const int64_t blocks = encode_grid(fn, ctx.num_sms, warps * 32);
    EncodeArgs ea{(const uint16_t *)x, (const uint16_t *)gamma, (const uint16_t *)beta, stats, P.m_tok, P.k,
                  P.meta_row_bytes, P.k / (P.fmt == kFmtNV ? 16 : 32), P.n, (uint8_t *)P.s_codes,
                  (uint8_t *)P.r_codes, (uint8_t *)P.s_scales, (uint8_t *)P.r_scales, (uint8_t *)P.meta};
    const unsigned *aw = words;
    float *sto = P.tensor_scale;
    int64_t sf_rows = P.sf_rows;
    void *args[] = {&ea, &aw, &sto, &sf_rows};
    cudaLaunchConfig_t cfg;
    memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3((unsigned)blocks, 1, 1);
    cfg.blockDim = dim3(kEncodeThreads, 1, 1);
    cfg.stream = ctx.stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = P.m_tok > 0 ? 1 : 0;
    SQ_CUDA_TRY(cudaLaunchKernelExC(&cfg, fn, args));
    ctx.launches++;
    return SHARQ_OK;
}

// Residual add and preparation: x_out = RN16(h + d) with its statistics in
// one pass, then the encode pass over x_out (a programmatic dependent).
sharq_status launch_prepare_add(LaunchCtx &ctx, const sharq_prep &P, const void *h, const void *d, void *x_out,
                                const void *gamma, const void *beta, float eps, int norm) {
    unsigned *words = reinterpret_cast<unsigned *>(P.tensor_scale) - 1;  // [0] amax bits, [1] s_t
    SQ_CUDA_TRY(cudaMemsetAsync(words, 0, sizeof(unsigned), ctx.stream));
    const bool meta_atomic = ((kUnit / P.m) * P.n * idx_bits(P.m)) % 8 != 0;
    if (meta_atomic && P.m_tok > 0)
        SQ_CUDA_TRY(cudaMemsetAsync(P.meta, 0, (size_t)(P.m_tok * P.meta_row_bytes), ctx.stream));
    float2 *stats = reinterpret_cast<float2 *>(P.scratch);
    const bool affine = gamma != nullptr || beta != nullptr;
    if (P.m_tok > 0) {
        const bool fast = P.k > 2048;
        void *fn;
        if (norm)
            fn = affine ? (fast ? (void *)add_stats_kernel<true, true, true> : (void *)add_stats_kernel<true, true, false>)
                        : (fast ? (void *)add_stats_kernel<false, true, true> : (void *)add_stats_kernel<false, true, false>);
        else
            fn = affine ? (fast ? (void *)add_stats_kernel<true, false, true> : (void *)add_stats_kernel<true, false, false>)
                        : (fast ? (void *)add_stats_kernel<false, false, true> : (void *)add_stats_kernel<false, false, false>);
        const int64_t need = (P.m_tok + (kStatsThreads / 32) - 1) / (kStatsThreads / 32);
        const unsigned grid = (unsigned)resident_grid(fn, ctx.num_sms, kStatsThreads, 0, need);
        const uint16_t *hh = (const uint16_t *)h, *dd = (const uint16_t *)d, *gg = (const uint16_t *)gamma,
                       *bb = (const uint16_t *)beta;
        uint16_t *xo = (uint16_t *)x_out;
        float e = eps;
        int64_t kk = P.k, mt = P.m_tok;
        void *args[] = {&hh, &dd, &xo, &gg, &bb, &e, &kk, &mt, &stats, &words};
        SQ_CUDA_TRY(cudaLaunchKernel(fn, dim3(grid), dim3(kStatsThreads), args, 0, ctx.stream));
        ctx.launches++;
    }
    void *fn = P.fmt == kFmtNV ? (affine ? encode_rows_fn<kFmtNV, true>(P.m, P.n) : encode_rows_fn<kFmtNV, false>(P.m, P.n))
                               : (affine ? encode_rows_fn<kFmtMX, true>(P.m, P.n) : encode_rows_fn<kFmtMX, false>(P.m, P.n));
    const int64_t chunks = (P.k / kUnit + 31) / 32;
    const int64_t warps = P.m_tok * chunks > 0 ? P.m_tok * chunks : 1;
    const int64_t blocks = encode_grid(fn, ctx.num_sms, warps * 32);
    EncodeArgs ea{(const uint16_t *)x_out, (const uint16_t *)gamma, (const uint16_t *)beta, stats, P.m_tok, P.k,
                  P.meta_row_bytes, P.k / (P.fmt == kFmtNV ? 16 : 32), P.n, (uint8_t *)P.s_codes,
                  (uint8_t *)P.r_codes, (uint8_t *)P.s_scales, (uint8_t *)P.r_scales, (uint8_t *)P.meta};
    const unsigned *aw = words;
    float *sto = P.tensor_scale;
    int64_t sf_rows = P.sf_rows;
    void *args[] = {&ea, &aw, &sto, &sf_rows};
    cudaLaunchConfig_t cfg;
    memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3((unsigned)blocks, 1, 1);
    cfg.blockDim = dim3(kEncodeThreads, 1, 1);
    cfg.stream = ctx.stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = P.m_tok > 0 ? 1 : 0;
    SQ_CUDA_TRY(cudaLaunchKernelExC(&cfg, fn, args));
    ctx.launches++;
    return SHARQ_OK;
}

// Preparation of `rows` rows in grouped order straight into a grouped prep P
// (P.m_tok = P.sf_rows = the grouped capacity): statistics over the source
// rows (kept in P's statistics area, indexed by source row), then the
// grouped encode pass.
sharq_status launch_prepare_grouped(LaunchCtx &ctx, const sharq_prep &P, const void *x, int64_t rows,
                                    const int32_t *offsets, int32_t groups, const void *gamma, const void *beta,
                                    float eps, int norm) {
    unsigned *words = reinterpret_cast<unsigned *>(P.tensor_scale) - 1;  // [0] amax bits, [1] s_t
    SQ_CUDA_TRY(cudaMemsetAsync(words, 0, sizeof(unsigned), ctx.stream));
    const bool meta_atomic = ((kUnit / P.m) * P.n * idx_bits(P.m)) % 8 != 0;
    if (meta_atomic && P.m_tok > 0)
        SQ_CUDA_TRY(cudaMemsetAsync(P.meta, 0, (size_t)(P.m_tok * P.meta_row_bytes), ctx.stream));
    float2 *stats = reinterpret_cast<float2 *>(P.scratch);
    sharq_prep src = P;  // the statistics pass sees the source rows
    src.m_tok = rows;
    const sharq_status sst = norm ? launch_stats<true>(ctx, src, x, gamma, beta, eps, stats, words)
                                  : launch_stats<false>(ctx, src, x, gamma, beta, eps, stats, words);
    if (sst != SHARQ_OK) return sst;
    void *fn = P.fmt == kFmtNV ? encode_grouped_fn<kFmtNV>(P.m, P.n) : encode_grouped_fn<kFmtMX>(P.m, P.n);
    const int64_t blocks = encode_grid(fn, ctx.num_sms, P.m_tok * (P.k / kUnit));
    EncodeArgs ea{(const uint16_t *)x, (const uint16_t *)gamma, (const uint16_t *)beta, stats, rows, P.k,
                  P.meta_row_bytes, P.k / (P.fmt == kFmtNV ? 16 : 32), P.n, (uint8_t *)P.s_codes,
                  (uint8_t *)P.r_codes, (uint8_t *)P.s_scales, (uint8_t *)P.r_scales, (uint8_t *)P.meta};
    const unsigned *aw = words;
    float *sto = P.tensor_scale;
    int64_t cap = P.m_tok, nrows = rows;
    int32_t ng = groups;
    unsigned *status = ctx.status;
    void *args[] = {&ea, &aw, &sto, &cap, &offsets, &ng, &nrows, &status};
    SQ_CUDA_TRY(cudaLaunchKernel(fn, dim3((unsigned)blocks), dim3(kEncodeThreads), args, 0, ctx.stream));
    ctx.launches++;
    return SHARQ_OK;
}

}  // namespace sq

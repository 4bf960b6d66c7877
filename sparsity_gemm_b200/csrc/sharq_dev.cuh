// Device helpers of the SharQ library: numeric steps shared by the
// preparation and weight kernels, and thin wrappers over the sm_100a PTX the
// GEMM uses (mbarrier, TMA, tcgen05). Every floating-point step is an
// explicit round-to-nearest intrinsic, so the compiler cannot contract a
// multiply and an add into one FMA.
#pragma once
#include <cuda_fp16.h>
#include <stdint.h>

#include "layout.h"

namespace sq {

// ---------------------------------------------------------------------------
// Status word: the first non-zero site code wins.
__device__ __forceinline__ void record_status(unsigned *status, unsigned site) {
    if (status) atomicCAS(status, 0u, site);
}

__device__ __forceinline__ unsigned read_status(const unsigned *status) {
    return status ? *(volatile const unsigned *)status : 0u;
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ---------------------------------------------------------------------------
// Numeric steps

// fp16 -> fp32 (exact).
__device__ __forceinline__ float h2f(uint16_t h) { return __half2float(__ushort_as_half(h)); }

// LayerNorm apply: RN32(RN32(RN32(x - mu) * rstd) * gamma) + beta.
__device__ __forceinline__ float ln_apply(float x, float mu, float rstd, bool has_g, float g, bool has_b,
                                          float b) {
    float t = __fsub_rn(x, mu);
    t = __fmul_rn(t, rstd);
    if (has_g) t = __fmul_rn(t, g);
    if (has_b) t = __fadd_rn(t, b);
    return t;
}

// E2M1 codes of (lo, hi) packed into one byte, lo in bits 0-3. The hardware
// conversion rounds to nearest even and saturates to 6; the sign bit is then
// forced from the operand so that values rounding to zero keep their sign.
__device__ __forceinline__ uint32_t e2m1x2(float lo, float hi) {
    uint32_t b;
    asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tcvt.u32.u8 %0, t;\n\t}"
        : "=r"(b) : "f"(hi), "f"(lo));
    b |= (__float_as_uint(lo) >> 31) << 3;
    b |= (__float_as_uint(hi) >> 31) << 7;
    return b;
}

// Values of two E2M1 codes in one byte (lo nibble first), as floats.
__device__ __forceinline__ float2 e2m1x2_value(uint32_t byte) {
    uint32_t h2;
    asm("{\n\t.reg .b8 t;\n\tcvt.u8.u32 t, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, t;\n\t}" : "=r"(h2) : "r"(byte));
    __half2 h = *reinterpret_cast<__half2 *>(&h2);
    return __half22float2(h);
}

// UE4M3 code of u >= 0: round to nearest even, saturate to 448.
__device__ __forceinline__ uint32_t ue4m3_code(float u) {
    uint16_t e;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(e) : "f"(0.0f), "f"(u));
    return e & 0xFFu;
}

// Value of a UE4M3 code (exact: every E4M3 value is an fp16 value).
__device__ __forceinline__ float ue4m3_value(uint32_t code) {
    uint32_t h2;
    uint16_t c = (uint16_t)code;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(c));
    return __half2float(__ushort_as_half((uint16_t)(h2 & 0xFFFF)));
}

// OCP MX block exponent: floor(log2 a) - 2 for a > 0, clamped to [-127, 127].
__device__ __forceinline__ int mx_exponent(float a) {
    uint32_t bits = __float_as_uint(a);
    int ex = (int)(bits >> 23);
    int fl = ex ? ex - 127 : (31 - __clz((int)(bits & 0x7FFFFF))) - 149;
    int e = fl - 2;
    return e < -127 ? -127 : (e > 127 ? 127 : e);
}

// 2^e as a float, e in [-127, 127] (2^-127 is subnormal).
__device__ __forceinline__ float pow2f(int e) {
    return e >= -126 ? __uint_as_float((uint32_t)(e + 127) << 23) : __uint_as_float(0x00400000u);
}

// Step d and scale code of one block with amax a (tensor scale s_t; c6 =
// RN32(6 s_t)). NVFP4: code = UE4M3(a / c6), d = RN32(value * s_t). MXFP4:
// code = e + 127, d = 2^e; a == 0 gives code 0 and d = 0.
template <int FMT>
__device__ __forceinline__ float block_step(float a, float s_t, float c6, uint32_t &code) {
    if (FMT == kFmtNV) {
        float u = __fdiv_rn(a, c6);
        code = ue4m3_code(u);
        return __fmul_rn(ue4m3_value(code), s_t);
    } else {
        if (a == 0.0f) {
            code = 0;
            return 0.0f;
        }
        int e = mx_exponent(a);
        code = (uint32_t)(e + 127);
        return pow2f(e);
    }
}

// ---------------------------------------------------------------------------
// Packed pairs of binary32 (sm_100 f32x2 instructions): one instruction for
// two independent IEEE operations, each rounded to nearest even. Code
// generation may fuse a packed multiply that feeds a packed add or subtract
// into one fused multiply-add (the product then goes unrounded), so callers
// use these only where no product feeds an add, or where the FMA is meant;
// rounded products that feed an add use the scalar __fmul_rn / __fadd_rn.

__device__ __forceinline__ uint64_t pk2(float a, float b) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ float2 up2(uint64_t r) {
    float2 f;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(f.x), "=f"(f.y) : "l"(r));
    return f;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t add2_rm(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("add.rm.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t sub2(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}

// Two fp16 values (one 32-bit word, low half first) as a packed float pair.
__device__ __forceinline__ uint64_t h2_to_f2(uint32_t w) {
    float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&w));
    return pk2(f.x, f.y);
}

// Correctly rounded quotients v / d of a packed pair, for d in [2^-90, 2^90]
// with y = RN(1/d) and |v / d| >= 2^-11 (smaller quotients come out within
// an ulp, which is all E2M1 and UE4M3 encoding need there). Markstein's correction (P. Markstein, "Computation of
// elementary functions on the IBM RISC System/6000 processor", IBM J. Res.
// Dev. 34(1), 1990): q0 = RN(v y); one FMA residual step makes the quotient
// faithful; with the remainder r = v - d q1 then exact, RN(q1 + r y) is the
// correctly rounded quotient. Zero quotients may lose their sign; callers
// take the sign from v.
__device__ __forceinline__ uint64_t div2(uint64_t v, uint64_t d2, uint64_t nd2, uint64_t y2) {
    uint64_t q = mul2(v, y2);
    uint64_t r = fma2(q, nd2, v);
    q = fma2(r, y2, q);
    r = fma2(q, nd2, v);
    return fma2(r, y2, q);
}

// The same correctly rounded quotient for one value (v / d, y = RN(1/d),
// d in [2^-90, 2^90], |v / d| >= 2^-11). The remainder v - d q1 is then a
// multiple of ulp(q1) ulp(d) >= 2^-147, hence exact even below the normal
// range.
__device__ __forceinline__ float div1(float v, float d, float y) {
    float q = __fmul_rn(v, y);
    float r = __fmaf_rn(q, -d, v);
    q = __fmaf_rn(r, y, q);
    r = __fmaf_rn(q, -d, v);
    return __fmaf_rn(r, y, q);
}

// E2M1 codes of eight quotients (four packed pairs) as one word, lowest
// nibble first, rounded to nearest even with saturation to 6. Each quotient
// first takes the sign bit of its dividend (sv: bit patterns), as in
// e2m1_pair below.
__device__ __forceinline__ uint32_t e2m1x8(const uint64_t *q, const float *sv) {
    float f[8];
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        const float2 t = up2(q[p]);
        f[2 * p] = __uint_as_float(__float_as_uint(t.x) | (__float_as_uint(sv[2 * p]) & 0x80000000u));
        f[2 * p + 1] = __uint_as_float(__float_as_uint(t.y) | (__float_as_uint(sv[2 * p + 1]) & 0x80000000u));
    }
    uint32_t r;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(r)
        : "f"(f[0]), "f"(f[1]), "f"(f[2]), "f"(f[3]), "f"(f[4]), "f"(f[5]), "f"(f[6]), "f"(f[7]));
    return r;
}

// E2M1 codes of eight quotients (four packed pairs) as one word, lowest
// nibble first, each with the sign of its quotient as it stands (the
// conversion keeps the sign of zeros and of values rounding to zero).
__device__ __forceinline__ uint32_t e2m1x8_as_is(const uint64_t *q) {
    float f[8];
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        const float2 t = up2(q[p]);
        f[2 * p] = t.x;
        f[2 * p + 1] = t.y;
    }
    uint32_t r;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(r)
        : "f"(f[0]), "f"(f[1]), "f"(f[2]), "f"(f[3]), "f"(f[4]), "f"(f[5]), "f"(f[6]), "f"(f[7]));
    return r;
}

// E2M1 codes of RN32(v_i / d) for eight values, lowest nibble first, for
// d in [2^-90, 2^90] with y = RN(1/d), ylo = RN(y (1 - 2^-21)) and
// yhi = RN(y (1 + 2^-21)) (packed pairs yl2, yh2, y2; d2 = (d, d),
// nd2 = (-d, -d)). Each relative error below is at most 2^-24 (RN of a
// normal number), so for v > 0
//   RN(v ylo) <= (v / d)(1 + 2^-24)^3 (1 - 2^-21) < v / d,
//   RN(v yhi) >= (v / d)(1 - 2^-24)^3 (1 + 2^-21) > v / d
// (mirrored for v < 0): the two products bracket the exact quotient, hence
// also RN32(v / d). Rounding to binary32 and encoding to E2M1 are both
// monotone, so when the two products give the same code word, every value
// between them has that code, RN32(v / d) included; where a product falls
// below the normal range, both it and the quotient are far below 1/4 and
// all of them give the zero code of v's sign. Products keep the sign of a
// zero dividend. Otherwise (a quotient within about 2^-21 of a rounding
// boundary) the correctly rounded quotients of div2 decide.
__device__ __forceinline__ uint32_t e2m1x8_div(const float *v, uint64_t yl2, uint64_t yh2, uint64_t d2, uint64_t nd2,
                                               uint64_t y2) {
    uint64_t ql[4], qh[4];
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        const uint64_t vv = pk2(v[2 * p], v[2 * p + 1]);
        ql[p] = mul2(vv, yl2);
        qh[p] = mul2(vv, yh2);
    }
    const uint32_t c = e2m1x8_as_is(ql);
    if (c == e2m1x8_as_is(qh)) return c;
    uint64_t q[4];
#pragma unroll
    for (int p = 0; p < 4; ++p) q[p] = div2(pk2(v[2 * p], v[2 * p + 1]), d2, nd2, y2);
    return e2m1x8(q, v);
}

// E2M1 byte of two quotients (lo nibble = q.x), rounded to nearest even with
// saturation to 6 by the hardware conversion, which keeps the sign of zeros.
// The quotients first take the sign bits of their dividends (sign_lo,
// sign_hi: bit patterns): that is the sign of the exact quotient, also where
// a zero dividend's quotient came out of the division as +0.
__device__ __forceinline__ uint32_t e2m1_pair(uint64_t q, uint32_t sign_lo, uint32_t sign_hi) {
    const float2 f = up2(q);
    const float lo = __uint_as_float(__float_as_uint(f.x) | (sign_lo & 0x80000000u));
    const float hi = __uint_as_float(__float_as_uint(f.y) | (sign_hi & 0x80000000u));
    uint32_t b;
    asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tcvt.u32.u8 %0, t;\n\t}"
        : "=r"(b) : "f"(hi), "f"(lo));
    return b;
}

// ---------------------------------------------------------------------------
// Programmatic dependent launch. A kernel launched with programmatic stream
// serialization may start while the kernel before it in the stream is still
// running; griddep_wait blocks until that kernel has completed and its memory
// is visible, so everything before it must not read what the previous kernel
// writes. griddep_launch lets the next kernel (if launched that way) start
// its own launch and set-up early.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// 32 bytes of global memory (p 32-byte aligned), streaming: read once.
__device__ __forceinline__ void ldg256_cs(const void *p, uint32_t (&r)[8]) {
    asm volatile("ld.global.cs.v8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "l"(p));
}

// ---------------------------------------------------------------------------
// Shared-memory and barrier primitives

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

// Per-thread asynchronous 16-byte copies global -> shared (L2 only), grouped
// by commit; wait_group<N> returns once at most N of this thread's groups are
// still in flight, after which the thread may read what it copied.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_fence_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait on a phase of an mbarrier. Gives up after `limit_ns` of
// global time, or as soon as another thread has recorded a status, and then
// records `site` (first writer wins) and returns false.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, unsigned *status, unsigned site,
                                          uint64_t limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 63u) == 0) {
            if (read_status(status) != 0u) return false;
            if (globaltimer_ns() - t0 > limit_ns) {
                record_status(status, site);
                return false;
            }
        }
    }
}

// ---------------------------------------------------------------------------
// Grouped (mixture-of-experts) launches. Group g owns grouped rows
// offsets[g] .. offsets[g+1]-1 and, in a grouped prep, the 128-row tiles
// tiles[g] .. tiles[g+1]-1, where tiles[g] counts ceil(size / 128) over the
// groups before g.

// Device-side argument codes (status word values 0x2xx).
enum : unsigned { kSiteBadOffsets = 0x201, kSiteBadRowIndex = 0x202 };

// Builds tiles[0 .. groups] in shared memory with the calling warp (all 32
// lanes must call). Returns, in every lane, whether the offsets are valid:
// offsets[0] == 0, nondecreasing, offsets[groups] == rows, and the padded
// rows 128 * tiles[groups] fit in cap_rows. Counts are clamped while
// scanning, so nothing overflows on invalid input; the table is then unused.
__device__ __forceinline__ bool build_tile_table(const int32_t *offsets, int groups, int64_t rows, int64_t cap_rows,
                                                 int32_t *tiles) {
    const int lane = threadIdx.x & 31;
    bool ok = offsets[0] == 0 && (int64_t)offsets[groups] == rows;
    int64_t carry = 0;
    if (lane == 0) tiles[0] = 0;
    for (int base = 0; base < groups; base += 32) {
        const int g = base + lane;
        int32_t t = 0;
        if (g < groups) {
            const int32_t a = offsets[g], b = offsets[g + 1];
            if (b < a) ok = false;
            const int64_t c = b >= a ? min((int64_t)b - a, rows) : 0;
            t = (int32_t)((c + 127) >> 7);
        }
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int32_t v = __shfl_up_sync(0xFFFFFFFFu, t, o);
            if (lane >= o) t += v;
        }
        if (g < groups) tiles[g + 1] = (int32_t)min(carry + t, (int64_t)0x7FFFFFFF);
        carry += __shfl_sync(0xFFFFFFFFu, t, 31);
    }
    if (carry * 128 > cap_rows) ok = false;
    return __all_sync(0xFFFFFFFFu, ok);
}

// The group whose tiles hold 128-row tile `tile` (< tiles[groups]): the
// largest g with tiles[g] <= tile (empty groups own no tile).
__device__ __forceinline__ int group_of_tile(const int32_t *tiles, int groups, int32_t tile) {
    int lo = 0, hi = groups;  // tiles[lo] <= tile < tiles[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (tiles[mid] <= tile) lo = mid;
        else hi = mid;
    }
    return lo;
}

// ---------------------------------------------------------------------------
// TMA and bulk copies (no multicast anywhere in this library).

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const void *tmap, int32_t c0, int32_t c1, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(tmap), "r"(c0), "r"(c1), "r"(bar)
        : "memory");
}

// 3-D tile load: coordinates (c0 innermost, c1, c2).
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const void *tmap, int32_t c0, int32_t c1, int32_t c2,
                                            uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
        "l"(tmap), "r"(c0), "r"(c1), "r"(c2), "r"(bar)
        : "memory");
}

__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const void *tmap) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(tmap) : "memory");
}

// ---------------------------------------------------------------------------
// Thread-block clusters (split-K reduction through distributed shared memory).

__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// Every thread of every CTA in the cluster: arrive (release), then wait
// (acquire).
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// The two halves of a cluster barrier: arrive without ordering (marks this
// thread as started; nothing before it needs to be visible), and the wait
// that returns once every thread of the cluster has arrived. After the wait,
// every CTA of the cluster is running, so its shared memory may be written.
__device__ __forceinline__ void cluster_arrive_relaxed() {
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.aligned;" ::: "memory"); }

// Store to shared memory of another CTA of the cluster (a mapa address).
__device__ __forceinline__ void st_cluster_u32(uint32_t addr, uint32_t v) {
    asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

// Address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}

__device__ __forceinline__ uint32_t ld_cluster_u32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
    return v;
}

__device__ __forceinline__ float4 ld_cluster_f4(uint32_t addr) {
    float4 v;
    asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(addr)
                 : "memory");
    return v;
}

// ---------------------------------------------------------------------------
// tcgen05 (5th-generation tensor core) wrappers, cta_group::1.

__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Arrive on `bar` once every tcgen05 operation this thread issued so far
// has completed.
__device__ __forceinline__ void tc_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

// Shared-memory matrix descriptor (tcgen05 format, version 1).
//   start: byte address >> 4 (bits 0-13); lbo: bits 16-29; sbo: bits 32-45;
//   version 1 at bits 46-47; layout type at bits 61-63 (2 = 128-byte swizzle,
//   0 = no swizzle).
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo_bytes, uint32_t sbo_bytes,
                                              uint32_t layout) {
    uint64_t d = (uint64_t)((addr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
    d |= 1ull << 46;
    d |= (uint64_t)layout << 61;
    return d;
}

// D[tmem] (+)= A[smem] * B[smem]^T with per-16 UE4M3 block scales (NVFP4).
__device__ __forceinline__ void tc_mma_nvf4(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                            uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
            d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
        : "memory");
}

// Same with per-32 E8M0 block scales (MXFP4).
__device__ __forceinline__ void tc_mma_mxf4(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                            uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.scale_vec::2X [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
            d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
        : "memory");
}

// Structured-sparse forms (pair-wise 4:8 A): D[tmem] (+)= A * B^T over 128
// logical K values, A's 64 kept values per row read from shared memory (the
// descriptor's K-compacted tile), its metadata (4 bits per group of 8, one
// row per tensor-memory lane, two columns per MMA) at e_tmem; one scale per
// 32 logical values (NVFP4: UE4M3) or per 64 (MXFP4: E8M0) on both operands.
__device__ __forceinline__ void tc_mma_sp_nvf4(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                               uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t e_tmem,
                                               uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.sp.cta_group::1.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], %1, %2, [%7], %3, [%5], [%6], p;\n\t}" ::"r"(
            d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem), "r"(e_tmem)
        : "memory");
}

__device__ __forceinline__ void tc_mma_sp_mxf4(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                               uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t e_tmem,
                                               uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.sp.cta_group::1.kind::mxf4.block_scale.scale_vec::2X [%0], %1, %2, [%7], %3, [%5], [%6], p;\n\t}" ::"r"(
            d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem), "r"(e_tmem)
        : "memory");
}

// ---------------------------------------------------------------------------
// CTA pairs (cta_group::2): one MMA over a 256-row tile whose A rows and W
// rows are split between the two CTAs of a cluster pair, issued by the even
// CTA. Its barriers collect both CTAs' copies and arrivals.

// Tensor-memory allocation shared by the pair (issued by the same warp of
// both CTAs, same destination slot).
__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// Tile load into this CTA's shared memory whose completed bytes count on a
// barrier of either CTA of the pair (bar: a shared::cluster address).
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const void *tmap, int32_t c0, int32_t c1, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(tmap), "r"(c0), "r"(c1), "r"(bar)
        : "memory");
}

// Arrive on a barrier of a CTA of the cluster (bar: a shared::cluster address).
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t bar) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar) : "memory");
}

// Arrive on the barrier at `bar` (this CTA's offset) in every CTA of `mask`
// once the pair MMAs this thread issued have completed.
__device__ __forceinline__ void tc_commit_pair(uint32_t bar, uint16_t mask) {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
                     bar),
                 "h"(mask)
                 : "memory");
}

__device__ __forceinline__ void tc_mma_nvf4_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                                 uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
            d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
        : "memory");
}

__device__ __forceinline__ void tc_mma_mxf4_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                                 uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::mxf4.block_scale.scale_vec::2X [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
            d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
        : "memory");
}

// 32 consecutive fp32 columns of this warp's 32 tensor-memory lanes.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}

// 16 consecutive fp32 columns of this warp's 32 tensor-memory lanes.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// 4 consecutive 32-bit columns of this warp's 32 tensor-memory lanes, from
// 4 registers per lane.
__device__ __forceinline__ void tmem_st4(uint32_t taddr, const uint4 &v) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1, %2, %3, %4};" ::"r"(taddr), "r"(v.x), "r"(v.y),
                 "r"(v.z), "r"(v.w)
                 : "memory");
}

// 2 consecutive 32-bit columns of this warp's 32 tensor-memory lanes.
__device__ __forceinline__ void tmem_st2(uint32_t taddr, uint32_t a, uint32_t b) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x2.b32 [%0], {%1, %2};" ::"r"(taddr), "r"(a), "r"(b) : "memory");
}

__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Store 32 bytes (one full sector) to global memory; p 32-byte aligned.
__device__ __forceinline__ void stg256(void *p, uint32_t a, uint32_t b, uint32_t c, uint32_t d, uint32_t e,
                                       uint32_t f, uint32_t g, uint32_t h) {
    asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(a), "r"(b), "r"(c),
                 "r"(d), "r"(e), "r"(f), "r"(g), "r"(h)
                 : "memory");
}

// Store 16 bytes to shared memory.
__device__ __forceinline__ void sts128(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

// 16 bytes of shared memory.
__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
    return v;
}

}  // namespace sq

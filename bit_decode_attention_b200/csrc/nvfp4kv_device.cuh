// nvfp4kv_device.cuh -- device-side building blocks of libnvfp4kv.so:
// E4M3 / E2M1 conversions written from the format definitions, the per-block
// FP8 lookup used to dequantize NVFP4 codes, and thin PTX wrappers for the
// sm_100a instructions the kernels use (mbarrier, bulk async copy, warp MMA,
// movmatrix).
//
// Formats ("NVIDIA解説: NVFP4 KV Cacheで長コンテキストLLM推論を最適化",
// section "E2M1 + 2レベルスケーリング"): E2M1 elements (sign/exp2/mant1,
// range +-6), one E4M3 scale per 16 elements, one fp32 tensor scale.
// E4M3 is the OCP E4M3FN byte: bias 7, largest finite 448, S.1111.111 = NaN.
#pragma once

#include <cmath>
#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/nvfp4kv.h"

namespace nvfp4kv {

// ---------------------------------------------------------------------------
// Division by a launch-invariant divisor (T. Granlund and P. Montgomery,
// "Division by Invariant Integers using Multiplication", 1994): for
// 1 <= d < 2^31 and 0 <= x < 2^31, x / d = (umulhi(x, m) + x) >> l with
// l = ceil(log2 d) and m = floor(2^32 (2^l - d) / d) + 1 (mod 2^32).  A
// runtime 32-bit division is a software routine of a few dozen instructions;
// this is two.  (umulhi(x, m) <= x, so the sum stays below 2^32.)
// ---------------------------------------------------------------------------
struct FastDiv {
    uint32_t d, m, l;
    FastDiv() = default;
    __host__ explicit FastDiv(uint32_t d_) : d(d_), m(0), l(0) {
        while ((1ull << l) < d) ++l;
        m = (uint32_t)((((1ull << 32) * ((1ull << l) - d)) / d + 1) & 0xFFFFFFFFull);
    }
    __host__ __device__ __forceinline__ uint32_t div(uint32_t x) const {
#ifdef __CUDA_ARCH__
        return (__umulhi(x, m) + x) >> l;
#else
        return (uint32_t)((((uint64_t)x * m) >> 32) + x) >> l;
#endif
    }
};

// ---------------------------------------------------------------------------
// status word: the first error wins
// ---------------------------------------------------------------------------
__device__ __forceinline__ void report(int32_t* status, int32_t code) {
    if (status != nullptr) atomicCAS(status, 0, code);
}

// ---------------------------------------------------------------------------
// E4M3 (E4M3FN) conversions
// ---------------------------------------------------------------------------
// float -> E4M3 byte, round to nearest (ties to even), finite overflow
// saturates to +-448, NaN -> 0x7F.  Integer rounding of the fp32 bit pattern:
// for normal results the 23-bit fraction is rounded to 3 bits (carry into the
// exponent is the correct next binade); below 2^-6 the result is a multiple
// of 2^-9 and |v| * 2^9 is rounded to an integer 0..8 (8 encodes 2^-6).
__device__ __forceinline__ uint32_t e4m3_from_float(float v) {
    const uint32_t bits = __float_as_uint(v);
    const uint32_t sign = (bits >> 24) & 0x80u;
    const uint32_t a = bits & 0x7FFFFFFFu;
    if (a > 0x7F800000u) return 0x7Fu;                 // NaN
    if (a >= 0x43E00000u) return sign | 0x7Eu;         // |v| >= 448 (incl. inf)
    if (a >= 0x3C800000u) {                            // |v| >= 2^-6: normal
        const uint32_t odd = (a >> 20) & 1u;
        uint32_t r = (a + 0x7FFFFu + odd) >> 20;       // exp32:3 | mant3, rounded
        r -= (127u - 7u) << 3;                         // rebias 127 -> 7
        return sign | (r > 0x7Eu ? 0x7Eu : r);
    }
    const float scaled = __uint_as_float(a) * 512.0f;  // exact (power of two)
    return sign | __float2uint_rn(scaled);             // 0..8, ties to even
}

// E4M3 byte (not NaN) -> float, exact.
__device__ __forceinline__ float e4m3_to_float(uint32_t b) {
    const uint32_t e = (b >> 3) & 0xFu;
    const uint32_t m = b & 7u;
    const float mag = (e == 0) ? (float)m * 0.001953125f                       // m * 2^-9
                               : __uint_as_float(((e + 120u) << 23) | (m << 20));
    return (b & 0x80u) ? -mag : mag;
}

// ---------------------------------------------------------------------------
// E2M1 conversions
// ---------------------------------------------------------------------------
// |code| -> value: 0, 0.5, 1, 1.5, 2, 3, 4, 6
__device__ __forceinline__ float e2m1_magnitude(uint32_t m3) {
    // exponent field e = m3 >> 1, mantissa bit = m3 & 1 (bias 1; e == 0 subnormal)
    const uint32_t e = m3 >> 1, mb = m3 & 1u;
    return e == 0 ? 0.5f * (float)mb : (1.0f + 0.5f * (float)mb) * (float)(1u << (e - 1));
}

// float -> E2M1 code: nearest grid value, ties to the even code, saturating at
// +-6; the sign bit is copied (negative values rounding to 0 give 0x8).  The
// comparisons are against the exact midpoints of the grid, strict where the
// lower neighbour has the even code and inclusive where the upper one has.
// NaN gives 0x7.
__device__ __forceinline__ uint32_t e2m1_from_float(float y) {
    if (y != y) return 0x7u;
    const float a = fabsf(y);
    uint32_t c = (a > 0.25f) + (a >= 0.75f) + (a > 1.25f) + (a >= 1.75f) +
                 (a > 2.5f) + (a >= 3.5f) + (a > 5.0f);
    return c | ((__float_as_uint(y) >> 28) & 0x8u);
}

// Two finite floats -> two E2M1 codes in one byte (lo in the low nibble), by
// the hardware conversion: round to nearest even, saturating at +-6, the sign
// kept on zero -- the rule of e2m1_from_float for every finite input.
__device__ __forceinline__ uint32_t e2m1x2_from_floats(float lo, float hi) {
    uint32_t r;
    asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tcvt.u32.u8 %0, t;\n\t}"
        : "=r"(r)
        : "f"(hi), "f"(lo));
    return r;
}

// Two lanes of fp32 in one 64-bit register, for the paired IEEE arithmetic
// of sm_100 (each lane rounded to nearest even on its own, no flush to zero).
__device__ __forceinline__ uint64_t f32x2_pack(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f32x2_unpack(uint64_t x, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(x));
}
__device__ __forceinline__ uint64_t f32x2_mul(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t f32x2_fma(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}

// a / b rounded to nearest even, from y = RN(1/b), for normal b and normal
// y with no overflow: Markstein's division by correction (P. Markstein, "IA-64
// and Elementary Functions", 2000).  One correction of q0 = RN(a y) leaves a
// quotient within one ulp of a/b, whose residual a - b q is then exact in a
// fused multiply-add; with y the correctly rounded reciprocal, the second
// correction RN(q + (a - b q) y) is the correctly rounded quotient.
// The residual is exact only while it is a multiple of 2^-149: with
// |b| >= 2^-90 that holds for every quotient of magnitude 2^-12 or more,
// which covers every rounding tie of E2M1 and of the E4M3 scale; a smaller
// quotient can be one ulp off but still lies below 2^-11, under the first tie
// of either, so its code is unchanged.  Below 2^-90 the residual underflows
// and quotients next to a tie round to the wrong side.  Above 2^125 the
// reciprocal would be subnormal.  Callers therefore divide by correction only
// for divisors in [kCorrectionMinDivisor, kCorrectionMaxDivisor].
// (Host-callable too, with the host's IEEE multiply and fused multiply-add,
// so that a host test can check the method on many quotients.)
constexpr float kCorrectionMinDivisor = 0x1p-90f;
constexpr float kCorrectionMaxDivisor = 0x1p125f;
__host__ __device__ __forceinline__ float div_rn_by_correction(float a, float b, float y) {
#ifdef __CUDA_ARCH__
    const float q0 = __fmul_rn(a, y);
    const float q1 = __fmaf_rn(__fmaf_rn(-q0, b, a), y, q0);
    return __fmaf_rn(__fmaf_rn(-q1, b, a), y, q1);
#else
    const float q0 = a * y;
    const float q1 = fmaf(fmaf(-q0, b, a), y, q0);
    return fmaf(fmaf(-q1, b, a), y, q1);
#endif
}
// The same for two dividends at once (yy = (y, y), nb = (-b, -b)); the
// quotients come back with the signs of their dividends, zeros included.
__device__ __forceinline__ uint64_t div2_rn_by_correction(uint64_t a, uint64_t nb, uint64_t yy) {
    const uint64_t q0 = f32x2_mul(a, yy);
    const uint64_t q1 = f32x2_fma(f32x2_fma(q0, nb, a), yy, q0);
    const uint64_t q2 = f32x2_fma(f32x2_fma(q1, nb, a), yy, q1);
    return q2 | (a & 0x8000000080000000ull);
}

// ---------------------------------------------------------------------------
// NVFP4 quantization of one 16-element micro-block (append path; also used by
// the fused append + attention kernel)
// ---------------------------------------------------------------------------
template <bool F32>
__device__ __forceinline__ void load16(const void* x, int64_t elem, float (&v)[16]) {
    if (F32) {
        const float4* p = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(x) + elem);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float4 f = __ldg(p + j);
            v[4 * j + 0] = f.x;
            v[4 * j + 1] = f.y;
            v[4 * j + 2] = f.z;
            v[4 * j + 3] = f.w;
        }
    } else {
        const uint4* p = reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(x) + elem);
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const uint4 w = __ldg(p + j);
            const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                v[8 * j + 2 * k + 0] = __uint_as_float(ws[k] << 16);          // bf16 -> fp32, exact
                v[8 * j + 2 * k + 1] = __uint_as_float(ws[k] & 0xFFFF0000u);
            }
        }
    }
}

// Quantize one micro-block: returns the scale byte, writes 8 packed bytes.
// The codes are E2M1(RN(v / den)) element by element.  A block with a NaN or
// an infinity, a saturated scale (amax / (6 s_tensor) > 448), or a den outside
// [2^-90, 2^125] (where division by correction is not exact) takes the IEEE
// division and the comparison encoder; every other block divides by correction from
// one reciprocal and encodes two elements per hardware conversion -- the same
// codes, bit for bit.
__device__ __forceinline__ uint32_t quantize_block(const float (&v)[16], float s_tensor, uint2& packed) {
    float amax = 0.0f;
    bool nan = false;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        amax = fmaxf(amax, fabsf(v[i]));
        nan |= v[i] != v[i];
    }
    const float d6 = __fmul_rn(6.0f, s_tensor);
    const float r = __fdiv_rn(amax, d6);
    const uint32_t sb = e4m3_from_float(r);
    const float den = __fmul_rn(e4m3_to_float(sb), s_tensor);
    uint32_t lo = 0, hi = 0;
    // r <= 448 bounds every |v / den| near 6, far from overflow
    if (!nan && r <= 448.0f && den >= kCorrectionMinDivisor && den <= kCorrectionMaxDivisor) {
        const float y = __frcp_rn(den);
        uint32_t byte[8];
        // copysignf: a zero quotient keeps the sign of its dividend (the
        // corrections add +0 to -0)
#pragma unroll
        for (int k = 0; k < 8; ++k)
            byte[k] = e2m1x2_from_floats(copysignf(div_rn_by_correction(v[2 * k], den, y), v[2 * k]),
                                         copysignf(div_rn_by_correction(v[2 * k + 1], den, y), v[2 * k + 1]));
        lo = __byte_perm(byte[0] | (byte[1] << 8), byte[2] | (byte[3] << 8), 0x5410);
        hi = __byte_perm(byte[4] | (byte[5] << 8), byte[6] | (byte[7] << 8), 0x5410);
    } else {
        uint32_t c[16];
        if (den == 0.0f) {
#pragma unroll
            for (int i = 0; i < 16; ++i) c[i] = (__float_as_uint(v[i]) >> 28) & 0x8u;
        } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) c[i] = e2m1_from_float(__fdiv_rn(v[i], den));
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            lo |= c[i] << (4 * i);
            hi |= c[8 + i] << (4 * i);
        }
    }
    packed = make_uint2(lo, hi);
    return sb;
}

// ---------------------------------------------------------------------------
// NVFP4 -> FP8 lookup
// ---------------------------------------------------------------------------
// The FP8 value of a code depends only on its 3-bit magnitude, the block's
// scale byte and the tensor scale:  E4M3(fl32(fl32(|c| * value(sb)) * s)).
// A block's 8 values fit two 32-bit words (byte m = magnitude m), which
// `byte_perm` then indexes with four 3-bit selectors at a time.
// |c| * value(sb) has at most 6 significant bits, so the first product is
// exact; the second is one fp32 rounding; the E4M3 conversion (the software
// one above, nearest even, saturating at 448) is the one the quantizer uses
// for its scale bytes, so the table needs no hardware conversion.
__device__ __forceinline__ uint2 lut_words(uint32_t sb, float s_tensor) {
    if ((sb & 0x7Fu) == 0x7Fu) return make_uint2(0u, 0u);   // never written by quantize
    const float v = e4m3_to_float(sb & 0x7Fu);
    uint32_t b[8];
#pragma unroll
    for (int m = 0; m < 8; ++m)
        b[m] = e4m3_from_float(__fmul_rn(__fmul_rn(e2m1_magnitude((uint32_t)m), v), s_tensor));
    return make_uint2(b[0] | (b[1] << 8) | (b[2] << 16) | (b[3] << 24),
                      b[4] | (b[5] << 8) | (b[6] << 16) | (b[7] << 24));
}

// Dequantize 8 packed codes (one 32-bit word; element k in nibble k) to 8 FP8
// bytes with the block's lookup words (lut_lo = magnitudes 0..3, lut_hi =
// 4..7).  out_lo = elements 0..3, out_hi = elements 4..7 (byte k = element k).
//   - magnitudes: byte_perm selects one lookup byte per 3-bit selector;
//   - signs: nibble msb k sits at bit 4k+3 and must land at bit 8k+7; the
//     byte permutes of (x << 4, x) move bits 3/7/11/15 (19/23/27/31) there.
__device__ __forceinline__ void dequant_word(uint32_t x, uint32_t lut_lo, uint32_t lut_hi,
                                             uint32_t& out_lo, uint32_t& out_hi) {
    const uint32_t sel_lo = x & 0x77777777u;
    const uint32_t sel_hi = __umulhi(sel_lo, 0x10000u);   // >> 16 on the multiply pipe
    const uint32_t mag_lo = __byte_perm(lut_lo, lut_hi, sel_lo);
    const uint32_t mag_hi = __byte_perm(lut_lo, lut_hi, sel_hi);
    const uint32_t xs = x * 16u;
    const uint32_t sgn_lo = __byte_perm(xs, x, 0x5140u);
    const uint32_t sgn_hi = __byte_perm(xs, x, 0x7362u);
    out_lo = mag_lo | (sgn_lo & 0x80808080u);
    out_hi = mag_hi | (sgn_hi & 0x80808080u);
}

// ---------------------------------------------------------------------------
// small PTX wrappers (sm_90+ / sm_100a)
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
                 : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// try_wait with a suspend-time hint: the thread may sleep up to `hint_ns`
// nanoseconds waiting for the phase instead of returning at once.
__device__ __forceinline__ bool mbar_try_wait_hint(uint64_t* bar, uint32_t parity, uint32_t hint_ns) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
        : "memory");
    return ok != 0;
}

// Bounded wait that sleeps between polls: at most `limit` polls of up to
// 20 us each.
__device__ __forceinline__ bool mbar_wait_sleep(uint64_t* bar, uint32_t parity, uint32_t limit) {
    for (uint32_t i = 0; i < limit; ++i)
        if (mbar_try_wait_hint(bar, parity, 20000u)) return true;
    return false;
}

// Wait for the phase with the given parity to complete; give up after
// `limit` polls (each poll may suspend the thread for a short while).
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, uint32_t limit) {
    for (uint32_t i = 0; i < limit; ++i)
        if (mbar_try_wait(bar, parity)) return true;
    return false;
}

// 1-D bulk copy global -> this CTA's shared memory, completing on `bar`.
// dst, src and bytes must be multiples of 16.  No cluster multicast.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
            "r"(smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// Order this thread's earlier generic-proxy shared-memory accesses before
// later async-proxy (bulk copy) writes to the same memory.
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Four E4M3 bytes -> two f16x2 (exact): lo = bytes (0, 1), hi = bytes (2, 3),
// the lower-addressed byte in the low half.
__device__ __forceinline__ void e4m3x4_to_f16x2x2(uint32_t x, uint32_t& lo, uint32_t& hi) {
    asm("{\n\t.reg .b16 a, b;\n\tmov.b32 {a, b}, %2;\n\t"
        "cvt.rn.f16x2.e4m3x2 %0, a;\n\tcvt.rn.f16x2.e4m3x2 %1, b;\n\t}"
        : "=r"(lo), "=r"(hi)
        : "r"(x));
}

// Two floats -> two E4M3 bytes (lo in the low byte), round to nearest even,
// finite overflow saturates.  Used for query operands only.
__device__ __forceinline__ uint32_t e4m3x2_from_floats(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// Two floats -> f16x2 (lo in the low half), round to nearest even.
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

__device__ __forceinline__ float f16_lo_to_float(uint32_t x) {
    float f;
    asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %1;\n\tcvt.f32.f16 %0, l;\n\t}" : "=f"(f) : "r"(x));
    return f;
}
__device__ __forceinline__ float f16_hi_to_float(uint32_t x) {
    float f;
    asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %1;\n\tcvt.f32.f16 %0, h;\n\t}" : "=f"(f) : "r"(x));
    return f;
}

// 8x8 b16 matrix transpose across the warp (fragment layout: lane holds row
// lane/4, columns 2*(lane%4), +1).
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
    uint32_t r;
    asm("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(r) : "r"(x));
    return r;
}

// D += A(16x16, f16, row) * B(16x8, f16, col), fp32 accumulate.
__device__ __forceinline__ void mma_f16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                              uint32_t a3, uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// D += A(16x32, e4m3, row) * B(32x8, e4m3, col), fp32 accumulate.
__device__ __forceinline__ void mma_e4m3_16832(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k32.row.col.f32.e4m3.e4m3.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ float fast_exp2(float x) {
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

}  // namespace nvfp4kv

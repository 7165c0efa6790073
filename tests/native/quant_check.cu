// Host-side check of two pieces of arithmetic the NVFP4 quantize kernels
// (nvfp4kv_device.cuh) take in place of runtime divisions:
//
//  * FastDiv, division by a launch-invariant divisor (Granlund and
//    Montgomery, "Division by Invariant Integers using Multiplication", 1994),
//    against the integer quotient x / d: every divisor up to 2^16 and random
//    divisors up to 2^31 - 1, with dividends at the ends of the range, around
//    every multiple tried, and at random below 2^31;
//  * div_rn_by_correction (Markstein's division by correction), against the
//    IEEE quotient a / b rounded to nearest even, over the operands the
//    quantizer gives it: block divisors b in [kCorrectionMinDivisor,
//    kCorrectionMaxDivisor] with dividends whose quotients lie near the E2M1
//    range (ties of the E2M1 grid and their neighbours included), and block
//    maxima over the whole finite range divided by 6 s.  Where the IEEE
//    quotient is at least 2^-12 and finite the two must agree bit for bit
//    (every rounding tie of E2M1 and of the E4M3 scale is at 2^-10 or
//    above); below, the method's result must be under 2^-11, which takes the
//    zero code in both formats, as the IEEE quotient does; where the IEEE
//    quotient overflows, the method's result must not pass the quantizer's
//    r <= 448 test.  Below kCorrectionMinDivisor the check counts E2M1 codes
//    that the method gets wrong next to a tie and requires some: the bound is
//    there for a reason.
//
// Compiled by nvcc (host code only runs) and run on the CPU; prints "ok" and
// exits 0 when every case agrees.
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstring>

#include "../../bit_decode_attention_b200/csrc/nvfp4kv_device.cuh"

using nvfp4kv::FastDiv;
using nvfp4kv::div_rn_by_correction;
using nvfp4kv::kCorrectionMaxDivisor;
using nvfp4kv::kCorrectionMinDivisor;

static long failures = 0, checked = 0;
#define CHECK(cond, ...)                                   \
    do {                                                   \
        ++checked;                                         \
        if (!(cond)) {                                     \
            if (failures < 20) std::printf(__VA_ARGS__);   \
            ++failures;                                    \
        }                                                  \
    } while (0)

// splitmix64 (Steele, Lea and Flood, "Fast Splittable Pseudorandom Number
// Generators", 2014)
static uint64_t rng_state = 0x5eed0f4b1dc0ffeeull;
static uint64_t next_u64() {
    uint64_t z = (rng_state += 0x9E3779B97F4A7C15ull);
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}
static uint32_t next_below(uint32_t n) { return (uint32_t)(next_u64() % n); }

static float bits_float(uint32_t u) {
    float f;
    std::memcpy(&f, &u, 4);
    return f;
}
static uint32_t float_bits(float f) {
    uint32_t u;
    std::memcpy(&u, &f, 4);
    return u;
}
// a float with the given unbiased exponent (normal range) and a random mantissa
static float random_with_exponent(int e, bool negative) {
    const uint32_t mant = (uint32_t)next_u64() & 0x7FFFFFu;
    return bits_float((negative ? 0x80000000u : 0u) | ((uint32_t)(e + 127) << 23) | mant);
}

// ---------------------------------------------------------------------------
// FastDiv
// ---------------------------------------------------------------------------
static void check_fastdiv(uint32_t d) {
    const FastDiv fd(d);
    const uint32_t top = 0x7FFFFFFFu;
    auto one = [&](uint32_t x) {
        CHECK(fd.div(x) == x / d, "FastDiv d=%u x=%u: %u vs %u\n", d, x, fd.div(x), x / d);
    };
    one(0);
    one(1);
    one(top);
    one(top - 1);
    one(d - 1);
    one(d);
    // around multiples of d spread over the range
    for (int k = 0; k < 16; ++k) {
        const uint64_t q = (uint64_t)next_below(top / d + 1);
        const uint64_t m = q * d;
        if (m <= top) one((uint32_t)m);
        if (m >= 1 && m - 1 <= top) one((uint32_t)(m - 1));
        if (m + 1 <= top) one((uint32_t)(m + 1));
    }
    for (int k = 0; k < 16; ++k) one(next_below(top) + 1u);
}

// ---------------------------------------------------------------------------
// division by correction
// ---------------------------------------------------------------------------
// one quotient: y = RN(1/b) as the quantizer computes it, the method's result
// with the sign of the dividend (as the kernels restore it), and the IEEE one
static void check_div(float a, float b) {
    const float y = 1.0f / b;
    const float q = std::copysign(div_rn_by_correction(a, b, y), a);
    const float ref = a / b;
    const float aref = std::fabs(ref);
    if (std::isinf(ref)) {
        CHECK(!(std::fabs(q) <= 448.0f), "overflow a=%a b=%a: %a passes r <= 448\n", a, b, q);
    } else if (aref < 0x1p-12f) {
        CHECK(std::fabs(q) < 0x1p-11f, "small quotient a=%a b=%a: %a vs %a\n", a, b, q, ref);
    } else {
        CHECK(float_bits(q) == float_bits(ref), "a=%a b=%a: %a vs %a\n", a, b, q, ref);
    }
}

// a divisor in the quantizer's correction range: exponent in [-90, 124]
static float random_divisor() {
    return random_with_exponent(-90 + (int)next_below(215), false);
}

// E2M1 magnitude index of x (0..7 for 0, 0.5, 1, 1.5, 2, 3, 4, 6), nearest,
// ties to the even index
static int e2m1_index(float x) {
    static const float grid[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};
    x = std::fabs(x);
    for (int i = 0; i < 7; ++i) {
        const float mid = 0.5f * (grid[i] + grid[i + 1]);
        if (x < mid) return i;
        if (x == mid) return (i % 2 == 0) ? i : i + 1;
    }
    return 7;
}

int main() {
    // FastDiv: every divisor up to 2^16, then random ones up to 2^31 - 1
    for (uint32_t d = 1; d <= 65536; ++d) check_fastdiv(d);
    for (int k = 0; k < 200000; ++k) check_fastdiv(next_below(0x7FFFFFFFu) + 1u);
    for (uint32_t d : {0x7FFFFFFFu, 0x7FFFFFFEu, 0x40000000u, 0x40000001u, 0x3FFFFFFFu, 3u, 5u, 7u, 641u, 6700417u})
        check_fastdiv(d);

    static_assert(kCorrectionMinDivisor == 0x1p-90f && kCorrectionMaxDivisor == 0x1p125f,
                  "the samplers below cover [2^-90, 2^125]");
    // element quotients: |a / b| from far below the E2M1 range to past it
    for (int k = 0; k < 3000000; ++k) {
        const float b = random_divisor();
        const int ea = (int)((float_bits(b) >> 23) & 0xFF) - 127 - 24 + (int)next_below(28);
        if (ea < -126) continue;
        check_div(random_with_exponent(ea, next_u64() & 1), b);
    }
    // rounding ties of E2M1 with full-mantissa divisors: a = RN(t b) and its
    // neighbours put a / b within a few ulps of the tie t
    const float e2m1_ties[] = {0.25f, 0.75f, 1.25f, 1.75f, 2.5f, 3.5f, 5.0f};
    for (int k = 0; k < 1000000; ++k) {
        const float b = random_divisor();
        const float a = e2m1_ties[next_below(7)] * b;
        for (int s = -2; s <= 2; ++s) check_div(bits_float(float_bits(a) + (uint32_t)s), b);
    }
    // exact E2M1 rounding ties (and their neighbours) times divisors with
    // short mantissas, where t * b is exact
    const float ties[] = {0.25f, 0.75f, 1.25f, 1.75f, 2.5f, 3.5f, 5.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};
    for (int k = 0; k < 400000; ++k) {
        const int eb = -90 + (int)next_below(215);
        const uint32_t mant = ((uint32_t)next_u64() & 0xFFFFu) << 7;   // 16 mantissa bits
        const float b = bits_float(((uint32_t)(eb + 127) << 23) | mant);
        const float t = ties[next_below(sizeof(ties) / sizeof(ties[0]))];
        const float a = t * b;                                    // exact: 3 + 17 bits
        for (int s = -3; s <= 3; ++s) {
            const float as = bits_float(float_bits(a) + (uint32_t)s);
            check_div(as, b);
            check_div(-as, b);
        }
    }
    // subnormal and zero dividends (inputs of any magnitude reach a block)
    for (int k = 0; k < 200000; ++k) {
        const float b = random_divisor();
        const float a = bits_float((uint32_t)(next_u64() & 0x7FFFFFu) | ((next_u64() & 1) ? 0x80000000u : 0u));
        check_div(a, b);
    }
    check_div(0.0f, 1.0f);
    check_div(-0.0f, 0x1p-90f);
    // rounding ties of the E4M3 scale (normal ones (1 + (2m+1)/16) 2^e and
    // subnormal ones (2k+1) 2^-10) for r = amax / d6, and their neighbours
    for (int k = 0; k < 1000000; ++k) {
        const float d6 = random_divisor();
        float t;
        if (next_below(4) == 0) {
            t = (float)(2 * next_below(8) + 1) * 0x1p-10f;
        } else {
            t = std::ldexp(1.0f + (float)(2 * next_below(8) + 1) / 16.0f, -6 + (int)next_below(15));
        }
        const float a = t * d6;
        if (std::isinf(a)) continue;
        for (int s = -2; s <= 2; ++s) check_div(bits_float(float_bits(a) + (uint32_t)s), d6);
    }
    // block maxima over the whole finite range divided by d6 = 6 s
    for (int k = 0; k < 2000000; ++k) {
        const float d6 = random_divisor();
        const float amax = random_with_exponent(-126 + (int)next_below(254), false);
        check_div(amax, d6);
    }
    check_div(3.4028234663852886e38f, 0x1p-90f);
    check_div(3.4028234663852886e38f, 0x1p125f);
    check_div(0x1p-126f, 0x1p125f);
    check_div(0x1p-149f, 0x1p-90f);
    check_div(0x1.fffffep-91f * 0.75f, 0x1.fffffep-91f);

    // below the range the residual underflows and E2M1 codes next to a tie
    // come out wrong: divisors in [2^-125, 2^-90)
    long flips = 0;
    for (int k = 0; k < 200000; ++k) {
        const float b = random_with_exponent(-125 + (int)next_below(35), false);
        const float a0 = e2m1_ties[next_below(7)] * b;
        for (int s = -2; s <= 2; ++s) {
            const float a = bits_float(float_bits(a0) + (uint32_t)s);
            flips += e2m1_index(div_rn_by_correction(a, b, 1.0f / b)) != e2m1_index(a / b);
        }
    }
    std::printf("%ld E2M1 codes wrong with divisors below the range\n", flips);
    CHECK(flips > 0, "no wrong code below the range: the bound is not what limits the method\n");

    std::printf("%ld checks, %ld failures\n", checked, failures);
    if (failures) return 1;
    std::printf("ok\n");
    return 0;
}

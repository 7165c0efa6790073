// GPU side of the exhaustive check of the format conversions the kernels use
// (nvfp4kv_device.cuh), hardware and software:
//
//  * e2m1x2_from_floats (cvt.rn.satfinite.e2m1x2.f32): the E2M1 codes of the
//    quantizer's fast path;
//  * e4m3x2_from_floats (cvt.rn.satfinite.e4m3x2.f32): the E4M3 terms of the
//    query and probability splits of the attention kernels;
//  * e4m3x4_to_f16x2x2 (cvt.rn.f16x2.e4m3x2): the exact FP8 -> f16 decode of
//    those splits;
//  * e2m1_from_float and e4m3_from_float, the software encoders of the
//    quantizer's general path, its scale bytes and the dequant tables;
//    e4m3_to_float and e2m1_magnitude, the software decoders.
//
// The test compiles this file into a shared library, calls it on device
// buffers and compares the bytes with the oracle's encoders, one chunk of
// fp32 bit patterns at a time, until every pattern has been converted.
#include <cstdint>
#include <cuda_runtime.h>

#include "../../bit_decode_attention_b200/csrc/nvfp4kv_device.cuh"

using namespace nvfp4kv;

namespace {

// patterns first .. first + 2 n_pairs - 1; pattern first + j goes to byte j
// of each output: hardware E2M1, hardware E4M3, software E2M1, software E4M3
__global__ void encode_patterns_kernel(uint32_t first, uint32_t n_pairs, uint8_t* hw_e2m1, uint8_t* hw_e4m3,
                                       uint8_t* sw_e2m1, uint8_t* sw_e4m3) {
    const uint32_t stride = gridDim.x * blockDim.x;
    for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < n_pairs; i += stride) {
        const float lo = __uint_as_float(first + 2u * i);
        const float hi = __uint_as_float(first + 2u * i + 1u);
        const uint32_t c = e2m1x2_from_floats(lo, hi);
        const uint32_t b = e4m3x2_from_floats(lo, hi);
        hw_e2m1[2u * i] = (uint8_t)(c & 0xFu);
        hw_e2m1[2u * i + 1u] = (uint8_t)((c >> 4) & 0xFu);
        hw_e4m3[2u * i] = (uint8_t)(b & 0xFFu);
        hw_e4m3[2u * i + 1u] = (uint8_t)((b >> 8) & 0xFFu);
        sw_e2m1[2u * i] = (uint8_t)e2m1_from_float(lo);
        sw_e2m1[2u * i + 1u] = (uint8_t)e2m1_from_float(hi);
        sw_e4m3[2u * i] = (uint8_t)e4m3_from_float(lo);
        sw_e4m3[2u * i + 1u] = (uint8_t)e4m3_from_float(hi);
    }
}

// out[0..255]: the 256 E4M3 bytes through the hardware f16 decode, widened to
// fp32 (exact); out[256..511]: the same bytes through e4m3_to_float (0 for
// the two NaN bytes, which it does not take); out[512..519]: e2m1_magnitude
// of the magnitude codes 0..7
__global__ void decode_bytes_kernel(float* out) {
    const uint32_t t = threadIdx.x;                      // 64 threads, 4 bytes each
    const uint32_t x = (4u * t) | ((4u * t + 1u) << 8) | ((4u * t + 2u) << 16) | ((4u * t + 3u) << 24);
    uint32_t lo, hi;
    e4m3x4_to_f16x2x2(x, lo, hi);
    out[4u * t] = f16_lo_to_float(lo);
    out[4u * t + 1u] = f16_hi_to_float(lo);
    out[4u * t + 2u] = f16_lo_to_float(hi);
    out[4u * t + 3u] = f16_hi_to_float(hi);
    for (uint32_t j = 0; j < 4; ++j) {
        const uint32_t byte = 4u * t + j;
        out[256u + byte] = (byte & 0x7Fu) == 0x7Fu ? 0.0f : e4m3_to_float(byte);
    }
    if (t < 8) out[512u + t] = e2m1_magnitude(t);
}

}  // namespace

// The four conversions of the n fp32 patterns first .. first + n - 1 into
// n-byte device buffers; n and first even, first + n <= 2^32.  Returns the
// CUDA error (0 = success) after the kernel has finished, -1 for bad
// arguments.
extern "C" int sweep_encode_patterns(uint32_t first, uint64_t n, uint8_t* d_hw_e2m1, uint8_t* d_hw_e4m3,
                                     uint8_t* d_sw_e2m1, uint8_t* d_sw_e4m3) {
    if (n == 0 || (n & 1u) || (first & 1u) || (uint64_t)first + n > (1ull << 32) || !d_hw_e2m1 || !d_hw_e4m3 ||
        !d_sw_e2m1 || !d_sw_e4m3)
        return -1;
    encode_patterns_kernel<<<148 * 8, 256>>>(first, (uint32_t)(n / 2), d_hw_e2m1, d_hw_e4m3, d_sw_e2m1,
                                             d_sw_e4m3);
    cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    return (int)e;
}

// the decoded values of decode_bytes_kernel into a 520-float device buffer
extern "C" int sweep_decode_bytes(float* d_out) {
    if (!d_out) return -1;
    decode_bytes_kernel<<<1, 64>>>(d_out);
    cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    return (int)e;
}

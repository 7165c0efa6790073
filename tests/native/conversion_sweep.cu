// GPU side of the exhaustive check of the hardware format conversions the
// kernels use (nvfp4kv_device.cuh):
//
//  * e2m1x2_from_floats (cvt.rn.satfinite.e2m1x2.f32): the E2M1 codes of the
//    quantizer's fast path;
//  * e4m3x2_from_floats (cvt.rn.satfinite.e4m3x2.f32): the E4M3 terms of the
//    query and probability splits of the attention kernels;
//  * e4m3x4_to_f16x2x2 (cvt.rn.f16x2.e4m3x2): the exact FP8 -> f16 decode of
//    those splits.
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
__global__ void encode_patterns_kernel(uint32_t first, uint32_t n_pairs, uint8_t* e2m1, uint8_t* e4m3) {
    const uint32_t stride = gridDim.x * blockDim.x;
    for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < n_pairs; i += stride) {
        const float lo = __uint_as_float(first + 2u * i);
        const float hi = __uint_as_float(first + 2u * i + 1u);
        const uint32_t c = e2m1x2_from_floats(lo, hi);
        const uint32_t b = e4m3x2_from_floats(lo, hi);
        e2m1[2u * i] = (uint8_t)(c & 0xFu);
        e2m1[2u * i + 1u] = (uint8_t)((c >> 4) & 0xFu);
        e4m3[2u * i] = (uint8_t)(b & 0xFFu);
        e4m3[2u * i + 1u] = (uint8_t)((b >> 8) & 0xFFu);
    }
}

// the 256 E4M3 bytes through the f16 decode, widened to fp32 (exact)
__global__ void decode_bytes_kernel(float* out) {
    const uint32_t t = threadIdx.x;                      // 64 threads, 4 bytes each
    const uint32_t x = (4u * t) | ((4u * t + 1u) << 8) | ((4u * t + 2u) << 16) | ((4u * t + 3u) << 24);
    uint32_t lo, hi;
    e4m3x4_to_f16x2x2(x, lo, hi);
    out[4u * t] = f16_lo_to_float(lo);
    out[4u * t + 1u] = f16_hi_to_float(lo);
    out[4u * t + 2u] = f16_lo_to_float(hi);
    out[4u * t + 3u] = f16_hi_to_float(hi);
}

}  // namespace

// E2M1 codes and E4M3 bytes of the n fp32 patterns first .. first + n - 1
// into n-byte device buffers; n and first even, first + n <= 2^32.  Returns
// the CUDA error (0 = success) after the kernel has finished, -1 for bad
// arguments.
extern "C" int sweep_encode_patterns(uint32_t first, uint64_t n, uint8_t* d_e2m1, uint8_t* d_e4m3) {
    if (n == 0 || (n & 1u) || (first & 1u) || (uint64_t)first + n > (1ull << 32) || !d_e2m1 || !d_e4m3)
        return -1;
    encode_patterns_kernel<<<148 * 8, 256>>>(first, (uint32_t)(n / 2), d_e2m1, d_e4m3);
    cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    return (int)e;
}

// the 256 decoded E4M3 values into a 256-float device buffer
extern "C" int sweep_decode_bytes(float* d_out) {
    if (!d_out) return -1;
    decode_bytes_kernel<<<1, 64>>>(d_out);
    cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    return (int)e;
}

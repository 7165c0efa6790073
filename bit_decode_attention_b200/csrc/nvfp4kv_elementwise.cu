// nvfp4kv_elementwise.cu -- the HBM-bound elementwise kernels of the NVFP4
// KV cache: tensor-scale calibration, quantize-and-append, and the standalone
// NVFP4 -> FP8 dequantization.
//
// "NVIDIA解説: NVFP4 KV Cacheで長コンテキストLLM推論を最適化":
//   "E2M1 + 2レベルスケーリング" -- x ~ x_q * s_block * s_tensor, E2M1
//     elements, one E4M3 s_block per 16 elements, one FP32 s_tensor;
//   "量子化・逆量子化フロー" -- quantize new K/V to NVFP4 in 16-element
//     blocks and append; dequantize NVFP4 -> FP8 at attention time.
#include <cuda_bf16.h>

#include "nvfp4kv_device.cuh"
#include "nvfp4kv_internal.h"

namespace nvfp4kv {

// ---------------------------------------------------------------------------
// Calibration: amax over the tensor, s_tensor = amax / (6 * 448).
// The running maximum is kept as the bit pattern of |x| in *d_s_tensor
// (non-negative floats order like their bit patterns; Inf/NaN patterns are
// above every finite one, so a non-finite element is seen by the finalize).
// ---------------------------------------------------------------------------
template <bool F32>
__global__ void __launch_bounds__(256) calib_amax_kernel(const void* __restrict__ x, int64_t n,
                                                          unsigned int* __restrict__ amax_bits) {
    uint32_t best = 0;
    const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t nthr = (int64_t)gridDim.x * blockDim.x;
    constexpr int kPer16 = F32 ? 4 : 8;  // elements per 16-byte load
    const bool aligned = (reinterpret_cast<uintptr_t>(x) & 15u) == 0;
    int64_t head = 0;
    if (aligned) {
        const int64_t nvec = n / kPer16;
        const uint4* v = reinterpret_cast<const uint4*>(x);
        for (int64_t i = tid; i < nvec; i += nthr) {
            const uint4 w = __ldg(v + i);
            const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                if (F32) {
                    best = max(best, ws[j] & 0x7FFFFFFFu);
                } else {
                    best = max(best, (ws[j] & 0x7FFFu) << 16);
                    best = max(best, (ws[j] >> 16 & 0x7FFFu) << 16);
                }
            }
        }
        head = nvec * kPer16;
    }
    for (int64_t i = head + tid; i < n; i += nthr) {
        uint32_t a;
        if (F32)
            a = reinterpret_cast<const uint32_t*>(x)[i] & 0x7FFFFFFFu;
        else
            a = (uint32_t)(reinterpret_cast<const uint16_t*>(x)[i] & 0x7FFFu) << 16;
        best = max(best, a);
    }
    best = __reduce_max_sync(0xFFFFFFFFu, best);
    if ((threadIdx.x & 31) == 0) atomicMax(amax_bits, best);
}

__global__ void calib_finalize_kernel(float* d_s_tensor, int32_t* status) {
    const uint32_t bits = *reinterpret_cast<const uint32_t*>(d_s_tensor);
    if (bits >= 0x7F800000u) {
        report(status, NVFP4_ERR_NONFINITE);
        *d_s_tensor = __uint_as_float(0x7FC00000u);
        return;
    }
    const float amax = __uint_as_float(bits);
    *d_s_tensor = (amax == 0.0f) ? 1.0f : __fdiv_rn(amax, 6.0f * 448.0f);
}

cudaError_t launch_calib(const void* x, bool f32, int64_t n, float* d_s_tensor, int32_t* d_status,
                         cudaStream_t stream) {
    cudaError_t e = cudaMemsetAsync(d_s_tensor, 0, sizeof(float), stream);
    if (e != cudaSuccess) return e;
    if (n > 0) {
        const int threads = 256;
        const int64_t want = (n / (f32 ? 4 : 8) + threads - 1) / threads;
        const int grid = (int)(want < 1 ? 1 : (want > 8L * device_sm_count() ? 8L * device_sm_count() : want));
        if (f32)
            calib_amax_kernel<true><<<grid, threads, 0, stream>>>(x, n, reinterpret_cast<unsigned*>(d_s_tensor));
        else
            calib_amax_kernel<false><<<grid, threads, 0, stream>>>(x, n, reinterpret_cast<unsigned*>(d_s_tensor));
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    calib_finalize_kernel<<<1, 1, 0, stream>>>(d_s_tensor, d_status);
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Quantize + append.  One thread per 16-element micro-block; threads are
// ordered (b, h, t, block) so that code and scale writes are contiguous in
// the [B][H_kv][S_max][...] planes.
// ---------------------------------------------------------------------------
// Quantize-append of one plane (a1-a4); `item` enumerates (b, t, h, blk)
// with blk fastest.  Index math in 32 bits when the item count fits.
template <bool F32, typename I>
__device__ __forceinline__ void quantize_append_item(
    const void* __restrict__ x_new, I i, int B, int n_new, int Hkv, int D,
    const int32_t* __restrict__ start_pos, int32_t* __restrict__ new_lens, float st, bool st_ok,
    uint8_t* __restrict__ codes, uint8_t* __restrict__ scales, int S_max, int32_t* __restrict__ status) {
    const int nblk = D / 16;
    const int blk = (int)(i % nblk);
    I r = i / nblk;
    const int t = (int)(r % n_new);
    r /= n_new;
    const int h = (int)(r % Hkv);
    const int b = (int)(r / Hkv);
    const bool leader = (t == 0 && h == 0 && blk == 0);
    if (!st_ok) {
        if (i == 0) report(status, NVFP4_ERR_NONFINITE);
        return;
    }
    const int start = start_pos[b];
    if (start < 0 || (int64_t)start + n_new > S_max) {
        if (leader) report(status, NVFP4_ERR_CAPACITY);
        return;
    }
    if (leader && new_lens != nullptr) new_lens[b] = start + n_new;
    float v[16];
    load16<F32>(x_new, (((int64_t)b * n_new + t) * Hkv + h) * D + 16 * blk, v);
    uint2 packed;
    const uint32_t sb = quantize_block(v, st, packed);
    const int64_t slot = ((int64_t)b * Hkv + h) * S_max + start + t;
    *reinterpret_cast<uint2*>(codes + slot * (D / 2) + 8 * blk) = packed;
    scales[slot * (D / 16) + blk] = (uint8_t)sb;
}

// One launch for the K and V planes of the same tokens: blockIdx.y selects the
// plane (0: K, which also writes new_lens; 1: V).
template <bool F32>
__global__ void __launch_bounds__(256) quantize_append_kv_kernel(
    const void* __restrict__ x_k, const void* __restrict__ x_v, int B, int n_new, int Hkv, int D,
    const int32_t* __restrict__ start_pos, int32_t* __restrict__ new_lens,
    const float* __restrict__ st_k_p, const float* __restrict__ st_v_p,
    uint8_t* __restrict__ codes_k, uint8_t* __restrict__ scales_k, uint8_t* __restrict__ codes_v,
    uint8_t* __restrict__ scales_v, int S_max, int32_t* __restrict__ status) {
    const bool is_v = blockIdx.y == 1;
    const float st = *(is_v ? st_v_p : st_k_p);
    const bool st_ok = st > 0.0f && st <= 3.4028234663852886e38f;  // finite and positive
    const int64_t total = (int64_t)B * Hkv * n_new * (D / 16);
    const void* x = is_v ? x_v : x_k;
    uint8_t* codes = is_v ? codes_v : codes_k;
    uint8_t* scales = is_v ? scales_v : scales_k;
    int32_t* nl = is_v ? nullptr : new_lens;
    if (total < (int64_t)INT32_MAX) {
        for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < (int)total; i += gridDim.x * blockDim.x)
            quantize_append_item<F32, int>(x, i, B, n_new, Hkv, D, start_pos, nl, st, st_ok, codes, scales,
                                           S_max, status);
    } else {
        for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
             i += (int64_t)gridDim.x * blockDim.x)
            quantize_append_item<F32, int64_t>(x, i, B, n_new, Hkv, D, start_pos, nl, st, st_ok, codes,
                                               scales, S_max, status);
    }
}

// With a block table (paged planes), token slot `pos` of sequence b is slot
// pos % page_tokens of pool page block_table[b * max_pages + pos / page_tokens]
// (pool layout [page][Hkv][page_tokens][...]) and S_max = max_pages * page_tokens.
template <bool F32>
__global__ void __launch_bounds__(256) quantize_append_kernel(
    const void* __restrict__ x_new, int B, int n_new, int Hkv, int D,
    const int32_t* __restrict__ start_pos, int32_t* __restrict__ new_lens,
    const float* __restrict__ s_tensor_p, uint8_t* __restrict__ codes, uint8_t* __restrict__ scales,
    int S_max, int32_t* __restrict__ status, const int32_t* __restrict__ block_table, int page_tokens,
    int max_pages, int num_pages) {
    const int nblk = D / 16;
    const int64_t total = (int64_t)B * Hkv * n_new * nblk;
    const float st = *s_tensor_p;
    const bool st_ok = st > 0.0f && st <= 3.4028234663852886e38f;  // finite and positive
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int blk = (int)(i % nblk);
        int64_t r = i / nblk;
        const int t = (int)(r % n_new);
        r /= n_new;
        const int h = (int)(r % Hkv);
        const int b = (int)(r / Hkv);
        const bool leader = (t == 0 && h == 0 && blk == 0);
        if (!st_ok) {
            if (i == 0) report(status, NVFP4_ERR_NONFINITE);
            continue;
        }
        const int start = start_pos[b];
        if (start < 0 || (int64_t)start + n_new > S_max) {
            if (leader) report(status, NVFP4_ERR_CAPACITY);
            continue;
        }
        if (leader && new_lens != nullptr) new_lens[b] = start + n_new;
        int64_t slot;
        if (block_table == nullptr) {
            slot = ((int64_t)b * Hkv + h) * S_max + start + t;
        } else {
            const int pos = start + t;
            const int page = block_table[(int64_t)b * max_pages + pos / page_tokens];
            if (page < 0 || page >= num_pages) {
                report(status, NVFP4_ERR_INVALID_ARG);
                continue;
            }
            slot = ((int64_t)page * Hkv + h) * page_tokens + pos % page_tokens;
        }
        float v[16];
        load16<F32>(x_new, (((int64_t)b * n_new + t) * Hkv + h) * D + 16 * blk, v);
        uint2 packed;
        const uint32_t sb = quantize_block(v, st, packed);
        *reinterpret_cast<uint2*>(codes + slot * (D / 2) + 8 * blk) = packed;
        scales[slot * (D / 16) + blk] = (uint8_t)sb;
    }
}

// ---------------------------------------------------------------------------
// MXFP4 quantize + append: the OCP MX format the NVFP4 page compares with
// ("MXFP4との比較": 32-element blocks, one E8M0 power-of-two scale each, no
// tensor scale).  One thread per block.
// The OCP exponent is floor(log2 amax) - 2, clamped to -127, and the E8M0 byte
// adds the bias 127.  For amax with fp32 exponent field E that is
// max(E - 129, -127) + 127 = max(E - 2, 0), subnormal and zero amax (E = 0)
// included.  Scaling by 2^(127 - byte) is then exact and leaves every element
// below 8 in magnitude; values past 6 saturate in the E2M1 conversion.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t mxfp4_quantize_block(const float (&a)[16], const float (&b)[16],
                                                         uint4& packed, bool& nonfinite) {
    float amax = 0.0f;
    bool bad = false;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const float x = fabsf(a[i]), y = fabsf(b[i]);
        bad |= !(x <= 3.4028234663852886e38f) || !(y <= 3.4028234663852886e38f);   // NaN or Inf
        amax = fmaxf(amax, fmaxf(x, y));
    }
    nonfinite = bad;
    if (bad) {                                       // E8M0 NaN scale, zero codes
        packed = make_uint4(0u, 0u, 0u, 0u);
        return 0xFFu;
    }
    const uint32_t E = __float_as_uint(amax) >> 23;
    const uint32_t sb = E >= 2u ? E - 2u : 0u;
    const float inv = __uint_as_float((254u - sb) << 23);   // 2^(127 - sb), a normal float
    uint32_t w[4] = {0u, 0u, 0u, 0u};
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        w[i / 8] |= e2m1_from_float(__fmul_rn(a[i], inv)) << (4 * (i % 8));
        w[2 + i / 8] |= e2m1_from_float(__fmul_rn(b[i], inv)) << (4 * (i % 8));
    }
    packed = make_uint4(w[0], w[1], w[2], w[3]);
    return sb;
}

template <bool F32>
__global__ void __launch_bounds__(256) mxfp4_quantize_append_kernel(
    const void* __restrict__ x_new, int B, int n_new, int Hkv, int D,
    const int32_t* __restrict__ start_pos, int32_t* __restrict__ new_lens, uint8_t* __restrict__ codes,
    uint8_t* __restrict__ scales, int S_max, int32_t* __restrict__ status) {
    const int nblk = D / 32;
    const int64_t total = (int64_t)B * Hkv * n_new * nblk;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int blk = (int)(i % nblk);
        int64_t r = i / nblk;
        const int t = (int)(r % n_new);
        r /= n_new;
        const int h = (int)(r % Hkv);
        const int b = (int)(r / Hkv);
        const bool leader = (t == 0 && h == 0 && blk == 0);
        const int start = start_pos[b];
        if (start < 0 || (int64_t)start + n_new > S_max) {
            if (leader) report(status, NVFP4_ERR_CAPACITY);
            continue;
        }
        if (leader && new_lens != nullptr) new_lens[b] = start + n_new;
        const int64_t elem = (((int64_t)b * n_new + t) * Hkv + h) * D + 32 * blk;
        float va[16], vb[16];
        load16<F32>(x_new, elem, va);
        load16<F32>(x_new, elem + 16, vb);
        uint4 packed;
        bool bad;
        const uint32_t sb = mxfp4_quantize_block(va, vb, packed, bad);
        if (bad) report(status, NVFP4_ERR_NONFINITE);
        const int64_t slot = ((int64_t)b * Hkv + h) * S_max + start + t;
        *reinterpret_cast<uint4*>(codes + slot * (D / 2) + 16 * blk) = packed;
        scales[slot * (D / 32) + blk] = (uint8_t)sb;
    }
}

cudaError_t launch_mxfp4_quantize_append(const void* x_new, bool f32, int n_new,
                                         const int32_t* d_start_pos, int32_t* d_new_lens,
                                         const nvfp4_kv_plane& pl, int32_t* d_status,
                                         cudaStream_t stream) {
    const int64_t total = (int64_t)pl.B * pl.H_kv * n_new * (pl.D / 32);
    if (total == 0) return cudaSuccess;
    const int threads = 256;
    int64_t grid = (total + threads - 1) / threads;
    const int64_t cap = 16L * device_sm_count();
    if (grid > cap) grid = cap;
    if (f32)
        mxfp4_quantize_append_kernel<true><<<(int)grid, threads, 0, stream>>>(
            x_new, pl.B, n_new, pl.H_kv, pl.D, d_start_pos, d_new_lens, pl.codes, pl.scales, pl.S_max,
            d_status);
    else
        mxfp4_quantize_append_kernel<false><<<(int)grid, threads, 0, stream>>>(
            x_new, pl.B, n_new, pl.H_kv, pl.D, d_start_pos, d_new_lens, pl.codes, pl.scales, pl.S_max,
            d_status);
    return cudaGetLastError();
}

cudaError_t launch_quantize_append_kv(const void* x_k, const void* x_v, bool f32, int n_new,
                                      const int32_t* d_start_pos, int32_t* d_new_lens,
                                      const float* d_st_k, const float* d_st_v,
                                      const nvfp4_kv_plane& pk, const nvfp4_kv_plane& pv,
                                      int32_t* d_status, cudaStream_t stream) {
    const int64_t total = (int64_t)pk.B * pk.H_kv * n_new * (pk.D / 16);
    if (total == 0) return cudaSuccess;
    const int threads = 256;
    int64_t grid = (total + threads - 1) / threads;
    const int64_t cap = 8L * device_sm_count();
    if (grid > cap) grid = cap;
    const dim3 g((unsigned)grid, 2);
    if (f32)
        quantize_append_kv_kernel<true><<<g, threads, 0, stream>>>(
            x_k, x_v, pk.B, n_new, pk.H_kv, pk.D, d_start_pos, d_new_lens, d_st_k, d_st_v, pk.codes,
            pk.scales, pv.codes, pv.scales, pk.S_max, d_status);
    else
        quantize_append_kv_kernel<false><<<g, threads, 0, stream>>>(
            x_k, x_v, pk.B, n_new, pk.H_kv, pk.D, d_start_pos, d_new_lens, d_st_k, d_st_v, pk.codes,
            pk.scales, pv.codes, pv.scales, pk.S_max, d_status);
    return cudaGetLastError();
}

cudaError_t launch_quantize_append(const void* x_new, bool f32, int n_new,
                                   const int32_t* d_start_pos, int32_t* d_new_lens,
                                   const float* d_s_tensor, const nvfp4_kv_plane& pl,
                                   int32_t* d_status, cudaStream_t stream) {
    const int64_t total = (int64_t)pl.B * pl.H_kv * n_new * (pl.D / 16);
    if (total == 0) return cudaSuccess;
    const int threads = 256;
    int64_t grid = (total + threads - 1) / threads;
    const int64_t cap = 16L * device_sm_count();
    if (grid > cap) grid = cap;
    if (f32)
        quantize_append_kernel<true><<<(int)grid, threads, 0, stream>>>(
            x_new, pl.B, n_new, pl.H_kv, pl.D, d_start_pos, d_new_lens, d_s_tensor, pl.codes,
            pl.scales, pl.S_max, d_status, nullptr, 0, 0, 0);
    else
        quantize_append_kernel<false><<<(int)grid, threads, 0, stream>>>(
            x_new, pl.B, n_new, pl.H_kv, pl.D, d_start_pos, d_new_lens, d_s_tensor, pl.codes,
            pl.scales, pl.S_max, d_status, nullptr, 0, 0, 0);
    return cudaGetLastError();
}

cudaError_t launch_quantize_append_paged(const void* x_new, bool f32, int n_new,
                                         const int32_t* d_start_pos, int32_t* d_new_lens,
                                         const float* d_s_tensor, const nvfp4_kv_paged_plane& pp,
                                         int32_t* d_status, cudaStream_t stream) {
    const int64_t total = (int64_t)pp.B * pp.H_kv * n_new * (pp.D / 16);
    if (total == 0) return cudaSuccess;
    const int threads = 256;
    int64_t grid = (total + threads - 1) / threads;
    const int64_t cap = 16L * device_sm_count();
    if (grid > cap) grid = cap;
    const int S_max = pp.max_pages * pp.page_tokens;   // fits: checked by the caller
    if (f32)
        quantize_append_kernel<true><<<(int)grid, threads, 0, stream>>>(
            x_new, pp.B, n_new, pp.H_kv, pp.D, d_start_pos, d_new_lens, d_s_tensor, pp.codes,
            pp.scales, S_max, d_status, pp.block_table, pp.page_tokens, pp.max_pages, pp.num_pages);
    else
        quantize_append_kernel<false><<<(int)grid, threads, 0, stream>>>(
            x_new, pp.B, n_new, pp.H_kv, pp.D, d_start_pos, d_new_lens, d_s_tensor, pp.codes,
            pp.scales, S_max, d_status, pp.block_table, pp.page_tokens, pp.max_pages, pp.num_pages);
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Standalone dequantization to FP8 (E4M3 bytes).  Each CTA first tabulates
// the FP8 value of every (scale byte, code magnitude) pair for this tensor
// scale (128 x 8 bytes); each thread then turns one 16-element block into 16
// FP8 bytes with two table words and byte permutes.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) dequant_fp8_kernel(
    const uint8_t* __restrict__ codes, const uint8_t* __restrict__ scales, int B, int Hkv,
    int S_max, int D, const float* __restrict__ s_tensor_p, const int32_t* __restrict__ seq_lens,
    uint8_t* __restrict__ out, int32_t* __restrict__ status) {
    __shared__ uint2 lut[128];
    const float st = *s_tensor_p;
    for (int sb = threadIdx.x; sb < 128; sb += blockDim.x) lut[sb] = lut_words((uint32_t)sb, st);
    if (blockIdx.x == 0 && threadIdx.x == 0 && !(st > 0.0f && st <= 3.4028234663852886e38f))
        report(status, NVFP4_ERR_NONFINITE);
    __syncthreads();
    const int nblk = D / 16;
    const int64_t total = (int64_t)B * Hkv * S_max * nblk;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int blk = (int)(i % nblk);
        const int64_t slot = i / nblk;                       // (b * Hkv + h) * S_max + t
        const int t = (int)(slot % S_max);
        const int b = (int)(slot / S_max / Hkv);
        int L = seq_lens[b];
        if (L > S_max || L < 0) {
            if (t == 0 && blk == 0 && (slot / S_max) % Hkv == 0) report(status, NVFP4_ERR_CAPACITY);
            L = L < 0 ? 0 : S_max;
        }
        if (t >= L) continue;
        const uint2 c = __ldg(reinterpret_cast<const uint2*>(codes + slot * (D / 2) + 8 * blk));
        const uint2 l = lut[scales[slot * nblk + blk] & 0x7F];
        uint4 o;
        dequant_word(c.x, l.x, l.y, o.x, o.y);
        dequant_word(c.y, l.x, l.y, o.z, o.w);
        *reinterpret_cast<uint4*>(out + slot * D + 16 * blk) = o;
    }
}

cudaError_t launch_dequant_fp8(const nvfp4_kv_plane& pl, const float* d_s_tensor,
                               const int32_t* d_seq_lens, uint8_t* out, int32_t* d_status,
                               cudaStream_t stream) {
    const int64_t total = (int64_t)pl.B * pl.H_kv * pl.S_max * (pl.D / 16);
    if (total == 0) return cudaSuccess;
    const int threads = 256;
    int64_t grid = (total + threads - 1) / threads;
    const int64_t cap = 4L * device_sm_count();
    if (grid > cap) grid = cap;
    dequant_fp8_kernel<<<(int)grid, threads, 0, stream>>>(pl.codes, pl.scales, pl.B, pl.H_kv,
                                                          pl.S_max, pl.D, d_s_tensor, d_seq_lens,
                                                          out, d_status);
    return cudaGetLastError();
}

}  // namespace nvfp4kv

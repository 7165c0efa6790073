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
// Index arithmetic: item indices are decoded with FastDiv (invariant
// divisors, nvfp4kv_device.cuh), never with a runtime division.
// ---------------------------------------------------------------------------
// launch-invariant shape of a quantize (nblk = elements per row / block size,
// a power of two)
struct QShape {
    int B, n_new, Hkv, D, S_max, lg_nblk;
    FastDiv fd_hkv, fd_new;
};

__host__ inline QShape make_qshape(int B, int n_new, int Hkv, int D, int S_max, int block) {
    QShape q;
    q.B = B; q.n_new = n_new; q.Hkv = Hkv; q.D = D; q.S_max = S_max;
    q.lg_nblk = 0;
    while ((block << q.lg_nblk) < D) ++q.lg_nblk;
    q.fd_hkv = FastDiv((uint32_t)Hkv);
    q.fd_new = FastDiv((uint32_t)n_new);
    return q;
}

// item i enumerates (b, t, h, blk), blk fastest: the order of the input
// [B][n_new][H_kv][D], so item i starts at element i * block
struct QItem {
    int b, t, h, blk;
};
__device__ __forceinline__ QItem decode_item(const QShape& q, uint32_t i) {
    QItem it;
    it.blk = (int)(i & ((1u << q.lg_nblk) - 1u));
    const uint32_t r = i >> q.lg_nblk;                 // (b * n_new + t) * Hkv + h
    const uint32_t bt = q.fd_hkv.div(r);
    it.h = (int)(r - bt * (uint32_t)q.Hkv);
    it.b = (int)q.fd_new.div(bt);
    it.t = (int)(bt - (uint32_t)it.b * (uint32_t)q.n_new);
    return it;
}
__device__ __forceinline__ QItem decode_item(const QShape& q, int64_t i) {
    QItem it;
    it.blk = (int)(i & ((1 << q.lg_nblk) - 1));
    int64_t r = i >> q.lg_nblk;
    it.h = (int)(r % q.Hkv);
    r /= q.Hkv;
    it.t = (int)(r % q.n_new);
    it.b = (int)(r / q.n_new);
    return it;
}

// ---------------------------------------------------------------------------
// Per-CTA constants of a tensor scale s: for every scale byte sb, the block
// divisor den = RN(value(sb) * s), its reciprocal RN(1/den) and whether den
// is in the range where quantize_block's division by correction applies; and
// the reciprocal of d6 = RN(6 s) with the same range test.
// ---------------------------------------------------------------------------
struct QTable {
    float den[128], rcp[128];
    uint32_t fast[4];                                  // bit sb: den in range
    float d6, rcp_d6;
    bool d6_fast;
};

__device__ __forceinline__ bool correction_range(float d) {
    return d >= kCorrectionMinDivisor && d <= kCorrectionMaxDivisor;
}

// all threads of the CTA; a barrier follows
__device__ __forceinline__ void build_qtable(QTable& tb, float st) {
    for (int sb = threadIdx.x; sb < 128; sb += blockDim.x) {
        const float den = __fmul_rn(e4m3_to_float((uint32_t)sb), st);
        tb.den[sb] = den;
        tb.rcp[sb] = correction_range(den) ? __frcp_rn(den) : 0.0f;
        const uint32_t bit = __ballot_sync(__activemask(), correction_range(den));
        if ((threadIdx.x & 31) == 0 && sb < 128) tb.fast[sb >> 5] = bit;
    }
    if (threadIdx.x == 0) {
        tb.d6 = __fmul_rn(6.0f, st);
        tb.d6_fast = correction_range(tb.d6);
        tb.rcp_d6 = tb.d6_fast ? __frcp_rn(tb.d6) : 0.0f;
    }
}

// quantize_block with the tensor-scale constants from the table: the same
// codes and scale byte, bit for bit (the per-block IEEE divisions are
// replaced by divisions by correction where those are exact)
__device__ __forceinline__ uint32_t quantize_block_tab(const float (&v)[16], const QTable& tb, float st,
                                                       uint2& packed) {
    // the block maximum, NaN if an element is NaN (max.NaN propagates it)
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) asm("max.NaN.f32 %0, %0, %1;" : "+f"(amax) : "f"(fabsf(v[i])));
    // r = RN(amax / d6): by correction when d6 is in range and amax finite; a
    // quotient past 448 (or an overflow, or a NaN) goes to the general path
    const float r = (tb.d6_fast && amax <= 3.4028234663852886e38f)
                        ? div_rn_by_correction(amax, tb.d6, tb.rcp_d6)
                        : 1e30f;
    if (r <= 448.0f) {
        const uint32_t sb = e4m3_from_float(r);
        if ((tb.fast[sb >> 5] >> (sb & 31)) & 1u) {
            const float den = tb.den[sb], y = tb.rcp[sb];
            const uint64_t nb = f32x2_pack(-den, -den), yy = f32x2_pack(y, y);
            uint32_t byte[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                float q0, q1;
                f32x2_unpack(div2_rn_by_correction(f32x2_pack(v[2 * k], v[2 * k + 1]), nb, yy), q0, q1);
                byte[k] = e2m1x2_from_floats(q0, q1);
            }
            packed = make_uint2(__byte_perm(byte[0] | (byte[1] << 8), byte[2] | (byte[3] << 8), 0x5410),
                                __byte_perm(byte[4] | (byte[5] << 8), byte[6] | (byte[7] << 8), 0x5410));
            return sb;
        }
    }
    return quantize_block(v, st, packed);
}

// ---------------------------------------------------------------------------
// Quantize + append.  One thread per 16-element micro-block; consecutive
// threads take consecutive blocks of the input, and the code and scale writes
// of a token row are contiguous in the [B][H_kv][S_max][...] planes.
// ---------------------------------------------------------------------------
// Quantize-append of one block (a1-a4).
template <bool F32, typename I>
__device__ __forceinline__ void quantize_append_item(
    const void* __restrict__ x_new, I i, const QShape& q, const int32_t* __restrict__ start_pos,
    int32_t* __restrict__ new_lens, float st, bool st_ok, const QTable& tb, uint8_t* __restrict__ codes,
    uint8_t* __restrict__ scales, int32_t* __restrict__ status) {
    const QItem it = decode_item(q, i);
    const bool leader = (it.t == 0 && it.h == 0 && it.blk == 0);
    if (!st_ok) {
        if (i == 0) report(status, NVFP4_ERR_NONFINITE);
        return;
    }
    const int start = start_pos[it.b];
    if (start < 0 || (int64_t)start + q.n_new > q.S_max) {
        if (leader) report(status, NVFP4_ERR_CAPACITY);
        return;
    }
    if (leader && new_lens != nullptr) new_lens[it.b] = start + q.n_new;
    float v[16];
    load16<F32>(x_new, (int64_t)i * 16, v);
    uint2 packed;
    const uint32_t sb = quantize_block_tab(v, tb, st, packed);
    const int64_t slot = ((int64_t)it.b * q.Hkv + it.h) * q.S_max + start + it.t;
    *reinterpret_cast<uint2*>(codes + slot * (q.D / 2) + 8 * it.blk) = packed;
    scales[slot * (q.D / 16) + it.blk] = (uint8_t)sb;
}

// One launch for the K and V planes of the same tokens: blockIdx.y selects the
// plane (0: K, which also writes new_lens; 1: V).
template <bool F32>
__global__ void __launch_bounds__(256) quantize_append_kv_kernel(
    const void* __restrict__ x_k, const void* __restrict__ x_v, const QShape q,
    const int32_t* __restrict__ start_pos, int32_t* __restrict__ new_lens,
    const float* __restrict__ st_k_p, const float* __restrict__ st_v_p,
    uint8_t* __restrict__ codes_k, uint8_t* __restrict__ scales_k, uint8_t* __restrict__ codes_v,
    uint8_t* __restrict__ scales_v, int32_t* __restrict__ status) {
    __shared__ QTable tb;
    const bool is_v = blockIdx.y == 1;
    const float st = *(is_v ? st_v_p : st_k_p);
    const bool st_ok = st > 0.0f && st <= 3.4028234663852886e38f;  // finite and positive
    build_qtable(tb, st);
    __syncthreads();
    const int64_t total = ((int64_t)q.B * q.Hkv * q.n_new) << q.lg_nblk;
    const void* x = is_v ? x_v : x_k;
    uint8_t* codes = is_v ? codes_v : codes_k;
    uint8_t* scales = is_v ? scales_v : scales_k;
    int32_t* nl = is_v ? nullptr : new_lens;
    if (total < (int64_t)INT32_MAX) {
        for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < (uint32_t)total; i += gridDim.x * blockDim.x)
            quantize_append_item<F32, uint32_t>(x, i, q, start_pos, nl, st, st_ok, tb, codes, scales, status);
    } else {
        for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
             i += (int64_t)gridDim.x * blockDim.x)
            quantize_append_item<F32, int64_t>(x, i, q, start_pos, nl, st, st_ok, tb, codes, scales, status);
    }
}

// With a block table (paged planes), token slot `pos` of sequence b is slot
// pos % page_tokens of pool page block_table[b * max_pages + pos / page_tokens]
// (pool layout [page][Hkv][page_tokens][...]) and S_max = max_pages * page_tokens.
template <bool F32, typename I>
__device__ __forceinline__ void quantize_append_paged_item(
    const void* __restrict__ x_new, I i, const QShape& q, const int32_t* __restrict__ start_pos,
    int32_t* __restrict__ new_lens, float st, bool st_ok, const QTable& tb, uint8_t* __restrict__ codes,
    uint8_t* __restrict__ scales, int32_t* __restrict__ status, const int32_t* __restrict__ block_table,
    int page_tokens, int max_pages, int num_pages) {
    const QItem it = decode_item(q, i);
    const bool leader = (it.t == 0 && it.h == 0 && it.blk == 0);
    if (!st_ok) {
        if (i == 0) report(status, NVFP4_ERR_NONFINITE);
        return;
    }
    const int start = start_pos[it.b];
    if (start < 0 || (int64_t)start + q.n_new > q.S_max) {
        if (leader) report(status, NVFP4_ERR_CAPACITY);
        return;
    }
    if (leader && new_lens != nullptr) new_lens[it.b] = start + q.n_new;
    int64_t slot;
    if (block_table == nullptr) {
        slot = ((int64_t)it.b * q.Hkv + it.h) * q.S_max + start + it.t;
    } else {
        const int pos = start + it.t;
        const int page = block_table[(int64_t)it.b * max_pages + pos / page_tokens];
        if (page < 0 || page >= num_pages) {
            report(status, NVFP4_ERR_INVALID_ARG);
            return;
        }
        slot = ((int64_t)page * q.Hkv + it.h) * page_tokens + pos % page_tokens;
    }
    float v[16];
    load16<F32>(x_new, (int64_t)i * 16, v);
    uint2 packed;
    const uint32_t sb = quantize_block_tab(v, tb, st, packed);
    *reinterpret_cast<uint2*>(codes + slot * (q.D / 2) + 8 * it.blk) = packed;
    scales[slot * (q.D / 16) + it.blk] = (uint8_t)sb;
}

template <bool F32>
__global__ void __launch_bounds__(256) quantize_append_kernel(
    const void* __restrict__ x_new, const QShape q, const int32_t* __restrict__ start_pos,
    int32_t* __restrict__ new_lens, const float* __restrict__ s_tensor_p, uint8_t* __restrict__ codes,
    uint8_t* __restrict__ scales, int32_t* __restrict__ status, const int32_t* __restrict__ block_table,
    int page_tokens, int max_pages, int num_pages) {
    __shared__ QTable tb;
    const int64_t total = ((int64_t)q.B * q.Hkv * q.n_new) << q.lg_nblk;
    const float st = *s_tensor_p;
    const bool st_ok = st > 0.0f && st <= 3.4028234663852886e38f;  // finite and positive
    build_qtable(tb, st);
    __syncthreads();
    if (total < (int64_t)INT32_MAX) {
        for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < (uint32_t)total; i += gridDim.x * blockDim.x)
            quantize_append_paged_item<F32, uint32_t>(x_new, i, q, start_pos, new_lens, st, st_ok, tb, codes, scales,
                                                      status, block_table, page_tokens, max_pages, num_pages);
    } else {
        for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
             i += (int64_t)gridDim.x * blockDim.x)
            quantize_append_paged_item<F32, int64_t>(x_new, i, q, start_pos, new_lens, st, st_ok, tb, codes, scales,
                                                     status, block_table, page_tokens, max_pages, num_pages);
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
    // two elements per hardware conversion (finite inputs: the rule of
    // e2m1_from_float)
    uint32_t by[16];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        by[k] = e2m1x2_from_floats(__fmul_rn(a[2 * k], inv), __fmul_rn(a[2 * k + 1], inv));
        by[8 + k] = e2m1x2_from_floats(__fmul_rn(b[2 * k], inv), __fmul_rn(b[2 * k + 1], inv));
    }
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
        w[j] = __byte_perm(by[4 * j] | (by[4 * j + 1] << 8), by[4 * j + 2] | (by[4 * j + 3] << 8), 0x5410);
    packed = make_uint4(w[0], w[1], w[2], w[3]);
    return sb;
}

template <bool F32, typename I>
__device__ __forceinline__ void mxfp4_quantize_append_item(
    const void* __restrict__ x_new, I i, const QShape& q, const int32_t* __restrict__ start_pos,
    int32_t* __restrict__ new_lens, uint8_t* __restrict__ codes, uint8_t* __restrict__ scales,
    int32_t* __restrict__ status) {
    const QItem it = decode_item(q, i);
    const bool leader = (it.t == 0 && it.h == 0 && it.blk == 0);
    const int start = start_pos[it.b];
    if (start < 0 || (int64_t)start + q.n_new > q.S_max) {
        if (leader) report(status, NVFP4_ERR_CAPACITY);
        return;
    }
    if (leader && new_lens != nullptr) new_lens[it.b] = start + q.n_new;
    const int64_t elem = (int64_t)i * 32;
    float va[16], vb[16];
    load16<F32>(x_new, elem, va);
    load16<F32>(x_new, elem + 16, vb);
    uint4 packed;
    bool bad;
    const uint32_t sb = mxfp4_quantize_block(va, vb, packed, bad);
    if (bad) report(status, NVFP4_ERR_NONFINITE);
    const int64_t slot = ((int64_t)it.b * q.Hkv + it.h) * q.S_max + start + it.t;
    *reinterpret_cast<uint4*>(codes + slot * (q.D / 2) + 16 * it.blk) = packed;
    scales[slot * (q.D / 32) + it.blk] = (uint8_t)sb;
}

template <bool F32>
__global__ void __launch_bounds__(256) mxfp4_quantize_append_kernel(
    const void* __restrict__ x_new, const QShape q, const int32_t* __restrict__ start_pos,
    int32_t* __restrict__ new_lens, uint8_t* __restrict__ codes, uint8_t* __restrict__ scales,
    int32_t* __restrict__ status) {
    const int64_t total = ((int64_t)q.B * q.Hkv * q.n_new) << q.lg_nblk;
    if (total < (int64_t)INT32_MAX) {
        for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < (uint32_t)total; i += gridDim.x * blockDim.x)
            mxfp4_quantize_append_item<F32, uint32_t>(x_new, i, q, start_pos, new_lens, codes, scales, status);
    } else {
        for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
             i += (int64_t)gridDim.x * blockDim.x)
            mxfp4_quantize_append_item<F32, int64_t>(x_new, i, q, start_pos, new_lens, codes, scales, status);
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
    const QShape q = make_qshape(pl.B, n_new, pl.H_kv, pl.D, pl.S_max, 32);
    if (f32)
        mxfp4_quantize_append_kernel<true><<<(int)grid, threads, 0, stream>>>(
            x_new, q, d_start_pos, d_new_lens, pl.codes, pl.scales, d_status);
    else
        mxfp4_quantize_append_kernel<false><<<(int)grid, threads, 0, stream>>>(
            x_new, q, d_start_pos, d_new_lens, pl.codes, pl.scales, d_status);
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
    const QShape q = make_qshape(pk.B, n_new, pk.H_kv, pk.D, pk.S_max, 16);
    if (f32)
        quantize_append_kv_kernel<true><<<g, threads, 0, stream>>>(
            x_k, x_v, q, d_start_pos, d_new_lens, d_st_k, d_st_v, pk.codes, pk.scales, pv.codes, pv.scales,
            d_status);
    else
        quantize_append_kv_kernel<false><<<g, threads, 0, stream>>>(
            x_k, x_v, q, d_start_pos, d_new_lens, d_st_k, d_st_v, pk.codes, pk.scales, pv.codes, pv.scales,
            d_status);
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
    const QShape q = make_qshape(pl.B, n_new, pl.H_kv, pl.D, pl.S_max, 16);
    if (f32)
        quantize_append_kernel<true><<<(int)grid, threads, 0, stream>>>(
            x_new, q, d_start_pos, d_new_lens, d_s_tensor, pl.codes, pl.scales, d_status, nullptr, 0, 0, 0);
    else
        quantize_append_kernel<false><<<(int)grid, threads, 0, stream>>>(
            x_new, q, d_start_pos, d_new_lens, d_s_tensor, pl.codes, pl.scales, d_status, nullptr, 0, 0, 0);
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
    const QShape q = make_qshape(pp.B, n_new, pp.H_kv, pp.D, S_max, 16);
    if (f32)
        quantize_append_kernel<true><<<(int)grid, threads, 0, stream>>>(
            x_new, q, d_start_pos, d_new_lens, d_s_tensor, pp.codes, pp.scales, d_status, pp.block_table,
            pp.page_tokens, pp.max_pages, pp.num_pages);
    else
        quantize_append_kernel<false><<<(int)grid, threads, 0, stream>>>(
            x_new, q, d_start_pos, d_new_lens, d_s_tensor, pp.codes, pp.scales, d_status, pp.block_table,
            pp.page_tokens, pp.max_pages, pp.num_pages);
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Standalone dequantization to FP8 (E4M3 bytes).  Each CTA first tabulates
// the FP8 value of every (scale byte, code magnitude) pair for this tensor
// scale (128 x 8 bytes); each thread then turns one 16-element block into 16
// FP8 bytes with two table words and byte permutes.
// ---------------------------------------------------------------------------
template <typename I>
__device__ __forceinline__ void dequant_fp8_item(I i, const uint8_t* __restrict__ codes,
                                                 const uint8_t* __restrict__ scales, int Hkv, int S_max, int D,
                                                 int lg_nblk, const FastDiv& fd_smax, const FastDiv& fd_hkv,
                                                 const int32_t* __restrict__ seq_lens, const uint2* lut,
                                                 uint8_t* __restrict__ out, int32_t* __restrict__ status) {
    const int blk = (int)(i & (I)((1 << lg_nblk) - 1));
    const I slot = i >> lg_nblk;                         // (b * Hkv + h) * S_max + t
    int t, b;
    bool h0;
    if constexpr (sizeof(I) == 4) {
        const uint32_t bh = fd_smax.div((uint32_t)slot);
        t = (int)((uint32_t)slot - bh * (uint32_t)S_max);
        b = (int)fd_hkv.div(bh);
        h0 = bh == (uint32_t)b * (uint32_t)Hkv;
    } else {
        t = (int)(slot % S_max);
        const int64_t bh = slot / S_max;
        b = (int)(bh / Hkv);
        h0 = bh % Hkv == 0;
    }
    int L = seq_lens[b];
    if (L > S_max || L < 0) {
        if (t == 0 && blk == 0 && h0) report(status, NVFP4_ERR_CAPACITY);
        L = L < 0 ? 0 : S_max;
    }
    if (t >= L) return;
    const int nblk = 1 << lg_nblk;
    const uint2 c = __ldg(reinterpret_cast<const uint2*>(codes + (int64_t)slot * (D / 2) + 8 * blk));
    const uint2 l = lut[scales[(int64_t)slot * nblk + blk] & 0x7F];
    uint4 o;
    dequant_word(c.x, l.x, l.y, o.x, o.y);
    dequant_word(c.y, l.x, l.y, o.z, o.w);
    *reinterpret_cast<uint4*>(out + (int64_t)slot * D + 16 * blk) = o;
}

__global__ void __launch_bounds__(256) dequant_fp8_kernel(
    const uint8_t* __restrict__ codes, const uint8_t* __restrict__ scales, int B, int Hkv,
    int S_max, int D, int lg_nblk, const FastDiv fd_smax, const FastDiv fd_hkv,
    const float* __restrict__ s_tensor_p, const int32_t* __restrict__ seq_lens,
    uint8_t* __restrict__ out, int32_t* __restrict__ status) {
    __shared__ uint2 lut[128];
    const float st = *s_tensor_p;
    for (int sb = threadIdx.x; sb < 128; sb += blockDim.x) lut[sb] = lut_words((uint32_t)sb, st);
    if (blockIdx.x == 0 && threadIdx.x == 0 && !(st > 0.0f && st <= 3.4028234663852886e38f))
        report(status, NVFP4_ERR_NONFINITE);
    __syncthreads();
    const int64_t total = ((int64_t)B * Hkv * S_max) << lg_nblk;
    if (total < (int64_t)INT32_MAX) {
        for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < (uint32_t)total; i += gridDim.x * blockDim.x)
            dequant_fp8_item<uint32_t>(i, codes, scales, Hkv, S_max, D, lg_nblk, fd_smax, fd_hkv, seq_lens, lut,
                                       out, status);
    } else {
        for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
             i += (int64_t)gridDim.x * blockDim.x)
            dequant_fp8_item<int64_t>(i, codes, scales, Hkv, S_max, D, lg_nblk, fd_smax, fd_hkv, seq_lens, lut,
                                      out, status);
    }
}

cudaError_t launch_dequant_fp8(const nvfp4_kv_plane& pl, const float* d_s_tensor,
                               const int32_t* d_seq_lens, uint8_t* out, int32_t* d_status,
                               cudaStream_t stream) {
    const int64_t total = (int64_t)pl.B * pl.H_kv * pl.S_max * (pl.D / 16);
    if (total == 0) return cudaSuccess;
    const int threads = 256;
    int64_t grid = (total + threads - 1) / threads;
    const int64_t cap = 8L * device_sm_count();
    if (grid > cap) grid = cap;
    int lg = 0;
    while ((16 << lg) < pl.D) ++lg;
    dequant_fp8_kernel<<<(int)grid, threads, 0, stream>>>(pl.codes, pl.scales, pl.B, pl.H_kv, pl.S_max, pl.D, lg,
                                                          FastDiv((uint32_t)pl.S_max), FastDiv((uint32_t)pl.H_kv),
                                                          d_s_tensor, d_seq_lens, out, d_status);
    return cudaGetLastError();
}

}  // namespace nvfp4kv

// nvfp4kv_internal.h -- host-side declarations shared by the .cu files of
// libnvfp4kv.so (launchers behind the C ABI in include/nvfp4kv.h).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/nvfp4kv.h"

namespace nvfp4kv {

// tokens per pipeline stage of the decode-attention kernel
constexpr int kTile = 32;
// sequences handled by one decode-attention launch
constexpr int kMaxBatchPerLaunch = 512;
// resident decode-attention CTAs per SM (the warp-MMA kernel is written for
// this); workspace partial slots are sized for the largest grid any of the
// decode-attention kernels launches (kMaxCtasPerSm x SM count)
constexpr int kCtasPerSm = 2;
constexpr int kMaxCtasPerSm = 3;

int device_sm_count();  // multiprocessor count of the current device (cached per device)

// Host-side argument checks of nvfp4_decode_attention (planes, shapes,
// pointers, alignment, dtype, softmax scale), without the workspace.
nvfp4_status attention_precheck(const void* q, nvfp4_dtype q_dtype, int H_q, const nvfp4_kv_plane* k,
                                const nvfp4_kv_plane* v, const float* d_s_tensor_k,
                                const float* d_s_tensor_v, const int32_t* d_seq_lens,
                                float softmax_scale, const float* out);

// cudaFuncSetAttribute(kernel, MaxDynamicSharedMemorySize, bytes) once per
// (kernel, device); `done` is the kernel's per-device flag array
cudaError_t ensure_smem_attribute(const void* kernel, int bytes, int* done_flags);
constexpr int kMaxDevices = 64;

// floats per split-K partial slot: O [g][D], m [g], l [g], padded to a whole
// float4 so that every slot starts 16-byte aligned
__host__ __device__ constexpr int64_t partial_slot_floats(int g, int D) {
    return ((int64_t)g * (D + 2) + 3) / 4 * 4;
}

cudaError_t launch_calib(const void* x, bool f32, int64_t n, float* d_s_tensor, int32_t* d_status,
                         cudaStream_t stream);

cudaError_t launch_quantize_append_paged(const void* x_new, bool f32, int n_new,
                                         const int32_t* d_start_pos, int32_t* d_new_lens,
                                         const float* d_s_tensor, const nvfp4_kv_paged_plane& pp,
                                         int32_t* d_status, cudaStream_t stream);
cudaError_t launch_mxfp4_quantize_append(const void* x_new, bool f32, int n_new,
                                         const int32_t* d_start_pos, int32_t* d_new_lens,
                                         const nvfp4_kv_plane& pl, int32_t* d_status,
                                         cudaStream_t stream);
cudaError_t launch_quantize_append(const void* x_new, bool f32, int n_new,
                                   const int32_t* d_start_pos, int32_t* d_new_lens,
                                   const float* d_s_tensor, const nvfp4_kv_plane& plane,
                                   int32_t* d_status, cudaStream_t stream);

cudaError_t launch_quantize_append_kv(const void* x_k, const void* x_v, bool f32, int n_new,
                                      const int32_t* d_start_pos, int32_t* d_new_lens,
                                      const float* d_st_k, const float* d_st_v,
                                      const nvfp4_kv_plane& pk, const nvfp4_kv_plane& pv,
                                      int32_t* d_status, cudaStream_t stream);

cudaError_t launch_dequant_fp8(const nvfp4_kv_plane& plane, const float* d_s_tensor,
                               const int32_t* d_seq_lens, uint8_t* out, int32_t* d_status,
                               cudaStream_t stream);

struct AttnLaunch {
    const void* q;
    bool q_f32;
    int B, Hq, Hkv, S_max, D;
    const uint8_t *kc, *ks, *vc, *vs;
    const float *st_k, *st_v;
    const int32_t* seq_lens;
    float softmax_scale;
    float* out;
    float* partials;     // [2 * grid] slots of partial_slot_floats(g, D)
    int32_t* counters;   // [B * Hkv], zero between calls
    int32_t* status;
    int grid;            // CTAs
    // paged cache: nullptr for contiguous planes (then S_max is the capacity)
    const int32_t* block_table;
    int page_tokens, max_pages, num_pages;
    uint32_t wait_polls;  // give-up limit of the tensor-core kernel's pipeline waits
    // append + attention (contiguous planes): start_pos != nullptr attends
    // start_pos[b] + 1 tokens after appending one new token per sequence from
    // x_k_new / x_v_new [B][1][Hkv][D] (fp32 when x_f32, else bf16) at slot
    // start_pos[b]; new_lens (optional) receives start_pos[b] + 1
    const int32_t* start_pos;
    int32_t* new_lens;
    const void* x_k_new;
    const void* x_v_new;
    bool x_f32;
};

cudaError_t launch_decode_attention(const AttnLaunch& a, cudaStream_t stream);

// chunked-prefill attention on the tensor cores (head_dim 128, contiguous planes)
cudaError_t launch_prefill_tc(const void* q, bool q_f32, int C, int H_q, const nvfp4_kv_plane& k,
                              const nvfp4_kv_plane& v, const float* d_st_k, const float* d_st_v,
                              const int32_t* d_start, float softmax_scale, float* out, int32_t* d_status,
                              uint32_t wait_polls, cudaStream_t stream);

// workspace layout of nvfp4_decode_attention for one shape
struct AttnWorkspace {
    size_t counters_bytes;  // B * H_kv int32, padded to 256 bytes
    size_t partial_floats;  // 2 * grid * partial_slot_floats(g, D)
    size_t total_bytes;
    int grid;
};
AttnWorkspace attention_workspace(int B, int Hq, int Hkv, int D);

}  // namespace nvfp4kv

// nvfp4kv_noalloc.cu -- nvfp4_decode_attention for callers that cannot
// allocate device memory.
//
// Some callers cannot call cudaMalloc or any allocating routine: code that
// runs inside a host or framework whose memory pool owns every device
// allocation, plugins that are handed only input and output buffers, or code
// paths that must not allocate while other work is in flight.  For them this
// entry point takes no workspace: the split-K partial results and arrival
// counters live in one file-scope device array of fixed size, which every
// GPU that loads this library holds until the process exits.
#include <cstdint>
#include <mutex>

#include <cuda_runtime.h>

#include "../../include/nvfp4kv.h"
#include "nvfp4kv_internal.h"

namespace {

// Built-in scratch: counters then partial results (the same layout
// nvfp4_decode_attention expects in its workspace argument).
constexpr size_t kNoAllocScratchBytes = NVFP4_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) uint8_t g_attention_scratch[kNoAllocScratchBytes];

// Device address of g_attention_scratch per device.  In host code the name
// g_attention_scratch is only a stand-in for the symbol; its device address
// must be looked up once per device with that device current.
std::mutex g_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

nvfp4_status scratch_for_current_device(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return NVFP4_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (g_scratch_ptr[dev] == nullptr) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_attention_scratch) != cudaSuccess || ptr == nullptr)
            return NVFP4_ERR_CUDA;
        g_scratch_ptr[dev] = ptr;
    }
    *out = g_scratch_ptr[dev];
    return NVFP4_OK;
}

}  // namespace

extern "C" nvfp4_status nvfp4_decode_attention_noalloc(
    const void* q, nvfp4_dtype q_dtype, int H_q, const nvfp4_kv_plane* k, const nvfp4_kv_plane* v,
    const float* d_s_tensor_k, const float* d_s_tensor_v, const int32_t* d_seq_lens,
    float softmax_scale, float* out, int32_t* d_status, nvfp4_stream_t stream) {
    // the same host checks as nvfp4_decode_attention, before anything is queued
    const nvfp4_status pre = nvfp4kv::attention_precheck(q, q_dtype, H_q, k, v, d_s_tensor_k, d_s_tensor_v,
                                                          d_seq_lens, softmax_scale, out);
    if (pre != NVFP4_OK) return pre;
    if (k->B == 0) return NVFP4_OK;
    const size_t need = nvfp4_decode_attention_workspace(k->B, H_q, k->H_kv, k->D);
    if (need == 0) return NVFP4_ERR_INVALID_ARG;
    if (need > kNoAllocScratchBytes) return NVFP4_ERR_WORKSPACE;   // shape too large for the buffer
    void* scratch = nullptr;
    const nvfp4_status st = scratch_for_current_device(&scratch);
    if (st != NVFP4_OK) return st;
    // the arrival counters must start at zero; clear them on the caller's
    // stream (a memset, not an allocation), so an earlier interrupted call
    // cannot leave stale counts behind
    const size_t counters = nvfp4kv::attention_workspace(k->B, H_q, k->H_kv, k->D).counters_bytes;
    if (cudaMemsetAsync(scratch, 0, counters, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
        return NVFP4_ERR_CUDA;
    return nvfp4_decode_attention(q, q_dtype, H_q, k, v, d_s_tensor_k, d_s_tensor_v, d_seq_lens,
                                  softmax_scale, out, scratch, kNoAllocScratchBytes, d_status, stream);
}

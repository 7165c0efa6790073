// nvfp4kv_api.cu -- the extern "C" entry points of libnvfp4kv.so declared in
// include/nvfp4kv.h: argument validation, workspace layout and launches.
// Every call is asynchronous on the caller's stream and allocates nothing.
#include <cmath>
#include <cstdint>
#include <cstring>
#include <atomic>
#include <mutex>

#include <cuda_runtime.h>

#include "../../include/nvfp4kv.h"
#include "nvfp4kv_internal.h"

namespace nvfp4kv {

namespace {
std::mutex g_dev_mutex;
int g_sm_count[kMaxDevices] = {};   // 0 = not looked up yet
}  // namespace

int device_sm_count() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return 148;
    if (dev >= kMaxDevices) {
        int n = 0;
        return (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && n > 0) ? n : 148;
    }
    std::lock_guard<std::mutex> lock(g_dev_mutex);
    if (g_sm_count[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
        g_sm_count[dev] = n;
    }
    return g_sm_count[dev];
}

cudaError_t ensure_smem_attribute(const void* kernel, int bytes, int* done_flags) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices)
        return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    std::lock_guard<std::mutex> lock(g_dev_mutex);
    if (!done_flags[dev]) {
        e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
        if (e != cudaSuccess) return e;
        done_flags[dev] = 1;
    }
    return cudaSuccess;
}

AttnWorkspace attention_workspace(int B, int Hq, int Hkv, int D) {
    AttnWorkspace w{};
    const int g = Hq / Hkv;
    w.grid = kMaxCtasPerSm * device_sm_count();
    w.counters_bytes = ((size_t)B * Hkv * sizeof(int32_t) + 255) / 256 * 256;
    w.partial_floats = (size_t)2 * w.grid * (size_t)partial_slot_floats(g, D);
    w.total_bytes = w.counters_bytes + w.partial_floats * sizeof(float);
    return w;
}

}  // namespace nvfp4kv

namespace {

using namespace nvfp4kv;

// Give-up limit of the tensor-core attention kernel's pipeline waits, in
// sleeping polls of up to 20 us each (2^16: about a second or more);
// nvfp4_set_wait_limit changes it (a testing hook).
constexpr uint32_t kDefaultWaitPolls = 1u << 16;
std::atomic<uint32_t> g_wait_polls{kDefaultWaitPolls};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool plane_ok(const nvfp4_kv_plane* pl) {
    if (pl == nullptr || pl->codes == nullptr || pl->scales == nullptr) return false;
    if (pl->B < 0 || pl->H_kv <= 0 || pl->S_max <= 0 || (pl->S_max % 16) != 0) return false;
    if (pl->D != 64 && pl->D != 128) return false;
    if (!aligned16(pl->codes) || !aligned16(pl->scales)) return false;
    return true;
}

nvfp4_status from_cuda(cudaError_t e) { return e == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA; }

bool paged_ok(const nvfp4_kv_paged_plane* pl) {
    if (pl == nullptr || pl->codes == nullptr || pl->scales == nullptr || pl->block_table == nullptr)
        return false;
    if (pl->B < 0 || pl->H_kv <= 0 || pl->num_pages <= 0 || pl->max_pages <= 0) return false;
    if (pl->page_tokens <= 0 || (pl->page_tokens % 128) != 0) return false;
    if ((int64_t)pl->max_pages * pl->page_tokens > (int64_t)INT32_MAX) return false;
    if (pl->D != 64 && pl->D != 128) return false;
    if (!aligned16(pl->codes) || !aligned16(pl->scales)) return false;
    return true;
}

// What a launch over sequences b0.. reads: contiguous planes advance by a
// sequence stride; paged planes keep their pools and advance the block table.
struct CacheView {
    const uint8_t *kc, *ks, *vc, *vs;
    size_t seq_code_bytes, seq_scale_bytes;
    const int32_t* block_table;
    int page_tokens, max_pages, num_pages;
};

// Validation and batch-chunked launches shared by the contiguous and the
// paged attention entry points (the planes are already validated).
// Argument checks shared by every attention entry point (the planes are
// already validated): dtype, group size, pointers, alignment, softmax scale,
// and the 32-bit tile count of one launch.
nvfp4_status check_attention_args(const void* q, nvfp4_dtype q_dtype, int H_q, int B, int H_kv, int S_max,
                                  const float* d_s_tensor_k, const float* d_s_tensor_v,
                                  const int32_t* d_seq_lens, float softmax_scale, const float* out) {
    if (q_dtype != NVFP4_IN_BF16 && q_dtype != NVFP4_IN_F32) return NVFP4_ERR_INVALID_ARG;
    if (H_q <= 0 || (H_q % H_kv) != 0) return NVFP4_ERR_INVALID_ARG;
    if (H_q / H_kv > 16) return NVFP4_ERR_UNSUPPORTED;
    if (d_s_tensor_k == nullptr || d_s_tensor_v == nullptr || d_seq_lens == nullptr)
        return NVFP4_ERR_INVALID_ARG;
    if (!(std::isfinite(softmax_scale)) || softmax_scale < 0.0f) return NVFP4_ERR_INVALID_ARG;
    if (B == 0) return NVFP4_OK;
    if (q == nullptr || out == nullptr || !aligned16(q) || !aligned16(out)) return NVFP4_ERR_INVALID_ARG;
    // the kernels split a launch's tiles (32 tokens at the smallest) of every
    // (sequence, KV head) with 32-bit prefix sums
    const int64_t launch_tiles = (int64_t)(B < kMaxBatchPerLaunch ? B : kMaxBatchPerLaunch) * H_kv *
                                 (((int64_t)S_max + 31) / 32);
    if (launch_tiles > (int64_t)INT32_MAX) return NVFP4_ERR_UNSUPPORTED;
    return NVFP4_OK;
}

// The new tokens of an append + attention call (nullptr: attention only).
struct AppendArgs {
    const void* x_k;
    const void* x_v;
    bool f32;
    const int32_t* start_pos;
    int32_t* new_lens;
};

nvfp4_status run_attention(const void* q, nvfp4_dtype q_dtype, int H_q, int B, int H_kv, int D,
                           int S_max, const CacheView& c, const float* d_s_tensor_k,
                           const float* d_s_tensor_v, const int32_t* d_seq_lens, float softmax_scale,
                           float* out, void* workspace, size_t workspace_bytes, int32_t* d_status,
                           nvfp4_stream_t stream, const AppendArgs* app = nullptr) {
    const nvfp4_status pre = check_attention_args(q, q_dtype, H_q, B, H_kv, S_max, d_s_tensor_k,
                                                  d_s_tensor_v, d_seq_lens, softmax_scale, out);
    if (pre != NVFP4_OK || B == 0) return pre;
    const AttnWorkspace ws = attention_workspace(B, H_q, H_kv, D);
    if (workspace == nullptr || workspace_bytes < ws.total_bytes || !aligned16(workspace))
        return NVFP4_ERR_WORKSPACE;

    const size_t esz = q_dtype == NVFP4_IN_F32 ? 4 : 2;
    AttnLaunch a{};
    a.q_f32 = q_dtype == NVFP4_IN_F32;
    a.Hq = H_q;
    a.Hkv = H_kv;
    a.S_max = S_max;
    a.D = D;
    a.st_k = d_s_tensor_k;
    a.st_v = d_s_tensor_v;
    a.softmax_scale = softmax_scale > 0.0f ? softmax_scale : 1.0f / std::sqrt((float)D);
    a.partials = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + ws.counters_bytes);
    a.status = d_status;
    a.grid = ws.grid;
    a.block_table = c.block_table;
    a.page_tokens = c.page_tokens;
    a.max_pages = c.max_pages;
    a.num_pages = c.num_pages;
    a.wait_polls = g_wait_polls.load();
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    for (int b0 = 0; b0 < B; b0 += kMaxBatchPerLaunch) {
        const int nb = (B - b0) < kMaxBatchPerLaunch ? (B - b0) : kMaxBatchPerLaunch;
        a.B = nb;
        a.q = static_cast<const uint8_t*>(q) + (size_t)b0 * H_q * D * esz;
        a.kc = c.kc + (size_t)b0 * c.seq_code_bytes;    // paged: offsets 0, the table moves
        a.ks = c.ks + (size_t)b0 * c.seq_scale_bytes;
        a.vc = c.vc + (size_t)b0 * c.seq_code_bytes;
        a.vs = c.vs + (size_t)b0 * c.seq_scale_bytes;
        if (c.block_table != nullptr) a.block_table = c.block_table + (size_t)b0 * c.max_pages;
        a.seq_lens = d_seq_lens + b0;
        a.out = out + (size_t)b0 * H_q * D;
        a.counters = static_cast<int32_t*>(workspace) + (size_t)b0 * H_kv;
        if (app != nullptr) {
            const size_t xsz = app->f32 ? 4 : 2;
            a.x_k_new = static_cast<const uint8_t*>(app->x_k) + (size_t)b0 * H_kv * D * xsz;
            a.x_v_new = static_cast<const uint8_t*>(app->x_v) + (size_t)b0 * H_kv * D * xsz;
            a.x_f32 = app->f32;
            a.start_pos = app->start_pos + b0;
            a.new_lens = app->new_lens != nullptr ? app->new_lens + b0 : nullptr;
        }
        cudaError_t e = launch_decode_attention(a, s);
        if (e != cudaSuccess) return NVFP4_ERR_CUDA;
    }
    return NVFP4_OK;
}


}  // namespace

namespace nvfp4kv {

nvfp4_status attention_precheck(const void* q, nvfp4_dtype q_dtype, int H_q, const nvfp4_kv_plane* k,
                                const nvfp4_kv_plane* v, const float* d_s_tensor_k,
                                const float* d_s_tensor_v, const int32_t* d_seq_lens,
                                float softmax_scale, const float* out) {
    if (!plane_ok(k) || !plane_ok(v)) return NVFP4_ERR_INVALID_ARG;
    if (k->B != v->B || k->H_kv != v->H_kv || k->S_max != v->S_max || k->D != v->D)
        return NVFP4_ERR_INVALID_ARG;
    return check_attention_args(q, q_dtype, H_q, k->B, k->H_kv, k->S_max, d_s_tensor_k, d_s_tensor_v,
                                d_seq_lens, softmax_scale, out);
}

}  // namespace nvfp4kv

extern "C" {

const char* nvfp4_status_string(int status) {
    switch (status) {
        case NVFP4_OK: return "ok";
        case NVFP4_ERR_INVALID_ARG: return "invalid argument";
        case NVFP4_ERR_UNSUPPORTED: return "unsupported";
        case NVFP4_ERR_CAPACITY: return "sequence past cache capacity";
        case NVFP4_ERR_NONFINITE: return "non-finite value or scale";
        case NVFP4_ERR_CUDA: return "CUDA error";
        case NVFP4_ERR_TIMEOUT: return "device wait timed out";
        case NVFP4_ERR_WORKSPACE: return "workspace missing or too small";
        default: return "unknown status";
    }
}

const char* nvfp4_version(void) { return "nvfp4kv 0.1.0 (sm_100a)"; }

void nvfp4_set_wait_limit(int64_t polls) {
    g_wait_polls.store(polls < 0 ? kDefaultWaitPolls
                                 : (polls > (int64_t)UINT32_MAX ? UINT32_MAX : (uint32_t)polls));
}

size_t nvfp4_cache_bytes(int B, int H_kv, int S_max, int D) {
    if (B < 0 || H_kv <= 0 || S_max < 0 || D <= 0 || (D % 16) != 0) return 0;
    return (size_t)B * H_kv * S_max * (size_t)(D / 2 + D / 16);
}

nvfp4_status nvfp4_calib_tensor_scale(const void* x, nvfp4_dtype dtype, int64_t n,
                                      float* d_s_tensor, int32_t* d_status, nvfp4_stream_t stream) {
    if (d_s_tensor == nullptr || n < 0 || (n > 0 && x == nullptr)) return NVFP4_ERR_INVALID_ARG;
    if (dtype != NVFP4_IN_BF16 && dtype != NVFP4_IN_F32) return NVFP4_ERR_INVALID_ARG;
    const size_t esz = dtype == NVFP4_IN_F32 ? 4 : 2;
    if ((reinterpret_cast<uintptr_t>(x) % esz) != 0) return NVFP4_ERR_INVALID_ARG;
    return from_cuda(launch_calib(x, dtype == NVFP4_IN_F32, n, d_s_tensor, d_status,
                                  reinterpret_cast<cudaStream_t>(stream)));
}

nvfp4_status nvfp4_kv_quantize_append(const void* x_new, nvfp4_dtype dtype, int n_new,
                                      const int32_t* d_start_pos, int32_t* d_new_lens,
                                      const float* d_s_tensor, const nvfp4_kv_plane* plane,
                                      int32_t* d_status, nvfp4_stream_t stream) {
    if (!plane_ok(plane) || n_new < 0 || d_s_tensor == nullptr || d_start_pos == nullptr)
        return NVFP4_ERR_INVALID_ARG;
    if (dtype != NVFP4_IN_BF16 && dtype != NVFP4_IN_F32) return NVFP4_ERR_INVALID_ARG;
    if (d_new_lens != nullptr && d_new_lens == d_start_pos) return NVFP4_ERR_INVALID_ARG;
    if (n_new == 0 || plane->B == 0) return NVFP4_OK;
    if (x_new == nullptr || !aligned16(x_new)) return NVFP4_ERR_INVALID_ARG;
    return from_cuda(launch_quantize_append(x_new, dtype == NVFP4_IN_F32, n_new, d_start_pos,
                                            d_new_lens, d_s_tensor, *plane, d_status,
                                            reinterpret_cast<cudaStream_t>(stream)));
}

nvfp4_status nvfp4_kv_quantize_append_paged(const void* x_new, nvfp4_dtype dtype, int n_new,
                                            const int32_t* d_start_pos, int32_t* d_new_lens,
                                            const float* d_s_tensor,
                                            const nvfp4_kv_paged_plane* plane, int32_t* d_status,
                                            nvfp4_stream_t stream) {
    if (!paged_ok(plane) || n_new < 0 || d_s_tensor == nullptr || d_start_pos == nullptr)
        return NVFP4_ERR_INVALID_ARG;
    if (dtype != NVFP4_IN_BF16 && dtype != NVFP4_IN_F32) return NVFP4_ERR_INVALID_ARG;
    if (d_new_lens != nullptr && d_new_lens == d_start_pos) return NVFP4_ERR_INVALID_ARG;
    if (n_new == 0 || plane->B == 0) return NVFP4_OK;
    if (x_new == nullptr || !aligned16(x_new)) return NVFP4_ERR_INVALID_ARG;
    return from_cuda(launch_quantize_append_paged(x_new, dtype == NVFP4_IN_F32, n_new, d_start_pos,
                                                  d_new_lens, d_s_tensor, *plane, d_status,
                                                  reinterpret_cast<cudaStream_t>(stream)));
}

nvfp4_status nvfp4_kv_quantize_append_kv(const void* x_k, const void* x_v, nvfp4_dtype dtype,
                                         int n_new, const int32_t* d_start_pos, int32_t* d_new_lens,
                                         const float* d_s_tensor_k, const float* d_s_tensor_v,
                                         const nvfp4_kv_plane* k, const nvfp4_kv_plane* v,
                                         int32_t* d_status, nvfp4_stream_t stream) {
    if (!plane_ok(k) || !plane_ok(v) || n_new < 0 || d_s_tensor_k == nullptr ||
        d_s_tensor_v == nullptr || d_start_pos == nullptr)
        return NVFP4_ERR_INVALID_ARG;
    if (k->B != v->B || k->H_kv != v->H_kv || k->S_max != v->S_max || k->D != v->D)
        return NVFP4_ERR_INVALID_ARG;
    if (dtype != NVFP4_IN_BF16 && dtype != NVFP4_IN_F32) return NVFP4_ERR_INVALID_ARG;
    if (d_new_lens != nullptr && d_new_lens == d_start_pos) return NVFP4_ERR_INVALID_ARG;
    if (n_new == 0 || k->B == 0) return NVFP4_OK;
    if (x_k == nullptr || x_v == nullptr || !aligned16(x_k) || !aligned16(x_v)) return NVFP4_ERR_INVALID_ARG;
    return from_cuda(launch_quantize_append_kv(x_k, x_v, dtype == NVFP4_IN_F32, n_new, d_start_pos,
                                               d_new_lens, d_s_tensor_k, d_s_tensor_v, *k, *v,
                                               d_status, reinterpret_cast<cudaStream_t>(stream)));
}

size_t mxfp4_cache_bytes(int B, int H_kv, int S_max, int D) {
    if (B < 0 || H_kv <= 0 || S_max < 0 || D <= 0 || (D % 32) != 0) return 0;
    return (size_t)B * H_kv * S_max * (size_t)(D / 2 + D / 32);
}

nvfp4_status mxfp4_kv_quantize_append(const void* x_new, nvfp4_dtype dtype, int n_new,
                                      const int32_t* d_start_pos, int32_t* d_new_lens,
                                      const nvfp4_kv_plane* plane, int32_t* d_status,
                                      nvfp4_stream_t stream) {
    if (!plane_ok(plane) || n_new < 0 || d_start_pos == nullptr) return NVFP4_ERR_INVALID_ARG;
    if (dtype != NVFP4_IN_BF16 && dtype != NVFP4_IN_F32) return NVFP4_ERR_INVALID_ARG;
    if (d_new_lens != nullptr && d_new_lens == d_start_pos) return NVFP4_ERR_INVALID_ARG;
    if (n_new == 0 || plane->B == 0) return NVFP4_OK;
    if (x_new == nullptr || !aligned16(x_new)) return NVFP4_ERR_INVALID_ARG;
    return from_cuda(launch_mxfp4_quantize_append(x_new, dtype == NVFP4_IN_F32, n_new, d_start_pos,
                                                  d_new_lens, *plane, d_status,
                                                  reinterpret_cast<cudaStream_t>(stream)));
}

nvfp4_status nvfp4_kv_dequant_fp8(const nvfp4_kv_plane* plane, const float* d_s_tensor,
                                  const int32_t* d_seq_lens, uint8_t* out_e4m3, int32_t* d_status,
                                  nvfp4_stream_t stream) {
    if (!plane_ok(plane) || d_s_tensor == nullptr || d_seq_lens == nullptr)
        return NVFP4_ERR_INVALID_ARG;
    if (plane->B == 0) return NVFP4_OK;
    if (out_e4m3 == nullptr || !aligned16(out_e4m3)) return NVFP4_ERR_INVALID_ARG;
    return from_cuda(launch_dequant_fp8(*plane, d_s_tensor, d_seq_lens, out_e4m3, d_status,
                                        reinterpret_cast<cudaStream_t>(stream)));
}

size_t nvfp4_decode_attention_workspace(int B, int H_q, int H_kv, int D) {
    if (B < 0 || H_kv <= 0 || H_q <= 0 || (H_q % H_kv) != 0 || H_q / H_kv > 16) return 0;
    if (D != 64 && D != 128) return 0;
    return attention_workspace(B, H_q, H_kv, D).total_bytes;
}

nvfp4_status nvfp4_decode_attention(const void* q, nvfp4_dtype q_dtype, int H_q,
                                    const nvfp4_kv_plane* k, const nvfp4_kv_plane* v,
                                    const float* d_s_tensor_k, const float* d_s_tensor_v,
                                    const int32_t* d_seq_lens, float softmax_scale, float* out,
                                    void* workspace, size_t workspace_bytes, int32_t* d_status,
                                    nvfp4_stream_t stream) {
    if (!plane_ok(k) || !plane_ok(v)) return NVFP4_ERR_INVALID_ARG;
    if (k->B != v->B || k->H_kv != v->H_kv || k->S_max != v->S_max || k->D != v->D)
        return NVFP4_ERR_INVALID_ARG;
    CacheView c{};
    c.kc = k->codes; c.ks = k->scales; c.vc = v->codes; c.vs = v->scales;
    const size_t plane_tok = (size_t)k->H_kv * k->S_max;  // token slots per sequence
    c.seq_code_bytes = plane_tok * (k->D / 2);
    c.seq_scale_bytes = plane_tok * (k->D / 16);
    return run_attention(q, q_dtype, H_q, k->B, k->H_kv, k->D, k->S_max, c, d_s_tensor_k, d_s_tensor_v,
                         d_seq_lens, softmax_scale, out, workspace, workspace_bytes, d_status, stream);
}

nvfp4_status nvfp4_decode_attention_append(const void* q, nvfp4_dtype q_dtype, int H_q,
                                           const void* x_k_new, const void* x_v_new, nvfp4_dtype x_dtype,
                                           const int32_t* d_start_pos, int32_t* d_new_lens,
                                           const nvfp4_kv_plane* k, const nvfp4_kv_plane* v,
                                           const float* d_s_tensor_k, const float* d_s_tensor_v,
                                           float softmax_scale, float* out, void* workspace,
                                           size_t workspace_bytes, int32_t* d_status,
                                           nvfp4_stream_t stream) {
    if (!plane_ok(k) || !plane_ok(v)) return NVFP4_ERR_INVALID_ARG;
    if (k->B != v->B || k->H_kv != v->H_kv || k->S_max != v->S_max || k->D != v->D)
        return NVFP4_ERR_INVALID_ARG;
    if (x_dtype != NVFP4_IN_BF16 && x_dtype != NVFP4_IN_F32) return NVFP4_ERR_INVALID_ARG;
    if (d_start_pos == nullptr || (d_new_lens != nullptr && d_new_lens == d_start_pos))
        return NVFP4_ERR_INVALID_ARG;
    if (k->B > 0 && (x_k_new == nullptr || x_v_new == nullptr || !aligned16(x_k_new) || !aligned16(x_v_new)))
        return NVFP4_ERR_INVALID_ARG;
    CacheView c{};
    c.kc = k->codes; c.ks = k->scales; c.vc = v->codes; c.vs = v->scales;
    const size_t plane_tok = (size_t)k->H_kv * k->S_max;
    c.seq_code_bytes = plane_tok * (k->D / 2);
    c.seq_scale_bytes = plane_tok * (k->D / 16);
    AppendArgs app{x_k_new, x_v_new, x_dtype == NVFP4_IN_F32, d_start_pos, d_new_lens};
    // the lengths come from d_start_pos (start + 1); it stands in for seq_lens in the checks
    return run_attention(q, q_dtype, H_q, k->B, k->H_kv, k->D, k->S_max, c, d_s_tensor_k, d_s_tensor_v,
                         d_start_pos, softmax_scale, out, workspace, workspace_bytes, d_status, stream, &app);
}

nvfp4_status nvfp4_decode_attention_paged(const void* q, nvfp4_dtype q_dtype, int H_q,
                                          const nvfp4_kv_paged_plane* k,
                                          const nvfp4_kv_paged_plane* v,
                                          const float* d_s_tensor_k, const float* d_s_tensor_v,
                                          const int32_t* d_seq_lens, float softmax_scale,
                                          float* out, void* workspace, size_t workspace_bytes,
                                          int32_t* d_status, nvfp4_stream_t stream) {
    if (!paged_ok(k) || !paged_ok(v)) return NVFP4_ERR_INVALID_ARG;
    if (k->block_table != v->block_table || k->B != v->B || k->H_kv != v->H_kv ||
        k->page_tokens != v->page_tokens || k->max_pages != v->max_pages || k->D != v->D)
        return NVFP4_ERR_INVALID_ARG;
    CacheView c{};
    c.kc = k->codes; c.ks = k->scales; c.vc = v->codes; c.vs = v->scales;
    c.block_table = k->block_table;
    c.page_tokens = k->page_tokens;
    c.max_pages = k->max_pages;
    c.num_pages = k->num_pages < v->num_pages ? k->num_pages : v->num_pages;
    return run_attention(q, q_dtype, H_q, k->B, k->H_kv, k->D, k->max_pages * k->page_tokens, c,
                         d_s_tensor_k, d_s_tensor_v, d_seq_lens, softmax_scale, out, workspace,
                         workspace_bytes, d_status, stream);
}

nvfp4_status nvfp4_prefill_attention(const void* q, nvfp4_dtype q_dtype, int C, int H_q,
                                     const nvfp4_kv_plane* k, const nvfp4_kv_plane* v,
                                     const float* d_s_tensor_k, const float* d_s_tensor_v,
                                     const int32_t* d_start_pos, float softmax_scale, float* out,
                                     int32_t* d_status, nvfp4_stream_t stream) {
    if (!plane_ok(k) || !plane_ok(v)) return NVFP4_ERR_INVALID_ARG;
    if (k->B != v->B || k->H_kv != v->H_kv || k->S_max != v->S_max || k->D != v->D)
        return NVFP4_ERR_INVALID_ARG;
    if (q_dtype != NVFP4_IN_BF16 && q_dtype != NVFP4_IN_F32) return NVFP4_ERR_INVALID_ARG;
    if (C < 0 || H_q <= 0 || (H_q % k->H_kv) != 0) return NVFP4_ERR_INVALID_ARG;
    if (d_s_tensor_k == nullptr || d_s_tensor_v == nullptr || d_start_pos == nullptr)
        return NVFP4_ERR_INVALID_ARG;
    if (!(std::isfinite(softmax_scale)) || softmax_scale < 0.0f) return NVFP4_ERR_INVALID_ARG;
    // the tensor-core prefill takes bf16 queries (exact in its f16 operand
    // after a power-of-two row scaling, down to 2^-31 of the row maximum); an
    // fp32 query would need a second f16 term and its shared memory
    if (k->D != 128 || H_q / k->H_kv > 128 || q_dtype != NVFP4_IN_BF16) return NVFP4_ERR_UNSUPPORTED;
    if (k->B == 0 || C == 0) return NVFP4_OK;
    if (q == nullptr || out == nullptr || !aligned16(q) || !aligned16(out)) return NVFP4_ERR_INVALID_ARG;
    const int g = H_q / k->H_kv, cq = 128 / g;
    if ((int64_t)k->B * k->H_kv * ((C + cq - 1) / cq) > (int64_t)INT32_MAX) return NVFP4_ERR_UNSUPPORTED;
    return from_cuda(launch_prefill_tc(q, q_dtype == NVFP4_IN_F32, C, H_q, *k, *v, d_s_tensor_k, d_s_tensor_v,
                                       d_start_pos, softmax_scale, out, d_status,
                                       g_wait_polls.load(std::memory_order_relaxed),
                                       reinterpret_cast<cudaStream_t>(stream)));
}

}  // extern "C"

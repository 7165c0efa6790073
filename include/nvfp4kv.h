/*
 * nvfp4kv.h -- C ABI of libnvfp4kv.so: an NVFP4 KV cache with fused
 * NVFP4 -> FP8 decode attention for NVIDIA B200 (sm_100a).
 *
 * What the library computes (sources are web pages, cited by title/section):
 *
 *   [NVFP4-KV] "NVIDIA解説: NVFP4 KV Cacheで長コンテキストLLM推論を最適化 --
 *              メモリ50%削減・TTFT 3倍高速化" (0h-n0.github.io; a summary of
 *              NVIDIA's technical blog on the NVFP4 KV cache).
 *   [rc17]     "TensorRT-LLM rc17 が SM121（DGX Spark）向けに NVFP4 MoE
 *              バックエンドと NVFP4 KV キャッシュを追加".
 *   [FR-lesson] "Compilation d'inferences spécialisées en matériel FP8 et
 *              NVFP4 sur Blackwell".
 *
 *   Storage ([NVFP4-KV] "E2M1 + 2レベルスケーリング"): every K or V element
 *   is an E2M1 code (sign 1, exponent 2, mantissa 1; values 0, 0.5, 1, 1.5,
 *   2, 3, 4, 6 and negatives), every 16 consecutive elements along head_dim
 *   share one E4M3 scale byte s_block, and the whole tensor shares one fp32
 *   scale s_tensor:  x ~ x_q * s_block * s_tensor.
 *   Flow ([NVFP4-KV] "量子化・逆量子化フロー", [rc17] "物語の KV キャッシュ側"):
 *   new tokens are quantized on append; at attention time the cache is
 *   dequantized to FP8 and FP8 attention runs with an FP32 accumulator
 *   ([FR-lesson] "Le type de Blackwell").
 *
 * Exact arithmetic (where the pages are silent, these are the readings):
 *   s_tensor = fl32(amax / 2688)          (2688 = 6 * 448; amax == 0 -> 1)
 *   d6       = fl32(6 * s_tensor)
 *   s_block  = E4M3(fl32(amax_blk / d6))  (round to nearest even, satfinite)
 *   den      = fl32(value(s_block) * s_tensor)
 *   code_i   = E2M1(fl32(x_i / den))      (nearest, ties to even code,
 *                                          saturating; sign copied, so a
 *                                          negative value rounding to zero
 *                                          gives code 0x8; den == 0 gives
 *                                          signed-zero codes)
 *   fp8_i    = E4M3(fl32(fl32(|code_i| * value(s_block)) * s_tensor)) with
 *              the code's sign as the FP8 sign bit
 *   out[b][h] = softmax(q[b][h] . K^T * softmax_scale) . V over the first
 *              seq_lens[b] tokens of KV head h / (H_q / H_kv), using the FP8
 *              values of K and V; an empty sequence gives a zero row.
 *
 * Memory layout of one cache plane (K or V; caller-owned device memory):
 *   codes  : uint8 [B][H_kv][S_max][D/2]; byte j of a token row holds
 *            element 2j in its low nibble and element 2j+1 in its high nibble
 *   scales : uint8 [B][H_kv][S_max][D/16]; byte j scales elements 16j..16j+15
 *   Both pointers 16-byte aligned; S_max a multiple of 16; D in {64, 128}.
 *
 * Conventions for every call:
 *   - All pointers named d_* or described as device memory are CUDA device
 *     pointers on the current device; plane structs and sizes are host data.
 *   - Calls are asynchronous on `stream` (0 = legacy default stream) and
 *     allocate nothing.  The return value reports host-side validation and
 *     launch errors only.
 *   - Conditions found on the device (a sequence past S_max, a non-finite
 *     or non-positive tensor scale, a pipeline wait that gave up) are written
 *     to *d_status (int32, device memory, may be NULL): the first error code
 *     is kept (compare-and-swap from 0); the caller zeroes it.
 *   - No call aborts, traps or throws.
 */
#ifndef NVFP4KV_H
#define NVFP4KV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* nvfp4_stream_t; /* same type as cudaStream_t */

typedef enum {
    NVFP4_OK = 0,
    NVFP4_ERR_INVALID_ARG = 1,  /* bad pointer, size, alignment or shape */
    NVFP4_ERR_UNSUPPORTED = 2,  /* valid request this build does not handle */
    NVFP4_ERR_CAPACITY = 3,     /* a sequence would pass S_max */
    NVFP4_ERR_NONFINITE = 4,    /* non-finite data or tensor scale */
    NVFP4_ERR_CUDA = 5,         /* a CUDA runtime call failed */
    NVFP4_ERR_TIMEOUT = 6,      /* a bounded device-side wait gave up */
    NVFP4_ERR_WORKSPACE = 7     /* workspace missing or too small */
} nvfp4_status;

typedef enum {
    NVFP4_IN_BF16 = 0,          /* bfloat16 inputs */
    NVFP4_IN_F32 = 1            /* float32 inputs */
} nvfp4_dtype;

/* One NVFP4 cache plane (K or V).  The struct lives in host memory; the
 * two arrays it points to live in device memory (layout above). */
typedef struct {
    uint8_t* codes;   /* [B][H_kv][S_max][D/2] */
    uint8_t* scales;  /* [B][H_kv][S_max][D/16] */
    int32_t B;        /* sequences */
    int32_t H_kv;     /* KV heads */
    int32_t S_max;    /* token capacity per sequence, multiple of 16 */
    int32_t D;        /* head_dim, 64 or 128 */
} nvfp4_kv_plane;

/* One paged NVFP4 cache plane ([NVFP4-KV] "学術研究との関連": vLLM's
 * PagedAttention block management is orthogonal to the NVFP4 cache and
 * combines with it).  A pool of pages, each holding page_tokens token slots
 * of every KV head, and a block table that maps (sequence, logical page) to a
 * pool page.  The struct lives in host memory; the arrays in device memory.
 *   codes       uint8 [num_pages][H_kv][page_tokens][D/2], 16-byte aligned
 *   scales      uint8 [num_pages][H_kv][page_tokens][D/16], 16-byte aligned
 *   block_table int32 [B][max_pages]: token t of sequence b lives in pool page
 *               block_table[b * max_pages + t / page_tokens], slot
 *               t % page_tokens; entries past a sequence's length are unread
 * Element encoding, packing and scales are those of nvfp4_kv_plane.  The
 * capacity of a sequence is max_pages * page_tokens tokens. */
typedef struct {
    uint8_t* codes;
    uint8_t* scales;
    const int32_t* block_table;
    int32_t num_pages;    /* pages in the pool, >= 1 */
    int32_t H_kv;         /* KV heads */
    int32_t page_tokens;  /* token slots per page, a multiple of 128 */
    int32_t D;            /* head_dim, 64 or 128 */
    int32_t B;            /* sequences (rows of the block table) */
    int32_t max_pages;    /* block-table entries per sequence, >= 1 */
} nvfp4_kv_paged_plane;

/* Human-readable name of a status value (static string). */
const char* nvfp4_status_string(int status);

/* Library version string (static). */
const char* nvfp4_version(void);

/* Testing hook for the failure path of the tensor-core attention kernel
 * (head_dim 128, bf16 queries).  Its pipeline waits (one role waiting for
 * another through a shared-memory barrier) give up after `polls` sleeping
 * polls of up to 20 us each: the kernel then reports NVFP4_ERR_TIMEOUT
 * through *d_status, skips its remaining work, waits (bounded) for the copies
 * and MMAs it has issued, releases its tensor memory and returns.  polls = 0
 * gives up at once unless the awaited phase has already completed; polls < 0
 * restores the default (65536).  Applies to later calls from every thread.
 * Host-only; needs no GPU. */
void nvfp4_set_wait_limit(int64_t polls);

/* Bytes of ONE plane (codes + scales) for the given shape: B * H_kv * S_max *
 * (D/2 + D/16).  Per element that is 4 code bits plus 8/16 scale bits = 4.5
 * bits, the format behind the memory table in [NVFP4-KV] "メモリ削減効果"
 * (3.5x smaller than FP16, about 1.8x smaller than FP8).  Returns 0 for
 * invalid shapes.  Host-only; needs no GPU. */
size_t nvfp4_cache_bytes(int B, int H_kv, int S_max, int D);

/* Calibrate the per-tensor scale ([NVFP4-KV] "E2M1 + 2レベルスケーリング",
 * level 2: one FP32 scale per tensor).
 *   x          device, n elements of `dtype` (any alignment)
 *   d_s_tensor device float, written with fl32(amax / 2688), or 1.0 when
 *              amax == 0.  If any element is Inf/NaN, *d_s_tensor is set to
 *              NaN and NVFP4_ERR_NONFINITE goes to *d_status.
 * Launches a 4-byte memset and two kernels on `stream`.  n == 0 gives 1.0. */
nvfp4_status nvfp4_calib_tensor_scale(const void* x, nvfp4_dtype dtype, int64_t n,
                                      float* d_s_tensor, int32_t* d_status,
                                      nvfp4_stream_t stream);

/* Quantize n_new tokens per sequence and append them to a plane
 * ([NVFP4-KV] "量子化・逆量子化フロー": new K/V are quantized to NVFP4 in
 * 16-element blocks and stored in the cache).
 *   x_new        device [B][n_new][H_kv][D] of `dtype`, 16-byte aligned
 *   d_start_pos  device int32 [B]: tokens go to slots start..start+n_new-1
 *   d_new_lens   device int32 [B] or NULL: written with start + n_new; must
 *                not alias d_start_pos
 *   d_s_tensor   device float, the tensor scale from calibration (> 0)
 *   plane        host struct describing the destination plane
 * A sequence with start < 0 or start + n_new > S_max is skipped entirely and
 * NVFP4_ERR_CAPACITY goes to *d_status; a non-finite or non-positive tensor
 * scale skips everything with NVFP4_ERR_NONFINITE.  n_new == 0 is a no-op. */
nvfp4_status nvfp4_kv_quantize_append(const void* x_new, nvfp4_dtype dtype, int n_new,
                                      const int32_t* d_start_pos, int32_t* d_new_lens,
                                      const float* d_s_tensor, const nvfp4_kv_plane* plane,
                                      int32_t* d_status, nvfp4_stream_t stream);

/* MXFP4 cache plane bytes: B * H_kv * S_max * (D/2 + D/32) -- 4 code bits
 * plus one E8M0 scale byte per 32 elements = 4.25 bits per element.  Returns
 * 0 for invalid sizes (D must be a multiple of 32). */
size_t mxfp4_cache_bytes(int B, int H_kv, int S_max, int D);

/* Quantize n_new tokens per sequence to MXFP4 and append them to a plane:
 * the OCP format that [NVFP4-KV] "MXFP4との比較" compares NVFP4 with --
 * 32-element blocks along head_dim, one E8M0 (power-of-two) scale per block,
 * no tensor scale.  The scale exponent is floor(log2(amax_blk)) - 2 clamped
 * to [-127, 127] (the OCP MX rule; the page fixes only block size and scale
 * type), stored as the E8M0 byte exponent + 127; codes are
 * E2M1_RNE_sat(x / 2^exponent), packed as for NVFP4.
 *   x_new, dtype, n_new, d_start_pos, d_new_lens, d_status, stream: as for
 *                nvfp4_kv_quantize_append
 *   plane        codes [B][H_kv][S_max][D/2] and scales [B][H_kv][S_max][D/32]
 *                (one E8M0 byte per 32 elements), both 16-byte aligned
 * A sequence with start < 0 or start + n_new > S_max is skipped and
 * NVFP4_ERR_CAPACITY goes to *d_status; a block holding NaN or Inf gets the
 * E8M0 NaN byte 0xFF and zero codes, and NVFP4_ERR_NONFINITE goes to
 * *d_status (the first error reported wins).  n_new == 0 is a no-op. */
nvfp4_status mxfp4_kv_quantize_append(const void* x_new, nvfp4_dtype dtype, int n_new,
                                      const int32_t* d_start_pos, int32_t* d_new_lens,
                                      const nvfp4_kv_plane* plane, int32_t* d_status,
                                      nvfp4_stream_t stream);

/* nvfp4_kv_quantize_append into a paged plane ([NVFP4-KV] "学術研究との関連":
 * PagedAttention's block management combines with the NVFP4 cache): the slot
 * of token t of sequence b is found through the block table.  Capacity errors as for
 * contiguous planes (start + n_new > max_pages * page_tokens); a block-table
 * entry outside [0, num_pages) skips that token's blocks and reports
 * NVFP4_ERR_INVALID_ARG through *d_status. */
nvfp4_status nvfp4_kv_quantize_append_paged(const void* x_new, nvfp4_dtype dtype, int n_new,
                                            const int32_t* d_start_pos, int32_t* d_new_lens,
                                            const float* d_s_tensor,
                                            const nvfp4_kv_paged_plane* plane, int32_t* d_status,
                                            nvfp4_stream_t stream);

/* Quantize-append the same new tokens into the K and the V plane in one
 * launch ([NVFP4-KV] "量子化・逆量子化フロー": K and V are both quantized
 * on append).  Same results, arguments and errors as two calls of
 * nvfp4_kv_quantize_append (K with d_s_tensor_k into k, V with d_s_tensor_v
 * into v); the planes must agree in B, H_kv, S_max and D.  d_new_lens, if
 * given, is written once. */
nvfp4_status nvfp4_kv_quantize_append_kv(const void* x_k, const void* x_v, nvfp4_dtype dtype,
                                         int n_new, const int32_t* d_start_pos, int32_t* d_new_lens,
                                         const float* d_s_tensor_k, const float* d_s_tensor_v,
                                         const nvfp4_kv_plane* k, const nvfp4_kv_plane* v,
                                         int32_t* d_status, nvfp4_stream_t stream);

/* Dequantize a plane to FP8 E4M3 bytes ([NVFP4-KV] "量子化・逆量子化フロー":
 * NVFP4 -> FP8 before attention).
 *   d_seq_lens device int32 [B]; only slots t < seq_lens[b] are written
 *   out_e4m3   device uint8 [B][H_kv][S_max][D], 16-byte aligned
 * Lengths past S_max are clamped and reported as NVFP4_ERR_CAPACITY. */
nvfp4_status nvfp4_kv_dequant_fp8(const nvfp4_kv_plane* plane, const float* d_s_tensor,
                                  const int32_t* d_seq_lens, uint8_t* out_e4m3,
                                  int32_t* d_status, nvfp4_stream_t stream);

/* Workspace bytes nvfp4_decode_attention needs on the current device for
 * this shape: the split-K partial results and per-(sequence, KV head)
 * arrival counters of the stream-K split ([llama.cpp digest] "CUDA/Vulkan/
 * HEXAGONの主要バグ修正": the split is sized to the GPU's SM count, so that
 * no SM idles).  The size depends on the current device's SM count: query
 * it on the device that will run the calls.  Returns 0 for invalid shapes.
 * The workspace must be zero-filled once after allocation; every completed
 * call leaves its counters at zero again, so it can be reused without
 * clearing.  Calls that share one workspace must not overlap on the GPU. */
size_t nvfp4_decode_attention_workspace(int B, int H_q, int H_kv, int D);

/* Decode attention over an NVFP4 cache with FP8 dequantization fused in
 * ([NVFP4-KV] "量子化・逆量子化フロー": FP8 attention and the context matmul
 * on the dequantized cache; [FR-lesson] "Le type de Blackwell": FP32
 * accumulator).  One query token per sequence, grouped-query attention.
 *   q            device [B][H_q][D] of `q_dtype`, 16-byte aligned
 *   H_q          query heads; H_q % H_kv == 0 and H_q / H_kv <= 16
 *   k, v         host structs of the K and V planes (same B, H_kv, S_max, D)
 *   d_s_tensor_k, d_s_tensor_v  device floats
 *   d_seq_lens   device int32 [B], tokens to attend per sequence (<= S_max)
 *   softmax_scale  0 selects 1/sqrt(D)
 *   out          device float [B][H_q][D], 16-byte aligned
 *   workspace    device, >= nvfp4_decode_attention_workspace(...) bytes,
 *                zero-filled once (see above), 16-byte aligned
 * Lengths past S_max are clamped and reported as NVFP4_ERR_CAPACITY.
 * Batches larger than 512 sequences are processed in launches of 512.
 * NVFP4_ERR_UNSUPPORTED when min(B, 512) * H_kv * ceil(S_max / 32) exceeds
 * 2^31 - 1 (the work split counts 32-token tiles in 32 bits). */
nvfp4_status nvfp4_decode_attention(const void* q, nvfp4_dtype q_dtype, int H_q,
                                    const nvfp4_kv_plane* k, const nvfp4_kv_plane* v,
                                    const float* d_s_tensor_k, const float* d_s_tensor_v,
                                    const int32_t* d_seq_lens, float softmax_scale,
                                    float* out, void* workspace, size_t workspace_bytes,
                                    int32_t* d_status, nvfp4_stream_t stream);

/* Chunked-prefill attention over the cache ([NVFP4-KV] "推論速度": the NVFP4
 * cache shortens time to first token, the prefill side; "量子化・逆量子化フロー":
 * attention runs over the cache dequantized to FP8).  A chunk of C prompt
 * tokens per sequence, already appended to the cache at slots start_pos[b] ..
 * start_pos[b] + C - 1, attends causally: query i of sequence b sees the
 * cache tokens t <= start_pos[b] + i.  Runs on the tensor cores (tcgen05,
 * f16 MMAs with fp32 accumulation; the cache's FP8 values are exact in f16,
 * and so is a bf16 query after a power-of-two row scaling, for every element
 * at least 2^-31 times the row's largest magnitude (smaller ones are rounded
 * to f16's subnormal grid); the probabilities enter as two f16 terms, about
 * 22 significant bits).
 *   q           device [B][C][H_q][128] bf16, 16-byte aligned (fp32 queries:
 *               NVFP4_ERR_UNSUPPORTED)
 *   C           chunk length (0: nothing to do)
 *   H_q         query heads, a multiple of H_kv with H_q / H_kv <= 128
 *   k, v        contiguous planes of head_dim 128 (other D: NVFP4_ERR_UNSUPPORTED)
 *   d_start_pos device int32 [B], the chunk's first position per sequence
 *   softmax_scale  0 selects 1 / sqrt(128)
 *   out         device float [B][C][H_q][128], overwritten
 * A sequence with start_pos < 0 or start_pos + C > S_max is skipped and
 * NVFP4_ERR_CAPACITY goes to *d_status (its output rows are left as they
 * were); a non-finite or non-positive tensor scale reports
 * NVFP4_ERR_NONFINITE.  Host errors as for nvfp4_decode_attention. */
nvfp4_status nvfp4_prefill_attention(const void* q, nvfp4_dtype q_dtype, int C, int H_q,
                                     const nvfp4_kv_plane* k, const nvfp4_kv_plane* v,
                                     const float* d_s_tensor_k, const float* d_s_tensor_v,
                                     const int32_t* d_start_pos, float softmax_scale, float* out,
                                     int32_t* d_status, nvfp4_stream_t stream);

/* Append one decode token per sequence, then attend over the cache including
 * it, in one call ([NVFP4-KV] "量子化・逆量子化フロー": the new K/V are
 * quantized to NVFP4 as they enter the cache, then FP8 attention runs over
 * the dequantized cache).  Equivalent to nvfp4_kv_quantize_append_kv with
 * n_new = 1 followed by nvfp4_decode_attention with seq_lens = start + 1, and
 * bit-identical to that pair: same codes, scale bytes and output.  On the
 * tensor-core path (head_dim 128, bf16 queries) it is ONE kernel launch (plus
 * the split-K merge): the CTA whose range holds a sequence's last tile
 * quantizes that sequence's new token before it loads the tile; other shapes
 * run the append kernel first.
 *   x_k_new, x_v_new  device [B][1][H_kv][D] of x_dtype, 16-byte aligned
 *   d_start_pos       device int32 [B]: the new token goes to slot start_pos[b]
 *                     and the attention covers start_pos[b] + 1 tokens
 *   d_new_lens        device int32 [B] or NULL: receives start_pos[b] + 1; must
 *                     not alias d_start_pos
 *   every other argument as for nvfp4_decode_attention (seq_lens excepted)
 * A sequence with start_pos < 0 or start_pos + 1 > S_max is not appended;
 * NVFP4_ERR_CAPACITY goes to *d_status and its attention length is clamped
 * to [0, S_max].  A non-finite or non-positive tensor scale skips the append
 * with NVFP4_ERR_NONFINITE. */
nvfp4_status nvfp4_decode_attention_append(const void* q, nvfp4_dtype q_dtype, int H_q,
                                           const void* x_k_new, const void* x_v_new, nvfp4_dtype x_dtype,
                                           const int32_t* d_start_pos, int32_t* d_new_lens,
                                           const nvfp4_kv_plane* k, const nvfp4_kv_plane* v,
                                           const float* d_s_tensor_k, const float* d_s_tensor_v,
                                           float softmax_scale, float* out, void* workspace,
                                           size_t workspace_bytes, int32_t* d_status,
                                           nvfp4_stream_t stream);

/* nvfp4_decode_attention over paged K and V planes.  k and v share one block
 * table (the same pointer) and agree in B, H_kv, page_tokens, max_pages, D;
 * their pools may differ.  Arguments, results and errors are those of
 * nvfp4_decode_attention with S_max = max_pages * page_tokens; the workspace
 * size is nvfp4_decode_attention_workspace(B, H_q, H_kv, D).  A block-table
 * entry outside [0, num_pages) is reported as NVFP4_ERR_INVALID_ARG through
 * *d_status and page 0 is read in its place (no access leaves the pool). */
nvfp4_status nvfp4_decode_attention_paged(const void* q, nvfp4_dtype q_dtype, int H_q,
                                          const nvfp4_kv_paged_plane* k,
                                          const nvfp4_kv_paged_plane* v,
                                          const float* d_s_tensor_k, const float* d_s_tensor_v,
                                          const int32_t* d_seq_lens, float softmax_scale,
                                          float* out, void* workspace, size_t workspace_bytes,
                                          int32_t* d_status, nvfp4_stream_t stream);

/* Decode attention for callers that cannot allocate device memory.
 *
 * The pages describe no such call; it exists for users of this library whose
 * code may not call cudaMalloc or any allocating routine -- code running inside
 * a framework or host whose memory pool owns every device allocation, plugins
 * that receive only their input and output buffers, or paths that must not
 * allocate while other work is in flight.
 *
 * Same arguments and results as nvfp4_decode_attention, without the workspace:
 * the split-K partial results and arrival counters live in one file-scope
 * device array of NVFP4_NOALLOC_SCRATCH_BYTES (8 MiB), held by every GPU that
 * loads this library until the process exits.  Behaviour:
 *   - Shapes whose workspace (nvfp4_decode_attention_workspace) exceeds the
 *     buffer are rejected with NVFP4_ERR_WORKSPACE before anything is queued.
 *   - The first call on each device looks up the buffer's device address with
 *     that device current; make that first call before any stream capture.
 *   - Each call clears the arrival counters with a memset on `stream`, then
 *     runs the same kernel as nvfp4_decode_attention.
 *   - Every call on a device shares the one buffer and leaves its contents
 *     behind: calls whose execution overlaps on the GPU (other streams, other
 *     host threads) race and give wrong results; serialize them.
 *   - Allocates nothing: no cudaMalloc, cudaFree or allocating library call. */
#define NVFP4_NOALLOC_SCRATCH_BYTES ((size_t)8 << 20)
nvfp4_status nvfp4_decode_attention_noalloc(const void* q, nvfp4_dtype q_dtype, int H_q,
                                            const nvfp4_kv_plane* k, const nvfp4_kv_plane* v,
                                            const float* d_s_tensor_k, const float* d_s_tensor_v,
                                            const int32_t* d_seq_lens, float softmax_scale,
                                            float* out, int32_t* d_status, nvfp4_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* NVFP4KV_H */

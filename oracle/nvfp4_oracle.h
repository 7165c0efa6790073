/*
 * nvfp4_oracle.h -- plain, slow CPU oracle for the NVFP4 KV-cache path.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference legs of bench.py may load this library.  The
 * product (libnvfp4kv.so and its Python binding) never calls it, and this
 * file shares no code, header, table or constant with the CUDA side.
 *
 * Sources (web pages; cited by title and section):
 *   [P3] "NVIDIA解説: NVFP4 KV Cacheで長コンテキストLLM推論を最適化 -- メモリ50%削減・
 *        TTFT 3倍高速化" (0h-n0.github.io, a summary of NVIDIA's technical blog).
 *        Sections used: "KV Cacheのメモリボトルネック" (memory formula),
 *        "E2M1 + 2レベルスケーリング" (format and two-level scaling),
 *        "量子化・逆量子化フロー" (quantize on append, dequantize to FP8,
 *        FP8 attention), "メモリ削減効果" (memory-reduction table),
 *        "MXFP4との比較" (MXFP4: 32-element blocks, E8M0 power-of-two scales).
 *   [P1] "TensorRT-LLM rc17 が SM121（DGX Spark）向けに NVFP4 MoE バックエンドと
 *        NVFP4 KV キャッシュを追加", section "物語の KV キャッシュ側"
 *        (values are dequantized from NVFP4 to FP8 before attention).
 *   [P5] "Compilation d'inferences spécialisées en matériel FP8 et NVFP4 sur
 *        Blackwell", section "Le type de Blackwell" (FP32 attention accumulator).
 *
 * Readings where the pages are silent (each one is listed with its reason in
 * the repository's design notes):
 *   R1  E2M1 code = sign bit 3, exponent bits 2..1 (bias 1), mantissa bit 0.
 *   R2  E4M3 is the OCP "E4M3FN" byte: bias 7, no infinity, 0x7F/0xFF = NaN,
 *       largest finite 448.  Conversions round to nearest, ties to even,
 *       and saturate finite overflow to +-448.
 *   R3  s_tensor = amax / (6 * 448) in fp32 (6 = largest E2M1, 448 = largest
 *       E4M3); amax == 0 gives s_tensor = 1.
 *   R4  Blocks are 16 consecutive elements along head_dim of one token.
 *   R5  Quantize: d6 = fl32(6*s_tensor); r = fl32(amax_blk/d6);
 *       sb = E4M3(r); den = fl32(value(sb)*s_tensor);
 *       code_i = E2M1(fl32(x_i/den)); den == 0 gives signed-zero codes.
 *   R6  Packing: byte j of a token row = code(2j) | code(2j+1) << 4.
 *   R7  Dequant to FP8: E4M3(fl32(fl32(|c|*value(sb)) * s_tensor)) with the
 *       code's sign bit copied to the FP8 sign bit (so -0 codes give 0x80).
 *   R8  Attention in fp64 over the FP8 values: query head h reads KV head
 *       h / (H_q/H_kv); empty sequences give a zero row.
 *   R13 MXFP4 scale: the pages fix only "E8M0, powers of two".  The OCP MX
 *       rule is taken: X = 2^e, e = floor(log2(amax_blk)) - 2 (2 is the
 *       exponent of E2M1's largest value 6 = 1.5 * 2^2), clamped to
 *       [-127, 127]; amax_blk == 0 gives e = -127.  E8M0 byte = e + 127.
 *   R14 MXFP4 codes: code_i = E2M1(x_i / X) (exact, X is a power of two),
 *       packed as R6; a block is 32 consecutive elements along head_dim of
 *       one token; there is no tensor scale.
 *   R15 A block holding NaN or +-Inf gets the E8M0 NaN byte 0xFF and zero
 *       codes, and the append reports ORACLE_ERR_NONFINITE.
 *   R17 Chunked prefill: query i of a chunk starting at position start sees
 *       cache tokens 0..start+i (causal, its own K/V appended first).
 */
#ifndef NVFP4_ORACLE_H
#define NVFP4_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Status values of the oracle (its own; unrelated to the product's). */
#define ORACLE_OK 0
#define ORACLE_ERR_ARG 1
#define ORACLE_ERR_NONFINITE 4
#define ORACLE_ERR_CAPACITY 3

/* ---- element formats ([P3] "E2M1 + 2レベルスケーリング") ---- */
double  oracle_e2m1_value(uint8_t code);            /* code 0..15 -> value */
double  oracle_e4m3_value(uint8_t byte);            /* byte -> value (NaN for 0x7F/0xFF) */
uint8_t oracle_e2m1_encode(float v);                /* RNE, ties to even, saturating */
uint8_t oracle_e4m3_encode(float v);                /* RNE, ties to even, satfinite */
void    oracle_e2m1_encode_array(const float* v, int64_t n, uint8_t* out);
void    oracle_e4m3_encode_array(const float* v, int64_t n, uint8_t* out);

/* ---- calibration of the per-tensor scale (R3) ---- */
int     oracle_tensor_scale(const float* x, int64_t n, float* s_tensor);

/* ---- one 16-element micro-block (R5, R6) ---- */
void    oracle_quantize_block(const float* x16, float s_tensor,
                              uint8_t* packed8, uint8_t* scale_byte);

/* ---- append n_new tokens into the cache planes ----
 * x_new   : fp32 [B][n_new][H_kv][D]
 * start   : int32 [B], first cache slot written for each sequence
 * codes   : uint8 [B][H_kv][S_max][D/2]
 * scales  : uint8 [B][H_kv][S_max][D/16]
 * Returns ORACLE_ERR_CAPACITY (and writes nothing for that sequence) when
 * start[b] + n_new > S_max. */
int     oracle_quantize_append(const float* x_new, int B, int n_new, int H_kv, int D,
                               const int32_t* start, float s_tensor,
                               uint8_t* codes, uint8_t* scales, int S_max);

/* ---- dequantize one code (R7) and whole planes ---- */
uint8_t oracle_dequant_fp8(uint8_t code, uint8_t scale_byte, float s_tensor);
/* out: uint8 [B][H_kv][S_max][D]; only slots t < seq_lens[b] are written. */
void    oracle_dequant_planes(const uint8_t* codes, const uint8_t* scales,
                              int B, int H_kv, int S_max, int D, float s_tensor,
                              const int32_t* seq_lens, uint8_t* out);

/* ---- decode attention over FP8 K/V (R8), fp64 ----
 * q      : fp32 [B][H_q][D]
 * k8, v8 : E4M3 bytes [B][H_kv][S_max][D]
 * out    : fp64 [B][H_q][D]
 * softmax_scale == 0 selects 1/sqrt(D). */
void    oracle_decode_attention_fp8(const float* q, const uint8_t* k8, const uint8_t* v8,
                                    int B, int H_q, int H_kv, int S_max, int D,
                                    const int32_t* seq_lens, double softmax_scale,
                                    double* out);

/* Full path from the NVFP4 planes: dequantize every needed element with
 * oracle_dequant_fp8 and run the fp64 attention above.  Same shapes. */
void    oracle_decode_attention_nvfp4(const float* q,
                                      const uint8_t* k_codes, const uint8_t* k_scales,
                                      const uint8_t* v_codes, const uint8_t* v_scales,
                                      float s_tensor_k, float s_tensor_v,
                                      int B, int H_q, int H_kv, int S_max, int D,
                                      const int32_t* seq_lens, double softmax_scale,
                                      double* out);

/* ---- the exact reconstruction x^ = value(code) * value(sb) * s_tensor
 * ([P3] "E2M1 + 2レベルスケーリング"), fp64 [B][H_kv][S_max][D], slots
 * t < seq_lens[b] only.  Used to measure quantization error. */
void    oracle_nvfp4_reconstruct_planes(const uint8_t* codes, const uint8_t* scales,
                                        int B, int H_kv, int S_max, int D, float s_tensor,
                                        const int32_t* seq_lens, double* out);

/* ---- MXFP4 ([P3] "MXFP4との比較"; readings R13-R15) ----
 * scales : uint8 [B][H_kv][S_max][D/32], one E8M0 byte per 32 elements;
 * codes  : uint8 [B][H_kv][S_max][D/2] as for NVFP4. */
double  oracle_e8m0_value(uint8_t byte);            /* 2^(byte - 127); NaN for 0xFF */
/* Returns ORACLE_OK, or ORACLE_ERR_NONFINITE for a block with NaN/Inf (R15). */
int     oracle_mxfp4_quantize_block(const float* x32, uint8_t* packed16, uint8_t* scale_byte);
/* Same placement and capacity rules as oracle_quantize_append; returns
 * ORACLE_ERR_CAPACITY or ORACLE_ERR_NONFINITE (capacity wins) or ORACLE_OK. */
int     oracle_mxfp4_quantize_append(const float* x_new, int B, int n_new, int H_kv, int D,
                                     const int32_t* start, uint8_t* codes, uint8_t* scales,
                                     int S_max);
/* x^ = value(code) * value(e8m0), fp64, slots t < seq_lens[b] only. */
void    oracle_mxfp4_reconstruct_planes(const uint8_t* codes, const uint8_t* scales,
                                        int B, int H_kv, int S_max, int D,
                                        const int32_t* seq_lens, double* out);
double  oracle_mxfp4_bits_per_element(void);

/* ---- chunked prefill attention (reading R17), fp64 ----
 * q     : fp32 [B][C][H_q][D], query i of sequence b at position start[b] + i
 * start : int32 [B]; the caller guarantees start[b] + C <= S_max
 * out   : fp64 [B][C][H_q][D]; query i attends to cache tokens
 *         0 .. start[b] + i (its own K/V included), FP8 values as R7. */
void    oracle_prefill_attention_nvfp4(const float* q,
                                       const uint8_t* k_codes, const uint8_t* k_scales,
                                       const uint8_t* v_codes, const uint8_t* v_scales,
                                       float s_tensor_k, float s_tensor_v,
                                       int B, int C, int H_q, int H_kv, int S_max, int D,
                                       const int32_t* start, double softmax_scale, double* out);

/* ---- memory model ([P3] "KV Cacheのメモリボトルネック") ----
 * KV bytes = 2 (K and V) * layers * n_h * s * b * bytes per head vector. */
double  oracle_kv_bytes(int64_t layers, int64_t n_h, int64_t d_h, int64_t s, int64_t b,
                        double bits_per_element);
double  oracle_nvfp4_bits_per_element(void);

void    oracle_set_threads(int n);
int     oracle_get_threads(void);

#ifdef __cplusplus
}
#endif
#endif

/*
 * nvfp4_oracle.c -- plain CPU oracle for the NVFP4 KV-cache path.
 *
 * TEST INFRASTRUCTURE ONLY (see nvfp4_oracle.h).  Every function is written
 * for a reader checking it against the pages by eye: no blocking, no fusion,
 * no lookup tables.  Conversions are "nearest representable value, ties to
 * the even code" searched over the format's value set; attention is a direct
 * fp64 softmax.  Build with -ffp-contract=off and without -ffast-math so that
 * every fp32 operation is one IEEE round-to-nearest-even operation.
 */
#include "nvfp4_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* --------------------------------------------------------------------------
 * E2M1: [P3] "E2M1 + 2レベルスケーリング" gives sign 1 bit, exponent 2 bits,
 * mantissa 1 bit and a range of about [-6, +6].  Reading R1: exponent bias 1,
 * exponent field 0 is subnormal with value mantissa * 0.5.
 * ------------------------------------------------------------------------ */
double oracle_e2m1_value(uint8_t code) {
    int sign = (code >> 3) & 1;
    int e = (code >> 1) & 3;
    int m = code & 1;
    double mag;
    if (e == 0)
        mag = 0.5 * m;                              /* subnormal: m * 2^(1-1) * 2^-1 */
    else
        mag = (1.0 + 0.5 * m) * ldexp(1.0, e - 1);  /* normal: (1 + m/2) * 2^(e-1) */
    return sign ? -mag : mag;
}

/* Nearest E2M1 magnitude, ties to the even code (mantissa bit 0).  Anything
 * past the largest value lands on it (saturation is the nearest point).
 * The sign bit is copied from v, so negative values that round to zero give
 * the code 0x8 (reading R5/R7).  NaN input is a caller error; it maps to 0x7. */
uint8_t oracle_e2m1_encode(float v) {
    if (isnan(v)) return 0x7;
    double a = fabs((double)v);
    int best = 0;
    double best_d = INFINITY;
    if (a >= oracle_e2m1_value(0x7)) {
        /* at or past the largest value: saturate.  (For huge |v| the two
         * distances to 4 and 6 round to the same double, so the search
         * below cannot be trusted there.) */
        best = 0x7;
        if (signbit(v)) best |= 0x8;
        return (uint8_t)best;
    }
    for (int c = 0; c < 8; ++c) {
        double d = fabs(a - oracle_e2m1_value((uint8_t)c));
        if (d < best_d || (d == best_d && (c & 1) == 0)) {
            best = c;
            best_d = d;
        }
    }
    if (signbit(v)) best |= 0x8;
    return (uint8_t)best;
}

/* --------------------------------------------------------------------------
 * E4M3: [P3] names "E4M3 FP8" as the micro-block scale format.  Reading R2:
 * the OCP E4M3FN encoding -- bias 7, exponent field 0 subnormal (m * 2^-9),
 * no infinity, S.1111.111 is NaN, largest finite 448.
 * ------------------------------------------------------------------------ */
double oracle_e4m3_value(uint8_t byte) {
    int sign = (byte >> 7) & 1;
    int e = (byte >> 3) & 0xF;
    int m = byte & 7;
    double mag;
    if (e == 15 && m == 7) return NAN;
    if (e == 0)
        mag = m * ldexp(1.0, -9);                      /* subnormal */
    else
        mag = (1.0 + m / 8.0) * ldexp(1.0, e - 7);     /* normal */
    return sign ? -mag : mag;
}

/* Nearest finite E4M3 magnitude, ties to the even code (mantissa lsb 0);
 * values past 448 (and +-inf) saturate to 448 ("satfinite"), NaN -> 0x7F.
 * The positive finite codes 0x00..0x7E are increasing in value, so the search
 * finds the last code not above |v| and compares it with the next one. */
uint8_t oracle_e4m3_encode(float v) {
    if (isnan(v)) return 0x7F;
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    double a = fabs((double)v);
    if (a >= oracle_e4m3_value(0x7E)) return (uint8_t)(sign | 0x7E);
    int lo = 0, hi = 0x7E;                 /* value(lo) <= a < value(hi) */
    while (hi - lo > 1) {
        int mid = (lo + hi) / 2;
        if (oracle_e4m3_value((uint8_t)mid) <= a) lo = mid; else hi = mid;
    }
    double dlo = a - oracle_e4m3_value((uint8_t)lo);
    double dhi = oracle_e4m3_value((uint8_t)hi) - a;
    int pick;
    if (dlo < dhi) pick = lo;
    else if (dhi < dlo) pick = hi;
    else pick = (lo & 1) == 0 ? lo : hi;   /* tie: even mantissa */
    return (uint8_t)(sign | pick);
}

void oracle_e2m1_encode_array(const float* v, int64_t n, uint8_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_e2m1_encode(v[i]);
}

void oracle_e4m3_encode_array(const float* v, int64_t n, uint8_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_e4m3_encode(v[i]);
}

/* --------------------------------------------------------------------------
 * Per-tensor scale.  [P3] "E2M1 + 2レベルスケーリング", level 2: one FP32
 * scale for the whole tensor; the pages only say it is calibrated (section
 * "TensorRT Model Optimizerによる実装").  Reading R3: amax maps onto the
 * largest product of an E2M1 value (6) and an E4M3 scale (448).
 * ------------------------------------------------------------------------ */
int oracle_tensor_scale(const float* x, int64_t n, float* s_tensor) {
    float amax = 0.0f;
    for (int64_t i = 0; i < n; ++i) {
        float a = fabsf(x[i]);
        if (!isfinite(a)) return ORACLE_ERR_NONFINITE;
        if (a > amax) amax = a;
    }
    if (amax == 0.0f) {
        *s_tensor = 1.0f;
        return ORACLE_OK;
    }
    const float six_times_448 = 6.0f * 448.0f;     /* 2688, exact in fp32 */
    *s_tensor = amax / six_times_448;
    return ORACLE_OK;
}

/* --------------------------------------------------------------------------
 * One micro-block.  [P3] "E2M1 + 2レベルスケーリング": x ~ x_q * s_block *
 * s_tensor with one E4M3 s_block per 16 elements.  Quantizing divides by the
 * scales (reading R5, the left-to-right order of the formula).
 * ------------------------------------------------------------------------ */
void oracle_quantize_block(const float* x16, float s_tensor,
                           uint8_t* packed8, uint8_t* scale_byte) {
    float amax_blk = 0.0f;
    for (int i = 0; i < 16; ++i) {
        float a = fabsf(x16[i]);
        if (a > amax_blk) amax_blk = a;
    }
    float d6 = 6.0f * s_tensor;
    float r = amax_blk / d6;
    uint8_t sb = oracle_e4m3_encode(r);
    float sb_value = (float)oracle_e4m3_value(sb);   /* exact in fp32 */
    float den = sb_value * s_tensor;
    uint8_t codes[16];
    for (int i = 0; i < 16; ++i) {
        if (den == 0.0f) {
            codes[i] = signbit(x16[i]) ? 0x8 : 0x0;
        } else {
            float y = x16[i] / den;
            codes[i] = oracle_e2m1_encode(y);
        }
    }
    /* reading R6: element 2j in the low nibble of byte j */
    for (int j = 0; j < 8; ++j)
        packed8[j] = (uint8_t)(codes[2 * j] | (codes[2 * j + 1] << 4));
    *scale_byte = sb;
}

/* [P3] "量子化・逆量子化フロー": a new token's K/V is quantized to NVFP4 in
 * 16-element blocks and appended to the cache. */
int oracle_quantize_append(const float* x_new, int B, int n_new, int H_kv, int D,
                           const int32_t* start, float s_tensor,
                           uint8_t* codes, uint8_t* scales, int S_max) {
    if (D % 16 != 0 || B < 0 || n_new < 0 || H_kv <= 0) return ORACLE_ERR_ARG;
    int status = ORACLE_OK;
    for (int b = 0; b < B; ++b) {
        if (start[b] < 0 || (int64_t)start[b] + n_new > S_max) {
            status = ORACLE_ERR_CAPACITY;
            continue;
        }
        for (int t = 0; t < n_new; ++t) {
            for (int h = 0; h < H_kv; ++h) {
                const float* row = x_new + (((int64_t)b * n_new + t) * H_kv + h) * D;
                int64_t slot = ((int64_t)b * H_kv + h) * S_max + (start[b] + t);
                for (int blk = 0; blk < D / 16; ++blk) {
                    oracle_quantize_block(row + 16 * blk, s_tensor,
                                          codes + slot * (D / 2) + 8 * blk,
                                          scales + slot * (D / 16) + blk);
                }
            }
        }
    }
    return status;
}

/* --------------------------------------------------------------------------
 * Dequantize to FP8.  [P3] "量子化・逆量子化フロー" and [P1] "物語の KV
 * キャッシュ側": at attention time the cache is dequantized from NVFP4 to FP8.
 * Reading R7: multiply in the formula's order, round once to fp32 per
 * product, then round the result to E4M3; the code's sign is the FP8 sign.
 * ------------------------------------------------------------------------ */
uint8_t oracle_dequant_fp8(uint8_t code, uint8_t scale_byte, float s_tensor) {
    float mag = (float)oracle_e2m1_value((uint8_t)(code & 0x7));
    float sb_value = (float)oracle_e4m3_value(scale_byte);
    float prod = mag * sb_value;           /* exact: at most 6 significant bits */
    float val = prod * s_tensor;
    uint8_t e = oracle_e4m3_encode(val);
    if (code & 0x8) e |= 0x80;
    return e;
}

void oracle_dequant_planes(const uint8_t* codes, const uint8_t* scales,
                           int B, int H_kv, int S_max, int D, float s_tensor,
                           const int32_t* seq_lens, uint8_t* out) {
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H_kv; ++h)
            for (int t = 0; t < seq_lens[b]; ++t) {
                int64_t slot = ((int64_t)b * H_kv + h) * S_max + t;
                for (int d = 0; d < D; ++d) {
                    uint8_t byte = codes[slot * (D / 2) + d / 2];
                    uint8_t code = (d % 2 == 0) ? (byte & 0xF) : (byte >> 4);
                    uint8_t sb = scales[slot * (D / 16) + d / 16];
                    out[slot * D + d] = oracle_dequant_fp8(code, sb, s_tensor);
                }
            }
}

/* The pages' reconstruction, x ~ x_q * s_block * s_tensor ([P3]
 * "E2M1 + 2レベルスケーリング"), in fp64 without the FP8 rounding of R7. */
void oracle_nvfp4_reconstruct_planes(const uint8_t* codes, const uint8_t* scales,
                                     int B, int H_kv, int S_max, int D, float s_tensor,
                                     const int32_t* seq_lens, double* out) {
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H_kv; ++h)
            for (int t = 0; t < seq_lens[b]; ++t) {
                int64_t slot = ((int64_t)b * H_kv + h) * S_max + t;
                for (int d = 0; d < D; ++d) {
                    uint8_t byte = codes[slot * (D / 2) + d / 2];
                    uint8_t code = (d % 2 == 0) ? (byte & 0xF) : (byte >> 4);
                    uint8_t sb = scales[slot * (D / 16) + d / 16];
                    out[slot * D + d] =
                        oracle_e2m1_value(code) * oracle_e4m3_value(sb) * (double)s_tensor;
                }
            }
}

/* --------------------------------------------------------------------------
 * MXFP4, the OCP format the pages compare NVFP4 with ([P3] "MXFP4との比較"):
 * blocks of 32 elements, one E8M0 scale that can only be a power of two, no
 * tensor scale.  E8M0 is a bare biased exponent: byte e + 127 is 2^e, 0xFF is
 * NaN (R13).
 * ------------------------------------------------------------------------ */
double oracle_e8m0_value(uint8_t byte) {
    if (byte == 0xFF) return NAN;
    return ldexp(1.0, (int)byte - 127);
}

int oracle_mxfp4_quantize_block(const float* x32, uint8_t* packed16, uint8_t* scale_byte) {
    double amax = 0.0;
    for (int i = 0; i < 32; ++i) {
        if (!isfinite(x32[i])) {                     /* R15 */
            for (int j = 0; j < 16; ++j) packed16[j] = 0;
            *scale_byte = 0xFF;
            return ORACLE_ERR_NONFINITE;
        }
        double a = fabs((double)x32[i]);
        if (a > amax) amax = a;
    }
    /* R13: X = 2^(floor(log2 amax) - 2), so amax / X lies in [4, 8): the
     * block's largest element lands on the top binade of E2M1 (4 or 6). */
    int e = -127;
    if (amax > 0.0) {
        int ex;
        frexp(amax, &ex);                            /* amax = m 2^ex, 0.5 <= m < 1 */
        e = (ex - 1) - 2;
        if (e < -127) e = -127;
        if (e > 127) e = 127;
    }
    double X = ldexp(1.0, e);
    uint8_t codes[32];
    for (int i = 0; i < 32; ++i)
        codes[i] = oracle_e2m1_encode((float)((double)x32[i] / X));   /* R14 */
    for (int j = 0; j < 16; ++j)                     /* R6 packing */
        packed16[j] = (uint8_t)(codes[2 * j] | (codes[2 * j + 1] << 4));
    *scale_byte = (uint8_t)(e + 127);
    return ORACLE_OK;
}

int oracle_mxfp4_quantize_append(const float* x_new, int B, int n_new, int H_kv, int D,
                                 const int32_t* start, uint8_t* codes, uint8_t* scales,
                                 int S_max) {
    if (D % 32 != 0 || B < 0 || n_new < 0 || H_kv <= 0) return ORACLE_ERR_ARG;
    int status = ORACLE_OK;
    for (int b = 0; b < B; ++b) {
        if (start[b] < 0 || (int64_t)start[b] + n_new > S_max) {
            status = ORACLE_ERR_CAPACITY;
            continue;
        }
        for (int t = 0; t < n_new; ++t)
            for (int h = 0; h < H_kv; ++h) {
                const float* row = x_new + (((int64_t)b * n_new + t) * H_kv + h) * D;
                int64_t slot = ((int64_t)b * H_kv + h) * S_max + (start[b] + t);
                for (int blk = 0; blk < D / 32; ++blk) {
                    int r = oracle_mxfp4_quantize_block(row + 32 * blk,
                                                        codes + slot * (D / 2) + 16 * blk,
                                                        scales + slot * (D / 32) + blk);
                    if (r != ORACLE_OK && status == ORACLE_OK) status = r;
                }
            }
    }
    return status;
}

void oracle_mxfp4_reconstruct_planes(const uint8_t* codes, const uint8_t* scales,
                                     int B, int H_kv, int S_max, int D,
                                     const int32_t* seq_lens, double* out) {
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H_kv; ++h)
            for (int t = 0; t < seq_lens[b]; ++t) {
                int64_t slot = ((int64_t)b * H_kv + h) * S_max + t;
                for (int d = 0; d < D; ++d) {
                    uint8_t byte = codes[slot * (D / 2) + d / 2];
                    uint8_t code = (d % 2 == 0) ? (byte & 0xF) : (byte >> 4);
                    uint8_t sb = scales[slot * (D / 32) + d / 32];
                    out[slot * D + d] = oracle_e2m1_value(code) * oracle_e8m0_value(sb);
                }
            }
}

/* --------------------------------------------------------------------------
 * Decode attention.  [P3] "量子化・逆量子化フロー": FP8 attention and the
 * context matmul run on the dequantized cache; [P5] "Le type de Blackwell":
 * the attention accumulator is FP32 -- the oracle uses fp64 throughout.
 * softmax(q K^T * scale) V for every (b, h) over the seq_lens[b] cached tokens.
 * ------------------------------------------------------------------------ */
static void attend_one(const float* q, const double* K, const double* V, int L, int D,
                       double scale, double* o) {
    if (L == 0) {
        for (int d = 0; d < D; ++d) o[d] = 0.0;
        return;
    }
    double* s = (double*)malloc(sizeof(double) * (size_t)L);
    double mx = -INFINITY;
    for (int t = 0; t < L; ++t) {
        double acc = 0.0;
        for (int d = 0; d < D; ++d) acc += (double)q[d] * K[(int64_t)t * D + d];
        s[t] = acc * scale;
        if (s[t] > mx) mx = s[t];
    }
    double l = 0.0;
    for (int t = 0; t < L; ++t) {
        s[t] = exp(s[t] - mx);
        l += s[t];
    }
    for (int d = 0; d < D; ++d) {
        double acc = 0.0;
        for (int t = 0; t < L; ++t) acc += s[t] * V[(int64_t)t * D + d];
        o[d] = acc / l;
    }
    free(s);
}

void oracle_decode_attention_fp8(const float* q, const uint8_t* k8, const uint8_t* v8,
                                 int B, int H_q, int H_kv, int S_max, int D,
                                 const int32_t* seq_lens, double softmax_scale,
                                 double* out) {
    double scale = softmax_scale != 0.0 ? softmax_scale : 1.0 / sqrt((double)D);
    int g = H_q / H_kv;
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int b = 0; b < B; ++b) {
        for (int hk = 0; hk < H_kv; ++hk) {
            int L = seq_lens[b];
            int64_t slot0 = ((int64_t)b * H_kv + hk) * S_max;
            double* K = (double*)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1) * D);
            double* V = (double*)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1) * D);
            for (int t = 0; t < L; ++t)
                for (int d = 0; d < D; ++d) {
                    K[(int64_t)t * D + d] = oracle_e4m3_value(k8[(slot0 + t) * D + d]);
                    V[(int64_t)t * D + d] = oracle_e4m3_value(v8[(slot0 + t) * D + d]);
                }
            for (int j = 0; j < g; ++j) {
                int h = hk * g + j;
                attend_one(q + ((int64_t)b * H_q + h) * D, K, V, L, D, scale,
                           out + ((int64_t)b * H_q + h) * D);
            }
            free(K);
            free(V);
        }
    }
}

void oracle_decode_attention_nvfp4(const float* q,
                                   const uint8_t* k_codes, const uint8_t* k_scales,
                                   const uint8_t* v_codes, const uint8_t* v_scales,
                                   float s_tensor_k, float s_tensor_v,
                                   int B, int H_q, int H_kv, int S_max, int D,
                                   const int32_t* seq_lens, double softmax_scale,
                                   double* out) {
    double scale = softmax_scale != 0.0 ? softmax_scale : 1.0 / sqrt((double)D);
    int g = H_q / H_kv;
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int b = 0; b < B; ++b) {
        for (int hk = 0; hk < H_kv; ++hk) {
            int L = seq_lens[b];
            int64_t slot0 = ((int64_t)b * H_kv + hk) * S_max;
            double* K = (double*)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1) * D);
            double* V = (double*)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1) * D);
            for (int t = 0; t < L; ++t) {
                int64_t slot = slot0 + t;
                for (int d = 0; d < D; ++d) {
                    uint8_t kb = k_codes[slot * (D / 2) + d / 2];
                    uint8_t vb = v_codes[slot * (D / 2) + d / 2];
                    uint8_t kc = (d % 2 == 0) ? (kb & 0xF) : (kb >> 4);
                    uint8_t vc = (d % 2 == 0) ? (vb & 0xF) : (vb >> 4);
                    uint8_t ks = k_scales[slot * (D / 16) + d / 16];
                    uint8_t vs = v_scales[slot * (D / 16) + d / 16];
                    K[(int64_t)t * D + d] = oracle_e4m3_value(oracle_dequant_fp8(kc, ks, s_tensor_k));
                    V[(int64_t)t * D + d] = oracle_e4m3_value(oracle_dequant_fp8(vc, vs, s_tensor_v));
                }
            }
            for (int j = 0; j < g; ++j) {
                int h = hk * g + j;
                attend_one(q + ((int64_t)b * H_q + h) * D, K, V, L, D, scale,
                           out + ((int64_t)b * H_q + h) * D);
            }
            free(K);
            free(V);
        }
    }
}

/* --------------------------------------------------------------------------
 * Chunked prefill over the cache.  [P1] and [P3] "推論速度" credit the NVFP4
 * cache with a faster time to first token, which is the prefill side: the
 * prompt is processed in chunks whose K/V are appended first, then each
 * query of the chunk attends to the cache.  Reading R17: query i of sequence
 * b sits at position start[b] + i and sees cache tokens t <= start[b] + i
 * (causal), over the same FP8 values as decode attention (R7, R8); so each
 * query is decode attention with its own length start[b] + i + 1.
 * ------------------------------------------------------------------------ */
void oracle_prefill_attention_nvfp4(const float* q,
                                    const uint8_t* k_codes, const uint8_t* k_scales,
                                    const uint8_t* v_codes, const uint8_t* v_scales,
                                    float s_tensor_k, float s_tensor_v,
                                    int B, int C, int H_q, int H_kv, int S_max, int D,
                                    const int32_t* start, double softmax_scale, double* out) {
    double scale = softmax_scale != 0.0 ? softmax_scale : 1.0 / sqrt((double)D);
    int g = H_q / H_kv;
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int b = 0; b < B; ++b) {
        for (int hk = 0; hk < H_kv; ++hk) {
            int L = start[b] + C;                     /* tokens any query of the chunk sees */
            int64_t slot0 = ((int64_t)b * H_kv + hk) * S_max;
            double* K = (double*)malloc(sizeof(double) * (size_t)L * D);
            double* V = (double*)malloc(sizeof(double) * (size_t)L * D);
            for (int t = 0; t < L; ++t) {
                int64_t slot = slot0 + t;
                for (int d = 0; d < D; ++d) {
                    uint8_t kb = k_codes[slot * (D / 2) + d / 2];
                    uint8_t vb = v_codes[slot * (D / 2) + d / 2];
                    uint8_t kc = (d % 2 == 0) ? (kb & 0xF) : (kb >> 4);
                    uint8_t vc = (d % 2 == 0) ? (vb & 0xF) : (vb >> 4);
                    uint8_t ks = k_scales[slot * (D / 16) + d / 16];
                    uint8_t vs = v_scales[slot * (D / 16) + d / 16];
                    K[(int64_t)t * D + d] = oracle_e4m3_value(oracle_dequant_fp8(kc, ks, s_tensor_k));
                    V[(int64_t)t * D + d] = oracle_e4m3_value(oracle_dequant_fp8(vc, vs, s_tensor_v));
                }
            }
            for (int i = 0; i < C; ++i)
                for (int j = 0; j < g; ++j) {
                    int h = hk * g + j;
                    int64_t row = (((int64_t)b * C + i) * H_q + h) * D;
                    attend_one(q + row, K, V, start[b] + i + 1, D, scale, out + row);
                }
            free(K);
            free(V);
        }
    }
}

/* --------------------------------------------------------------------------
 * Memory model.  [P3] "KV Cacheのメモリボトルネック": KV_mem = 2 * L * n_h *
 * d_h * s * b * sizeof(dtype).  For NVFP4 the per-element size is 4 code bits
 * plus one 8-bit scale shared by 16 elements ("E2M1 + 2レベルスケーリング");
 * the single fp32 tensor scale is negligible and left out.
 * ------------------------------------------------------------------------ */
double oracle_nvfp4_bits_per_element(void) { return 4.0 + 8.0 / 16.0; }

/* MXFP4 ([P3] "MXFP4との比較"): 4 code bits plus one 8-bit E8M0 scale per 32. */
double oracle_mxfp4_bits_per_element(void) { return 4.0 + 8.0 / 32.0; }

double oracle_kv_bytes(int64_t layers, int64_t n_h, int64_t d_h, int64_t s, int64_t b,
                       double bits_per_element) {
    return 2.0 * (double)layers * (double)n_h * (double)d_h * (double)s * (double)b *
           (bits_per_element / 8.0);
}

void oracle_set_threads(int n) {
#ifdef _OPENMP
    omp_set_num_threads(n > 0 ? n : 1);
#else
    (void)n;
#endif
}

int oracle_get_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

// nvfp4kv_prefill_attention_tc.cu -- chunked-prefill attention over the NVFP4
// KV cache on the sm_100a tensor cores (tcgen05).
//
// "NVIDIA解説: NVFP4 KV Cacheで長コンテキストLLM推論を最適化", "推論速度": the
// NVFP4 cache shortens time to first token, which is the prefill side; and
// "量子化・逆量子化フロー": the cache is dequantized to FP8 at attention time.
// A prompt is processed in chunks of C tokens whose K/V are appended first;
// query i of sequence b sits at position start[b] + i and attends to the cache
// tokens t <= start[b] + i, over the same FP8 values as decode attention.
//
// Unlike decode, a chunk gives the MMAs real width: a CTA takes 128 rows =
// (query, head) pairs of one (sequence, KV head) -- floor(128 / g) queries x
// the GQA group g -- and walks the cache in tiles of 128 tokens:
//     S = Q . K^T     M = 128 rows, N = 128 tokens, K = 128 head_dim
//     O += P . V      M = 128 rows, N = 128 head_dim, K = 128 tokens
// both as kind::f16 MMAs with fp32 accumulators in tensor memory.  Every
// E4M3 value is exact in f16, so K and V are the cache's FP8 values (LUT
// dequant, then an exact E4M3 -> f16 conversion).  q (bf16) is scaled per row
// by a power of two, which leaves it exact in f16; P is
// split into two f16 terms, P_hi = f16(p) and P_lo = f16(p - P_hi) (about
// 22 significant bits), each with its own P.V into O.
//
// Warp roles (one CTA per SM: 209 KB of shared memory):
//   warps 0-3  softmax: thread r owns row r (tensor-memory lane r) -- the
//              query operand in the prologue, the online softmax, the output
//   warps 4-7  dequant: thread t owns token t of the tile -- K -> f16 rows,
//              V -> f16 (MN-major)
//   warp 8     bulk copies of the raw codes and scales into a 2-stage ring
//   warp 9     MMA issue (one elected lane): S(k + 1) = Q.K^T is issued
//              before O += P(k).V(k), so the next scores are ready when the
//              softmax finishes a tile
// S is double-buffered in tensor memory (2 x 128 columns) next to O (128).
// Every thread that writes an MMA operand (Q, K, V, P), reads S or reads a
// ring stage fences and arrives on the barrier itself (arrival counts of 128):
// the tiles are consumed (or refilled) right after they are produced (or
// read), and per-warp arrivals after __syncwarp let the tensor core and the
// bulk copies race with other lanes' accesses in testing.
#include <cuda_bf16.h>

#include "nvfp4kv_device.cuh"
#include "nvfp4kv_internal.h"
#include "nvfp4kv_pipeline.cuh"
#include "nvfp4kv_tcgen05.cuh"

namespace nvfp4kv {

namespace {

constexpr int PT = 128;                               // tokens per tile, rows per CTA
constexpr int PD = 128;                               // head_dim
constexpr int kKB = PD / 2, kSB = PD / 16;            // code / scale bytes per token
constexpr int PSTAGE = PT * (2 * kKB + 2 * kSB);      // 18432
constexpr int P_OFF_VC = PT * kKB;
constexpr int P_OFF_KS = 2 * PT * kKB;
constexpr int P_OFF_VS = 2 * PT * kKB + PT * kSB;
constexpr int kPThreads = 10 * 32;
constexpr int kDqWarp0 = 4, kLdWarp = 8, kMmaWarp = 9;
constexpr int kPLutCopies = 4;
constexpr uint32_t COL_S = 0, COL_O = 2 * PT, kPTmemCols = 512;
// O is rescaled only when a row's running max grows by more than this (base-2
// units), so P = 2^(s - m) <= 2^8 stays well inside f16
constexpr float kPSlack = 8.0f;

struct PrefillParams {
    const void* q;                                    // [B][C][H_q][128], bf16 or fp32
    bool q_f32;
    const uint8_t *kc, *ks, *vc, *vs;                 // contiguous planes [B][H_kv][S_max][...]
    const float *st_k, *st_v;
    const int32_t* start;                             // [B]
    float* out;                                       // [B][C][H_q][128]
    int32_t* status;
    int B, C, Hq, Hkv, g, S_max, cq, nqb;             // cq queries per CTA, nqb CTAs per (b, KV head)
    float softmax_scale;
    uint32_t wait_polls;
};

// Canonical non-swizzled layouts (byte offsets, 2-byte elements), 8-row x
// 16-byte core matrices: K-major rows r with K index k: (r/8)*2048 +
// (k/8)*128 + (r%8)*16 + (k%8)*2; MN-major: (mn/8)*2048 + (k/8)*128 +
// (k%8)*16 + (mn%8)*2.  LBO = 128 (along K), SBO = 2048.
struct __align__(1024) PSmem {
    uint8_t ring[2][PSTAGE];
    uint8_t q[PT * PD * 2];                           // A of Q.K^T, K-major (row, d)
    uint8_t k[PT * PD * 2];                           // B of Q.K^T, K-major (token, d)
    uint8_t v[PT * PD * 2];                           // B of P.V,   MN-major (d, token)
    uint8_t p[2][PT * PT * 2];                        // A of P.V,   K-major (row, token): P_hi, P_lo
    uint2 lut[2][128][kPLutCopies];
    uint64_t full[2], empty[2];
    uint64_t kready, vready, pvdone, sready[2], sfree[2], pready, qready, mma_done;
    float cscale[PT];
    uint32_t tmem_base;
    int32_t abort_flag;
};

__device__ __forceinline__ uint32_t pack_f16x2_rn(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// 8 codes -> 8 f16 values (16 bytes), through the FP8 lookup words
__device__ __forceinline__ uint4 dequant8_f16(uint32_t x, uint2 l) {
    uint32_t lo, hi;
    dequant_word(x, l.x, l.y, lo, hi);                // E4M3 bytes of elements 0-3, 4-7
    uint4 o;
    e4m3x4_to_f16x2x2(lo, o.x, o.y);
    e4m3x4_to_f16x2x2(hi, o.z, o.w);
    return o;
}

// Eight kind::f16 MMAs (K = 16 each, descriptors advancing 256 bytes per
// step) into one accumulator, in one instruction sequence; the first
// accumulates only when `acc` is non-zero.
__device__ __forceinline__ void mma8_f16(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p0, p1;\n\t"
        "setp.ne.b32 p0, %3, 0;\n\t"
        "setp.eq.b32 p1, %3, %3;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %4, p0;\n\t"
        "add.s64 %1, %1, 16;\n\tadd.s64 %2, %2, 16;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %4, p1;\n\t"
        "add.s64 %1, %1, 16;\n\tadd.s64 %2, %2, 16;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %4, p1;\n\t"
        "add.s64 %1, %1, 16;\n\tadd.s64 %2, %2, 16;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %4, p1;\n\t"
        "add.s64 %1, %1, 16;\n\tadd.s64 %2, %2, 16;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %4, p1;\n\t"
        "add.s64 %1, %1, 16;\n\tadd.s64 %2, %2, 16;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %4, p1;\n\t"
        "add.s64 %1, %1, 16;\n\tadd.s64 %2, %2, 16;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %4, p1;\n\t"
        "add.s64 %1, %1, 16;\n\tadd.s64 %2, %2, 16;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %4, p1;\n\t}"
        : "+r"(d), "+l"(a), "+l"(b)
        : "r"(acc), "r"(idesc)
        : "memory");
}

__global__ void __launch_bounds__(kPThreads, 1) prefill_attention_tc_kernel(const PrefillParams p) {
    extern __shared__ uint8_t smem_raw[];
    PSmem& sm = *reinterpret_cast<PSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    // ---- the unit: (sequence b, KV head hk, query block qb) ----
    const int qb = (int)(blockIdx.x % (unsigned)p.nqb);
    const int bh = (int)(blockIdx.x / (unsigned)p.nqb);
    const int hk = bh % p.Hkv, b = bh / p.Hkv;
    const int start = p.start[b];
    if (start < 0 || (int64_t)start + p.C > p.S_max) {
        if (tid == 0 && qb == 0 && hk == 0) report(p.status, NVFP4_ERR_CAPACITY);
        return;
    }
    const int i0 = qb * p.cq;
    const int nq = min(p.cq, p.C - i0);                // queries of this CTA
    const int rows = nq * p.g;
    const int T_end = start + i0 + nq;                 // tokens the last query sees
    const int ntiles = (T_end + PT - 1) / PT;
    const float st_k = *p.st_k, st_v = *p.st_v;
    const uint32_t polls = p.wait_polls;

    // ---- prologue ----
    if (warp == kMmaWarp) {
        tc::tmem_alloc(&sm.tmem_base, kPTmemCols);
        tc::tmem_relinquish();
    }
    if (warp == kLdWarp && lane == 0) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], 128);
        }
        mbar_init(&sm.kready, 128);
        mbar_init(&sm.vready, 128);
        mbar_init(&sm.pvdone, 1);
        mbar_init(&sm.sready[0], 1);
        mbar_init(&sm.sready[1], 1);
        mbar_init(&sm.sfree[0], 128);
        mbar_init(&sm.sfree[1], 128);
        mbar_init(&sm.pready, 128);
        mbar_init(&sm.qready, 128);
        mbar_init(&sm.mma_done, 1);
        fence_mbar_init();
        sm.abort_flag = 0;
    }
    // lookup tables: 2 planes x 128 scale bytes, by the 192 threads from warp 4 on
    for (int e = tid - kDqWarp0 * 32; e >= 0 && e < 256; e += kPThreads - kDqWarp0 * 32) {
        const int plane = e >> 7;
        const uint2 w = lut_words((uint32_t)(e & 127), plane ? st_v : st_k);
#pragma unroll
        for (int c = 0; c < kPLutCopies; ++c) sm.lut[plane][e & 127][c] = w;
    }
    if (tid == 0 && blockIdx.x == 0) {
        const bool ok = st_k > 0.f && st_k <= 3.4028234663852886e38f && st_v > 0.f &&
                        st_v <= 3.4028234663852886e38f;
        if (!ok) report(p.status, NVFP4_ERR_NONFINITE);
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tbase = sm.tmem_base;
    int32_t* const abort_flag = &sm.abort_flag;
    const int64_t slot0 = ((int64_t)b * p.Hkv + hk) * p.S_max;

    if (warp == kLdWarp) {
        // ================= bulk copies of tile k into stage k % 2 =================
        if (lane == 0) {
            int k = 0;
            for (; k < ntiles; ++k) {
                const int s = k & 1;
                if (k >= 2 && !wait_one(&sm.empty[s], ((k >> 1) - 1) & 1, abort_flag, p.status, polls)) break;
                const int t0 = k * PT;
                const int n = min(PT, T_end - t0);
                const int ncopy = (n + 3) & ~3;        // every copy a multiple of 16 bytes
                const uint32_t cb = (uint32_t)ncopy * kKB, sb = (uint32_t)ncopy * kSB;
                mbar_arrive_expect_tx(&sm.full[s], 2 * (cb + sb));
                const int64_t tok = slot0 + t0;
                uint8_t* st = sm.ring[s];
                bulk_g2s(st, p.kc + tok * kKB, cb, &sm.full[s]);
                bulk_g2s(st + P_OFF_VC, p.vc + tok * kKB, cb, &sm.full[s]);
                bulk_g2s(st + P_OFF_KS, p.ks + tok * kSB, sb, &sm.full[s]);
                bulk_g2s(st + P_OFF_VS, p.vs + tok * kSB, sb, &sm.full[s]);
            }
            // every issued copy lands before the CTA exits
            for (int i = k > 2 ? k - 2 : 0; i < k; ++i)
                if (!mbar_wait_sleep(&sm.full[i & 1], (i >> 1) & 1, 1u << 16)) {
                    report(p.status, NVFP4_ERR_TIMEOUT);
                    break;
                }
        }
    } else if (warp == kMmaWarp) {
        // ================= MMA issue =================
        const uint32_t idesc_qk = tc::idesc_e4m3(128, 128, false, false, false);   // f16 x f16 -> f32
        const uint32_t idesc_pv = tc::idesc_e4m3(128, 128, false, true, false);    // B = V MN-major
        const uint64_t dq = tc::smem_desc(tc::smem_addr(sm.q), 128, 2048);
        const uint64_t dk = tc::smem_desc(tc::smem_addr(sm.k), 128, 2048);
        const uint64_t dv = tc::smem_desc(tc::smem_addr(sm.v), 128, 2048);
        const uint64_t dp = tc::smem_desc(tc::smem_addr(sm.p[0]), 128, 2048);
        const uint64_t dp2 = tc::smem_desc(tc::smem_addr(sm.p[1]), 128, 2048);
        bool ok = wait_warp(&sm.qready, 0, abort_flag, p.status, polls);
        // S(k) = Q . K(k)^T into S buffer k % 2; one commit, to sready[k % 2]
        // (its completion also frees the K buffer: the dequant warps wait on it)
        auto issue_qk = [&](int k) -> bool {
            if (!wait_warp(&sm.kready, k & 1, abort_flag, p.status, polls)) return false;
            if (k >= 2 && !wait_warp(&sm.sfree[k & 1], ((k >> 1) - 1) & 1, abort_flag, p.status, polls))
                return false;
            tc::fence_after_sync();
            if (tc::elect_one()) {
                mma8_f16(tbase + COL_S + PT * (k & 1), dq, dk, idesc_qk, 0u);
                tc::mma_commit(&sm.sready[k & 1]);
            }
            __syncwarp();
            return true;
        };
        if (ok) ok = issue_qk(0);
        for (int k = 0; ok && k < ntiles; ++k) {
            if (k + 1 < ntiles && !issue_qk(k + 1)) break;
            // O += P(k) . V(k); commit: pvdone
            if (!wait_warp(&sm.pready, k & 1, abort_flag, p.status, polls)) break;
            if (!wait_warp(&sm.vready, k & 1, abort_flag, p.status, polls)) break;
            tc::fence_after_sync();
            if (tc::elect_one()) {
                mma8_f16(tbase + COL_O, dp, dv, idesc_pv, k > 0 ? 1u : 0u);
                mma8_f16(tbase + COL_O, dp2, dv, idesc_pv, 1u);
                tc::mma_commit(&sm.pvdone);
            }
            __syncwarp();
        }
        // every issued MMA completes before tensor memory is released (one
        // commit per barrier: a second commit of the same MMAs is not relied on)
        if (tc::elect_one()) tc::mma_commit(&sm.mma_done);
        __syncwarp();
    } else if (warp >= kDqWarp0 && warp < kDqWarp0 + 4) {
        // ================= dequant: token t of each tile =================
        const int t = tid - kDqWarp0 * 32;
        const uint2* lut_k = &sm.lut[0][0][lane & (kPLutCopies - 1)];
        const uint2* lut_v = &sm.lut[1][0][lane & (kPLutCopies - 1)];
        for (int k = 0; k < ntiles; ++k) {
            const int s = k & 1;
            if (!wait_warp(&sm.full[s], (k >> 1) & 1, abort_flag, p.status, polls)) break;
            const uint8_t* st = sm.ring[s];
            uint4 kc[4], vc[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                kc[j] = *reinterpret_cast<const uint4*>(st + t * kKB + 16 * j);
                vc[j] = *reinterpret_cast<const uint4*>(st + P_OFF_VC + t * kKB + 16 * j);
            }
            const uint2 ksb = *reinterpret_cast<const uint2*>(st + P_OFF_KS + t * kSB);
            const uint2 vsb = *reinterpret_cast<const uint2*>(st + P_OFF_VS + t * kSB);
            // the next bulk copy into this stage (async proxy) comes after these reads
            fence_proxy_async_smem();
            mbar_arrive(&sm.empty[s]);
            // Q.K^T of tile k - 1 has read the K buffer (its commit to sready)
            if (k >= 1 && !wait_warp(&sm.sready[(k - 1) & 1], ((k - 1) >> 1) & 1, abort_flag, p.status, polls))
                break;
            uint8_t* kd = sm.k + (t / 8) * 2048 + (t % 8) * 16;
#pragma unroll
            for (int j = 0; j < 4; ++j) {              // codes 32j .. 32j + 31 = two blocks
                const uint32_t sc = j < 2 ? ksb.x : ksb.y;
                const uint2 la = lut_k[((sc >> (16 * (j & 1))) & 0x7F) * kPLutCopies];
                const uint2 lb = lut_k[((sc >> (16 * (j & 1) + 8)) & 0x7F) * kPLutCopies];
                const uint32_t w[4] = {kc[j].x, kc[j].y, kc[j].z, kc[j].w};
#pragma unroll
                for (int c = 0; c < 4; ++c)              // 8 head_dim values each
                    *reinterpret_cast<uint4*>(kd + (4 * j + c) * 128) = dequant8_f16(w[c], c < 2 ? la : lb);
            }
            fence_proxy_async_smem();
            mbar_arrive(&sm.kready);
            // P.V of tile k - 1 has read the V buffer
            if (k >= 1 && !wait_warp(&sm.pvdone, (k - 1) & 1, abort_flag, p.status, polls)) break;
            uint8_t* vd = sm.v + (t / 8) * 128 + (t % 8) * 16;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint32_t sc = j < 2 ? vsb.x : vsb.y;
                const uint2 la = lut_v[((sc >> (16 * (j & 1))) & 0x7F) * kPLutCopies];
                const uint2 lb = lut_v[((sc >> (16 * (j & 1) + 8)) & 0x7F) * kPLutCopies];
                const uint32_t w[4] = {vc[j].x, vc[j].y, vc[j].z, vc[j].w};
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    *reinterpret_cast<uint4*>(vd + (4 * j + c) * 2048) = dequant8_f16(w[c], c < 2 ? la : lb);
            }
            fence_proxy_async_smem();
            mbar_arrive(&sm.vready);
        }
    } else {
        // ================= softmax: row r = (query i0 + r / g, head hk * g + r % g) =================
        const int r = tid;
        const uint32_t trow = tbase + ((uint32_t)(32 * warp) << 16);
        const bool live = r < rows;
        const int qi = i0 + r / p.g;                   // query index in the chunk
        const int lim = live ? start + qi + 1 : 0;     // tokens this row sees
        // query operand: q * 2^e rounded to f16, e from the row's amax (two
        // passes over the row, so that it never sits in registers whole)
        {
            const int64_t row = (((int64_t)b * p.C + (live ? qi : 0)) * p.Hq + (int64_t)hk * p.g + r % p.g) * PD;
            auto load8 = [&](int c, float (&x)[8]) {       // head_dim 8c .. 8c + 7
                if (!live) {
#pragma unroll
                    for (int j = 0; j < 8; ++j) x[j] = 0.0f;
                } else if (p.q_f32) {
                    const float4* src = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(p.q) + row) + 2 * c;
                    const float4 f0 = src[0], f1 = src[1];
                    x[0] = f0.x; x[1] = f0.y; x[2] = f0.z; x[3] = f0.w;
                    x[4] = f1.x; x[5] = f1.y; x[6] = f1.z; x[7] = f1.w;
                } else {
                    const uint4 u = reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(p.q) + row)[c];
                    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        x[2 * j] = __uint_as_float(w[j] << 16);
                        x[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
                    }
                }
            };
            float amax = 0.0f;
            for (int c = 0; c < PD / 8; ++c) {
                float x[8];
                load8(c, x);
#pragma unroll
                for (int j = 0; j < 8; ++j) amax = fmaxf(amax, fabsf(x[j]));
            }
            int e = 0;
            if (amax > 0.0f && amax <= 3.4028234663852886e38f) {
                int ex;
                frexpf(amax, &ex);                     // amax < 2^ex
                e = 15 - ex;                           // max |q * 2^e| < 2^15
                e = e < -126 ? -126 : (e > 126 ? 126 : e);
            }
            const float up = __uint_as_float((uint32_t)(127 + e) << 23);
            uint8_t* qd = sm.q + (r / 8) * 2048 + (r % 8) * 16;
            for (int c = 0; c < PD / 8; ++c) {
                float x[8];
                load8(c, x);
                uint4 o;
                o.x = pack_f16x2_rn(x[0] * up, x[1] * up);
                o.y = pack_f16x2_rn(x[2] * up, x[3] * up);
                o.z = pack_f16x2_rn(x[4] * up, x[5] * up);
                o.w = pack_f16x2_rn(x[6] * up, x[7] * up);
                *reinterpret_cast<uint4*>(qd + c * 128) = o;
            }
            const float scale = p.softmax_scale > 0.0f ? p.softmax_scale : rsqrtf((float)PD);
            sm.cscale[r] = scale * 1.4426950408889634f * __uint_as_float((uint32_t)(127 - e) << 23);
        }
        fence_proxy_async_smem();
        mbar_arrive(&sm.qready);
        const float cs = sm.cscale[r];
        float m_run = -INFINITY, l_run = 0.0f;
        bool ok = true;
        for (int k = 0; ok && k < ntiles; ++k) {
            const int sb = k & 1;
            if (!wait_warp(&sm.sready[sb], (k >> 1) & 1, abort_flag, p.status, polls)) {
                ok = false;
                break;
            }
            tc::fence_after_sync();
            const int t0 = k * PT;
            const uint32_t scol = trow + COL_S + PT * sb;
            // pass 1: the row's max over the tile's visible tokens
            float mt = -INFINITY;
#pragma unroll 1
            for (int c = 0; c < PT / 32; ++c) {
                uint32_t v[32];
                tc::tmem_ld_x16(scol + 32 * c, v);
                tc::tmem_ld_x16(scol + 32 * c + 16, v + 16);
                tc::tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    if (t0 + 32 * c + j < lim) mt = fmaxf(mt, __uint_as_float(v[j]) * cs);
            }
            float m_use = m_run;
            if (mt > m_run + kPSlack || m_run == -INFINITY) m_use = fmaxf(m_run, mt);
            // P and O: P.V of tile k - 1 is done with the P buffer and with O
            if (k >= 1 && !wait_warp(&sm.pvdone, (k - 1) & 1, abort_flag, p.status, polls)) {
                ok = false;
                break;
            }
            tc::fence_after_sync();
            float f = 1.0f;                            // this row's O and l factor
            if (m_use != m_run) {
                f = m_run == -INFINITY ? 0.0f : fast_exp2(m_run - m_use);
                l_run *= f;
                m_run = m_use;
            }
            // tcgen05.ld/st are warp-wide (.sync.aligned): the whole warp rescales
            // when any of its rows must, the others by 1
            if (k >= 1 && __any_sync(0xFFFFFFFFu, f != 1.0f)) {
#pragma unroll 1
                for (int c = 0; c < PD / 32; ++c) {
                    uint32_t o[32];
                    tc::tmem_ld_x16(trow + COL_O + 32 * c, o);
                    tc::tmem_ld_x16(trow + COL_O + 32 * c + 16, o + 16);
                    tc::tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * f);
                    tc::tmem_st_x32(trow + COL_O + 32 * c, o);
                }
                tc::tmem_wait_st();
            }
            // pass 2: P = 2^(s - m) as two f16 terms (P_hi + P_lo, ~22 bits), l over the row
            uint8_t* pd = sm.p[0] + (r / 8) * 2048 + (r % 8) * 16;
            uint8_t* pd2 = sm.p[1] + (r / 8) * 2048 + (r % 8) * 16;
#pragma unroll 1
            for (int c = 0; c < PT / 32; ++c) {
                uint32_t v[32];
                tc::tmem_ld_x16(scol + 32 * c, v);
                tc::tmem_ld_x16(scol + 32 * c + 16, v + 16);
                tc::tmem_wait_ld();
                float pv[32];
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const bool vis = t0 + 32 * c + j < lim && m_run != -INFINITY;
                    pv[j] = vis ? fast_exp2(__uint_as_float(v[j]) * cs - m_run) : 0.0f;
                    l_run += pv[j];
                }
#pragma unroll
                for (int j = 0; j < 4; ++j) {          // 8 tokens per 16-byte chunk
                    uint32_t hi[4], lo[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float a = pv[8 * j + 2 * e], b2 = pv[8 * j + 2 * e + 1];
                        hi[e] = pack_f16x2_rn(a, b2);
                        lo[e] = pack_f16x2_rn(a - f16_lo_to_float(hi[e]), b2 - f16_hi_to_float(hi[e]));
                    }
                    *reinterpret_cast<uint4*>(pd + (4 * c + j) * 128) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
                    *reinterpret_cast<uint4*>(pd2 + (4 * c + j) * 128) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
                }
            }
            tc::fence_before_sync();
            mbar_arrive(&sm.sfree[sb]);
            fence_proxy_async_smem();
            mbar_arrive(&sm.pready);
        }
        // ---- output: O / l ----
        if (ok && wait_warp(&sm.pvdone, (ntiles - 1) & 1, abort_flag, p.status, polls)) {
            tc::fence_after_sync();
            const float inv = l_run > 0.0f ? 1.0f / l_run : 0.0f;
            float* dst = p.out + (((int64_t)b * p.C + qi) * p.Hq + (int64_t)hk * p.g + r % p.g) * PD;
#pragma unroll 1
            for (int c = 0; c < PD / 32; ++c) {
                uint32_t o[32];
                tc::tmem_ld_x16(trow + COL_O + 32 * c, o);
                tc::tmem_ld_x16(trow + COL_O + 32 * c + 16, o + 16);
                tc::tmem_wait_ld();
                if (live) {
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        reinterpret_cast<float4*>(dst + 32 * c)[j] =
                            make_float4(__uint_as_float(o[4 * j]) * inv, __uint_as_float(o[4 * j + 1]) * inv,
                                        __uint_as_float(o[4 * j + 2]) * inv, __uint_as_float(o[4 * j + 3]) * inv);
                }
            }
        }
    }

    // ---- release tensor memory once every MMA has completed ----
    if (warp == kMmaWarp) {
        if (!mbar_wait_sleep(&sm.mma_done, 0, 1u << 16)) report(p.status, NVFP4_ERR_TIMEOUT);
        __syncwarp();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (warp == kMmaWarp) tc::tmem_dealloc(tbase, kPTmemCols);
}

}  // namespace

cudaError_t launch_prefill_tc(const void* q, bool q_f32, int C, int H_q, const nvfp4_kv_plane& k,
                              const nvfp4_kv_plane& v, const float* d_st_k, const float* d_st_v,
                              const int32_t* d_start, float softmax_scale, float* out, int32_t* d_status,
                              uint32_t wait_polls, cudaStream_t stream) {
    PrefillParams p;
    p.q = q;
    p.q_f32 = q_f32;
    p.kc = k.codes; p.ks = k.scales; p.vc = v.codes; p.vs = v.scales;
    p.st_k = d_st_k; p.st_v = d_st_v;
    p.start = d_start;
    p.out = out;
    p.status = d_status;
    p.B = k.B; p.C = C; p.Hq = H_q; p.Hkv = k.H_kv; p.g = H_q / k.H_kv; p.S_max = k.S_max;
    p.cq = PT / p.g;
    p.nqb = (C + p.cq - 1) / p.cq;
    p.softmax_scale = softmax_scale;
    p.wait_polls = wait_polls;
    const int64_t grid = (int64_t)p.B * p.Hkv * p.nqb;
    if (grid == 0) return cudaSuccess;
    const int smem = (int)sizeof(PSmem) + 1024;
    static int configured[kMaxDevices] = {};          // the attribute is set once per device
    cudaError_t e =
        ensure_smem_attribute(reinterpret_cast<const void*>(prefill_attention_tc_kernel), smem, configured);
    if (e != cudaSuccess) return e;
    prefill_attention_tc_kernel<<<(unsigned)grid, kPThreads, smem, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace nvfp4kv

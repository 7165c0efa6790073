// nvfp4kv_decode_attention.cu -- fused NVFP4 -> FP8 decode attention.
//
// What it computes ("NVIDIA解説: NVFP4 KV Cacheで長コンテキストLLM推論を最適化",
// "量子化・逆量子化フロー"; "TensorRT-LLM rc17 ...", "物語の KV キャッシュ側";
// "Compilation d'inferences ... NVFP4 sur Blackwell", "Le type de Blackwell"):
// the NVFP4 cache is dequantized to FP8 and FP8 attention runs with an FP32
// accumulator:  out[b][h] = softmax(q . K^T * scale) . V  over seq_lens[b]
// tokens of KV head h / g.  The speed-up the pages describe comes from the
// smaller memory traffic, so the kernel is built around streaming the 4.5-bit
// cache from HBM once:
//
//  * Split-K across the whole GPU (stream-K style): the (sequence, KV head,
//    32-token tile) list is cut into gridDim.x equal contiguous ranges, one
//    per CTA (gridDim.x = 2 x SM count), so every SM gets the same number of
//    tiles whatever the mix of lengths.  A CTA range crosses (sequence, head)
//    units; a unit shared by several CTAs is merged by the last CTA to finish
//    with it (arrival counter), never by waiting.
//  * Each of the 4 warps of a CTA streams its own tiles through a private
//    4-stage ring in shared memory, filled by 1-D bulk async copies (codes and
//    scale bytes are contiguous per (sequence, head)) that complete on an
//    mbarrier.  Every wait is bounded.
//  * Dequantization happens in registers: per 16-element block, two lookup
//    words (the FP8 bytes of the 8 code magnitudes for that scale byte) from a
//    per-CTA table, four byte permutes per 8 codes, then an exact E4M3 -> f16
//    convert.  The FP8 values are therefore exactly those of
//    nvfp4_kv_dequant_fp8.
//  * Q.K^T and P.V run on tensor cores (mma.sync m16n8k16, f16 inputs, f32
//    accumulate) with tokens on M for Q.K^T and head_dim on M for P.V, so a
//    GQA group of up to 8 (16) query heads is one (two) 8-wide N tiles.
//    f16 holds every E4M3 value and every bf16 query (after a power-of-two
//    rescale per head) exactly; P is split into an f16 high and low part so
//    the weights keep ~22 bits.  The C fragment of the score MMA is turned
//    into the B fragment of the P.V MMA with movmatrix (8x8 transpose).
//  * Online softmax in base 2 with a lazily updated running max (rescale only
//    when a score passes the max by more than 2^8), so the common tile does
//    no accumulator rescaling.
#include <cuda_bf16.h>

#include "nvfp4kv_device.cuh"
#include "nvfp4kv_internal.h"

namespace nvfp4kv {

namespace {

constexpr int kWarps = 4;
// ring depth per warp: 4 stages, 3 when the GQA group needs two 8-wide tiles
// (keeps two CTAs resident per SM)
template <int NT>
struct Ring { static constexpr int kStages = NT == 1 ? 4 : 3; };
constexpr uint32_t kWaitLimit = 1u << 22;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleSlack = 8.0f;  // log2 units

template <int D>
struct Geometry {
    static constexpr int KB = D / 2;                 // code bytes per token
    static constexpr int SB = D / 16;                // scale bytes per token
    static constexpr int KS = D / 16;                // k-steps of Q.K^T = m-tiles of P.V
    static constexpr int EK = D / 4;                 // K elements per lane per token
    static constexpr int WK = EK / 8;                // K code words per lane per token
    static constexpr int EV = D / 8;                 // V channels per lane
    static constexpr int WV = EV / 8;                // V code words per lane per token
    static constexpr int STAGE = kTile * (2 * KB + 2 * SB);
    static constexpr int OFF_VC = kTile * KB;
    static constexpr int OFF_KS = 2 * kTile * KB;
    static constexpr int OFF_VS = 2 * kTile * KB + kTile * SB;
    static_assert(STAGE % 16 == 0, "stage must keep 16-byte alignment");
};

template <int D, int NT>
struct __align__(16) Smem {
    static constexpr int kStages = Ring<NT>::kStages;
    uint8_t ring[kWarps][kStages][Geometry<D>::STAGE];
    float merge_o[kWarps][8 * NT][D];
    uint2 lut_k[128];
    uint2 lut_v[128];
    uint64_t bar[kWarps][kStages];
    int32_t lens[kMaxBatchPerLaunch];
    int32_t prefix[kMaxBatchPerLaunch + 1];
    float merge_m[kWarps][8 * NT];
    float merge_l[kWarps][8 * NT];
    int32_t warp_tot[kWarps];
    int32_t last_flag;
};

struct Params {
    const void* q;
    const uint8_t* kc;
    const uint8_t* ks;
    const uint8_t* vc;
    const uint8_t* vs;
    const float* st_k;
    const float* st_v;
    const int32_t* seq_lens;
    float* out;
    float* partials;
    int32_t* counters;
    int32_t* status;
    int B, Hq, Hkv, g, S_max;
    float softmax_scale;
};

// Global tile index -> (sequence, head, first tile of the unit, length).
struct Unit {
    int b, h, L, ntb;
    int64_t U0, U1;  // global tile range of the unit
};

__device__ __forceinline__ Unit find_unit(const int32_t* prefix, const int32_t* lens, int B, int Hkv,
                                          int64_t gt) {
    int lo = 0, hi = B;  // prefix[lo] <= gt < prefix[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (prefix[mid] <= gt) lo = mid; else hi = mid;
    }
    Unit u;
    u.b = lo;
    u.L = lens[lo];
    u.ntb = u.L > 0 ? (u.L + kTile - 1) / kTile : 1;
    const int64_t r = gt - prefix[lo];
    u.h = (int)(r / u.ntb);
    u.U0 = prefix[lo] + (int64_t)u.h * u.ntb;
    u.U1 = u.U0 + u.ntb;
    (void)Hkv;
    return u;
}

// CTA c owns global tiles [range_start(c), range_start(c + 1)).
__device__ __forceinline__ int64_t range_start(int64_t c, int64_t T, int64_t N) {
    return c * T / N;
}

// CTA owning global tile t when T tiles are cut into N equal ranges.
__device__ __forceinline__ int64_t cta_of(int64_t t, int64_t T, int64_t N) {
    return ((t + 1) * N - 1) / T;
}

// Partial-result slot of CTA cc for a unit starting at global tile U0: a CTA
// can share at most two units with other CTAs -- the one holding its first
// tile (slot 2cc) and the one holding its last tile (slot 2cc + 1).
__device__ __forceinline__ int64_t partial_slot(int64_t cc, int64_t U0, int64_t T, int64_t N) {
    return (U0 <= range_start(cc, T, N)) ? 2 * cc : 2 * cc + 1;
}

// Per-warp walk over its tiles: in each segment [seg_lo, seg_hi) of the
// CTA range the warp takes tiles seg_lo + warp, seg_lo + warp + kWarps, ...
struct Cursor {
    int64_t seg_lo, seg_hi, gt, t_end;
    Unit u;
    bool done;
};

__device__ __forceinline__ void cursor_enter(Cursor& c, const int32_t* prefix, const int32_t* lens,
                                             int B, int Hkv, int warp) {
    // find the next segment (from c.seg_lo) holding a tile for this warp
    while (c.seg_lo < c.t_end) {
        c.u = find_unit(prefix, lens, B, Hkv, c.seg_lo);
        c.seg_hi = c.u.U1 < c.t_end ? c.u.U1 : c.t_end;
        c.gt = c.seg_lo + warp;
        if (c.gt < c.seg_hi) return;
        c.seg_lo = c.seg_hi;
    }
    c.done = true;
}

__device__ __forceinline__ void cursor_next(Cursor& c, const int32_t* prefix, const int32_t* lens,
                                            int B, int Hkv, int warp) {
    c.gt += kWarps;
    if (c.gt < c.seg_hi) return;
    c.seg_lo = c.seg_hi;
    cursor_enter(c, prefix, lens, B, Hkv, warp);
}

// Issue the bulk copies of one tile into a ring stage (one lane).
template <int D>
__device__ __forceinline__ void issue_tile(const Params& p, const Unit& u, int64_t gt, uint8_t* stage,
                                           uint64_t* bar) {
    using G = Geometry<D>;
    const int t0 = (int)(gt - u.U0) * kTile;
    int n = u.L - t0;
    n = n < 0 ? 0 : (n > kTile ? kTile : n);
    const int ncopy = (n + 3) & ~3;  // keeps every copy a multiple of 16 bytes
    const uint32_t code_bytes = (uint32_t)ncopy * G::KB;
    const uint32_t scale_bytes = (uint32_t)ncopy * G::SB;
    mbar_arrive_expect_tx(bar, 2 * (code_bytes + scale_bytes));
    if (ncopy > 0) {
        const int64_t tok = ((int64_t)u.b * p.Hkv + u.h) * p.S_max + t0;
        bulk_g2s(stage, p.kc + tok * G::KB, code_bytes, bar);
        bulk_g2s(stage + G::OFF_VC, p.vc + tok * G::KB, code_bytes, bar);
        bulk_g2s(stage + G::OFF_KS, p.ks + tok * G::SB, scale_bytes, bar);
        bulk_g2s(stage + G::OFF_VS, p.vs + tok * G::SB, scale_bytes, bar);
    }
}

__device__ __forceinline__ uint32_t pow2_bits(int e) {  // 2^e as fp32 bits, e in [-126, 127]
    return (uint32_t)(127 + e) << 23;
}

// Load the query fragments of unit (b, h) for this lane.  Lane (gid, tig)
// holds query row j = 8*nt + gid, elements [EK*tig, EK*tig + EK) as f16
// pairs in natural order: qf[s][nt][0] = elements (4s, 4s+1),
// qf[s][nt][1] = (4s+2, 4s+3) -- the same order the K fragments use.
// Each row is scaled by 2^e so that its largest |q| lands below 2^14;
// cscale[nt][c] = softmax_scale * log2(e) * 2^-e of the row in column
// 2*tig + c.
template <int D, int NT, bool QF32>
__device__ __forceinline__ void load_q(const Params& p, int b, int h, int gid, int tig,
                                       uint32_t (&qf)[D / 16][NT][2], uint32_t (&ql)[D / 16][NT][2],
                                       float (&cscale)[NT][2]) {
    using G = Geometry<D>;
    const float base = p.softmax_scale * kLog2e;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const int j = 8 * nt + gid;
        const bool valid = j < p.g;
        float v[G::EK];
        const int64_t row = ((int64_t)b * p.Hq + (int64_t)h * p.g + (valid ? j : 0)) * D + G::EK * tig;
        if (QF32) {
            const float4* src = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(p.q) + row);
#pragma unroll
            for (int i = 0; i < G::EK / 4; ++i) {
                const float4 f = valid ? __ldg(src + i) : make_float4(0.f, 0.f, 0.f, 0.f);
                v[4 * i + 0] = f.x; v[4 * i + 1] = f.y; v[4 * i + 2] = f.z; v[4 * i + 3] = f.w;
            }
        } else {
            const uint4* src = reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(p.q) + row);
#pragma unroll
            for (int i = 0; i < G::EK / 8; ++i) {
                const uint4 w = valid ? __ldg(src + i) : make_uint4(0, 0, 0, 0);
                const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    v[8 * i + 2 * k + 0] = __uint_as_float(ws[k] << 16);
                    v[8 * i + 2 * k + 1] = __uint_as_float(ws[k] & 0xFFFF0000u);
                }
            }
        }
        float amax = 0.0f;
#pragma unroll
        for (int i = 0; i < G::EK; ++i) amax = fmaxf(amax, fabsf(v[i]));
        amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 1));
        amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 2));
        int e = 0;
        if (amax > 0.0f && amax <= 3.4028234663852886e38f) {
            int ex;
            frexpf(amax, &ex);                 // amax < 2^ex
            e = 14 - ex;
            e = e < -126 ? -126 : (e > 126 ? 126 : e);
        }
        const float up = __uint_as_float(pow2_bits(e));
        const float down = __uint_as_float(pow2_bits(-e));
#pragma unroll
        for (int s = 0; s < G::KS; ++s) {
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const float x0 = v[4 * s + 2 * k] * up, x1 = v[4 * s + 2 * k + 1] * up;
                const uint32_t hi = pack_f16x2(x0, x1);
                qf[s][nt][k] = hi;
                if (QF32) ql[s][nt][k] = pack_f16x2(x0 - f16_lo_to_float(hi), x1 - f16_hi_to_float(hi));
            }
        }
        // the score columns of this lane are query rows 2*tig and 2*tig+1 of n-tile nt,
        // whose scale factors live in lanes (gid = 2*tig (+1), tig = 0)
        const float f0 = __shfl_sync(0xFFFFFFFFu, down, (2 * tig) * 4);
        const float f1 = __shfl_sync(0xFFFFFFFFu, down, (2 * tig + 1) * 4);
        cscale[nt][0] = base * f0;
        cscale[nt][1] = base * f1;
    }
}

template <int D, int NT, bool QF32>
__global__ void __launch_bounds__(kWarps * 32, kCtasPerSm) decode_attention_kernel(const Params p) {
    using G = Geometry<D>;
    constexpr int KS = G::KS;
    constexpr int kStages = Ring<NT>::kStages;
    extern __shared__ __align__(128) uint8_t smem_raw[];
    Smem<D, NT>& sm = *reinterpret_cast<Smem<D, NT>*>(smem_raw);

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int gid = lane >> 2;
    const int tig = lane & 3;
    const int B = p.B;

    // ---- prologue: lookup tables, barriers, sequence lengths ----------------
    const float st_k = *p.st_k;
    const float st_v = *p.st_v;
    {
        uint8_t* lk = reinterpret_cast<uint8_t*>(sm.lut_k);
        uint8_t* lv = reinterpret_cast<uint8_t*>(sm.lut_v);
        for (int e = tid; e < 1024; e += kWarps * 32) {
            lk[e] = (uint8_t)lut_entry((uint32_t)(e >> 3), (uint32_t)(e & 7), st_k);
            lv[e] = (uint8_t)lut_entry((uint32_t)(e >> 3), (uint32_t)(e & 7), st_v);
        }
    }
    if (tid == 0 && blockIdx.x == 0) {
        const bool ok = st_k > 0.f && st_k <= 3.4028234663852886e38f && st_v > 0.f &&
                        st_v <= 3.4028234663852886e38f;
        if (!ok) report(p.status, NVFP4_ERR_NONFINITE);
    }
    if (lane == 0) {
#pragma unroll
        for (int s = 0; s < kStages; ++s) mbar_init(&sm.bar[warp][s], 1);
        fence_mbar_init();
    }
    // lengths and the per-sequence tile prefix (units of one sequence are contiguous)
    {
        constexpr int per = (kMaxBatchPerLaunch + kWarps * 32 - 1) / (kWarps * 32);
        int tiles[per];
        int run = 0;
#pragma unroll
        for (int i = 0; i < per; ++i) {
            const int b = tid * per + i;
            int L = 0;
            if (b < B) {
                L = p.seq_lens[b];
                if (L < 0 || L > p.S_max) {
                    if (blockIdx.x == 0) report(p.status, NVFP4_ERR_CAPACITY);
                    L = L < 0 ? 0 : p.S_max;
                }
                sm.lens[b] = L;
            }
            tiles[i] = (b < B) ? p.Hkv * (L > 0 ? (L + kTile - 1) / kTile : 1) : 0;
            run += tiles[i];
        }
        // exclusive scan of `run` over the CTA
        int incl = run;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
            if (lane >= o) incl += y;
        }
        if (lane == 31) sm.warp_tot[warp] = incl;
        __syncthreads();
        int before = 0;
        for (int w = 0; w < warp; ++w) before += sm.warp_tot[w];
        int acc = before + incl - run;
#pragma unroll
        for (int i = 0; i < per; ++i) {
            const int b = tid * per + i;
            if (b < B) sm.prefix[b] = acc;
            acc += tiles[i];
        }
        if (tid == kWarps * 32 - 1) sm.prefix[B] = acc;
    }
    __syncthreads();

    const int64_t T = sm.prefix[B];
    const int64_t N = gridDim.x;
    const int64_t c = blockIdx.x;
    const int64_t t_begin = range_start(c, T, N);
    const int64_t t_end = range_start(c + 1, T, N);
    if (t_begin >= t_end) return;

    // ---- producer: lane 0 of each warp fills the warp's ring ---------------
    Cursor prod;
    prod.seg_lo = t_begin;
    prod.t_end = t_end;
    prod.done = false;
    cursor_enter(prod, sm.prefix, sm.lens, B, p.Hkv, warp);
    uint32_t issued = 0;
    if (lane == 0) {
        for (int s = 0; s < kStages && !prod.done; ++s) {
            issue_tile<D>(p, prod.u, prod.gt, sm.ring[warp][s], &sm.bar[warp][s]);
            ++issued;
            cursor_next(prod, sm.prefix, sm.lens, B, p.Hkv, warp);
        }
    }

    uint32_t consumed = 0;
    bool aborted = false;

    // ---- segments of the CTA range, processed by all warps together --------
    int64_t seg_lo = t_begin;
    while (seg_lo < t_end) {
        const Unit u = find_unit(sm.prefix, sm.lens, B, p.Hkv, seg_lo);
        const int64_t seg_hi = u.U1 < t_end ? u.U1 : t_end;

        uint32_t qf[KS][NT][2], ql[KS][NT][2];
        float cscale[NT][2];
        load_q<D, NT, QF32>(p, u.b, u.h, gid, tig, qf, ql, cscale);

        float o[KS][NT][4];
        float m_run[NT][2], l_run[NT][2];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                m_run[nt][k] = -INFINITY;
                l_run[nt][k] = 0.0f;
            }
#pragma unroll
            for (int i = 0; i < KS; ++i)
#pragma unroll
                for (int k = 0; k < 4; ++k) o[i][nt][k] = 0.0f;
        }

        for (int64_t gt = seg_lo + warp; gt < seg_hi; gt += kWarps) {
            const int stage = (int)(consumed % kStages);
            const uint32_t parity = (consumed / kStages) & 1u;
            {
                // every lane polls; the warp gives up together so that the
                // warp-collective instructions below stay converged
                const bool ok = mbar_wait_bounded(&sm.bar[warp][stage], parity, kWaitLimit);
                if (!__all_sync(0xFFFFFFFFu, ok)) {
                    if (!aborted && lane == 0) report(p.status, NVFP4_ERR_TIMEOUT);
                    aborted = true;
                }
            }
            const int t0 = (int)(gt - u.U0) * kTile;
            int valid = u.L - t0;
            valid = valid > kTile ? kTile : valid;
            const uint8_t* st = sm.ring[warp][stage];
            const uint8_t* kc_s = st;
            const uint8_t* vc_s = st + G::OFF_VC;
            const uint8_t* ks_s = st + G::OFF_KS;
            const uint8_t* vs_s = st + G::OFF_VS;

#pragma unroll
            for (int sub = 0; sub < kTile / 16; ++sub) {
                if (aborted || sub * 16 >= valid) break;
                // ---------------- K: dequantize this lane's A fragments -------------
                const int r0 = sub * 16 + gid;
                uint32_t fk[2][2 * G::WK];  // [token r0 / r0+8][fp8x4 words]
#pragma unroll
                for (int rr = 0; rr < 2; ++rr) {
                    const int r = r0 + 8 * rr;
                    uint32_t w[G::WK];
                    if constexpr (D == 128) {
                        const uint4 x = *reinterpret_cast<const uint4*>(kc_s + r * G::KB + 16 * tig);
                        w[0] = x.x; w[1] = x.y; w[2] = x.z; w[3] = x.w;
                    } else {
                        const uint2 x = *reinterpret_cast<const uint2*>(kc_s + r * G::KB + 8 * tig);
                        w[0] = x.x; w[1] = x.y;
                    }
#pragma unroll
                    for (int j = 0; j < G::WK; ++j) {
                        const int blk = (G::EK * tig + 8 * j) / 16;
                        const uint2 lut = sm.lut_k[ks_s[r * G::SB + blk] & 0x7F];
                        dequant_word(w[j], lut.x, lut.y, fk[rr][2 * j], fk[rr][2 * j + 1]);
                    }
                }
                // ---------------- S^T = K Q^T on tensor cores -----------------------
                float sacc[NT][4];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int k = 0; k < 4; ++k) sacc[nt][k] = 0.0f;
#pragma unroll
                for (int s = 0; s < KS; ++s) {
                    const uint32_t a0 = lo16_to_f16x2(fk[0][s]);
                    const uint32_t a2 = hi16_to_f16x2(fk[0][s]);
                    const uint32_t a1 = lo16_to_f16x2(fk[1][s]);
                    const uint32_t a3 = hi16_to_f16x2(fk[1][s]);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        mma_f16_16816(sacc[nt], a0, a1, a2, a3, qf[s][nt][0], qf[s][nt][1]);
                        if (QF32) mma_f16_16816(sacc[nt], a0, a1, a2, a3, ql[s][nt][0], ql[s][nt][1]);
                    }
                }
                // ---------------- online softmax (base 2, lazy max) -----------------
                const bool row0_ok = (sub * 16 + gid) < valid;
                const bool row1_ok = (sub * 16 + gid + 8) < valid;
                bool need = false;
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    sacc[nt][0] = row0_ok ? sacc[nt][0] * cscale[nt][0] : -INFINITY;
                    sacc[nt][1] = row0_ok ? sacc[nt][1] * cscale[nt][1] : -INFINITY;
                    sacc[nt][2] = row1_ok ? sacc[nt][2] * cscale[nt][0] : -INFINITY;
                    sacc[nt][3] = row1_ok ? sacc[nt][3] * cscale[nt][1] : -INFINITY;
                    need |= fmaxf(sacc[nt][0], sacc[nt][2]) > m_run[nt][0] + kRescaleSlack;
                    need |= fmaxf(sacc[nt][1], sacc[nt][3]) > m_run[nt][1] + kRescaleSlack;
                }
                if (__any_sync(0xFFFFFFFFu, need)) {
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
                        for (int k = 0; k < 2; ++k) {
                            float mx = fmaxf(sacc[nt][k], sacc[nt][k + 2]);
                            mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 4));
                            mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 8));
                            mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 16));
                            const float m_new = fmaxf(m_run[nt][k], mx);
                            const float f = (m_run[nt][k] == -INFINITY) ? 0.0f : fast_exp2(m_run[nt][k] - m_new);
                            m_run[nt][k] = m_new;
                            l_run[nt][k] *= f;
#pragma unroll
                            for (int i = 0; i < KS; ++i) {
                                o[i][nt][k] *= f;
                                o[i][nt][k + 2] *= f;
                            }
                        }
                    }
                }
                uint32_t bph[NT][2], bpl[NT][2];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    float pv[4];
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        pv[k] = fast_exp2(sacc[nt][k] - m_run[nt][k & 1]);
                        l_run[nt][k & 1] += pv[k];
                    }
                    const uint32_t h01 = pack_f16x2(pv[0], pv[1]);
                    const uint32_t h23 = pack_f16x2(pv[2], pv[3]);
                    const uint32_t l01 = pack_f16x2(pv[0] - f16_lo_to_float(h01), pv[1] - f16_hi_to_float(h01));
                    const uint32_t l23 = pack_f16x2(pv[2] - f16_lo_to_float(h23), pv[3] - f16_hi_to_float(h23));
                    bph[nt][0] = movmatrix_trans(h01);
                    bph[nt][1] = movmatrix_trans(h23);
                    bpl[nt][0] = movmatrix_trans(l01);
                    bpl[nt][1] = movmatrix_trans(l23);
                }
                // ---------------- V: dequantize token pairs for the A fragments -----
                // lane (gid, tig) covers tokens 2tig, 2tig+1, 2tig+8, 2tig+9 of the
                // sub-tile and channels [EV*gid, EV*gid + EV) (one scale block)
                uint32_t gv[4][2 * G::WV];
#pragma unroll
                for (int tt = 0; tt < 4; ++tt) {
                    const int r = sub * 16 + 2 * tig + (tt & 1) + 8 * (tt >> 1);
                    const uint2 lut = sm.lut_v[vs_s[r * G::SB + (G::EV * gid) / 16] & 0x7F];
                    if constexpr (D == 128) {
                        const uint2 x = *reinterpret_cast<const uint2*>(vc_s + r * G::KB + 8 * gid);
                        dequant_word(x.x, lut.x, lut.y, gv[tt][0], gv[tt][1]);
                        dequant_word(x.y, lut.x, lut.y, gv[tt][2], gv[tt][3]);
                    } else {
                        const uint32_t x = *reinterpret_cast<const uint32_t*>(vc_s + r * G::KB + 4 * gid);
                        dequant_word(x, lut.x, lut.y, gv[tt][0], gv[tt][1]);
                    }
                }
                // ---------------- O^T += V^T P^T on tensor cores --------------------
#pragma unroll
                for (int i = 0; i < KS; ++i) {
                    // row gid <-> channel i, row gid + 8 <-> channel KS + i (of the lane's EV)
                    const int e0 = i, e1 = KS + i;
                    const uint32_t sel0 = (e0 & 2) ? 0x7362u : 0x5140u;
                    const uint32_t sel1 = (e1 & 2) ? 0x7362u : 0x5140u;
                    const uint32_t p00 = __byte_perm(gv[0][e0 >> 2], gv[1][e0 >> 2], sel0);
                    const uint32_t p01 = __byte_perm(gv[0][e1 >> 2], gv[1][e1 >> 2], sel1);
                    const uint32_t p10 = __byte_perm(gv[2][e0 >> 2], gv[3][e0 >> 2], sel0);
                    const uint32_t p11 = __byte_perm(gv[2][e1 >> 2], gv[3][e1 >> 2], sel1);
                    const uint32_t a0 = (e0 & 1) ? hi16_to_f16x2(p00) : lo16_to_f16x2(p00);
                    const uint32_t a1 = (e1 & 1) ? hi16_to_f16x2(p01) : lo16_to_f16x2(p01);
                    const uint32_t a2 = (e0 & 1) ? hi16_to_f16x2(p10) : lo16_to_f16x2(p10);
                    const uint32_t a3 = (e1 & 1) ? hi16_to_f16x2(p11) : lo16_to_f16x2(p11);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        mma_f16_16816(o[i][nt], a0, a1, a2, a3, bph[nt][0], bph[nt][1]);
                        mma_f16_16816(o[i][nt], a0, a1, a2, a3, bpl[nt][0], bpl[nt][1]);
                    }
                }
            }
            ++consumed;
            // ---- refill this stage with the warp's next tile ----
            __syncwarp();
            if (lane == 0 && !prod.done) {
                fence_proxy_async_smem();
                issue_tile<D>(p, prod.u, prod.gt, sm.ring[warp][stage], &sm.bar[warp][stage]);
                ++issued;
                cursor_next(prod, sm.prefix, sm.lens, B, p.Hkv, warp);
            }
        }

        // ---- merge the warps of this CTA for the segment -------------------
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                float l = l_run[nt][k];
                l += __shfl_xor_sync(0xFFFFFFFFu, l, 4);
                l += __shfl_xor_sync(0xFFFFFFFFu, l, 8);
                l += __shfl_xor_sync(0xFFFFFFFFu, l, 16);
                if (gid == 0) {
                    sm.merge_m[warp][8 * nt + 2 * tig + k] = m_run[nt][k];
                    sm.merge_l[warp][8 * nt + 2 * tig + k] = l;
                }
            }
#pragma unroll
            for (int i = 0; i < KS; ++i) {
                const int d0 = G::EV * gid + i;
                const int d1 = G::EV * gid + KS + i;
                const int q0 = 8 * nt + 2 * tig;
                sm.merge_o[warp][q0][d0] = o[i][nt][0];
                sm.merge_o[warp][q0 + 1][d0] = o[i][nt][1];
                sm.merge_o[warp][q0][d1] = o[i][nt][2];
                sm.merge_o[warp][q0 + 1][d1] = o[i][nt][3];
            }
        }
        __syncthreads();

        const bool whole = (u.U0 >= t_begin) && (u.U1 <= t_end);
        const int g = p.g;
        const int64_t slot = partial_slot(c, u.U0, T, N);
        const int64_t slot_floats = (int64_t)g * (D + 2);
        for (int idx = tid; idx < g * D; idx += kWarps * 32) {
            const int q = idx / D, d = idx - q * D;
            float M = -INFINITY;
#pragma unroll
            for (int w = 0; w < kWarps; ++w) M = fmaxf(M, sm.merge_m[w][q]);
            float acc = 0.0f, l = 0.0f;
            if (M != -INFINITY) {
#pragma unroll
                for (int w = 0; w < kWarps; ++w) {
                    const float mw = sm.merge_m[w][q];
                    if (mw == -INFINITY) continue;
                    const float f = fast_exp2(mw - M);
                    acc += f * sm.merge_o[w][q][d];
                    l += f * sm.merge_l[w][q];
                }
            }
            if (whole) {
                p.out[((int64_t)u.b * p.Hq + (int64_t)u.h * g + q) * D + d] = (l > 0.0f) ? acc / l : 0.0f;
            } else {
                float* part = p.partials + slot * slot_floats;
                part[q * D + d] = acc;
                if (d == 0) {
                    part[g * D + q] = M;
                    part[g * D + g + q] = l;
                }
            }
        }
        if (!whole) {
            __threadfence();
            __syncthreads();
            if (tid == 0) {
                // contributors: the CTAs with a non-empty range inside the unit's
                // span (ranges are empty only when there are fewer tiles than CTAs)
                const int64_t c_first = cta_of(u.U0, T, N);
                const int64_t c_last = cta_of(u.U1 - 1, T, N);
                int contributors = 0;
                for (int64_t cc = c_first; cc <= c_last; ++cc)
                    contributors += range_start(cc, T, N) < range_start(cc + 1, T, N);
                const int prev = atomicAdd(&p.counters[(int64_t)u.b * p.Hkv + u.h], 1);
                sm.last_flag = (prev == contributors - 1);
            }
            __syncthreads();
            if (sm.last_flag) {
                __threadfence();
                const int64_t c_first = cta_of(u.U0, T, N);
                const int64_t c_last = cta_of(u.U1 - 1, T, N);
                for (int idx = tid; idx < g * D; idx += kWarps * 32) {
                    const int q = idx / D, d = idx - q * D;
                    float M = -INFINITY;
                    for (int64_t cc = c_first; cc <= c_last; ++cc) {
                        if (range_start(cc, T, N) == range_start(cc + 1, T, N)) continue;
                        const int64_t sl = partial_slot(cc, u.U0, T, N);
                        M = fmaxf(M, __ldcg(p.partials + sl * slot_floats + g * D + q));
                    }
                    float acc = 0.0f, l = 0.0f;
                    if (M != -INFINITY) {
                        for (int64_t cc = c_first; cc <= c_last; ++cc) {
                            if (range_start(cc, T, N) == range_start(cc + 1, T, N)) continue;
                            const int64_t sl = partial_slot(cc, u.U0, T, N);
                            const float* part = p.partials + sl * slot_floats;
                            const float mw = __ldcg(part + g * D + q);
                            if (mw == -INFINITY) continue;
                            const float f = fast_exp2(mw - M);
                            acc += f * __ldcg(part + q * D + d);
                            l += f * __ldcg(part + g * D + g + q);
                        }
                    }
                    p.out[((int64_t)u.b * p.Hq + (int64_t)u.h * g + q) * D + d] = (l > 0.0f) ? acc / l : 0.0f;
                }
                if (tid == 0) atomicExch(&p.counters[(int64_t)u.b * p.Hkv + u.h], 0);
            }
        }
        __syncthreads();  // merge buffers are reused by the next segment
        seg_lo = seg_hi;
    }

    // ---- drain: no bulk copy may still target this CTA's memory ------------
    while (consumed < issued) {
        const int stage = (int)(consumed % kStages);
        const uint32_t parity = (consumed / kStages) & 1u;
        if (!mbar_wait_bounded(&sm.bar[warp][stage], parity, kWaitLimit)) {
            report(p.status, NVFP4_ERR_TIMEOUT);
            break;
        }
        ++consumed;
    }
}

template <int D, int NT, bool QF32>
cudaError_t launch_instance(const Params& p, int grid, cudaStream_t stream) {
    auto kern = decode_attention_kernel<D, NT, QF32>;
    const int smem = (int)sizeof(Smem<D, NT>);
    static int configured_device = -1;
    int dev = 0;
    cudaGetDevice(&dev);
    if (configured_device != dev) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        configured_device = dev;
    }
    kern<<<grid, kWarps * 32, smem, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode_attention(const AttnLaunch& a, cudaStream_t stream) {
    Params p;
    p.q = a.q;
    p.kc = a.kc; p.ks = a.ks; p.vc = a.vc; p.vs = a.vs;
    p.st_k = a.st_k; p.st_v = a.st_v;
    p.seq_lens = a.seq_lens;
    p.out = a.out;
    p.partials = a.partials;
    p.counters = a.counters;
    p.status = a.status;
    p.B = a.B; p.Hq = a.Hq; p.Hkv = a.Hkv; p.g = a.Hq / a.Hkv; p.S_max = a.S_max;
    p.softmax_scale = a.softmax_scale;
    const bool two = p.g > 8;
    if (a.D == 128) {
        if (!two) return a.q_f32 ? launch_instance<128, 1, true>(p, a.grid, stream)
                                 : launch_instance<128, 1, false>(p, a.grid, stream);
        return a.q_f32 ? launch_instance<128, 2, true>(p, a.grid, stream)
                       : launch_instance<128, 2, false>(p, a.grid, stream);
    }
    if (!two) return a.q_f32 ? launch_instance<64, 1, true>(p, a.grid, stream)
                             : launch_instance<64, 1, false>(p, a.grid, stream);
    return a.q_f32 ? launch_instance<64, 2, true>(p, a.grid, stream)
                   : launch_instance<64, 2, false>(p, a.grid, stream);
}

size_t attention_smem_bytes(int D, int NT) {
    if (D == 128) return NT == 1 ? sizeof(Smem<128, 1>) : sizeof(Smem<128, 2>);
    return NT == 1 ? sizeof(Smem<64, 1>) : sizeof(Smem<64, 2>);
}

}  // namespace nvfp4kv

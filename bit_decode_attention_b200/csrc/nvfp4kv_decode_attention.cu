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
#include "nvfp4kv_tcgen05.cuh"

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

// scratch of the split-K merge (see combine_partials)
struct CombineSmem {
    int32_t slot[32];         // partial slot of chunk contributor j, -1 if none
    float w[16][32];          // weight of contributor j for query q
    float M[16];
    float l[16];
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
    CombineSmem comb;
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

template <int TILE = kTile>
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
    u.ntb = u.L > 0 ? (u.L + TILE - 1) / TILE : 1;
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

template <int TILE = kTile, int STRIDE = kWarps>
__device__ __forceinline__ void cursor_enter(Cursor& c, const int32_t* prefix, const int32_t* lens,
                                             int B, int Hkv, int warp) {
    // find the next segment (from c.seg_lo) holding a tile for this warp
    while (c.seg_lo < c.t_end) {
        c.u = find_unit<TILE>(prefix, lens, B, Hkv, c.seg_lo);
        c.seg_hi = c.u.U1 < c.t_end ? c.u.U1 : c.t_end;
        c.gt = c.seg_lo + warp;
        if (c.gt < c.seg_hi) return;
        c.seg_lo = c.seg_hi;
    }
    c.done = true;
}

template <int TILE = kTile, int STRIDE = kWarps>
__device__ __forceinline__ void cursor_next(Cursor& c, const int32_t* prefix, const int32_t* lens,
                                            int B, int Hkv, int warp) {
    c.gt += STRIDE;
    if (c.gt < c.seg_hi) return;
    c.seg_lo = c.seg_hi;
    cursor_enter<TILE, STRIDE>(c, prefix, lens, B, Hkv, warp);
}

// Issue the bulk copies of one tile into a ring stage (one lane).
template <int D, int TILE = kTile>
__device__ __forceinline__ void issue_tile(const Params& p, const Unit& u, int64_t gt, uint8_t* stage,
                                           uint64_t* bar) {
    using G = Geometry<D>;
    constexpr int OFF_VC = TILE * G::KB;
    constexpr int OFF_KS = 2 * TILE * G::KB;
    constexpr int OFF_VS = 2 * TILE * G::KB + TILE * G::SB;
    const int t0 = (int)(gt - u.U0) * TILE;
    int n = u.L - t0;
    n = n < 0 ? 0 : (n > TILE ? TILE : n);
    const int ncopy = (n + 3) & ~3;  // keeps every copy a multiple of 16 bytes
    const uint32_t code_bytes = (uint32_t)ncopy * G::KB;
    const uint32_t scale_bytes = (uint32_t)ncopy * G::SB;
    mbar_arrive_expect_tx(bar, 2 * (code_bytes + scale_bytes));
    if (ncopy > 0) {
        const int64_t tok = ((int64_t)u.b * p.Hkv + u.h) * p.S_max + t0;
        bulk_g2s(stage, p.kc + tok * G::KB, code_bytes, bar);
        bulk_g2s(stage + OFF_VC, p.vc + tok * G::KB, code_bytes, bar);
        bulk_g2s(stage + OFF_KS, p.ks + tok * G::SB, scale_bytes, bar);
        bulk_g2s(stage + OFF_VS, p.vs + tok * G::SB, scale_bytes, bar);
    }
}

__device__ __forceinline__ uint32_t pow2_bits(int e) {  // 2^e as fp32 bits, e in [-126, 127]
    return (uint32_t)(127 + e) << 23;
}

// ---------------------------------------------------------------------------
// Query operands.  Lane (gid, tig) holds query row j = 8*nt + gid, head_dim
// elements [EK*tig, EK*tig + EK): the same elements its K fragments carry,
// in the same order, so the contraction runs over a permutation of head_dim
// that both operands share.
//
//  * bf16 queries -> FP8 (E4M3) MMA operands: every bf16 value (8 significant
//    bits) is split exactly into hi = E4M3(q') and lo = E4M3((q' - hi) * 16),
//    q' = q * 2^e with e chosen per row so that max |q'| < 256.  The two
//    products go to separate accumulators: s = s_hi + s_lo / 16.
//  * fp32 queries -> f16 MMA operands: hi = f16(q'), lo = f16(q' - hi)
//    (22 bits), q' scaled so that max |q'| < 2^14; both accumulate together.
// cscale[nt][c] = softmax_scale * log2(e) * 2^-e of the row in score column
// 2*tig + c.
// ---------------------------------------------------------------------------
template <int D, int NT, bool QF32>
struct QueryFrags;

template <int D, int NT>
struct QueryFrags<D, NT, false> {
    static constexpr int S = D / 32;          // k32 steps
    uint32_t hi[S][NT][2], lo[S][NT][2];
    float cscale[NT][2];
};

template <int D, int NT>
struct QueryFrags<D, NT, true> {
    static constexpr int S = D / 16;          // k16 steps
    uint32_t hi[S][NT][2], lo[S][NT][2];
    float cscale[NT][2];
};

template <int D, int NT, bool QF32>
__device__ __forceinline__ void load_q(const Params& p, int b, int h, int gid, int tig,
                                       QueryFrags<D, NT, QF32>& qf) {
    using G = Geometry<D>;
    const float base = p.softmax_scale * kLog2e;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const int j = 8 * nt + gid;
        const bool valid = j < p.g;
        float v[G::EK];
        const int64_t row = ((int64_t)b * p.Hq + (int64_t)h * p.g + (valid ? j : 0)) * D + G::EK * tig;
        if constexpr (QF32) {
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
        constexpr int kTopExp = QF32 ? 14 : 8;   // max |q'| < 2^kTopExp
        int e = 0;
        if (amax > 0.0f && amax <= 3.4028234663852886e38f) {
            int ex;
            frexpf(amax, &ex);                    // amax < 2^ex
            e = kTopExp - ex;
            e = e < -126 ? -126 : (e > 126 ? 126 : e);
        }
        const float up = __uint_as_float(pow2_bits(e));
        const float down = __uint_as_float(pow2_bits(-e));
#pragma unroll
        for (int i = 0; i < G::EK; ++i) v[i] *= up;
        if constexpr (QF32) {
#pragma unroll
            for (int s = 0; s < G::KS; ++s) {
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    const float x0 = v[4 * s + 2 * k], x1 = v[4 * s + 2 * k + 1];
                    const uint32_t hi = pack_f16x2(x0, x1);
                    qf.hi[s][nt][k] = hi;
                    qf.lo[s][nt][k] = pack_f16x2(x0 - f16_lo_to_float(hi), x1 - f16_hi_to_float(hi));
                }
            }
        } else {
#pragma unroll
            for (int s = 0; s < D / 32; ++s) {
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    const float* x = v + 8 * s + 4 * k;
                    const uint32_t h01 = e4m3x2_from_floats(x[0], x[1]);
                    const uint32_t h23 = e4m3x2_from_floats(x[2], x[3]);
                    uint32_t f01, f23;
                    e4m3x4_to_f16x2x2(h01 | (h23 << 16), f01, f23);
                    const uint32_t l01 = e4m3x2_from_floats((x[0] - f16_lo_to_float(f01)) * 16.0f,
                                                            (x[1] - f16_hi_to_float(f01)) * 16.0f);
                    const uint32_t l23 = e4m3x2_from_floats((x[2] - f16_lo_to_float(f23)) * 16.0f,
                                                            (x[3] - f16_hi_to_float(f23)) * 16.0f);
                    qf.hi[s][nt][k] = h01 | (h23 << 16);
                    qf.lo[s][nt][k] = l01 | (l23 << 16);
                }
            }
        }
        // score column c of this lane is query row 2*tig + c; its scale lives
        // in lanes (gid = 2*tig + c, tig = 0)
        const float f0 = __shfl_sync(0xFFFFFFFFu, down, (2 * tig) * 4);
        const float f1 = __shfl_sync(0xFFFFFFFFu, down, (2 * tig + 1) * 4);
        qf.cscale[nt][0] = base * f0;
        qf.cscale[nt][1] = base * f1;
    }
}

// K operands of one 16-token sub-tile: lane (gid, tig) dequantizes tokens
// gid and gid + 8, head_dim elements [EK*tig, EK*tig + EK) (EK/16 blocks).
// fk[rr][w] = FP8 bytes of elements 4w .. 4w+3 of token gid + 8*rr.
template <int D>
__device__ __forceinline__ void dequant_k(const uint8_t* kc_s, const uint8_t* ks_s, const uint2* lut,
                                          int sub, int gid, int tig, uint32_t (&fk)[2][D / 8]) {
    using G = Geometry<D>;
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
        const int r = sub * 16 + gid + 8 * rr;
        if constexpr (D == 128) {
            const uint4 x = *reinterpret_cast<const uint4*>(kc_s + r * G::KB + 16 * tig);
            const uint32_t sb = *reinterpret_cast<const uint16_t*>(ks_s + r * G::SB + 2 * tig);
            const uint2 l0 = lut[sb & 0x7F];
            const uint2 l1 = lut[(sb >> 8) & 0x7F];
            dequant_word(x.x, l0.x, l0.y, fk[rr][0], fk[rr][1]);
            dequant_word(x.y, l0.x, l0.y, fk[rr][2], fk[rr][3]);
            dequant_word(x.z, l1.x, l1.y, fk[rr][4], fk[rr][5]);
            dequant_word(x.w, l1.x, l1.y, fk[rr][6], fk[rr][7]);
        } else {
            const uint2 x = *reinterpret_cast<const uint2*>(kc_s + r * G::KB + 8 * tig);
            const uint2 l0 = lut[ks_s[r * G::SB + tig] & 0x7F];
            dequant_word(x.x, l0.x, l0.y, fk[rr][0], fk[rr][1]);
            dequant_word(x.y, l0.x, l0.y, fk[rr][2], fk[rr][3]);
        }
    }
}

// V operands of one 16-token sub-tile: lane (gid, tig) dequantizes tokens
// 2tig, 2tig+1, 2tig+8, 2tig+9 over channels [EV*gid, EV*gid + EV) (one
// block); gv[tt][w] = FP8 bytes of channels 4w .. 4w+3 of token tt.
template <int D>
__device__ __forceinline__ void dequant_v(const uint8_t* vc_s, const uint8_t* vs_s, const uint2* lut,
                                          int sub, int gid, int tig, int valid,
                                          uint32_t (&gv)[4][D / 32]) {
    using G = Geometry<D>;
#pragma unroll
    for (int tt = 0; tt < 4; ++tt) {
        const int r = sub * 16 + 2 * tig + (tt & 1) + 8 * (tt >> 1);
        uint2 l = lut[vs_s[r * G::SB + (G::EV * gid) / 16] & 0x7F];
        // bytes past the sequence may hold anything (a NaN scale): P is 0
        // there, and a zero table makes V +-0 so that 0 * V stays 0
        if (r >= valid) l = make_uint2(0u, 0u);
        if constexpr (D == 128) {
            const uint2 x = *reinterpret_cast<const uint2*>(vc_s + r * G::KB + 8 * gid);
            dequant_word(x.x, l.x, l.y, gv[tt][0], gv[tt][1]);
            dequant_word(x.y, l.x, l.y, gv[tt][2], gv[tt][3]);
        } else {
            const uint32_t x = *reinterpret_cast<const uint32_t*>(vc_s + r * G::KB + 4 * gid);
            dequant_word(x, l.x, l.y, gv[tt][0], gv[tt][1]);
        }
    }
}

// ---------------------------------------------------------------------------
// Split-K merge of one (sequence, KV head) unit by the last CTA to finish with
// it.  The contributors are CTAs c_first..c_last (those with non-empty ranges);
// each left (m, l, O) per query in its partial slot.  Out = sum_c w_c O_c /
// sum_c w_c l_c with w_c = 2^(m_c - M), M = max_c m_c.  Contributors are
// walked in chunks of 32 whose slot indices are computed once per chunk.
// ---------------------------------------------------------------------------
template <int D, int NT, int THREADS = kWarps * 32>
__device__ __noinline__ void combine_partials(const Params& p, CombineSmem& cs, const Unit& u,
                                                 int64_t T, int64_t N, int64_t c_first,
                                                 int64_t c_last, int64_t slot_floats, int tid,
                                                 int warp, int lane) {
    constexpr int kThreads = THREADS;                // every thread of the CTA calls this
    constexpr int kNumWarps = THREADS / 32;
    constexpr int kMaxOut = 8 * NT * D / kThreads;   // outputs per thread for g <= 8 * NT
    const int g = p.g;
    const int ncc = (int)(c_last - c_first + 1);
    float acc[kMaxOut];
#pragma unroll
    for (int k = 0; k < kMaxOut; ++k) acc[k] = 0.0f;
    for (int q = tid; q < g; q += kThreads) {
        cs.M[q] = -INFINITY;
        cs.l[q] = 0.0f;
    }
    for (int pass = 0; pass < 2; ++pass) {
        for (int base = 0; base < ncc; base += 32) {
            __syncthreads();
            if (warp == 0) {
                int sl = -1;
                if (base + lane < ncc) {
                    const int64_t cc = c_first + base + lane;
                    if (range_start(cc, T, N) < range_start(cc + 1, T, N))
                        sl = (int)partial_slot(cc, u.U0, T, N);
                }
                cs.slot[lane] = sl;
            }
            __syncthreads();
            const int sl = cs.slot[lane];
            for (int q = warp; q < g; q += kNumWarps) {
                const float* part = p.partials + (int64_t)(sl < 0 ? 0 : sl) * slot_floats;
                const float m = sl < 0 ? -INFINITY : __ldcg(part + g * D + q);
                if (pass == 0) {
                    float mx = m;
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
                    if (lane == 0) cs.M[q] = fmaxf(cs.M[q], mx);
                } else {
                    const float M = cs.M[q];
                    const float w = (m == -INFINITY) ? 0.0f : fast_exp2(m - M);
                    cs.w[q][lane] = w;
                    float lw = (w == 0.0f) ? 0.0f : w * __ldcg(part + g * D + g + q);
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) lw += __shfl_xor_sync(0xFFFFFFFFu, lw, o);
                    if (lane == 0) cs.l[q] += lw;
                }
            }
            if (pass == 1) {
                __syncthreads();
                const int nj = ncc - base < 32 ? ncc - base : 32;
#pragma unroll
                for (int k = 0; k < kMaxOut; ++k) {
                    const int idx = tid + k * kThreads;
                    if (idx >= g * D) break;
                    const int q = idx / D, d = idx - q * D;
                    float a = acc[k];
#pragma unroll 4
                    for (int j = 0; j < nj; ++j) {
                        const int s2 = cs.slot[j];
                        if (s2 < 0) continue;
                        a += cs.w[q][j] * __ldcg(p.partials + (int64_t)s2 * slot_floats + q * D + d);
                    }
                    acc[k] = a;
                }
            }
        }
        __syncthreads();
    }
#pragma unroll
    for (int k = 0; k < kMaxOut; ++k) {
        const int idx = tid + k * kThreads;
        if (idx >= g * D) break;
        const int q = idx / D, d = idx - q * D;
        const float l = cs.l[q];
        p.out[((int64_t)u.b * p.Hq + (int64_t)u.h * g + q) * D + d] = (l > 0.0f) ? acc[k] / l : 0.0f;
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

    // ---- prologue 1: barriers, sequence lengths, this CTA's tile range -----
    const float st_k = *p.st_k;
    const float st_v = *p.st_v;
    if (lane == 0) {
#pragma unroll
        for (int s = 0; s < kStages; ++s) mbar_init(&sm.bar[warp][s], 1);
        fence_mbar_init();
    }
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

    // ---- prologue 2: lane 0 of each warp starts filling the warp's ring ----
    Cursor prod;
    prod.seg_lo = t_begin;
    prod.t_end = t_end;
    prod.done = false;
    uint32_t issued = 0;
    if (lane == 0) {
        cursor_enter(prod, sm.prefix, sm.lens, B, p.Hkv, warp);
        for (int s = 0; s < kStages && !prod.done; ++s) {
            issue_tile<D>(p, prod.u, prod.gt, sm.ring[warp][s], &sm.bar[warp][s]);
            ++issued;
            cursor_next(prod, sm.prefix, sm.lens, B, p.Hkv, warp);
        }
    }

    // ---- prologue 3: FP8 lookup tables, built while the first copies fly ---
    for (int sb = tid; sb < 128; sb += kWarps * 32) {
        sm.lut_k[sb] = lut_words((uint32_t)sb, st_k);
        sm.lut_v[sb] = lut_words((uint32_t)sb, st_v);
    }
    if (tid == 0 && blockIdx.x == 0) {
        const bool ok = st_k > 0.f && st_k <= 3.4028234663852886e38f && st_v > 0.f &&
                        st_v <= 3.4028234663852886e38f;
        if (!ok) report(p.status, NVFP4_ERR_NONFINITE);
    }
    __syncthreads();

    uint32_t consumed = 0;
    bool aborted = false;

    // ---- segments of the CTA range, processed by all warps together --------
    int64_t seg_lo = t_begin;
    while (seg_lo < t_end) {
        const Unit u = find_unit(sm.prefix, sm.lens, B, p.Hkv, seg_lo);
        const int64_t seg_hi = u.U1 < t_end ? u.U1 : t_end;

        QueryFrags<D, NT, QF32> qf;
        load_q<D, NT, QF32>(p, u.b, u.h, gid, tig, qf);

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
            const bool sub1 = valid > 16;

            if (!aborted && valid > 0) {
                // ---------------- S^T = K Q^T for both 16-token sub-tiles -----------
                float sc[2][NT][4];
#pragma unroll
                for (int sub = 0; sub < 2; ++sub) {
                    if (sub == 1 && !sub1) break;
                    uint32_t fk[2][D / 8];
                    dequant_k<D>(kc_s, ks_s, sm.lut_k, sub, gid, tig, fk);
                    float sh[NT][4], sl[NT][4];
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                        for (int k = 0; k < 4; ++k) sh[nt][k] = sl[nt][k] = 0.0f;
                    if constexpr (QF32) {
#pragma unroll
                        for (int s = 0; s < KS; ++s) {
                            uint32_t a0, a2, a1, a3;
                            e4m3x4_to_f16x2x2(fk[0][s], a0, a2);
                            e4m3x4_to_f16x2x2(fk[1][s], a1, a3);
#pragma unroll
                            for (int nt = 0; nt < NT; ++nt) {
                                mma_f16_16816(sh[nt], a0, a1, a2, a3, qf.hi[s][nt][0], qf.hi[s][nt][1]);
                                mma_f16_16816(sl[nt], a0, a1, a2, a3, qf.lo[s][nt][0], qf.lo[s][nt][1]);
                            }
                        }
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                            for (int k = 0; k < 4; ++k) sc[sub][nt][k] = sh[nt][k] + sl[nt][k];
                    } else {
#pragma unroll
                        for (int s = 0; s < D / 32; ++s) {
#pragma unroll
                            for (int nt = 0; nt < NT; ++nt) {
                                mma_e4m3_16832(sh[nt], fk[0][2 * s], fk[1][2 * s], fk[0][2 * s + 1],
                                               fk[1][2 * s + 1], qf.hi[s][nt][0], qf.hi[s][nt][1]);
                                mma_e4m3_16832(sl[nt], fk[0][2 * s], fk[1][2 * s], fk[0][2 * s + 1],
                                               fk[1][2 * s + 1], qf.lo[s][nt][0], qf.lo[s][nt][1]);
                            }
                        }
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                            for (int k = 0; k < 4; ++k) sc[sub][nt][k] = fmaf(sl[nt][k], 0.0625f, sh[nt][k]);
                    }
                }
                // ---------------- online softmax over the 32 tokens (base 2) -------
                bool need = false;
#pragma unroll
                for (int sub = 0; sub < 2; ++sub) {
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const int row = sub * 16 + gid + 8 * (k >> 1);
                            const float v = (sub == 0 || sub1) ? sc[sub][nt][k] : 0.0f;
                            sc[sub][nt][k] = row < valid ? v * qf.cscale[nt][k & 1] : -INFINITY;
                            need |= sc[sub][nt][k] > m_run[nt][k & 1] + kRescaleSlack;
                        }
                    }
                }
                if (__any_sync(0xFFFFFFFFu, need)) {
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
                        for (int col = 0; col < 2; ++col) {
                            float mx = fmaxf(fmaxf(sc[0][nt][col], sc[0][nt][col + 2]),
                                             fmaxf(sc[1][nt][col], sc[1][nt][col + 2]));
                            mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 4));
                            mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 8));
                            mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 16));
                            const float m_new = fmaxf(m_run[nt][col], mx);
                            const float f = (m_run[nt][col] == -INFINITY) ? 0.0f : fast_exp2(m_run[nt][col] - m_new);
                            m_run[nt][col] = m_new;
                            l_run[nt][col] *= f;
#pragma unroll
                            for (int i = 0; i < KS; ++i) {
                                o[i][nt][col] *= f;
                                o[i][nt][col + 2] *= f;
                            }
                        }
                    }
                }
                // ---------------- P (hi + lo f16) and O^T += V^T P^T ---------------
#pragma unroll
                for (int sub = 0; sub < 2; ++sub) {
                    if (sub == 1 && !sub1) break;
                    uint32_t bph[NT][2], bpl[NT][2];
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        float pv[4];
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            pv[k] = fast_exp2(sc[sub][nt][k] - m_run[nt][k & 1]);
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
                    uint32_t gv[4][D / 32];
                    dequant_v<D>(vc_s, vs_s, sm.lut_v, sub, gid, tig, valid, gv);
                    // m-tile i: row gid <-> channel i, row gid + 8 <-> channel KS + i
                    // (of the lane's EV channels); consecutive tokens pair up in f16x2
#pragma unroll
                    for (int i = 0; i < KS; i += 2) {
                        const int e0 = i, e1 = KS + i;
                        const uint32_t sel0 = (e0 & 2) ? 0x7362u : 0x5140u;
                        const uint32_t sel1 = (e1 & 2) ? 0x7362u : 0x5140u;
                        uint32_t a0[2], a1[2], a2[2], a3[2];
                        e4m3x4_to_f16x2x2(__byte_perm(gv[0][e0 >> 2], gv[1][e0 >> 2], sel0), a0[0], a0[1]);
                        e4m3x4_to_f16x2x2(__byte_perm(gv[0][e1 >> 2], gv[1][e1 >> 2], sel1), a1[0], a1[1]);
                        e4m3x4_to_f16x2x2(__byte_perm(gv[2][e0 >> 2], gv[3][e0 >> 2], sel0), a2[0], a2[1]);
                        e4m3x4_to_f16x2x2(__byte_perm(gv[2][e1 >> 2], gv[3][e1 >> 2], sel1), a3[0], a3[1]);
#pragma unroll
                        for (int ii = 0; ii < 2; ++ii) {
#pragma unroll
                            for (int nt = 0; nt < NT; ++nt) {
                                mma_f16_16816(o[i + ii][nt], a0[ii], a1[ii], a2[ii], a3[ii], bph[nt][0], bph[nt][1]);
                                mma_f16_16816(o[i + ii][nt], a0[ii], a1[ii], a2[ii], a3[ii], bpl[nt][0], bpl[nt][1]);
                            }
                        }
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
                    const float f = (mw == -INFINITY) ? 0.0f : fast_exp2(mw - M);
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
            const int64_t c_first = cta_of(u.U0, T, N);
            const int64_t c_last = cta_of(u.U1 - 1, T, N);
            if (tid == 0) {
                // contributors: the CTAs with a non-empty range inside the unit's
                // span (ranges are empty only when there are fewer tiles than CTAs)
                int contributors = 0;
                for (int64_t cc = c_first; cc <= c_last; ++cc)
                    contributors += range_start(cc, T, N) < range_start(cc + 1, T, N);
                const int prev = atomicAdd(&p.counters[(int64_t)u.b * p.Hkv + u.h], 1);
                sm.last_flag = (prev == contributors - 1);
            }
            __syncthreads();
            if (sm.last_flag) {
                __threadfence();
                combine_partials<D, NT>(p, sm.comb, u, T, N, c_first, c_last, slot_floats, tid, warp, lane);
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

// ===========================================================================
// v4: the same decode attention on the fifth-generation tensor cores.
//
// One CTA = one warpgroup (128 threads); thread t owns token t of each
// 128-token tile and, at the end of a segment, head_dim row t of the output.
// Per tile:
//   1. K codes -> sign-split FP8 magnitudes K+ (positive codes) and K- (the
//      magnitudes of negative codes), written to tensor memory as the A
//      operand (lane = token, 4 bytes of head_dim per column).  Two byte
//      permutes per 4 codes and no sign arithmetic.
//   2. V codes -> signed FP8 V, written to shared memory as the MN-major A
//      operand of P.V (V^T: head_dim contiguous per token).
//   3. S^T[token][n] = K+ . Q'^T - K- . Q'^T on tcgen05 (kind::f8f6f4,
//      M = 128 tokens, B-negate for K-); the query operand holds hi and lo
//      E4M3 parts of each (power-of-two scaled) bf16 query, so s = hi + lo/16
//      is exact.
//   4. Each thread reads its score row from tensor memory, updates the online
//      softmax (base 2, running max shared by the CTA, raised lazily), and
//      writes P as four E4M3 terms p ~ t0 + t1/16 + t2/256 + t3/4096 to shared
//      memory (MN-major B operand).
//   5. O^T[d][term, q] += V^T . P^T on tcgen05 into tensor memory.
// ===========================================================================
namespace tcattn {

// ===========================================================================
// Decode attention on the fifth-generation tensor cores.
//
// A CTA is two warpgroups (256 threads).  Thread (h, t) -- warpgroup h, index
// t in 0..127 -- owns token t of each 128-token tile and tensor-memory lane t:
// it dequantizes head_dim half h of that token's K and V rows and runs the
// softmax of half h of the GQA group.  Per tile:
//   1. K codes -> sign-split FP8 magnitudes K+ (positive codes) and K- (the
//      magnitudes of negative codes), stored to tensor memory as the A
//      operand (lane = token, 4 bytes of head_dim per column).  Two byte
//      permutes per 4 codes and no sign arithmetic.
//   2. S^T[token][n] = K+ . Q'^T - K- . Q'^T on tcgen05 (kind::f8f6f4,
//      M = 128 tokens, B-negate for K-).  The query operand holds hi and lo
//      E4M3 parts of each (power-of-two scaled) bf16 query: s = hi + lo/16
//      exactly.  While it runs:
//   3. V codes -> signed FP8 V stored to shared memory as the MN-major A
//      operand of P.V (V^T: head_dim contiguous per token).
//   4. Each thread reads its score row, updates the online softmax (base 2,
//      running max shared by the CTA and raised lazily), and stores P as four
//      E4M3 terms p ~ t0 + t1/16 + t2/256 + t3/4096 (MN-major B operand).
//   5. O^T[d][term, q] += V^T . P^T on tcgen05 into tensor memory.
// ===========================================================================

constexpr int TILE = 128;
constexpr int kThreads = 256;
constexpr int kStages = 2;
constexpr int kKB = 64, kSB = 8;                       // D = 128: code / scale bytes per token
constexpr int STAGE = TILE * (2 * kKB + 2 * kSB);      // 18432
constexpr int OFF_VC = TILE * kKB;
constexpr int OFF_KS = 2 * TILE * kKB;
constexpr int OFF_VS = 2 * TILE * kKB + TILE * kSB;
constexpr int NTERM = 4;
constexpr uint32_t kTcWaitLimit = 1u << 16;         // sleeping polls (<= 20 us each) per bounded wait

template <int NT>
struct Cfg {
    static constexpr int NQ = 8 * NT;                  // query rows (padded)
    static constexpr int NQH = NQ / 2;                 // query rows per warpgroup
    static constexpr int NS = 2 * NQ;                  // score columns: hi, lo
    static constexpr int NP = NTERM * NQ;              // P columns: term-major
    static constexpr int kCtasPerSm = 2;
    static constexpr uint32_t kTmemCols = NT == 1 ? 128 : 256;
    static constexpr uint32_t COL_KP = 0, COL_KN = 32, COL_S = 64, COL_O = 64 + NS;
    static_assert(COL_O + NP <= kTmemCols, "tensor memory columns");
};

template <int NT>
struct __align__(1024) TcSmem {
    uint8_t ring[kStages][STAGE];
    uint8_t vt[128 * TILE];                            // V^T, MN-major: (d/16)*2048 + (t/8)*128 + (t%8)*16 + d%16
    uint8_t pb[Cfg<NT>::NP * TILE];                    // P^T, MN-major: (n/16)*2048 + (t/8)*128 + (t%8)*16 + n%16
    uint8_t qb[Cfg<NT>::NS * 128];                     // Q', K-major: (n/8)*1024 + (d/16)*128 + (n%8)*16 + d%16
    uint2 lut_k[128];
    uint2 lut_v[128];
    uint64_t bar_full[kStages];
    uint64_t bar_s;
    uint64_t bar_o;
    int32_t lens[kMaxBatchPerLaunch];
    int32_t prefix[kMaxBatchPerLaunch + 1];
    float cscale[Cfg<NT>::NQ];
    float red[8][Cfg<NT>::NQH];                        // [warp][query of the warp's half]
    int32_t warp_tot[8];
    CombineSmem comb;
    uint32_t tmem_base;
    int32_t last_flag;
    int32_t abort_flag;
};

// PTX byte permute in its default mode: each selector nibble picks one of
// the 8 bytes of {b, a} with bits 2..0 and, when bit 3 is set, replicates
// that byte's most significant bit over the output byte instead.
__device__ __forceinline__ uint32_t prmt_sx(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
    return r;
}

// K+ / K- for 8 codes (one word, element k in nibble k): positive codes select
// their magnitude byte and negative codes give 0 (the selector's sign bit
// replicates the msb of a lookup byte, which is 0); flipping the sign bits
// swaps the roles.  The upper 4 codes are brought down with a multiply-high
// (a shift on the FMA pipe).
__device__ __forceinline__ void dequant_split(uint32_t x, uint32_t lut_lo, uint32_t lut_hi,
                                              uint32_t& p_lo, uint32_t& p_hi, uint32_t& n_lo,
                                              uint32_t& n_hi) {
    const uint32_t xh = __umulhi(x, 0x10000u);
    const uint32_t xn = x ^ 0x88888888u;
    const uint32_t xnh = __umulhi(xn, 0x10000u);
    p_lo = prmt_sx(lut_lo, lut_hi, x);
    p_hi = prmt_sx(lut_lo, lut_hi, xh);
    n_lo = prmt_sx(lut_lo, lut_hi, xn);
    n_hi = prmt_sx(lut_lo, lut_hi, xnh);
}

__device__ __forceinline__ void tmem_ld_x4(uint32_t taddr, uint32_t* r) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(taddr)
                 : "memory");
}
__device__ __forceinline__ void tmem_st_x4(uint32_t taddr, const uint32_t* r) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1, %2, %3, %4};" ::"r"(taddr),
                 "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3])
                 : "memory");
}
__device__ __forceinline__ void tmem_st_x16(uint32_t taddr, const uint32_t* r) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15, %16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15])
        : "memory");
}
// NQH (4 or 8) consecutive columns of this thread's lane
template <int N>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t* r) {
    if constexpr (N == 4) tmem_ld_x4(taddr, r);
    else tc::tmem_ld_x8(taddr, r);
}
template <int N>
__device__ __forceinline__ void tmem_st_cols(uint32_t taddr, const uint32_t* r) {
    if constexpr (N == 4) tmem_st_x4(taddr, r);
    else tc::tmem_st_x8(taddr, r);
}

// Query operand of unit (b, h): hi/lo E4M3 rows and per-row score scales.
// fetch_q issues the global loads (so they can start a segment early);
// build_q turns them into the K-major operand rows and the score scales.
template <int NT>
struct QRaw {
    static constexpr int PER = Cfg<NT>::NQ * 128 / kThreads;   // bf16 elements per thread: 4 or 8
    uint32_t w[PER / 2];
};

template <int NT>
__device__ __forceinline__ void fetch_q(const Params& p, int b, int h, int tid, QRaw<NT>& raw) {
    constexpr int PER = QRaw<NT>::PER;
    constexpr int TPQ = 128 / PER;                     // threads per query row: 32 or 16
    const int q = tid / TPQ;
    const int d0 = (tid % TPQ) * PER;
    const bool valid = q < p.g;
    const int64_t row = ((int64_t)b * p.Hq + (int64_t)h * p.g + (valid ? q : 0)) * 128 + d0;
    const uint16_t* src = reinterpret_cast<const uint16_t*>(p.q) + row;
    if constexpr (PER == 4) {
        const uint2 w = valid ? __ldg(reinterpret_cast<const uint2*>(src)) : make_uint2(0, 0);
        raw.w[0] = w.x;
        raw.w[1] = w.y;
    } else {
        const uint4 w = valid ? __ldg(reinterpret_cast<const uint4*>(src)) : make_uint4(0, 0, 0, 0);
        raw.w[0] = w.x;
        raw.w[1] = w.y;
        raw.w[2] = w.z;
        raw.w[3] = w.w;
    }
}

template <int NT>
__device__ __forceinline__ void build_q(const Params& p, TcSmem<NT>& sm, const QRaw<NT>& raw, int tid) {
    using C = Cfg<NT>;
    constexpr int PER = QRaw<NT>::PER;
    constexpr int TPQ = 128 / PER;
    const int q = tid / TPQ;
    const int d0 = (tid % TPQ) * PER;
    float v[PER];
#pragma unroll
    for (int k = 0; k < PER / 2; ++k) {
        v[2 * k + 0] = __uint_as_float(raw.w[k] << 16);
        v[2 * k + 1] = __uint_as_float(raw.w[k] & 0xFFFF0000u);
    }
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < PER; ++i) amax = fmaxf(amax, fabsf(v[i]));
#pragma unroll
    for (int o = 1; o < TPQ; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
    int e = 0;
    if (amax > 0.0f && amax <= 3.4028234663852886e38f) {
        int ex;
        frexpf(amax, &ex);                             // amax < 2^ex
        e = 8 - ex;                                    // max |q'| < 256
        e = e < -126 ? -126 : (e > 126 ? 126 : e);
    }
    const float up = __uint_as_float(pow2_bits(e));
    uint32_t hw[PER / 4], lw[PER / 4];
#pragma unroll
    for (int i = 0; i < PER; i += 4) {
        const float x0 = v[i] * up, x1 = v[i + 1] * up, x2 = v[i + 2] * up, x3 = v[i + 3] * up;
        const uint32_t h01 = e4m3x2_from_floats(x0, x1);
        const uint32_t h23 = e4m3x2_from_floats(x2, x3);
        uint32_t f01, f23;
        e4m3x4_to_f16x2x2(h01 | (h23 << 16), f01, f23);
        const uint32_t l01 = e4m3x2_from_floats((x0 - f16_lo_to_float(f01)) * 16.0f,
                                                (x1 - f16_hi_to_float(f01)) * 16.0f);
        const uint32_t l23 = e4m3x2_from_floats((x2 - f16_lo_to_float(f23)) * 16.0f,
                                                (x3 - f16_hi_to_float(f23)) * 16.0f);
        hw[i / 4] = h01 | (h23 << 16);
        lw[i / 4] = l01 | (l23 << 16);
    }
    // K-major rows n = q (hi) and n = NQ + q (lo); d0 is a multiple of PER
    const int nh = q, nl = C::NQ + q;
    uint8_t* dh = sm.qb + (nh / 8) * 1024 + (d0 / 16) * 128 + (nh % 8) * 16 + d0 % 16;
    uint8_t* dl = sm.qb + (nl / 8) * 1024 + (d0 / 16) * 128 + (nl % 8) * 16 + d0 % 16;
    if constexpr (PER == 4) {
        *reinterpret_cast<uint32_t*>(dh) = hw[0];
        *reinterpret_cast<uint32_t*>(dl) = lw[0];
    } else {
        *reinterpret_cast<uint2*>(dh) = make_uint2(hw[0], hw[1]);
        *reinterpret_cast<uint2*>(dl) = make_uint2(lw[0], lw[1]);
    }
    if (tid % TPQ == 0)
        sm.cscale[q] = p.softmax_scale * kLog2e * __uint_as_float(pow2_bits(-e));
}

// Four E4M3 terms of p (in pairs): p ~ t0 + t1/16 + t2/256 + t3/4096.
__device__ __forceinline__ void p_terms(float p0, float p1, uint32_t (&t)[NTERM]) {
#pragma unroll
    for (int k = 0; k < NTERM; ++k) {
        const uint32_t b = e4m3x2_from_floats(p0, p1);
        t[k] = b;
        if (k + 1 < NTERM) {
            uint32_t f, unused;
            e4m3x4_to_f16x2x2(b, f, unused);
            p0 = (p0 - f16_lo_to_float(f)) * 16.0f;
            p1 = (p1 - f16_hi_to_float(f)) * 16.0f;
        }
    }
}

template <int NT>
__global__ void __launch_bounds__(kThreads, Cfg<NT>::kCtasPerSm) decode_attention_tc_kernel(const Params p) {
    using C = Cfg<NT>;
    constexpr int NQ = C::NQ;
    constexpr int NQH = C::NQH;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    TcSmem<NT>& sm = *reinterpret_cast<TcSmem<NT>*>(smem_raw);
    const int tid = threadIdx.x;
    const int warp = tid >> 5;                         // 0..7
    const int lane = tid & 31;
    const int hg = tid >> 7;                           // warpgroup: head_dim half / query half
    const int t = tid & 127;                           // token (and tensor-memory lane)
    const int wq = warp & 3;                           // lane quarter
    const int B = p.B;

    // ---- lengths, tile prefix over sequences, this CTA's range ----
    {
        constexpr int per = (kMaxBatchPerLaunch + kThreads - 1) / kThreads;
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
            tiles[i] = (b < B) ? p.Hkv * (L > 0 ? (L + TILE - 1) / TILE : 1) : 0;
            run += tiles[i];
        }
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
        if (tid == kThreads - 1) sm.prefix[B] = acc;
    }
    __syncthreads();
    const int64_t T = sm.prefix[B];
    const int64_t N = gridDim.x;
    const int64_t c = blockIdx.x;
    const int64_t t_begin = range_start(c, T, N);
    const int64_t t_end = range_start(c + 1, T, N);
    if (t_begin >= t_end) return;

    // ---- tensor memory, barriers, first copies, lookup tables ----
    if (warp == 0) {
        tc::tmem_alloc(&sm.tmem_base, C::kTmemCols);
        tc::tmem_relinquish();
    }
    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) mbar_init(&sm.bar_full[s], 1);
        mbar_init(&sm.bar_s, 1);
        mbar_init(&sm.bar_o, 1);
        fence_mbar_init();
        sm.abort_flag = 0;
    }
    __syncthreads();
    Cursor prod;
    prod.seg_lo = t_begin;
    prod.t_end = t_end;
    prod.done = false;
    uint32_t issued = 0;
    if (tid == 0) {
        cursor_enter<TILE, 1>(prod, sm.prefix, sm.lens, B, p.Hkv, 0);
        for (int s = 0; s < kStages && !prod.done; ++s) {
            issue_tile<128, TILE>(p, prod.u, prod.gt, sm.ring[s], &sm.bar_full[s]);
            ++issued;
            cursor_next<TILE, 1>(prod, sm.prefix, sm.lens, B, p.Hkv, 0);
        }
    }
    const float st_k = *p.st_k;
    const float st_v = *p.st_v;
    if (tid < 128) sm.lut_k[tid] = lut_words((uint32_t)tid, st_k);
    else sm.lut_v[tid - 128] = lut_words((uint32_t)(tid - 128), st_v);
    if (tid == 0 && blockIdx.x == 0) {
        const bool ok = st_k > 0.f && st_k <= 3.4028234663852886e38f && st_v > 0.f &&
                        st_v <= 3.4028234663852886e38f;
        if (!ok) report(p.status, NVFP4_ERR_NONFINITE);
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tbase = sm.tmem_base;
    const uint32_t trow = tbase + ((uint32_t)(32 * wq) << 16);    // this thread's lane
    const uint32_t idesc_qk = tc::idesc_e4m3(128, C::NS, false, false, false);
    const uint32_t idesc_qk_neg = tc::idesc_e4m3(128, C::NS, false, false, true);
    const uint32_t idesc_pv = tc::idesc_e4m3(128, C::NP, true, true, false);
    const uint32_t qb_addr = tc::smem_addr(sm.qb);
    const uint32_t vt_addr = tc::smem_addr(sm.vt);
    const uint32_t pb_addr = tc::smem_addr(sm.pb);
    const int q0 = hg * NQH;                           // first query row of this warpgroup

    uint32_t consumed = 0;      // ring stages consumed
    uint32_t mma_it = 0;        // tiles with MMAs issued (phases of bar_s / bar_o)
    bool aborted = false;

    QRaw<NT> qnext;
    {
        const Unit u0 = find_unit<TILE>(sm.prefix, sm.lens, B, p.Hkv, t_begin);
        fetch_q<NT>(p, u0.b, u0.h, tid, qnext);
    }
    int64_t seg_lo = t_begin;
    while (seg_lo < t_end) {
        const Unit u = find_unit<TILE>(sm.prefix, sm.lens, B, p.Hkv, seg_lo);
        const int64_t seg_hi = u.U1 < t_end ? u.U1 : t_end;
        build_q<NT>(p, sm, qnext, tid);
        if (seg_hi < t_end) {       // start the next segment's query loads now
            const Unit un = find_unit<TILE>(sm.prefix, sm.lens, B, p.Hkv, seg_hi);
            fetch_q<NT>(p, un.b, un.h, tid, qnext);
        }
        fence_proxy_async_smem();
        __syncthreads();
        float cs[NQH], m_run[NQH], l_run[NQH];
#pragma unroll
        for (int i = 0; i < NQH; ++i) {
            cs[i] = sm.cscale[q0 + i];
            m_run[i] = -INFINITY;
            l_run[i] = 0.0f;
        }
        bool any_pv = false;

        for (int64_t gt = seg_lo; gt < seg_hi; ++gt) {
            const int stage = (int)(consumed % kStages);
            const uint32_t parity = (consumed / kStages) & 1u;
            if (!aborted && !mbar_wait_sleep(&sm.bar_full[stage], parity, kTcWaitLimit))
                sm.abort_flag = 1;
            const int t0 = (int)(gt - u.U0) * TILE;
            int valid = u.L - t0;
            valid = valid > TILE ? TILE : valid;
            const uint8_t* st = sm.ring[stage];
            bool work = !aborted && valid > 0;            // CTA-uniform

            // ---------------- K half-row -> K+ / K- in tensor memory -------------
            if (work) {
                const uint4* kc = reinterpret_cast<const uint4*>(st + t * kKB + 32 * hg);
                const uint32_t sw = *reinterpret_cast<const uint32_t*>(st + OFF_KS + t * kSB + 4 * hg);
                uint32_t kp[16], kn[16];
#pragma unroll
                for (int j = 0; j < 2; ++j) {              // 16 bytes = 32 codes = 2 blocks
                    const uint4 x = kc[j];
                    const uint2 l0 = sm.lut_k[(sw >> (16 * j)) & 0x7F];
                    const uint2 l1 = sm.lut_k[(sw >> (16 * j + 8)) & 0x7F];
                    dequant_split(x.x, l0.x, l0.y, kp[8 * j + 0], kp[8 * j + 1], kn[8 * j + 0], kn[8 * j + 1]);
                    dequant_split(x.y, l0.x, l0.y, kp[8 * j + 2], kp[8 * j + 3], kn[8 * j + 2], kn[8 * j + 3]);
                    dequant_split(x.z, l1.x, l1.y, kp[8 * j + 4], kp[8 * j + 5], kn[8 * j + 4], kn[8 * j + 5]);
                    dequant_split(x.w, l1.x, l1.y, kp[8 * j + 6], kp[8 * j + 7], kn[8 * j + 6], kn[8 * j + 7]);
                }
                tmem_st_x16(trow + C::COL_KP + 16 * hg, kp);
                tmem_st_x16(trow + C::COL_KN + 16 * hg, kn);
                tc::tmem_wait_st();
                tc::fence_before_sync();
            }
            __syncthreads();                                  // (A) K operand complete
            if (sm.abort_flag) {
                if (!aborted && tid == 0) report(p.status, NVFP4_ERR_TIMEOUT);
                aborted = true;
                work = false;
            }
            tc::fence_after_sync();
            if (tid == 0 && work) {
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    tc::mma_e4m3_ts(tbase + C::COL_S, tbase + C::COL_KP + 8 * ks,
                                    tc::smem_desc(qb_addr + ks * 256, 128, 1024), idesc_qk, ks > 0);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    tc::mma_e4m3_ts(tbase + C::COL_S, tbase + C::COL_KN + 8 * ks,
                                    tc::smem_desc(qb_addr + ks * 256, 128, 1024), idesc_qk_neg, true);
                tc::mma_commit(&sm.bar_s);
            }

            if (work) {
                // ---------------- V half-row -> V^T operand (while Q.K^T runs) -------
                bool ok = true;
                const bool live = t < valid;
                if (mma_it > 0)     // the previous P.V must be done reading vt / pb
                    ok = mbar_wait_sleep(&sm.bar_o, (mma_it - 1) & 1u, kTcWaitLimit);
                {
                    const uint4* vc = reinterpret_cast<const uint4*>(st + OFF_VC + t * kKB + 32 * hg);
                    const uint32_t sw = *reinterpret_cast<const uint32_t*>(st + OFF_VS + t * kSB + 4 * hg);
                    uint8_t* dst = sm.vt + (4 * hg) * 2048 + (t / 8) * 128 + (t % 8) * 16;
#pragma unroll
                    for (int j = 0; j < 2; ++j) {          // head_dim 64hg + 32j .. +31
                        const uint4 x = vc[j];
                        uint2 l0 = sm.lut_v[(sw >> (16 * j)) & 0x7F];
                        uint2 l1 = sm.lut_v[(sw >> (16 * j + 8)) & 0x7F];
                        if (!live) {        // bytes past the sequence may hold anything (a NaN
                            l0 = make_uint2(0u, 0u);    // scale): P is 0 there and V must be +-0
                            l1 = l0;
                        }
                        uint4 o0, o1;
                        dequant_word(x.x, l0.x, l0.y, o0.x, o0.y);
                        dequant_word(x.y, l0.x, l0.y, o0.z, o0.w);
                        dequant_word(x.z, l1.x, l1.y, o1.x, o1.y);
                        dequant_word(x.w, l1.x, l1.y, o1.z, o1.w);
                        *reinterpret_cast<uint4*>(dst + (2 * j) * 2048) = o0;
                        *reinterpret_cast<uint4*>(dst + (2 * j + 1) * 2048) = o1;
                    }
                }
                // ---------------- scores -> online softmax -> P terms -----------------
                ok = ok && mbar_wait_sleep(&sm.bar_s, mma_it & 1u, kTcWaitLimit);
                if (!ok) sm.abort_flag = 1;
                tc::fence_after_sync();
                float s[NQH];
                {
                    uint32_t rh[NQH], rl[NQH];
                    tmem_ld_cols<NQH>(trow + C::COL_S + q0, rh);
                    tmem_ld_cols<NQH>(trow + C::COL_S + NQ + q0, rl);
                    tc::tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < NQH; ++i)
                        s[i] = live ? fmaf(__uint_as_float(rl[i]), 0.0625f, __uint_as_float(rh[i])) * cs[i]
                                    : -INFINITY;
                }
                bool need = false;
#pragma unroll
                for (int i = 0; i < NQH; ++i) need |= s[i] > m_run[i] + kRescaleSlack;
                if (__syncthreads_or(need)) {
                    // raise the shared running max to the tile max (per query, over
                    // this warpgroup's 128 tokens), rescale l and O
#pragma unroll
                    for (int i = 0; i < NQH; ++i) {
                        float mx = s[i];
#pragma unroll
                        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
                        if (lane == 0) sm.red[warp][i] = mx;
                    }
                    __syncthreads();
                    float f[NQH];
#pragma unroll
                    for (int i = 0; i < NQH; ++i) {
                        const int w0 = 4 * hg;
                        const float mt = fmaxf(fmaxf(sm.red[w0][i], sm.red[w0 + 1][i]),
                                               fmaxf(sm.red[w0 + 2][i], sm.red[w0 + 3][i]));
                        const float mn = fmaxf(m_run[i], mt);
                        f[i] = (m_run[i] == -INFINITY) ? 0.0f : fast_exp2(m_run[i] - mn);
                        m_run[i] = mn;
                        l_run[i] *= f[i];
                    }
                    if (any_pv) {      // the previous P.V has completed (waited above)
#pragma unroll
                        for (int k = 0; k < NTERM; ++k) {
                            uint32_t r[NQH];
                            tmem_ld_cols<NQH>(trow + C::COL_O + k * NQ + q0, r);
                            tc::tmem_wait_ld();
#pragma unroll
                            for (int i = 0; i < NQH; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * f[i]);
                            tmem_st_cols<NQH>(trow + C::COL_O + k * NQ + q0, r);
                        }
                        tc::tmem_wait_st();
                    }
                }
                {
                    // P terms of this warpgroup's queries: columns n = k * NQ + q0 + i
                    uint32_t tw[NTERM][NQH / 2];     // two bytes (queries i, i+1) per entry
#pragma unroll
                    for (int i = 0; i < NQH; i += 2) {
                        const float p0 = (m_run[i] == -INFINITY) ? 0.0f : fast_exp2(s[i] - m_run[i]);
                        const float p1 = (m_run[i + 1] == -INFINITY) ? 0.0f : fast_exp2(s[i + 1] - m_run[i + 1]);
                        l_run[i] += p0;
                        l_run[i + 1] += p1;
                        uint32_t tt[NTERM];
                        p_terms(p0, p1, tt);
#pragma unroll
                        for (int k = 0; k < NTERM; ++k) tw[k][i / 2] = tt[k];
                    }
                    uint8_t* dst = sm.pb + (t / 8) * 128 + (t % 8) * 16;
#pragma unroll
                    for (int k = 0; k < NTERM; ++k) {
                        const int n = k * NQ + q0;
                        if constexpr (NQH == 4) {
                            *reinterpret_cast<uint32_t*>(dst + (n / 16) * 2048 + (n % 16)) =
                                tw[k][0] | (tw[k][1] << 16);
                        } else {
                            *reinterpret_cast<uint2*>(dst + (n / 16) * 2048 + (n % 16)) =
                                make_uint2(tw[k][0] | (tw[k][1] << 16), tw[k][2] | (tw[k][3] << 16));
                        }
                    }
                }
                fence_proxy_async_smem();
                tc::fence_before_sync();
            }
            __syncthreads();                                  // (B) V^T and P complete, stage read
            if (sm.abort_flag && work) {
                if (!aborted && tid == 0) report(p.status, NVFP4_ERR_TIMEOUT);
                aborted = true;
                work = false;
            }
            tc::fence_after_sync();
            if (tid == 0) {
                if (work) {
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        tc::mma_e4m3_ss(tbase + C::COL_O, tc::smem_desc(vt_addr + ks * 512, 128, 2048),
                                        tc::smem_desc(pb_addr + ks * 512, 128, 2048), idesc_pv,
                                        any_pv || ks > 0);
                    tc::mma_commit(&sm.bar_o);
                }
                // every thread has read this stage's codes and scales: refill it
                if (!prod.done) {
                    fence_proxy_async_smem();
                    issue_tile<128, TILE>(p, prod.u, prod.gt, sm.ring[stage], &sm.bar_full[stage]);
                    ++issued;
                    cursor_next<TILE, 1>(prod, sm.prefix, sm.lens, B, p.Hkv, 0);
                }
            }
            ++consumed;
            if (work) {
                any_pv = true;
                ++mma_it;
            }
        }

        // ---- segment end: O^T row (head_dim d = t) for this warpgroup's queries ----
        float o[NQH];
#pragma unroll
        for (int i = 0; i < NQH; ++i) o[i] = 0.0f;
        if (any_pv && !aborted) {
            const bool ok = mbar_wait_sleep(&sm.bar_o, (mma_it - 1) & 1u, kTcWaitLimit);
            if (!ok) report(p.status, NVFP4_ERR_TIMEOUT);
            tc::fence_after_sync();
            float scale = 1.0f;
#pragma unroll
            for (int k = 0; k < NTERM; ++k) {
                uint32_t r[NQH];
                tmem_ld_cols<NQH>(trow + C::COL_O + k * NQ + q0, r);
                tc::tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < NQH; ++i) o[i] = fmaf(__uint_as_float(r[i]), scale, o[i]);
                scale *= 0.0625f;
            }
        }
        // l over the warpgroup's tokens (per-thread partials; the running max is shared)
#pragma unroll
        for (int i = 0; i < NQH; ++i) {
            float l = l_run[i];
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) l += __shfl_xor_sync(0xFFFFFFFFu, l, off);
            if (lane == 0) sm.red[warp][i] = l;
        }
        __syncthreads();
        float lt[NQH];
#pragma unroll
        for (int i = 0; i < NQH; ++i) {
            const int w0 = 4 * hg;
            lt[i] = (sm.red[w0][i] + sm.red[w0 + 1][i]) + (sm.red[w0 + 2][i] + sm.red[w0 + 3][i]);
        }

        const bool whole = (u.U0 >= t_begin) && (u.U1 <= t_end);
        const int g = p.g;
        const int64_t slot_floats = (int64_t)g * (128 + 2);
        if (whole) {
#pragma unroll
            for (int i = 0; i < NQH; ++i)
                if (q0 + i < g)
                    p.out[((int64_t)u.b * p.Hq + (int64_t)u.h * g + q0 + i) * 128 + t] =
                        (lt[i] > 0.0f) ? o[i] / lt[i] : 0.0f;
        } else {
            float* part = p.partials + partial_slot(c, u.U0, T, N) * slot_floats;
#pragma unroll
            for (int i = 0; i < NQH; ++i)
                if (q0 + i < g) part[(q0 + i) * 128 + t] = o[i];
            if (t == 0) {
#pragma unroll
                for (int i = 0; i < NQH; ++i)
                    if (q0 + i < g) {
                        part[g * 128 + q0 + i] = m_run[i];
                        part[g * 128 + g + q0 + i] = lt[i];
                    }
            }
            __threadfence();
            __syncthreads();
            const int64_t c_first = cta_of(u.U0, T, N);
            const int64_t c_last = cta_of(u.U1 - 1, T, N);
            if (tid == 0) {
                int contributors = 0;
                for (int64_t cc = c_first; cc <= c_last; ++cc)
                    contributors += range_start(cc, T, N) < range_start(cc + 1, T, N);
                const int prev = atomicAdd(&p.counters[(int64_t)u.b * p.Hkv + u.h], 1);
                sm.last_flag = (prev == contributors - 1);
            }
            __syncthreads();
            if (sm.last_flag) {
                __threadfence();
                combine_partials<128, NT, kThreads>(p, sm.comb, u, T, N, c_first, c_last, slot_floats,
                                                    tid, warp, lane);
                if (tid == 0) atomicExch(&p.counters[(int64_t)u.b * p.Hkv + u.h], 0);
            }
        }
        __syncthreads();
        seg_lo = seg_hi;
    }

    // ---- drain copies still in flight, release tensor memory ----
    if (tid == 0) {
        while (consumed < issued) {
            const int stage = (int)(consumed % kStages);
            if (!mbar_wait_sleep(&sm.bar_full[stage], (consumed / kStages) & 1u, kTcWaitLimit)) {
                report(p.status, NVFP4_ERR_TIMEOUT);
                break;
            }
            ++consumed;
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (warp == 0) tc::tmem_dealloc(tbase, C::kTmemCols);
}

template <int NT>
cudaError_t launch_tc(const Params& p, int grid, cudaStream_t stream) {
    auto kern = decode_attention_tc_kernel<NT>;
    const int smem = (int)sizeof(TcSmem<NT>);
    static int configured_device = -1;
    int dev = 0;
    cudaGetDevice(&dev);
    if (configured_device != dev) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        configured_device = dev;
    }
    kern<<<grid, kThreads, smem, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace tcattn

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
    const int sms = device_sm_count();
    if (a.D == 128 && !a.q_f32) {
        // fifth-generation tensor cores: the main path
        return two ? tcattn::launch_tc<2>(p, tcattn::Cfg<2>::kCtasPerSm * sms, stream)
                   : tcattn::launch_tc<1>(p, tcattn::Cfg<1>::kCtasPerSm * sms, stream);
    }
    const int grid = kCtasPerSm * sms;   // warp-MMA kernel: fp32 queries or head_dim 64
    if (a.D == 128) {
        if (!two) return a.q_f32 ? launch_instance<128, 1, true>(p, grid, stream)
                                 : launch_instance<128, 1, false>(p, grid, stream);
        return a.q_f32 ? launch_instance<128, 2, true>(p, grid, stream)
                       : launch_instance<128, 2, false>(p, grid, stream);
    }
    if (!two) return a.q_f32 ? launch_instance<64, 1, true>(p, grid, stream)
                             : launch_instance<64, 1, false>(p, grid, stream);
    return a.q_f32 ? launch_instance<64, 2, true>(p, grid, stream)
                   : launch_instance<64, 2, false>(p, grid, stream);
}

size_t attention_smem_bytes(int D, int NT) {
    if (D == 128) return NT == 1 ? sizeof(Smem<128, 1>) : sizeof(Smem<128, 2>);
    return NT == 1 ? sizeof(Smem<64, 1>) : sizeof(Smem<64, 2>);
}

}  // namespace nvfp4kv

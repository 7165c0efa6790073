// nvfp4kv_decode_attention.cu -- fused NVFP4 -> FP8 decode attention on the
// warp-level MMA path (mma.sync): fp32 queries and head_dim 64.  Head_dim 128
// with bf16 queries goes to the tcgen05 kernel (nvfp4kv_decode_attention_tc.cu);
// launch_decode_attention below picks the kernel.
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

#include "nvfp4kv_attention_common.cuh"

namespace nvfp4kv {

namespace {

using namespace attn;

constexpr int kWarps = 4;
// ring depth per warp: 4 stages, 3 when the GQA group needs two 8-wide tiles
// (keeps two CTAs resident per SM)
template <int NT>
struct Ring { static constexpr int kStages = NT == 1 ? 4 : 3; };
constexpr uint32_t kWaitLimit = 1u << 22;

template <int D>
struct Geometry {
    static constexpr int KB = D / 2;                 // code bytes per token
    static constexpr int SB = D / 16;                // scale bytes per token
    static constexpr int KS = D / 16;                // k-steps of Q.K^T = m-tiles of P.V
    static constexpr int EK = D / 4;                 // K elements per lane per token
    static constexpr int EV = D / 8;                 // V channels per lane
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
    CombineSmem comb;
    int32_t warp_tot[kWarps];
    int32_t last_flag;
};

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
                bool bad;
                L = attended_len(p, b, &bad);
                if (bad && blockIdx.x == 0) report(p.status, NVFP4_ERR_CAPACITY);
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
        const int64_t slot_floats = partial_slot_floats(g, D);
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
            __syncthreads();
            if (tid == 0) {
                const int prev = arrive_split_unit(&p.counters[(int64_t)u.b * p.Hkv + u.h]);
                sm.last_flag = (prev == unit_contributors(u.U0, u.U1, T, N) - 1);
            }
            __syncthreads();
            if (sm.last_flag) {
                combine_partials<D, NT, kWarps * 32>(p, sm.comb, u, T, N, slot_floats, tid, warp, lane);
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
template <int D, int NT, bool QF32>
cudaError_t launch_instance(const Params& p, int grid, cudaStream_t stream) {
    auto kern = decode_attention_kernel<D, NT, QF32>;
    const int smem = (int)sizeof(Smem<D, NT>);
    static int configured[kMaxDevices] = {};
    cudaError_t e0 = ensure_smem_attribute(reinterpret_cast<const void*>(kern), smem, configured);
    if (e0 != cudaSuccess) return e0;
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
    p.block_table = a.block_table;
    p.page_tokens = a.page_tokens;
    p.max_pages = a.max_pages;
    p.num_pages = a.num_pages;
    p.wait_polls = a.wait_polls;
    p.len_from_start = a.start_pos != nullptr ? 1 : 0;
    p.start_pos = a.start_pos;
    p.new_lens = a.new_lens;
    p.x_f32 = a.x_f32 ? 1 : 0;
    p.x_k_new = nullptr;
    p.x_v_new = nullptr;
    const bool two = p.g > 8;
    const int sms = device_sm_count();
    if (a.D == 128 && !a.q_f32) {   // fifth-generation tensor cores: the main path
        p.x_k_new = a.x_k_new;       // the kernel appends the new tokens itself
        p.x_v_new = a.x_v_new;
        return launch_decode_attention_tc(p, sms, stream);
    }
    if (a.x_k_new != nullptr) {      // warp-MMA path: the append runs as its own launch first
        nvfp4_kv_plane pk{}, pv{};
        pk.codes = const_cast<uint8_t*>(a.kc); pk.scales = const_cast<uint8_t*>(a.ks);
        pv.codes = const_cast<uint8_t*>(a.vc); pv.scales = const_cast<uint8_t*>(a.vs);
        pk.B = pv.B = a.B; pk.H_kv = pv.H_kv = a.Hkv; pk.S_max = pv.S_max = a.S_max; pk.D = pv.D = a.D;
        cudaError_t e = launch_quantize_append_kv(a.x_k_new, a.x_v_new, a.x_f32, 1, a.start_pos, a.new_lens,
                                                  a.st_k, a.st_v, pk, pv, a.status, stream);
        if (e != cudaSuccess) return e;
        p.new_lens = nullptr;
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

}  // namespace nvfp4kv

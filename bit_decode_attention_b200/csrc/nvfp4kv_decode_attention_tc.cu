// nvfp4kv_decode_attention_tc.cu -- NVFP4 -> FP8 decode attention on the
// fifth-generation tensor cores (tcgen05), head_dim 128, bf16 queries.
//
// What it computes ("NVIDIA解説: NVFP4 KV Cacheで長コンテキストLLM推論を最適化",
// "量子化・逆量子化フロー"; "TensorRT-LLM rc17 ...", "物語の KV キャッシュ側"):
// the NVFP4 cache is dequantized to FP8 (E4M3) and attention runs on FP8
// tensor-core MMAs with FP32 accumulation,
//     out[b][h] = softmax(q . K^T * scale) . V   over seq_lens[b] tokens.
//
// Work split: the (sequence, KV head, 128-token tile) list is cut into one
// contiguous range per CTA, one CTA per SM (stream-K).  A (sequence, head)
// unit that crosses a range boundary leaves one partial (O, m, l) per CTA in
// the workspace; a second, small kernel (launched as a programmatic dependent
// of this one, so it is resident before this grid ends) merges them.  The
// attention kernel itself therefore has no atomics, counters or merge code.
//
// Inside a CTA every stage of a tile has its own warps, and the stages of
// consecutive tiles overlap; they hand tiles to each other through
// mbarriers, never through CTA-wide barriers:
//
//   load warp   : bulk copies of K/V codes and scale bytes into a 4-stage ring
//   dequant warps 0-3 and 8-11: thread t of group h = token t, head_dim half
//                 h.  K codes -> signed FP8 K in tensor memory lane t (the A
//                 operand of Q.K^T); V codes -> FP8 V^T in shared memory (the
//                 MN-major A operand of P.V)
//   MMA thread  : a fixed schedule, one tile ahead on Q.K^T:
//                   S^T(w+1) = K(w+1) . Q'^T,   then   O^T += V^T(w) . P^T(w)
//                 four MMAs and one commit per product; every wait blocks on
//                 one barrier (no polling of several)
//   softmax 4-7 : thread t reads score row t, online softmax in base 2 with a
//                 lazily raised running max, P as three E4M3 terms
//                 p ~ t0 + t1/16 + t2/256 (MN-major B operand); at the end of
//                 a unit thread d reads O^T row d and writes the output row or
//                 the split-K partial
//
// Four buffers of every kind: tile w uses K/S buffer w % 4 (tensor memory)
// and V^T/P buffer w % 4 (shared memory).  One commit after Q.K^T(w) both
// publishes S(w) and frees K(w); one after P.V(w) publishes O and frees V^T(w)
// and P(w).
//
// The query operand Q' holds, per query row, an exact two-term E4M3 split of
// the bf16 query scaled by a power of two: q * 2^e = hi + lo / 16, so the
// scores are exact sums of FP8 products (up to fp32 accumulation order).
#include <cuda_bf16.h>

#include "nvfp4kv_attention_common.cuh"
#include "nvfp4kv_pipeline.cuh"
#include "nvfp4kv_tcgen05.cuh"

namespace nvfp4kv {

namespace {

using namespace attn;

constexpr int TILE = 128;                             // tokens per tile = MMA M
constexpr int kKB = 64, kSB = 8;                      // code / scale bytes per token
constexpr int STAGE = TILE * (2 * kKB + 2 * kSB);     // 18432
constexpr int OFF_VC = TILE * kKB;
constexpr int OFF_KS = 2 * TILE * kKB;
constexpr int OFF_VS = 2 * TILE * kKB + TILE * kSB;
constexpr int kStages = 4;                            // bulk-copy ring
constexpr int kBuf = 4;                               // K/S and V^T/P operand buffers
constexpr int NTERM = 3;                              // E4M3 terms of P

// Hand-offs: every thread that produced (or last read) what a barrier
// guards fences and arrives on it itself (arrival counts of 128 per group):
// a per-warp arrival after __syncwarp let the tensor core and the bulk copies
// race with the other lanes' accesses in the prefill kernel built the same way.
//
// warp roles, in warpgroups of four (warp w reaches tensor-memory lanes
// 32 * (w % 4) .. +31, so every group covers the 128 token lanes):
//   warps  0- 3, 8-11, 12-15, 16-19  dequant groups 0..3: group i takes the
//                tiles w = i (mod 4), K and V of one token per thread; it owns
//                ring stage i and operand buffer i
//   warps  4- 7  softmax group 0 (queries 0 .. NQ/2-1)
//   warps 20-23  softmax group 1 (NQ/2 .. NQ-1)
//   warp 24 loads, 25 Q.K^T MMAs, 26 P.V MMAs, 27 the fused append's new tokens
constexpr int kS0Warp0 = 4;
constexpr int kS1Warp0 = 20;
static_assert(kStages == 4 && kBuf == 4, "one ring stage and one operand buffer per dequant group");
constexpr int kLoadWarp = 24;
constexpr int kMmaWarp = 25;                          // Q.K^T
constexpr int kPvWarp = 26;                           // P.V
constexpr int kAppendWarp = 27;                       // new tokens of the fused append
constexpr int kThreads = 28 * 32;
// registers per thread after the prologue (setmaxnreg); the launch holds
// kThreads x 72, and 128 x (2 x 112 + 4 x 56 + 56) = 64,512 of them
constexpr uint32_t kRegsSoftmax = 112, kRegsDequant = 56, kRegsMisc = 56;

constexpr uint32_t kWaitPolls = 1u << 16;             // sleeping polls (<= 20 us each) per wait

template <int NT>
struct Cfg {
    static constexpr int NQ = 8 * NT;                 // query rows (padded GQA group)
    static constexpr int NS = 2 * NQ;                 // score columns: hi, lo
    static constexpr int NP = (NTERM * NQ + 15) / 16 * 16;   // P columns (MMA N), term-major
    static constexpr uint32_t COL_K = 0;              // kBuf buffers x 32 columns (4 FP8 each)
    static constexpr uint32_t COL_S = 32 * kBuf;      // kBuf buffers x NS
    static constexpr uint32_t COL_O = COL_S + kBuf * NS;   // NP
    static constexpr uint32_t kTmemCols = COL_O + NP <= 128 ? 128 : (COL_O + NP <= 256 ? 256 : 512);
    static_assert(COL_O + NP <= kTmemCols, "tensor memory columns");
};

// lookup tables: [plane][scale byte & 0x7F][copy]; lane l reads copy l % 16, so
// the 16 lanes of a half-warp always hit 16 different bank pairs
constexpr int kLutCopies = 16;

template <int NT>
struct __align__(1024) Smem {
    using C = Cfg<NT>;
    uint8_t ring[kStages][STAGE];
    uint8_t vt[kBuf][128 * TILE];                     // V^T: (d/16)*2048 + (t/8)*128 + (t%8)*16 + d%16
    uint8_t pb[kBuf][C::NP * TILE];                   // P^T: (n/16)*2048 + (t/8)*128 + (t%8)*16 + n%16
    uint8_t qb[2][C::NS * 128];                       // Q':  (n/8)*1024 + (d/16)*128 + (n%8)*16 + d%16
    uint2 lut[2][128][kLutCopies];
    uint64_t full[kStages], empty[kStages];
    uint64_t kfull[kBuf], qkdone[kBuf], sempty[kBuf];
    uint64_t vfull[kBuf], pfull[kBuf], pvdone[kBuf];
    uint64_t qfull[2];
    uint64_t mma_done;
    uint64_t appended;                                // the fused append's new tokens are written
    int32_t lens[kMaxBatchPerLaunch];
    int32_t prefix[kMaxBatchPerLaunch + 1];
    float cscale[2][C::NQ];
    alignas(16) uint8_t qraw[2][128][16];             // next unit's query loads, per softmax thread
    float red[4][C::NQ];
    int32_t warp_tot[kThreads / 32];
    int32_t warp_empty[kThreads / 32];
    uint32_t tmem_base;
    int32_t abort_flag;
};

// ---------------------------------------------------------------------------
// small helpers
// ---------------------------------------------------------------------------

// A wait of a 128-thread group: one warp polls the barrier while the other
// three wait on the group's named barrier without issuing, which then hands
// every thread the outcome (an AND over the group).
__device__ __forceinline__ bool group_wait(uint64_t* bar, uint32_t parity, bool poller, int bar_id,
                                           int32_t* abort_flag, int32_t* status, uint32_t polls) {
    const bool ok = poller ? wait_warp(bar, parity, abort_flag, status, polls) : true;
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred pi, po;\n\tsetp.ne.u32 pi, %1, 0;\n\t"
        "bar.red.and.pred po, %2, 128, pi;\n\tselp.u32 %0, 1, 0, po;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)ok), "r"(bar_id)
        : "memory");
    return r != 0;
}

// the softmax warps' named barrier, plain and as an OR-reduction
// (named barrier 1 + group, 128 threads each)
__device__ __forceinline__ void softmax_sync(int bar_id) {
    asm volatile("bar.sync %0, 128;" ::"r"(bar_id) : "memory");
}
__device__ __forceinline__ bool softmax_any(bool v, int bar_id) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred pi, po;\n\tsetp.ne.u32 pi, %1, 0;\n\t"
        "bar.red.or.pred po, %2, 128, pi;\n\tselp.u32 %0, 1, 0, po;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v), "r"(bar_id)
        : "memory");
    return r != 0;
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
// N consecutive 32-bit columns of this thread's lane (N = 8, 16, 32)
template <int N>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t* r) {
    if constexpr (N == 4) {
        tc::tmem_ld_x4(taddr, r);
    } else if constexpr (N == 8) {
        tc::tmem_ld_x8(taddr, r);
    } else if constexpr (N == 16) {
        tc::tmem_ld_x16(taddr, r);
    } else {
        static_assert(N == 32, "columns");
        tc::tmem_ld_x16(taddr, r);
        tc::tmem_ld_x16(taddr + 16, r + 16);
    }
}
template <int N>
__device__ __forceinline__ void tmem_st_cols(uint32_t taddr, const uint32_t* r) {
    if constexpr (N == 4) {
        tc::tmem_st_x4(taddr, r);
    } else if constexpr (N == 8) {
        tc::tmem_st_x8(taddr, r);
    } else {
        static_assert(N == 16, "columns");
        tc::tmem_st_x8(taddr, r);
        tc::tmem_st_x8(taddr + 8, r + 8);
    }
}

// Registers per thread of this warpgroup (all four warps execute it).
template <uint32_t N>
__device__ __forceinline__ void regs_inc() {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <uint32_t N>
__device__ __forceinline__ void regs_dec() {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}

// Allow the dependent grid (the split-K merge) to be scheduled.
__device__ __forceinline__ void launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
// Wait until the grids this one depends on have completed and their memory
// operations are visible.
__device__ __forceinline__ void wait_prerequisites() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

// Three E4M3 terms of two non-negative weights (two bytes each, lo weight in
// the low byte): p ~ t0 + t1/16 + t2/256, relative error <= 2^-12.
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

// ---------------------------------------------------------------------------
// Query operand of unit (b, h), built by the 128 softmax threads: per query
// row q (padded to NQ rows; rows past the group are zero) the exact split
// q * 2^e = hi + lo / 16 into two E4M3 rows (n = q and n = NQ + q) of the
// K-major B operand, with max |q * 2^e| < 256; cscale[q] = scale * log2(e) *
// 2^-e turns the MMA result into a base-2 score.
// ---------------------------------------------------------------------------
template <int NT>
struct QRaw {
    static constexpr int PER = Cfg<NT>::NQ / 2;       // bf16 elements per thread: 4 or 8
    uint32_t w[PER / 2];
};

// Query rows q0 .. q0 + NQ/2 - 1 of unit (b, h), by the 128 threads of one
// softmax group: thread t holds row q0 + t / TPQ, head_dim d0 .. d0 + PER - 1.
template <int NT>
__device__ __forceinline__ void fetch_q(const Params& p, int b, int h, int q0, int t, QRaw<NT>& raw) {
    constexpr int PER = QRaw<NT>::PER;
    constexpr int TPQ = 128 / PER;                    // threads per query row
    const int q = q0 + t / TPQ;
    const int d0 = (t % TPQ) * PER;
    const bool valid = q < p.g;
    const int64_t row = ((int64_t)b * p.Hq + (int64_t)h * p.g + (valid ? q : 0)) * 128 + d0;
    const uint16_t* src = reinterpret_cast<const uint16_t*>(p.q) + row;
    if constexpr (PER == 8) {
        const uint4 v = valid ? __ldg(reinterpret_cast<const uint4*>(src)) : make_uint4(0, 0, 0, 0);
        raw.w[0] = v.x; raw.w[1] = v.y; raw.w[2] = v.z; raw.w[3] = v.w;
    } else {
        const uint2 v = valid ? __ldg(reinterpret_cast<const uint2*>(src)) : make_uint2(0, 0);
        raw.w[0] = v.x; raw.w[1] = v.y;
    }
}

// The same loads as fetch_q, but asynchronous into this thread's 16-byte slot
// of shared memory (rows past the group are zero-filled), so that no register
// holds them while the segment runs; take_q waits for them and reads them.
template <int NT>
__device__ __forceinline__ void fetch_q_async(const Params& p, int b, int h, int q0, int t, uint8_t* slot) {
    constexpr int PER = QRaw<NT>::PER;
    constexpr int TPQ = 128 / PER;
    const int q = q0 + t / TPQ;
    const int d0 = (t % TPQ) * PER;
    const bool valid = q < p.g;
    const int64_t row = ((int64_t)b * p.Hq + (int64_t)h * p.g + (valid ? q : 0)) * 128 + d0;
    const uint16_t* src = reinterpret_cast<const uint16_t*>(p.q) + row;
    asm volatile("cp.async.ca.shared.global [%0], [%1], %2, %3;\n\tcp.async.commit_group;" ::"r"(smem_u32(slot)),
                 "l"(src), "n"(PER * 2), "r"(valid ? PER * 2 : 0)
                 : "memory");
}
template <int NT>
__device__ __forceinline__ void take_q(const uint8_t* slot, QRaw<NT>& raw) {
    asm volatile("cp.async.wait_all;" ::: "memory");
#pragma unroll
    for (int k = 0; k < QRaw<NT>::PER / 2; ++k) raw.w[k] = reinterpret_cast<const uint32_t*>(slot)[k];
}

template <int NT>
__device__ __forceinline__ void build_q(const Params& p, uint8_t* qb, float* cscale, const QRaw<NT>& raw,
                                        int q0, int t) {
    using C = Cfg<NT>;
    constexpr int PER = QRaw<NT>::PER;
    constexpr int TPQ = 128 / PER;
    const int q = q0 + t / TPQ;
    const int d0 = (t % TPQ) * PER;
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
    for (int o = 1; o < TPQ && o < 32; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
    int e = 0;
    if (amax > 0.0f && amax <= 3.4028234663852886e38f) {
        int ex;
        frexpf(amax, &ex);                            // amax < 2^ex
        e = 8 - ex;                                   // max |q'| < 256
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
    // K-major rows n = q (hi) and n = NQ + q (lo); d0 is a multiple of 4
    const int nh = q, nl = C::NQ + q;
#pragma unroll
    for (int c = 0; c < PER / 4; ++c) {
        const int d = d0 + 4 * c;
        *reinterpret_cast<uint32_t*>(qb + (nh / 8) * 1024 + (d / 16) * 128 + (nh % 8) * 16 + d % 16) = hw[c];
        *reinterpret_cast<uint32_t*>(qb + (nl / 8) * 1024 + (d / 16) * 128 + (nl % 8) * 16 + d % 16) = lw[c];
    }
    if (t % TPQ == 0) cscale[q] = p.softmax_scale * kLog2e * __uint_as_float(pow2_bits(-e));
}

// Valid tokens of global tile gt of unit u (<= 0 for the empty tile of a
// zero-length sequence).
__device__ __forceinline__ int tile_valid(const Unit& u, int64_t gt) {
    const int t0 = (int)(gt - u.U0) * TILE;
    const int v = u.L - t0;
    return v > TILE ? TILE : v;
}

// Walk over the tiles with work (valid > 0) of a CTA range, in order.  The
// segment ordinal counts every segment (unit) of the range, empty ones too.
struct TileWalker {
    int64_t seg_hi, gt, t_end;
    Unit u;
    int64_t last;                                     // the tile returned by next()
    int32_t j;                                        // its segment ordinal
    bool first;                                       // first tile with work of its segment
    bool fresh;

    __device__ __forceinline__ void start(int64_t t_begin, int64_t t_end_) {
        seg_hi = gt = t_begin;
        t_end = t_end_;
        j = -1;
        fresh = true;
    }
    // advance to the next tile with work; false at the end of the range
    __device__ __forceinline__ bool next(const int32_t* prefix, const int32_t* lens, int B, int Hkv) {
        for (;;) {
            if (gt < seg_hi) {
                const int64_t cur = gt++;
                if (tile_valid(u, cur) > 0) {
                    last = cur;
                    first = fresh;
                    fresh = false;
                    return true;
                }
                continue;
            }
            if (seg_hi >= t_end) return false;
            const int64_t seg_lo = seg_hi;
            u = find_unit<TILE>(prefix, lens, B, Hkv, seg_lo);
            seg_hi = u.U1 < t_end ? u.U1 : t_end;
            gt = seg_lo;
            ++j;
            fresh = true;
        }
    }
};

// ---------------------------------------------------------------------------
// Fused append (a2-a4 for one token), by one warp: every unit whose last tile
// lies in [t_begin, t_end) gets its new token -- K and V, 8 blocks each, one
// lane per block (half-warp h of the warp takes every second such unit; lanes
// 0-7 of a half K, 8-15 V) -- quantized with the same block quantizer as
// nvfp4_kv_quantize_append and written at slot start_pos[b].  A sequence whose
// slot is out of range is skipped (the prologue reported it); a non-finite or
// non-positive tensor scale skips everything with NVFP4_ERR_NONFINITE.  Every
// writer then orders its global stores before later async-proxy reads (the
// load warp's bulk copies, after the caller's barrier arrive).
// ---------------------------------------------------------------------------
__device__ __forceinline__ void append_new_tokens(const Params& p, const int32_t* prefix, const int32_t* lens,
                                                  int B, int64_t t_begin, int64_t t_end, float st_k,
                                                  float st_v, int lane) {
    const bool ok_k = st_k > 0.0f && st_k <= 3.4028234663852886e38f;
    const bool ok_v = st_v > 0.0f && st_v <= 3.4028234663852886e38f;
    if (!(ok_k && ok_v) && lane == 0) report(p.status, NVFP4_ERR_NONFINITE);
    const int half = lane >> 4;
    const bool is_v = (lane & 15) >= 8;
    const int blk = lane & 7;
    int ui = 0;
    for (int64_t seg_lo = t_begin; seg_lo < t_end;) {
        const Unit u = find_unit<TILE>(prefix, lens, B, p.Hkv, seg_lo);
        if (u.U1 <= t_end) {
            if ((ui & 1) == half) {
                const int start = p.start_pos[u.b];
                const bool in_range = start >= 0 && start + 1 <= p.S_max;
                if (in_range && (is_v ? ok_v : ok_k)) {
                    float v[16];
                    const int64_t elem = ((int64_t)u.b * p.Hkv + u.h) * 128 + 16 * blk;
                    if (p.x_f32) load16<true>(is_v ? p.x_v_new : p.x_k_new, elem, v);
                    else load16<false>(is_v ? p.x_v_new : p.x_k_new, elem, v);
                    uint2 packed;
                    const uint32_t sb = quantize_block(v, is_v ? st_v : st_k, packed);
                    const int64_t slot = ((int64_t)u.b * p.Hkv + u.h) * p.S_max + start;
                    uint8_t* codes = const_cast<uint8_t*>(is_v ? p.vc : p.kc);
                    uint8_t* scales = const_cast<uint8_t*>(is_v ? p.vs : p.ks);
                    *reinterpret_cast<uint2*>(codes + slot * 64 + 8 * blk) = packed;
                    scales[slot * 8 + blk] = (uint8_t)sb;
                    if (!is_v && blk == 0 && u.h == 0 && p.new_lens != nullptr) p.new_lens[u.b] = start + 1;
                }
            }
            ++ui;
        }
        seg_lo = u.U1 < t_end ? u.U1 : t_end;
    }
    asm volatile("fence.proxy.async.global;" ::: "memory");
}

// ---------------------------------------------------------------------------
// the attention kernel
// ---------------------------------------------------------------------------
template <int NT>
__global__ void __launch_bounds__(kThreads, 1) decode_attention_tc_kernel(const Params p) {
    using C = Cfg<NT>;
    constexpr int NQ = C::NQ;
    constexpr int NS = C::NS;
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte aligned view; pointer arithmetic on the __shared__ array (not
    // an integer round trip) keeps every access a shared-memory instruction
    Smem<NT>& sm = *reinterpret_cast<Smem<NT>*>(smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u));
    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int B = p.B;
    const uint32_t polls = p.wait_polls;
    const float st_k = __ldg(p.st_k);                 // loads in flight during the prefix scan
    const float st_v = __ldg(p.st_v);

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
                bool bad;
                L = attended_len(p, b, &bad);
                if (bad && blockIdx.x == 0) report(p.status, NVFP4_ERR_CAPACITY);
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
    {
        // every tile of a unit has work except the single tile of an empty
        // sequence's unit: count those inside this CTA's range
        constexpr int per = (kMaxBatchPerLaunch + kThreads - 1) / kThreads;
        int empty = 0;
#pragma unroll
        for (int i = 0; i < per; ++i) {
            const int b = tid * per + i;
            if (b < B && sm.lens[b] == 0) {
                const int64_t lo = sm.prefix[b] > t_begin ? sm.prefix[b] : t_begin;
                const int64_t hi = (int64_t)sm.prefix[b] + p.Hkv < t_end ? (int64_t)sm.prefix[b] + p.Hkv : t_end;
                empty += hi > lo ? (int)(hi - lo) : 0;
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) empty += __shfl_xor_sync(0xFFFFFFFFu, empty, o);
        if (lane == 0) sm.warp_empty[warp] = empty;
    }

    // softmax groups with real queries: the second group (queries NQ/2 ..)
    // has none when the GQA group fits the first one's
    const int n_sgrp = p.g > NQ / 2 ? 2 : 1;

    // ---- tensor memory, barriers, lookup tables, zeroed P buffers ----
    if (warp == kMmaWarp) {
        tc::tmem_alloc(&sm.tmem_base, C::kTmemCols);
        tc::tmem_relinquish();
    }
    // the load warp sets up every barrier and starts the first copies at once
    TileWalker load_walk;
    load_walk.start(t_begin, t_end);
    uint32_t load_w = 0;
    bool load_pending = false;                        // the walker's current tile is not issued yet
    if (warp == kLoadWarp && lane == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], 128);
        }
        for (int b = 0; b < kBuf; ++b) {
            mbar_init(&sm.kfull[b], 128);
            mbar_init(&sm.qkdone[b], 1);
            mbar_init(&sm.sempty[b], 128 * n_sgrp);
            mbar_init(&sm.vfull[b], 128);
            mbar_init(&sm.pfull[b], 128 * n_sgrp);
            mbar_init(&sm.pvdone[b], 1);
        }
        mbar_init(&sm.qfull[0], 4 * n_sgrp);
        mbar_init(&sm.qfull[1], 4 * n_sgrp);
        mbar_init(&sm.mma_done, 2);                   // both MMA warps commit
        mbar_init(&sm.appended, 32);                  // every lane of the append warp
        fence_mbar_init();
        sm.abort_flag = 0;
        // the first two tiles only: the CTA barrier below waits for this lane;
        // in the fused append mode a unit's last tile (it holds the new token)
        // waits for the append warp
        while (load_w < 2u && load_walk.next(sm.prefix, sm.lens, B, p.Hkv)) {
            if (p.x_k_new != nullptr && load_walk.last == load_walk.u.U1 - 1) {
                load_pending = true;
                break;
            }
            issue_tile<128, TILE>(p, load_walk.u, load_walk.last, sm.ring[load_w], &sm.full[load_w]);
            ++load_w;
        }
    }
    QRaw<NT> q_first;                                 // query loads in flight during the table build
    const int wg = warp >> 2;                          // warpgroup
    const bool is_softmax = wg == kS0Warp0 / 4 || wg == kS1Warp0 / 4;
    const int sgrp = wg == kS1Warp0 / 4 ? 1 : 0;       // softmax group
    if (is_softmax && sgrp < n_sgrp) {
        const Unit u0 = find_unit<TILE>(sm.prefix, sm.lens, B, p.Hkv, t_begin);
        fetch_q<NT>(p, u0.b, u0.h, sgrp * (NQ / 2), 32 * (warp & 3) + lane, q_first);
    }
    if (tid < 256) {
        const int plane = tid >> 7;
        const uint2 w = lut_words((uint32_t)(tid & 127), plane ? st_v : st_k);
#pragma unroll
        for (int cp = 0; cp < kLutCopies; ++cp) sm.lut[plane][tid & 127][cp] = w;
    }
    {
        uint4* pz = reinterpret_cast<uint4*>(&sm.pb[0][0]);
        for (int i = tid; i < (int)(sizeof(sm.pb) / 16); i += kThreads) pz[i] = make_uint4(0, 0, 0, 0);
    }
    if (tid == 0 && blockIdx.x == 0) {
        const bool ok = st_k > 0.f && st_k <= 3.4028234663852886e38f && st_v > 0.f &&
                        st_v <= 3.4028234663852886e38f;
        if (!ok) report(p.status, NVFP4_ERR_NONFINITE);
    }
    fence_proxy_async_smem();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tbase = sm.tmem_base;
    int32_t* const abort_flag = &sm.abort_flag;
    launch_dependents();                              // the merge grid may be scheduled now
    int n_work = (int)(t_end - t_begin);              // tiles with work in this CTA's range
#pragma unroll
    for (int i = 0; i < kThreads / 32; ++i) n_work -= sm.warp_empty[i];

    // each role sets its warpgroup's register count first (setmaxnreg); the
    // loader's and the MMA warp's group also holds the two idle warps
    if (wg == kLoadWarp / 4) {
        regs_dec<kRegsMisc>();
    }
    if (warp == kLoadWarp) {
        // ================= bulk copies into the ring =================
        if (lane == 0) {
            uint32_t w = load_w;                       // the first stages went out in the prologue
            bool appended = p.x_k_new == nullptr;
            while (load_pending || load_walk.next(sm.prefix, sm.lens, B, p.Hkv)) {
                load_pending = false;
                const int s = (int)(w % kStages);
                if (w >= (uint32_t)kStages &&
                    !wait_one(&sm.empty[s], ((w / kStages) - 1) & 1u, abort_flag, p.status, polls))
                    break;
                if (!appended && load_walk.last == load_walk.u.U1 - 1) {
                    if (!wait_one(&sm.appended, 0, abort_flag, p.status, polls)) break;
                    appended = true;
                }
                issue_tile<128, TILE>(p, load_walk.u, load_walk.last, sm.ring[s], &sm.full[s]);
                ++w;
            }
            // every issued copy must land before the CTA exits
            const uint32_t first = w > (uint32_t)kStages ? w - kStages : 0u;
            for (uint32_t i = first; i < w; ++i) {
                if (!mbar_wait_sleep(&sm.full[i % kStages], (i / kStages) & 1u, kWaitPolls)) {
                    report(p.status, NVFP4_ERR_TIMEOUT);
                    break;
                }
            }
        }
    } else if (warp == kMmaWarp || warp == kPvWarp) {
        // ================= tensor-core MMAs =================
        // Two issuing warps, so that neither product waits behind the other:
        // warp kMmaWarp issues Q.K^T as soon as a tile's K is in tensor
        // memory, warp kPvWarp issues P.V as soon as its P and V^T are in
        // shared memory (a commit tracks the issuing thread's own MMAs).  The
        // whole warp runs the schedule and its waits (every value stays
        // warp-uniform); one elected lane issues each group of four MMAs
        // together with its commit.
        TileWalker walk;
        walk.start(t_begin, t_end);
        bool ok = true;
        if (warp == kMmaWarp) {
            const uint32_t idesc_qk = tc::idesc_e4m3(128, NS, false, false, false);
            // descriptor of buffer 0; buffer and k-step add to the start-address
            // field (16-byte units, no carry out of its 14 bits)
            const uint64_t qdesc0 = tc::smem_desc(tc::smem_addr(sm.qb[0]), 128, 1024);
            constexpr uint64_t kQStep = (C::NS * 128) >> 4;
            int32_t q_seg = -1;                        // segment whose query operand is in place
            // Q.K^T of tile w: S(b) = K(b) . Q'^T, then commit to qkdone[b]
            for (uint32_t w = 0; ok && walk.next(sm.prefix, sm.lens, B, p.Hkv); ++w) {
                const int32_t jq = walk.j;
                const int b = (int)(w % kBuf);
                const uint32_t ph = (w / kBuf) & 1u;
                if (q_seg != jq) {
                    ok = wait_warp(&sm.qfull[jq & 1], ((uint32_t)jq >> 1) & 1u, abort_flag, p.status, polls);
                    q_seg = jq;
                }
                ok = ok && wait_warp(&sm.kfull[b], ph, abort_flag, p.status, polls);
                ok = ok && (w < (uint32_t)kBuf || wait_warp(&sm.sempty[b], ph ^ 1u, abort_flag, p.status, polls));
                if (!ok) break;
                tc::fence_after_sync();
                const uint64_t qd = qdesc0 + (uint64_t)(jq & 1) * kQStep;
                const uint64_t bq[4] = {qd, qd + 16, qd + 32, qd + 48};
                if (tc::elect_one())
                    tc::mma4_ts_commit(tbase + C::COL_S + NS * b, tbase + C::COL_K + 32 * b, bq, idesc_qk, 0u,
                                       &sm.qkdone[b]);
                __syncwarp();
            }
        } else {
            const uint32_t idesc_pv = tc::idesc_e4m3(128, C::NP, true, true, false);
            const uint64_t vdesc0 = tc::smem_desc(tc::smem_addr(sm.vt[0]), 128, 2048);
            const uint64_t pdesc0 = tc::smem_desc(tc::smem_addr(sm.pb[0]), 128, 2048);
            constexpr uint64_t kVStep = (128 * TILE) >> 4, kPStep = (C::NP * TILE) >> 4;
            // P.V of tile w: O += V^T(b) . P^T(b), then commit to pvdone[b]; O
            // restarts with the first tile of each unit
            for (uint32_t w = 0; ok && walk.next(sm.prefix, sm.lens, B, p.Hkv); ++w) {
                const int b = (int)(w % kBuf);
                const uint32_t ph = (w / kBuf) & 1u;
                ok = wait_warp(&sm.pfull[b], ph, abort_flag, p.status, polls) &&
                     wait_warp(&sm.vfull[b], ph, abort_flag, p.status, polls);
                if (!ok) break;
                tc::fence_after_sync();
                const uint64_t vd = vdesc0 + (uint64_t)b * kVStep;
                const uint64_t pd = pdesc0 + (uint64_t)b * kPStep;
                const uint64_t av[4] = {vd, vd + 32, vd + 64, vd + 96};
                const uint64_t bp[4] = {pd, pd + 32, pd + 64, pd + 96};
                if (tc::elect_one())
                    tc::mma4_ss_commit(tbase + C::COL_O, av, bp, idesc_pv, walk.first ? 0u : 1u, &sm.pvdone[b]);
                __syncwarp();
            }
        }
        // every issued MMA must complete before tensor memory is released
        if (tc::elect_one()) tc::mma_commit(&sm.mma_done);
        __syncwarp();
        if (!mbar_wait_sleep(&sm.mma_done, 0, kWaitPolls)) report(p.status, NVFP4_ERR_TIMEOUT);
        __syncwarp();
    } else if (warp == kAppendWarp) {
        // ================= the fused append's new tokens =================
        if (p.x_k_new != nullptr) {
            append_new_tokens(p, sm.prefix, sm.lens, B, t_begin, t_end, st_k, st_v, lane);
            mbar_arrive(&sm.appended);                 // after this lane's async-proxy fence
        }
    } else if (!is_softmax) {
        // ======== dequant group i: tiles w = i (mod 4), K and V of token t ========
        // A group has four tile periods for each of its tiles, so the latency
        // of its loads, tensor-memory stores and barriers is spread over four
        // tiles in flight.  K goes first (its Q.K^T runs ahead of P.V); the
        // ring stage is released once V's raw data is in registers.
        regs_dec<kRegsDequant>();
        const int i = wg == 0 ? 0 : wg - 1;                // wg 0, 2, 3, 4 -> 0, 1, 2, 3
        const int t = 32 * (warp & 3) + lane;              // token, tensor-memory lane
        const uint32_t trow = tbase + ((uint32_t)(32 * (warp & 3)) << 16);
        const uint2* lut_k = &sm.lut[0][0][lane & (kLutCopies - 1)];
        const uint2* lut_v = &sm.lut[1][0][lane & (kLutCopies - 1)];
        const uint8_t* st = sm.ring[i];
        uint8_t* const vdst = sm.vt[i] + (t / 8) * 128 + (t % 8) * 16;
        const bool poller = (warp & 3) == 0;
        const int gbar = 3 + i;                            // named barriers 3..6
        for (int w = i; w < n_work; w += 4) {
            const uint32_t ph = ((uint32_t)w >> 2) & 1u;
            if (!group_wait(&sm.full[i], ph, poller, gbar, abort_flag, p.status, polls)) break;
            // Q.K^T of tile w - 4 has read this K buffer
            if (w >= 4 && !group_wait(&sm.qkdone[i], ph ^ 1u, poller, gbar, abort_flag, p.status, polls)) break;
            const uint2 sk = *reinterpret_cast<const uint2*>(st + OFF_KS + t * kSB);
            uint4 kc[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) kc[j] = *reinterpret_cast<const uint4*>(st + t * kKB + 16 * j);
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {               // head_dim 64hh .. 64hh + 63
                const uint32_t sc = hh ? sk.y : sk.x;
                uint2 l[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) l[k] = lut_k[((sc >> (8 * k)) & 0x7F) * kLutCopies];
                const uint4 c0 = kc[2 * hh], c1 = kc[2 * hh + 1];
                uint32_t kf[16];                           // 64 codes -> 16 columns (4 FP8 each)
                dequant_word(c0.x, l[0].x, l[0].y, kf[0], kf[1]);
                dequant_word(c0.y, l[0].x, l[0].y, kf[2], kf[3]);
                dequant_word(c0.z, l[1].x, l[1].y, kf[4], kf[5]);
                dequant_word(c0.w, l[1].x, l[1].y, kf[6], kf[7]);
                dequant_word(c1.x, l[2].x, l[2].y, kf[8], kf[9]);
                dequant_word(c1.y, l[2].x, l[2].y, kf[10], kf[11]);
                dequant_word(c1.z, l[3].x, l[3].y, kf[12], kf[13]);
                dequant_word(c1.w, l[3].x, l[3].y, kf[14], kf[15]);
                tmem_st_x16(trow + C::COL_K + 32 * i + 16 * hh, kf);
            }
            const uint2 sv = *reinterpret_cast<const uint2*>(st + OFF_VS + t * kSB);
            uint4 vc[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) vc[j] = *reinterpret_cast<const uint4*>(st + OFF_VC + t * kKB + 16 * j);
            tc::tmem_wait_st();
            tc::fence_before_sync();
            mbar_arrive(&sm.kfull[i]);                     // Q.K^T of tile w may start
            fence_proxy_async_smem();                      // these ring reads come before the refill
            mbar_arrive(&sm.empty[i]);                     // the loader may refill stage i
            // P.V of tile w - 4 has read this V^T buffer
            if (w >= 4 && !group_wait(&sm.pvdone[i], ph ^ 1u, poller, gbar, abort_flag, p.status, polls)) break;
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const uint32_t sc = hh ? sv.y : sv.x;
                uint2 l[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) l[k] = lut_v[((sc >> (8 * k)) & 0x7F) * kLutCopies];
#pragma unroll
                for (int j = 0; j < 2; ++j) {              // 32 codes -> 2 rows of 16 head_dim bytes of V^T
                    const uint4 c = vc[2 * hh + j];
                    uint4 o0, o1;
                    dequant_word(c.x, l[2 * j].x, l[2 * j].y, o0.x, o0.y);
                    dequant_word(c.y, l[2 * j].x, l[2 * j].y, o0.z, o0.w);
                    dequant_word(c.z, l[2 * j + 1].x, l[2 * j + 1].y, o1.x, o1.y);
                    dequant_word(c.w, l[2 * j + 1].x, l[2 * j + 1].y, o1.z, o1.w);
                    *reinterpret_cast<uint4*>(vdst + (4 * hh + 2 * j) * 2048) = o0;
                    *reinterpret_cast<uint4*>(vdst + (4 * hh + 2 * j + 1) * 2048) = o1;
                }
            }
            fence_proxy_async_smem();
            mbar_arrive(&sm.vfull[i]);                     // P.V of tile w may start
        }
    } else if (is_softmax && sgrp >= n_sgrp) {
        // a group with padding queries only: nothing to do (its P columns stay
        // the zeros of the prologue)
        regs_inc<kRegsSoftmax>();
    } else if (is_softmax) {
        // ============ softmax, P, output: group sgrp owns queries q0 .. q0 + NH - 1 ============
        regs_inc<kRegsSoftmax>();
        constexpr int NH = NQ / 2;
        const int q0 = sgrp * NH;
        const int bar_id = 1 + sgrp;
        const int sw = warp & 3;                           // lane quadrant
        const int t = 32 * sw + lane;                      // token of the score row; head_dim of O
        const uint32_t trow = tbase + ((uint32_t)(32 * sw) << 16);
        bool aborted = false;
        uint32_t w = 0;
        uint32_t j = 0;
        {   // query operand of the first unit (loads issued in the prologue)
            build_q<NT>(p, sm.qb[0], sm.cscale[0], q_first, q0, t);
            fence_proxy_async_smem();
            softmax_sync(bar_id);
            if (lane == 0) mbar_arrive(&sm.qfull[0]);
        }
        // Each unit's query operand is built when the unit BEFORE it starts, so
        // that Q.K^T of a unit's first tile never waits for the softmax of the
        // previous unit's last tile (the pipeline does not drain at a unit
        // boundary); its loads are issued one unit earlier still.
        uint8_t* const qslot = sm.qraw[sgrp][t];
        {
            const Unit u0 = find_unit<TILE>(sm.prefix, sm.lens, B, p.Hkv, t_begin);
            if (u0.U1 < t_end) {
                const Unit u1 = find_unit<TILE>(sm.prefix, sm.lens, B, p.Hkv, u0.U1);
                fetch_q_async<NT>(p, u1.b, u1.h, q0, t, qslot);
            }
        }
        for (int64_t seg_lo = t_begin; seg_lo < t_end; ++j) {
            const Unit u = find_unit<TILE>(sm.prefix, sm.lens, B, p.Hkv, seg_lo);
            const int64_t seg_hi = u.U1 < t_end ? u.U1 : t_end;
            const bool has_next = seg_hi < t_end;
            float cs[NH], m_run[NH], l_run[NH];
#pragma unroll
            for (int q = 0; q < NH; ++q) cs[q] = sm.cscale[j & 1u][q0 + q];
            if (has_next) {
                // query rows of the next unit; their buffer was last read by the
                // Q.K^T MMAs of the unit before this one, all complete by now
                // (this group has read every score of that unit)
                {
                    QRaw<NT> qnext;
                    take_q<NT>(qslot, qnext);
                    build_q<NT>(p, sm.qb[(j + 1) & 1u], sm.cscale[(j + 1) & 1u], qnext, q0, t);
                }
                fence_proxy_async_smem();
                softmax_sync(bar_id);
                if (lane == 0) mbar_arrive(&sm.qfull[(j + 1) & 1u]);
                const Unit un = find_unit<TILE>(sm.prefix, sm.lens, B, p.Hkv, seg_hi);
                if (un.U1 < t_end) {                       // loads for the unit after it
                    const Unit un2 = find_unit<TILE>(sm.prefix, sm.lens, B, p.Hkv, un.U1);
                    fetch_q_async<NT>(p, un2.b, un2.h, q0, t, qslot);
                }
            }
#pragma unroll
            for (int q = 0; q < NH; ++q) {
                m_run[q] = -INFINITY;
                l_run[q] = 0.0f;
            }
            bool any_pv = false;
            // Two tiles per pass where the segment has them: every wait, barrier
            // and fence of the pass is shared by both, so its latency is paid
            // once per 256 tokens.
            for (int64_t gt = seg_lo; gt < seg_hi;) {
                const int valid0 = tile_valid(u, gt);
                if (valid0 <= 0) {                         // the empty tile of a zero-length sequence
                    ++gt;
                    continue;
                }
                // every other tile of a unit is full or its last, so the second
                // tile (when the segment has one) has work too
                const bool two = gt + 1 < seg_hi;
                const int valid1 = two ? tile_valid(u, gt + 1) : 0;
                const int b0 = (int)(w % kBuf), b1 = (int)((w + 1) % kBuf);
                const uint32_t ph0 = (w / kBuf) & 1u, ph1 = ((w + 1) / kBuf) & 1u;
                float s0[NH], s1[NH];
                if (!aborted && !wait_warp(&sm.qkdone[b0], ph0, abort_flag, p.status, polls)) aborted = true;
                if (!aborted && two && !wait_warp(&sm.qkdone[b1], ph1, abort_flag, p.status, polls)) aborted = true;
                if (!aborted) {
                    tc::fence_after_sync();
                    uint32_t rh0[NH], rl0[NH], rh1[NH], rl1[NH];
                    tmem_ld_cols<NH>(trow + C::COL_S + NS * b0 + q0, rh0);
                    tmem_ld_cols<NH>(trow + C::COL_S + NS * b0 + NQ + q0, rl0);
                    if (two) {
                        tmem_ld_cols<NH>(trow + C::COL_S + NS * b1 + q0, rh1);
                        tmem_ld_cols<NH>(trow + C::COL_S + NS * b1 + NQ + q0, rl1);
                    }
                    tc::tmem_wait_ld();
                    tc::fence_before_sync();
                    mbar_arrive(&sm.sempty[b0]);
                    if (two) mbar_arrive(&sm.sempty[b1]);
                    const bool live0 = t < valid0, live1 = t < valid1;
#pragma unroll
                    for (int q = 0; q < NH; ++q) {
                        s0[q] = live0 ? fmaf(__uint_as_float(rl0[q]), 0.0625f, __uint_as_float(rh0[q])) * cs[q]
                                      : -INFINITY;
                        s1[q] = live1 ? fmaf(__uint_as_float(rl1[q]), 0.0625f, __uint_as_float(rh1[q])) * cs[q]
                                      : -INFINITY;
                    }
                } else {
#pragma unroll
                    for (int q = 0; q < NH; ++q) s0[q] = s1[q] = -INFINITY;
                }
                bool need = false;
#pragma unroll
                for (int q = 0; q < NH; ++q) need |= fmaxf(s0[q], s1[q]) > m_run[q] + kRescaleSlack;
                if (softmax_any(need, bar_id)) {
                    // raise the running max to the max over the pass's tokens (per
                    // query), rescale l and this group's O columns
#pragma unroll
                    for (int q = 0; q < NH; ++q) {
                        float mx = fmaxf(s0[q], s1[q]);
#pragma unroll
                        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
                        if (lane == 0) sm.red[sw][q0 + q] = mx;
                    }
                    softmax_sync(bar_id);
                    float f[NH];
#pragma unroll
                    for (int q = 0; q < NH; ++q) {
                        const float mt = fmaxf(fmaxf(sm.red[0][q0 + q], sm.red[1][q0 + q]),
                                               fmaxf(sm.red[2][q0 + q], sm.red[3][q0 + q]));
                        const float mn = fmaxf(m_run[q], mt);
                        f[q] = (m_run[q] == -INFINITY) ? 0.0f : fast_exp2(m_run[q] - mn);
                        m_run[q] = mn;
                        l_run[q] *= f[q];
                    }
                    softmax_sync(bar_id);                  // red is reused
                    if (any_pv && !aborted) {
                        // the previous P.V must have landed in O before it is rescaled
                        const uint32_t v = w - 1;
                        if (!wait_warp(&sm.pvdone[v % kBuf], (v / kBuf) & 1u, abort_flag, p.status, polls))
                            aborted = true;
                        if (!aborted) {
                            tc::fence_after_sync();
#pragma unroll
                            for (int k = 0; k < NTERM; ++k) {
                                uint32_t r[NH];
                                tmem_ld_cols<NH>(trow + C::COL_O + k * NQ + q0, r);
                                tc::tmem_wait_ld();
#pragma unroll
                                for (int q = 0; q < NH; ++q) r[q] = __float_as_uint(__uint_as_float(r[q]) * f[q]);
                                tmem_st_cols<NH>(trow + C::COL_O + k * NQ + q0, r);
                            }
                            tc::tmem_wait_st();
                        }
                    }
                }
                // P terms of this thread's token in both tiles for this group's
                // queries: column n = k * NQ + q0 + q
                uint32_t tw0[NTERM][NH / 4], tw1[NTERM][NH / 4];
#pragma unroll
                for (int q = 0; q < NH; q += 4) {
                    uint32_t ta[NTERM], tb[NTERM], tc_[NTERM], td[NTERM];
                    float pa[4], pb_[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const bool none = m_run[q + i] == -INFINITY;
                        pa[i] = none ? 0.0f : fast_exp2(s0[q + i] - m_run[q + i]);
                        pb_[i] = none ? 0.0f : fast_exp2(s1[q + i] - m_run[q + i]);
                        l_run[q + i] += pa[i] + pb_[i];
                    }
                    p_terms(pa[0], pa[1], ta);
                    p_terms(pa[2], pa[3], tb);
                    p_terms(pb_[0], pb_[1], tc_);
                    p_terms(pb_[2], pb_[3], td);
#pragma unroll
                    for (int k = 0; k < NTERM; ++k) {
                        tw0[k][q / 4] = ta[k] | (tb[k] << 16);
                        tw1[k][q / 4] = tc_[k] | (td[k] << 16);
                    }
                }
                // P.V of tiles w - kBuf and w + 1 - kBuf have read these P buffers
                if (!aborted && w >= (uint32_t)kBuf &&
                    !wait_warp(&sm.pvdone[b0], ph0 ^ 1u, abort_flag, p.status, polls))
                    aborted = true;
                if (!aborted && two && w + 1 >= (uint32_t)kBuf &&
                    !wait_warp(&sm.pvdone[b1], ph1 ^ 1u, abort_flag, p.status, polls))
                    aborted = true;
                if (!aborted) {
                    uint8_t* dst0 = sm.pb[b0] + (t / 8) * 128 + (t % 8) * 16;
                    uint8_t* dst1 = sm.pb[b1] + (t / 8) * 128 + (t % 8) * 16;
#pragma unroll
                    for (int k = 0; k < NTERM; ++k) {
                        const int n = k * NQ + q0;
                        if constexpr (NH == 4) {
                            *reinterpret_cast<uint32_t*>(dst0 + (n / 16) * 2048 + (n % 16)) = tw0[k][0];
                            if (two) *reinterpret_cast<uint32_t*>(dst1 + (n / 16) * 2048 + (n % 16)) = tw1[k][0];
                        } else {
                            *reinterpret_cast<uint2*>(dst0 + (n / 16) * 2048 + (n % 16)) =
                                make_uint2(tw0[k][0], tw0[k][1]);
                            if (two)
                                *reinterpret_cast<uint2*>(dst1 + (n / 16) * 2048 + (n % 16)) =
                                    make_uint2(tw1[k][0], tw1[k][1]);
                        }
                    }
                    fence_proxy_async_smem();
                    tc::fence_before_sync();
                    mbar_arrive(&sm.pfull[b0]);
                    if (two) mbar_arrive(&sm.pfull[b1]);
                }
                any_pv = true;
                w += two ? 2u : 1u;
                gt += two ? 2 : 1;
            }

            // ---- segment end ----
            float o[NH];
#pragma unroll
            for (int q = 0; q < NH; ++q) o[q] = 0.0f;
            if (any_pv && !aborted) {
                const uint32_t v = w - 1;
                if (!wait_warp(&sm.pvdone[v % kBuf], (v / kBuf) & 1u, abort_flag, p.status, polls))
                    aborted = true;
                if (!aborted) {
                    tc::fence_after_sync();
                    float scale = 1.0f;
#pragma unroll
                    for (int k = 0; k < NTERM; ++k) {
                        uint32_t r[NH];
                        tmem_ld_cols<NH>(trow + C::COL_O + k * NQ + q0, r);
                        tc::tmem_wait_ld();
#pragma unroll
                        for (int q = 0; q < NH; ++q) o[q] = fmaf(__uint_as_float(r[q]), scale, o[q]);
                        scale *= 0.0625f;
                    }
                    tc::fence_before_sync();
                }
            }
            // l over the 128 tokens (per-thread partials; the running max is shared)
#pragma unroll
            for (int q = 0; q < NH; ++q) {
                float l = l_run[q];
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) l += __shfl_xor_sync(0xFFFFFFFFu, l, off);
                if (lane == 0) sm.red[sw][q0 + q] = l;
            }
            softmax_sync(bar_id);
            float lt[NH];
#pragma unroll
            for (int q = 0; q < NH; ++q)
                lt[q] = (sm.red[0][q0 + q] + sm.red[1][q0 + q]) + (sm.red[2][q0 + q] + sm.red[3][q0 + q]);

            const bool whole = (u.U0 >= t_begin) && (u.U1 <= t_end);
            const int g = p.g;
            if (whole) {
#pragma unroll
                for (int q = 0; q < NH; ++q)
                    if (q0 + q < g)
                        p.out[((int64_t)u.b * p.Hq + (int64_t)u.h * g + q0 + q) * 128 + t] =
                            (lt[q] > 0.0f) ? o[q] / lt[q] : 0.0f;
            } else {
                // split unit: this CTA's partial; the merge kernel combines them
                float* part = p.partials + partial_slot(c, u.U0, T, N) * partial_slot_floats(g, 128);
#pragma unroll
                for (int q = 0; q < NH; ++q)
                    if (q0 + q < g) part[(q0 + q) * 128 + t] = o[q];
                if (t == 0) {
#pragma unroll
                    for (int q = 0; q < NH; ++q)
                        if (q0 + q < g) {
                            part[g * 128 + q0 + q] = m_run[q];
                            part[g * 128 + g + q0 + q] = lt[q];
                        }
                }
            }
            softmax_sync(bar_id);
            seg_lo = seg_hi;
        }
    }

    // ---- release tensor memory once every role is done ----
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (warp == kMmaWarp) tc::tmem_dealloc(tbase, C::kTmemCols);
}

// ---------------------------------------------------------------------------
// Split-K merge of the units the attention grid left in partials:
//     out = sum_j w_j O_j / sum_j w_j l_j,   w_j = 2^(m_j - M),  M = max_j m_j
// over the contributors j of a unit (m in base-2 score units).  CTA c of this
// grid stands for attention CTA c: for each split unit that CTA holds (at most
// its first and its last), it merges slice jc of the unit's g x 128 outputs,
// jc being c's index among the unit's contributors -- so a unit spread over
// many CTAs is merged by as many.  Each output is one thread's single pass
// over the contributors (running max, batches of loads in flight), with no
// CTA barrier.  The grid is a programmatic dependent of the attention
// grid: its prologue (the length scan) overlaps the attention tail, and
// griddepcontrol.wait holds it until every attention CTA has finished and its
// partial stores are visible.
// ---------------------------------------------------------------------------
constexpr int kMergeThreads = 256;
constexpr int kMergeBatch = 8;                        // contributors per batch of loads

__global__ void __launch_bounds__(kMergeThreads, 1) merge_split_units_kernel(const Params p, int n_attn) {
    __shared__ int32_t s_lens[kMaxBatchPerLaunch];
    __shared__ int32_t s_prefix[kMaxBatchPerLaunch + 1];
    __shared__ int32_t s_warp_tot[kMergeThreads / 32];
    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int B = p.B;
    // the lengths are final before the attention grid starts (stream order),
    // so the split is recomputed while that grid still runs
    {
        constexpr int per = (kMaxBatchPerLaunch + kMergeThreads - 1) / kMergeThreads;
        int tiles[per];
        int run = 0;
#pragma unroll
        for (int i = 0; i < per; ++i) {
            const int b = tid * per + i;
            int L = 0;
            if (b < B) {
                L = attended_len(p, b, nullptr);
                s_lens[b] = L;
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
        if (lane == 31) s_warp_tot[warp] = incl;
        __syncthreads();
        int before = 0;
        for (int w = 0; w < warp; ++w) before += s_warp_tot[w];
        int acc = before + incl - run;
#pragma unroll
        for (int i = 0; i < per; ++i) {
            const int b = tid * per + i;
            if (b < B) s_prefix[b] = acc;
            acc += tiles[i];
        }
        if (tid == kMergeThreads - 1) s_prefix[B] = acc;
    }
    __syncthreads();
    const int64_t T = s_prefix[B];
    const int64_t N = n_attn;
    const int64_t c = blockIdx.x;
    const int64_t t_begin = range_start(c, T, N);
    const int64_t t_end = range_start(c + 1, T, N);
    if (t_begin >= t_end) return;
    const int g = p.g;
    const int64_t slot_floats = partial_slot_floats(g, 128);
    const bool dense = T >= N;                            // every CTA range non-empty
    bool waited = false;
    // the units holding this range's first and last tiles: the only ones it can share
    for (int which = 0; which < 2; ++which) {
        const int64_t gt = which == 0 ? t_begin : t_end - 1;
        const Unit u = find_unit<TILE>(s_prefix, s_lens, B, p.Hkv, gt);
        if (which == 1 && u.U0 <= t_begin) break;          // the same unit as the first
        const int64_t c_first = cta_of(u.U0, T, N);
        if (cta_of(u.U1 - 1, T, N) == c_first) continue;   // inside one range: not split
        const int ncc = unit_contributors(u.U0, u.U1, T, N);
        const bool first_odd = range_start(c_first, T, N) < u.U0;   // the unit is c_first's second unit
        // this CTA's contributor index, and its slice of the g x 128 outputs
        const int jc = dense ? (int)(c - c_first) : (int)(t_begin - u.U0);
        const int per = (g * 128 + ncc - 1) / ncc;
        const int o0 = jc * per;
        const int o1 = o0 + per < g * 128 ? o0 + per : g * 128;
        const float* base = p.partials + 2 * c_first * slot_floats;
        auto part_of = [&](int j) -> const float* {
            if (dense) return base + (2 * (int64_t)j + ((j == 0 && first_odd) ? 1 : 0)) * slot_floats;
            return p.partials + contributor_slot(j, u.U0, c_first, first_odd, dense, T, N) * slot_floats;
        };
        if (!waited) {
            wait_prerequisites();                         // partials are complete and visible from here
            waited = true;
        }
        for (int o = o0 + tid; o < o1; o += kMergeThreads) {
            const int q = o >> 7, d = o & 127;
            // one pass over the contributors with a running max (batches of loads in flight)
            float M = -INFINITY, acc = 0.0f, L = 0.0f;
            for (int j0 = 0; j0 < ncc; j0 += kMergeBatch) {
                float m[kMergeBatch], l[kMergeBatch], v[kMergeBatch];
#pragma unroll
                for (int k = 0; k < kMergeBatch; ++k) {
                    const bool in = j0 + k < ncc;
                    const float* pp = in ? part_of(j0 + k) : base;
                    m[k] = in ? __ldcg(pp + g * 128 + q) : -INFINITY;
                    l[k] = in ? __ldcg(pp + g * 128 + g + q) : 0.0f;
                    v[k] = in ? __ldcg(pp + q * 128 + d) : 0.0f;
                }
                float Mb = M;
#pragma unroll
                for (int k = 0; k < kMergeBatch; ++k) Mb = fmaxf(Mb, m[k]);
                if (Mb == -INFINITY) continue;
                const float f = M == -INFINITY ? 0.0f : fast_exp2(M - Mb);
                acc *= f;
                L *= f;
#pragma unroll
                for (int k = 0; k < kMergeBatch; ++k) {
                    const float wk = m[k] == -INFINITY ? 0.0f : fast_exp2(m[k] - Mb);
                    L = fmaf(wk, l[k], L);
                    acc = fmaf(wk, v[k], acc);
                }
                M = Mb;
            }
            p.out[((int64_t)u.b * p.Hq + (int64_t)u.h * g + q) * 128 + d] = L > 0.0f ? acc / L : 0.0f;
        }
    }
}

template <int NT>
cudaError_t launch_tc(const Params& p, int grid, cudaStream_t stream) {
    auto kern = decode_attention_tc_kernel<NT>;
    const int smem = (int)sizeof(Smem<NT>) + 1024;   // + alignment slack
    static int configured[kMaxDevices] = {};
    cudaError_t e0 = ensure_smem_attribute(reinterpret_cast<const void*>(kern), smem, configured);
    if (e0 != cudaSuccess) return e0;
    kern<<<grid, kThreads, smem, stream>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    // the merge grid, launched as a programmatic dependent of the attention grid
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kMergeThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, merge_split_units_kernel, p, grid);
}

}  // namespace

cudaError_t launch_decode_attention_tc(const attn::Params& p, int sms, cudaStream_t stream) {
    return p.g > 8 ? launch_tc<2>(p, sms, stream) : launch_tc<1>(p, sms, stream);
}

}  // namespace nvfp4kv

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
// contiguous range per CTA, one CTA per SM (stream-K); a (sequence, head)
// unit shared by several CTAs is merged by the last one to finish with it.
//
// Inside a CTA every stage of a tile has its own warps, and the stages of
// consecutive tiles overlap; they hand tiles to each other through
// mbarriers (double-buffered operands), never through CTA-wide barriers:
//
//   load warp   : bulk copies of K/V codes and scale bytes into a 4-stage ring
//   dequant warps 0-3 and 8-11: thread t of group h = token t, head_dim half
//                 h.  K codes -> signed FP8 K in tensor memory lane t (the A
//                 operand of Q.K^T); V codes -> FP8 V^T in shared memory (the
//                 MN-major A operand of P.V).  K and V^T have 5 buffers
//   MMA warp    : S^T[t][n] = K . Q'^T,  O^T[d][n] += V^T . P^T
//                 (a tcgen05 MMA costs about the same for any N up to 256:
//                 the instruction count per tile, 4 + 4, sets the pace)
//   softmax 4-7 : thread t reads score row t, online softmax in base 2 with a
//                 lazily raised running max, P as three E4M3 terms
//                 p ~ t0 + t1/16 + t2/256 (MN-major B operand); at the end of
//                 a unit thread d reads O^T row d and writes the output
//
// The query operand Q' holds, per query row, an exact two-term E4M3 split of
// the bf16 query scaled by a power of two: q * 2^e = hi + lo / 16, so the
// scores are exact sums of FP8 products (up to fp32 accumulation order).
#include <cuda_bf16.h>

#include "nvfp4kv_attention_common.cuh"
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
constexpr int kStages = 4;
// operand buffers: K (tensor memory) and V^T (shared memory) let the dequant
// warps run ahead of the softmax; S (tensor memory) lets Q.K^T run ahead
constexpr int kKBuf = 5, kVBuf = 5, kSBuf = 3, kPBuf = 3;
constexpr int NTERM = 3;                              // E4M3 terms of P

// warp roles
constexpr int kSWarp0 = 4;                            // warps 4-7: softmax / output
constexpr int kVWarp0 = 8;                            // warps 0-3 and 8-11: dequant
constexpr int kLoadWarp = 12;
constexpr int kMmaWarp = 13;
constexpr int kThreads = 14 * 32;
constexpr int kSoftmaxBar = 1;                        // named barrier of the softmax warps

constexpr uint32_t kWaitPolls = 1u << 16;             // sleeping polls (<= 20 us each) per wait
constexpr uint32_t kMmaIdlePolls = 1u << 25;          // idle polls (~32 ns sleep each) of the MMA thread

template <int NT>
struct Cfg {
    static constexpr int NQ = 8 * NT;                 // query rows (padded GQA group)
    static constexpr int NS = 2 * NQ;                 // score columns: hi, lo
    static constexpr int NP = (NTERM * NQ + 15) / 16 * 16;   // P columns (MMA N), term-major
    static constexpr uint32_t COL_K = 0;              // kKBuf buffers x 32 columns (4 FP8 each)
    static constexpr uint32_t COL_S = 32 * kKBuf;     // kSBuf buffers x NS
    static constexpr uint32_t COL_O = COL_S + kSBuf * NS;  // NP
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
    uint8_t vt[kVBuf][128 * TILE];                        // V^T: (d/16)*2048 + (t/8)*128 + (t%8)*16 + d%16
    uint8_t pb[kPBuf][C::NP * TILE];                      // P^T: (n/16)*2048 + (t/8)*128 + (t%8)*16 + n%16
    uint8_t qb[2][C::NS * 128];                       // Q':  (n/8)*1024 + (d/16)*128 + (n%8)*16 + d%16
    uint2 lut[2][128][kLutCopies];
    uint64_t full[kStages], empty[kStages];
    uint64_t kfull[kKBuf], kempty[kKBuf], vfull[kVBuf], vtfree[kVBuf];
    uint64_t sfull[kSBuf], sempty[kSBuf], pfull[kPBuf], pvdone[kPBuf];
    uint64_t qfull[2];
    uint64_t mma_done;
    int32_t lens[kMaxBatchPerLaunch];
    int32_t prefix[kMaxBatchPerLaunch + 1];
    float cscale[2][C::NQ];
    float red[4][C::NQ];
    int32_t warp_tot[kThreads / 32];
    CombineSmem comb;
    uint32_t tmem_base;
    int32_t n_sig;                                    // split units whose partial this CTA wrote
    int32_t n_pend;                                   // units this CTA must merge at its end
    int64_t sig_gt[2];
    int64_t pend_gt[2];
    int32_t abort_flag;
};

// ---------------------------------------------------------------------------
// small helpers
// ---------------------------------------------------------------------------

// non-blocking test of the phase with the given parity
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Bounded wait of one thread: gives up when the CTA's abort flag is set or
// after kWaitPolls sleeping polls (then sets the flag and reports a timeout).
// Inlined: a call would spill the live registers of the caller.
__device__ __forceinline__ bool wait_one(uint64_t* bar, uint32_t parity, int32_t* abort_flag,
                                         int32_t* status) {
    if (mbar_test_wait(bar, parity)) return true;
    for (uint32_t i = 0; i < kWaitPolls; ++i) {
        if (mbar_try_wait_hint(bar, parity, 20000u)) return true;
        if (*reinterpret_cast<volatile int32_t*>(abort_flag)) return false;
    }
    atomicExch(abort_flag, 1);
    report(status, NVFP4_ERR_TIMEOUT);
    return false;
}

// The same for a whole warp; the result is warp-uniform.
__device__ __forceinline__ bool wait_warp(uint64_t* bar, uint32_t parity, int32_t* abort_flag,
                                          int32_t* status) {
    const bool ok = wait_one(bar, parity, abort_flag, status);
    return __all_sync(0xFFFFFFFFu, ok);
}

// the softmax warps' named barrier, plain and as an OR-reduction
__device__ __forceinline__ void softmax_sync() {
    asm volatile("bar.sync %0, 128;" ::"n"(kSoftmaxBar) : "memory");
}
__device__ __forceinline__ bool softmax_any(bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred pi, po;\n\tsetp.ne.u32 pi, %1, 0;\n\t"
        "bar.red.or.pred po, %2, 128, pi;\n\tselp.u32 %0, 1, 0, po;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v), "n"(kSoftmaxBar)
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
    if constexpr (N == 8) {
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
    if constexpr (N == 8) {
        tc::tmem_st_x8(taddr, r);
    } else {
        static_assert(N == 16, "columns");
        tc::tmem_st_x8(taddr, r);
        tc::tmem_st_x8(taddr + 8, r + 8);
    }
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
    static constexpr int PER = Cfg<NT>::NQ;           // bf16 elements per thread: 8 or 16
    uint4 w[PER / 8];
};

template <int NT>
__device__ __forceinline__ void fetch_q(const Params& p, int b, int h, int t, QRaw<NT>& raw) {
    constexpr int PER = QRaw<NT>::PER;
    constexpr int TPQ = 128 / PER;                    // threads per query row
    const int q = t / TPQ;
    const int d0 = (t % TPQ) * PER;
    const bool valid = q < p.g;
    const int64_t row = ((int64_t)b * p.Hq + (int64_t)h * p.g + (valid ? q : 0)) * 128 + d0;
    const uint4* src = reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(p.q) + row);
#pragma unroll
    for (int i = 0; i < PER / 8; ++i) raw.w[i] = valid ? __ldg(src + i) : make_uint4(0, 0, 0, 0);
}

template <int NT>
__device__ __forceinline__ void build_q(const Params& p, uint8_t* qb, float* cscale, const QRaw<NT>& raw,
                                        int t) {
    using C = Cfg<NT>;
    constexpr int PER = QRaw<NT>::PER;
    constexpr int TPQ = 128 / PER;
    const int q = t / TPQ;
    const int d0 = (t % TPQ) * PER;
    float v[PER];
#pragma unroll
    for (int i = 0; i < PER / 8; ++i) {
        const uint32_t w[4] = {raw.w[i].x, raw.w[i].y, raw.w[i].z, raw.w[i].w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            v[8 * i + 2 * k + 0] = __uint_as_float(w[k] << 16);
            v[8 * i + 2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
        }
    }
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < PER; ++i) amax = fmaxf(amax, fabsf(v[i]));
#pragma unroll
    for (int o = 1; o < TPQ; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
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
    // K-major rows n = q (hi) and n = NQ + q (lo); d0 is a multiple of 8
    const int nh = q, nl = C::NQ + q;
#pragma unroll
    for (int c = 0; c < PER / 8; ++c) {
        const int d = d0 + 8 * c;
        uint8_t* dh = qb + (nh / 8) * 1024 + (d / 16) * 128 + (nh % 8) * 16 + d % 16;
        uint8_t* dl = qb + (nl / 8) * 1024 + (d / 16) * 128 + (nl % 8) * 16 + d % 16;
        *reinterpret_cast<uint2*>(dh) = make_uint2(hw[2 * c], hw[2 * c + 1]);
        *reinterpret_cast<uint2*>(dl) = make_uint2(lw[2 * c], lw[2 * c + 1]);
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
    int64_t seg_lo, seg_hi, gt, t_end;
    Unit u;
    int64_t last;                                     // the tile returned by next()
    int32_t j;                                        // its segment ordinal
    bool first;                                       // first tile with work of its segment
    bool fresh;

    __device__ __forceinline__ void start(int64_t t_begin, int64_t t_end_) {
        seg_lo = seg_hi = gt = t_begin;
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
            seg_lo = seg_hi;
            u = find_unit<TILE>(prefix, lens, B, Hkv, seg_lo);
            seg_hi = u.U1 < t_end ? u.U1 : t_end;
            gt = seg_lo;
            ++j;
            fresh = true;
        }
    }
};

// ---------------------------------------------------------------------------
// the kernel
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

    // ---- tensor memory, barriers, lookup tables, zeroed P buffers ----
    if (warp == kMmaWarp) {
        tc::tmem_alloc(&sm.tmem_base, C::kTmemCols);
        tc::tmem_relinquish();
    }
    // the load warp sets up every barrier and starts the first copies at once
    TileWalker load_walk;
    load_walk.start(t_begin, t_end);
    uint32_t load_w = 0;
    if (warp == kLoadWarp && lane == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], 8);
        }
        for (int b = 0; b < kKBuf; ++b) {
            mbar_init(&sm.kfull[b], 8);
            mbar_init(&sm.kempty[b], 1);
        }
        for (int b = 0; b < kVBuf; ++b) {
            mbar_init(&sm.vfull[b], 8);
            mbar_init(&sm.vtfree[b], 1);
        }
        for (int b = 0; b < kSBuf; ++b) {
            mbar_init(&sm.sfull[b], 1);
            mbar_init(&sm.sempty[b], 4);
        }
        for (int b = 0; b < kPBuf; ++b) {
            mbar_init(&sm.pfull[b], 4);
            mbar_init(&sm.pvdone[b], 1);
        }
        mbar_init(&sm.qfull[0], 4);
        mbar_init(&sm.qfull[1], 4);
        mbar_init(&sm.mma_done, 1);
        fence_mbar_init();
        sm.abort_flag = 0;
        sm.n_sig = 0;
        sm.n_pend = 0;
        // the first two tiles only: the CTA barrier below waits for this lane
        while (load_w < 2u && load_walk.next(sm.prefix, sm.lens, B, p.Hkv)) {
            issue_tile<128, TILE>(p, load_walk.u, load_walk.last, sm.ring[load_w], &sm.full[load_w]);
            ++load_w;
        }
    }
    QRaw<NT> q_first;                                 // query loads in flight during the table build
    if (warp >= kSWarp0 && warp < kVWarp0) {
        const Unit u0 = find_unit<TILE>(sm.prefix, sm.lens, B, p.Hkv, t_begin);
        fetch_q<NT>(p, u0.b, u0.h, tid - 32 * kSWarp0, q_first);
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

    if (warp == kLoadWarp) {
        // ================= bulk copies into the ring =================
        if (lane == 0) {
            uint32_t w = load_w;                       // the first stages went out in the prologue
            while (load_walk.next(sm.prefix, sm.lens, B, p.Hkv)) {
                const int s = (int)(w % kStages);
                if (w >= (uint32_t)kStages && !wait_one(&sm.empty[s], ((w / kStages) - 1) & 1u, abort_flag, p.status))
                    break;
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
    } else if (warp == kMmaWarp) {
        // ================= tensor-core MMAs (one thread) =================
        // Q.K^T runs ahead of the softmax as far as the S buffers allow; P.V
        // follows the softmax.  Both streams are polled, so neither waits
        // behind the other.
        if (lane == 0) {
            const uint32_t idesc_qk = tc::idesc_e4m3(128, NS, false, false, false);
            const uint32_t idesc_pv = tc::idesc_e4m3(128, C::NP, true, true, false);
            TileWalker qk, pv;
            qk.start(t_begin, t_end);
            pv.start(t_begin, t_end);
            bool qk_more = qk.next(sm.prefix, sm.lens, B, p.Hkv);
            bool pv_more = pv.next(sm.prefix, sm.lens, B, p.Hkv);
            uint32_t wq = 0, wp = 0;                   // work tiles issued per stream
            int32_t q_seg = -1;                        // segment whose query operand is in place
            uint32_t idle = 0;
            bool ok = true;
            while (ok && (qk_more || pv_more)) {
                bool progress = false;
                if (pv_more && wp < wq) {
                    const int bv = (int)(wp % kVBuf), bp = (int)(wp % kPBuf);
                    if (mbar_test_wait(&sm.vfull[bv], (wp / kVBuf) & 1u) &&
                        mbar_test_wait(&sm.pfull[bp], (wp / kPBuf) & 1u)) {
                        tc::fence_after_sync();
                        const uint32_t va = tc::smem_addr(sm.vt[bv]);
                        const uint32_t pa = tc::smem_addr(sm.pb[bp]);
                        const bool first = pv.first;   // O restarts with each unit
#pragma unroll
                        for (int ks = 0; ks < 4; ++ks)
                            tc::mma_e4m3_ss(tbase + C::COL_O, tc::smem_desc(va + ks * 512, 128, 2048),
                                            tc::smem_desc(pa + ks * 512, 128, 2048), idesc_pv,
                                            !first || ks > 0);
                        tc::mma_commit(&sm.pvdone[bp]);
                        tc::mma_commit(&sm.vtfree[bv]);
                        ++wp;
                        pv_more = pv.next(sm.prefix, sm.lens, B, p.Hkv);
                        progress = true;
                    }
                }
                if (qk_more) {
                    const int bk = (int)(wq % kKBuf), bs = (int)(wq % kSBuf);
                    const int32_t jq = qk.j;
                    const bool q_ok = q_seg == jq || mbar_test_wait(&sm.qfull[jq & 1], (jq >> 1) & 1u);
                    if (q_ok) q_seg = jq;
                    if (q_ok && mbar_test_wait(&sm.kfull[bk], (wq / kKBuf) & 1u) &&
                        (wq < (uint32_t)kSBuf || mbar_test_wait(&sm.sempty[bs], ((wq / kSBuf) - 1) & 1u))) {
                        tc::fence_after_sync();
                        const uint32_t qa = tc::smem_addr(sm.qb[jq & 1]);
                        const uint32_t kcol = tbase + C::COL_K + 32 * bk;
                        const uint32_t scol = tbase + C::COL_S + NS * bs;
#pragma unroll
                        for (int ks = 0; ks < 4; ++ks)
                            tc::mma_e4m3_ts(scol, kcol + 8 * ks, tc::smem_desc(qa + ks * 256, 128, 1024),
                                            idesc_qk, ks > 0);
                        tc::mma_commit(&sm.sfull[bs]);
                        tc::mma_commit(&sm.kempty[bk]);
                        ++wq;
                        qk_more = qk.next(sm.prefix, sm.lens, B, p.Hkv);
                        progress = true;
                    }
                }
                if (progress) {
                    idle = 0;
                } else {
                    if (*reinterpret_cast<volatile int32_t*>(abort_flag)) break;
                    if (++idle > kMmaIdlePolls) {
                        atomicExch(abort_flag, 1);
                        report(p.status, NVFP4_ERR_TIMEOUT);
                        ok = false;
                    }
                    __nanosleep(32);
                }
            }
            // every issued MMA must complete before tensor memory is released
            tc::mma_commit(&sm.mma_done);
            if (!mbar_wait_sleep(&sm.mma_done, 0, kWaitPolls)) report(p.status, NVFP4_ERR_TIMEOUT);
        }
        __syncwarp();
    } else if (warp < kSWarp0 || warp >= kVWarp0) {
        // ======== dequant: head_dim half h of the K and V rows of token t ========
        const int h = warp >= kVWarp0 ? 1 : 0;            // head_dim [64h, 64h + 64)
        const int t = tid - (h ? 32 * kVWarp0 : 0);        // token, tensor-memory lane
        const uint32_t trow = tbase + ((uint32_t)(32 * (warp & 3)) << 16);
        const int rot = (t >> 1) & 1;                      // V chunk order: fewer bank conflicts
        const uint2* lut_k = &sm.lut[0][0][lane & (kLutCopies - 1)];
        const uint2* lut_v = &sm.lut[1][0][lane & (kLutCopies - 1)];
        uint32_t w = 0;
        bool ok = true;
        for (int64_t seg_lo = t_begin; seg_lo < t_end && ok;) {
            const Unit u = find_unit<TILE>(sm.prefix, sm.lens, B, p.Hkv, seg_lo);
            const int64_t seg_hi = u.U1 < t_end ? u.U1 : t_end;
            for (int64_t gt = seg_lo; gt < seg_hi && ok; ++gt) {
                if (tile_valid(u, gt) <= 0) continue;
                const int s = (int)(w % kStages);
                const int bk = (int)(w % kKBuf), bv = (int)(w % kVBuf);
                ok = wait_warp(&sm.full[s], (w / kStages) & 1u, abort_flag, p.status);
                if (ok && w >= kKBuf)      // Q.K^T of tile w - kKBuf has read this K buffer
                    ok = wait_warp(&sm.kempty[bk], ((w / kKBuf) - 1) & 1u, abort_flag, p.status);
                if (!ok) break;
                const uint8_t* st = sm.ring[s];
                uint4 xk[2], xv[2];
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    xk[j] = *reinterpret_cast<const uint4*>(st + t * kKB + 32 * h + 16 * j);
                    xv[j] = *reinterpret_cast<const uint4*>(st + OFF_VC + t * kKB + 32 * h + 16 * (j ^ rot));
                }
                const uint32_t sk = *reinterpret_cast<const uint32_t*>(st + OFF_KS + t * kSB + 4 * h);
                const uint32_t sv = *reinterpret_cast<const uint32_t*>(st + OFF_VS + t * kSB + 4 * h);
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.empty[s]);
                // K: 64 codes -> 16 tensor-memory columns (4 FP8 each)
                uint32_t kf[16];
#pragma unroll
                for (int j = 0; j < 2; ++j) {              // 16 bytes = 32 codes = 2 blocks
                    const uint2 l0 = lut_k[((sk >> (16 * j)) & 0x7F) * kLutCopies];
                    const uint2 l1 = lut_k[((sk >> (16 * j + 8)) & 0x7F) * kLutCopies];
                    dequant_word(xk[j].x, l0.x, l0.y, kf[8 * j + 0], kf[8 * j + 1]);
                    dequant_word(xk[j].y, l0.x, l0.y, kf[8 * j + 2], kf[8 * j + 3]);
                    dequant_word(xk[j].z, l1.x, l1.y, kf[8 * j + 4], kf[8 * j + 5]);
                    dequant_word(xk[j].w, l1.x, l1.y, kf[8 * j + 6], kf[8 * j + 7]);
                }
                tmem_st_x16(trow + C::COL_K + 32 * bk + 16 * h, kf);
                tc::tmem_wait_st();
                tc::fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.kfull[bk]);  // Q.K^T may start before V is done
                // P.V of tile w - kVBuf has read this V^T buffer
                if (w >= kVBuf && !wait_warp(&sm.vtfree[bv], ((w / kVBuf) - 1) & 1u, abort_flag, p.status)) {
                    ok = false;
                    break;
                }
                // V: 64 codes -> 4 rows of 16 head_dim bytes of V^T
                uint8_t* dst = sm.vt[bv] + (4 * h) * 2048 + (t / 8) * 128 + (t % 8) * 16;
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const int cc = j ^ rot;                // head_dim 64h + 32cc .. +31
                    const uint2 l0 = lut_v[((sv >> (16 * cc)) & 0x7F) * kLutCopies];
                    const uint2 l1 = lut_v[((sv >> (16 * cc + 8)) & 0x7F) * kLutCopies];
                    uint4 o0, o1;
                    dequant_word(xv[j].x, l0.x, l0.y, o0.x, o0.y);
                    dequant_word(xv[j].y, l0.x, l0.y, o0.z, o0.w);
                    dequant_word(xv[j].z, l1.x, l1.y, o1.x, o1.y);
                    dequant_word(xv[j].w, l1.x, l1.y, o1.z, o1.w);
                    *reinterpret_cast<uint4*>(dst + (2 * cc) * 2048) = o0;
                    *reinterpret_cast<uint4*>(dst + (2 * cc + 1) * 2048) = o1;
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.vfull[bv]);
                ++w;
            }
            seg_lo = seg_hi;
        }
    } else {
        // ================= softmax, P, output (warps 4-7) =================
        const int t = tid - 32 * kSWarp0;                  // token of the score row; head_dim of O
        const int sw = warp - kSWarp0;
        const uint32_t trow = tbase + ((uint32_t)(32 * sw) << 16);
        bool aborted = false;
        uint32_t w = 0;
        uint32_t j = 0;
        {   // query operand of the first unit (loads issued in the prologue)
            build_q<NT>(p, sm.qb[0], sm.cscale[0], q_first, t);
            fence_proxy_async_smem();
            softmax_sync();
            if (lane == 0) mbar_arrive(&sm.qfull[0]);
        }
        for (int64_t seg_lo = t_begin; seg_lo < t_end; ++j) {
            const Unit u = find_unit<TILE>(sm.prefix, sm.lens, B, p.Hkv, seg_lo);
            const int64_t seg_hi = u.U1 < t_end ? u.U1 : t_end;
            const bool has_next = seg_hi < t_end;
            QRaw<NT> qnext;
            if (has_next) {                                // loads in flight during this segment
                const Unit un = find_unit<TILE>(sm.prefix, sm.lens, B, p.Hkv, seg_hi);
                fetch_q<NT>(p, un.b, un.h, t, qnext);
            }
            float cs[NQ], m_run[NQ], l_run[NQ];
#pragma unroll
            for (int q = 0; q < NQ; ++q) {
                cs[q] = sm.cscale[j & 1u][q];
                m_run[q] = -INFINITY;
                l_run[q] = 0.0f;
            }
            bool any_pv = false;
            for (int64_t gt = seg_lo; gt < seg_hi; ++gt) {
                const int valid = tile_valid(u, gt);
                if (valid <= 0) continue;
                const int bs = (int)(w % kSBuf), bp = (int)(w % kPBuf);
                float s[NQ];
                if (!aborted && !wait_warp(&sm.sfull[bs], (w / kSBuf) & 1u, abort_flag, p.status)) aborted = true;
                if (!aborted) {
                    tc::fence_after_sync();
                    uint32_t r[NS];
                    tmem_ld_cols<NS>(trow + C::COL_S + NS * bs, r);
                    tc::tmem_wait_ld();
                    tc::fence_before_sync();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&sm.sempty[bs]);
                    const bool live = t < valid;
#pragma unroll
                    for (int q = 0; q < NQ; ++q)
                        s[q] = live ? fmaf(__uint_as_float(r[NQ + q]), 0.0625f, __uint_as_float(r[q])) * cs[q]
                                    : -INFINITY;
                } else {
#pragma unroll
                    for (int q = 0; q < NQ; ++q) s[q] = -INFINITY;
                }
                bool need = false;
#pragma unroll
                for (int q = 0; q < NQ; ++q) need |= s[q] > m_run[q] + kRescaleSlack;
                if (softmax_any(need)) {
                    // raise the running max to the tile max (per query over the 128
                    // tokens), rescale l and O
#pragma unroll
                    for (int q = 0; q < NQ; ++q) {
                        float mx = s[q];
#pragma unroll
                        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
                        if (lane == 0) sm.red[sw][q] = mx;
                    }
                    softmax_sync();
                    float f[NQ];
#pragma unroll
                    for (int q = 0; q < NQ; ++q) {
                        const float mt = fmaxf(fmaxf(sm.red[0][q], sm.red[1][q]), fmaxf(sm.red[2][q], sm.red[3][q]));
                        const float mn = fmaxf(m_run[q], mt);
                        f[q] = (m_run[q] == -INFINITY) ? 0.0f : fast_exp2(m_run[q] - mn);
                        m_run[q] = mn;
                        l_run[q] *= f[q];
                    }
                    softmax_sync();                        // red is reused
                    if (any_pv && !aborted) {
                        // the previous P.V must have landed in O before it is rescaled
                        const uint32_t v = w - 1;
                        if (!wait_warp(&sm.pvdone[v % kPBuf], (v / kPBuf) & 1u, abort_flag, p.status)) aborted = true;
                        if (!aborted) {
                            tc::fence_after_sync();
#pragma unroll
                            for (int k = 0; k < NTERM; ++k) {
                                uint32_t r[NQ];
                                tmem_ld_cols<NQ>(trow + C::COL_O + k * NQ, r);
                                tc::tmem_wait_ld();
#pragma unroll
                                for (int q = 0; q < NQ; ++q) r[q] = __float_as_uint(__uint_as_float(r[q]) * f[q]);
                                tmem_st_cols<NQ>(trow + C::COL_O + k * NQ, r);
                            }
                            tc::tmem_wait_st();
                        }
                    }
                }
                // P terms of this token for every query: column n = k * NQ + q
                uint32_t tw[NTERM][NQ / 4];
#pragma unroll
                for (int q = 0; q < NQ; q += 4) {
                    uint32_t ta[NTERM], tb[NTERM];
                    float pq[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        pq[i] = (m_run[q + i] == -INFINITY) ? 0.0f : fast_exp2(s[q + i] - m_run[q + i]);
                        l_run[q + i] += pq[i];
                    }
                    p_terms(pq[0], pq[1], ta);
                    p_terms(pq[2], pq[3], tb);
#pragma unroll
                    for (int k = 0; k < NTERM; ++k) tw[k][q / 4] = ta[k] | (tb[k] << 16);
                }
                if (!aborted && w >= kPBuf &&
                    !wait_warp(&sm.pvdone[bp], ((w / kPBuf) - 1) & 1u, abort_flag, p.status))
                    aborted = true;
                if (!aborted) {
                    uint8_t* dst = sm.pb[bp] + (t / 8) * 128 + (t % 8) * 16;
#pragma unroll
                    for (int k = 0; k < NTERM; ++k) {
                        const int n = k * NQ;
                        if constexpr (NQ == 8) {
                            *reinterpret_cast<uint2*>(dst + (n / 16) * 2048 + (n % 16)) =
                                make_uint2(tw[k][0], tw[k][1]);
                        } else {
                            *reinterpret_cast<uint4*>(dst + (n / 16) * 2048) =
                                make_uint4(tw[k][0], tw[k][1], tw[k][2], tw[k][3]);
                        }
                    }
                    fence_proxy_async_smem();
                    tc::fence_before_sync();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&sm.pfull[bp]);
                }
                any_pv = true;
                ++w;
            }

            // ---- segment end ----
            if (has_next) {
                // query operand of the next unit; its buffer was last read by the
                // Q.K^T MMAs of the unit before this one, all complete by now
                build_q<NT>(p, sm.qb[(j + 1) & 1u], sm.cscale[(j + 1) & 1u], qnext, t);
                fence_proxy_async_smem();
                softmax_sync();
                if (lane == 0) mbar_arrive(&sm.qfull[(j + 1) & 1u]);
            }
            float o[NQ];
#pragma unroll
            for (int q = 0; q < NQ; ++q) o[q] = 0.0f;
            if (any_pv && !aborted) {
                const uint32_t v = w - 1;
                if (!wait_warp(&sm.pvdone[v % kPBuf], (v / kPBuf) & 1u, abort_flag, p.status)) aborted = true;
                if (!aborted) {
                    tc::fence_after_sync();
                    float scale = 1.0f;
#pragma unroll
                    for (int k = 0; k < NTERM; ++k) {
                        uint32_t r[NQ];
                        tmem_ld_cols<NQ>(trow + C::COL_O + k * NQ, r);
                        tc::tmem_wait_ld();
#pragma unroll
                        for (int q = 0; q < NQ; ++q) o[q] = fmaf(__uint_as_float(r[q]), scale, o[q]);
                        scale *= 0.0625f;
                    }
                    tc::fence_before_sync();
                }
            }
            // l over the 128 tokens (per-thread partials; the running max is shared)
#pragma unroll
            for (int q = 0; q < NQ; ++q) {
                float l = l_run[q];
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) l += __shfl_xor_sync(0xFFFFFFFFu, l, off);
                if (lane == 0) sm.red[sw][q] = l;
            }
            softmax_sync();
            float lt[NQ];
#pragma unroll
            for (int q = 0; q < NQ; ++q) lt[q] = (sm.red[0][q] + sm.red[1][q]) + (sm.red[2][q] + sm.red[3][q]);

            const bool whole = (u.U0 >= t_begin) && (u.U1 <= t_end);
            const int g = p.g;
            const int64_t slot_floats = partial_slot_floats(g, 128);
            if (whole) {
#pragma unroll
                for (int q = 0; q < NQ; ++q)
                    if (q < g)
                        p.out[((int64_t)u.b * p.Hq + (int64_t)u.h * g + q) * 128 + t] =
                            (lt[q] > 0.0f) ? o[q] / lt[q] : 0.0f;
            } else {
                float* part = p.partials + partial_slot(c, u.U0, T, N) * slot_floats;
#pragma unroll
                for (int q = 0; q < NQ; ++q)
                    if (q < g) part[q * 128 + t] = o[q];
                if (t == 0) {
#pragma unroll
                    for (int q = 0; q < NQ; ++q)
                        if (q < g) {
                            part[g * 128 + q] = m_run[q];
                            part[g * 128 + g + q] = lt[q];
                        }
                }
                // arrival is counted after the roles finish, so that the
                // atomic (and the wait for its release) stays off this CTA's
                // tile pipeline; a CTA splits at most its first and last unit
                if (t == 0) sm.sig_gt[sm.n_sig++] = u.U0;
            }
            softmax_sync();
            seg_lo = seg_hi;
        }
    }

    // ---- release tensor memory once every role is done ----
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (warp == kMmaWarp) tc::tmem_dealloc(tbase, C::kTmemCols);

    // ---- split-K: count this CTA's arrival at each split unit (one lane per
    // unit, atomics in flight together); the last to arrive merges the unit
    // on every thread ----
    if (warp == 0) {
        const int n_sig = sm.n_sig;
        bool last = false;
        int64_t gt = 0;
        if (lane < n_sig) {
            gt = sm.sig_gt[lane];
            const Unit u = find_unit<TILE>(sm.prefix, sm.lens, B, p.Hkv, gt);
            const int prev = arrive_split_unit(&p.counters[(int64_t)u.b * p.Hkv + u.h]);
            last = prev == unit_contributors(u.U0, u.U1, T, N) - 1;
        }
        const uint32_t lm = __ballot_sync(0xFFFFFFFFu, last);
        if (last) sm.pend_gt[__popc(lm & ((1u << lane) - 1u))] = gt;
        if (lane == 0) sm.n_pend = __popc(lm);
    }
    __syncthreads();
    const int n_pend = sm.n_pend;
    for (int i = 0; i < n_pend; ++i) {
        const Unit u = find_unit<TILE>(sm.prefix, sm.lens, B, p.Hkv, sm.pend_gt[i]);
        combine_partials<128, NT, kThreads, 0>(p, sm.comb, u, T, N, partial_slot_floats(p.g, 128), tid,
                                               warp, lane);
        if (tid == 0) atomicExch(&p.counters[(int64_t)u.b * p.Hkv + u.h], 0);
    }
}

template <int NT>
cudaError_t launch_tc(const Params& p, int grid, cudaStream_t stream) {
    auto kern = decode_attention_tc_kernel<NT>;
    const int smem = (int)sizeof(Smem<NT>) + 1024;   // + alignment slack
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

}  // namespace

cudaError_t launch_decode_attention_tc(const attn::Params& p, int sms, cudaStream_t stream) {
    return p.g > 8 ? launch_tc<2>(p, sms, stream) : launch_tc<1>(p, sms, stream);
}

}  // namespace nvfp4kv

// nvfp4kv_attention_common.cuh -- pieces shared by the decode-attention
// kernels: launch parameters, the stream-K split of the (sequence, KV head,
// tile) list over CTAs, the bulk copies of one tile, and the merge of units
// split between CTAs.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "nvfp4kv_device.cuh"
#include "nvfp4kv_internal.h"

namespace nvfp4kv {
namespace attn {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleSlack = 8.0f;  // log2 units: the running max is raised only past this

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
    // paged cache (block_table != nullptr): token t of sequence b sits in page
    // block_table[b * max_pages + t / page_tokens], slot t % page_tokens, of a
    // pool laid out [page][Hkv][page_tokens][...]; S_max = max_pages * page_tokens
    const int32_t* block_table;
    int page_tokens, max_pages, num_pages;
    // sleeping polls (each up to 20 us) after which a pipeline wait of the
    // tensor-core kernel gives up and reports NVFP4_ERR_TIMEOUT
    uint32_t wait_polls;
    // append + attention: with len_from_start the attention covers
    // start_pos[b] + 1 tokens (seq_lens is not read); with x_k_new != nullptr
    // as well (tensor-core kernel, contiguous planes) the kernel itself first
    // quantizes one new token per sequence, x_k_new / x_v_new [B][1][Hkv][D]
    // (bf16, or fp32 when x_f32), into slot start_pos[b] of the K and V planes
    // (new_lens, if given, receives start_pos[b] + 1)
    int len_from_start;
    const void* x_k_new;
    const void* x_v_new;
    const int32_t* start_pos;
    int32_t* new_lens;
    int x_f32;
};

// Tokens to attend for sequence b: seq_lens[b], or start_pos[b] + 1 after an
// append; clamped to [0, S_max] (the caller reports past-capacity).
__device__ __forceinline__ int attended_len(const Params& p, int b, bool* out_of_range) {
    const int L = p.len_from_start ? p.start_pos[b] + 1 : p.seq_lens[b];
    const bool bad = L < 0 || L > p.S_max || (p.len_from_start && L < 1);
    if (out_of_range) *out_of_range = bad;
    return L < 0 ? 0 : (L > p.S_max ? p.S_max : L);
}

// Global tile index -> (sequence, head, first tile of the unit, length).
struct Unit {
    int b, h, L, ntb;
    int64_t U0, U1;  // global tile range of the unit
};

template <int TILE = kTile>
__host__ __device__ __forceinline__ Unit find_unit(const int32_t* prefix, const int32_t* lens, int B, int Hkv,
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
    // r < H_kv * ntb <= the launch's tile count < 2^31: a 32-bit division
    // (a 64-bit one is a long software routine)
    const uint32_t r = (uint32_t)(gt - prefix[lo]);
    u.h = (int)(r / (uint32_t)u.ntb);
    u.U0 = prefix[lo] + (int64_t)u.h * u.ntb;
    u.U1 = u.U0 + u.ntb;
    (void)Hkv;
    return u;
}

// floor(a / n) for 0 <= a < 2^53 and 0 < n < 2^53.  The correctly rounded
// double quotient is within one of the exact one (its error is below
// a / n * 2^-53 < 1), and one integer step each way fixes it.  This replaces
// the software routine of a 64-bit integer division, which costs a few
// hundred cycles.
__host__ __device__ __forceinline__ int64_t div_floor(int64_t a, int64_t n) {
    int64_t q = (int64_t)((double)a / (double)n);
    if (q * n > a) {
        --q;
    } else if ((q + 1) * n <= a) {
        ++q;
    }
    return q;
}

// CTA c owns global tiles [range_start(c), range_start(c + 1)).
// (c <= N < 2^16 and T < 2^31, so c * T < 2^47.)
__host__ __device__ __forceinline__ int64_t range_start(int64_t c, int64_t T, int64_t N) {
    return div_floor(c * T, N);
}

// CTA owning global tile t when T tiles are cut into N equal ranges.
__host__ __device__ __forceinline__ int64_t cta_of(int64_t t, int64_t T, int64_t N) {
    return div_floor((t + 1) * N - 1, T);
}

// Partial-result slot of CTA cc for a unit starting at global tile U0: a CTA
// can share at most two units with other CTAs -- the one holding its first
// tile (slot 2cc) and the one holding its last tile (slot 2cc + 1).
__host__ __device__ __forceinline__ int64_t partial_slot(int64_t cc, int64_t U0, int64_t T, int64_t N) {
    return (U0 <= range_start(cc, T, N)) ? 2 * cc : 2 * cc + 1;
}

// Issue the bulk copies of one tile into a ring stage (one lane).
// Stage layout: K codes [TILE][D/2], V codes [TILE][D/2], K scales
// [TILE][D/16], V scales [TILE][D/16].  Only the tokens below the sequence
// length are copied (rounded up to 4 so every copy is a multiple of 16 bytes).
template <int D, int TILE = kTile>
__device__ __forceinline__ void issue_tile(const Params& p, const Unit& u, int64_t gt, uint8_t* stage,
                                           uint64_t* bar) {
    constexpr int KB = D / 2, SB = D / 16;   // code / scale bytes per token
    constexpr int OFF_VC = TILE * KB;
    constexpr int OFF_KS = 2 * TILE * KB;
    constexpr int OFF_VS = 2 * TILE * KB + TILE * SB;
    const int t0 = (int)(gt - u.U0) * TILE;
    int n = u.L - t0;
    n = n < 0 ? 0 : (n > TILE ? TILE : n);
    const int ncopy = (n + 3) & ~3;  // keeps every copy a multiple of 16 bytes
    const uint32_t code_bytes = (uint32_t)ncopy * KB;
    const uint32_t scale_bytes = (uint32_t)ncopy * SB;
    mbar_arrive_expect_tx(bar, 2 * (code_bytes + scale_bytes));
    if (ncopy > 0) {
        int64_t tok;
        if (p.block_table == nullptr) {
            tok = ((int64_t)u.b * p.Hkv + u.h) * p.S_max + t0;
        } else {
            // a tile never straddles two pages (page_tokens is a multiple of
            // 128, a multiple of every tile size); an entry outside the pool is
            // reported and read from page 0, so no copy leaves the pool
            int page = __ldg(p.block_table + (int64_t)u.b * p.max_pages + t0 / p.page_tokens);
            if (page < 0 || page >= p.num_pages) {
                report(p.status, NVFP4_ERR_INVALID_ARG);
                page = 0;
            }
            tok = ((int64_t)page * p.Hkv + u.h) * p.page_tokens + t0 % p.page_tokens;
        }
        bulk_g2s(stage, p.kc + tok * KB, code_bytes, bar);
        bulk_g2s(stage + OFF_VC, p.vc + tok * KB, code_bytes, bar);
        bulk_g2s(stage + OFF_KS, p.ks + tok * SB, scale_bytes, bar);
        bulk_g2s(stage + OFF_VS, p.vs + tok * SB, scale_bytes, bar);
    }
}

__device__ __forceinline__ uint32_t pow2_bits(int e) {  // 2^e as fp32 bits, e in [-126, 127]
    return (uint32_t)(127 + e) << 23;
}

// Barrier over a group of THREADS threads: named barrier BAR, or the whole CTA
// when BAR is 0.
template <int THREADS, int BAR>
__device__ __forceinline__ void group_sync() {
    if constexpr (BAR == 0) {
        __syncthreads();
    } else {
        asm volatile("bar.sync %0, %1;" ::"n"(BAR), "n"(THREADS) : "memory");
    }
}

// scratch of the split-K merge (see combine_partials)
struct CombineSmem {
    float w[16][32];          // w_j = 2^(m_j - M) of chunk contributor j for query q
    float L[16];              // sum_j w_j l_j over every contributor
};

// Number of CTAs holding a partial of the unit of global tiles [U0, U1).
// With T >= N every range is non-empty, so each CTA from cta_of(U0) to
// cta_of(U1 - 1) holds one; with T < N a non-empty range is a single tile,
// so there is one CTA per tile.  (No loop over CTAs: a 64-bit division costs
// a few hundred cycles, and the count sits on the critical path of the merge.)
__host__ __device__ __forceinline__ int unit_contributors(int64_t U0, int64_t U1, int64_t T, int64_t N) {
    return T >= N ? (int)(cta_of(U1 - 1, T, N) - cta_of(U0, T, N) + 1) : (int)(U1 - U0);
}

// Partial slot of contributor j (in CTA order) of the unit starting at global
// tile U0, whose first contributor is CTA c_first.  dense: T >= N (every CTA
// range non-empty, contributors are consecutive CTAs); first_odd: the unit
// starts inside c_first's range, so that CTA stored it as its second unit.
// The writer of the partial uses partial_slot(); both must agree.
__host__ __device__ __forceinline__ int64_t contributor_slot(int j, int64_t U0, int64_t c_first,
                                                             bool first_odd, bool dense, int64_t T,
                                                             int64_t N) {
    const int64_t cc = dense ? c_first + j : cta_of(U0 + j, T, N);
    return 2 * cc + ((j == 0 && first_odd) ? 1 : 0);
}

// Count one CTA's arrival at a split unit.  The CTA's partial stores are
// ordered before this by a CTA barrier; the release half of the atomic
// publishes them (it is cumulative over the barrier), and its acquire half
// makes the other contributors' stores visible to a CTA that arrives last,
// once a second CTA barrier follows.  One atomic per CTA replaces a fence on
// every thread: a sequentially consistent GPU fence costs about a
// microsecond, and they do not overlap.
__device__ __forceinline__ int arrive_split_unit(int32_t* counter) {
    int prev;
    asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], 1;" : "=r"(prev) : "l"(counter) : "memory");
    return prev;
}

// ---------------------------------------------------------------------------
// Split-K merge of one (sequence, KV head) unit by the last CTA to finish with
// it.  Contributor j (0 <= j < unit_contributors) left (m, l, O) per query in
// its partial slot.  Out = sum_j w_j O_j / sum_j w_j l_j with
// w_j = 2^(m_j - M), M = max_j m_j.
//
// The partials sit in L2, so the merge is a handful of L2 round trips:
// every thread issues its float4 loads of the first batch of O partials at
// once, together with the (m, l) loads (warp q, lane j: query q of
// contributor j), and only then waits.  Contributors are taken 32 at a time
// (one lane each); a thread keeps up to 16 O loads in flight.
// The merge runs on a group of THREADS threads (tid, warp, lane relative to
// the group) that synchronizes on named barrier BAR (0: the whole CTA).
// ---------------------------------------------------------------------------
template <int D, int NT, int THREADS, int BAR = 0>
__device__ __noinline__ void combine_partials(const Params& p, CombineSmem& cs, const Unit& u,
                                                 int64_t T, int64_t N, int64_t slot_floats, int tid,
                                                 int warp, int lane) {
    constexpr int kQ = 8 * NT;                                    // g <= kQ
    constexpr int kWarps = THREADS / 32;
    constexpr int kQW = (kQ + kWarps - 1) / kWarps;               // queries per warp
    constexpr int kOut4 = (kQ * D / 4 + THREADS - 1) / THREADS;   // float4 outputs per thread
    constexpr int kBatch = kOut4 >= 4 ? 4 : 16 / kOut4;          // contributors per batch of loads
    const int g = p.g;
    const int n4 = g * D / 4;                        // float4 outputs of the unit
    const bool dense = T >= N;                       // every CTA range non-empty
    const int64_t c_first = cta_of(u.U0, T, N);
    const int ncc = unit_contributors(u.U0, u.U1, T, N);
    // the first contributor's slot is odd when the unit starts inside its range
    const bool first_odd = range_start(c_first, T, N) < u.U0;
    auto part_of = [&](int j) -> const float* {
        return p.partials + contributor_slot(j, u.U0, c_first, first_odd, dense, T, N) * slot_floats;
    };
    float4 acc[kOut4];
    float4 v[kOut4][kBatch];
#pragma unroll
    for (int k = 0; k < kOut4; ++k) acc[k] = make_float4(0.f, 0.f, 0.f, 0.f);
    // O loads of contributors j0 .. j0 + kBatch - 1 (those below jlim)
    auto issue = [&](int j0, int jlim) {
#pragma unroll
        for (int k = 0; k < kOut4; ++k) {
            const int i4 = tid + k * THREADS;
#pragma unroll
            for (int jj = 0; jj < kBatch; ++jj) {
                const int j = j0 + jj;
                v[k][jj] = (j < jlim && i4 < n4)
                               ? __ldcg(reinterpret_cast<const float4*>(part_of(j)) + i4)
                               : make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
    };
    // weighted sum of the batch; w of chunk position jc0 + jj
    auto consume = [&](int jc0) {
#pragma unroll
        for (int k = 0; k < kOut4; ++k) {
            const int i4 = tid + k * THREADS;
            const int q = i4 < n4 ? (i4 * 4) / D : 0;
#pragma unroll
            for (int jj = 0; jj < kBatch; ++jj) {
                const float w = (jc0 + jj < 32) ? cs.w[q][jc0 + jj] : 0.0f;
                acc[k].x = fmaf(w, v[k][jj].x, acc[k].x);
                acc[k].y = fmaf(w, v[k][jj].y, acc[k].y);
                acc[k].z = fmaf(w, v[k][jj].z, acc[k].z);
                acc[k].w = fmaf(w, v[k][jj].w, acc[k].w);
            }
        }
    };
    const int nj0 = ncc < 32 ? ncc : 32;
    issue(0, nj0);                                   // in flight with the (m, l) loads below

    // M per query (warp-uniform); the first chunk's (m, l) stay in registers
    float Mq[kQW], m0[kQW], l0[kQW], Lq[kQW];
#pragma unroll
    for (int qi = 0; qi < kQW; ++qi) {
        const int q = warp + qi * kWarps;
        Mq[qi] = -INFINITY;
        m0[qi] = -INFINITY;
        l0[qi] = 0.0f;
        Lq[qi] = 0.0f;
        if (q < g) {
            for (int base = 0; base < ncc; base += 32) {
                const int j = base + lane;
                float m = -INFINITY, l = 0.0f;
                if (j < ncc) {
                    const float* pp = part_of(j);
                    m = __ldcg(pp + g * D + q);
                    l = __ldcg(pp + g * D + g + q);
                }
                if (base == 0) {
                    m0[qi] = m;
                    l0[qi] = l;
                }
                Mq[qi] = fmaxf(Mq[qi], m);
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) Mq[qi] = fmaxf(Mq[qi], __shfl_xor_sync(0xFFFFFFFFu, Mq[qi], o));
        }
    }

    for (int base = 0; base < ncc; base += 32) {
        const int nj = ncc - base < 32 ? ncc - base : 32;
        if (base > 0) group_sync<THREADS, BAR>();   // the previous chunk's weights are consumed
#pragma unroll
        for (int qi = 0; qi < kQW; ++qi) {
            const int q = warp + qi * kWarps;
            if (q < g) {
                float m = m0[qi], l = l0[qi];
                if (base > 0) {
                    m = -INFINITY;
                    l = 0.0f;
                    if (lane < nj) {
                        const float* pp = part_of(base + lane);
                        m = __ldcg(pp + g * D + q);
                        l = __ldcg(pp + g * D + g + q);
                    }
                }
                const float w = (m == -INFINITY) ? 0.0f : fast_exp2(m - Mq[qi]);
                float wl = w * l;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) wl += __shfl_xor_sync(0xFFFFFFFFu, wl, o);
                Lq[qi] += wl;
                cs.w[q][lane] = w;
            }
        }
        group_sync<THREADS, BAR>();
        for (int j0 = 0; j0 < nj; j0 += kBatch) {
            if (base > 0 || j0 > 0) issue(base + j0, base + nj);
            consume(j0);
        }
    }
#pragma unroll
    for (int qi = 0; qi < kQW; ++qi) {
        const int q = warp + qi * kWarps;
        if (q < g && lane == 0) cs.L[q] = Lq[qi];
    }
    group_sync<THREADS, BAR>();
#pragma unroll
    for (int k = 0; k < kOut4; ++k) {
        const int i4 = tid + k * THREADS;
        if (i4 < n4) {
            const int q = (i4 * 4) / D;
            const float L = cs.L[q];
            const float4 a = acc[k];
            const float4 o = L > 0.0f ? make_float4(a.x / L, a.y / L, a.z / L, a.w / L)
                                      : make_float4(0.f, 0.f, 0.f, 0.f);
            float* dst = p.out + ((int64_t)u.b * p.Hq + (int64_t)u.h * g) * D + (int64_t)i4 * 4;
            *reinterpret_cast<float4*>(dst) = o;
        }
    }
}

}  // namespace attn

// Launch of the tensor-core (tcgen05) kernel for head_dim 128 and bf16
// queries; grid = one CTA per SM.
cudaError_t launch_decode_attention_tc(const attn::Params& p, int sms, cudaStream_t stream);

}  // namespace nvfp4kv

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
        const int64_t tok = ((int64_t)u.b * p.Hkv + u.h) * p.S_max + t0;
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
    int32_t slot[32];         // partial slot of chunk contributor j, -1 if none
    float m[16][32];          // running max m_j of contributor j for query q
    float l[16][32];          // l_j, then w_j = 2^(m_j - M) once M is known
    float M[16];
    float L[16];
};

// ---------------------------------------------------------------------------
// Split-K merge of one (sequence, KV head) unit by the last CTA to finish with
// it.  The contributors are CTAs c_first..c_last (those with non-empty ranges);
// each left (m, l, O) per query in its partial slot.  Out = sum_c w_c O_c /
// sum_c w_c l_c with w_c = 2^(m_c - M), M = max_c m_c.
//
// The partials sit in L2; the merge is written so that every load of a round
// is independent (one L2 latency per round, not one per contributor):
// contributors are taken 32 at a time; their (m, l) pairs are fetched by all
// threads at once into shared memory, and each thread then loads float4
// slices of the O partials of up to 16 contributors per batch.
// The merge runs on a group of THREADS threads (tid, warp, lane relative to
// the group) that synchronizes on named barrier BAR (0: the whole CTA).
// ---------------------------------------------------------------------------
template <int D, int NT, int THREADS, int BAR = 0>
__device__ __noinline__ void combine_partials(const Params& p, CombineSmem& cs, const Unit& u,
                                                 int64_t T, int64_t N, int64_t c_first,
                                                 int64_t c_last, int64_t slot_floats, int tid,
                                                 int warp, int lane) {
    constexpr int kQ = 8 * NT;                       // g <= kQ
    constexpr int kOut4 = (kQ * D / 4 + THREADS - 1) / THREADS;   // float4 outputs per thread
    constexpr int kBatch = kOut4 >= 4 ? 4 : 16 / kOut4;          // contributors per batch of loads
    const int g = p.g;
    const int n4 = g * D / 4;                        // float4 outputs of the unit
    const int ncc = (int)(c_last - c_first + 1);
    float4 acc[kOut4];
#pragma unroll
    for (int k = 0; k < kOut4; ++k) acc[k] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (tid < kQ) {
        cs.M[tid] = -INFINITY;
        cs.L[tid] = 0.0f;
    }
    // one chunk of up to 32 contributors: slots, then (m, l) of every query
    auto load_chunk = [&](int base) {
        group_sync<THREADS, BAR>();
        if (warp == 0) {
            int sl = -1;
            if (base + lane < ncc) {
                const int64_t cc = c_first + base + lane;
                if (range_start(cc, T, N) < range_start(cc + 1, T, N))
                    sl = (int)partial_slot(cc, u.U0, T, N);
            }
            cs.slot[lane] = sl;
        }
        group_sync<THREADS, BAR>();
        for (int i = tid; i < 32 * kQ; i += THREADS) {
            const int j = i & 31, q = i >> 5;
            const int sl = cs.slot[j];
            float m = -INFINITY, l = 0.0f;
            if (sl >= 0 && q < g) {
                const float* part = p.partials + (int64_t)sl * slot_floats;
                m = __ldcg(part + g * D + q);
                l = __ldcg(part + g * D + g + q);
            }
            cs.m[q][j] = m;
            cs.l[q][j] = l;
        }
        group_sync<THREADS, BAR>();
    };
    // pass 1: M = max over every contributor
    for (int base = 0; base < ncc; base += 32) {
        load_chunk(base);
        if (tid < g) {
            float mx = cs.M[tid];
            for (int j = 0; j < 32; ++j) mx = fmaxf(mx, cs.m[tid][j]);
            cs.M[tid] = mx;
        }
    }
    // pass 2: weights, L and the weighted sum of the O partials
    for (int base = 0; base < ncc; base += 32) {
        if (ncc > 32) load_chunk(base);      // a single chunk is still in place
        group_sync<THREADS, BAR>();
        if (tid < g) {
            const float M = cs.M[tid];
            float lsum = cs.L[tid];
            for (int j = 0; j < 32; ++j) {
                const float mj = cs.m[tid][j];
                const float w = (mj == -INFINITY) ? 0.0f : fast_exp2(mj - M);
                lsum += w * cs.l[tid][j];
                cs.l[tid][j] = w;                // l is replaced by the weight
            }
            cs.L[tid] = lsum;
        }
        group_sync<THREADS, BAR>();
        const int nj = ncc - base < 32 ? ncc - base : 32;
        for (int j0 = 0; j0 < nj; j0 += kBatch) {
            float4 v[kOut4][kBatch];
            float w[kOut4][kBatch];
#pragma unroll
            for (int k = 0; k < kOut4; ++k) {          // every load of the batch in flight at once
                const int i4 = tid + k * THREADS;
                const int q = i4 < n4 ? (i4 * 4) / D : 0;
#pragma unroll
                for (int jj = 0; jj < kBatch; ++jj) {
                    const int j = j0 + jj;
                    const int sl = (j < nj && i4 < n4) ? cs.slot[j] : -1;
                    w[k][jj] = sl >= 0 ? cs.l[q][j] : 0.0f;
                    v[k][jj] = sl >= 0 ? __ldcg(reinterpret_cast<const float4*>(
                                             p.partials + (int64_t)sl * slot_floats) + i4)
                                       : make_float4(0.f, 0.f, 0.f, 0.f);
                }
            }
#pragma unroll
            for (int k = 0; k < kOut4; ++k)
#pragma unroll
                for (int jj = 0; jj < kBatch; ++jj) {
                    acc[k].x = fmaf(w[k][jj], v[k][jj].x, acc[k].x);
                    acc[k].y = fmaf(w[k][jj], v[k][jj].y, acc[k].y);
                    acc[k].z = fmaf(w[k][jj], v[k][jj].z, acc[k].z);
                    acc[k].w = fmaf(w[k][jj], v[k][jj].w, acc[k].w);
                }
        }
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

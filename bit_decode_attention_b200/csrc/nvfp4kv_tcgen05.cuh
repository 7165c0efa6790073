// nvfp4kv_tcgen05.cuh -- thin wrappers for the sm_100a fifth-generation
// tensor core instructions (tcgen05.*) used by the decode-attention kernel:
// tensor-memory allocation, register <-> tensor-memory moves, FP8 (E4M3)
// MMAs with operands in shared or tensor memory, and their completion.
//
// Tensor-memory addresses: bits 31..16 lane, bits 15..0 column (32-bit
// columns).  A warp may only touch lanes 32*(warp % 4) .. +31.
//
// Shared-memory matrix descriptors here use the non-swizzled canonical
// layouts, built from 8 x 16-byte "core matrices" (128 contiguous bytes):
//   K-major  (rows = M or N, 16-byte chunks along K):
//     byte(r, k) = (r / 8) * SBO + (k / 16) * LBO + (r % 8) * 16 + k % 16
//   MN-major (rows = K, 16-byte chunks along M or N):
//     byte(mn, k) = (mn / 16) * SBO + (k / 8) * LBO + (k % 8) * 16 + mn % 16
#pragma once

#include <cstdint>

namespace nvfp4kv {
namespace tc {

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---- tensor memory allocation (whole warp) ----
__device__ __forceinline__ void tmem_alloc(uint32_t* smem_result, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr(smem_result)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

// ---- ordering of tcgen05 operations around thread synchronization ----
__device__ __forceinline__ void fence_before_sync() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_after_sync() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// ---- registers <-> tensor memory, 32 lanes x 32 bits, N columns ----
__device__ __forceinline__ void tmem_st_x8(uint32_t taddr, const uint32_t* r) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
        : "memory");
}
__device__ __forceinline__ void tmem_st_x32(uint32_t taddr, const uint32_t* r) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, "
        "%29, %30, %31, %32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
        "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
        "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}
__device__ __forceinline__ void tmem_st_x4(uint32_t taddr, const uint32_t* r) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1, %2, %3, %4};" ::"r"(taddr), "r"(r[0]),
                 "r"(r[1]), "r"(r[2]), "r"(r[3])
                 : "memory");
}
__device__ __forceinline__ void tmem_ld_x4(uint32_t taddr, uint32_t* r) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(taddr)
                 : "memory");
}
__device__ __forceinline__ void tmem_ld_x8(uint32_t taddr, uint32_t* r) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                   "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr)
                 : "memory");
}
__device__ __forceinline__ void tmem_ld_x16(uint32_t taddr, uint32_t* r) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
        "%12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_ld() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// ---- descriptors ----
// Instruction descriptor for kind::f8f6f4 with E4M3 A and B, fp32 D.
__host__ __device__ constexpr uint32_t idesc_e4m3(int M, int N, bool a_mn_major, bool b_mn_major,
                                                  bool negate_b) {
    return (1u << 4)                                   // D format: F32
           | (0u << 7) | (0u << 10)                    // A, B format: E4M3
           | ((negate_b ? 1u : 0u) << 14)              // negate B
           | ((a_mn_major ? 1u : 0u) << 15)            // A major-ness
           | ((b_mn_major ? 1u : 0u) << 16)            // B major-ness
           | ((uint32_t)(N >> 3) << 17)                // N / 8
           | ((uint32_t)(M >> 4) << 24);               // M / 16
}

// Shared-memory matrix descriptor, non-swizzled canonical layout (see top).
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);          // start address, bits 0..13
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;       // leading byte offset, bits 16..29
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;       // stride byte offset, bits 32..45
    d |= (uint64_t)1u << 46;                           // descriptor version (sm_100)
    return d;                                          // base offset 0, no swizzle
}

// ---- MMAs (issued by one thread) ----
// D(tmem) (+)= A(tmem) * B(smem)
__device__ __forceinline__ void mma_e4m3_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                            uint32_t idesc, bool accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate ? 1u : 0u)
        : "memory");
}
// D(tmem) (+)= A(smem) * B(smem)
__device__ __forceinline__ void mma_e4m3_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                            uint32_t idesc, bool accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate ? 1u : 0u)
        : "memory");
}
// Four MMAs accumulating into one D and the commit that signals their
// completion, in one instruction sequence (separate asm statements per MMA
// cost several times more issue cycles: each moves its operands into uniform
// registers on its own).  D(tmem) (+)= A_k(tmem) * B_k(smem) for k = 0..3,
// A_k at column a + 8k (K = 32 FP8 bytes each), B_k = b[k]; the first MMA
// accumulates only when `acc` is non-zero; then one arrive on `bar` when all
// MMAs this thread issued so far have completed.
__device__ __forceinline__ void mma4_ts_commit(uint32_t d, uint32_t a, const uint64_t (&b)[4], uint32_t idesc,
                                               uint32_t acc, uint64_t* bar) {
    asm volatile(
        "{\n\t.reg .pred p0, p1;\n\t"
        "setp.ne.b32 p0, %9, 0;\n\t"
        "setp.eq.b32 p1, %9, %9;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %5, %10, p0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%2], %6, %10, p1;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%3], %7, %10, p1;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%4], %8, %10, p1;\n\t"
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%11];\n\t}"
        ::"r"(d), "r"(a), "r"(a + 8), "r"(a + 16), "r"(a + 24), "l"(b[0]), "l"(b[1]), "l"(b[2]), "l"(b[3]),
          "r"(acc), "r"(idesc), "r"(smem_addr(bar))
        : "memory");
}
// The same with A from shared memory: D(tmem) (+)= A_k(smem) * B_k(smem).
__device__ __forceinline__ void mma4_ss_commit(uint32_t d, const uint64_t (&a)[4], const uint64_t (&b)[4],
                                               uint32_t idesc, uint32_t acc, uint64_t* bar) {
    asm volatile(
        "{\n\t.reg .pred p0, p1;\n\t"
        "setp.ne.b32 p0, %9, 0;\n\t"
        "setp.eq.b32 p1, %9, %9;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %5, %10, p0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %2, %6, %10, p1;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %3, %7, %10, p1;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %4, %8, %10, p1;\n\t"
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%11];\n\t}"
        ::"r"(d), "l"(a[0]), "l"(a[1]), "l"(a[2]), "l"(a[3]), "l"(b[0]), "l"(b[1]), "l"(b[2]), "l"(b[3]),
          "r"(acc), "r"(idesc), "r"(smem_addr(bar))
        : "memory");
}

// One lane of the (converged) warp: true in exactly one lane.
__device__ __forceinline__ bool elect_one() {
    uint32_t pred = 0;
    asm volatile(
        "{\n\t.reg .pred p;\n\telect.sync _|p, 0xffffffff;\n\tselp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(pred));
    return pred != 0;
}

// Arrive once on the mbarrier when every MMA this thread issued so far has completed.
__device__ __forceinline__ void mma_commit(uint64_t* mbar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_addr(mbar))
                 : "memory");
}

}  // namespace tc
}  // namespace nvfp4kv

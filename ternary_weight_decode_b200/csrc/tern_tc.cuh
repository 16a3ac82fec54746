// tern_tc.cuh -- 5th-generation tensor-core (tcgen05) helpers for sm_100a:
// tensor-memory allocation, register <-> tensor-memory moves, the int8 MMA
// with A in tensor memory or shared memory and B in shared memory, commit to
// an mbarrier, and the descriptors these instructions take.
//
// Conventions used throughout libtern:
//  * cta_group::1, M = 128: tensor-memory lane i holds row i of A and of the
//    accumulator D.  A 32-bit tensor-memory column holds 4 consecutive 8-bit
//    K elements (A) or one int32 accumulator (D).  Warp w of a warpgroup
//    reaches lanes 32*(w%4) .. 32*(w%4)+31.
//  * B (N x K, 8-bit) sits in shared memory K-major without swizzle, as
//    "core matrices" of 8 rows x 16 bytes (128 contiguous bytes, rows 16 B
//    apart).  Core matrices adjacent along K are LBO bytes apart, along N
//    SBO bytes apart.
#pragma once

#include <stdint.h>

#include "tern_common.cuh"

namespace tern {

// ---------------------------------------------------------------- allocation
// Warp-collective: allocates `ncols` (power of two, 32..512) tensor-memory
// columns and writes their base address to *dst (shared memory).
__device__ __forceinline__ void tmem_alloc(uint32_t *dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(dst)),
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

// ---------------------------------------------------------------- fences
__device__ __forceinline__ void tc_fence_before_sync() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after_sync() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// ---------------------------------------------------------------- st / ld
// Lane (taddr.lane + laneid) of the warp's quarter, 8 consecutive columns.
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&v)[8]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
        : "memory");
}

__device__ __forceinline__ void tmem_st2(uint32_t taddr, uint32_t a, uint32_t b) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x2.b32 [%0], {%1, %2};" ::"r"(taddr), "r"(a), "r"(b)
                 : "memory");
}

__device__ __forceinline__ void tmem_wait_st() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_ld2(uint32_t taddr, uint32_t &a, uint32_t &b) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x2.b32 {%0, %1}, [%2];"
                 : "=r"(a), "=r"(b)
                 : "r"(taddr)
                 : "memory");
}

__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t (&v)[8]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]),
                   "=r"(v[6]), "=r"(v[7])
                 : "r"(taddr)
                 : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}


__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
        : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
                 : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
                 : "r"(taddr)
                 : "memory");
}

__device__ __forceinline__ void tmem_ld4(uint32_t taddr, uint32_t (&v)[4]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3])
                 : "r"(taddr)
                 : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
        "%12, %13, %14, %15}, [%16];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
          "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]),
          "=r"(v[14]), "=r"(v[15])
        : "r"(taddr)
        : "memory");
}

// Reads the first NR (<= 32) accumulator columns of this thread's lane.
template <int NR>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t (&v)[NR]) {
    if constexpr (NR == 1) {
        uint32_t b;
        tmem_ld2(taddr, v[0], b);
    } else if constexpr (NR == 2) {
        tmem_ld2(taddr, v[0], v[1]);
    } else if constexpr (NR <= 4) {
        uint32_t t[4];
        tmem_ld4(taddr, t);
#pragma unroll
        for (int i = 0; i < NR; ++i) v[i] = t[i];
    } else if constexpr (NR <= 8) {
        uint32_t t[8];
        tmem_ld8(taddr, t);
#pragma unroll
        for (int i = 0; i < NR; ++i) v[i] = t[i];
    } else if constexpr (NR <= 16) {
        uint32_t t[16];
        tmem_ld16(taddr, t);
#pragma unroll
        for (int i = 0; i < NR; ++i) v[i] = t[i];
    } else {
        uint32_t t[32];
        tmem_ld32(taddr, t);
#pragma unroll
        for (int i = 0; i < NR; ++i) v[i] = t[i];
    }
}

// Named barrier over the 128 threads of one warpgroup (id 0 is __syncthreads).
__device__ __forceinline__ void warpgroup_sync(int id) {
    asm volatile("bar.sync %0, 128;" ::"r"(id) : "memory");
}

// ---------------------------------------------------------------- descriptors
// Instruction descriptor of a dense kind::i8 MMA with an int32 accumulator,
// A and B K-major.  a_signed / b_signed select s8 (1) or u8 (0).
//   bits [4,6) accumulator format (2 = s32), [7,10) A format, [10,13) B format,
//   bit 15 / 16 A / B major (0 = K), [17,23) N >> 3, [24,29) M >> 4.
__host__ __device__ constexpr uint32_t idesc_i8(int M, int N, int a_signed, int b_signed) {
    return (2u << 4) | (static_cast<uint32_t>(a_signed) << 7) |
           (static_cast<uint32_t>(b_signed) << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
           (static_cast<uint32_t>(M >> 4) << 24);
}

// Shared-memory matrix descriptor, no swizzle:
//   bits [0,14) start address >> 4, [16,30) LBO >> 4, [32,46) SBO >> 4,
//   [46,48) = 1 (descriptor version), [61,64) = 0 (no swizzle).
__device__ __forceinline__ uint64_t smem_desc_noswizzle(uint32_t saddr, uint32_t lbo,
                                                        uint32_t sbo) {
    return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) |
           (static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16) |
           (static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46);
}

// Shared-memory matrix descriptor, K-major with 128-byte swizzle: rows of
// 128 bytes (128 8-bit K elements), 16-byte chunk c of row r stored at chunk
// c ^ (r % 8) (the pattern TMA writes with CU_TENSOR_MAP_SWIZZLE_128B), 8-row
// groups 1024 bytes apart (SBO); the tile base 1024-byte aligned.  Steps of
// 32 K elements inside the 128-byte row advance the start address by 32.
//   layout type [61,64) = 2 (128-byte swizzle), LBO unused (16).
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr) {
    return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) | (static_cast<uint64_t>(1u) << 16) |
           (static_cast<uint64_t>(1024u >> 4) << 32) | (1ull << 46) | (2ull << 61);
}

// Byte offset of element (r, k) (k < 128) in a 128-byte-swizzled K-major tile.
__host__ __device__ constexpr uint32_t sw128_offset(uint32_t r, uint32_t k) {
    return r * 128u + ((((k >> 4) ^ (r & 7u)) & 7u) << 4) + (k & 15u);
}

// ---------------------------------------------------------------- MMA
// D[tmem] (+)= A[tmem] * B[smem]^T, issued by one thread.
__device__ __forceinline__ void mma_i8_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.u32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, issued by one thread.
__device__ __forceinline__ void mma_i8_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.u32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem), "l"(a_desc),
        "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrives once on `bar` when every tcgen05 operation this thread issued so
// far has completed.
__device__ __forceinline__ void tc_commit(uint64_t *bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
            smem_u32(bar))
        : "memory");
}

// Byte offset of element (n, k) of an N x K (8-bit) operand in the no-swizzle
// K-major core-matrix layout with LBO = (N/8)*128 and SBO = 128.
__host__ __device__ constexpr uint32_t core_offset(uint32_t n, uint32_t k, uint32_t N) {
    return (k >> 4) * (N >> 3) * 128u + (n >> 3) * 128u + (n & 7u) * 16u + (k & 15u);
}

}  // namespace tern

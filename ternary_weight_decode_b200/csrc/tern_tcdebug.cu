// tern_tcdebug.cu -- test hook for the tcgen05 int8 MMA path: one CTA
// computes D = A * B^T for a 128 x K int8 A and an N x K int8 B, with A taken
// from tensor memory (written by tcgen05.st, as the decode kernels write
// their decoded operand) or from shared memory, B from shared memory in the
// no-swizzle core-matrix layout -- or (mode 2) both from shared memory in the
// 128-byte-swizzled K-major layout the prefill GEMM uses.  Used by the tests
// to pin the descriptor encodings against a plain integer product.
#include "tern_common.cuh"
#include "tern_internal.h"
#include "tern_tc.cuh"

namespace tern {

constexpr int kDbgDCol = 256;  // accumulator columns start here; A uses < 256

__global__ void __launch_bounds__(128)
    debug_mma_kernel(int a_in_smem, const int8_t *__restrict__ A, int a_signed,
                     const int8_t *__restrict__ B, int b_signed, int32_t *__restrict__ D, int K,
                     int N) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
    __shared__ uint32_t tmem_slot;
    __shared__ __align__(8) uint64_t bar;
    const int tid = threadIdx.x, warp = tid >> 5;
    uint8_t *sb = smem;                   // B: N x K
    uint8_t *sa = smem + N * K;           // A: 128 x K (shared-memory variant)

    if (warp == 0) tmem_alloc(&tmem_slot, 512);
    if (tid == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    const bool sw = a_in_smem == 2;
    // mode 2: 128-K blocks, each an [rows][128 B] swizzled tile
    for (int idx = tid; idx < N * K; idx += 128) {
        const int n = idx / K, k = idx % K;
        sb[sw ? (k >> 7) * N * 128 + sw128_offset(n, k & 127) : core_offset(n, k, N)] =
            static_cast<uint8_t>(B[idx]);
    }
    if (a_in_smem)
        for (int idx = tid; idx < 128 * K; idx += 128) {
            const int r = idx / K, k = idx % K;
            sa[sw ? (k >> 7) * 128 * 128 + sw128_offset(r, k & 127) : core_offset(r, k, 128)] =
                static_cast<uint8_t>(A[idx]);
        }
    fence_proxy_async_smem();
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tbase = tmem_slot;
    const uint32_t lane_base = static_cast<uint32_t>(32 * warp) << 16;

    if (!a_in_smem) {
        // row tid of A into tensor-memory lane tid, 4 K elements per column
        const uint32_t *arow = reinterpret_cast<const uint32_t *>(A + static_cast<int64_t>(tid) * K);
        for (int c0 = 0; c0 < K / 4; c0 += 8) {
            uint32_t v[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) v[j] = arow[c0 + j];
            tmem_st8(tbase + lane_base + c0, v);
        }
        tmem_wait_st();
    }
    tc_fence_before_sync();
    __syncthreads();

    if (tid == 0) {
        tc_fence_after_sync();
        const uint32_t idesc = idesc_i8(128, N, a_signed, b_signed);
        for (int ks = 0; ks < K / 32; ++ks) {
            if (sw) {
                const int kb = ks >> 2, kk = (ks & 3) * 32;
                const uint64_t bd = smem_desc_sw128(smem_u32(sb) + kb * N * 128 + kk);
                const uint64_t ad = smem_desc_sw128(smem_u32(sa) + kb * 128 * 128 + kk);
                mma_i8_ss(tbase + kDbgDCol, ad, bd, idesc, ks > 0);
                continue;
            }
            const uint64_t bd = smem_desc_noswizzle(smem_u32(sb) + ks * 2 * (N / 8) * 128,
                                                    (N / 8) * 128, 128);
            if (a_in_smem) {
                const uint64_t ad = smem_desc_noswizzle(smem_u32(sa) + ks * 2 * 16 * 128, 16 * 128, 128);
                mma_i8_ss(tbase + kDbgDCol, ad, bd, idesc, ks > 0);
            } else {
                mma_i8_ts(tbase + kDbgDCol, tbase + ks * 8, bd, idesc, ks > 0);
            }
        }
        tc_commit(&bar);
    }
    const bool ok = mbar_wait_bounded(&bar, 0);
    tc_fence_after_sync();
    for (int c = 0; c < N; c += 8) {
        uint32_t v[8];
        tmem_ld8(tbase + lane_base + kDbgDCol + c, v);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 8; ++j)
            D[static_cast<int64_t>(tid) * N + c + j] = ok ? static_cast<int32_t>(v[j]) : 0;
    }
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        tmem_relinquish();
        tmem_dealloc(tbase, 512);
    }
}

cudaError_t launch_debug_mma(int a_in_smem, const int8_t *A, int a_signed, const int8_t *B,
                             int b_signed, int32_t *D, int K, int N, cudaStream_t s) {
    // A fixed, generous allocation: the operands sit at its start, so a
    // misread descriptor stride still reads inside this CTA's shared memory.
    const size_t smem = 200 * 1024;
    cudaError_t e = cudaFuncSetAttribute(debug_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    debug_mma_kernel<<<1, 128, smem, s>>>(a_in_smem, A, a_signed, B, b_signed, D, K, N);
    return cudaGetLastError();
}

}  // namespace tern

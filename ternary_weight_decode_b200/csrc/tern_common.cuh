// tern_common.cuh -- device helpers shared by the sm_100a kernels of libtern:
// shared-memory addresses, mbarriers with bounded waits, TMA tile loads
// (no multicast), thread-block-cluster barriers and distributed shared
// memory, programmatic dependent launch, and the integer dot product.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace tern {

// Device error word: a bounded wait that runs out records a code here and
// the kernel carries on to a clean exit instead of hanging the GPU.
extern __device__ int g_device_error;

enum : int {
    kErrTmaTimeout = 1,
};

// Budget of a bounded wait, in SM clock cycles (about 0.5 s at 2 GHz).
constexpr long long kWaitBudgetCycles = 1000000000LL;
// Back-off between polls of a wait that is not yet satisfied (ns).
constexpr unsigned kWaitBackoffNs = 32;

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
                 : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Waits for phase `parity` of `bar` to complete, at most `budget` SM cycles.
// Returns false (and records kErrTmaTimeout) when the budget runs out.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity,
                                                  long long budget = kWaitBudgetCycles) {
    if (mbar_try_wait(bar, parity)) return true;
    long long start = clock64();
    while (!mbar_try_wait(bar, parity)) {
        __nanosleep(kWaitBackoffNs);  // leave the issue slots to warps with work
        if (clock64() - start > budget) {
            atomicExch(&g_device_error, kErrTmaTimeout);
            return false;
        }
    }
    return true;
}

// ---------------------------------------------------------------- TMA
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// A warp hands a TMA-filled shared-memory buffer back to its producer: each
// lane's reads of it (generic proxy) are ordered before the producer's next
// TMA write into it (async proxy) by a proxy fence, then one arrival on the
// buffer's empty barrier for the whole warp.  Without the fence the refill
// may land before a lane's read of the old contents.
__device__ __forceinline__ void release_to_tma(uint64_t *empty_bar, int lane) {
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(empty_bar);
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap *map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 2-D tiled TMA load of one box into this CTA's shared memory, completing
// `bytes` on `bar`.  x is the innermost (byte) coordinate.
__device__ __forceinline__ void tma_load_2d(void *smem_dst, const CUtensorMap *map, int x, int y,
                                            uint64_t *bar, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

// 3-D tiled TMA load (x innermost, bytes).
__device__ __forceinline__ void tma_load_3d(void *smem_dst, const CUtensorMap *map, int x, int y, int z,
                                            uint64_t *bar, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

// The same without a cache hint (operands that other CTAs read again).
__device__ __forceinline__ void tma_load_2d_nohint(void *smem_dst, const CUtensorMap *map, int x, int y,
                                                   uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

// L2 policy for data read exactly once (the weight stream).
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// ---------------------------------------------------------------- clusters
__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\t"
                 "barrier.cluster.wait.acquire.aligned;" ::
                     : "memory");
}

// Address of `p` (this CTA's shared memory) in the shared memory of CTA
// `rank` of the cluster.
__device__ __forceinline__ uint32_t map_shared_rank(const void *p, uint32_t rank) {
    uint32_t out;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(out) : "r"(smem_u32(p)), "r"(rank));
    return out;
}

__device__ __forceinline__ uint32_t cluster_nctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
    return r;
}

// Split cluster barrier: every thread of every CTA of the cluster arrives
// once, and may wait later.
__device__ __forceinline__ void cluster_arrive() {
    asm volatile("barrier.cluster.arrive.release;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
    asm volatile("barrier.cluster.wait.acquire;" ::: "memory");
}

// Asynchronous store of 4 / 8 bytes into the shared memory of a CTA of the
// cluster (addresses from map_shared_rank); completes the bytes on that
// CTA's mbarrier `remote_bar`.
__device__ __forceinline__ void st_async_u32(uint32_t remote_addr, uint32_t v, uint32_t remote_bar) {
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.u32 [%0], %1, [%2];" ::"r"(
                     remote_addr),
                 "r"(v), "r"(remote_bar)
                 : "memory");
}
__device__ __forceinline__ void st_async_v2f32(uint32_t remote_addr, float a, float b,
                                               uint32_t remote_bar) {
    asm volatile(
        "st.async.shared::cluster.mbarrier::complete_tx::bytes.v2.f32 [%0], {%1, %2}, [%3];" ::"r"(
            remote_addr),
        "f"(a), "f"(b), "r"(remote_bar)
        : "memory");
}

// Bulk copy of `bytes` (multiple of 16, both addresses 16-byte aligned) from
// this CTA's shared memory into the shared memory of a CTA of the cluster,
// completing the bytes on that CTA's mbarrier.  The source must have been
// made visible to the async proxy (fence_proxy_async_smem) by its writers.
__device__ __forceinline__ void bulk_copy_s2cluster(uint32_t remote_dst, const void *src,
                                                    uint32_t bytes, uint32_t remote_bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            remote_dst),
        "r"(smem_u32(src)), "r"(bytes), "r"(remote_bar)
        : "memory");
}

// 8-byte relaxed accesses at GPU scope: single-copy atomic, so a (value,
// tag) pair packed into one 64-bit word is seen whole or not at all.
__device__ __forceinline__ void st_relaxed_gpu_u64(unsigned long long *p, unsigned long long v) {
    asm volatile("st.relaxed.gpu.global.b64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ unsigned long long ld_relaxed_gpu_u64(const unsigned long long *p) {
    unsigned long long v;
    asm volatile("ld.relaxed.gpu.global.b64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

// Reads the 64-bit word at p once its tag (high half) is nonzero, waiting at
// most `budget` SM cycles for another CTA to publish it.  When the budget
// runs out it records kErrTmaTimeout and returns the word as it stands (tag
// still 0).
__device__ __forceinline__ unsigned long long wait_tagged_word(const unsigned long long *p,
                                                               long long budget = kWaitBudgetCycles) {
    unsigned long long w = ld_relaxed_gpu_u64(p);
    if ((w >> 32) != 0) return w;
    const long long start = clock64();
    while (((w = ld_relaxed_gpu_u64(p)) >> 32) == 0) {
        __nanosleep(kWaitBackoffNs);
        if (clock64() - start > budget) {
            atomicExch(&g_device_error, kErrTmaTimeout);
            break;
        }
    }
    return w;
}

// Waits (bounded, like mbar_wait_bounded) for a phase completed by other CTAs
// of the cluster, with acquire at cluster scope.
__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ bool mbar_wait_cluster_bounded(uint64_t *bar, uint32_t parity) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    long long start = clock64();
    while (!mbar_try_wait_cluster(bar, parity)) {
        __nanosleep(kWaitBackoffNs);
        if (clock64() - start > kWaitBudgetCycles) {
            atomicExch(&g_device_error, kErrTmaTimeout);
            return false;
        }
    }
    return true;
}

__device__ __forceinline__ float ld_shared_cluster_f32(uint32_t addr) {
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
    return v;
}

// ---------------------------------------------------------------- PDL
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------- integer dot
// Four u8 x s8 products summed into c (the 2-bit masked fields exceed s8).
__device__ __forceinline__ int dp4a_us(uint32_t a_u8x4, uint32_t b_s8x4, int c) {
    int d;
    asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a_u8x4), "r"(b_s8x4), "r"(c));
    return d;
}

__device__ __forceinline__ int dp4a_ss(uint32_t a, uint32_t b, int c) {
    return __dp4a(static_cast<int>(a), static_cast<int>(b), c);
}

__device__ __forceinline__ uint4 lds128(const void *p) {
    return *reinterpret_cast<const uint4 *>(p);
}

// ---------------------------------------------------------------- Hadamard
// Unnormalised 128-point Sylvester Hadamard transform of one block held by a
// warp, lane l owning elements 4l..4l+3 in r[0..3]: radix-2 butterflies
// (a, b) -> (a + b, a - b) in stage order h = 1, 2, 4, ..., 64, each output a
// single fp32 add or subtract.  Every kernel that rotates uses this routine,
// so all of them produce the same bits.
__device__ __forceinline__ void fwht128_warp(float (&r)[4], int lane) {
    float a0 = __fadd_rn(r[0], r[1]), a1 = __fsub_rn(r[0], r[1]);  // h = 1
    float a2 = __fadd_rn(r[2], r[3]), a3 = __fsub_rn(r[2], r[3]);
    r[0] = __fadd_rn(a0, a2);  // h = 2
    r[1] = __fadd_rn(a1, a3);
    r[2] = __fsub_rn(a0, a2);
    r[3] = __fsub_rn(a1, a3);
#pragma unroll
    for (int mask = 1; mask < 32; mask <<= 1) {  // h = 4 mask
        const bool upper = (lane & mask) != 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float other = __shfl_xor_sync(0xffffffffu, r[i], mask);
            r[i] = upper ? __fsub_rn(other, r[i]) : __fadd_rn(r[i], other);
        }
    }
}

// Named barrier over `count` threads (a multiple of 32; id 0 is __syncthreads).
__device__ __forceinline__ void warpgroup_sync_n(int id, int count) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ int warp_sum_int(int v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Statistics of one 128-element block (lane l holds elements 4l..4l+3):
// {max |v|, max |H v|, sum v^2}.  Feeds the fused quantisation of a
// consumer kernel, which recomputes H v with fwht128_warp bit for bit.
__device__ __forceinline__ float3 block_stats128(float (&r)[4], int lane) {
    float amax = fmaxf(fmaxf(fabsf(r[0]), fabsf(r[1])), fmaxf(fabsf(r[2]), fabsf(r[3])));
    float ss = fmaf(r[3], r[3], fmaf(r[2], r[2], fmaf(r[1], r[1], r[0] * r[0])));
    amax = warp_max(amax);
    ss = warp_sum(ss);
    fwht128_warp(r, lane);
    float amaxh = fmaxf(fmaxf(fabsf(r[0]), fabsf(r[1])), fmaxf(fabsf(r[2]), fabsf(r[3])));
    amaxh = warp_max(amaxh);
    return make_float3(amax, amaxh, ss);
}

constexpr float kInvSqrt128 = 0.0883883476483184405501f;

}  // namespace tern

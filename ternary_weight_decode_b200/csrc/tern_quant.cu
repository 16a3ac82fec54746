// tern_quant.cu -- per-token int8 activation quantisation with an optional
// 128-point Walsh-Hadamard rotation (Bonsai page, "Decode 为什么只能算一般":
// the FFN input is rotated once and shared by gate and up; activations are
// re-quantised per token between matmuls).
//
// Arithmetic (fp32, reproduced bit for bit by the CPU oracle):
//   x^ = x, or per 128-block the unnormalised Sylvester butterflies, stages
//        h = 1, 2, ..., 64, (a, b) -> (a + b, a - b);
//   amax = max |x^|, inv = 127/amax, q = clamp(rint(x^ * inv), -127, 127),
//   s_x = amax/127 (times fp32(1/sqrt(128)) when rotated).
// One CTA per token row; the row is staged in shared memory.  A warp owns a
// 128-block: lane l holds elements 4l..4l+3, so stages h = 1, 2 are local and
// h = 4..64 are butterflies across lanes l ^ (h/4).
#include "tern_common.cuh"
#include "tern_internal.h"

namespace tern {

constexpr int kQuantThreads = 512;

template <bool FP16>
__global__ void __launch_bounds__(kQuantThreads)
    act_quant_kernel(const void *__restrict__ x, int K, int ldx, int fwht, int rmsnorm,
                     int8_t *__restrict__ q, int ldq, float *__restrict__ s_x) {
    extern __shared__ __align__(16) float v[];
    __shared__ float warp_max[kQuantThreads / 32];
    __shared__ float warp_ss[kQuantThreads / 32];
    const int m = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    constexpr int nwarps = kQuantThreads / 32;

    pdl_wait();  // x is written by the previous kernel on the stream
    pdl_launch_dependents();

    // ---- stage the row as fp32
    if (FP16) {
        const __half *row = static_cast<const __half *>(x) + static_cast<int64_t>(m) * ldx;
        for (int k = tid * 4; k < K; k += kQuantThreads * 4) {
            if (k + 4 <= K) {
                uint2 raw = *reinterpret_cast<const uint2 *>(row + k);
                __half2 a = *reinterpret_cast<__half2 *>(&raw.x);
                __half2 b = *reinterpret_cast<__half2 *>(&raw.y);
                float2 fa = __half22float2(a), fb = __half22float2(b);
                *reinterpret_cast<float4 *>(v + k) = make_float4(fa.x, fa.y, fb.x, fb.y);
            } else {
                for (int e = k; e < K; ++e) v[e] = __half2float(row[e]);
            }
        }
    } else {
        const float *row = static_cast<const float *>(x) + static_cast<int64_t>(m) * ldx;
        for (int k = tid * 4; k < K; k += kQuantThreads * 4) {
            if (k + 4 <= K) {
                *reinterpret_cast<float4 *>(v + k) = *reinterpret_cast<const float4 *>(row + k);
            } else {
                for (int e = k; e < K; ++e) v[e] = row[e];
            }
        }
    }
    __syncthreads();

    // ---- sum of squares of the unrotated row (weightless RMSNorm fold)
    float ss = 0.0f;
    if (rmsnorm) {
        for (int k = tid; k < K; k += kQuantThreads) ss = fmaf(v[k], v[k], ss);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        if (lane == 0) warp_ss[warp] = ss;
    }
    __syncthreads();

    // ---- optional Hadamard rotation, one 128-block per warp at a time
    if (fwht) {
        for (int b = warp; b < K / 128; b += nwarps) {
            float4 *p = reinterpret_cast<float4 *>(v + 128 * b + 4 * lane);
            float4 e = *p;
            float r[4] = {e.x, e.y, e.z, e.w};
            fwht128_warp(r, lane);
            *p = make_float4(r[0], r[1], r[2], r[3]);
        }
        __syncthreads();
    }

    // ---- amax
    float mx = 0.0f;
    for (int k = tid; k < K; k += kQuantThreads) mx = fmaxf(mx, fabsf(v[k]));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if (lane == 0) warp_max[warp] = mx;
    __syncthreads();
    float amax = 0.0f;
#pragma unroll
    for (int w = 0; w < nwarps; ++w) amax = fmaxf(amax, warp_max[w]);

    float inv = 0.0f, s = 0.0f;
    if (amax > 0.0f) {
        inv = __fdiv_rn(127.0f, amax);
        s = __fdiv_rn(amax, 127.0f);
        if (fwht) s = __fmul_rn(s, kInvSqrt128);
    }
    if (rmsnorm) {
        float tot = 0.0f;
#pragma unroll
        for (int w = 0; w < nwarps; ++w) tot += warp_ss[w];
        s = s / sqrtf(tot / static_cast<float>(K) + 1e-6f);
    }

    // ---- quantise, 16 bytes per thread-iteration, zero past K up to ldq
    int8_t *qrow = q + static_cast<int64_t>(m) * ldq;
    for (int k0 = tid * 16; k0 < ldq; k0 += kQuantThreads * 16) {
        uint32_t words[4];
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            uint32_t packed = 0;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                int k = k0 + 4 * w + e;
                int qi = 0;
                if (k < K && amax > 0.0f) {
                    qi = __float2int_rn(__fmul_rn(v[k], inv));
                    qi = max(-127, min(127, qi));
                }
                packed |= (static_cast<uint32_t>(qi) & 0xffu) << (8 * e);
            }
            words[w] = packed;
        }
        *reinterpret_cast<uint4 *>(qrow + k0) = make_uint4(words[0], words[1], words[2], words[3]);
    }
    if (tid == 0) s_x[m] = s;
}

cudaError_t launch_act_quant(const void *x, bool fp16, int M, int K, int ldx, int fwht_block,
                             int flags, int8_t *q, int ldq, float *s_x, cudaStream_t s) {
    const int rmsnorm = (flags & TERN_QUANT_RMSNORM) ? 1 : 0;
    size_t smem = static_cast<size_t>(K) * sizeof(float);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(M);
    cfg.blockDim = dim3(kQuantThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    // The shared-memory limit is a property of the kernel on each device:
    // set once per device (thread-safe), for both input types.
    static DeviceOnce once;
    int dev = 0;
    cudaError_t e = current_device(&dev);
    if (e != cudaSuccess) return e;
    e = once.run(dev, []() {
        cudaError_t r = cudaFuncSetAttribute(act_quant_kernel<true>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
        if (r != cudaSuccess) return r;
        return cudaFuncSetAttribute(act_quant_kernel<false>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
    });
    if (e != cudaSuccess) return e;
    if (fp16)
        e = cudaLaunchKernelEx(&cfg, act_quant_kernel<true>, x, K, ldx, fwht_block, rmsnorm, q, ldq, s_x);
    else
        e = cudaLaunchKernelEx(&cfg, act_quant_kernel<false>, x, K, ldx, fwht_block, rmsnorm, q, ldq, s_x);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace tern

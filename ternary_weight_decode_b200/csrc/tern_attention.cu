// tern_attention.cu -- decode attention over a Q4_0 KV cache (Bonsai page,
// "先交代机器和配置": K and V cached as Q4_0 with Flash Attention; the passage
// before "PQ2 会不会快很多": the Q4 data is decoded inside attention).
//
// Cache layout (tern_kv_cache): per KV head, per token, the D/2 code bytes of
// K (Q4_0 blocks of 32 along D: byte j of a block holds element j in its low
// nibble and element j + 16 in its high nibble) and the D/32 fp16 block
// scales, in two arrays so that a token's codes are one aligned 64-byte row
// (D = 128).  V alike.
//
//  * kv_append_kernel: quantises the new token's k and v, one thread per
//    block of 32, in the fp32 steps of the definition (d = m / -8 with m the
//    value of largest magnitude, code = min(15, trunc(x / d + 8.5))).
//  * attn_split_kernel: split-context flash decoding.  A CTA owns one KV head
//    and a chunk of tokens and serves all Hq/Hkv query heads of that group,
//    so each cached byte is read once per token.  Scores: a thread per token
//    (its codes as four 16-byte loads), sum_b d_b (sum_i q_i c_i - 8 sum_i q_i)
//    with the per-block query sums precomputed.  Values: the pass's V rows
//    copied into shared memory (cp.async) while the scores are formed, then
//    a warp per token, a lane per four dimensions, p_t d_b (c - 8)
//    accumulated in fp32.  The CTA
//    writes its chunk's max score, exp-sum and unnormalised output.  The
//    codes become floats as the bits of 2^23 + c less 2^23 (no conversion
//    instruction); one thread starts a bulk L2 prefetch of the K and V rows
//    two passes ahead, so each pass's loads find them in L2.  Chunks are
//    sized from the CTAs an SM holds at once so that the grid fills whole
//    waves of the SMs.
//  * attn_combine_kernel: per query head, the chunks' partial results merged
//    with the running-max rule: the chunk weights once in shared memory,
//    then four chunk lanes per dimension, each in chunk order, added in lane
//    order (a fixed order: the result does not depend on timing).
#include "tern_common.cuh"
#include "tern_internal.h"

namespace tern {
namespace {

constexpr int kAttD = 128;         // head dimension
constexpr int kAttThreads = 128;   // 4 warps
constexpr int kAttMaxChunks = 8192;  // chunks of the context per KV head

__global__ void kv_append_kernel(const float *__restrict__ x, int H, int D, int pos, int capacity,
                                 uint8_t *__restrict__ codes, uint16_t *__restrict__ scales) {
    const int nb = D / 32;
    const int blk = blockIdx.x * blockDim.x + threadIdx.x;  // (head, block)
    if (blk >= H * nb) return;
    const int h = blk / nb, b = blk % nb;
    const float *v = x + static_cast<int64_t>(h) * D + 32 * b;
    float amax = 0.0f, m = 0.0f;
    for (int j = 0; j < 32; ++j) {
        const float a = fabsf(v[j]);
        if (a > amax) {
            amax = a;
            m = v[j];
        }
    }
    const float d = __fdiv_rn(m, -8.0f);
    const float id = d != 0.0f ? __fdiv_rn(1.0f, d) : 0.0f;
    const int64_t row = static_cast<int64_t>(h) * capacity + pos;
    uint8_t *c = codes + row * (D / 2) + 16 * b;
    for (int j = 0; j < 16; ++j) {
        const int c0 = min(15, __float2int_rz(__fadd_rn(__fmul_rn(v[j], id), 8.5f)));
        const int c1 = min(15, __float2int_rz(__fadd_rn(__fmul_rn(v[j + 16], id), 8.5f)));
        c[j] = static_cast<uint8_t>(c0 | (c1 << 4));
    }
    scales[row * nb + b] = __half_as_ushort(__float2half_rn(d));
}

// Codes as floats without the conversion unit: byte e of `nib` (a nibble,
// 0..15) becomes the low byte of the bit pattern of 2^23 + c, from which
// one subtraction leaves c - bias exactly (every value here is an integer
// below 2^24, where one ulp is 1).
constexpr uint32_t kNibMagic = 0x4B000000u;  // 2^23 as fp32 bits
__device__ __forceinline__ float nib_float(uint32_t nib, int e, float bias) {
    return __fsub_rn(__uint_as_float(__byte_perm(nib, kNibMagic, 0x7640 + e)), 8388608.0f + bias);
}

// Nibble values of a 32-bit word as floats: lo[e] = byte e & 15, hi[e] = byte e >> 4.
__device__ __forceinline__ void nibbles(uint32_t w, float (&lo)[4], float (&hi)[4]) {
    const uint32_t l = w & 0x0F0F0F0Fu, h = (w >> 4) & 0x0F0F0F0Fu;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        lo[e] = nib_float(l, e, 0.0f);
        hi[e] = nib_float(h, e, 0.0f);
    }
}

// Bulk prefetch into L2 (no shared memory, no completion): `bytes` from a
// 16-byte aligned address, a multiple of 16.
__device__ __forceinline__ void prefetch_l2(const void *p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(reinterpret_cast<uint64_t>(p)), "r"(bytes)
                 : "memory");
}

// The K and V rows (codes, and scales when `scales16`: both scale arrays
// 16-byte aligned) of tokens [t, t + n) of one head, into L2.  Scale rows
// are 8 bytes: the range is shrunk to whole 16-byte pairs inside it.
__device__ __forceinline__ void prefetch_rows(int64_t row, int n, const uint8_t *kc, const uint16_t *ks,
                                              const uint8_t *vc, const uint16_t *vs, bool scales16) {
    if (n <= 0) return;
    prefetch_l2(kc + row * (kAttD / 2), static_cast<uint32_t>(n) * (kAttD / 2));
    prefetch_l2(vc + row * (kAttD / 2), static_cast<uint32_t>(n) * (kAttD / 2));
    const int64_t r0 = (row + 1) & ~static_cast<int64_t>(1), r1 = (row + n) & ~static_cast<int64_t>(1);
    if (scales16 && r1 > r0) {
        constexpr int NB = kAttD / 32;
        prefetch_l2(ks + r0 * NB, static_cast<uint32_t>(r1 - r0) * NB * 2);
        prefetch_l2(vs + r0 * NB, static_cast<uint32_t>(r1 - r0) * NB * 2);
    }
}

// Asynchronous copies global -> shared (no registers held while in flight).
__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)),
                 "l"(reinterpret_cast<uint64_t>(src))
                 : "memory");
}
__device__ __forceinline__ void cp_async8(void *dst, const void *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(smem_u32(dst)),
                 "l"(reinterpret_cast<uint64_t>(src))
                 : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// Launch flags of the split kernel: alignment of the scale arrays.
constexpr int kScales16 = 1;  // both scale arrays 16-byte aligned (L2 prefetch of scales)
constexpr int kVScales8 = 2;  // v_scales 8-byte aligned (one 8-byte copy per token)

template <int GQ>
__global__ void __launch_bounds__(kAttThreads)
    attn_split_kernel(const float *__restrict__ q, int Hkv, int capacity, int L, int chunk,
                      const uint8_t *__restrict__ kc, const uint16_t *__restrict__ ks,
                      const uint8_t *__restrict__ vc, const uint16_t *__restrict__ vs,
                      float *__restrict__ part, int nchunks, int flags) {
    constexpr int D = kAttD, NB = D / 32;
    __shared__ __align__(16) float qs[GQ][D];  // the group's queries
    __shared__ float qsum[GQ][NB];       // sum of q over each block of 32
    __shared__ float p[GQ][kAttThreads]; // scores, then exp(score - max), of one pass
    __shared__ float red[GQ][4][D];      // the warps' partial outputs
    __shared__ float wmax[GQ][4], wsum[GQ][4];
    __shared__ __align__(16) uint8_t vt[kAttThreads][D / 2];  // the pass's V codes
    __shared__ __align__(16) uint16_t vst[kAttThreads][NB];   // and their block scales
    const bool scales16 = (flags & kScales16) != 0;
    const int g = blockIdx.y, ck = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int t0 = ck * chunk, t1 = min(L, t0 + chunk);
    const float inv_sqrt_d = 0.08838834764831845f;  // 1/sqrt(128) rounded to fp32
    const int64_t head_row = static_cast<int64_t>(g) * capacity;
    // The first two passes' rows start towards L2 before the wait (L2 is
    // coherent: the token the previous kernel appends is read after it).
    if (tid == 0)
        prefetch_rows(head_row + t0, min(2 * kAttThreads, t1 - t0), kc, ks, vc, vs, scales16);
    pdl_wait();  // q (and the appended token) come from earlier kernels
    for (int i = tid; i < GQ * D; i += kAttThreads) (&qs[0][0])[i] = q[static_cast<int64_t>(g) * GQ * D + i];
    __syncthreads();
    if (tid < GQ * NB) {
        const int h = tid / NB, b = tid % NB;
        float s = 0.0f;
        for (int i = 0; i < 32; ++i) s += qs[h][32 * b + i];
        qsum[h][b] = s;
    }
    float m_run[GQ], z_run[GQ];
    float2 acc[GQ][2];  // the lane's four dimensions, two per packed instruction
#pragma unroll
    for (int h = 0; h < GQ; ++h) {
        m_run[h] = -INFINITY;
        z_run[h] = 0.0f;
#pragma unroll
        for (int e = 0; e < 2; ++e) acc[h][e] = make_float2(0.0f, 0.0f);
    }
    __syncthreads();
    // passes of kAttThreads tokens: scores, then the value accumulation;
    // the pass two ahead is prefetched into L2 as each one starts
    for (int tb = t0; tb < t1; tb += kAttThreads) {
        const int t = tb + tid;
        if (tid == 0) {
            const int tp = tb + 2 * kAttThreads;
            prefetch_rows(head_row + tp, min(kAttThreads, t1 - tp), kc, ks, vc, vs, scales16);
        }
        const int nt = min(kAttThreads, t1 - tb);
        // this pass's V rows into shared memory, in flight while the scores
        // are formed (the previous pass's readers are past its last barrier)
        for (int i = tid; i < nt * 4; i += kAttThreads)
            cp_async16(&vt[i >> 2][16 * (i & 3)], vc + (head_row + tb + (i >> 2)) * (D / 2) + 16 * (i & 3));
        if (tid < nt) {
            const uint16_t *src = vs + (head_row + tb + tid) * NB;
            if (flags & kVScales8) {
                cp_async8(&vst[tid][0], src);
            } else {
#pragma unroll
                for (int b = 0; b < NB; ++b) vst[tid][b] = __ldg(src + b);
            }
        }
        float sc[GQ];
        if (t < t1) {
            const uint4 *krow = reinterpret_cast<const uint4 *>(kc + (head_row + t) * (D / 2));
            const uint16_t *kd = ks + (head_row + t) * NB;
#pragma unroll
            for (int h = 0; h < GQ; ++h) sc[h] = 0.0f;
#pragma unroll
            for (int b = 0; b < NB; ++b) {
                const uint4 w = __ldg(krow + b);
                const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
                // per head, even and odd elements in the two halves of a packed pair
                float2 dot[GQ];
#pragma unroll
                for (int h = 0; h < GQ; ++h) dot[h] = make_float2(0.0f, 0.0f);
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    float lo[4], hi[4];
                    nibbles(ww[c], lo, hi);
#pragma unroll
                    for (int h = 0; h < GQ; ++h) {
                        // elements 4c..4c+3 (low nibbles) and 16+4c.. (high nibbles)
                        const float4 ql = *reinterpret_cast<const float4 *>(&qs[h][32 * b + 4 * c]);
                        const float4 qh = *reinterpret_cast<const float4 *>(&qs[h][32 * b + 16 + 4 * c]);
                        float2 d = dot[h];
                        d = __ffma2_rn(make_float2(ql.x, ql.y), make_float2(lo[0], lo[1]), d);
                        d = __ffma2_rn(make_float2(ql.z, ql.w), make_float2(lo[2], lo[3]), d);
                        d = __ffma2_rn(make_float2(qh.x, qh.y), make_float2(hi[0], hi[1]), d);
                        d = __ffma2_rn(make_float2(qh.z, qh.w), make_float2(hi[2], hi[3]), d);
                        dot[h] = d;
                    }
                }
                const float db = __half2float(__ushort_as_half(__ldg(kd + b)));
#pragma unroll
                for (int h = 0; h < GQ; ++h)
                    sc[h] = fmaf(db, fmaf(-8.0f, qsum[h][b], dot[h].x + dot[h].y), sc[h]);
            }
#pragma unroll
            for (int h = 0; h < GQ; ++h) sc[h] *= inv_sqrt_d;
        } else {
#pragma unroll
            for (int h = 0; h < GQ; ++h) sc[h] = -INFINITY;
        }
        // this pass's max per head, the running max, and the rescale of what came before
        float mp[GQ];
#pragma unroll
        for (int h = 0; h < GQ; ++h) {
            float v = warp_max(sc[h]);
            if (lane == 0) wmax[h][warp] = v;
        }
        __syncthreads();
#pragma unroll
        for (int h = 0; h < GQ; ++h) {
            mp[h] = fmaxf(fmaxf(wmax[h][0], wmax[h][1]), fmaxf(wmax[h][2], wmax[h][3]));
            const float mn = fmaxf(m_run[h], mp[h]);
            const float r = m_run[h] == -INFINITY ? 0.0f : expf(m_run[h] - mn);
            z_run[h] *= r;
#pragma unroll
            for (int e = 0; e < 2; ++e) acc[h][e] = make_float2(acc[h][e].x * r, acc[h][e].y * r);
            m_run[h] = mn;
            p[h][tid] = t < t1 ? expf(sc[h] - mn) : 0.0f;
        }
        cp_async_wait_all();  // this thread's V copies have landed
        __syncthreads();
        // values: warp w takes tokens w, w+4, ... of the pass; lane = dims 4l..4l+3
        const int b = lane >> 3;               // block of the lane's dims
        const int e0 = (4 * lane) & 31;        // first element inside the block
        const int word = (e0 & 15) >> 2;       // code word of the block holding them
        const bool high = e0 >= 16;
        // four tokens per step, from shared memory
        constexpr int U = 4;
        for (int j0 = warp; j0 < nt; j0 += 4 * U) {
            uint32_t w[U];
            float db[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int j = j0 + 4 * u;
                w[u] = 0;
                db[u] = 0.0f;
                if (j < nt) {
                    w[u] = *reinterpret_cast<const uint32_t *>(&vt[j][16 * b + 4 * word]);
                    db[u] = __half2float(__ushort_as_half(vst[j][b]));
                }
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int j = j0 + 4 * u;
                if (j >= nt) break;
                // only the lane's four nibbles, as c - 8
                const uint32_t nib = (w[u] >> (high ? 4 : 0)) & 0x0F0F0F0Fu;
                float cv[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) cv[e] = nib_float(nib, e, 8.0f);
#pragma unroll
                for (int h = 0; h < GQ; ++h) {
                    const float pd = p[h][j] * db[u];
#pragma unroll
                    for (int e = 0; e < 2; ++e)
                        acc[h][e] = __ffma2_rn(make_float2(pd, pd), make_float2(cv[2 * e], cv[2 * e + 1]), acc[h][e]);
                }
            }
        }
        // exp-sum of the pass
#pragma unroll
        for (int h = 0; h < GQ; ++h) {
            const float v = warp_sum(p[h][tid]);
            if (lane == 0) wsum[h][warp] = v;
        }
        __syncthreads();
#pragma unroll
        for (int h = 0; h < GQ; ++h) z_run[h] += (wsum[h][0] + wsum[h][1]) + (wsum[h][2] + wsum[h][3]);
    }
    // the warps' outputs, summed in warp order
#pragma unroll
    for (int h = 0; h < GQ; ++h)
#pragma unroll
        for (int e = 0; e < 4; ++e) red[h][warp][4 * lane + e] = (e & 1) ? acc[h][e >> 1].y : acc[h][e >> 1].x;
    __syncthreads();
    for (int i = tid; i < GQ * D; i += kAttThreads) {
        const int h = i / D, d = i % D;
        const float v = (red[h][0][d] + red[h][1][d]) + (red[h][2][d] + red[h][3][d]);
        part[((static_cast<int64_t>(g) * GQ + h) * nchunks + ck) * (D + 2) + d] = v;
    }
    if (tid < GQ) {
        float *rec = part + ((static_cast<int64_t>(g) * GQ + tid) * nchunks + ck) * (D + 2);
        rec[D] = m_run[tid];
        rec[D + 1] = z_run[tid];
    }
    pdl_launch_dependents();
}

// Merge of one query head's chunk records: lane j of dimension d (S lanes
// per dimension) sums chunks j, j + S, ... in order; the S partial sums are
// added in lane order, so the result does not depend on timing.  The chunk
// weights exp(m_c - M) are formed once, in shared memory.
constexpr int kCombSplit = 4;
constexpr int kCombThreads = kAttD * kCombSplit;

__global__ void __launch_bounds__(kCombThreads)
    attn_combine_kernel(const float *__restrict__ part, int nchunks, float *__restrict__ out) {
    constexpr int D = kAttD;
    extern __shared__ float wch[];  // [nchunks] chunk weights
    __shared__ float wmax[kCombThreads / 32];
    __shared__ float pnum[kCombSplit][D], pden[kCombSplit][D];
    const int h = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int d = tid % D, j = tid / D;
    pdl_wait();
    const float *base = part + static_cast<int64_t>(h) * nchunks * (D + 2);
    float m = -INFINITY;
    for (int c = tid; c < nchunks; c += kCombThreads) m = fmaxf(m, base[c * (D + 2) + D]);
    m = warp_max(m);
    if (lane == 0) wmax[warp] = m;
    __syncthreads();
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kCombThreads / 32; ++w) M = fmaxf(M, wmax[w]);
    for (int c = tid; c < nchunks; c += kCombThreads) {
        const float mc = base[c * (D + 2) + D];
        wch[c] = mc == -INFINITY ? 0.0f : expf(mc - M);  // an empty chunk weighs nothing
    }
    __syncthreads();
    float num = 0.0f, den = 0.0f;
#pragma unroll 4
    for (int c = j; c < nchunks; c += kCombSplit) {
        const float *rec = base + c * (D + 2);
        const float w = wch[c];
        num = fmaf(w, rec[d], num);
        den = fmaf(w, rec[D + 1], den);
    }
    pnum[j][d] = num;
    pden[j][d] = den;
    __syncthreads();
    if (j == 0) {
        float n = pnum[0][d], z = pden[0][d];
#pragma unroll
        for (int i = 1; i < kCombSplit; ++i) {
            n += pnum[i][d];
            z += pden[i][d];
        }
        out[static_cast<int64_t>(h) * D + d] = n / z;
    }
}

template <int GQ>
cudaError_t launch_split(const float *q, int Hkv, int capacity, int L, int chunk, int nchunks,
                         const tern_kv_cache &C, float *part, cudaStream_t s) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(nchunks, Hkv, 1);
    cfg.blockDim = dim3(kAttThreads, 1, 1);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const auto ks = reinterpret_cast<uintptr_t>(C.k_scales), vs = reinterpret_cast<uintptr_t>(C.v_scales);
    const int flags = (ks % 16 == 0 && vs % 16 == 0 ? kScales16 : 0) | (vs % 8 == 0 ? kVScales8 : 0);
    return cudaLaunchKernelEx(&cfg, attn_split_kernel<GQ>, q, Hkv, capacity, L, chunk, C.k_codes,
                              C.k_scales, C.v_codes, C.v_scales, part, nchunks, flags);
}

// Split CTAs one SM holds at once (registers and shared memory of the
// instantiation for GQ query heads per KV head); 1 for an unsupported GQ.
int split_ctas_per_sm(int GQ) {
    const void *k = nullptr;
    switch (GQ) {
        case 1: k = reinterpret_cast<const void *>(attn_split_kernel<1>); break;
        case 2: k = reinterpret_cast<const void *>(attn_split_kernel<2>); break;
        case 4: k = reinterpret_cast<const void *>(attn_split_kernel<4>); break;
        case 5: k = reinterpret_cast<const void *>(attn_split_kernel<5>); break;
        case 8: k = reinterpret_cast<const void *>(attn_split_kernel<8>); break;
        default: return 1;
    }
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k, kAttThreads, 0) != cudaSuccess || n < 1) {
        (void)cudaGetLastError();
        return 1;
    }
    return n;
}

}  // namespace

int attention_chunk(int L, int Hkv, int GQ, int num_sms) {
    // Chunks of at least one pass, beyond that of whole warps' worth of
    // tokens (the last pass may be partial), chosen so that the CTAs fill
    // whole waves of the SMs: the least tokens that one resident CTA slot has
    // to stream (waves x chunk), the fewer CTAs on a tie.  (Chunks shorter
    // than a pass measured slower: a CTA's fixed work and the merge grow.)
    // At most kAttMaxChunks chunks (the merge keeps one weight per chunk in
    // shared memory).
    const long long slots = static_cast<long long>(split_ctas_per_sm(GQ)) * num_sms;
    constexpr long long kGrain = 32;
    auto whole_passes = [](long long t) {
        return t <= kAttThreads ? static_cast<long long>(kAttThreads) : (t + kGrain - 1) / kGrain * kGrain;
    };
    long long best = whole_passes((L + kAttMaxChunks - 1) / kAttMaxChunks), best_cost = -1;
    for (long long w = 1; w <= 64; ++w) {
        const long long per_head = w * slots / Hkv > 0 ? w * slots / Hkv : 1;
        const long long chunk = whole_passes((L + per_head - 1) / per_head);
        if ((L + chunk - 1) / chunk > kAttMaxChunks) continue;
        const long long ctas = (L + chunk - 1) / chunk * Hkv;
        const long long cost = (ctas + slots - 1) / slots * chunk;
        if (best_cost < 0 || cost < best_cost || (cost == best_cost && chunk > best)) {
            best = chunk;
            best_cost = cost;
        }
    }
    return static_cast<int>(best);
}

size_t attention_workspace_bytes(int Hq, int L, int Hkv, int num_sms) {
    const int chunk = attention_chunk(L, Hkv, Hq / Hkv, num_sms);
    const size_t nchunks = static_cast<size_t>((L + chunk - 1) / chunk);
    return static_cast<size_t>(Hq) * nchunks * (kAttD + 2) * sizeof(float);
}

cudaError_t launch_kv_append(const float *k, const float *v, int pos, const tern_kv_cache &C,
                             cudaStream_t s) {
    const int blocks = C.Hkv * (C.D / 32);
    kv_append_kernel<<<(blocks + 63) / 64, 64, 0, s>>>(k, C.Hkv, C.D, pos, C.capacity, C.k_codes,
                                                       C.k_scales);
    kv_append_kernel<<<(blocks + 63) / 64, 64, 0, s>>>(v, C.Hkv, C.D, pos, C.capacity, C.v_codes,
                                                       C.v_scales);
    return cudaGetLastError();
}

cudaError_t launch_attention(const float *q, int Hq, const tern_kv_cache &C, int L, float *out,
                             float *part, int num_sms, cudaStream_t s, const char **why) {
    const int GQ = Hq / C.Hkv;
    const int chunk = attention_chunk(L, C.Hkv, GQ, num_sms);
    const int nchunks = (L + chunk - 1) / chunk;
    cudaError_t e;
    switch (GQ) {
        case 1: e = launch_split<1>(q, C.Hkv, C.capacity, L, chunk, nchunks, C, part, s); break;
        case 2: e = launch_split<2>(q, C.Hkv, C.capacity, L, chunk, nchunks, C, part, s); break;
        case 4: e = launch_split<4>(q, C.Hkv, C.capacity, L, chunk, nchunks, C, part, s); break;
        case 5: e = launch_split<5>(q, C.Hkv, C.capacity, L, chunk, nchunks, C, part, s); break;
        case 8: e = launch_split<8>(q, C.Hkv, C.capacity, L, chunk, nchunks, C, part, s); break;
        default: *why = "query heads per KV head must be 1, 2, 4, 5 or 8"; return cudaErrorInvalidValue;
    }
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(Hq, 1, 1);
    cfg.blockDim = dim3(kCombThreads, 1, 1);
    cfg.dynamicSmemBytes = static_cast<size_t>(nchunks) * sizeof(float);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, attn_combine_kernel, static_cast<const float *>(part), nchunks, out);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace tern

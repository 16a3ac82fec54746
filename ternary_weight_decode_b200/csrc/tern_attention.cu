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
//    with the per-block query sums precomputed.  Values: a warp per token, a
//    lane per four dimensions, p_t d_b (c - 8) accumulated in fp32.  The CTA
//    writes its chunk's max score, exp-sum and unnormalised output.  Chunks
//    are sized for about eight resident CTAs per SM, so the loads of many
//    warps are in flight at once.
//  * attn_combine_kernel: per query head, the chunks' partial results merged
//    in chunk order with the running-max rule (a fixed order: the result
//    does not depend on timing).
#include "tern_common.cuh"
#include "tern_internal.h"

namespace tern {
namespace {

constexpr int kAttD = 128;         // head dimension
constexpr int kAttThreads = 128;   // 4 warps
constexpr int kAttMaxGroup = 8;    // query heads per KV head

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

// Nibble values of a 32-bit word as floats: lo[e] = byte e & 15, hi[e] = byte e >> 4.
__device__ __forceinline__ void nibbles(uint32_t w, float (&lo)[4], float (&hi)[4]) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        lo[e] = static_cast<float>((w >> (8 * e)) & 15u);
        hi[e] = static_cast<float>((w >> (8 * e + 4)) & 15u);
    }
}

template <int GQ>
__global__ void __launch_bounds__(kAttThreads)
    attn_split_kernel(const float *__restrict__ q, int Hkv, int capacity, int L, int chunk,
                      const uint8_t *__restrict__ kc, const uint16_t *__restrict__ ks,
                      const uint8_t *__restrict__ vc, const uint16_t *__restrict__ vs,
                      float *__restrict__ part, int nchunks) {
    constexpr int D = kAttD, NB = D / 32;
    __shared__ __align__(16) float qs[GQ][D];  // the group's queries
    __shared__ float qsum[GQ][NB];       // sum of q over each block of 32
    __shared__ float p[GQ][kAttThreads]; // scores, then exp(score - max), of one pass
    __shared__ float red[GQ][4][D];      // the warps' partial outputs
    __shared__ float wmax[GQ][4], wsum[GQ][4];
    const int g = blockIdx.y, ck = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int t0 = ck * chunk, t1 = min(L, t0 + chunk);
    const float inv_sqrt_d = 0.08838834764831845f;  // 1/sqrt(128) rounded to fp32
    pdl_wait();  // q (and the appended token) come from earlier kernels
    for (int i = tid; i < GQ * D; i += kAttThreads) (&qs[0][0])[i] = q[static_cast<int64_t>(g) * GQ * D + i];
    __syncthreads();
    if (tid < GQ * NB) {
        const int h = tid / NB, b = tid % NB;
        float s = 0.0f;
        for (int i = 0; i < 32; ++i) s += qs[h][32 * b + i];
        qsum[h][b] = s;
    }
    float m_run[GQ], z_run[GQ], acc[GQ][4];
#pragma unroll
    for (int h = 0; h < GQ; ++h) {
        m_run[h] = -INFINITY;
        z_run[h] = 0.0f;
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[h][e] = 0.0f;
    }
    __syncthreads();
    const int64_t head_row = static_cast<int64_t>(g) * capacity;
    // passes of kAttThreads tokens: scores, then the value accumulation
    for (int tb = t0; tb < t1; tb += kAttThreads) {
        const int t = tb + tid;
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
                float dot[GQ];
#pragma unroll
                for (int h = 0; h < GQ; ++h) dot[h] = 0.0f;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    float lo[4], hi[4];
                    nibbles(ww[c], lo, hi);
#pragma unroll
                    for (int h = 0; h < GQ; ++h) {
                        // elements 4c..4c+3 (low nibbles) and 16+4c.. (high nibbles)
                        const float4 ql = *reinterpret_cast<const float4 *>(&qs[h][32 * b + 4 * c]);
                        const float4 qh = *reinterpret_cast<const float4 *>(&qs[h][32 * b + 16 + 4 * c]);
                        float d = dot[h];
                        d = fmaf(ql.x, lo[0], d);
                        d = fmaf(ql.y, lo[1], d);
                        d = fmaf(ql.z, lo[2], d);
                        d = fmaf(ql.w, lo[3], d);
                        d = fmaf(qh.x, hi[0], d);
                        d = fmaf(qh.y, hi[1], d);
                        d = fmaf(qh.z, hi[2], d);
                        d = fmaf(qh.w, hi[3], d);
                        dot[h] = d;
                    }
                }
                const float db = __half2float(__ushort_as_half(__ldg(kd + b)));
#pragma unroll
                for (int h = 0; h < GQ; ++h) sc[h] = fmaf(db, fmaf(-8.0f, qsum[h][b], dot[h]), sc[h]);
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
            for (int e = 0; e < 4; ++e) acc[h][e] *= r;
            m_run[h] = mn;
            p[h][tid] = t < t1 ? expf(sc[h] - mn) : 0.0f;
        }
        __syncthreads();
        // values: warp w takes tokens w, w+4, ... of the pass; lane = dims 4l..4l+3
        const int b = lane >> 3;               // block of the lane's dims
        const int e0 = (4 * lane) & 31;        // first element inside the block
        const int word = (e0 & 15) >> 2;       // code word of the block holding them
        const bool high = e0 >= 16;
        const int nt = min(kAttThreads, t1 - tb);
        // four tokens per step, their loads issued before any is used
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
                    const int64_t r = head_row + tb + j;
                    w[u] = __ldg(reinterpret_cast<const uint32_t *>(vc + r * (D / 2) + 16 * b) + word);
                    db[u] = __half2float(__ushort_as_half(__ldg(vs + r * NB + b)));
                }
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int j = j0 + 4 * u;
                if (j >= nt) break;
                float lo[4], hi[4];
                nibbles(w[u], lo, hi);
#pragma unroll
                for (int h = 0; h < GQ; ++h) {
                    const float pd = p[h][j] * db[u];
#pragma unroll
                    for (int e = 0; e < 4; ++e) acc[h][e] = fmaf(pd, (high ? hi[e] : lo[e]) - 8.0f, acc[h][e]);
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
        for (int e = 0; e < 4; ++e) red[h][warp][4 * lane + e] = acc[h][e];
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

__global__ void attn_combine_kernel(const float *__restrict__ part, int nchunks, float *__restrict__ out) {
    constexpr int D = kAttD;
    const int h = blockIdx.x, d = threadIdx.x;
    pdl_wait();
    const float *base = part + static_cast<int64_t>(h) * nchunks * (D + 2);
    float M = -INFINITY;
    for (int c = 0; c < nchunks; ++c) M = fmaxf(M, base[c * (D + 2) + D]);
    float num = 0.0f, den = 0.0f;
    for (int c = 0; c < nchunks; ++c) {
        const float *rec = base + c * (D + 2);
        if (rec[D] == -INFINITY) continue;  // an empty chunk
        const float w = expf(rec[D] - M);
        num = fmaf(w, rec[d], num);
        den = fmaf(w, rec[D + 1], den);
    }
    out[static_cast<int64_t>(h) * D + d] = num / den;
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
    return cudaLaunchKernelEx(&cfg, attn_split_kernel<GQ>, q, Hkv, capacity, L, chunk, C.k_codes,
                              C.k_scales, C.v_codes, C.v_scales, part, nchunks);
}

}  // namespace

int attention_chunk(int L, int Hkv, int num_sms) {
    // chunks of whole passes, as many CTAs as about eight per SM hold at once
    // (128 threads and under 32 KB of shared memory each)
    int chunk = kAttThreads;
    while (static_cast<long long>((L + chunk - 1) / chunk) * Hkv > 8LL * num_sms && chunk < (1 << 20))
        chunk *= 2;
    return chunk;
}

size_t attention_workspace_bytes(int Hq, int L, int Hkv, int num_sms) {
    const int chunk = attention_chunk(L, Hkv, num_sms);
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
    const int chunk = attention_chunk(L, C.Hkv, num_sms);
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
    cfg.blockDim = dim3(kAttD, 1, 1);
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

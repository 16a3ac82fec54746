// tern_gemv_common.cuh -- pieces shared by the two GEMV engines of libtern
// (CUDA-core dp4a in tern_gemv.cu, tensor-core tcgen05 in tern_gemv_tc.cu):
// launch parameters, the D3 digit decode, staging of scales and activations
// (including the in-kernel quantisation from producer statistics), and the
// epilogue (cluster reduction of K-split partials, outputs, statistics).
//
// Work decomposition (both engines): a CTA of 4 warps owns 128 consecutive
// output rows -- warp w rows 32w..32w+31, one per lane -- over a K range
// made of 128-byte superblocks of each row (640 positions = 5 scale groups in
// D3, 512 = 4 groups in D2); a longer K is split across a thread-block
// cluster whose rank 0 sums the CTAs' fp32 row partials in rank order.
#pragma once

#include "tern_common.cuh"
#include "tern_internal.h"

namespace tern {

constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr int kRowsCta = kWarps * 32;
constexpr int kSBBytes = 128;
constexpr int kTile = 32 * kSBBytes;  // bytes of one matrix per warp stage

template <int FMT>
struct Fmt;
template <>
struct Fmt<TERN_FMT_BASE3> {
    static constexpr int kPos = 640;  // K positions per superblock
    static constexpr int kGroups = 5;
};
template <>
struct Fmt<TERN_FMT_2BIT> {
    static constexpr int kPos = 512;
    static constexpr int kGroups = 4;
};
template <>
struct Fmt<TERN_FMT_BITPLANE> {  // every engine but the tensor-core GEMV
    static constexpr int kPos = 512;
    static constexpr int kGroups = 4;
};

struct GemvParams {
    int N, K, G;
    int SB;          // superblocks per row
    int sb_per_cta;  // superblocks per K split
    int nsplit;
    int M;
    int prefetch_ok;
    int stages;
    const uint16_t *scales0;
    const uint16_t *scales1;
    // int8 input
    const int8_t *q;
    int ldq;
    const float *s_x;
    // fp32 input with producer statistics
    const float *x;
    int ldx;
    const float *x_stats;
    int x_stats_ld;  // blocks between token rows of x_stats
    int qflags;
    // output
    const float *residual;
    void *out;
    int ldo;
    float *y_stats;
    int y_stats_ld;
};

__host__ __device__ constexpr int align128(int v) { return (v + 127) & ~127; }

// D3 word -> five int8x4 words of leading-digit numbers D_i (word i aligned
// with the activation word at K = 20w + 4i): a code byte y = ceil(256 V/243)
// gives D_i = floor(y 3^(i+1) / 256).  Two bytes share one 32-bit multiply
// (16-bit lanes, y 3^(i+1) < 2^16); PRMT gathers the four high bytes.
// 3 z as a shift and an add: integer ALU work, leaving the multiply pipe
// (shared with dp4a) to the dot product.  Exact: 3 z = z + 2 z mod 2^32.
__device__ __forceinline__ uint32_t times3(uint32_t z) {
    uint32_t r;
    asm("{\n\t.reg .u32 t;\n\tshl.b32 t, %1, 1;\n\tadd.u32 %0, t, %1;\n\t}" : "=r"(r) : "r"(z));
    return r;
}

__device__ __forceinline__ void decode_d3_D(uint32_t X, uint32_t (&D)[5]) {
    uint32_t ze = X & 0x00FF00FFu;              // bytes 0 and 2
    uint32_t zo = __byte_perm(X, 0u, 0x4341);  // bytes 1 and 3: one permute, not a shift and a mask
#pragma unroll
    for (int i = 0; i < 5; ++i) {
        ze = times3(ze);
        zo = times3(zo);
        D[i] = __byte_perm(ze, zo, 0x7351);
    }
}

// D3 word -> five int8x4 words of digits t_i = D_i - 3 D_(i-1) (0..2).
__device__ __forceinline__ void decode_d3(uint32_t X, uint32_t (&t)[5]) {
    uint32_t D[5];
    decode_d3_D(X, D);
    t[0] = D[0];
#pragma unroll
    for (int i = 1; i < 5; ++i) t[i] = D[i] - 3u * D[i - 1];
}

// ---------------------------------------------------------------- scales
template <int NMAT>
__device__ __forceinline__ void stage_scales(float *sc, int sc_stride, const GemvParams &p, int rg,
                                             int g0, int GS, int tid) {
    const int total = NMAT * kRowsCta * GS;
    for (int idx = tid; idx < total; idx += kThreads) {
        const int mat = idx / (kRowsCta * GS);
        const int r = (idx / GS) % kRowsCta;
        const int gl = idx % GS;
        const int n = rg * kRowsCta + r, gg = g0 + gl;
        float v = 0.0f;
        if (n < p.N && gg < p.G) {
            const uint16_t *s = mat ? p.scales1 : p.scales0;
            v = __half2float(__ushort_as_half(s[static_cast<int64_t>(n) * p.G + gg]));
        }
        sc[(mat * kRowsCta + r) * sc_stride + gl] = v;
    }
}

// ---------------------------------------------------------------- activations
// int8 input: the K slice [k0, k0 + KS) of q (zero past K) in 16-byte chunks,
// handed to put16(m, local k, chunk), and the per-group sums of q.
template <int MT, typename Put16>
__device__ __forceinline__ void stage_q(int *sq, const GemvParams &p, int k0, int KS, int GS,
                                        int tid, Put16 put16) {
    const int nchunks = KS / 16;  // a scale group is 8 chunks
    for (int m = 0; m < MT; ++m) {
        for (int base = 0; base < nchunks; base += kThreads) {
            const int c = base + tid;
            const bool valid = c < nchunks;
            uint4 v = make_uint4(0, 0, 0, 0);
            const int k = k0 + c * 16;
            if (valid && m < p.M && k < p.K) {
                const int8_t *src = p.q + static_cast<int64_t>(m) * p.ldq + k;
                if (k + 16 <= p.K) {
                    v = *reinterpret_cast<const uint4 *>(src);
                } else {
                    uint32_t w[4] = {0, 0, 0, 0};
                    for (int e = 0; e < 16 && k + e < p.K; ++e)
                        w[e >> 2] |= static_cast<uint32_t>(static_cast<uint8_t>(src[e])) << (8 * (e & 3));
                    v = make_uint4(w[0], w[1], w[2], w[3]);
                }
            }
            if (valid) put16(m, c * 16, v);
            int s = dp4a_ss(v.x, 0x01010101u, 0);
            s = dp4a_ss(v.y, 0x01010101u, s);
            s = dp4a_ss(v.z, 0x01010101u, s);
            s = dp4a_ss(v.w, 0x01010101u, s);
            s += __shfl_xor_sync(0xffffffffu, s, 1);
            s += __shfl_xor_sync(0xffffffffu, s, 2);
            s += __shfl_xor_sync(0xffffffffu, s, 4);
            if (valid && (c & 7) == 0) sq[m * GS + (c >> 3)] = s;
        }
    }
}

// fp32 input: row scale and its inverse (sx[m], sx[MT + m]) from the
// producer's block statistics -- the arithmetic of act_quant_fwht.
template <int MT>
__device__ __forceinline__ void row_scales(float *sx, const GemvParams &p, int tid) {
    const int lane = tid & 31, warp = tid >> 5;
    const bool rotate = (p.qflags & TERN_QUANT_FWHT128) != 0;
    const bool rms = (p.qflags & TERN_QUANT_RMSNORM) != 0;
    const int nb = (p.K + 127) / 128;
    for (int m = warp; m < MT; m += kWarps) {
        float amax = 0.0f, ss = 0.0f;
        if (m < p.M) {
            const float *st = p.x_stats + static_cast<int64_t>(m) * p.x_stats_ld * 4;
            for (int b = lane; b < nb; b += 32) {
                const float4 v = *reinterpret_cast<const float4 *>(st + 4 * b);
                amax = fmaxf(amax, rotate ? v.y : v.x);
                ss += v.z;
            }
            amax = warp_max(amax);
            ss = warp_sum(ss);
        }
        if (lane == 0) {
            float inv = 0.0f, s = 0.0f;
            if (amax > 0.0f) {
                inv = __fdiv_rn(127.0f, amax);
                s = __fdiv_rn(amax, 127.0f);
                if (rotate) s = __fmul_rn(s, kInvSqrt128);
            }
            if (rms) s = s / sqrtf(ss / static_cast<float>(p.K) + 1e-6f);
            sx[m] = s;
            sx[MT + m] = inv;
        }
    }
}

// fp32 input: each warp quantises 128-blocks of the K slice (4 elements per
// lane, rotated first when asked), hands 4 bytes at a time to
// put4(m, local k, word) and records the per-group sums.  Needs row_scales
// and a CTA barrier before it.
template <int MT, typename Put4>
__device__ __forceinline__ void quantise_slice(int *sq, const float *sx, const GemvParams &p,
                                               int k0, int KS, int GS, int tid, Put4 put4) {
    const int lane = tid & 31, warp = tid >> 5;
    const bool rotate = (p.qflags & TERN_QUANT_FWHT128) != 0;
    const int nblk = KS / 128;
    for (int job = warp; job < MT * nblk; job += kWarps) {
        const int m = job / nblk, blk = job % nblk;
        const int k = k0 + 128 * blk + 4 * lane;
        float r[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        if (m < p.M && k < p.K) {
            const float *src = p.x + static_cast<int64_t>(m) * p.ldx + k;
            if (k + 4 <= p.K) {
                const float4 v = *reinterpret_cast<const float4 *>(src);
                r[0] = v.x;
                r[1] = v.y;
                r[2] = v.z;
                r[3] = v.w;
            } else {
                for (int e = 0; e < 4 && k + e < p.K; ++e) r[e] = src[e];
            }
        }
        if (rotate) fwht128_warp(r, lane);
        const float inv = sx[MT + m];
        uint32_t packed = 0;
        int qsum = 0;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            int qi = 0;
            if (k + e < p.K && inv > 0.0f) {
                qi = __float2int_rn(__fmul_rn(r[e], inv));
                qi = max(-127, min(127, qi));
            }
            qsum += qi;
            packed |= (static_cast<uint32_t>(qi) & 0xffu) << (8 * e);
        }
        put4(m, 128 * blk + 4 * lane, packed);
        qsum = warp_sum_int(qsum);
        if (lane == 0) sq[m * GS + blk] = qsum;
    }
}

// ---------------------------------------------------------------- epilogue
// part[(mat*MT + m)*128 + row] holds this CTA's fp32 partial of row `row`;
// rank 0 of the cluster adds the other ranks' partials, writes y / h and,
// optionally, the statistics of the 128 outputs.  Returns on ranks != 0.
template <int MT, int NMAT, int MODE, int XIN>
__device__ __forceinline__ void gemv_epilogue(float *part, const float *sx, const GemvParams &p,
                                              int split, int rg, int tid) {
    const int lane = tid & 31, warp = tid >> 5, row = tid;
    const int n = rg * kRowsCta + row;
    constexpr int NPART = NMAT * MT * kRowsCta;
    if (p.nsplit > 1) {
        cluster_sync();
        if (split == 0) {
            for (int i = tid; i < NPART; i += kThreads) {
                float s = part[i];
                for (int r = 1; r < p.nsplit; ++r) s += ld_shared_cluster_f32(map_shared_rank(&part[i], r));
                part[i] = s;
            }
        }
        cluster_sync();  // remote shared memory stays valid until rank 0 is done
    } else {
        __syncthreads();
    }
    if (split != 0) return;

    for (int m = 0; m < MT; ++m) {
        float v = 0.0f;
        if (m < p.M && n < p.N) {
            const float sxm = XIN ? sx[m] : p.s_x[m];
            const int64_t o = static_cast<int64_t>(m) * p.ldo + n;
            if (MODE == kModeGemv) {
                v = sxm * part[m * kRowsCta + row];
                if (p.residual) v += p.residual[o];
            } else {
                const float g = sxm * part[m * kRowsCta + row];
                const float u = sxm * part[(MT + m) * kRowsCta + row];
                v = g * (1.0f / (1.0f + expf(-g))) * u;
            }
            static_cast<float *>(p.out)[o] = v;
        }
        part[m * kRowsCta + row] = v;  // rows past N count as 0 in the statistics
    }
    if (p.y_stats) {
        __syncthreads();
        for (int m = warp; m < MT && m < p.M; m += kWarps) {
            const float4 v = *reinterpret_cast<const float4 *>(&part[m * kRowsCta + 4 * lane]);
            float r[4] = {v.x, v.y, v.z, v.w};
            const float3 st = block_stats128(r, lane);
            if (lane == 0)
                *reinterpret_cast<float4 *>(p.y_stats + (static_cast<int64_t>(m) * p.y_stats_ld + rg) * 4) =
                    make_float4(st.x, st.y, st.z, 0.0f);
        }
    }
}

// ---------------------------------------------------------------- host helpers
bool make_weight_tmap(CUtensorMap *map, const void *packed, int64_t row_bytes, int N,
                      int64_t row_stride);

// Fills the parameters shared by both engines from the launch description.
void fill_params(GemvParams &p, const GemvLaunch &L);

}  // namespace tern

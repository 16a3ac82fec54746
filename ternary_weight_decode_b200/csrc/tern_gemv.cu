// tern_gemv.cu -- ternary GEMV / skinny GEMM for decode (M = 1..16 token
// rows), the fused gate/up + SwiGLU form, the integer-partials test hook,
// and the activation statistics that let a GEMV quantise its own input.
//
// The method (Bonsai page, "Decode 为什么只能算一般"): stream the packed codes
// once, restore -1/0/+1 in registers, integer dot with the int8 activation,
// apply the FP16 group scale (4sapi page, section 三), never materialising
// dequantised weights; gate/up + SwiGLU fused; activations re-quantised per
// token (after a 128-point Hadamard rotation for the FFN input).
//
// Kernel shape (B200, sm_100a):
//  * A CTA owns 128 consecutive output rows; warp w takes rows 32w..32w+31,
//    one per lane, over the CTA's whole K range, so no two warps share a row.
//    The K range is a run of 128-byte "superblocks" of each row (640
//    positions = 5 scale groups in D3, 512 = 4 groups in D2).  A longer K is
//    split across a thread-block cluster (<= 8 CTAs); rank 0 sums the CTAs'
//    fp32 row partials in rank order through distributed shared memory.
//  * Each warp streams its superblocks through its own ring of shared-memory
//    stages filled by TMA (a 32 x 128 B box per matrix, 128-byte swizzle,
//    L2 evict-first; no multicast).
//  * Input, either form:
//      - int8 q + s_x (tern_gemv): the CTA copies its K slice and per-group
//        sums of q into shared memory;
//      - fp32 x + per-128-block statistics of x (tern_gemv_fused): the CTA
//        forms the row scale from the statistics and quantises its own K
//        slice (optionally Hadamard-rotated) itself -- bit for bit what
//        act_quant_fwht computes -- so no separate quantisation launch sits
//        between two GEMVs.
//  * D3 decode: a code byte y = ceil(256 V / 243) gives the leading-digit
//    numbers D_i = floor(y 3^(i+1) / 256) and digits t_i = D_i - 3 D_(i-1).
//    Two bytes share one 32-bit multiply (16-bit lanes); PRMT gathers the
//    D_i bytes of a word's four code bytes into an int8x4 word aligned with
//    the activation word at K = 20w + 4i.  dp4a gives sum t q, and
//    sum w q = sum t q - sum q per group.
//  * D2 decode: (X >> 2i) & 0x03030303 is an int8x4 word of digits.
//  * Epilogue: y = s_x * sum_g s_w P (+ residual), or h = g sigmoid(g) u;
//    optionally the statistics of the 128 outputs {max|y|, max|H y|, sum y^2}
//    for the next fused call.
//  * Programmatic dependent launch: with static matrices the weight stream
//    and the scale staging start before the previous kernel on the stream
//    has finished; inputs are read and outputs written only after it has.
#include <mutex>

#include "tern_common.cuh"
#include "tern_internal.h"

namespace tern {

__device__ int g_device_error = 0;

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

struct SmemLayout {
    int stage_bytes, act_off, sq_off, sc_off, part_off, sx_off, bar_off, total;
    int KS, GS, sc_stride;
};

// Every region starts on a 128-byte boundary (the epilogue reads `part` and
// the staging writes `act` with 16-byte vector accesses).
__host__ __device__ constexpr int align128(int v) { return (v + 127) & ~127; }

template <int FMT, int MT, int NMAT>
__host__ __device__ inline SmemLayout smem_layout(int sb_per_cta, int stages) {
    SmemLayout L;
    L.KS = sb_per_cta * Fmt<FMT>::kPos;
    L.GS = sb_per_cta * Fmt<FMT>::kGroups;
    L.sc_stride = L.GS + 1;  // odd float stride: conflict-free per-lane scale reads
    L.stage_bytes = NMAT * kTile;
    int off = kWarps * stages * L.stage_bytes;
    L.act_off = off;
    off = align128(off + MT * L.KS);
    L.sq_off = off;
    off = align128(off + MT * L.GS * 4);
    L.sc_off = off;
    off = align128(off + NMAT * kRowsCta * L.sc_stride * 4);
    L.part_off = off;
    off = align128(off + NMAT * MT * kRowsCta * 4);
    L.sx_off = off;
    off = align128(off + 2 * MT * 4);
    L.bar_off = off;
    off += kWarps * stages * 8;
    L.total = off + 1024;  // slack for aligning the base to 1024 bytes (128B swizzle)
    return L;
}

// ---------------------------------------------------------------- decode
// D3 word -> five int8x4 words of digits t (0..2); word i is aligned with the
// activation word at K = 20w + 4i.
__device__ __forceinline__ void decode_d3(uint32_t X, uint32_t (&t)[5]) {
    uint32_t ze = X & 0x00FF00FFu;         // bytes 0 and 2 in 16-bit lanes
    uint32_t zo = (X >> 8) & 0x00FF00FFu;  // bytes 1 and 3
    uint32_t prev = 0;
#pragma unroll
    for (int i = 0; i < 5; ++i) {
        ze *= 3u;  // y * 3^(i+1) < 2^16 per lane
        zo *= 3u;
        uint32_t D = __byte_perm(ze, zo, 0x7351);  // high bytes -> [b0, b1, b2, b3]
        t[i] = (i == 0) ? D : D - 3u * prev;
        prev = D;
    }
}

// Adds one finished group to the fp32 accumulators (or stores its partials).
template <int MT, int NMAT, int MODE>
__device__ __forceinline__ void finish_group(int (&acc)[NMAT][MT], float (&yacc)[NMAT][MT], int m,
                                             int gl, int row, const int *sq, int GS,
                                             const float *sc, int sc_stride,
                                             const GemvParams &p, int n, int gg) {
    const int s = sq[m * GS + gl];
#pragma unroll
    for (int mat = 0; mat < NMAT; ++mat) {
        const int P = acc[mat][m] - s;
        if (MODE == kModePartials) {
            if (n < p.N && gg < p.G && m < p.M)
                static_cast<int *>(p.out)[(static_cast<int64_t>(m) * p.N + n) * p.G + gg] = P;
        } else {
            yacc[mat][m] = fmaf(sc[(mat * kRowsCta + row) * sc_stride + gl], static_cast<float>(P),
                                yacc[mat][m]);
        }
        acc[mat][m] = 0;
    }
}

template <int MT, int NMAT, int MODE>
__device__ __forceinline__ void process_d3(const uint8_t *stage, int sbl, int lane, int row,
                                           const uint8_t *act, int KS, const int *sq, int GS,
                                           const float *sc, int sc_stride,
                                           float (&yacc)[NMAT][MT], const GemvParams &p, int n,
                                           int g_base) {
    int acc[NMAT][MT];
#pragma unroll
    for (int mat = 0; mat < NMAT; ++mat)
#pragma unroll
        for (int m = 0; m < MT; ++m) acc[mat][m] = 0;
    const int rsw = lane & 7;
    const int gl0 = sbl * 5;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        uint32_t t[NMAT][20];
#pragma unroll
        for (int mat = 0; mat < NMAT; ++mat) {
            uint4 wv = lds128(stage + mat * kTile + lane * kSBBytes + ((c ^ rsw) << 4));
            uint32_t words[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
            for (int wi = 0; wi < 4; ++wi) {
                uint32_t tw[5];
                decode_d3(words[wi], tw);
#pragma unroll
                for (int i = 0; i < 5; ++i) t[mat][5 * wi + i] = tw[i];
            }
        }
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            const uint8_t *a = act + m * KS + sbl * 640 + c * 80;
            uint32_t aw[20];
#pragma unroll
            for (int j = 0; j < 5; ++j) {
                uint4 v = lds128(a + 16 * j);
                aw[4 * j + 0] = v.x;
                aw[4 * j + 1] = v.y;
                aw[4 * j + 2] = v.z;
                aw[4 * j + 3] = v.w;
            }
#pragma unroll
            for (int d = 0; d < 20; ++d) {
                const int dd = c * 20 + d;  // digit-word index in the superblock
                if (dd > 0 && (dd & 31) == 0)
                    finish_group<MT, NMAT, MODE>(acc, yacc, m, gl0 + (dd >> 5) - 1, row, sq, GS, sc,
                                                 sc_stride, p, n, g_base + (dd >> 5) - 1);
#pragma unroll
                for (int mat = 0; mat < NMAT; ++mat) acc[mat][m] = dp4a_ss(t[mat][d], aw[d], acc[mat][m]);
            }
        }
    }
#pragma unroll
    for (int m = 0; m < MT; ++m)
        finish_group<MT, NMAT, MODE>(acc, yacc, m, gl0 + 4, row, sq, GS, sc, sc_stride, p, n,
                                     g_base + 4);
}

template <int MT, int NMAT, int MODE>
__device__ __forceinline__ void process_d2(const uint8_t *stage, int sbl, int lane, int row,
                                           const uint8_t *act, int KS, const int *sq, int GS,
                                           const float *sc, int sc_stride,
                                           float (&yacc)[NMAT][MT], const GemvParams &p, int n,
                                           int g_base) {
    int acc[NMAT][MT];
#pragma unroll
    for (int mat = 0; mat < NMAT; ++mat)
#pragma unroll
        for (int m = 0; m < MT; ++m) acc[mat][m] = 0;
    const int rsw = lane & 7;
    const int gl0 = sbl * 4;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        uint32_t words[NMAT][4];
#pragma unroll
        for (int mat = 0; mat < NMAT; ++mat) {
            uint4 wv = lds128(stage + mat * kTile + lane * kSBBytes + ((c ^ rsw) << 4));
            words[mat][0] = wv.x;
            words[mat][1] = wv.y;
            words[mat][2] = wv.z;
            words[mat][3] = wv.w;
        }
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            const uint8_t *a = act + m * KS + sbl * 512 + c * 64;
            uint32_t aw[16];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                uint4 v = lds128(a + 16 * j);
                aw[4 * j + 0] = v.x;
                aw[4 * j + 1] = v.y;
                aw[4 * j + 2] = v.z;
                aw[4 * j + 3] = v.w;
            }
#pragma unroll
            for (int mat = 0; mat < NMAT; ++mat) {
                if (MT <= 2) {
                    // masked fields: lane values 4^i * t, summed separately and
                    // rescaled (exactly) by arithmetic shifts
                    int a4[4] = {0, 0, 0, 0};
#pragma unroll
                    for (int wi = 0; wi < 4; ++wi)
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            a4[i] = dp4a_us(words[mat][wi] & (0x03030303u << (2 * i)), aw[4 * wi + i],
                                            a4[i]);
                    acc[mat][m] += a4[0] + (a4[1] >> 2) + (a4[2] >> 4) + (a4[3] >> 6);
                } else {
#pragma unroll
                    for (int wi = 0; wi < 4; ++wi)
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            acc[mat][m] = dp4a_ss((words[mat][wi] >> (2 * i)) & 0x03030303u,
                                                  aw[4 * wi + i], acc[mat][m]);
                }
            }
            if (c & 1)
                finish_group<MT, NMAT, MODE>(acc, yacc, m, gl0 + (c >> 1), row, sq, GS, sc,
                                             sc_stride, p, n, g_base + (c >> 1));
        }
    }
}

// ---------------------------------------------------------------- input staging
// int8 input: copy the K slice [k0, k0 + KS) of q (zero past K) and its
// per-group sums.
template <int MT>
__device__ __forceinline__ void stage_q(uint8_t *act, int *sq, const GemvParams &p, int k0, int KS,
                                        int GS, int tid) {
    const int nchunks = KS / 16;  // 16-byte chunks; a scale group is 8 chunks
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
            if (valid) *reinterpret_cast<uint4 *>(act + m * KS + c * 16) = v;
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

// fp32 input: row scales from the producer's block statistics, then each warp
// quantises 128-blocks of the K slice -- the arithmetic of act_quant_fwht.
template <int MT>
__device__ __forceinline__ void stage_x(uint8_t *act, int *sq, float *sx, const GemvParams &p,
                                        int k0, int KS, int GS, int tid) {
    const int lane = tid & 31, warp = tid >> 5;
    const bool rotate = (p.qflags & TERN_QUANT_FWHT128) != 0;
    const bool rms = (p.qflags & TERN_QUANT_RMSNORM) != 0;
    const int nb = (p.K + 127) / 128;
    // ---- row scales: warp m % 4 reduces the statistics of row m
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
    __syncthreads();
    // ---- quantise: one 128-block per warp-iteration, 4 elements per lane
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
        *reinterpret_cast<uint32_t *>(act + m * KS + 128 * blk + 4 * lane) = packed;
        qsum = warp_sum_int(qsum);
        if (lane == 0) sq[m * GS + blk] = qsum;
    }
}

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

// ---------------------------------------------------------------- kernel
template <int FMT, int MT, int MODE, int XIN>
__global__ void __launch_bounds__(kThreads)
    gemv_kernel(const __grid_constant__ CUtensorMap tm0, const __grid_constant__ CUtensorMap tm1,
                const GemvParams p) {
    constexpr int NMAT = (MODE == kModeSwiglu) ? 2 : 1;
    constexpr int POS = Fmt<FMT>::kPos;
    constexpr int GPS = Fmt<FMT>::kGroups;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);

    const int S = p.stages;
    const SmemLayout L = smem_layout<FMT, MT, NMAT>(p.sb_per_cta, S);
    uint8_t *stages = smem;
    uint8_t *act = smem + L.act_off;
    int *sq = reinterpret_cast<int *>(smem + L.sq_off);
    float *sc = reinterpret_cast<float *>(smem + L.sc_off);
    float *part = reinterpret_cast<float *>(smem + L.part_off);
    float *sx = reinterpret_cast<float *>(smem + L.sx_off);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L.bar_off);

    const int split = blockIdx.x, rg = blockIdx.y;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int row = warp * 32 + lane;  // row within the CTA
    const int n = rg * kRowsCta + row;
    const int sb0 = split * p.sb_per_cta;
    const int nsb = min(p.sb_per_cta, p.SB - sb0);

    if (tid == 0) {
        prefetch_tmap(&tm0);
        if (NMAT == 2) prefetch_tmap(&tm1);
        for (int i = 0; i < kWarps * S; ++i) mbar_init(&bars[i], 1);
        fence_mbar_init();
    }
    __syncthreads();

    if (!p.prefetch_ok) pdl_wait();
    pdl_launch_dependents();

    const uint64_t policy = l2_policy_evict_first();
    uint64_t *wbars = bars + warp * S;
    uint8_t *wstages = stages + warp * S * L.stage_bytes;
    auto issue = [&](int it) {
        const int st = it % S;
        const int sb = sb0 + it;
        uint8_t *dst = wstages + st * L.stage_bytes;
        mbar_arrive_expect_tx(&wbars[st], NMAT * kTile);
        tma_load_2d(dst, &tm0, sb * kSBBytes, rg * kRowsCta + warp * 32, &wbars[st], policy);
        if (NMAT == 2)
            tma_load_2d(dst + kTile, &tm1, sb * kSBBytes, rg * kRowsCta + warp * 32, &wbars[st], policy);
    };
    int issued = min(S, nsb);
    if (lane == 0)
        for (int it = 0; it < issued; ++it) issue(it);

    stage_scales<NMAT>(sc, L.sc_stride, p, rg, sb0 * GPS, L.GS, tid);
    if (p.prefetch_ok) pdl_wait();
    if (XIN)
        stage_x<MT>(act, sq, sx, p, sb0 * POS, L.KS, L.GS, tid);
    else
        stage_q<MT>(act, sq, p, sb0 * POS, L.KS, L.GS, tid);
    __syncthreads();

    float yacc[NMAT][MT];
#pragma unroll
    for (int mat = 0; mat < NMAT; ++mat)
#pragma unroll
        for (int m = 0; m < MT; ++m) yacc[mat][m] = 0.0f;

    bool aborted = false;
    int consumed = 0;
    for (int it = 0; it < nsb; ++it) {
        const int st = it % S;
        const bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(&wbars[st], (it / S) & 1));
        if (!ok) {
            aborted = true;
            break;
        }
        consumed = it + 1;
        const uint8_t *stg = wstages + st * L.stage_bytes;
        if (FMT == TERN_FMT_BASE3)
            process_d3<MT, NMAT, MODE>(stg, it, lane, row, act, L.KS, sq, L.GS, sc, L.sc_stride,
                                       yacc, p, n, (sb0 + it) * GPS);
        else
            process_d2<MT, NMAT, MODE>(stg, it, lane, row, act, L.KS, sq, L.GS, sc, L.sc_stride,
                                       yacc, p, n, (sb0 + it) * GPS);
        __syncwarp();
        if (it + S < nsb) {
            if (lane == 0) {
                fence_proxy_async_smem();
                issue(it + S);
            }
            ++issued;
        }
    }
    if (aborted) {
        // Let copies still in flight land (each wait bounded) before exiting.
        for (int it = consumed; it < issued; ++it) mbar_wait_bounded(&wbars[it % S], (it / S) & 1);
    }

    if constexpr (MODE != kModePartials) {
#pragma unroll
        for (int mat = 0; mat < NMAT; ++mat)
#pragma unroll
            for (int m = 0; m < MT; ++m) part[(mat * MT + m) * kRowsCta + row] = yacc[mat][m];
        constexpr int NPART = NMAT * MT * kRowsCta;
        if (p.nsplit > 1) {
            cluster_sync();
            if (split == 0) {
                for (int i = tid; i < NPART; i += kThreads) {
                    float s = part[i];
                    for (int r = 1; r < p.nsplit; ++r)
                        s += ld_shared_cluster_f32(map_shared_rank(&part[i], r));
                    part[i] = s;
                }
            }
            cluster_sync();  // remote shared memory stays valid until rank 0 is done
        } else {
            __syncthreads();
        }
        if (split != 0) return;

        // ---- outputs: thread = row
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
        // ---- statistics of the 128 outputs, for the next fused call
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
}

// Statistics {max|x|, max|H x|, sum x^2} of each 128-block of an fp32 row
// (the first fused call of a chain has no producer to compute them).
__global__ void __launch_bounds__(128) act_stats_kernel(const float *__restrict__ x, int K, int ldx,
                                                        float *__restrict__ stats, int ld) {
    const int lane = threadIdx.x & 31;
    const int b = blockIdx.x * 4 + (threadIdx.x >> 5);
    const int m = blockIdx.y;
    pdl_wait();
    pdl_launch_dependents();
    if (b * 128 >= K) return;
    const int k = b * 128 + 4 * lane;
    const float *src = x + static_cast<int64_t>(m) * ldx + k;
    float r[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    if (k + 4 <= K) {
        const float4 v = *reinterpret_cast<const float4 *>(src);
        r[0] = v.x;
        r[1] = v.y;
        r[2] = v.z;
        r[3] = v.w;
    } else {
        for (int e = 0; e < 4 && k + e < K; ++e) r[e] = src[e];
    }
    const float3 st = block_stats128(r, lane);
    if (lane == 0)
        *reinterpret_cast<float4 *>(stats + (static_cast<int64_t>(m) * ld + b) * 4) =
            make_float4(st.x, st.y, st.z, 0.0f);
}

// ---------------------------------------------------------------- host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult qr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &qr) ==
                cudaSuccess &&
            qr == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    });
    return fn;
}

static bool make_tmap(CUtensorMap *map, const void *packed, int64_t row_bytes, int N,
                      int64_t row_stride) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(row_bytes), static_cast<cuuint64_t>(N)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(row_stride)};
    cuuint32_t box[2] = {kSBBytes, 32};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(packed), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

constexpr int kMaxDevices = 64;
constexpr int kTargetCtas = 3 * 148;

template <int FMT, int MT, int MODE, int XIN>
static cudaError_t launch_impl(const GemvLaunch &Lh, cudaStream_t s, const char **why) {
    constexpr int NMAT = (MODE == kModeSwiglu) ? 2 : 1;
    constexpr int POS = Fmt<FMT>::kPos;
    static int smem_set[kMaxDevices] = {0};

    GemvParams p = {};
    p.N = Lh.N;
    p.K = Lh.K;
    p.G = Lh.G;
    p.SB = static_cast<int>(ceil_div(Lh.row_bytes, kSBBytes));
    p.M = Lh.M;
    p.prefetch_ok = Lh.prefetch_ok;
    p.scales0 = Lh.scales[0];
    p.scales1 = Lh.scales[1];
    p.q = Lh.q;
    p.ldq = Lh.ldq;
    p.s_x = Lh.s_x;
    p.x = Lh.x;
    p.ldx = Lh.ldx;
    p.x_stats = Lh.x_stats;
    p.x_stats_ld = Lh.x_stats_ld;
    p.qflags = Lh.qflags;
    p.residual = Lh.residual;
    p.out = Lh.out;
    p.ldo = Lh.ldo;
    p.y_stats = Lh.y_stats;
    p.y_stats_ld = Lh.y_stats_ld;

    // K split: at least what keeps the CTA's activation slice <= 48 KB, then
    // widened (cluster of <= 8) towards about three CTAs per SM.
    const int rowgroups = static_cast<int>(ceil_div(Lh.N, kRowsCta));
    int sb_max = (48 * 1024) / (MT * POS);
    if (sb_max < 1) sb_max = 1;
    int nsplit = static_cast<int>(ceil_div(p.SB, sb_max));
    int want = static_cast<int>(ceil_div(kTargetCtas, rowgroups));
    if (want > 8) want = 8;
    if (nsplit < want) nsplit = want;
    if (nsplit > p.SB) nsplit = p.SB;
    p.sb_per_cta = static_cast<int>(ceil_div(p.SB, nsplit));
    p.nsplit = static_cast<int>(ceil_div(p.SB, p.sb_per_cta));
    if (MODE != kModePartials && p.nsplit > 8) {
        *why = "K too large for an 8-CTA cluster split at this M";
        return cudaErrorInvalidValue;
    }
    p.stages = p.sb_per_cta < 3 ? p.sb_per_cta : 3;

    const SmemLayout L = smem_layout<FMT, MT, NMAT>(p.sb_per_cta, p.stages);
    if (L.total > 227 * 1024) {
        *why = "shared memory plan exceeds 227 KB";
        return cudaErrorInvalidValue;
    }

    CUtensorMap tm0, tm1;
    if (!make_tmap(&tm0, Lh.packed[0], Lh.row_bytes, Lh.N, Lh.row_stride) ||
        !make_tmap(&tm1, Lh.packed[NMAT - 1], Lh.row_bytes, Lh.N, Lh.row_stride)) {
        *why = "cuTensorMapEncodeTiled failed or is unavailable";
        return cudaErrorInvalidValue;
    }

    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < kMaxDevices && !smem_set[dev]) {
        e = cudaFuncSetAttribute(gemv_kernel<FMT, MT, MODE, XIN>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
        if (e != cudaSuccess) return e;
        smem_set[dev] = 1;
    }

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.nsplit, rowgroups, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = L.total;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    int na = 0;
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
    if (p.nsplit > 1 && MODE != kModePartials) {
        attr[na].id = cudaLaunchAttributeClusterDimension;
        attr[na].val.clusterDim.x = p.nsplit;
        attr[na].val.clusterDim.y = 1;
        attr[na].val.clusterDim.z = 1;
        ++na;
    }
    cfg.attrs = attr;
    cfg.numAttrs = na;
    e = cudaLaunchKernelEx(&cfg, gemv_kernel<FMT, MT, MODE, XIN>, tm0, tm1, p);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

template <int FMT, int MODE, int XIN>
static cudaError_t launch_mt(const GemvLaunch &L, cudaStream_t s, const char **why) {
    if (L.M <= 1) return launch_impl<FMT, 1, MODE, XIN>(L, s, why);
    if (L.M <= 2) return launch_impl<FMT, 2, MODE, XIN>(L, s, why);
    if (L.M <= 4) return launch_impl<FMT, 4, MODE, XIN>(L, s, why);
    if (L.M <= 8) return launch_impl<FMT, 8, MODE, XIN>(L, s, why);
    return launch_impl<FMT, 16, MODE, XIN>(L, s, why);
}

template <int FMT>
static cudaError_t launch_fmt(const GemvLaunch &L, cudaStream_t s, const char **why) {
    if (L.x) {
        if (L.mode == kModeSwiglu) return launch_mt<FMT, kModeSwiglu, 1>(L, s, why);
        return launch_mt<FMT, kModeGemv, 1>(L, s, why);
    }
    switch (L.mode) {
        case kModeGemv: return launch_mt<FMT, kModeGemv, 0>(L, s, why);
        case kModeSwiglu: return launch_mt<FMT, kModeSwiglu, 0>(L, s, why);
        default: return launch_mt<FMT, kModePartials, 0>(L, s, why);
    }
}

cudaError_t launch_gemv(const GemvLaunch &L, cudaStream_t s, const char **why) {
    if (L.fmt == TERN_FMT_BASE3) return launch_fmt<TERN_FMT_BASE3>(L, s, why);
    return launch_fmt<TERN_FMT_2BIT>(L, s, why);
}

cudaError_t launch_act_stats(const float *x, int M, int K, int ldx, float *stats, int ld,
                             cudaStream_t s) {
    const int nb = static_cast<int>(ceil_div(K, 128));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(ceil_div(nb, 4)), M, 1);
    cfg.blockDim = dim3(128, 1, 1);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, act_stats_kernel, x, K, ldx, stats, ld);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

cudaError_t read_clear_device_error(int *value, cudaStream_t s) {
    int zero = 0;
    cudaError_t e = cudaMemcpyFromSymbolAsync(value, g_device_error, sizeof(int), 0,
                                              cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess)
        e = cudaMemcpyToSymbolAsync(g_device_error, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    return e;
}

}  // namespace tern

// tern_gemv.cu -- ternary GEMV / skinny GEMM for decode (M = 1..16 token
// rows), the fused gate/up + SwiGLU form, and the integer-partials test hook.
//
// The method (Bonsai page, "Decode 为什么只能算一般"): stream the packed codes
// once, restore -1/0/+1 in registers, integer dot with the int8 activation,
// apply the FP16 group scale (4sapi page, section 三), never materialising
// dequantised weights.
//
// Kernel shape (B200, sm_100a):
//  * A CTA owns 32 output rows (one per lane) and a K-range made of 128-byte
//    "superblocks" of each row (640 positions in D3 = 5 scale groups,
//    512 in D2 = 4 groups), so every scale group lies inside one superblock.
//  * Each of the 4 warps streams its own superblocks through a ring of
//    shared-memory stages filled by TMA (one 32 x 128 B box per matrix,
//    128-byte swizzle, L2 evict-first; no multicast).  Lane l reads row l.
//  * The CTA stages its slice of the int8 activations and their per-group
//    sums in shared memory; lanes read activation words with warp-uniform
//    addresses (broadcast).
//  * D3 decode: a code byte y = ceil(256 V / 243) gives the leading-digit
//    numbers D_i = floor(y 3^(i+1) / 256) (i = 0..4) and digits
//    t_i = D_i - 3 D_(i-1).  Two bytes are handled per 32-bit multiply
//    (16-bit lanes); PRMT gathers the D_i bytes of the four code bytes of a
//    word into one int8x4 word aligned with the activation word
//    K = 20w + 4i + (0..3).  dp4a gives sum t q; sum w q = sum t q - sum q.
//  * D2 decode: fields (X >> 2i) & 0x03030303 are int8x4 words of t.
//  * Int32 partials are exact per group; the epilogue does
//    y += s_w[n][g] * (P - 0) in fp32, sums warps in a fixed order and, for a
//    K split over a thread-block cluster, sums the CTAs' partials through
//    distributed shared memory in rank order (deterministic).
//  * Programmatic dependent launch: when the matrices are marked static, the
//    weight stream starts before the previous kernel on the stream has
//    finished; activations are read and outputs written only after it has.
#include <mutex>

#include "tern_common.cuh"
#include "tern_internal.h"

namespace tern {

__device__ int g_device_error = 0;

constexpr int kRows = 32;
constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr int kSBBytes = 128;
constexpr int kTile = kRows * kSBBytes;  // bytes of one matrix per stage

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
    const int8_t *q;
    int ldq;
    const float *s_x;
    const float *residual;
    void *out;
    int ldo;
};

struct SmemLayout {
    int stage_bytes, stages_off, act_off, sq_off, sc_off, red_off, part_off, bar_off, total;
    int KS, GS, sc_stride;
};

template <int FMT, int MT, int NMAT>
__host__ __device__ inline SmemLayout smem_layout(int sb_per_cta, int stages) {
    SmemLayout L;
    L.KS = sb_per_cta * Fmt<FMT>::kPos;
    L.GS = sb_per_cta * Fmt<FMT>::kGroups;
    L.sc_stride = L.GS + 1;  // odd float stride: conflict-free per-lane scale reads
    L.stage_bytes = NMAT * kTile;
    L.stages_off = 0;
    int off = kWarps * stages * L.stage_bytes;
    L.act_off = off;
    off += MT * L.KS;
    L.sq_off = off;
    off += MT * L.GS * 4;
    L.sc_off = off;
    off += NMAT * kRows * L.sc_stride * 4;
    L.red_off = off;
    off += kWarps * NMAT * MT * kRows * 4;
    L.part_off = off;
    off += NMAT * MT * kRows * 4;
    off = (off + 7) & ~7;
    L.bar_off = off;
    off += kWarps * stages * 8;
    L.total = off + 1024;  // slack for aligning the base to 1024 bytes (128B swizzle)
    return L;
}

// ---------------------------------------------------------------- decode
// D3 word -> five int8x4 words of digits t (0..2), word i aligned with the
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
                                             int gl, int lane, const int *sq, int GS,
                                             const float *sc, int sc_stride,
                                             const GemvParams &p, int n, int gg) {
    int s = sq[m * GS + gl];
#pragma unroll
    for (int mat = 0; mat < NMAT; ++mat) {
        int P = acc[mat][m] - s;
        if (MODE == kModePartials) {
            if (n < p.N && gg < p.G && m < p.M)
                static_cast<int *>(p.out)[(static_cast<int64_t>(m) * p.N + n) * p.G + gg] = P;
        } else {
            yacc[mat][m] = fmaf(sc[(mat * kRows + lane) * sc_stride + gl], static_cast<float>(P),
                                yacc[mat][m]);
        }
        acc[mat][m] = 0;
    }
}

template <int MT, int NMAT, int MODE>
__device__ __forceinline__ void process_d3(const uint8_t *stage, int sbl, int lane,
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
                    finish_group<MT, NMAT, MODE>(acc, yacc, m, gl0 + (dd >> 5) - 1, lane, sq, GS,
                                                 sc, sc_stride, p, n, g_base + (dd >> 5) - 1);
#pragma unroll
                for (int mat = 0; mat < NMAT; ++mat) acc[mat][m] = dp4a_ss(t[mat][d], aw[d], acc[mat][m]);
            }
        }
    }
#pragma unroll
    for (int m = 0; m < MT; ++m)
        finish_group<MT, NMAT, MODE>(acc, yacc, m, gl0 + 4, lane, sq, GS, sc, sc_stride, p, n,
                                     g_base + 4);
}

template <int MT, int NMAT, int MODE>
__device__ __forceinline__ void process_d2(const uint8_t *stage, int sbl, int lane,
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
                finish_group<MT, NMAT, MODE>(acc, yacc, m, gl0 + (c >> 1), lane, sq, GS, sc,
                                             sc_stride, p, n, g_base + (c >> 1));
        }
    }
}

// ---------------------------------------------------------------- staging
template <int FMT, int MT>
__device__ __forceinline__ void stage_activations(uint8_t *act, int *sq, const GemvParams &p,
                                                  int k0, int KS, int GS, int tid) {
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
                    uint8_t b[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) b[e] = (k + e < p.K) ? static_cast<uint8_t>(src[e]) : 0;
                    v.x = b[0] | (b[1] << 8) | (b[2] << 16) | (static_cast<uint32_t>(b[3]) << 24);
                    v.y = b[4] | (b[5] << 8) | (b[6] << 16) | (static_cast<uint32_t>(b[7]) << 24);
                    v.z = b[8] | (b[9] << 8) | (b[10] << 16) | (static_cast<uint32_t>(b[11]) << 24);
                    v.w = b[12] | (b[13] << 8) | (b[14] << 16) | (static_cast<uint32_t>(b[15]) << 24);
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

template <int NMAT>
__device__ __forceinline__ void stage_scales(float *sc, int sc_stride, const GemvParams &p, int rb,
                                             int g0, int GS, int tid) {
    const int total = NMAT * kRows * GS;
    for (int idx = tid; idx < total; idx += kThreads) {
        const int mat = idx / (kRows * GS);
        const int r = (idx / GS) % kRows;
        const int gl = idx % GS;
        const int n = rb * kRows + r, gg = g0 + gl;
        float v = 0.0f;
        if (n < p.N && gg < p.G) {
            const uint16_t *s = mat ? p.scales1 : p.scales0;
            v = __half2float(__ushort_as_half(s[static_cast<int64_t>(n) * p.G + gg]));
        }
        sc[(mat * kRows + r) * sc_stride + gl] = v;
    }
}

// ---------------------------------------------------------------- kernel
template <int FMT, int MT, int MODE>
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
    uint8_t *stages = smem + L.stages_off;
    uint8_t *act = smem + L.act_off;
    int *sq = reinterpret_cast<int *>(smem + L.sq_off);
    float *sc = reinterpret_cast<float *>(smem + L.sc_off);
    float *red = reinterpret_cast<float *>(smem + L.red_off);
    float *part = reinterpret_cast<float *>(smem + L.part_off);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L.bar_off);

    const int split = blockIdx.x, rb = blockIdx.y;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int sb0 = split * p.sb_per_cta;
    const int nsb = min(p.sb_per_cta, p.SB - sb0);
    const int my_n = (nsb > warp) ? (nsb - warp + kWarps - 1) / kWarps : 0;

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
        const int sb = sb0 + warp + it * kWarps;
        uint8_t *dst = wstages + st * L.stage_bytes;
        mbar_arrive_expect_tx(&wbars[st], NMAT * kTile);
        tma_load_2d(dst, &tm0, sb * kSBBytes, rb * kRows, &wbars[st], policy);
        if (NMAT == 2) tma_load_2d(dst + kTile, &tm1, sb * kSBBytes, rb * kRows, &wbars[st], policy);
    };
    int issued = 0;
    if (lane == 0)
        for (; issued < min(S, my_n); ++issued) issue(issued);
    issued = __shfl_sync(0xffffffffu, issued, 0);

    stage_scales<NMAT>(sc, L.sc_stride, p, rb, sb0 * GPS, L.GS, tid);
    if (p.prefetch_ok) pdl_wait();
    stage_activations<FMT, MT>(act, sq, p, sb0 * POS, L.KS, L.GS, tid);
    __syncthreads();

    float yacc[NMAT][MT];
#pragma unroll
    for (int mat = 0; mat < NMAT; ++mat)
#pragma unroll
        for (int m = 0; m < MT; ++m) yacc[mat][m] = 0.0f;

    const int n = rb * kRows + lane;
    bool aborted = false;
    int consumed = 0;
    for (int it = 0; it < my_n; ++it) {
        const int st = it % S;
        const bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(&wbars[st], (it / S) & 1));
        if (!ok) {
            aborted = true;
            break;
        }
        consumed = it + 1;
        const int sbl = warp + it * kWarps;
        const uint8_t *stg = wstages + st * L.stage_bytes;
        if (FMT == TERN_FMT_BASE3)
            process_d3<MT, NMAT, MODE>(stg, sbl, lane, act, L.KS, sq, L.GS, sc, L.sc_stride, yacc,
                                       p, n, (sb0 + sbl) * GPS);
        else
            process_d2<MT, NMAT, MODE>(stg, sbl, lane, act, L.KS, sq, L.GS, sc, L.sc_stride, yacc,
                                       p, n, (sb0 + sbl) * GPS);
        __syncwarp();
        if (it + S < my_n) {
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

    if (MODE == kModePartials) return;  // partials were stored group by group

#pragma unroll
    for (int mat = 0; mat < NMAT; ++mat)
#pragma unroll
        for (int m = 0; m < MT; ++m) red[((warp * NMAT + mat) * MT + m) * kRows + lane] = yacc[mat][m];
    __syncthreads();
    constexpr int NPART = NMAT * MT * kRows;
    for (int i = tid; i < NPART; i += kThreads) {
        float s = 0.0f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) s += red[w * NPART + i];
        part[i] = s;
    }
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
    for (int i = tid; i < MT * kRows; i += kThreads) {
        const int m = i / kRows, r = i % kRows, row = rb * kRows + r;
        if (m >= p.M || row >= p.N) continue;
        const float sx = p.s_x[m];
        const int64_t o = static_cast<int64_t>(m) * p.ldo + row;
        if (MODE == kModeGemv) {
            float v = sx * part[m * kRows + r];
            if (p.residual) v += p.residual[o];
            static_cast<float *>(p.out)[o] = v;
        } else {
            const float g = sx * part[m * kRows + r];
            const float u = sx * part[(MT + m) * kRows + r];
            const float sig = 1.0f / (1.0f + expf(-g));
            static_cast<float *>(p.out)[o] = g * sig * u;
        }
    }
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
    cuuint32_t box[2] = {kSBBytes, kRows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(packed), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

constexpr int kMaxDevices = 64;

template <int FMT, int MT, int MODE>
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
    p.residual = Lh.residual;
    p.out = Lh.out;
    p.ldo = Lh.ldo;

    // K split: bounded by the activation slice a CTA stages, then widened
    // (up to a cluster of 8) while the grid is short of two CTAs per SM.
    const int rowblocks = static_cast<int>(ceil_div(Lh.N, kRows));
    const int act_budget = 48 * 1024;
    int sb_max = act_budget / (MT * POS);
    if (sb_max < 1) sb_max = 1;
    int nsplit = static_cast<int>(ceil_div(p.SB, sb_max));
    if (MODE != kModePartials) {
        while (nsplit < 8 && rowblocks * nsplit < 2 * 148 && ceil_div(p.SB, nsplit + 1) >= kWarps)
            ++nsplit;
    }
    if (nsplit > 8) {
        *why = "K too large for an 8-CTA cluster split at this M";
        return cudaErrorInvalidValue;
    }
    p.sb_per_cta = static_cast<int>(ceil_div(p.SB, nsplit));
    p.nsplit = static_cast<int>(ceil_div(p.SB, p.sb_per_cta));
    if (MODE == kModePartials) p.nsplit = nsplit = static_cast<int>(ceil_div(p.SB, p.sb_per_cta));
    const int per_warp = static_cast<int>(ceil_div(p.sb_per_cta, kWarps));
    p.stages = (NMAT == 1) ? 4 : 3;
    if (p.stages > per_warp) p.stages = per_warp;
    if (p.stages < 1) p.stages = 1;

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
        e = cudaFuncSetAttribute(gemv_kernel<FMT, MT, MODE>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
        if (e != cudaSuccess) return e;
        smem_set[dev] = 1;
    }

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.nsplit, rowblocks, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = L.total;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    int na = 0;
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
    if (p.nsplit > 1) {
        attr[na].id = cudaLaunchAttributeClusterDimension;
        attr[na].val.clusterDim.x = p.nsplit;
        attr[na].val.clusterDim.y = 1;
        attr[na].val.clusterDim.z = 1;
        ++na;
    }
    cfg.attrs = attr;
    cfg.numAttrs = na;
    e = cudaLaunchKernelEx(&cfg, gemv_kernel<FMT, MT, MODE>, tm0, tm1, p);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

template <int FMT, int MODE>
static cudaError_t launch_mt(const GemvLaunch &L, cudaStream_t s, const char **why) {
    if (L.M <= 1) return launch_impl<FMT, 1, MODE>(L, s, why);
    if (L.M <= 2) return launch_impl<FMT, 2, MODE>(L, s, why);
    if (L.M <= 4) return launch_impl<FMT, 4, MODE>(L, s, why);
    if (L.M <= 8) return launch_impl<FMT, 8, MODE>(L, s, why);
    return launch_impl<FMT, 16, MODE>(L, s, why);
}

template <int FMT>
static cudaError_t launch_fmt(const GemvLaunch &L, cudaStream_t s, const char **why) {
    switch (L.mode) {
        case kModeGemv: return launch_mt<FMT, kModeGemv>(L, s, why);
        case kModeSwiglu: return launch_mt<FMT, kModeSwiglu>(L, s, why);
        default: return launch_mt<FMT, kModePartials>(L, s, why);
    }
}

cudaError_t launch_gemv(const GemvLaunch &L, cudaStream_t s, const char **why) {
    if (L.fmt == TERN_FMT_BASE3) return launch_fmt<TERN_FMT_BASE3>(L, s, why);
    return launch_fmt<TERN_FMT_2BIT>(L, s, why);
}

}  // namespace tern

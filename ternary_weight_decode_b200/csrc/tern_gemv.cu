// tern_gemv.cu -- CUDA-core engine of the ternary GEMV (dp4a on decoded
// digits), the activation-statistics kernel, the host-side helpers both
// engines use, and the engine dispatch.
//
// The method (Bonsai page, "Decode 为什么只能算一般"): stream the packed codes
// once, restore -1/0/+1 in registers, integer dot with the int8 activation,
// apply the FP16 group scale (4sapi page, section 三), never materialising
// dequantised weights; gate/up + SwiGLU fused; activations re-quantised per
// token (after a 128-point Hadamard rotation for the FFN input).
//
// This engine decodes a D3 word into five int8x4 digit words t_i = D_i -
// 3 D_(i-1) and dots them with dp4a (sum w q = sum t q - sum q per group);
// D2 fields are (X >> 2i) & 0x03030303.  A DB (bit-plane) pair is dotted
// plane by plane, the nonzero plane and the negative one (nonzero AND sign)
// masked one bit per byte (sum w q = sum n q - 2 sum (n s) q, nothing to
// subtract per group).  Each warp streams its own
// superblocks through a ring of TMA stages (32 x 128 B box per matrix,
// 128-byte swizzle, L2 evict-first, no multicast).  This is the default
// engine; the tensor-core engine (tern_gemv_tc.cu) replaces the dp4a with
// tcgen05 and is selected with tern_debug_select_engine.
#include <mutex>

#include "tern_gemv_common.cuh"

namespace tern {

__device__ int g_device_error = 0;

namespace {

struct CcLayout {
    int stage_bytes, act_off, sq_off, sc_off, part_off, sx_off, bar_off, total;
    int KS, GS, sc_stride;
};

template <int FMT, int MT, int NMAT>
__host__ __device__ inline CcLayout cc_layout(int sb_per_cta, int stages) {
    CcLayout L;
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

// Adds one finished group to the fp32 accumulators (or stores its partials).
// SUBQ: the accumulators hold sum t q with t = w + 1 (D3, D2), so the group
// sum of q is subtracted; a DB accumulator already holds sum w q.
template <int MT, int NMAT, int MODE, bool SUBQ = true>
__device__ __forceinline__ void finish_group(int (&acc)[NMAT][MT], float (&yacc)[NMAT][MT], int m,
                                             int gl, int row, const int *sq, int GS,
                                             const float *sc, int sc_stride,
                                             const GemvParams &p, int n, int gg) {
    const int s = SUBQ ? sq[m * GS + gl] : 0;
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
        // several token rows: the digit words once per chunk, shared by
        // every row (as the D3 path does)
        uint32_t t[NMAT][16];
        if (MT > 2) {
#pragma unroll
            for (int mat = 0; mat < NMAT; ++mat)
#pragma unroll
                for (int wi = 0; wi < 4; ++wi)
#pragma unroll
                    for (int i = 0; i < 4; ++i) t[mat][4 * wi + i] = (words[mat][wi] >> (2 * i)) & 0x03030303u;
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
                    for (int d = 0; d < 16; ++d) acc[mat][m] = dp4a_ss(t[mat][d], aw[d], acc[mat][m]);
                }
            }
            if (c & 1)
                finish_group<MT, NMAT, MODE>(acc, yacc, m, gl0 + (c >> 1), row, sq, GS, sc,
                                             sc_stride, p, n, g_base + (c >> 1));
        }
    }
}

// DB: each 16-byte chunk holds two word pairs (nonzero plane n, sign plane
// s) of 32 positions; bit 8j + i of a word is position 4i + j of its pair,
// so the byte mask 0x01010101 << i lines the pair's bits up with activation
// word i of the pair.
template <int MT, int NMAT, int MODE>
__device__ __forceinline__ void process_db(const uint8_t *stage, int sbl, int lane, int row,
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
        // several token rows: signed weight words once per chunk (a + 0xFE b
        // per byte: 1, -1 or 0, no carries), shared by every row
        uint32_t wq[NMAT][16];
        if (MT > 2) {
#pragma unroll
            for (int mat = 0; mat < NMAT; ++mat)
#pragma unroll
                for (int pr = 0; pr < 2; ++pr) {
                    const uint32_t nz = words[mat][2 * pr], ng = nz & words[mat][2 * pr + 1];
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        wq[mat][8 * pr + i] = ((nz >> i) & 0x01010101u) + 0xFEu * ((ng >> i) & 0x01010101u);
                }
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
                int sn = 0, sg = 0;
                if (MT <= 2) {
                    // masked bits: lane values 2^i * bit, summed per i and
                    // rescaled (exactly) by arithmetic shifts
                    int an[8] = {0, 0, 0, 0, 0, 0, 0, 0}, as[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll
                    for (int pr = 0; pr < 2; ++pr) {
                        const uint32_t nz = words[mat][2 * pr], ng = nz & words[mat][2 * pr + 1];
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            an[i] = dp4a_us(nz & (0x01010101u << i), aw[8 * pr + i], an[i]);
                            as[i] = dp4a_us(ng & (0x01010101u << i), aw[8 * pr + i], as[i]);
                        }
                    }
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        sn += an[i] >> i;
                        sg += as[i] >> i;
                    }
                    acc[mat][m] += sn - 2 * sg;
                } else {
#pragma unroll
                    for (int d = 0; d < 16; ++d) acc[mat][m] = dp4a_ss(wq[mat][d], aw[d], acc[mat][m]);
                }
            }
            if (c & 1)
                finish_group<MT, NMAT, MODE, false>(acc, yacc, m, gl0 + (c >> 1), row, sq, GS, sc,
                                                    sc_stride, p, n, g_base + (c >> 1));
        }
    }
}

template <int FMT, int MT, int MODE, int XIN>
__global__ void __launch_bounds__(kThreads)
    gemv_cc_kernel(const __grid_constant__ CUtensorMap tm0, const __grid_constant__ CUtensorMap tm1,
                   const GemvParams p) {
    constexpr int NMAT = (MODE == kModeSwiglu) ? 2 : 1;
    constexpr int POS = Fmt<FMT>::kPos;
    constexpr int GPS = Fmt<FMT>::kGroups;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);

    const int S = p.stages;
    const CcLayout L = cc_layout<FMT, MT, NMAT>(p.sb_per_cta, S);
    uint8_t *stages = smem;
    uint8_t *act = smem + L.act_off;
    int *sq = reinterpret_cast<int *>(smem + L.sq_off);
    float *sc = reinterpret_cast<float *>(smem + L.sc_off);
    float *part = reinterpret_cast<float *>(smem + L.part_off);
    float *sx = reinterpret_cast<float *>(smem + L.sx_off);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L.bar_off);

    const int split = blockIdx.x, rg = blockIdx.y;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int row = tid;
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
    const int KS = L.KS;
    if (XIN) {
        row_scales<MT>(sx, p, tid);
        __syncthreads();
        quantise_slice<MT>(sq, sx, p, sb0 * POS, KS, L.GS, tid, [&](int m, int k, uint32_t w) {
            *reinterpret_cast<uint32_t *>(act + m * KS + k) = w;
        });
    } else {
        stage_q<MT>(sq, p, sb0 * POS, KS, L.GS, tid, [&](int m, int k, uint4 v) {
            *reinterpret_cast<uint4 *>(act + m * KS + k) = v;
        });
    }
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
            process_d3<MT, NMAT, MODE>(stg, it, lane, row, act, KS, sq, L.GS, sc, L.sc_stride, yacc,
                                       p, n, (sb0 + it) * GPS);
        else if (FMT == TERN_FMT_BITPLANE)
            process_db<MT, NMAT, MODE>(stg, it, lane, row, act, KS, sq, L.GS, sc, L.sc_stride, yacc,
                                       p, n, (sb0 + it) * GPS);
        else
            process_d2<MT, NMAT, MODE>(stg, it, lane, row, act, KS, sq, L.GS, sc, L.sc_stride, yacc,
                                       p, n, (sb0 + it) * GPS);
        // every lane's reads of the stage ordered before its TMA refill
        fence_proxy_async_smem();
        __syncwarp();
        if (it + S < nsb) {
            if (lane == 0) issue(it + S);
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
        gemv_epilogue<MT, NMAT, MODE, XIN>(part, sx, p, split, rg, tid);
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

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
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

constexpr int kTargetCtas = 3 * 148;

template <int FMT, int MT, int MODE, int XIN>
cudaError_t launch_cc(const GemvLaunch &Lh, cudaStream_t s, const char **why) {
    constexpr int NMAT = (MODE == kModeSwiglu) ? 2 : 1;
    constexpr int POS = Fmt<FMT>::kPos;
    static DeviceOnce once;  // kernel attributes, set once per device

    GemvParams p;
    fill_params(p, Lh);
    const int rowgroups = static_cast<int>(ceil_div(Lh.N, kRowsCta));
    int sb_max = (48 * 1024) / (MT * POS);
    if (sb_max < 1) sb_max = 1;
    int nsplit = static_cast<int>(ceil_div(p.SB, sb_max));
    int want = static_cast<int>(ceil_div(kTargetCtas, rowgroups));
    if (want > 8) want = 8;
    if (nsplit < want) nsplit = want;
    if (nsplit > p.SB) nsplit = p.SB;
    nsplit = even_split(p.SB, nsplit);
    p.sb_per_cta = static_cast<int>(ceil_div(p.SB, nsplit));
    p.nsplit = static_cast<int>(ceil_div(p.SB, p.sb_per_cta));
    if (MODE != kModePartials && p.nsplit > 8) {
        *why = "K too large for an 8-CTA cluster split at this M";
        return cudaErrorInvalidValue;
    }
    p.stages = p.sb_per_cta < 3 ? p.sb_per_cta : 3;

    const CcLayout L = cc_layout<FMT, MT, NMAT>(p.sb_per_cta, p.stages);
    if (L.total > 227 * 1024) {
        *why = "shared memory plan exceeds 227 KB";
        return cudaErrorInvalidValue;
    }
    CUtensorMap tm0, tm1;
    if (!make_weight_tmap(&tm0, Lh.packed[0], Lh.row_bytes, Lh.N, Lh.row_stride) ||
        !make_weight_tmap(&tm1, Lh.packed[NMAT - 1], Lh.row_bytes, Lh.N, Lh.row_stride)) {
        *why = "cuTensorMapEncodeTiled failed or is unavailable";
        return cudaErrorInvalidValue;
    }
    int dev = 0;
    cudaError_t e = current_device(&dev);
    if (e != cudaSuccess) return e;
    e = once.run(dev, []() {
        cudaError_t r = cudaFuncSetAttribute(gemv_cc_kernel<FMT, MT, MODE, XIN>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
        if (r != cudaSuccess) return r;
        // The largest shared-memory split for every launch, so that a launch
        // waiting on its predecessor (programmatic launch) can share its SMs:
        // launches whose splits differ cannot, and the SM drains first.
        return cudaFuncSetAttribute(gemv_cc_kernel<FMT, MT, MODE, XIN>,
                                    cudaFuncAttributePreferredSharedMemoryCarveout,
                                    cudaSharedmemCarveoutMaxShared);
    });
    if (e != cudaSuccess) return e;
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
    e = cudaLaunchKernelEx(&cfg, gemv_cc_kernel<FMT, MT, MODE, XIN>, tm0, tm1, p);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

template <int FMT, int MODE, int XIN>
cudaError_t launch_cc_mt(const GemvLaunch &L, cudaStream_t s, const char **why) {
    if (L.M <= 1) return launch_cc<FMT, 1, MODE, XIN>(L, s, why);
    if (L.M <= 2) return launch_cc<FMT, 2, MODE, XIN>(L, s, why);
    if (L.M <= 4) return launch_cc<FMT, 4, MODE, XIN>(L, s, why);
    if (L.M <= 8) return launch_cc<FMT, 8, MODE, XIN>(L, s, why);
    return launch_cc<FMT, 16, MODE, XIN>(L, s, why);
}

template <int FMT>
cudaError_t launch_cc_fmt(const GemvLaunch &L, cudaStream_t s, const char **why) {
    if (L.x) {
        if (L.mode == kModeSwiglu) return launch_cc_mt<FMT, kModeSwiglu, 1>(L, s, why);
        return launch_cc_mt<FMT, kModeGemv, 1>(L, s, why);
    }
    switch (L.mode) {
        case kModeGemv: return launch_cc_mt<FMT, kModeGemv, 0>(L, s, why);
        case kModeSwiglu: return launch_cc_mt<FMT, kModeSwiglu, 0>(L, s, why);
        default: return launch_cc_mt<FMT, kModePartials, 0>(L, s, why);
    }
}

int g_engine = 1;  // 0: tensor cores, 1: CUDA cores (default); set by a test hook

}  // namespace

bool make_u8_tmap_2d(CUtensorMap *map, const void *base, uint64_t inner, uint64_t rows,
                     uint64_t stride, uint32_t box_inner, uint32_t box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(stride)};
    cuuint32_t box[2] = {box_inner, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool make_weight_tmap3d(CUtensorMap *map, const void *packed, int N, int64_t row_stride,
                        int sb_full, int box_sb) {
    EncodeTiledFn fn = encode_fn();
    if (!fn || sb_full < 1) return false;
    // (byte in superblock, row, superblock): only whole superblocks, so no
    // box reaches past a row's used bytes
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(kSBBytes), static_cast<cuuint64_t>(N),
                          static_cast<cuuint64_t>(sb_full)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(row_stride), static_cast<cuuint64_t>(kSBBytes)};
    cuuint32_t box[3] = {kSBBytes, 32, static_cast<cuuint32_t>(box_sb)};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(packed), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool make_weight_tmap(CUtensorMap *map, const void *packed, int64_t row_bytes, int N,
                      int64_t row_stride) {
    return make_u8_tmap_2d(map, packed, static_cast<uint64_t>(row_bytes), static_cast<uint64_t>(N),
                           static_cast<uint64_t>(row_stride), kSBBytes, 32);
}

void fill_params(GemvParams &p, const GemvLaunch &L) {
    p = GemvParams{};
    p.N = L.N;
    p.K = L.K;
    p.G = L.G;
    p.SB = static_cast<int>(ceil_div(L.row_bytes, kSBBytes));
    p.M = L.M;
    p.prefetch_ok = L.prefetch_ok;
    p.scales0 = L.scales[0];
    p.scales1 = L.scales[1];
    p.q = L.q;
    p.ldq = L.ldq;
    p.s_x = L.s_x;
    p.x = L.x;
    p.ldx = L.ldx;
    p.x_stats = L.x_stats;
    p.x_stats_ld = L.x_stats_ld;
    p.qflags = L.qflags;
    p.residual = L.residual;
    p.out = L.out;
    p.ldo = L.ldo;
    p.y_stats = L.y_stats;
    p.y_stats_ld = L.y_stats_ld;
}

void select_engine(int engine) { g_engine = engine; }

cudaError_t launch_gemv(const GemvLaunch &L, cudaStream_t s, const char **why) {
    if (g_engine == 0 && L.mode != kModePartials) {
        if (L.fmt == TERN_FMT_BITPLANE) {
            *why = "the tensor-core GEMV engine has no bit-plane form";
            return cudaErrorInvalidValue;
        }
        return launch_gemv_tc(L, s, why);
    }
    if (L.fmt == TERN_FMT_BASE3) return launch_cc_fmt<TERN_FMT_BASE3>(L, s, why);
    if (L.fmt == TERN_FMT_BITPLANE) return launch_cc_fmt<TERN_FMT_BITPLANE>(L, s, why);
    return launch_cc_fmt<TERN_FMT_2BIT>(L, s, why);
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

// tern_gemm.cu -- prefill GEMM of a ternary weight matrix with int8
// activations on the 5th-generation tensor cores (tcgen05.mma kind::i8).
//
//   Y[m][n] = s_x[m] * sum_g s_w[n][g] * P[m][n][g],
//   P[m][n][g] = sum_{k in group g} w[n][k] q[m][k]          (exact int32)
//
// (Bonsai page, "Decode 为什么只能算一般": prefill is a large matrix multiply
// over the same packed weights; 4sapi page, section 三: integer products of
// the signs, then one FP16 scale per group of 128.)
//
// One CTA computes a 128-row (n) x 128-token (m) tile of Y over all of K:
//  * warp 0 (TMA): per 128-byte superblock of codes, the 128 x 128 B code
//    tile; per group of 128 K, the 128 x 128 B activation tile -- both with
//    128-byte swizzle, no multicast;
//  * warps 2..5 (decode, one weight row per thread): the row's 32 code words
//    of the superblock into registers, then per group the signed int8
//    weights w = t - 1 into a 128 x 128 B tile in the 128-byte-swizzled
//    K-major layout the MMA reads (trits never leave the SM);
//  * warp 1 (MMA, one thread): per group four tcgen05.mma (K = 32 each), A =
//    weights, B = activations, int32 accumulator in tensor memory -- two
//    accumulator buffers of 128 columns, so group g+1 is multiplied while
//    group g is drained;
//  * warps 6..13 (epilogue, two per tensor-memory lane quarter, 64 token
//    columns each): per group tcgen05.ld of the int32 partials, exact int ->
//    float, acc += s_w[n][g] * P in fp32 registers (group order, as the
//    definition reads); at the end Y = s_x[m] * acc.
// The per-group scale is why the accumulator is drained every 128 K: the
// tensor cores accumulate only the exact integer partial of one group.
#include "tern_gemv_common.cuh"
#include "tern_tc.cuh"

namespace tern {
namespace {

constexpr int kGmTileN = 128;   // weight rows per CTA (MMA M)
constexpr int kGmTileM = 128;   // tokens per CTA (MMA N)
constexpr int kGmTile = 128 * 128;  // bytes of one 128 x 128 B int8 tile
constexpr int kGmCodeStages = 2;
constexpr int kGmActStages = 4;
constexpr int kGmAStages = 2;
constexpr int kGmDecodeWarps = 4;
constexpr int kGmEpiWarps = 8;
constexpr int kGmWarps = 2 + kGmDecodeWarps + kGmEpiWarps;
constexpr int kGmThreads = 32 * kGmWarps;
constexpr int kGmTmemCols = 256;  // two 128-column int32 accumulators

struct GemmParams {
    int N, K, M, G, SB;
    const uint16_t *scales;  // fp16 [N][G]
    const float *s_x;        // [M]
    float *y;
    int ldy;
};

struct GemmSmem {
    uint8_t code[kGmCodeStages][kGmTile];
    uint8_t act[kGmActStages][kGmTile];
    uint8_t a[kGmAStages][kGmTile];
    uint64_t code_full[kGmCodeStages], code_empty[kGmCodeStages];
    uint64_t act_full[kGmActStages], act_empty[kGmActStages];
    uint64_t a_full[kGmAStages], a_empty[kGmAStages];
    uint64_t acc_full[2], acc_empty[2];
    uint32_t tmem_base;
};

// w = t - 1 on four packed digits t in {0, 1, 2}: no byte carries.
__device__ __forceinline__ uint32_t signed_trits(uint32_t t) { return (t + 0x7F7F7F7Fu) ^ 0x80808080u; }

// Exact int -> float for |v| < 2^22 on the full-rate pipes.
__device__ __forceinline__ float int_to_float_exact(uint32_t v) {
    return __int_as_float(static_cast<int>(v) + 0x4B400000) - 12582912.0f;
}

template <int FMT>
__global__ void __launch_bounds__(kGmThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_q,
                const GemmParams p) {
    constexpr int GPS = FMT == TERN_FMT_BASE3 ? 5 : 4;  // groups per superblock
    extern __shared__ uint8_t smem_raw[];
    GemmSmem &S = *reinterpret_cast<GemmSmem *>(
        smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023));
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int n0 = blockIdx.x * kGmTileN, m0 = blockIdx.y * kGmTileM;
    const int G = p.G;
    // After a failed wait anywhere (recorded in the device error word) the
    // remaining CTAs leave at once instead of timing out one by one.
    if (*reinterpret_cast<volatile int *>(&g_device_error) != 0) return;

    if (tid == 0) {
        prefetch_tmap(&tm_w);
        prefetch_tmap(&tm_q);
        for (int i = 0; i < kGmCodeStages; ++i) {
            mbar_init(&S.code_full[i], 1);
            mbar_init(&S.code_empty[i], kGmDecodeWarps);
        }
        for (int i = 0; i < kGmActStages; ++i) {
            mbar_init(&S.act_full[i], 1);
            mbar_init(&S.act_empty[i], 1);
        }
        for (int i = 0; i < kGmAStages; ++i) {
            mbar_init(&S.a_full[i], kGmDecodeWarps);
            mbar_init(&S.a_empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&S.acc_full[i], 1);
            mbar_init(&S.acc_empty[i], kGmEpiWarps);
        }
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&S.tmem_base, kGmTmemCols);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = S.tmem_base;
    pdl_launch_dependents();

    if (warp == 0) {
        // ------------------------------------------------------------- TMA
        if (lane == 0) {
            pdl_wait();
            int g = 0;
            for (int sb = 0; sb < p.SB && g < G; ++sb) {
                const int cs = sb % kGmCodeStages;
                if (sb >= kGmCodeStages &&
                    !mbar_wait_bounded(&S.code_empty[cs], ((sb / kGmCodeStages) - 1) & 1))
                    break;
                mbar_arrive_expect_tx(&S.code_full[cs], kGmTile);
                tma_load_2d_nohint(S.code[cs], &tm_w, sb * 128, n0, &S.code_full[cs]);
                for (int gg = 0; gg < GPS && g < G; ++gg, ++g) {
                    const int as = g % kGmActStages;
                    if (g >= kGmActStages &&
                        !mbar_wait_bounded(&S.act_empty[as], ((g / kGmActStages) - 1) & 1))
                        break;
                    mbar_arrive_expect_tx(&S.act_full[as], kGmTile);
                    tma_load_2d_nohint(S.act[as], &tm_q, g * 128, m0, &S.act_full[as]);
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------- MMA
        if (lane == 0) {
            const uint32_t idesc = idesc_i8(kGmTileN, kGmTileM, 1, 1);
            for (int g = 0; g < G; ++g) {
                const int as = g % kGmAStages, qs = g % kGmActStages, buf = g & 1;
                bool ok = mbar_wait_bounded(&S.a_full[as], (g / kGmAStages) & 1);
                ok = ok && mbar_wait_bounded(&S.act_full[qs], (g / kGmActStages) & 1);
                if (g >= 2) ok = ok && mbar_wait_bounded(&S.acc_empty[buf], ((g >> 1) - 1) & 1);
                if (!ok) break;
                tc_fence_after_sync();
                const uint32_t a0 = smem_u32(S.a[as]), b0 = smem_u32(S.act[qs]);
#pragma unroll
                for (int s = 0; s < 4; ++s)
                    mma_i8_ss(tmem + buf * 128, smem_desc_sw128(a0 + 32 * s),
                              smem_desc_sw128(b0 + 32 * s), idesc, s > 0);
                tc_commit(&S.acc_full[buf]);
                tc_commit(&S.a_empty[as]);
                tc_commit(&S.act_empty[qs]);
            }
        }
    } else if (warp < 2 + kGmDecodeWarps) {
        // ---------------------------------------------------------- decode
        const int r = tid - 64;  // weight row of the tile, 0..127
        int g = 0;
        for (int sb = 0; sb < p.SB && g < G; ++sb) {
            const int cs = sb % kGmCodeStages;
            if (!__all_sync(0xffffffffu,
                            mbar_wait_bounded(&S.code_full[cs], (sb / kGmCodeStages) & 1)))
                break;
            uint32_t words[32];
            const uint8_t *row = S.code[cs] + r * 128;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const uint4 v = lds128(row + ((c ^ (r & 7)) << 4));
                words[4 * c + 0] = v.x;
                words[4 * c + 1] = v.y;
                words[4 * c + 2] = v.z;
                words[4 * c + 3] = v.w;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&S.code_empty[cs]);
#pragma unroll
            for (int gg = 0; gg < GPS; ++gg) {
                if (g >= G) break;
                const int as = g % kGmAStages;
                if (g >= kGmAStages &&
                    !__all_sync(0xffffffffu,
                                mbar_wait_bounded(&S.a_empty[as], ((g / kGmAStages) - 1) & 1)))
                    break;
                uint8_t *arow = S.a[as] + r * 128;
                // 32 words of 4 signed weights = this row's 128 K of group g
                uint32_t wq[32];
                if constexpr (FMT == TERN_FMT_BASE3) {
                    // D3: t-word d of the superblock (positions 4d..4d+3) is
                    // digit d % 5 of code word d / 5
#pragma unroll
                    for (int cw = (32 * gg) / 5; cw <= (32 * gg + 31) / 5; ++cw) {
                        uint32_t t[5];
                        decode_d3(words[cw], t);
#pragma unroll
                        for (int i = 0; i < 5; ++i) {
                            const int d = 5 * cw + i - 32 * gg;
                            if (d >= 0 && d < 32) wq[d] = signed_trits(t[i]);
                        }
                    }
                } else {
                    // D2: code word w holds positions 16w + 4i + j in bits
                    // [2i, 2i+1] of byte j; group gg = words 8gg .. 8gg+7
#pragma unroll
                    for (int w8 = 0; w8 < 8; ++w8) {
                        const uint32_t X = words[8 * gg + w8];
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            wq[4 * w8 + i] = signed_trits((X >> (2 * i)) & 0x03030303u);
                    }
                }
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    uint4 v;
                    v.x = wq[4 * c + 0];
                    v.y = wq[4 * c + 1];
                    v.z = wq[4 * c + 2];
                    v.w = wq[4 * c + 3];
                    *reinterpret_cast<uint4 *>(arow + ((c ^ (r & 7)) << 4)) = v;
                }
                fence_proxy_async_smem();  // read by the tensor cores
                __syncwarp();
                if (lane == 0) mbar_arrive(&S.a_full[as]);
                ++g;
            }
        }
    } else {
        // -------------------------------------------------------- epilogue
        const int e = warp - 2 - kGmDecodeWarps;  // 0..7
        const int quarter = warp & 3;             // tensor-memory lanes it reaches
        const int half = e >> 2;                  // token columns [64 half, 64 half + 64)
        const int n = n0 + 32 * quarter + lane;
        const uint32_t lane_addr = static_cast<uint32_t>(32 * quarter) << 16;
        float acc[64];
#pragma unroll
        for (int c = 0; c < 64; ++c) acc[c] = 0.0f;
        const uint16_t *srow = p.scales + static_cast<int64_t>(n < p.N ? n : 0) * G;
        float s_next = n < p.N ? __half2float(__ushort_as_half(__ldg(srow))) : 0.0f;
        for (int g = 0; g < G; ++g) {
            const int buf = g & 1;
            const float s = s_next;
            if (g + 1 < G && n < p.N) s_next = __half2float(__ushort_as_half(__ldg(srow + g + 1)));
            const bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(&S.acc_full[buf], (g >> 1) & 1));
            if (!ok) break;
            tc_fence_after_sync();
            uint32_t v[32];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                tmem_ld32(tmem + lane_addr + buf * 128 + 64 * half + 32 * h, v);
                tmem_wait_ld();
                if (h == 1) {
                    tc_fence_before_sync();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&S.acc_empty[buf]);
                }
#pragma unroll
                for (int c = 0; c < 32; ++c)
                    acc[32 * h + c] = fmaf(s, int_to_float_exact(v[c]), acc[32 * h + c]);
            }
        }
        pdl_wait();  // s_x comes from the previous kernel
        if (n < p.N) {
#pragma unroll
            for (int c = 0; c < 64; ++c) {
                const int m = m0 + 64 * half + c;
                if (m < p.M) p.y[static_cast<int64_t>(m) * p.ldy + n] = __ldg(p.s_x + m) * acc[c];
            }
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, kGmTmemCols);
    }
}

bool make_tmap_2d(CUtensorMap *map, const void *base, uint64_t inner, uint64_t rows, uint64_t stride,
                  uint32_t box_rows) {
    return make_u8_tmap_2d(map, base, inner, rows, stride, 128, box_rows);
}

size_t gemm_smem_bytes() { return sizeof(GemmSmem) + 1024; }

}  // namespace

cudaError_t launch_gemm(const GemmLaunch &L, cudaStream_t s, const char **why) {
    GemmParams p = {};
    p.N = L.N;
    p.K = L.K;
    p.M = L.M;
    p.G = static_cast<int>(ceil_div(L.K, 128));
    p.SB = static_cast<int>(ceil_div(L.row_bytes, 128));
    p.scales = L.scales;
    p.s_x = L.s_x;
    p.y = L.y;
    p.ldy = L.ldy;
    CUtensorMap tm_w, tm_q;
    if (!make_tmap_2d(&tm_w, L.packed, static_cast<uint64_t>(L.row_bytes), static_cast<uint64_t>(L.N),
                      static_cast<uint64_t>(L.row_stride), kGmTileN) ||
        !make_tmap_2d(&tm_q, L.q, static_cast<uint64_t>(L.K), static_cast<uint64_t>(L.M),
                      static_cast<uint64_t>(L.ldq), kGmTileM)) {
        *why = "cuTensorMapEncodeTiled failed or is unavailable";
        return cudaErrorInvalidValue;
    }
    const size_t smem = gemm_smem_bytes();
    cudaError_t e;
    auto kern = L.fmt == TERN_FMT_BASE3 ? gemm_kernel<TERN_FMT_BASE3> : gemm_kernel<TERN_FMT_2BIT>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(ceil_div(L.N, kGmTileN)),
                       static_cast<unsigned>(ceil_div(L.M, kGmTileM)), 1);
    cfg.blockDim = dim3(kGmThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, tm_w, tm_q, p);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace tern

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
// One CTA computes a 128-row (n) x 256-token (m) tile of Y over all of K,
// with 22 warps:
//  * warp 0 (TMA): per 128-byte superblock of codes, the 128 x 128 B code
//    tile; per group of 128 K, the 256 x 128 B activation tile -- both with
//    128-byte swizzle, no multicast;
//  * warp 1 (MMA, one thread): per group four tcgen05.mma (M = 128, N = 256,
//    K = 32 each), A = decoded weights, B = activations, int32 accumulator in
//    tensor memory -- two accumulator buffers of 256 columns (all 512), so
//    the tensor cores run one group ahead of the epilogue;
//  * warps 2..5 (decode; a thread = one weight row): the row's 32 code words
//    of the superblock into registers, then per group the signed int8
//    weights (w = t - 1 for D3 and D2; from the two bit planes for DB)
//    into a 128 x 128 B tile in the 128-byte-swizzled
//    K-major layout the MMA reads (trits never leave the SM), two tiles in
//    flight;
//  * warps 6..21 (epilogue, four per tensor-memory lane quarter, 64 token
//    columns each): the tile's group scales into shared memory once, then
//    per group tcgen05.ld of the int32 partials, int -> float (exact: the
//    partials are below 2^15), acc += s_w[n][g] * P in fp32 registers (group
//    order, as the definition reads); at the end Y = s_x[m] * acc.
// The per-group scale is why the accumulator is drained every 128 K: the
// tensor cores accumulate only the exact integer partial of one group.  The
// test-hook instantiation (DBG) also writes every partial P[m][n][g].
//
// Multi-token verify (Bonsai page, "后面还有没有优化空间": one weight read
// serving several candidate tokens) runs the same kernel with a narrower
// token tile, TM = 64 or 128 tokens (MMA N = TM), so that 17..128 token rows
// do not pay for a 256-token tile.  When the weight-row tiles are too few to
// fill the SMs (N = 5120: 40 tiles), a thread-block cluster of C CTAs splits
// the superblocks of K between its ranks; each rank accumulates its groups
// in fp32 as above, leaves its partial tile in shared memory, and rank 0
// adds the ranks' tiles in rank order (distributed shared memory) before
// the s_x multiply -- a fixed order, so the result does not depend on timing.
#include "tern_gemv_common.cuh"
#include "tern_tc.cuh"

namespace tern {
namespace {

constexpr int kGmTileN = 128;   // weight rows per CTA (MMA M)
constexpr int kGmTile = 128 * 128;  // bytes of one 128 x 128 B int8 tile (codes, decoded A)
constexpr int kGmCodeStages = 2;
constexpr int kGmDecodeWarps = 4;
constexpr int kGmEpiWarps = 16;
constexpr int kGmWarps = 2 + kGmDecodeWarps + kGmEpiWarps;
constexpr int kGmThreads = 32 * kGmWarps;
constexpr int kGmBand = 8;                     // weight-row tiles per raster band
constexpr int kGmEpiBar = 1;                   // named barrier of the epilogue warps
constexpr int kGmMaxSplit = 8;                 // portable cluster size

// Sizes that follow from the token tile TM (MMA N): 64, 128 or 256 tokens.
// The 64-token tile has little MMA and drain work per group: the time of a
// group there is the latency of decode -> MMA -> drain, so it keeps four
// groups in flight (activation tiles, decoded weight tiles, accumulators);
// the wider tiles keep two or three.
template <int TM>
struct GmShape {
    static_assert(TM == 64 || TM == 128 || TM == 256, "token tile");
    static constexpr int kActStages = TM == 64 ? 4 : 3;
    static constexpr int kAStages = TM == 64 ? 4 : 2;
    static constexpr int kAccBufs = TM == 64 ? 4 : 2;
    static constexpr int kActTile = TM * 128;          // one TM x 128 B activation tile
    static constexpr int kEpiCols = TM * 4 / kGmEpiWarps;  // token columns per epilogue warp
    static constexpr int kTmemCols = TM * kAccBufs;    // accumulators (a power of two)
    static_assert(kTmemCols <= 512, "tensor memory holds 512 columns");
};

struct GemmParams {
    int N, K, M, G, SB;
    const uint16_t *scales;  // fp16 [N][G]
    const float *s_x;        // [M]
    float *y;
    int ldy;
    int32_t *dbg_P;  // DBG kernels only: P [M][N][G]
};

template <int TM>
struct GemmSmem {
    uint8_t code[kGmCodeStages][kGmTile];
    uint8_t act[GmShape<TM>::kActStages][GmShape<TM>::kActTile];
    uint8_t a[GmShape<TM>::kAStages][kGmTile];
    uint64_t code_full[kGmCodeStages], code_empty[kGmCodeStages];
    uint64_t act_full[GmShape<TM>::kActStages], act_empty[GmShape<TM>::kActStages];
    uint64_t a_full[GmShape<TM>::kAStages], a_empty[GmShape<TM>::kAStages];
    uint64_t acc_full[GmShape<TM>::kAccBufs], acc_empty[GmShape<TM>::kAccBufs];
    uint32_t tmem_base;
    // followed, with a split of K, by this rank's fp32 partial tile [TM][128]
    // (token-major), then by the tile's group scales, fp16 [GL][128]
};

// w = t - 1 on four packed digits t in {0, 1, 2}: no byte carries.
__device__ __forceinline__ uint32_t signed_trits(uint32_t t) { return (t + 0x7F7F7F7Fu) ^ 0x80808080u; }

// One half (64 K) of group gg of a weight row: its 16 words of four signed
// weights, stored as four 16-byte chunks of the swizzled A tile row.
template <int FMT, int H>
__device__ __forceinline__ void decode_half(const uint32_t (&words)[32], int gg, uint8_t *arow, int r) {
    uint32_t wq[16];
    if constexpr (FMT == TERN_FMT_BASE3) {
        // D3: t-word d of the superblock (positions 4d..4d+3) is digit d % 5
        // of code word d / 5
        const int d0 = 32 * gg + 16 * H;
#pragma unroll
        for (int cw = d0 / 5; cw <= (d0 + 15) / 5; ++cw) {
            uint32_t t[5];
            decode_d3(words[cw], t);
#pragma unroll
            for (int i = 0; i < 5; ++i) {
                const int d = 5 * cw + i - d0;
                if (d >= 0 && d < 16) wq[d] = signed_trits(t[i]);
            }
        }
    } else if constexpr (FMT == TERN_FMT_BITPLANE) {
        // DB: word pair p (nonzero plane n, sign plane s) holds positions
        // 32p + 4i + j in bit 8j + i; group gg = pairs 4gg .. 4gg+3.  With
        // a = the n bits and b = the (n AND s) bits of four positions (one
        // per byte), w = a + 0xFE b is 0x01, 0xFF or 0 per byte: no carries.
#pragma unroll
        for (int pr = 0; pr < 2; ++pr) {
            const uint32_t nz = words[8 * gg + 4 * H + 2 * pr];
            const uint32_t ng = nz & words[8 * gg + 4 * H + 2 * pr + 1];
#pragma unroll
            for (int i = 0; i < 8; ++i)
                wq[8 * pr + i] = ((nz >> i) & 0x01010101u) + 0xFEu * ((ng >> i) & 0x01010101u);
        }
    } else {
        // D2: code word w holds positions 16w + 4i + j in bits [2i, 2i+1] of
        // byte j; group gg = words 8gg .. 8gg+7
#pragma unroll
        for (int w4 = 0; w4 < 4; ++w4) {
            const uint32_t X = words[8 * gg + 4 * H + w4];
#pragma unroll
            for (int i = 0; i < 4; ++i) wq[4 * w4 + i] = signed_trits((X >> (2 * i)) & 0x03030303u);
        }
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        uint4 v;
        v.x = wq[4 * c + 0];
        v.y = wq[4 * c + 1];
        v.z = wq[4 * c + 2];
        v.w = wq[4 * c + 3];
        *reinterpret_cast<uint4 *>(arow + (((4 * H + c) ^ (r & 7)) << 4)) = v;
    }
}

template <int FMT, bool DBG, int TM>
__global__ void __launch_bounds__(kGmThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_q,
                const GemmParams p) {
    using Sh = GmShape<TM>;
    constexpr int GPS = FMT == TERN_FMT_BASE3 ? 5 : 4;  // groups per superblock
    constexpr int EC = Sh::kEpiCols;
    constexpr int kGmActStages = Sh::kActStages;
    constexpr int kGmAStages = Sh::kAStages;
    constexpr int kGmAccBufs = Sh::kAccBufs;
    extern __shared__ uint8_t smem_raw[];
    GemmSmem<TM> &S = *reinterpret_cast<GemmSmem<TM> *>(
        smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023));
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // A cluster of C CTAs shares one output tile and splits its superblocks.
    const int C = static_cast<int>(cluster_nctarank());
    const int rank = static_cast<int>(cluster_ctarank());
    const int tile = blockIdx.x / C;
    // Tile order: bands of kGmBand weight-row tiles, token tiles fastest
    // inside a band, so the CTAs resident at one time cover a patch of about
    // kGmBand x (148 / kGmBand) tiles: each activation tile is read by about
    // kGmBand CTAs at once, not by every weight-row tile of the grid.
    const int tiles_n = (p.N + kGmTileN - 1) / kGmTileN, tiles_m = (p.M + TM - 1) / TM;
    const int band = tile / (kGmBand * tiles_m);
    const int band_w = min(kGmBand, tiles_n - band * kGmBand);
    const int in_band = tile - band * kGmBand * tiles_m;
    const int n0 = (band * kGmBand + in_band % band_w) * kGmTileN;
    const int m0 = (in_band / band_w) * TM;
    const int G = p.G;
    // this rank's superblocks and groups (C <= SB: every rank has some)
    const int sb_lo = p.SB * rank / C, sb_hi = p.SB * (rank + 1) / C;
    const int g_lo = min(G, sb_lo * GPS), g_hi = min(G, sb_hi * GPS);
    const int GL = g_hi - g_lo;
    // After a failed wait anywhere (recorded in the device error word) the
    // remaining CTAs leave at once instead of timing out one by one (not in
    // a cluster, whose peers would wait for the leaver).
    if (C == 1 && *reinterpret_cast<volatile int *>(&g_device_error) != 0) return;

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
        for (int i = 0; i < kGmAccBufs; ++i) {
            mbar_init(&S.acc_full[i], 1);
            mbar_init(&S.acc_empty[i], kGmEpiWarps);
        }
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&S.tmem_base, Sh::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = S.tmem_base;
    pdl_launch_dependents();
    // with a split of K: this rank's fp32 partial tile, at the same offset in
    // every rank (rank 0 reads the others' through distributed shared memory)
    float *red = reinterpret_cast<float *>(&S + 1);
    uint16_t *ssc = reinterpret_cast<uint16_t *>(red + (C > 1 ? TM * kGmTileN : 0));

    if (warp == 0) {
        // ------------------------------------------------------------- TMA
        if (lane == 0) {
            pdl_wait();
            int gl = 0;
            for (int sb = sb_lo; sb < sb_hi && gl < GL; ++sb) {
                const int sl = sb - sb_lo, cs = sl % kGmCodeStages;
                if (sl >= kGmCodeStages &&
                    !mbar_wait_bounded(&S.code_empty[cs], ((sl / kGmCodeStages) - 1) & 1))
                    break;
                mbar_arrive_expect_tx(&S.code_full[cs], kGmTile);
                tma_load_2d_nohint(S.code[cs], &tm_w, sb * 128, n0, &S.code_full[cs]);
                for (int gg = 0; gg < GPS && gl < GL; ++gg, ++gl) {
                    const int as = gl % kGmActStages;
                    if (gl >= kGmActStages &&
                        !mbar_wait_bounded(&S.act_empty[as], ((gl / kGmActStages) - 1) & 1))
                        break;
                    mbar_arrive_expect_tx(&S.act_full[as], Sh::kActTile);
                    tma_load_2d_nohint(S.act[as], &tm_q, (g_lo + gl) * 128, m0, &S.act_full[as]);
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------- MMA
        if (lane == 0) {
            // The issuing thread shares its scheduler with busy decode and
            // epilogue warps, so its loop is kept short: stage indices and
            // barrier parities advance incrementally, and the descriptors are
            // a stage's base plus 2 per 32-byte K step (the start-address
            // field counts 16-byte units and stays inside its 14 bits).
            const uint32_t idesc = idesc_i8(kGmTileN, TM, 1, 1);
            const uint64_t a_desc0 = smem_desc_sw128(smem_u32(S.a[0]));
            const uint64_t q_desc0 = smem_desc_sw128(smem_u32(S.act[0]));
            constexpr uint64_t kAStep = kGmTile >> 4, kQStep = Sh::kActTile >> 4;
            int as = 0, qs = 0, buf = 0;
            uint32_t pa = 0, pq = 0, pe = 1;
            for (int gl = 0; gl < GL; ++gl) {
                bool ok = mbar_wait_bounded(&S.a_full[as], pa);
                ok = ok && mbar_wait_bounded(&S.act_full[qs], pq);
                if (gl >= kGmAccBufs) ok = ok && mbar_wait_bounded(&S.acc_empty[buf], pe);
                if (!ok) break;
                tc_fence_after_sync();
                const uint64_t ad = a_desc0 + as * kAStep, qd = q_desc0 + qs * kQStep;
                const uint32_t d = tmem + buf * TM;
#pragma unroll
                for (int s = 0; s < 4; ++s) mma_i8_ss(d, ad + 2 * s, qd + 2 * s, idesc, s > 0);
                tc_commit(&S.acc_full[buf]);
                tc_commit(&S.a_empty[as]);
                tc_commit(&S.act_empty[qs]);
                if (++as == kGmAStages) {
                    as = 0;
                    pa ^= 1;
                }
                if (++qs == kGmActStages) {
                    qs = 0;
                    pq ^= 1;
                }
                if (++buf == kGmAccBufs) {
                    buf = 0;
                    pe ^= 1;
                }
            }
        }
    } else if (warp < 2 + kGmDecodeWarps) {
        // ---------------------------------------------------------- decode
        const int dt = tid - 64;
        const int r = dt & (kGmTileN - 1);  // weight row of the tile
        const int half = dt >> 7;           // which 64 K of each group (warp-uniform)
        int gl = 0;
        for (int sb = sb_lo; sb < sb_hi && gl < GL; ++sb) {
            const int sl = sb - sb_lo, cs = sl % kGmCodeStages;
            if (!__all_sync(0xffffffffu,
                            mbar_wait_bounded(&S.code_full[cs], (sl / kGmCodeStages) & 1)))
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
            release_to_tma(&S.code_empty[cs], lane);
#pragma unroll
            for (int gg = 0; gg < GPS; ++gg) {
                if (gl >= GL) break;
                const int as = gl % kGmAStages;
                if (gl >= kGmAStages &&
                    !__all_sync(0xffffffffu,
                                mbar_wait_bounded(&S.a_empty[as], ((gl / kGmAStages) - 1) & 1)))
                    break;
                uint8_t *arow = S.a[as] + r * 128;
                if constexpr (kGmDecodeWarps == 4) {
                    decode_half<FMT, 0>(words, gg, arow, r);  // a thread = one row, whole group
                    decode_half<FMT, 1>(words, gg, arow, r);
                } else if (half == 0) {
                    decode_half<FMT, 0>(words, gg, arow, r);
                } else {
                    decode_half<FMT, 1>(words, gg, arow, r);
                }
                fence_proxy_async_smem();  // read by the tensor cores
                __syncwarp();
                if (lane == 0) mbar_arrive(&S.a_full[as]);
                ++gl;
            }
        }
    } else {
        // -------------------------------------------------------- epilogue
        const int e = warp - 2 - kGmDecodeWarps;      // 0 .. kGmEpiWarps-1
        const int quarter = warp & 3;                  // tensor-memory lanes it reaches
        const int c0 = (e >> 2) * EC;                  // its token columns
        const int r = 32 * quarter + lane;             // tile row
        const int n = n0 + r;
        const uint32_t lane_addr = static_cast<uint32_t>(32 * quarter) << 16;
        // this rank's scales of the tile, group-major (conflict-free reads below)
        for (int idx = tid - 32 * (2 + kGmDecodeWarps); idx < kGmTileN * GL; idx += 32 * kGmEpiWarps) {
            const int rr = idx / GL, gg = idx % GL;
            ssc[gg * kGmTileN + rr] =
                n0 + rr < p.N ? p.scales[static_cast<int64_t>(n0 + rr) * G + g_lo + gg] : 0;
        }
        warpgroup_sync_n(kGmEpiBar, 32 * kGmEpiWarps);
        float acc[EC];
#pragma unroll
        for (int c = 0; c < EC; ++c) acc[c] = 0.0f;
        for (int gl = 0; gl < GL; ++gl) {
            const int buf = gl % kGmAccBufs;
            const float s = __half2float(__ushort_as_half(ssc[gl * kGmTileN + r]));
            const bool ok =
                __all_sync(0xffffffffu, mbar_wait_bounded(&S.acc_full[buf], (gl / kGmAccBufs) & 1));
            if (!ok) break;
            tc_fence_after_sync();
            uint32_t v[8];
#pragma unroll
            for (int h = 0; h < EC / 8; ++h) {
                tmem_ld8(tmem + lane_addr + buf * TM + c0 + 8 * h, v);
                tmem_wait_ld();
                if (h == EC / 8 - 1) {
                    tc_fence_before_sync();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&S.acc_empty[buf]);
                }
                // acc += s * float(P), two columns per packed FMA (each lane
                // rounds as fmaf does)
#pragma unroll
                for (int c = 0; c < 8; c += 2) {
                    const float2 a2 = __ffma2_rn(make_float2(s, s),
                                                 make_float2(__int2float_rn(static_cast<int>(v[c])),
                                                             __int2float_rn(static_cast<int>(v[c + 1]))),
                                                 make_float2(acc[8 * h + c], acc[8 * h + c + 1]));
                    acc[8 * h + c] = a2.x;
                    acc[8 * h + c + 1] = a2.y;
                }
                if constexpr (DBG) {
                    // test hook: the exact partials of this group
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        const int m = m0 + c0 + 8 * h + c;
                        if (m < p.M && n < p.N)
                            p.dbg_P[(static_cast<int64_t>(m) * p.N + n) * G + g_lo + gl] =
                                static_cast<int>(v[c]);
                    }
                }
            }
        }
        if (C == 1) {
            pdl_wait();  // s_x comes from the previous kernel
            if (n < p.N) {
#pragma unroll
                for (int c = 0; c < EC; ++c) {
                    const int m = m0 + c0 + c;
                    if (m < p.M) p.y[static_cast<int64_t>(m) * p.ldy + n] = __ldg(p.s_x + m) * acc[c];
                }
            }
        } else {
            // this rank's partial tile, token-major (lanes write consecutive rows)
#pragma unroll
            for (int c = 0; c < EC; ++c) red[(c0 + c) * kGmTileN + r] = acc[c];
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    if (C > 1) {
        cluster_sync();  // every rank's partial tile is in its shared memory
        if (rank == 0 && warp >= 2 + kGmDecodeWarps) {
            const int e = warp - 2 - kGmDecodeWarps;
            const int c0 = (e >> 2) * EC, r = 32 * (warp & 3) + lane, n = n0 + r;
            pdl_wait();
#pragma unroll 4
            for (int c = 0; c < EC; ++c) {
                float* own = red + (c0 + c) * kGmTileN + r;
                float v = *own;
                for (int q = 1; q < C; ++q) v += ld_shared_cluster_f32(map_shared_rank(own, q));
                const int m = m0 + c0 + c;
                if (n < p.N && m < p.M) p.y[static_cast<int64_t>(m) * p.ldy + n] = __ldg(p.s_x + m) * v;
            }
        }
        cluster_sync();  // peers keep their shared memory until rank 0 has read it
    }
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, Sh::kTmemCols);
    }
}

bool make_tmap_2d(CUtensorMap *map, const void *base, uint64_t inner, uint64_t rows, uint64_t stride,
                  uint32_t box_rows) {
    return make_u8_tmap_2d(map, base, inner, rows, stride, 128, box_rows);
}

template <int TM>
size_t gemm_smem_bytes(int GL, bool split) {
    return sizeof(GemmSmem<TM>) + (split ? static_cast<size_t>(TM) * kGmTileN * 4 : 0) +
           static_cast<size_t>(GL) * kGmTileN * 2 + 1024;
}

template <int TM>
cudaError_t launch_gemm_tm(const GemmLaunch &L, const GemmParams &p, int C, cudaStream_t s,
                           const char **why) {
    CUtensorMap tm_w, tm_q;
    if (!make_tmap_2d(&tm_w, L.packed, static_cast<uint64_t>(L.row_bytes), static_cast<uint64_t>(L.N),
                      static_cast<uint64_t>(L.row_stride), kGmTileN) ||
        !make_tmap_2d(&tm_q, L.q, static_cast<uint64_t>(L.K), static_cast<uint64_t>(L.M),
                      static_cast<uint64_t>(L.ldq), TM)) {
        *why = "cuTensorMapEncodeTiled failed or is unavailable";
        return cudaErrorInvalidValue;
    }
    const int GPS = L.fmt == TERN_FMT_BASE3 ? 5 : 4;
    const int per_rank = static_cast<int>(ceil_div(p.SB, C)) * GPS;  // groups of the widest rank
    const int GL_max = per_rank < p.G ? per_rank : p.G;
    const size_t smem = gemm_smem_bytes<TM>(GL_max, C > 1);
    if (smem > 227 * 1024) {
        *why = "K too large for the shared-memory scale block of the prefill GEMM (K <= 40960)";
        return cudaErrorInvalidValue;
    }
    auto kern = L.dbg_P ? (L.fmt == TERN_FMT_BASE3      ? gemm_kernel<TERN_FMT_BASE3, true, TM>
                           : L.fmt == TERN_FMT_BITPLANE ? gemm_kernel<TERN_FMT_BITPLANE, true, TM>
                                                        : gemm_kernel<TERN_FMT_2BIT, true, TM>)
                        : (L.fmt == TERN_FMT_BASE3      ? gemm_kernel<TERN_FMT_BASE3, false, TM>
                           : L.fmt == TERN_FMT_BITPLANE ? gemm_kernel<TERN_FMT_BITPLANE, false, TM>
                                                        : gemm_kernel<TERN_FMT_2BIT, false, TM>);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    const long long tiles = ceil_div(L.N, kGmTileN) * ceil_div(L.M, TM);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(tiles * C), 1, 1);
    cfg.blockDim = dim3(kGmThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = C;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = C > 1 ? 2 : 1;
    e = cudaLaunchKernelEx(&cfg, kern, tm_w, tm_q, p);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace

// Token tile and split of K for M token rows: the narrowest tile that holds
// them (64, 128; 256 beyond), and, for TM <= 128, a cluster split of K when
// the output tiles alone would leave most SMs idle.
void gemm_plan(int N, int M, int SB, int num_sms, int *TM, int *C) {
    *TM = M <= 64 ? 64 : (M <= 128 ? 128 : 256);
    *C = 1;
    const long long tiles = ceil_div(N, kGmTileN) * ceil_div(M, *TM);
    if (*TM <= 128 && tiles * 3 < 2LL * num_sms) {
        long long c = num_sms / tiles;
        if (c > kGmMaxSplit) c = kGmMaxSplit;
        if (c > SB) c = SB;
        if (c < 1) c = 1;
        *C = static_cast<int>(c);
    }
}

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
    p.dbg_P = L.dbg_P;
    int dev = 0, sms = 148;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    int TM = 256, C = 1;
    gemm_plan(L.N, L.M, p.SB, sms, &TM, &C);
    if (TM == 64) return launch_gemm_tm<64>(L, p, C, s, why);
    if (TM == 128) return launch_gemm_tm<128>(L, p, C, s, why);
    return launch_gemm_tm<256>(L, p, C, s, why);
}

}  // namespace tern

// tern_gemv_tc.cu -- tensor-core engine of the ternary GEMV.
//
// Same method and work decomposition as the CUDA-core engine (see
// tern_gemv_common.cuh); the integer dot product runs on the 5th-generation
// tensor cores instead of dp4a, which is what lets the decode keep pace
// with HBM on B200 (the CUDA-core instruction mix tops out below it).
//
//  * Each lane decodes its own row.  The decoded operand goes to tensor
//    memory (tcgen05.st, lane = row): 32-bit column c of a 128-position
//    scale group holds the four 8-bit values for K positions 4c..4c+3.
//  * D3 ("D-form"): the column holds the leading-digit numbers
//    D_i = floor(y 3^(i+1) / 256) of the code bytes, not the digits; the
//    activation operand B (shared memory) carries, per token m, row 2m =
//    q_m and row 2m+1 = q_m shifted by 4 positions (0 on the last digit of
//    each 20-position word), so one MMA yields sum D_i q_i and
//    sum D_i q_(i+1), and sum t q = acc[2m] - 3 acc[2m+1] since
//    t_i = D_i - 3 D_(i-1).  The digit subtraction never runs on the ALUs.
//  * D2: the column holds the digits t = (X >> 2i) & 0x03030303; B row m = q_m.
//  * sum w q = sum t q - sum q per group; the epilogue applies the fp16
//    group scale in fp32 (4sapi page, section 三).
//  * Pipeline per group (128 K positions): all lanes store their 32 columns,
//    a warpgroup barrier, one thread issues 4 MMAs (M = 128, N = 16 or 32,
//    K = 32 bytes each, kind::i8, A from tensor memory, B from shared
//    memory) and commits to an mbarrier; two tensor-memory slots alternate,
//    so the decode of group g+1 overlaps the MMA of group g, and group g's
//    accumulators are read back while g+2 is being decoded.
//  * Tensor memory is allocated before this kernel lets its dependents
//    launch, so a later kernel cannot hold columns this one waits for.
#include "tern_gemv_common.cuh"
#include "tern_tc.cuh"

namespace tern {
namespace {

template <int FMT, int MT>
struct TcShape {
    static constexpr int NR = (FMT == TERN_FMT_BASE3) ? 2 * MT : MT;  // accumulator columns used
    static constexpr int NB = NR <= 16 ? 16 : 32;                       // MMA N = rows of B
};

struct TcLayout {
    int stage_bytes, b_off, sq_off, sc_off, part_off, sx_off, bar_off, mbar_off, slot_off, total;
    int KS, GS, sc_stride;
};

template <int FMT, int MT, int NMAT>
__host__ __device__ inline TcLayout tc_layout(int sb_per_cta, int stages) {
    constexpr int NB = TcShape<FMT, MT>::NB;
    TcLayout L;
    L.KS = sb_per_cta * Fmt<FMT>::kPos;
    L.GS = sb_per_cta * Fmt<FMT>::kGroups;
    L.sc_stride = L.GS + 1;
    L.stage_bytes = NMAT * kTile;
    int off = kWarps * stages * L.stage_bytes;
    L.b_off = off;
    off = align128(off + NB * L.KS);
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
    L.mbar_off = off;
    off += 2 * 8;
    L.slot_off = off;
    off += 16;
    L.total = off + 1024;
    return L;
}

template <int NMAT>
__host__ __device__ constexpr int tmem_cols() {
    return NMAT == 1 ? 128 : 256;
}

// Tensor-memory columns: A slots first, then accumulator slots.
template <int NMAT, int NB>
__device__ __forceinline__ uint32_t a_col(int mat, int slot) {
    return static_cast<uint32_t>((mat * 2 + slot) * 32);
}
template <int NMAT, int NB>
__device__ __forceinline__ uint32_t acc_col(int mat, int slot) {
    return static_cast<uint32_t>(NMAT * 64 + (mat * 2 + slot) * NB);
}

struct TcCtx {
    uint32_t tbase, lane_base;
    uint32_t b_addr;  // shared-memory address of the B operand
    const uint8_t *b_ptr;
    uint64_t *mbar;   // two MMA-completion barriers
    const int *sq;
    const float *sc;
    int GS, sc_stride, row, tid;
};

// Reads the accumulators of CTA-local group gl (slot `slot`) into yacc.
// corr: the D3 cross term of the group's first digit-word (see
// process_superblock), added to the shifted column.
template <int FMT, int MT, int NMAT>
__device__ __forceinline__ void consume_group(const TcCtx &c, int gl, int slot,
                                              const int (&corr)[NMAT][MT],
                                              float (&yacc)[NMAT][MT]) {
    constexpr int NR = TcShape<FMT, MT>::NR;
    constexpr int NB = TcShape<FMT, MT>::NB;
    uint32_t v[NMAT][NR];
#pragma unroll
    for (int mat = 0; mat < NMAT; ++mat)
        tmem_ld_cols<NR>(c.tbase + c.lane_base + acc_col<NMAT, NB>(mat, slot), v[mat]);
    tmem_wait_ld();
#pragma unroll
    for (int m = 0; m < MT; ++m) {
        const int s = c.sq[m * c.GS + gl];
#pragma unroll
        for (int mat = 0; mat < NMAT; ++mat) {
            int P;
            if (FMT == TERN_FMT_BASE3)
                P = static_cast<int>(v[mat][2 * m]) -
                    3 * (static_cast<int>(v[mat][2 * m + 1]) + corr[mat][m]) - s;
            else
                P = static_cast<int>(v[mat][m]) - s;
            yacc[mat][m] = fmaf(c.sc[(mat * kRowsCta + c.row) * c.sc_stride + gl],
                                static_cast<float>(P), yacc[mat][m]);
        }
    }
}

// Stores group gl's operand columns, then one thread issues its MMAs.  First
// retires group gl - 2, whose MMA used the same tensor-memory slot.
template <int FMT, int MT, int NMAT>
__device__ __forceinline__ void flush_group(const TcCtx &c, int gl, uint32_t (&cur)[NMAT][32],
                                            int (&corr_slot)[2][NMAT][MT],
                                            const int (&corr_cur)[NMAT][MT],
                                            float (&yacc)[NMAT][MT]) {
    constexpr int NB = TcShape<FMT, MT>::NB;
    const int slot = gl & 1;
    if (gl >= 2) {
        mbar_wait_bounded(&c.mbar[slot], ((gl >> 1) - 1) & 1);
        tc_fence_after_sync();
        consume_group<FMT, MT, NMAT>(c, gl - 2, slot, corr_slot[slot], yacc);
    }
#pragma unroll
    for (int mat = 0; mat < NMAT; ++mat)
#pragma unroll
        for (int m = 0; m < MT; ++m) corr_slot[slot][mat][m] = corr_cur[mat][m];
#pragma unroll
    for (int mat = 0; mat < NMAT; ++mat)
        tmem_st32(c.tbase + c.lane_base + a_col<NMAT, NB>(mat, slot), cur[mat]);
    tmem_wait_st();
    tc_fence_before_sync();
    warpgroup_sync(1);
    if (c.tid == 0) {
        tc_fence_after_sync();
        constexpr uint32_t idesc = idesc_i8(128, NB, 0, 1);  // A unsigned (D or t), B signed (q)
        constexpr uint32_t lbo = (NB / 8) * 128;
#pragma unroll
        for (int mat = 0; mat < NMAT; ++mat)
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const uint64_t bd = smem_desc_noswizzle(c.b_addr + (8 * gl + 2 * kk) * lbo, lbo, 128);
                mma_i8_ts(c.tbase + acc_col<NMAT, NB>(mat, slot),
                          c.tbase + a_col<NMAT, NB>(mat, slot) + 8 * kk, bd, idesc, kk > 0);
            }
        tc_commit(&c.mbar[slot]);
    }
}

// One superblock (8 chunks of 16 bytes per row) of every matrix: decode into
// operand columns, flushing each 32-column group as it completes.
//
// D3 cross term: digit i+1 of a code byte contributes -3 D_i q_(i+1), which
// the MMA collects in the shifted column of digit i's position.  When a
// group boundary falls between digits i and i+1 of the same word (128 is not
// a multiple of 20), that term belongs to the next group: B's shifted row is
// zero there, and the term is formed here with one dp4a from the D word in
// registers and handed to the next group as its correction.
template <int FMT, int MT, int NMAT>
__device__ __forceinline__ void process_superblock(const TcCtx &c, const uint8_t *stage, int lane,
                                                   int g0, int sbl, int (&corr_slot)[2][NMAT][MT],
                                                   float (&yacc)[NMAT][MT]) {
    constexpr int NB = TcShape<FMT, MT>::NB;
    const int rsw = lane & 7;
    uint32_t cur[NMAT][32];
    int corr_cur[NMAT][MT];  // correction of the group being decoded
#pragma unroll
    for (int mat = 0; mat < NMAT; ++mat)
#pragma unroll
        for (int m = 0; m < MT; ++m) corr_cur[mat][m] = 0;  // superblocks start on a word boundary
#pragma unroll
    for (int ch = 0; ch < 8; ++ch) {
        uint32_t words[NMAT][4];
#pragma unroll
        for (int mat = 0; mat < NMAT; ++mat) {
            const uint4 wv = lds128(stage + mat * kTile + lane * kSBBytes + ((ch ^ rsw) << 4));
            words[mat][0] = wv.x;
            words[mat][1] = wv.y;
            words[mat][2] = wv.z;
            words[mat][3] = wv.w;
        }
#pragma unroll
        for (int wi = 0; wi < 4; ++wi) {
            if constexpr (FMT == TERN_FMT_BASE3) {
                uint32_t D[NMAT][5];
#pragma unroll
                for (int mat = 0; mat < NMAT; ++mat) decode_d3_D(words[mat][wi], D[mat]);
                // a word's five columns may straddle a group boundary: flush
                // as soon as a group's last column is in place
#pragma unroll
                for (int i = 0; i < 5; ++i) {
                    const int col = 20 * ch + 5 * wi + i;
#pragma unroll
                    for (int mat = 0; mat < NMAT; ++mat) cur[mat][col & 31] = D[mat][i];
                    if ((col & 31) == 31) {
                        int nxt[NMAT][MT];
#pragma unroll
                        for (int mat = 0; mat < NMAT; ++mat)
#pragma unroll
                            for (int m = 0; m < MT; ++m) nxt[mat][m] = 0;
                        if (i < 4) {  // digit i+1 of this word opens the next group
                            const int qpos = sbl * 640 + 4 * (col + 1);
#pragma unroll
                            for (int m = 0; m < MT; ++m) {
                                const uint32_t qw = *reinterpret_cast<const uint32_t *>(
                                    c.b_ptr + core_offset(2 * m, qpos, NB));
#pragma unroll
                                for (int mat = 0; mat < NMAT; ++mat) nxt[mat][m] = dp4a_us(D[mat][i], qw, 0);
                            }
                        }
                        flush_group<FMT, MT, NMAT>(c, g0 + (col >> 5), cur, corr_slot, corr_cur, yacc);
#pragma unroll
                        for (int mat = 0; mat < NMAT; ++mat)
#pragma unroll
                            for (int m = 0; m < MT; ++m) corr_cur[mat][m] = nxt[mat][m];
                    }
                }
            } else {
#pragma unroll
                for (int mat = 0; mat < NMAT; ++mat)
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        cur[mat][(16 * ch + 4 * wi + i) & 31] = (words[mat][wi] >> (2 * i)) & 0x03030303u;
                const int col = 16 * ch + 4 * wi + 3;
                if ((col & 31) == 31)
                    flush_group<FMT, MT, NMAT>(c, g0 + (col >> 5), cur, corr_slot, corr_cur, yacc);
            }
        }
    }
}

template <int FMT, int MT, int MODE, int XIN>
__global__ void __launch_bounds__(kThreads, 1)
    gemv_tc_kernel(const __grid_constant__ CUtensorMap tm0, const __grid_constant__ CUtensorMap tm1,
                   const GemvParams p) {
    constexpr int NMAT = (MODE == kModeSwiglu) ? 2 : 1;
    constexpr int POS = Fmt<FMT>::kPos;
    constexpr int GPS = Fmt<FMT>::kGroups;
    constexpr int NB = TcShape<FMT, MT>::NB;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);

    const int S = p.stages;
    const TcLayout L = tc_layout<FMT, MT, NMAT>(p.sb_per_cta, S);
    uint8_t *stages = smem;
    uint8_t *bop = smem + L.b_off;
    int *sq = reinterpret_cast<int *>(smem + L.sq_off);
    float *sc = reinterpret_cast<float *>(smem + L.sc_off);
    float *part = reinterpret_cast<float *>(smem + L.part_off);
    float *sx = reinterpret_cast<float *>(smem + L.sx_off);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L.bar_off);
    uint64_t *mbar = reinterpret_cast<uint64_t *>(smem + L.mbar_off);
    uint32_t *slot = reinterpret_cast<uint32_t *>(smem + L.slot_off);

    const int split = blockIdx.x, rg = blockIdx.y;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int sb0 = split * p.sb_per_cta;
    const int nsb = min(p.sb_per_cta, p.SB - sb0);

    if (tid == 0) {
        prefetch_tmap(&tm0);
        if (NMAT == 2) prefetch_tmap(&tm1);
        for (int i = 0; i < kWarps * S; ++i) mbar_init(&bars[i], 1);
        mbar_init(&mbar[0], 1);
        mbar_init(&mbar[1], 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(slot, tmem_cols<NMAT>());
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tbase = *slot;

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

    // ---- activation operand B (rows x KS bytes, core-matrix layout)
    const int KS = L.KS;
    constexpr int kRowOf = (FMT == TERN_FMT_BASE3) ? 2 : 1;  // B row of token m = kRowOf * m
    if (XIN) {
        row_scales<MT>(sx, p, tid);
        __syncthreads();
        quantise_slice<MT>(sq, sx, p, sb0 * POS, KS, L.GS, tid, [&](int m, int k, uint32_t w) {
            *reinterpret_cast<uint32_t *>(bop + core_offset(kRowOf * m, k, NB)) = w;
        });
    } else {
        stage_q<MT>(sq, p, sb0 * POS, KS, L.GS, tid, [&](int m, int k, uint4 v) {
            *reinterpret_cast<uint4 *>(bop + core_offset(kRowOf * m, k, NB)) = v;
        });
    }
    if constexpr (FMT == TERN_FMT_BASE3) {
        // row 2m+1: q_m shifted by 4 positions; 0 on the last digit of each
        // 20-position word and where the next digit opens a new scale group
        // (that cross term is added by the decode loop instead).  The K slice
        // starts on a word and group boundary.
        __syncthreads();
        const int words = KS / 4;
        for (int idx = tid; idx < MT * words; idx += kThreads) {
            const int m = idx / words, k = 4 * (idx % words);
            uint32_t w = 0;
            if (k % 20 < 16 && k % 128 != 124)
                w = *reinterpret_cast<const uint32_t *>(bop + core_offset(2 * m, k + 4, NB));
            *reinterpret_cast<uint32_t *>(bop + core_offset(2 * m + 1, k, NB)) = w;
        }
    }
    fence_proxy_async_smem();  // generic-proxy writes of B, read by the tensor cores
    __syncthreads();

    TcCtx ctx;
    ctx.tbase = tbase;
    ctx.lane_base = static_cast<uint32_t>(32 * warp) << 16;
    ctx.b_addr = smem_u32(bop);
    ctx.b_ptr = bop;
    ctx.mbar = mbar;
    ctx.sq = sq;
    ctx.sc = sc;
    ctx.GS = L.GS;
    ctx.sc_stride = L.sc_stride;
    ctx.row = tid;
    ctx.tid = tid;

    float yacc[NMAT][MT];
#pragma unroll
    for (int mat = 0; mat < NMAT; ++mat)
#pragma unroll
        for (int m = 0; m < MT; ++m) yacc[mat][m] = 0.0f;

    int corr_slot[2][NMAT][MT];
#pragma unroll
    for (int sl = 0; sl < 2; ++sl)
#pragma unroll
        for (int mat = 0; mat < NMAT; ++mat)
#pragma unroll
            for (int m = 0; m < MT; ++m) corr_slot[sl][mat][m] = 0;
    int consumed = 0;
    int groups = 0;
    for (int it = 0; it < nsb; ++it) {
        const int st = it % S;
        const bool ok = mbar_wait_bounded(&wbars[st], (it / S) & 1);
        if (__syncthreads_or(!ok)) break;  // CTA-uniform: every warp takes the same barriers
        consumed = it + 1;
        process_superblock<FMT, MT, NMAT>(ctx, wstages + st * L.stage_bytes, lane, groups, it,
                                          corr_slot, yacc);
        groups += GPS;
        // every lane's reads of the stage ordered before its TMA refill
        fence_proxy_async_smem();
        __syncwarp();
        if (it + S < nsb) {
            if (lane == 0) issue(it + S);
            ++issued;
        }
    }
    // retire the last two groups
    for (int g = max(0, groups - 2); g < groups; ++g) {
        mbar_wait_bounded(&mbar[g & 1], (g >> 1) & 1);
        tc_fence_after_sync();
        consume_group<FMT, MT, NMAT>(ctx, g, g & 1, corr_slot[g & 1], yacc);
    }
    // copies still in flight after an aborted stream land before exit
    for (int it = consumed; it < issued; ++it) mbar_wait_bounded(&wbars[it % S], (it / S) & 1);

    tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tbase, tmem_cols<NMAT>());

#pragma unroll
    for (int mat = 0; mat < NMAT; ++mat)
#pragma unroll
        for (int m = 0; m < MT; ++m) part[(mat * MT + m) * kRowsCta + tid] = yacc[mat][m];
    gemv_epilogue<MT, NMAT, MODE, XIN>(part, sx, p, split, rg, tid);
}

constexpr int kTargetCtas = 3 * 148;

template <int FMT, int MT, int MODE, int XIN>
cudaError_t launch_tc(const GemvLaunch &Lh, cudaStream_t s, const char **why) {
    constexpr int NMAT = (MODE == kModeSwiglu) ? 2 : 1;
    constexpr int POS = Fmt<FMT>::kPos;
    constexpr int NB = TcShape<FMT, MT>::NB;
    static DeviceOnce once;  // kernel attribute, set once per device

    GemvParams p;
    fill_params(p, Lh);
    const int rowgroups = static_cast<int>(ceil_div(Lh.N, kRowsCta));
    int sb_max = (96 * 1024) / (NB * POS);  // the B operand of a CTA's K slice
    if (sb_max < 1) sb_max = 1;
    int nsplit = static_cast<int>(ceil_div(p.SB, sb_max));
    int want = static_cast<int>(ceil_div(kTargetCtas, rowgroups));
    if (want > 8) want = 8;
    if (nsplit < want) nsplit = want;
    if (nsplit > p.SB) nsplit = p.SB;
    nsplit = even_split(p.SB, nsplit);  // as the CUDA-core engine: the same sum order
    p.sb_per_cta = static_cast<int>(ceil_div(p.SB, nsplit));
    p.nsplit = static_cast<int>(ceil_div(p.SB, p.sb_per_cta));
    if (p.nsplit > 8) {
        *why = "K too large for an 8-CTA cluster split at this M";
        return cudaErrorInvalidValue;
    }
    p.stages = p.sb_per_cta < 3 ? p.sb_per_cta : 3;
    const TcLayout L = tc_layout<FMT, MT, NMAT>(p.sb_per_cta, p.stages);
    if (L.total > 227 * 1024) {
        *why = "shared memory plan exceeds 227 KB";
        return cudaErrorInvalidValue;
    }
    // Never more CTAs on an SM than its 512 tensor-memory columns can serve at
    // once: a CTA waiting in tcgen05.alloc while its cluster peers wait for it
    // could otherwise deadlock against another cluster.  The shared-memory
    // request enforces the cap.
    const int max_ctas = 512 / tmem_cols<NMAT>();
    int smem_req = L.total;
    const int cap_req = 233472 / (max_ctas + 1) + 1024;
    if (smem_req < cap_req) smem_req = cap_req;
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
        return cudaFuncSetAttribute(gemv_tc_kernel<FMT, MT, MODE, XIN>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
    });
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.nsplit, rowgroups, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem_req;
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
    e = cudaLaunchKernelEx(&cfg, gemv_tc_kernel<FMT, MT, MODE, XIN>, tm0, tm1, p);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

template <int FMT, int MODE, int XIN>
cudaError_t launch_tc_mt(const GemvLaunch &L, cudaStream_t s, const char **why) {
    if (L.M <= 1) return launch_tc<FMT, 1, MODE, XIN>(L, s, why);
    if (L.M <= 2) return launch_tc<FMT, 2, MODE, XIN>(L, s, why);
    if (L.M <= 4) return launch_tc<FMT, 4, MODE, XIN>(L, s, why);
    if (L.M <= 8) return launch_tc<FMT, 8, MODE, XIN>(L, s, why);
    return launch_tc<FMT, 16, MODE, XIN>(L, s, why);
}

template <int FMT>
cudaError_t launch_tc_fmt(const GemvLaunch &L, cudaStream_t s, const char **why) {
    if (L.x) {
        if (L.mode == kModeSwiglu) return launch_tc_mt<FMT, kModeSwiglu, 1>(L, s, why);
        return launch_tc_mt<FMT, kModeGemv, 1>(L, s, why);
    }
    if (L.mode == kModeSwiglu) return launch_tc_mt<FMT, kModeSwiglu, 0>(L, s, why);
    return launch_tc_mt<FMT, kModeGemv, 0>(L, s, why);
}

}  // namespace

cudaError_t launch_gemv_tc(const GemvLaunch &L, cudaStream_t s, const char **why) {
    if (L.fmt == TERN_FMT_BASE3) return launch_tc_fmt<TERN_FMT_BASE3>(L, s, why);
    return launch_tc_fmt<TERN_FMT_2BIT>(L, s, why);
}

}  // namespace tern

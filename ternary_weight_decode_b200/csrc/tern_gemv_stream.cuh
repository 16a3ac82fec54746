// tern_gemv_stream.cuh -- streamed (persistent, evenly split) ternary GEMV for
// batch-1 / 2-token decode: the kernel and its launcher, as templates.  The
// release instantiations live in tern_gemv_stream.cu, the test-hook ones
// (DBG = true: they also write the int8 input, the row scales and every
// exact int32 group partial) in tern_debug_stream.cu.
//
// The method is that of tern_gemv.cu (Bonsai page, "Decode 为什么只能算一般":
// stream the packed codes once, restore -1/0/+1 in registers, integer dot,
// FP16 group scale -- 4sapi page, section 三); this file changes how the
// work is laid over the GPU so that one projection costs about its bytes:
//
//  * A "unit" is 32 rows x one 128-byte superblock of codes; an "item" is one
//    unit of one matrix (gate and up are two items of the same unit).  The
//    units of a matrix (row-block major) are cut into equal contiguous ranges,
//    one per CTA, one CTA per SM -- so every SM streams the same bytes.
//  * Warp 0 of a CTA is a producer: from the first instruction (before the
//    previous kernel on the stream has finished, when the matrix is static)
//    it streams its items into a ring of shared-memory slots: the 32 x 128 B
//    code tile by TMA (128-byte swizzle, L2 evict-first, no multicast) and the
//    unit's 32 x GPS scales, re-tiled at load time into unit order, by a bulk
//    copy.
//  * Warps 1..16 are consumers.  The input is quantised once per cluster of C
//    CTAs: each CTA takes 1/C of the 128-blocks of the fp32 input, forms its
//    share of max |x| (max |H x| with the Hadamard rotation) and of sum x^2,
//    sends it to every CTA of the cluster (st.async into their shared
//    memory), then quantises its blocks with the cluster-wide row scale and
//    sends the int8 codes and group sums to every CTA the same way.
//  * Consumers then take items round-robin: lane = row; decode + dp4a as in
//    tern_gemv.cu; one fp32 partial per (item, row, token).  A 2-bit item is
//    copied to registers and its ring slot handed back at once, so the whole
//    ring stays in flight; a base-3 item, whose decode outlasts the refill of
//    a slot, is read from the slot as it is decoded and handed back after.
//  * Row blocks inside a CTA's range are summed in unit order and written.
//    A row block cut by a range boundary belongs to two CTAs.  The one that
//    holds its end (its first units) publishes its partial as soon as those
//    units are done: value and tag in one 64-bit store into the workspace.
//    The one that holds its start adds that partial to its own at its end
//    (lower + upper: fixed order, so the result does not depend on timing)
//    with one relaxed 64-bit load, waiting (bounded) only if the tag is not
//    there yet, then clears the word -- the workspace is zero again after
//    every call.
#pragma once

#include "tern_gemv_common.cuh"

namespace tern {
namespace {

constexpr int kSkConsumers = 16;
constexpr int kSkThreads = 32 * (kSkConsumers + 1);
constexpr int kSkBar = 1;   // named barrier of the consumer warps
// Input blocks a consumer warp loads at once (one round) and keeps in
// registers between the two passes: a K of 5 x 16 warps x 128 = 10240 per
// CTA is one round; a longer share takes several, the earlier ones loaded
// again for the second pass.  The prologue is unrolled over a round and runs
// once per launch: rounds of 9 measured slower (with 8 consumer warps), their
// code costing more than the reloads they save.
constexpr int kSkKeep = 5;
constexpr int kSkMaxCluster = 4;
// One CTA per SM with 16 consumer warps and a ring of up to 40 unit slots.
// Measured on B200 against two CTAs per SM with 8 consumer warps and a
// 24-slot ring (which let the next launch's CTA prefetch beside this one):
// 2.73 vs 3.05 ms per base-3 decode step, 2.34 vs 2.46 ms for 2-bit.  The
// small projections (12 and 9 units per CTA) then decode every item at once
// instead of two after another; 20 consumer warps spill, 24 or 48 slots
// gain nothing.
constexpr int kSkSmemBudget = 200 * 1024;
constexpr int kSkMinRing = 8, kSkMaxRing = 40;  // unit slots, multiples of kSkChunk
constexpr int kSkChunk = 4;                      // unit slots filled by one chunk of loads

template <int FMT>
__host__ __device__ constexpr int scb() {
    return 32 * Fmt<FMT>::kGroups * 2;  // bytes of one unit's scales
}

struct SkParams {
    int N, K, SB, SBF, RB, R;  // SBF: whole superblocks per row
    long long U;
    int nCTA, M, prefetch_ok, qflags;
    const uint16_t *tsc0;
    const uint16_t *tsc1;
    const float *x;
    int ldx;
    const float *residual;
    float *out;
    int ldo;
    unsigned long long *ws_tag;  // tagged partials of cut row blocks, zero at rest
    // test hook (DBG kernels only): CTA 0's int8 input [M][dbg_ldq] and row
    // scales [M]; every exact group partial [NMAT][M][N][G]
    int8_t *dbg_q;
    int dbg_ldq;
    float *dbg_sx;
    int32_t *dbg_P;
    int G;
};

struct SkLayout {
    int ring_s_off, act_off, sq_off, xred_off, sx_off, red_off, misc_off, slots_off, bar_off, total;
    int Kpad, GT;
};

// Shared memory plan: ring of R slots (code tile + scales), the int8 input
// over the padded K (MT rows), its group sums (one per 16 bytes, so that a
// CTA's share is one aligned bulk copy), the cluster's partials of the row
// scale, row scales, per-warp partials, a counter, per-(item, token) row
// partials, barriers.
template <int FMT, int MT>
__host__ __device__ inline SkLayout sk_layout(int SB, int items_max, int R) {
    SkLayout L;
    L.Kpad = SB * Fmt<FMT>::kPos;
    L.GT = SB * Fmt<FMT>::kGroups;  // 128-blocks of the padded K
    int off = R * kTile;            // code tiles, 1024-aligned slots (128-byte swizzle)
    L.ring_s_off = off;
    off = align128(off + R * scb<FMT>());
    L.act_off = off;
    off = align128(off + MT * L.Kpad);
    L.sq_off = off;
    off = align128(off + MT * L.GT * 16);
    L.xred_off = off;
    off = align128(off + kSkMaxCluster * MT * 2 * 4);
    L.sx_off = off;
    off = align128(off + 2 * MT * 4);
    L.red_off = off;
    off = align128(off + kSkConsumers * MT * 2 * 4);
    L.misc_off = off;
    off = align128(off + 16);
    L.slots_off = off;
    off = align128(off + items_max * MT * 32 * 4);
    L.bar_off = off;
    off += (2 * R + 2) * 8;
    L.total = off + 1024;
    return L;
}

__device__ __forceinline__ void bulk_copy_g2s(void *dst, const void *src, uint32_t bytes,
                                              uint64_t *bar, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

// One item (this lane's row, one superblock of one matrix): the decode and
// dp4a of tern_gemv.cu.  words4(c): the row's code words 4c .. 4c+3 (bytes
// 16c .. 16c+15 of its 128, K order); sc: the row's GPS group scales; sq_sb:
// group sums of the input, one per 4 ints.  sink(m, g, P) sees every exact
// group partial P (a no-op outside the test hook).
template <int FMT, int MT, typename Words4, typename Sink>
__device__ __forceinline__ void sk_item(Words4 words4, const float (&sc)[Fmt<FMT>::kGroups],
                                        const uint8_t *act_sb, int Kpad, const int *sq_sb, int GT,
                                        float (&yacc)[MT], Sink sink) {
    // Two integer chains (base-3: even and odd digit words), so that one
    // dp4a need not wait for the one before; their sum is exact.
    int acc[MT], acc2[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) {
        acc[m] = 0;
        acc2[m] = 0;
        yacc[m] = 0.0f;
    }
    // sum w q = sum t q - sum q over the group (t = w + 1); the bit-plane
    // path accumulates sum w q itself
    auto finish = [&](int m, int g) {
        const int S = acc[m] + acc2[m];
        const int P = FMT == TERN_FMT_BITPLANE ? S : S - sq_sb[(m * GT + g) * 4];
        sink(m, g, P);
        yacc[m] = fmaf(sc[g], static_cast<float>(P), yacc[m]);
        acc[m] = 0;
        acc2[m] = 0;
    };
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        const uint4 wv = words4(c);
        const uint32_t words[4] = {wv.x, wv.y, wv.z, wv.w};
        if constexpr (FMT == TERN_FMT_BASE3) {
            uint32_t t[20];
#pragma unroll
            for (int wi = 0; wi < 4; ++wi) {
                uint32_t tw[5];
                decode_d3(words[wi], tw);
#pragma unroll
                for (int i = 0; i < 5; ++i) t[5 * wi + i] = tw[i];
            }
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                const uint8_t *a = act_sb + m * Kpad + c * 80;
                uint32_t aw[20];
#pragma unroll
                for (int j = 0; j < 5; ++j) {
                    const uint4 v = lds128(a + 16 * j);
                    aw[4 * j + 0] = v.x;
                    aw[4 * j + 1] = v.y;
                    aw[4 * j + 2] = v.z;
                    aw[4 * j + 3] = v.w;
                }
#pragma unroll
                for (int d = 0; d < 20; ++d) {
                    const int dd = c * 20 + d;
                    if (dd > 0 && (dd & 31) == 0) finish(m, (dd >> 5) - 1);
                    if (d & 1)
                        acc2[m] = dp4a_ss(t[d], aw[d], acc2[m]);
                    else
                        acc[m] = dp4a_ss(t[d], aw[d], acc[m]);
                }
            }
        } else if constexpr (FMT == TERN_FMT_BITPLANE) {
            // two word pairs (nonzero n, sign s) of 32 positions: bit 8j + i
            // of a word is position 4i + j of its pair, so the masked word
            // n & (0x01010101 << i) is 2^i times a 0/1 byte vector aligned
            // with activation word i; w = n (1 - 2 s).
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                const uint8_t *a = act_sb + m * Kpad + c * 64;
                uint32_t aw[16];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint4 v = lds128(a + 16 * j);
                    aw[4 * j + 0] = v.x;
                    aw[4 * j + 1] = v.y;
                    aw[4 * j + 2] = v.z;
                    aw[4 * j + 3] = v.w;
                }
                int an[8] = {0, 0, 0, 0, 0, 0, 0, 0}, as[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll
                for (int pr = 0; pr < 2; ++pr) {
                    const uint32_t nz = words[2 * pr], ng = words[2 * pr] & words[2 * pr + 1];
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        an[i] = dp4a_us(nz & (0x01010101u << i), aw[8 * pr + i], an[i]);
                        as[i] = dp4a_us(ng & (0x01010101u << i), aw[8 * pr + i], as[i]);
                    }
                }
                int sn = 0, sg = 0;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    sn += an[i] >> i;  // exact: an[i] is a multiple of 2^i
                    sg += as[i] >> i;
                }
                acc[m] += sn - 2 * sg;
                if (c & 1) finish(m, c >> 1);
            }
        } else {
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                const uint8_t *a = act_sb + m * Kpad + c * 64;
                uint32_t aw[16];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint4 v = lds128(a + 16 * j);
                    aw[4 * j + 0] = v.x;
                    aw[4 * j + 1] = v.y;
                    aw[4 * j + 2] = v.z;
                    aw[4 * j + 3] = v.w;
                }
                int a4[4] = {0, 0, 0, 0};
#pragma unroll
                for (int wi = 0; wi < 4; ++wi)
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        a4[i] = dp4a_us(words[wi] & (0x03030303u << (2 * i)), aw[4 * wi + i], a4[i]);
                acc[m] += a4[0] + (a4[1] >> 2) + (a4[2] >> 4) + (a4[3] >> 6);
                if (c & 1) finish(m, c >> 1);
            }
        }
    }
    if constexpr (FMT == TERN_FMT_BASE3) {
#pragma unroll
        for (int m = 0; m < MT; ++m) finish(m, 4);
    }
}

// Four floats at p (16-byte aligned) when `pred`, else zeros; one
// predicated L2 load, never reordered against the other volatile loads.
__device__ __forceinline__ void ld_cg_f32x4_pred(const float *p, bool pred, float (&r)[4]) {
    asm volatile(
        "{\n\t.reg .pred q;\n\t"
        "setp.ne.b32 q, %5, 0;\n\t"
        "mov.b32 %0, 0;\n\tmov.b32 %1, 0;\n\tmov.b32 %2, 0;\n\tmov.b32 %3, 0;\n\t"
        "@q ld.global.cg.v4.f32 {%0, %1, %2, %3}, [%4];\n\t}"
        : "=f"(r[0]), "=f"(r[1]), "=f"(r[2]), "=f"(r[3])
        : "l"(p), "r"(static_cast<int>(pred)));
}

// Lane's 4 values of 128-block b of token row m (zero past K and for m >= M).
__device__ __forceinline__ void load_block(const SkParams &p, int m, int b, int lane, float (&r)[4]) {
    r[0] = r[1] = r[2] = r[3] = 0.0f;
    const int k = 128 * b + 4 * lane;
    if (m >= p.M || k >= p.K) return;
    const float *src = p.x + static_cast<int64_t>(m) * p.ldx + k;
    if (k + 4 <= p.K) {
        const float4 v = __ldcg(reinterpret_cast<const float4 *>(src));
        r[0] = v.x;
        r[1] = v.y;
        r[2] = v.z;
        r[3] = v.w;
    } else {
        for (int e = 0; e < 4 && k + e < p.K; ++e) r[e] = __ldcg(src + e);
    }
}

__device__ __forceinline__ float sumsq4(const float (&r)[4]) {
    return fmaf(r[3], r[3], fmaf(r[2], r[2], fmaf(r[1], r[1], r[0] * r[0])));
}
__device__ __forceinline__ float amax4(const float (&r)[4]) {
    return fmaxf(fmaxf(fabsf(r[0]), fabsf(r[1])), fmaxf(fabsf(r[2]), fabsf(r[3])));
}

// Ring order of the items: chunk k holds units kCH .. kCH+CH-1 of matrix 0,
// then the same units of matrix 1.  Item (unit ul of the range, matrix).
template <int CH>
__host__ __device__ __forceinline__ int sk_item_index(int ul, int mat) {
    return (ul / CH) * kSkChunk + mat * CH + ul % CH;
}
template <int NMAT>
__host__ __device__ inline int sk_items_max(long long U, int nCTA) {
    const int units = static_cast<int>((U + nCTA - 1) / nCTA);
    return (units + kSkChunk / NMAT - 1) / (kSkChunk / NMAT) * kSkChunk;
}

// Index of the tagged partial of (row block, matrix, token, lane).
template <int NMAT, int MT>
__device__ __forceinline__ int64_t tag_index(int rb, int mat, int m, int lane) {
    return ((static_cast<int64_t>(rb) * NMAT + mat) * MT + m) * 32 + lane;
}

template <int FMT, int MT, int MODE, bool DBG>
__global__ void __launch_bounds__(kSkThreads, 1)
    gemv_stream_kernel(const __grid_constant__ CUtensorMap tm0,
                       const __grid_constant__ CUtensorMap tm1,
                       const __grid_constant__ CUtensorMap tm3_0,
                       const __grid_constant__ CUtensorMap tm3_1, const SkParams p) {
    constexpr int NMAT = (MODE == kModeSwiglu) ? 2 : 1;
    constexpr int CH = kSkChunk / NMAT;  // units of one matrix per ring chunk
    // Base-3 with one token row processes every slot of a round (see pass 1):
    // the rotated gate/up input takes rounds of 3 (one round up to K = 6144),
    // which waste fewer rotations on empty slots than rounds of 5 (gate/up
    // 16.2 -> 15.7 us); the unrotated projections keep rounds of 5, which
    // spare the down projection (K = 17408) a second round (12.3 vs 13.1 us).
    constexpr int KEEP = (MT == 1 && FMT == TERN_FMT_BASE3 && MODE == kModeSwiglu) ? 3 : kSkKeep;
    constexpr int POS = Fmt<FMT>::kPos;
    constexpr int GPS = Fmt<FMT>::kGroups;
    constexpr int SCB = scb<FMT>();
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);

    const int R = p.R;
    const long long U = p.U;
    const int c = blockIdx.x;
    const long long u0 = U * c / p.nCTA, u1 = U * (c + 1) / p.nCTA;
    const int nunits = static_cast<int>(u1 - u0);
    const int items_max = sk_items_max<NMAT>(U, p.nCTA);
    const SkLayout L = sk_layout<FMT, MT>(p.SB, items_max, R);
    const int RC = R / kSkChunk;  // chunks in the ring
    uint8_t *ring_w = smem;
    uint8_t *ring_s = smem + L.ring_s_off;
    uint8_t *act = smem + L.act_off;
    int *sq = reinterpret_cast<int *>(smem + L.sq_off);
    float *xred = reinterpret_cast<float *>(smem + L.xred_off);
    float *sx = reinterpret_cast<float *>(smem + L.sx_off);
    float *red = reinterpret_cast<float *>(smem + L.red_off);
    int *first_cnt = reinterpret_cast<int *>(smem + L.misc_off);
    float *slots = reinterpret_cast<float *>(smem + L.slots_off);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + L.bar_off);  // per chunk
    uint64_t *empty = full + RC;
    uint64_t *qbar1 = empty + RC;  // the peers' partials of the row scale arrived
    uint64_t *qbar2 = qbar1 + 1;  // the peers' int8 input and group sums arrived

    const int C = static_cast<int>(cluster_nctarank());
    const int rank = static_cast<int>(cluster_ctarank());
    // This CTA's share of the 128-blocks of the padded input.
    const int b_lo = L.GT * rank / C, b_hi = L.GT * (rank + 1) / C;
    const int nown = b_hi - b_lo;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid == 0) {
        prefetch_tmap(&tm0);
        prefetch_tmap(&tm3_0);
        if (NMAT == 2) {
            prefetch_tmap(&tm1);
            prefetch_tmap(&tm3_1);
        }
        for (int i = 0; i < RC; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], kSkChunk);
        }
        *first_cnt = 0;
        mbar_init(qbar1, 1);
        mbar_init(qbar2, 1);
        mbar_arrive_expect_tx(qbar1, (C - 1) * MT * 8);
        mbar_arrive_expect_tx(qbar2, MT * (L.GT - nown) * (128 + 16));
        fence_mbar_init();
    }
    // Every CTA of the cluster has its barriers ready before any peer sends.
    cluster_sync();
    pdl_launch_dependents();

    if (warp == 0) {
        // ---------------------------------------------------------- producer
        // The whole warp walks the ring (one lane issues), so that no lane
        // of it spins elsewhere while the copies are being issued.
        cluster_arrive();  // sends nothing: the exit barrier's arrival
        if (!p.prefetch_ok) pdl_wait();
        const uint64_t policy = l2_policy_evict_first();
        // A chunk is CH consecutive units of each matrix: one 3-D box of CH
        // whole superblocks when they lie in one row block (one TMA
        // instruction per 16 KB: the tile issue rate, not HBM, bounds small
        // boxes), else one 2-D box per unit; their scales in one bulk copy.
        // Positions advance incrementally: no division inside the loop.
        const int nchunks = (nunits + CH - 1) / CH;
        int cs = 0, round = 0;
        int rb = static_cast<int>(u0 / p.SB), sb = static_cast<int>(u0 % p.SB);
        const uint8_t *sc_unit[2] = {reinterpret_cast<const uint8_t *>(p.tsc0) + u0 * SCB,
                                     reinterpret_cast<const uint8_t *>(p.tsc1) + u0 * SCB};
        for (int k = 0; k < nchunks; ++k) {
            if (round > 0 &&
                !__all_sync(0xffffffffu, mbar_wait_bounded(&empty[cs], (round - 1) & 1)))
                break;
            const int nu = min(CH, nunits - k * CH);
            if (lane == 0) {
                mbar_arrive_expect_tx(&full[cs], nu * NMAT * (kTile + SCB));
                const bool whole = nu == CH && sb + CH <= p.SBF;
#pragma unroll
                for (int mat = 0; mat < NMAT; ++mat) {
                    const int slot0 = cs * kSkChunk + mat * CH;
                    if (whole) {
                        tma_load_3d(ring_w + slot0 * kTile, mat ? &tm3_1 : &tm3_0, 0, rb * 32, sb,
                                    &full[cs], policy);
                    } else {
                        int r2 = rb, s2 = sb;
                        for (int i = 0; i < nu; ++i) {
                            tma_load_2d(ring_w + (slot0 + i) * kTile, mat ? &tm1 : &tm0,
                                        s2 * kSBBytes, r2 * 32, &full[cs], policy);
                            if (++s2 == p.SB) {
                                s2 = 0;
                                ++r2;
                            }
                        }
                    }
                    bulk_copy_g2s(ring_s + slot0 * SCB, sc_unit[mat], nu * SCB, &full[cs], policy);
                }
            }
            __syncwarp();
            sc_unit[0] += CH * SCB;
            sc_unit[1] += CH * SCB;
            sb += CH;
            while (sb >= p.SB) {
                sb -= p.SB;
                ++rb;
            }
            if (++cs == RC) {
                cs = 0;
                ++round;
            }
        }
    } else {
        // ---------------------------------------------------------- consumers
        const int cw = warp - 1, ctid = tid - 32;
        const int rb_lo = static_cast<int>(u0 / p.SB);
        const int rb_hi = static_cast<int>((u1 - 1) / p.SB);
        // A cut first row block is published (its end is here), a cut last
        // row block is finished here (its start is here).
        const bool publish = static_cast<long long>(rb_lo) * p.SB < u0;
        const bool combine = static_cast<long long>(rb_hi + 1) * p.SB > u1;
        pdl_wait();
        // Residual of the first row block this warp finishes, fetched early.
        float res0[MT];
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            res0[m] = 0.0f;
            const int n = (rb_lo + cw) * 32 + lane;
            if (MODE == kModeGemv && p.residual && rb_lo + cw <= rb_hi && n < p.N && m < p.M)
                res0[m] = __ldcg(p.residual + static_cast<int64_t>(m) * p.ldo + n);
        }
        const bool rotate = (p.qflags & TERN_QUANT_FWHT128) != 0;
        const bool rms = (p.qflags & TERN_QUANT_RMSNORM) != 0;

        // The warp's blocks of this CTA's share are b_lo + cw + 8 (KEEP r + j),
        // taken in rounds r of KEEP.  A round's full 4-value loads are all
        // issued before any is used (predicated volatile loads: the compiler
        // may not interleave them with their uses); a block ending past K is
        // read by load_block afterwards.
        float v[MT][KEEP][4];
        auto blk = [&](int r, int j) { return b_lo + cw + kSkConsumers * (KEEP * r + j); };
        auto load_round = [&](int r) {
#pragma unroll
            for (int m = 0; m < MT; ++m)
#pragma unroll
                for (int j = 0; j < KEEP; ++j) {
                    const int b = blk(r, j);
                    const int k = 128 * b + 4 * lane;
                    const bool full = b < b_hi && m < p.M && k + 4 <= p.K;
                    ld_cg_f32x4_pred(p.x + static_cast<int64_t>(m) * p.ldx + k, full, v[m][j]);
                }
#pragma unroll
            for (int m = 0; m < MT; ++m)
#pragma unroll
                for (int j = 0; j < KEEP; ++j) {
                    const int b = blk(r, j);
                    const int k = 128 * b + 4 * lane;
                    if (b < b_hi && m < p.M && k < p.K && k + 4 > p.K) load_block(p, m, b, lane, v[m][j]);
                }
        };
        const int nblk = b_hi > b_lo + cw ? (b_hi - b_lo - cw + kSkConsumers - 1) / kSkConsumers : 0;
        const int nrounds = nblk > KEEP ? (nblk + KEEP - 1) / KEEP : 1;

        // pass 1: the rotation, max |.| and sum x^2 of the warp's blocks; the
        // last round stays in registers
        float amax[MT], ss[MT];
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            amax[m] = 0.0f;
            ss[m] = 0.0f;
        }
        // Base-3 with one token row processes every slot of a round, an
        // unused one holding zeros (which add nothing): no branch per block,
        // so the rotations' shuffle chains of a round overlap (measured:
        // base-3 step -1.5 %).  The other formats and two rows keep one loop
        // with a branch per block (the split loops measured +0.7 % for 2-bit).
        constexpr bool kAllSlots = MT == 1 && FMT == TERN_FMT_BASE3;
#pragma unroll 1
        for (int r = 0; r < nrounds; ++r) {
            load_round(r);
            if constexpr (kAllSlots) {
#pragma unroll
                for (int j = 0; j < KEEP; ++j) ss[0] += sumsq4(v[0][j]);
                if (rotate) {
#pragma unroll
                    for (int j = 0; j < KEEP; ++j) fwht128_warp(v[0][j], lane);
                }
#pragma unroll
                for (int j = 0; j < KEEP; ++j) amax[0] = fmaxf(amax[0], amax4(v[0][j]));
            } else {
#pragma unroll
                for (int m = 0; m < MT; ++m)
#pragma unroll
                    for (int j = 0; j < KEEP; ++j) {
                        if (blk(r, j) >= b_hi) continue;
                        ss[m] += sumsq4(v[m][j]);
                        if (rotate) fwht128_warp(v[m][j], lane);
                        amax[m] = fmaxf(amax[m], amax4(v[m][j]));
                    }
            }
        }
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            // max of non-negative floats = max of their bit patterns
            const float a = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(amax[m])));
            const float s = warp_sum(ss[m]);
            if (lane == 0) {
                red[(cw * MT + m) * 2 + 0] = a;
                red[(cw * MT + m) * 2 + 1] = s;
            }
        }
        warpgroup_sync_n(kSkBar, kSkConsumers * 32);
        // This CTA's share: lane w holds warp w's, combined across the lanes
        // by the same butterfly in every warp (hence the same sum in every
        // lane, warp and CTA).
        static_assert(kSkConsumers <= 32, "one consumer warp per lane");
        float amax_c[MT], ss_c[MT];
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            float a = 0.0f, s = 0.0f;
            if (lane < kSkConsumers) {
                a = red[(lane * MT + m) * 2 + 0];
                s = red[(lane * MT + m) * 2 + 1];
            }
            amax_c[m] = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(a)));
            ss_c[m] = warp_sum(s);
        }
        bool ok1 = true;
        if (C > 1) {
            // shares of the cluster: sent to the peers, combined in rank order
            if (ctid < MT) {
                const int m = ctid;
                xred[(rank * MT + m) * 2 + 0] = amax_c[m];
                xred[(rank * MT + m) * 2 + 1] = ss_c[m];
                for (int q = 0; q < C; ++q)
                    if (q != rank)
                        st_async_v2f32(map_shared_rank(xred + (rank * MT + m) * 2, q), amax_c[m],
                                       ss_c[m], map_shared_rank(qbar1, q));
            }
            warpgroup_sync_n(kSkBar, kSkConsumers * 32);
            ok1 = mbar_wait_cluster_bounded(qbar1, 0);
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                float a = 0.0f, s = 0.0f;
                for (int q = 0; q < C; ++q) {
                    const bool have = ok1 || q == rank;
                    a = fmaxf(a, have ? xred[(q * MT + m) * 2 + 0] : 0.0f);
                    s += have ? xred[(q * MT + m) * 2 + 1] : 0.0f;
                }
                amax_c[m] = a;
                ss_c[m] = s;
            }
        }
        // Row scale (the same in every CTA).
        float inv[MT];
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            const float a = amax_c[m], s = ss_c[m];
            float iv = 0.0f, sc = 0.0f;
            // The arithmetic of act_quant_fwht and of the fused entry points:
            // IEEE division for inv (it decides every int8 code) and for the
            // scale, IEEE square root for the RMS factor.
            if (a > 0.0f) {
                iv = __fdiv_rn(127.0f, a);
                sc = __fdiv_rn(a, 127.0f);
                if (rotate) sc = __fmul_rn(sc, kInvSqrt128);
            }
            if (rms) sc = sc / sqrtf(s / static_cast<float>(p.K) + 1e-6f);
            inv[m] = iv;
            if (ctid == 0) sx[m] = sc;
        }

        // pass 2: int8 codes and group sums of this CTA's blocks, written
        // here, then one bulk copy of the share to each peer
        auto quant_block = [&](int m, int b, const float (&r)[4]) {
            // q = rint(x * inv) (half to even), by the float adder: exact
            // for |x * inv| < 2^22; inv = 0 (all-zero row) gives q = 0
            int qi[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float t = __fadd_rn(__fmul_rn(r[e], inv[m]), 12582912.0f);
                qi[e] = max(-127, min(127, __float_as_int(t) - 0x4B400000));
            }
            const uint32_t packed =
                __byte_perm(__byte_perm(qi[0], qi[1], 0x0040), __byte_perm(qi[2], qi[3], 0x0040), 0x5410);
            const int qsum = __reduce_add_sync(0xffffffffu, dp4a_ss(packed, 0x01010101u, 0));
            *reinterpret_cast<uint32_t *>(act + m * L.Kpad + 128 * b + 4 * lane) = packed;
            if (lane == 0) sq[(m * L.GT + b) * 4] = qsum;
        };
        // the last round from registers; earlier ones loaded again, a round
        // at a time
#pragma unroll
        for (int m = 0; m < MT; ++m)
#pragma unroll
            for (int j = 0; j < KEEP; ++j) {
                const int b = blk(nrounds - 1, j);
                if (b < b_hi) quant_block(m, b, v[m][j]);
            }
#pragma unroll 1
        for (int r = 0; r + 1 < nrounds; ++r) {
            load_round(r);
#pragma unroll
            for (int m = 0; m < MT; ++m)
#pragma unroll
                for (int j = 0; j < KEEP; ++j) {
                    const int b = blk(r, j);
                    if (b >= b_hi) continue;
                    if (rotate) fwht128_warp(v[m][j], lane);
                    quant_block(m, b, v[m][j]);
                }
        }
        if (C > 1) fence_proxy_async_smem();  // the share is read by the bulk copies
        warpgroup_sync_n(kSkBar, kSkConsumers * 32);
        if (ctid == 0 && nown > 0) {
            for (int q = 0; q < C; ++q) {
                if (q == rank) continue;
                const uint32_t bar = map_shared_rank(qbar2, q);
                for (int m = 0; m < MT; ++m) {
                    uint8_t *a = act + m * L.Kpad + 128 * b_lo;
                    int *g = sq + (m * L.GT + b_lo) * 4;
                    bulk_copy_s2cluster(map_shared_rank(a, q), a, 128 * nown, bar);
                    bulk_copy_s2cluster(map_shared_rank(g, q), g, 16 * nown, bar);
                }
            }
        }
        const bool ok2 = mbar_wait_cluster_bounded(qbar2, 0);
        // Everything sent to this CTA has landed: its exit no longer waits
        // on it (and the peers' copies out of their shared memory are done).
        cluster_arrive();
        if constexpr (DBG) {
            // test hook: the int8 input and row scales as CTA 0 holds them
            if (blockIdx.x == 0) {
                for (int m = 0; m < p.M; ++m)
                    for (int k = ctid; k < p.K; k += kSkConsumers * 32)
                        p.dbg_q[static_cast<int64_t>(m) * p.dbg_ldq + k] =
                            static_cast<int8_t>(act[m * L.Kpad + k]);
                if (ctid < p.M) p.dbg_sx[ctid] = sx[ctid];
            }
        }

        // items, round-robin over the consumer warps (a warp always takes the
        // same position in a chunk, hence the same matrix); the item is copied
        // to registers and its chunk slot handed back at once.  Chunk, phase
        // and superblock advance incrementally (two chunks a step).
        const int pos = cw % kSkChunk, uoff = pos % CH;
        int kc = cw / kSkChunk;
        int kcs = kc % RC, phase = (kc / RC) & 1;
        int sb = static_cast<int>((u0 + kc * CH + uoff) % p.SB);
        const int n_first = publish ? static_cast<int>(static_cast<long long>(rb_lo + 1) * p.SB - u0) : 0;
        for (;; kc += kSkConsumers / kSkChunk) {
            const int ul = kc * CH + uoff;
            if (ul >= nunits) break;
            const int j = kc * kSkChunk + pos;
            const bool ok =
                ok2 && __all_sync(0xffffffffu, mbar_wait_bounded(&full[kcs], phase));
            const int slot = kcs * kSkChunk + pos;
            float yacc[MT];
            // test hook: every exact group partial of the item
            auto sink = [&](int m, int g, int P) {
                if constexpr (DBG) {
                    const int n = static_cast<int>((u0 + ul) / p.SB) * 32 + lane;
                    const int gg = sb * GPS + g;
                    if (m < p.M && n < p.N && gg < p.G)
                        p.dbg_P[(static_cast<int64_t>((pos / CH) * p.M + m) * p.N + n) * p.G + gg] = P;
                }
            };
            if (ok) {
                // the lane's row of the slot: 8 chunks of 16 bytes, 128-byte swizzle
                const uint8_t *wt = ring_w + slot * kTile + lane * kSBBytes;
                const int rsw = lane & 7;
                float sc[GPS];
                const uint16_t *st =
                    reinterpret_cast<const uint16_t *>(ring_s + slot * SCB) + lane * GPS;
#pragma unroll
                for (int g = 0; g < GPS; ++g) sc[g] = __half2float(__ushort_as_half(st[g]));
                if constexpr (FMT == TERN_FMT_BASE3) {
                    // The decode takes longer than the slot takes to refill:
                    // the words are read from the slot as they are used
                    // (fewer live registers for the decode), and the slot is
                    // handed back when the item is done.
                    sk_item<FMT, MT>([&](int cc) { return lds128(wt + ((cc ^ rsw) << 4)); }, sc,
                                     act + sb * POS, L.Kpad, sq + sb * GPS * 4, L.GT, yacc, sink);
                    release_to_tma(&empty[kcs], lane);
                } else {
                    // copied to registers, the slot handed back at once
                    uint4 wv[8];
#pragma unroll
                    for (int cc = 0; cc < 8; ++cc) wv[cc] = lds128(wt + ((cc ^ rsw) << 4));
                    release_to_tma(&empty[kcs], lane);
                    sk_item<FMT, MT>([&](int cc) { return wv[cc]; }, sc, act + sb * POS, L.Kpad,
                                     sq + sb * GPS * 4, L.GT, yacc, sink);
                }
            } else {
                release_to_tma(&empty[kcs], lane);
#pragma unroll
                for (int m = 0; m < MT; ++m) yacc[m] = 0.0f;
            }
#pragma unroll
            for (int m = 0; m < MT; ++m) slots[(j * MT + m) * 32 + lane] = yacc[m];
            kcs += kSkConsumers / kSkChunk;
            if (kcs >= RC) {
                kcs -= RC;
                phase ^= 1;
            }
            sb += (kSkConsumers / kSkChunk) * CH;
            while (sb >= p.SB) sb -= p.SB;
            if (ul < n_first) {
                // The last warp to finish an item of the cut first row block
                // publishes that row block's partial (value and tag in one
                // 64-bit store) for the CTA holding its start.
                __syncwarp();
                int done = 0;
                if (lane == 0) {
                    __threadfence_block();
                    done = atomicAdd(first_cnt, 1);
                }
                done = __shfl_sync(0xffffffffu, done, 0);
                if (done == n_first * NMAT - 1) {
                    __threadfence_block();
#pragma unroll
                    for (int mat = 0; mat < NMAT; ++mat)
#pragma unroll
                        for (int m = 0; m < MT; ++m) {
                            float s = 0.0f;
                            for (int uu = 0; uu < n_first; ++uu)
                                s += slots[(sk_item_index<CH>(uu, mat) * MT + m) * 32 + lane];
                            st_relaxed_gpu_u64(p.ws_tag + tag_index<NMAT, MT>(rb_lo, mat, m, lane),
                                               (1ull << 32) | __float_as_uint(s));
                        }
                }
            }
        }
        // The warp that finishes the cut last row block reads the partial its
        // neighbour published before the barrier, so that the load's latency
        // overlaps the wait for the slowest warp; if the tag is not there yet
        // it waits below.  (Every tag seen after the dependency wait is this
        // launch's: each launch clears the words it used before it ends.)
        unsigned long long early[NMAT][MT];
        const bool combine_here = combine && (rb_hi - rb_lo) % kSkConsumers == cw && !(rb_hi == rb_lo && publish);
#pragma unroll
        for (int mat = 0; mat < NMAT; ++mat)
#pragma unroll
            for (int m = 0; m < MT; ++m)
                early[mat][m] = combine_here ? ld_relaxed_gpu_u64(p.ws_tag + tag_index<NMAT, MT>(rb_hi, mat, m, lane))
                                             : 0ull;
        warpgroup_sync_n(kSkBar, kSkConsumers * 32);

        // row blocks of this range: sum units in order; finish
        int i = 0;
        for (int rb = rb_lo + cw; rb <= rb_hi; rb += kSkConsumers, ++i) {
            if (rb == rb_lo && publish) continue;
            const long long ua = max(u0, static_cast<long long>(rb) * p.SB);
            const long long ub = min(u1, static_cast<long long>(rb + 1) * p.SB);
            float tot[NMAT][MT];
#pragma unroll
            for (int mat = 0; mat < NMAT; ++mat)
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    float s = 0.0f;
                    for (long long u = ua; u < ub; ++u)
                        s += slots[(sk_item_index<CH>(static_cast<int>(u - u0), mat) * MT + m) * 32 + lane];
                    tot[mat][m] = s;
                }
            if (rb == rb_hi && combine) {
                // this CTA holds the start: add the partial the next CTA
                // published (bounded wait), then clear it for the next call
#pragma unroll
                for (int mat = 0; mat < NMAT; ++mat)
#pragma unroll
                    for (int m = 0; m < MT; ++m) {
                        unsigned long long *t = p.ws_tag + tag_index<NMAT, MT>(rb, mat, m, lane);
                        const unsigned long long w =
                            (early[mat][m] >> 32) != 0 ? early[mat][m] : wait_tagged_word(t);
                        tot[mat][m] = tot[mat][m] + __uint_as_float(static_cast<uint32_t>(w));
                        st_relaxed_gpu_u64(t, 0ull);
                    }
            }
            const int n = rb * 32 + lane;
            if (n >= p.N) continue;
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                if (m >= p.M) continue;
                const int64_t o = static_cast<int64_t>(m) * p.ldo + n;
                float val;
                if (MODE == kModeGemv) {
                    val = sx[m] * tot[0][m];
                    if (p.residual) val += (i == 0) ? res0[m] : p.residual[o];
                } else {
                    const float g = sx[m] * tot[0][m];
                    const float up = sx[m] * tot[NMAT - 1][m];
                    val = g * (1.0f / (1.0f + expf(-g))) * up;
                }
                p.out[o] = val;
            }
        }
        if (!ok2) mbar_wait_cluster_bounded(qbar2, 0);  // let late copies land before exit
    }
    // No CTA leaves while a peer of its cluster may still copy into it.
    cluster_wait();
}

// Cluster size for the input quantisation: the largest of {4, 2} whose
// clusters keep at least 97% of the SMs busy with one CTA each, else 1.
// Returns the size and (in *ncta) the CTAs that are resident at once.
template <typename Kern>
int choose_cluster(Kern kern, int num_sms, int *ncta) {
    for (int C : {4, 2}) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((num_sms / C) * C, 1, 1);
        cfg.blockDim = dim3(kSkThreads, 1, 1);
        cfg.dynamicSmemBytes = 200 * 1024;  // one CTA per SM
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = C;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int nclusters = 0;
        if (cudaOccupancyMaxActiveClusters(&nclusters, kern, &cfg) != cudaSuccess) {
            (void)cudaGetLastError();
            continue;
        }
        const int n = nclusters * C;
        if (n * 100 >= num_sms * 97) {
            *ncta = n < num_sms ? n : num_sms;
            return C;
        }
    }
    *ncta = num_sms;
    return 1;
}

template <int FMT, int MT, int MODE, bool DBG>
cudaError_t launch_sk(const StreamLaunch &S, cudaStream_t s, const char **why) {
    constexpr int NMAT = (MODE == kModeSwiglu) ? 2 : 1;
    // per device: cluster size and resident CTAs, set once (thread-safe)
    static DeviceOnce once;
    static int plan_c[DeviceOnce::kMaxDevices] = {0}, plan_n[DeviceOnce::kMaxDevices] = {0};
    SkParams p = {};
    p.N = S.N;
    p.K = S.K;
    p.SB = static_cast<int>(ceil_div(S.row_bytes, kSBBytes));
    p.SBF = static_cast<int>(S.row_bytes / kSBBytes);
    p.RB = static_cast<int>(ceil_div(S.N, 32));
    p.U = static_cast<long long>(p.RB) * p.SB;
    p.M = S.M;
    p.prefetch_ok = S.prefetch_ok;
    p.qflags = S.qflags;
    p.tsc0 = S.scales_tiled[0];
    p.tsc1 = S.scales_tiled[1];
    p.x = S.x;
    p.ldx = S.ldx;
    p.residual = S.residual;
    p.out = S.out;
    p.ldo = S.ldo;
    p.ws_tag = static_cast<unsigned long long *>(S.workspace);
    p.dbg_q = S.dbg_q;
    p.dbg_ldq = S.dbg_ldq;
    p.dbg_sx = S.dbg_sx;
    p.dbg_P = S.dbg_P;
    p.G = static_cast<int>(ceil_div(S.K, 128));

    int dev = 0;
    cudaError_t e = current_device(&dev);
    if (e != cudaSuccess) return e;
    auto kern = gemv_stream_kernel<FMT, MT, MODE, DBG>;
    e = once.run(dev, [&]() {
        cudaError_t r = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
        if (r != cudaSuccess) return r;
        // Every launch of the library takes the largest shared-memory split
        // of the SM, so that consecutive launches never need the SM to be
        // reconfigured (a split that differs from the previous launch's
        // waits until the SM has drained).
        r = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 cudaSharedmemCarveoutMaxShared);
        if (r != cudaSuccess) return r;
        plan_c[dev] = choose_cluster(kern, S.num_sms, &plan_n[dev]);
        return cudaSuccess;
    });
    if (e != cudaSuccess) return e;
    // The smallest cluster whose CTAs hold their share of the input blocks in
    // registers (no reloads); a single CTA needs no exchange at all.
    const int GT = p.SB * Fmt<FMT>::kGroups;
    int C = 1;
    while (C < plan_c[dev] && ceil_div(ceil_div(GT, C), kSkConsumers) > kSkKeep) C *= 2;
    // every range holds >= SB units, so a row block meets at most 2 ranges
    long long want = p.U / p.SB;
    if (want > (C > 1 ? plan_n[dev] : S.num_sms)) want = C > 1 ? plan_n[dev] : S.num_sms;
    if (want < 1) want = 1;
    while (C > 1 && want < C) C /= 2;
    p.nCTA = static_cast<int>((want / C) * C);
    const int items_max = sk_items_max<NMAT>(p.U, p.nCTA);
    // ring depth: as many whole chunks as fit the shared-memory budget of
    // one CTA per SM
    int R = kSkMaxRing;
    while (R > kSkMinRing && sk_layout<FMT, MT>(p.SB, items_max, R).total > kSkSmemBudget)
        R -= kSkChunk;
    p.R = R;
    const SkLayout L = sk_layout<FMT, MT>(p.SB, items_max, R);
    if (L.total > 227 * 1024) {
        *why = "shared memory plan of the streamed kernel exceeds 227 KB";
        return cudaErrorInvalidValue;
    }
    CUtensorMap tm0, tm1, tm3_0, tm3_1;
    constexpr int CH = kSkChunk / NMAT;
    if (!make_weight_tmap(&tm0, S.packed[0], S.row_bytes, S.N, S.row_stride) ||
        !make_weight_tmap(&tm1, S.packed[NMAT - 1], S.row_bytes, S.N, S.row_stride)) {
        *why = "cuTensorMapEncodeTiled failed or is unavailable";
        return cudaErrorInvalidValue;
    }
    if (p.SBF >= 1) {
        if (!make_weight_tmap3d(&tm3_0, S.packed[0], S.N, S.row_stride, p.SBF, CH) ||
            !make_weight_tmap3d(&tm3_1, S.packed[NMAT - 1], S.N, S.row_stride, p.SBF, CH)) {
            *why = "cuTensorMapEncodeTiled (3-D) failed";
            return cudaErrorInvalidValue;
        }
    } else {
        tm3_0 = tm0;  // never used: no whole superblock, every chunk takes 2-D boxes
        tm3_1 = tm1;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.nCTA, 1, 1);
    cfg.blockDim = dim3(kSkThreads, 1, 1);
    cfg.dynamicSmemBytes = L.total;
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
    e = cudaLaunchKernelEx(&cfg, kern, tm0, tm1, tm3_0, tm3_1, p);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

template <int FMT, int MODE, bool DBG>
cudaError_t launch_sk_mt(const StreamLaunch &S, cudaStream_t s, const char **why) {
    if (S.M <= 1) return launch_sk<FMT, 1, MODE, DBG>(S, s, why);
    return launch_sk<FMT, 2, MODE, DBG>(S, s, why);
}

template <bool DBG>
cudaError_t launch_sk_any(const StreamLaunch &S, cudaStream_t s, const char **why) {
    if (S.fmt == TERN_FMT_BASE3)
        return S.swiglu ? launch_sk_mt<TERN_FMT_BASE3, kModeSwiglu, DBG>(S, s, why)
                        : launch_sk_mt<TERN_FMT_BASE3, kModeGemv, DBG>(S, s, why);
    if (S.fmt == TERN_FMT_BITPLANE)
        return S.swiglu ? launch_sk_mt<TERN_FMT_BITPLANE, kModeSwiglu, DBG>(S, s, why)
                        : launch_sk_mt<TERN_FMT_BITPLANE, kModeGemv, DBG>(S, s, why);
    return S.swiglu ? launch_sk_mt<TERN_FMT_2BIT, kModeSwiglu, DBG>(S, s, why)
                    : launch_sk_mt<TERN_FMT_2BIT, kModeGemv, DBG>(S, s, why);
}

}  // namespace
}  // namespace tern

// tern_gemv_stream.cu -- streamed (persistent, evenly split) ternary GEMV for
// batch-1 / 2-token decode.
//
// The method is that of tern_gemv.cu (Bonsai page, "Decode 为什么只能算一般":
// stream the packed codes once, restore -1/0/+1 in registers, integer dot,
// FP16 group scale -- 4sapi page, section 三); this file changes how the
// work is laid over the GPU so that one projection costs about its bytes:
//
//  * A "unit" is 32 rows x one 128-byte superblock of codes.  The U units of
//    a matrix (row-block major) are cut into equal contiguous ranges, one per
//    CTA, one CTA per SM -- so every SM streams the same number of bytes.
//  * Warp 0 of a CTA is a producer: from the first instruction (before the
//    previous kernel on the stream has finished, when the matrix is static)
//    it streams its units into a ring of shared-memory slots: the 32 x 128 B
//    code tile by TMA (128-byte swizzle, L2 evict-first, no multicast) and
//    the unit's 32 x GPS scales, re-tiled at load time into unit order, by a
//    bulk copy.  A CTA of the next kernel, resident beside this one under
//    programmatic dependent launch, fills its own ring meanwhile.
//  * Warps 1..8 are consumers.  After the previous kernel finishes they
//    quantise the fp32 input once per CTA (two passes: row scale from max|x|
//    -- or max|H x| with the Hadamard rotation -- then the int8 codes and
//    per-group sums), then take units round-robin: lane = row, decode +
//    dp4a as in tern_gemv.cu, one fp32 partial per (unit, row).
//  * Row blocks inside a CTA's range are summed in unit order and written.
//    A row block cut by a range boundary belongs to two CTAs: each writes
//    its partial to the workspace (from its start) and increments the row
//    block's counter (counters sit at the end of the workspace, so calls of
//    any size that share it agree on where each counter is);
//    the second one adds lower + upper (fixed order, so the result does not
//    depend on which finishes first), writes the output and resets the
//    counter, so the workspace is zero again for the next call.
#include "tern_gemv_common.cuh"

namespace tern {
namespace {

constexpr int kSkConsumers = 8;
constexpr int kSkThreads = 32 * (kSkConsumers + 1);
constexpr int kSkBar = 1;  // named barrier of the consumer warps

template <int FMT>
__host__ __device__ constexpr int scb() {
    return 32 * Fmt<FMT>::kGroups * 2;  // bytes of one unit's scales
}
template <int NMAT>
__host__ __device__ constexpr int sk_ring() {
    return NMAT == 1 ? 16 : 8;
}

struct SkParams {
    int N, K, G, SB, RB;
    long long U;
    int nCTA, M, prefetch_ok, qflags;
    const uint16_t *tsc0;
    const uint16_t *tsc1;
    const float *x;
    int ldx;
    const float *residual;
    float *out;
    int ldo;
    float *ws_part;
    int *ws_cnt_end;  // counter of row block rb is ws_cnt_end[-1 - rb]
};

struct SkLayout {
    int ring_s_off, act_off, sq_off, sx_off, red_off, slots_off, bar_off, total;
    int Kpad, GT, umax;
};

template <int FMT, int MT, int NMAT>
__host__ __device__ inline SkLayout sk_layout(int SB, int umax) {
    constexpr int R = sk_ring<NMAT>();
    SkLayout L;
    L.Kpad = SB * Fmt<FMT>::kPos;
    L.GT = SB * Fmt<FMT>::kGroups;
    L.umax = umax;
    int off = R * NMAT * kTile;  // code tiles, 1024-aligned slots (128-byte swizzle)
    L.ring_s_off = off;
    off = align128(off + R * NMAT * scb<FMT>());
    L.act_off = off;
    off = align128(off + MT * L.Kpad);
    L.sq_off = off;
    off = align128(off + MT * L.GT * 4);
    L.sx_off = off;
    off = align128(off + 2 * MT * 4);
    L.red_off = off;
    off = align128(off + kSkConsumers * MT * 2 * 4);
    L.slots_off = off;
    off = align128(off + umax * NMAT * MT * 32 * 4);
    L.bar_off = off;
    off += 2 * R * 8;
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

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ float unit_scale(const uint8_t *s, int lane, int gps, int g) {
    return __half2float(
        __ushort_as_half(reinterpret_cast<const uint16_t *>(s)[lane * gps + g]));
}

// One unit (this lane's row, one superblock) of NMAT matrices: the decode and
// dp4a of tern_gemv.cu with the unit's scales from its ring slot.
template <int FMT, int MT, int NMAT>
__device__ __forceinline__ void sk_unit(const uint8_t *wtile, const uint8_t *stile, int lane,
                                        const uint8_t *act_sb, int Kpad, const int *sq_sb, int GT,
                                        float (&yacc)[NMAT][MT]) {
    constexpr int GPS = Fmt<FMT>::kGroups;
    constexpr int SCB = scb<FMT>();
    const int rsw = lane & 7;
    int acc[NMAT][MT];
#pragma unroll
    for (int mat = 0; mat < NMAT; ++mat)
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            acc[mat][m] = 0;
            yacc[mat][m] = 0.0f;
        }
    auto finish = [&](int m, int g) {
        const int s = sq_sb[m * GT + g];
#pragma unroll
        for (int mat = 0; mat < NMAT; ++mat) {
            yacc[mat][m] = fmaf(unit_scale(stile + mat * SCB, lane, GPS, g),
                                static_cast<float>(acc[mat][m] - s), yacc[mat][m]);
            acc[mat][m] = 0;
        }
    };
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        uint32_t words[NMAT][4];
#pragma unroll
        for (int mat = 0; mat < NMAT; ++mat) {
            const uint4 wv = lds128(wtile + mat * kTile + lane * kSBBytes + ((c ^ rsw) << 4));
            words[mat][0] = wv.x;
            words[mat][1] = wv.y;
            words[mat][2] = wv.z;
            words[mat][3] = wv.w;
        }
        if constexpr (FMT == TERN_FMT_BASE3) {
            uint32_t t[NMAT][20];
#pragma unroll
            for (int mat = 0; mat < NMAT; ++mat)
#pragma unroll
                for (int wi = 0; wi < 4; ++wi) {
                    uint32_t tw[5];
                    decode_d3(words[mat][wi], tw);
#pragma unroll
                    for (int i = 0; i < 5; ++i) t[mat][5 * wi + i] = tw[i];
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
#pragma unroll
                    for (int mat = 0; mat < NMAT; ++mat) acc[mat][m] = dp4a_ss(t[mat][d], aw[d], acc[mat][m]);
                }
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
#pragma unroll
                for (int mat = 0; mat < NMAT; ++mat) {
                    int a4[4] = {0, 0, 0, 0};
#pragma unroll
                    for (int wi = 0; wi < 4; ++wi)
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            a4[i] = dp4a_us(words[mat][wi] & (0x03030303u << (2 * i)), aw[4 * wi + i], a4[i]);
                    acc[mat][m] += a4[0] + (a4[1] >> 2) + (a4[2] >> 4) + (a4[3] >> 6);
                }
                if (c & 1) finish(m, c >> 1);
            }
        }
    }
    if constexpr (FMT == TERN_FMT_BASE3) {
#pragma unroll
        for (int m = 0; m < MT; ++m) finish(m, 4);
    }
}

template <int FMT, int MT, int MODE>
__global__ void __launch_bounds__(kSkThreads, 1)
    gemv_stream_kernel(const __grid_constant__ CUtensorMap tm0,
                       const __grid_constant__ CUtensorMap tm1, const SkParams p) {
    constexpr int NMAT = (MODE == kModeSwiglu) ? 2 : 1;
    constexpr int POS = Fmt<FMT>::kPos;
    constexpr int GPS = Fmt<FMT>::kGroups;
    constexpr int SCB = scb<FMT>();
    constexpr int R = sk_ring<NMAT>();
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);

    const long long U = p.U;
    const int c = blockIdx.x;
    const long long u0 = U * c / p.nCTA, u1 = U * (c + 1) / p.nCTA;
    const int nu = static_cast<int>(u1 - u0);
    const int umax = static_cast<int>((U + p.nCTA - 1) / p.nCTA);
    const SkLayout L = sk_layout<FMT, MT, NMAT>(p.SB, umax);
    uint8_t *ring_w = smem;
    uint8_t *ring_s = smem + L.ring_s_off;
    uint8_t *act = smem + L.act_off;
    int *sq = reinterpret_cast<int *>(smem + L.sq_off);
    float *sx = reinterpret_cast<float *>(smem + L.sx_off);
    float *red = reinterpret_cast<float *>(smem + L.red_off);
    float *slots = reinterpret_cast<float *>(smem + L.slots_off);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + L.bar_off);
    uint64_t *empty = full + R;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid == 0) {
        prefetch_tmap(&tm0);
        if (NMAT == 2) prefetch_tmap(&tm1);
        for (int i = 0; i < R; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        fence_mbar_init();
    }
    __syncthreads();
    pdl_launch_dependents();

    if (warp == 0) {
        // ---------------------------------------------------------- producer
        if (!p.prefetch_ok) pdl_wait();
        if (lane == 0) {
            const uint64_t policy = l2_policy_evict_first();
            for (int j = 0; j < nu; ++j) {
                const int slot = j % R, round = j / R;
                if (round > 0 && !mbar_wait_bounded(&empty[slot], (round - 1) & 1)) break;
                const long long u = u0 + j;
                const int rb = static_cast<int>(u / p.SB), sb = static_cast<int>(u % p.SB);
                mbar_arrive_expect_tx(&full[slot], NMAT * (kTile + SCB));
#pragma unroll
                for (int mat = 0; mat < NMAT; ++mat) {
                    tma_load_2d(ring_w + (slot * NMAT + mat) * kTile, mat ? &tm1 : &tm0,
                                sb * kSBBytes, rb * 32, &full[slot], policy);
                    const uint16_t *tsc = mat ? p.tsc1 : p.tsc0;
                    bulk_copy_g2s(ring_s + (slot * NMAT + mat) * SCB,
                                  reinterpret_cast<const uint8_t *>(tsc) + u * SCB, SCB, &full[slot],
                                  policy);
                }
            }
        }
    } else {
        // ---------------------------------------------------------- consumers
        const int cw = warp - 1, ctid = tid - 32;
        pdl_wait();
        const bool rotate = (p.qflags & TERN_QUANT_FWHT128) != 0;
        const bool rms = (p.qflags & TERN_QUANT_RMSNORM) != 0;
        const int nb = (p.K + 127) / 128;    // blocks holding input
        const int nbpad = L.Kpad / 128;      // blocks of the padded activation
        // pass 1: max |x| (or |H x|) and sum x^2 per token row
        for (int m = 0; m < MT; ++m) {
            float amax = 0.0f, ss = 0.0f;
            if (m < p.M) {
                for (int b = cw; b < nb; b += kSkConsumers) {
                    const int k = 128 * b + 4 * lane;
                    float r[4] = {0.0f, 0.0f, 0.0f, 0.0f};
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
                    ss += fmaf(r[3], r[3], fmaf(r[2], r[2], fmaf(r[1], r[1], r[0] * r[0])));
                    if (rotate) fwht128_warp(r, lane);
                    amax = fmaxf(amax, fmaxf(fmaxf(fabsf(r[0]), fabsf(r[1])), fmaxf(fabsf(r[2]), fabsf(r[3]))));
                }
            }
            amax = warp_max(amax);
            ss = warp_sum(ss);
            if (lane == 0) {
                red[(cw * MT + m) * 2 + 0] = amax;
                red[(cw * MT + m) * 2 + 1] = ss;
            }
        }
        warpgroup_sync_n(kSkBar, kSkConsumers * 32);
        if (ctid < MT) {
            const int m = ctid;
            float amax = 0.0f, ss = 0.0f;
            for (int w = 0; w < kSkConsumers; ++w) {
                amax = fmaxf(amax, red[(w * MT + m) * 2 + 0]);
                ss += red[(w * MT + m) * 2 + 1];
            }
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
        warpgroup_sync_n(kSkBar, kSkConsumers * 32);
        // pass 2: int8 codes of every block and the per-group sums
        for (int job = cw; job < MT * nbpad; job += kSkConsumers) {
            const int m = job / nbpad, b = job % nbpad;
            const int k = 128 * b + 4 * lane;
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
            *reinterpret_cast<uint32_t *>(act + m * L.Kpad + k) = packed;
            qsum = warp_sum_int(qsum);
            if (lane == 0) sq[m * L.GT + b] = qsum;
        }
        warpgroup_sync_n(kSkBar, kSkConsumers * 32);

        // units, round-robin over the consumer warps
        for (int j = cw; j < nu; j += kSkConsumers) {
            const int slot = j % R;
            const bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(&full[slot], (j / R) & 1));
            float yacc[NMAT][MT];
            if (ok) {
                const long long u = u0 + j;
                const int sb = static_cast<int>(u % p.SB);
                sk_unit<FMT, MT, NMAT>(ring_w + slot * NMAT * kTile, ring_s + slot * NMAT * SCB, lane,
                                       act + sb * POS, L.Kpad, sq + sb * GPS, L.GT, yacc);
            } else {
#pragma unroll
                for (int mat = 0; mat < NMAT; ++mat)
#pragma unroll
                    for (int m = 0; m < MT; ++m) yacc[mat][m] = 0.0f;
            }
#pragma unroll
            for (int mat = 0; mat < NMAT; ++mat)
#pragma unroll
                for (int m = 0; m < MT; ++m) slots[((j * NMAT + mat) * MT + m) * 32 + lane] = yacc[mat][m];
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[slot]);
        }
        warpgroup_sync_n(kSkBar, kSkConsumers * 32);

        // row blocks of this range: sum units in order; finish or combine
        const int rb_lo = static_cast<int>(u0 / p.SB);
        const int rb_hi = static_cast<int>((u1 - 1) / p.SB);
        for (int rb = rb_lo + cw; rb <= rb_hi; rb += kSkConsumers) {
            const long long ua = max(u0, static_cast<long long>(rb) * p.SB);
            const long long ub = min(u1, static_cast<long long>(rb + 1) * p.SB);
            float tot[NMAT][MT];
#pragma unroll
            for (int mat = 0; mat < NMAT; ++mat)
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    float s = 0.0f;
                    for (long long u = ua; u < ub; ++u)
                        s += slots[(((u - u0) * NMAT + mat) * MT + m) * 32 + lane];
                    tot[mat][m] = s;
                }
            const bool lower_cut = static_cast<long long>(rb) * p.SB < u0;
            const bool upper_cut = static_cast<long long>(rb + 1) * p.SB > u1;
            bool finish_here = true;
            if (lower_cut || upper_cut) {
                const int side = lower_cut ? 1 : 0;  // 0: this CTA holds the row block's start
#pragma unroll
                for (int mat = 0; mat < NMAT; ++mat)
#pragma unroll
                    for (int m = 0; m < MT; ++m)
                        p.ws_part[((((static_cast<int64_t>(rb) * 2 + side) * NMAT + mat) * MT + m) * 32) +
                                  lane] = tot[mat][m];
                __threadfence();
                __syncwarp();
                int old = 0;
                if (lane == 0) old = atomicAdd(&p.ws_cnt_end[-1 - rb], 1);
                old = __shfl_sync(0xffffffffu, old, 0);
                finish_here = (old == 1);
                if (finish_here) {
                    __threadfence();
#pragma unroll
                    for (int mat = 0; mat < NMAT; ++mat)
#pragma unroll
                        for (int m = 0; m < MT; ++m) {
                            const int64_t base = (((static_cast<int64_t>(rb) * 2) * NMAT + mat) * MT + m) * 32 + lane;
                            const float lo = __ldcg(p.ws_part + base);
                            const float hi = __ldcg(p.ws_part + base + static_cast<int64_t>(NMAT) * MT * 32);
                            tot[mat][m] = lo + hi;
                        }
                    if (lane == 0) p.ws_cnt_end[-1 - rb] = 0;
                }
            }
            if (!finish_here) continue;
            const int n = rb * 32 + lane;
            if (n >= p.N) continue;
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                if (m >= p.M) continue;
                const int64_t o = static_cast<int64_t>(m) * p.ldo + n;
                float v;
                if (MODE == kModeGemv) {
                    v = sx[m] * tot[0][m];
                    if (p.residual) v += p.residual[o];
                } else {
                    const float g = sx[m] * tot[0][m];
                    const float u = sx[m] * tot[NMAT - 1][m];
                    v = g * (1.0f / (1.0f + expf(-g))) * u;
                }
                p.out[o] = v;
            }
        }
    }
    __syncthreads();
}

constexpr int kMaxDevices = 64;

template <int FMT, int MT, int MODE>
cudaError_t launch_sk(const StreamLaunch &S, cudaStream_t s, const char **why) {
    constexpr int NMAT = (MODE == kModeSwiglu) ? 2 : 1;
    static int smem_set[kMaxDevices] = {0};
    SkParams p = {};
    p.N = S.N;
    p.K = S.K;
    p.G = static_cast<int>(ceil_div(S.K, 128));
    p.SB = static_cast<int>(ceil_div(S.row_bytes, kSBBytes));
    p.RB = static_cast<int>(ceil_div(S.N, 32));
    p.U = static_cast<long long>(p.RB) * p.SB;
    long long ncta = p.U / p.SB;  // every range holds >= SB units: a row block meets <= 2 ranges
    if (ncta > S.num_sms) ncta = S.num_sms;
    if (ncta < 1) ncta = 1;
    p.nCTA = static_cast<int>(ncta);
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
    // Partial sums from the start of the workspace, counters from its end:
    // every call finds counter rb at the same place, whatever its own size.
    p.ws_part = static_cast<float *>(S.workspace);
    p.ws_cnt_end = reinterpret_cast<int *>(static_cast<char *>(S.workspace) + (S.ws_bytes & ~size_t(3)));
    const int umax = static_cast<int>((p.U + p.nCTA - 1) / p.nCTA);
    const SkLayout L = sk_layout<FMT, MT, NMAT>(p.SB, umax);
    if (L.total > 227 * 1024) {
        *why = "shared memory plan of the streamed kernel exceeds 227 KB";
        return cudaErrorInvalidValue;
    }
    CUtensorMap tm0, tm1;
    if (!make_weight_tmap(&tm0, S.packed[0], S.row_bytes, S.N, S.row_stride) ||
        !make_weight_tmap(&tm1, S.packed[NMAT - 1], S.row_bytes, S.N, S.row_stride)) {
        *why = "cuTensorMapEncodeTiled failed or is unavailable";
        return cudaErrorInvalidValue;
    }
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < kMaxDevices && !smem_set[dev]) {
        e = cudaFuncSetAttribute(gemv_stream_kernel<FMT, MT, MODE>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
        if (e != cudaSuccess) return e;
        smem_set[dev] = 1;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.nCTA, 1, 1);
    cfg.blockDim = dim3(kSkThreads, 1, 1);
    cfg.dynamicSmemBytes = L.total;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, gemv_stream_kernel<FMT, MT, MODE>, tm0, tm1, p);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

template <int FMT, int MODE>
cudaError_t launch_sk_mt(const StreamLaunch &S, cudaStream_t s, const char **why) {
    if (S.M <= 1) return launch_sk<FMT, 1, MODE>(S, s, why);
    return launch_sk<FMT, 2, MODE>(S, s, why);
}

}  // namespace

size_t stream_workspace_bytes(int fmt, int N, int M, int nmat) {
    (void)fmt;
    const int MT = M <= 1 ? 1 : 2;
    const size_t RB = static_cast<size_t>(ceil_div(N, 32));
    return RB * 2 * nmat * MT * 32 * sizeof(float) + RB * sizeof(int);
}

cudaError_t launch_gemv_stream(const StreamLaunch &S, cudaStream_t s, const char **why) {
    if (S.fmt == TERN_FMT_BASE3)
        return S.swiglu ? launch_sk_mt<TERN_FMT_BASE3, kModeSwiglu>(S, s, why)
                        : launch_sk_mt<TERN_FMT_BASE3, kModeGemv>(S, s, why);
    return S.swiglu ? launch_sk_mt<TERN_FMT_2BIT, kModeSwiglu>(S, s, why)
                    : launch_sk_mt<TERN_FMT_2BIT, kModeGemv>(S, s, why);
}

}  // namespace tern

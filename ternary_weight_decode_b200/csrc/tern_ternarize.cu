// tern_ternarize.cu -- producer-side ternarisation of float weights: per
// group of 128 consecutive K positions of a row, two thresholds -D / +D
// (values between them become 0, the sides -1 / +1) and one FP16 scale,
// chosen to make the residual of the weights small (pwwt.cn/news/5175886,
// section 1.2: per-block thresholds and a scale that minimises the
// residual; m.nxbn.cn/news/172464, section 1.2: threshold plus one scale
// per group).  No calibration data: the residual is sum (w - alpha t)^2.
//
// For thresholds at a magnitude, the best scale is the mean of the kept
// |w|, and the residual is sum w^2 - S^2 / k (k kept values, S their sum),
// so the best cut keeps the k largest |w| maximising S^2 / k.  A warp owns
// one (row, group); lane l holds the four values at 4l .. 4l+3 and
// evaluates the four cuts "keep everything ranked at or above value j"
// (rank: larger |w| first, lower index first among equals).  Its sum S(j)
// adds the kept |w| in index order in fp32, exactly as the definition
// states it, so the integer decisions (which cut, which trits) are the same
// on every implementation that follows that order.  The warp then takes the
// largest S^2 / k (smallest k among equals; k = 0 when nothing scores above
// 0), writes t = sign(w) on the kept entries and alpha = fp16(S / k).
#include "tern_common.cuh"
#include "tern_internal.h"

namespace tern {
namespace {

constexpr int kTzWarps = 8;

__global__ void __launch_bounds__(kTzWarps * 32)
    ternarize_kernel(const float *__restrict__ w, int N, int K, int ldw, int G,
                     int8_t *__restrict__ trits, uint16_t *__restrict__ scales) {
    __shared__ float mag[kTzWarps][128];
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const long long job = static_cast<long long>(blockIdx.x) * kTzWarps + wid;
    if (job >= static_cast<long long>(N) * G) return;
    const int n = static_cast<int>(job / G), g = static_cast<int>(job % G);
    const int k0 = 128 * g;
    const int len = min(128, K - k0);
    const float *row = w + static_cast<int64_t>(n) * ldw + k0;

    float v[4], a[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const int i = 4 * lane + e;
        v[e] = i < len ? row[i] : 0.0f;
        a[e] = fabsf(v[e]);
        mag[wid][i] = a[e];
    }
    __syncwarp();

    // the four cuts of this lane: S(j) and k(j), index-order fp32 sums
    float sum[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    int cnt[4] = {0, 0, 0, 0};
    for (int i = 0; i < len; ++i) {
        const float ai = mag[wid][i];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int j = 4 * lane + e;
            const bool keep = ai > a[e] || (ai == a[e] && i <= j);
            if (keep) {
                sum[e] = __fadd_rn(sum[e], ai);
                ++cnt[e];
            }
        }
    }
    // best cut of the lane, then of the warp: largest score, smallest k
    float best_score = 0.0f, best_sum = 0.0f;
    int best_cnt = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        if (4 * lane + e >= len) continue;
        const float score = __fdiv_rn(__fmul_rn(sum[e], sum[e]), static_cast<float>(cnt[e]));
        if (score > best_score || (score == best_score && cnt[e] < best_cnt)) {
            best_score = score;
            best_cnt = cnt[e];
            best_sum = sum[e];
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float s2 = __shfl_xor_sync(0xffffffffu, best_score, o);
        const int c2 = __shfl_xor_sync(0xffffffffu, best_cnt, o);
        const float u2 = __shfl_xor_sync(0xffffffffu, best_sum, o);
        if (s2 > best_score || (s2 == best_score && c2 < best_cnt)) {
            best_score = s2;
            best_cnt = c2;
            best_sum = u2;
        }
    }
    // kept entries: rank < best_cnt (rank counted against the whole group)
    int8_t *trow = trits + static_cast<int64_t>(n) * K + k0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const int i = 4 * lane + e;
        if (i >= len) continue;
        int rank = 0;
        for (int j = 0; j < len; ++j) {
            const float aj = mag[wid][j];
            rank += (aj > a[e] || (aj == a[e] && j < i)) ? 1 : 0;
        }
        const int s = v[e] > 0.0f ? 1 : (v[e] < 0.0f ? -1 : 0);
        trow[i] = static_cast<int8_t>(rank < best_cnt ? s : 0);
    }
    if (lane == 0) {
        const float alpha = best_cnt ? __fdiv_rn(best_sum, static_cast<float>(best_cnt)) : 0.0f;
        scales[static_cast<int64_t>(n) * G + g] = __half_as_ushort(__float2half_rn(alpha));
    }
}

}  // namespace

cudaError_t launch_ternarize(const float *w, int N, int K, int ldw, int8_t *trits, uint16_t *scales,
                             cudaStream_t s) {
    const int G = static_cast<int>(ceil_div(K, 128));
    const long long jobs = static_cast<long long>(N) * G;
    const long long blocks = (jobs + kTzWarps - 1) / kTzWarps;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
    ternarize_kernel<<<static_cast<unsigned>(blocks), kTzWarps * 32, 0, s>>>(w, N, K, ldw, G, trits,
                                                                              scales);
    return cudaGetLastError();
}

}  // namespace tern

// tern_internal.h -- declarations shared between the C-ABI layer and the
// kernel launchers of libtern (not installed; the public ABI is tern.h).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <mutex>

#include "../../include/tern.h"

namespace tern {

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// K split of the fused GEMV engines: nsplit, or the next count up to 8 (a
// portable cluster) that divides the SB superblocks evenly, so that the
// ranks of a cluster finish together (2-bit gate/up at K = 5120: 10
// superblocks as 5 x 2, not 3 + 3 + 3 + 1).  Both engines take the same
// split, hence the same sum order.
inline int even_split(int SB, int nsplit) {
    for (int n = nsplit; SB % nsplit != 0 && n <= 8 && n <= SB; ++n)
        if (SB % n == 0) nsplit = n;
    return nsplit;
}

// One-time set-up of a launch site on each device (kernel attributes, launch
// plans).  Safe when several host threads make their first call at once: the
// first caller on a device runs `setup` under a lock, later callers see its
// result through an acquire load without locking.  A set-up that fails is
// tried again on the next call.  Use as a function-local static.
class DeviceOnce {
  public:
    static constexpr int kMaxDevices = 64;
    template <typename F>
    cudaError_t run(int dev, F &&setup) {
        if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
        if (done_[dev].load(std::memory_order_acquire)) return cudaSuccess;
        std::lock_guard<std::mutex> lock(mu_);
        if (done_[dev].load(std::memory_order_relaxed)) return cudaSuccess;
        const cudaError_t e = setup();
        if (e == cudaSuccess) done_[dev].store(1, std::memory_order_release);
        return e;
    }

  private:
    std::mutex mu_;
    std::atomic<int> done_[kMaxDevices]{};
};

// The current device, checked against DeviceOnce's range.
inline cudaError_t current_device(int *dev) {
    cudaError_t e = cudaGetDevice(dev);
    if (e != cudaSuccess) return e;
    if (*dev < 0 || *dev >= DeviceOnce::kMaxDevices) return cudaErrorInvalidDevice;
    return cudaSuccess;
}

inline int64_t device_row_bytes(int fmt, int64_t K) {
    if (fmt == TERN_FMT_BASE3) return 4 * ((K + 19) / 20);
    if (fmt == TERN_FMT_2BIT) return 4 * ((K + 15) / 16);
    if (fmt == TERN_FMT_BITPLANE) return 8 * ((K + 31) / 32);
    return -1;
}

inline int64_t canonical_row_bytes(int fmt, int64_t K) {
    if (fmt == TERN_FMT_BASE3) return (K + 4) / 5;
    if (fmt == TERN_FMT_2BIT) return (K + 3) / 4;
    if (fmt == TERN_FMT_BITPLANE) return 2 * ((K + 7) / 8);
    return -1;
}

// ---------------------------------------------------------------- format
cudaError_t launch_pack(int fmt, const int8_t *trits, int N, int K, void *out, int64_t row_stride,
                        int32_t *d_invalid, cudaStream_t s);
cudaError_t launch_unpack(int fmt, const void *packed, int N, int K, int64_t row_stride,
                          int8_t *trits, int32_t *d_invalid, cudaStream_t s);
cudaError_t launch_import(int fmt, const uint8_t *canon, int N, int K, void *out,
                          int64_t row_stride, int32_t *d_invalid, cudaStream_t s);
cudaError_t launch_export(int fmt, const void *packed, int N, int K, int64_t row_stride,
                          uint8_t *canon, int32_t *d_invalid, cudaStream_t s);
cudaError_t launch_retile_scales(int fmt, const uint16_t *sc, int N, int K, uint16_t *out,
                                 cudaStream_t s);

inline int64_t tiled_scales_bytes(int fmt, int64_t N, int64_t K) {
    const int64_t SB = ceil_div(device_row_bytes(fmt, K), 128);
    const int64_t gps = (fmt == TERN_FMT_BASE3) ? 5 : 4;
    return ceil_div(N, 32) * SB * 32 * gps * 2;
}

// ---------------------------------------------------------------- ternarisation
cudaError_t launch_ternarize(const float *w, int N, int K, int ldw, int8_t *trits, uint16_t *scales,
                             cudaStream_t s);

// ---------------------------------------------------------------- attention
cudaError_t launch_kv_append(const float *k, const float *v, int pos, const tern_kv_cache &C,
                             cudaStream_t s);
int attention_chunk(int L, int Hkv, int GQ, int num_sms);
size_t attention_workspace_bytes(int Hq, int L, int Hkv, int num_sms);
cudaError_t launch_attention(const float *q, int Hq, const tern_kv_cache &C, int L, float *out,
                             float *part, int num_sms, cudaStream_t s, const char **why);

// ---------------------------------------------------------------- quant
cudaError_t launch_act_quant(const void *x, bool fp16, int M, int K, int ldx, int fwht_block,
                             int flags, int8_t *q, int ldq, float *s_x, cudaStream_t s);

// ---------------------------------------------------------------- gemv
enum GemvMode : int { kModeGemv = 0, kModeSwiglu = 1, kModePartials = 2 };

struct GemvLaunch {
    int mode;
    int fmt;
    int N, K, G;
    int64_t row_bytes;  // used bytes per row (the TMA box's x extent)
    int64_t row_stride;
    const void *packed[2];
    const uint16_t *scales[2];
    int prefetch_ok;  // both matrices carry TERN_MATRIX_STATIC
    const int8_t *q;
    int ldq;
    const float *s_x;
    int M;
    const float *residual;
    void *out;  // y, h (fp32) or partials (int32)
    int ldo;
    // fp32 input quantised inside the kernel (x != nullptr selects this form)
    const float *x;
    int ldx;
    const float *x_stats;
    int x_stats_ld;
    int qflags;
    // optional statistics of the output, per 128-row block
    float *y_stats;
    int y_stats_ld;
};

cudaError_t launch_gemv(const GemvLaunch &L, cudaStream_t s, const char **why);

// Streamed (persistent, evenly split) GEMV of tern_gemv_stream.cu.
struct StreamLaunch {
    int fmt, swiglu;
    int N, K;
    int64_t row_bytes, row_stride;
    const void *packed[2];
    const uint16_t *scales_tiled[2];
    int prefetch_ok;
    const float *x;
    int ldx, qflags, M;
    const float *residual;
    float *out;
    int ldo;
    void *workspace;
    size_t ws_bytes;
    int num_sms;
    // test hook only (launch_gemv_stream_debug): the int8 input codes [M][dbg_ldq]
    // and row scales [M] as CTA 0 holds them, and every exact int32 group
    // partial [NMAT][M][N][ceil(K/128)]
    int8_t *dbg_q;
    int dbg_ldq;
    float *dbg_sx;
    int32_t *dbg_P;
};
size_t stream_workspace_bytes(int fmt, int N, int M, int nmat);
cudaError_t launch_gemv_stream(const StreamLaunch &S, cudaStream_t s, const char **why);
// The same kernels instantiated with the test-hook outputs (S.dbg_*).
cudaError_t launch_gemv_stream_debug(const StreamLaunch &S, cudaStream_t s, const char **why);
// Host-side checks of a streamed call, everything but the workspace (W1 is
// the up matrix of the SwiGLU form, else NULL).  Sets tern_last_error().
tern_status check_streamed_call(const tern_matrix *W0, const tern_matrix *W1, const float *x,
                                int32_t ldx, int32_t qflags, int32_t M, const float *residual,
                                const float *out, int32_t ldo, const char *name);
cudaError_t launch_gemv_tc(const GemvLaunch &L, cudaStream_t s, const char **why);
void select_engine(int engine);  // 0: tensor cores, 1: CUDA cores (default)
cudaError_t launch_act_stats(const float *x, int M, int K, int ldx, float *stats, int ld,
                             cudaStream_t s);
cudaError_t read_clear_device_error(int *value, cudaStream_t s);
// Test hook: one bounded wait that nothing satisfies (kind 0: an mbarrier
// phase, kind 1: a tagged global word), with the given budget in SM cycles.
cudaError_t launch_debug_wait(int kind, long long budget_cycles, cudaStream_t s);

// 3-D view (byte in superblock, row, superblock) of a packed matrix's whole
// superblocks: one box = box_sb consecutive superblocks of 32 rows.
bool make_weight_tmap3d(CUtensorMap *map, const void *packed, int N, int64_t row_stride,
                        int sb_full, int box_sb);
// 2-D uint8 tensor map with 128-byte swizzle (tern_gemv.cu).
bool make_u8_tmap_2d(CUtensorMap *map, const void *base, uint64_t inner, uint64_t rows,
                     uint64_t stride, uint32_t box_inner, uint32_t box_rows);

// ---------------------------------------------------------------- prefill GEMM
struct GemmLaunch {
    int fmt;
    int N, K, M;
    int64_t row_bytes, row_stride;
    const void *packed;
    const uint16_t *scales;
    const int8_t *q;
    int ldq;
    const float *s_x;
    float *y;
    int ldy;
    int32_t *dbg_P;  // test hook only: exact int32 group partials [M][N][ceil(K/128)]
};
cudaError_t launch_gemm(const GemmLaunch &L, cudaStream_t s, const char **why);
// Token tile (64, 128 or 256 tokens) and cluster split of K of tern_gemm for
// an N x K matrix (SB superblocks) and M token rows.
void gemm_plan(int N, int M, int SB, int num_sms, int *TM, int *C);

// Sets the message tern_last_error() returns on the calling host thread.
tern_status set_last_error(tern_status s, const char *message);

// ---------------------------------------------------------------- tcgen05 test hook
cudaError_t launch_debug_mma(int a_in_smem, const int8_t *A, int a_signed, const int8_t *B,
                             int b_signed, int32_t *D, int K, int N, cudaStream_t s);

}  // namespace tern

/*
 * tern.h -- C ABI of libtern.so, the B200 (sm_100a) ternary-weight path.
 *
 * What the library computes (the pages this method is described on):
 *  - "Ternary Bonsai 2 27B: 8GB 显卡硬塞 27B 三元模型，能跑，但我大概率不会真用"
 *    (171host.com), section "Decode 为什么只能算一般": batch-1 decode reads the
 *    packed weights once per token; the kernel unpacks base-3 codes, restores
 *    -1/0/+1, reads the group scale and takes an integer dot product with the
 *    quantised activation, never writing dequantised weights back to memory;
 *    gate/up + SwiGLU run as one fused kernel sharing the Hadamard-rotated,
 *    quantised input; activations are re-quantised per token between matmuls.
 *  - "三值权重 27B 压到 5.9GB｜本地部署成本账单重算" (blog.4sapi.com), section 三:
 *    weights in {-1, 0, +1} with one FP16 scale per group; add/subtract by
 *    sign, then multiply by the group scale.
 *  - Same Bonsai page, section "后面还有没有优化空间": re-tile codes and scales
 *    at load time into the order the integer dot product consumes them.
 *
 * Conventions for every call:
 *  - Every pointer argument marked "device" is CUDA device memory owned by
 *    the caller.  The library allocates nothing, frees nothing and never
 *    synchronises the device; every call is asynchronous on `stream`
 *    (a cudaStream_t; NULL = legacy default stream) and may be captured in a
 *    CUDA graph.
 *  - Arguments are validated on the host before any launch; a violation
 *    returns TERN_EINVAL and launches nothing.  A failed launch returns
 *    TERN_ECUDA; tern_last_error() then holds the CUDA message.  No call
 *    aborts, throws or exits.  There is no CPU fallback.
 *  - Compute kernels are launched with programmatic dependent launch: they
 *    may begin before the previous kernel on the stream has finished, but
 *    read activations and write outputs only after it has.
 */
#ifndef TERN_H
#define TERN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    TERN_OK = 0,
    TERN_EINVAL = 1,       /* bad argument (shape, alignment, pointer, format) */
    TERN_ECUDA = 2,        /* a CUDA launch or query failed */
    TERN_EUNSUPPORTED = 3, /* valid request this build does not implement */
    TERN_ETIMEOUT = 4      /* a bounded device-side wait ran out */
} tern_status;

/* Weight formats.  Each holds one trit per weight, t = w + 1 in {0, 1, 2}. */
typedef enum {
    TERN_FMT_BASE3 = 0,   /* 5 trits per byte (PTQ1_0-style), 1.6 bit/trit */
    TERN_FMT_2BIT = 1,    /* 4 trits per byte (PQ2-style), 2 bit/trit */
    TERN_FMT_BITPLANE = 2 /* a nonzero bit and a sign bit per weight, 2 bit/trit (Bonsai
                             page, "后面还有没有优化空间"); every call takes it except
                             the tensor-core GEMV engine of tern_debug_select_engine,
                             which returns TERN_EUNSUPPORTED for it */
} tern_format;

/* Bit 0 of tern_matrix.flags: the packed codes and scales are not written by
 * any work still pending on the stream, so a compute kernel may start
 * streaming them before the previous kernel on the stream has finished. */
#define TERN_MATRIX_STATIC 1

/* act_quant_fwht flag: fold a weightless RMSNorm of the (unrotated) row into
 * the scale, s_x *= fp32(1/sqrt(mean_k x_k^2 + 1e-6)); q is unchanged. */
#define TERN_QUANT_RMSNORM 1

/* Fused-quantisation flag (tern_gemv_fused, tern_gateup_swiglu_fused): rotate
 * the input by the 128-point Hadamard transform before quantising it, exactly
 * as act_quant_fwht with fwht_block = 128. */
#define TERN_QUANT_FWHT128 2

/*
 * A packed weight matrix W [N][K] in the device layout written by tern_pack
 * or tern_import:
 *   TERN_FMT_BASE3 (D3): 4-byte word w of a row covers K in [20w, 20w+20);
 *     byte j of the word holds the trits at K = 20w + j + 4i, i = 0..4, as
 *     y = ceil(256 V / 243) with V = sum_i t_i 3^(4-i).  Row bytes used:
 *     4*ceil(K/20).
 *   TERN_FMT_2BIT (D2): 4-byte word w covers K in [16w, 16w+16); bits
 *     [2i, 2i+1] of byte j hold t for K = 16w + 4i + j.  Row bytes used:
 *     4*ceil(K/16).
 *   TERN_FMT_BITPLANE (DB): 4-byte words in pairs; pair p covers K in
 *     [32p, 32p+32): word 2p holds the nonzero bits (w != 0), word 2p+1 the
 *     sign bits (w < 0), bit 8j + i of each for K = 32p + 4i + j.  Row bytes
 *     used: 8*ceil(K/32).
 *   Positions past K hold w = 0; bytes past the used row bytes are 0.
 * scales: fp16 bit patterns [N][ceil(K/group)], one per group of `group`
 * consecutive K positions of a row (the last group may be partial).
 */
typedef struct tern_matrix {
    int32_t fmt;           /* tern_format */
    int32_t N;             /* output rows, >= 1 */
    int32_t K;             /* input length, >= 1 */
    int32_t group;         /* scale group along K; this build supports 128 */
    int64_t row_stride;    /* bytes between rows of `packed`: a multiple of 16,
                              >= the used row bytes */
    const void *packed;    /* device, 16-byte aligned, N * row_stride bytes */
    const uint16_t *scales;/* device, 2-byte aligned, N * ceil(K/group) fp16 */
    const uint16_t *scales_tiled; /* optional, device, 16-byte aligned: the same
                              scales re-tiled by tern_retile_scales; required
                              by the streamed entry points, else may be NULL */
    int32_t flags;         /* TERN_MATRIX_STATIC or 0 */
    int32_t reserved;      /* must be 0 */
} tern_matrix;

/*
 * Load-time re-tile of the group scales into the order the streamed kernels
 * consume them (Bonsai page, "后面还有没有优化空间": re-tile codes and
 * scales at load time).  A "unit" is 32 rows x one 128-byte superblock of
 * codes (640 positions = 5 groups in TERN_FMT_BASE3, 512 = 4 groups in
 * TERN_FMT_2BIT); units are numbered rb * SB + sb with rb = row / 32 and SB =
 * ceil(used row bytes / 128).  Unit u holds 32 rows x GPS fp16 scales
 * (GPS = 5 or 4), row-major, zero past N and past ceil(K/128):
 *   out[(u * 32 + r) * GPS + g] = scales[(32 rb + r) * G + GPS sb + g].
 * out: device, 16-byte aligned, tern_tiled_scales_bytes() bytes.
 */
tern_status tern_tiled_scales_bytes(int32_t fmt, int32_t N, int32_t K, size_t *bytes);
/* Errors (both): TERN_EINVAL for an unknown format, N or K < 1, a NULL or
 * misaligned pointer; tern_retile_scales returns TERN_ECUDA when its launch
 * fails. */
tern_status tern_retile_scales(const tern_matrix *W, uint16_t *out, void *stream);

/* Human-readable name of a status code (static storage).  Library plumbing:
 * the pages have no counterpart. */
const char *tern_status_string(tern_status s);

/* Message of the last failure on the calling host thread ("" if none).
 * Library plumbing: the pages have no counterpart. */
const char *tern_last_error(void);

/*
 * Sizes of the device layout for an N x K matrix: the minimal row stride
 * (used row bytes rounded up to 16), the packed bytes N*row_stride and the
 * scale bytes 2*N*ceil(K/group).  Any output pointer may be NULL.
 * The two densities are the pages': base-3 close to 1.6 bit per trit (Bonsai
 * page, "后面还有没有优化空间"; a trit carries log2 3 = 1.585 bits, page
 * pwwt.cn/news/5175886 section 1.1) and 2 bit per trit in a 2-bit field
 * (same section; Bonsai page, "PQ2 会不会快很多"), plus one FP16 scale per
 * group (4sapi page, section 三).  Errors: TERN_EINVAL for an unknown format
 * or N, K, group < 1.
 */
tern_status tern_packed_size(int32_t fmt, int32_t N, int32_t K, int32_t group,
                             int64_t *row_stride, size_t *packed_bytes,
                             size_t *scale_bytes);

/* Bytes per row of the canonical (file) encodings: base-3 = ceil(K/5)
 * (byte value sum_{i<5} t_i 3^i over K = 5j+i, least significant digit
 * first), 2-bit = ceil(K/4) (bits [2i,2i+1] of byte j hold K = 4j+i),
 * bit-plane = 2*ceil(K/8) (the nonzero plane, then the sign plane, bit k mod
 * 8 of byte k/8; the Bonsai page, "后面还有没有优化空间").  These
 * are the PTQ1_0-style (5 trits a byte) and PQ2-style (4 trits a byte) rows
 * of the Bonsai page ("Decode 为什么只能算一般", "PQ2 会不会快很多"); the
 * digit order is this library's reading, the pages give none.  Errors:
 * TERN_EINVAL for an unknown format, K < 1 or a NULL `bytes`. */
tern_status tern_canonical_row_bytes(int32_t fmt, int32_t K, int64_t *bytes);

/*
 * Pack trits into the device layout: the packing step that ends post-training
 * ternarisation (page pwwt.cn/news/5175886, section 1.2: quantised weights
 * and scales are packed in a fixed format), in the order the decode kernels
 * consume the codes (Bonsai page, "后面还有没有优化空间": re-tile codes at
 * load time into consumption order).
 *  trits: device int8 [N][K] in {-1, 0, +1}.
 *  packed_out: device, 16-byte aligned, N*row_stride bytes (row_stride as in
 *    tern_matrix).  Every byte of every row is written.
 *  d_invalid: optional device int32 counter (may be NULL); the number of
 *    trits outside {-1,0,+1} is added to it (they are packed as 0).
 */
tern_status tern_pack(int32_t fmt, const int8_t *trits, int32_t N, int32_t K,
                      void *packed_out, int64_t row_stride, int32_t *d_invalid,
                      void *stream);

/* Inverse of tern_pack: trits_out device int8 [N][K] -- the "unpack base-3,
 * restore -1/0/+1" step of the Bonsai page ("Decode 为什么只能算一般"),
 * written out to memory for tests.  Invalid codes (D3 bytes that are no
 * code, D2 fields equal to 3, padding digits other than t = 1) are counted in
 * d_invalid (may be NULL) and unpacked as 0.  Errors: TERN_EINVAL for a bad
 * matrix or a NULL output. */
tern_status tern_unpack(const tern_matrix *W, int8_t *trits_out,
                        int32_t *d_invalid, void *stream);

/* Load-time re-tile (Bonsai page, "后面还有没有优化空间": rearrange the codes
 * at load time in the order the integer dot product consumes them):
 * canonical bytes (device [N][canonical row bytes], rows contiguous) into
 * the device layout.  Invalid canonical codes are counted in d_invalid (may
 * be NULL).  Errors: TERN_EINVAL for bad shapes, strides or pointers. */
tern_status tern_import(int32_t fmt, const uint8_t *canonical, int32_t N,
                        int32_t K, void *packed_out, int64_t row_stride,
                        int32_t *d_invalid, void *stream);

/* Device layout back to canonical bytes (device [N][canonical row bytes]):
 * the inverse of tern_import (same passage).  Errors as tern_unpack. */
tern_status tern_export(const tern_matrix *W, uint8_t *canonical_out,
                        int32_t *d_invalid, void *stream);

/*
 * Producer-side ternarisation of float weights, no calibration data (page
 * pwwt.cn/news/5175886, section 1.2: per block two thresholds -- values
 * between them become 0, the two sides +1 and -1 -- and a scale that keeps
 * the residual small; m.nxbn.cn/news/172464, section 1.2: threshold plus one
 * scale per group; 4sapi page, section 三: one FP16 scale per group).  Per
 * group of `group` (= 128) consecutive K positions of row n of w:
 *   keep the k largest |w| (larger first, lower index first among equals),
 *   t = sign(w) on them and 0 elsewhere, alpha = fp16(S / k) (round to
 *   nearest even), for the k that maximises S^2 / k, S = the fp32 sum of
 *   the kept |w| added in index order, score = fp32(fp32(S * S) / k); the
 *   largest score wins, the smallest k among equal scores; k = 0 (t = 0,
 *   alpha = 0) when no score is above 0.  This is the cut that minimises
 *   sum (w - alpha t)^2 over all thresholds.
 *  w: device fp32 [N][ldw], ldw >= K, finite values.
 *  trits: device int8 [N][K] in {-1, 0, +1} (the input of tern_pack).
 *  scales: device fp16 bits [N][ceil(K/128)], 2-byte aligned.
 * Errors: TERN_EINVAL for bad shapes or pointers, TERN_EUNSUPPORTED for a
 * group other than 128, TERN_ECUDA when the launch fails.
 */
tern_status tern_ternarize(const float *w, int32_t N, int32_t K, int32_t ldw, int32_t group,
                           int8_t *trits, uint16_t *scales, void *stream);

/*
 * Per-token int8 activation quantisation with an optional 128-point
 * Walsh-Hadamard rotation (Bonsai page, "Decode 为什么只能算一般": the FFN
 * input is Hadamard-rotated once for gate and up; activations are quantised
 * per token).  Row m of x (ldx elements apart, fp16 if x_is_fp16 else fp32):
 *   x^ = x, or x^ = H x per 128-block (unnormalised Sylvester butterflies in
 *        fp32, stages h = 1..64) when fwht_block == 128 (needs K % 128 == 0);
 *   amax = max_k |x^_k|;  inv = 127/amax (IEEE fp32 division);
 *   q[m][k] = clamp(rint_half_even(x^_k * inv), -127, 127) for k < K,
 *   q[m][k] = 0 for K <= k < ldq;
 *   s_x[m] = amax/127, times fp32(1/sqrt(128)) when rotated;
 *   amax == 0 gives s_x = 0 and q = 0;
 *   with TERN_QUANT_RMSNORM in flags, s_x is also divided by the row's rms.
 *  x: device, 16-byte aligned, ldx a multiple of 8 (fp16) or 4 (fp32).
 *  q: device int8 [M][ldq], 16-byte aligned, ldq >= K, ldq % 16 == 0.
 *  s_x: device fp32 [M].  Inputs must be finite.
 */
tern_status act_quant_fwht(const void *x, int32_t x_is_fp16, int32_t M,
                           int32_t K, int32_t ldx, int32_t fwht_block,
                           int32_t flags, int8_t *q, int32_t ldq, float *s_x,
                           void *stream);

/*
 * Ternary GEMV / skinny GEMM for decode, M = 1..16 token rows (Bonsai page,
 * "Decode 为什么只能算一般": batch-1 decode is a matrix-vector product that
 * reads every packed weight once per token; the kernel unpacks the codes,
 * restores -1/0/+1, reads the group scale and takes an integer dot product,
 * never writing dequantised weights back; 4sapi page, section 三: add or
 * subtract by sign, then multiply by the FP16 group scale):
 *   y[m][n] = residual[m][n] + s_x[m] * sum_g s_w[n][g] * P[m][n][g],
 *   P[m][n][g] = sum_{k in group g} w[n][k] * q[m][k]   (exact int32),
 * with residual taken as 0 when `residual` is NULL.
 * Errors: TERN_EINVAL for a bad matrix, M outside 1..16, misaligned or NULL
 * buffers or strides; TERN_ECUDA when the launch fails.
 *  q: device int8 [M][ldq], 16-byte aligned, ldq >= K, ldq % 16 == 0
 *     (bytes past K are ignored).  s_x: device fp32 [M].
 *  residual, y: device fp32 [M][ldy], ldy >= N; residual may equal y.
 */
tern_status tern_gemv(const tern_matrix *W, const int8_t *q, int32_t ldq,
                      const float *s_x, int32_t M, const float *residual,
                      float *y, int32_t ldy, void *stream);

/*
 * Prefill GEMM on the tensor cores (Bonsai page, "Decode 为什么只能算一般":
 * prefill is a large matrix multiply over the same packed weights), any
 * number of token rows M >= 1:
 *   y[m][n] = s_x[m] * sum_g s_w[n][g] * P[m][n][g],
 *   P[m][n][g] = sum_{k in group g} w[n][k] * q[m][k]   (exact int32),
 * the product of tern_gemv without a residual.  The trits are expanded to
 * int8 in shared memory and multiplied by tcgen05.mma kind::i8 into int32
 * tensor memory, one 128-K group at a time; the fp32 epilogue applies the
 * group scales in group order.
 *  q: device int8 [M][ldq], 16-byte aligned, ldq >= K, ldq % 16 == 0
 *     (bytes past K are ignored).  s_x: device fp32 [M].
 *  y: device fp32 [M][ldy], ldy >= N; must not overlap q.
 * The caller owns every buffer; nothing is allocated.  While the device
 * error word is set (a bounded wait in an earlier kernel ran out; see
 * tern_device_error) the kernel returns without computing.
 */
tern_status tern_gemm(const tern_matrix *W, const int8_t *q, int32_t ldq,
                      const float *s_x, int32_t M, float *y, int32_t ldy,
                      void *stream);

/*
 * Fused gate/up + SwiGLU (Bonsai page, "Decode 为什么只能算一般"):
 *   g = Wg x^, u = Wu x^ (each as in tern_gemv, same q and s_x),
 *   h[m][n] = g * sigmoid(g) * u,  sigmoid(z) = 1/(1+exp(-z)).
 *  Wg and Wu must have the same fmt, N, K and group.  h: device fp32
 *  [M][ldh], ldh >= N.
 */
tern_status tern_gateup_swiglu(const tern_matrix *Wg, const tern_matrix *Wu,
                               const int8_t *q, int32_t ldq, const float *s_x,
                               int32_t M, float *h, int32_t ldh, void *stream);

/*
 * Test hook: the exact integer group partials P[m][n][g] (device int32
 * [M][N][ceil(K/group)]) of the integer dot product of tern_gemv (Bonsai
 * page, "Decode 为什么只能算一般": integer dot of the restored trits with the
 * quantised activation), as the CUDA-core engine computes them.
 */
tern_status tern_debug_group_partials(const tern_matrix *W, const int8_t *q,
                                      int32_t ldq, int32_t M, int32_t *P,
                                      void *stream);

/*
 * Activation statistics, the input of the fused quantisation below (Bonsai
 * page, "Decode 为什么只能算一般": activations are re-quantised between the
 * matmuls of a layer, so a producer can hand its consumer the statistics
 * that quantisation needs).  For each
 * token row m of x (fp32 [M][ldx], 16-byte aligned, ldx % 4 == 0) and each
 * 128-element block b of its first K elements (the last block zero-padded):
 *   stats[(m*stats_ld + b)*4 + 0] = max |x_b|
 *   stats[(m*stats_ld + b)*4 + 1] = max |H x_b|   (H: act_quant_fwht's rotation)
 *   stats[(m*stats_ld + b)*4 + 2] = sum x_b^2     (fp32)
 *   stats[(m*stats_ld + b)*4 + 3] = 0
 * stats: device fp32, 16-byte aligned, stats_ld >= ceil(K/128).
 */
tern_status tern_act_stats(const float *x, int32_t M, int32_t K, int32_t ldx,
                           float *stats, int32_t stats_ld, void *stream);

/*
 * tern_gemv with the per-token quantisation of its input done inside the
 * kernel: x is the fp32 activation [M][ldx] (16-byte aligned, ldx % 4 == 0,
 * ldx >= K; must not overlap y), x_stats its block statistics (as written by
 * tern_act_stats, or by the y_stats of the call that produced x; row stride
 * x_stats_ld blocks).  With qflags TERN_QUANT_FWHT128 and/or
 * TERN_QUANT_RMSNORM, q and s_x are those act_quant_fwht(x, fwht_block =
 * 128 if FWHT128, flags = RMSNORM) gives -- q bit for bit; s_x with RMSNORM
 * up to the summation order of the squares.  Then y as tern_gemv computes
 * it.  y_stats (optional, 16-byte aligned, y_stats_ld >= ceil(N/128)) receives
 * the statistics of y, so the next call can quantise y without a separate
 * launch (the Bonsai page's chain of re-quantised activations).
 */
tern_status tern_gemv_fused(const tern_matrix *W, const float *x, int32_t ldx,
                            const float *x_stats, int32_t x_stats_ld,
                            int32_t qflags, int32_t M, const float *residual,
                            float *y, int32_t ldy, float *y_stats,
                            int32_t y_stats_ld, void *stream);

/* tern_gateup_swiglu with the fused input quantisation of tern_gemv_fused;
 * h_stats (optional) receives the statistics of h. */
tern_status tern_gateup_swiglu_fused(const tern_matrix *Wg, const tern_matrix *Wu,
                                     const float *x, int32_t ldx,
                                     const float *x_stats, int32_t x_stats_ld,
                                     int32_t qflags, int32_t M, float *h,
                                     int32_t ldh, float *h_stats,
                                     int32_t h_stats_ld, void *stream);

/*
 * Streamed forms of tern_gemv_fused / tern_gateup_swiglu_fused for decode
 * with M = 1 or 2 token rows (Bonsai page, "Decode 为什么只能算一般": at batch
 * 1 the memory controller spends decode moving weights, so each projection
 * should cost about its bytes), same results and arguments apart from these:
 *  - the activation statistics are not needed: every CTA forms the row
 *    scale from x itself (max |x|, or max |H x| with TERN_QUANT_FWHT128);
 *  - W->scales_tiled must hold the re-tiled scales (tern_retile_scales);
 *  - workspace: device, 16-byte aligned, >= tern_stream_workspace_bytes()
 *    bytes, all zero before its first use.  It carries, from its start, the
 *    partial sums of the 32-row blocks that two CTAs share (one 64-bit word
 *    per row, matrix and token: fp32 value and a tag); every call clears
 *    what it wrote, so the workspace is all zero again after each call and
 *    one workspace, sized for the largest call, serves a whole chain of
 *    calls of any sizes on one stream (calls that may overlap need separate
 *    workspaces).  The exception is a call whose bounded wait ran out
 *    (tern_device_error reports it): a partial published after the wait
 *    gave up can stay behind, so zero the workspace again before reusing it.
 * One CTA per SM streams an equal share of the matrix's 32-row x 128-byte
 * tiles; with TERN_MATRIX_STATIC the tiles start streaming before the
 * previous kernel on the stream has finished.  x must not overlap y / h.
 */
tern_status tern_stream_workspace_bytes(int32_t fmt, int32_t N, int32_t M,
                                        int32_t two_matrices, size_t *bytes);
tern_status tern_gemv_streamed(const tern_matrix *W, const float *x, int32_t ldx,
                               int32_t qflags, int32_t M, const float *residual,
                               float *y, int32_t ldy, void *workspace,
                               size_t ws_bytes, void *stream);
tern_status tern_gateup_swiglu_streamed(const tern_matrix *Wg, const tern_matrix *Wu,
                                        const float *x, int32_t ldx, int32_t qflags,
                                        int32_t M, float *h, int32_t ldh,
                                        void *workspace, size_t ws_bytes,
                                        void *stream);

/*
 * tern_gemv_streamed without a caller workspace (the pages have no
 * counterpart: this is a convenience of the library).  Some callers cannot
 * call cudaMalloc: a plug-in whose host program owns all device memory
 * through its own pool or a fixed budget, or code on a latency-critical
 * path where cudaMalloc's implicit device-wide synchronisation would stall
 * other streams.  This entry point allocates nothing.  The kernel's scratch
 * -- the partial sums of the row blocks that two CTAs share -- is a fixed array of TERN_NOALLOC_SCRATCH_BYTES (1 MiB) inside the
 * library, held on every GPU that loads the library until the process exits.
 * Arguments, results and errors are those of tern_gemv_streamed.  Also:
 *  - sizes whose scratch exceeds the array are rejected with TERN_EINVAL
 *    (N <= 129024 at M = 1, N <= 65024 at M = 2);
 *  - the first call on a device looks up the array's device address there
 *    (that device current) and keeps it; make that first call before any
 *    stream capture;
 *  - each call first clears the part of the array it uses (an asynchronous
 *    memset on `stream`, then the kernel); every call on a device shares
 *    the one array, so calls that may overlap on the GPU (other streams,
 *    other host threads) race and give wrong results: serialise them.
 */
#define TERN_NOALLOC_SCRATCH_BYTES (1u << 20)
tern_status tern_gemv_streamed_noalloc(const tern_matrix *W, const float *x, int32_t ldx,
                                       int32_t qflags, int32_t M, const float *residual,
                                       float *y, int32_t ldy, void *stream);

/*
 * Q4_0 KV cache of one layer for decode attention (Bonsai page, "先交代机器和
 * 配置": K and V cached as Q4_0; the passage before "PQ2 会不会快很多": the Q4
 * data is decoded inside attention).  Q4_0 blocks of 32 values along the head
 * dimension: an fp16 scale d and 32 4-bit codes, value = (code - 8) d;
 * byte j of a block holds element j (low nibble) and element j + 16 (high
 * nibble).  Per KV head g and token t:
 *   k_codes[(g * capacity + t) * D/2 ..]   the D/2 code bytes of K,
 *   k_scales[(g * capacity + t) * D/32 ..] its D/32 fp16 block scales,
 * and v_codes / v_scales alike.  All device memory owned by the caller;
 * codes 16-byte aligned, scales 2-byte aligned.  This build takes D = 128.
 */
typedef struct tern_kv_cache {
    int32_t Hkv;       /* KV heads */
    int32_t D;         /* head dimension (128) */
    int32_t capacity;  /* tokens the arrays hold */
    int32_t reserved;  /* must be 0 */
    uint8_t *k_codes;
    uint16_t *k_scales;
    uint8_t *v_codes;
    uint16_t *v_scales;
} tern_kv_cache;

/*
 * Appends one token at position pos (< capacity): k and v are device fp32
 * [Hkv][D] (the K and V parts of the QKV projection's output), quantised to
 * Q4_0 with d = m / -8 (m: the value of largest magnitude in the block, the
 * first on ties) and code = min(15, trunc(x / d + 8.5)) in fp32 (code 8 when
 * d = 0), d stored as fp16 rounded to nearest.  Errors: TERN_EINVAL for a bad
 * cache or position, TERN_ECUDA when a launch fails.
 */
tern_status tern_kv_append_q4_0(const float *k, const float *v, int32_t pos,
                                const tern_kv_cache *cache, void *stream);

/* Workspace bytes of tern_attention_decode_q4_0 for Hq query heads over L
 * cached tokens on the current device. */
tern_status tern_attention_workspace_bytes(int32_t Hq, int32_t L, const tern_kv_cache *cache,
                                           size_t *bytes);

/*
 * Decode attention of one new token over the first L tokens of the cache:
 * query head h (q: device fp32 [Hq][D]) reads KV head h * Hkv / Hq and
 *   out[h] = sum_t softmax_t(q_h . k_t / sqrt(D)) v_t,
 * with k_t, v_t the dequantised Q4_0 rows (no rotary embedding or mask).
 * Split-context flash decoding: chunks of the context per CTA, merged in
 * chunk order by a second kernel.  Hq / Hkv must be 1, 2, 4, 5 or 8.
 *  out: device fp32 [Hq][D]; workspace: device, 16-byte aligned, at least
 *  tern_attention_workspace_bytes() bytes (no initial contents needed).
 * Errors: TERN_EINVAL for bad shapes, pointers or workspace,
 * TERN_EUNSUPPORTED for D != 128 or another group size, TERN_ECUDA.
 */
tern_status tern_attention_decode_q4_0(const float *q, int32_t Hq, const tern_kv_cache *cache,
                                       int32_t L, float *out, void *workspace, size_t ws_bytes,
                                       void *stream);

/*
 * Test hook of the streamed kernels (the integer dot product and the
 * in-kernel quantisation of the Bonsai page, "Decode 为什么只能算一般"): runs
 * tern_gemv_streamed (W1 == NULL, no residual) or tern_gateup_swiglu_streamed
 * (W1 = up matrix) with the same arguments and the same kernel, instantiated
 * to also write
 *   q_out[m][k] (k < K, row stride ldq_out >= K): the int8 input codes, and
 *   s_x_out[m]: the row scales, both as CTA 0 holds them after quantising;
 *   P_out[((mat * M + m) * N + n) * G + g] (G = ceil(K/128), mat 0 = W0,
 *   1 = W1): every exact int32 group partial sum_{k in g} w[n][k] q[m][k].
 * Outputs are device buffers owned by the caller; errors as
 * tern_gemv_streamed, and TERN_EINVAL when an output is missing.
 */
tern_status tern_debug_streamed(const tern_matrix *W0, const tern_matrix *W1, const float *x,
                                int32_t ldx, int32_t qflags, int32_t M, float *out, int32_t ldo,
                                int8_t *q_out, int32_t ldq_out, float *s_x_out, int32_t *P_out,
                                void *workspace, size_t ws_bytes, void *stream);

/*
 * Test hook of the prefill GEMM (the tensor-core product of the Bonsai page,
 * "Decode 为什么只能算一般": prefill is a large matrix multiply): tern_gemm
 * with the same arguments and kernel, instantiated to also write every exact
 * int32 group partial P[(m * N + n) * ceil(K/128) + g] as the tensor cores
 * accumulated it.  P: device int32, caller-owned.  Errors as tern_gemm.
 */
tern_status tern_debug_gemm_partials(const tern_matrix *W, const int8_t *q, int32_t ldq,
                                     const float *s_x, int32_t M, float *y, int32_t ldy, int32_t *P,
                                     void *stream);

/*
 * Test hook of the bounded waits (no counterpart on the pages): one kernel
 * waits on something nothing will ever complete -- kind 0: an mbarrier phase
 * (the form of the weight-ring and cluster waits), kind 1: a tagged 64-bit
 * word (the form of the wait for a neighbour's partial) -- for at most
 * budget_cycles SM cycles (1 .. 2e8), then records the timeout in the
 * device error word and returns.  tern_device_error then reports it.
 * Errors: TERN_EINVAL for a bad kind or budget.
 */
tern_status tern_debug_bounded_wait(int32_t kind, int64_t budget_cycles, void *stream);

/*
 * Test hook for the tensor-core path (no counterpart on the pages; it pins
 * the tcgen05 encodings the kernels use): one CTA computes
 *   D[m][n] = sum_k A[m][k] * B[n][k]   (int32, exact)
 * for A int8 [128][K] (row-major; read as unsigned bytes when a_signed == 0)
 * and B int8 [N][K] (row-major; unsigned when b_signed == 0), with A taken
 * from tensor memory (a_in_smem == 0) or shared memory (1), B from shared
 * memory without swizzle; mode 2: A and B both from shared memory in the
 * 128-byte-swizzled K-major layout of tern_gemm (then K % 128 == 0).
 * K in 32..512, a multiple of 32; N in 16..256, a multiple of 16.
 * A, B: device, 16-byte aligned; D: device int32 [128][N].
 */
tern_status tern_debug_mma_i8(int32_t a_in_smem, const int8_t *A, int32_t a_signed,
                              const int8_t *B, int32_t b_signed, int32_t *D,
                              int32_t K, int32_t N, void *stream);

/*
 * Test hook: selects the engine of the GEMV entry points for the calling
 * process -- 0: tensor cores (tcgen05), 1: CUDA cores (dp4a, the default).
 * Both compute the same integers; the tests compare them.  The tensor-core
 * engine has no bit-plane form: with it selected, a bit-plane matrix gives
 * TERN_EUNSUPPORTED.  tern_debug_group_partials always uses the CUDA-core
 * engine.
 */
tern_status tern_debug_select_engine(int32_t engine);

/*
 * Reads and clears the device error word of the current device: 0 when no
 * bounded wait in a kernel ran out since the last call, else a nonzero code
 * (1: a wait on an mbarrier, a cluster peer or a neighbour's partial ran
 * out).  Synchronises `stream`.  Library plumbing (no counterpart on the
 * pages).  After a nonzero code, zero every streamed workspace the failed
 * calls used before using it again.
 */
tern_status tern_device_error(int32_t *code_out, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* TERN_H */

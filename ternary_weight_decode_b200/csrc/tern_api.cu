// tern_api.cu -- the extern "C" boundary of libtern (declared in tern.h):
// argument validation on the host, then one launch per call on the caller's
// stream.  No allocation, no synchronisation, no CPU fallback.
#include <stdio.h>
#include <string.h>

#include "tern_common.cuh"
#include "tern_internal.h"

namespace {

thread_local char g_last_error[512] = "";

tern_status fail(tern_status s, const char *fmt, const char *detail = "") {
    snprintf(g_last_error, sizeof(g_last_error), fmt, detail);
    return s;
}

tern_status cuda_status(cudaError_t e, const char *what) {
    if (e == cudaSuccess) return TERN_OK;
    snprintf(g_last_error, sizeof(g_last_error), "%s: %s", what, cudaGetErrorString(e));
    return TERN_ECUDA;
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool valid_fmt(int32_t fmt) {
    return fmt == TERN_FMT_BASE3 || fmt == TERN_FMT_2BIT || fmt == TERN_FMT_BITPLANE;
}

tern_status check_matrix(const tern_matrix *W, const char *name) {
    if (!W) return fail(TERN_EINVAL, "%s: null matrix", name);
    if (!valid_fmt(W->fmt)) return fail(TERN_EINVAL, "%s: unknown format", name);
    if (W->N < 1 || W->K < 1) return fail(TERN_EINVAL, "%s: N and K must be >= 1", name);
    if (W->group != 128) return fail(TERN_EUNSUPPORTED, "%s: only group = 128 is supported", name);
    if (W->row_stride % 16 != 0 || W->row_stride < tern::device_row_bytes(W->fmt, W->K))
        return fail(TERN_EINVAL, "%s: row_stride must be a multiple of 16 and >= the used row bytes",
                    name);
    if (!W->packed || !aligned(W->packed, 16))
        return fail(TERN_EINVAL, "%s: packed must be a 16-byte aligned device pointer", name);
    if (!W->scales || !aligned(W->scales, 2))
        return fail(TERN_EINVAL, "%s: scales must be a 2-byte aligned device pointer", name);
    if (W->scales_tiled && !aligned(W->scales_tiled, 16))
        return fail(TERN_EINVAL, "%s: scales_tiled must be 16-byte aligned", name);
    if (W->flags & ~TERN_MATRIX_STATIC) return fail(TERN_EINVAL, "%s: unknown flag bits", name);
    if (W->reserved != 0) return fail(TERN_EINVAL, "%s: reserved must be 0", name);
    return TERN_OK;
}

tern_status check_activations(const int8_t *q, int32_t ldq, int32_t K, const float *s_x,
                              int32_t M) {
    if (M < 1 || M > 16) return fail(TERN_EINVAL, "M must be in 1..16%s");
    if (!q || !aligned(q, 16)) return fail(TERN_EINVAL, "q must be a 16-byte aligned device pointer%s");
    if (ldq < K || ldq % 16 != 0) return fail(TERN_EINVAL, "ldq must be >= K and a multiple of 16%s");
    if (!s_x || !aligned(s_x, 4)) return fail(TERN_EINVAL, "s_x must be a 4-byte aligned device pointer%s");
    return TERN_OK;
}

}  // namespace

namespace tern {
tern_status set_last_error(tern_status s, const char *message) {
    snprintf(g_last_error, sizeof(g_last_error), "%s", message);
    return s;
}
}  // namespace tern

extern "C" {

const char *tern_status_string(tern_status s) {
    switch (s) {
        case TERN_OK: return "TERN_OK";
        case TERN_EINVAL: return "TERN_EINVAL (invalid argument)";
        case TERN_ECUDA: return "TERN_ECUDA (CUDA error)";
        case TERN_EUNSUPPORTED: return "TERN_EUNSUPPORTED (not supported by this build)";
        case TERN_ETIMEOUT: return "TERN_ETIMEOUT (bounded device wait ran out)";
    }
    return "unknown tern_status";
}

const char *tern_last_error(void) { return g_last_error; }

tern_status tern_packed_size(int32_t fmt, int32_t N, int32_t K, int32_t group, int64_t *row_stride,
                             size_t *packed_bytes, size_t *scale_bytes) {
    if (!valid_fmt(fmt)) return fail(TERN_EINVAL, "unknown format%s");
    if (N < 1 || K < 1 || group < 1) return fail(TERN_EINVAL, "N, K and group must be >= 1%s");
    int64_t stride = (tern::device_row_bytes(fmt, K) + 15) / 16 * 16;
    if (row_stride) *row_stride = stride;
    if (packed_bytes) *packed_bytes = static_cast<size_t>(stride) * static_cast<size_t>(N);
    if (scale_bytes)
        *scale_bytes = 2u * static_cast<size_t>(N) * static_cast<size_t>(tern::ceil_div(K, group));
    return TERN_OK;
}

tern_status tern_canonical_row_bytes(int32_t fmt, int32_t K, int64_t *bytes) {
    if (!valid_fmt(fmt)) return fail(TERN_EINVAL, "unknown format%s");
    if (K < 1 || !bytes) return fail(TERN_EINVAL, "K must be >= 1 and bytes non-null%s");
    *bytes = tern::canonical_row_bytes(fmt, K);
    return TERN_OK;
}

tern_status tern_tiled_scales_bytes(int32_t fmt, int32_t N, int32_t K, size_t *bytes) {
    if (!valid_fmt(fmt)) return fail(TERN_EINVAL, "tern_tiled_scales_bytes: unknown format%s");
    if (N < 1 || K < 1 || !bytes) return fail(TERN_EINVAL, "tern_tiled_scales_bytes: bad arguments%s");
    *bytes = static_cast<size_t>(tern::tiled_scales_bytes(fmt, N, K));
    return TERN_OK;
}

tern_status tern_retile_scales(const tern_matrix *W, uint16_t *out, void *stream) {
    tern_status st = check_matrix(W, "tern_retile_scales");
    if (st != TERN_OK) return st;
    if (!out || !aligned(out, 16)) return fail(TERN_EINVAL, "tern_retile_scales: out must be 16-byte aligned%s");
    return cuda_status(tern::launch_retile_scales(W->fmt, W->scales, W->N, W->K, out,
                                                  static_cast<cudaStream_t>(stream)),
                       "tern_retile_scales");
}

tern_status tern_pack(int32_t fmt, const int8_t *trits, int32_t N, int32_t K, void *packed_out,
                      int64_t row_stride, int32_t *d_invalid, void *stream) {
    if (!valid_fmt(fmt)) return fail(TERN_EINVAL, "tern_pack: unknown format%s");
    if (N < 1 || K < 1) return fail(TERN_EINVAL, "tern_pack: N and K must be >= 1%s");
    if (!trits || !packed_out || !aligned(packed_out, 16))
        return fail(TERN_EINVAL, "tern_pack: null pointer or packed_out not 16-byte aligned%s");
    if (row_stride % 16 != 0 || row_stride < tern::device_row_bytes(fmt, K))
        return fail(TERN_EINVAL, "tern_pack: bad row_stride%s");
    return cuda_status(tern::launch_pack(fmt, trits, N, K, packed_out, row_stride, d_invalid,
                                         static_cast<cudaStream_t>(stream)),
                       "tern_pack");
}

tern_status tern_unpack(const tern_matrix *W, int8_t *trits_out, int32_t *d_invalid, void *stream) {
    tern_status st = check_matrix(W, "tern_unpack");
    if (st != TERN_OK) return st;
    if (!trits_out) return fail(TERN_EINVAL, "tern_unpack: null output%s");
    return cuda_status(tern::launch_unpack(W->fmt, W->packed, W->N, W->K, W->row_stride, trits_out,
                                           d_invalid, static_cast<cudaStream_t>(stream)),
                       "tern_unpack");
}

tern_status tern_import(int32_t fmt, const uint8_t *canonical, int32_t N, int32_t K,
                        void *packed_out, int64_t row_stride, int32_t *d_invalid, void *stream) {
    if (!valid_fmt(fmt)) return fail(TERN_EINVAL, "tern_import: unknown format%s");
    if (N < 1 || K < 1) return fail(TERN_EINVAL, "tern_import: N and K must be >= 1%s");
    if (!canonical || !packed_out || !aligned(packed_out, 16))
        return fail(TERN_EINVAL, "tern_import: null pointer or packed_out not 16-byte aligned%s");
    if (row_stride % 16 != 0 || row_stride < tern::device_row_bytes(fmt, K))
        return fail(TERN_EINVAL, "tern_import: bad row_stride%s");
    return cuda_status(tern::launch_import(fmt, canonical, N, K, packed_out, row_stride, d_invalid,
                                           static_cast<cudaStream_t>(stream)),
                       "tern_import");
}

tern_status tern_export(const tern_matrix *W, uint8_t *canonical_out, int32_t *d_invalid,
                        void *stream) {
    tern_status st = check_matrix(W, "tern_export");
    if (st != TERN_OK) return st;
    if (!canonical_out) return fail(TERN_EINVAL, "tern_export: null output%s");
    return cuda_status(tern::launch_export(W->fmt, W->packed, W->N, W->K, W->row_stride,
                                           canonical_out, d_invalid,
                                           static_cast<cudaStream_t>(stream)),
                       "tern_export");
}

tern_status tern_ternarize(const float *w, int32_t N, int32_t K, int32_t ldw, int32_t group,
                           int8_t *trits, uint16_t *scales, void *stream) {
    if (N < 1 || K < 1) return fail(TERN_EINVAL, "tern_ternarize: N and K must be >= 1%s");
    if (group != 128) return fail(TERN_EUNSUPPORTED, "tern_ternarize: only group = 128 is supported%s");
    if (!w || !aligned(w, 4) || ldw < K) return fail(TERN_EINVAL, "tern_ternarize: bad w or ldw%s");
    if (!trits || !scales || !aligned(scales, 2))
        return fail(TERN_EINVAL, "tern_ternarize: null or misaligned output%s");
    return cuda_status(tern::launch_ternarize(w, N, K, ldw, trits, scales, static_cast<cudaStream_t>(stream)),
                       "tern_ternarize");
}

static tern_status check_cache(const tern_kv_cache *C, const char *name) {
    if (!C || C->Hkv < 1 || C->capacity < 1 || C->reserved != 0)
        return fail(TERN_EINVAL, "%s: bad cache (Hkv, capacity >= 1, reserved = 0)", name);
    if (C->D != 128) return fail(TERN_EUNSUPPORTED, "%s: this build takes head dimension 128", name);
    if (!C->k_codes || !C->v_codes || !aligned(C->k_codes, 16) || !aligned(C->v_codes, 16) ||
        !C->k_scales || !C->v_scales || !aligned(C->k_scales, 2) || !aligned(C->v_scales, 2))
        return fail(TERN_EINVAL, "%s: cache arrays missing or misaligned", name);
    return TERN_OK;
}

static cudaError_t device_sms(int *sms) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(sms, cudaDevAttrMultiProcessorCount, dev);
    return e;
}

tern_status tern_kv_append_q4_0(const float *k, const float *v, int32_t pos, const tern_kv_cache *cache,
                                void *stream) {
    tern_status st = check_cache(cache, "tern_kv_append_q4_0");
    if (st != TERN_OK) return st;
    if (pos < 0 || pos >= cache->capacity) return fail(TERN_EINVAL, "tern_kv_append_q4_0: pos outside the cache%s");
    if (!k || !v || !aligned(k, 4) || !aligned(v, 4)) return fail(TERN_EINVAL, "tern_kv_append_q4_0: bad k or v%s");
    return cuda_status(tern::launch_kv_append(k, v, pos, *cache, static_cast<cudaStream_t>(stream)),
                       "tern_kv_append_q4_0");
}

tern_status tern_attention_workspace_bytes(int32_t Hq, int32_t L, const tern_kv_cache *cache, size_t *bytes) {
    tern_status st = check_cache(cache, "tern_attention_workspace_bytes");
    if (st != TERN_OK) return st;
    if (Hq < 1 || L < 1 || !bytes) return fail(TERN_EINVAL, "tern_attention_workspace_bytes: bad arguments%s");
    int sms = 0;
    cudaError_t e = device_sms(&sms);
    if (e != cudaSuccess) return cuda_status(e, "tern_attention_workspace_bytes");
    *bytes = tern::attention_workspace_bytes(Hq, L, cache->Hkv, sms);
    return TERN_OK;
}

tern_status tern_attention_decode_q4_0(const float *q, int32_t Hq, const tern_kv_cache *cache, int32_t L,
                                       float *out, void *workspace, size_t ws_bytes, void *stream) {
    const char *name = "tern_attention_decode_q4_0";
    tern_status st = check_cache(cache, name);
    if (st != TERN_OK) return st;
    if (Hq < 1 || Hq % cache->Hkv != 0) return fail(TERN_EINVAL, "%s: Hq must be a multiple of Hkv", name);
    if (L < 1 || L > cache->capacity) return fail(TERN_EINVAL, "%s: L must be in 1..capacity", name);
    if (!q || !aligned(q, 16) || !out || !aligned(out, 4))
        return fail(TERN_EINVAL, "%s: q (16-byte aligned) and out are required", name);
    int sms = 0;
    cudaError_t e = device_sms(&sms);
    if (e != cudaSuccess) return cuda_status(e, name);
    if (!workspace || !aligned(workspace, 16) || ws_bytes < tern::attention_workspace_bytes(Hq, L, cache->Hkv, sms))
        return fail(TERN_EINVAL, "%s: workspace missing, misaligned or too small", name);
    const char *why = nullptr;
    e = tern::launch_attention(q, Hq, *cache, L, out, static_cast<float *>(workspace), sms,
                               static_cast<cudaStream_t>(stream), &why);
    if (why) return fail(TERN_EUNSUPPORTED, "tern_attention_decode_q4_0: %s", why);
    return cuda_status(e, name);
}

tern_status act_quant_fwht(const void *x, int32_t x_is_fp16, int32_t M, int32_t K, int32_t ldx,
                           int32_t fwht_block, int32_t flags, int8_t *q, int32_t ldq, float *s_x,
                           void *stream) {
    if (M < 1 || K < 1) return fail(TERN_EINVAL, "act_quant_fwht: M and K must be >= 1%s");
    if (K > 49152) return fail(TERN_EUNSUPPORTED, "act_quant_fwht: K > 49152 is not supported%s");
    if (fwht_block != 0 && fwht_block != 128)
        return fail(TERN_EINVAL, "act_quant_fwht: fwht_block must be 0 or 128%s");
    if (flags & ~TERN_QUANT_RMSNORM) return fail(TERN_EINVAL, "act_quant_fwht: unknown flag bits%s");
    if (fwht_block == 128 && K % 128 != 0)
        return fail(TERN_EINVAL, "act_quant_fwht: the Hadamard rotation needs K %% 128 == 0%s");
    if (!x || !aligned(x, 16)) return fail(TERN_EINVAL, "act_quant_fwht: x must be 16-byte aligned%s");
    if (ldx < K || ldx % (x_is_fp16 ? 8 : 4) != 0)
        return fail(TERN_EINVAL, "act_quant_fwht: ldx must be >= K and keep rows 16-byte aligned%s");
    if (!q || !aligned(q, 16) || ldq < K || ldq % 16 != 0)
        return fail(TERN_EINVAL, "act_quant_fwht: q must be 16-byte aligned with ldq >= K, ldq %% 16 == 0%s");
    if (!s_x || !aligned(s_x, 4)) return fail(TERN_EINVAL, "act_quant_fwht: bad s_x%s");
    return cuda_status(tern::launch_act_quant(x, x_is_fp16 != 0, M, K, ldx, fwht_block, flags, q, ldq, s_x,
                                              static_cast<cudaStream_t>(stream)),
                       "act_quant_fwht");
}

static tern_status run_gemv(tern::GemvLaunch &L, const char *name, cudaStream_t s) {
    const char *why = nullptr;
    cudaError_t e = tern::launch_gemv(L, s, &why);
    if (why) return fail(TERN_EUNSUPPORTED, "%s", why);
    return cuda_status(e, name);
}

tern_status tern_gemv(const tern_matrix *W, const int8_t *q, int32_t ldq, const float *s_x,
                      int32_t M, const float *residual, float *y, int32_t ldy, void *stream) {
    tern_status st = check_matrix(W, "tern_gemv");
    if (st != TERN_OK) return st;
    st = check_activations(q, ldq, W->K, s_x, M);
    if (st != TERN_OK) return st;
    if (!y || !aligned(y, 4) || ldy < W->N) return fail(TERN_EINVAL, "tern_gemv: bad y or ldy%s");
    if (residual && !aligned(residual, 4)) return fail(TERN_EINVAL, "tern_gemv: bad residual%s");
    tern::GemvLaunch L = {};
    L.mode = tern::kModeGemv;
    L.fmt = W->fmt;
    L.N = W->N;
    L.K = W->K;
    L.G = static_cast<int>(tern::ceil_div(W->K, W->group));
    L.row_bytes = tern::device_row_bytes(W->fmt, W->K);
    L.row_stride = W->row_stride;
    L.packed[0] = L.packed[1] = W->packed;
    L.scales[0] = L.scales[1] = W->scales;
    L.prefetch_ok = (W->flags & TERN_MATRIX_STATIC) ? 1 : 0;
    L.q = q;
    L.ldq = ldq;
    L.s_x = s_x;
    L.M = M;
    L.residual = residual;
    L.out = y;
    L.ldo = ldy;
    return run_gemv(L, "tern_gemv", static_cast<cudaStream_t>(stream));
}

tern_status tern_gateup_swiglu(const tern_matrix *Wg, const tern_matrix *Wu, const int8_t *q,
                               int32_t ldq, const float *s_x, int32_t M, float *h, int32_t ldh,
                               void *stream) {
    tern_status st = check_matrix(Wg, "tern_gateup_swiglu (gate)");
    if (st != TERN_OK) return st;
    st = check_matrix(Wu, "tern_gateup_swiglu (up)");
    if (st != TERN_OK) return st;
    if (Wg->fmt != Wu->fmt || Wg->N != Wu->N || Wg->K != Wu->K || Wg->group != Wu->group ||
        Wg->row_stride != Wu->row_stride)
        return fail(TERN_EINVAL, "tern_gateup_swiglu: gate and up must share fmt, N, K, group, row_stride%s");
    st = check_activations(q, ldq, Wg->K, s_x, M);
    if (st != TERN_OK) return st;
    if (!h || !aligned(h, 4) || ldh < Wg->N) return fail(TERN_EINVAL, "tern_gateup_swiglu: bad h or ldh%s");
    tern::GemvLaunch L = {};
    L.mode = tern::kModeSwiglu;
    L.fmt = Wg->fmt;
    L.N = Wg->N;
    L.K = Wg->K;
    L.G = static_cast<int>(tern::ceil_div(Wg->K, Wg->group));
    L.row_bytes = tern::device_row_bytes(Wg->fmt, Wg->K);
    L.row_stride = Wg->row_stride;
    L.packed[0] = Wg->packed;
    L.packed[1] = Wu->packed;
    L.scales[0] = Wg->scales;
    L.scales[1] = Wu->scales;
    L.prefetch_ok = ((Wg->flags & Wu->flags) & TERN_MATRIX_STATIC) ? 1 : 0;
    L.q = q;
    L.ldq = ldq;
    L.s_x = s_x;
    L.M = M;
    L.residual = nullptr;
    L.out = h;
    L.ldo = ldh;
    return run_gemv(L, "tern_gateup_swiglu", static_cast<cudaStream_t>(stream));
}

tern_status tern_debug_group_partials(const tern_matrix *W, const int8_t *q, int32_t ldq, int32_t M,
                                      int32_t *P, void *stream) {
    tern_status st = check_matrix(W, "tern_debug_group_partials");
    if (st != TERN_OK) return st;
    if (M < 1 || M > 16) return fail(TERN_EINVAL, "tern_debug_group_partials: M must be in 1..16%s");
    if (!q || !aligned(q, 16) || ldq < W->K || ldq % 16 != 0)
        return fail(TERN_EINVAL, "tern_debug_group_partials: bad q or ldq%s");
    if (!P || !aligned(P, 4)) return fail(TERN_EINVAL, "tern_debug_group_partials: bad P%s");
    tern::GemvLaunch L = {};
    L.mode = tern::kModePartials;
    L.fmt = W->fmt;
    L.N = W->N;
    L.K = W->K;
    L.G = static_cast<int>(tern::ceil_div(W->K, W->group));
    L.row_bytes = tern::device_row_bytes(W->fmt, W->K);
    L.row_stride = W->row_stride;
    L.packed[0] = L.packed[1] = W->packed;
    L.scales[0] = L.scales[1] = W->scales;
    L.prefetch_ok = 0;
    L.q = q;
    L.ldq = ldq;
    L.s_x = nullptr;
    L.M = M;
    L.out = P;
    L.ldo = 0;
    return run_gemv(L, "tern_debug_group_partials", static_cast<cudaStream_t>(stream));
}

tern_status tern_device_error(int32_t *code_out, void *stream) {
    if (!code_out) return fail(TERN_EINVAL, "tern_device_error: null code_out%s");
    int value = 0;
    cudaError_t e = tern::read_clear_device_error(&value, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_status(e, "tern_device_error");
    *code_out = value;
    return TERN_OK;
}

tern_status tern_act_stats(const float *x, int32_t M, int32_t K, int32_t ldx, float *stats,
                           int32_t stats_ld, void *stream) {
    if (M < 1 || K < 1) return fail(TERN_EINVAL, "tern_act_stats: M and K must be >= 1%s");
    if (!x || !aligned(x, 16) || ldx < K || ldx % 4 != 0)
        return fail(TERN_EINVAL, "tern_act_stats: x must be 16-byte aligned, ldx >= K, ldx %% 4 == 0%s");
    if (!stats || !aligned(stats, 16) || stats_ld < tern::ceil_div(K, 128))
        return fail(TERN_EINVAL, "tern_act_stats: bad stats or stats_ld%s");
    return cuda_status(tern::launch_act_stats(x, M, K, ldx, stats, stats_ld,
                                              static_cast<cudaStream_t>(stream)),
                       "tern_act_stats");
}

tern_status tern_debug_mma_i8(int32_t a_in_smem, const int8_t *A, int32_t a_signed, const int8_t *B,
                              int32_t b_signed, int32_t *D, int32_t K, int32_t N, void *stream) {
    if (K < 32 || K > 512 || K % 32 != 0) return fail(TERN_EINVAL, "tern_debug_mma_i8: K must be 32..512, a multiple of 32%s");
    if (N < 16 || N > 256 || N % 16 != 0) return fail(TERN_EINVAL, "tern_debug_mma_i8: N must be 16..256, a multiple of 16%s");
    if (!A || !B || !D || !aligned(A, 16) || !aligned(B, 16) || !aligned(D, 16))
        return fail(TERN_EINVAL, "tern_debug_mma_i8: pointers must be 16-byte aligned%s");
    if (a_in_smem < 0 || a_in_smem > 2) return fail(TERN_EINVAL, "tern_debug_mma_i8: mode must be 0, 1 or 2%s");
    if (a_in_smem == 2 && K % 128 != 0)
        return fail(TERN_EINVAL, "tern_debug_mma_i8: mode 2 needs K %% 128 == 0%s");
    return cuda_status(tern::launch_debug_mma(a_in_smem, A, a_signed ? 1 : 0, B, b_signed ? 1 : 0,
                                              D, K, N, static_cast<cudaStream_t>(stream)),
                       "tern_debug_mma_i8");
}

tern_status tern_stream_workspace_bytes(int32_t fmt, int32_t N, int32_t M, int32_t two_matrices,
                                        size_t *bytes) {
    if (!valid_fmt(fmt) || N < 1 || M < 1 || M > 2 || !bytes)
        return fail(TERN_EINVAL, "tern_stream_workspace_bytes: bad arguments (M must be 1 or 2)%s");
    *bytes = tern::stream_workspace_bytes(fmt, N, M, two_matrices ? 2 : 1);
    return TERN_OK;
}

}  // extern "C"

namespace tern {
tern_status check_streamed_call(const tern_matrix *W0, const tern_matrix *W1, const float *x,
                                int32_t ldx, int32_t qflags, int32_t M, const float *residual,
                                const float *out, int32_t ldo, const char *name) {
    tern_status st = check_matrix(W0, name);
    if (st != TERN_OK) return st;
    if (W1) {
        st = check_matrix(W1, name);
        if (st != TERN_OK) return st;
        if (W0->fmt != W1->fmt || W0->N != W1->N || W0->K != W1->K || W0->group != W1->group ||
            W0->row_stride != W1->row_stride)
            return fail(TERN_EINVAL, "%s: gate and up must share fmt, N, K, group, row_stride", name);
    }
    if (M < 1 || M > 2) return fail(TERN_EUNSUPPORTED, "%s: the streamed kernels take M = 1 or 2", name);
    if (!W0->scales_tiled || (W1 && !W1->scales_tiled))
        return fail(TERN_EINVAL, "%s: scales_tiled is required (tern_retile_scales)", name);
    if (!x || !aligned(x, 16) || ldx < W0->K || ldx % 4 != 0)
        return fail(TERN_EINVAL, "%s: x must be 16-byte aligned, ldx >= K, ldx %% 4 == 0", name);
    if (qflags & ~(TERN_QUANT_FWHT128 | TERN_QUANT_RMSNORM)) return fail(TERN_EINVAL, "%s: unknown qflags", name);
    if ((qflags & TERN_QUANT_FWHT128) && W0->K % 128 != 0)
        return fail(TERN_EINVAL, "%s: the Hadamard rotation needs K %% 128 == 0", name);
    if (!out || !aligned(out, 4) || ldo < W0->N) return fail(TERN_EINVAL, "%s: bad output or its stride", name);
    if (residual && !aligned(residual, 4)) return fail(TERN_EINVAL, "%s: bad residual", name);
    return TERN_OK;
}
}  // namespace tern

namespace {
struct StreamDebug {
    int8_t *q;
    int32_t ldq;
    float *s_x;
    int32_t *P;
};

tern_status run_streamed(const tern_matrix *W0, const tern_matrix *W1, const float *x, int32_t ldx,
                         int32_t qflags, int32_t M, const float *residual, float *out, int32_t ldo,
                         void *workspace, size_t ws_bytes, void *stream, const char *name,
                         const StreamDebug *dbg = nullptr) {
    tern_status st = tern::check_streamed_call(W0, W1, x, ldx, qflags, M, residual, out, ldo, name);
    if (st != TERN_OK) return st;
    const size_t need = tern::stream_workspace_bytes(W0->fmt, W0->N, M, W1 ? 2 : 1);
    if (!workspace || !aligned(workspace, 16) || ws_bytes < need)
        return fail(TERN_EINVAL, "%s: workspace missing, misaligned or too small", name);
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_status(e, name);
    tern::StreamLaunch S = {};
    S.fmt = W0->fmt;
    S.swiglu = W1 ? 1 : 0;
    S.N = W0->N;
    S.K = W0->K;
    S.row_bytes = tern::device_row_bytes(W0->fmt, W0->K);
    S.row_stride = W0->row_stride;
    S.packed[0] = W0->packed;
    S.packed[1] = W1 ? W1->packed : W0->packed;
    S.scales_tiled[0] = W0->scales_tiled;
    S.scales_tiled[1] = W1 ? W1->scales_tiled : W0->scales_tiled;
    S.prefetch_ok = ((W0->flags & (W1 ? W1->flags : W0->flags)) & TERN_MATRIX_STATIC) ? 1 : 0;
    S.x = x;
    S.ldx = ldx;
    S.qflags = qflags;
    S.M = M;
    S.residual = residual;
    S.out = out;
    S.ldo = ldo;
    S.workspace = workspace;
    S.ws_bytes = ws_bytes;
    S.num_sms = sms;
    const char *why = nullptr;
    if (dbg) {
        S.dbg_q = dbg->q;
        S.dbg_ldq = dbg->ldq;
        S.dbg_sx = dbg->s_x;
        S.dbg_P = dbg->P;
        e = tern::launch_gemv_stream_debug(S, static_cast<cudaStream_t>(stream), &why);
    } else {
        e = tern::launch_gemv_stream(S, static_cast<cudaStream_t>(stream), &why);
    }
    if (why) return fail(TERN_EUNSUPPORTED, "%s", why);
    return cuda_status(e, name);
}
}  // namespace

extern "C" {

tern_status tern_gemv_streamed(const tern_matrix *W, const float *x, int32_t ldx, int32_t qflags,
                               int32_t M, const float *residual, float *y, int32_t ldy,
                               void *workspace, size_t ws_bytes, void *stream) {
    return run_streamed(W, nullptr, x, ldx, qflags, M, residual, y, ldy, workspace, ws_bytes, stream,
                        "tern_gemv_streamed");
}

tern_status tern_gateup_swiglu_streamed(const tern_matrix *Wg, const tern_matrix *Wu, const float *x,
                                        int32_t ldx, int32_t qflags, int32_t M, float *h,
                                        int32_t ldh, void *workspace, size_t ws_bytes,
                                        void *stream) {
    return run_streamed(Wg, Wu, x, ldx, qflags, M, nullptr, h, ldh, workspace, ws_bytes, stream,
                        "tern_gateup_swiglu_streamed");
}

tern_status tern_debug_streamed(const tern_matrix *W0, const tern_matrix *W1, const float *x,
                                int32_t ldx, int32_t qflags, int32_t M, float *out, int32_t ldo,
                                int8_t *q_out, int32_t ldq_out, float *s_x_out, int32_t *P_out,
                                void *workspace, size_t ws_bytes, void *stream) {
    const char *name = "tern_debug_streamed";
    if (!W0) return fail(TERN_EINVAL, "%s: null matrix", name);
    if (!q_out || ldq_out < W0->K || !s_x_out || !aligned(s_x_out, 4) || !P_out || !aligned(P_out, 4))
        return fail(TERN_EINVAL, "%s: q_out (ldq_out >= K), s_x_out and P_out are required", name);
    const StreamDebug dbg = {q_out, ldq_out, s_x_out, P_out};
    return run_streamed(W0, W1, x, ldx, qflags, M, nullptr, out, ldo, workspace, ws_bytes, stream, name,
                        &dbg);
}

static tern_status run_gemm(const tern_matrix *W, const int8_t *q, int32_t ldq, const float *s_x,
                            int32_t M, float *y, int32_t ldy, int32_t *dbg_P, void *stream) {
    tern_status st = check_matrix(W, "tern_gemm");
    if (st != TERN_OK) return st;
    if (M < 1) return fail(TERN_EINVAL, "tern_gemm: M must be >= 1%s");
    if (!q || !aligned(q, 16) || ldq < W->K || ldq % 16 != 0)
        return fail(TERN_EINVAL, "tern_gemm: q must be 16-byte aligned with ldq >= K, ldq %% 16 == 0%s");
    if (!s_x || !aligned(s_x, 4)) return fail(TERN_EINVAL, "tern_gemm: bad s_x%s");
    if (!y || !aligned(y, 4) || ldy < W->N) return fail(TERN_EINVAL, "tern_gemm: bad y or ldy%s");
    tern::GemmLaunch L = {};
    L.fmt = W->fmt;
    L.N = W->N;
    L.K = W->K;
    L.M = M;
    L.row_bytes = tern::device_row_bytes(W->fmt, W->K);
    L.row_stride = W->row_stride;
    L.packed = W->packed;
    L.scales = W->scales;
    L.q = q;
    L.ldq = ldq;
    L.s_x = s_x;
    L.y = y;
    L.ldy = ldy;
    L.dbg_P = dbg_P;
    const char *why = nullptr;
    cudaError_t e = tern::launch_gemm(L, static_cast<cudaStream_t>(stream), &why);
    if (why) return fail(TERN_EUNSUPPORTED, "tern_gemm: %s", why);
    return cuda_status(e, "tern_gemm");
}

tern_status tern_gemm(const tern_matrix *W, const int8_t *q, int32_t ldq, const float *s_x,
                      int32_t M, float *y, int32_t ldy, void *stream) {
    return run_gemm(W, q, ldq, s_x, M, y, ldy, nullptr, stream);
}

tern_status tern_debug_gemm_partials(const tern_matrix *W, const int8_t *q, int32_t ldq,
                                     const float *s_x, int32_t M, float *y, int32_t ldy, int32_t *P,
                                     void *stream) {
    if (!P || !aligned(P, 4)) return fail(TERN_EINVAL, "tern_debug_gemm_partials: bad P%s");
    return run_gemm(W, q, ldq, s_x, M, y, ldy, P, stream);
}

tern_status tern_debug_bounded_wait(int32_t kind, int64_t budget_cycles, void *stream) {
    if (kind != 0 && kind != 1) return fail(TERN_EINVAL, "tern_debug_bounded_wait: kind must be 0 or 1%s");
    if (budget_cycles < 1 || budget_cycles > 200000000LL)
        return fail(TERN_EINVAL, "tern_debug_bounded_wait: budget must be 1 .. 2e8 cycles%s");
    return cuda_status(tern::launch_debug_wait(kind, budget_cycles, static_cast<cudaStream_t>(stream)),
                       "tern_debug_bounded_wait");
}

tern_status tern_debug_select_engine(int32_t engine) {
    if (engine != 0 && engine != 1) return fail(TERN_EINVAL, "tern_debug_select_engine: engine must be 0 or 1%s");
    tern::select_engine(engine);
    return TERN_OK;
}

static tern_status check_fused_input(const float *x, int32_t ldx, int32_t K, const float *x_stats,
                                     int32_t x_stats_ld, int32_t qflags, int32_t M) {
    if (M < 1 || M > 16) return fail(TERN_EINVAL, "fused: M must be in 1..16%s");
    if (!x || !aligned(x, 16) || ldx < K || ldx % 4 != 0)
        return fail(TERN_EINVAL, "fused: x must be 16-byte aligned, ldx >= K, ldx %% 4 == 0%s");
    if (!x_stats || !aligned(x_stats, 16) || x_stats_ld < tern::ceil_div(K, 128))
        return fail(TERN_EINVAL, "fused: bad x_stats or x_stats_ld%s");
    if (qflags & ~(TERN_QUANT_FWHT128 | TERN_QUANT_RMSNORM))
        return fail(TERN_EINVAL, "fused: unknown qflags bits%s");
    if ((qflags & TERN_QUANT_FWHT128) && K % 128 != 0)
        return fail(TERN_EINVAL, "fused: the Hadamard rotation needs K %% 128 == 0%s");
    return TERN_OK;
}

tern_status tern_gemv_fused(const tern_matrix *W, const float *x, int32_t ldx, const float *x_stats,
                            int32_t x_stats_ld, int32_t qflags, int32_t M, const float *residual,
                            float *y, int32_t ldy, float *y_stats, int32_t y_stats_ld,
                            void *stream) {
    tern_status st = check_matrix(W, "tern_gemv_fused");
    if (st != TERN_OK) return st;
    st = check_fused_input(x, ldx, W->K, x_stats, x_stats_ld, qflags, M);
    if (st != TERN_OK) return st;
    if (!y || !aligned(y, 4) || ldy < W->N) return fail(TERN_EINVAL, "tern_gemv_fused: bad y or ldy%s");
    if (residual && !aligned(residual, 4)) return fail(TERN_EINVAL, "tern_gemv_fused: bad residual%s");
    if (y_stats && (!aligned(y_stats, 16) || y_stats_ld < tern::ceil_div(W->N, 128)))
        return fail(TERN_EINVAL, "tern_gemv_fused: bad y_stats or y_stats_ld%s");
    tern::GemvLaunch L = {};
    L.mode = tern::kModeGemv;
    L.fmt = W->fmt;
    L.N = W->N;
    L.K = W->K;
    L.G = static_cast<int>(tern::ceil_div(W->K, W->group));
    L.row_bytes = tern::device_row_bytes(W->fmt, W->K);
    L.row_stride = W->row_stride;
    L.packed[0] = L.packed[1] = W->packed;
    L.scales[0] = L.scales[1] = W->scales;
    L.prefetch_ok = (W->flags & TERN_MATRIX_STATIC) ? 1 : 0;
    L.M = M;
    L.residual = residual;
    L.out = y;
    L.ldo = ldy;
    L.x = x;
    L.ldx = ldx;
    L.x_stats = x_stats;
    L.x_stats_ld = x_stats_ld;
    L.qflags = qflags;
    L.y_stats = y_stats;
    L.y_stats_ld = y_stats_ld;
    return run_gemv(L, "tern_gemv_fused", static_cast<cudaStream_t>(stream));
}

tern_status tern_gateup_swiglu_fused(const tern_matrix *Wg, const tern_matrix *Wu, const float *x,
                                     int32_t ldx, const float *x_stats, int32_t x_stats_ld,
                                     int32_t qflags, int32_t M, float *h, int32_t ldh,
                                     float *h_stats, int32_t h_stats_ld, void *stream) {
    tern_status st = check_matrix(Wg, "tern_gateup_swiglu_fused (gate)");
    if (st != TERN_OK) return st;
    st = check_matrix(Wu, "tern_gateup_swiglu_fused (up)");
    if (st != TERN_OK) return st;
    if (Wg->fmt != Wu->fmt || Wg->N != Wu->N || Wg->K != Wu->K || Wg->group != Wu->group ||
        Wg->row_stride != Wu->row_stride)
        return fail(TERN_EINVAL, "tern_gateup_swiglu_fused: gate and up must share fmt, N, K, group, row_stride%s");
    st = check_fused_input(x, ldx, Wg->K, x_stats, x_stats_ld, qflags, M);
    if (st != TERN_OK) return st;
    if (!h || !aligned(h, 4) || ldh < Wg->N) return fail(TERN_EINVAL, "tern_gateup_swiglu_fused: bad h or ldh%s");
    if (h_stats && (!aligned(h_stats, 16) || h_stats_ld < tern::ceil_div(Wg->N, 128)))
        return fail(TERN_EINVAL, "tern_gateup_swiglu_fused: bad h_stats or h_stats_ld%s");
    tern::GemvLaunch L = {};
    L.mode = tern::kModeSwiglu;
    L.fmt = Wg->fmt;
    L.N = Wg->N;
    L.K = Wg->K;
    L.G = static_cast<int>(tern::ceil_div(Wg->K, Wg->group));
    L.row_bytes = tern::device_row_bytes(Wg->fmt, Wg->K);
    L.row_stride = Wg->row_stride;
    L.packed[0] = Wg->packed;
    L.packed[1] = Wu->packed;
    L.scales[0] = Wg->scales;
    L.scales[1] = Wu->scales;
    L.prefetch_ok = ((Wg->flags & Wu->flags) & TERN_MATRIX_STATIC) ? 1 : 0;
    L.M = M;
    L.out = h;
    L.ldo = ldh;
    L.x = x;
    L.ldx = ldx;
    L.x_stats = x_stats;
    L.x_stats_ld = x_stats_ld;
    L.qflags = qflags;
    L.y_stats = h_stats;
    L.y_stats_ld = h_stats_ld;
    return run_gemv(L, "tern_gateup_swiglu_fused", static_cast<cudaStream_t>(stream));
}

}  // extern "C"

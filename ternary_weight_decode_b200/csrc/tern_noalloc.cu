// tern_noalloc.cu -- tern_gemv_streamed for callers that cannot allocate
// device memory: the streamed kernel's scratch (partial sums of the row
// blocks cut between two CTAs) lives in a fixed array that the library
// itself holds on every device that loads it.
#include <stdio.h>

#include <mutex>

#include "tern_common.cuh"
#include "tern_internal.h"

namespace {

// Held on every device that loads the library, for as long as the process
// runs.  Shared by every call on that device; each call clears the part it
// uses before its kernel runs.
static __device__ __align__(256) unsigned char g_noalloc_scratch[TERN_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void *g_scratch_addr[kMaxDevices] = {};

// The device address of g_noalloc_scratch on the current device.  In host
// code the array's name only stands for it, so the address is looked up once
// per device (with that device current) and cached.
cudaError_t scratch_address(void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        if (!p) return cudaErrorInvalidSymbol;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return cudaSuccess;
}

}  // namespace

tern_status tern_gemv_streamed_noalloc(const tern_matrix *W, const float *x, int32_t ldx,
                                       int32_t qflags, int32_t M, const float *residual,
                                       float *y, int32_t ldy, void *stream) {
    // Every host-side check of the streamed entry point first, so that a
    // call that is rejected leaves the shared array untouched.
    const tern_status st = tern::check_streamed_call(W, nullptr, x, ldx, qflags, M, residual, y, ldy,
                                                     "tern_gemv_streamed_noalloc");
    if (st != TERN_OK) return st;
    const size_t bytes = TERN_NOALLOC_SCRATCH_BYTES;
    const size_t need = tern::stream_workspace_bytes(W->fmt, W->N, M, 1);
    if (need > bytes) {
        char msg[256];
        snprintf(msg, sizeof(msg),
                 "tern_gemv_streamed_noalloc: N = %d, M = %d needs %zu bytes of scratch, more than "
                 "the %zu the library holds (N <= 129024 at M = 1, N <= 65024 at M = 2)",
                 W->N, M, need, bytes);
        return tern::set_last_error(TERN_EINVAL, msg);
    }
    void *scratch = nullptr;
    cudaError_t e = scratch_address(&scratch);
    if (e != cudaSuccess) {
        char msg[256];
        snprintf(msg, sizeof(msg), "tern_gemv_streamed_noalloc: scratch set-up: %s",
                 cudaGetErrorString(e));
        return tern::set_last_error(TERN_ECUDA, msg);
    }
    // The kernel expects the scratch it uses to start at zero; clear it,
    // whatever an earlier (possibly failed) call left there.
    e = cudaMemsetAsync(scratch, 0, need, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) {
        char msg[256];
        snprintf(msg, sizeof(msg), "tern_gemv_streamed_noalloc: clearing the counters: %s",
                 cudaGetErrorString(e));
        return tern::set_last_error(TERN_ECUDA, msg);
    }
    return tern_gemv_streamed(W, x, ldx, qflags, M, residual, y, ldy, scratch, bytes, stream);
}

// tern_debug.cu -- test hooks that need kernels of their own:
//  * the streamed GEMV instantiated with its debug outputs (the int8 input
//    and row scales as CTA 0 holds them, every exact int32 group partial);
//  * a bounded wait that nothing satisfies, so that a test can watch the
//    timeout path record its error code and return, with the context intact.
#include "tern_gemv_stream.cuh"

namespace tern {
namespace {

// Never published by anything: the tagged-word wait below always runs out.
__device__ unsigned long long g_never_published = 0;

__global__ void debug_wait_kernel(int kind, long long budget) {
    __shared__ __align__(8) uint64_t bar;
    if (kind == 0) {
        if (threadIdx.x == 0) {
            mbar_init(&bar, 1);
            fence_mbar_init();
        }
        __syncwarp();
        // nobody arrives: the phase never completes
        (void)__all_sync(0xffffffffu, mbar_wait_bounded(&bar, 0, budget));
    } else if (threadIdx.x == 0) {
        (void)wait_tagged_word(&g_never_published, budget);
    }
}

}  // namespace

cudaError_t launch_gemv_stream_debug(const StreamLaunch &S, cudaStream_t s, const char **why) {
    return launch_sk_any<true>(S, s, why);
}

cudaError_t launch_debug_wait(int kind, long long budget_cycles, cudaStream_t s) {
    debug_wait_kernel<<<1, 32, 0, s>>>(kind, budget_cycles);
    return cudaGetLastError();
}

}  // namespace tern

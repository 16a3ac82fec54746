// tern_gemv_stream.cu -- release instantiations of the streamed GEMV
// (tern_gemv_stream.cuh) and its workspace size.
#include "tern_gemv_stream.cuh"

namespace tern {

size_t stream_workspace_bytes(int fmt, int N, int M, int nmat) {
    (void)fmt;
    const int MT = M <= 1 ? 1 : 2;
    const size_t RB = static_cast<size_t>(ceil_div(N, 32));
    return RB * 2 * nmat * MT * 32 * sizeof(float) + RB * sizeof(int);
}

cudaError_t launch_gemv_stream(const StreamLaunch &S, cudaStream_t s, const char **why) {
    return launch_sk_any<false>(S, s, why);
}

}  // namespace tern

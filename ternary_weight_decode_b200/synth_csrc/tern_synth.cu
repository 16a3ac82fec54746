// tern_synth.cu -- device side of the seeded input generator (libtern_synth).
//
// Input generation only: no packing, quantisation or dot-product arithmetic.
// Implements the same definition as ternary_weight_decode_b200/synth.py:
//   mix64   = SplitMix64 output function (Steele, Lea & Flood, OOPSLA 2014;
//             S. Vigna's public-domain reference code);
//   h(idx)  = mix64(key + (idx + 1) * 0x9E3779B97F4A7C15), key passed in
//             (key = mix64(seed * GAMMA + stream), computed on the host);
//   trit    = -1 if (h >> 32) < 1288490189, +1 if (h >> 32) >= 3006477108, else 0;
//   scale   = fp16(fp32(fp32((h >> 40) * 2^-24) * 0.045) + 0.005), each fp32
//             step rounded to nearest.
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace {

constexpr uint64_t kGamma = 0x9E3779B97F4A7C15ull;

__device__ __forceinline__ uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

__global__ void synth_trits_kernel(uint64_t key, int64_t row0, int64_t N, int64_t K, int8_t *out) {
    int64_t total = N * K;
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        uint64_t idx = static_cast<uint64_t>(row0 * K + i);
        uint32_t u = static_cast<uint32_t>(mix64(key + (idx + 1) * kGamma) >> 32);
        out[i] = u < 1288490189u ? -1 : (u >= 3006477108u ? 1 : 0);
    }
}

__global__ void synth_scales_kernel(uint64_t key, int64_t N, int64_t G, uint16_t *out) {
    int64_t total = N * G;
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        uint64_t h = mix64(key + (static_cast<uint64_t>(i) + 1) * kGamma);
        float a = __fmul_rn(static_cast<float>(static_cast<uint32_t>(h >> 40)), 5.9604644775390625e-8f);
        float b = __fmul_rn(a, 0.045f);
        float c = __fadd_rn(b, 0.005f);
        out[i] = __half_as_ushort(__float2half_rn(c));
    }
}

int grid_for(int64_t total) {
    int64_t b = (total + 255) / 256;
    if (b < 1) b = 1;
    if (b > 148 * 32) b = 148 * 32;
    return static_cast<int>(b);
}

}  // namespace

extern "C" {

// Trits of rows [row0, row0 + N) of the K-wide matrix with stream key `key`,
// written to out (device int8 [N][K]).  Returns a cudaError_t value.
int tern_synth_trits(uint64_t key, int64_t row0, int64_t N, int64_t K, int8_t *out, void *stream) {
    synth_trits_kernel<<<grid_for(N * K), 256, 0, static_cast<cudaStream_t>(stream)>>>(key, row0, N, K, out);
    return static_cast<int>(cudaGetLastError());
}

// fp16 scale bit patterns [N][G] for stream key `key` (device uint16).
int tern_synth_scales(uint64_t key, int64_t N, int64_t G, uint16_t *out, void *stream) {
    synth_scales_kernel<<<grid_for(N * G), 256, 0, static_cast<cudaStream_t>(stream)>>>(key, N, G, out);
    return static_cast<int>(cudaGetLastError());
}

}  // extern "C"

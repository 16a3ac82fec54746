// tern_format.cu -- load-time kernels: trits <-> device layout, canonical
// file encodings <-> device layout (the load-time re-tile of the Bonsai page,
// section "后面还有没有优化空间").  Not on the per-token hot path.
//
// Device layouts (see include/tern.h):
//   D3: word w covers K in [20w, 20w+20); byte j holds K = 20w + j + 4i,
//       i = 0..4, as y = ceil(256 V / 243), V = sum_i t_i 3^(4-i).
//   D2: word w covers K in [16w, 16w+16); bits [2i,2i+1] of byte j hold t
//       for K = 16w + 4i + j.
//   DB: word pair p covers K in [32p, 32p+32): word 2p is the nonzero plane
//       (w != 0), word 2p+1 the sign plane (w < 0); bit 8j + i holds
//       K = 32p + 4i + j.
// Canonical encodings:
//   base-3: byte j = sum_{i<5} t_{5j+i} 3^i;  2-bit: byte j bits [2i,2i+1]
//   = t_{4j+i}.  Both pad K with t = 1.  Bit-plane: ceil(K/8) bytes of the
//   nonzero plane, then ceil(K/8) bytes of the sign plane, bit k mod 8 of
//   byte k/8, zero past K.
// In the bit-plane format a sign bit without its nonzero bit, and a nonzero
// bit past K, are invalid.
#include "tern_internal.h"

namespace tern {

__device__ __forceinline__ int d3_encode(int V) { return (256 * V + 242) / 243; }

// Returns V for a valid D3 code y, else -1.
__device__ __forceinline__ int d3_decode(int y) {
    int V = (243 * y) >> 8;
    return (V <= 242 && d3_encode(V) == y) ? V : -1;
}

__device__ __forceinline__ int trit_digit(const int8_t *row, int64_t k, int K, int &bad) {
    if (k >= K) return 1;
    int t = row[k] + 1;
    if (t < 0 || t > 2) {
        ++bad;
        return 1;
    }
    return t;
}

// Position of bit i (0..7) of byte b of a DB row (b inside a word pair).
__device__ __forceinline__ int64_t db_position(int64_t b, int i) {
    return 32 * (b >> 3) + 4 * i + (b & 3);
}

// Digit t (0..2) from a nonzero and a sign bit; counts a sign without nonzero.
__device__ __forceinline__ int db_digit(int nz, int sg, int &bad) {
    if (sg && !nz) {
        ++bad;
        return 1;
    }
    return nz ? (sg ? 0 : 2) : 1;
}

__global__ void pack_kernel(int fmt, const int8_t *__restrict__ trits, int N, int K,
                            uint8_t *__restrict__ out, int64_t row_stride, int64_t used,
                            int32_t *d_invalid) {
    int64_t total = static_cast<int64_t>(N) * row_stride;
    int bad = 0;
    for (int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; idx < total;
         idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        int64_t n = idx / row_stride, b = idx % row_stride;
        uint8_t code = 0;
        if (b < used) {
            const int8_t *row = trits + n * K;
            int64_t wd = b >> 2;
            int j = static_cast<int>(b & 3);
            if (fmt == TERN_FMT_BASE3) {
                int V = 0;
                for (int i = 0; i < 5; ++i) V = 3 * V + trit_digit(row, 20 * wd + j + 4 * i, K, bad);
                code = static_cast<uint8_t>(d3_encode(V));
            } else if (fmt == TERN_FMT_2BIT) {
                int c = 0;
                for (int i = 0; i < 4; ++i) c |= trit_digit(row, 16 * wd + 4 * i + j, K, bad) << (2 * i);
                code = static_cast<uint8_t>(c);
            } else {
                const bool sign_word = (b & 4) != 0;
                int c = 0;
                for (int i = 0; i < 8; ++i) {
                    const int t = trit_digit(row, db_position(b, i), K, bad);
                    c |= (sign_word ? (t == 0) : (t != 1)) << i;
                }
                code = static_cast<uint8_t>(c);
            }
        }
        out[idx] = code;
    }
    if (bad && d_invalid) atomicAdd(d_invalid, bad);
}

__global__ void unpack_kernel(int fmt, const uint8_t *__restrict__ packed, int N, int K,
                              int64_t row_stride, int64_t used, int8_t *__restrict__ trits,
                              int32_t *d_invalid) {
    int64_t total = static_cast<int64_t>(N) * used;
    int bad = 0;
    for (int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; idx < total;
         idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        int64_t n = idx / used, b = idx % used;
        int code = packed[n * row_stride + b];
        int64_t wd = b >> 2;
        int j = static_cast<int>(b & 3);
        int8_t *row = trits + n * K;
        if (fmt == TERN_FMT_BITPLANE) {
            if (b & 4) continue;  // sign bytes are read with their nonzero byte
            const int sign = packed[n * row_stride + b + 4];
            for (int i = 0; i < 8; ++i) {
                const int nz = (code >> i) & 1;
                const int t = db_digit(nz, (sign >> i) & 1, bad);
                const int64_t k = db_position(b, i);
                if (k < K)
                    row[k] = static_cast<int8_t>(t - 1);
                else if (nz)
                    ++bad;
            }
        } else if (fmt == TERN_FMT_BASE3) {
            int V = d3_decode(code);
            if (V < 0) {
                ++bad;
                V = 121;  // all digits 1 (w = 0)
            }
            for (int i = 4; i >= 0; --i) {  // digit 4 is the least significant
                int t = V % 3;
                V /= 3;
                int64_t k = 20 * wd + j + 4 * i;
                if (k < K)
                    row[k] = static_cast<int8_t>(t - 1);
                else if (t != 1)
                    ++bad;
            }
        } else {
            for (int i = 0; i < 4; ++i) {
                int t = (code >> (2 * i)) & 3;
                if (t == 3) {
                    ++bad;
                    t = 1;
                }
                int64_t k = 16 * wd + 4 * i + j;
                if (k < K)
                    row[k] = static_cast<int8_t>(t - 1);
                else if (t != 1)
                    ++bad;
            }
        }
    }
    if (bad && d_invalid) atomicAdd(d_invalid, bad);
}

// Digit t (0..2) of canonical position k of a row; counts invalid codes and
// (for positions past K) padding digits other than 1.
__device__ __forceinline__ int canonical_digit(int fmt, const uint8_t *row, int64_t k, int K,
                                               int64_t cbytes, int &bad) {
    if (fmt == TERN_FMT_BITPLANE) {
        const int64_t P = cbytes / 2;
        if (k / 8 >= P) return 1;
        const int nz = (row[k / 8] >> (k % 8)) & 1, sg = (row[P + k / 8] >> (k % 8)) & 1;
        const int t = db_digit(nz, sg, bad);
        if (k >= K) {
            if (nz) ++bad;
            return 1;
        }
        return t;
    }
    int per = (fmt == TERN_FMT_BASE3) ? 5 : 4;
    int64_t byte = k / per;
    if (byte >= cbytes) return 1;  // beyond the canonical row: padding of the device layout
    int code = row[byte];
    int i = static_cast<int>(k % per);
    int t;
    if (fmt == TERN_FMT_BASE3) {
        if (code >= 243) {
            ++bad;
            return 1;
        }
        for (int s = 0; s < i; ++s) code /= 3;
        t = code % 3;
    } else {
        t = (code >> (2 * i)) & 3;
        if (t == 3) {
            ++bad;
            return 1;
        }
    }
    if (k >= K) {
        if (t != 1) ++bad;
        return 1;
    }
    return t;
}

__global__ void import_kernel(int fmt, const uint8_t *__restrict__ canon, int N, int K,
                              int64_t cbytes, uint8_t *__restrict__ out, int64_t row_stride,
                              int64_t used, int32_t *d_invalid) {
    int64_t total = static_cast<int64_t>(N) * row_stride;
    int bad = 0;
    for (int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; idx < total;
         idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        int64_t n = idx / row_stride, b = idx % row_stride;
        uint8_t code = 0;
        if (b < used) {
            const uint8_t *row = canon + n * cbytes;
            int64_t wd = b >> 2;
            int j = static_cast<int>(b & 3);
            if (fmt == TERN_FMT_BASE3) {
                int V = 0;
                for (int i = 0; i < 5; ++i)
                    V = 3 * V + canonical_digit(fmt, row, 20 * wd + j + 4 * i, K, cbytes, bad);
                code = static_cast<uint8_t>(d3_encode(V));
            } else if (fmt == TERN_FMT_BITPLANE) {
                // both words of a pair read the same positions: only the
                // nonzero word's reads count invalid bits
                const bool sign_word = (b & 4) != 0;
                int uncounted = 0;
                int c = 0;
                for (int i = 0; i < 8; ++i) {
                    const int t = canonical_digit(fmt, row, db_position(b, i), K, cbytes,
                                                  sign_word ? uncounted : bad);
                    c |= (sign_word ? (t == 0) : (t != 1)) << i;
                }
                code = static_cast<uint8_t>(c);
            } else {
                int c = 0;
                for (int i = 0; i < 4; ++i)
                    c |= canonical_digit(fmt, row, 16 * wd + 4 * i + j, K, cbytes, bad) << (2 * i);
                code = static_cast<uint8_t>(c);
            }
        }
        out[idx] = code;
    }
    if (bad && d_invalid) atomicAdd(d_invalid, bad);
}

// Digit t of position k < K of a device-layout row.
__device__ __forceinline__ int device_digit(int fmt, const uint8_t *row, int64_t k, int &bad) {
    if (fmt == TERN_FMT_BITPLANE) {
        const int64_t p = k / 32;
        const int r = static_cast<int>(k % 32), i = r >> 2, j = r & 3;
        return db_digit((row[8 * p + j] >> i) & 1, (row[8 * p + 4 + j] >> i) & 1, bad);
    }
    if (fmt == TERN_FMT_BASE3) {
        int64_t wd = k / 20;
        int r = static_cast<int>(k % 20);
        int j = r & 3, i = r >> 2;
        int V = d3_decode(row[4 * wd + j]);
        if (V < 0) {
            ++bad;
            return 1;
        }
        for (int s = i; s < 4; ++s) V /= 3;  // digit i has weight 3^(4-i)
        return V % 3;
    }
    int64_t wd = k / 16;
    int r = static_cast<int>(k % 16);
    int j = r & 3, i = r >> 2;
    int t = (row[4 * wd + j] >> (2 * i)) & 3;
    if (t == 3) {
        ++bad;
        return 1;
    }
    return t;
}

__global__ void export_kernel(int fmt, const uint8_t *__restrict__ packed, int N, int K,
                              int64_t row_stride, uint8_t *__restrict__ canon, int64_t cbytes,
                              int32_t *d_invalid) {
    int64_t total = static_cast<int64_t>(N) * cbytes;
    int per = (fmt == TERN_FMT_BASE3) ? 5 : 4;
    int bad = 0;
    for (int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; idx < total;
         idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        int64_t n = idx / cbytes, cb = idx % cbytes;
        const uint8_t *row = packed + n * row_stride;
        if (fmt == TERN_FMT_BITPLANE) {
            const int64_t P = cbytes / 2;
            const bool sign_plane = cb >= P;
            const int64_t k0 = 8 * (sign_plane ? cb - P : cb);
            int value = 0;
            for (int i = 0; i < 8; ++i) {
                const int64_t k = k0 + i;
                const int t = (k < K) ? device_digit(fmt, row, k, bad) : 1;
                value |= (sign_plane ? (t == 0) : (t != 1)) << i;
            }
            canon[idx] = static_cast<uint8_t>(value);
            continue;
        }
        int value = 0;
        for (int i = per - 1; i >= 0; --i) {
            int64_t k = cb * per + i;
            int t = (k < K) ? device_digit(fmt, row, k, bad) : 1;
            value = (fmt == TERN_FMT_BASE3) ? value * 3 + t : (value << 2) | t;
        }
        canon[idx] = static_cast<uint8_t>(value);
    }
    if (bad && d_invalid) atomicAdd(d_invalid, bad);
}

// Unit-major scales: unit u = rb * SB + sb holds 32 rows x gps scales.
__global__ void retile_scales_kernel(const uint16_t *__restrict__ sc, int N, int G, int SB, int gps,
                                     int64_t units, uint16_t *__restrict__ out) {
    const int64_t total = units * 32 * gps;
    for (int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; idx < total;
         idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t u = idx / (32 * gps);
        const int r = static_cast<int>((idx / gps) % 32);
        const int g = static_cast<int>(idx % gps);
        const int64_t rb = u / SB, sb = u % SB;
        const int64_t n = rb * 32 + r, gg = sb * gps + g;
        out[idx] = (n < N && gg < G) ? sc[n * G + gg] : static_cast<uint16_t>(0);
    }
}

static int grid_for(int64_t total) {
    int64_t blocks = (total + 255) / 256;
    if (blocks < 1) blocks = 1;
    if (blocks > 148 * 64) blocks = 148 * 64;
    return static_cast<int>(blocks);
}

cudaError_t launch_pack(int fmt, const int8_t *trits, int N, int K, void *out, int64_t row_stride,
                        int32_t *d_invalid, cudaStream_t s) {
    int64_t used = device_row_bytes(fmt, K);
    pack_kernel<<<grid_for(static_cast<int64_t>(N) * row_stride), 256, 0, s>>>(
        fmt, trits, N, K, static_cast<uint8_t *>(out), row_stride, used, d_invalid);
    return cudaGetLastError();
}

cudaError_t launch_unpack(int fmt, const void *packed, int N, int K, int64_t row_stride,
                          int8_t *trits, int32_t *d_invalid, cudaStream_t s) {
    int64_t used = device_row_bytes(fmt, K);
    unpack_kernel<<<grid_for(static_cast<int64_t>(N) * used), 256, 0, s>>>(
        fmt, static_cast<const uint8_t *>(packed), N, K, row_stride, used, trits, d_invalid);
    return cudaGetLastError();
}

cudaError_t launch_import(int fmt, const uint8_t *canon, int N, int K, void *out,
                          int64_t row_stride, int32_t *d_invalid, cudaStream_t s) {
    int64_t used = device_row_bytes(fmt, K);
    int64_t cbytes = canonical_row_bytes(fmt, K);
    import_kernel<<<grid_for(static_cast<int64_t>(N) * row_stride), 256, 0, s>>>(
        fmt, canon, N, K, cbytes, static_cast<uint8_t *>(out), row_stride, used, d_invalid);
    return cudaGetLastError();
}

cudaError_t launch_retile_scales(int fmt, const uint16_t *sc, int N, int K, uint16_t *out,
                                 cudaStream_t s) {
    const int G = static_cast<int>(ceil_div(K, 128));
    const int SB = static_cast<int>(ceil_div(device_row_bytes(fmt, K), 128));
    const int gps = (fmt == TERN_FMT_BASE3) ? 5 : 4;  // 512 positions a superblock otherwise
    const int64_t units = ceil_div(N, 32) * SB;
    retile_scales_kernel<<<grid_for(units * 32 * gps), 256, 0, s>>>(sc, N, G, SB, gps, units, out);
    return cudaGetLastError();
}

cudaError_t launch_export(int fmt, const void *packed, int N, int K, int64_t row_stride,
                          uint8_t *canon, int32_t *d_invalid, cudaStream_t s) {
    int64_t cbytes = canonical_row_bytes(fmt, K);
    export_kernel<<<grid_for(static_cast<int64_t>(N) * cbytes), 256, 0, s>>>(
        fmt, static_cast<const uint8_t *>(packed), N, K, row_stride, canon, cbytes, d_invalid);
    return cudaGetLastError();
}

}  // namespace tern

/*
 * tern_oracle.c -- plain CPU oracle for the ternary weight path.
 *
 * TEST INFRASTRUCTURE.  Only the tests, the smoke check and the CPU-baseline
 * leg of the benchmark may load this file's library.  It shares no code,
 * header, table or helper with the CUDA library; it is written from the
 * definitions below, slowly and plainly, so that a reader can check it
 * against them by eye.
 *
 * Sources (the pages this method is described on):
 *  [BONSAI]  "Ternary Bonsai 2 27B: 8GB 显卡硬塞 27B 三元模型，能跑，但我大概率
 *            不会真用" (171host.com), section "Decode 为什么只能算一般":
 *            base-3 unpack, restore -1/0/+1, read the scale, integer dot;
 *            gate/up + SwiGLU fused, Hadamard transform shared by gate and up;
 *            activations quantised per token (about 1.1 us per call).
 *  [4SAPI]   "三值权重 27B 压到 5.9GB｜本地部署成本账单重算" (blog.4sapi.com),
 *            section 三: weights in {-1,0,+1} with one FP16 scale per group;
 *            restore by adding/subtracting by sign, then multiply by the
 *            group scale.
 *  [PWWT1]   pwwt.cn/news/4940051, section 1.1: a weight is -1, 0 or +1, so
 *            the multiply becomes negate / zero / keep; activations go to
 *            4 or 8 bits.
 *  [PWWT2]   pwwt.cn/news/5175886, section 1.1: log2(3) ~ 1.585 bit of
 *            information per ternary weight; 2-bit storage in practice.
 *
 * Readings where the pages are silent (each also listed in the design notes):
 *  R1 trit <-> digit: digit t = w + 1 in {0,1,2}.
 *  R2 canonical base-3 byte: value = sum_{i=0..4} t_i * 3^i, t_i the weight
 *     at K index 5j+i (least significant digit first); rows contiguous along
 *     K, K padded to a multiple of 5 with digit 1 (w = 0).
 *  R3 invalid codes: base-3 bytes 243..255, 2-bit field value 3, and padding
 *     digits other than 1 are rejected (error 1).
 *  R4 canonical 2-bit: field t = w + 1 in bits [2i, 2i+1] of byte k/4,
 *     i = k mod 4; K padded to a multiple of 4 with t = 1.
 *  R5 scale groups: 128 consecutive K positions per output row, the last
 *     group partial when K mod 128 != 0.
 *  R6 activation quantisation (the pages give only "per token, int8"):
 *     fp32 arithmetic, amax = max |x^|, inv = 127/amax (correctly rounded),
 *     q = clamp(rint_half_even(x^ * inv), -127, 127), s_x = amax/127;
 *     amax == 0 gives s_x = 0, q = 0.
 *  R7 Hadamard (the pages name only "Hadamard"): Sylvester order, 128-point
 *     blocks along K, unnormalised radix-2 butterflies in fp32 in stage order
 *     h = 1, 2, ..., 64 with (a, b) -> (a + b, a - b); the orthonormal
 *     1/sqrt(128) is folded into s_x (s_x = fp32(fp32(amax/127) * fp32(1/sqrt(128)))).
 *  R8 SwiGLU: h = g * sigmoid(g) * u, sigmoid(z) = 1 / (1 + exp(-z)).
 *  R9 decode chain glue (the pages give no norm or attention detail): a
 *     weightless RMSNorm of the unrotated row folded into the scale only,
 *     s_x / sqrt(mean(x^2) + 1e-6), which leaves every int8 code unchanged.
 *  R11 bit-plane format (Bonsai page, "后面还有没有优化空间", first direction:
 *     split the weights into a "nonzero" and a "sign" bit plane, about 2 bits
 *     per weight, for a cheaper decode): n = (w != 0), s = (w < 0).
 *     Canonical row: ceil(K/8) bytes of the n plane, then ceil(K/8) bytes of
 *     the s plane, bit k mod 8 of byte k/8; bits past K are 0; an s bit set
 *     where n is 0 is invalid (error 1).
 *  R12 decode attention over a Q4_0 KV cache (Bonsai page, "先交代机器和配置":
 *     K and V cached as Q4_0, Flash Attention on; the passage before "PQ2 会不会
 *     快很多": the Q4 data is decoded inside attention).  Q4_0 is the block
 *     format of the llama.cpp family the pages run: blocks of 32 values along
 *     the head dimension, one fp16 scale d and 32 4-bit codes; with m the
 *     value of largest magnitude (first one on ties), d = m / -8,
 *     code = min(15, trunc(x / d + 8.5)) (0 when d = 0), value = (code - 8) d;
 *     codes j and j + 16 share byte j (low and high nibble).  Attention for
 *     one new token: query head h reads KV head h * Hkv / Hq (grouped
 *     query attention), s_t = (q . k_t) / sqrt(D) over the L cached tokens,
 *     out = sum_t softmax(s)_t v_t, in fp64 from the dequantised cache.  No
 *     rotary embedding or mask (the pages give none; this is the product the
 *     kernel computes).
 *  R10 ternarisation (pwwt.cn/news/5175886, section 1.2: per block, two
 *     thresholds -- values between them become 0, the two sides +1 / -1 --
 *     and a scale chosen to make the residual small; m.nxbn.cn/news/172464,
 *     section 1.2: threshold plus one scale per group; no calibration data
 *     here, so the residual is that of the weights themselves).  Per group of
 *     128 consecutive K positions of a row: the thresholds are -D and +D and
 *     the scale alpha is the one that minimises sum (w - alpha t)^2, i.e.
 *     keep the k largest |w| (ties: lower index first) for the k that
 *     maximises S_k^2 / k, S_k = their sum.  Arithmetic fixed in fp32 so
 *     that the integer decisions are reproducible: S_k is the fp32 sum of
 *     the kept |w| in index order, score = fp32(fp32(S_k * S_k) / k), the
 *     largest score wins and among equal scores the smallest k (k = 0,
 *     score 0, when nothing beats it); alpha = fp16(fp32(S_k / k)), rounded
 *     to nearest even.
 *
 * Device layouts (the "load-time retile into consumption order" suggested on
 * [BONSAI], section "后面还有没有优化空间"):
 *  D3 (base-3): a 4-byte word w of a row covers K in [20w, 20w+20).  Byte j
 *     (0..3) holds the five trits at K = 20w + j + 4i, i = 0..4, as the
 *     fixed-point code y = ceil(256 * V / 243), V = sum_i t_i * 3^(4-i)
 *     (digit i = 0 most significant).  Row bytes used: 4*ceil(K/20).
 *  D2 (2-bit): a 4-byte word w covers K in [16w, 16w+16).  Bits [2i, 2i+1]
 *     of byte j hold t for K = 16w + 4i + j.  Row bytes used: 4*ceil(K/16).
 *  DB (bit-plane): 4-byte words in pairs; pair p of a row covers K in
 *     [32p, 32p+32): word 2p is the n plane, word 2p+1 the s plane, and bit
 *     8j + i of each holds K = 32p + 4i + j (i = 0..7, j = 0..3).  Row bytes
 *     used: 8*ceil(K/32).
 *  D3, D2: positions past K hold t = 1; DB: positions past K hold n = s = 0
 *  (w = 0).  Bytes past the used row bytes up to the row stride are 0.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_EINVAL 1

/* ------------------------------------------------------------------ */
/* fp16 bits -> double (IEEE binary16: 1 sign, 5 exponent, 10 fraction) */
double oracle_half_to_double(uint16_t h) {
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int m = h & 0x3ff;
    double v;
    if (e == 0)
        v = ldexp((double)m, -24);               /* subnormal: m * 2^-24 */
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + m), e - 25);   /* (1 + m/1024) * 2^(e-15) */
    return sign ? -v : v;
}

/* ------------------------------------------------------------------ */
/* Canonical base-3: 5 trits per byte, least significant digit first (R2). */
int64_t oracle_base3_row_bytes(int64_t K) { return (K + 4) / 5; }

int oracle_pack_base3(const int8_t *w, int64_t N, int64_t K, uint8_t *out) {
    int64_t B = oracle_base3_row_bytes(K);
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t j = 0; j < B; ++j) {
            int value = 0, power = 1;
            for (int i = 0; i < 5; ++i) {
                int64_t k = 5 * j + i;
                int t = 1;
                if (k < K) {
                    t = w[n * K + k] + 1;
                    if (t < 0 || t > 2) return ORACLE_EINVAL;
                }
                value += t * power;
                power *= 3;
            }
            out[n * B + j] = (uint8_t)value;
        }
    }
    return ORACLE_OK;
}

int oracle_unpack_base3(const uint8_t *b, int64_t N, int64_t K, int8_t *w) {
    int64_t B = oracle_base3_row_bytes(K);
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t j = 0; j < B; ++j) {
            int value = b[n * B + j];
            if (value >= 243) return ORACLE_EINVAL;
            for (int i = 0; i < 5; ++i) {
                int t = value % 3;
                value /= 3;
                int64_t k = 5 * j + i;
                if (k < K)
                    w[n * K + k] = (int8_t)(t - 1);
                else if (t != 1)
                    return ORACLE_EINVAL;
            }
        }
    }
    return ORACLE_OK;
}

/* Canonical 2-bit: 4 trits per byte, field i in bits [2i, 2i+1] (R4). */
int64_t oracle_2bit_row_bytes(int64_t K) { return (K + 3) / 4; }

int oracle_pack_2bit(const int8_t *w, int64_t N, int64_t K, uint8_t *out) {
    int64_t B = oracle_2bit_row_bytes(K);
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t j = 0; j < B; ++j) {
            int byte = 0;
            for (int i = 0; i < 4; ++i) {
                int64_t k = 4 * j + i;
                int t = 1;
                if (k < K) {
                    t = w[n * K + k] + 1;
                    if (t < 0 || t > 2) return ORACLE_EINVAL;
                }
                byte |= t << (2 * i);
            }
            out[n * B + j] = (uint8_t)byte;
        }
    }
    return ORACLE_OK;
}

int oracle_unpack_2bit(const uint8_t *b, int64_t N, int64_t K, int8_t *w) {
    int64_t B = oracle_2bit_row_bytes(K);
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t j = 0; j < B; ++j) {
            int byte = b[n * B + j];
            for (int i = 0; i < 4; ++i) {
                int t = (byte >> (2 * i)) & 3;
                if (t == 3) return ORACLE_EINVAL;
                int64_t k = 4 * j + i;
                if (k < K)
                    w[n * K + k] = (int8_t)(t - 1);
                else if (t != 1)
                    return ORACLE_EINVAL;
            }
        }
    }
    return ORACLE_OK;
}

/* Canonical bit-plane: the n plane then the s plane, 1 bit per weight (R11). */
int64_t oracle_bitplane_row_bytes(int64_t K) { return 2 * ((K + 7) / 8); }

int oracle_pack_bitplane(const int8_t *w, int64_t N, int64_t K, uint8_t *out) {
    int64_t P = (K + 7) / 8, B = 2 * P;
    for (int64_t n = 0; n < N; ++n) {
        memset(out + n * B, 0, (size_t)B);
        for (int64_t k = 0; k < K; ++k) {
            int v = w[n * K + k];
            if (v < -1 || v > 1) return ORACLE_EINVAL;
            if (v != 0) out[n * B + k / 8] |= (uint8_t)(1u << (k % 8));
            if (v < 0) out[n * B + P + k / 8] |= (uint8_t)(1u << (k % 8));
        }
    }
    return ORACLE_OK;
}

int oracle_unpack_bitplane(const uint8_t *b, int64_t N, int64_t K, int8_t *w) {
    int64_t P = (K + 7) / 8, B = 2 * P;
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t k = 0; k < 8 * P; ++k) {
            int nz = (b[n * B + k / 8] >> (k % 8)) & 1;
            int sg = (b[n * B + P + k / 8] >> (k % 8)) & 1;
            if (sg && !nz) return ORACLE_EINVAL;
            if (k < K)
                w[n * K + k] = (int8_t)(nz ? (sg ? -1 : 1) : 0);
            else if (nz)
                return ORACLE_EINVAL;
        }
    }
    return ORACLE_OK;
}

/* ------------------------------------------------------------------ */
/* Device layouts D3 / D2 / DB (see the header comment). fmt 0 = D3,
 * 1 = D2, 2 = DB.                                                         */
int64_t oracle_device_row_bytes(int fmt, int64_t K) {
    if (fmt == 0) return 4 * ((K + 19) / 20);
    if (fmt == 1) return 4 * ((K + 15) / 16);
    if (fmt == 2) return 8 * ((K + 31) / 32);
    return -1;
}

/* The D3 fixed-point code of a 5-digit value V (0..242): ceil(256 V / 243). */
int oracle_d3_encode_value(int V) { return (256 * V + 242) / 243; }

/* Inverse: returns V, or -1 when y is not the code of any V.  The digits of
 * V are read most significant first, digit i = floor(y * 3^(i+1) / 256) mod 3;
 * here V itself is recovered as floor(243 y / 256) and checked by re-encoding. */
int oracle_d3_decode_value(int y) {
    int V = (243 * y) / 256;
    if (V > 242 || oracle_d3_encode_value(V) != y) return -1;
    return V;
}

int oracle_pack_device(int fmt, const int8_t *w, int64_t N, int64_t K,
                       int64_t row_stride, uint8_t *out) {
    int64_t used = oracle_device_row_bytes(fmt, K);
    if (used < 0 || row_stride < used) return ORACLE_EINVAL;
    for (int64_t n = 0; n < N; ++n) {
        uint8_t *row = out + n * row_stride;
        memset(row, 0, (size_t)row_stride);
        if (fmt == 2) {
            for (int64_t k = 0; k < K; ++k) {
                int v = w[n * K + k];
                if (v < -1 || v > 1) return ORACLE_EINVAL;
                int64_t p = k / 32;
                int i = (int)((k % 32) / 4), j = (int)(k % 4);
                int bit = 8 * j + i;
                if (v != 0) row[8 * p + bit / 8] |= (uint8_t)(1u << (bit % 8));
                if (v < 0) row[8 * p + 4 + bit / 8] |= (uint8_t)(1u << (bit % 8));
            }
            continue;
        }
        for (int64_t wd = 0; wd < used / 4; ++wd) {
            for (int j = 0; j < 4; ++j) {
                int code = 0;
                if (fmt == 0) {
                    int V = 0;
                    for (int i = 0; i < 5; ++i) {
                        int64_t k = 20 * wd + j + 4 * i;
                        int t = 1;
                        if (k < K) {
                            t = w[n * K + k] + 1;
                            if (t < 0 || t > 2) return ORACLE_EINVAL;
                        }
                        V = 3 * V + t; /* digit i = 0 ends most significant */
                    }
                    code = oracle_d3_encode_value(V);
                } else {
                    for (int i = 0; i < 4; ++i) {
                        int64_t k = 16 * wd + 4 * i + j;
                        int t = 1;
                        if (k < K) {
                            t = w[n * K + k] + 1;
                            if (t < 0 || t > 2) return ORACLE_EINVAL;
                        }
                        code |= t << (2 * i);
                    }
                }
                row[4 * wd + j] = (uint8_t)code;
            }
        }
    }
    return ORACLE_OK;
}

int oracle_unpack_device(int fmt, const uint8_t *b, int64_t N, int64_t K,
                         int64_t row_stride, int8_t *w) {
    int64_t used = oracle_device_row_bytes(fmt, K);
    if (used < 0 || row_stride < used) return ORACLE_EINVAL;
    for (int64_t n = 0; n < N; ++n) {
        const uint8_t *row = b + n * row_stride;
        if (fmt == 2) {
            for (int64_t k = 0; k < used * 4; ++k) { /* 32 positions per 8 bytes */
                int64_t p = k / 32;
                int i = (int)((k % 32) / 4), j = (int)(k % 4);
                int bit = 8 * j + i;
                int nz = (row[8 * p + bit / 8] >> (bit % 8)) & 1;
                int sg = (row[8 * p + 4 + bit / 8] >> (bit % 8)) & 1;
                if (sg && !nz) return ORACLE_EINVAL;
                if (k < K)
                    w[n * K + k] = (int8_t)(nz ? (sg ? -1 : 1) : 0);
                else if (nz)
                    return ORACLE_EINVAL;
            }
            continue;
        }
        for (int64_t wd = 0; wd < used / 4; ++wd) {
            for (int j = 0; j < 4; ++j) {
                int code = row[4 * wd + j];
                if (fmt == 0) {
                    int V = oracle_d3_decode_value(code);
                    if (V < 0) return ORACLE_EINVAL;
                    int digits[5];
                    for (int i = 4; i >= 0; --i) { /* least significant = digit 4 */
                        digits[i] = V % 3;
                        V /= 3;
                    }
                    for (int i = 0; i < 5; ++i) {
                        int64_t k = 20 * wd + j + 4 * i;
                        if (k < K)
                            w[n * K + k] = (int8_t)(digits[i] - 1);
                        else if (digits[i] != 1)
                            return ORACLE_EINVAL;
                    }
                } else {
                    for (int i = 0; i < 4; ++i) {
                        int t = (code >> (2 * i)) & 3;
                        if (t == 3) return ORACLE_EINVAL;
                        int64_t k = 16 * wd + 4 * i + j;
                        if (k < K)
                            w[n * K + k] = (int8_t)(t - 1);
                        else if (t != 1)
                            return ORACLE_EINVAL;
                    }
                }
            }
        }
    }
    return ORACLE_OK;
}

/* ------------------------------------------------------------------ */
/* Activation quantisation, fp32 as the kernel computes it (R6, R7).      */
/* 1/sqrt(128) rounded to fp32. */
static const float INV_SQRT128_F = 0.0883883476483184405501f;

void oracle_fwht128_f32(float *v) {
    for (int h = 1; h < 128; h <<= 1)
        for (int i = 0; i < 128; i += 2 * h)
            for (int j = i; j < i + h; ++j) {
                float a = v[j], b = v[j + h];
                v[j] = a + b;
                v[j + h] = a - b;
            }
}

void oracle_fwht128_f64(double *v) {
    for (int h = 1; h < 128; h <<= 1)
        for (int i = 0; i < 128; i += 2 * h)
            for (int j = i; j < i + h; ++j) {
                double a = v[j], b = v[j + h];
                v[j] = a + b;
                v[j + h] = a - b;
            }
}

/* x: fp32 [M][K] (fp16 inputs are passed as their exact fp32 values).
 * q: int8 [M][K]; s_x: fp32 [M]. */
int oracle_act_quant(const float *x, int64_t M, int64_t K, int fwht_block,
                     int rmsnorm, int8_t *q, float *s_x) {
    if (fwht_block != 0 && fwht_block != 128) return ORACLE_EINVAL;
    if (fwht_block == 128 && K % 128 != 0) return ORACLE_EINVAL;
    float *v = (float *)malloc((size_t)(K > 0 ? K : 1) * sizeof(float));
    if (!v) return ORACLE_EINVAL;
    for (int64_t m = 0; m < M; ++m) {
        memcpy(v, x + m * K, (size_t)K * sizeof(float));
        double inv_rms = 1.0;
        if (rmsnorm) {
            double ss = 0.0;
            for (int64_t k = 0; k < K; ++k) ss += (double)v[k] * (double)v[k];
            inv_rms = 1.0 / sqrt(ss / (double)K + 1e-6);
        }
        if (fwht_block == 128)
            for (int64_t b = 0; b < K / 128; ++b) oracle_fwht128_f32(v + 128 * b);
        float amax = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            float a = fabsf(v[k]);
            if (a > amax) amax = a;
        }
        if (amax == 0.0f) {
            s_x[m] = 0.0f;
            for (int64_t k = 0; k < K; ++k) q[m * K + k] = 0;
            continue;
        }
        volatile float inv = 127.0f / amax;
        for (int64_t k = 0; k < K; ++k) {
            volatile float t = v[k] * inv;
            float r = rintf(t); /* default rounding mode: nearest, ties to even */
            if (r > 127.0f) r = 127.0f;
            if (r < -127.0f) r = -127.0f;
            q[m * K + k] = (int8_t)r;
        }
        volatile float s = amax / 127.0f;
        if (fwht_block == 128) s = s * INV_SQRT128_F;
        s_x[m] = rmsnorm ? (float)((double)s * inv_rms) : s;
    }
    free(v);
    return ORACLE_OK;
}

/* ------------------------------------------------------------------ */
/* Integer group partials: P[m][n][g] = sum_{k in group g} w[n][k] q[m][k]. */
int64_t oracle_groups(int64_t K, int64_t group) { return (K + group - 1) / group; }

int oracle_group_partials(const int8_t *w, int64_t N, int64_t K, int64_t group,
                          const int8_t *q, int64_t M, int64_t *P) {
    if (group <= 0) return ORACLE_EINVAL;
    int64_t G = oracle_groups(K, group);
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n)
            for (int64_t g = 0; g < G; ++g) {
                int64_t acc = 0;
                int64_t k1 = (g + 1) * group < K ? (g + 1) * group : K;
                for (int64_t k = g * group; k < k1; ++k)
                    acc += (int64_t)w[n * K + k] * (int64_t)q[m * K + k];
                P[(m * N + n) * G + g] = acc;
            }
    return ORACLE_OK;
}

/* y[m][n] = s_x[m] * sum_g s_w[n][g] * P[m][n][g], in fp64 ([4SAPI] §三:
 * add/subtract by sign, then multiply by the group scale).  Output rows are
 * independent and are spread over threads when OpenMP is on. */
int oracle_gemv(const int8_t *w, const uint16_t *scales, int64_t N, int64_t K,
                int64_t group, const int8_t *q, const float *s_x, int64_t M,
                double *y) {
    if (group <= 0) return ORACLE_EINVAL;
    int64_t G = oracle_groups(K, group);
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t m = 0; m < M; ++m) {
            double acc = 0.0;
            for (int64_t g = 0; g < G; ++g) {
                int64_t P = 0;
                int64_t k1 = (g + 1) * group < K ? (g + 1) * group : K;
                for (int64_t k = g * group; k < k1; ++k)
                    P += (int64_t)w[n * K + k] * (int64_t)q[m * K + k];
                acc += oracle_half_to_double(scales[n * G + g]) * (double)P;
            }
            y[m * N + n] = (double)s_x[m] * acc;
        }
    }
    return ORACLE_OK;
}

/* SwiGLU of [BONSAI]: h = g * sigmoid(g) * u (R8). */
void oracle_swiglu(const double *g, const double *u, int64_t n, double *h) {
    for (int64_t i = 0; i < n; ++i) {
        double sig = 1.0 / (1.0 + exp(-g[i]));
        h[i] = g[i] * sig * u[i];
    }
}

/* Fused gate/up + SwiGLU: both projections read the same quantised input. */
int oracle_gateup_swiglu(const int8_t *wg, const uint16_t *sg, const int8_t *wu,
                         const uint16_t *su, int64_t N, int64_t K, int64_t group,
                         const int8_t *q, const float *s_x, int64_t M, double *h) {
    double *g = (double *)malloc((size_t)(M * N > 0 ? M * N : 1) * sizeof(double));
    double *u = (double *)malloc((size_t)(M * N > 0 ? M * N : 1) * sizeof(double));
    if (!g || !u) { free(g); free(u); return ORACLE_EINVAL; }
    int rc = oracle_gemv(wg, sg, N, K, group, q, s_x, M, g);
    if (rc == ORACLE_OK) rc = oracle_gemv(wu, su, N, K, group, q, s_x, M, u);
    if (rc == ORACLE_OK) oracle_swiglu(g, u, M * N, h);
    free(g);
    free(u);
    return rc;
}

/* ------------------------------------------------------------------ */
/* fp32 -> IEEE binary16 bits, round to nearest, ties to even, written from
 * the format's definition: 1 sign bit, 5 exponent bits (bias 15), 10
 * fraction bits; subnormals below 2^-14; overflow to infinity.           */
uint16_t oracle_float_to_half(float f) {
    uint32_t x;
    memcpy(&x, &f, 4);
    uint16_t sign = (uint16_t)((x >> 16) & 0x8000u);
    uint32_t e = (x >> 23) & 0xffu;
    uint32_t m = x & 0x7fffffu;
    if (e == 0xffu) return (uint16_t)(sign | 0x7c00u | (m ? 0x200u : 0u)); /* inf / nan */
    double a = fabs((double)f);                        /* exact */
    if (a == 0.0) return sign;
    /* value = a = q * 2^E with the fp16 quantum of a's binade */
    int ex;
    frexp(a, &ex);                                     /* a = f * 2^ex, f in [0.5, 1) */
    int E = ex - 1;                                    /* a in [2^E, 2^(E+1)) */
    if (E < -14) E = -14;                              /* subnormal range: quantum 2^-24 */
    double quantum = ldexp(1.0, E - 10);
    double qv = a / quantum;                           /* exact (power-of-two scaling) */
    double r = floor(qv);
    double rem = qv - r;
    if (rem > 0.5 || (rem == 0.5 && fmod(r, 2.0) != 0.0)) r += 1.0;
    double v = r * quantum;                            /* rounded magnitude */
    if (v >= 65520.0 || v > 65504.0) return (uint16_t)(sign | 0x7c00u);
    /* encode v */
    if (v < ldexp(1.0, -14)) return (uint16_t)(sign | (uint16_t)(v / ldexp(1.0, -24)));
    frexp(v, &ex);
    E = ex - 1;
    uint32_t frac = (uint32_t)(v / ldexp(1.0, E - 10)) - 1024u;
    return (uint16_t)(sign | (uint16_t)((E + 15) << 10) | (uint16_t)frac);
}

/* Ternarisation of one matrix (R10).  w: fp32 [N][K] (finite), row stride
 * ldw; t: int8 [N][K] in {-1,0,+1}; scales: fp16 bits [N][ceil(K/group)]. */
int oracle_ternarize(const float *w, int64_t N, int64_t K, int64_t ldw, int64_t group,
                     int8_t *t, uint16_t *scales) {
    if (group <= 0 || ldw < K) return ORACLE_EINVAL;
    int64_t G = oracle_groups(K, group);
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t g = 0; g < G; ++g) {
            int64_t k0 = g * group, k1 = (g + 1) * group < K ? (g + 1) * group : K;
            const float *v = w + n * ldw;
            /* candidate j keeps every i ranked at or above j: |w_i| > |w_j|,
             * or |w_i| == |w_j| with i <= j; it keeps cnt(j) = rank(j) + 1 */
            int64_t best_cnt = 0;
            float best_score = 0.0f, best_sum = 0.0f;
            for (int64_t j = k0; j < k1; ++j) {
                float aj = fabsf(v[j]);
                volatile float sum = 0.0f;
                int64_t cnt = 0;
                for (int64_t i = k0; i < k1; ++i) {
                    float ai = fabsf(v[i]);
                    if (ai > aj || (ai == aj && i <= j)) {
                        sum = sum + ai;
                        ++cnt;
                    }
                }
                volatile float sq = sum * sum;
                volatile float score = sq / (float)cnt;
                if (score > best_score || (score == best_score && cnt < best_cnt)) {
                    best_score = score;
                    best_cnt = cnt;
                    best_sum = sum;
                }
            }
            /* keep the best_cnt largest |w| (same rank order) */
            for (int64_t i = k0; i < k1; ++i) {
                int64_t rank = 0;
                float ai = fabsf(v[i]);
                for (int64_t j = k0; j < k1; ++j) {
                    float aj = fabsf(v[j]);
                    if (aj > ai || (aj == ai && j < i)) ++rank;
                }
                int8_t s = v[i] > 0.0f ? 1 : (v[i] < 0.0f ? -1 : 0);
                t[n * K + i] = rank < best_cnt ? s : 0;
            }
            volatile float alpha = best_cnt ? best_sum / (float)best_cnt : 0.0f;
            scales[n * G + g] = oracle_float_to_half(alpha);
        }
    }
    return ORACLE_OK;
}

/* ------------------------------------------------------------------ */
/* Q4_0 blocks (R12).  x: n floats (n a multiple of 32); d: n/32 fp16
 * scale bits; qs: 16 bytes per block.                                   */
int oracle_q4_0_quantize(const float *x, int64_t n, uint16_t *d, uint8_t *qs) {
    if (n % 32 != 0) return ORACLE_EINVAL;
    for (int64_t b = 0; b < n / 32; ++b) {
        const float *v = x + 32 * b;
        float amax = 0.0f, m = 0.0f;
        for (int j = 0; j < 32; ++j)
            if (fabsf(v[j]) > amax) {
                amax = fabsf(v[j]);
                m = v[j];
            }
        volatile float dd = m / -8.0f;
        volatile float id = dd != 0.0f ? 1.0f / dd : 0.0f;
        d[b] = oracle_float_to_half(dd);
        for (int j = 0; j < 16; ++j) {
            int c[2];
            for (int h = 0; h < 2; ++h) {
                volatile float t = v[j + 16 * h] * id;
                volatile float u = t + 8.5f;
                int code = (int)u; /* truncation toward zero; u >= 0.5 */
                c[h] = code > 15 ? 15 : code;
            }
            qs[16 * b + j] = (uint8_t)(c[0] | (c[1] << 4));
        }
    }
    return ORACLE_OK;
}

void oracle_q4_0_dequantize(const uint16_t *d, const uint8_t *qs, int64_t n, double *out) {
    for (int64_t b = 0; b < n / 32; ++b) {
        double s = oracle_half_to_double(d[b]);
        for (int j = 0; j < 16; ++j) {
            out[32 * b + j] = ((qs[16 * b + j] & 15) - 8) * s;
            out[32 * b + j + 16] = ((qs[16 * b + j] >> 4) - 8) * s;
        }
    }
}

/* Decode attention (R12).  q: fp32 [Hq][D]; the cache of KV head g holds L
 * tokens, token t's K at kd/kq block (g * L + t) * (D/32) .. (and V alike);
 * out: fp64 [Hq][D].                                                    */
int oracle_attention_decode(const float *q, const uint16_t *kd, const uint8_t *kq,
                            const uint16_t *vd, const uint8_t *vq, int64_t L, int64_t Hkv,
                            int64_t Hq, int64_t D, double *out) {
    if (D % 32 != 0 || Hkv < 1 || Hq % Hkv != 0 || L < 1) return ORACLE_EINVAL;
    int64_t nb = D / 32;
    double *k = (double *)malloc((size_t)D * sizeof(double));
    double *v = (double *)malloc((size_t)D * sizeof(double));
    double *s = (double *)malloc((size_t)L * sizeof(double));
    if (!k || !v || !s) { free(k); free(v); free(s); return ORACLE_EINVAL; }
    for (int64_t h = 0; h < Hq; ++h) {
        int64_t g = h * Hkv / Hq;
        double smax = -INFINITY;
        for (int64_t t = 0; t < L; ++t) {
            int64_t blk = (g * L + t) * nb;
            oracle_q4_0_dequantize(kd + blk, kq + 16 * blk, D, k);
            double dot = 0.0;
            for (int64_t i = 0; i < D; ++i) dot += (double)q[h * D + i] * k[i];
            s[t] = dot / sqrt((double)D);
            if (s[t] > smax) smax = s[t];
        }
        double z = 0.0;
        for (int64_t i = 0; i < D; ++i) out[h * D + i] = 0.0;
        for (int64_t t = 0; t < L; ++t) {
            double p = exp(s[t] - smax);
            z += p;
            int64_t blk = (g * L + t) * nb;
            oracle_q4_0_dequantize(vd + blk, vq + 16 * blk, D, v);
            for (int64_t i = 0; i < D; ++i) out[h * D + i] += p * v[i];
        }
        for (int64_t i = 0; i < D; ++i) out[h * D + i] /= z;
    }
    free(k);
    free(v);
    free(s);
    return ORACLE_OK;
}

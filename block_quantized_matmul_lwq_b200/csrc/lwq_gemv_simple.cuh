// Simple GEMV for the shapes the tensor-core paths do not take: K not a
// multiple of 256 (only Q8_0 and Q4_0 allow that), and Q6_K or Q2_K matrices
// that are not a whole number of 16-byte units (N * row bytes; their row
// slots need it), at any M.  One warp per
// weight row; lanes stride over 32-weight units, decode them with byte loads
// and accumulate in fp32 for up to 16 activation rows; a warp shuffle
// reduction finishes each output.  Correct for every valid shape, not tuned.
#pragma once

#include "lwq_gemv.cuh"

namespace lwq {

template <int XT>
__device__ __forceinline__ float load_x1(const void *x, long idx) {
    if constexpr (XT == X_F32)
        return static_cast<const float *>(x)[idx];
    else if constexpr (XT == X_F16)
        return __half2float(static_cast<const __half *>(x)[idx]);
    else
        return bf16_bits_to_float(static_cast<const uint16_t *>(x)[idx]);
}

__device__ __forceinline__ uint32_t ld_u16(const uint8_t *p) { return (uint32_t)p[0] | ((uint32_t)p[1] << 8); }

// Decode 32 weights (unit u of the row) into w[32], in element order.
template <int FMT>
__device__ __forceinline__ void decode_unit(const uint8_t *row, int u, float (&w)[32]) {
    if constexpr (FMT == F_Q8_0) {
        const uint8_t *b = row + (size_t)u * 34;
        const float d = f16_bits_to_float(ld_u16(b));
#pragma unroll
        for (int i = 0; i < 32; ++i) w[i] = d * (float)(int8_t)b[2 + i];
    } else if constexpr (FMT == F_Q4_0) {
        const uint8_t *b = row + (size_t)u * 18;
        const float d = f16_bits_to_float(ld_u16(b));
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const int v = b[2 + i];
            w[i] = d * (float)((v & 15) - 8);
            w[i + 16] = d * (float)((v >> 4) - 8);
        }
    } else if constexpr (FMT == F_Q6_K) {
        // unit u: elements 32j .. 32j+31 of superblock u/8 (j = u%8 = 4n + g)
        const uint8_t *b = row + (size_t)(u >> 3) * 210;
        const int j = u & 7, n = j >> 2, g = j & 3;
        const float d = f16_bits_to_float(ld_u16(b + 208));
        const uint8_t *ql = b + 64 * n + 32 * (g & 1), *qh = b + 128 + 32 * n;
        const int8_t *sc = reinterpret_cast<const int8_t *>(b + 192);
        const float s0 = d * (float)sc[2 * j], s1 = d * (float)sc[2 * j + 1];   // exact in fp32
#pragma unroll
        for (int l = 0; l < 32; ++l) {
            const int q = ((ql[l] >> (4 * (g >> 1))) & 15) | (((qh[l] >> (2 * g)) & 3) << 4);
            w[l] = (l < 16 ? s0 : s1) * (float)(q - 32);                          // exact in fp32
        }
    } else if constexpr (FMT == F_Q5_K) {
        const uint8_t *b = row + (size_t)(u >> 3) * 176;
        const int j = u & 7, g = j >> 1, h = j & 1;   // sub-block j
        const float d = f16_bits_to_float(ld_u16(b));
        const float dmin = f16_bits_to_float(ld_u16(b + 2));
        const uint8_t *s = b + 4;
        int sc, m;
        if (j < 4) {
            sc = s[j] & 63;
            m = s[j + 4] & 63;
        } else {
            sc = (s[j + 4] & 15) | ((s[j - 4] >> 6) << 4);
            m = (s[j + 4] >> 4) | ((s[j] >> 6) << 4);
        }
        const float ds = d * (float)sc, dm = dmin * (float)m;  // both exact in fp32
        const uint8_t *qh = b + 16, *qs = b + 48 + 32 * g;
#pragma unroll
        for (int l = 0; l < 32; ++l)
            w[l] = fmaf(ds, (float)(((qs[l] >> (4 * h)) & 15) | (((qh[l] >> (2 * g + h)) & 1) << 4)), -dm);
    } else if constexpr (FMT == F_Q2_K) {
        // unit u: elements 32j .. 32j+31 of superblock u/8 (j = 4n + field)
        const uint8_t *b = row + (size_t)(u >> 3) * 84;
        const int j = u & 7, n = j >> 2, f = j & 3;
        const float d = f16_bits_to_float(ld_u16(b + 80));
        const float dmin = f16_bits_to_float(ld_u16(b + 82));
        const uint8_t *qs = b + 16 + 32 * n;
        const int s0 = b[2 * j], s1 = b[2 * j + 1];
        const float ds0 = d * (float)(s0 & 15), dm0 = dmin * (float)(s0 >> 4);   // exact in fp32
        const float ds1 = d * (float)(s1 & 15), dm1 = dmin * (float)(s1 >> 4);
#pragma unroll
        for (int l = 0; l < 32; ++l) {
            const float q = (float)((qs[l] >> (2 * f)) & 3);
            w[l] = l < 16 ? fmaf(ds0, q, -dm0) : fmaf(ds1, q, -dm1);
        }
    } else {
        const uint8_t *b = row + (size_t)(u >> 3) * 144;
        const int j = u & 7;  // sub-block
        const float d = f16_bits_to_float(ld_u16(b));
        const float dmin = f16_bits_to_float(ld_u16(b + 2));
        const uint8_t *s = b + 4;
        int sc, m;
        if (j < 4) {
            sc = s[j] & 63;
            m = s[j + 4] & 63;
        } else {
            sc = (s[j + 4] & 15) | ((s[j - 4] >> 6) << 4);
            m = (s[j + 4] >> 4) | ((s[j] >> 6) << 4);
        }
        const float ds = d * (float)sc, dm = dmin * (float)m;  // both exact in fp32
        const uint8_t *q = b + 16 + 32 * (j >> 1);
        const int sh = (j & 1) * 4;
#pragma unroll
        for (int l = 0; l < 32; ++l) w[l] = fmaf(ds, (float)((q[l] >> sh) & 15), -dm);
    }
}

template <int FMT, int XT>
__global__ void __launch_bounds__(256) gemv_simple_kernel(const uint8_t *__restrict__ Wq, const void *__restrict__ x,
                                                          float *__restrict__ y, int M, int N, int K, long rb) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int row = blockIdx.x * (blockDim.x >> 5) + warp;
    if (row >= N) return;
    const uint8_t *wr = Wq + (size_t)row * rb;
    float acc[16];
#pragma unroll
    for (int m = 0; m < 16; ++m) acc[m] = 0.f;
    const int units = K / 32;
    for (int u = lane; u < units; u += 32) {
        float w[32];
        decode_unit<FMT>(wr, u, w);
        const long k0 = (long)u * 32;
#pragma unroll
        for (int m = 0; m < 16; ++m) {
            if (m < M) {
                float s = 0.f;
#pragma unroll
                for (int i = 0; i < 32; ++i) s = fmaf(w[i], load_x1<XT>(x, (long)m * K + k0 + i), s);
                acc[m] += s;
            }
        }
    }
#pragma unroll
    for (int m = 0; m < 16; ++m) {
        if (m < M) {
            float v = acc[m];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
            if (lane == 0) y[(size_t)m * N + row] = v;
        }
    }
}

}  // namespace lwq

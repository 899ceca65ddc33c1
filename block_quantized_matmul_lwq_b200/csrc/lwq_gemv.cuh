// Decode GEMV (M <= 16): y[M,N] = x[M,K] . dequant(Wq)^T.
//
// Design (sm_100a):
//  * A persistent grid.  CTA (split s, row group r) owns a fixed slice of K
//    (split-K factor S) and walks the row tiles r, r+G, r+2G, ... (16 weight
//    rows per tile).
//  * One producer warp stages, per row tile, one [16 rows][256 weights]
//    packed box per compute warp with 2-D TMA loads into a ring of shared
//    memory stages (mbarrier full/empty pairs).
//  * Each compute warp owns one 256-weight "chunk" of K for the whole kernel
//    and keeps the activations of that chunk in registers, already laid out
//    as tensor-core B fragments.  Per row tile it decodes the packed bytes in
//    registers straight into A fragments (nibbles -> 16-bit values with
//    exponent-bias tricks, no conversion instructions) and issues
//    mma.sync m16n8k16 with the weight rows as the MMA's M dimension and the
//    up-to-16 activation rows as its N dimension.  Block scales are applied
//    to the fp32 MMA results (Q4_0, Q8_0) or folded exactly into the fp16
//    A values (Q4_K sub-block scales, with the mins added by one extra MMA).
//  * A reducer warp sums the compute warps' partials in a fixed order and
//    writes y, or, with split-K, fp32 partials to the workspace; the last
//    split to finish a row tile (per-tile arrival counter) adds the splits
//    in order and writes y.  Results are bitwise deterministic.
//
// This is the matrix-vector half of the co-designed dequantization in
// "Resumo Tecnico: Llamas na Web", "3. Design de Shader Consciente de
// Quantizacao" (decode directly in registers), with tensor cores and
// asynchronous memory loads (the native advantages named in its "Desempenho
// Nativo vs. Navegador" result).
#pragma once

#include "lwq_ptx.cuh"

namespace lwq {

enum { F_Q8_0 = 1, F_Q4_0 = 2, F_Q4_K = 3 };
enum { X_F32 = 0, X_F16 = 1, X_BF16 = 2 };

constexpr int GEMV_ROWS = 16;      // weight rows per tile (the MMA's M)
constexpr int CHUNK = 256;         // weights of K per compute warp

template <int FMT>
struct FmtInfo;
template <>
struct FmtInfo<F_Q8_0> { static constexpr int chunk_bytes = 272; };
template <>
struct FmtInfo<F_Q4_0> { static constexpr int chunk_bytes = 144; };
template <>
struct FmtInfo<F_Q4_K> { static constexpr int chunk_bytes = 144; };

struct GemvArgs {
    const void *x;
    float *y;
    float *partial;       // [S][M][N] fp32 (split-K only)
    unsigned *counters;   // [row_tiles] (split-K only), zero between calls
    int M, N, K;
    int nchunks;          // K / 256
    int splits;           // S
    int chunks_per_split; // ceil(nchunks / S)
    int row_tiles;        // ceil(N / 16)
    int stages;
    unsigned long long timeout_ns;
};

// --------------------------------------------------------------- constants
// fp16 constants (two copies packed)
constexpr uint32_t H2_ONE = 0x3C003C00u;
constexpr uint32_t H2_SIXTEENTH = 0x2C002C00u;
constexpr uint32_t H2_M1032 = 0xE408E408u;  // -1032
constexpr uint32_t H2_M72 = 0xD480D480u;    // -72
constexpr uint32_t H2_M1152 = 0xE480E480u;  // -1152
constexpr uint32_t H2_M1024 = 0xE400E400u;  // -1024
constexpr uint32_t H2_M64 = 0xD400D400u;    // -64
constexpr uint32_t H2_MAGIC = 0x64006400u;  // 1024
// bf16 constants
constexpr uint32_t B2_ONE = 0x3F803F80u;
constexpr uint32_t B2_M136 = 0xC308C308u;  // -136
constexpr uint32_t B2_MAGIC = 0x43004300u; // 128

// ------------------------------------------------------- activation frags
// Two activations (elements e0, e1 of column b) as one packed register in the
// MMA's 16-bit type; fp32 activations become a (hi, lo) bf16 pair whose sum
// carries 16 significant bits (relative representation error <= 2^-17).
template <int XT>
struct XFrag {
    static constexpr int parts = (XT == X_F32) ? 2 : 1;
};

template <int XT>
__device__ __forceinline__ void load_pair(uint32_t (&out)[XFrag<XT>::parts], const void *x, int M, int K, int b,
                                          long k0, int e0, int e1) {
    if (b >= M) {
#pragma unroll
        for (int p = 0; p < XFrag<XT>::parts; ++p) out[p] = 0u;
        return;
    }
    if constexpr (XT == X_F32) {
        const float *xf = static_cast<const float *>(x) + (long)b * K + k0;
        float v0 = xf[e0], v1 = xf[e1];
        __nv_bfloat16 h0 = __float2bfloat16_rn(v0), h1 = __float2bfloat16_rn(v1);
        float r0 = v0 - __bfloat162float(h0), r1 = v1 - __bfloat162float(h1);
        out[0] = pack_bf16x2(__bfloat162float(h0), __bfloat162float(h1));
        out[1] = pack_bf16x2(r0, r1);
    } else {
        const uint16_t *xh = static_cast<const uint16_t *>(x) + (long)b * K + k0;
        out[0] = (uint32_t)xh[e0] | ((uint32_t)xh[e1] << 16);
    }
}

template <int XT>
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    if constexpr (XT == X_F16)
        mma_f16_16816(d, a, b0, b1, d);
    else
        mma_bf16_16816(d, a, b0, b1, d);
}

// Nibble pair decode into the MMA's 16-bit type.  `w` holds 4 bytes; the
// result holds (byte0 field, byte2 field) for the low nibbles at bits 0-3 /
// 16-19 of w (HI=false) or the high nibbles (HI=true), minus `bias`.
template <int XT, bool HI>
__device__ __forceinline__ uint32_t nib_pair_minus8(uint32_t w) {
    if constexpr (XT == X_F16) {
        if constexpr (!HI)
            return hfma2_f16(and_or(w, 0x000F000Fu, H2_MAGIC), H2_ONE, H2_M1032);       // (1024+q)-1032
        else
            return hfma2_f16(and_or(w, 0x00F000F0u, H2_MAGIC), H2_SIXTEENTH, H2_M72);  // (1024+16q)/16-72
    } else {
        uint32_t v = HI ? (w >> 4) : w;
        return hfma2_bf16(and_or(v, 0x000F000Fu, B2_MAGIC), B2_ONE, B2_M136);           // (128+q)-136
    }
}

// ---------------------------------------------------------------- Q4_0
// Per block (32 weights, 2 k-steps), lane t (= lane % 4) of weight row g
// (= lane / 4) takes nibble bytes 4t..4t+3: elements 4t+j (low nibbles) and
// 4t+j+16 (high nibbles).  k-step A uses elements (4t, 4t+2 | 4t+1, 4t+3),
// k-step B (4t+16, 4t+18 | 4t+17, 4t+19).
template <int XT, int NT>
struct Q40 {
    static constexpr int P = XFrag<XT>::parts;
    // xf[nt][blk][step][reg][part]
    uint32_t xf[NT][8][2][2][P];

    __device__ __forceinline__ void load_x(const void *x, int M, int K, long k0, int lane) {
        const int g = lane >> 2, t = lane & 3;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int blk = 0; blk < 8; ++blk) {
                const int e = blk * 32 + 4 * t;
                load_pair<XT>(xf[nt][blk][0][0], x, M, K, g + 8 * nt, k0, e, e + 2);
                load_pair<XT>(xf[nt][blk][0][1], x, M, K, g + 8 * nt, k0, e + 1, e + 3);
                load_pair<XT>(xf[nt][blk][1][0], x, M, K, g + 8 * nt, k0, e + 16, e + 18);
                load_pair<XT>(xf[nt][blk][1][1], x, M, K, g + 8 * nt, k0, e + 17, e + 19);
            }
    }

    // tb: this warp's [16 rows][144 B] box.  acc[nt][4] accumulates.
    __device__ __forceinline__ void compute(const uint8_t *tb, float (&acc)[NT][4], int lane) const {
        const int g = lane >> 2, t = lane & 3;
        const uint32_t *r0 = reinterpret_cast<const uint32_t *>(tb + g * 144);
        const uint32_t *r1 = reinterpret_cast<const uint32_t *>(tb + (g + 8) * 144);
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            uint32_t nw[2][2];   // [block in pair][row]
            float dd[2][2];
            {
                const int b = 9 * p;
                uint32_t a0 = r0[b + t], a1 = r0[b + t + 1], c0 = r1[b + t], c1 = r1[b + t + 1];
                nw[0][0] = __funnelshift_r(a0, a1, 16);
                nw[0][1] = __funnelshift_r(c0, c1, 16);
                nw[1][0] = r0[b + 5 + t];
                nw[1][1] = r1[b + 5 + t];
                dd[0][0] = f16_bits_to_float(r0[b]);
                dd[0][1] = f16_bits_to_float(r1[b]);
                dd[1][0] = f16_bits_to_float(r0[b + 4] >> 16);
                dd[1][1] = f16_bits_to_float(r1[b + 4] >> 16);
            }
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int blk = 2 * p + h;
                const uint32_t w0 = nw[h][0], w1 = nw[h][1];
                const uint32_t w0s = w0 >> 8, w1s = w1 >> 8;
                uint32_t aA[4] = {nib_pair_minus8<XT, false>(w0), nib_pair_minus8<XT, false>(w1),
                                  nib_pair_minus8<XT, false>(w0s), nib_pair_minus8<XT, false>(w1s)};
                uint32_t aB[4] = {nib_pair_minus8<XT, true>(w0), nib_pair_minus8<XT, true>(w1),
                                  nib_pair_minus8<XT, true>(w0s), nib_pair_minus8<XT, true>(w1s)};
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int q = 0; q < P; ++q) {
                        mma16816<XT>(c, aA, xf[nt][blk][0][0][q], xf[nt][blk][0][1][q]);
                        mma16816<XT>(c, aB, xf[nt][blk][1][0][q], xf[nt][blk][1][1][q]);
                    }
                    acc[nt][0] = fmaf(dd[h][0], c[0], acc[nt][0]);
                    acc[nt][1] = fmaf(dd[h][0], c[1], acc[nt][1]);
                    acc[nt][2] = fmaf(dd[h][1], c[2], acc[nt][2]);
                    acc[nt][3] = fmaf(dd[h][1], c[3], acc[nt][3]);
                }
            }
        }
    }
};

// ---------------------------------------------------------------- Q8_0
// Per block (32 int8, 2 k-steps), lane t takes bytes 8t..8t+7:
// k-step A = elements (8t, 8t+1 | 8t+2, 8t+3), k-step B = (8t+4, 8t+5 | 8t+6, 8t+7).
template <int XT>
__device__ __forceinline__ void q8_pairs(uint32_t w, uint32_t &lo, uint32_t &hi) {
    const uint32_t u = w ^ 0x80808080u;   // biased bytes u = q + 128
    if constexpr (XT == X_F16) {
        lo = hfma2_f16(prmt(u, 0x6400u, 0x5150u), H2_ONE, H2_M1152);   // bytes 0,1
        hi = hfma2_f16(prmt(u, 0x6400u, 0x5352u), H2_ONE, H2_M1152);   // bytes 2,3
    } else {
        const float bias = 8388736.0f;  // 2^23 + 128
        float f0 = __uint_as_float(prmt(u, 0x4B000000u, 0x7440u)) - bias;
        float f1 = __uint_as_float(prmt(u, 0x4B000000u, 0x7441u)) - bias;
        float f2 = __uint_as_float(prmt(u, 0x4B000000u, 0x7442u)) - bias;
        float f3 = __uint_as_float(prmt(u, 0x4B000000u, 0x7443u)) - bias;
        lo = pack_bf16x2(f0, f1);
        hi = pack_bf16x2(f2, f3);
    }
}

template <int XT, int NT>
struct Q80 {
    static constexpr int P = XFrag<XT>::parts;
    uint32_t xf[NT][8][2][2][P];

    __device__ __forceinline__ void load_x(const void *x, int M, int K, long k0, int lane) {
        const int g = lane >> 2, t = lane & 3;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int blk = 0; blk < 8; ++blk) {
                const int e = blk * 32 + 8 * t;
                load_pair<XT>(xf[nt][blk][0][0], x, M, K, g + 8 * nt, k0, e, e + 1);
                load_pair<XT>(xf[nt][blk][0][1], x, M, K, g + 8 * nt, k0, e + 2, e + 3);
                load_pair<XT>(xf[nt][blk][1][0], x, M, K, g + 8 * nt, k0, e + 4, e + 5);
                load_pair<XT>(xf[nt][blk][1][1], x, M, K, g + 8 * nt, k0, e + 6, e + 7);
            }
    }

    __device__ __forceinline__ void compute(const uint8_t *tb, float (&acc)[NT][4], int lane) const {
        const int g = lane >> 2, t = lane & 3;
        const uint32_t *r0 = reinterpret_cast<const uint32_t *>(tb + g * 272);
        const uint32_t *r1 = reinterpret_cast<const uint32_t *>(tb + (g + 8) * 272);
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            const int b = 17 * p;
            uint32_t qw[2][2][2];  // [block in pair][row][word]
            float dd[2][2];
            {
                uint32_t a0 = r0[b + 2 * t], a1 = r0[b + 2 * t + 1], a2 = r0[b + 2 * t + 2];
                uint32_t c0 = r1[b + 2 * t], c1 = r1[b + 2 * t + 1], c2 = r1[b + 2 * t + 2];
                qw[0][0][0] = __funnelshift_r(a0, a1, 16);
                qw[0][0][1] = __funnelshift_r(a1, a2, 16);
                qw[0][1][0] = __funnelshift_r(c0, c1, 16);
                qw[0][1][1] = __funnelshift_r(c1, c2, 16);
                qw[1][0][0] = r0[b + 9 + 2 * t];
                qw[1][0][1] = r0[b + 10 + 2 * t];
                qw[1][1][0] = r1[b + 9 + 2 * t];
                qw[1][1][1] = r1[b + 10 + 2 * t];
                dd[0][0] = f16_bits_to_float(r0[b]);
                dd[0][1] = f16_bits_to_float(r1[b]);
                dd[1][0] = f16_bits_to_float(r0[b + 8] >> 16);
                dd[1][1] = f16_bits_to_float(r1[b + 8] >> 16);
            }
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int blk = 2 * p + h;
                uint32_t aA[4], aB[4];
                q8_pairs<XT>(qw[h][0][0], aA[0], aA[2]);
                q8_pairs<XT>(qw[h][1][0], aA[1], aA[3]);
                q8_pairs<XT>(qw[h][0][1], aB[0], aB[2]);
                q8_pairs<XT>(qw[h][1][1], aB[1], aB[3]);
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int q = 0; q < P; ++q) {
                        mma16816<XT>(c, aA, xf[nt][blk][0][0][q], xf[nt][blk][0][1][q]);
                        mma16816<XT>(c, aB, xf[nt][blk][1][0][q], xf[nt][blk][1][1][q]);
                    }
                    acc[nt][0] = fmaf(dd[h][0], c[0], acc[nt][0]);
                    acc[nt][1] = fmaf(dd[h][0], c[1], acc[nt][1]);
                    acc[nt][2] = fmaf(dd[h][1], c[2], acc[nt][2]);
                    acc[nt][3] = fmaf(dd[h][1], c[3], acc[nt][3]);
                }
            }
        }
    }
};

// ---------------------------------------------------------------- Q4_K
// fp16 activations only.  Lane t owns nibble group t of the superblock
// (sub-blocks 2t and 2t+1) for its two weight rows, so the sub-block scales
// enter the fp16 A values exactly (sc*q <= 945) and all 16 k-steps of a
// superblock accumulate into one MMA result: C = sum_j sc_j sum_i q_i x_i.
// k-step 2i+h uses word i of the group: h=0 low nibbles (sub-block 2t),
// h=1 high nibbles (sub-block 2t+1); slots (2t,2t+1 | 2t+8,2t+9) hold
// elements (4i, 4i+2 | 4i+1, 4i+3) of that sub-block.  The mins enter
// through one more MMA: A = (m_2t, m_2t+1) per row, B = the sub-block sums
// of x (as an fp16 hi + lo pair).  y += d*C - dmin*Cmin.
template <int NT>
struct Q4K {
    uint32_t xf[NT][8][2][2];   // [nt][word i][h][reg]
    uint32_t xs[NT][2];         // sub-block sums (X_2t, X_2t+1) of column g: hi, lo

    __device__ __forceinline__ void load_x(const void *x, int M, int K, long k0, int lane) {
        const int g = lane >> 2, t = lane & 3;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int b = g + 8 * nt;
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int e = 32 * (2 * t + h) + 4 * i;
                    uint32_t r[1];
                    load_pair<X_F16>(r, x, M, K, b, k0, e, e + 2);
                    xf[nt][i][h][0] = r[0];
                    load_pair<X_F16>(r, x, M, K, b, k0, e + 1, e + 3);
                    xf[nt][i][h][1] = r[0];
                }
            float s0 = 0.f, s1 = 0.f;
            if (b < M) {
                const __half *xh = static_cast<const __half *>(x) + (long)b * K + k0;
                for (int l = 0; l < 32; ++l) {
                    s0 += __half2float(xh[32 * (2 * t) + l]);
                    s1 += __half2float(xh[32 * (2 * t + 1) + l]);
                }
            }
            const __half h0 = __float2half_rn(s0), h1 = __float2half_rn(s1);
            const float l0 = s0 - __half2float(h0), l1 = s1 - __half2float(h1);
            xs[nt][0] = (uint32_t)__half_as_ushort(h0) | ((uint32_t)__half_as_ushort(h1) << 16);
            xs[nt][1] = pack_f16x2(l0, l1);
        }
    }

    __device__ __forceinline__ void compute(const uint8_t *tb, float (&acc)[NT][4], int lane) const {
        const int g = lane >> 2, t = lane & 3;
        const uint4 *r0 = reinterpret_cast<const uint4 *>(tb + g * 144);
        const uint4 *r1 = reinterpret_cast<const uint4 *>(tb + (g + 8) * 144);
        const uint4 hd[2] = {r0[0], r1[0]};
        const uint4 qa[2] = {r0[1 + 2 * t], r1[1 + 2 * t]};
        const uint4 qb[2] = {r0[2 + 2 * t], r1[2 + 2 * t]};
        // scales and mins of sub-blocks 2t, 2t+1 for both rows
        uint32_t slo[2], tlo[2], shi[2], thi[2], mpair[2];
        float d[2], dmin[2];
        const uint32_t sel_sc = (t & 1) ? 0x5352u : 0x5150u;  // bytes (2(t&1), 2(t&1)+1) -> halves
        const uint32_t sel_a = (t & 1) ? 0x5252u : 0x5050u;   // byte 2(t&1) in both halves
        const uint32_t sel_b = (t & 1) ? 0x5353u : 0x5151u;   // byte 2(t&1)+1 in both halves
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const uint32_t s0 = hd[r].y, s1 = hd[r].z, s2 = hd[r].w;
            const uint32_t sc_w = (t < 2) ? (s0 & 0x3F3F3F3Fu) : ((s2 & 0x0F0F0F0Fu) | ((s0 >> 2) & 0x30303030u));
            const uint32_t m_w = (t < 2) ? (s1 & 0x3F3F3F3Fu) : (((s2 >> 4) & 0x0F0F0F0Fu) | ((s1 >> 2) & 0x30303030u));
            // (1024 + v) as fp16, then minus 1024
            const uint32_t sa = hfma2_f16(prmt(sc_w, 0x6400u, sel_a), H2_ONE, H2_M1024);   // sc_2t (both halves)
            const uint32_t sb16 = hfma2_f16(prmt(sc_w, 0x6400u, sel_b), H2_SIXTEENTH, H2_M64);  // sc_2t+1 / 16
            slo[r] = sa;
            tlo[r] = hfma2_f16(sa, H2_M1024, 0u);       // -1024 sc
            shi[r] = sb16;
            thi[r] = hfma2_f16(sb16, H2_M1024, 0u);     // -64 sc
            mpair[r] = hfma2_f16(prmt(m_w, 0x6400u, sel_sc), H2_ONE, H2_M1024);  // (m_2t, m_2t+1)
            d[r] = f16_bits_to_float(hd[r].x);
            dmin[r] = f16_bits_to_float(hd[r].x >> 16);
        }
        float c[NT][4];
        float cm[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int j = 0; j < 4; ++j) c[nt][j] = cm[nt][j] = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const uint32_t w0 = (i < 4) ? (&qa[0].x)[i] : (&qb[0].x)[i - 4];
            const uint32_t w1 = (i < 4) ? (&qa[1].x)[i] : (&qb[1].x)[i - 4];
            const uint32_t w0s = w0 >> 8, w1s = w1 >> 8;
            uint32_t al[4] = {hfma2_f16(and_or(w0, 0x000F000Fu, H2_MAGIC), slo[0], tlo[0]),
                              hfma2_f16(and_or(w1, 0x000F000Fu, H2_MAGIC), slo[1], tlo[1]),
                              hfma2_f16(and_or(w0s, 0x000F000Fu, H2_MAGIC), slo[0], tlo[0]),
                              hfma2_f16(and_or(w1s, 0x000F000Fu, H2_MAGIC), slo[1], tlo[1])};
            uint32_t ah[4] = {hfma2_f16(and_or(w0, 0x00F000F0u, H2_MAGIC), shi[0], thi[0]),
                              hfma2_f16(and_or(w1, 0x00F000F0u, H2_MAGIC), shi[1], thi[1]),
                              hfma2_f16(and_or(w0s, 0x00F000F0u, H2_MAGIC), shi[0], thi[0]),
                              hfma2_f16(and_or(w1s, 0x00F000F0u, H2_MAGIC), shi[1], thi[1])};
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                mma_f16_16816(c[nt], al, xf[nt][i][0][0], xf[nt][i][0][1], c[nt]);
                mma_f16_16816(c[nt], ah, xf[nt][i][1][0], xf[nt][i][1][1], c[nt]);
            }
        }
        const uint32_t am[4] = {mpair[0], mpair[1], 0u, 0u};
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            mma_f16_16816(cm[nt], am, xs[nt][0], 0u, cm[nt]);
            mma_f16_16816(cm[nt], am, xs[nt][1], 0u, cm[nt]);
            acc[nt][0] += d[0] * c[nt][0] - dmin[0] * cm[nt][0];
            acc[nt][1] += d[0] * c[nt][1] - dmin[0] * cm[nt][1];
            acc[nt][2] += d[1] * c[nt][2] - dmin[1] * cm[nt][2];
            acc[nt][3] += d[1] * c[nt][3] - dmin[1] * cm[nt][3];
        }
    }
};

template <int FMT, int XT, int NT>
struct GemvImpl;
template <int XT, int NT>
struct GemvImpl<F_Q4_0, XT, NT> : Q40<XT, NT> {};
template <int XT, int NT>
struct GemvImpl<F_Q8_0, XT, NT> : Q80<XT, NT> {};
template <int XT, int NT>
struct GemvImpl<F_Q4_K, XT, NT> : Q4K<NT> {
    static_assert(XT == X_F16, "Q4_K tensor-core GEMV takes fp16 activations");
};

// ------------------------------------------------------------------ kernel
// blockDim = (NW + 2) * 32: warps 0..NW-1 compute, NW produces, NW+1 reduces.
// Register budget: an SM has four 16K-register sub-partitions and a CTA's
// warps are spread over them, so 18 warps (5 on some sub-partitions) allow
// 96 registers per thread and 16 warps allow 128: NT=1 kernels run up to 16
// compute warps at 96 registers, NT=2 kernels up to 14 at 128.
// Dynamic shared memory: stages * NW * 16 * CB bytes of packed boxes, then
// stages * NW * 16 * 8NT fp32 partials, then 3 * stages mbarriers.
template <int FMT, int XT, int NT>
__global__ void __maxnreg__(NT == 1 ? 96 : 128)
    gemv_tc_kernel(const __grid_constant__ CUtensorMap wmap, const GemvArgs a) {
    constexpr int CB = FmtInfo<FMT>::chunk_bytes;
    constexpr int BOX = GEMV_ROWS * CB;
    constexpr int RED = GEMV_ROWS * 8 * NT;  // floats per warp per stage
    extern __shared__ __align__(128) uint8_t smem[];

    const int NW = blockDim.x / 32 - 2;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int S = a.splits;
    const int split = blockIdx.x % S;
    const int rgrp = blockIdx.x / S;
    const int G = gridDim.x / S;
    const int c_begin = split * a.chunks_per_split;
    const int c_end = min(c_begin + a.chunks_per_split, a.nchunks);
    const int nact = c_end - c_begin;  // compute warps with a chunk
    const int stages = a.stages;

    uint8_t *boxes = smem;
    float *red = reinterpret_cast<float *>(smem + (size_t)stages * NW * BOX);
    uint64_t *bars = reinterpret_cast<uint64_t *>(reinterpret_cast<uint8_t *>(red) + (size_t)stages * NW * RED * 4);
    uint64_t *full = bars, *empty = bars + stages, *redfull = bars + 2 * stages;

    if (threadIdx.x == 0) {
        for (int s = 0; s < stages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], nact + 1);
            mbar_init(&redfull[s], nact);
        }
        fence_mbar_init();
    }
    __syncthreads();
    if (nact <= 0 || rgrp >= G) return;

    if (warp == NW) {
        // ---------------- producer
        if (lane == 0) {
            tma_prefetch_desc(&wmap);
            int it = 0;
            for (int tile = rgrp; tile < a.row_tiles; tile += G, ++it) {
                const int s = it % stages;
                if (it >= stages && !mbar_wait(&empty[s], ((it / stages) - 1) & 1, a.timeout_ns, DEVERR_GEMV_WAIT))
                    break;
                mbar_arrive_expect_tx(&full[s], (uint32_t)(nact * BOX));
                for (int w = 0; w < nact; ++w)
                    tma_load_2d(boxes + ((size_t)s * NW + w) * BOX, &wmap, &full[s], (c_begin + w) * (CB / 2),
                                tile * GEMV_ROWS);
            }
            // drain: every issued stage's load lands before the CTA may exit
            const int issued = it;
            for (int j = max(0, issued - stages); j < issued; ++j)
                mbar_wait(&full[j % stages], (j / stages) & 1, a.timeout_ns, DEVERR_GEMV_WAIT);
        }
        return;
    }

    if (warp == NW + 1) {
        // ---------------- reducer
        const int M = a.M, N = a.N;
        const int nout = GEMV_ROWS * M;  // outputs per tile: 16 rows x M columns
        int it = 0;
        for (int tile = rgrp; tile < a.row_tiles; tile += G, ++it) {
            const int s = it % stages;
            if (!mbar_wait(&redfull[s], (it / stages) & 1, a.timeout_ns, DEVERR_GEMV_WAIT)) break;
            const float *rs = red + (size_t)s * NW * RED;
            for (int o = lane; o < nout; o += 32) {
                const int r = o % GEMV_ROWS, b = o / GEMV_ROWS;
                float sum = 0.f;
                for (int w = 0; w < nact; ++w) sum += rs[w * RED + r * (8 * NT) + b];
                const int row = tile * GEMV_ROWS + r;
                if (row < N) {
                    if (S == 1)
                        a.y[(size_t)b * N + row] = sum;
                    else
                        a.partial[((size_t)split * M + b) * N + row] = sum;
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
            if (S > 1) {
                // deterministic split-K fix-up: the last split to arrive adds all splits in order
                __threadfence();
                __syncwarp();
                unsigned old = 0;
                if (lane == 0) old = atomicAdd(&a.counters[tile], 1u);
                old = __shfl_sync(0xffffffffu, old, 0);
                if (old == (unsigned)(S - 1)) {
                    __threadfence();
                    for (int o = lane; o < nout; o += 32) {
                        const int r = o % GEMV_ROWS, b = o / GEMV_ROWS;
                        const int row = tile * GEMV_ROWS + r;
                        if (row < N) {
                            float sum = 0.f;
                            for (int sp = 0; sp < S; ++sp) sum += __ldcg(&a.partial[((size_t)sp * M + b) * N + row]);
                            a.y[(size_t)b * N + row] = sum;
                        }
                    }
                    __syncwarp();
                    if (lane == 0) a.counters[tile] = 0u;
                }
            }
        }
        return;
    }

    // ---------------- compute warps
    if (warp >= nact) return;
    GemvImpl<FMT, XT, NT> impl;
    impl.load_x(a.x, a.M, a.K, (long)(c_begin + warp) * CHUNK, lane);
    const int g = lane >> 2, t = lane & 3;
    int it = 0;
    for (int tile = rgrp; tile < a.row_tiles; tile += G, ++it) {
        const int s = it % stages;
        if (!mbar_wait(&full[s], (it / stages) & 1, a.timeout_ns, DEVERR_GEMV_WAIT)) break;
        float acc[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[nt][j] = 0.f;
        impl.compute(boxes + ((size_t)s * NW + warp) * BOX, acc, lane);
        float *rw = red + ((size_t)s * NW + warp) * RED;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            *reinterpret_cast<float2 *>(&rw[g * (8 * NT) + 8 * nt + 2 * t]) = make_float2(acc[nt][0], acc[nt][1]);
            *reinterpret_cast<float2 *>(&rw[(g + 8) * (8 * NT) + 8 * nt + 2 * t]) =
                make_float2(acc[nt][2], acc[nt][3]);
        }
        __syncwarp();
        if (lane == 0) {
            mbar_arrive(&redfull[s]);
            mbar_arrive(&empty[s]);
        }
    }
}

}  // namespace lwq

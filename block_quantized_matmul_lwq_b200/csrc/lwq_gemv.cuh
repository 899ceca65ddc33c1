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
//    as tensor-core B fragments in fp16.  Per row tile it decodes the packed
//    bytes in registers straight into fp16 A fragments (nibble | 0x6400 is
//    1024 + q: one LOP3 and one packed FMA per two weights, no conversion
//    instructions) and issues mma.sync m16n8k16 with the weight rows as the
//    MMA's M dimension.
//  * Activations: fp16 as they are; bf16 and fp32 scaled by one power of two
//    per warp so that the warp's largest |x| lands in [2^13, 2^14), then fp16
//    (bf16's 8-bit significand fits fp16's 11) or an fp16 hi + lo pair (22
//    significant bits) for fp32.  The scale is undone exactly on the fp32
//    results.
//  * Two lane mappings.  Several activation rows (M >= 2): the MMA's N
//    dimension carries the activation rows; the four lanes of a weight row
//    share a block per k-step, and block scales multiply the fp32 MMA
//    results.  One activation row (M = 1): each lane owns whole blocks, and
//    the N dimension carries blocks instead: lane t's k-slots feed column 2t
//    (its first block) or 2t+1 (its second), so one MMA chain covers eight
//    blocks and each block scale is applied once per row tile.  Q4_K: each
//    lane owns one nibble group (two sub-blocks); the sub-block scales enter
//    the fp16 A values exactly (sc*q <= 945), the mins through one more MMA.
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
    int overlap;          // host side: launch with programmatic stream serialization
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

// ------------------------------------------------------------- activations
template <int XT>
struct XFrag {
    static constexpr int parts = (XT == X_F32) ? 2 : 1;  // fp32 -> fp16 hi + lo
};

// Four consecutive activations (row b, elements e..e+3 of the chunk) as fp32
// (zeros when b >= M): one 16-byte (fp32) or 8-byte (fp16/bf16) load.
template <int XT>
__device__ __forceinline__ float4 load4(const void *x, int M, int K, int b, long k0, int e) {
    if (b >= M) return make_float4(0.f, 0.f, 0.f, 0.f);
    if constexpr (XT == X_F32) {
        return __ldg(reinterpret_cast<const float4 *>(static_cast<const float *>(x) + (long)b * K + k0 + e));
    } else {
        const uint2 u = __ldg(reinterpret_cast<const uint2 *>(static_cast<const uint16_t *>(x) + (long)b * K + k0 + e));
        if constexpr (XT == X_F16)
            return make_float4(f16_bits_to_float(u.x), f16_bits_to_float(u.x >> 16), f16_bits_to_float(u.y),
                               f16_bits_to_float(u.y >> 16));
        else
            return make_float4(bf16_bits_to_float(u.x), bf16_bits_to_float(u.x >> 16), bf16_bits_to_float(u.y),
                               bf16_bits_to_float(u.y >> 16));
    }
}

__device__ __forceinline__ float absmax4(float4 v) {
    return fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
}

// Power-of-two scale s (and 1/s) that puts the warp's largest |x| in
// [2^13, 2^14); fp16 activations are used as they are (s = 1).
template <int XT>
__device__ __forceinline__ void warp_scale(float local_max, float &s, float &inv) {
    float m = local_max;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    s = inv = 1.f;
    if (XT == X_F16 || !(m > 0.f) || !(m <= 3.0e38f)) return;
    const int e = (int)((__float_as_uint(m) >> 23) & 0xFF) - 127;
    int es = 13 - e;
    es = es > 126 ? 126 : (es < -126 ? -126 : es);
    s = __uint_as_float((uint32_t)(127 + es) << 23);
    inv = __uint_as_float((uint32_t)(127 - es) << 23);
}

// Two scaled activations as fp16 pair(s): exact for fp16 (s = 1) and for
// bf16 (8 significant bits); fp32 splits into hi + lo (22 bits together).
template <int XT>
__device__ __forceinline__ void pack2(uint32_t (&out)[XFrag<XT>::parts], float a, float b, float s) {
    a *= s;
    b *= s;
    const uint32_t hi = pack_f16x2(a, b);
    out[0] = hi;
    if constexpr (XT == X_F32) {
        const float ha = __half2float(__ushort_as_half((unsigned short)(hi & 0xFFFFu)));
        const float hb = __half2float(__ushort_as_half((unsigned short)(hi >> 16)));
        out[1] = pack_f16x2(a - ha, b - hb);
    }
}

// ----------------------------------------------------------- weight decode
// (byte0, byte2) low nibbles (bits 0-3, 16-19) minus 8, as fp16x2:
// (1024 + q) - 1032.
__device__ __forceinline__ uint32_t nib_lo(uint32_t w) {
    return hfma2_f16(and_or(w, 0x000F000Fu, H2_MAGIC), H2_ONE, H2_M1032);
}
// (byte0, byte2) high nibbles (bits 4-7, 20-23) minus 8: (1024 + 16q)/16 - 72.
__device__ __forceinline__ uint32_t nib_hi(uint32_t w) {
    return hfma2_f16(and_or(w, 0x00F000F0u, H2_MAGIC), H2_SIXTEENTH, H2_M72);
}
// Q8_0 codes of bytes (0,1) and (2,3) as exact fp16x2: (1024 + (q+128)) - 1152.
__device__ __forceinline__ void q8_pairs(uint32_t w, uint32_t &lo, uint32_t &hi) {
    const uint32_t u = w ^ 0x80808080u;
    lo = hfma2_f16(prmt(u, 0x6400u, 0x5150u), H2_ONE, H2_M1152);
    hi = hfma2_f16(prmt(u, 0x6400u, 0x5352u), H2_ONE, H2_M1152);
}

__device__ __forceinline__ void mma(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    mma_f16_16816(d, a, b0, b1, d);
}

// ------------------------------------------------- Q4_0, several activation rows
// Per block (32 weights, 2 k-steps), lane t (= lane % 4) of weight row g
// (= lane / 4) takes nibble bytes 4t..4t+3: k-step A uses elements
// (4t, 4t+2 | 4t+1, 4t+3), k-step B (4t+16, 4t+18 | 4t+17, 4t+19).
template <int XT, int NT>
struct Q40 {
    static constexpr int P = XFrag<XT>::parts;
    uint32_t xf[NT][8][2][2][P];   // [nt][block][step][reg][part]
    float inv;

    __device__ __forceinline__ void load_x(const void *x, int M, int K, long k0, int lane) {
        const int g = lane >> 2, t = lane & 3;
        float mx = 0.f, s;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int blk = 0; blk < 8; ++blk) {
                mx = fmaxf(mx, absmax4(load4<XT>(x, M, K, g + 8 * nt, k0, blk * 32 + 4 * t)));
                mx = fmaxf(mx, absmax4(load4<XT>(x, M, K, g + 8 * nt, k0, blk * 32 + 16 + 4 * t)));
            }
        warp_scale<XT>(mx, s, inv);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int blk = 0; blk < 8; ++blk)
#pragma unroll
                for (int st = 0; st < 2; ++st) {
                    const float4 v = load4<XT>(x, M, K, g + 8 * nt, k0, blk * 32 + 16 * st + 4 * t);
                    pack2<XT>(xf[nt][blk][st][0], v.x, v.z, s);
                    pack2<XT>(xf[nt][blk][st][1], v.y, v.w, s);
                }
    }

    // tb: this warp's [16 rows][144 B] box.  acc[nt][4] accumulates (scaled).
    __device__ __forceinline__ void compute(uint32_t tb, float (&acc)[NT][4], int lane) const {
        const int g = lane >> 2, t = lane & 3;
        const uint32_t r0 = tb + g * 144, r1 = tb + (g + 8) * 144;   // shared addresses of rows g, g+8
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            uint32_t nw[2][2];   // [block in pair][row]
            float dd[2][2];
            {
                const uint32_t b = 36 * p;
                const uint32_t a0 = lds32(r0 + b + 4 * t), a1 = lds32(r0 + b + 4 * t + 4);
                const uint32_t c0 = lds32(r1 + b + 4 * t), c1 = lds32(r1 + b + 4 * t + 4);
                nw[0][0] = __funnelshift_r(a0, a1, 16);
                nw[0][1] = __funnelshift_r(c0, c1, 16);
                nw[1][0] = lds32(r0 + b + 20 + 4 * t);
                nw[1][1] = lds32(r1 + b + 20 + 4 * t);
                dd[0][0] = f16_bits_to_float(lds32(r0 + b));
                dd[0][1] = f16_bits_to_float(lds32(r1 + b));
                dd[1][0] = f16_bits_to_float(lds32(r0 + b + 16) >> 16);
                dd[1][1] = f16_bits_to_float(lds32(r1 + b + 16) >> 16);
            }
            uint32_t aA[2][4], aB[2][4];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const uint32_t w0 = nw[h][0], w1 = nw[h][1];
                const uint32_t w0s = w0 >> 8, w1s = w1 >> 8;
                aA[h][0] = nib_lo(w0);
                aA[h][1] = nib_lo(w1);
                aA[h][2] = nib_lo(w0s);
                aA[h][3] = nib_lo(w1s);
                aB[h][0] = nib_hi(w0);
                aB[h][1] = nib_hi(w1);
                aB[h][2] = nib_hi(w0s);
                aB[h][3] = nib_hi(w1s);
            }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                // two independent chains (one per block), each over both parts
                float c0[4] = {0.f, 0.f, 0.f, 0.f}, c1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int q = 0; q < P; ++q) {
                    mma(c0, aA[0], xf[nt][2 * p][0][0][q], xf[nt][2 * p][0][1][q]);
                    mma(c1, aA[1], xf[nt][2 * p + 1][0][0][q], xf[nt][2 * p + 1][0][1][q]);
                    mma(c0, aB[0], xf[nt][2 * p][1][0][q], xf[nt][2 * p][1][1][q]);
                    mma(c1, aB[1], xf[nt][2 * p + 1][1][0][q], xf[nt][2 * p + 1][1][1][q]);
                }
                acc[nt][0] = fmaf(dd[0][0], c0[0], fmaf(dd[1][0], c1[0], acc[nt][0]));
                acc[nt][1] = fmaf(dd[0][0], c0[1], fmaf(dd[1][0], c1[1], acc[nt][1]));
                acc[nt][2] = fmaf(dd[0][1], c0[2], fmaf(dd[1][1], c1[2], acc[nt][2]));
                acc[nt][3] = fmaf(dd[0][1], c0[3], fmaf(dd[1][1], c1[3], acc[nt][3]));
            }
        }
    }
};

// --------------------------------------------------- one activation row (M = 1)
// Lane (g, t) owns blocks 2t and 2t+1 of the chunk for weight rows g and g+8.
// k-step s (0..15) takes four weights of block 2t + s/8 from every lane t;
// the B operand is block-diagonal: column c holds the activations of block c
// in the k-slots of the lane that owns block c, zeros elsewhere.  So C[r][c]
// is block c's partial dot product for row r, and lane (g, t) holds exactly
// its own two blocks (columns 2t, 2t+1).  The activation registers of lane
// (g, t) are non-zero only when g is 2t or 2t+1 (then they hold block g).
template <int FMT, int XT>
struct OneRow {
    static constexpr int P = XFrag<XT>::parts;
    uint32_t xf[16][2][P];   // [k-step][reg][part]
    float inv;

    __device__ __forceinline__ void load_x(const void *x, int M, int K, long k0, int lane) {
        const int g = lane >> 2, t = lane & 3;
        const int h = g - 2 * t;                  // which half of the k-steps this lane's B feeds
        const bool own = (h == 0 || h == 1);
        float4 v[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            // Q4_0: v[0..3] = elements 4i..4i+3 (low nibbles), v[4..7] = 16+4i.. (high)
            // Q8_0: v[i] = elements 4i..4i+3
            const int e = (FMT == F_Q4_0) ? ((i < 4) ? 4 * i : 16 + 4 * (i - 4)) : 4 * i;
            v[i] = own ? load4<XT>(x, M, K, 0, k0, 32 * g + e) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        float mx = 0.f, s;
#pragma unroll
        for (int i = 0; i < 8; ++i) mx = fmaxf(mx, absmax4(v[i]));
        warp_scale<XT>(mx, s, inv);
        // pack the lane's own half (8 k-steps) once, then place it in half h
        uint32_t pk[8][2][P];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            // Q4_0: word j/2, low (j even) or high (j odd) nibbles; Q8_0: word j
            const int vi = (FMT == F_Q4_0) ? ((j >> 1) + 4 * (j & 1)) : j;
            if constexpr (FMT == F_Q4_0) {
                pack2<XT>(pk[j][0], v[vi].x, v[vi].z, s);
                pack2<XT>(pk[j][1], v[vi].y, v[vi].w, s);
            } else {
                pack2<XT>(pk[j][0], v[vi].x, v[vi].y, s);
                pack2<XT>(pk[j][1], v[vi].z, v[vi].w, s);
            }
        }
#pragma unroll
        for (int st = 0; st < 16; ++st) {
            const bool live = own && ((st >> 3) == h);
#pragma unroll
            for (int r = 0; r < 2; ++r)
#pragma unroll
                for (int q = 0; q < P; ++q) xf[st][r][q] = live ? pk[st & 7][r][q] : 0u;
        }
    }

    __device__ __forceinline__ void compute(uint32_t tb, float (&acc)[1][4], int lane) const {
        const int g = lane >> 2, t = lane & 3;
        constexpr int CB = FmtInfo<FMT>::chunk_bytes;
        const uint32_t r0 = tb + g * CB, r1 = tb + (g + 8) * CB;   // shared addresses of rows g, g+8
        // four independent chains: [block of the pair][even / odd k-step]
        float c[2][2][4];
#pragma unroll
        for (int a = 0; a < 2; ++a)
#pragma unroll
            for (int b = 0; b < 2; ++b)
#pragma unroll
                for (int j = 0; j < 4; ++j) c[a][b][j] = 0.f;
        float d[2][2];   // [block][row]
        if constexpr (FMT == F_Q4_0) {
            // lane t's block pair: 36 bytes (9 words) at word 9t of each row;
            // block 2t: d in word 0 (low half), nibbles at bytes 2..17;
            // block 2t+1: d in word 4 (high half), nibbles in words 5..8
#pragma unroll
            for (int hb = 0; hb < 2; ++hb) {
                uint32_t W0[5], W1[5];
#pragma unroll
                for (int i = 0; i < 5; ++i) {
                    W0[i] = lds32(r0 + 4 * (9 * t + 4 * hb + i));
                    W1[i] = lds32(r1 + 4 * (9 * t + 4 * hb + i));
                }
                d[hb][0] = f16_bits_to_float(hb ? (W0[0] >> 16) : W0[0]);
                d[hb][1] = f16_bits_to_float(hb ? (W1[0] >> 16) : W1[0]);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const uint32_t n0 = hb ? W0[1 + i] : __funnelshift_r(W0[i], W0[i + 1], 16);
                    const uint32_t n1 = hb ? W1[1 + i] : __funnelshift_r(W1[i], W1[i + 1], 16);
                    const uint32_t n0s = n0 >> 8, n1s = n1 >> 8;
                    const uint32_t al[4] = {nib_lo(n0), nib_lo(n1), nib_lo(n0s), nib_lo(n1s)};
                    const uint32_t ah[4] = {nib_hi(n0), nib_hi(n1), nib_hi(n0s), nib_hi(n1s)};
                    const int st = 8 * hb + 2 * i;
#pragma unroll
                    for (int q = 0; q < P; ++q) {
                        mma(c[hb][0], al, xf[st][0][q], xf[st][1][q]);
                        mma(c[hb][1], ah, xf[st + 1][0][q], xf[st + 1][1][q]);
                    }
                }
            }
        } else {
            // lane t's block pair: 68 bytes (17 words) at word 17t of each row;
            // block 2t: d in word 0 (low half), codes at bytes 2..33;
            // block 2t+1: d in word 8 (high half), codes in words 9..16
#pragma unroll
            for (int hb = 0; hb < 2; ++hb) {
                uint32_t W0[9], W1[9];
#pragma unroll
                for (int i = 0; i < 9; ++i) {
                    W0[i] = lds32(r0 + 4 * (17 * t + 8 * hb + i));
                    W1[i] = lds32(r1 + 4 * (17 * t + 8 * hb + i));
                }
                d[hb][0] = f16_bits_to_float(hb ? (W0[0] >> 16) : W0[0]);
                d[hb][1] = f16_bits_to_float(hb ? (W1[0] >> 16) : W1[0]);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const uint32_t q0 = hb ? W0[1 + i] : __funnelshift_r(W0[i], W0[i + 1], 16);
                    const uint32_t q1 = hb ? W1[1 + i] : __funnelshift_r(W1[i], W1[i + 1], 16);
                    uint32_t a[4];
                    q8_pairs(q0, a[0], a[2]);
                    q8_pairs(q1, a[1], a[3]);
                    const int st = 8 * hb + i;
#pragma unroll
                    for (int q = 0; q < P; ++q) mma(c[hb][i & 1], a, xf[st][0][q], xf[st][1][q]);
                }
            }
        }
        // column 2t (block 2t) lives in c[0][*], column 2t+1 (block 2t+1) in c[1][*]
        float yg = d[0][0] * (c[0][0][0] + c[0][1][0]) + d[1][0] * (c[1][0][1] + c[1][1][1]);
        float yg8 = d[0][1] * (c[0][0][2] + c[0][1][2]) + d[1][1] * (c[1][0][3] + c[1][1][3]);
        yg += __shfl_xor_sync(0xffffffffu, yg, 1);
        yg8 += __shfl_xor_sync(0xffffffffu, yg8, 1);
        yg += __shfl_xor_sync(0xffffffffu, yg, 2);
        yg8 += __shfl_xor_sync(0xffffffffu, yg8, 2);
        acc[0][0] += yg;
        acc[0][2] += yg8;
    }
};

// ------------------------------------------------- Q8_0, several activation rows
// Per block (32 int8, 2 k-steps), lane t takes bytes 8t..8t+7:
// k-step A = elements (8t, 8t+1 | 8t+2, 8t+3), k-step B = (8t+4, 8t+5 | 8t+6, 8t+7).
template <int XT, int NT>
struct Q80 {
    static constexpr int P = XFrag<XT>::parts;
    uint32_t xf[NT][8][2][2][P];
    float inv;

    __device__ __forceinline__ void load_x(const void *x, int M, int K, long k0, int lane) {
        const int g = lane >> 2, t = lane & 3;
        float mx = 0.f, s;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int blk = 0; blk < 8; ++blk)
#pragma unroll
                for (int st = 0; st < 2; ++st)
                    mx = fmaxf(mx, absmax4(load4<XT>(x, M, K, g + 8 * nt, k0, blk * 32 + 8 * t + 4 * st)));
        warp_scale<XT>(mx, s, inv);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int blk = 0; blk < 8; ++blk)
#pragma unroll
                for (int st = 0; st < 2; ++st) {
                    const float4 v = load4<XT>(x, M, K, g + 8 * nt, k0, blk * 32 + 8 * t + 4 * st);
                    pack2<XT>(xf[nt][blk][st][0], v.x, v.y, s);
                    pack2<XT>(xf[nt][blk][st][1], v.z, v.w, s);
                }
    }

    __device__ __forceinline__ void compute(uint32_t tb, float (&acc)[NT][4], int lane) const {
        const int g = lane >> 2, t = lane & 3;
        const uint32_t r0 = tb + g * 272, r1 = tb + (g + 8) * 272;   // shared addresses of rows g, g+8
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            const uint32_t b = 68 * p;
            uint32_t qw[2][2][2];  // [block in pair][row][word]
            float dd[2][2];
            {
                const uint32_t a0 = lds32(r0 + b + 8 * t), a1 = lds32(r0 + b + 8 * t + 4), a2 = lds32(r0 + b + 8 * t + 8);
                const uint32_t c0 = lds32(r1 + b + 8 * t), c1 = lds32(r1 + b + 8 * t + 4), c2 = lds32(r1 + b + 8 * t + 8);
                qw[0][0][0] = __funnelshift_r(a0, a1, 16);
                qw[0][0][1] = __funnelshift_r(a1, a2, 16);
                qw[0][1][0] = __funnelshift_r(c0, c1, 16);
                qw[0][1][1] = __funnelshift_r(c1, c2, 16);
                qw[1][0][0] = lds32(r0 + b + 36 + 8 * t);
                qw[1][0][1] = lds32(r0 + b + 40 + 8 * t);
                qw[1][1][0] = lds32(r1 + b + 36 + 8 * t);
                qw[1][1][1] = lds32(r1 + b + 40 + 8 * t);
                dd[0][0] = f16_bits_to_float(lds32(r0 + b));
                dd[0][1] = f16_bits_to_float(lds32(r1 + b));
                dd[1][0] = f16_bits_to_float(lds32(r0 + b + 32) >> 16);
                dd[1][1] = f16_bits_to_float(lds32(r1 + b + 32) >> 16);
            }
            uint32_t aA[2][4], aB[2][4];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                q8_pairs(qw[h][0][0], aA[h][0], aA[h][2]);
                q8_pairs(qw[h][1][0], aA[h][1], aA[h][3]);
                q8_pairs(qw[h][0][1], aB[h][0], aB[h][2]);
                q8_pairs(qw[h][1][1], aB[h][1], aB[h][3]);
            }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                float c0[4] = {0.f, 0.f, 0.f, 0.f}, c1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int q = 0; q < P; ++q) {
                    mma(c0, aA[0], xf[nt][2 * p][0][0][q], xf[nt][2 * p][0][1][q]);
                    mma(c1, aA[1], xf[nt][2 * p + 1][0][0][q], xf[nt][2 * p + 1][0][1][q]);
                    mma(c0, aB[0], xf[nt][2 * p][1][0][q], xf[nt][2 * p][1][1][q]);
                    mma(c1, aB[1], xf[nt][2 * p + 1][1][0][q], xf[nt][2 * p + 1][1][1][q]);
                }
                acc[nt][0] = fmaf(dd[0][0], c0[0], fmaf(dd[1][0], c1[0], acc[nt][0]));
                acc[nt][1] = fmaf(dd[0][0], c0[1], fmaf(dd[1][0], c1[1], acc[nt][1]));
                acc[nt][2] = fmaf(dd[0][1], c0[2], fmaf(dd[1][1], c1[2], acc[nt][2]));
                acc[nt][3] = fmaf(dd[0][1], c0[3], fmaf(dd[1][1], c1[3], acc[nt][3]));
            }
        }
    }
};

// ---------------------------------------------------------------- Q4_K
// Lane t owns nibble group t of the superblock (sub-blocks 2t and 2t+1) for
// its two weight rows, so the sub-block scales enter the fp16 A values
// exactly (sc*q <= 945) and all 16 k-steps of a superblock accumulate into
// one MMA result C = sum_j sc_j sum_i q_i x_i.  k-step 2i+h uses word i of
// the group: h=0 low nibbles (sub-block 2t), h=1 high nibbles (sub-block
// 2t+1); slots (2t,2t+1 | 2t+8,2t+9) hold elements (4i, 4i+2 | 4i+1, 4i+3)
// of that sub-block.  The mins enter through one more MMA: A = (m_2t,
// m_2t+1) x 64 per row, B = the sub-block sums of x / 64 (an fp16 hi + lo pair).
// y += d*C - dmin*Cmin.
template <int XT, int NT>
struct Q4K {
    static constexpr int P = XFrag<XT>::parts;
    uint32_t xf[NT][8][2][2][P];   // [nt][word i][h][reg][part]
    uint32_t xs[NT][2];            // scaled sub-block sums (X_2t, X_2t+1) of column g: hi, lo
    float inv;

    __device__ __forceinline__ void load_x(const void *x, int M, int K, long k0, int lane) {
        const int g = lane >> 2, t = lane & 3;
        float mx = 0.f, s;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    mx = fmaxf(mx, absmax4(load4<XT>(x, M, K, g + 8 * nt, k0, 32 * (2 * t + h) + 4 * i)));
        warp_scale<XT>(mx, s, inv);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            float sum[2] = {0.f, 0.f};
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float4 v = load4<XT>(x, M, K, g + 8 * nt, k0, 32 * (2 * t + h) + 4 * i);
                    pack2<XT>(xf[nt][i][h][0], v.x, v.z, s);
                    pack2<XT>(xf[nt][i][h][1], v.y, v.w, s);
                    sum[h] += ((v.x + v.y) + (v.z + v.w)) * s;
                }
            // sums of up to 32 scaled activations can exceed fp16's range: carry them / 64
            sum[0] *= 0.015625f;
            sum[1] *= 0.015625f;
            const __half h0 = __float2half_rn(sum[0]), h1 = __float2half_rn(sum[1]);
            const float l0 = sum[0] - __half2float(h0), l1 = sum[1] - __half2float(h1);
            xs[nt][0] = (uint32_t)__half_as_ushort(h0) | ((uint32_t)__half_as_ushort(h1) << 16);
            xs[nt][1] = pack_f16x2(l0, l1);
        }
    }

    __device__ __forceinline__ void compute(uint32_t tb, float (&acc)[NT][4], int lane) const {
        const int g = lane >> 2, t = lane & 3;
        const uint32_t r0 = tb + g * 144, r1 = tb + (g + 8) * 144;   // shared addresses of rows g, g+8
        const uint4 hd[2] = {lds128(r0), lds128(r1)};
        const uint4 qa[2] = {lds128(r0 + 16 + 32 * t), lds128(r1 + 16 + 32 * t)};
        const uint4 qb[2] = {lds128(r0 + 32 + 32 * t), lds128(r1 + 32 + 32 * t)};
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
            const uint32_t sa = hfma2_f16(prmt(sc_w, 0x6400u, sel_a), H2_ONE, H2_M1024);        // sc_2t
            const uint32_t sb16 = hfma2_f16(prmt(sc_w, 0x6400u, sel_b), H2_SIXTEENTH, H2_M64);  // sc_2t+1 / 16
            slo[r] = sa;
            tlo[r] = hfma2_f16(sa, H2_M1024, 0u);       // -1024 sc
            shi[r] = sb16;
            thi[r] = hfma2_f16(sb16, H2_M1024, 0u);     // -64 sc
            // (64 m_2t, 64 m_2t+1): exact (<= 4032); the B side carries the sums / 64
            mpair[r] = hmul2_f16(hfma2_f16(prmt(m_w, 0x6400u, sel_sc), H2_ONE, H2_M1024), 0x54005400u);
            d[r] = f16_bits_to_float(hd[r].x);
            dmin[r] = f16_bits_to_float(hd[r].x >> 16);
        }
        // four independent accumulation chains: (word parity) x (low / high nibbles)
        float c[NT][2][2][4];
        float cm[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                cm[nt][j] = 0.f;
                c[nt][0][0][j] = c[nt][0][1][j] = c[nt][1][0][j] = c[nt][1][1][j] = 0.f;
            }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const uint32_t w0 = (i < 4) ? (&qa[0].x)[i] : (&qb[0].x)[i - 4];
            const uint32_t w1 = (i < 4) ? (&qa[1].x)[i] : (&qb[1].x)[i - 4];
            const uint32_t w0s = w0 >> 8, w1s = w1 >> 8;
            const uint32_t al[4] = {hfma2_f16(and_or(w0, 0x000F000Fu, H2_MAGIC), slo[0], tlo[0]),
                                    hfma2_f16(and_or(w1, 0x000F000Fu, H2_MAGIC), slo[1], tlo[1]),
                                    hfma2_f16(and_or(w0s, 0x000F000Fu, H2_MAGIC), slo[0], tlo[0]),
                                    hfma2_f16(and_or(w1s, 0x000F000Fu, H2_MAGIC), slo[1], tlo[1])};
            const uint32_t ah[4] = {hfma2_f16(and_or(w0, 0x00F000F0u, H2_MAGIC), shi[0], thi[0]),
                                    hfma2_f16(and_or(w1, 0x00F000F0u, H2_MAGIC), shi[1], thi[1]),
                                    hfma2_f16(and_or(w0s, 0x00F000F0u, H2_MAGIC), shi[0], thi[0]),
                                    hfma2_f16(and_or(w1s, 0x00F000F0u, H2_MAGIC), shi[1], thi[1])};
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int q = 0; q < P; ++q) {
                    mma(c[nt][i & 1][0], al, xf[nt][i][0][0][q], xf[nt][i][0][1][q]);
                    mma(c[nt][i & 1][1], ah, xf[nt][i][1][0][q], xf[nt][i][1][1][q]);
                }
        }
        const uint32_t am[4] = {mpair[0], mpair[1], 0u, 0u};
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            mma(cm[nt], am, xs[nt][0], 0u);
            mma(cm[nt], am, xs[nt][1], 0u);
            float cs[4];
#pragma unroll
            for (int j = 0; j < 4; ++j)
                cs[j] = (c[nt][0][0][j] + c[nt][1][0][j]) + (c[nt][0][1][j] + c[nt][1][1][j]);
            acc[nt][0] += d[0] * cs[0] - dmin[0] * cm[nt][0];
            acc[nt][1] += d[0] * cs[1] - dmin[0] * cm[nt][1];
            acc[nt][2] += d[1] * cs[2] - dmin[1] * cm[nt][2];
            acc[nt][3] += d[1] * cs[3] - dmin[1] * cm[nt][3];
        }
    }
};

// FMT x activation type x n8 tiles x one-row mapping
template <int FMT, int XT, int NT, bool ONE>
struct GemvImpl;
template <int XT, int NT>
struct GemvImpl<F_Q4_0, XT, NT, false> : Q40<XT, NT> {};
template <int XT, int NT>
struct GemvImpl<F_Q8_0, XT, NT, false> : Q80<XT, NT> {};
template <int XT>
struct GemvImpl<F_Q4_0, XT, 1, true> : OneRow<F_Q4_0, XT> {};
template <int XT>
struct GemvImpl<F_Q8_0, XT, 1, true> : OneRow<F_Q8_0, XT> {};
template <int XT, int NT>
struct GemvImpl<F_Q4_K, XT, NT, false> : Q4K<XT, NT> {};

// ------------------------------------------------------------------ kernel
// blockDim = (NW + 2) * 32: warps 0..NW-1 compute, warp NW produces (TMA),
// warp NW+1 reduces.  A dedicated producer refills a stage the moment its
// consumers release it, and a dedicated reducer keeps the per-tile reduction
// off the compute warps; both measured faster than folding these duties into
// compute warps.  Register budget: an SM has four 16K-register sub-partitions
// and a CTA's warps are spread over them, so 18 warps (5 on some
// sub-partitions) allow 96 registers per thread and 16 warps allow 128: NT=1
// kernels run up to 16 compute warps at 96 registers, NT=2 kernels up to 14 at
// 128.
// Shared memory: stages * NW * 16 * CB bytes of packed boxes, stages * NW *
// 16 * 8NT fp32 partials, then 3 * stages mbarriers.
template <int FMT, int XT, int NT, bool ONE>
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
        // the next kernel on the stream (launched with programmatic serialization)
        // may begin its own weight prefetch while this one runs
        pdl_launch_dependents();
    }
    __syncthreads();
    if (nact <= 0 || rgrp >= G) return;

    if (warp == NW) {
        // ---------------- producer: reads only Wq, which callers that allow
        // overlap promise is not written by the preceding work
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
        // ---------------- reducer: y and the workspace only after the preceding work completed
        pdl_wait();
        const int M = a.M, N = a.N;
        const int nout = GEMV_ROWS * M;  // outputs per tile: 16 rows x M columns
        int it = 0;
        for (int tile = rgrp; tile < a.row_tiles; tile += G, ++it) {
            const int s = it % stages;
            if (!mbar_wait(&redfull[s], (it / stages) & 1, a.timeout_ns, DEVERR_GEMV_WAIT)) break;
            const uint32_t rs = smem_u32(red) + (uint32_t)(s * NW * RED * 4);
            for (int o = lane; o < nout; o += 32) {
                const int r = o % GEMV_ROWS, b = o / GEMV_ROWS;
                float sum = 0.f;
                for (int w = 0; w < nact; ++w) sum += ldsf(rs + 4 * (w * RED + r * (8 * NT) + b));
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
    GemvImpl<FMT, XT, NT, ONE> impl;
    pdl_wait();   // x may be the preceding kernel's output
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
        impl.compute(smem_u32(boxes) + (uint32_t)((s * NW + warp) * BOX), acc, lane);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[nt][j] *= impl.inv;   // undo the activation scale (exact)
        const uint32_t rw = smem_u32(red) + (uint32_t)(((s * NW + warp) * RED) * 4);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            sts_f2(rw + 4 * (g * (8 * NT) + 8 * nt + 2 * t), acc[nt][0], acc[nt][1]);
            sts_f2(rw + 4 * ((g + 8) * (8 * NT) + 8 * nt + 2 * t), acc[nt][2], acc[nt][3]);
        }
        __syncwarp();
        if (lane == 0) {
            mbar_arrive(&redfull[s]);
            mbar_arrive(&empty[s]);
        }
    }
}

}  // namespace lwq

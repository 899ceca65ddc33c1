// Decode GEMV (M <= 16): y[M,N] = x[M,K] . dequant(Wq)^T.
//
// Design (sm_100a):
//  * A persistent grid.  CTA (split s, row group r) owns a fixed slice of K
//    (split-K factor S) and walks the row tiles r, r+G, r+2G, ... (16 weight
//    rows per tile).
//  * One producer warp stages, per row tile, the tile's packed rows for all
//    of the CTA's K chunks with one 3-D TMA load (dimensions: bytes of a
//    chunk, weight row, chunk), which lands as one [16 rows][256 weights] box
//    per compute warp, into a ring of shared-memory stages (mbarrier
//    full/empty pairs).  One load per stage keeps the producer's issue time
//    small; 2-D boxes of one chunk each cost about as much to issue as a
//    stage takes to arrive.
//  * Each compute warp owns one 256-weight "chunk" of K for the whole kernel
//    and keeps the activations of that chunk in registers, already laid out
//    as tensor-core B fragments in fp16.  Per row tile it decodes the packed
//    bytes in registers straight into fp16 A fragments (nibble | 0x6400 is
//    1024 + q: one LOP3 and one packed FMA per two weights, no conversion
//    instructions) and issues mma.sync m16n8k16 with the weight rows as the
//    MMA's M dimension.
//  * Activations are scaled by one power of two per warp so that the warp's
//    largest |x| lands in [2^13, 2^14), then held as fp16 (fp16 and bf16
//    inputs: exact, bf16's 8-bit significand fits fp16's 11) or as an fp16
//    hi + lo pair (22 significant bits) for fp32.  The scale is undone exactly
//    on the fp32 results.
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
//    writes y, or, with split-K, fp32 partials to the workspace, which a
//    small follow-up kernel (a programmatic dependent launch) adds in split
//    order.  Results are bitwise deterministic.
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
    float *partial;       // [S][M][N] fp32 (split-K only; gemv_splitk_sum_kernel adds the splits)
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
// [2^13, 2^14).  Exact for fp16 and bf16 activations (bar elements that fall
// below fp16's normal range, 2^-27 of the largest), and it keeps x / 16 (the
// high-nibble k-steps) in the normal range too.
template <int XT>
__device__ __forceinline__ void warp_scale(float local_max, float &s, float &inv) {
    float m = local_max;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    s = inv = 1.f;
    if (!(m > 0.f) || !(m <= 3.0e38f)) return;
    const int e = (int)((__float_as_uint(m) >> 23) & 0xFF) - 127;
    int es = 13 - e;
    es = es > 126 ? 126 : (es < -126 ? -126 : es);
    s = __uint_as_float((uint32_t)(127 + es) << 23);
    inv = __uint_as_float((uint32_t)(127 - es) << 23);
}

// Two scaled activations as fp16 pair(s): exact for fp16 and
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

// D = A * B (+0), A 16x32 s8 (row), B 32x8 s8 (col), s32 accumulate.
__device__ __forceinline__ void imma_s8_16832(int (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%10, %10, %10, %10};"
        : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "r"(0));
}

// ------------------------------------------------- Q4_0, several activation rows
// The MMA's N dimension carries activation columns; lane (g, t) of weight
// rows g, g+8 takes code word t of every block (4 code bytes, 8 weights), and
// each block is two k-steps: its low nibbles, then its high nibbles.  Word t
// of an odd block (word-aligned in the 36-byte block pair) is read as it
// lies; word t of an even block holds code bytes 4t-2..4t+1 (t > 0) or
// (14, 15, 0, 1) (t = 0).  A register of code bytes (b0, b2) or (b1, b3) of
// the word feeds k-slots (2t, 2t+1) or (2t+8, 2t+9).
//
// Codes enter the MMA as fp16 subnormals (see the one-row mapping below): the
// low nibble u is u * 2^-24 and the high nibble, left in place, 16u * 2^-24,
// so the high-nibble k-step takes its activations divided by 16.  Per block,
// C_b = sum_k u_k x_k * 2^-24 and y += d_b C_b; the offset 8 comes off once
// per tile through one more MMA: A = the block scales d (fp16, exact),
// B = the block sums of x / 64 as an fp16 hi + lo pair, so
// y = 2^24 sum_b d_b C_b - 8 * 64 * sum_b d_b (X_b / 64).
//
// Column tiles (NT): 16-bit activations: tile nt holds activation rows
// 8nt..8nt+7.  fp32 activations (hi + lo fp16 parts): NT = 1 holds up to 4
// rows, column g = part g >> 2 of row g & 3 (the reducer adds columns b and
// b + 4); NT = 2 holds up to 8 rows with the two parts in the two tiles, both
// accumulated into one result (so only the first output tile is written).
// Two consecutive activations as loaded (fp32 pair, or one word of two
// 16-bit codes) and as fp32.
template <int XT>
struct RawPair {
    using T = uint32_t;
    __device__ static __forceinline__ T zero() { return 0u; }
    __device__ static __forceinline__ T load(const void *x, long off) {
        return __ldg(reinterpret_cast<const uint32_t *>(static_cast<const uint16_t *>(x) + off));
    }
    __device__ static __forceinline__ float2 get(T u) {
        if constexpr (XT == X_F16)
            return make_float2(f16_bits_to_float(u), f16_bits_to_float(u >> 16));
        else
            return make_float2(bf16_bits_to_float(u), bf16_bits_to_float(u >> 16));
    }
};
template <>
struct RawPair<X_F32> {
    using T = float2;
    __device__ static __forceinline__ T zero() { return make_float2(0.f, 0.f); }
    __device__ static __forceinline__ T load(const void *x, long off) {
        return __ldg(reinterpret_cast<const float2 *>(static_cast<const float *>(x) + off));
    }
    __device__ static __forceinline__ float2 get(T v) { return v; }
};

template <int XT, int NT>
struct Q40 {
    static constexpr int P = XFrag<XT>::parts;
    static constexpr bool MERGED = (XT == X_F32 && NT == 1);
    static constexpr bool PART_TILES = (XT == X_F32 && NT == 2);
    uint32_t xf[NT][8][2][2];   // [tile][block][k-step][reg]
    uint32_t xs[NT][2];         // correction B: block sums / 64 of blocks (2t, 2t+1), hi and lo
    float inv;

    __device__ static __forceinline__ int cb0(int hb, int j) { return hb ? 4 * j : (j ? 4 * j - 2 : 14); }
    __device__ static __forceinline__ int cb2(int hb, int j) { return hb ? 4 * j + 2 : 4 * j; }

    __device__ static __forceinline__ float2 load2(const void *x, long off) {
        if constexpr (XT == X_F32) {
            return __ldg(reinterpret_cast<const float2 *>(static_cast<const float *>(x) + off));
        } else {
            const uint32_t u = __ldg(reinterpret_cast<const uint32_t *>(static_cast<const uint16_t *>(x) + off));
            if constexpr (XT == X_F16)
                return make_float2(f16_bits_to_float(u), f16_bits_to_float(u >> 16));
            else
                return make_float2(bf16_bits_to_float(u), bf16_bits_to_float(u >> 16));
        }
    }

    // Part p of the fp16 pair (a, b).
    __device__ static __forceinline__ uint32_t part(float a, float b, int p) {
        const uint32_t hi = pack_f16x2(a, b);
        if (P == 1 || p == 0) return hi;
        return pack_f16x2(a - f16_bits_to_float(hi), b - f16_bits_to_float(hi >> 16));
    }

    // The two element pairs of this lane's writer units in block b (zeros for absent rows).
    __device__ static __forceinline__ void fetch_round(const void *x, int M, int K, long k0, int lane, int b,
                                                       typename RawPair<XT>::T (&r)[(MERGED ? 4 : (PART_TILES ? 8 : 8 * NT)) / 4][2]) {
#pragma unroll
        for (int k = 0; k < (MERGED ? 4 : (PART_TILES ? 8 : 8 * NT)) / 4; ++k) {
            const int u = lane + 32 * k, m = u >> 3, tu = (u >> 1) & 3, h = u & 1;
            r[k][0] = r[k][1] = RawPair<XT>::zero();
            if (m < M) {
                const long e = (long)m * K + k0 + 32 * b + 16 * h;
                r[k][0] = RawPair<XT>::load(x, e + cb0(b & 1, tu));
                r[k][1] = RawPair<XT>::load(x, e + cb2(b & 1, tu));
            }
        }
    }

    // Activation rows in this pass's column tiles, and writer units per lane:
    // a unit is (row m, code word t, nibble half h) of one block, 4 elements.
    static constexpr int ROWS = MERGED ? 4 : (PART_TILES ? 8 : 8 * NT);
    static constexpr int UPL = ROWS * 8 / 32;   // units per lane per block
    static constexpr int OT = PART_TILES ? 1 : NT;

    // Tile nt of a block's B in the staging area: [lane][h][reg], 512 bytes.
    __device__ static __forceinline__ uint32_t stage_addr(uint32_t stage0, uint32_t pstride, int nt) {
        return (OT == NT) ? stage0 + 512u * nt : stage0 + pstride * nt;
    }
    // Column tile and column of part p of row m.
    __device__ static __forceinline__ void place(int m, int p, int &nt, int &g) {
        if (MERGED) {
            nt = 0;
            g = m + 4 * p;
        } else if (PART_TILES) {
            nt = p;
            g = m;
        } else {
            nt = m >> 3;
            g = m & 7;
        }
    }

    // Activation row of column g in tile nt, and the fp16 part it carries.
    __device__ static __forceinline__ int col_row(int g, int nt) {
        return MERGED ? (g & 3) : (PART_TILES ? g : g + 8 * nt);
    }
    __device__ static __forceinline__ int col_part(int g, int nt) { return MERGED ? (g >> 2) : (PART_TILES ? nt : 0); }

    // Fast path, one pass with scale 1 (exact whenever the warp's largest |x|
    // lies in [2^-8, 2^15]: every fp16 value, x / 16 included, stays in range
    // and tiny elements lose only bits far below the largest's): each lane
    // builds its own column's fragments straight from its loads (word t of
    // every block of its row), with no dependence on a maximum first, so all
    // its loads can be in flight together.  Returns false, leaving the
    // fragments to be rebuilt, when the range check fails.
    __device__ __forceinline__ bool load_x_direct(const void *x, int M, int K, long k0, int lane) {
        const int g = lane >> 2, t = lane & 3;
        constexpr int LT = PART_TILES ? 1 : NT;   // tiles with distinct rows
        float mx = 0.f;
#pragma unroll
        for (int nt = 0; nt < LT; ++nt) {
            const int r = col_row(g, nt);
            const bool live = r < M;
            const long base = (long)r * K + k0;
            const bool lo_part = (P == 2 && !PART_TILES && col_part(g, nt) == 1);
            float bsum[8];
            // The loads of BPP blocks are issued together before any of them is
            // used: with the fragments already taking 32-64 registers, leaving
            // the order to the compiler let only a few loads be in flight at a
            // time, several L2 round trips where one or two suffice.
            constexpr int BPP = (XT == X_F32) ? 4 : 8;
            using Raw = typename RawPair<XT>::T;
#pragma unroll
            for (int b0 = 0; b0 < 8; b0 += BPP) {
            Raw rp[BPP][2], rq[BPP][2];
#pragma unroll
            for (int bb = 0; bb < BPP; ++bb)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int b = b0 + bb;
                    rp[bb][h] = rq[bb][h] = RawPair<XT>::zero();
                    if (live) {
                        rp[bb][h] = RawPair<XT>::load(x, base + 32 * b + 16 * h + cb0(b & 1, t));
                        rq[bb][h] = RawPair<XT>::load(x, base + 32 * b + 16 * h + cb2(b & 1, t));
                    }
                }
#pragma unroll
            for (int bb = 0; bb < BPP; ++bb) {
                const int b = b0 + bb;
                bsum[b] = 0.f;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    float2 p = RawPair<XT>::get(rp[bb][h]), q = RawPair<XT>::get(rq[bb][h]);
                    mx = fmaxf(mx, fmaxf(fmaxf(fabsf(p.x), fabsf(p.y)), fmaxf(fabsf(q.x), fabsf(q.y))));
                    const float2 pq = __fadd2_rn(p, q);
                    bsum[b] += pq.x + pq.y;
                    if (h) {   // high-nibble step: x / 16 (exact)
                        p = __fmul2_rn(p, make_float2(0.0625f, 0.0625f));
                        q = __fmul2_rn(q, make_float2(0.0625f, 0.0625f));
                    }
                    if constexpr (P == 1) {
                        xf[nt][b][h][0] = pack_f16x2(p.x, q.x);
                        xf[nt][b][h][1] = pack_f16x2(p.y, q.y);
                    } else {
                        // hi = the top 11 significant bits (exact in fp16), lo = x - hi
                        const float2 ph = make_float2(__uint_as_float(__float_as_uint(p.x) & 0xFFFFE000u),
                                                      __uint_as_float(__float_as_uint(p.y) & 0xFFFFE000u));
                        const float2 qh = make_float2(__uint_as_float(__float_as_uint(q.x) & 0xFFFFE000u),
                                                      __uint_as_float(__float_as_uint(q.y) & 0xFFFFE000u));
                        if constexpr (PART_TILES) {
                            const float2 pl = __ffma2_rn(ph, make_float2(-1.f, -1.f), p);
                            const float2 ql = __ffma2_rn(qh, make_float2(-1.f, -1.f), q);
                            xf[0][b][h][0] = pack_f16x2(ph.x, qh.x);
                            xf[0][b][h][1] = pack_f16x2(ph.y, qh.y);
                            xf[1][b][h][0] = pack_f16x2(pl.x, ql.x);
                            xf[1][b][h][1] = pack_f16x2(pl.y, ql.y);
                        } else if (lo_part) {
                            const float2 pl = __ffma2_rn(ph, make_float2(-1.f, -1.f), p);
                            const float2 ql = __ffma2_rn(qh, make_float2(-1.f, -1.f), q);
                            xf[nt][b][h][0] = pack_f16x2(pl.x, ql.x);
                            xf[nt][b][h][1] = pack_f16x2(pl.y, ql.y);
                        } else {
                            xf[nt][b][h][0] = pack_f16x2(ph.x, qh.x);
                            xf[nt][b][h][1] = pack_f16x2(ph.y, qh.y);
                        }
                    }
                }
                // the block's sum over the four lanes (code words) of this column
                bsum[b] += __shfl_xor_sync(0xffffffffu, bsum[b], 1);
                bsum[b] += __shfl_xor_sync(0xffffffffu, bsum[b], 2);
            }
            }
            // correction B: sums of blocks (2t, 2t+1) / 64, hi + lo; only part-0 columns carry them
            float s0 = 0.f, s1 = 0.f;
#pragma unroll
            for (int j = 0; j < 4; ++j)
                if (j == t) {
                    s0 = bsum[2 * j];
                    s1 = bsum[2 * j + 1];
                }
            if (!live || col_part(g, nt) != 0) s0 = s1 = 0.f;
            s0 *= 0.015625f;
            s1 *= 0.015625f;
            const uint32_t hh = pack_f16x2(s0, s1);
            xs[nt][0] = hh;
            xs[nt][1] = pack_f16x2(s0 - f16_bits_to_float(hh), s1 - f16_bits_to_float(hh >> 16));
        }
        if constexpr (PART_TILES) xs[1][0] = xs[1][1] = 0u;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        inv = 1.f;
        // all-zero activations are exact too; NaN and Inf take the other path
        return mx == 0.f || (mx >= 0.00390625f && mx <= 32768.f);
    }

    // One block at a time, every lane packs UPL units (each element of the
    // pass's rows once, both fp16 parts) into the warp's staging area, then
    // reads back its own B fragments; the block sums ride along for the offset
    // correction.
    // Up to 4 fp32 rows, two columns share a row (hi and lo parts), so the
    // staged path converts each element once; otherwise every lane converts
    // its own column directly.  Both first try scale 1 in a single pass.
    __device__ __forceinline__ void load_x(const void *x, int M, int K, long k0, int lane, uint32_t stage0,
                                           uint32_t pstride) {
        if constexpr (MERGED) {
            if (!load_x_staged<true>(x, M, K, k0, lane, stage0, pstride))
                load_x_staged<false>(x, M, K, k0, lane, stage0, pstride);
        } else {
            if (!load_x_direct(x, M, K, k0, lane)) load_x_staged<false>(x, M, K, k0, lane, stage0, pstride);
        }
    }

    // Staged path: one block per round through the staging area.  UNIT: scale
    // 1 in one pass, returning false when the range check of the direct path
    // fails; else a per-warp power-of-two scale from a first pass over the chunk.
    template <bool UNIT>
    __device__ __forceinline__ bool load_x_staged(const void *x, int M, int K, long k0, int lane, uint32_t stage0,
                                                  uint32_t pstride) {
        const int g = lane >> 2, t = lane & 3;
        // pass 1: the warp's largest |x|
        float mx = 0.f;
#pragma unroll
        for (int k = 0; k < (UNIT ? 0 : UPL); ++k) {
            const int u = lane + 32 * k, m = u >> 3, tu = (u >> 1) & 3, h = u & 1;
            if (m < M) {
                const long base = (long)m * K + k0 + 16 * h;
#pragma unroll
                for (int b = 0; b < 8; ++b) {
                    const float2 p = load2(x, base + 32 * b + cb0(b & 1, tu));
                    const float2 q = load2(x, base + 32 * b + cb2(b & 1, tu));
                    mx = fmaxf(mx, fmaxf(fmaxf(fabsf(p.x), fabsf(p.y)), fmaxf(fabsf(q.x), fabsf(q.y))));
                }
            }
        }
        float s = 1.f;
        if (UNIT)
            inv = 1.f;
        else
            warp_scale<XT>(mx, s, inv);
        // correction sums of blocks (2t, 2t+1) for each tile's column g (part 0 only)
        float cs[NT][2];
        int crow[NT];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            cs[nt][0] = cs[nt][1] = 0.f;
            const int row = MERGED ? (g & 3) : (PART_TILES ? g : g + 8 * nt);
            const bool part0 = MERGED ? (g < 4) : (PART_TILES ? nt == 0 : true);
            crow[nt] = (part0 && row < M) ? row : -1;
        }
        // pass 2, one block per round.  Each round ends in shared-memory stores
        // and a warp barrier that loads may not pass, so the raw activations of
        // round b + PF - 1 are requested at the start of round b: with one unit
        // per lane all eight rounds' loads are in flight before the first is used.
        using Raw = typename RawPair<XT>::T;
        constexpr int PF = (UPL == 1) ? 8 : 3;
        Raw raw[PF][UPL][2];
#pragma unroll
        for (int b = 0; b < PF - 1; ++b) fetch_round(x, M, K, k0, lane, b, raw[b]);
#pragma unroll
        for (int b = 0; b < 8; ++b) {
            if (b + PF - 1 < 8) fetch_round(x, M, K, k0, lane, b + PF - 1, raw[(b + PF - 1) % PF]);
#pragma unroll
            for (int k = 0; k < UPL; ++k) {
                const int u = lane + 32 * k, m = u >> 3, tu = (u >> 1) & 3, h = u & 1;
                float2 p = RawPair<XT>::get(raw[b % PF][k][0]), q = RawPair<XT>::get(raw[b % PF][k][1]);
                if (UNIT) mx = fmaxf(mx, fmaxf(fmaxf(fabsf(p.x), fabsf(p.y)), fmaxf(fabsf(q.x), fabsf(q.y))));
                // high-nibble step: x / 16 (exact: a power of two)
                const float sc = h ? s * 0.0625f : s;
                p.x *= sc;
                p.y *= sc;
                q.x *= sc;
                q.y *= sc;
                float bs = h ? 16.f * ((p.x + p.y) + (q.x + q.y)) : (p.x + p.y) + (q.x + q.y);
                // the block sum of row m: its 8 units sit in lanes 8(m & 3) .. 8(m & 3) + 7
                bs += __shfl_xor_sync(0xffffffffu, bs, 1);
                bs += __shfl_xor_sync(0xffffffffu, bs, 2);
                bs += __shfl_xor_sync(0xffffffffu, bs, 4);
#pragma unroll
                for (int pp = 0; pp < P; ++pp) {
                    int nt, gg;
                    place(m, pp, nt, gg);
                    const uint32_t dst = stage_addr(stage0, pstride, nt) + (uint32_t)((4 * gg + tu) * 16 + 8 * h);
                    asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(dst), "r"(part(p.x, q.x, pp)),
                                 "r"(part(p.y, q.y, pp))
                                 : "memory");
                }
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const int r = crow[nt] < 0 ? 0 : crow[nt];
                    const float v = __shfl_sync(0xffffffffu, bs, 8 * (r & 3));
                    if (crow[nt] >= 0 && (crow[nt] >> 2) == k && (b >> 1) == t) cs[nt][b & 1] = v;
                }
            }
            __syncwarp();
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const uint4 v = lds128(stage_addr(stage0, pstride, nt) + (uint32_t)(lane * 16));
                xf[nt][b][0][0] = v.x;
                xf[nt][b][0][1] = v.y;
                xf[nt][b][1][0] = v.z;
                xf[nt][b][1][1] = v.w;
            }
            __syncwarp();
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const float s0 = cs[nt][0] * 0.015625f, s1 = cs[nt][1] * 0.015625f;
            const uint32_t hh = pack_f16x2(s0, s1);
            xs[nt][0] = hh;
            xs[nt][1] = pack_f16x2(s0 - f16_bits_to_float(hh), s1 - f16_bits_to_float(hh >> 16));
        }
        if constexpr (UNIT) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            return mx == 0.f || (mx >= 0.00390625f && mx <= 32768.f);
        } else {
            return true;
        }
    }

    // tb: this warp's [16 rows][144 B] box.
    __device__ __forceinline__ void compute(uint32_t tb, float (&acc)[NT][4], int lane) const {
        const int g = lane >> 2, t = lane & 3;
        const uint32_t r0 = tb + g * 144, r1 = r0 + 8 * 144;   // rows g, g+8
        const uint32_t sel = t ? 0x3210u : 0x3254u;            // word t of an even block
        float m[OT][4];
#pragma unroll
        for (int o = 0; o < OT; ++o)
#pragma unroll
            for (int j = 0; j < 4; ++j) m[o][j] = 0.f;
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            const uint32_t pb = 36 * p;
            const uint32_t w00 = lds32(r0 + pb), w10 = lds32(r1 + pb);             // d(2p), codes
            const uint32_t w04 = lds32(r0 + pb + 16), w14 = lds32(r1 + pb + 16);   // codes, d(2p+1)
            uint32_t u[2][2];   // [block of the pair][row]
            u[0][0] = prmt(lds32(r0 + pb + 4 * t), w04, sel);
            u[0][1] = prmt(lds32(r1 + pb + 4 * t), w14, sel);
            u[1][0] = lds32(r0 + pb + 20 + 4 * t);
            u[1][1] = lds32(r1 + pb + 20 + 4 * t);
            const float d[2][2] = {{f16_bits_to_float(w00), f16_bits_to_float(w10)},
                                   {f16_bits_to_float(w04 >> 16), f16_bits_to_float(w14 >> 16)}};
#pragma unroll
            for (int hb = 0; hb < 2; ++hb) {
                const uint32_t a0 = u[hb][0], a1 = u[hb][1], s0 = a0 >> 8, s1 = a1 >> 8;
                const uint32_t al[4] = {a0 & 0x000F000Fu, a1 & 0x000F000Fu, s0 & 0x000F000Fu, s1 & 0x000F000Fu};
                const uint32_t ah[4] = {a0 & 0x00F000F0u, a1 & 0x00F000F0u, s0 & 0x00F000F0u, s1 & 0x00F000F0u};
                const int b = 2 * p + hb;
                float c[OT][4];
#pragma unroll
                for (int o = 0; o < OT; ++o)
#pragma unroll
                    for (int j = 0; j < 4; ++j) c[o][j] = 0.f;
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const int o = PART_TILES ? 0 : nt;
                    mma(c[o], al, xf[nt][b][0][0], xf[nt][b][0][1]);
                    mma(c[o], ah, xf[nt][b][1][0], xf[nt][b][1][1]);
                }
#pragma unroll
                for (int o = 0; o < OT; ++o) {
                    m[o][0] = fmaf(d[hb][0], c[o][0], m[o][0]);
                    m[o][1] = fmaf(d[hb][0], c[o][1], m[o][1]);
                    m[o][2] = fmaf(d[hb][1], c[o][2], m[o][2]);
                    m[o][3] = fmaf(d[hb][1], c[o][3], m[o][3]);
                }
            }
        }
        // offset correction: A = (d(2t), d(2t+1)) of rows g, g+8, twice (hi and lo sums)
        const uint32_t q0 = prmt(lds32(r0 + 36 * t), lds32(r0 + 36 * t + 16), 0x7610u);
        const uint32_t q1 = prmt(lds32(r1 + 36 * t), lds32(r1 + 36 * t + 16), 0x7610u);
        const uint32_t ad[4] = {q0, q1, q0, q1};
#pragma unroll
        for (int o = 0; o < OT; ++o) {
            float cm[4] = {0.f, 0.f, 0.f, 0.f};
            mma(cm, ad, xs[o][0], xs[o][1]);
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[o][j] += fmaf(m[o][j], 16777216.f, -512.f * cm[j]);
        }
    }
};

// ------------------------------------- Q4_0, int8 activation blocks (LWQ_FLAG_ACT_I8)
// "Quantized arithmetic without runtime dequantization" ("Compute Shaders con
// WebGPU para Inferencia ML", on why to write the kernels by hand): each run of
// 32 activations of a row becomes int8 codes q with one fp32 scale d
// (d = amax/127, q = rint(x * 127/amax); zero below 2^-100), and one
// mma.m16n8k32 (s8 x s8 -> s32) takes a whole block for 8 activation rows.
// A Q4_0 code u enters as the signed byte 16(u - 8): a high nibble in place
// is (byte & 0xF0) ^ 0x80, a low nibble the same after a 4-bit shift.  So the
// block's integer dot product is 16 * sum (u - 8) q, exact in s32, and
// y += d_w * (d_x / 16) * C per block in fp32.
//
// Lane (g, t) reads code word t of every block, as the fp16 several-row
// mapping does: byte j of the word is code byte e(t, j), with e(t, j) = 4t + j
// for odd blocks and (4t - 2 + j) mod 16 for even ones (the even block starts
// 2 bytes into its word).  Its low nibbles are weights e(t, 0..3) and feed
// MMA k-slots 4t..4t+3; its high nibbles, weights e(t, .) + 16, feed k-slots
// 16 + 4t..  The B fragment of the lane (activation row g) holds the
// activation codes of the same weights in the same slots.
template <int XT>
struct Q40I8 {
    uint32_t xq[8][2];   // [block][k-slots 4t.. / 16+4t..]: int8 codes of activation row g
    float dx[8][2];      // [block][column 2t, 2t+1]: d_x / 16 of activation rows 2t, 2t+1
    float inv;           // 1: no activation scale to undo

    __device__ static __forceinline__ int cb0(int hb, int j) { return hb ? 4 * j : (j ? 4 * j - 2 : 14); }
    __device__ static __forceinline__ int cb2(int hb, int j) { return hb ? 4 * j + 2 : 4 * j; }

    __device__ static __forceinline__ uint32_t pack_s8(int a, int b, int c, int d) {
        return (uint32_t)(a & 0xFF) | ((uint32_t)(b & 0xFF) << 8) | ((uint32_t)(c & 0xFF) << 16) |
               ((uint32_t)d << 24);
    }
    __device__ static __forceinline__ int q8(float v, float s) {
        return max(-127, min(127, __float2int_rn(v * s)));
    }

    __device__ __forceinline__ void load_x(const void *x, int M, int K, long k0, int lane, uint32_t, uint32_t) {
        const int g = lane >> 2, t = lane & 3;
        const bool live = g < M;
        const long base = (long)g * K + k0;
        using Raw = typename RawPair<XT>::T;
        inv = 1.f;
#pragma unroll
        for (int b0 = 0; b0 < 8; b0 += 4) {
            // all loads of four blocks in flight before any is used
            Raw r[4][4];   // [block][pairs: e(t,0..1), e(t,2..3), +16, +16]
#pragma unroll
            for (int bb = 0; bb < 4; ++bb) {
                const int b = b0 + bb;
#pragma unroll
                for (int i = 0; i < 4; ++i) r[bb][i] = RawPair<XT>::zero();
                if (live) {
                    const long e = base + 32 * b;
                    r[bb][0] = RawPair<XT>::load(x, e + cb0(b & 1, t));
                    r[bb][1] = RawPair<XT>::load(x, e + cb2(b & 1, t));
                    r[bb][2] = RawPair<XT>::load(x, e + 16 + cb0(b & 1, t));
                    r[bb][3] = RawPair<XT>::load(x, e + 16 + cb2(b & 1, t));
                }
            }
#pragma unroll
            for (int bb = 0; bb < 4; ++bb) {
                const int b = b0 + bb;
                float v[8];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float2 f = RawPair<XT>::get(r[bb][i]);
                    v[2 * i] = f.x;
                    v[2 * i + 1] = f.y;
                }
                float amax = 0.f;
#pragma unroll
                for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[i]));
                // the block's 32 elements of row g lie in lanes 4g .. 4g+3
                amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
                amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
                const bool zero = !(amax >= 7.888609052210118e-31f);   // 2^-100
                const float d = zero ? 0.f : amax / 127.f;
                const float sc = zero ? 0.f : 127.f / amax;
                xq[b][0] = pack_s8(q8(v[0], sc), q8(v[1], sc), q8(v[2], sc), q8(v[3], sc));
                xq[b][1] = pack_s8(q8(v[4], sc), q8(v[5], sc), q8(v[6], sc), q8(v[7], sc));
                // columns 2t and 2t+1 carry activation rows 2t, 2t+1 (lanes 8t and 8t+4)
                dx[b][0] = 0.0625f * __shfl_sync(0xffffffffu, d, 8 * t);
                dx[b][1] = 0.0625f * __shfl_sync(0xffffffffu, d, 8 * t + 4);
            }
        }
    }

    // tb: this warp's [16 rows][144 B] box.
    __device__ __forceinline__ void compute(uint32_t tb, float (&acc)[1][4], int lane) const {
        const int g = lane >> 2, t = lane & 3;
        const uint32_t r0 = tb + g * 144, r1 = r0 + 8 * 144;   // rows g, g+8
        const uint32_t sel = t ? 0x3210u : 0x3254u;            // word t of an even block
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            const uint32_t pb = 36 * p;
            const uint32_t w00 = lds32(r0 + pb), w10 = lds32(r1 + pb);             // d(2p), codes
            const uint32_t w04 = lds32(r0 + pb + 16), w14 = lds32(r1 + pb + 16);   // codes, d(2p+1)
            uint32_t u[2][2];   // [block of the pair][row]
            u[0][0] = prmt(lds32(r0 + pb + 4 * t), w04, sel);
            u[0][1] = prmt(lds32(r1 + pb + 4 * t), w14, sel);
            u[1][0] = lds32(r0 + pb + 20 + 4 * t);
            u[1][1] = lds32(r1 + pb + 20 + 4 * t);
            const float d[2][2] = {{f16_bits_to_float(w00), f16_bits_to_float(w10)},
                                   {f16_bits_to_float(w04 >> 16), f16_bits_to_float(w14 >> 16)}};
#pragma unroll
            for (int hb = 0; hb < 2; ++hb) {
                const int b = 2 * p + hb;
                const uint32_t a0 = u[hb][0], a1 = u[hb][1];
                // signed bytes 16 (u - 8): low nibbles of rows g, g+8, then high nibbles
                const uint32_t a[4] = {((a0 << 4) & 0xF0F0F0F0u) ^ 0x80808080u, ((a1 << 4) & 0xF0F0F0F0u) ^ 0x80808080u,
                                       (a0 & 0xF0F0F0F0u) ^ 0x80808080u, (a1 & 0xF0F0F0F0u) ^ 0x80808080u};
                int c[4];
                imma_s8_16832(c, a, xq[b][0], xq[b][1]);
                acc[0][0] = fmaf(d[hb][0] * dx[b][0], (float)c[0], acc[0][0]);
                acc[0][1] = fmaf(d[hb][0] * dx[b][1], (float)c[1], acc[0][1]);
                acc[0][2] = fmaf(d[hb][1] * dx[b][0], (float)c[2], acc[0][2]);
                acc[0][3] = fmaf(d[hb][1] * dx[b][1], (float)c[3], acc[0][3]);
            }
        }
    }
};

// --------------------------------------------------- one activation row (M = 1)
// Lane (g, t) owns blocks 2t and 2t+1 of the chunk for weight rows g and g+8
// and runs them one after the other, 8 k-steps each.  Every k-slot of lane t
// holds a weight of its own block, so the B operand is block-diagonal: column
// 2t+p carries part p of the activations of lane t's current block in lane
// t's k-slots and zeros elsewhere (p = 0: the fp16 activation, or the hi half
// of an fp32 one; p = 1: the lo half, zero for fp16/bf16 activations).  Then
// C[r][2t+p] is part p of the block's dot product for row r, held by lane
// (g, t) itself, and fp32 activations take no extra MMAs.
//
// Codes enter the MMA as fp16 subnormals: the bit pattern of an unsigned code
// u is the fp16 value u * 2^-24 (exact, as is every product with an fp16
// activation), so one LOP3 (Q4_0: a nibble of each half, the high nibble left
// in place as 16u * 2^-24) or one PRMT (Q8_0: a byte of each half) makes two
// weights with no arithmetic.  The codes' offset o (8 for Q4_0; 128 for Q8_0,
// whose int8 codes are read as u = q + 128) is removed once per block:
// sum (u - o) x = sum u x - o * sum x.
//
// Code words: lane t's two blocks span CB/16 words per row.  Block 2t starts
// 2 bytes into the first word, so its codes are read as word 0 = (last two
// code bytes, first two code bytes) and words 1.. as they lie; block 2t+1's
// codes are word-aligned.  Byte b of code word j is code byte cb(hb, j) + b
// for b = 0, 1 and cb2(hb, j) + b - 2 for b = 2, 3.
template <int FMT, int XT>
struct OneRow {
    static constexpr int P = XFrag<XT>::parts;
    static constexpr int NC = (FMT == F_Q4_0) ? 16 : 32;   // code bytes per block
    static constexpr int NWB = NC / 4;                       // code words per block and row
    static constexpr float OFFSET = (FMT == F_Q4_0) ? 8.f : 128.f;
    uint32_t xb[2][8][2];   // [block 2t + hb][k-step][reg]: this lane's column of B
    float corr[2];          // -OFFSET * (sum of the block's scaled activations)
    float inv;

    __device__ static __forceinline__ int cb0(int hb, int j) { return hb ? 4 * j : (j ? 4 * j - 2 : NC - 2); }
    __device__ static __forceinline__ int cb2(int hb, int j) { return hb ? 4 * j + 2 : 4 * j; }

    // Element pairs (e, e+1) of activation row 0 as fp32.
    __device__ static __forceinline__ float2 load2(const void *x, long k0, int e) {
        if constexpr (XT == X_F32) {
            return __ldg(reinterpret_cast<const float2 *>(static_cast<const float *>(x) + k0 + e));
        } else {
            const uint32_t u = __ldg(reinterpret_cast<const uint32_t *>(static_cast<const uint16_t *>(x) + k0 + e));
            if constexpr (XT == X_F16)
                return make_float2(f16_bits_to_float(u), f16_bits_to_float(u >> 16));
            else
                return make_float2(bf16_bits_to_float(u), bf16_bits_to_float(u >> 16));
        }
    }

    // Part p (0: hi, 1: lo) of the fp16 pair (a, b), a in the low half.
    __device__ static __forceinline__ uint32_t part(float a, float b, int p) {
        const uint32_t hi = pack_f16x2(a, b);
        if (P == 1 || p == 0) return hi;
        return pack_f16x2(a - f16_bits_to_float(hi), b - f16_bits_to_float(hi >> 16));
    }

    // Each lane packs 8 activations (two k-steps of one block) into the warp's
    // staging area [p][t][hb][k-step][reg] (slot p at stage0 + p * pstride),
    // then the owner lanes (g >> 1 == t) read their column of B from it.
    __device__ __forceinline__ void load_x(const void *x, int M, int K, long k0, int lane, uint32_t stage0,
                                           uint32_t pstride) {
        (void)M;
        (void)K;
        const int blk = lane >> 2, q = lane & 3;   // block of the chunk and quarter of it
        const int hb = blk & 1, tb = blk >> 1;
        // Q4_0: code word q, k-steps 2q (low nibbles) and 2q+1 (high nibbles);
        // Q8_0: code words 2q and 2q+1, one k-step each
        float2 v[4];
        if constexpr (FMT == F_Q4_0) {
            const int e0 = cb0(hb, q), e2 = cb2(hb, q);
            v[0] = load2(x, k0 + 32 * blk, e0);
            v[1] = load2(x, k0 + 32 * blk, e2);
            v[2] = load2(x, k0 + 32 * blk, 16 + e0);
            v[3] = load2(x, k0 + 32 * blk, 16 + e2);
        } else {
            v[0] = load2(x, k0 + 32 * blk, cb0(hb, 2 * q));
            v[1] = load2(x, k0 + 32 * blk, cb2(hb, 2 * q));
            v[2] = load2(x, k0 + 32 * blk, cb0(hb, 2 * q + 1));
            v[3] = load2(x, k0 + 32 * blk, cb2(hb, 2 * q + 1));
        }
        float mx = 0.f;
#pragma unroll
        for (int i = 0; i < 4; ++i) mx = fmaxf(mx, fmaxf(fabsf(v[i].x), fabsf(v[i].y)));
        float s;
        warp_scale<XT>(mx, s, inv);
        float sum = 0.f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            v[i].x *= s;
            v[i].y *= s;
            sum += v[i].x + v[i].y;
        }
        // the block's sum over its four lanes
        sum += __shfl_xor_sync(0xffffffffu, sum, 1);
        sum += __shfl_xor_sync(0xffffffffu, sum, 2);
#pragma unroll
        for (int p = 0; p < P; ++p) {
            uint32_t r[4];
            if constexpr (FMT == F_Q4_0) {
                // k-step 2q: reg 0 = code bytes (0, 2) of word q, reg 1 = bytes (1, 3); low nibbles
                r[0] = part(v[0].x, v[1].x, p);
                r[1] = part(v[0].y, v[1].y, p);
                r[2] = part(v[2].x, v[3].x, p);   // k-step 2q+1: the high nibbles (elements + 16)
                r[3] = part(v[2].y, v[3].y, p);
            } else {
                // k-step j: reg 0 = code bytes (0, 1) of word j, reg 1 = bytes (2, 3)
                r[0] = part(v[0].x, v[0].y, p);
                r[1] = part(v[1].x, v[1].y, p);
                r[2] = part(v[2].x, v[2].y, p);
                r[3] = part(v[3].x, v[3].y, p);
            }
            // k-steps 2q and 2q+1 of block (tb, hb): 4 consecutive words
            st_shared_v4(stage0 + p * pstride + (uint32_t)(((tb * 2 + hb) * 16 + 4 * q) * 4), r[0], r[1], r[2], r[3]);
        }
        __syncwarp();
        const int g = lane >> 2, t = lane & 3;
        corr[0] = -OFFSET * __shfl_sync(0xffffffffu, sum, 8 * t);
        corr[1] = -OFFSET * __shfl_sync(0xffffffffu, sum, 8 * t + 4);
        if ((g >> 1) == t && (g & 1) < P) {
            const uint32_t src = stage0 + (g & 1) * pstride + (uint32_t)(t * 128);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const uint4 u = lds128(src + 16 * i);
                xb[i >> 2][(i & 3) * 2][0] = u.x;
                xb[i >> 2][(i & 3) * 2][1] = u.y;
                xb[i >> 2][(i & 3) * 2 + 1][0] = u.z;
                xb[i >> 2][(i & 3) * 2 + 1][1] = u.w;
            }
        } else {
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int j = 0; j < 8; ++j) xb[h][j][0] = xb[h][j][1] = 0u;
        }
        __syncwarp();
    }

    __device__ __forceinline__ void compute(uint32_t tb, float (&acc)[1][4], int lane) const {
        const int g = lane >> 2, t = lane & 3;
        constexpr int CB = FmtInfo<FMT>::chunk_bytes;
        constexpr int PW = CB / 16;   // words of lane t's block pair per row (2 * NWB + 1)
        const uint32_t r0 = tb + g * CB + 4 * PW * t, r1 = r0 + 8 * CB;   // rows g, g+8
        float y0 = 0.f, y1 = 0.f;
#pragma unroll
        for (int hb = 0; hb < 2; ++hb) {
            uint32_t u0[NWB], u1[NWB];   // code words of the block, rows g and g+8
            float d0, d1;
            if (hb == 0) {
                const uint32_t a0 = lds32(r0), a1 = lds32(r1);
                const uint32_t b0 = lds32(r0 + 4 * NWB), b1 = lds32(r1 + 4 * NWB);
                u0[0] = prmt(a0, b0, 0x3254u);
                u1[0] = prmt(a1, b1, 0x3254u);
#pragma unroll
                for (int j = 1; j < NWB; ++j) {
                    u0[j] = lds32(r0 + 4 * j);
                    u1[j] = lds32(r1 + 4 * j);
                }
                d0 = f16_bits_to_float(a0);
                d1 = f16_bits_to_float(a1);
            } else {
                const uint32_t b0 = lds32(r0 + 4 * NWB), b1 = lds32(r1 + 4 * NWB);
#pragma unroll
                for (int j = 0; j < NWB; ++j) {
                    u0[j] = lds32(r0 + 4 * (NWB + 1 + j));
                    u1[j] = lds32(r1 + 4 * (NWB + 1 + j));
                }
                d0 = f16_bits_to_float(b0 >> 16);
                d1 = f16_bits_to_float(b1 >> 16);
            }
            float c[2][4];   // two independent chains
#pragma unroll
            for (int i = 0; i < 2; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) c[i][j] = 0.f;
            float S0, S1;
            if constexpr (FMT == F_Q4_0) {
                // chain 0: low nibbles (u * 2^-24), chain 1: high nibbles (16u * 2^-24)
#pragma unroll
                for (int j = 0; j < NWB; ++j) {
                    const uint32_t s0 = u0[j] >> 8, s1 = u1[j] >> 8;
                    const uint32_t al[4] = {u0[j] & 0x000F000Fu, u1[j] & 0x000F000Fu, s0 & 0x000F000Fu,
                                            s1 & 0x000F000Fu};
                    const uint32_t ah[4] = {u0[j] & 0x00F000F0u, u1[j] & 0x00F000F0u, s0 & 0x00F000F0u,
                                            s1 & 0x00F000F0u};
                    mma(c[0], al, xb[hb][2 * j][0], xb[hb][2 * j][1]);
                    mma(c[1], ah, xb[hb][2 * j + 1][0], xb[hb][2 * j + 1][1]);
                }
                const float lo0 = (P == 2) ? c[0][0] + c[0][1] : c[0][0];
                const float lo1 = (P == 2) ? c[0][2] + c[0][3] : c[0][2];
                const float hi0 = (P == 2) ? c[1][0] + c[1][1] : c[1][0];
                const float hi1 = (P == 2) ? c[1][2] + c[1][3] : c[1][2];
                S0 = fmaf(hi0, 0.0625f, lo0);
                S1 = fmaf(hi1, 0.0625f, lo1);
            } else {
#pragma unroll
                for (int j = 0; j < NWB; ++j) {
                    const uint32_t v0 = u0[j] ^ 0x80808080u, v1 = u1[j] ^ 0x80808080u;
                    const uint32_t a[4] = {prmt(v0, 0u, 0x4140u), prmt(v1, 0u, 0x4140u), prmt(v0, 0u, 0x4342u),
                                           prmt(v1, 0u, 0x4342u)};
                    mma(c[j & 1], a, xb[hb][j][0], xb[hb][j][1]);
                }
                S0 = (P == 2) ? (c[0][0] + c[1][0]) + (c[0][1] + c[1][1]) : c[0][0] + c[1][0];
                S1 = (P == 2) ? (c[0][2] + c[1][2]) + (c[0][3] + c[1][3]) : c[0][2] + c[1][2];
            }
            // block value in scaled-activation units: d * (2^24 S - OFFSET * sum x)
            y0 = fmaf(d0, fmaf(S0, 16777216.f, corr[hb]), y0);
            y1 = fmaf(d1, fmaf(S1, 16777216.f, corr[hb]), y1);
        }
        // lane t's share of rows g, g+8 goes to column 2t; the reducer adds the four
        acc[0][0] += y0;
        acc[0][2] += y1;
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

    __device__ __forceinline__ void load_x(const void *x, int M, int K, long k0, int lane, uint32_t, uint32_t) {
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

    __device__ __forceinline__ void load_x(const void *x, int M, int K, long k0, int lane, uint32_t, uint32_t) {
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

// ------------------------------------------------- Q4_K, one activation row
// The one-row mapping for superblocks: lane (g, t) owns nibble group t (32
// code bytes: sub-block 2t in the low nibbles, 2t+1 in the high nibbles) of
// weight rows g, g+8, and B is block-diagonal as in the Q4_0/Q8_0 one-row
// mapping (column 2t+p = part p of lane t's activations), so C[r][2t+p] is a
// plain dot product of codes and activations per sub-block.  Two chains per
// nibble half keep the low-nibble (sub-block 2t) and high-nibble (2t+1)
// results apart; the high-nibble k-steps take x / 16, matching their
// in-place codes (16u * 2^-24).  Per row, in fp32:
//   y = d * 2^24 * (sc_2t C_2t + sc_2t+1 C_2t+1) - dmin * (m_2t X_2t + m_2t+1 X_2t+1)
// with X_j the sub-block sums of the scaled activations.  k-slots (2t, 2t+1)
// and (2t+8, 2t+9) of k-step (word i, half h) hold code bytes (0, 2) and
// (1, 3) of word i, i.e. elements (4i, 4i+2) and (4i+1, 4i+3) of sub-block
// 2t+h.
template <int XT>
struct OneRowK {
    static constexpr int P = XFrag<XT>::parts;
    uint32_t xb[8][2][2];   // [code word][nibble half][reg]: this lane's column of B
    float xsum[2];          // X_2t, X_2t+1
    float inv;

    __device__ static __forceinline__ float2 load2(const void *x, long e) {
        if constexpr (XT == X_F32) {
            return __ldg(reinterpret_cast<const float2 *>(static_cast<const float *>(x) + e));
        } else {
            const uint32_t u = __ldg(reinterpret_cast<const uint32_t *>(static_cast<const uint16_t *>(x) + e));
            if constexpr (XT == X_F16)
                return make_float2(f16_bits_to_float(u), f16_bits_to_float(u >> 16));
            else
                return make_float2(bf16_bits_to_float(u), bf16_bits_to_float(u >> 16));
        }
    }
    __device__ static __forceinline__ uint32_t part(float a, float b, int p) {
        const uint32_t hi = pack_f16x2(a, b);
        if (P == 1 || p == 0) return hi;
        return pack_f16x2(a - f16_bits_to_float(hi), b - f16_bits_to_float(hi >> 16));
    }

    // Each lane packs 8 activations (code words 2q, 2q+1 of sub-block j) into
    // the staging area [p][t][h][word][reg]; owner lanes then read their column.
    __device__ __forceinline__ void load_x(const void *x, int M, int K, long k0, int lane, uint32_t stage0,
                                           uint32_t pstride) {
        (void)M;
        (void)K;
        const int j = lane >> 2, q = lane & 3;   // sub-block, quarter
        float2 v[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) v[i] = load2(x, k0 + 32 * j + 8 * q + 2 * i);
        float mx = 0.f;
#pragma unroll
        for (int i = 0; i < 4; ++i) mx = fmaxf(mx, fmaxf(fabsf(v[i].x), fabsf(v[i].y)));
        float s;
        warp_scale<XT>(mx, s, inv);
        float sum = 0.f;
        const float sb = (j & 1) ? s * 0.0625f : s;   // high-nibble sub-blocks: x / 16
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            sum += v[i].x * s + v[i].y * s;
            v[i].x *= sb;
            v[i].y *= sb;
        }
        sum += __shfl_xor_sync(0xffffffffu, sum, 1);
        sum += __shfl_xor_sync(0xffffffffu, sum, 2);
#pragma unroll
        for (int p = 0; p < P; ++p) {
            // word 2q: elements 8q..8q+3 -> reg 0 = (e0, e2), reg 1 = (e1, e3); word 2q+1 likewise
            const uint32_t r0 = part(v[0].x, v[1].x, p), r1 = part(v[0].y, v[1].y, p);
            const uint32_t r2 = part(v[2].x, v[3].x, p), r3 = part(v[2].y, v[3].y, p);
            st_shared_v4(stage0 + p * pstride + (uint32_t)((((j >> 1) * 2 + (j & 1)) * 8 + 2 * q) * 2 * 4), r0, r1, r2,
                         r3);
        }
        __syncwarp();
        const int g = lane >> 2, t = lane & 3;
        xsum[0] = __shfl_sync(0xffffffffu, sum, 8 * t);
        xsum[1] = __shfl_sync(0xffffffffu, sum, 8 * t + 4);
        if ((g >> 1) == t && (g & 1) < P) {
            const uint32_t src = stage0 + (g & 1) * pstride + (uint32_t)(t * 128);
#pragma unroll
            for (int i = 0; i < 8; ++i) {   // [h][word pair]
                const uint4 u = lds128(src + 16 * i);
                const int h = i >> 2, w = 2 * (i & 3);
                xb[w][h][0] = u.x;
                xb[w][h][1] = u.y;
                xb[w + 1][h][0] = u.z;
                xb[w + 1][h][1] = u.w;
            }
        } else {
#pragma unroll
            for (int w = 0; w < 8; ++w)
#pragma unroll
                for (int h = 0; h < 2; ++h) xb[w][h][0] = xb[w][h][1] = 0u;
        }
        __syncwarp();
    }

    // Byte k of w as an exact float (0..255): 2^23 + b, minus 2^23.
    __device__ static __forceinline__ float byte_f(uint32_t w, uint32_t sel) {
        return __uint_as_float(prmt(w, 0x4B000000u, sel)) - 8388608.f;
    }

    __device__ __forceinline__ void compute(uint32_t tb, float (&acc)[1][4], int lane) const {
        const int g = lane >> 2, t = lane & 3;
        const uint32_t r0 = tb + g * 144, r1 = r0 + 8 * 144;   // rows g, g+8
        uint32_t w[2][8];
        {
            const uint4 a0 = lds128(r0 + 16 + 32 * t), b0 = lds128(r0 + 32 + 32 * t);
            const uint4 a1 = lds128(r1 + 16 + 32 * t), b1 = lds128(r1 + 32 + 32 * t);
            w[0][0] = a0.x; w[0][1] = a0.y; w[0][2] = a0.z; w[0][3] = a0.w;
            w[0][4] = b0.x; w[0][5] = b0.y; w[0][6] = b0.z; w[0][7] = b0.w;
            w[1][0] = a1.x; w[1][1] = a1.y; w[1][2] = a1.z; w[1][3] = a1.w;
            w[1][4] = b1.x; w[1][5] = b1.y; w[1][6] = b1.z; w[1][7] = b1.w;
        }
        float c[2][2][4];   // [nibble half][word parity]
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int e = 0; e < 2; ++e)
#pragma unroll
                for (int j = 0; j < 4; ++j) c[h][e][j] = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const uint32_t s0 = w[0][i] >> 8, s1 = w[1][i] >> 8;
            const uint32_t al[4] = {w[0][i] & 0x000F000Fu, w[1][i] & 0x000F000Fu, s0 & 0x000F000Fu, s1 & 0x000F000Fu};
            const uint32_t ah[4] = {w[0][i] & 0x00F000F0u, w[1][i] & 0x00F000F0u, s0 & 0x00F000F0u, s1 & 0x00F000F0u};
            mma(c[0][i & 1], al, xb[i][0][0], xb[i][0][1]);
            mma(c[1][i & 1], ah, xb[i][1][0], xb[i][1][1]);
        }
        // sub-block results per row (units of 2^-24): columns 2t (part 0) and 2t+1 (part 1)
        float C[2][2];   // [row][half]
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            C[0][h] = (c[h][0][0] + c[h][1][0]);
            C[1][h] = (c[h][0][2] + c[h][1][2]);
            if (P == 2) {
                C[0][h] += (c[h][0][1] + c[h][1][1]);
                C[1][h] += (c[h][0][3] + c[h][1][3]);
            }
        }
        // scales and mins of sub-blocks 2t, 2t+1 (6-bit, packed as in the format)
        const uint32_t sel_lo = 0x7540u | (uint32_t)(2 * (t & 1)), sel_hi = sel_lo + 1u;
        float y[2];
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const uint4 hd = lds128(r ? r1 : r0);
            const uint32_t s0 = hd.y, s1 = hd.z, s2 = hd.w;
            const uint32_t sc_w = (t < 2) ? (s0 & 0x3F3F3F3Fu) : ((s2 & 0x0F0F0F0Fu) | ((s0 >> 2) & 0x30303030u));
            const uint32_t m_w = (t < 2) ? (s1 & 0x3F3F3F3Fu) : (((s2 >> 4) & 0x0F0F0F0Fu) | ((s1 >> 2) & 0x30303030u));
            const float sc0 = byte_f(sc_w, sel_lo), sc1 = byte_f(sc_w, sel_hi);
            const float m0 = byte_f(m_w, sel_lo), m1 = byte_f(m_w, sel_hi);
            const float d = f16_bits_to_float(hd.x) * 16777216.f, dmin = f16_bits_to_float(hd.x >> 16);
            const float a = fmaf(sc1, C[r][1], sc0 * C[r][0]);
            const float b = fmaf(m1, xsum[1], m0 * xsum[0]);
            y[r] = fmaf(d, a, -dmin * b);
        }
        // lane t's share of rows g, g+8 goes to column 2t; the reducer adds the four
        acc[0][0] += y[0];
        acc[0][2] += y[1];
    }
};

// FMT x activation type x n8 tiles x one-row mapping
template <int FMT, int XT, int NT, bool ONE, bool I8 = false>
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
template <int XT>
struct GemvImpl<F_Q4_K, XT, 1, true> : OneRowK<XT> {};
template <int XT>
struct GemvImpl<F_Q4_0, XT, 1, false, true> : Q40I8<XT> {};

// ------------------------------------------------------------------ kernel
// Registers per thread: 96 lets a CTA run 16 compute warps (+ producer and
// reducer); kernels whose activation fragments need more take 128 and at most
// 14 compute warps.  fp32 Q4_0 with two column tiles fits 96 (a few bytes of
// prologue spill).
constexpr int gemv_max_regs(int fmt, int xt, int nt) { return (nt == 1 || (fmt == F_Q4_0 && xt == X_F32)) ? 96 : 128; }

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
template <int FMT, int XT, int NT, bool ONE, bool I8 = false>
__global__ void __maxnreg__(gemv_max_regs(FMT, XT, NT))
    gemv_tc_kernel(const __grid_constant__ CUtensorMap wmap, const GemvArgs a) {
    constexpr int CB = FmtInfo<FMT>::chunk_bytes;
    constexpr int BOX = GEMV_ROWS * CB;
    // fp32 activations keep one output tile (their two fp16 parts are merged
    // before the reducer: in the MMA chain for NT = 2, by the reducer for NT = 1)
    constexpr int OT = (XT == X_F32) ? 1 : NT;
    constexpr bool MERGED = (XT == X_F32 && NT == 1 && !ONE && !I8 && FMT == F_Q4_0);
    constexpr int RED = GEMV_ROWS * 8 * OT;  // floats per warp per stage
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
            // stage index and phase parity tracked incrementally (no division per tile)
            int it = 0, s = 0;
            uint32_t ph = 0;
            for (int tile = rgrp; tile < a.row_tiles; tile += G, ++it) {
                if (it >= stages && !mbar_wait(&empty[s], ph ^ 1u, a.timeout_ns, DEVERR_GEMV_WAIT)) break;
                // one 3-D box per stage: [chunks of this split][16 rows][chunk bytes]; the last
                // split's box may run past the last chunk, where it reads zeros (no traffic)
                mbar_arrive_expect_tx(&full[s], (uint32_t)(a.chunks_per_split * BOX));
                tma_load_3d(boxes + (size_t)s * NW * BOX, &wmap, &full[s], 0, tile * GEMV_ROWS, c_begin);
                if (++s == stages) {
                    s = 0;
                    ph ^= 1u;
                }
            }
            // drain: every issued stage's load lands before the CTA may exit
            const int n_issued = it;
            for (int j = max(0, n_issued - stages); j < n_issued; ++j)
                mbar_wait(&full[j % stages], (j / stages) & 1, a.timeout_ns, DEVERR_GEMV_WAIT);
        }
        return;
    }

    if (warp == NW + 1) {
        // ---------------- reducer: y and the workspace only after the preceding work completed.
        // Lane (r, half) sums 4-column groups half, half + 2, ... of row r over the
        // compute warps with 16-byte loads, in warp order (deterministic).
        pdl_wait();
        const int M = a.M, N = a.N;
        constexpr int GPL = OT;   // column groups per lane: 2 * OT groups over two half-warps
        const int r = lane & 15, half = lane >> 4;
        int s = 0;
        uint32_t ph = 0;
        for (int tile = rgrp; tile < a.row_tiles; tile += G) {
            if (!mbar_wait(&redfull[s], ph, a.timeout_ns, DEVERR_GEMV_WAIT)) break;
            const uint32_t rs = smem_u32(red) + (uint32_t)(s * NW * RED * 4) + (uint32_t)(r * 8 * OT * 4);
            float4 v[GPL];
#pragma unroll
            for (int j = 0; j < GPL; ++j) v[j] = make_float4(0.f, 0.f, 0.f, 0.f);
            // four warps' loads in flight at a time; the sums still run in warp order
            int w = 0;
#pragma unroll 1
            for (; w + 4 <= nact; w += 4) {
                uint4 u[4][GPL];
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int j = 0; j < GPL; ++j) u[i][j] = lds128(rs + (uint32_t)((w + i) * RED * 4 + (half + 2 * j) * 16));
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int j = 0; j < GPL; ++j) {
                        v[j].x += __uint_as_float(u[i][j].x);
                        v[j].y += __uint_as_float(u[i][j].y);
                        v[j].z += __uint_as_float(u[i][j].z);
                        v[j].w += __uint_as_float(u[i][j].w);
                    }
            }
#pragma unroll 1
            for (; w < nact; ++w) {
#pragma unroll
                for (int j = 0; j < GPL; ++j) {
                    const uint4 u = lds128(rs + (uint32_t)(w * RED * 4 + (half + 2 * j) * 16));
                    v[j].x += __uint_as_float(u.x);
                    v[j].y += __uint_as_float(u.y);
                    v[j].z += __uint_as_float(u.z);
                    v[j].w += __uint_as_float(u.w);
                }
            }
            if (ONE) {
                // one-row mappings leave lane t's share of each row in column 2t
                float t = v[0].x + v[0].z;
                t += __shfl_xor_sync(0xffffffffu, t, 16);
                v[0].x = t;
            } else if (MERGED) {
                // fp32 parts: column b + 4 holds the lo half of column b
                v[0].x += __shfl_xor_sync(0xffffffffu, v[0].x, 16);
                v[0].y += __shfl_xor_sync(0xffffffffu, v[0].y, 16);
                v[0].z += __shfl_xor_sync(0xffffffffu, v[0].z, 16);
                v[0].w += __shfl_xor_sync(0xffffffffu, v[0].w, 16);
            }
            const int row = tile * GEMV_ROWS + r;
            if (row < N && (half == 0 || !(ONE || MERGED))) {
#pragma unroll
                for (int j = 0; j < GPL; ++j) {
                    const float o[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int b = 4 * (half + 2 * j) + i;
                        if (b < M) {
                            if (S == 1)
                                a.y[(size_t)b * N + row] = o[i];
                            else
                                a.partial[((size_t)split * M + b) * N + row] = o[i];
                        }
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
            if (++s == stages) {
                s = 0;
                ph ^= 1u;
            }
        }
        return;
    }

    // ---------------- compute warps
    if (warp >= nact) return;
    GemvImpl<FMT, XT, NT, ONE, I8> impl;
    pdl_wait();   // x may be the preceding kernel's output
    // staging for the activation layout: this warp's partial-sum slots of stages 0 and 1,
    // which it first writes after its first tile
    impl.load_x(a.x, a.M, a.K, (long)(c_begin + warp) * CHUNK, lane, smem_u32(red) + (uint32_t)(warp * RED * 4),
                (uint32_t)(NW * RED * 4));
    const int g = lane >> 2, t = lane & 3;
    int s = 0;
    uint32_t ph = 0;
    for (int tile = rgrp; tile < a.row_tiles; tile += G) {
        if (!mbar_wait(&full[s], ph, a.timeout_ns, DEVERR_GEMV_WAIT)) break;
        float acc[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[nt][j] = 0.f;
        impl.compute(smem_u32(boxes) + (uint32_t)((s * NW + warp) * BOX), acc, lane);
#pragma unroll
        for (int nt = 0; nt < OT; ++nt)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[nt][j] *= impl.inv;   // undo the activation scale (exact)
        const uint32_t rw = smem_u32(red) + (uint32_t)(((s * NW + warp) * RED) * 4);
#pragma unroll
        for (int nt = 0; nt < OT; ++nt) {
            sts_f2(rw + 4 * (g * (8 * OT) + 8 * nt + 2 * t), acc[nt][0], acc[nt][1]);
            sts_f2(rw + 4 * ((g + 8) * (8 * OT) + 8 * nt + 2 * t), acc[nt][2], acc[nt][3]);
        }
        __syncwarp();
        if (lane == 0) {
            mbar_arrive(&redfull[s]);
            mbar_arrive(&empty[s]);
        }
        if (++s == stages) {
            s = 0;
            ph ^= 1u;
        }
    }
}

// Split-K: y[i] = sum over s (in order) of partial[s][i], i over the M*N
// outputs of one pass.  Launched as a programmatic dependent of the GEMV: it
// waits for the GEMV's partials, and lets the next kernel on the stream start.
static __global__ void __launch_bounds__(256) gemv_splitk_sum_kernel(const float *__restrict__ partial,
                                                                     float *__restrict__ y, int S, long mn) {
    if (threadIdx.x == 0) pdl_launch_dependents();
    pdl_wait();
    const long stride = (long)gridDim.x * blockDim.x;
    if ((mn & 3) == 0) {
        const long n4 = mn >> 2;
        for (long i = (long)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += stride) {
            float4 acc = __ldcg(reinterpret_cast<const float4 *>(partial) + i);
            for (int sp = 1; sp < S; ++sp) {
                const float4 v = __ldcg(reinterpret_cast<const float4 *>(partial + (long)sp * mn) + i);
                acc.x += v.x;
                acc.y += v.y;
                acc.z += v.z;
                acc.w += v.w;
            }
            reinterpret_cast<float4 *>(y)[i] = acc;
        }
    } else {
        for (long i = (long)blockIdx.x * blockDim.x + threadIdx.x; i < mn; i += stride) {
            float acc = __ldcg(partial + i);
            for (int sp = 1; sp < S; ++sp) acc += __ldcg(partial + (long)sp * mn + i);
            y[i] = acc;
        }
    }
}

inline int splitk_sum_blocks(long mn) {
    const long n = ((mn & 3) == 0 ? mn / 4 : mn);
    long b = (n + 255) / 256;
    return (int)(b < 1 ? 1 : (b > 1184 ? 1184 : b));
}

}  // namespace lwq

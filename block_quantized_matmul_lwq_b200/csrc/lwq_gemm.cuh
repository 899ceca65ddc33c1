// Prefill GEMM (M > 16 activation rows): y[M,N] = x[M,K] . dequant(Wq)^T
// on the 5th-generation tensor cores (tcgen05, accumulators in TMEM).
//
// This is the matrix-matrix half of the co-designed dequantization in
// "Resumo Tecnico: Llamas na Web", "3. Design de Shader Consciente de
// Quantizacao": quantized tiles are loaded, dequantized in shared memory and
// reused across rows; here they are reused across up to 256 activation rows
// per MMA, so the decode work per flop shrinks with the token tile.
//
// Roles (one persistent CTA per SM, warp-specialized):
//   warp 0      TMA producer: packed weight chunks [128 or 256 rows][256 weights]
//   warp 1      TMEM allocator and single-thread UMMA issuer
//   warps 2..17 dequantizers: packed chunk -> bf16/fp16 weight tile
//               [128 rows][64 k] per half in the UMMA K-major 128-byte-swizzle layout
//   warps 18-21 epilogue: TMEM -> registers -> y (fp32), coalesced along N
//   warp 22     TMA producer: activation tiles [BN tokens][64 k] (128-byte swizzle)
//               (a warp of its own: two producers in one warp's lanes delayed each
//               other's requests while one of them waited)
// Weight tile: 128 rows (one UMMA per K step) or 256 rows (two, one per
// 128-row half, sharing the activation tile: half the L2 traffic of
// activations per flop, which bounds the 128-row tiles).  UMMA shape: M = 128
// weight rows, N = BN tokens (a multiple of 16 from 32 to 256), K = 16.  The
// tile pair is chosen per shape from a model of the persistent grid's rounds
// and a tile's shared-memory, tensor and L2 time.  Accumulators are
// double-buffered in TMEM where two fit (the epilogue of one tile overlaps
// the main loop of the next).  Every wait is bounded (device error word).
#pragma once

#include "../../include/lwq.h"
#include "lwq_gemv.cuh"
#include "lwq_ptx.cuh"

namespace lwq {

constexpr int GEMM_WROWS = 128;       // weight rows per tile (UMMA M)
constexpr int GEMM_BK = 64;           // k per k-block (one 128-byte swizzle atom of 16-bit values)
constexpr int GEMM_KB_PER_CHUNK = 4;  // k-blocks per packed 256-weight chunk
constexpr int GEMM_DQ_WARPS = 16;
constexpr int GEMM_EPI_WARPS = 4;
constexpr int GEMM_THREADS = (3 + GEMM_DQ_WARPS + GEMM_EPI_WARPS) * 32;
constexpr int GEMM_ACT_WARP = 2 + GEMM_DQ_WARPS + GEMM_EPI_WARPS;

struct GemmPlan {
    int warps, stages, ctas, tile_n, tile_m, splits;
    size_t smem;
};

struct GemmArgs {
    float *y;
    float *partial;   // split-K: [splits][M][N] fp32 (gemv_splitk_sum_kernel adds them), else unused
    int splits;       // K slices per tile (1: write y directly)
    int cps;          // chunks per K slice
    int M, N, K;
    int nchunks;      // K / 256
    int n_wtiles;     // ceil(N / 128)
    int n_ttiles;     // ceil(M / BN)
    int bn;           // token tile (UMMA N)
    int a_stages;     // dequantized weight k-blocks (produced on chip)
    int b_stages;     // activation k-blocks (TMA from L2/HBM)
    int p_stages;     // packed weight chunks (TMA from HBM)
    unsigned long long timeout_ns;
    int overlap;      // host side: launch with programmatic stream serialization
    // Q6_K and Q2_K rows that are not 16-byte multiples: row slots.  The dequantizer warps
    // fetch their own rows: each row's superblock of a chunk is copied as the 16-byte units that
    // hold it (cp.async, 16 bytes per thread and copy) into the row's place in the stage
    // (chunk_bytes apart), so the superblock starts (n rb + sb c) mod 16 bytes in.  Rows past N
    // copy row N - 1 (their outputs are not stored).
    int slots;
    const void *wq;   // the packed weights (row slots only)
    long row_bytes;   // rb
};

template <int FMT>
struct GemmFmt;
template <>
struct GemmFmt<F_Q4_0> { static constexpr int chunk_bytes = 144; };
template <>
struct GemmFmt<F_Q8_0> { static constexpr int chunk_bytes = 272; };
template <>
struct GemmFmt<F_Q4_K> { static constexpr int chunk_bytes = 144; };
template <>
struct GemmFmt<F_Q5_K> { static constexpr int chunk_bytes = 176; };
// Q6_K: a 240-byte box per row and superblock, from the 16-byte boundary at or
// below the 210-byte superblock (which starts 2 * ((105 c) & 7) bytes in)
template <>
struct GemmFmt<F_Q6_K> { static constexpr int chunk_bytes = 240; };
// Q2_K: a 96-byte box per row and superblock, from the 16-byte boundary at or
// below the 84-byte superblock (which starts 2 * ((42 c) & 7) bytes in: 0, 4, 8
// or 12, so its words stay aligned); rows of 16-byte multiples need K % 1024 == 0
template <>
struct GemmFmt<F_Q2_K> { static constexpr int chunk_bytes = 96; };

__host__ __device__ constexpr size_t gemm_a_bytes() { return (size_t)GEMM_WROWS * 128; }
__host__ __device__ constexpr size_t gemm_b_bytes(int bn) { return (size_t)bn * 128; }
// one B stage, rounded up to the 1024-byte alignment of 128-byte-swizzle atoms (A stages are 16 KB)
__host__ __device__ constexpr size_t gemm_bstage_bytes(int bn) { return (gemm_b_bytes(bn) + 1023) & ~(size_t)1023; }
// Accumulator buffers: two (the epilogue of one tile overlaps the main loop of
// the next) when both fit the 512 TMEM columns, else one.
__host__ __device__ constexpr int gemm_nbuf(int h, int bn) { return 2 * h * bn <= 512 ? 2 : 1; }
// TMEM columns allocated: a power of two >= 32 holding nbuf x h accumulators of bn fp32 columns
__host__ __device__ constexpr uint32_t gemm_tmem_cols(int h, int bn) {
    const int need = gemm_nbuf(h, bn) * h * bn;
    return need <= 32 ? 32u : (need <= 64 ? 64u : (need <= 128 ? 128u : (need <= 256 ? 256u : 512u)));
}

// Shared memory: [a stages x h x A 16 KB] [b stages x B bn*128 B] [p stages x h*128*CB] [barriers] [tmem addr]
__host__ __device__ inline size_t gemm_smem_bytes(int cb, int bn, int h, int a_stages, int b_stages, int p_stages) {
    size_t s = (size_t)a_stages * h * gemm_a_bytes() + (size_t)b_stages * gemm_bstage_bytes(bn);
    s += (size_t)p_stages * h * GEMM_WROWS * cb;
    s = (s + 7) & ~(size_t)7;
    s += (size_t)(2 * a_stages + 2 * b_stages + 2 * p_stages + 4 + 1) * 8 + 16;
    return s + 1024;  // slack to align the base to 1024 B
}

// Byte offset of 16-bit element (row r, k) inside a [rows][64] K-major tile
// in the 128-byte swizzle layout: row r at r*128, 16-byte chunk j = k/8 stored
// at chunk position j ^ (r % 8).
__device__ __forceinline__ uint32_t sw128_chunk_offset(int r, int j) {
    return (uint32_t)(r * 128 + ((j ^ (r & 7)) << 4));
}

// ------------------------------------------------------------- dequantizers
// One thread writes the four 16-byte chunks (32 weights) of unit (row, h) of
// a k-block: h selects the first or second 32 weights of the block's 64.

// exact (q - 8) pairs in the target type for the low nibbles of bytes b0, b1
// at bits 0-3 and 16-19 of `v`
template <int XT>
__device__ __forceinline__ uint32_t q4_pair(uint32_t v) {
    if constexpr (XT == X_F16)
        return hfma2_f16(and_or(v, 0x000F000Fu, H2_MAGIC), H2_ONE, H2_M1032);
    else
        return hfma2_bf16(and_or(v, 0x000F000Fu, B2_MAGIC), B2_ONE, B2_M136);
}

// w = d * (q - 8), rounded once to the 16-bit type.
// fp16: d is exact in fp16, one rounding in the multiply.
// bf16: d = d_hi + d_lo with both parts exact in bf16 and (q-8)*d_lo exact,
//       so fma((q-8), d_hi, (q-8)*d_lo) rounds the exact product once.
template <int XT>
__device__ __forceinline__ uint32_t scale_pair(uint32_t qm8, uint32_t dh2, uint32_t dl2) {
    if constexpr (XT == X_F16)
        return hmul2_f16(qm8, dh2);
    else
        return hfma2_bf16(qm8, dh2, hmul2_bf16(qm8, dl2));
}

template <int XT>
__device__ __forceinline__ void split_scale(float d, uint32_t &dh2, uint32_t &dl2) {
    if constexpr (XT == X_F16) {
        const uint32_t h = __half_as_ushort(__float2half_rn(d));  // d came from fp16: exact
        dh2 = h | (h << 16);
        dl2 = 0;
    } else {
        const __nv_bfloat16 hi = __float2bfloat16_rn(d);
        const __nv_bfloat16 lo = __float2bfloat16_rn(d - __bfloat162float(hi));  // exact (<= 4 bits)
        const uint32_t a = __bfloat16_as_ushort(hi), b = __bfloat16_as_ushort(lo);
        dh2 = a | (a << 16);
        dl2 = b | (b << 16);
    }
}

template <int FMT, int XT>
struct Dequant;

// One dequant thread produces 16 weights of a k-block for one weight row r:
// h selects the first or second 32 weights of the k-block's 64, v the 16-B
// output chunks {2v, 2v+1} of those 32 (the chunk pairs are chosen so that a
// thread's two chunks come from the same packed bytes).

// Q4_0: k-block kb of a chunk = blocks 2kb (h=0) and 2kb+1 (h=1).  Block
// bytes 8v..8v+7 hold elements 8v..8v+7 (low nibbles, output chunk v) and
// 16+8v..16+8v+7 (high nibbles, output chunk 2+v).
template <int XT>
struct Dequant<F_Q4_0, XT> {
    static __device__ __forceinline__ void run(uint32_t prow, int kb, int h, int v, uint32_t a_base, int r) {
        // block 2kb+h starts at byte 36kb + 18h; its nibbles at +2, so bytes 8v..8v+7 are at 36kb+18h+2+8v:
        // word 9kb+2v, 2 bytes in (h=0), or exactly word 9kb+5+2v (h=1).  Rows lie 36 words apart, so a
        // warp's h=0 lanes read even banks and its h=1 lanes odd ones: no two lanes of a load share a bank
        // (the third load of an h=1 lane repeats its first)
        const uint32_t w = prow + 4 * (9 * kb + 2 * v + (h ? 5 : 0));
        const uint32_t W0 = lds32(w), W1 = lds32(w + 4), W2 = lds32(h ? w : w + 8);
        const uint32_t q0 = h ? W0 : __funnelshift_r(W0, W1, 16), q1 = h ? W1 : __funnelshift_r(W1, W2, 16);
        const uint32_t dw = lds32(prow + 4 * (9 * kb + 4 * h));
        const float d = f16_bits_to_float(h ? (dw >> 16) : dw);
        uint32_t dh2, dl2;
        split_scale<XT>(d, dh2, dl2);
        // bytes (0,1), (2,3) of q0 and q1 as 16-bit halves, shared by the low and high chunks
        const uint32_t p0 = prmt(q0, 0u, 0x4140u), p1 = prmt(q0, 0u, 0x4342u);
        const uint32_t p2 = prmt(q1, 0u, 0x4140u), p3 = prmt(q1, 0u, 0x4342u);
        st_shared_v4(a_base + sw128_chunk_offset(r, 4 * h + v),
                     scale_pair<XT>(q4_pair<XT>(p0), dh2, dl2), scale_pair<XT>(q4_pair<XT>(p1), dh2, dl2),
                     scale_pair<XT>(q4_pair<XT>(p2), dh2, dl2), scale_pair<XT>(q4_pair<XT>(p3), dh2, dl2));
        st_shared_v4(a_base + sw128_chunk_offset(r, 4 * h + 2 + v),
                     scale_pair<XT>(q4_pair<XT>(p0 >> 4), dh2, dl2), scale_pair<XT>(q4_pair<XT>(p1 >> 4), dh2, dl2),
                     scale_pair<XT>(q4_pair<XT>(p2 >> 4), dh2, dl2), scale_pair<XT>(q4_pair<XT>(p3 >> 4), dh2, dl2));
    }
};

// Codes to the 16-bit type, 8 at a time: n0 and n1 hold one code per
// byte (codes 0-3 and 4-7).  Byte b becomes the fp32 2^23 + code (one PRMT
// with the exponent byte 0x4B), then, two at a time with packed fp32
// arithmetic, (2^23 + code) + off (exact: code + off) and w = s * that + c,
// rounded once to fp32 as fmaf(s, code + off, c) would be; then each pair is
// rounded once to the 16-bit type.
template <int XT>
__device__ __forceinline__ void kq_codes_to_chunk(uint32_t n0, uint32_t n1, float s, float off, float c, uint32_t (&o)[4]) {
    const float2 s2 = make_float2(s, s), c2 = make_float2(c, c), off2 = make_float2(off, off);
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        const uint32_t nw = (p < 2) ? n0 : n1;
        const uint32_t b = 2u * (uint32_t)(p & 1);
        const float2 fq = make_float2(__uint_as_float(prmt(nw, 0x4B000000u, 0x7440u + b)),
                                      __uint_as_float(prmt(nw, 0x4B000000u, 0x7441u + b)));
        const float2 t = __fadd2_rn(fq, off2);   // exact
        const float2 w = __ffma2_rn(s2, t, c2);
        o[p] = (XT == X_F16) ? pack_f16x2(w.x, w.y) : pack_bf16x2(w.x, w.y);
    }
}

// Q8_0: k-block kb = blocks 2kb (h=0) and 2kb+1 (h=1); codes 16v..16v+15
// of the block become output chunks 4h+2v and 4h+2v+1.
template <int XT>
struct Dequant<F_Q8_0, XT> {
    static __device__ __forceinline__ void run(uint32_t prow, int kb, int h, int v, uint32_t a_base, int r) {
        // block 2kb+h starts at byte 68kb + 34h; its codes at +2
        const uint32_t w = prow + 4 * (17 * kb + 8 * h + 4 * v);
        uint32_t W[5];
#pragma unroll
        for (int i = 0; i < 5; ++i) W[i] = lds32(w + 4 * i);
        const uint32_t s = h ? 32u : 16u;
        const uint32_t dw = lds32(prow + 4 * (17 * kb + 8 * h));
        const float d = f16_bits_to_float(h ? (dw >> 16) : dw);
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            const uint32_t q0 = __funnelshift_rc(W[2 * c], W[2 * c + 1], s) ^ 0x80808080u;
            const uint32_t q1 = __funnelshift_rc(W[2 * c + 1], W[2 * c + 2], s) ^ 0x80808080u;
            uint32_t o[4];
            if constexpr (XT == X_F16) {
                const uint32_t h16 = __half_as_ushort(__float2half_rn(d));
                const uint32_t d2 = h16 | (h16 << 16);
                o[0] = hmul2_f16(hfma2_f16(prmt(q0, 0x6400u, 0x5150u), H2_ONE, H2_M1152), d2);
                o[1] = hmul2_f16(hfma2_f16(prmt(q0, 0x6400u, 0x5352u), H2_ONE, H2_M1152), d2);
                o[2] = hmul2_f16(hfma2_f16(prmt(q1, 0x6400u, 0x5150u), H2_ONE, H2_M1152), d2);
                o[3] = hmul2_f16(hfma2_f16(prmt(q1, 0x6400u, 0x5352u), H2_ONE, H2_M1152), d2);
            } else {
                // (2^23 + (q + 128)) - (2^23 + 128) = q, then d * q rounded once
                kq_codes_to_chunk<XT>(q0, q1, d, -8388736.0f, -0.0f, o);
            }
            st_shared_v4(a_base + sw128_chunk_offset(r, 4 * h + 2 * v + c), o[0], o[1], o[2], o[3]);
        }
    }
};

// Q4_K: chunk = one superblock; k-block kb = nibble group kb: h=0 sub-block
// 2kb (low nibbles), h=1 sub-block 2kb+1 (high nibbles); elements 16v..16v+15
// of the sub-block (bytes 32kb+16v..+15) become output chunks 4h+2v, 4h+2v+1.
template <int XT>
struct Dequant<F_Q4_K, XT> {
    static __device__ __forceinline__ void run(uint32_t prow, int kb, int h, int v, uint32_t a_base, int r) {
        const uint4 hd = lds128(prow);
        const uint4 qv = lds128(prow + 16 + 32 * kb + 16 * v);
        const int j = 2 * kb + h;
        const uint32_t s0 = hd.y, s1 = hd.z, s2 = hd.w;
        uint32_t scw, mw;
        if (j < 4) {
            scw = s0 & 0x3F3F3F3Fu;
            mw = s1 & 0x3F3F3F3Fu;
        } else {
            scw = (s2 & 0x0F0F0F0Fu) | ((s0 >> 2) & 0x30303030u);
            mw = ((s2 >> 4) & 0x0F0F0F0Fu) | ((s1 >> 2) & 0x30303030u);
        }
        const int sc = (scw >> (8 * (j & 3))) & 63, m = (mw >> (8 * (j & 3))) & 63;
        const float ds = f16_bits_to_float(hd.x) * (float)sc;           // exact in fp32
        const float dm = f16_bits_to_float(hd.x >> 16) * (float)m;      // exact in fp32
        const uint32_t qw[4] = {qv.x, qv.y, qv.z, qv.w};
        const uint32_t sh = 4u * h;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            // w = ds * q - dm, q the nibbles h of the 8 bytes
            uint32_t o[4];
            kq_codes_to_chunk<XT>((qw[2 * c] >> sh) & 0x0F0F0F0Fu, (qw[2 * c + 1] >> sh) & 0x0F0F0F0Fu, ds,
                                  -8388608.0f, -dm, o);
            st_shared_v4(a_base + sw128_chunk_offset(r, 4 * h + 2 * v + c), o[0], o[1], o[2], o[3]);
        }
    }
};

// Q5_K: as Q4_K, with the nibbles at 48 and a fifth bit per code: bit j of
// qh[l] for element l of sub-block j's 32 (qh[32] at 16).
template <int XT>
struct Dequant<F_Q5_K, XT> {
    static __device__ __forceinline__ void run(uint32_t prow, int kb, int h, int v, uint32_t a_base, int r) {
        const uint4 hd = lds128(prow);
        const uint4 qv = lds128(prow + 48 + 32 * kb + 16 * v);
        const uint4 hv = lds128(prow + 16 + 16 * v);
        const int j = 2 * kb + h;
        const uint32_t s0 = hd.y, s1 = hd.z, s2 = hd.w;
        uint32_t scw, mw;
        if (j < 4) {
            scw = s0 & 0x3F3F3F3Fu;
            mw = s1 & 0x3F3F3F3Fu;
        } else {
            scw = (s2 & 0x0F0F0F0Fu) | ((s0 >> 2) & 0x30303030u);
            mw = ((s2 >> 4) & 0x0F0F0F0Fu) | ((s1 >> 2) & 0x30303030u);
        }
        const int sc = (scw >> (8 * (j & 3))) & 63, m = (mw >> (8 * (j & 3))) & 63;
        const float ds = f16_bits_to_float(hd.x) * (float)sc;           // exact in fp32
        const float dm = f16_bits_to_float(hd.x >> 16) * (float)m;      // exact in fp32
        const uint32_t qw[4] = {qv.x, qv.y, qv.z, qv.w};
        const uint32_t hw[4] = {hv.x, hv.y, hv.z, hv.w};
        const uint32_t sh = 4u * h;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            // q = nibble h | (bit j of the qh byte) << 4, four bytes at a time
            uint32_t n[2];
#pragma unroll
            for (int w = 0; w < 2; ++w)
                n[w] = ((qw[2 * c + w] >> sh) & 0x0F0F0F0Fu) | (((hw[2 * c + w] >> j) << 4) & 0x10101010u);
            uint32_t o[4];
            kq_codes_to_chunk<XT>(n[0], n[1], ds, -8388608.0f, -dm, o);
            st_shared_v4(a_base + sw128_chunk_offset(r, 4 * h + 2 * v + c), o[0], o[1], o[2], o[3]);
        }
    }
};

// 16 bytes at a 2-byte-aligned shared address (5 aligned words and PRMTs when
// the address is 2 mod 4).
__device__ __forceinline__ uint4 lds128_a2(uint32_t addr) {
    const uint32_t b = addr & ~3u;
    const uint32_t w0 = lds32(b), w1 = lds32(b + 4), w2 = lds32(b + 8), w3 = lds32(b + 12);
    if (!(addr & 2)) return make_uint4(w0, w1, w2, w3);
    const uint32_t w4 = lds32(b + 16);
    return make_uint4(prmt(w0, w1, 0x5432u), prmt(w1, w2, 0x5432u), prmt(w2, w3, 0x5432u), prmt(w3, w4, 0x5432u));
}

// Q6_K: k-block kb = sub-blocks 4kb .. 4kb+3 of 16 weights; (h, v) takes
// sub-block j = 4kb + 2h + v, whose codes are nibble g>>1 of
// ql[64n + 32(g&1) + 16(j&1) + i] and bits 2g, 2g+1 of qh[32n + 16(j&1) + i]
// (n = j/8, g = (j/2)%4, i < 16), scale int8 sc[j], w = d * sc * (q - 32),
// exact in fp32 and rounded once to the 16-bit type.  prow: the row's
// superblock (2-byte aligned).
template <int XT>
struct Dequant<F_Q6_K, XT> {
    static __device__ __forceinline__ void run(uint32_t prow, int kb, int h, int v, uint32_t a_base, int r) {
        const int j = 4 * kb + 2 * h + v, n = j >> 3, g = (j >> 1) & 3, l0 = 16 * (j & 1);
        const uint4 qlv = lds128_a2(prow + 64 * n + 32 * (g & 1) + l0);
        const uint4 qhv = lds128_a2(prow + 128 + 32 * n + l0);
        const uint32_t dw = lds32((prow + 208) & ~3u), sw = lds32((prow + 192 + j) & ~3u);
        const float d = f16_bits_to_float(((prow + 208) & 2) ? (dw >> 16) : dw);
        const int sc = (int)(int8_t)(sw >> (8 * ((prow + 192 + j) & 3)));
        const float ds = d * (float)sc;   // exact in fp32
        const uint32_t ql[4] = {qlv.x, qlv.y, qlv.z, qlv.w}, qh[4] = {qhv.x, qhv.y, qhv.z, qhv.w};
        const uint32_t ls = 4u * (g >> 1), hs = 2u * g;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            // q = nibble g>>1 of the ql byte | bits 2g, 2g+1 of the qh byte << 4; w = ds * (q - 32), exact
            uint32_t n[2];
#pragma unroll
            for (int w = 0; w < 2; ++w)
                n[w] = ((ql[2 * c + w] >> ls) & 0x0F0F0F0Fu) | (((qh[2 * c + w] >> hs) << 4) & 0x30303030u);
            uint32_t o[4];
            kq_codes_to_chunk<XT>(n[0], n[1], ds, -8388640.0f, -0.0f, o);   // + (-0): ds * t exactly, signed zeros too
            st_shared_v4(a_base + sw128_chunk_offset(r, 4 * h + 2 * v + c), o[0], o[1], o[2], o[3]);
        }
    }
};

// Q2_K: k-block kb = elements 64kb .. 64kb+63 of the superblock; (h, v) takes the
// 16-weight sub-block 4kb + 2h + v, elements 128n + 32j + 16v + i (n = kb/2,
// j = 2(kb & 1) + h, i < 16), whose codes are bits 2j, 2j+1 of qs[32n + 16v + i]
// (qs at 16), scale and min the nibbles of s[4kb + 2h + v]; w = d sc q - dmin m,
// rounded once.  prow: the row's superblock (4-byte aligned).
template <int XT>
struct Dequant<F_Q2_K, XT> {
    static __device__ __forceinline__ void run(uint32_t prow, int kb, int h, int v, uint32_t a_base, int r) {
        const int n = kb >> 1, j = 2 * (kb & 1) + h, sb = 4 * kb + 2 * h + v;
        const uint32_t dw = lds32(prow + 80);                       // d | dmin
        const uint32_t sbyte = (lds32(prow + (uint32_t)(sb & ~3)) >> (8 * (sb & 3))) & 0xFFu;
        const float ds = f16_bits_to_float(dw) * (float)(sbyte & 15u);           // exact in fp32
        const float dm = f16_bits_to_float(dw >> 16) * (float)(sbyte >> 4);      // exact in fp32
        const uint32_t q = prow + 16u + 32u * (uint32_t)n + 16u * (uint32_t)v;
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) w[i] = (lds32(q + 4 * i) >> (2 * j)) & 0x03030303u;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            uint32_t o[4];
            kq_codes_to_chunk<XT>(w[2 * c], w[2 * c + 1], ds, -8388608.0f, -dm, o);
            st_shared_v4(a_base + sw128_chunk_offset(r, 4 * h + 2 * v + c), o[0], o[1], o[2], o[3]);
        }
    }
};

// -------------------------------------------------------------------- kernel
// H = 128-row halves of a weight tile (1 or 2).  With H = 2 the tile is 256
// weight rows: two UMMAs per K step (one per half, into two accumulators)
// share each activation tile, so activations stream from L2 once per 256
// weight rows instead of once per 128.
template <int FMT, int XT, int H>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap wmap, const __grid_constant__ CUtensorMap xmap,
                   const GemmArgs a) {
    constexpr int CB = GemmFmt<FMT>::chunk_bytes;
    constexpr uint32_t AH_BYTES = (uint32_t)gemm_a_bytes();       // one half's k-block tile
    constexpr uint32_t A_BYTES = H * AH_BYTES;
    constexpr uint32_t PH_BYTES = (uint32_t)GEMM_WROWS * CB;      // one half's packed chunk
    constexpr uint32_t P_BYTES = H * PH_BYTES;
    constexpr int WR = H * GEMM_WROWS;                            // weight rows per tile
    // dequantized k-blocks per batch (one proxy fence and warp barrier per batch):
    // two when the A ring has 4 stages, one with the 2-stage ring of 256-row tiles
    constexpr int BATCH = H == 1 ? 2 : 1;
    const int BN = a.bn;
    const uint32_t B_BYTES = (uint32_t)gemm_b_bytes(BN);
    const uint32_t BS_BYTES = (uint32_t)gemm_bstage_bytes(BN);
    const int NBUF = gemm_nbuf(H, BN);
    const uint32_t TMEM_COLS = gemm_tmem_cols(H, BN);
    const uint32_t BUF_COLS = TMEM_COLS / (uint32_t)NBUF;          // columns per accumulator buffer
    const uint32_t IDESC = umma_idesc_f16(XT == X_F16 ? 0 : 1, GEMM_WROWS, BN);

    extern __shared__ uint8_t smem_raw[];
    // 1024-byte aligned base (128-byte swizzle atoms)
    const uint32_t raw_addr = smem_u32(smem_raw);
    uint8_t *smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
    const int SA = a.a_stages, SB = a.b_stages, P = a.p_stages;
    uint8_t *As = smem;
    uint8_t *Bs = As + (size_t)SA * A_BYTES;
    uint8_t *pk = Bs + (size_t)SB * BS_BYTES;
    uint64_t *bars = reinterpret_cast<uint64_t *>(pk + (((size_t)P * P_BYTES + 7) & ~(size_t)7));
    uint64_t *a_full = bars, *a_empty = bars + SA;
    uint64_t *b_full = bars + 2 * SA, *b_empty = bars + 2 * SA + SB;
    uint64_t *p_full = bars + 2 * SA + 2 * SB, *p_empty = p_full + P;
    uint64_t *acc_full = p_empty + P, *acc_empty = acc_full + 2;
    uint64_t *mma_done = acc_full + 4;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(mma_done + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // work items: (output tile, K slice); a tile's slices write fp32 partials when K is split
    const int n_items = a.n_wtiles * a.n_ttiles * a.splits;

    if (threadIdx.x == 0) {
        for (int s = 0; s < SA; ++s) {
            mbar_init(&a_full[s], GEMM_DQ_WARPS);
            mbar_init(&a_empty[s], 1);
        }
        for (int s = 0; s < SB; ++s) {
            mbar_init(&b_full[s], 1);
            mbar_init(&b_empty[s], 1);
        }
        for (int s = 0; s < P; ++s) {
            mbar_init(&p_full[s], 1);
            mbar_init(&p_empty[s], GEMM_DQ_WARPS);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&acc_full[s], 1);
            mbar_init(&acc_empty[s], GEMM_EPI_WARPS);
        }
        mbar_init(mma_done, 1);
        fence_mbar_init();
        pdl_launch_dependents();
    }
    if (warp == 1) {
        tmem_alloc(tmem_holder, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer: weights
        // Lane 0 streams the packed weight chunks (p ring) as far ahead as the ring
        // allows: a chunk is requested as soon as its slot frees.  The activation
        // k-blocks have their own producer warp (GEMM_ACT_WARP), so neither
        // producer's waits hold up the other's requests.  With row slots the
        // dequantizer warps fetch the weights themselves (this warp idles).
        bool slot_mode = false;
        if constexpr (FMT == F_Q6_K || FMT == F_Q2_K) slot_mode = a.slots != 0;
        if (lane == 0 && !slot_mode) {
            tma_prefetch_desc(&wmap);
            int ci = 0, ps = 0;
            uint32_t pph = 0;
            bool ok = true;
            for (int item = blockIdx.x; ok && item < n_items; item += gridDim.x) {
                const int tile = item / a.splits, ks = item % a.splits;
                const int wt = tile / a.n_ttiles;
                const int c0 = ks * a.cps, c1 = min(a.nchunks, c0 + a.cps);
                for (int c = c0; c < c1; ++c, ++ci) {
                    // Wq only: callers that allow overlap promise it is not written by preceding work
                    if (ci >= P && !(ok = mbar_wait(&p_empty[ps], pph ^ 1u, a.timeout_ns, DEVERR_GEMM_WAIT))) break;
                    mbar_arrive_expect_tx(&p_full[ps], P_BYTES);
                    // Q6_K, Q2_K: the box starts at the 16-byte boundary at or below the superblock
                    const int x0 = FMT == F_Q6_K ? (105 * c) & ~7 : (FMT == F_Q2_K ? (42 * c) & ~7 : c * (CB / 2));
#pragma unroll
                    for (int hh = 0; hh < H; ++hh)   // rows past N read zeros
                        tma_load_2d(pk + (size_t)ps * P_BYTES + hh * PH_BYTES, &wmap, &p_full[ps], x0,
                                    wt * WR + hh * GEMM_WROWS);
                    if (++ps == P) {
                        ps = 0;
                        pph ^= 1u;
                    }
                }
            }
            // drain: the last loads land before the CTA may exit (runs once; divisions are fine here)
            for (int j = max(0, ci - P); j < ci; ++j)
                mbar_wait(&p_full[j % P], (j / P) & 1, a.timeout_ns, DEVERR_GEMM_WAIT);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------- UMMA issuer
        if (lane == 0) {
            int ti = 0, sa = 0, sb = 0;
            uint32_t pha = 0, phb = 0;
            bool ok = true;
            for (int item = blockIdx.x; ok && item < n_items; item += gridDim.x, ++ti) {
                const int ks = item % a.splits;
                const int kbn = (min(a.nchunks, (ks + 1) * a.cps) - ks * a.cps) * GEMM_KB_PER_CHUNK;
                const int as = ti % NBUF, use = ti / NBUF;   // buffer, and how often it was used before
                if (use >= 1 && !(ok = mbar_wait(&acc_empty[as], (uint32_t)((use - 1) & 1), a.timeout_ns, DEVERR_GEMM_WAIT)))
                    break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)as * BUF_COLS;
                for (int k = 0; k < kbn; ++k) {
                    if (!(ok = mbar_wait(&b_full[sb], phb, a.timeout_ns, DEVERR_GEMM_WAIT))) break;
                    if (!(ok = mbar_wait(&a_full[sa], pha, a.timeout_ns, DEVERR_GEMM_WAIT))) break;
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(As + (size_t)sa * A_BYTES);
                    const uint32_t b_addr = smem_u32(Bs + (size_t)sb * BS_BYTES);
#pragma unroll
                    for (int kk = 0; kk < GEMM_BK / 16; ++kk)
#pragma unroll
                        for (int hh = 0; hh < H; ++hh)   // half hh accumulates at columns hh * BN of the buffer
                            umma_f16(d_tmem + (uint32_t)(hh * BN), umma_desc_sw128(a_addr + hh * AH_BYTES + kk * 32),
                                     umma_desc_sw128(b_addr + kk * 32), IDESC, (k | kk) ? 1u : 0u);
                    umma_commit(&a_empty[sa]);
                    umma_commit(&b_empty[sb]);
                    if (++sa == SA) {
                        sa = 0;
                        pha ^= 1u;
                    }
                    if (++sb == SB) {
                        sb = 0;
                        phb ^= 1u;
                    }
                }
                if (!ok) break;
                umma_commit(&acc_full[as]);
            }
            // every issued MMA completes before TMEM is released
            umma_commit(mma_done);
            mbar_wait(mma_done, 0, a.timeout_ns, DEVERR_GEMM_WAIT);
        }
    } else if (warp == GEMM_ACT_WARP) {
        // --------------------------------------------- TMA producer: activations
        // Lane 0 streams the activation k-blocks (b ring) as far ahead as it allows.
        if (lane == 0) {
            tma_prefetch_desc(&xmap);
            pdl_wait();   // x may be the preceding kernel's output
            int kbi = 0, s = 0;
            uint32_t ph = 0;
            bool ok = true;
            for (int item = blockIdx.x; ok && item < n_items; item += gridDim.x) {
                const int tile = item / a.splits, ks = item % a.splits;
                const int tt = tile % a.n_ttiles;
                const int k0 = ks * a.cps * GEMM_KB_PER_CHUNK;
                const int k1 = min(a.nchunks, (ks + 1) * a.cps) * GEMM_KB_PER_CHUNK;
                for (int k = k0; k < k1; ++k, ++kbi) {
                    if (kbi >= SB && !(ok = mbar_wait(&b_empty[s], ph ^ 1u, a.timeout_ns, DEVERR_GEMM_WAIT))) break;
                    mbar_arrive_expect_tx(&b_full[s], B_BYTES);
                    tma_load_2d(Bs + (size_t)s * BS_BYTES, &xmap, &b_full[s], k * GEMM_BK, tt * BN);
                    if (++s == SB) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
            }
            for (int j = max(0, kbi - SB); j < kbi; ++j)
                mbar_wait(&b_full[j % SB], (j / SB) & 1, a.timeout_ns, DEVERR_GEMM_WAIT);
        }
    } else if (warp < 2 + GEMM_DQ_WARPS) {
        // ------------------------------------------------------ dequantizers
        // Warp i of the 16 takes weight rows 8i..8i+7 of each half, all four (h, v) slices of each:
        // its packed-chunk loads then spread over the shared-memory banks (rows lie 144 bytes apart,
        // which a warp of 32 rows would fold onto 8 banks), and each quarter-warp's 16-byte stores
        // (8 rows, one chunk column) fall on distinct swizzled positions.
        const int t = threadIdx.x - 64;          // 0..511
        const int r = 8 * (t >> 5) + (t & 7);    // weight row within the half
        const int h = (t >> 3) & 1;              // which 32 of the k-block's 64 weights
        const int v = (t >> 4) & 1;              // which 16 of those 32
        int kbi = 0, s = 0, ps = 0;
        uint32_t ph = 0, pph = 0;
        bool ok = true;
        // the four k-blocks of one packed chunk (row r's superblock at prow)
        auto dequant_chunk = [&](uint32_t prow) {
            // BATCH k-blocks per batch; the A ring's depth is a multiple of BATCH, so a batch never wraps
            for (int kb = 0; kb < GEMM_KB_PER_CHUNK; kb += BATCH, kbi += BATCH) {
                if (kbi >= SA) {
#pragma unroll
                    for (int j = 0; j < BATCH; ++j)
                        if (ok && !(ok = mbar_wait(&a_empty[s + j], ph ^ 1u, a.timeout_ns, DEVERR_GEMM_WAIT))) break;
                    if (!ok) break;
                }
#pragma unroll
                for (int j = 0; j < BATCH; ++j)
#pragma unroll
                    for (int hh = 0; hh < H; ++hh)
                        Dequant<FMT, XT>::run(prow + hh * PH_BYTES, kb + j, h, v,
                                              smem_u32(As + (size_t)(s + j) * A_BYTES + hh * AH_BYTES), r);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
#pragma unroll
                    for (int j = 0; j < BATCH; ++j) mbar_arrive(&a_full[s + j]);
                }
                if ((s += BATCH) == SA) {
                    s = 0;
                    ph ^= 1u;
                }
            }
        };
        bool slot_mode = false;
        if constexpr (FMT == F_Q6_K || FMT == F_Q2_K) slot_mode = a.slots != 0;
        if (slot_mode) {
            if constexpr (FMT == F_Q6_K || FMT == F_Q2_K) {
                // Row slots: this warp's rows (8 of each half) are fetched by the warp itself, P - 1
                // chunks ahead along the CTA's (item, chunk) sequence, with 16-byte cp.async: a warp
                // reads only its own rows, so a warp barrier orders the copies and the reads.
                constexpr int SBB = FMT == F_Q6_K ? 210 : 84;           // superblock bytes
                constexpr int UMAX = (SBB + 15 + 15) / 16;              // 16-byte units a row's copy may take
                const uint8_t *wq = static_cast<const uint8_t *>(a.wq);
                const int w8 = 8 * (t >> 5);                            // the warp's first row
                int f_item = blockIdx.x, f_c = (blockIdx.x % a.splits) * a.cps;
                auto fetch = [&](int slot) {
                    if (f_item < n_items) {
                        const int wt_f = f_item / a.splits / a.n_ttiles;
                        // lane: row (lane >> 2) of the warp's 8 in each half, units (lane & 3) + 4 i of it
#pragma unroll
                        for (int hh = 0; hh < H; ++hh) {
                            const int rr = w8 + (lane >> 2);
                            const long n = min(wt_f * WR + hh * GEMM_WROWS + rr, a.N - 1);
                            const long b0 = n * a.row_bytes + (long)SBB * f_c;
                            const int o = (int)(b0 & 15);
                            const int units = (o + SBB + 15) / 16;
                            const uint8_t *src = wq + (b0 - o);
                            const uint32_t dst = smem_u32(pk) + (uint32_t)(slot * P_BYTES + hh * PH_BYTES + rr * CB);
#pragma unroll
                            for (int i = 0; i < (UMAX + 3) / 4; ++i) {
                                const int u = (lane & 3) + 4 * i;
                                if (u < units) cp_async_cg16(dst + 16 * u, src + 16 * u);
                            }
                        }
                        const int c1_f = min(a.nchunks, (f_item % a.splits) * a.cps + a.cps);
                        if (++f_c >= c1_f) {
                            f_item += gridDim.x;
                            f_c = (f_item % a.splits) * a.cps;
                        }
                    }
                    cp_async_commit();   // an empty group past the end keeps the counting uniform
                };
                for (int j = 0; j < P - 1; ++j) fetch(j);
                int seq = 0;
                for (int item = blockIdx.x; ok && item < n_items; item += gridDim.x) {
                    const int ks = item % a.splits;
                    const int wt = item / a.splits / a.n_ttiles;
                    const int c0 = ks * a.cps, c1 = min(a.nchunks, c0 + a.cps);
                    for (int c = c0; ok && c < c1; ++c, ++seq) {
                        fetch((seq + P - 1) % P);   // the slot the previous chunk freed
                        cp_async_wait_n(P - 1);     // this chunk's copies (this thread's) have landed
                        __syncwarp();               // ... and every lane's
                        const long n = min(wt * WR + r, a.N - 1);
                        const uint32_t off = (uint32_t)((n * a.row_bytes + (long)SBB * c) & 15);
                        dequant_chunk(smem_u32(pk) + (uint32_t)((seq % P) * P_BYTES + r * CB) + off);
                        __syncwarp();               // every lane is done with the slot before it is refilled
                    }
                }
                cp_async_wait<0>();                 // no copy still lands after the warp is done
            }
        } else {
            for (int item = blockIdx.x; ok && item < n_items; item += gridDim.x) {
                const int ks = item % a.splits;
                const int c0 = ks * a.cps, c1 = min(a.nchunks, c0 + a.cps);
                for (int c = c0; ok && c < c1; ++c) {
                    if (!(ok = mbar_wait(&p_full[ps], pph, a.timeout_ns, DEVERR_GEMM_WAIT))) break;
                    // (Q6_K, Q2_K: the superblock lies 2 * ((105 c) & 7), 2 * ((42 c) & 7) bytes into its box)
                    const uint32_t off = FMT == F_Q6_K ? 2u * (uint32_t)((105 * c) & 7)
                                                       : (FMT == F_Q2_K ? 2u * (uint32_t)((42 * c) & 7) : 0u);
                    dequant_chunk(smem_u32(pk) + (uint32_t)(ps * P_BYTES + r * CB) + off);
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&p_empty[ps]);
                    if (++ps == P) {
                        ps = 0;
                        pph ^= 1u;
                    }
                }
            }
        }
    } else {
        // --------------------------------------------------------- epilogue
        pdl_wait();              // y only after the preceding work completed
        const int q = warp & 3;  // TMEM lane quarter this warp may access
        const int N = a.N, M = a.M;
        int ti = 0;
        for (int item = blockIdx.x; item < n_items; item += gridDim.x, ++ti) {
            const int tile = item / a.splits, ks = item % a.splits;
            const int tt = tile % a.n_ttiles, wt = tile / a.n_ttiles;
            float *out = a.splits > 1 ? a.partial + (size_t)ks * M * N : a.y;
            const int as = ti % NBUF, use = ti / NBUF;
            if (!mbar_wait(&acc_full[as], (uint32_t)(use & 1), a.timeout_ns, DEVERR_GEMM_WAIT)) break;
            tc_fence_after();
#pragma unroll 1
            for (int hh = 0; hh < H; ++hh) {
                const int n = wt * WR + hh * GEMM_WROWS + q * 32 + lane;
                const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)as * BUF_COLS + (uint32_t)(hh * BN);
#pragma unroll 1
                for (int c0 = 0; c0 < BN; c0 += 32) {
                    uint32_t v[32];
                    if (BN - c0 >= 32) {
                        tmem_ld_32x32b_x32(taddr + c0, v);
                    } else {
                        tmem_ld_32x32b_x16(taddr + c0, *reinterpret_cast<uint32_t(*)[16]>(v));
#pragma unroll
                        for (int j = 16; j < 32; ++j) v[j] = 0u;
                    }
                    tmem_wait_ld();
                    const int m0 = tt * BN + c0;
                    const int mcols = min(32, BN - c0);
                    if (n < N) {
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            if (j < mcols && m0 + j < M) out[(size_t)(m0 + j) * N + n] = __uint_as_float(v[j]);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[as]);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

// ---------------------------------------------------------------- host side
// Formats with a tcgen05 GEMM decoder (all of them); gemm_eligible adds the
// conditions of their weight streams.
inline bool gemm_format(int wf) {
    return wf == LWQ_Q8_0 || wf == LWQ_Q4_0 || wf == LWQ_Q4_K || wf == LWQ_Q5_K || wf == LWQ_Q6_K || wf == LWQ_Q2_K;
}
// Q6_K (210-byte superblocks) and Q2_K (84) rows are 16-byte multiples, which a tensor map can take
// as its rows, when K % 2048 and K % 1024 == 0; other K stream as row slots (GemmArgs::slots), whose
// copies need the whole matrix to be 16-byte units
inline bool gemm_row_slots(int wf, long K) {
    return (wf == LWQ_Q6_K && K % 2048 != 0) || (wf == LWQ_Q2_K && K % 1024 != 0);
}
inline bool gemm_eligible(int wf, int xt, long N, long K) {
    if (!gemm_format(wf) || (xt != X_F16 && xt != X_BF16) || K % 256 != 0) return false;
    if (gemm_row_slots(wf, K)) return (N * (K / 256) * (wf == LWQ_Q6_K ? 210 : 84)) % 16 == 0;
    return true;
}

// bytes of one row of a packed chunk in a stage (Q6_K, Q2_K: their 240- and 96-byte boxes)
inline int gemm_chunk_bytes(int wf) {
    return wf == LWQ_Q8_0 ? 272 : (wf == LWQ_Q5_K ? 176 : (wf == LWQ_Q6_K ? 240 : (wf == LWQ_Q2_K ? 96 : 144)));
}

// Ring depths.  128-row tiles: 4 dequantized A stages (made on chip, two per
// batch), 3 packed chunk stages (each feeds four k-blocks; 2 when shared
// memory is short), and as many activation B stages as fit, up to 8 (B tiles
// arrive from L2 at ~60 bytes per cycle of a busy tensor pipe, so their ring
// covers the load latency).  256-row tiles: 2 A stages (one per batch) and 2
// chunk stages, the rest for B.  A forced stage count fixes the B ring.
constexpr int GEMM_A_STAGES = 4;   // 128-row tiles; even: the dequantizers fill two stages per batch
inline int gemm_a_stages(int h) { return h == 1 ? GEMM_A_STAGES : 2; }
inline bool gemm_rings(int cb, int bn, int h, const lwq_config *force, int *na, int *nb, int *np) {
    *na = gemm_a_stages(h);
    for (int p = h == 1 ? 3 : 2; p >= 2; --p) {
        int b = force && force->stages ? force->stages : 8;
        while (!(force && force->stages) && b > 2 && gemm_smem_bytes(cb, bn, h, *na, b, p) > 232448) --b;
        *nb = b;
        *np = p;
        if (gemm_smem_bytes(cb, bn, h, *na, b, p) <= 232448) return true;
    }
    return false;
}

// Modelled time (ns) of one k-block (64 of K) of a tile on one SM, the
// slowest of: shared-memory traffic at 128 B per cycle (the UMMAs' operand
// reads, the TMA writes of activations and packed weights, the dequantizers'
// reads and writes), the tensor pipe at this machine's measured bf16 rate per
// SM, the activation stream from L2 at its measured aggregate share, and the
// B ring's cover of the L2 latency.
inline double gemm_kblock_ns(int cb, int bn, int h, int nb) {
    const double smem = h * (16384.0 + bn * 128.0) + bn * 128.0 + h * 128.0 * cb / 4.0 * 2.0 + h * 16384.0;
    const double t_smem = smem / 243.0;        // 128 B/clk at 1.9 GHz
    const double t_mma = h * bn * 1.46;        // 2*128*bn*64 flops at 11.2 TFLOP/s
    const double t_l2 = bn * 128.0 / 81.0;     // ~12 TB/s over 148 SMs
    const double t_lat = 1000.0 / nb;          // ~1 us of L2 latency over nb stages
    double t = t_smem;
    if (t_mma > t) t = t_mma;
    if (t_l2 > t) t = t_l2;
    if (t_lat > t) t = t_lat;
    return t;
}

inline int gemm_plan(int wf, int xt, int M, int N, int K, const lwq_config *force, int sms, GemmPlan *g) {
    (void)xt;
    const int nchunks = K / 256;
    const int cb = gemm_chunk_bytes(wf);
    // K slices for a tile count: split when the tiles fill at most half the SMs, keeping >= 4 chunks a slice
    auto slices = [&](long tiles) -> int {
        if (force && force->splits) return force->splits;
        if (2 * tiles > sms) return 1;
        long sp = (sms + tiles - 1) / tiles;
        if (sp > nchunks / 4) sp = nchunks / 4;
        return sp < 1 ? 1 : (int)sp;
    };
    if (force && force->tile_n && force->tile_n != 128 && force->tile_n != 256) return LWQ_ERR_UNSUPPORTED;
    if (force && force->tile_m && (force->tile_m < 32 || force->tile_m > 256 || force->tile_m % 16))
        return LWQ_ERR_UNSUPPORTED;
    // weight tile (128 or 256 rows) and token tile (a multiple of 16 from 32 to 256): the least
    // modelled time, rounds of the persistent grid x the time of one work item (a tile's K slice)
    double best = -1;
    int bh = 0, bn = 0;
    for (int h = 1; h <= 2; ++h) {
        if (force && force->tile_n && force->tile_n != 128 * h) continue;
        const int hi = force && force->tile_m ? force->tile_m : (M < 256 ? ((M + 15) / 16) * 16 : 256);
        const int lo = force && force->tile_m ? force->tile_m : 32;
        for (int c = hi; c >= lo; c -= 16) {
            int na = 0, nb = 0, np = 0;
            if (!gemm_rings(cb, c, h, force, &na, &nb, &np)) continue;
            const long tiles = (long)((N + 128 * h - 1) / (128 * h)) * ((M + c - 1) / c);
            const int sp = slices(tiles);
            const long rounds = (tiles * sp + sms - 1) / sms;
            const double kbs = (double)((nchunks + sp - 1) / sp) * GEMM_KB_PER_CHUNK;
            double item = kbs * gemm_kblock_ns(cb, c, h, nb) + 1500.0;
            if (gemm_nbuf(h, c) == 1 && rounds > 1) item += h * c * 512.0 / 100.0;   // epilogue not overlapped
            const double cost = (double)rounds * item;
            if (best < 0 || cost < best * 0.999) {
                best = cost;
                bh = h;
                bn = c;
            }
        }
    }
    if (!bh) return LWQ_ERR_UNSUPPORTED;
    int na = 0, nb = 0, np = 0;
    if (!gemm_rings(cb, bn, bh, force, &na, &nb, &np) || nb < 2) return LWQ_ERR_UNSUPPORTED;
    const int tiles = ((N + 128 * bh - 1) / (128 * bh)) * ((M + bn - 1) / bn);
    int splits = slices(tiles);
    if (splits < 1 || splits > nchunks) return LWQ_ERR_UNSUPPORTED;
    const int cps = (nchunks + splits - 1) / splits;
    splits = (nchunks + cps - 1) / cps;   // drop empty slices
    const int items = tiles * splits;
    int ctas = force && force->ctas ? force->ctas : sms;
    if (ctas > items) ctas = items;
    if (ctas < 1) ctas = 1;
    g->splits = splits;
    g->warps = GEMM_DQ_WARPS;
    g->stages = nb;
    g->ctas = ctas;
    g->tile_n = 128 * bh;
    g->tile_m = bn;
    g->smem = gemm_smem_bytes(cb, bn, bh, na, nb, np);
    return LWQ_OK;
}

}  // namespace lwq

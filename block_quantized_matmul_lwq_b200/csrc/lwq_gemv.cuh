// Decode GEMV (M <= 16): y[M,N] = x[M,K] . dequant(Wq)^T, exact in x.
//
// Design (sm_100a):
//  * A persistent grid of one CTA per SM per call (16 compute warps, a TMA
//    producer and two or four reducers).  Every CTA triggers its programmatic dependents
//    at once, so the next call on the stream (a programmatic dependent
//    launch) is scheduled as early as possible and takes each SM as soon as
//    this call's CTA there exits.
//  * CTA (split s, row group r) owns a slice of K (split-K factor S) and
//    walks the 16-row weight tiles r, r+G, r+2G, ...  A producer warp stages,
//    per tile, the tile's packed rows for all of the CTA's K chunks (256
//    weights each) with one 3-D TMA load into a ring of shared-memory stages
//    (Q6_K: one 2-D box per chunk; row slots: one box per row).
//  * Sixteen compute warps each own 256 (or 128) weights of the CTA's K slice
//    and keep that slice of x in registers for the whole kernel, laid out as
//    tensor-core B fragments.  Per tile a warp decodes its packed bytes in
//    registers straight into A fragments holding the codes exactly (q - 8 for
//    Q4_0, q for Q8_0, q - 32 for Q6_K, the unsigned code for Q4_K, Q5_K and
//    Q2_K) and runs one
//    two-step mma.sync chain per 32-weight block, then adds d_block * chain
//    into its fp32 accumulators.  A code of zero weight therefore contributes
//    exactly nothing, however large the activation it meets.
//  * Activations reach the MMA exactly.  fp16 x: fp16 MMA, x as it is.  bf16
//    x: bf16 MMA, x as it is.  fp32 x: bf16 MMA with x split into three bf16
//    parts hi + mid + lo, which together hold all 24 significand bits (each
//    part is a truncation, so the split is exact).  The parts are separate
//    MMA columns: column c of the B operand is activation row c / P, part
//    c % P (P = 3 for fp32, else 1); 8 columns per n8 tile.  bf16 keeps fp32's
//    exponent range, so no element of x is crushed by its neighbours.  fp32
//    and bf16 x whose largest element in a warp's slice is far outside
//    [2^-60, 2^60] are scaled by a power of two first (exact), and the scale
//    is undone on the fp32 results.
//  * Q4_K (Q5_K, Q2_K): per sub-block j, y += (d * sc_j) * (sum q x) in fp32
//    (d * sc_j is exact in fp32), and once per tile y -= dmin * sum_j m_j S_j
//    with S_j the sub-block sums of x (kept in shared memory), as three bf16
//    MMAs with S split into exact parts.
//  * Two reducer warps (8 rows each; four of 4 rows for Q4_0 and Q8_0 at three
//    column tiles) sum the compute warps' partial tiles in a fixed order
//    and the parts of each activation row, and writes y, or, with split-K,
//    fp32 partials to the workspace, which a small follow-up kernel (a
//    programmatic dependent launch) adds in split order.  Results are
//    bitwise deterministic.
//
// This is the matrix-vector half of the co-designed dequantization in
// "Resumo Tecnico: Llamas na Web", "3. Design de Shader Consciente de
// Quantizacao" (decode directly in registers), with tensor cores and
// asynchronous memory loads (the native advantages named in its "Desempenho
// Nativo vs. Navegador" result).
#pragma once

#include "lwq_ptx.cuh"

namespace lwq {

// F_Q6_KS: Q6_K rows that are not 16-byte multiples, streamed as row slots
enum { F_Q8_0 = 1, F_Q4_0 = 2, F_Q4_K = 3, F_Q6_K = 4, F_Q5_K = 5, F_Q2_K = 6, F_Q6_KS = 7 };
enum { X_F32 = 0, X_F16 = 1, X_BF16 = 2 };

constexpr int GEMV_ROWS = 16;                     // weight rows per tile (the MMA's M)
constexpr int CHUNK = 256;                        // weights per TMA chunk of a row
constexpr int GEMV_W = 16;                        // compute warps per CTA
// Reducer warps: two (rows 8j .. 8j + 7 each), or four (rows 4j .. 4j + 3) for
// the one-scale formats at three n8 tiles (fp32 x with 6..8 activation rows),
// where the reduction is then the longest stage of a tile.  Four reducers make
// 21 warps, which caps every thread at 80 registers: the K-quant decoders spill
// there and lose more than the shorter reduction gains.
__host__ __device__ constexpr int gemv_red(int fmt, int nt) {
    return nt == 3 && (fmt == F_Q4_0 || fmt == F_Q8_0) ? 4 : 2;
}
__host__ __device__ constexpr int gemv_threads(int fmt, int nt) { return (GEMV_W + 1 + gemv_red(fmt, nt)) * 32; }
constexpr int GEMV_RSTAGES = 2;                   // depth of the reduction-slot ring

template <int FMT>
struct FmtInfo;
template <>
struct FmtInfo<F_Q8_0> { static constexpr int chunk_bytes = 272; };
template <>
struct FmtInfo<F_Q4_0> { static constexpr int chunk_bytes = 144; };
template <>
struct FmtInfo<F_Q4_K> { static constexpr int chunk_bytes = 144; };
template <>
struct FmtInfo<F_Q5_K> { static constexpr int chunk_bytes = 176; };
// Q6_K superblocks are 210 bytes, not a 16-byte multiple: each chunk is its own
// TMA box of 120 16-bit words (240 bytes) starting at the 16-byte boundary at
// or below the superblock, which lies 2 * ((105 c) & 7) bytes into the box.
template <>
struct FmtInfo<F_Q6_K> { static constexpr int chunk_bytes = 240; };
// Q2_K superblocks are 84 bytes: a row of K = 11008 (3612 bytes) is not a
// 16-byte multiple, so no tensor map can take the rows as its second
// dimension.  Its weights stream as row slots instead (fmt_row_slots).
template <>
struct FmtInfo<F_Q2_K> { static constexpr int chunk_bytes = 84; };
template <>
struct FmtInfo<F_Q6_KS> { static constexpr int chunk_bytes = 210; };
// Formats with a per-sub-block min (the S_j sums of x enter the result), and
// the number of those sums per 256-weight chunk (sub-blocks of 32 or 16).
__host__ __device__ constexpr int fmt_sums(int fmt) {
    return (fmt == F_Q4_K || fmt == F_Q5_K) ? 8 : (fmt == F_Q2_K ? 16 : 0);
}
__host__ __device__ constexpr bool fmt_has_min(int fmt) { return fmt_sums(fmt) > 0; }
// Row slots: the weight matrix is read as one flat array of 16-byte units (a
// tensor map of [bytes / 16][16]); per stage, row r of the tile is one box of
// whole units into its own 128-byte aligned slot, starting r mod 8 units before
// the unit that holds the row's first byte of the split.  The slice then lies
// 16 (r mod 8) + ((n rb + cb c) mod 16) bytes into the slot, and the 8 rows
// that a warp's lane groups read at once fall on distinct bank quads.  The
// second term is 0, 4, 8 or 12 for Q2_K (cb = 84), so its 32-bit words stay
// aligned; Q6_K (cb = 210) may start 2 bytes off a word.
__host__ __device__ constexpr bool fmt_row_slots(int fmt) { return fmt == F_Q2_K || fmt == F_Q6_KS; }
__host__ __device__ constexpr int gemv_slot_units(int chunk_bytes, int cps) {   // units per row box
    return (chunk_bytes * cps + 15 + 15) / 16 + 7;
}
__host__ __device__ constexpr int gemv_slot_bytes(int chunk_bytes, int cps) {   // slot stride
    return (16 * gemv_slot_units(chunk_bytes, cps) + 127) / 128 * 128;
}

struct GemvArgs {
    const void *x;
    float *y;
    float *partial;       // [S][M][N] fp32 (split-K only; gemv_splitk_sum_kernel adds the splits)
    int M, N, K;
    int nchunks;          // K / 256
    int splits;           // S
    int cps;              // chunks per split (the depth of one TMA box)
    int row_tiles;        // ceil(N / 16)
    int wstages;          // weight ring depth
    unsigned long long timeout_ns;
    int overlap;          // host side: launch with programmatic stream serialization
};

// Activation parts per element: fp32 x is split into three bf16 parts.
__host__ __device__ constexpr int gemv_parts(int xt, bool i8) { return (xt == X_F32 && !i8) ? 3 : 1; }
// Weights of K per compute warp: one chunk with up to two n8 column tiles,
// half a chunk with three (their B fragments take 32 registers per tile and
// chunk).  A whole chunk per warp means fewer, larger tiles per CTA and K up
// to 4096 in one CTA (no split-K): measured faster at two tiles even with a
// few registers spilled (fp32, M = 4: 17.2 -> 14.4 us).  The planner takes
// half a chunk at two tiles too when a CTA's K slice has 8 chunks or fewer,
// which a warp per chunk would leave to half the warps.
__host__ __device__ constexpr int gemv_kw(int nt) { return nt <= 2 ? 256 : 128; }
// Floats per row of a reduction slot: the tile's 8 NT columns and 4 of padding,
// which spreads the rows of a slot over the shared-memory banks.
__host__ __device__ constexpr int gemv_rs(int nt) { return 8 * nt + 4; }

// Padding (16-bit elements) after each row of the activation planes: with K
// slices of whole chunks it makes the row stride 8 words mod 32, so four rows
// in a row fall on distinct bank groups (the split planes also swap the two
// words of each pair in rows 4-7 of every 8, which separates the next four).
constexpr int GEMV_XPAD = 16;

// Shared-memory layout (bytes): ring | the CTA's slice of x | reduction slots |
// Q4_K sub-block sums of x | reducer scratch | CTA maximum | mbarriers.
//  * The slice of x (fp path): P planes [part][activation row][K slice + pad]
//    of 16-bit values -- the bf16 parts of fp32 x, or 16-bit x as it is.
//    Int8 activation blocks stage the raw slice [row][K slice].
//  * The K-quant sums: [activation row][sub-block of the slice] fp32 (sub-blocks
//    of 32 weights; Q2_K: 16).
struct GemvSmem {
    size_t stage, slot, tx, ring, xs, red, sx, scratch, xmax, bars, total;   // tx: bytes a stage's loads bring
};
__host__ __device__ inline GemvSmem gemv_smem_layout(int chunk_bytes, int cps, int wstages, int nt, int sums,
                                                     int parts, int m, int xelem, bool i8, bool slots) {
    GemvSmem s;
    s.slot = slots ? (size_t)gemv_slot_bytes(chunk_bytes, cps) : 0;
    s.stage = slots ? GEMV_ROWS * s.slot : (size_t)cps * GEMV_ROWS * chunk_bytes;
    s.tx = slots ? (size_t)GEMV_ROWS * 16 * gemv_slot_units(chunk_bytes, cps) : s.stage;
    s.ring = (size_t)wstages * s.stage;
    s.xs = i8 ? (size_t)m * cps * CHUNK * xelem : (size_t)parts * m * (cps * CHUNK + GEMV_XPAD) * 2;
    s.xs = (s.xs + 15) & ~(size_t)15;
    s.red = (size_t)GEMV_RSTAGES * GEMV_W * GEMV_ROWS * gemv_rs(nt) * 4;
    s.sx = (size_t)m * cps * sums * 4;
    s.scratch = parts > 1 ? (size_t)GEMV_ROWS * gemv_rs(nt) * 4 : 0;
    s.xmax = 16 * 4;
    s.bars = (size_t)(2 * wstages + 2 * GEMV_RSTAGES + 1) * 8;
    s.total = s.ring + s.xs + s.red + s.sx + s.scratch + s.xmax + s.bars;
    return s;
}

// --------------------------------------------------------------- constants
constexpr uint32_t H2_ONE = 0x3C003C00u;
constexpr uint32_t H2_SIXTEENTH = 0x2C002C00u;
constexpr uint32_t H2_MAGIC = 0x64006400u;   // 1024
constexpr uint32_t H2_M1032 = 0xE408E408u;   // -1032
constexpr uint32_t H2_M72 = 0xD480D480u;     // -72
constexpr uint32_t H2_M1024 = 0xE400E400u;   // -1024
constexpr uint32_t H2_M64 = 0xD400D400u;     // -64
constexpr uint32_t H2_M1152 = 0xE480E480u;   // -1152
constexpr uint32_t B2_ONE = 0x3F803F80u;
constexpr uint32_t B2_MAGIC = 0x43004300u;   // 128
constexpr uint32_t B2_M136 = 0xC308C308u;    // -136
constexpr uint32_t B2_M128 = 0xC300C300u;    // -128
constexpr uint32_t B2_M128_OR_256 = 0xC300C300u;   // -128, or -256 with bit 7 of each half set

// ----------------------------------------------------------- code decode
// Each decoder turns two codes of a 32-bit code word (bytes 0 and 2, or with
// the word shifted right by 8, bytes 1 and 3) into a packed pair of exact
// fp16 or bf16 values.  Magic-number decodes: for fp16, 0x6400 | v is 1024 + v
// for v < 1024; for bf16, 0x4300 | v is 128 + v for v < 128.  One LOP3 and
// one packed FMA per two codes (bf16 nibbles in bits 4-7 need a shift first,
// since bit 7 of a bf16 half is an exponent bit).
template <bool BF>
__device__ __forceinline__ uint32_t q40_lo(uint32_t w) {   // low nibbles, minus 8
    if constexpr (BF) return hfma2_bf16(and_or(w, 0x000F000Fu, B2_MAGIC), B2_ONE, B2_M136);
    else return hfma2_f16(and_or(w, 0x000F000Fu, H2_MAGIC), H2_ONE, H2_M1032);
}
template <bool BF>
__device__ __forceinline__ uint32_t q40_hi(uint32_t w) {   // high nibbles, minus 8
    if constexpr (BF) return hfma2_bf16(and_or(w >> 4, 0x000F000Fu, B2_MAGIC), B2_ONE, B2_M136);
    else return hfma2_f16(and_or(w, 0x00F000F0u, H2_MAGIC), H2_SIXTEENTH, H2_M72);   // (1024+16q)/16 - 72
}
template <bool BF>
__device__ __forceinline__ uint32_t q4k_lo(uint32_t w) {   // low nibbles, unsigned
    if constexpr (BF) return hfma2_bf16(and_or(w, 0x000F000Fu, B2_MAGIC), B2_ONE, B2_M128);
    else return hfma2_f16(and_or(w, 0x000F000Fu, H2_MAGIC), H2_ONE, H2_M1024);
}
template <bool BF>
__device__ __forceinline__ uint32_t q4k_hi(uint32_t w) {   // high nibbles, unsigned
    if constexpr (BF) return hfma2_bf16(and_or(w >> 4, 0x000F000Fu, B2_MAGIC), B2_ONE, B2_M128);
    else return hfma2_f16(and_or(w, 0x00F000F0u, H2_MAGIC), H2_SIXTEENTH, H2_M64);
}
// Q6_K: the 6-bit codes of bytes 0 and 2, minus 32.
template <bool BF>
__device__ __forceinline__ uint32_t q6k_pair(uint32_t v) {
    if constexpr (BF) return hfma2_bf16(and_or(v, 0x003F003Fu, B2_MAGIC), B2_ONE, 0xC320C320u);   // 128 + v - 160
    else return hfma2_f16(and_or(v, 0x003F003Fu, H2_MAGIC), H2_ONE, 0xE420E420u);                 // 1024 + v - 1056
}
// Q5_K: the 5-bit codes of bytes 0 and 2, unsigned.
template <bool BF>
__device__ __forceinline__ uint32_t q5k_pair(uint32_t v) {
    if constexpr (BF) return hfma2_bf16(and_or(v, 0x001F001Fu, B2_MAGIC), B2_ONE, B2_M128);
    else return hfma2_f16(and_or(v, 0x001F001Fu, H2_MAGIC), H2_ONE, H2_M1024);
}
// Q2_K: the 2-bit codes in bits 0-1 of bytes 0 and 2, unsigned.
template <bool BF>
__device__ __forceinline__ uint32_t q2k_pair(uint32_t v) {
    if constexpr (BF) return hfma2_bf16(and_or(v, 0x00030003u, B2_MAGIC), B2_ONE, B2_M128);
    else return hfma2_f16(and_or(v, 0x00030003u, H2_MAGIC), H2_ONE, H2_M1024);
}
// Q4_K / Q5_K: two 6-bit mins (bits 0-5 of each half) as exact bf16 values.
__device__ __forceinline__ uint32_t min6_pair_bf16(uint32_t v) {
    return hfma2_bf16(and_or(v, 0x003F003Fu, B2_MAGIC), B2_ONE, B2_M128);
}
// Q8_0: the int8 codes of bytes 0 and 2.  fp16: (1024 + (q + 128)) - 1152.
// bf16 has room for 7 bits only: (128 + (q & 127)) plus -128 or -256 from the
// sign bit, which lands on the exponent bit of 0xC300 (0xC380 is -256).
template <bool BF>
__device__ __forceinline__ uint32_t q80_pair(uint32_t w) {
    if constexpr (BF) return hfma2_bf16(and_or(w, 0x007F007Fu, B2_MAGIC), B2_ONE, and_or(w, 0x00800080u, B2_M128_OR_256));
    else return hfma2_f16(and_or(w ^ 0x00800080u, 0x00FF00FFu, H2_MAGIC), H2_ONE, H2_M1152);
}

// D = A.B (C = 0) and D += A.B, bf16 or fp16 operands, fp32 accumulate.
template <bool BF>
__device__ __forceinline__ void mma_zero(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    if constexpr (BF)
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
            "{%10,%10,%10,%10};"
            : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(0.f));
    else
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
            "{%10,%10,%10,%10};"
            : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(0.f));
}
template <bool BF>
__device__ __forceinline__ void mma_acc(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    if constexpr (BF) mma_bf16_16816(d, a, b0, b1, d);
    else mma_f16_16816(d, a, b0, b1, d);
}

// fp32 value (an exact bf16 value, or a truncation of one) whose top 16 bits
// are the bf16 code.
__device__ __forceinline__ float trunc_bf16(float v) { return __uint_as_float(__float_as_uint(v) & 0xFFFF0000u); }

// 2^23 + byte jj of v as fp32: PRMT into the fp32 pattern 0x4B0000xx.
__device__ __forceinline__ float byte_magic(uint32_t v, int jj) {
    return __uint_as_float(prmt(v, 0x4B000000u, 0x7650u | (uint32_t)jj));
}

// ------------------------------------------------------------- exact fp path
// Element layout of a lane's B fragments.  For block b of the chunk (32
// weights; a Q4_K sub-block), MMA step h (16 weights) and lane t, the lane's
// four k-slots 2t, 2t+1, 2t+8, 2t+9 carry the weights of bytes j = 0, 2, 1, 3
// of its code word (so one mask takes bytes 0 and 2 and the same mask after
// an 8-bit shift takes bytes 1 and 3).  Bytes (0, 1) and (2, 3) of the word
// are consecutive elements; elem() is the element of byte 2q.
//  * Q4_K, and odd blocks of Q4_0 and Q8_0 (word-aligned codes): the word is
//    code bytes 16h + 4t .. (Q8_0) or 4t .. (Q4_0: low nibbles are step 0,
//    high nibbles elements + 16 in step 1).  Q4_K nibbles come from the
//    32-byte group of sub-blocks 2g (low) and 2g + 1 (high).
//  * Even blocks of Q4_0 and Q8_0 start 2 bytes into a word: lane t reads the
//    aligned word that holds code bytes 4i - 2 .. 4i + 1 (i = t, or 4h + t for
//    Q8_0), and the first lane, whose word would hold the block scale, takes
//    the last two code bytes of the block in its place (one PRMT).
template <int FMT>
__device__ __forceinline__ int elem(int bb, int h, int t, int q) {
    if (FMT == F_Q4_K || FMT == F_Q5_K || FMT == F_Q6_K || FMT == F_Q6_KS || FMT == F_Q2_K || (bb & 1))
        return 32 * bb + 16 * h + 4 * t + 2 * q;
    if (FMT == F_Q4_0) return 32 * bb + 16 * h + ((4 * t - 2 + 2 * q) & 15);
    return 32 * bb + ((16 * h + 4 * t - 2 + 2 * q) & 31);
}

template <int FMT, int XT, int NT, int KW>
struct Exact {
    static constexpr bool BF = (XT != X_F16);
    static constexpr int P = gemv_parts(XT, false);
    static constexpr int NB = KW / 32;       // blocks (Q4_K: sub-blocks) per warp
    static constexpr int CB = FmtInfo<FMT>::chunk_bytes;
    uint32_t xf[NT][NB][2][2];               // [tile][block][step][reg]
    float inv;                               // 1 / the activation scale (a power of two)
    uint32_t q6o = 0;                        // Q6_K: byte offset of the superblock in its chunk box
    uint32_t sr0 = 0, sr1 = 0;               // row slots: the superblock in rows g and g + 8 of the stage

    // ---------------------------------------------------------- prologue
    // The CTA's slice of x is prepared once, by all nact compute warps
    // together (thread i of nthr), into the part planes in shared memory;
    // then every warp loads its B fragments from them.  Returns false when a
    // bounded wait gave up.
    //  * fp32 x: loaded from global memory (after the wait for the preceding
    //    kernel), each element once, split into hi / mid / lo bf16 parts.
    //  * 16-bit x: the reducer's bulk copies stage it in plane 0 as it is.
    //  * Scale: the CTA's largest |x| far outside [2^-60, 2^60] (and finite)
    //    scales the slice by a power of two (exact), undone on the results.
    //  * Q4_K: the sub-block sums S_j of the (scaled) slice go to sx.
    // Plane rows: row m * P + p holds part p of activation row m (the 8
    // columns of an n8 tile are 8 consecutive plane rows).  Split planes (fp32
    // x) swap the words of each word pair in rows r with r & 4 set (bank
    // spread); staged 16-bit rows lie as copied.
    struct Slice {
        uint16_t *xp;    // plane rows [M * P][rs]
        float *sx;       // Q4_K sums [M][nk / 32]
        float *xmax;     // 16 per-warp maxima
        int M, nk, rs;   // rows, K slice, plane row stride (16-bit elements)
    };
    __device__ static __forceinline__ int swz(int r) { return (P > 1 && (r & 4)) ? 2 : 0; }   // element offset XOR

    // bf16 bits of the three parts of v (truncations: hi + mid + lo == v)
    __device__ static __forceinline__ void split3(float v, uint32_t &hi, uint32_t &mid, uint32_t &lo) {
        const uint32_t h = __float_as_uint(v) & 0xFFFF0000u;
        const float r = v - __uint_as_float(h);   // exact
        const uint32_t md = __float_as_uint(r) & 0xFFFF0000u;
        const float l = r - __uint_as_float(md);  // exact, at most 8 significant bits
        hi = h >> 16;
        mid = md >> 16;
        lo = __float_as_uint(l) >> 16;
    }

    // CTA-wide maximum of the threads' mx: per-warp maxima in shared memory, one named barrier.
    __device__ static __forceinline__ float cta_max(float mx, const Slice &S, int nact, int warp, int lane) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        if (lane == 0) S.xmax[warp] = mx;
        named_bar_sync(1, nact * 32);
        float m = 0.f;
        for (int w = 0; w < nact; ++w) m = fmaxf(m, S.xmax[w]);
        return m;
    }

    // Power-of-two scale that puts m in [1, 2), or 1 when m is in range, zero or not finite.
    __device__ static __forceinline__ float pick_scale(float m, float &inv_out) {
        inv_out = 1.f;
        if (!(m > 0.f && m <= 3.0e38f && (m < 8.673617e-19f || m > 1.1529215e18f))) return 1.f;
        const int e = (int)((__float_as_uint(m) >> 23) & 0xFF) - 127;
        const int es = e < -126 ? 126 : (e > 126 ? -126 : -e);
        inv_out = __uint_as_float((uint32_t)(127 - es) << 23);
        return __uint_as_float((uint32_t)(127 + es) << 23);
    }

    // Q4_K: the sum of a 32-element sub-block lies in 8 consecutive lanes (4
    // elements each; a group of 8 lanes is valid or not as a whole).
    // Q2_K: of a 16-element sub-block, in 4 consecutive lanes.
    __device__ static __forceinline__ void store_sum(float v, const Slice &S, long e, bool ok, int lane) {
        v += __shfl_xor_sync(0xffffffffu, v, 1);
        v += __shfl_xor_sync(0xffffffffu, v, 2);
        if constexpr (FMT == F_Q2_K) {
            if (ok && (lane & 3) == 0) S.sx[e / 16] = v;   // row-major [M][nk/16] == element index / 16
        } else {
            v += __shfl_xor_sync(0xffffffffu, v, 4);
            if (ok && (lane & 7) == 0) S.sx[e / 32] = v;   // row-major [M][nk/32] == element index / 32
        }
    }

    // |v| outside [2^-60, 2^60] and not zero (or not finite): the slice needs the power-of-two scale
    __device__ static __forceinline__ bool out_of_range(float v) {
        const float a = fabsf(v);
        return a != 0.f && !(a >= 8.673617e-19f && a <= 1.1529215e18f);
    }

    // hi / mid / lo bf16 parts of (a, b), each packed as one register (a in the low half)
    __device__ static __forceinline__ void split_pair(float a, float b, uint32_t &hi, uint32_t &mid, uint32_t &lo) {
        const uint32_t ha = __float_as_uint(a) & 0xFFFF0000u, hb = __float_as_uint(b) & 0xFFFF0000u;
        // a - hi and r - mid as packed fp32 FMAs with -1 (exact: the results are representable)
        const float2 r = __ffma2_rn(make_float2(__uint_as_float(ha), __uint_as_float(hb)), make_float2(-1.f, -1.f),
                                    make_float2(a, b));
        const uint32_t ma = __float_as_uint(r.x) & 0xFFFF0000u, mb = __float_as_uint(r.y) & 0xFFFF0000u;
        const float2 l = __ffma2_rn(make_float2(__uint_as_float(ma), __uint_as_float(mb)), make_float2(-1.f, -1.f), r);
        hi = prmt(ha, hb, 0x7632u);
        mid = prmt(ma, mb, 0x7632u);
        lo = prmt(__float_as_uint(l.x), __float_as_uint(l.y), 0x7632u);
    }

    __device__ __forceinline__ bool prologue(const GemvArgs &a, const Slice &S, int c_begin, uint64_t *xfull,
                                             int nact, int warp, int lane, unsigned long long timeout) {
        const int nthr = nact * 32, tid = warp * 32 + lane;
        // 4-element units of fp32 x per thread: M * nk / 4 over nact warps with
        // nact * KW = nk, i.e. 2M with a chunk per warp and M with half a chunk,
        // M being at most 8 NT / P for this kernel
        constexpr int VPT = (8 * NT / P) * (KW == CHUNK ? 2 : 1);
        int *flag = reinterpret_cast<int *>(S.xmax + 15);   // set (to 1) when a rescale is needed
        inv = 1.f;
        if constexpr (XT == X_F32) {
            pdl_wait();   // x may be the preceding kernel's output
            // thread tid takes units tid, tid + nthr, ... in row-major order: (row, unit in row)
            // advance without divisions
            const int upr = S.nk / 4, nu = S.M * upr;
            const int dm = nthr / upr, dk = nthr % upr;
            int m = tid / upr, k4 = tid % upr;
            float4 v[VPT];
            int mk[VPT];   // m << 16 | unit in row
            // every load is issued before any value is used, so they are all in flight
            // at once; a unit past the end reloads the thread's first unit (always one of
            // the slice: M * nk / 4 >= nthr) and is zeroed below
            const float *xb = static_cast<const float *>(a.x) + (long)c_begin * CHUNK;
            const long first = (long)m * a.K + 4 * k4;
#pragma unroll
            for (int j = 0; j < VPT; ++j) {
                mk[j] = (m << 16) | k4;
                const bool ok = j * nthr + tid < nu;
                v[j] = __ldcg(reinterpret_cast<const float4 *>(xb + (ok ? (long)m * a.K + 4 * k4 : first)));
                k4 += dk;
                m += dm;
                if (k4 >= upr) {
                    k4 -= upr;
                    ++m;
                }
            }
            bool out = false;
#pragma unroll
            for (int j = 0; j < VPT; ++j) {
                if (j * nthr + tid >= nu) v[j] = make_float4(0.f, 0.f, 0.f, 0.f);
                out |= out_of_range(v[j].x) | out_of_range(v[j].y) | out_of_range(v[j].z) | out_of_range(v[j].w);
            }
            if (out) *flag = 1;
            // the planes (and Q4_K sums) of the slice scaled by sc
            auto emit = [&](float sc) {
#pragma unroll
                for (int j = 0; j < VPT; ++j) {
                    if (j * nthr >= nu) break;   // uniform across the CTA
                    const bool ok = j * nthr + tid < nu;
                    const int mm = mk[j] >> 16, k = 4 * (mk[j] & 0xFFFF);
                    const float4 w = make_float4(v[j].x * sc, v[j].y * sc, v[j].z * sc, v[j].w * sc);
                    if constexpr (fmt_has_min(FMT)) store_sum((w.x + w.y) + (w.z + w.w), S, (long)mm * S.nk + k, ok, lane);
                    if (ok) {
                        uint32_t pr[3][2];
                        split_pair(w.x, w.y, pr[0][0], pr[1][0], pr[2][0]);
                        split_pair(w.z, w.w, pr[0][1], pr[1][1], pr[2][1]);
#pragma unroll
                        for (int q = 0; q < 3; ++q) {
                            const int r = mm * P + q;
                            const bool sw = swz(r) != 0;   // words of the pair swapped
                            *reinterpret_cast<uint2 *>(S.xp + (size_t)r * S.rs + k) =
                                sw ? make_uint2(pr[q][1], pr[q][0]) : make_uint2(pr[q][0], pr[q][1]);
                        }
                    }
                }
            };
            emit(1.f);
            named_bar_sync(1, nthr);
            if (*flag) {
                // rare: the largest |x| of the CTA's slice sets a power-of-two scale; split again
                float mx = 0.f;
#pragma unroll
                for (int j = 0; j < VPT; ++j)
                    mx = fmaxf(mx, fmaxf(fmaxf(fabsf(v[j].x), fabsf(v[j].y)), fmaxf(fabsf(v[j].z), fabsf(v[j].w))));
                const float sc = pick_scale(cta_max(mx, S, nact, warp, lane), inv);
                if (sc != 1.f) {
                    emit(sc);
                    named_bar_sync(1, nthr);
                }
            }
        } else {
            if (!mbar_wait(xfull, 0, timeout, DEVERR_GEMV_WAIT)) return false;
            if constexpr (XT == X_BF16 || fmt_has_min(FMT)) {
                // 4-element units of plane 0 ([m][rs], nk / 4 units per row): the range check
                // (bf16), a rescale in place when needed (rare), and the Q4_K sums
                const int upr4 = S.nk / 4, nu4 = S.M * upr4;
                float sc = 1.f;
                if constexpr (XT == X_BF16) {
                    bool out = false;
                    for (int u = tid; u < nu4; u += nthr) {
                        const uint2 q = *reinterpret_cast<const uint2 *>(S.xp + (size_t)(u / upr4) * S.rs + 4 * (u % upr4));
                        out |= out_of_range(bf16_bits_to_float(q.x)) | out_of_range(bf16_bits_to_float(q.x >> 16)) |
                               out_of_range(bf16_bits_to_float(q.y)) | out_of_range(bf16_bits_to_float(q.y >> 16));
                    }
                    if (out) *flag = 1;
                    named_bar_sync(1, nthr);
                    if (*flag) {
                        float mx = 0.f;
                        for (int u = tid; u < nu4; u += nthr) {
                            const uint2 q = *reinterpret_cast<const uint2 *>(S.xp + (size_t)(u / upr4) * S.rs + 4 * (u % upr4));
                            mx = fmaxf(mx, fmaxf(fmaxf(fabsf(bf16_bits_to_float(q.x)), fabsf(bf16_bits_to_float(q.x >> 16))),
                                                 fmaxf(fabsf(bf16_bits_to_float(q.y)), fabsf(bf16_bits_to_float(q.y >> 16)))));
                        }
                        sc = pick_scale(cta_max(mx, S, nact, warp, lane), inv);
                    }
                }
                if (sc != 1.f || fmt_has_min(FMT)) {
                    for (int u0 = 0; u0 < nu4; u0 += nthr) {   // uniform trip count (shuffles inside)
                        const int u = u0 + tid;
                        const bool ok = u < nu4;
                        const int m = ok ? u / upr4 : 0, k = ok ? 4 * (u % upr4) : 0;
                        uint16_t *p = S.xp + (size_t)m * S.rs + k;
                        uint2 q = ok ? *reinterpret_cast<const uint2 *>(p) : make_uint2(0u, 0u);
                        float f[4];
                        if constexpr (XT == X_F16) {
                            f[0] = f16_lo(q.x); f[1] = f16_hi(q.x);
                            f[2] = f16_lo(q.y); f[3] = f16_hi(q.y);
                        } else {
                            f[0] = bf16_bits_to_float(q.x) * sc; f[1] = bf16_bits_to_float(q.x >> 16) * sc;
                            f[2] = bf16_bits_to_float(q.y) * sc; f[3] = bf16_bits_to_float(q.y >> 16) * sc;
                            if (sc != 1.f && ok)
                                *reinterpret_cast<uint2 *>(p) =
                                    make_uint2(prmt(__float_as_uint(f[0]), __float_as_uint(f[1]), 0x7632u),
                                               prmt(__float_as_uint(f[2]), __float_as_uint(f[3]), 0x7632u));
                        }
                        if constexpr (fmt_has_min(FMT)) store_sum((f[0] + f[1]) + (f[2] + f[3]), S, (long)m * S.nk + k, ok, lane);
                    }
                    named_bar_sync(1, nthr);
                }
            }
        }
        return true;
    }

    // This warp's B fragments from the planes: the chunk starts at element k0
    // of the slice, blocks half*NB ..
    __device__ __forceinline__ void load_frags(const Slice &S, int k0, int half, int lane) {
        const int g = lane >> 2, t = lane & 3;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int c = 8 * nt + g, m = c / P;
            const bool live = m < S.M;
            const int r = live ? c : 0;   // plane row m * P + p == column c
            const uint16_t *row = S.xp + ((size_t)r * S.rs + k0);
            const int sw = swz(r);
#pragma unroll
            for (int b = 0; b < NB; ++b)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    // unconditional loads (a dead column reads plane row 0), zeroed after:
                    // no load waits behind a branch on the previous one
                    uint32_t l0 = *reinterpret_cast<const uint32_t *>(row + (elem<FMT>(half * NB + b, h, t, 0) ^ sw));
                    uint32_t l1 = *reinterpret_cast<const uint32_t *>(row + (elem<FMT>(half * NB + b, h, t, 1) ^ sw));
                    l0 = live ? l0 : 0u;
                    l1 = live ? l1 : 0u;
                    // slots (2t, 2t+1) take bytes 0 and 2, slots (2t+8, 2t+9) bytes 1 and 3
                    xf[nt][b][h][0] = prmt(l0, l1, 0x5410u);
                    xf[nt][b][h][1] = prmt(l0, l1, 0x7632u);
                }
        }
    }

    // One block's chain: d * (A0 . B[step 0] + A1 . B[step 1]) into acc, for
    // every column tile; s0, s1 scale rows g and g + 8.
    __device__ __forceinline__ void block(const uint32_t (&a0)[4], const uint32_t (&a1)[4], int b, float s0, float s1,
                                          float (&acc)[NT][4]) const {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            float c[4];
            mma_zero<BF>(c, a0, xf[nt][b][0][0], xf[nt][b][0][1]);
            mma_acc<BF>(c, a1, xf[nt][b][1][0], xf[nt][b][1][1]);
            acc[nt][0] = fmaf(s0, c[0], acc[nt][0]);
            acc[nt][1] = fmaf(s0, c[1], acc[nt][1]);
            acc[nt][2] = fmaf(s1, c[2], acc[nt][2]);
            acc[nt][3] = fmaf(s1, c[3], acc[nt][3]);
        }
    }

    // Q6_K: 32-bit word at byte q6o + off of a row (q6o even; MIS: q6o = 2 mod 4,
    // the word straddles two aligned words)
    // Q6_K: 32-bit word at byte off of a superblock.  MIS 0 / 1: the superblock
    // starts q6o bytes into the row's chunk box, q6o = 0 / 2 mod 4 (one load, or
    // two aligned loads and a PRMT); MIS 2 (row slots): row is the superblock's
    // own address, even, with each row's alignment its own (two loads and a PRMT
    // whose selector follows the row).
    template <int MIS>
    __device__ __forceinline__ uint32_t q6w(uint32_t row, uint32_t off) const {
        if constexpr (MIS == 2) {
            const uint32_t a = (row + off) & ~3u;
            return prmt(lds32(a), lds32(a + 4), (row & 2) ? 0x5432u : 0x3210u);
        } else if constexpr (MIS == 1) {
            return prmt(lds32(row + q6o - 2 + off), lds32(row + q6o + 2 + off), 0x5432u);
        } else {
            return lds32(row + q6o + off);
        }
    }
    // Q6_K (210-byte superblock = the warp's chunk; with KW = 128 the warp takes
    // half `half` of it).  For half n and l0 in {0, 16}, lane t's words
    // A = ql[64n + l0 + 4t], B = ql[64n + 32 + l0 + 4t] and H = qh[32n + l0 + 4t]
    // give the 6-bit codes of elements 16j + 4t .. 16j + 4t + 3 of the four
    // sub-blocks j = 8n + 2g + l0/16 (g = 0..3: low nibbles of A, of B, high
    // nibbles of A, of B; high bits 2g, 2g+1 of H).  A sub-block of 16 weights has
    // one int8 scale: one MMA step, then y += d * sc_j * C.
    template <int MIS>
    __device__ __forceinline__ void compute_q6(uint32_t r0, uint32_t r1, int half, float (&acc)[NT][4], int t) const {
        const float d0 = f16_lo(q6w<MIS>(r0, 208)), d1 = f16_lo(q6w<MIS>(r1, 208));
        constexpr int NH = NB / 4;                                    // halves of the superblock: 2 or 1
#pragma unroll
        for (int hh = 0; hh < NH; ++hh) {
            const int n = NH == 2 ? hh : half;
            // int8 scales of sub-blocks 8n .. 8n + 7, biased by 128 (so a byte is an unsigned magic)
            const uint32_t sa0 = q6w<MIS>(r0, 192 + 8 * n) ^ 0x80808080u, sb0 = q6w<MIS>(r0, 196 + 8 * n) ^ 0x80808080u;
            const uint32_t sa1 = q6w<MIS>(r1, 192 + 8 * n) ^ 0x80808080u, sb1 = q6w<MIS>(r1, 196 + 8 * n) ^ 0x80808080u;
#pragma unroll
            for (int lq = 0; lq < 2; ++lq) {
                const uint32_t l0 = 16 * lq;
                const uint32_t A0 = q6w<MIS>(r0, 64 * n + l0 + 4 * t), A1 = q6w<MIS>(r1, 64 * n + l0 + 4 * t);
                const uint32_t B0 = q6w<MIS>(r0, 64 * n + 32 + l0 + 4 * t), B1 = q6w<MIS>(r1, 64 * n + 32 + l0 + 4 * t);
                const uint32_t H0 = q6w<MIS>(r0, 128 + 32 * n + l0 + 4 * t), H1 = q6w<MIS>(r1, 128 + 32 * n + l0 + 4 * t);
#pragma unroll
                for (int g6 = 0; g6 < 4; ++g6) {
                    auto code = [&](uint32_t A, uint32_t B, uint32_t H) {
                        const uint32_t lo = ((g6 & 1) ? B : A) >> (4 * (g6 >> 1));
                        const uint32_t hi = g6 == 0 ? (H << 4) : g6 == 1 ? (H << 2) : g6 == 2 ? H : (H >> 2);
                        return (lo & 0x0F0F0F0Fu) | (hi & 0x30303030u);
                    };
                    const uint32_t v0 = code(A0, B0, H0), v1 = code(A1, B1, H1);
                    const int j = 2 * g6 + lq;                 // sub-block within half n (0..7)
                    // sc_j = (2^23 + (sc + 128)) - (2^23 + 128), exact; d * sc_j has <= 19 bits: exact
                    const float s0 = (byte_magic(j < 4 ? sa0 : sb0, j & 3) - 8388736.f) * d0;
                    const float s1 = (byte_magic(j < 4 ? sa1 : sb1, j & 3) - 8388736.f) * d1;
                    const uint32_t a[4] = {q6k_pair<BF>(v0), q6k_pair<BF>(v1), q6k_pair<BF>(v0 >> 8),
                                           q6k_pair<BF>(v1 >> 8)};
                    const int jl = 8 * hh + j;                 // sub-block of this warp: block jl / 2, step jl % 2
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        float c[4];
                        mma_zero<BF>(c, a, xf[nt][jl >> 1][jl & 1][0], xf[nt][jl >> 1][jl & 1][1]);
                        acc[nt][0] = fmaf(s0, c[0], acc[nt][0]);
                        acc[nt][1] = fmaf(s0, c[1], acc[nt][1]);
                        acc[nt][2] = fmaf(s1, c[2], acc[nt][2]);
                        acc[nt][3] = fmaf(s1, c[3], acc[nt][3]);
                    }
                }
            }
        }
    }

    // Q2_K (84-byte superblock = the warp's chunk; with KW = 128 the warp takes
    // half `half` of it).  Rows g and g + 8 lie at box + sr0 and box + sr1
    // (row slots).  Sub-block 8n + 2j + h (16 weights: elements 128n + 32j +
    // 16h ..) has its codes in bits 2j, 2j+1 of qs[32n + 16h ..]: lane t's word
    // qs[32n + 16h + 4t ..] gives elements 4t .. 4t + 3 of it, bytes 0 and 2
    // shifted by 2j into the even pair, bytes 1 and 3 by 2j + 8 into the odd
    // one.  One MMA step per sub-block, then y += d * sc * C; the mins enter
    // once per tile, y -= dmin * sum m S over the part-0 columns.
    __device__ __forceinline__ void compute_q2(uint32_t box, int half, float (&acc)[NT][4], int g, int t, int M,
                                               const float *sxw, int sstride) const {
        const uint32_t r0 = box + sr0, r1 = box + sr1;
        const uint32_t h0 = lds32(r0 + 80), h1 = lds32(r1 + 80);   // d | dmin
        const float d0 = f16_lo(h0), d1 = f16_lo(h1);
        const float nd0 = d0 * -8388608.f, nd1 = d1 * -8388608.f;   // -2^23 d (exact)
        constexpr int NH = NB / 4;                                    // halves of the superblock: 2 or 1
        uint32_t sc[NH][2][2];                                        // [half][row][word]: s[8n .. 8n + 7]
#pragma unroll
        for (int hh = 0; hh < NH; ++hh) {
            const int n = NH == 2 ? hh : half;
            sc[hh][0][0] = lds32(r0 + 8 * n);
            sc[hh][0][1] = lds32(r0 + 8 * n + 4);
            sc[hh][1][0] = lds32(r1 + 8 * n);
            sc[hh][1][1] = lds32(r1 + 8 * n + 4);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const uint32_t W0 = lds32(r0 + 16 + 32 * n + 16 * h + 4 * t);
                const uint32_t W1 = lds32(r1 + 16 + 32 * n + 16 * h + 4 * t);
                const uint32_t V0 = W0 >> 8, V1 = W1 >> 8;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int sb = 2 * j + h;   // scale byte of the sub-block in s[8n ..]
                    const float s0 = fmaf(byte_magic(sc[hh][0][sb >> 2] & 0x0F0F0F0Fu, sb & 3), d0, nd0);   // d * sc
                    const float s1 = fmaf(byte_magic(sc[hh][1][sb >> 2] & 0x0F0F0F0Fu, sb & 3), d1, nd1);
                    const uint32_t a[4] = {q2k_pair<BF>(W0 >> (2 * j)), q2k_pair<BF>(W1 >> (2 * j)),
                                           q2k_pair<BF>(V0 >> (2 * j)), q2k_pair<BF>(V1 >> (2 * j))};
                    const int bl = 4 * hh + j;   // the warp's 32-element block: step h of it
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        float c[4];
                        mma_zero<BF>(c, a, xf[nt][bl][h][0], xf[nt][bl][h][1]);
                        acc[nt][0] = fmaf(s0, c[0], acc[nt][0]);
                        acc[nt][1] = fmaf(s0, c[1], acc[nt][1]);
                        acc[nt][2] = fmaf(s1, c[2], acc[nt][2]);
                        acc[nt][3] = fmaf(s1, c[3], acc[nt][3]);
                    }
                }
            }
        }
        // mins: the warp's sub-blocks q = 0 .. 2 NB - 1 in element order are s bytes 8n + q (n =
        // the warp's first half), sums sxw[m * sstride + q].  y -= dmin * sum_q m_q S_q on the tensor
        // cores: k-slot q holds sub-block q (A: the 4-bit mins of rows g, g + 8; B: S of column g's
        // activation row as three exact bf16 parts, zero on the other parts' columns).
        const float m0f = f16_hi(h0), m1f = f16_hi(h1);
        const uint32_t msel = (t & 1) ? 0x4342u : 0x4140u;   // bytes 2t, 2t+1 (mod 4) to halves 0 and 1
        uint32_t am[4];
#pragma unroll
        for (int hi = 0; hi < 2; ++hi) {   // k-slots 2t, 2t+1 (hi = 0) and 2t+8, 2t+9 (hi = 1)
            const bool kin = hi == 0 || NB == 8;
            // (the lane's word index puts sc in local memory; a select in its place measured slower:
            // 11008 x 4096 at M = 1, 12.7 -> 13.4 us, and M = 9..12, 4-7 %)
            am[2 * hi] = kin ? min6_pair_bf16(prmt((sc[hi & (NH - 1)][0][t >> 1] >> 4) & 0x0F0F0F0Fu, 0u, msel)) : 0u;
            am[2 * hi + 1] = kin ? min6_pair_bf16(prmt((sc[hi & (NH - 1)][1][t >> 1] >> 4) & 0x0F0F0F0Fu, 0u, msel)) : 0u;
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int c = 8 * nt + g, m = c / P;
            const bool live = (c - m * P == 0) && m < M;
            uint32_t b[2][3];   // [k-slot half][part]
#pragma unroll
            for (int hi = 0; hi < 2; ++hi) {
                const bool kin = live && (hi == 0 || NB == 8);
                const float2 sv = kin ? *reinterpret_cast<const float2 *>(sxw + m * sstride + 2 * t + 8 * hi)
                                      : make_float2(0.f, 0.f);
                uint32_t h0p, m0p, l0p, h1p, m1p, l1p;
                split3(sv.x, h0p, m0p, l0p);
                split3(sv.y, h1p, m1p, l1p);
                b[hi][0] = h0p | (h1p << 16);
                b[hi][1] = m0p | (m1p << 16);
                b[hi][2] = l0p | (l1p << 16);
            }
            float cz[4];
            mma_zero<true>(cz, am, b[0][0], b[1][0]);
            mma_acc<true>(cz, am, b[0][1], b[1][1]);
            mma_acc<true>(cz, am, b[0][2], b[1][2]);
            acc[nt][0] = fmaf(-m0f, cz[0], acc[nt][0]);
            acc[nt][1] = fmaf(-m0f, cz[1], acc[nt][1]);
            acc[nt][2] = fmaf(-m1f, cz[2], acc[nt][2]);
            acc[nt][3] = fmaf(-m1f, cz[3], acc[nt][3]);
        }
    }

    // box: this warp's chunk, row 0, in the stage; half: which half of the
    // chunk (KW = 128); sxw: the x sums of this warp's first sub-block, rows
    // sstride apart (Q4_K).
    __device__ __forceinline__ void compute(uint32_t box, int half, float (&acc)[NT][4], int lane, int M,
                                            const float *sxw, int sstride) const {
        const int g = lane >> 2, t = lane & 3;
        const uint32_t r0 = box + g * CB, r1 = r0 + 8 * CB;   // rows g, g + 8
        if constexpr (FMT == F_Q4_0) {
            const uint32_t sel = t ? 0x3210u : 0x3254u;
#pragma unroll
            for (int pp = 0; pp < NB / 2; ++pp) {
                const uint32_t o = 36u * (uint32_t)(half * (NB / 2) + pp);   // the block pair
                const uint32_t w0 = lds32(r0 + o), w1 = lds32(r1 + o);             // d(even), codes 0, 1
                const uint32_t v0 = lds32(r0 + o + 16), v1 = lds32(r1 + o + 16);   // codes 14, 15, d(odd)
                const uint32_t e0 = prmt(lds32(r0 + o + 4 * t), v0, sel), e1 = prmt(lds32(r1 + o + 4 * t), v1, sel);
                const uint32_t u0 = lds32(r0 + o + 20 + 4 * t), u1 = lds32(r1 + o + 20 + 4 * t);
                {
                    const uint32_t a0[4] = {q40_lo<BF>(e0), q40_lo<BF>(e1), q40_lo<BF>(e0 >> 8), q40_lo<BF>(e1 >> 8)};
                    const uint32_t a1[4] = {q40_hi<BF>(e0), q40_hi<BF>(e1), q40_hi<BF>(e0 >> 8), q40_hi<BF>(e1 >> 8)};
                    block(a0, a1, 2 * pp, f16_lo(w0), f16_lo(w1), acc);
                }
                {
                    const uint32_t a0[4] = {q40_lo<BF>(u0), q40_lo<BF>(u1), q40_lo<BF>(u0 >> 8), q40_lo<BF>(u1 >> 8)};
                    const uint32_t a1[4] = {q40_hi<BF>(u0), q40_hi<BF>(u1), q40_hi<BF>(u0 >> 8), q40_hi<BF>(u1 >> 8)};
                    block(a0, a1, 2 * pp + 1, f16_hi(v0), f16_hi(v1), acc);
                }
            }
        } else if constexpr (FMT == F_Q2_K) {
            compute_q2(box, half, acc, g, t, M, sxw, sstride);
        } else if constexpr (FMT == F_Q6_KS) {
            compute_q6<2>(box + sr0, box + sr1, half, acc, t);
        } else if constexpr (FMT == F_Q6_K) {
            if (q6o & 2) compute_q6<1>(r0, r1, half, acc, t);
            else compute_q6<0>(r0, r1, half, acc, t);
        } else if constexpr (FMT == F_Q8_0) {
#pragma unroll
            for (int pp = 0; pp < NB / 2; ++pp) {
                const uint32_t o = 68u * (uint32_t)(half * (NB / 2) + pp);
                const uint32_t w0 = lds32(r0 + o), w1 = lds32(r1 + o);             // d(even), codes 0, 1
                const uint32_t v0 = lds32(r0 + o + 32), v1 = lds32(r1 + o + 32);   // codes 30, 31, d(odd)
                uint32_t e[2][2], u[2][2];   // [step][row]
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const uint32_t sel = (4 * h + t) ? 0x3210u : 0x3254u;
                    e[h][0] = prmt(lds32(r0 + o + 16 * h + 4 * t), v0, sel);
                    e[h][1] = prmt(lds32(r1 + o + 16 * h + 4 * t), v1, sel);
                    u[h][0] = lds32(r0 + o + 36 + 16 * h + 4 * t);
                    u[h][1] = lds32(r1 + o + 36 + 16 * h + 4 * t);
                }
                {
                    const uint32_t a0[4] = {q80_pair<BF>(e[0][0]), q80_pair<BF>(e[0][1]), q80_pair<BF>(e[0][0] >> 8),
                                            q80_pair<BF>(e[0][1] >> 8)};
                    const uint32_t a1[4] = {q80_pair<BF>(e[1][0]), q80_pair<BF>(e[1][1]), q80_pair<BF>(e[1][0] >> 8),
                                            q80_pair<BF>(e[1][1] >> 8)};
                    block(a0, a1, 2 * pp, f16_lo(w0), f16_lo(w1), acc);
                }
                {
                    const uint32_t a0[4] = {q80_pair<BF>(u[0][0]), q80_pair<BF>(u[0][1]), q80_pair<BF>(u[0][0] >> 8),
                                            q80_pair<BF>(u[0][1] >> 8)};
                    const uint32_t a1[4] = {q80_pair<BF>(u[1][0]), q80_pair<BF>(u[1][1]), q80_pair<BF>(u[1][0] >> 8),
                                            q80_pair<BF>(u[1][1] >> 8)};
                    block(a0, a1, 2 * pp + 1, f16_hi(v0), f16_hi(v1), acc);
                }
            }
        } else {
            // Q4_K and Q5_K: header words d|dmin, scales s[0..3], s[4..7], s[8..11];
            // Q5_K's fifth bits (qh[32]) follow at 16 and its nibbles at 48
            constexpr bool K5 = FMT == F_Q5_K;
            constexpr uint32_t QS = K5 ? 48u : 16u;
            const uint32_t h0 = lds32(r0), h1 = lds32(r1);
            const float d0 = f16_lo(h0), d1 = f16_lo(h1);
            const float nd0 = d0 * -8388608.f, nd1 = d1 * -8388608.f;   // -2^23 d (exact)
            const uint32_t s10 = lds32(r0 + 4), s11 = lds32(r1 + 4);
            const uint32_t s20 = lds32(r0 + 8), s21 = lds32(r1 + 8);
            const uint32_t s30 = lds32(r0 + 12), s31 = lds32(r1 + 12);
            // 6-bit scales of this warp's sub-blocks, one per byte (sub-blocks 0-3: s[j] & 63;
            // 4-7: s[j+4] & 15 | (s[j-4] >> 6) << 4)
            const uint32_t sc0 = half == 0 ? (s10 & 0x3F3F3F3Fu) : ((s30 & 0x0F0F0F0Fu) | ((s10 >> 2) & 0x30303030u));
            const uint32_t sc1 = half == 0 ? (s11 & 0x3F3F3F3Fu) : ((s31 & 0x0F0F0F0Fu) | ((s11 >> 2) & 0x30303030u));
            uint32_t sch0 = 0, sch1 = 0;   // KW = 256: the upper four scales too
            if constexpr (NB == 8) {
                sch0 = (s30 & 0x0F0F0F0Fu) | ((s10 >> 2) & 0x30303030u);
                sch1 = (s31 & 0x0F0F0F0Fu) | ((s11 >> 2) & 0x30303030u);
            }
            // Q5_K: qh bytes of elements 16h + 4t .. 16h + 4t + 3 of every group (bit 2g + nibble)
            uint32_t hq0[2] = {0u, 0u}, hq1[2] = {0u, 0u};
            if constexpr (K5) {
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    hq0[h] = lds32(r0 + 16 + 16 * h + 4 * t);
                    hq1[h] = lds32(r1 + 16 + 16 * h + 4 * t);
                }
            }
#pragma unroll
            for (int gq = 0; gq < NB / 2; ++gq) {
                const int grp = half * (NB / 2) + gq;
                uint32_t c0[2], c1[2];
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    c0[h] = lds32(r0 + QS + 32 * grp + 16 * h + 4 * t);
                    c1[h] = lds32(r1 + QS + 32 * grp + 16 * h + 4 * t);
                }
#pragma unroll
                for (int hi = 0; hi < 2; ++hi) {
                    const int b = 2 * gq + hi;                           // sub-block of this warp
                    const uint32_t sv0 = (NB == 8 && b >= 4) ? sch0 : sc0, sv1 = (NB == 8 && b >= 4) ? sch1 : sc1;
                    const float s0 = fmaf(byte_magic(sv0, b & 3), d0, nd0);   // d * sc (exact)
                    const float s1 = fmaf(byte_magic(sv1, b & 3), d1, nd1);
                    if constexpr (K5) {
                        // 5-bit codes, one per byte: nibble hi of the code byte | bit 2 grp + hi of qh << 4
                        const int sh = 2 * grp + hi;
                        uint32_t v0[2], v1[2];
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            v0[h] = ((c0[h] >> (4 * hi)) & 0x0F0F0F0Fu) | (((hq0[h] >> sh) & 0x01010101u) << 4);
                            v1[h] = ((c1[h] >> (4 * hi)) & 0x0F0F0F0Fu) | (((hq1[h] >> sh) & 0x01010101u) << 4);
                        }
                        const uint32_t a0[4] = {q5k_pair<BF>(v0[0]), q5k_pair<BF>(v1[0]), q5k_pair<BF>(v0[0] >> 8),
                                                q5k_pair<BF>(v1[0] >> 8)};
                        const uint32_t a1[4] = {q5k_pair<BF>(v0[1]), q5k_pair<BF>(v1[1]), q5k_pair<BF>(v0[1] >> 8),
                                                q5k_pair<BF>(v1[1] >> 8)};
                        block(a0, a1, b, s0, s1, acc);
                    } else if (hi == 0) {
                        const uint32_t a0[4] = {q4k_lo<BF>(c0[0]), q4k_lo<BF>(c1[0]), q4k_lo<BF>(c0[0] >> 8),
                                                q4k_lo<BF>(c1[0] >> 8)};
                        const uint32_t a1[4] = {q4k_lo<BF>(c0[1]), q4k_lo<BF>(c1[1]), q4k_lo<BF>(c0[1] >> 8),
                                                q4k_lo<BF>(c1[1] >> 8)};
                        block(a0, a1, b, s0, s1, acc);
                    } else {
                        const uint32_t a0[4] = {q4k_hi<BF>(c0[0]), q4k_hi<BF>(c1[0]), q4k_hi<BF>(c0[0] >> 8),
                                                q4k_hi<BF>(c1[0] >> 8)};
                        const uint32_t a1[4] = {q4k_hi<BF>(c0[1]), q4k_hi<BF>(c1[1]), q4k_hi<BF>(c0[1] >> 8),
                                                q4k_hi<BF>(c1[1] >> 8)};
                        block(a0, a1, b, s0, s1, acc);
                    }
                }
            }
            // mins: y -= dmin * sum_j m_j S_j on the part-0 column of each activation row
            // (sub-blocks 0-3: m = s[j+4] & 63; 4-7: s[j+4] >> 4 | (s[j] >> 6) << 4), on the tensor
            // cores: C = A B with A = the mins of rows g, g + 8 at k-slots 2t, 2t + 1 (the warp's
            // sub-blocks 2t, 2t + 1; slots 8-15 empty) and B = the sums S of column g's activation
            // row as three exact bf16 parts (zero on the other parts' columns); products exact,
            // fp32 sums.  bf16 MMAs whatever the activation type (S needs fp32's exponent range).
            const float m0f = f16_hi(h0), m1f = f16_hi(h1);
            const uint32_t mn0 = half == 0 ? (s20 & 0x3F3F3F3Fu) : (((s30 >> 4) & 0x0F0F0F0Fu) | ((s20 >> 2) & 0x30303030u));
            const uint32_t mn1 = half == 0 ? (s21 & 0x3F3F3F3Fu) : (((s31 >> 4) & 0x0F0F0F0Fu) | ((s21 >> 2) & 0x30303030u));
            uint32_t mnh0 = 0, mnh1 = 0;
            if constexpr (NB == 8) {
                mnh0 = ((s30 >> 4) & 0x0F0F0F0Fu) | ((s20 >> 2) & 0x30303030u);
                mnh1 = ((s31 >> 4) & 0x0F0F0F0Fu) | ((s21 >> 2) & 0x30303030u);
            }
            const bool kin = 2 * t < NB;                          // k-slots 2t, 2t+1 hold sub-blocks of this warp
            const uint32_t msel = (t & 1) ? 0x4342u : 0x4140u;    // bytes 2t, 2t+1 (mod 4) to halves 0 and 1
            const uint32_t w0 = (NB == 8 && t >= 2) ? mnh0 : mn0, w1 = (NB == 8 && t >= 2) ? mnh1 : mn1;
            const uint32_t am[4] = {kin ? min6_pair_bf16(prmt(w0, 0u, msel)) : 0u,
                                    kin ? min6_pair_bf16(prmt(w1, 0u, msel)) : 0u, 0u, 0u};
            const int g = lane >> 2;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const int c = 8 * nt + g, m = c / P;
                const bool live = kin && (c - m * P == 0) && m < M;
                const float2 sv = live ? *reinterpret_cast<const float2 *>(sxw + m * sstride + 2 * t)
                                       : make_float2(0.f, 0.f);
                uint32_t ph0, pm0, pl0, ph1, pm1, pl1;
                split3(sv.x, ph0, pm0, pl0);
                split3(sv.y, ph1, pm1, pl1);
                float cz[4];
                mma_zero<true>(cz, am, ph0 | (ph1 << 16), 0u);
                mma_acc<true>(cz, am, pm0 | (pm1 << 16), 0u);
                mma_acc<true>(cz, am, pl0 | (pl1 << 16), 0u);
                acc[nt][0] = fmaf(-m0f, cz[0], acc[nt][0]);
                acc[nt][1] = fmaf(-m0f, cz[1], acc[nt][1]);
                acc[nt][2] = fmaf(-m1f, cz[2], acc[nt][2]);
                acc[nt][3] = fmaf(-m1f, cz[3], acc[nt][3]);
            }
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
// y += d_w * (d_x / 16) * C per block in fp32.  B column g is activation row g.
//
// Lane (g, t) reads code word t of every block: byte j of the word is code
// byte e(t, j), with e(t, j) = 4t + j for odd blocks and (4t - 2 + j) mod 16
// for even ones (the even block starts 2 bytes into its word).  Its low
// nibbles are weights e(t, 0..3) and feed MMA k-slots 4t..4t+3; its high
// nibbles, weights e(t, .) + 16, feed k-slots 16 + 4t..  The B fragment of the
// lane (activation row g) holds the activation codes of the same weights in
// the same slots.
__device__ __forceinline__ void imma_s8_16832(int (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%10, %10, %10, %10};"
        : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "r"(0));
}

template <int XT>
struct RawPair {
    using T = uint32_t;
    __device__ static __forceinline__ T zero() { return 0u; }
    __device__ static __forceinline__ T load(const void *x, long off) {   // the staged slice of x
        return *reinterpret_cast<const uint32_t *>(static_cast<const uint16_t *>(x) + off);
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
    __device__ static __forceinline__ T load(const void *x, long off) {   // the staged slice of x
        return *reinterpret_cast<const float2 *>(static_cast<const float *>(x) + off);
    }
    __device__ static __forceinline__ float2 get(T v) { return v; }
};

// Q8_0 weights take the same path with their int8 codes as they are: lane t
// holds codes 4t..4t+3 and 16+4t..16+4t+3 of each block (the even block of a
// pair starts 2 bytes into a word: two words and a PRMT), the activations in
// the same natural order, and y += d_w * d_x * C.
template <int XT, int FMT = F_Q4_0>
struct Q40I8 {
    static constexpr bool Q8 = FMT == F_Q8_0;
    static constexpr bool QK = FMT == F_Q4_K;   // Q4_K: unsigned codes, sub-block scale and min
    static constexpr int CB = FmtInfo<FMT>::chunk_bytes;
    uint32_t xq[8][2];   // [block][k-slots 4t.. / 16+4t..]: int8 codes of activation row g
    float dx[8][2];      // [block][column 2t, 2t+1]: d_x (Q4_0: d_x / 16) of activation rows 2t, 2t+1
    float inv;           // 1: no activation scale to undo

    // activation element of k-slot pair (4t, 4t+1) and (4t+2, 4t+3) of block parity hb
    __device__ static __forceinline__ int cb0(int hb, int j) { return (Q8 || QK || hb) ? 4 * j : (j ? 4 * j - 2 : 14); }
    __device__ static __forceinline__ int cb2(int hb, int j) { return (Q8 || QK || hb) ? 4 * j + 2 : 4 * j; }

    __device__ static __forceinline__ uint32_t pack_s8(int a, int b, int c, int d) {
        return (uint32_t)(a & 0xFF) | ((uint32_t)(b & 0xFF) << 8) | ((uint32_t)(c & 0xFF) << 16) |
               ((uint32_t)d << 24);
    }
    // |v| <= amax and s = RN(127 / amax), so |v s| rounds to at most 127 (1 + 2^-23) < 127.5:
    // the code never leaves [-127, 127] and needs no clamp
    __device__ static __forceinline__ int q8(float v, float s) { return __float2int_rn(v * s); }

    struct Slice {
        uint8_t *xp;     // the raw slice [M][nk] in shared memory
        float *sx, *xmax;
        int M, nk, rs;
    };
    __device__ __forceinline__ bool prologue(const GemvArgs &, const Slice &, int, uint64_t *xfull, int, int, int,
                                             unsigned long long timeout) {
        return mbar_wait(xfull, 0, timeout, DEVERR_GEMV_WAIT);
    }
    __device__ __forceinline__ void load_frags(const Slice &S, int k0, int, int lane) {
        load_x(S.xp, S.M, S.nk, k0, lane);
    }

    // One block of one activation row: lanes 4G .. 4G+3 (t = lane & 3) take its 32
    // elements, 8 each at the k-slots of their B fragment; returns the lane's two
    // code words and the block's scale d.
    __device__ static __forceinline__ void quant_block(const void *x, long e, int hb, int t, uint32_t &q0,
                                                       uint32_t &q1, float &d) {
        using Raw = typename RawPair<XT>::T;
        const Raw r0 = RawPair<XT>::load(x, e + cb0(hb, t)), r1 = RawPair<XT>::load(x, e + cb2(hb, t));
        const Raw r2 = RawPair<XT>::load(x, e + 16 + cb0(hb, t)), r3 = RawPair<XT>::load(x, e + 16 + cb2(hb, t));
        const float2 f0 = RawPair<XT>::get(r0), f1 = RawPair<XT>::get(r1), f2 = RawPair<XT>::get(r2),
                     f3 = RawPair<XT>::get(r3);
        const float v[8] = {f0.x, f0.y, f1.x, f1.y, f2.x, f2.y, f3.x, f3.y};
        float amax = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[i]));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
        const bool zero = !(amax >= 7.888609052210118e-31f);   // 2^-100
        d = zero ? 0.f : amax / 127.f;
        const float sc = zero ? 0.f : 127.f / amax;
        q0 = pack_s8(q8(v[0], sc), q8(v[1], sc), q8(v[2], sc), q8(v[3], sc));
        q1 = pack_s8(q8(v[4], sc), q8(v[5], sc), q8(v[6], sc), q8(v[7], sc));
    }

    __device__ __forceinline__ void load_x(const void *x, int M, int K, long k0, int lane) {
        const int g = lane >> 2, t = lane & 3;
        constexpr float DSF = (Q8 || QK) ? 1.f : 0.0625f;   // Q4_0 codes enter as 16 (u - 8)
        if (M <= 4) {
            // Few rows: lane group G quantizes block G of every row (M blocks in a row of
            // dependent steps instead of 8), then the codes move to the lanes whose B
            // fragments hold them (row g, block b: group b's result for row g) and the
            // scales to the lanes whose columns they scale (rows 2t, 2t + 1).
            inv = 1.f;
            uint32_t tq[4][2];
            float td[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                if (j < M) quant_block(x, (long)j * K + k0 + 32 * g, g & 1, t, tq[j][0], tq[j][1], td[j]);
                else tq[j][0] = tq[j][1] = 0u, td[j] = 0.f;
            }
#pragma unroll
            for (int b = 0; b < 8; ++b) {
                uint32_t q0 = 0u, q1 = 0u;
                float d0 = 0.f, d1 = 0.f;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    if (j >= M) break;   // uniform
                    const uint32_t a0 = __shfl_sync(0xffffffffu, tq[j][0], 4 * b + t);
                    const uint32_t a1 = __shfl_sync(0xffffffffu, tq[j][1], 4 * b + t);
                    const float dj = __shfl_sync(0xffffffffu, td[j], 4 * b);
                    if (g == j) {
                        q0 = a0;
                        q1 = a1;
                    }
                    if (2 * t == j) d0 = dj;
                    if (2 * t + 1 == j) d1 = dj;
                }
                xq[b][0] = q0;
                xq[b][1] = q1;
                dx[b][0] = DSF * d0;
                dx[b][1] = DSF * d1;
            }
            return;
        }
        const bool live = g < M;
        const long base = (live ? (long)g * K : 0L) + k0;   // a dead column reads row 0, zeroed below
        using Raw = typename RawPair<XT>::T;
        inv = 1.f;
#pragma unroll
        for (int b0 = 0; b0 < 8; b0 += 4) {
            // all loads of four blocks in flight before any is used
            Raw r[4][4];   // [block][pairs: e(t,0..1), e(t,2..3), +16, +16]
#pragma unroll
            for (int bb = 0; bb < 4; ++bb) {
                const int b = b0 + bb;
                const long e = base + 32 * b;
                r[bb][0] = RawPair<XT>::load(x, e + cb0(b & 1, t));
                r[bb][1] = RawPair<XT>::load(x, e + cb2(b & 1, t));
                r[bb][2] = RawPair<XT>::load(x, e + 16 + cb0(b & 1, t));
                r[bb][3] = RawPair<XT>::load(x, e + 16 + cb2(b & 1, t));
            }
            if (!live) {
#pragma unroll
                for (int bb = 0; bb < 4; ++bb)
#pragma unroll
                    for (int i = 0; i < 4; ++i) r[bb][i] = RawPair<XT>::zero();
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
                constexpr float DS = (Q8 || QK) ? 1.f : 0.0625f;   // Q4_0 codes enter as 16 (u - 8)
                dx[b][0] = DS * __shfl_sync(0xffffffffu, d, 8 * t);
                dx[b][1] = DS * __shfl_sync(0xffffffffu, d, 8 * t + 4);
            }
        }
    }

    // box: this warp's [16 rows][CB] chunk.
    __device__ __forceinline__ void compute(uint32_t box, int, float (&acc)[1][4], int lane, int, const float *,
                                            int) const {
        const int g = lane >> 2, t = lane & 3;
        const uint32_t r0 = box + g * CB, r1 = r0 + 8 * CB;   // rows g, g+8
        if constexpr (QK) {
            // Q4_K superblock: sub-block b (32 weights) takes nibble b & 1 of qs[32 (b / 2) ..]; its
            // codes u enter as they are (0..15), so C = sum u q_x, and a second MMA with A = 1
            // gives the code sums Q = sum q_x of each activation row:
            //   y += d_x (d sc_b C - dmin m_b Q)
            const uint32_t h0 = lds32(r0), h1 = lds32(r1);                 // d | dmin
            const float d0 = f16_lo(h0), d1 = f16_lo(h1), n0 = -f16_hi(h0), n1 = -f16_hi(h1);
            const uint32_t s10 = lds32(r0 + 4), s11 = lds32(r1 + 4), s20 = lds32(r0 + 8), s21 = lds32(r1 + 8);
            const uint32_t s30 = lds32(r0 + 12), s31 = lds32(r1 + 12);
            // 6-bit scales and mins, one per byte: sub-blocks 0-3 and 4-7
            const uint32_t sc[2][2] = {{s10 & 0x3F3F3F3Fu, (s30 & 0x0F0F0F0Fu) | ((s10 >> 2) & 0x30303030u)},
                                       {s11 & 0x3F3F3F3Fu, (s31 & 0x0F0F0F0Fu) | ((s11 >> 2) & 0x30303030u)}};
            const uint32_t mn[2][2] = {{s20 & 0x3F3F3F3Fu, ((s30 >> 4) & 0x0F0F0F0Fu) | ((s20 >> 2) & 0x30303030u)},
                                       {s21 & 0x3F3F3F3Fu, ((s31 >> 4) & 0x0F0F0F0Fu) | ((s21 >> 2) & 0x30303030u)}};
            const uint32_t ones[4] = {0x01010101u, 0x01010101u, 0x01010101u, 0x01010101u};
#pragma unroll
            for (int gq = 0; gq < 4; ++gq) {
                const uint32_t o = 16u + 32u * (uint32_t)gq + 4u * (uint32_t)t;
                const uint32_t lo0 = lds32(r0 + o), lo1 = lds32(r1 + o), hi0 = lds32(r0 + o + 16), hi1 = lds32(r1 + o + 16);
#pragma unroll
                for (int hb = 0; hb < 2; ++hb) {
                    const int b = 2 * gq + hb;
                    const int sh = 4 * hb;
                    const uint32_t a[4] = {(lo0 >> sh) & 0x0F0F0F0Fu, (lo1 >> sh) & 0x0F0F0F0Fu,
                                           (hi0 >> sh) & 0x0F0F0F0Fu, (hi1 >> sh) & 0x0F0F0F0Fu};
                    int c[4], q[4];
                    imma_s8_16832(c, a, xq[b][0], xq[b][1]);
                    imma_s8_16832(q, ones, xq[b][0], xq[b][1]);
                    const float s0 = d0 * (float)((sc[0][b >> 2] >> (8 * (b & 3))) & 0xFFu);   // exact
                    const float s1 = d1 * (float)((sc[1][b >> 2] >> (8 * (b & 3))) & 0xFFu);
                    const float m0 = n0 * (float)((mn[0][b >> 2] >> (8 * (b & 3))) & 0xFFu);
                    const float m1 = n1 * (float)((mn[1][b >> 2] >> (8 * (b & 3))) & 0xFFu);
                    acc[0][0] = fmaf(dx[b][0], fmaf(s0, (float)c[0], m0 * (float)q[0]), acc[0][0]);
                    acc[0][1] = fmaf(dx[b][1], fmaf(s0, (float)c[1], m0 * (float)q[1]), acc[0][1]);
                    acc[0][2] = fmaf(dx[b][0], fmaf(s1, (float)c[2], m1 * (float)q[2]), acc[0][2]);
                    acc[0][3] = fmaf(dx[b][1], fmaf(s1, (float)c[3], m1 * (float)q[3]), acc[0][3]);
                }
            }
            return;
        }
        if constexpr (Q8) {
#pragma unroll
            for (int p = 0; p < 4; ++p) {
                const uint32_t pb = 68 * p;   // the block pair: d(2p) codes(2p) | d(2p+1) codes(2p+1)
                const uint32_t w00 = lds32(r0 + pb), w10 = lds32(r1 + pb);             // d(2p)
                const uint32_t w08 = lds32(r0 + pb + 32), w18 = lds32(r1 + pb + 32);   // d(2p+1) in the high half
                uint32_t u[2][2][2];   // [block of the pair][row][codes 4t.. / 16+4t..]
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const uint32_t o = pb + 16 * h + 4 * t;
                    u[0][0][h] = prmt(lds32(r0 + o), lds32(r0 + o + 4), 0x5432u);
                    u[0][1][h] = prmt(lds32(r1 + o), lds32(r1 + o + 4), 0x5432u);
                    u[1][0][h] = lds32(r0 + o + 36);
                    u[1][1][h] = lds32(r1 + o + 36);
                }
                const float d[2][2] = {{f16_bits_to_float(w00), f16_bits_to_float(w10)},
                                       {f16_bits_to_float(w08 >> 16), f16_bits_to_float(w18 >> 16)}};
#pragma unroll
                for (int hb = 0; hb < 2; ++hb) {
                    const int b = 2 * p + hb;
                    const uint32_t a[4] = {u[hb][0][0], u[hb][1][0], u[hb][0][1], u[hb][1][1]};
                    int c[4];
                    imma_s8_16832(c, a, xq[b][0], xq[b][1]);
                    acc[0][0] = fmaf(d[hb][0] * dx[b][0], (float)c[0], acc[0][0]);
                    acc[0][1] = fmaf(d[hb][0] * dx[b][1], (float)c[1], acc[0][1]);
                    acc[0][2] = fmaf(d[hb][1] * dx[b][0], (float)c[2], acc[0][2]);
                    acc[0][3] = fmaf(d[hb][1] * dx[b][1], (float)c[3], acc[0][3]);
                }
            }
            return;
        }
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

// KW: weights of K per compute warp and chunk (256: a warp per chunk; 128: two)
template <int FMT, int XT, int NT, bool I8, int KW = (I8 ? 256 : gemv_kw(NT))>
struct GemvImpl : Exact<FMT, XT, NT, KW> {};
template <int XT>
struct GemvImpl<F_Q4_0, XT, 1, true, 256> : Q40I8<XT> {};
template <int XT>
struct GemvImpl<F_Q8_0, XT, 1, true, 256> : Q40I8<XT, F_Q8_0> {};
template <int XT>
struct GemvImpl<F_Q4_K, XT, 1, true, 256> : Q40I8<XT, F_Q4_K> {};

// ------------------------------------------------------------------ kernel
// blockDim = gemv_threads(FMT, NT): warps 0..15 compute, warp 16 produces (TMA), the
// rest reduce; one CTA per SM (at most 96 registers per thread with 19 warps
// over four 16K-register sub-partitions, 80 with 21).  Every wait is
// bounded; a wait that gives up sets a bit of the device error word and ends
// its warp's loop.
template <int FMT, int XT, int NT, bool I8, int KW = (I8 ? 256 : gemv_kw(NT))>
__global__ void __launch_bounds__(gemv_threads(FMT, NT), 1)
    gemv_kernel(const __grid_constant__ CUtensorMap wmap, const GemvArgs a) {
    constexpr int CB = FmtInfo<FMT>::chunk_bytes;
    constexpr int WPC = CHUNK / KW;            // compute warps per chunk
    constexpr int P = gemv_parts(XT, I8);
    constexpr int RS = gemv_rs(NT);            // floats per row of a reduction slot
    constexpr int RED = gemv_red(FMT, NT);
    extern __shared__ __align__(128) uint8_t smem[];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int S = a.splits;
    const int split = blockIdx.x % S;
    const int rgrp = blockIdx.x / S;
    const int G = gridDim.x / S;
    const int c_begin = split * a.cps;
    const int c_end = min(c_begin + a.cps, a.nchunks);
    const int nact = (c_end - c_begin) * WPC;   // compute warps with work (<= GEMV_W)
    const int ws = a.wstages;

    constexpr int XE = (XT == X_F32) ? 4 : 2;
    // the reducer stages x raw with bulk copies, except fp32 x on the fp path (the compute warps split it)
    constexpr bool STAGE = I8 || XT != X_F32;
    const GemvSmem L = gemv_smem_layout(CB, a.cps, ws, NT, fmt_sums(FMT), P, a.M, XE, I8, fmt_row_slots(FMT));
    uint8_t *ring = smem;
    uint8_t *xs = smem + L.ring;
    float *red = reinterpret_cast<float *>(xs + L.xs);
    float *sx = reinterpret_cast<float *>(xs + L.xs + L.red);
    float *scratch = reinterpret_cast<float *>(xs + L.xs + L.red + L.sx);
    float *xmax = reinterpret_cast<float *>(xs + L.xs + L.red + L.sx + L.scratch);
    uint64_t *bars = reinterpret_cast<uint64_t *>(xs + L.xs + L.red + L.sx + L.scratch + L.xmax);
    uint64_t *full = bars, *empty = bars + ws, *redfull = bars + 2 * ws, *redempty = bars + 2 * ws + GEMV_RSTAGES;
    uint64_t *xfull = redempty + GEMV_RSTAGES;
    const int nk = (c_end - c_begin) * CHUNK;   // elements of K in this CTA's slice
    const int rs = I8 ? nk : a.cps * CHUNK + GEMV_XPAD;   // row stride of the staged slice (elements)

    if (threadIdx.x == 0) {
        for (int s = 0; s < ws; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], nact > 0 ? nact : 1);
        }
        for (int s = 0; s < GEMV_RSTAGES; ++s) {
            mbar_init(&redfull[s], nact > 0 ? nact : 1);
            mbar_init(&redempty[s], RED);
        }
        mbar_init(xfull, 1);
        fence_mbar_init();
        reinterpret_cast<int *>(xmax)[15] = 0;   // the activation rescale flag
    }
    __syncthreads();
    // the next kernel on the stream (a programmatic dependent) may become
    // resident now and start its own weight stream while this one runs
    pdl_launch_dependents();
    if (nact <= 0 || rgrp >= G) return;

    if (warp == GEMV_W) {
        // ---------------- producer: reads only Wq, which callers that allow
        // overlap promise is not written by the preceding work
        if (lane == 0) {
            tma_prefetch_desc(&wmap);
            int it = 0, s = 0;
            uint32_t ph = 0;
            for (int tile = rgrp; tile < a.row_tiles; tile += G, ++it) {
                if (it >= ws && !mbar_wait(&empty[s], ph ^ 1u, a.timeout_ns, DEVERR_GEMV_WAIT)) break;
                // first pass through the ring: one stage in flight at a time, so that the
                // first stage (and the prologue's activation loads) are not queued behind
                // every SM's whole ring of weight requests
                if (it > 0 && it < ws && !mbar_wait(&full[it - 1], 0u, a.timeout_ns, DEVERR_GEMV_WAIT)) break;
                // one 3-D box per stage: [chunks of this split][16 rows][chunk bytes]; the
                // last split's box may run past the last chunk, where it reads zeros
                mbar_arrive_expect_tx(&full[s], (uint32_t)L.tx);
                if constexpr (fmt_row_slots(FMT)) {
                    // one box per row of the tile: whole 16-byte units from r mod 8 units before
                    // the one holding the row's first byte of this split (rows past the end
                    // read zeros; row 0, the only one that could start before the matrix, starts
                    // at its own unit)
                    const long rb = (long)a.nchunks * CB;
                    for (int r = 0; r < GEMV_ROWS; ++r) {
                        const long b0 = (long)(tile * GEMV_ROWS + r) * rb + (long)c_begin * CB;
                        tma_load_2d(ring + (size_t)s * L.stage + (size_t)r * L.slot, &wmap, &full[s], 0,
                                    (int)((b0 >> 4) - (r & 7)));
                    }
                } else if constexpr (FMT == F_Q6_K) {
                    // one 2-D box per chunk, [16 rows][120 words] from the 16-byte boundary at or
                    // below the superblock (chunks past the end read zeros)
                    for (int ci = 0; ci < a.cps; ++ci)
                        tma_load_2d(ring + (size_t)s * L.stage + (size_t)ci * GEMV_ROWS * CB, &wmap, &full[s],
                                    (105 * (c_begin + ci)) & ~7, tile * GEMV_ROWS);
                } else {
                    tma_load_3d(ring + (size_t)s * L.stage, &wmap, &full[s], 0, tile * GEMV_ROWS, c_begin);
                }
                if (++s == ws) {
                    s = 0;
                    ph ^= 1u;
                }
            }
            // drain: every issued stage's load lands before the CTA may exit
            for (int j = max(0, it - ws); j < it; ++j)
                mbar_wait(&full[j % ws], (uint32_t)((j / ws) & 1), a.timeout_ns, DEVERR_GEMV_WAIT);
        }
        return;
    }

    if (warp > GEMV_W) {
        // ---------------- reducers: touch y and the workspace only after the
        // preceding work has completed.  Reducer j takes RR rows of each tile
        // from row RR j; lane (row, column group) sums the compute warps'
        // 4-column groups in warp order (deterministic), then the parts of each
        // activation row.
        const int j = warp - GEMV_W - 1;
        pdl_wait();
        const int M = a.M, N = a.N;
        if (j == 0 && STAGE && lane == 0) {
            // the CTA's slice of x, one bulk copy per activation row, into shared memory
            mbar_arrive_expect_tx(xfull, (uint32_t)(M * nk * XE));
            for (int m = 0; m < M; ++m)
                bulk_load(xs + (size_t)m * rs * XE,
                          static_cast<const uint8_t *>(a.x) + ((size_t)m * a.K + (size_t)c_begin * CHUNK) * XE,
                          (uint32_t)(nk * XE), xfull);
        }
        __syncwarp();
        constexpr int RR = GEMV_ROWS / RED, NCG = 32 / RR;   // rows per reducer, column groups in parallel
        const int row = RR * j + (lane % RR), cgl = lane / RR;
        float *dst = (S == 1) ? a.y : a.partial + (size_t)split * M * N;
        int r = 0;
        uint32_t rph = 0;
        for (int tile = rgrp; tile < a.row_tiles; tile += G) {
            if (!mbar_wait(&redfull[r], rph, a.timeout_ns, DEVERR_GEMV_WAIT)) break;
            const uint32_t rs0 = smem_u32(red) + (uint32_t)(r * GEMV_W * GEMV_ROWS * RS * 4);
            const int n = tile * GEMV_ROWS + row;
#pragma unroll
            for (int k = 0; k < (2 * NT + NCG - 1) / NCG; ++k) {
                const int cg = cgl + NCG * k;
                if (cg < 2 * NT) {
                    const uint32_t addr = rs0 + (uint32_t)((row * RS + 4 * cg) * 4);
                    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
                    // all of the warps' loads in flight at once, summed in warp order
                    uint4 u[GEMV_W];
#pragma unroll
                    for (int w = 0; w < GEMV_W; ++w)
                        u[w] = w < nact ? lds128(addr + (uint32_t)(w * GEMV_ROWS * RS * 4)) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
                    for (int w = 0; w < GEMV_W; ++w) {
                        v.x += __uint_as_float(u[w].x);
                        v.y += __uint_as_float(u[w].y);
                        v.z += __uint_as_float(u[w].z);
                        v.w += __uint_as_float(u[w].w);
                    }
                    if constexpr (P == 1) {
                        // column = activation row
                        const float o[4] = {v.x, v.y, v.z, v.w};
                        if (n < N) {
#pragma unroll
                            for (int i = 0; i < 4; ++i)
                                if (4 * cg + i < M) dst[(size_t)(4 * cg + i) * N + n] = o[i];
                        }
                    } else {
                        st_shared_v4(smem_u32(scratch) + (uint32_t)((row * RS + 4 * cg) * 4), __float_as_uint(v.x),
                                     __float_as_uint(v.y), __float_as_uint(v.z), __float_as_uint(v.w));
                    }
                }
            }
            if constexpr (P > 1) {
                __syncwarp();
                for (int o = lane; o < RR * M; o += 32) {
                    const int rr = RR * j + (o % RR), m = o / RR, nn = tile * GEMV_ROWS + rr;
                    const float *sp = scratch + rr * RS + m * P;
                    const float val = (sp[0] + sp[1]) + sp[2];
                    if (nn < N) dst[(size_t)m * N + nn] = val;
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&redempty[r]);
            if (++r == GEMV_RSTAGES) {
                r = 0;
                rph ^= 1u;
            }
        }
        // the bulk copies of x land before the CTA may exit
        if (j == 0 && STAGE) mbar_wait(xfull, 0, a.timeout_ns, DEVERR_GEMV_WAIT);
        return;
    }

    // ---------------- compute warps
    if (warp >= nact) return;
    const int ci = warp / WPC, half = warp % WPC;
    using Impl = GemvImpl<FMT, XT, NT, I8, KW>;
    Impl impl;
    typename Impl::Slice sl;
    sl.xp = reinterpret_cast<decltype(sl.xp)>(xs);
    sl.sx = sx;
    sl.xmax = xmax;
    sl.M = a.M;
    sl.nk = nk;
    sl.rs = rs;
    if (!impl.prologue(a, sl, c_begin, xfull, nact, warp, lane, a.timeout_ns)) return;
    impl.load_frags(sl, ci * CHUNK, half, lane);
    if constexpr (FMT == F_Q6_K && !I8) impl.q6o = 2u * (uint32_t)((105 * (c_begin + ci)) & 7);
    constexpr int SUB = FMT == F_Q2_K ? 16 : 32;   // weights per sum of x
    const float *sxw = sx + ci * (CHUNK / SUB) + half * (KW / SUB);
    const int sstride = nk / SUB;
    const int g = lane >> 2, t = lane & 3;
    int s = 0, r = 0, rit = 0;
    uint32_t ph = 0, rph = 0;
    for (int tile = rgrp; tile < a.row_tiles; tile += G, ++rit) {
        if (!mbar_wait(&full[s], ph, a.timeout_ns, DEVERR_GEMV_WAIT)) break;
        float acc[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[nt][j] = 0.f;
        uint32_t box;
        if constexpr (fmt_row_slots(FMT)) {
            // rows g and g + 8 of the tile: their slots, the slice's offset in them, this warp's chunk
            const long rb = (long)a.nchunks * CB;
            const long b0 = (long)(tile * GEMV_ROWS + g) * rb + (long)c_begin * CB, b1 = b0 + 8 * rb;
            impl.sr0 = (uint32_t)(g * L.slot + 16 * g) + (uint32_t)(b0 & 15) + (uint32_t)(ci * CB);
            impl.sr1 = (uint32_t)((g + 8) * L.slot + 16 * g) + (uint32_t)(b1 & 15) + (uint32_t)(ci * CB);
            box = smem_u32(ring) + (uint32_t)((size_t)s * L.stage);
        } else {
            box = smem_u32(ring) + (uint32_t)((size_t)s * L.stage + (size_t)ci * GEMV_ROWS * CB);
        }
        impl.compute(box, half, acc, lane, a.M, sxw, sstride);
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
        if (++s == ws) {
            s = 0;
            ph ^= 1u;
        }
        if (rit >= GEMV_RSTAGES && !mbar_wait(&redempty[r], rph ^ 1u, a.timeout_ns, DEVERR_GEMV_WAIT)) break;
        const uint32_t rw = smem_u32(red) + (uint32_t)(((r * GEMV_W + warp) * GEMV_ROWS) * RS * 4);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            sts_f2(rw + 4 * (g * RS + 8 * nt + 2 * t), acc[nt][0] * impl.inv, acc[nt][1] * impl.inv);
            sts_f2(rw + 4 * ((g + 8) * RS + 8 * nt + 2 * t), acc[nt][2] * impl.inv, acc[nt][3] * impl.inv);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&redfull[r]);
        if (++r == GEMV_RSTAGES) {
            r = 0;
            rph ^= 1u;
        }
    }
}

// Split-K: y[i] = sum over s (in order) of partial[s][i], i over the M*N
// outputs of one pass.  Launched as a programmatic dependent of the GEMV: it
// waits for the GEMV's partials, and lets the next kernel on the stream start.
static __global__ void __launch_bounds__(256) gemv_splitk_sum_kernel(const float *__restrict__ partial,
                                                                     float *__restrict__ y, int S, long mn) {
    pdl_launch_dependents();
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

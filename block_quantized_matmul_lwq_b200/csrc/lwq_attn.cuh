// Decode attention: one query token per sequence and head against that
// sequence's key/value cache, with the softmax fused into the single pass over
// the keys (the running-maximum "online softmax" of "Compute Shaders con
// WebGPU para Inferencia ML", "El Mecanismo de Atencion"), split over the
// sequence as flash-decoding does so that a few long sequences still fill the
// GPU, and the splits' partial results merged by a second kernel.
//
//   s_j = scale * (q . k_j),  out = sum_j softmax(s)_j v_j
//
// Layouts: q [B][H][D] and the caches [B][Hkv][Lmax][D] in fp16 or bf16,
// out [B][H][D] fp32; query head h reads kv head h / G, G = H / Hkv.
//
// The pass is HBM-bound (every key and value row is read once per kv head;
// the G query heads of a kv head share the read), so it runs on the CUDA
// cores: lane i of a warp holds elements [E*i, E*i + E) of the head dimension
// (E = D / 32), a key row is one coalesced warp-wide load, and the G x 4 dot
// products of a step (4 keys, G query heads) are finished together by one
// transposed butterfly of warp shuffles.  Scores are kept in the log2 domain
// (q, or the score, multiplied by scale * log2(e)) so that every exponential
// is one exp2.  Grouped query heads (G > 1) take a tensor-core form of the
// same pass (attn_split_tc_kernel, below).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <math.h>
#include <stdint.h>

#include "lwq_gemv.cuh"

namespace lwq {

constexpr int ATTN_WARPS = 4;   // warps per CTA; each walks its own 4-key groups of the split
constexpr int ATTN_U = 4;       // keys per warp per step (their K and V rows in flight together)

// E consecutive 16-bit elements of a row as fp32 (E = 2 or 4), coherent loads
// (the cache may have been written by the preceding kernel).
template <int XT, int E>
__device__ __forceinline__ void load_row(const uint16_t *p, float (&f)[E]) {
    uint32_t w[E / 2];
    if constexpr (E == 4) {
        const uint2 u = __ldcg(reinterpret_cast<const uint2 *>(p));
        w[0] = u.x;
        w[1] = u.y;
    } else {
        w[0] = __ldcg(reinterpret_cast<const unsigned int *>(p));
    }
#pragma unroll
    for (int i = 0; i < E / 2; ++i) {
        if constexpr (XT == X_F16) {
            const float2 v = __half22float2(*reinterpret_cast<const __half2 *>(&w[i]));
            f[2 * i] = v.x;
            f[2 * i + 1] = v.y;
        } else {
            f[2 * i] = __uint_as_float(w[i] << 16);
            f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
        }
    }
}

// Sums over the 32 lanes of V = 2^k values at once, in (V - 1) + (5 - k)
// shuffles instead of 5 V: each round halves the values a lane keeps (the
// lower half where the round's lane bit is 0, else the upper half) and adds
// its partner's copy of that half.  Afterwards lane L holds the total of
// value (L >> (5 - k)) & (V - 1), in val[0].
template <int V>
__device__ __forceinline__ void transpose_reduce(float (&val)[V], int lane) {
    constexpr int K = V >= 32 ? 5 : (V >= 16 ? 4 : (V >= 8 ? 3 : (V >= 4 ? 2 : (V >= 2 ? 1 : 0))));
    static_assert((1 << K) == V && K <= 5, "V must be a power of two <= 32");
#pragma unroll
    for (int r = 0; r < K; ++r) {
        const int half = V >> (r + 1), bit = 16 >> r;
        const bool upper = (lane & bit) != 0;
#pragma unroll
        for (int i = 0; i < half; ++i) {
            const float send = upper ? val[i] : val[i + half];
            const float keep = upper ? val[i + half] : val[i];
            val[i] = keep + __shfl_xor_sync(0xffffffffu, send, bit);
        }
    }
#pragma unroll
    for (int bit = 16 >> K; bit > 0; bit >>= 1) val[0] += __shfl_xor_sync(0xffffffffu, val[0], bit);
}

// Asynchronous global -> shared copies (cp.async) of 4, 8 or 16 bytes, grouped
// per thread; a warp barrier after the wait makes them visible to the warp.

struct AttnArgs {
    const uint16_t *q, *k, *v;
    const int *lens;     // [B] or null (every sequence Lmax long)
    float *out;          // [B][H][D]
    float *part;         // [B][H][S][D + 2]: m (log2 domain), l, acc[D] per split (S > 1)
    int B, H, Hkv, Lmax, S, chunk;
    float qscale;        // scale * log2(e)
};

// One CTA: split s of sequence b, kv head g, all G query heads of g (used with
// G = 1; grouped heads take attn_split_tc_kernel).  With one query head per kv
// head, direct coalesced row loads keep HBM busy (measured 0.99 of peak).
template <int XT, int D, int G>
__global__ void __launch_bounds__(ATTN_WARPS * 32) attn_split_kernel(const AttnArgs a) {
    constexpr int E = D / 32;
    const int s = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int len = a.lens ? a.lens[b] : a.Lmax;
    len = len < 1 ? 1 : (len > a.Lmax ? a.Lmax : len);
    const int j0 = s * a.chunk, j1 = min(j0 + a.chunk, len);

    float qf[G][E];
#pragma unroll
    for (int h = 0; h < G; ++h) {
        load_row<XT, E>(a.q + ((size_t)b * a.H + (size_t)g * G + h) * D + E * lane, qf[h]);
#pragma unroll
        for (int e = 0; e < E; ++e) qf[h][e] *= a.qscale;
    }
    float m[G], l[G], acc[G][E];
#pragma unroll
    for (int h = 0; h < G; ++h) {
        m[h] = -INFINITY;
        l[h] = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) acc[h][e] = 0.f;
    }
    const uint16_t *kb = a.k + ((size_t)b * a.Hkv + g) * (size_t)a.Lmax * D + E * lane;
    const uint16_t *vb = a.v + ((size_t)b * a.Hkv + g) * (size_t)a.Lmax * D + E * lane;

    constexpr int STRIDE = ATTN_U * ATTN_WARPS;
    const int jfirst = j0 + ATTN_U * warp;
    const int nsteps = jfirst < j1 ? (j1 - jfirst + STRIDE - 1) / STRIDE : 0;
    for (int i = 0; i < nsteps; ++i) {
        const int jg = jfirst + i * STRIDE;
        float kf[ATTN_U][E], vf[ATTN_U][E];
#pragma unroll
        for (int u = 0; u < ATTN_U; ++u) {
            const int j = min(jg + u, j1 - 1);   // a key past the split reloads the last one (masked below)
            load_row<XT, E>(kb + (size_t)j * D, kf[u]);
            load_row<XT, E>(vb + (size_t)j * D, vf[u]);
        }
        // the G x U dot products: lane partials, summed over the warp together
        constexpr int V = G * ATTN_U;
        constexpr int KV = V >= 32 ? 5 : (V >= 16 ? 4 : (V >= 8 ? 3 : 2));
        float part[V];
#pragma unroll
        for (int h = 0; h < G; ++h)
#pragma unroll
            for (int u = 0; u < ATTN_U; ++u) {
                float p = 0.f;
#pragma unroll
                for (int e = 0; e < E; ++e) p = fmaf(qf[h][e], kf[u][e], p);
                part[h * ATTN_U + u] = p;
            }
        transpose_reduce<V>(part, lane);
#pragma unroll
        for (int h = 0; h < G; ++h) {
            float sc[ATTN_U];
#pragma unroll
            for (int u = 0; u < ATTN_U; ++u) {
                const float p = __shfl_sync(0xffffffffu, part[0], (h * ATTN_U + u) << (5 - KV));
                sc[u] = (jg + u < j1) ? p : -INFINITY;
            }
            float mn = m[h];
#pragma unroll
            for (int u = 0; u < ATTN_U; ++u) mn = fmaxf(mn, sc[u]);   // finite: key jg is in the split
            const float corr = exp2f(m[h] - mn);                      // 0 on the first step (m = -inf)
            float ps = 0.f;
#pragma unroll
            for (int e = 0; e < E; ++e) acc[h][e] *= corr;
#pragma unroll
            for (int u = 0; u < ATTN_U; ++u) {
                const float p = exp2f(sc[u] - mn);                    // 0 for a masked key
                ps += p;
#pragma unroll
                for (int e = 0; e < E; ++e) acc[h][e] = fmaf(p, vf[u][e], acc[h][e]);
            }
            l[h] = fmaf(l[h], corr, ps);
            m[h] = mn;
        }
    }

    // merge the warps: per head the largest running maximum, the others rescaled to it
    __shared__ float sm[ATTN_WARPS][G], sl[ATTN_WARPS][G], sacc[ATTN_WARPS][G][D];
#pragma unroll
    for (int h = 0; h < G; ++h) {
        if (lane == 0) {
            sm[warp][h] = m[h];
            sl[warp][h] = l[h];
        }
#pragma unroll
        for (int e = 0; e < E; ++e) sacc[warp][h][E * lane + e] = acc[h][e];
    }
    __syncthreads();
    for (int i = threadIdx.x; i < G * D; i += ATTN_WARPS * 32) {
        const int h = i / D, d = i % D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < ATTN_WARPS; ++w) M = fmaxf(M, sm[w][h]);
        float L = 0.f, A = 0.f;
        if (M != -INFINITY) {   // an empty split (past the sequence) keeps m = -inf, l = 0, acc = 0
#pragma unroll
            for (int w = 0; w < ATTN_WARPS; ++w) {
                const float f = exp2f(sm[w][h] - M);
                L = fmaf(sl[w][h], f, L);
                A = fmaf(sacc[w][h][d], f, A);
            }
        }
        const size_t bh = (size_t)b * a.H + (size_t)g * G + h;
        if (a.S == 1) {
            a.out[bh * D + d] = A / L;
        } else {
            float *pp = a.part + (bh * a.S + s) * (D + 2);
            if (d == 0) {
                pp[0] = M;
                pp[1] = L;
            }
            pp[2 + d] = A;
        }
    }
    pdl_launch_dependents();
}

// ----------------------------------------------------- grouped heads: tensor cores
// With G > 1 query heads per kv head the scores and the weighted values are
// small matrix products, which the tensor cores take (mma.sync m16n8k16 in
// fp16/bf16, fp32 accumulate): per step of 16 keys a warp computes
// S = Q K^T (MMA rows: the G query heads, exact 16-bit q; columns: keys) and
// O += P V (rows: the heads' probabilities; columns: head dimensions).  P is
// carried as two 16-bit parts, hi in MMA rows 0..7 and lo = p - hi in rows
// 8..15 (16 of p's bits in bf16, 22 in fp16): O's rows g and g + 8 add up to
// the product with p to that precision, where a single 16-bit P would lose
// 2^-8.  K and V tiles [16 keys][D] stream through a per-warp cp.async ring in
// a 128-byte-swizzled layout (chunk c of key r at c ^ (r & 7)), read by
// ldmatrix (V transposed) without bank conflicts.
constexpr int ATTN_TC_STAGES = 3;

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

// two fp32 values rounded to nearest into a 16-bit pair (lo in the low half)
template <int XT>
__device__ __forceinline__ uint32_t pack16(float a, float b) {
    if constexpr (XT == X_F16) {
        const __half2 h = __floats2half2_rn(a, b);
        return *reinterpret_cast<const uint32_t *>(&h);
    } else {
        const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
        return *reinterpret_cast<const uint32_t *>(&h);
    }
}
template <int XT>
__device__ __forceinline__ float lo16(uint32_t v) {
    return XT == X_F16 ? __half2float(__ushort_as_half((unsigned short)(v & 0xFFFFu))) : __uint_as_float(v << 16);
}
template <int XT>
__device__ __forceinline__ float hi16(uint32_t v) {
    return XT == X_F16 ? __half2float(__ushort_as_half((unsigned short)(v >> 16))) : __uint_as_float(v & 0xFFFF0000u);
}

template <int D>
constexpr size_t attn_tc_smem() { return (size_t)ATTN_WARPS * ATTN_TC_STAGES * 2 * 16 * 2 * D; }

template <int XT, int D, int G>
__global__ void __launch_bounds__(ATTN_WARPS * 32) attn_split_tc_kernel(const AttnArgs a) {
    static_assert(G >= 2 && G <= 8, "grouped heads only");
    constexpr int NCH = D / 8;                 // 16-byte chunks per row
    constexpr uint32_t ROWB = 2 * D, TILEB = 16 * ROWB, STAGEB = 2 * TILEB;
    constexpr int STRIDE = 16 * ATTN_WARPS;
    extern __shared__ __align__(128) uint8_t dsm[];
    const int s = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gr = lane >> 2, t = lane & 3;
    int len = a.lens ? a.lens[b] : a.Lmax;
    len = len < 1 ? 1 : (len > a.Lmax ? a.Lmax : len);
    const int j0 = s * a.chunk, j1 = min(j0 + a.chunk, len);

    // Q as the A operand of S: row gr is query head g G + gr (rows >= G and 8..15 are zero)
    uint32_t qa[D / 16][2];
    {
        const bool live = gr < G;
        const uint16_t *qr = a.q + ((size_t)b * a.H + (size_t)g * G + (live ? gr : 0)) * D;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
            const uint32_t x0 = __ldcg(reinterpret_cast<const unsigned int *>(qr + 16 * ks + 2 * t));
            const uint32_t x1 = __ldcg(reinterpret_cast<const unsigned int *>(qr + 16 * ks + 8 + 2 * t));
            qa[ks][0] = live ? x0 : 0u;
            qa[ks][1] = live ? x1 : 0u;
        }
    }
    float o[D / 8][4];
#pragma unroll
    for (int n = 0; n < D / 8; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) o[n][e] = 0.f;
    float m = -INFINITY, l = 0.f;   // running maximum of row gr (log2 domain); this lane's part of its sum

    const uint16_t *kb = a.k + ((size_t)b * a.Hkv + g) * (size_t)a.Lmax * D;
    const uint16_t *vb = a.v + ((size_t)b * a.Hkv + g) * (size_t)a.Lmax * D;
    const uint32_t ring = (uint32_t)__cvta_generic_to_shared(dsm) + (uint32_t)warp * ATTN_TC_STAGES * STAGEB;
    const int jfirst = j0 + 16 * warp;
    const int nsteps = jfirst < j1 ? (j1 - jfirst + STRIDE - 1) / STRIDE : 0;
    auto issue = [&](int i) {   // step i into stage i % STAGES (an empty group past the end)
        if (i < nsteps) {
            const uint32_t st = ring + (uint32_t)(i % ATTN_TC_STAGES) * STAGEB;
            const int jg = jfirst + i * STRIDE;
#pragma unroll
            for (int q = lane; q < 2 * 16 * NCH; q += 32) {
                const int which = q / (16 * NCH), rem = q % (16 * NCH), r = rem / NCH, c = rem % NCH;
                const int j = min(jg + r, j1 - 1);   // a key past the split reloads the last one (masked below)
                cp_async<16>(st + which * TILEB + r * ROWB + ((c ^ (r & 7)) << 4), (which ? vb : kb) + (size_t)j * D + 8 * c);
            }
        }
        cp_async_commit();
    };
#pragma unroll
    for (int i = 0; i < ATTN_TC_STAGES - 1; ++i) issue(i);
    for (int i = 0; i < nsteps; ++i) {
        issue(i + ATTN_TC_STAGES - 1);
        cp_async_wait<ATTN_TC_STAGES - 1>();
        __syncwarp();   // every lane's copies of step i are in and visible to the warp
        const uint32_t st = ring + (uint32_t)(i % ATTN_TC_STAGES) * STAGEB;
        const int jg = jfirst + i * STRIDE;
        // S = Q K^T: n-tile 0 = keys 0..7, 1 = keys 8..15
        float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        {
            const int key = (lane & 7) + ((lane >> 4) << 3), hcol = (lane >> 3) & 1;
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
                uint32_t r[4];
                const int ch = 2 * ks + hcol;
                ldsm_x4(st + key * ROWB + ((ch ^ (key & 7)) << 4), r);
                const uint32_t aq[4] = {qa[ks][0], 0u, qa[ks][1], 0u};
                if constexpr (XT == X_F16) {
                    mma_f16_16816(sc[0], aq, r[0], r[1], sc[0]);
                    mma_f16_16816(sc[1], aq, r[2], r[3], sc[1]);
                } else {
                    mma_bf16_16816(sc[0], aq, r[0], r[1], sc[0]);
                    mma_bf16_16816(sc[1], aq, r[2], r[3], sc[1]);
                }
            }
        }
        // row gr's scores of keys 2t, 2t+1, 8+2t, 9+2t, in the log2 domain; keys past the split masked
        float v4[4] = {sc[0][0], sc[0][1], sc[1][0], sc[1][1]};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int key = 8 * (e >> 1) + 2 * t + (e & 1);
            v4[e] = (jg + key < j1) ? v4[e] * a.qscale : -INFINITY;
        }
        float mx = fmaxf(fmaxf(v4[0], v4[1]), fmaxf(v4[2], v4[3]));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        const float mn = fmaxf(m, mx);          // finite: key jg is in the split
        const float corr = exp2f(m - mn);       // 0 on the first step (m = -inf)
        float p[4], ps = 0.f;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            p[e] = exp2f(v4[e] - mn);           // 0 for a masked key
            ps += p[e];
        }
        l = fmaf(l, corr, ps);
        m = mn;
        // P: hi parts in rows 0..7, lo parts (p - hi) in rows 8..15
        const uint32_t h0 = pack16<XT>(p[0], p[1]), h1 = pack16<XT>(p[2], p[3]);
        const uint32_t l0 = pack16<XT>(p[0] - lo16<XT>(h0), p[1] - hi16<XT>(h0));
        const uint32_t l1 = pack16<XT>(p[2] - lo16<XT>(h1), p[3] - hi16<XT>(h1));
        const uint32_t ap[4] = {h0, l0, h1, l1};
        {
            const int key = (lane & 7) + (((lane >> 3) & 1) << 3), hcol = lane >> 4;
#pragma unroll
            for (int p2 = 0; p2 < D / 16; ++p2) {
                uint32_t r[4];
                const int ch = 2 * p2 + hcol;
                ldsm_x4_t(st + TILEB + key * ROWB + ((ch ^ (key & 7)) << 4), r);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    o[2 * p2][e] *= corr;
                    o[2 * p2 + 1][e] *= corr;
                }
                if constexpr (XT == X_F16) {
                    mma_f16_16816(o[2 * p2], ap, r[0], r[1], o[2 * p2]);
                    mma_f16_16816(o[2 * p2 + 1], ap, r[2], r[3], o[2 * p2 + 1]);
                } else {
                    mma_bf16_16816(o[2 * p2], ap, r[0], r[1], o[2 * p2]);
                    mma_bf16_16816(o[2 * p2 + 1], ap, r[2], r[3], o[2 * p2 + 1]);
                }
            }
        }
        __syncwarp();   // the stage is read before a later step's copies refill it
    }
    l += __shfl_xor_sync(0xffffffffu, l, 1);
    l += __shfl_xor_sync(0xffffffffu, l, 2);

    // merge the warps (the ring's space is free after the barrier): as in the single-head kernel
    __syncthreads();
    float(*sm)[G] = reinterpret_cast<float(*)[G]>(dsm);
    float(*sl)[G] = reinterpret_cast<float(*)[G]>(dsm + ATTN_WARPS * G * 4);
    float(*sacc)[G][D] = reinterpret_cast<float(*)[G][D]>(dsm + 2 * ATTN_WARPS * G * 4);
    if (gr < G) {
        if (t == 0) {
            sm[warp][gr] = m;
            sl[warp][gr] = l;
        }
#pragma unroll
        for (int n = 0; n < D / 8; ++n) {
            sacc[warp][gr][8 * n + 2 * t] = o[n][0] + o[n][2];       // hi rows + lo rows
            sacc[warp][gr][8 * n + 2 * t + 1] = o[n][1] + o[n][3];
        }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < G * D; i += ATTN_WARPS * 32) {
        const int h = i / D, d = i % D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < ATTN_WARPS; ++w) M = fmaxf(M, sm[w][h]);
        float L = 0.f, A = 0.f;
        if (M != -INFINITY) {
#pragma unroll
            for (int w = 0; w < ATTN_WARPS; ++w) {
                const float f = exp2f(sm[w][h] - M);
                L = fmaf(sl[w][h], f, L);
                A = fmaf(sacc[w][h][d], f, A);
            }
        }
        const size_t bh = (size_t)b * a.H + (size_t)g * G + h;
        if (a.S == 1) {
            a.out[bh * D + d] = A / L;
        } else {
            float *pp = a.part + (bh * a.S + s) * (D + 2);
            if (d == 0) {
                pp[0] = M;
                pp[1] = L;
            }
            pp[2 + d] = A;
        }
    }
    pdl_launch_dependents();
}

// out[b][h][d] from the S partial results of (b, h).  A CTA takes one (b, h)
// and 32 of its D columns (lane = column) with NG = ceil(S / 8) warps (at most
// 16): warp j takes slots j, j + NG, ... in order with 8 slots' loads in
// flight, keeping a running maximum and rescaling its weight and weighted
// values when the maximum grows (an empty split, m = -inf, adds nothing); the
// warps' results are then rescaled to the largest maximum, added in warp order
// and divided by the total weight.  S alone fixes the order of every addition.
// (One thread walking all S splits, twice, made the merge of a long sequence's
// 32 splits cost more than a tenth of the call.)
constexpr int ATTN_COMBINE_U = 8;
inline int attn_combine_warps(int S) {
    const int ng = (S + ATTN_COMBINE_U - 1) / ATTN_COMBINE_U;
    return ng < 1 ? 1 : (ng > 16 ? 16 : ng);
}
template <int D>
__global__ void __launch_bounds__(512) attn_combine_kernel(const float *__restrict__ part, float *__restrict__ out,
                                                            int S) {
    constexpr int U = ATTN_COMBINE_U;
    __shared__ float gm[16], gl[16], ga[16][32];
    pdl_wait();
    const int NG = blockDim.x >> 5;
    const size_t bh = blockIdx.x / (D / 32);
    const int j = threadIdx.x >> 5, c = threadIdx.x & 31, d = 32 * (blockIdx.x % (D / 32)) + c;
    const float *p = part + bh * S * (D + 2);
    float M = -INFINITY, L = 0.f, A = 0.f;
    for (int s0 = j; s0 < S; s0 += NG * U) {
        float mv[U], lv[U], av[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {   // a slot past S reads slot 0 and is skipped below
            const int s = s0 + u * NG;
            const float *ps = p + (size_t)(s < S ? s : 0) * (D + 2);
            mv[u] = s < S ? __ldcg(ps) : -INFINITY;
            lv[u] = __ldcg(ps + 1);
            av[u] = __ldcg(ps + 2 + d);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            if (mv[u] == -INFINITY) continue;
            const float mn = fmaxf(M, mv[u]);
            const float fo = exp2f(M - mn), fn = exp2f(mv[u] - mn);   // fo = 0 while M = -inf
            L = fmaf(L, fo, lv[u] * fn);
            A = fmaf(A, fo, av[u] * fn);
            M = mn;
        }
    }
    if (NG == 1) {   // split 0 holds key 0: M is finite
        out[bh * D + d] = A / L;
        return;
    }
    if (c == 0) {
        gm[j] = M;
        gl[j] = L;
    }
    ga[j][c] = A;
    __syncthreads();
    if (j == 0) {   // warp 0 holds split 0: Mt is finite
        float Mt = -INFINITY;
        for (int g = 0; g < NG; ++g) Mt = fmaxf(Mt, gm[g]);
        float Lt = 0.f, At = 0.f;
        for (int g = 0; g < NG; ++g) {
            if (gm[g] == -INFINITY) continue;
            const float f = exp2f(gm[g] - Mt);
            Lt = fmaf(gl[g], f, Lt);
            At = fmaf(ga[g][c], f, At);
        }
        out[bh * D + d] = At / Lt;
    }
}

// Splits of the sequence (each at least 64 keys, a multiple of 16).  A small
// problem (few sequences and heads) thus still spreads over many CTAs: each
// warp's chain of dependent key steps, not bandwidth, sets its time.
//  * One query head per kv head: enough CTAs for ~4 per SM (up to ~9 are
//    resident: many short waves).
//  * Grouped heads (the tensor-core pass, 2 CTAs resident per SM): the split
//    count with the least modelled time, waves x (keys per split + 128), the
//    128 standing for a CTA's ramp; a last wave that leaves most SMs idle
//    costs a whole wave.  With 8 or fewer (sequence, kv head) pairs, one CTA
//    per SM instead (splits = SMs / pairs).
inline void attn_splits(int B, int H, int Hkv, int Lmax, int sms, int *S, int *chunk) {
    const long pairs = (long)B * Hkv;
    const long smax = (Lmax + 63) / 64;
    long best_s = 1;
    if (H == Hkv) {
        best_s = (4L * sms + pairs - 1) / pairs;
    } else if (pairs <= 8) {
        // few (sequence, kv head) pairs, i.e. long sequences: one CTA per SM.  Two per SM on half the keys each
        // measured slower (1 x 32768 keys, 8 kv heads: 18 splits 28.9 us, 37 splits 30.9 us; 2 x 16384, 4 kv
        // heads: 20.5 and 22.3 us): the SM's bandwidth is shared, and the merge has twice the splits.
        best_s = sms / pairs;
    } else {
        const long slots = 2L * sms;
        double best = -1.0;
        for (long s = 1; s <= smax; ++s) {
            long c = (Lmax + s - 1) / s;
            c = (c + 15) & ~15L;
            const long se = (Lmax + c - 1) / c;
            const long waves = (pairs * se + slots - 1) / slots;
            const double cost = (double)waves * (double)(c + 128);
            if (best < 0 || cost < best) {
                best = cost;
                best_s = se;
            }
        }
    }
    if (best_s > smax) best_s = smax;
    if (best_s < 1) best_s = 1;
    int c = (int)((Lmax + best_s - 1) / best_s);
    c = (c + 15) & ~15;
    *chunk = c;
    *S = (Lmax + c - 1) / c;
}

}  // namespace lwq

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
// transposed butterfly of warp shuffles.  Scores are kept in the
// log2 domain (q is pre-multiplied by scale * log2(e)) so that every
// exponential is one exp2.
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

// Asynchronous global -> shared copies of 4 or 8 bytes (cp.async), grouped;
// a thread reads back only what it copied itself, after waiting for its group.
template <int BYTES>
__device__ __forceinline__ void cp_async(uint32_t dst, const void *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], %2;" ::"r"(dst), "l"(src), "n"(BYTES) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// E 16-bit elements of a row, already in shared memory, as fp32.
template <int XT, int E>
__device__ __forceinline__ void smem_row(uint32_t addr, float (&f)[E]) {
    uint32_t w[E / 2];
    if constexpr (E == 4) {
        asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(w[0]), "=r"(w[1]) : "r"(addr));
    } else {
        asm volatile("ld.shared.u32 %0, [%1];" : "=r"(w[0]) : "r"(addr));
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

constexpr int ATTN_RING = 4;   // steps of K and V rows in flight per warp (shared-memory ring)

struct AttnArgs {
    const uint16_t *q, *k, *v;
    const int *lens;     // [B] or null (every sequence Lmax long)
    float *out;          // [B][H][D]
    float *part;         // [B][H][S][D + 2]: m (log2 domain), l, acc[D] per split (S > 1)
    int B, H, Hkv, Lmax, S, chunk;
    float qscale;        // scale * log2(e)
};

// One CTA: split s of sequence b, kv head g, all G query heads of g.
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

    // Each warp streams its steps (4 keys' K and V rows) through a ring of
    // ATTN_RING shared-memory stages with cp.async: several steps are in flight
    // without holding registers.  Lane i copies, and later reads, bytes
    // [2E i, 2E i + 2E) of each row.  Stage layout: [key u][K, V][lane][E].
    constexpr int STRIDE = ATTN_U * ATTN_WARPS;
    constexpr uint32_t ROWB = 2 * D, STAGEB = ATTN_U * 2 * ROWB;
    // the ring, later reused for the warps' merge
    // one query head per kv head (G = 1): the direct loads keep HBM busy without the ring (measured
    // 0.98 of peak against 0.81 with it); with G > 1 the per-step math is longer and the ring's
    // deeper stream pays
    constexpr bool RING = G > 1;
    constexpr uint32_t RINGB = RING ? ATTN_WARPS * ATTN_RING * STAGEB : 0;
    constexpr uint32_t MERGEB = (2 * ATTN_WARPS * G + ATTN_WARPS * G * D) * 4;
    __shared__ __align__(16) uint8_t smraw[RINGB > MERGEB ? RINGB : MERGEB];
    const uint32_t ring0 = (uint32_t)__cvta_generic_to_shared(smraw) + (uint32_t)warp * ATTN_RING * STAGEB + 2 * E * lane;
    const int jfirst = j0 + ATTN_U * warp;
    const int nsteps = jfirst < j1 ? (j1 - jfirst + STRIDE - 1) / STRIDE : 0;
    auto issue = [&](int i) {   // step i of this warp into stage i % ATTN_RING (an empty group past the end)
        if (i < nsteps) {
            const uint32_t st = ring0 + (uint32_t)(i % ATTN_RING) * STAGEB;
            const int jg = jfirst + i * STRIDE;
#pragma unroll
            for (int u = 0; u < ATTN_U; ++u) {
                const int j = min(jg + u, j1 - 1);   // a key past the split reloads the last one (masked below)
                cp_async<2 * E>(st + (2 * u) * ROWB, kb + (size_t)j * D);
                cp_async<2 * E>(st + (2 * u + 1) * ROWB, vb + (size_t)j * D);
            }
        }
        cp_async_commit();
    };
    if constexpr (RING) {
#pragma unroll
        for (int i = 0; i < ATTN_RING - 1; ++i) issue(i);
    }
    for (int i = 0; i < nsteps; ++i) {
        const int jg = jfirst + i * STRIDE;
        float kf[ATTN_U][E], vf[ATTN_U][E];
        if constexpr (RING) {
            issue(i + ATTN_RING - 1);
            cp_async_wait<ATTN_RING - 1>();   // step i's group has landed
            const uint32_t st = ring0 + (uint32_t)(i % ATTN_RING) * STAGEB;
#pragma unroll
            for (int u = 0; u < ATTN_U; ++u) {
                smem_row<XT, E>(st + (2 * u) * ROWB, kf[u]);
                smem_row<XT, E>(st + (2 * u + 1) * ROWB, vf[u]);
            }
        } else {
#pragma unroll
            for (int u = 0; u < ATTN_U; ++u) {
                const int j = min(jg + u, j1 - 1);   // a key past the split reloads the last one (masked below)
                load_row<XT, E>(kb + (size_t)j * D, kf[u]);
                load_row<XT, E>(vb + (size_t)j * D, vf[u]);
            }
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
    // (every warp's copies have landed and been read: the ring's space is free after the barrier)
    __syncthreads();
    float(*sm)[G] = reinterpret_cast<float(*)[G]>(smraw);
    float(*sl)[G] = reinterpret_cast<float(*)[G]>(smraw + ATTN_WARPS * G * 4);
    float(*sacc)[G][D] = reinterpret_cast<float(*)[G][D]>(smraw + 2 * ATTN_WARPS * G * 4);
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

// out[b][h][d] from the S partial results of (b, h): rescale each split to the
// largest maximum, add in split order, divide by the total weight.
template <int D>
__global__ void __launch_bounds__(D) attn_combine_kernel(const float *__restrict__ part, float *__restrict__ out,
                                                          int S) {
    pdl_wait();
    const size_t bh = blockIdx.x;
    const int d = threadIdx.x;
    const float *p = part + bh * S * (D + 2);
    float M = -INFINITY;
    for (int s = 0; s < S; ++s) M = fmaxf(M, __ldcg(p + (size_t)s * (D + 2)));
    float L = 0.f, A = 0.f;
    for (int s = 0; s < S; ++s) {
        const float *ps = p + (size_t)s * (D + 2);
        const float f = exp2f(__ldcg(ps) - M);   // 0 for an empty split
        L = fmaf(__ldcg(ps + 1), f, L);
        A = fmaf(__ldcg(ps + 2 + d), f, A);
    }
    out[bh * D + d] = A / L;
}

// Splits of the sequence: enough CTAs for ~4 per SM, each split at least 256
// keys (a multiple of 16).
inline void attn_splits(int B, int Hkv, int Lmax, int sms, int *S, int *chunk) {
    const long pairs = (long)B * Hkv;
    long s = (4L * sms + pairs - 1) / pairs;
    const long smax = (Lmax + 255) / 256;
    if (s > smax) s = smax;
    if (s < 1) s = 1;
    int c = (int)((Lmax + s - 1) / s);
    c = (c + 15) & ~15;
    *chunk = c;
    *S = (Lmax + c - 1) / c;
}

}  // namespace lwq

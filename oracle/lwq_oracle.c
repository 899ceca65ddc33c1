/*
 * CPU oracle for y[M,N] = x[M,K] . dequant(Wq[N,K])^T  --  TEST INFRASTRUCTURE.
 *
 * This file is the plain, slow, obviously correct definition that the CUDA
 * library is checked against.  Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg load it; the library never does.  It shares no
 * code, header or table with the CUDA path.
 *
 * What it computes (the plain definition; quantization is in the data, not in
 * the algorithm):
 *
 *   w_hat[n][k] = exact value of weight (n,k) decoded from its block, rounded
 *                 once to fp32;
 *   y[m][n]     = sum_{k=0..K-1} x[m][k] * w_hat[n][k]   in fp64, ascending k;
 *   den[m][n]   = sum_{k=0..K-1} |x[m][k] * w_hat[n][k]| in fp64.
 *
 * Formats (llama.cpp's legacy and K-quant block families, named in "Resumo
 * Tecnico: Llamas na Web", "Declaracao do Problema" item 3 and "3. Design de
 * Shader Consciente de Quantizacao"; the pages give the family names only,
 * and the byte layouts below are the ones this library is specified with):
 *
 *   Q8_0: block of 32 weights, 34 bytes: fp16 d (little endian), int8 q[32];
 *         w = d * q.
 *   Q4_0: block of 32 weights, 18 bytes: fp16 d, 16 bytes b[16];
 *         element i    = (b[i] & 15) - 8,  element i+16 = (b[i] >> 4) - 8;
 *         w = d * element.
 *   Q4_K: superblock of 256 weights, 144 bytes: fp16 d, fp16 dmin,
 *         s[12] (eight 6-bit scales sc_j and eight 6-bit mins m_j),
 *         qs[128].  For j < 4: sc_j = s[j] & 63, m_j = s[j+4] & 63; for
 *         j >= 4: sc_j = (s[j+4] & 15) | ((s[j-4] >> 6) << 4),
 *                 m_j  = (s[j+4] >> 4) | ((s[j]   >> 6) << 4).
 *         Nibbles: 4 groups g of 32 bytes; element 64g+l = qs[32g+l] & 15
 *         (sub-block 2g) and element 64g+32+l = qs[32g+l] >> 4 (sub-block
 *         2g+1), l < 32.  w = d*sc_j*q - dmin*m_j for element in sub-block j.
 *   Q6_K: superblock of 256 weights, 210 bytes: ql[128] (low 4 bits of the
 *         6-bit codes), qh[64] (high 2 bits), int8 sc[16] (one scale per 16
 *         weights), fp16 d last.  Element e = 128n + 32g + l (n < 2, g < 4,
 *         l < 32): low bits = nibble (g >> 1) of ql[64n + 32(g & 1) + l]
 *         (0 = low, 1 = high), high bits = bits 2g, 2g+1 of qh[32n + l];
 *         q = low | high << 4 in [0, 64); w = d * sc[e / 16] * (q - 32).
 *   Q5_K: superblock of 256 weights, 176 bytes: fp16 d, fp16 dmin, s[12]
 *         (scales and mins packed as for Q4_K), qh[32], qs[128].  Element
 *         e = 64g + 32h + l (g < 4, h < 2, l < 32): low bits = nibble h of
 *         qs[32g + l], fifth bit = bit 2g + h of qh[l]; sub-block j = 2g + h;
 *         w = d*sc_j*q - dmin*m_j.
 *   Q2_K: superblock of 256 weights, 84 bytes: s[16] (per 16 weights: scale
 *         in the low nibble, min in the high nibble), qs[64], fp16 d, fp16
 *         dmin.  Element e = 128n + 32j + l (n < 2, j < 4, l < 32): q = bits
 *         2j, 2j+1 of qs[32n + l]; w = d*(s[e/16] & 15)*q - dmin*(s[e/16] >> 4).
 *
 * Activations x are fp32, fp16 or bf16 codes; each is decoded exactly from
 * its IEEE-754 bit fields.
 *
 * Build: gcc -O2 -fopenmp -ffp-contract=off -shared -fPIC (no FMA
 * contraction, so every product and sum is an individually rounded fp64
 * operation in the order written).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Own codes; the Python wrapper maps format names onto them. */
#define OR_Q8_0 1
#define OR_Q4_0 2
#define OR_Q4_K 3
#define OR_Q6_K 4
#define OR_Q5_K 5
#define OR_Q2_K 6
#define OR_ACT_F32 0
#define OR_ACT_F16 1
#define OR_ACT_BF16 2

/* IEEE-754 binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
double lwq_oracle_f16(uint16_t h) {
    int s = h >> 15;
    int e = (h >> 10) & 31;
    int f = h & 1023;
    double v;
    if (e == 0)
        v = ldexp((double)f, -24);                 /* subnormal: f * 2^-14 * 2^-10 */
    else if (e == 31)
        v = f ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + f), e - 25);     /* (1 + f/2^10) * 2^(e-15) */
    return s ? -v : v;
}

/* bfloat16: 1 sign bit, 8 exponent bits (bias 127), 7 fraction bits. */
double lwq_oracle_bf16(uint16_t h) {
    int s = h >> 15;
    int e = (h >> 7) & 255;
    int f = h & 127;
    double v;
    if (e == 0)
        v = ldexp((double)f, -133);                /* f * 2^-126 * 2^-7 */
    else if (e == 255)
        v = f ? NAN : INFINITY;
    else
        v = ldexp((double)(128 + f), e - 134);     /* (1 + f/2^7) * 2^(e-127) */
    return s ? -v : v;
}

static uint16_t rd16(const uint8_t *p) { return (uint16_t)(p[0] | (p[1] << 8)); }

long lwq_oracle_block_weights(int fmt) {
    switch (fmt) {
    case OR_Q8_0: return 32;
    case OR_Q4_0: return 32;
    case OR_Q4_K:
    case OR_Q6_K:
    case OR_Q5_K:
    case OR_Q2_K: return 256;
    default: return -1;
    }
}

long lwq_oracle_block_bytes(int fmt) {
    switch (fmt) {
    case OR_Q8_0: return 34;
    case OR_Q4_0: return 18;
    case OR_Q4_K: return 144;
    case OR_Q6_K: return 210;
    case OR_Q5_K: return 176;
    case OR_Q2_K: return 84;
    default: return -1;
    }
}

long lwq_oracle_row_bytes(int fmt, long K) {
    long bw = lwq_oracle_block_weights(fmt);
    if (bw <= 0 || K <= 0 || K % bw) return -1;
    return K / bw * lwq_oracle_block_bytes(fmt);
}

/* The j-th (scale, min) pair of a Q4_K superblock, j in [0, 8). */
void lwq_oracle_q4k_scale_min(const uint8_t *s, int j, int *sc, int *m) {
    if (j < 4) {
        *sc = s[j] & 63;
        *m = s[j + 4] & 63;
    } else {
        *sc = (s[j + 4] & 15) | ((s[j - 4] >> 6) << 4);
        *m = (s[j + 4] >> 4) | ((s[j] >> 6) << 4);
    }
}

static void decode_q8_0(const uint8_t *b, float *w) {
    double d = lwq_oracle_f16(rd16(b));
    for (int i = 0; i < 32; i++) {
        int q = (int8_t)b[2 + i];
        w[i] = (float)(d * (double)q);
    }
}

static void decode_q4_0(const uint8_t *b, float *w) {
    double d = lwq_oracle_f16(rd16(b));
    for (int i = 0; i < 16; i++) {
        int lo = b[2 + i] & 15;
        int hi = b[2 + i] >> 4;
        w[i] = (float)(d * (double)(lo - 8));
        w[i + 16] = (float)(d * (double)(hi - 8));
    }
}

static void decode_q4_k(const uint8_t *b, float *w) {
    double d = lwq_oracle_f16(rd16(b));
    double dmin = lwq_oracle_f16(rd16(b + 2));
    const uint8_t *s = b + 4;
    const uint8_t *qs = b + 16;
    for (int g = 0; g < 4; g++) {
        int sc0, m0, sc1, m1;
        lwq_oracle_q4k_scale_min(s, 2 * g, &sc0, &m0);
        lwq_oracle_q4k_scale_min(s, 2 * g + 1, &sc1, &m1);
        for (int l = 0; l < 32; l++) {
            int qlo = qs[32 * g + l] & 15;
            int qhi = qs[32 * g + l] >> 4;
            /* d*sc*q (<= 21 significant bits) and dmin*m (<= 17) are exact in
               fp64; their difference is exact whenever the exponents of d and
               dmin are within 32 binades (always, for d, dmin in (0, 0.01]
               as fp16 normals), and is then rounded once to fp32. */
            w[64 * g + l] = (float)(d * (double)sc0 * (double)qlo - dmin * (double)m0);
            w[64 * g + 32 + l] = (float)(d * (double)sc1 * (double)qhi - dmin * (double)m1);
        }
    }
}

static void decode_q6_k(const uint8_t *b, float *w) {
    const uint8_t *ql = b, *qh = b + 128;
    const int8_t *sc = (const int8_t *)(b + 192);
    double d = lwq_oracle_f16(rd16(b + 208));
    for (int e = 0; e < 256; e++) {
        int n = e / 128, g = (e % 128) / 32, l = e % 32;
        int low = (ql[64 * n + 32 * (g & 1) + l] >> (4 * (g >> 1))) & 15;
        int high = (qh[32 * n + l] >> (2 * g)) & 3;
        int q = low | (high << 4);
        /* d (11 bits) * sc (8) * (q - 32) (6): exact in fp64 and in fp32 */
        w[e] = (float)(d * (double)sc[e / 16] * (double)(q - 32));
    }
}

static void decode_q5_k(const uint8_t *b, float *w) {
    double d = lwq_oracle_f16(rd16(b));
    double dmin = lwq_oracle_f16(rd16(b + 2));
    const uint8_t *s = b + 4, *qh = b + 16, *qs = b + 48;
    for (int e = 0; e < 256; e++) {
        int g = e / 64, h = (e % 64) / 32, l = e % 32;
        int q = ((qs[32 * g + l] >> (4 * h)) & 15) | (((qh[l] >> (2 * g + h)) & 1) << 4);
        int sc, m;
        lwq_oracle_q4k_scale_min(s, 2 * g + h, &sc, &m);
        /* d*sc*q (<= 22 significant bits) and dmin*m (<= 17) exact in fp64, as for Q4_K */
        w[e] = (float)(d * (double)sc * (double)q - dmin * (double)m);
    }
}

static void decode_q2_k(const uint8_t *b, float *w) {
    const uint8_t *s = b, *qs = b + 16;
    double d = lwq_oracle_f16(rd16(b + 80));
    double dmin = lwq_oracle_f16(rd16(b + 82));
    for (int e = 0; e < 256; e++) {
        int n = e / 128, j = (e % 128) / 32, l = e % 32;
        int q = (qs[32 * n + l] >> (2 * j)) & 3;
        int sc = s[e / 16] & 15, m = s[e / 16] >> 4;
        w[e] = (float)(d * (double)sc * (double)q - dmin * (double)m);
    }
}

/* Decode one packed row of K weights into fp32.  Returns 0, or -1 on bad args. */
int lwq_oracle_dequant_row(int fmt, const uint8_t *row, long K, float *out) {
    long bw = lwq_oracle_block_weights(fmt);
    long bb = lwq_oracle_block_bytes(fmt);
    if (bw <= 0 || K <= 0 || K % bw) return -1;
    for (long blk = 0; blk < K / bw; blk++) {
        const uint8_t *b = row + blk * bb;
        float *w = out + blk * bw;
        switch (fmt) {
        case OR_Q8_0: decode_q8_0(b, w); break;
        case OR_Q4_0: decode_q4_0(b, w); break;
        case OR_Q4_K: decode_q4_k(b, w); break;
        case OR_Q6_K: decode_q6_k(b, w); break;
        case OR_Q5_K: decode_q5_k(b, w); break;
        default: decode_q2_k(b, w); break;
        }
    }
    return 0;
}

static double act_value(int act, const void *x, long idx) {
    if (act == OR_ACT_F32) return (double)((const float *)x)[idx];
    if (act == OR_ACT_F16) return lwq_oracle_f16(((const uint16_t *)x)[idx]);
    return lwq_oracle_bf16(((const uint16_t *)x)[idx]);
}

/* Decode all of x[M][K] into fp64 (exact). */
static double *decode_x(int act, const void *x, long M, long K) {
    double *xd = (double *)malloc(sizeof(double) * (size_t)M * (size_t)K);
    if (!xd) return NULL;
    for (long i = 0; i < M * K; i++) xd[i] = act_value(act, x, i);
    return xd;
}

static int check_args(int fmt, int act, long M, long N, long K) {
    if (lwq_oracle_row_bytes(fmt, K) < 0) return -1;
    if (act != OR_ACT_F32 && act != OR_ACT_F16 && act != OR_ACT_BF16) return -1;
    if (M <= 0 || N <= 0) return -1;
    return 0;
}

/* One output: fp64 dot product of x row m with decoded weight row w, ascending k. */
static void dot_row(const double *xm, const float *w, long K, double *y, double *den) {
    double acc = 0.0, acc_abs = 0.0;
    for (long k = 0; k < K; k++) {
        double p = xm[k] * (double)w[k];
        acc += p;
        acc_abs += fabs(p);
    }
    *y = acc;
    *den = acc_abs;
}

/*
 * Full product: y and den are [M][N] fp64 (den may be NULL).  nthreads <= 0
 * means the OpenMP default.  Returns 0, or -1 on bad args / no memory.
 */
int lwq_oracle_matmul(int fmt, int act, const uint8_t *Wq, const void *x,
                      long M, long N, long K, double *y, double *den, int nthreads) {
    if (check_args(fmt, act, M, N, K)) return -1;
    long rb = lwq_oracle_row_bytes(fmt, K);
    double *xd = decode_x(act, x, M, K);
    if (!xd) return -1;
    int fail = 0;
#ifdef _OPENMP
    if (nthreads <= 0) nthreads = omp_get_max_threads();
#pragma omp parallel num_threads(nthreads) reduction(| : fail)
#endif
    {
        float *w = (float *)malloc(sizeof(float) * (size_t)K);
        if (!w) {
            fail = 1;
        } else {
#ifdef _OPENMP
#pragma omp for schedule(static)
#endif
            for (long n = 0; n < N; n++) {
                lwq_oracle_dequant_row(fmt, Wq + n * rb, K, w);
                for (long m = 0; m < M; m++) {
                    double dd;
                    dot_row(xd + m * K, w, K, &y[m * N + n], &dd);
                    if (den) den[m * N + n] = dd;
                }
            }
            free(w);
        }
    }
    free(xd);
    return fail ? -1 : 0;
}

/*
 * Selected outputs only: for i < count, y[i] and den[i] are output
 * (ms[i], ns[i]).  Same arithmetic and order as lwq_oracle_matmul.
 */
int lwq_oracle_matmul_sampled(int fmt, int act, const uint8_t *Wq, const void *x,
                              long M, long N, long K, const long *ms, const long *ns,
                              long count, double *y, double *den, int nthreads) {
    if (check_args(fmt, act, M, N, K) || count < 0) return -1;
    for (long i = 0; i < count; i++)
        if (ms[i] < 0 || ms[i] >= M || ns[i] < 0 || ns[i] >= N) return -1;
    long rb = lwq_oracle_row_bytes(fmt, K);
    int fail = 0;
#ifdef _OPENMP
    if (nthreads <= 0) nthreads = omp_get_max_threads();
#pragma omp parallel num_threads(nthreads) reduction(| : fail)
#endif
    {
        float *w = (float *)malloc(sizeof(float) * (size_t)K);
        double *xm = (double *)malloc(sizeof(double) * (size_t)K);
        if (!w || !xm) {
            fail = 1;
        } else {
#ifdef _OPENMP
#pragma omp for schedule(static)
#endif
            for (long i = 0; i < count; i++) {
                lwq_oracle_dequant_row(fmt, Wq + ns[i] * rb, K, w);
                for (long k = 0; k < K; k++) xm[k] = act_value(act, x, ms[i] * K + k);
                double dd;
                dot_row(xm, w, K, &y[i], &dd);
                if (den) den[i] = dd;
            }
        }
        free(w);
        free(xm);
    }
    return fail ? -1 : 0;
}

int lwq_oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * Decode attention (one query per sequence and head) -- the plain definition
 * behind "Compute Shaders con WebGPU para Inferencia ML", "El Mecanismo de
 * Atencion": scores s_j = scale * (q . k_j), weights p_j = softmax(s)_j,
 * out = sum_j p_j v_j.  The page fuses the softmax into the pass over the keys
 * with a running maximum (online softmax); that reaches this same result up to
 * rounding, so the oracle is the definition written out, in fp64:
 *
 *   m = max_j s_j;  p_j = exp(s_j - m);  out[d] = (sum_j p_j v_j[d]) / (sum_j p_j)
 *   den[d] = (sum_j p_j |v_j[d]|) / (sum_j p_j)      (the error scale)
 *
 * Layouts (16-bit codes of dtype act: OR_ACT_F16 or OR_ACT_BF16):
 *   q   [B][H][D]
 *   k,v [B][Hkv][Lmax][D]   (key j of sequence b and kv head g at [b][g][j])
 *   out, den [B][H][D] fp64
 * Query head h reads kv head h / (H / Hkv).  Sequence b has len[b] keys
 * (1 <= len[b] <= Lmax).  Returns 0, or -1 on bad arguments.
 */
int lwq_oracle_attention(int act, const uint16_t *q, const uint16_t *k, const uint16_t *v, const int *len,
                         long B, long H, long Hkv, long Lmax, long D, double scale, double *out, double *den) {
    if ((act != OR_ACT_F16 && act != OR_ACT_BF16) || B <= 0 || H <= 0 || Hkv <= 0 || H % Hkv || Lmax <= 0 ||
        D <= 0)
        return -1;
    for (long b = 0; b < B; b++)
        if (len[b] < 1 || len[b] > Lmax) return -1;
    long G = H / Hkv;
    int fail = 0;
#ifdef _OPENMP
#pragma omp parallel for schedule(static) reduction(| : fail)
#endif
    for (long bh = 0; bh < B * H; bh++) {
        long b = bh / H, h = bh % H, g = h / G;
        long n = len[b];
        double *s = (double *)malloc(sizeof(double) * (size_t)n);
        if (!s) {
            fail = 1;
            continue;
        }
        const uint16_t *qh = q + (b * H + h) * D;
        const uint16_t *kb = k + (b * Hkv + g) * Lmax * D;
        const uint16_t *vb = v + (b * Hkv + g) * Lmax * D;
        double m = -INFINITY;
        for (long j = 0; j < n; j++) {
            double dot = 0.0;
            for (long d = 0; d < D; d++) {
                double qd = act == OR_ACT_F16 ? lwq_oracle_f16(qh[d]) : lwq_oracle_bf16(qh[d]);
                double kd = act == OR_ACT_F16 ? lwq_oracle_f16(kb[j * D + d]) : lwq_oracle_bf16(kb[j * D + d]);
                dot += qd * kd;
            }
            s[j] = scale * dot;
            if (s[j] > m) m = s[j];
        }
        double sum = 0.0;
        for (long j = 0; j < n; j++) {
            s[j] = exp(s[j] - m);
            sum += s[j];
        }
        for (long d = 0; d < D; d++) {
            double acc = 0.0, acc_abs = 0.0;
            for (long j = 0; j < n; j++) {
                double vd = act == OR_ACT_F16 ? lwq_oracle_f16(vb[j * D + d]) : lwq_oracle_bf16(vb[j * D + d]);
                acc += s[j] * vd;
                acc_abs += s[j] * fabs(vd);
            }
            out[(b * H + h) * D + d] = acc / sum;
            if (den) den[(b * H + h) * D + d] = acc_abs / sum;
        }
        free(s);
    }
    return fail ? -1 : 0;
}

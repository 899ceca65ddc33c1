// C ABI of the block-quantized matmul library (see include/lwq.h).
//
// Host side of the path: argument checks, the per-device workspace registry
// (one caller-owned arena per device, registered once), TMA descriptor
// encoding, the per-shape configuration table and the kernel launches.
// Nothing here allocates device memory or synchronizes the host inside
// lwq_matmul.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include <mutex>
#include <utility>

#include "../../include/lwq.h"
#include "lwq_gemm.cuh"
#include "lwq_gemv.cuh"
#include "lwq_gemv_simple.cuh"
#include "lwq_attn.cuh"

namespace lwq {
namespace {

constexpr int kMaxDevices = 64;
constexpr size_t kSmemLimit = 232448;  // 227 KB opt-in dynamic shared memory per block on sm_100
constexpr unsigned long long kTimeoutNs = 2000000000ull;  // bounded waits give up after 2 s

struct DeviceState {
    void *ws = nullptr;
    size_t ws_bytes = 0;
    bool registered = false;
    int sms = 0;
};

DeviceState g_dev[kMaxDevices];
std::mutex g_mu;
thread_local int t_last_launches = 0;

// ------------------------------------------------------- driver entry point
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

int current_device(int *dev) {
    if (cudaGetDevice(dev) != cudaSuccess || *dev < 0 || *dev >= kMaxDevices) return LWQ_ERR_CUDA;
    return LWQ_OK;
}

int sm_count(int dev) {
    if (g_dev[dev].sms == 0) {
        int v = 0;
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) v = 148;
        g_dev[dev].sms = v;
    }
    return g_dev[dev].sms;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int block_weights(int wf) {
    switch (wf) {
    case LWQ_Q8_0:
    case LWQ_Q4_0: return 32;
    case LWQ_Q4_K:
    case LWQ_Q6_K:
    case LWQ_Q5_K:
    case LWQ_Q2_K: return 256;
    default: return 0;
    }
}
int block_bytes(int wf) {
    switch (wf) {
    case LWQ_Q8_0: return 34;
    case LWQ_Q4_0: return 18;
    case LWQ_Q4_K: return 144;
    case LWQ_Q6_K: return 210;
    case LWQ_Q5_K: return 176;
    case LWQ_Q2_K: return 84;
    default: return 0;
    }
}
int act_code(int fmt) {
    switch (fmt & LWQ_ACT_MASK) {
    case LWQ_ACT_F32: return X_F32;
    case LWQ_ACT_F16: return X_F16;
    case LWQ_ACT_BF16: return X_BF16;
    default: return -1;
    }
}

int check_fmt_k(int fmt, long K) {
    const int wf = fmt & LWQ_FMT_MASK;
    if (fmt & ~(LWQ_FMT_MASK | LWQ_ACT_MASK | LWQ_FLAG_OVERLAP | LWQ_FLAG_ACT_I8)) return LWQ_ERR_UNSUPPORTED;
    if (block_weights(wf) == 0 || act_code(fmt) < 0) return LWQ_ERR_UNSUPPORTED;
    if (K <= 0 || K % block_weights(wf)) return LWQ_ERR_INVALID_ARG;
    return LWQ_OK;
}

// ---------------------------------------------------------- configuration
struct Plan {
    lwq_config cfg;
    int nt;          // GEMV n8 column tiles (activation rows x parts / 8)
    bool i8;         // GEMV with int8 activation blocks (LWQ_FLAG_ACT_I8)
    int m_group;     // activation rows per pass
    int cps;         // GEMV: chunks of 256 weights per split (the depth of one TMA box)
    int kw;          // GEMV: weights of K per compute warp and chunk at nt column tiles (256 or 128)
    size_t smem;
    size_t ws_need;  // workspace bytes for one pass
};

// n8 column tiles of the GEMV for a pass of mg activation rows: each row takes
// P columns (P = 3 bf16 parts for fp32 activations, else 1), 8 columns per tile.
inline int gemv_nt(int xt, bool i8, int mg) { return i8 ? 1 : (mg * gemv_parts(xt, i8) + 7) / 8; }
// bytes of one row of a chunk in a GEMV stage (Q6_K: its 240-byte box, see FmtInfo)
// The GEMV kernel format of a call: the library's format codes equal the
// kernels' (LWQ_Q8_0 == F_Q8_0, ...), except Q6_K rows that are not 16-byte
// multiples, which stream as row slots (F_Q6_KS).
inline int gemv_kfmt(int wf, long K) { return (wf == LWQ_Q6_K && K % 2048 != 0) ? F_Q6_KS : wf; }
inline int gemv_chunk_bytes(int kf) {
    switch (kf) {
    case F_Q8_0: return 272;
    case F_Q5_K: return 176;
    case F_Q6_K: return 240;
    case F_Q6_KS: return 210;
    case F_Q2_K: return 84;
    default: return 144;
    }
}
inline size_t gemv_smem(int kf, int cps, int stages, int nt, bool i8, int xt, int m) {
    return gemv_smem_layout(gemv_chunk_bytes(kf), cps, stages, nt, fmt_sums(kf), gemv_parts(xt, i8), m,
                            xt == X_F32 ? 4 : 2, i8, fmt_row_slots(kf))
        .total;
}

// Formats with a tensor-core GEMV decoder (all of them); tc_gemv_eligible adds
// the shape conditions of their weight streams.
bool tc_gemv_format(int wf) {
    return wf == LWQ_Q8_0 || wf == LWQ_Q4_0 || wf == LWQ_Q4_K || wf == LWQ_Q5_K || wf == LWQ_Q2_K || wf == LWQ_Q6_K;
}
// Q6_K rows are 210 bytes per superblock: with K a multiple of 2048 (8
// superblocks) they are 16-byte multiples and a tensor map takes them as its
// rows; otherwise, like Q2_K's 84-byte superblocks, they stream as row slots of
// the flat matrix, whose tensor map needs the whole matrix to be 16-byte units.
bool tc_gemv_eligible(int wf, long N, long K) {
    if (K % 256 != 0) return false;
    if (wf == LWQ_Q6_K) return K % 2048 == 0 || (N * (K / 256) * 210) % 16 == 0;
    if (wf == LWQ_Q2_K) return (N * (K / 256) * 84) % 16 == 0;
    return tc_gemv_format(wf);
}

// Workspace layout: fp32 split-K partials [S][m_group][N].  Nothing in it
// needs to start at any particular value.
size_t splitk_ws(int S, int m, int N) {
    if (S <= 1) return 0;
    return (size_t)S * m * N * 4;
}

int make_plan(int fmt, int M, int N, int K, const lwq_config *force, int sms, Plan *p) {
    const int wf = fmt & LWQ_FMT_MASK, xt = act_code(fmt);
    memset(p, 0, sizeof(*p));
    int path = force && force->path ? force->path : 0;
    if (fmt & LWQ_FLAG_ACT_I8) {
        // int8 activation blocks: tensor-core GEMV only
        if (path && path != 1) return LWQ_ERR_UNSUPPORTED;
        path = 1;
    }
    if (!path) {
        if (M > 16 && xt != X_F32 && gemm_eligible(wf, xt, N, K))
            path = 2;
        else if (tc_gemv_eligible(wf, N, K))
            path = 1;
        else
            path = 3;
    }
    p->cfg.path = path;
    if (path == 2) {
        if (!gemm_eligible(wf, xt, N, K)) return LWQ_ERR_UNSUPPORTED;
        GemmPlan gp;
        int rc = gemm_plan(wf, xt, M, N, K, force, sms, &gp);
        if (rc) return rc;
        p->cfg.warps = gp.warps;
        p->cfg.stages = gp.stages;
        p->cfg.splits = gp.splits;
        p->cfg.ctas = gp.ctas;
        p->cfg.tile_n = gp.tile_n;
        p->cfg.tile_m = gp.tile_m;
        p->smem = gp.smem;
        p->m_group = M;
        p->ws_need = splitk_ws(gp.splits, M, N);
        return LWQ_OK;
    }
    if (path == 3) {
        p->m_group = M < 16 ? M : 16;
        p->cfg.warps = 8;
        p->cfg.ctas = (N + 7) / 8;
        p->cfg.splits = 1;
        return LWQ_OK;
    }
    if (path != 1 || !tc_gemv_eligible(wf, N, K)) return LWQ_ERR_UNSUPPORTED;
    p->i8 = (fmt & LWQ_FLAG_ACT_I8) != 0;
    // int8 activation blocks: Q4_0, Q8_0 and Q4_K weights, any M (passes of 8 rows; every pass streams
    // the weights again, so a prefill-sized M reads them M / 8 times)
    if (p->i8 && wf != LWQ_Q4_0 && wf != LWQ_Q8_0 && wf != LWQ_Q4_K) return LWQ_ERR_UNSUPPORTED;
    // rows per pass: 8 with fp32 activations (3 parts, 24 columns) or int8 blocks, else 16
    const int mmax = (xt == X_F32 || p->i8) ? 8 : 16;
    p->m_group = M < mmax ? M : mmax;
    p->nt = gemv_nt(xt, p->i8, p->m_group);
    // K per warp and chunk: gemv_kw, except the K-quants at two tiles with K <= 4096, which take half a chunk:
    // their decoders spill with a whole chunk's B fragments (68-132 bytes), and two K splits of half chunks
    // measured faster than one of whole chunks (M = 9..12 of 16-bit x, M = 3, 4 of fp32 x: Q4_K 1.06-1.16x,
    // Q2_K up to 1.12x, none slower).  At K = 11008 the same choice was mixed (0.89-1.17x).
    const bool kq = wf == LWQ_Q4_K || wf == LWQ_Q5_K || wf == LWQ_Q6_K || wf == LWQ_Q2_K;
    const bool half = p->nt == 2 && kq && K <= 4096 && !(force && force->warps);
    const int kw = p->i8 ? 256 : (half ? CHUNK / 2 : gemv_kw(p->nt));
    const int wpc = CHUNK / kw;              // compute warps per chunk
    const int cmax = GEMV_W / wpc;           // chunks a CTA can hold
    const int nchunks = K / 256;
    int cpc = cmax;
    if (force && force->warps) {
        if (force->warps < 1 || force->warps > GEMV_W) return LWQ_ERR_UNSUPPORTED;
        cpc = force->warps / wpc > 0 ? force->warps / wpc : 1;
    }
    int S = force && force->splits ? force->splits : (nchunks + cpc - 1) / cpc;
    if (!(force && force->splits) && S > 1) {
        // K spans several CTAs: up to two more splits than the fewest when that lowers the
        // busiest CTA's work, tiles x (chunks + 4), the 4 standing for a tile's fixed cost
        // (its reduction and barrier round trips).  Q4_K, K = 11008, N = 4096: 3 splits leave
        // a CTA 6 tiles x 15 chunks, 4 splits 7 x 11.
        const int rt = (N + GEMV_ROWS - 1) / GEMV_ROWS;
        long best = -1;
        const int s_min = S;
        for (int s = s_min; s <= s_min + 2; ++s) {
            const int c = (nchunks + s - 1) / s;
            const int se = (nchunks + c - 1) / c;   // splits left after dropping empty ones
            const int g = sms / se;
            if (g < 1) continue;
            const long cost = (long)((rt + g - 1) / g) * (c + 4);
            if (best < 0 || cost < best) {
                best = cost;
                S = se;
            }
        }
    }
    if (S < 1) return LWQ_ERR_UNSUPPORTED;
    int cps = (nchunks + S - 1) / S;
    if (cps > cmax) return LWQ_ERR_UNSUPPORTED;  // every chunk of a split needs its warps
    // weight ring: 4 stages, fewer where shared memory is short (Q8_0 chunks
    // are twice as large, and the CTA's slice of x is staged too); with 2 stages
    // still too large, the CTA takes fewer chunks; a forced depth only has to fit
    const int mg = p->m_group;
    int stages = force && force->stages ? force->stages : 4;
    if (!(force && force->stages)) {
        while (stages > 2 && gemv_smem(gemv_kfmt(wf, K), cps, stages, p->nt, p->i8, xt, mg) > kSmemLimit) --stages;
        while (cps > 1 && !(force && force->splits) && gemv_smem(gemv_kfmt(wf, K), cps, stages, p->nt, p->i8, xt, mg) > kSmemLimit)
            --cps;
    }
    if (stages < 2 || gemv_smem(gemv_kfmt(wf, K), cps, stages, p->nt, p->i8, xt, mg) > kSmemLimit) return LWQ_ERR_UNSUPPORTED;
    S = (nchunks + cps - 1) / cps;               // drop empty splits
    if (!(force && force->splits)) {
        // even splits: shared memory that limited a CTA to cps chunks (K = 4096, 16 rows of 16-bit
        // x: 14) would otherwise leave the last split a remainder (2), and its CTAs idle beside the
        // others; the smaller slice may also leave room for more weight stages
        cps = (nchunks + S - 1) / S;
        if (!(force && force->stages))
            while (stages < 4 && gemv_smem(gemv_kfmt(wf, K), cps, stages + 1, p->nt, p->i8, xt, mg) <= kSmemLimit)
                ++stages;
    }
    const int row_tiles = (N + GEMV_ROWS - 1) / GEMV_ROWS;
    // one CTA per SM
    int groups = force && force->ctas ? force->ctas / S : sms / S;
    if (groups < 1) groups = 1;
    if (groups > row_tiles) groups = row_tiles;
    // Two column tiles whose K slice is 8 chunks or fewer (16-bit x with 9..16 rows, or fp32 x with 4 or 5 rows
    // where the staged slice leaves room for no more): half a chunk per warp, so that all 16 compute warps
    // work and each holds half the B fragments.  A warp per chunk left 8 warps idle and spilled registers.
    int kwe = kw;
    if (!p->i8 && p->nt == 2 && kw == CHUNK && 2 * cps <= GEMV_W && !(force && force->warps)) kwe = CHUNK / 2;
    p->kw = kwe;
    p->cps = cps;
    p->cfg.warps = cps * (CHUNK / kwe);
    p->cfg.stages = stages;
    p->cfg.splits = S;
    p->cfg.ctas = S * groups;
    p->smem = gemv_smem(gemv_kfmt(wf, K), cps, stages, p->nt, p->i8, xt, mg);
    p->ws_need = splitk_ws(S, p->m_group, N);
    return LWQ_OK;
}

// A GEMV plan whose split-K partials exceed the `have` bytes of workspace (none registered: 0) gives way to
// the plan with a warp per chunk, where that one needs no more: the K-quants' half chunks split K where a warp
// per chunk would not, and a call that fits without them still runs.  Forced configurations are kept.
int fit_plan(int fmt, int M, int N, int K, const lwq_config *force, int sms, size_t have, Plan *p) {
    if (force || p->cfg.path != 1 || p->ws_need <= have) return LWQ_OK;
    lwq_config whole = {};
    whole.path = 1;
    whole.warps = GEMV_W;
    Plan q;
    if (make_plan(fmt, M, N, K, &whole, sms, &q) == LWQ_OK && q.ws_need <= have) *p = q;
    return LWQ_OK;
}

// --------------------------------------------------------------- launches
// Launch on `st`; with `overlap`, as a programmatic dependent launch, so that
// the kernel may start (and prefetch weights) before the preceding kernel on
// the stream completes -- its other warps wait for that completion in-kernel.
template <typename... KArgs, typename... Args>
cudaError_t launch_k(void (*kern)(KArgs...), int ctas, int threads, size_t smem, cudaStream_t st, bool overlap,
                     Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)ctas);
    cfg.blockDim = dim3((unsigned)threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    if (overlap) {
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
    }
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// Raise a kernel's dynamic shared-memory limit once per (device, kernel), so
// that launches captured into CUDA graphs make no attribute calls.
cudaError_t ensure_smem(const void *kern, size_t smem) {
    struct Entry {
        int dev;
        const void *kern;
        size_t smem;
    };
    static Entry cache[256];
    static int n = 0;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lk(g_mu);
    for (int i = 0; i < n; ++i)
        if (cache[i].dev == dev && cache[i].kern == kern && cache[i].smem >= smem) return cudaSuccess;
    const size_t want = kSmemLimit;  // set the maximum once; any smaller launch fits
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)want);
    if (e != cudaSuccess) return e;
    if (n < 256) cache[n++] = Entry{dev, kern, want};
    return cudaSuccess;
}

template <int FMT, int XT, int NT, bool I8 = false, int KW = (I8 ? 256 : gemv_kw(NT))>
cudaError_t launch_gemv(const CUtensorMap &map, const GemvArgs &a, int ctas, size_t smem, cudaStream_t st) {
    auto kern = gemv_kernel<FMT, XT, NT, I8, KW>;
    cudaError_t e = ensure_smem(reinterpret_cast<const void *>(kern), smem);
    if (e != cudaSuccess) return e;
    return launch_k(kern, ctas, gemv_threads(FMT, NT), smem, st, a.overlap != 0, map, a);
}

// NT = n8 column tiles: fp32 activations take 1..3 (3 parts per row, 8 rows
// at most), 16-bit ones 1..2 (16 rows at most); int8 blocks one.  kw: the
// plan's K per warp and chunk at two tiles (128 or 256).
template <int FMT, int XT>
cudaError_t launch_gemv_nt(int nt, int kw, const CUtensorMap &map, const GemvArgs &a, int ctas, size_t smem,
                           cudaStream_t st) {
    if (nt == 1) return launch_gemv<FMT, XT, 1>(map, a, ctas, smem, st);
    if (nt == 2)
        return kw == CHUNK / 2 ? launch_gemv<FMT, XT, 2, false, CHUNK / 2>(map, a, ctas, smem, st)
                               : launch_gemv<FMT, XT, 2>(map, a, ctas, smem, st);
    if constexpr (XT == X_F32) {
        if (nt == 3) return launch_gemv<FMT, XT, 3>(map, a, ctas, smem, st);
    }
    return cudaErrorInvalidValue;
}

cudaError_t dispatch_gemv(int wf, int xt, int nt, int kw, bool i8, const CUtensorMap &map, const GemvArgs &a,
                          int ctas, size_t smem, cudaStream_t st) {
    if (i8) {
        if (nt != 1) return cudaErrorInvalidValue;
        if (wf == LWQ_Q4_0) {
            if (xt == X_F32) return launch_gemv<F_Q4_0, X_F32, 1, true>(map, a, ctas, smem, st);
            if (xt == X_F16) return launch_gemv<F_Q4_0, X_F16, 1, true>(map, a, ctas, smem, st);
            return launch_gemv<F_Q4_0, X_BF16, 1, true>(map, a, ctas, smem, st);
        }
        if (wf == LWQ_Q8_0) {
            if (xt == X_F32) return launch_gemv<F_Q8_0, X_F32, 1, true>(map, a, ctas, smem, st);
            if (xt == X_F16) return launch_gemv<F_Q8_0, X_F16, 1, true>(map, a, ctas, smem, st);
            return launch_gemv<F_Q8_0, X_BF16, 1, true>(map, a, ctas, smem, st);
        }
        if (wf == LWQ_Q4_K) {
            if (xt == X_F32) return launch_gemv<F_Q4_K, X_F32, 1, true>(map, a, ctas, smem, st);
            if (xt == X_F16) return launch_gemv<F_Q4_K, X_F16, 1, true>(map, a, ctas, smem, st);
            return launch_gemv<F_Q4_K, X_BF16, 1, true>(map, a, ctas, smem, st);
        }
        return cudaErrorInvalidValue;
    }
#define LWQ_GV(F)                                                                       \
    if (xt == X_F32) return launch_gemv_nt<F, X_F32>(nt, kw, map, a, ctas, smem, st);  \
    if (xt == X_F16) return launch_gemv_nt<F, X_F16>(nt, kw, map, a, ctas, smem, st);  \
    return launch_gemv_nt<F, X_BF16>(nt, kw, map, a, ctas, smem, st);
    switch (wf) {
    case LWQ_Q4_0: { LWQ_GV(F_Q4_0) }
    case LWQ_Q8_0: { LWQ_GV(F_Q8_0) }
    case LWQ_Q4_K: { LWQ_GV(F_Q4_K) }
    case LWQ_Q5_K: { LWQ_GV(F_Q5_K) }
    case LWQ_Q6_K: {
        if (a.K % 2048 != 0) { LWQ_GV(F_Q6_KS) }
        LWQ_GV(F_Q6_K)
    }
    case LWQ_Q2_K: { LWQ_GV(F_Q2_K) }
    }
#undef LWQ_GV
    return cudaErrorInvalidValue;
}

template <int FMT, int XT>
cudaError_t launch_simple(const uint8_t *W, const void *x, float *y, int M, int N, int K, long rb,
                          cudaStream_t st) {
    gemv_simple_kernel<FMT, XT><<<(N + 7) / 8, 256, 0, st>>>(W, x, y, M, N, K, rb);
    return cudaGetLastError();
}

cudaError_t dispatch_simple(int wf, int xt, const uint8_t *W, const void *x, float *y, int M, int N, int K, long rb,
                            cudaStream_t st) {
#define LWQ_SIMPLE(F)                                                                        \
    if (xt == X_F32) return launch_simple<F, X_F32>(W, x, y, M, N, K, rb, st);              \
    if (xt == X_F16) return launch_simple<F, X_F16>(W, x, y, M, N, K, rb, st);              \
    return launch_simple<F, X_BF16>(W, x, y, M, N, K, rb, st);
    switch (wf) {
    case LWQ_Q8_0: { LWQ_SIMPLE(F_Q8_0) }
    case LWQ_Q4_0: { LWQ_SIMPLE(F_Q4_0) }
    case LWQ_Q4_K: { LWQ_SIMPLE(F_Q4_K) }
    case LWQ_Q6_K: { LWQ_SIMPLE(F_Q6_K) }
    case LWQ_Q5_K: { LWQ_SIMPLE(F_Q5_K) }
    case LWQ_Q2_K: { LWQ_SIMPLE(F_Q2_K) }
    }
#undef LWQ_SIMPLE
    return cudaErrorInvalidValue;
}

// Tensor maps are encoded on the host for every call.  A map depends only on
// its arguments, so a small per-thread cache keyed by all of them (address,
// sizes, strides, box, type, swizzle) returns the same map again for a
// repeated call, as in a decode loop, without the driver call.
struct MapReq {
    void *p;
    uint32_t dtype, rank, swizzle, pad;
    cuuint64_t dims[3], strides[2];
    cuuint32_t box[3], pad2;
};
struct MapEntry {
    MapReq req;
    CUtensorMap map;
    bool valid;
};
constexpr int kMapCache = 16;
thread_local MapEntry t_maps[kMapCache];
thread_local int t_map_next = 0;

int encode_cached(const MapReq &r, CUtensorMap *out) {
    for (int i = 0; i < kMapCache; ++i)
        if (t_maps[i].valid && memcmp(&t_maps[i].req, &r, sizeof(MapReq)) == 0) {
            *out = t_maps[i].map;
            return LWQ_OK;
        }
    EncodeTiledFn enc = encode_fn();
    if (!enc) return LWQ_ERR_CUDA;
    const cuuint32_t estr[3] = {1, 1, 1};
    if (enc(out, (CUtensorMapDataType)r.dtype, r.rank, r.p, r.dims, r.strides, r.box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, (CUtensorMapSwizzle)r.swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return LWQ_ERR_CUDA;
    MapEntry &e = t_maps[t_map_next];
    t_map_next = (t_map_next + 1) % kMapCache;
    e.req = r;
    e.map = *out;
    e.valid = true;
    return LWQ_OK;
}

MapReq map_req(const void *p, CUtensorMapDataType dtype, int rank, CUtensorMapSwizzle swz) {
    MapReq r;
    memset(&r, 0, sizeof(r));   // the padding takes part in the comparison
    r.p = const_cast<void *>(p);
    r.dtype = (uint32_t)dtype;
    r.rank = (uint32_t)rank;
    r.swizzle = (uint32_t)swz;
    return r;
}

// The GEMV's view of Wq: 3-D, (8-byte word of a 256-weight chunk, weight row,
// chunk), strides (row_bytes, chunk_bytes); a box of (all words, 16 rows, cps
// chunks) lands as cps consecutive [16 rows][chunk bytes] boxes, one GEMV stage.
int encode_weight_map(CUtensorMap *map, const void *Wq, int wf, int N, long K, long rb, int cps) {
    const int kf = gemv_kfmt(wf, K);
    if (fmt_row_slots(kf)) {
        // row slots: the flat matrix as [N rb / 16 units][16 bytes], a box of whole units
        // covering one row's slice of a split and up to 7 units before it
        MapReq r = map_req(Wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, CU_TENSOR_MAP_SWIZZLE_NONE);
        r.dims[0] = 16;
        r.dims[1] = (cuuint64_t)((long)N * rb / 16);
        r.strides[0] = 16;
        r.box[0] = 16;
        r.box[1] = (cuuint32_t)gemv_slot_units(gemv_chunk_bytes(kf), cps);
        return encode_cached(r, map);
    }
    if (wf == LWQ_Q6_K) {
        // [N rows][rb / 2 words] with a box of [16 rows][120 words], one per chunk
        MapReq r = map_req(Wq, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, CU_TENSOR_MAP_SWIZZLE_NONE);
        r.dims[0] = (cuuint64_t)(rb / 2);
        r.dims[1] = (cuuint64_t)N;
        r.strides[0] = (cuuint64_t)rb;
        r.box[0] = 120;
        r.box[1] = (cuuint32_t)GEMV_ROWS;
        return encode_cached(r, map);
    }
    const int cb = gemv_chunk_bytes(kf);
    MapReq r = map_req(Wq, CU_TENSOR_MAP_DATA_TYPE_UINT64, 3, CU_TENSOR_MAP_SWIZZLE_NONE);
    r.dims[0] = (cuuint64_t)(cb / 8);
    r.dims[1] = (cuuint64_t)N;
    r.dims[2] = (cuuint64_t)(rb / cb);
    r.strides[0] = (cuuint64_t)rb;
    r.strides[1] = (cuuint64_t)cb;
    r.box[0] = (cuuint32_t)(cb / 8);
    r.box[1] = (cuuint32_t)GEMV_ROWS;
    r.box[2] = (cuuint32_t)cps;
    return encode_cached(r, map);
}

// ------------------------------------------------------------- prefill GEMM
template <int FMT, int XT, int H>
cudaError_t launch_gemm_tc(const CUtensorMap &wm, const CUtensorMap &xm, const GemmArgs &a, int ctas, size_t smem,
                           cudaStream_t st) {
    auto kern = gemm_tc_kernel<FMT, XT, H>;
    cudaError_t e = ensure_smem(reinterpret_cast<const void *>(kern), smem);
    if (e != cudaSuccess) return e;
    return launch_k(kern, ctas, GEMM_THREADS, smem, st, a.overlap != 0, wm, xm, a);
}

// h = 128-row halves of a weight tile
template <int FMT>
cudaError_t launch_gemm_xt(int xt, int h, const CUtensorMap &wm, const CUtensorMap &xm, const GemmArgs &a, int ctas,
                           size_t smem, cudaStream_t st) {
    if (xt == X_F16)
        return h == 2 ? launch_gemm_tc<FMT, X_F16, 2>(wm, xm, a, ctas, smem, st)
                      : launch_gemm_tc<FMT, X_F16, 1>(wm, xm, a, ctas, smem, st);
    return h == 2 ? launch_gemm_tc<FMT, X_BF16, 2>(wm, xm, a, ctas, smem, st)
                  : launch_gemm_tc<FMT, X_BF16, 1>(wm, xm, a, ctas, smem, st);
}

// Returns the kernels launched (1, or 2 with the split-K sum) through *launches.
int gemm_launch(int wf, int xt, const void *Wq, const void *x, float *y, int M, int N, int K, long rb,
                const lwq_config &cfg, size_t smem, unsigned long long timeout_ns, int overlap, float *partial,
                cudaStream_t st, int *launches) {
    const int cb = gemm_chunk_bytes(wf);
    const int bn = cfg.tile_m;
    const bool slots = gemm_row_slots(wf, K);
    CUtensorMap wm, xm;
    if (slots) {
        // row slots copy without a tensor map; the kernel's map argument is then this flat view
        // of the matrix as 16-byte units, which it does not read
        MapReq r = map_req(Wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, CU_TENSOR_MAP_SWIZZLE_NONE);
        r.dims[0] = 16;
        r.dims[1] = (cuuint64_t)((long)N * rb / 16);
        r.strides[0] = 16;
        r.box[0] = 16;
        r.box[1] = 1;
        if (encode_cached(r, &wm)) return LWQ_ERR_CUDA;
    } else {
        MapReq r = map_req(Wq, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, CU_TENSOR_MAP_SWIZZLE_NONE);
        r.dims[0] = (cuuint64_t)(rb / 2);
        r.dims[1] = (cuuint64_t)N;
        r.strides[0] = (cuuint64_t)rb;
        r.box[0] = (cuuint32_t)(cb / 2);
        r.box[1] = (cuuint32_t)GEMM_WROWS;
        if (encode_cached(r, &wm)) return LWQ_ERR_CUDA;
    }
    {
        MapReq r = map_req(x, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, CU_TENSOR_MAP_SWIZZLE_128B);
        r.dims[0] = (cuuint64_t)K;
        r.dims[1] = (cuuint64_t)M;
        r.strides[0] = (cuuint64_t)K * 2;
        r.box[0] = (cuuint32_t)GEMM_BK;
        r.box[1] = (cuuint32_t)bn;
        if (encode_cached(r, &xm)) return LWQ_ERR_CUDA;
    }
    GemmArgs a;
    a.y = y;
    a.splits = cfg.splits > 1 ? cfg.splits : 1;
    a.cps = (K / 256 + a.splits - 1) / a.splits;
    a.partial = partial;
    a.M = M;
    a.N = N;
    a.K = K;
    a.nchunks = K / 256;
    const int h = cfg.tile_n / GEMM_WROWS;   // 128-row halves of a weight tile
    if (h != 1 && h != 2) return LWQ_ERR_UNSUPPORTED;
    a.n_wtiles = (N + cfg.tile_n - 1) / cfg.tile_n;
    a.n_ttiles = (M + bn - 1) / bn;
    a.bn = bn;
    {
        // the same ring depths gemm_plan chose (its B ring is the configuration's stage count)
        lwq_config f = cfg;
        int na = 0, nb = 0, np = 0;
        if (!gemm_rings(gemm_chunk_bytes(wf), bn, h, &f, &na, &nb, &np)) return LWQ_ERR_UNSUPPORTED;
        a.a_stages = na;
        a.b_stages = nb;
        a.p_stages = np;
    }
    a.timeout_ns = timeout_ns;
    a.overlap = overlap;
    a.slots = slots ? 1 : 0;
    a.wq = Wq;
    a.row_bytes = rb;
    cudaError_t e;
    switch (wf) {
    case LWQ_Q4_0: e = launch_gemm_xt<F_Q4_0>(xt, h, wm, xm, a, cfg.ctas, smem, st); break;
    case LWQ_Q8_0: e = launch_gemm_xt<F_Q8_0>(xt, h, wm, xm, a, cfg.ctas, smem, st); break;
    case LWQ_Q5_K: e = launch_gemm_xt<F_Q5_K>(xt, h, wm, xm, a, cfg.ctas, smem, st); break;
    case LWQ_Q6_K: e = launch_gemm_xt<F_Q6_K>(xt, h, wm, xm, a, cfg.ctas, smem, st); break;
    case LWQ_Q2_K: e = launch_gemm_xt<F_Q2_K>(xt, h, wm, xm, a, cfg.ctas, smem, st); break;
    default: e = launch_gemm_xt<F_Q4_K>(xt, h, wm, xm, a, cfg.ctas, smem, st); break;
    }
    if (e != cudaSuccess) return LWQ_ERR_CUDA;
    *launches = 1;
    if (a.splits > 1) {
        // add the K slices in order: a programmatic dependent launch after the GEMM
        const long mn = (long)M * N;
        e = launch_k(gemv_splitk_sum_kernel, splitk_sum_blocks(mn), 256, 0, st, true,
                     static_cast<const float *>(partial), y, a.splits, mn);
        if (e != cudaSuccess) return LWQ_ERR_CUDA;
        *launches = 2;
    }
    return LWQ_OK;
}

// The GEMV passes of one call (shared by lwq_matmul and lwq_matmul_noalloc):
// one kernel per pass of m_group activation rows, plus the split-K sum kernel
// when K is split; `partial` holds that pass's [S][m][N] partial sums.
int gemv_run(const Plan &p, int fmt, const void *Wq, const void *x, float *y, int M, int N, int K, float *partial,
             int overlap, cudaStream_t st, int *launches) {
    const int wf = fmt & LWQ_FMT_MASK, xt = act_code(fmt);
    const long rb = (long)K / block_weights(wf) * block_bytes(wf);
    const size_t xelem = (xt == X_F32) ? 4 : 2;
    const int S = p.cfg.splits;
    CUtensorMap map;
    int rc = encode_weight_map(&map, Wq, wf, N, K, rb, p.cps);
    if (rc) return rc;
    int n = 0;
    for (int m0 = 0; m0 < M; m0 += p.m_group) {
        const int mg = (M - m0) < p.m_group ? (M - m0) : p.m_group;
        GemvArgs a;
        a.x = static_cast<const uint8_t *>(x) + (size_t)m0 * K * xelem;
        a.y = y + (size_t)m0 * N;
        a.partial = partial;
        a.M = mg;
        a.N = N;
        a.K = K;
        a.nchunks = K / 256;
        a.splits = S;
        a.cps = p.cps;
        a.row_tiles = (N + GEMV_ROWS - 1) / GEMV_ROWS;
        a.wstages = p.cfg.stages;
        a.timeout_ns = kTimeoutNs;
        a.overlap = overlap;
        const int nt = gemv_nt(xt, p.i8, mg);
        const int kw = nt == p.nt ? p.kw : gemv_kw(nt);   // a last, shorter pass may take fewer tiles
        cudaError_t e = dispatch_gemv(wf, xt, nt, kw, p.i8, map, a, p.cfg.ctas,
                                      gemv_smem(gemv_kfmt(wf, K), p.cps, p.cfg.stages, nt, p.i8, xt, mg), st);
        if (e != cudaSuccess) return LWQ_ERR_CUDA;
        ++n;
        if (S > 1) {
            const long mn = (long)mg * N;
            e = launch_k(gemv_splitk_sum_kernel, splitk_sum_blocks(mn), 256, 0, st, true,
                         static_cast<const float *>(partial), a.y, S, mn);
            if (e != cudaSuccess) return LWQ_ERR_CUDA;
            ++n;
        }
    }
    *launches = n;
    return LWQ_OK;
}

int run(int fmt, const void *Wq, const void *x, float *y, int M, int N, int K, const lwq_config *force,
        void *stream) {
    t_last_launches = 0;
    if (!Wq || !x || !y) return LWQ_ERR_INVALID_ARG;
    if (M <= 0 || N <= 0 || K <= 0) return LWQ_ERR_INVALID_ARG;
    int rc = check_fmt_k(fmt, K);
    if (rc) return rc;
    if (!aligned16(Wq) || !aligned16(x) || !aligned16(y)) return LWQ_ERR_MISALIGNED;
    int dev;
    if ((rc = current_device(&dev))) return rc;
    const int wf = fmt & LWQ_FMT_MASK, xt = act_code(fmt);
    const int overlap = (fmt & LWQ_FLAG_OVERLAP) ? 1 : 0;
    Plan p;
    if ((rc = make_plan(fmt, M, N, K, force, sm_count(dev), &p))) return rc;
    fit_plan(fmt, M, N, K, force, sm_count(dev), g_dev[dev].registered ? g_dev[dev].ws_bytes : 0, &p);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const long rb = (long)K / block_weights(wf) * block_bytes(wf);
    const size_t xelem = (xt == X_F32) ? 4 : 2;
    int launches = 0;

    if (p.cfg.path == 2) {
        DeviceState &ds = g_dev[dev];
        if (p.ws_need > 0) {
            if (!ds.registered) return LWQ_ERR_NOT_INITIALIZED;
            if (ds.ws_bytes < p.ws_need) return LWQ_ERR_WORKSPACE_TOO_SMALL;
        }
        int n = 0;
        rc = gemm_launch(wf, xt, Wq, x, y, M, N, K, rb, p.cfg, p.smem, kTimeoutNs, overlap,
                         static_cast<float *>(ds.ws), st, &n);
        if (rc) return rc;
        t_last_launches = n;
        return LWQ_OK;
    }
    if (p.cfg.path == 3) {
        for (int m0 = 0; m0 < M; m0 += 16) {
            const int mg = (M - m0) < 16 ? (M - m0) : 16;
            cudaError_t e = dispatch_simple(wf, xt, static_cast<const uint8_t *>(Wq),
                                            static_cast<const uint8_t *>(x) + (size_t)m0 * K * xelem,
                                            y + (size_t)m0 * N, mg, N, K, rb, st);
            if (e != cudaSuccess) return LWQ_ERR_CUDA;
            ++launches;
        }
        t_last_launches = launches;
        return LWQ_OK;
    }

    // tensor-core GEMV, in passes of m_group activation rows
    DeviceState &ds = g_dev[dev];
    if (p.ws_need > 0) {
        if (!ds.registered) return LWQ_ERR_NOT_INITIALIZED;
        if (ds.ws_bytes < p.ws_need) return LWQ_ERR_WORKSPACE_TOO_SMALL;
    }
    rc = gemv_run(p, fmt, Wq, x, y, M, N, K, static_cast<float *>(ds.ws), overlap, st, &launches);
    if (rc) return rc;
    t_last_launches = launches;
    return LWQ_OK;
}

// ------------------------------------------------------- decode attention
template <int XT, int D, int G>
cudaError_t launch_attn(const AttnArgs &a, cudaStream_t st) {
    const dim3 grid((unsigned)a.S, (unsigned)a.Hkv, (unsigned)a.B);
    if constexpr (G == 1) {
        attn_split_kernel<XT, D, G><<<grid, ATTN_WARPS * 32, 0, st>>>(a);
    } else {
        // grouped heads: the tensor-core pass (its K/V ring is dynamic shared memory)
        auto kern = attn_split_tc_kernel<XT, D, G>;
        constexpr size_t smem = attn_tc_smem<D>();
        cudaError_t e = ensure_smem(reinterpret_cast<const void *>(kern), smem);
        if (e != cudaSuccess) return e;
        kern<<<grid, ATTN_WARPS * 32, smem, st>>>(a);
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess || a.S == 1) return e;
    // the splits' merge: a programmatic dependent launch that waits for the split kernel; a CTA per
    // (sequence, head) and 32 columns
    return launch_k(attn_combine_kernel<D>, a.B * a.H * (D / 32), 32 * attn_combine_warps(a.S), 0, st, true,
                    (const float *)a.part, a.out, a.S);
}

template <int XT, int D>
cudaError_t launch_attn_g(int G, const AttnArgs &a, cudaStream_t st) {
    switch (G) {
    case 1: return launch_attn<XT, D, 1>(a, st);
    case 2: return launch_attn<XT, D, 2>(a, st);
    case 4: return launch_attn<XT, D, 4>(a, st);
    case 8: return launch_attn<XT, D, 8>(a, st);
    default: return cudaErrorInvalidValue;
    }
}

size_t attn_ws_bytes(int B, int H, int S, int D) { return S > 1 ? (size_t)B * H * S * (D + 2) * 4 : 0; }

int attn_check(int dtype, int B, int H, int Hkv, int Lmax, int D) {
    if (B <= 0 || H <= 0 || Hkv <= 0 || Lmax <= 0 || D <= 0) return LWQ_ERR_INVALID_ARG;
    if (dtype != LWQ_ACT_F16 && dtype != LWQ_ACT_BF16) return LWQ_ERR_UNSUPPORTED;
    if (D != 64 && D != 128) return LWQ_ERR_UNSUPPORTED;
    if (H % Hkv) return LWQ_ERR_INVALID_ARG;
    const int G = H / Hkv;
    if (G != 1 && G != 2 && G != 4 && G != 8) return LWQ_ERR_UNSUPPORTED;
    if (B > 65535 || Hkv > 65535) return LWQ_ERR_UNSUPPORTED;
    return LWQ_OK;
}

__global__ void selftest_timeout_kernel(unsigned long long timeout_ns) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        // nothing arrives on `bar`: the bounded wait must give up and report
        if (!mbar_wait(&bar, 0, timeout_ns, DEVERR_SELFTEST)) return;
    }
}

}  // namespace
}  // namespace lwq

using namespace lwq;

namespace lwq_noalloc {
void forget_device(int dev);   // lwq_noalloc.cuh: drop the cached scratch address
}

extern "C" {

size_t lwq_row_bytes(int fmt, int64_t K) {
    const int wf = fmt & LWQ_FMT_MASK;
    if (block_weights(wf) == 0 || K <= 0 || K % block_weights(wf)) return 0;
    return (size_t)(K / block_weights(wf)) * block_bytes(wf);
}

size_t lwq_workspace_size(int fmt, int max_M, int max_N, int max_K) {
    if (max_M <= 0 || max_N <= 0 || max_K <= 0) return 0;
    if (check_fmt_k(fmt, max_K)) return 0;
    int dev = 0;
    int sms = 148;
    if (current_device(&dev) == LWQ_OK) sms = sm_count(dev);
    // the need grows with M (up to one pass), N and K: evaluate at the maxima
    // and at every pass size the M loop can use
    size_t need = 0;
    for (int m = 1; m <= max_M && m <= 16; ++m) {
        Plan p;
        if (make_plan(fmt, m, max_N, max_K, nullptr, sms, &p) == LWQ_OK && p.ws_need > need) need = p.ws_need;
    }
    // The GEMM splits K only while its output tiles fill at most half the SMs, into
    // S <= ceil(sms / tiles) <= K / 1024 slices, so S * tiles <= 1.5 sms and each tile holds at most
    // 256 x 256 outputs: its partials never exceed 4 * 1.5 * sms * 65536 bytes, nor 4 * (K/1024) * M * N.
    if (max_M > 16 && (fmt & LWQ_ACT_MASK) != LWQ_ACT_F32) {
        const size_t by_grid = (size_t)6 * sms * 65536;
        const size_t by_shape = (size_t)4 * (max_K / 1024) * max_M * max_N;
        const size_t g = by_grid < by_shape ? by_grid : by_shape;
        if (g > need) need = g;
    }
    if (need < 256) need = 256;
    return need;
}

int lwq_init(void *d_workspace, size_t bytes) {
    int dev;
    int rc = current_device(&dev);
    if (rc) return rc;
    if (bytes > 0 && (!d_workspace || !aligned16(d_workspace))) return d_workspace ? LWQ_ERR_MISALIGNED : LWQ_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lk(g_mu);
    g_dev[dev].ws = bytes ? d_workspace : nullptr;
    g_dev[dev].ws_bytes = bytes;
    g_dev[dev].registered = true;
    return LWQ_OK;
}

int lwq_shutdown(void) {
    int dev;
    if (current_device(&dev) == LWQ_OK) {
        {
            std::lock_guard<std::mutex> lk(g_mu);
            g_dev[dev] = DeviceState{};
        }
        lwq_noalloc::forget_device(dev);
    }
    return LWQ_OK;
}

int lwq_matmul(int fmt, const void *Wq, const void *x, float *y, int M, int N, int K, void *stream) {
    return run(fmt, Wq, x, y, M, N, K, nullptr, stream);
}

int lwq_matmul_config(int fmt, const void *Wq, const void *x, float *y, int M, int N, int K, const lwq_config *cfg,
                      void *stream) {
    return run(fmt, Wq, x, y, M, N, K, cfg, stream);
}

int lwq_select_config(int fmt, int M, int N, int K, lwq_config *cfg) {
    if (!cfg || M <= 0 || N <= 0 || K <= 0) return LWQ_ERR_INVALID_ARG;
    int rc = check_fmt_k(fmt, K);
    if (rc) return rc;
    int dev = 0, sms = 148;
    if (current_device(&dev) == LWQ_OK) sms = sm_count(dev);
    Plan p;
    if ((rc = make_plan(fmt, M, N, K, nullptr, sms, &p))) return rc;
    *cfg = p.cfg;
    return LWQ_OK;
}

const char *lwq_status_string(int s) {
    switch (s) {
    case LWQ_OK: return "ok";
    case LWQ_ERR_INVALID_ARG: return "invalid argument";
    case LWQ_ERR_UNSUPPORTED: return "unsupported format, dtype or configuration";
    case LWQ_ERR_MISALIGNED: return "pointer not 16-byte aligned";
    case LWQ_ERR_NOT_INITIALIZED: return "workspace not registered (call lwq_init)";
    case LWQ_ERR_WORKSPACE_TOO_SMALL: return "workspace too small (see lwq_workspace_size)";
    case LWQ_ERR_CUDA: return "CUDA error";
    case LWQ_ERR_DEVICE_TIMEOUT: return "a kernel gave up a bounded wait";
    default: return "unknown status";
    }
}

int lwq_get_device_error(void) {
    unsigned v = 0;
    if (cudaMemcpyFromSymbol(&v, g_dev_error, sizeof(v)) != cudaSuccess) return LWQ_ERR_CUDA;
    if (v == 0) return LWQ_OK;
    unsigned zero = 0;
    if (cudaMemcpyToSymbol(g_dev_error, &zero, sizeof(zero)) != cudaSuccess) return LWQ_ERR_CUDA;
    return LWQ_ERR_DEVICE_TIMEOUT;
}

int lwq_selftest_timeout(unsigned timeout_us, void *stream) {
    selftest_timeout_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        (unsigned long long)timeout_us * 1000ull);
    return cudaGetLastError() == cudaSuccess ? LWQ_OK : LWQ_ERR_CUDA;
}

int lwq_last_launch_count(void) { return t_last_launches; }

size_t lwq_attention_workspace_size(int B, int H, int Hkv, int Lmax, int D) {
    if (attn_check(LWQ_ACT_F16, B, H, Hkv, Lmax, D)) return 0;
    int dev = 0, sms = 148;
    if (current_device(&dev) == LWQ_OK) sms = sm_count(dev);
    int S = 1, chunk = 0;
    attn_splits(B, H, Hkv, Lmax, sms, &S, &chunk);
    return attn_ws_bytes(B, H, S, D);
}

int lwq_attention_decode(int dtype, const void *q, const void *k, const void *v, const int32_t *seq_lens, float *out,
                         int B, int H, int Hkv, int Lmax, int D, float scale, void *stream) {
    t_last_launches = 0;
    if (!q || !k || !v || !out) return LWQ_ERR_INVALID_ARG;
    int rc = attn_check(dtype, B, H, Hkv, Lmax, D);
    if (rc) return rc;
    if (!isfinite(scale)) return LWQ_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) ||
        (reinterpret_cast<uintptr_t>(seq_lens) & 3u))
        return LWQ_ERR_MISALIGNED;
    int dev;
    if ((rc = current_device(&dev))) return rc;
    AttnArgs a;
    a.q = static_cast<const uint16_t *>(q);
    a.k = static_cast<const uint16_t *>(k);
    a.v = static_cast<const uint16_t *>(v);
    a.lens = seq_lens;
    a.out = out;
    a.B = B;
    a.H = H;
    a.Hkv = Hkv;
    a.Lmax = Lmax;
    a.qscale = scale * 1.4426950408889634f;   // log2(e): the kernels take exponentials as exp2
    attn_splits(B, H, Hkv, Lmax, sm_count(dev), &a.S, &a.chunk);
    DeviceState &ds = g_dev[dev];
    a.part = nullptr;
    const size_t need = attn_ws_bytes(B, H, a.S, D);
    if (need > 0) {
        if (!ds.registered) return LWQ_ERR_NOT_INITIALIZED;
        if (ds.ws_bytes < need) return LWQ_ERR_WORKSPACE_TOO_SMALL;
        a.part = static_cast<float *>(ds.ws);
    }
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int G = H / Hkv;
    cudaError_t e;
    if (dtype == LWQ_ACT_F16)
        e = D == 64 ? launch_attn_g<X_F16, 64>(G, a, st) : launch_attn_g<X_F16, 128>(G, a, st);
    else
        e = D == 64 ? launch_attn_g<X_BF16, 64>(G, a, st) : launch_attn_g<X_BF16, 128>(G, a, st);
    if (e != cudaSuccess) return LWQ_ERR_CUDA;
    t_last_launches = a.S > 1 ? 2 : 1;
    return LWQ_OK;
}

int lwq_version(void) { return 0x000100; }

}  // extern "C"

// The allocation-free entry point shares this translation unit, so the whole
// library is one device module: one copy of each kernel and of the device
// error word that every bounded wait sets.
#include "lwq_noalloc.cuh"

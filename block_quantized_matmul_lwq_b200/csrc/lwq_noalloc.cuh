// lwq_matmul_noalloc: the decode GEMV for callers that cannot allocate device
// memory.
//
// The regular entry point takes its split-K scratch from a workspace that the
// caller allocates and registers with lwq_init.  Some callers cannot do that:
// code running where the CUDA allocator may not be called (inside a custom
// allocator's own callbacks, in a process whose memory pool is fixed and fully
// handed out at start-up, or in a plugin that receives only input and output
// pointers from its host).  This variant needs nothing from them but Wq, x
// and y: its scratch is one static device array in this file, created when
// the library is loaded on a device and held until the process exits.
//
// Limits and behaviour:
//  * The scratch is kScratchBytes (4 MiB) of fp32 split-K partial sums.  A
//    call whose configuration needs more (lwq_workspace_size(fmt, M, N, K)
//    bytes) is rejected with LWQ_ERR_WORKSPACE_TOO_SMALL.
//  * Only the tensor-core GEMV is offered (M <= 16 and the shapes it takes);
//    other shapes return LWQ_ERR_UNSUPPORTED.
//  * The device address of the array is looked up once per device, with that
//    device current, on the first call made on it.  Make that first call
//    before any stream capture on the device.
//  * Every call shares the one array and it keeps the previous call's
//    contents; nothing in it needs to start at any value (partial sums are
//    written before they are read).  Calls whose kernels overlap on the GPU
//    (different streams without ordering between them) race on the array.
//  * Nothing here calls cudaMalloc, cudaFree or any allocating routine.
//  * A bounded wait that gives up in these kernels sets the library's device
//    error word, as in lwq_matmul (lwq_get_device_error); the call's outputs
//    are then not all written.
//
// This file is included by lwq_api.cu: the library is a single translation
// unit, so that the kernels it shares with lwq_matmul and the device error
// word each exist once.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <mutex>

#include "../../include/lwq.h"
#include "lwq_gemv.cuh"

namespace lwq_noalloc {

using namespace lwq;

constexpr size_t kScratchBytes = 4u << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

struct DevSlot {
    void *ptr = nullptr;
    bool ready = false;
};
static DevSlot g_slots[kMaxDevices];
static std::mutex g_mu;

// Device address of g_scratch on the current device (looked up once per device).
static int scratch_ptr(void **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return LWQ_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_slots[dev].ready) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || p == nullptr) return LWQ_ERR_CUDA;
        g_slots[dev].ptr = p;
        g_slots[dev].ready = true;
    }
    *out = g_slots[dev].ptr;
    return LWQ_OK;
}

static size_t smem_bytes(int wf, int nw, int stages, int ot) { return lwq::gemv_smem(wf, nw, stages, ot); }

}  // namespace lwq_noalloc

extern "C" int lwq_matmul_noalloc(int fmt, const void *Wq, const void *x, float *y, int M, int N, int K,
                                  void *stream) {
    using namespace lwq_noalloc;
    if (!Wq || !x || !y || M <= 0 || N <= 0 || K <= 0) return LWQ_ERR_INVALID_ARG;
    if (((uintptr_t)Wq | (uintptr_t)x | (uintptr_t)y) & 15u) return LWQ_ERR_MISALIGNED;
    lwq_config cfg;
    int rc = lwq_select_config(fmt, M, N, K, &cfg);  // argument checks and the configuration table
    if (rc) return rc;
    if (cfg.path != 1 || M > 16) return LWQ_ERR_UNSUPPORTED;
    const int wf = fmt & LWQ_FMT_MASK;
    const int xt = (fmt & LWQ_ACT_MASK) == LWQ_ACT_F32 ? X_F32 : ((fmt & LWQ_ACT_MASK) == LWQ_ACT_F16 ? X_F16 : X_BF16);
    const bool i8 = (fmt & LWQ_FLAG_ACT_I8) != 0;
    const int m_group = (xt == X_F32 || i8) ? (M < 8 ? M : 8) : M;
    const int S = cfg.splits;
    const int row_tiles = (N + GEMV_ROWS - 1) / GEMV_ROWS;
    if (S > 1 && (size_t)S * m_group * N * 4 > kScratchBytes) return LWQ_ERR_WORKSPACE_TOO_SMALL;
    void *scratch = nullptr;
    if ((rc = scratch_ptr(&scratch))) return rc;
    const long rb = (long)lwq_row_bytes(fmt, K);
    const int nchunks = K / 256;
    const int cps = (nchunks + S - 1) / S;
    CUtensorMap map;   // one box per stage, as lwq_matmul's
    if ((rc = lwq::encode_weight_map(&map, Wq, wf, N, rb, cps))) return rc;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const size_t xelem = (xt == X_F32) ? 4 : 2;
    for (int m0 = 0; m0 < M; m0 += m_group) {
        const int mg = (M - m0) < m_group ? (M - m0) : m_group;
        GemvArgs a;
        a.x = static_cast<const uint8_t *>(x) + (size_t)m0 * K * xelem;
        a.y = y + (size_t)m0 * N;
        a.partial = static_cast<float *>(scratch);
        a.M = mg;
        a.N = N;
        a.K = K;
        a.nchunks = nchunks;
        a.splits = S;
        a.chunks_per_split = cps;
        a.row_tiles = row_tiles;
        a.stages = cfg.stages;
        a.timeout_ns = lwq::kTimeoutNs;   // the library's 2 s wait bound
        a.overlap = 0;
        // n8 column tiles, as lwq_matmul picks them
        const int nt = i8 ? 1 : lwq::gemv_nt(wf, xt, mg);
        const int ot = lwq::gemv_ot(xt, nt);
        cudaError_t e = lwq::dispatch_gemv_tc(wf, xt, nt, mg == 1 && !i8, i8, map, a, cfg.ctas, cfg.warps,
                                 smem_bytes(wf, cfg.warps, cfg.stages, ot), st);
        if (e != cudaSuccess) return LWQ_ERR_CUDA;
        if (S > 1) {
            // add the splits in order: a programmatic dependent launch after the GEMV
            const long mn = (long)mg * N;
            cudaLaunchConfig_t lc = {};
            lc.gridDim = dim3((unsigned)splitk_sum_blocks(mn));
            lc.blockDim = dim3(256u);
            lc.stream = st;
            cudaLaunchAttribute at[1];
            at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
            at[0].val.programmaticStreamSerializationAllowed = 1;
            lc.attrs = at;
            lc.numAttrs = 1;
            if (cudaLaunchKernelEx(&lc, gemv_splitk_sum_kernel, static_cast<const float *>(a.partial), a.y, S, mn) !=
                cudaSuccess)
                return LWQ_ERR_CUDA;
        }
    }
    return LWQ_OK;
}

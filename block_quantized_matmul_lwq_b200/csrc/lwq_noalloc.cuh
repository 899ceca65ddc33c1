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
//    before any stream capture on the device.  lwq_shutdown forgets the
//    address on the current device (call it after a device reset, which can
//    move the array); the next call looks it up again.
//  * LWQ_FLAG_OVERLAP is honoured as in lwq_matmul: the kernels then wait for
//    the preceding work on the stream before they read x or write y or the
//    scratch.
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

// Drop the cached address of the current device (lwq_shutdown).
void forget_device(int dev) {
    if (dev < 0 || dev >= kMaxDevices) return;
    std::lock_guard<std::mutex> lk(g_mu);
    g_slots[dev] = DevSlot{};
}

}  // namespace lwq_noalloc

extern "C" int lwq_matmul_noalloc(int fmt, const void *Wq, const void *x, float *y, int M, int N, int K,
                                  void *stream) {
    using namespace lwq_noalloc;
    if (!Wq || !x || !y || M <= 0 || N <= 0 || K <= 0) return LWQ_ERR_INVALID_ARG;
    int rc = lwq::check_fmt_k(fmt, K);
    if (rc) return rc;
    if (((uintptr_t)Wq | (uintptr_t)x | (uintptr_t)y) & 15u) return LWQ_ERR_MISALIGNED;
    int dev = 0;
    if ((rc = lwq::current_device(&dev))) return rc;
    lwq::Plan p;
    if ((rc = lwq::make_plan(fmt, M, N, K, nullptr, lwq::sm_count(dev), &p))) return rc;
    lwq::fit_plan(fmt, M, N, K, nullptr, lwq::sm_count(dev), kScratchBytes, &p);
    if (p.cfg.path != 1 || M > 16) return LWQ_ERR_UNSUPPORTED;
    if (p.ws_need > kScratchBytes) return LWQ_ERR_WORKSPACE_TOO_SMALL;
    void *scratch = nullptr;
    if ((rc = scratch_ptr(&scratch))) return rc;
    int launches = 0;
    return lwq::gemv_run(p, fmt, Wq, x, y, M, N, K, static_cast<float *>(scratch),
                         (fmt & LWQ_FLAG_OVERLAP) ? 1 : 0, reinterpret_cast<cudaStream_t>(stream), &launches);
}

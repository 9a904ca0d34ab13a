// Candidate scoring for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc (or any allocator) at request time: a
// serving runtime that forbids allocation on its hot path, or a host that
// manages all GPU memory through a pool it does not share with this library.
// ot_score_candidates needs a caller-provided workspace; this entry point
// instead uses a fixed scratch array that is part of the library's device
// image.  The array exists on every GPU that loads the library and stays
// there until the process exits.
//
// Set-up: in host code the array's name is only a host-side stand-in, not a
// device address.  The first call on a device (with that device current)
// asks the runtime for the array's address there (cudaGetSymbolAddress) and
// keeps it for that device and its current context; a call that finds a
// different context (the old one was torn down, e.g. by cudaDeviceReset)
// does the set-up again.  That first call should come before any stream
// capture.  Every call on a device shares the one array and leaves its
// contents behind; nothing in the scoring path reads scratch it has not
// first written in the same call, so no clearing is needed.  Calls that
// overlap on the GPU (other streams, other host threads) race on the array
// and must be serialised by the caller.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <mutex>

#include "ot_internal.h"

static __device__ __align__(256) unsigned char ot_noalloc_scratch[OT_NOALLOC_SCRATCH_BYTES];

namespace {
constexpr int kMaxDevices = 64;

struct ScratchSlot {
    void *addr;                  // device address of the array, or null
    unsigned long long ctx_id;   // the context it was looked up in
};
ScratchSlot g_slot[kMaxDevices];
std::mutex g_scratch_mu;
PFN_cuCtxGetCurrent_v4000 g_ctx_current = nullptr;
PFN_cuCtxGetId_v12000 g_ctx_id = nullptr;

// Unique id of the calling thread's current context (0 if unavailable).
unsigned long long current_ctx_id()
{
    if (!g_ctx_current || !g_ctx_id) {
        void *f1 = nullptr, *f2 = nullptr;
        cudaDriverEntryPointQueryResult q1, q2;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f1, cudaEnableDefault, &q1) != cudaSuccess ||
            cudaGetDriverEntryPoint("cuCtxGetId", &f2, cudaEnableDefault, &q2) != cudaSuccess ||
            q1 != cudaDriverEntryPointSuccess || q2 != cudaDriverEntryPointSuccess || !f1 || !f2)
            return 0;
        g_ctx_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(f1);
        g_ctx_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(f2);
    }
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (g_ctx_current(&ctx) != CUDA_SUCCESS || !ctx || g_ctx_id(ctx, &id) != CUDA_SUCCESS) return 0;
    return id;
}
} // namespace

extern "C" ot_status ot_score_candidates_noalloc(ot_model *m, const void *kv_cache, int U,
                                                 const void *ns, int C, void *out_ns, void *stream)
{
    if (!m || !kv_cache || !ns || !out_ns || U < 1 || C < 1) return OT_ERR_ARG;
    // the checks ot_score_candidates makes, before the scratch size
    auto aligned16 = [](const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; };
    if (!aligned16(kv_cache) || !aligned16(ns) || !aligned16(out_ns)) return OT_ERR_ALIGN;
    const long long n_ns = ot::internal_n_ns(m);
    if (static_cast<long long>(U) * C * n_ns > (1LL << 31) - 1) return OT_ERR_SHAPE;
    if (static_cast<long long>(C) * n_ns > (1LL << 30)) return OT_ERR_SHAPE;
    // per-launch profiling would create CUDA events during the call
    if (ot::internal_profiling(m)) return OT_ERR_UNSUPPORTED;
    const size_t need = ot::internal_score_ws_bytes(m, U, C);
    if (need == 0) return OT_ERR_SHAPE;
    if (need > OT_NOALLOC_SCRATCH_BYTES) return OT_ERR_WORKSPACE_TOO_SMALL;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return OT_ERR_CUDA;
    if (dev != ot::internal_device(m)) return OT_ERR_ARG;
    const unsigned long long ctx = current_ctx_id();
    if (ctx == 0) return OT_ERR_CUDA;
    void *scratch = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_scratch_mu);
        ScratchSlot &slot = g_slot[dev];
        if (!slot.addr || slot.ctx_id != ctx) {
            // set-up for this device and context, with the device current
            void *p = nullptr;
            if (cudaGetSymbolAddress(&p, ot_noalloc_scratch) != cudaSuccess || !p) return OT_ERR_CUDA;
            slot.addr = p;
            slot.ctx_id = ctx;
        }
        scratch = slot.addr;
    }
    return ot_score_candidates(m, kv_cache, U, ns, C, out_ns, scratch, OT_NOALLOC_SCRATCH_BYTES,
                               stream);
}

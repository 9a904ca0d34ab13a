// Candidate scoring for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc (or any allocator) at request time: a
// serving runtime that forbids allocation on its hot path, code running while
// a stream is being captured, or a host that manages GPU memory through a
// pool it does not share with this library.  ot_score_candidates needs a
// caller-provided workspace; this entry point instead uses a fixed scratch
// array that is part of the library's device image.  The array exists on
// every GPU that loads the library and stays there until the process exits.
//
// Set-up: the first call on a device (with that device current) looks up the
// array's device address with cudaGetSymbolAddress and caches it for the
// device.  That first call should come before any stream capture.
// Every call on a device shares the one array and leaves its contents behind;
// nothing in the scoring path reads scratch it has not first written, so no
// clearing is needed.  Calls that overlap on the GPU (other streams, other
// host threads) race on the array and must be serialised by the caller.
#include <cuda_runtime.h>

#include <mutex>

#include "ot_internal.h"

static __device__ __align__(256) unsigned char ot_noalloc_scratch[OT_NOALLOC_SCRATCH_BYTES];

namespace {
constexpr int kMaxDevices = 64;
void *g_scratch_by_device[kMaxDevices];
std::mutex g_scratch_mu;
} // namespace

extern "C" ot_status ot_score_candidates_noalloc(ot_model *m, const void *kv_cache, int U,
                                                 const void *ns, int C, void *out_ns, void *stream)
{
    if (!m || !kv_cache || !ns || !out_ns || U < 1 || C < 1) return OT_ERR_ARG;
    // per-launch profiling would create CUDA events during the call
    if (ot::internal_profiling(m)) return OT_ERR_UNSUPPORTED;
    const size_t need = ot::internal_score_ws_bytes(m, U, C);
    if (need == 0) return OT_ERR_SHAPE;
    if (need > OT_NOALLOC_SCRATCH_BYTES) return OT_ERR_WORKSPACE_TOO_SMALL;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return OT_ERR_CUDA;
    if (dev != ot::internal_device(m)) return OT_ERR_ARG;
    void *scratch = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_scratch_mu);
        scratch = g_scratch_by_device[dev];
        if (!scratch) {
            // the host-side name of the array is not a device address: ask the
            // runtime for this device's copy once, with the device current
            if (cudaGetSymbolAddress(&scratch, ot_noalloc_scratch) != cudaSuccess || !scratch)
                return OT_ERR_CUDA;
            g_scratch_by_device[dev] = scratch;
        }
    }
    return ot_score_candidates(m, kv_cache, U, ns, C, out_ns, scratch, OT_NOALLOC_SCRATCH_BYTES,
                               stream);
}

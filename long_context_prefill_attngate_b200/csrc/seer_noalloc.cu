// seer_noalloc.cu — seer_gate_scores_noalloc: the AttnGate scores call for
// callers that cannot allocate device memory.
//
// Who needs it: code embedded in a host application whose memory pool owns
// all device memory and forbids side allocations, and latency-critical paths
// where cudaMalloc (which may synchronise the device) or a pool round trip is
// not acceptable.  Such callers can still pass their inputs and outputs, but
// cannot provide the gate's workspace.  This entry point supplies it from a
// fixed array compiled into the library instead.
//
// The array is a file-scope device variable of kNoAllocScratchBytes (24 MiB):
// every GPU that loads the library holds it until the process exits.  It is
// enough for a layer with (B*Hq*(d + d_gate) + B*Hkv*(dk + d_gate)) * (S/64) * 4
// bytes of gate workspace up to 24 MiB, dk = d (average K pooling) or 2d
// (max+min K pooling) — for example the 32k-token Llama-3.1-8B layer, 32/8
// heads, d = d_gate = 128: 21 MB (23 MB with max+min).  Larger shapes are rejected with
// SEER_ERR_UNSUPPORTED before anything is launched.
//
// All calls share the one array and it keeps whatever the last call left in
// it.  Nothing in it has to start at zero: every byte the kernels read is
// written earlier in the same call.  Two calls whose kernels overlap on the
// GPU (for example on two streams without ordering between them) race on the
// array and give wrong results; order them on one stream or with events.
//
// The device address of the array is looked up once per device, with that
// device current, on the first call made on it (cudaGetSymbolAddress; host
// code must not hand the array's host-side name to a kernel).  Make that first
// call before any stream capture.  No memory is allocated by this file.
#include <mutex>

#include <cuda_runtime.h>

#include "../../include/seer.h"
#include "seer_internal.h"

namespace seer {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(24) << 20;

static __device__ __align__(256) unsigned char g_gate_scratch[kNoAllocScratchBytes];

// Per-device address of g_gate_scratch, resolved with the device current.
void *scratch_address(cudaError_t *err)
{
    static std::mutex mu;
    static void *cache[64] = {nullptr};
    int dev = 0;
    *err = cudaGetDevice(&dev);
    if (*err != cudaSuccess)
        return nullptr;
    if (dev < 0 || dev >= 64) {
        *err = cudaErrorInvalidDevice;
        return nullptr;
    }
    std::lock_guard<std::mutex> lk(mu);
    if (cache[dev] == nullptr) {
        void *p = nullptr;
        *err = cudaGetSymbolAddress(&p, g_gate_scratch);
        if (*err != cudaSuccess)
            return nullptr;
        cache[dev] = p;
    }
    return cache[dev];
}

} // namespace
} // namespace seer

extern "C" seer_status seer_gate_scores_noalloc(const seer_shape *shape, const void *q, const void *k,
                                                const void *wq, const void *wk, const seer_gate_params *gp,
                                                float *scores, void *stream)
{
    using namespace seer;
    // Shapes the workspace call would reject are passed on to it unchanged,
    // so the error text is the same; only the size limit is checked here.
    if (shape != nullptr && gp != nullptr && shape->B > 0 && shape->Hq > 0 && shape->Hkv > 0 &&
        shape->S > 0 && shape->d > 0 && gp->d_gate > 0) {
        const size_t need = gate_workspace_bytes(shape->B, shape->Hq, shape->Hkv, shape->S, shape->d, gp->d_gate,
                                                 gp->k_pooling == SEER_KPOOL_MAXMIN);
        if (need > kNoAllocScratchBytes)
            return set_last_error(SEER_ERR_UNSUPPORTED,
                                  "seer_gate_scores_noalloc: this shape needs %zu bytes of gate scratch; the "
                                  "library's fixed scratch holds %zu bytes (use seer_gate_scores with a workspace)",
                                  need, kNoAllocScratchBytes);
    }
    cudaError_t err = cudaSuccess;
    void *scratch = scratch_address(&err);
    if (scratch == nullptr)
        return set_last_error(SEER_ERR_CUDA, "seer_gate_scores_noalloc: cannot resolve the scratch address: %s",
                              cudaGetErrorString(err));
    return seer_gate_scores(shape, q, k, wq, wk, gp, scores, scratch, kNoAllocScratchBytes, stream);
}

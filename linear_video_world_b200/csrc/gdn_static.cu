// hlta_gdn_chunk_fwd_static: the chunkwise gated delta rule for callers that are not allowed
// to allocate device memory. Its scratch (the chunk workspace that hlta_gdn_chunk_fwd takes as
// an argument) lives in a fixed array compiled into this library instead of caller memory.
//
// Who needs this: code that runs inside a host application that owns the whole device-memory
// budget and hands plugins only their inputs and outputs, or a latency-critical loop that must
// never enter the allocator (an allocation can block, fragment the heap or fail under memory
// pressure in the middle of a rollout). Such callers pass inputs and outputs only.
//
// The array is part of this library's device image, so every GPU on which the library is used
// keeps HLTA_STATIC_SCRATCH_BYTES reserved until the process exits.
#include "hlta.h"
#include "hlta_internal.cuh"

#include <mutex>

namespace hlta {
namespace {

constexpr size_t kStaticScratchBytes = (size_t)HLTA_STATIC_SCRATCH_BYTES;

// The shared scratch. In host code this name is only a stand-in for the symbol, never a
// device address: the device address is looked up per device with cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_gdn_scratch[kStaticScratchBytes];

constexpr int kMaxDev = 64;
void *g_scratch_addr[kMaxDev];
std::mutex g_scratch_mu;

// Device address of the scratch on the current device (looked up once per device).
hlta_status scratch_address(void **out)
{
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return record_error(HLTA_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    if (dev < 0 || dev >= kMaxDev) return record_error(HLTA_ERR_UNSUPPORTED, "device %d", dev);
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    if (!g_scratch_addr[dev]) {
        void *ptr = nullptr;
        e = cudaGetSymbolAddress(&ptr, g_gdn_scratch);
        if (e != cudaSuccess || !ptr)
            return record_error(HLTA_ERR_CUDA, "cudaGetSymbolAddress(static scratch): %s",
                                cudaGetErrorString(e));
        g_scratch_addr[dev] = ptr;
    }
    *out = g_scratch_addr[dev];
    return HLTA_OK;
}

}  // namespace
}  // namespace hlta

extern "C" hlta_status hlta_gdn_chunk_fwd_static(const void *q, const void *k, const void *v,
                                                 const float *a, const float *b, void *o,
                                                 const float *S0, float *S_out, int B, int H,
                                                 long L, int d, int chunk, hlta_dtype dt,
                                                 void *stream)
{
    using namespace hlta;
    const size_t need = hlta_gdn_workspace_bytes(B, H, L, d, chunk, dt);
    if (need > kStaticScratchBytes)
        return record_error(HLTA_ERR_INVALID_ARG,
                            "this problem needs %zu bytes of scratch; the built-in scratch of "
                            "hlta_gdn_chunk_fwd_static holds %zu bytes (use hlta_gdn_chunk_fwd "
                            "with a caller-provided workspace)",
                            need, kStaticScratchBytes);
    void *scratch = nullptr;
    hlta_status st = scratch_address(&scratch);
    if (st != HLTA_OK) return st;
    // Nothing in the scratch has to start at zero: the chunk preparation writes every
    // element the state pass reads. Stale contents of an earlier call are simply overwritten.
    return hlta_gdn_chunk_fwd(q, k, v, a, b, o, S0, S_out, B, H, L, d, chunk, scratch,
                              kStaticScratchBytes, dt, stream);
}

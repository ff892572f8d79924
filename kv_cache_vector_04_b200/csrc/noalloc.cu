// tq_attend_noalloc: decode attention whose scratch lives in a static device
// array, for callers that cannot allocate device memory.
//
// tq_attend needs a workspace (the query fragments and the split-K partial
// results). Most callers pass one they allocated. Some cannot: runtimes whose
// memory is owned by a caching allocator they do not control, and real-time
// serving loops that forbid allocation after start-up. This entry point takes
// its scratch from a file-scope __device__ array of TQ_NOALLOC_SCRATCH_BYTES
// instead. The array exists on every GPU that loads this library, for as long
// as the process runs.
//
// Rules that follow from sharing one array:
//  - Calls that overlap on a GPU (other streams, other threads, other
//    contexts of this library) race on the array: serialize them.
//  - The array keeps whatever the last call wrote; nothing in it has to
//    start at zero, because every call writes all the scratch it reads.
//  - The host cannot pass the array's name to a kernel (in host code it is
//    only a stand-in): its device address is looked up with
//    cudaGetSymbolAddress once per device, on the first call made with that
//    device current, and kept for the life of the process. A cudaDeviceReset (which also
//    invalidates every context's tables) can move the array: do not use the
//    library across one.
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>

#include "device_common.cuh"
#include "kernels.h"
#include "tq.h"

// The scratch: 16 MiB covers, e.g., 16 sequences x 8 kv heads at any context
// length (split-K partials grow with the number of splits, which is bounded
// by the SM count, not by the context).
static __device__ __align__(256) unsigned char g_noalloc_scratch[TQ_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::atomic<void*> g_scratch_addr[kMaxDevices];

// Device address of the scratch on the current device (looked up once).
int scratch_for_current_device(void** out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return TQ_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return TQ_ERR_DEVICE;
    void* p = g_scratch_addr[dev].load(std::memory_order_acquire);
    if (!p) {
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return TQ_ERR_CUDA;
        g_scratch_addr[dev].store(p, std::memory_order_release);
    }
    *out = p;
    return TQ_OK;
}

}  // namespace

extern "C" int tq_attend_noalloc(tq_ctx* ctx, const void* q, int q_dtype, int B, int Hq,
                                 const tq_cache* cache, const int32_t* seq_len, int max_len,
                                 float* out, void* stream)
{
    if (!ctx || !cache) return TQ_ERR_INVALID_ARG;
    if (B <= 0 || Hq <= 0 || cache->Hkv <= 0 || Hq % cache->Hkv != 0 || max_len < 0)
        return TQ_ERR_INVALID_ARG;
    size_t need = 0;
    int rc = tq_attend_workspace(ctx, B, Hq, cache->Hkv, max_len, &need);
    if (rc != TQ_OK) return rc;
    if (need > (size_t)TQ_NOALLOC_SCRATCH_BYTES) return TQ_ERR_WORKSPACE;
    void* scratch = nullptr;
    if ((rc = scratch_for_current_device(&scratch)) != TQ_OK) return rc;
    return tq_attend(ctx, q, q_dtype, B, Hq, cache, seq_len, max_len, out, scratch,
                     (size_t)TQ_NOALLOC_SCRATCH_BYTES, stream);
}

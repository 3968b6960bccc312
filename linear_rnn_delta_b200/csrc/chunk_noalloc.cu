// Allocation-free variant of the split form of the chunked forward: the
// workspace lives in a fixed, file-scope device array instead of memory the
// caller or the library allocates.
//
// Who needs it: callers that may not allocate device memory at call time --
// an engine whose allocator has reserved all of HBM up front and hands out no
// more, a runtime with a hard device-memory budget, or a latency-critical
// loop that cannot absorb cudaMalloc's cost and the implicit device
// synchronisation it may bring.  They pass inputs and outputs only.
//
// Cost of the array: every GPU that loads this library holds it, 64 MiB,
// until the process exits.
#include <mutex>

#include "common.cuh"

namespace kda {
namespace {

// Room for 64 MiB / 82944 B = 809 (chunk slot, head) pairs of the split form.
constexpr size_t NOALLOC_SCRATCH_BYTES = 64ull << 20;
static __device__ __align__(256) unsigned char g_chunk_scratch[NOALLOC_SCRATCH_BYTES];

// Device address of the array on the current device.  In host code the
// array's name is only a host-side stand-in, so the address must come from
// cudaGetSymbolAddress, once per device, with that device current.  The
// address is kept for the life of the process: a cudaDeviceReset, which
// unloads the module, makes it stale (the header forbids calls after one).
cudaError_t scratch_address(void **ptr)
{
    static std::mutex mu;
    static void *addr[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_chunk_scratch);
        if (e != cudaSuccess) return e;
        addr[dev] = p;
    }
    *ptr = addr[dev];
    return cudaSuccess;
}

}  // namespace

size_t chunk_noalloc_capacity() { return NOALLOC_SCRATCH_BYTES; }

cudaError_t launch_chunk_split_noalloc(const FwdArgs &a, cudaStream_t st)
{
    void *ws = nullptr;
    cudaError_t e = scratch_address(&ws);
    if (e != cudaSuccess) return e;
    // Nothing in the workspace has to start at zero: each slot is written in
    // full before it is read, and a slot left over from an earlier call
    // carries that call's epoch tag, which the chain kernel rejects.
    return launch_chunk_split_sm100(a, ws, st);
}

}  // namespace kda

// noalloc.cu -- small-M forward that needs no memory from the caller's allocator.
//
// bsl_forward_stream needs a scratch buffer for the fp32 partial sums of block
// rows that are cut between warps.  Some callers cannot hand one over: code
// that must not call cudaMalloc once it is running (a serving loop with a
// fixed memory budget, where an allocation can block on the device or fail
// under fragmentation), plug-ins and custom operators inside another
// framework that owns all device memory and gives the library no allocator,
// and setups where device allocation is forbidden after start-up.  For them,
// bsl_forward_stream_noalloc runs the same kernels with the scratch taken
// from a fixed array in this library's own device memory.
//
// The array is a file-scope __device__ variable.  The runtime loads it on a
// device the first time this file's module is used there (this entry
// point's first call on that device), which takes BSL_NOALLOC_SCRATCH_BYTES
// of device memory and can fail if the device is full; the device then keeps
// it until the process exits.  Host code must not use the array's name as a
// device address (on the host it only names a host-side stand-in), so the
// device address is looked up once per device with cudaGetSymbolAddress,
// with that device current, cached, and passed to the kernel.  The cache
// assumes the device's primary context lives as long as the process.
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace bsl {
namespace {

static __device__ __align__(256) unsigned char g_scratch[BSL_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxScratchDevices = 64;
void *g_scratch_addr[kMaxScratchDevices] = {nullptr};
std::mutex g_scratch_mutex;

// Device address of g_scratch on the current device (looked up on first use).
bsl_status scratch_address(void **out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return BSL_ERR_NO_DEVICE;
    if (dev >= kMaxScratchDevices) return BSL_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_scratch);
        if (e != cudaSuccess || !p) return cuda_status(e != cudaSuccess ? e : cudaErrorInvalidSymbol);
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return BSL_OK;
}

}  // namespace
}  // namespace bsl

using namespace bsl;

extern "C" bsl_status bsl_forward_stream_noalloc(const void *X, int32_t M, const bsl_bsr *W, void *Y, void *stream)
{
    const bsl_status st = check_bsr(W);
    if (st != BSL_OK) return st;
    if (!X || !Y || M <= 0) return BSL_ERR_INVALID_ARG;
    if (M > bsl_small_m_max()) return BSL_ERR_UNSUPPORTED;
    // the scratch lives on the device that owns X: make it current first
    DeviceGuard guard;
    bsl_status b = guard.bind(X);
    if (b != BSL_OK) return b;
    if ((b = check_device()) != BSL_OK) return b;
    if (stream_workspace_bytes(M, W) > BSL_NOALLOC_SCRATCH_BYTES) return BSL_ERR_SCRATCH_TOO_SMALL;
    void *scratch = nullptr;
    if ((b = scratch_address(&scratch)) != BSL_OK) return b;
    return bsl_forward_stream(X, M, W, nullptr, Y, scratch, BSL_NOALLOC_SCRATCH_BYTES, stream);
}

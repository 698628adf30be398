// api.cu -- the extern "C" entry points of libbsl: argument checks, tensor
// map encoding, dispatch to the kernels.  No entry point allocates memory.
#include <stdio.h>
#include <stdlib.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace bsl {

namespace {

constexpr int kMaxDevices = 64;
constexpr int32_t kSmallMMax = 32;

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
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

uint64_t g_timeout_ns = 0;
std::once_flag g_timeout_once;

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

bsl_status check_matrix(const void *p, int64_t rows)
{
    if (rows > 0 && (!p || !aligned(p, 16))) return BSL_ERR_INVALID_ARG;
    return BSL_OK;
}

#define BSL_TRY(expr)                          \
    do {                                       \
        const bsl_status st_ = (expr);         \
        if (st_ != BSL_OK) return st_;         \
    } while (0)

}  // namespace

// device must be sm_100 (B200 family); result cached per device
bsl_status check_device()
{
    static int ok_cache[kMaxDevices] = {0};  // 0 unknown, 1 ok, 2 bad
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return BSL_ERR_NO_DEVICE;
    if (dev < kMaxDevices && ok_cache[dev]) return ok_cache[dev] == 1 ? BSL_OK : BSL_ERR_NO_DEVICE;
    int major = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
        return BSL_ERR_NO_DEVICE;
    const bool ok = major == 10;
    if (dev < kMaxDevices) ok_cache[dev] = ok ? 1 : 2;
    return ok ? BSL_OK : BSL_ERR_NO_DEVICE;
}

// Make the device that owns `p` current for this host thread (this also
// binds its primary context, which a fresh thread may not have yet), and
// reject pointers that are not device memory.  The call is made even when the
// runtime already reports that device: on a thread that has made no runtime
// call yet (PyTorch's autograd thread, for one) no context is bound, and the
// driver-level tensor-map encoding would then fail.
bsl_status bind_device(const void *p)
{
    cudaPointerAttributes a;
    if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
        cudaGetLastError();  // clear the non-sticky error
        return BSL_ERR_INVALID_ARG;
    }
    if (a.type != cudaMemoryTypeDevice && a.type != cudaMemoryTypeManaged) return BSL_ERR_INVALID_ARG;
    if (cudaSetDevice(a.device) != cudaSuccess) return BSL_ERR_NO_DEVICE;
    return BSL_OK;
}

bsl_status check_bsr(const bsl_bsr *W)
{
    if (!W) return BSL_ERR_INVALID_ARG;
    if (W->b != 32 && W->b != 64) return BSL_ERR_UNSUPPORTED;
    if (W->N <= 0 || W->K <= 0 || W->N % W->b || W->K % W->b || W->nnz < 0) return BSL_ERR_INVALID_ARG;
    const int64_t R = W->N / W->b, C = W->K / W->b;
    if (W->nnz > R * C) return BSL_ERR_INVALID_ARG;
    if (R >= (1 << 24) || C >= (1 << 24)) return BSL_ERR_UNSUPPORTED;  // plan entries hold 24-bit coordinates
    const void *ptrs[] = {W->row_ptr, W->col_ptr, W->row_order, W->col_order, W->rgrp_ptr,
                          W->rgrp_bptr, W->cgrp_ptr, W->cgrp_bptr, W->status, W->sched, W->sbounds};
    for (const void *p : ptrs)
        if (!p || !aligned(p, 4)) return BSL_ERR_INVALID_ARG;
    if (W->nnz > 0) {
        const void *nz[] = {W->col_idx, W->row_idx, W->csc_to_bsr, W->rgrp_ent, W->rgrp_blk, W->cgrp_ent,
                            W->cgrp_blk};
        for (const void *p : nz)
            if (!p || !aligned(p, 4)) return BSL_ERR_INVALID_ARG;
        if (!W->values || !aligned(W->values, 16)) return BSL_ERR_INVALID_ARG;
    }
    return BSL_OK;
}

bsl_status check_semi24(const bsl_semi24 *W)
{
    if (!W) return BSL_ERR_INVALID_ARG;
    if (W->N <= 0 || W->K <= 0 || W->N % 8 || W->K % 64) return BSL_ERR_INVALID_ARG;
    if (!W->values || !aligned(W->values, 16) || !W->meta || !aligned(W->meta, 16) || !W->status ||
        !aligned(W->status, 4))
        return BSL_ERR_INVALID_ARG;
    return BSL_OK;
}

namespace {
thread_local int g_last_cuda_error = 0;  // last CUDA error seen by this host thread
}

bsl_status cuda_status(cudaError_t e)
{
    if (e == cudaSuccess) return BSL_OK;
    g_last_cuda_error = static_cast<int>(e);
    return BSL_ERR_CUDA;
}

void note_driver_error(int code) { g_last_cuda_error = -code; }

int num_sms()
{
    static int cache[kMaxDevices] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < kMaxDevices && cache[dev]) return cache[dev];
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 1;
    if (dev < kMaxDevices) cache[dev] = n;
    return n;
}

bsl_status set_smem_once(const void *func, int bytes)
{
    struct Entry {
        const void *func;
        int dev;
    };
    static Entry done[64];
    static int ndone = 0;
    static std::mutex mu;
    int dev = 0;
    cudaGetDevice(&dev);
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < ndone; ++i)
        if (done[i].func == func && done[i].dev == dev) return BSL_OK;
    const cudaError_t e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return cuda_status(e);
    if (ndone < 64) done[ndone++] = Entry{func, dev};
    return BSL_OK;
}

uint64_t wait_timeout_ns()
{
    std::call_once(g_timeout_once, [] {
        if (g_timeout_ns == 0) {
            uint64_t us = 2000000ull;
            if (const char *e = getenv("BSL_WAIT_TIMEOUT_US")) {
                const unsigned long long v = strtoull(e, nullptr, 10);
                if (v > 0) us = v;
            }
            g_timeout_ns = us * 1000ull;
        }
    });
    return g_timeout_ns;
}

bool make_map_2d(CUtensorMap *map, const void *base, uint64_t inner, uint64_t outer, uint64_t row_bytes,
                 uint32_t box_inner, uint32_t box_outer, int swizzle_bytes)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) {
        note_driver_error(999);
        return false;
    }
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {row_bytes};
    const cuuint32_t box[2] = {box_inner, box_outer};
    const cuuint32_t estr[2] = {1, 1};
    const CUtensorMapSwizzle sw = swizzle_bytes == 128  ? CU_TENSOR_MAP_SWIZZLE_128B
                                  : swizzle_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                  : swizzle_bytes == 32 ? CU_TENSOR_MAP_SWIZZLE_32B
                                                        : CU_TENSOR_MAP_SWIZZLE_NONE;
    const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box,
                          estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) note_driver_error(static_cast<int>(r));
    return r == CUDA_SUCCESS;
}

bool make_map_3d(CUtensorMap *map, const void *base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t stride1,
                 uint64_t stride2, uint32_t box0, uint32_t box1, int swizzle_bytes)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) {
        note_driver_error(999);
        return false;
    }
    const cuuint64_t dims[3] = {d0, d1, d2 > 0 ? d2 : 1};
    const cuuint64_t strides[2] = {stride1, stride2};
    const cuuint32_t box[3] = {box0, box1, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    const CUtensorMapSwizzle sw = swizzle_bytes == 128  ? CU_TENSOR_MAP_SWIZZLE_128B
                                  : swizzle_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                  : swizzle_bytes == 32 ? CU_TENSOR_MAP_SWIZZLE_32B
                                                        : CU_TENSOR_MAP_SWIZZLE_NONE;
    const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box,
                          estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) note_driver_error(static_cast<int>(r));
    return r == CUDA_SUCCESS;
}

bool make_block_map(CUtensorMap *map, const void *values, int32_t b, int32_t nblocks, uint32_t box_rows)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) {
        note_driver_error(999);
        return false;
    }
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(b), static_cast<cuuint64_t>(b),
                                static_cast<cuuint64_t>(nblocks > 0 ? nblocks : 1)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(b) * 2, static_cast<cuuint64_t>(b) * b * 2};
    const cuuint32_t box[3] = {static_cast<cuuint32_t>(b), box_rows, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(values), dims, strides, box,
                          estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          b == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) note_driver_error(static_cast<int>(r));
    return r == CUDA_SUCCESS;
}

namespace {
__global__ void k_debug_wait(int32_t *status, uint64_t timeout_ns)
{
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);  // nothing ever arrives on it
        fence_barrier_init();
        if (!mbar_wait(&bar, 0, timeout_ns, nullptr)) set_status(status, BSL_ERR_TIMEOUT);
    }
}
}  // namespace

bsl_status launch_debug_wait(int32_t *status, uint64_t timeout_ns, cudaStream_t s)
{
    k_debug_wait<<<1, 32, 0, s>>>(status, timeout_ns);
    return cuda_status(cudaGetLastError());
}

}  // namespace bsl

using namespace bsl;

extern "C" {

const char *bsl_status_string(bsl_status s)
{
    switch (s) {
    case BSL_OK: return "BSL_OK";
    case BSL_ERR_INVALID_ARG: return "BSL_ERR_INVALID_ARG";
    case BSL_ERR_UNSUPPORTED: return "BSL_ERR_UNSUPPORTED";
    case BSL_ERR_CUDA: return "BSL_ERR_CUDA";
    case BSL_ERR_TIMEOUT: return "BSL_ERR_TIMEOUT";
    case BSL_ERR_NNZ_MISMATCH: return "BSL_ERR_NNZ_MISMATCH";
    case BSL_ERR_NO_DEVICE: return "BSL_ERR_NO_DEVICE";
    case BSL_ERR_SCRATCH_TOO_SMALL: return "BSL_ERR_SCRATCH_TOO_SMALL";
    case BSL_ERR_NOT_2_4: return "BSL_ERR_NOT_2_4";
    }
    return "BSL_ERR_UNKNOWN";
}

const char *bsl_last_cuda_error(void)
{
    thread_local char buf[160];
    const int e = g_last_cuda_error;
    if (e == 0) return "none";
    if (e > 0)
        snprintf(buf, sizeof buf, "cuda runtime error %d (%s)", e, cudaGetErrorName(static_cast<cudaError_t>(e)));
    else
        snprintf(buf, sizeof buf, "cuda driver error %d (tensor map encoding)", -e);
    return buf;
}

bsl_status bsl_pack_count(const uint8_t *mask, int32_t R, int32_t C, int32_t *row_ptr, int32_t *nnz_host,
                          void *stream)
{
    if (!mask || !row_ptr || !nnz_host || R <= 0 || C <= 0) return BSL_ERR_INVALID_ARG;
    DeviceGuard guard;
    BSL_TRY(guard.bind(row_ptr));
    BSL_TRY(check_device());
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    BSL_TRY(launch_pack_count(mask, R, C, row_ptr, s));
    BSL_TRY(cuda_status(cudaMemcpyAsync(nnz_host, row_ptr + R, sizeof(int32_t), cudaMemcpyDeviceToHost, s)));
    return cuda_status(cudaStreamSynchronize(s));
}

bsl_status bsl_pack(const void *W, const uint8_t *mask, const bsl_bsr *out, void *stream)
{
    BSL_TRY(check_bsr(out));
    if (!mask || check_matrix(W, out->N) != BSL_OK) return BSL_ERR_INVALID_ARG;
    DeviceGuard guard;
    BSL_TRY(guard.bind(W));
    BSL_TRY(check_device());
    return launch_pack(W, mask, out, static_cast<cudaStream_t>(stream));
}

int32_t bsl_small_m_max(void) { return kSmallMMax; }

size_t bsl_forward_workspace_bytes(int32_t M, const bsl_bsr *W)
{
    if (check_bsr(W) != BSL_OK || M <= 0 || M > kSmallMMax) return 0;
    return stream_workspace_bytes(M, W);
}

bsl_status bsl_forward_tc(const void *X, int32_t M, const bsl_bsr *W, const void *bias, void *Y, void *stream)
{
    BSL_TRY(check_bsr(W));
    if (M <= 0 || check_matrix(X, M) != BSL_OK || check_matrix(Y, M) != BSL_OK) return BSL_ERR_INVALID_ARG;
    if (bias && !aligned(bias, 16)) return BSL_ERR_INVALID_ARG;
    DeviceGuard guard;
    BSL_TRY(guard.bind(X));
    BSL_TRY(check_device());
    return launch_spmm_tc(X, M, W->K, W, false, bias, Y, W->N, static_cast<cudaStream_t>(stream));
}

bsl_status bsl_forward_stream(const void *X, int32_t M, const bsl_bsr *W, const void *bias, void *Y,
                              void *workspace, size_t workspace_bytes, void *stream)
{
    BSL_TRY(check_bsr(W));
    if (M <= 0 || check_matrix(X, M) != BSL_OK || check_matrix(Y, M) != BSL_OK) return BSL_ERR_INVALID_ARG;
    if (bias && !aligned(bias, 16)) return BSL_ERR_INVALID_ARG;
    if (M > kSmallMMax) return BSL_ERR_UNSUPPORTED;
    DeviceGuard guard;
    BSL_TRY(guard.bind(X));
    BSL_TRY(check_device());
    if (!workspace || !aligned(workspace, 16) || workspace_bytes < stream_workspace_bytes(M, W))
        return BSL_ERR_INVALID_ARG;
    return launch_stream_fwd(X, M, W, bias, Y, workspace, static_cast<cudaStream_t>(stream));
}

bsl_status bsl_forward(const void *X, int32_t M, const bsl_bsr *W, const void *bias, void *Y, void *workspace,
                       size_t workspace_bytes, void *stream)
{
    if (M > 0 && M <= kSmallMMax)
        return bsl_forward_stream(X, M, W, bias, Y, workspace, workspace_bytes, stream);
    return bsl_forward_tc(X, M, W, bias, Y, stream);
}

bsl_status bsl_backward_input(const void *dY, int32_t M, const bsl_bsr *W, void *dX, void *stream)
{
    BSL_TRY(check_bsr(W));
    if (M <= 0 || check_matrix(dY, M) != BSL_OK || check_matrix(dX, M) != BSL_OK) return BSL_ERR_INVALID_ARG;
    DeviceGuard guard;
    BSL_TRY(guard.bind(dY));
    BSL_TRY(check_device());
    return launch_spmm_tc(dY, M, W->N, W, true, nullptr, dX, W->K, static_cast<cudaStream_t>(stream));
}

bsl_status bsl_bias_grad(const void *dY, int32_t M, int32_t N, void *dbias, void *stream)
{
    if (M <= 0 || N <= 0 || N % 32 || check_matrix(dY, M) != BSL_OK || !dbias || !aligned(dbias, 16))
        return BSL_ERR_INVALID_ARG;
    DeviceGuard guard;
    BSL_TRY(guard.bind(dY));
    BSL_TRY(check_device());
    return launch_bias_grad(dY, M, N, dbias, static_cast<cudaStream_t>(stream));
}

bsl_status bsl_backward_weight(const void *dY, const void *X, int32_t M, const bsl_bsr *W, void *dW_values,
                               void *stream)
{
    BSL_TRY(check_bsr(W));
    if (M <= 0 || check_matrix(dY, M) != BSL_OK || check_matrix(X, M) != BSL_OK) return BSL_ERR_INVALID_ARG;
    if (W->nnz > 0 && (!dW_values || !aligned(dW_values, 16))) return BSL_ERR_INVALID_ARG;
    DeviceGuard guard;
    BSL_TRY(guard.bind(dY));
    BSL_TRY(check_device());
    return launch_sddmm_tc(dY, X, M, W, dW_values, static_cast<cudaStream_t>(stream));
}

bsl_status bsl_get_device_status(const bsl_bsr *W, int32_t *status_host, void *stream)
{
    if (!W || !W->status || !status_host) return BSL_ERR_INVALID_ARG;
    DeviceGuard guard;
    BSL_TRY(guard.bind(W->status));
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    BSL_TRY(cuda_status(cudaMemcpyAsync(status_host, W->status, sizeof(int32_t), cudaMemcpyDeviceToHost, s)));
    BSL_TRY(cuda_status(cudaMemsetAsync(W->status, 0, sizeof(int32_t), s)));
    return cuda_status(cudaStreamSynchronize(s));
}

bsl_status bsl_semi24_compress(const void *W, const bsl_semi24 *out, void *stream)
{
    BSL_TRY(check_semi24(out));
    if (check_matrix(W, out->N) != BSL_OK) return BSL_ERR_INVALID_ARG;
    DeviceGuard guard;
    BSL_TRY(guard.bind(W));
    BSL_TRY(check_device());
    return launch_compress24(W, out, static_cast<cudaStream_t>(stream));
}

bsl_status bsl_semi24_forward(const void *X, int32_t M, const bsl_semi24 *W, const void *bias, void *Y,
                              void *stream)
{
    BSL_TRY(check_semi24(W));
    if (M <= 0 || check_matrix(X, M) != BSL_OK || check_matrix(Y, M) != BSL_OK) return BSL_ERR_INVALID_ARG;
    if (bias && !aligned(bias, 16)) return BSL_ERR_INVALID_ARG;
    DeviceGuard guard;
    BSL_TRY(guard.bind(X));
    BSL_TRY(check_device());
    return launch_semi24_fwd(X, M, W, bias, Y, static_cast<cudaStream_t>(stream));
}

bsl_status bsl_bsr24_compress(const bsl_bsr *W, void *values24, uint16_t *meta24, void *stream)
{
    BSL_TRY(check_bsr(W));
    if (!values24 || !aligned(values24, 16) || (W->nnz > 0 && (!meta24 || !aligned(meta24, 16))))
        return BSL_ERR_INVALID_ARG;
    DeviceGuard guard;
    BSL_TRY(guard.bind(values24));
    BSL_TRY(check_device());
    return launch_bsr24_compress(W, values24, meta24, static_cast<cudaStream_t>(stream));
}

bsl_status bsl_bsr24_forward(const void *X, int32_t M, const bsl_bsr *W, const void *values24,
                             const uint16_t *meta24, const void *bias, void *Y, void *stream)
{
    BSL_TRY(check_bsr(W));
    if (M <= 0 || check_matrix(X, M) != BSL_OK || check_matrix(Y, M) != BSL_OK) return BSL_ERR_INVALID_ARG;
    if (!values24 || !aligned(values24, 16) || (W->nnz > 0 && (!meta24 || !aligned(meta24, 16))))
        return BSL_ERR_INVALID_ARG;
    if (bias && !aligned(bias, 16)) return BSL_ERR_INVALID_ARG;
    DeviceGuard guard;
    BSL_TRY(guard.bind(X));
    BSL_TRY(check_device());
    return launch_bsr24_fwd(X, M, W, values24, meta24, bias, Y, static_cast<cudaStream_t>(stream));
}

bsl_status bsl_semi24_get_status(const bsl_semi24 *W, int32_t *status_host, void *stream)
{
    if (!W || !W->status || !status_host) return BSL_ERR_INVALID_ARG;
    DeviceGuard guard;
    BSL_TRY(guard.bind(W->status));
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    BSL_TRY(cuda_status(cudaMemcpyAsync(status_host, W->status, sizeof(int32_t), cudaMemcpyDeviceToHost, s)));
    BSL_TRY(cuda_status(cudaMemsetAsync(W->status, 0, sizeof(int32_t), s)));
    return cuda_status(cudaStreamSynchronize(s));
}

void bsl_set_wait_timeout_us(uint64_t timeout_us)
{
    wait_timeout_ns();  // settle the environment default first
    g_timeout_ns = (timeout_us ? timeout_us : 1) * 1000ull;
}

bsl_status bsl_debug_wait_timeout(int32_t *status, uint64_t timeout_us, void *stream)
{
    if (!status || !aligned(status, 4)) return BSL_ERR_INVALID_ARG;
    DeviceGuard guard;
    BSL_TRY(guard.bind(status));
    BSL_TRY(check_device());
    return launch_debug_wait(status, timeout_us * 1000ull, static_cast<cudaStream_t>(stream));
}

}  // extern "C"

// internal.h -- host-side declarations shared by the libbsl translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <utility>

#include "bsl.h"

namespace bsl {

// Encode a 2-D bf16 tensor map: `inner` contiguous elements per row, `outer`
// rows, `row_bytes` between rows, box of box_inner x box_outer elements.
// swizzle_bytes: 0, 64 or 128.  Returns false if the driver rejects it.
bool make_map_2d(CUtensorMap *map, const void *base, uint64_t inner, uint64_t outer, uint64_t row_bytes,
                 uint32_t box_inner, uint32_t box_outer, int swizzle_bytes);

// Encode a 3-D bf16 tensor map: d0 contiguous elements, d1 rows `stride1`
// bytes apart, d2 planes `stride2` bytes apart; box of box0 x box1 x 1.
bool make_map_3d(CUtensorMap *map, const void *base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t stride1,
                 uint64_t stride2, uint32_t box0, uint32_t box1, int swizzle_bytes);

// Encode the packed weight values bf16 [nblocks][b][b] as a 3-D tensor map
// (x = column inside a block, y = row inside a block, z = block) with a
// box of b columns x box_rows rows x 1 block, swizzled like the kernels'
// shared-memory operands (128-byte rows for b = 64, 64-byte rows for b = 32).
bool make_block_map(CUtensorMap *map, const void *values, int32_t b, int32_t nblocks, uint32_t box_rows);

int num_sms();
// Argument and device checks shared by the entry points (api.cu).
bsl_status bind_device(const void *p);  // make the device owning p current

// Makes the device owning a pointer current for the duration of an entry
// point and puts the caller's current device back when it goes out of scope.
class DeviceGuard {
public:
    DeviceGuard() { cudaGetDevice(&prev_); }
    ~DeviceGuard()
    {
        int now = -1;
        if (cudaGetDevice(&now) == cudaSuccess && now != prev_) cudaSetDevice(prev_);
    }
    bsl_status bind(const void *p) { return bind_device(p); }
    DeviceGuard(const DeviceGuard &) = delete;
    DeviceGuard &operator=(const DeviceGuard &) = delete;

private:
    int prev_ = 0;
};

// Launch a kernel that may begin while the previous kernel in the stream is
// finishing (programmatic stream serialization).  The kernel must wait for
// the prior grid (wait_for_prior_grid, common.cuh) before its first global
// memory access; results and ordering are those of a plain launch.
template <typename... KArgs, typename... Args>
cudaError_t launch_dependent(void (*kern)(KArgs...), unsigned grid, unsigned block, size_t smem, cudaStream_t s,
                             Args &&...args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// cudaFuncSetAttribute(MaxDynamicSharedMemorySize) once per kernel and device.
bsl_status set_smem_once(const void *func, int bytes);
bsl_status check_device();              // current device is sm_100
bsl_status check_bsr(const bsl_bsr *W);
bsl_status check_semi24(const bsl_semi24 *W);
uint64_t wait_timeout_ns();
bsl_status cuda_status(cudaError_t e);
void note_driver_error(int code);

// Kernel launchers (defined next to their kernels).
bsl_status launch_pack(const void *W, const uint8_t *mask, const bsl_bsr *out, cudaStream_t s);
bsl_status launch_pack_count(const uint8_t *mask, int32_t R, int32_t C, int32_t *row_ptr, cudaStream_t s);

// Forward (A = X, segments = block rows) and input gradient (A = dY,
// segments = block columns through the CSC index) share one engine.
// bias: bf16 [out_cols] added to every output row (forward only; may be null).
bsl_status launch_spmm_tc(const void *A, int32_t M, int32_t a_cols, const bsl_bsr *W, bool transposed,
                          const void *bias, void *out, int32_t out_cols, cudaStream_t s);

bsl_status launch_sddmm_tc(const void *dY, const void *X, int32_t M, const bsl_bsr *W, void *dW,
                           cudaStream_t s);

size_t stream_workspace_bytes(int32_t M, const bsl_bsr *W);
bsl_status launch_stream_fwd(const void *X, int32_t M, const bsl_bsr *W, const void *bias, void *Y, void *ws,
                             cudaStream_t s);
bsl_status launch_bias_grad(const void *dY, int32_t M, int32_t N, void *dbias, cudaStream_t s);

// 2:4 semi-structured weight: compress a dense weight, forward on the sparse MMA.
bsl_status launch_compress24(const void *W, const bsl_semi24 *out, cudaStream_t s);
bsl_status launch_semi24_fwd(const void *X, int32_t M, const bsl_semi24 *W, const void *bias, void *Y,
                             cudaStream_t s);

// Block-sparse weight with 2:4 inside its blocks: compress the kept blocks,
// forward on the sparse MMA driven by the row-group plan.
bsl_status launch_bsr24_compress(const bsl_bsr *W, void *values24, uint16_t *meta24, cudaStream_t s);
bsl_status launch_bsr24_fwd(const void *X, int32_t M, const bsl_bsr *W, const void *values24,
                            const uint16_t *meta24, const void *bias, void *Y, cudaStream_t s);

bsl_status launch_debug_wait(int32_t *status, uint64_t timeout_ns, cudaStream_t s);

}  // namespace bsl

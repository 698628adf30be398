// internal.h -- host-side declarations shared by the libbsl translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "bsl.h"

namespace bsl {

// Encode a 2-D bf16 tensor map: `inner` contiguous elements per row, `outer`
// rows, `row_bytes` between rows, box of box_inner x box_outer elements.
// swizzle_bytes: 0, 64 or 128.  Returns false if the driver rejects it.
bool make_map_2d(CUtensorMap *map, const void *base, uint64_t inner, uint64_t outer, uint64_t row_bytes,
                 uint32_t box_inner, uint32_t box_outer, int swizzle_bytes);

int num_sms();
// Argument and device checks shared by the entry points (api.cu).
bsl_status bind_device(const void *p);  // make the device owning p current
bsl_status check_device();              // current device is sm_100
bsl_status check_bsr(const bsl_bsr *W);
uint64_t wait_timeout_ns();
bsl_status cuda_status(cudaError_t e);
void note_driver_error(int code);

// Kernel launchers (defined next to their kernels).
bsl_status launch_pack(const void *W, const uint8_t *mask, const bsl_bsr *out, cudaStream_t s);
bsl_status launch_pack_count(const uint8_t *mask, int32_t R, int32_t C, int32_t *row_ptr, cudaStream_t s);

// Forward (A = X, segments = block rows) and input gradient (A = dY,
// segments = block columns through the CSC index) share one engine.
bsl_status launch_spmm_tc(const void *A, int32_t M, int32_t a_cols, const bsl_bsr *W, bool transposed,
                          void *out, int32_t out_cols, cudaStream_t s);

bsl_status launch_sddmm_tc(const void *dY, const void *X, int32_t M, const bsl_bsr *W, void *dW,
                           cudaStream_t s);

size_t stream_workspace_bytes(int32_t M, const bsl_bsr *W);
bsl_status launch_stream_fwd(const void *X, int32_t M, const bsl_bsr *W, void *Y, void *ws, cudaStream_t s);

bsl_status launch_debug_wait(int32_t *status, uint64_t timeout_ns, cudaStream_t s);

}  // namespace bsl

/*
 * bsl.h -- C ABI of libbsl, the B200 (sm_100a) block-sparse linear layer.
 *
 * The layer is Hugging Face pytorch_block_sparse's BlockSparseLinear
 * (release note, "Block-Sparse Implementation and Usage"): a weight W[N,K]
 * that keeps only its nonzero b x b blocks, multiplied with dense
 * activations.  The library computes, in bf16 with fp32 accumulation:
 *
 *   forward          Y  = X  . W~^T      X [M,K] -> Y [M,N]
 *   input gradient   dX = dY . W~        dY[M,N] -> dX[M,K]
 *   weight gradient  dW = dY^T . X, only at the stored blocks
 *
 * where W~ is W with zeros outside the block mask.  The pruned weight is
 * handed over as a dense tensor with zeros in place plus a block mask, and
 * the sparse product equals the dense product with that tensor (torchao
 * sparsity README, introduction).  The stored form is BSR: data blocks plus
 * the block row pointer / column index arrays (torchao README, Table 4.1,
 * BSR and CSR rows), with a transposed (CSC) index over the same blocks
 * (Table 4.1, CSC row).  The masked weight gradient is dW (.) Mask
 * (torchao README, "Pruning Criteria", out-of-place mask updates).
 *
 * Conventions for every entry point:
 *  - All pointers are DEVICE pointers owned by the caller, unless a
 *    parameter says "host".  The library never frees caller memory and
 *    allocates nothing.
 *  - Matrices are row-major and contiguous (row stride = number of
 *    columns); bf16 is IEEE bfloat16 (2 bytes), passed as void *.
 *  - Every pointer must be 16-byte aligned.
 *  - Kernels run on the device that owns the first data pointer of the
 *    call (X, dY, W or the status word); the library makes that device
 *    current for the calling host thread (binding its primary context, so
 *    calls from fresh threads work) and returns BSL_ERR_INVALID_ARG for a
 *    pointer that is not device or managed memory.
 *  - `stream` is a cudaStream_t (NULL = legacy default stream).  Calls are
 *    asynchronous on it unless stated otherwise.
 *  - Arguments are checked on the host before any launch; a failed check
 *    returns a status and launches nothing.  Launch failures return
 *    BSL_ERR_CUDA.  Problems found on the device (a wait that ran out, a
 *    packed size that does not match the mask) are written to the device
 *    status word of the bsl_bsr (first error wins); read it with
 *    bsl_get_device_status.
 *  - Outputs are overwritten, never accumulated into.
 *  - Block size b must be 32 or 64; N and K must be multiples of b.
 */
#ifndef BSL_H_
#define BSL_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define BSL_API __attribute__((visibility("default")))
#else
#define BSL_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    BSL_OK = 0,
    BSL_ERR_INVALID_ARG = 1,   /* null pointer, bad shape, misalignment */
    BSL_ERR_UNSUPPORTED = 2,   /* block size or size outside what is built */
    BSL_ERR_CUDA = 3,          /* a CUDA runtime / driver call failed */
    BSL_ERR_TIMEOUT = 4,       /* a device-side wait ran out of time (device status) */
    BSL_ERR_NNZ_MISMATCH = 5,  /* mask block count != bsl_bsr.nnz (device status) */
    BSL_ERR_NO_DEVICE = 6,     /* no sm_100 device current */
    BSL_ERR_SCRATCH_TOO_SMALL = 7, /* bsl_forward_stream_noalloc: the call needs more
                                      scratch than BSL_NOALLOC_SCRATCH_BYTES */
    BSL_ERR_NOT_2_4 = 8            /* bsl_semi24_compress: a group of four holds more than
                                      two nonzeros (device status) */
} bsl_status;

/* Bytes of device memory that libbsl keeps, on every GPU that loads it, as
 * the scratch of bsl_forward_stream_noalloc. */
#define BSL_NOALLOC_SCRATCH_BYTES (16u * 1024u * 1024u)

/* Length (int32 entries) of bsl_bsr.sbounds: room for the CTA ranges of a
 * weight-streaming grid of up to 1024 CTAs (one CTA per SM). */
#define BSL_SBOUNDS_LEN 1026

/* Packed block-sparse weight.  The caller allocates every array (device
 * memory) with the sizes below, R = N/b, C = K/b; bsl_pack fills them. */
typedef struct {
    int32_t N, K, b, nnz;
    int32_t *row_ptr;     /* [R+1] BSR row pointer: blocks of block row r are row_ptr[r]..row_ptr[r+1]-1 */
    int32_t *col_idx;     /* [nnz] block column of each block, ascending inside a row */
    void *values;         /* bf16 [nnz][b][b]; block p row-major, in BSR order */
    int32_t *col_ptr;     /* [C+1] CSC column pointer over the same blocks */
    int32_t *row_idx;     /* [nnz] block row of each CSC entry, ascending inside a column */
    int32_t *csc_to_bsr;  /* [nnz] BSR position of each CSC entry (values are not duplicated) */
    int32_t *row_order;   /* [R] block rows by block count, largest first, ties lower id first */
    int32_t *col_order;   /* [C] block columns, same order rule */
    /* Work plan of the tensor-core forward: block rows taken G = 128/b at a
     * time in row_order ("row groups", ceil(R/G) of them).  For each group
     * the members' block columns are merged into one ascending list of
     * entries; entry = block column | (member mask << 24), bit i set when the
     * i-th member of the group holds a block in that column.  The blocks of
     * the present members are listed entry by entry, members in order. */
    int32_t *rgrp_ptr;    /* [ceil(R/G)+1] entry range of each row group in rgrp_ent */
    int32_t *rgrp_bptr;   /* [ceil(R/G)+1] block range of each row group in rgrp_blk */
    int32_t *rgrp_ent;    /* [nnz] entries (at most nnz) */
    int32_t *rgrp_blk;    /* [nnz] BSR block of each present member */
    /* The same plan for the input gradient over block columns (col_order, CSC
     * index), G = 128/b columns per group; entry = block row | (member mask << 24). */
    int32_t *cgrp_ptr;    /* [ceil(C/G)+1] */
    int32_t *cgrp_bptr;   /* [ceil(C/G)+1] */
    int32_t *cgrp_ent;    /* [nnz] */
    int32_t *cgrp_blk;    /* [nnz] */
    int32_t *status;      /* [1] device status word; must be zeroed once at allocation */
    int32_t *sched;       /* [8] work counters of the persistent tensor-core kernels: zeroed by
                           * bsl_pack, and every call (one that ran out of time included) leaves
                           * them at zero again, so no memset precedes a launch.  Two calls of the
                           * same contraction on one weight must not run at the same time: they
                           * would share a counter. */
    int32_t *sbounds;     /* [BSL_SBOUNDS_LEN] block ranges of the weight-streaming forward's CTAs:
                           * [0] = U, the CTA count of the device bsl_pack ran on (its SM
                           * count), [1 + c] = first block of CTA c, c = 0..U ([1 + U] = nnz).
                           * Bound c lies within q = nnz / (2U) blocks of floor(c * nnz / U):
                           * on a block-row start inside that window when there is one (among
                           * those, the choice that minimises the largest CTA range), else at
                           * floor(c * nnz / U) itself: block rows of up to 2q + 1 blocks are
                           * never split between CTAs. */
} bsl_bsr;

/* Human-readable name of a status code (static string). */
BSL_API const char *bsl_status_string(bsl_status s);

/* Description of the last CUDA error this host thread saw inside the
 * library (the cause behind a BSL_ERR_CUDA), or "none".  The string lives in
 * thread-local storage until the next call from the same thread. */
BSL_API const char *bsl_last_cuda_error(void);

/* Count the mask's blocks.  mask: uint8 [R][C], nonzero = block kept.
 * row_ptr: int32 [R+1] device scratch that receives the BSR row pointer.
 * nnz_host: HOST int32 that receives the count.  SYNCHRONOUS: waits for the
 * stream, so the caller can size the packed arrays before bsl_pack. */
BSL_API bsl_status bsl_pack_count(const uint8_t *mask, int32_t R, int32_t C, int32_t *row_ptr,
                          int32_t *nnz_host, void *stream);

/* Build the packed weight from a dense bf16 W [N][K] (zeros in place or
 * not: entries outside the mask are dropped) and a uint8 mask [N/b][K/b].
 * Fills every array of *out (N, K, b, nnz and the pointers set by the
 * caller).  If the mask holds a different number of blocks than out->nnz,
 * the device status becomes BSL_ERR_NNZ_MISMATCH and no array is written
 * past its size.  A masked-in block is stored even if all its values are 0. */
BSL_API bsl_status bsl_pack(const void *W, const uint8_t *mask, const bsl_bsr *out, void *stream);

/* Y [M][N] = X [M][K] . W~^T (+ bias).  BlockSparseLinear is a drop-in for
 * nn.Linear (release note, "Block-Sparse Implementation and Usage"), so the
 * forward takes nn.Linear's bias: bias is bf16 [N] added to every row of Y
 * in fp32 before the one rounding to bf16, or NULL for none.  Picks the
 * weight-streaming kernel for M <= bsl_small_m_max() and the tensor-core
 * kernel otherwise.  workspace: device scratch of
 * bsl_forward_workspace_bytes(M, W) bytes (may be NULL when that size is 0). */
BSL_API bsl_status bsl_forward(const void *X, int32_t M, const bsl_bsr *W, const void *bias, void *Y,
                       void *workspace, size_t workspace_bytes, void *stream);

/* Largest M routed to the weight-streaming kernel by bsl_forward. */
BSL_API int32_t bsl_small_m_max(void);

/* Scratch bytes bsl_forward needs for this M (0 for the tensor-core path). */
BSL_API size_t bsl_forward_workspace_bytes(int32_t M, const bsl_bsr *W);

/* Tensor-core forward for any M >= 1 (persistent tcgen05 kernel; TMA
 * loads of X tiles and weight blocks, fp32 accumulators in TMEM).  bias:
 * bf16 [N] or NULL, as for bsl_forward. */
BSL_API bsl_status bsl_forward_tc(const void *X, int32_t M, const bsl_bsr *W, const void *bias, void *Y,
                          void *stream);

/* Weight-streaming forward ("load and sparse expand", lecture summary at
 * 48:12) for 1 <= M <= bsl_small_m_max(): each warp streams a contiguous,
 * equal share of its CTA's range of packed blocks once (the ranges in
 * W->sbounds); block rows split between warps or CTAs are summed in a fixed
 * order.  workspace: bsl_forward_workspace_bytes(M, W) bytes, zeroed once
 * when it is allocated; every call leaves its counters (at the start of the
 * workspace, the same place for every M) at zero again, a call that ran out
 * of time included, so one workspace serves later calls of any M and weight
 * without being cleared.  Calls that use one workspace must not overlap on
 * the GPU.  bias: bf16 [N] or NULL, as for bsl_forward. */
BSL_API bsl_status bsl_forward_stream(const void *X, int32_t M, const bsl_bsr *W, const void *bias, void *Y,
                              void *workspace, size_t workspace_bytes, void *stream);

/* Same computation and kernels as bsl_forward_stream, for callers that cannot
 * allocate device memory: code that must not call cudaMalloc once running
 * (a serving loop with a fixed memory budget, where an allocation can block
 * or fail), or a plug-in inside another framework that owns all device
 * memory and gives the library no allocator.  The pages have no counterpart
 * of this entry point; it exists only for such callers.
 *
 * The scratch is a fixed array of BSL_NOALLOC_SCRATCH_BYTES in libbsl's own
 * device memory.  The CUDA runtime loads the array, like the library's
 * kernels, the first time it is used on a device: the first call of this
 * entry point on each device takes those 16 MiB from the device and fails
 * with BSL_ERR_CUDA if the device has no room left, so make one call at
 * start-up, before the memory budget is spent.  From then on the device keeps
 * the array until the process exits.  The entry point allocates nothing
 * itself and calls no cudaMalloc / cudaFree.  It returns
 * BSL_ERR_SCRATCH_TOO_SMALL, launching nothing, when the call would need more
 * scratch than that.  The need is bsl_forward_workspace_bytes(M, W) =
 * about SMs x (4 + 2 x b x M' x 4) bytes, M' = 16 for M <= 16, else 32: at most
 * 2.4 MB on a 148-SM B200 (b = 64, M <= 32), so every supported call fits
 * there; only a device with more than about 1000 SMs would be turned away.
 *
 * The first call on each device also looks up the array's device address
 * (cudaGetSymbolAddress) and keeps it for the life of the process, so make
 * that first call outside any stream capture; calls after the device's
 * primary context was destroyed and re-created (cudaDeviceReset) are not
 * supported.  Every call on a device shares the one array, which starts at
 * zero when it is loaded; each call writes every partial sum before reading
 * it and leaves the counters at zero again.  Calls whose kernels overlap
 * on the GPU (different streams without ordering between them) race on the
 * array: serialise them.  X, Y, W: as for bsl_forward_stream; the kernels
 * run on the device that owns X. */
BSL_API bsl_status bsl_forward_stream_noalloc(const void *X, int32_t M, const bsl_bsr *W, void *Y, void *stream);

/* dX [M][K] = dY [M][N] . W~ (tensor-core kernel over the CSC index). */
BSL_API bsl_status bsl_backward_input(const void *dY, int32_t M, const bsl_bsr *W, void *dX, void *stream);

/* dW_values [nnz][b][b] = blocks of dY^T . X at the stored blocks, in BSR
 * order (sampled dense-dense product over M; tensor-core kernel). */
BSL_API bsl_status bsl_backward_weight(const void *dY, const void *X, int32_t M, const bsl_bsr *W,
                               void *dW_values, void *stream);

/* dbias [N] = sum over the M rows of dY [M][N]: the gradient of the forward's
 * bias (nn.Linear's bias, which BlockSparseLinear keeps as a drop-in;
 * release note, "Block-Sparse Implementation and Usage").  fp32 sums in a
 * fixed order (identical results run to run), rounded once to bf16.  N must
 * be a multiple of 32; dbias is bf16 [N], 16-byte aligned.  Needs no
 * scratch. */
BSL_API bsl_status bsl_bias_grad(const void *dY, int32_t M, int32_t N, void *dbias, void *stream);

/* ---------------------------------------------------------------- 2:4 semi-structured
 *
 * A linear layer whose weight has the 2:4 semi-structured pattern: in every
 * group of four consecutive elements of a row (along K) at most two are
 * nonzero (torchao sparsity README, introduction and Table 4.1; "Lecture 11:
 * Sparsity" summary, 8:02 and 12:52).  The weight is stored in the
 * compressed form of Table 4.1, row "NVIDIA 2:4 compressed representation":
 * a dense matrix of half the width holding the unpruned elements, plus
 * 2-bit indices.  Y = X . W^T runs on the sparse tensor-core MMA. */
typedef struct {
    int32_t N, K;       /* dense shape of W: N output features, K input features;
                         * N a multiple of 8, K a multiple of 64 */
    void *values;       /* bf16 [N][K/2]: group g of row n (columns 4g .. 4g+3) keeps two
                         * elements, at values[n][2g] and values[n][2g+1], in column order */
    uint16_t *meta;     /* [N][K/16]: positions of the kept elements; entry (n, c) covers
                         * groups 4c .. 4c+3 of row n, group 4c+j in bits 4j .. 4j+3 as
                         * i0 | i1 << 2, the two positions inside the group with i0 < i1 */
    int32_t *status;    /* [1] device status word; must be zeroed once at allocation */
} bsl_semi24;

/* Compress a dense bf16 weight W [N][K] with zeros in place (the handoff
 * format of the torchao README's introduction) into out->values / out->meta
 * (caller-allocated, 16-byte aligned).  The kept positions of a group are
 * its nonzeros (+0 and -0 count as zero), completed by its lowest-indexed
 * zeros when it has fewer than two; kept elements are copied bit for bit.
 * A group with more than two nonzeros sets BSL_ERR_NOT_2_4 in the device
 * status (its outputs are then unspecified); read it with
 * bsl_semi24_get_status. */
BSL_API bsl_status bsl_semi24_compress(const void *W, const bsl_semi24 *out, void *stream);

/* Y [M][N] = X [M][K] . W^T (+ bias) with W the weight the compressed form
 * stands for, in bf16 with fp32 accumulation (the sparse product is the
 * dense product with zeros in place: torchao README, introduction).  bias is
 * bf16 [N] added in fp32 before the one rounding to bf16, or NULL.  M >= 1.
 * Tensor-core kernel (tcgen05.mma.sp), persistent, one CTA per SM. */
BSL_API bsl_status bsl_semi24_forward(const void *X, int32_t M, const bsl_semi24 *W, const void *bias, void *Y,
                                      void *stream);

/* ---------------------------------------------------------------- 2:4 inside blocks
 *
 * A block-sparse weight (bsl_bsr, packed by bsl_pack) whose kept blocks carry
 * the 2:4 pattern along K: the "50% sparse pattern within blocks" of the
 * release note's "Future Development Roadmap" and the "blocks of 2:4" of the
 * "Lecture 11: Sparsity" summary (43:51).  The kept blocks are stored
 * compressed beside the packed weight:
 *   values24  bf16 [nnz + 1][b][b/2]: block p in BSR order, each row's two kept
 *             elements of every group of four in column order; block nnz is
 *             zeros (written by bsl_bsr24_compress);
 *   meta24    uint16 [nnz][b][b/16]: the positions, per row as bsl_semi24.meta.
 * Both caller-allocated, 16-byte aligned. */

/* Compress the packed weight's kept blocks (W->values) into values24 and
 * meta24, with the kept positions chosen as bsl_semi24_compress does.  A
 * group with more than two nonzeros sets BSL_ERR_NOT_2_4 in W's device status
 * (read it with bsl_get_device_status). */
BSL_API bsl_status bsl_bsr24_compress(const bsl_bsr *W, void *values24, uint16_t *meta24, void *stream);

/* Y [M][N] = X [M][K] . W~^T (+ bias), W~ the block-sparse weight with zeros
 * outside its blocks, the blocks read from values24 / meta24 (the dense
 * product with zeros in place: torchao README, introduction).  bf16 in, fp32
 * accumulation, bias bf16 [N] or NULL.  b = 32 or 64.  Sparse tensor-core
 * kernel driven by W's row-group plan, persistent, one CTA per SM. */
BSL_API bsl_status bsl_bsr24_forward(const void *X, int32_t M, const bsl_bsr *W, const void *values24,
                                     const uint16_t *meta24, const void *bias, void *Y, void *stream);

/* SYNCHRONOUS: waits for the stream, copies the device status word of W to
 * *status_host (a bsl_status value) and resets it to BSL_OK. */
BSL_API bsl_status bsl_semi24_get_status(const bsl_semi24 *W, int32_t *status_host, void *stream);

/* SYNCHRONOUS: waits for the stream, copies the device status word of W to
 * *status_host (a bsl_status value) and resets it to BSL_OK. */
BSL_API bsl_status bsl_get_device_status(const bsl_bsr *W, int32_t *status_host, void *stream);

/* Upper bound, in microseconds, on any device-side wait of the kernels
 * launched after this call (default 2,000,000, or BSL_WAIT_TIMEOUT_US from
 * the environment at first use).  A wait that runs out sets
 * BSL_ERR_TIMEOUT in the device status and the kernel returns. */
BSL_API void bsl_set_wait_timeout_us(uint64_t timeout_us);

/* Test hook for the bounded waits: launches one block that waits on a
 * barrier nothing arrives at, for at most timeout_us, then writes
 * BSL_ERR_TIMEOUT to *status (device int32, zeroed by the caller). */
BSL_API bsl_status bsl_debug_wait_timeout(int32_t *status, uint64_t timeout_us, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* BSL_H_ */

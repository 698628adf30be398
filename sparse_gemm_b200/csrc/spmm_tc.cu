// spmm_tc.cu -- block-sparse x dense products on the sm_100a tensor cores.
//
// One engine computes both contractions of the layer that have a dense
// activation operand and a sparse weight operand:
//
//   forward         Y [M,N]  = X  [M,K] . W~^T   segment = block row r,
//                   entries = the row's blocks (BSR order), A tile = X[:, c-block]
//   input gradient  dX[M,K]  = dY [M,N] . W~     segment = block column c,
//                   entries = the column's blocks (CSC index -> BSR block),
//                   A tile = dY[:, r-block], weight block used untransposed
//
// (Hugging Face pytorch_block_sparse release note, "Block-Sparse
// Implementation and Usage": BlockSparseLinear keeps only the nonzero blocks
// of the weight; torchao sparsity README, Table 4.1: BSR and CSC indices.)
// Only stored blocks are touched; an output tile whose segment has no block
// is written as zeros.
//
// Work unit = (segment, 128-row tile of M).  The grid is persistent (one CTA
// per SM); units are dealt round-robin, m-tile-major (CTAs busy at the same
// time share one tile of activation rows in L2) and longest segment first
// inside a tile (heavy block rows of Zipf-skewed masks start early).  Each
// CTA caches its unit descriptors in shared memory at start.  Per CTA:
//   warp 0      TMA producer: X/dY tile (128 x b) + weight block (b x b) per
//               stored block into an smem ring (swizzled, 64 B or 128 B rows)
//   warp 1      allocates TMEM; one thread issues tcgen05.mma (M=128, N=b,
//               K=16 per instruction, bf16 in, fp32 accumulators in TMEM)
//   warps 2..5  epilogue: TMEM -> registers -> bf16 (RNE) -> swizzled smem ->
//               TMA store; 4 TMEM accumulators let the epilogue of one unit
//               overlap the MMAs of the next ones.
// Every wait is bounded in time; on expiry the kernel records
// BSL_ERR_TIMEOUT, lets its own copies and MMAs drain, frees TMEM and exits.
#include "common.cuh"
#include "internal.h"

namespace bsl {
namespace {

template <int B>
struct SpmmCfg {
    static constexpr int BM = 128;                      // rows of M per tile (= MMA M)
    static constexpr int ROW_BYTES = B * 2;             // one tile row: 64 B (b=32) or 128 B (b=64)
    static constexpr int A_BYTES = BM * ROW_BYTES;      // activation tile
    static constexpr int W_BYTES = B * ROW_BYTES;       // weight block
    static constexpr int STAGE_BYTES = A_BYTES + W_BYTES;
    static constexpr int STAGES = B == 64 ? 7 : 16;
    static constexpr int OUT_BYTES = BM * ROW_BYTES;    // epilogue staging tile
    static constexpr int OUT_BUFS = 2;
    static constexpr int ACC = 4;                       // TMEM accumulators
    static constexpr int TMEM_COLS = ACC * B;           // 128 or 256 (power of two)
    static constexpr uint32_t LAYOUT = B == 64 ? kLayoutSw128 : kLayoutSw64;
    static constexpr uint32_t SBO = 8 * ROW_BYTES;      // stride of 8-row core-matrix groups
    static constexpr int NUM_BARS = 2 * STAGES + 2 * ACC + 1;
    static constexpr int TABLE = 1024;                  // unit descriptors cached in smem per CTA
    static constexpr int SMEM_BYTES =
        STAGES * STAGE_BYTES + OUT_BUFS * OUT_BYTES + TABLE * 16 + NUM_BARS * 8 + 16 + 1024;
    static_assert(TMEM_COLS == 128 || TMEM_COLS == 256, "TMEM allocation must be a power of two");
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

struct SpmmArgs {
    int32_t M, nseg, mtiles;
    const int32_t *seg_ptr;    // [nseg+1]
    const int32_t *seg_idx;    // [nnz] block coordinate of the A tile for each entry
    const int32_t *blk_map;    // [nnz] entry -> BSR block, or null (entry j is block j)
    const int32_t *seg_order;  // [nseg] longest-first
    int32_t *status;
    uint64_t timeout_ns;
};

// Unit i of this CTA (global unit u = blockIdx.x + i * gridDim.x).  Units
// run m-tile-major: all segments of one 128-row tile of M before the next
// tile, so the CTAs working at the same time share the tile's rows of the
// activation in L2; inside a tile, segments go longest first.
__device__ __forceinline__ int4 unit_info(const SpmmArgs &a, int i)
{
    const int u = blockIdx.x + i * gridDim.x;
    const int mt = u / a.nseg;
    const int seg = a.seg_order[u - mt * a.nseg];
    return make_int4(seg, mt * 128, a.seg_ptr[seg], a.seg_ptr[seg + 1]);
}

__device__ __forceinline__ uint8_t *align1024(uint8_t *p)
{
    return reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// 16-byte chunk position inside a swizzled tile row (matches the TMA
// 128-byte / 64-byte swizzle patterns for 1024-byte aligned tiles).
template <int B>
__device__ __forceinline__ int swz_chunk(int chunk, int row)
{
    if constexpr (B == 64) return chunk ^ (row & 7);
    else return chunk ^ ((row >> 1) & 3);
}

template <int B, bool TRANS>
__global__ void __launch_bounds__(192, 1)
    k_spmm_tc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmW,
              const __grid_constant__ CUtensorMap tmO, const SpmmArgs args)
{
    using Cfg = SpmmCfg<B>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align1024(smem_raw);
    uint8_t *stages = smem;
    uint8_t *outbuf = smem + Cfg::STAGES * Cfg::STAGE_BYTES;
    int4 *table = reinterpret_cast<int4 *>(outbuf + Cfg::OUT_BUFS * Cfg::OUT_BYTES);
    uint64_t *bars = reinterpret_cast<uint64_t *>(table + Cfg::TABLE);
    uint64_t *full = bars;
    uint64_t *empty = full + Cfg::STAGES;
    uint64_t *tfull = empty + Cfg::STAGES;
    uint64_t *tempty = tfull + Cfg::ACC;
    uint64_t *drain = tempty + Cfg::ACC;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    volatile int *epi_go = abort_flag + 1;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint64_t tmo = args.timeout_ns;

    if (threadIdx.x == 0) {
        for (int s = 0; s < Cfg::STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < Cfg::ACC; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], 128);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        *epi_go = 0;
        fence_barrier_init();
        tma_prefetch_map(&tmA);
        tma_prefetch_map(&tmW);
        tma_prefetch_map(&tmO);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
        tmem_relinquish();
    }
    const int units = args.nseg * args.mtiles;
    const int nlocal = blockIdx.x < units ? (units - 1 - blockIdx.x) / gridDim.x + 1 : 0;
    const int ncached = nlocal < Cfg::TABLE ? nlocal : Cfg::TABLE;
    for (int i = threadIdx.x; i < ncached; i += blockDim.x) table[i] = unit_info(args, i);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    auto unit = [&](int i) { return i < Cfg::TABLE ? table[i] : unit_info(args, i); };

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        // The warp loads up to 32 entries' indices at once (coalesced); lane 0
        // waits for free stages and issues the copies.
        uint32_t stage = 0, phase = 0, issued = 0, issued_par = 0;
        bool ok = true;
        for (int i = 0; i < nlocal && ok; ++i) {
            const int4 ui = unit(i);
            for (int jb = ui.z; jb < ui.w && ok; jb += 32) {
                const int j = jb + lane;
                int acol = 0, blk = 0;
                if (j < ui.w) {
                    acol = args.seg_idx[j];
                    blk = args.blk_map ? args.blk_map[j] : j;
                }
                const int cnt = min(32, ui.w - jb);
                for (int t = 0; t < cnt; ++t) {
                    const int a_t = __shfl_sync(0xffffffffu, acol, t);
                    const int b_t = __shfl_sync(0xffffffffu, blk, t);
                    int good = 1;
                    if (lane == 0) {
                        good = mbar_wait(&empty[stage], phase ^ 1, tmo, abort_flag);
                        if (good) {
                            uint8_t *sa = stages + stage * Cfg::STAGE_BYTES;
                            mbar_arrive_expect_tx(&full[stage], Cfg::STAGE_BYTES);
                            tma_load_2d(sa, &tmA, &full[stage], a_t * B, ui.y);
                            tma_load_2d(sa + Cfg::A_BYTES, &tmW, &full[stage], 0, b_t * B);
                            issued |= 1u << stage;
                            issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
                        }
                    }
                    if (!__shfl_sync(0xffffffffu, good, 0)) {
                        ok = false;
                        break;
                    }
                    if (++stage == Cfg::STAGES) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
            }
        }
        if (lane == 0) {
            if (!ok) {
                *abort_flag = 1;
                set_status(args.status, BSL_ERR_TIMEOUT);
            }
            // every load this CTA issued must land before its smem is released
            for (int s = 0; s < Cfg::STAGES; ++s)
                if ((issued >> s) & 1u) mbar_wait(&full[s], (issued_par >> s) & 1u, tmo, nullptr);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = make_idesc_bf16(128, B, false, TRANS);
            uint32_t stage = 0, phase = 0, acc = 0, acc_phase = 0;
            bool ok = true, any = false;
            for (int i = 0; i < nlocal && ok; ++i) {
                const int4 ui = unit(i);
                const int beg = ui.z, end = ui.w;
                if (!mbar_wait(&tempty[acc], acc_phase ^ 1, tmo, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d = tmem_base + acc * B;
                for (int j = beg; j < end; ++j) {
                    if (!mbar_wait(&full[stage], phase, tmo, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a0 = smem_u32(stages + stage * Cfg::STAGE_BYTES);
                    const uint32_t w0 = a0 + Cfg::A_BYTES;
#pragma unroll
                    for (int k = 0; k < B / 16; ++k) {
                        const uint64_t ad = make_sdesc(a0 + k * 32, 16, Cfg::SBO, Cfg::LAYOUT);
                        const uint64_t wd =
                            TRANS ? make_sdesc(w0 + k * 16 * Cfg::ROW_BYTES, Cfg::W_BYTES, Cfg::SBO, Cfg::LAYOUT)
                                  : make_sdesc(w0 + k * 32, 16, Cfg::SBO, Cfg::LAYOUT);
                        umma_bf16(d, ad, wd, idesc, (j > beg || k > 0) ? 1u : 0u);
                    }
                    umma_commit(&empty[stage]);
                    any = true;
                    if (++stage == Cfg::STAGES) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
                if (!ok) break;
                if (end > beg) umma_commit(&tfull[acc]);
                else mbar_arrive(&tfull[acc]);
                if (++acc == Cfg::ACC) {
                    acc = 0;
                    acc_phase ^= 1;
                }
            }
            if (!ok) {
                *abort_flag = 1;
                set_status(args.status, BSL_ERR_TIMEOUT);
            }
            if (any) {  // all MMAs of this thread complete before TMEM is freed
                umma_commit(drain);
                mbar_wait(drain, 0, tmo, nullptr);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue
        const int et = threadIdx.x - 64;  // 0..127
        const int q = warp & 3;           // TMEM lane quarter this warp may access
        const int row = q * 32 + lane;    // tile row = TMEM lane
        uint32_t acc = 0, acc_phase = 0, ob = 0;
        for (int i = 0; i < nlocal; ++i) {
            const int4 ui = unit(i);
            const int seg = ui.x, m0 = ui.y;
            const bool nonempty = ui.w > ui.z;
            if (et == 0) {
                bool go = mbar_wait(&tfull[acc], acc_phase, tmo, abort_flag);
                if (go) bulk_wait_group_read<Cfg::OUT_BUFS - 1>();  // staging buffer `ob` is free
                else {
                    *abort_flag = 1;
                    set_status(args.status, BSL_ERR_TIMEOUT);
                }
                *epi_go = go ? 1 : 0;
            }
            named_bar_sync(1, 128);
            if (!*epi_go) break;
            tc_fence_after();
            uint32_t v[B];
            if (nonempty) {
                const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * B;
#pragma unroll
                for (int c = 0; c < B / 16; ++c)
                    tmem_ld16(taddr + c * 16, *reinterpret_cast<uint32_t(*)[16]>(&v[c * 16]));
                tmem_wait_ld();
            } else {
#pragma unroll
                for (int i = 0; i < B; ++i) v[i] = 0u;
            }
            tc_fence_before();
            mbar_arrive(&tempty[acc]);
            uint8_t *dst = outbuf + ob * Cfg::OUT_BYTES + row * Cfg::ROW_BYTES;
#pragma unroll
            for (int c = 0; c < B / 8; ++c) {
                uint4 pk;
                pk.x = pack_bf16x2(__uint_as_float(v[8 * c + 0]), __uint_as_float(v[8 * c + 1]));
                pk.y = pack_bf16x2(__uint_as_float(v[8 * c + 2]), __uint_as_float(v[8 * c + 3]));
                pk.z = pack_bf16x2(__uint_as_float(v[8 * c + 4]), __uint_as_float(v[8 * c + 5]));
                pk.w = pack_bf16x2(__uint_as_float(v[8 * c + 6]), __uint_as_float(v[8 * c + 7]));
                *reinterpret_cast<uint4 *>(dst + swz_chunk<B>(c, row) * 16) = pk;
            }
            fence_async_smem();
            named_bar_sync(1, 128);
            if (et == 0) {
                tma_store_2d(&tmO, outbuf + ob * Cfg::OUT_BYTES, seg * B, m0);
                bulk_commit_group();
            }
            ob ^= 1;
            if (++acc == Cfg::ACC) {
                acc = 0;
                acc_phase ^= 1;
            }
        }
        if (et == 0) bulk_wait_group<0>();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
    }
}

template <int B, bool TRANS>
bsl_status run(const CUtensorMap &a, const CUtensorMap &w, const CUtensorMap &o, const SpmmArgs &args,
               cudaStream_t s)
{
    using Cfg = SpmmCfg<B>;
    auto kern = k_spmm_tc<B, TRANS>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM_BYTES);
    if (e != cudaSuccess) return cuda_status(e);
    const int units = args.nseg * args.mtiles;
    const int grid = units < num_sms() ? units : num_sms();
    kern<<<grid, 192, Cfg::SMEM_BYTES, s>>>(a, w, o, args);
    return cuda_status(cudaGetLastError());
}

}  // namespace

bsl_status launch_spmm_tc(const void *A, int32_t M, int32_t a_cols, const bsl_bsr *W, bool transposed,
                          void *out, int32_t out_cols, cudaStream_t s)
{
    const int B = W->b;
    if (W->nnz == 0)
        return cuda_status(cudaMemsetAsync(out, 0, static_cast<size_t>(M) * out_cols * 2, s));
    CUtensorMap ma, mw, mo;
    if (!make_map_2d(&ma, A, a_cols, M, static_cast<uint64_t>(a_cols) * 2, B, 128, 2 * B) ||
        !make_map_2d(&mw, W->values, B, static_cast<uint64_t>(W->nnz) * B, 2 * B, B, B, 2 * B) ||
        !make_map_2d(&mo, out, out_cols, M, static_cast<uint64_t>(out_cols) * 2, B, 128, 2 * B))
        return BSL_ERR_CUDA;
    SpmmArgs args;
    args.M = M;
    args.mtiles = (M + 127) / 128;
    args.nseg = transposed ? W->K / B : W->N / B;
    args.seg_ptr = transposed ? W->col_ptr : W->row_ptr;
    args.seg_idx = transposed ? W->row_idx : W->col_idx;
    args.blk_map = transposed ? W->csc_to_bsr : nullptr;
    args.seg_order = transposed ? W->col_order : W->row_order;
    args.status = W->status;
    args.timeout_ns = wait_timeout_ns();
    if (B == 64) return transposed ? run<64, true>(ma, mw, mo, args, s) : run<64, false>(ma, mw, mo, args, s);
    return transposed ? run<32, true>(ma, mw, mo, args, s) : run<32, false>(ma, mw, mo, args, s);
}

}  // namespace bsl

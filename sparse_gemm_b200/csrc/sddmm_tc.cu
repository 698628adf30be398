// sddmm_tc.cu -- masked weight gradient on the sm_100a tensor cores.
//
// dW = dY^T . X is needed only at the stored blocks (torchao sparsity README,
// "Pruning Criteria", out-of-place mask updates: the weight gradient is
// dW (.) Mask), so this is an output-sparse (sampled dense-dense) product:
// for each stored block p = (r, c),
//     dW_p[u][v] = sum_m dY[m][r*b+u] * X[m][c*b+v]      (u, v < b)
// written as bf16 into dW_values[p] (BSR order), reduction over all M rows in
// fp32.
//
// MMA shape: the blocks of one block column c share the X strip X[:, c-block],
// so a work unit ("group") stacks G = 128/b blocks of the same column along
// MMA M: A = [dY[:, r_1-block] | ... | dY[:, r_G-block]]^T (128 x 128 rows of
// M per stage, MN-major in smem: the dY tiles are loaded untransposed),
// B = X[:, c-block]^T (b x 128, MN-major), D = 128 x b fp32 in TMEM.  Groups
// are listed per column by the pack's dw_gptr prefix (ceil(count/G) per
// column); a column's last group may hold fewer than G blocks, and its
// unused accumulator lanes are never stored.
//
// Roles: warps 0..P-1 TMA producers (one thread cannot start copies fast
// enough, so k-step i is issued by warp i % P; the stage ring is partitioned
// so that slot i % STAGES is only ever filled by that warp), warp P TMEM
// owner + MMA issuer, warps P+1..P+4 epilogue (TMEM -> bf16 -> 16-byte
// global stores).
#include "common.cuh"
#include "internal.h"

namespace bsl {
namespace {

// Rows of M per stage: copies are the bottleneck of this kernel (one thread
// starts only about four per microsecond), so each copy moves a tall strip.
constexpr int kSddmmRows = 128;

template <int B>
struct SddmmCfg {
    static constexpr int G = 128 / B;                    // blocks stacked along MMA M
    static constexpr int MK = kSddmmRows;                // rows of M reduced per stage
    static constexpr int ROW_BYTES = B * 2;
    static constexpr int T_BYTES = MK * ROW_BYTES;       // one strip tile (MK x b)
    static constexpr int STAGE_BYTES = (G + 1) * T_BYTES;
    static constexpr int STAGES = 4;
    static constexpr int P = 4;                          // producer warps (STAGES % P == 0)
    static constexpr int THREADS = (P + 5) * 32;
    static_assert(STAGES % P == 0, "each stage slot belongs to one producer warp");
    static constexpr int ACC = 2;
    static constexpr int TMEM_COLS = ACC * B;            // 64 or 128
    static constexpr uint32_t LAYOUT = B == 64 ? kLayoutSw128 : kLayoutSw64;
    static constexpr uint32_t SBO = 8 * ROW_BYTES;
    static constexpr int NUM_BARS = 2 * STAGES + 2 * ACC + 1;
    static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + NUM_BARS * 8 + 16 + 1024;
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

struct SddmmArgs {
    int32_t M, C, ksteps;
    const int32_t *col_ptr, *row_idx, *csc_to_bsr, *dw_gptr;
    __nv_bfloat16 *dW;
    int32_t *status;
    uint64_t timeout_ns;
};

__device__ __forceinline__ uint8_t *align1024(uint8_t *p)
{
    return reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// column c of group g: last c with dw_gptr[c] <= g
__device__ __forceinline__ int group_column(const int32_t *gptr, int C, int g)
{
    int lo = 0, hi = C;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (gptr[mid] <= g) lo = mid;
        else hi = mid;
    }
    return lo;
}

template <int B>
__global__ void __launch_bounds__(SddmmCfg<B>::THREADS, 1)
    k_sddmm_tc(const __grid_constant__ CUtensorMap tmDY, const __grid_constant__ CUtensorMap tmX,
               const SddmmArgs args)
{
    using Cfg = SddmmCfg<B>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *stages = align1024(smem_raw);
    uint64_t *bars = reinterpret_cast<uint64_t *>(stages + Cfg::STAGES * Cfg::STAGE_BYTES);
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
        tma_prefetch_map(&tmDY);
        tma_prefetch_map(&tmX);
    }
    if (warp == Cfg::P) {
        tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int ngroups = args.dw_gptr[args.C];

    if (warp < Cfg::P) {
        // k-step i (counted over all groups of this CTA) uses slot i % STAGES and
        // is issued by warp i % P; the slot's previous fill, step i - STAGES,
        // was issued by the same warp, so every wait is on the warp's own fills
        if (lane == 0) {
            uint32_t issued = 0, issued_par = 0;
            bool ok = true;
            int i = 0;
            for (int g = blockIdx.x; g < ngroups && ok; g += gridDim.x) {
                const int c = group_column(args.dw_gptr, args.C, g);
                const int j0 = args.col_ptr[c] + (g - args.dw_gptr[c]) * Cfg::G;
                const int cnt = min(Cfg::G, args.col_ptr[c + 1] - j0);
                int rows[Cfg::G];
#pragma unroll
                for (int q = 0; q < Cfg::G; ++q) rows[q] = q < cnt ? args.row_idx[j0 + q] : 0;
                for (int ks = 0; ks < args.ksteps; ++ks, ++i) {
                    if (i % Cfg::P != warp) continue;
                    const int stage = i % Cfg::STAGES;
                    const uint32_t phase = (i / Cfg::STAGES) & 1;
                    if (!mbar_wait(&empty[stage], phase ^ 1, tmo, abort_flag)) {
                        ok = false;
                        break;
                    }
                    uint8_t *sa = stages + stage * Cfg::STAGE_BYTES;
                    mbar_arrive_expect_tx(&full[stage], (cnt + 1) * Cfg::T_BYTES);
#pragma unroll
                    for (int q = 0; q < Cfg::G; ++q)
                        if (q < cnt)
                            tma_load_2d(sa + q * Cfg::T_BYTES, &tmDY, &full[stage], rows[q] * B, ks * Cfg::MK);
                    tma_load_2d(sa + Cfg::G * Cfg::T_BYTES, &tmX, &full[stage], c * B, ks * Cfg::MK);
                    issued |= 1u << stage;
                    issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
                }
            }
            if (!ok) {
                *abort_flag = 1;
                set_status(args.status, BSL_ERR_TIMEOUT);
            }
            for (int sl = 0; sl < Cfg::STAGES; ++sl)
                if (((issued >> sl) & 1u) && !mbar_wait(&full[sl], (issued_par >> sl) & 1u, tmo, nullptr))
                    set_status(args.status, BSL_ERR_TIMEOUT);
        }
        __syncwarp();
    } else if (warp == Cfg::P) {
        if (lane == 0) {
            constexpr uint32_t idesc = make_idesc_bf16(128, B, true, true);
            uint32_t stage = 0, phase = 0, acc = 0, acc_phase = 0;
            bool ok = true, any = false;
            for (int g = blockIdx.x; g < ngroups && ok; g += gridDim.x) {
                if (!mbar_wait(&tempty[acc], acc_phase ^ 1, tmo, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d = tmem_base + acc * B;
                for (int ks = 0; ks < args.ksteps; ++ks) {
                    if (!mbar_wait(&full[stage], phase, tmo, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a0 = smem_u32(stages + stage * Cfg::STAGE_BYTES);
                    const uint32_t x0 = a0 + Cfg::G * Cfg::T_BYTES;
#pragma unroll
                    for (int k = 0; k < Cfg::MK / 16; ++k) {
                        const uint64_t ad =
                            make_sdesc(a0 + k * 16 * Cfg::ROW_BYTES, Cfg::T_BYTES, Cfg::SBO, Cfg::LAYOUT);
                        const uint64_t xd =
                            make_sdesc(x0 + k * 16 * Cfg::ROW_BYTES, Cfg::T_BYTES, Cfg::SBO, Cfg::LAYOUT);
                        umma_bf16(d, ad, xd, idesc, (ks > 0 || k > 0) ? 1u : 0u);
                    }
                    umma_commit(&empty[stage]);
                    any = true;
                    if (++stage == Cfg::STAGES) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
                if (!ok) break;
                umma_commit(&tfull[acc]);
                if (++acc == Cfg::ACC) {
                    acc = 0;
                    acc_phase ^= 1;
                }
            }
            if (!ok) {
                *abort_flag = 1;
                set_status(args.status, BSL_ERR_TIMEOUT);
            }
            if (any) {
                umma_commit(drain);
                if (!mbar_wait(drain, 0, tmo, nullptr)) set_status(args.status, BSL_ERR_TIMEOUT);
            }
        }
        __syncwarp();
    } else {
        const int et = threadIdx.x - (Cfg::P + 1) * 32;
        const int q = warp & 3;
        const int l = q * 32 + lane;      // accumulator row = TMEM lane
        const int blk_in_group = l / B, u = l % B;
        uint32_t acc = 0, acc_phase = 0;
        for (int g = blockIdx.x; g < ngroups; g += gridDim.x) {
            const int c = group_column(args.dw_gptr, args.C, g);
            const int j0 = args.col_ptr[c] + (g - args.dw_gptr[c]) * Cfg::G;
            const int cnt = min(Cfg::G, args.col_ptr[c + 1] - j0);
            if (et == 0) {
                const bool go = mbar_wait(&tfull[acc], acc_phase, tmo, abort_flag);
                if (!go) {
                    *abort_flag = 1;
                    set_status(args.status, BSL_ERR_TIMEOUT);
                }
                *epi_go = go ? 1 : 0;
            }
            named_bar_sync(1, 128);
            if (!*epi_go) break;
            tc_fence_after();
            uint32_t v[B];
            const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * B;
#pragma unroll
            for (int k = 0; k < B / 16; ++k)
                tmem_ld16(taddr + k * 16, *reinterpret_cast<uint32_t(*)[16]>(&v[k * 16]));
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(&tempty[acc]);
            if (blk_in_group < cnt) {
                const int p = args.csc_to_bsr[j0 + blk_in_group];
                uint4 *dst = reinterpret_cast<uint4 *>(args.dW + (static_cast<int64_t>(p) * B + u) * B);
#pragma unroll
                for (int k = 0; k < B / 8; ++k) {
                    uint4 pk;
                    pk.x = pack_bf16x2(__uint_as_float(v[8 * k + 0]), __uint_as_float(v[8 * k + 1]));
                    pk.y = pack_bf16x2(__uint_as_float(v[8 * k + 2]), __uint_as_float(v[8 * k + 3]));
                    pk.z = pack_bf16x2(__uint_as_float(v[8 * k + 4]), __uint_as_float(v[8 * k + 5]));
                    pk.w = pack_bf16x2(__uint_as_float(v[8 * k + 6]), __uint_as_float(v[8 * k + 7]));
                    dst[k] = pk;
                }
            }
            named_bar_sync(1, 128);  // everyone has read epi_go before it is rewritten
            if (++acc == Cfg::ACC) {
                acc = 0;
                acc_phase ^= 1;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == Cfg::P) {
        tc_fence_after();
        tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
    }
}

template <int B>
bsl_status run(const CUtensorMap &dy, const CUtensorMap &x, const SddmmArgs &args, int ngroups_max,
               cudaStream_t s)
{
    using Cfg = SddmmCfg<B>;
    auto kern = k_sddmm_tc<B>;
    const bsl_status sa = set_smem_once(reinterpret_cast<const void *>(kern), Cfg::SMEM_BYTES);
    if (sa != BSL_OK) return sa;
    const int grid = ngroups_max < num_sms() ? ngroups_max : num_sms();
    kern<<<grid, Cfg::THREADS, Cfg::SMEM_BYTES, s>>>(dy, x, args);
    return cuda_status(cudaGetLastError());
}

}  // namespace

bsl_status launch_sddmm_tc(const void *dY, const void *X, int32_t M, const bsl_bsr *W, void *dW, cudaStream_t s)
{
    const int B = W->b;
    if (W->nnz == 0) return BSL_OK;
    CUtensorMap mdy, mx;
    if (!make_map_2d(&mdy, dY, W->N, M, static_cast<uint64_t>(W->N) * 2, B, kSddmmRows, 2 * B) ||
        !make_map_2d(&mx, X, W->K, M, static_cast<uint64_t>(W->K) * 2, B, kSddmmRows, 2 * B))
        return BSL_ERR_CUDA;
    SddmmArgs args;
    args.M = M;
    args.C = W->K / B;
    args.ksteps = (M + kSddmmRows - 1) / kSddmmRows;
    args.col_ptr = W->col_ptr;
    args.row_idx = W->row_idx;
    args.csc_to_bsr = W->csc_to_bsr;
    args.dw_gptr = W->dw_gptr;
    args.dW = static_cast<__nv_bfloat16 *>(dW);
    args.status = W->status;
    args.timeout_ns = wait_timeout_ns();
    // groups <= nnz; the kernel reads the exact count from dw_gptr[C]
    const int G = 128 / B;
    const int gmax = W->nnz < args.C * ((W->N / B + G - 1) / G) ? W->nnz : args.C * ((W->N / B + G - 1) / G);
    return B == 64 ? run<64>(mdy, mx, args, gmax, s) : run<32>(mdy, mx, args, gmax, s);
}

}  // namespace bsl

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
// Tiles.  The block grid is cut into tiles of GR x GC blocks (GR*b = 128 rows
// of dW, GC*b = 128 columns).  For a tile, every stage brings in 128 rows of
// M of two 64-column strips of dY (the tile's 128 dY columns) and two of X,
// and one tcgen05.mma of M = 128, N = 128 per 16 rows computes the whole
// 128 x 128 tile of dY^T . X (fp32 in TMEM).  A strip is one block column
// for b = 64 and two for b = 32: its 128-byte rows move at the copy engine's
// full rate, where 64-byte rows move at about 70 % of it.  Only strips that
// hold a stored block of the tile are copied (a skipped strip leaves old data
// in shared memory, which only reaches accumulator entries that are never
// stored), only stored blocks are written out, and tiles without a stored
// block are skipped.  Each strip is read once per tile instead of once per
// stored block, and every MMA is full width.
//
// Roles: warps 0..P-1 TMA producers (stage i of this CTA is filled by warp
// i % P, which owns that stage slot alone), warp P TMEM owner + MMA issuer,
// warps P+1..P+4 epilogue (TMEM -> bf16 -> 16-byte global stores of the
// stored blocks).  Tiles go round-robin over the CTAs, consecutive tiles
// sharing their block rows (their dY strips stay in L2).  Results do not
// depend on the schedule: every output is one fixed-order fp32 reduction.
#include "common.cuh"
#include "internal.h"

namespace bsl {
namespace {

template <int B>
struct SddmmCfg {
    static constexpr int GR = 128 / B;                   // block rows per tile (MMA M = 128)
    static constexpr int GC = 128 / B;                   // block columns per tile (MMA N = 128)
    static constexpr int MK = 128;                       // rows of M reduced per stage
    static constexpr int SW = 64;                        // strip width (columns): 128-byte rows
    static constexpr int NS = 128 / SW;                  // strips per operand
    static constexpr int BPS = SW / B;                   // block columns per strip
    static constexpr int ROW_BYTES = SW * 2;
    static constexpr int T_BYTES = MK * ROW_BYTES;       // one strip tile (MK x 64)
    static constexpr int STAGE_BYTES = 2 * NS * T_BYTES;
    static constexpr int STAGES = 3;
    static constexpr int P = STAGES;                     // producer warps: one per stage slot
    static constexpr int THREADS = (P + 5) * 32;
    static constexpr int ACC = 2;
    static constexpr int ACC_COLS = GC * B;              // 128
    static constexpr int TMEM_COLS = ACC * ACC_COLS;     // 256
    static constexpr uint32_t LAYOUT = kLayoutSw128;
    static constexpr uint32_t SBO = 8 * ROW_BYTES;
    static constexpr int NUM_BARS = 2 * STAGES + 2 * ACC + 1;
    static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + NUM_BARS * 8 + 16 + 1024;
    static_assert(STAGES % P == 0, "each stage slot belongs to one producer warp");
    static_assert(GR * GC <= 32, "one lane per block of a tile");
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

struct SddmmArgs {
    int32_t M, R, C, ksteps, nrg, ncg, ntiles;
    const int32_t *row_ptr, *col_idx;
    __nv_bfloat16 *dW;
    int32_t *status;
    uint64_t timeout_ns;
};

__device__ __forceinline__ uint8_t *align1024(uint8_t *p)
{
    return reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Stored blocks of tile t, found by the whole warp (lane l < GR*GC looks up
// block (i, j) = (l / GC, l % GC) in its block row's ascending columns):
// returns the lane's BSR position (-1: not stored) and the tile's block-row /
// block-column masks.
template <int B>
__device__ __forceinline__ int tile_blocks(const SddmmArgs &a, int t, int lane, uint32_t *rmask, uint32_t *cmask,
                                           int *rg_out, int *cg_out)
{
    using Cfg = SddmmCfg<B>;
    const int rg = t / a.ncg, cg = t - (t / a.ncg) * a.ncg;
    *rg_out = rg;
    *cg_out = cg;
    int pos = -1;
    if (lane < Cfg::GR * Cfg::GC) {
        const int i = lane / Cfg::GC, j = lane % Cfg::GC;
        const int r = rg * Cfg::GR + i, c = cg * Cfg::GC + j;
        if (r < a.R && c < a.C) {
            int lo = a.row_ptr[r], hi = a.row_ptr[r + 1];
            while (lo < hi) {  // first position with column >= c
                const int mid = (lo + hi) >> 1;
                if (a.col_idx[mid] < c) lo = mid + 1;
                else hi = mid;
            }
            if (lo < a.row_ptr[r + 1] && a.col_idx[lo] == c) pos = lo;
        }
    }
    const uint32_t present = __ballot_sync(0xffffffffu, pos >= 0);
    uint32_t rm = 0, cm = 0;
#pragma unroll
    for (int l = 0; l < Cfg::GR * Cfg::GC; ++l)
        if ((present >> l) & 1u) {
            rm |= 1u << (l / Cfg::GC);
            cm |= 1u << (l % Cfg::GC);
        }
    *rmask = rm;
    *cmask = cm;
    return pos;
}

// Strips holding any of the tile's blocks in `blocks` (bit i = block i).
template <int B>
__device__ __forceinline__ uint32_t strip_mask(uint32_t blocks)
{
    using Cfg = SddmmCfg<B>;
    uint32_t m = 0;
#pragma unroll
    for (int q = 0; q < Cfg::NS; ++q)
        if ((blocks >> (q * Cfg::BPS)) & ((1u << Cfg::BPS) - 1u)) m |= 1u << q;
    return m;
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

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint64_t tmo = args.timeout_ns;
    dependents_may_launch();

    if (threadIdx.x == 0) {
        for (int s = 0; s < Cfg::STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < Cfg::ACC; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], 4);  // one arrival per epilogue warp
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
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
    wait_for_prior_grid();  // set-up above touched no global memory

    if (warp < Cfg::P) {
        // ------------------------------------------------------------ producers
        // stage i (counted over this CTA's non-empty tiles) uses slot i % STAGES
        // and is filled by warp i % P; the slot's previous fill, stage
        // i - STAGES, came from the same warp, so every wait is on its own fills
        uint32_t issued = 0, issued_par = 0;
        bool ok = true;
        int i = 0;
        for (int t = blockIdx.x; t < args.ntiles && ok; t += gridDim.x) {
            uint32_t rm, cm;
            int rg, cg;
            tile_blocks<B>(args, t, lane, &rm, &cm, &rg, &cg);
            if (!rm) continue;
            const uint32_t rs = strip_mask<B>(rm), cs = strip_mask<B>(cm);
            const uint32_t nstrips = __popc(rs) + __popc(cs);
            for (int ks = 0; ks < args.ksteps; ++ks, ++i) {
                if (i % Cfg::P != warp) continue;
                const int stage = i % Cfg::STAGES;
                const uint32_t phase = (i / Cfg::STAGES) & 1;
                int good = 1;
                if (lane == 0) {
                    if (!mbar_wait(&empty[stage], phase ^ 1, tmo, abort_flag)) {
                        good = 0;
                    } else {
                        uint8_t *sa = stages + stage * Cfg::STAGE_BYTES;
                        mbar_arrive_expect_tx(&full[stage], nstrips * Cfg::T_BYTES);
#pragma unroll
                        for (int q = 0; q < Cfg::NS; ++q)
                            if ((rs >> q) & 1u)
                                tma_load_2d(sa + q * Cfg::T_BYTES, &tmDY, &full[stage],
                                            rg * Cfg::GR * B + q * Cfg::SW, ks * Cfg::MK);
#pragma unroll
                        for (int q = 0; q < Cfg::NS; ++q)
                            if ((cs >> q) & 1u)
                                tma_load_2d(sa + (Cfg::NS + q) * Cfg::T_BYTES, &tmX, &full[stage],
                                            cg * Cfg::GC * B + q * Cfg::SW, ks * Cfg::MK);
                        issued |= 1u << stage;
                        issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
                    }
                }
                if (!__shfl_sync(0xffffffffu, good, 0)) {
                    ok = false;
                    break;
                }
            }
        }
        if (lane == 0) {
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
        // ------------------------------------------------------------ MMA issuer
        constexpr uint32_t idesc = make_idesc_bf16(128, Cfg::GC * B, true, true);
        uint32_t stage = 0, phase = 0, acc = 0, acc_phase = 0;
        bool ok = true, any = false;
        const uint32_t lead = lane == 0 ? 1u : 0u;
        for (int t = blockIdx.x; t < args.ntiles && ok; t += gridDim.x) {
            uint32_t rm, cm;
            int rg, cg;
            tile_blocks<B>(args, t, lane, &rm, &cm, &rg, &cg);
            if (!rm) continue;
            if (__any_sync(0xffffffffu, !mbar_wait(&tempty[acc], acc_phase ^ 1, tmo, abort_flag))) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t d = tmem_base + acc * Cfg::ACC_COLS;
            for (int ks = 0; ks < args.ksteps; ++ks) {
                if (__any_sync(0xffffffffu, !mbar_wait(&full[stage], phase, tmo, abort_flag))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t a0 = smem_u32(stages + stage * Cfg::STAGE_BYTES);
                const uint32_t x0 = a0 + Cfg::NS * Cfg::T_BYTES;
                // A: the dY strips side by side along M (MN-major, T_BYTES apart);
                // B: the X strips along N; K = 16 rows of M per instruction
                const uint64_t ad0 = make_sdesc(a0, Cfg::T_BYTES, Cfg::SBO, Cfg::LAYOUT);
                const uint64_t xd0 = make_sdesc(x0, Cfg::T_BYTES, Cfg::SBO, Cfg::LAYOUT);
                const uint32_t alo = static_cast<uint32_t>(ad0), ahi = static_cast<uint32_t>(ad0 >> 32);
                const uint32_t xlo = static_cast<uint32_t>(xd0), xhi = static_cast<uint32_t>(xd0 >> 32);
                constexpr uint32_t KSTEP = (16 * Cfg::ROW_BYTES) >> 4;
#pragma unroll
                for (int k = 0; k < Cfg::MK / 16; ++k)
                    umma_bf16_lo_lead(lead, d, alo + k * KSTEP, ahi, xlo + k * KSTEP, xhi, idesc,
                                      (ks > 0 || k > 0) ? 1u : 0u);
                umma_commit_lead(lead, &empty[stage]);
                any = true;
                if (++stage == Cfg::STAGES) {
                    stage = 0;
                    phase ^= 1;
                }
            }
            if (!ok) break;
            umma_commit_lead(lead, &tfull[acc]);
            __syncwarp();
            if (++acc == Cfg::ACC) {
                acc = 0;
                acc_phase ^= 1;
            }
        }
        if (lane == 0 && !ok) {
            *abort_flag = 1;
            set_status(args.status, BSL_ERR_TIMEOUT);
        }
        if (any) {
            umma_commit_lead(lead, drain);
            if (lane == 0 && !mbar_wait(drain, 0, tmo, nullptr)) set_status(args.status, BSL_ERR_TIMEOUT);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue
        // warp q reads TMEM lanes 32q..32q+31 = dW rows u of block row i of
        // the tile (i = 32q / b, u = 32q % b + lane) and writes the stored
        // blocks of that row: one 2b-byte row of each per thread.
        const int q = warp & 3;
        const int i = (32 * q) / B;
        const int u = (32 * q) % B + lane;
        uint32_t acc = 0, acc_phase = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < args.ntiles; t += gridDim.x) {
            uint32_t rm, cm;
            int rg, cg;
            const int pos = tile_blocks<B>(args, t, lane, &rm, &cm, &rg, &cg);
            if (!rm) continue;
            int go = 1;
            if (lane == 0) go = mbar_wait(&tfull[acc], acc_phase, tmo, abort_flag);
            if (!__shfl_sync(0xffffffffu, go, 0)) {
                ok = false;
                break;
            }
            tc_fence_after();
#pragma unroll 1
            for (int j = 0; j < Cfg::GC; ++j) {
                const int p = __shfl_sync(0xffffffffu, pos, i * Cfg::GC + j);
                if (p < 0) continue;
                uint32_t v[B];
                const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * Cfg::ACC_COLS + j * B;
#pragma unroll
                for (int k = 0; k < B / 16; ++k)
                    tmem_ld16(taddr + k * 16, *reinterpret_cast<uint32_t(*)[16]>(&v[k * 16]));
                tmem_wait_ld();
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
            // every TMEM read of this accumulator is complete (each was waited)
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[acc]);
            if (++acc == Cfg::ACC) {
                acc = 0;
                acc_phase ^= 1;
            }
        }
        if (lane == 0 && !ok) {
            *abort_flag = 1;
            set_status(args.status, BSL_ERR_TIMEOUT);
        }
        __syncwarp();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == Cfg::P) {
        tc_fence_after();
        tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
    }
}

template <int B>
bsl_status run(const CUtensorMap &dy, const CUtensorMap &x, const SddmmArgs &args, cudaStream_t s)
{
    using Cfg = SddmmCfg<B>;
    auto kern = k_sddmm_tc<B>;
    const bsl_status sa = set_smem_once(reinterpret_cast<const void *>(kern), Cfg::SMEM_BYTES);
    if (sa != BSL_OK) return sa;
    const int grid = args.ntiles < num_sms() ? args.ntiles : num_sms();
    return cuda_status(launch_dependent(kern, grid, Cfg::THREADS, Cfg::SMEM_BYTES, s, dy, x, args));
}

}  // namespace

bsl_status launch_sddmm_tc(const void *dY, const void *X, int32_t M, const bsl_bsr *W, void *dW, cudaStream_t s)
{
    const int B = W->b;
    if (W->nnz == 0) return BSL_OK;
    CUtensorMap mdy, mx;
    // 64-column strips (128-byte rows, 128-byte swizzle); a strip that reaches
    // past the last column reads zeros there
    if (!make_map_2d(&mdy, dY, W->N, M, static_cast<uint64_t>(W->N) * 2, 64, 128, 128) ||
        !make_map_2d(&mx, X, W->K, M, static_cast<uint64_t>(W->K) * 2, 64, 128, 128))
        return BSL_ERR_CUDA;
    const int G = 128 / B;
    SddmmArgs args;
    args.M = M;
    args.R = W->N / B;
    args.C = W->K / B;
    args.ksteps = (M + 127) / 128;
    args.nrg = (args.R + G - 1) / G;
    args.ncg = (args.C + G - 1) / G;
    args.ntiles = args.nrg * args.ncg;
    args.row_ptr = W->row_ptr;
    args.col_idx = W->col_idx;
    args.dW = static_cast<__nv_bfloat16 *>(dW);
    args.status = W->status;
    args.timeout_ns = wait_timeout_ns();
    return B == 64 ? run<64>(mdy, mx, args, s) : run<32>(mdy, mx, args, s);
}

}  // namespace bsl

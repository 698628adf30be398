// spmm_tc.cu -- block-sparse x dense products on the sm_100a tensor cores.
//
// One engine computes both contractions of the layer that have a dense
// activation operand and a sparse weight operand:
//
//   forward         Y [M,N]  = X  [M,K] . W~^T   segments = block rows,
//                   activation tile = X[:, c-block] for block column c
//   input gradient  dX[M,K]  = dY [M,N] . W~     segments = block columns (CSC),
//                   activation tile = dY[:, r-block], weight block untransposed
//
// (Hugging Face pytorch_block_sparse release note, "Block-Sparse
// Implementation and Usage": BlockSparseLinear keeps only the nonzero blocks
// of the weight; torchao sparsity README, Table 4.1: BSR and CSC indices.)
// Only stored blocks are touched; output blocks of segments without blocks
// are written as zeros.
//
// Data flow.  On B200 the L2 -> SM fabric, not the tensor core, limits a
// block-sparse product whose activation tile feeds one b-wide block: every
// 128 x b activation tile would be fetched once per block.  So segments are
// processed G = 256/b at a time ("groups", fixed by the pack in longest-
// first order): for each group the pack merged the members' block
// coordinates into ascending entries with a member mask.  A work unit is
// (128-row tile of M, group); per entry the activation tile is fetched once
// and the weight blocks of the present members follow it into a separate
// ring, so each activation tile feeds every member that needs it.  Present
// members that are consecutive in the group and whose blocks sit in
// consecutive ring slots form a "run" whose blocks are stacked along N: one
// tcgen05.mma of N = run * b per 16-wide K step, writing the members'
// accumulator columns directly (runs are also split where a member is
// written for the first time in the unit, since that MMA must overwrite).
// The accumulator of a unit is G*b = 256 fp32 columns of TMEM; two of them
// let the epilogue of one unit overlap the MMAs of the next.
//
// Copies are issued from several warps: one thread can start only a few TMA
// copies per microsecond, far below what the fabric delivers, so entry e is
// issued by producer warp e % P.  The weight blocks of an entry sit
// contiguously in the pack's plan-ordered copy of the values, stored in the
// swizzled shared-memory image, so they arrive with one 1-D bulk copy into
// consecutive W-ring slots (an entry never wraps around the ring).
//
// Roles per CTA (persistent grid, one CTA per SM, units dealt round-robin,
// m-tile-major so concurrent CTAs share activation rows in L2):
//   warps 0..P-1   producers: TMA tile copy of the activation tile (X ring),
//                  bulk copy of the entry's weight blocks (W ring)
//   warp P         TMEM owner; lane 0 issues the MMAs (bf16 in, fp32 in TMEM)
//   warps P+1..P+4 epilogue: TMEM -> registers -> bf16 (RNE) -> swizzled smem
//                  -> TMA store, one 128 x b chunk per member
// Every wait is bounded in time; on expiry the kernel records
// BSL_ERR_TIMEOUT, lets its own copies and MMAs drain, frees TMEM and exits.
#include "common.cuh"
#include "internal.h"

namespace bsl {
namespace {

template <int B>
struct SpmmCfg {
    static constexpr int BM = 128;                      // rows of M per tile (= MMA M)
    static constexpr int G = 256 / B;                   // members per group
    static constexpr int ROW_BYTES = B * 2;             // one tile row: 64 B (b=32) or 128 B (b=64)
    static constexpr int A_BYTES = BM * ROW_BYTES;      // activation tile
    static constexpr int W_BYTES = B * ROW_BYTES;       // weight block
    static constexpr int P = 4;                         // producer warps
    static constexpr int THREADS = (P + 5) * 32;        // producers, MMA warp, 4 epilogue warps
    static constexpr int XS = B == 64 ? 5 : 10;         // activation ring slots (= entries in flight)
    static constexpr int WS = B == 64 ? 12 : 48;        // weight ring slots
    static constexpr int OUT_BYTES = BM * ROW_BYTES;    // epilogue staging chunk
    static constexpr int OUT_BUFS = 2;
    static constexpr int ACC = 2;                       // TMEM accumulators
    static constexpr int ACC_COLS = G * B;              // 256
    static constexpr int TMEM_COLS = ACC * ACC_COLS;    // 512
    static constexpr uint32_t LAYOUT = B == 64 ? kLayoutSw128 : kLayoutSw64;
    static constexpr uint32_t SBO = 8 * ROW_BYTES;      // stride of 8-row core-matrix groups
    static constexpr int TABLE = 256;                   // unit descriptors cached per CTA
    static constexpr int NUM_BARS = 2 * XS + 2 * ACC + 1;
    static constexpr int SMEM_BYTES = XS * A_BYTES + WS * W_BYTES + OUT_BUFS * OUT_BYTES + TABLE * 20 +
                                      P * (WS + XS + 1) * 4 + NUM_BARS * 8 + 32 + 1024;
    static_assert(ACC_COLS == 256 && TMEM_COLS == 512, "TMEM layout");
    static_assert(G <= 8, "member mask is 8 bits");
    static_assert(XS <= 32, "issue bookkeeping uses a 32-bit mask");
    static_assert(WS >= G, "one entry's blocks must fit the weight ring");
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

struct SpmmArgs {
    int32_t M, nseg, ngroups, mtiles, nblk;
    const int32_t *seg_ptr;    // [nseg+1] blocks per segment (empty segments give zero output)
    const int32_t *seg_order;  // [nseg] longest first; group g = seg_order[g*G .. g*G+G-1]
    const int32_t *grp_ptr;    // [ngroups+1] entry range per group
    const int32_t *grp_bptr;   // [ngroups+1] block range per group
    const int32_t *grp_ent;    // entries: coordinate | (mask << 24)
    const uint8_t *grp_vals;   // weight blocks in plan order, swizzled smem image
    int32_t *status;
    uint64_t timeout_ns;
};

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

// Unit i of this CTA: global unit u = blockIdx.x + i * gridDim.x, m-tile-major.
// x = group, y = first row of the m-tile, z/w = entry range; first block in *bstart.
__device__ __forceinline__ int4 unit_info(const SpmmArgs &a, int i, int *bstart)
{
    const int u = blockIdx.x + i * gridDim.x;
    const int mt = u / a.ngroups;
    const int g = u - mt * a.ngroups;
    *bstart = a.grp_bptr[g];
    return make_int4(g, mt * 128, a.grp_ptr[g], a.grp_ptr[g + 1]);
}

// Ring cursor: slot index + phase parity.
struct Ring {
    uint32_t slot = 0, phase = 0;
    __device__ __forceinline__ void next(uint32_t n)
    {
        if (++slot == n) {
            slot = 0;
            phase ^= 1;
        }
    }
};

template <int B, bool TRANS>
__global__ void __launch_bounds__(SpmmCfg<B>::THREADS, 1)
    k_spmm_tc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmW,
              const __grid_constant__ CUtensorMap tmO, const SpmmArgs args)
{
    using Cfg = SpmmCfg<B>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align1024(smem_raw);
    uint8_t *xring = smem;
    uint8_t *wring = xring + Cfg::XS * Cfg::A_BYTES;
    uint8_t *outbuf = wring + Cfg::WS * Cfg::W_BYTES;
    int4 *table = reinterpret_cast<int4 *>(outbuf + Cfg::OUT_BUFS * Cfg::OUT_BYTES);
    int *btable = reinterpret_cast<int *>(table + Cfg::TABLE);
    int *wowner_all = btable + Cfg::TABLE;  // per producer warp: entry that last filled each weight slot
    int *xlast_all = wowner_all + Cfg::P * Cfg::WS;  // per producer warp: last entry it issued per X slot
    uint64_t *bars = reinterpret_cast<uint64_t *>(xlast_all + Cfg::P * Cfg::XS + (Cfg::P * Cfg::XS) % 2);
    uint64_t *xfull = bars;   // all copies of an entry (activation tile + weight blocks)
    uint64_t *xempty = xfull + Cfg::XS;  // MMAs of the entry done: its X slot and weight slots are free
    uint64_t *tfull = xempty + Cfg::XS;
    uint64_t *tempty = tfull + Cfg::ACC;
    uint64_t *drain = tempty + Cfg::ACC;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    volatile int *epi_go = abort_flag + 1;
    volatile int *turn = epi_go + 1;  // next entry whose producer may check slot reuse

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint64_t tmo = args.timeout_ns;

    if (threadIdx.x == 0) {
        for (int s = 0; s < Cfg::XS; ++s) {
            mbar_init(&xfull[s], 1);
            mbar_init(&xempty[s], 1);
        }
        for (int s = 0; s < Cfg::P * Cfg::WS; ++s) wowner_all[s] = -1;
        for (int s = 0; s < Cfg::P * Cfg::XS; ++s) xlast_all[s] = -1;
        for (int a = 0; a < Cfg::ACC; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], 128);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        *epi_go = 0;
        *turn = 0;
        fence_barrier_init();
        tma_prefetch_map(&tmA);
        tma_prefetch_map(&tmW);
        tma_prefetch_map(&tmO);
    }
    if (warp == Cfg::P) {
        tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
        tmem_relinquish();
    }
    const int units = args.ngroups * args.mtiles;
    const int nlocal = blockIdx.x < units ? (units - 1 - blockIdx.x) / gridDim.x + 1 : 0;
    const int ncached = nlocal < Cfg::TABLE ? nlocal : Cfg::TABLE;
    for (int i = threadIdx.x; i < ncached; i += blockDim.x) table[i] = unit_info(args, i, &btable[i]);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    auto unit = [&](int i, int *bstart) {
        if (i < Cfg::TABLE) {
            *bstart = btable[i];
            return table[i];
        }
        return unit_info(args, i, bstart);
    };

    if (warp < Cfg::P) {
        // ------------------------------------------------------------ producers
        // Every producer warp walks all entries (ring cursors and slot owners
        // stay identical across warps) and issues the copies of entries
        // e % P == warp.  Entry e uses X slot e % XS; its copies complete on
        // xfull of that slot, and the MMA warp's one commit per entry frees the
        // X slot and the entry's weight slots.  A slot is refilled once the
        // entry that last used it has completed (entries complete in order).
        // The reuse checks run in entry order (`turn`), so each waits on a
        // barrier at most one phase ahead of the entry it waits for; the
        // copies themselves are then issued by the warps concurrently.
        int *wowner = wowner_all + warp * Cfg::WS;
        int *xlast = xlast_all + warp * Cfg::XS;
        Ring xr;
        uint32_t ws = 0;                 // weight ring cursor
        int e = 0, done = -1;            // entries walked; highest entry known complete
        bool ok = true;
        for (int i = 0; i < nlocal && ok; ++i) {
            int bcur;
            const int4 ui = unit(i, &bcur);
            for (int eb = ui.z; eb < ui.w && ok; eb += 32) {
                const int el = eb + lane < ui.w ? args.grp_ent[eb + lane] : 0;
                const int n = min(32, ui.w - eb);
                for (int t = 0; t < n; ++t, ++e) {
                    const uint32_t ent = static_cast<uint32_t>(__shfl_sync(0xffffffffu, el, t));
                    const int coord = static_cast<int>(ent & 0xFFFFFFu);
                    const uint32_t k = __popc(ent >> 24);
                    if (ws + k > Cfg::WS) ws = 0;  // an entry's blocks never wrap
                    int good = 1;
                    if (lane == 0 && e % Cfg::P == warp) {
                        // wait for this entry's turn (all earlier entries passed their checks)
                        if (*turn != e) {
                            const uint64_t t0 = globaltimer_ns();
                            for (uint32_t spin = 1; *turn != e; ++spin) {
                                // the clock is slow to read: look at it (and the abort flag) rarely
                                if ((spin & 255u) == 0 && (*abort_flag || globaltimer_ns() - t0 > tmo)) {
                                    good = 0;
                                    break;
                                }
                            }
                        }
                        // entry e-1 passed its checks, which made entry e-1-XS complete, and
                        // entries complete in order; so any remaining owner is at least
                        // e - XS and its X-slot barrier is at most one phase ahead of it
                        done = max(done, e - 1 - Cfg::XS);
                        if (good && e >= Cfg::XS && e - Cfg::XS > done) {  // X slot: entry e - XS done
                            good = mbar_wait(&xempty[xr.slot], xr.phase ^ 1, tmo, abort_flag);
                            done = e - Cfg::XS;
                        }
                        for (uint32_t q = 0; q < k && good; ++q) {  // weight slots: last users done
                            const int owner = wowner[ws + q];
                            if (owner > done) {
                                good = mbar_wait(&xempty[owner % Cfg::XS], (owner / Cfg::XS) & 1, tmo, abort_flag);
                                done = owner;
                            }
                        }
                        if (good) {
                            __threadfence_block();
                            *turn = e + 1;  // the next entry may check its slots
                            uint64_t *bar = &xfull[xr.slot];
                            mbar_arrive_expect_tx(bar, Cfg::A_BYTES + k * Cfg::W_BYTES);
                            tma_load_2d(xring + xr.slot * Cfg::A_BYTES, &tmA, bar, coord * B, ui.y);
                            if (k)
                                bulk_load(wring + ws * Cfg::W_BYTES,
                                          args.grp_vals + static_cast<int64_t>(bcur) * Cfg::W_BYTES,
                                          k * Cfg::W_BYTES, bar);
                            xlast[xr.slot] = e;
                        }
                    }
                    if (!__shfl_sync(0xffffffffu, good, 0)) {
                        ok = false;
                        break;
                    }
                    if (lane == 0)
                        for (uint32_t q = 0; q < k; ++q) wowner[ws + q] = e;
                    ws += k;
                    bcur += static_cast<int>(k);
                    xr.next(Cfg::XS);
                }
            }
        }
        if (lane == 0) {
            if (!ok) {
                *abort_flag = 1;
                set_status(args.status, BSL_ERR_TIMEOUT);
            }
            // every copy this warp issued must land before the CTA's smem is released.
            // If entry x + XS passed its reuse check, x was consumed already; otherwise
            // x is the last fill of its slot and the parity wait is unambiguous.
            for (int sl = 0; sl < Cfg::XS; ++sl) {
                const int x = xlast[sl];
                if (x >= 0 && *turn <= x + Cfg::XS && !mbar_wait(&xfull[sl], (x / Cfg::XS) & 1, tmo, nullptr))
                    set_status(args.status, BSL_ERR_TIMEOUT);
            }
        }
        __syncwarp();
    } else if (warp == Cfg::P) {
        // ------------------------------------------------------------ MMA issuer
        // The warp walks the entries (cached 32 at a time); lane 0 waits and issues.
        Ring xr, ar;
        uint32_t ws = 0;  // weight ring cursor (same allocation rule as the producers)
        bool ok = true, any = false;
        for (int i = 0; i < nlocal && ok; ++i) {
            int bdummy;
            const int4 ui = unit(i, &bdummy);
            int good = 1;
            if (lane == 0) good = mbar_wait(&tempty[ar.slot], ar.phase ^ 1, tmo, abort_flag);
            if (!__shfl_sync(0xffffffffu, good, 0)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t d0 = tmem_base + ar.slot * Cfg::ACC_COLS;
            uint32_t seen = 0;  // members already written in this unit
            for (int eb = ui.z; eb < ui.w && ok; eb += 32) {
                const int el = eb + lane < ui.w ? args.grp_ent[eb + lane] : 0;
                const int n = min(32, ui.w - eb);
                for (int t = 0; t < n; ++t) {
                    const uint32_t mask = static_cast<uint32_t>(__shfl_sync(0xffffffffu, el, t)) >> 24;
                    const uint32_t k = __popc(mask);
                    if (ws + k > Cfg::WS) ws = 0;
                    if (lane == 0) {
                        good = mbar_wait(&xfull[xr.slot], xr.phase, tmo, abort_flag);
                        if (good) {
                            tc_fence_after();
                            const uint32_t a0 = smem_u32(xring + xr.slot * Cfg::A_BYTES);
                            // runs: consecutive present members with the same first-write
                            // status (their blocks sit in consecutive slots)
                            uint32_t slot = ws;
                            int mbr = 0;
                            while (mbr < Cfg::G) {
                                if (!((mask >> mbr) & 1u)) {
                                    ++mbr;
                                    continue;
                                }
                                const int first = mbr;
                                const uint32_t first_slot = slot;
                                const uint32_t st = (seen >> mbr) & 1u;
                                int len = 1;
                                ++mbr;
                                ++slot;
                                while (mbr < Cfg::G && ((mask >> mbr) & 1u) && ((seen >> mbr) & 1u) == st) {
                                    ++len;
                                    ++mbr;
                                    ++slot;
                                }
                                const uint32_t idesc = make_idesc_bf16(128, len * B, false, TRANS);
                                const uint32_t w0 = smem_u32(wring + first_slot * Cfg::W_BYTES);
#pragma unroll
                                for (int kk = 0; kk < B / 16; ++kk) {
                                    const uint64_t ad = make_sdesc(a0 + kk * 32, 16, Cfg::SBO, Cfg::LAYOUT);
                                    const uint64_t wd =
                                        TRANS ? make_sdesc(w0 + kk * 16 * Cfg::ROW_BYTES, Cfg::W_BYTES, Cfg::SBO,
                                                           Cfg::LAYOUT)
                                              : make_sdesc(w0 + kk * 32, 16, Cfg::SBO, Cfg::LAYOUT);
                                    umma_bf16(d0 + first * B, ad, wd, idesc, (kk > 0 || st) ? 1u : 0u);
                                }
                            }
                            // the entry's X slot and weight slots are free once these MMAs finish
                            umma_commit(&xempty[xr.slot]);
                            any = true;
                        }
                    }
                    if (!__shfl_sync(0xffffffffu, good, 0)) {
                        ok = false;
                        break;
                    }
                    seen |= mask;
                    xr.next(Cfg::XS);
                    ws += k;
                }
            }
            if (!ok) break;
            if (lane == 0) {
                if (ui.w > ui.z) umma_commit(&tfull[ar.slot]);
                else mbar_arrive(&tfull[ar.slot]);
            }
            ar.next(Cfg::ACC);
        }
        if (lane == 0) {
            if (!ok) {
                *abort_flag = 1;
                set_status(args.status, BSL_ERR_TIMEOUT);
            }
            if (any) {  // all MMAs of this thread complete before TMEM is freed
                umma_commit(drain);
                if (!mbar_wait(drain, 0, tmo, nullptr)) set_status(args.status, BSL_ERR_TIMEOUT);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue
        const int et = threadIdx.x - (Cfg::P + 1) * 32;  // 0..127
        const int q = warp & 3;           // TMEM lane quarter this warp may access
        const int row = q * 32 + lane;    // tile row = TMEM lane
        Ring ar;
        uint32_t ob = 0;
        for (int i = 0; i < nlocal; ++i) {
            int bdummy;
            const int4 ui = unit(i, &bdummy);
            const int g = ui.x, m0 = ui.y;
            // members of the group and whether they hold any block (lane i < G)
            const int mi = g * Cfg::G + lane;
            int mseg = -1, mnz = 0;
            if (lane < Cfg::G && mi < args.nseg) {
                mseg = args.seg_order[mi];
                mnz = args.seg_ptr[mseg + 1] > args.seg_ptr[mseg];
            }
            if (et == 0) {
                const bool go = mbar_wait(&tfull[ar.slot], ar.phase, tmo, abort_flag);
                if (!go) {
                    *abort_flag = 1;
                    set_status(args.status, BSL_ERR_TIMEOUT);
                }
                *epi_go = go ? 1 : 0;
            }
            named_bar_sync(1, 128);
            if (!*epi_go) break;
            tc_fence_after();
            for (int mbr = 0; mbr < Cfg::G; ++mbr) {
                const int seg = __shfl_sync(0xffffffffu, mseg, mbr);
                const int nz = __shfl_sync(0xffffffffu, mnz, mbr);
                if (seg < 0) break;
                uint32_t v[B];
                if (nz) {
                    const uint32_t taddr =
                        tmem_base + (static_cast<uint32_t>(q * 32) << 16) + ar.slot * Cfg::ACC_COLS + mbr * B;
#pragma unroll
                    for (int c = 0; c < B / 16; ++c)
                        tmem_ld16(taddr + c * 16, *reinterpret_cast<uint32_t(*)[16]>(&v[c * 16]));
                    tmem_wait_ld();
                } else {
#pragma unroll
                    for (int c = 0; c < B; ++c) v[c] = 0u;
                }
                if (et == 0) bulk_wait_group_read<Cfg::OUT_BUFS - 1>();  // staging chunk `ob` is free
                named_bar_sync(1, 128);
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
            }
            // every TMEM read of this accumulator is complete (each was waited)
            tc_fence_before();
            mbar_arrive(&tempty[ar.slot]);
            ar.next(Cfg::ACC);
        }
        if (et == 0) bulk_wait_group<0>();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == Cfg::P) {
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
    const int units = args.ngroups * args.mtiles;
    const int grid = units < num_sms() ? units : num_sms();
    kern<<<grid, Cfg::THREADS, Cfg::SMEM_BYTES, s>>>(a, w, o, args);
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
    const int G = 256 / B;
    SpmmArgs args;
    args.M = M;
    args.mtiles = (M + 127) / 128;
    args.nseg = transposed ? W->K / B : W->N / B;
    args.ngroups = (args.nseg + G - 1) / G;
    args.nblk = W->nnz;
    args.seg_ptr = transposed ? W->col_ptr : W->row_ptr;
    args.seg_order = transposed ? W->col_order : W->row_order;
    args.grp_ptr = transposed ? W->cgrp_ptr : W->rgrp_ptr;
    args.grp_bptr = transposed ? W->cgrp_bptr : W->rgrp_bptr;
    args.grp_ent = transposed ? W->cgrp_ent : W->rgrp_ent;
    args.grp_vals = static_cast<const uint8_t *>(transposed ? W->values_cg : W->values_rg);
    args.status = W->status;
    args.timeout_ns = wait_timeout_ns();
    if (B == 64) return transposed ? run<64, true>(ma, mw, mo, args, s) : run<64, false>(ma, mw, mo, args, s);
    return transposed ? run<32, true>(ma, mw, mo, args, s) : run<32, false>(ma, mw, mo, args, s);
}

}  // namespace bsl

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
// Data flow.  At low density each stored block needs a whole activation
// tile, so tile traffic (L2 -> shared memory) and the count of narrow MMAs,
// not tensor-core arithmetic, set the pace; reuse is raised both ways.
// A work unit is (256-row tile of M, group of G = 128/b segments); the pack
// fixed the groups (longest-first order) and merged the members' block
// coordinates into ascending entries with a member mask.  Per entry one
// 256 x b activation tile is fetched and feeds every present member, and
// every weight block feeds both 128-row halves of the tile.  Present members
// that are consecutive in the group and share their first-write status form
// a "run" whose blocks are stacked along N: per 128-row half and 16-wide K
// step one tcgen05.mma of N = run * b (runs are split where a member is
// written for the first time in the unit, since that MMA must overwrite).
// For b = 32 an MMA costs about the same whatever its N, so every entry is
// instead one run of all G members (N = 128): each member's block sits at
// its own slot position, positions of absent members hold zeros, and the
// unit's first entry overwrites the whole accumulator.  Shared memory is the
// bound for b = 64: per entry the activation tile is written by TMA and read
// by both halves' MMAs, the weight blocks written once and read twice.
// A unit's accumulator is 2 x G*b = 256 fp32 columns of TMEM; two of them
// let the epilogue of one unit overlap the MMAs of the next.
//
// Entry slots.  Each entry in flight owns one shared-memory slot: its
// activation tile and room for G weight blocks.  Each present member's
// block comes straight from the packed values (the weight is stored once,
// in BSR order) by a 3-D tensor copy that swizzles it on the way into the
// slot; the group plan lists the BSR block ids of every entry, which the
// producer warp stages in shared memory a chunk of entries at a time.  The
// producer also writes the entry's MMA runs (TMEM column,
// block, instruction descriptor, overwrite flag) into a small slot header:
// the MMA pipe barely runs ahead of the thread that issues it, so that
// thread does nothing per entry but wait, read the header and issue.  One
// thread starts only about four TMA copies per microsecond, so entry e goes
// to slot e % S and its copies are issued by producer warp e % P, which owns
// that slot alone (S a multiple of P): every slot is a single-producer,
// single-consumer ring.
//
// Scheduling.  Units are taken from a per-weight atomic counter in the
// order of decode_unit (heaviest first inside chunks of m-tiles), so the SMs
// stay balanced under skewed block rows.  A scheduler warp takes a unit only
// once a chunk slot is free (the CTA holds at most one unit beyond the one
// its producers issue) and publishes it to the other roles through a small
// ring in shared memory.  The CTA that makes the launch's last take past the
// final unit sets the counter back to zero, and a CTA that ran out of time
// first takes the remaining units, so every launch leaves the counter at zero
// and no memset precedes the kernel; two launches of the same contraction on
// one weight must not run at the same time (they would share the counter).
// CTA i's first unit is unit i, with no atomic round trip before its first
// plan load; a launch with no more units than CTAs leaves the counter alone.
//
// Roles per CTA (persistent grid, one CTA per SM):
//   warps 0..P-1   producers: TMA tile copies of the activation tile and of
//                  the entry's weight blocks, into the entry's slot
//   warp P         TMEM owner; runs converged, lane 0 issues the MMAs and commits
//                  (bf16 in, fp32 accumulators in TMEM)
//   warps P+1..P+4 epilogue: TMEM -> registers -> bf16 (RNE) -> swizzled smem
//                  -> TMA store; each warp its own 32 rows of every chunk
// Every wait is bounded in time; on expiry the kernel records
// BSL_ERR_TIMEOUT, lets its own copies and MMAs drain, frees TMEM and exits.
#include "common.cuh"
#include "internal.h"

namespace bsl {
namespace {

template <int B>
struct SpmmCfg {
    static constexpr int BM = 128;                      // rows of one MMA (M)
    static constexpr int MSUB = 2;                      // MMA row blocks per unit
    static constexpr int MT = BM * MSUB;                // rows of M per unit
    static constexpr int G = 128 / B;                   // members per group
    // b = 32: every entry is one MMA of all G members (N = 128), absent
    // members' blocks read as zeros; b = 64: runs of present members only
    static constexpr bool PAD = B == 32;
    static constexpr int ROW_BYTES = B * 2;             // one tile row: 64 B (b=32) or 128 B (b=64)
    static constexpr int SUB_BYTES = BM * ROW_BYTES;    // one 128-row half of the activation tile
    static constexpr int X_BYTES = MT * ROW_BYTES;      // activation tile
    static constexpr int W_BYTES = B * ROW_BYTES;       // weight block
    static constexpr int SLOT_BYTES = X_BYTES + G * W_BYTES;
    static constexpr int S = B == 64 ? 4 : 8;           // entry slots (= entries in flight)
    static constexpr int S_LOG = B == 64 ? 2 : 3;
    static constexpr int P = 4;                         // producer warps
    static constexpr int UR = 16;                       // unit ring (id, entry count)
    static constexpr int W_MMA = P;                     // then 4 epilogue warps
    static constexpr int W_SCHED = P + 5;               // then the scheduler
    static constexpr int THREADS = (P + 6) * 32;
    static constexpr int D = 2;                         // staged chunks of entries
    static constexpr int CH_BYTES = 16 + 32 * 8 + 32 * G * 4;  // header, entries, aux, block ids
    static constexpr int WARP_OUT = 32 * ROW_BYTES;     // one epilogue warp's staging chunk (32 rows)
    static constexpr int OUT_BYTES = 4 * 2 * WARP_OUT;  // 4 warps x 2 chunks
    static constexpr int ACC = 2;                       // TMEM accumulators
    static constexpr int HALF_COLS = G * B;             // 128 columns per row block
    static constexpr int ACC_COLS = MSUB * HALF_COLS;   // 256
    static constexpr int TMEM_COLS = ACC * ACC_COLS;    // 512
    static constexpr uint32_t LAYOUT = B == 64 ? kLayoutSw128 : kLayoutSw64;
    static constexpr uint32_t SBO = 8 * ROW_BYTES;      // stride of 8-row core-matrix groups
    static constexpr int NUM_BARS = 2 * S + 2 * ACC + 2 * UR + 2 * D + 1;
    static constexpr int HDR_V4 = (G + 1) / 2;          // 16-byte header words per slot (two runs each)
    static constexpr int HDR_BYTES = S * HDR_V4 * 16;
    static constexpr int SMEM_BYTES =
        S * SLOT_BYTES + OUT_BYTES + NUM_BARS * 8 + HDR_BYTES + UR * 8 + D * CH_BYTES + 64 + 1024;
    static_assert((1 << S_LOG) == S && S % P == 0 && (P & (P - 1)) == 0, "slot ownership");
    static_assert(ACC_COLS == 256 && TMEM_COLS == 512, "TMEM layout");
    static_assert(G <= 8, "member mask is 8 bits");
    static_assert((D & (D - 1)) == 0 && CH_BYTES % 16 == 0, "chunk ring");
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

struct SpmmArgs {
    int32_t M, nseg, ngroups, mtiles, units;  // units = ngroups * mtiles
    const int32_t *seg_ptr;    // [nseg+1] blocks per segment (empty segments give zero output)
    const int32_t *seg_order;  // [nseg] longest first; group g = seg_order[g*G .. g*G+G-1]
    const int32_t *grp_ptr;    // [ngroups+1] entry range per group
    const int32_t *grp_bptr;   // [ngroups+1] block range per group
    const int32_t *grp_ent;    // entries: coordinate | (mask << 24)
    const int32_t *grp_blk;    // BSR block of every present member, entry by entry
    int32_t *sched;            // [1] next unit (zero between launches: each launch resets it)
    const __nv_bfloat16 *bias; // [nseg * b] added to every output row (forward only; null: none)
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

// Work order: m-tiles in chunks of CHUNK (4096 rows: the activation rows a
// chunk needs stay in L2), and inside a chunk group-major, groups in
// longest-first order, so every chunk starts with its heaviest units and
// ends with the lightest: the SMs that finish first pick up the small units
// of the tail.  (Measured: 16 m-tiles per chunk matches 8 on the 8192-row
// layer and is ~4 % faster on the 4096-row one; 2 and 4 are slower.)
constexpr int CHUNK = 16;
__device__ __forceinline__ void decode_unit(const SpmmArgs &a, int ord, int *mt, int *g)
{
    const int per_chunk = CHUNK * a.ngroups;
    const int ch = ord / per_chunk;
    const int mt0 = ch * CHUNK;
    const int nmt = min(CHUNK, a.mtiles - mt0);
    const int r = ord - ch * per_chunk;
    *g = r / nmt;
    *mt = mt0 + (r - *g * nmt);
}

// Take the next unit from the per-weight counter (-1: none left).  Units
// 0 .. gridDim.x - 1 are the CTAs' first units, taken without the counter,
// so the counter hands out units from gridDim.x on.  Every CTA ends with
// exactly one take past the last unit: units atomic takes in all, and the
// one that finds units - 1 (unit units + gridDim.x - 1) is the last of the
// launch, so that CTA sets the counter back to zero for the next launch
// (stream order makes the store visible to it).
__device__ __forceinline__ int take_unit(int32_t *sched, int units)
{
    const int ord = atomicAdd(sched, 1) + static_cast<int>(gridDim.x);
    if (ord < units) return ord;
    if (ord == units + static_cast<int>(gridDim.x) - 1) *reinterpret_cast<volatile int32_t *>(sched) = 0;
    return -1;
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

// Consumer side of the unit ring: the j-th unit id of this CTA (-1: no more
// units) and its entry count.  Returns false if the wait ran out or the
// kernel aborted.
template <int UR>
__device__ __forceinline__ bool unit_take(uint64_t *ufull, uint64_t *uempty, const volatile int *uring, int j,
                                          int *uid, int *nent, uint64_t tmo, const volatile int *abort_flag)
{
    const int s = j % UR;
    if (!mbar_wait(&ufull[s], (j / UR) & 1, tmo, abort_flag)) return false;
    *uid = uring[2 * s];
    *nent = uring[2 * s + 1];
    mbar_arrive(&uempty[s]);
    return true;
}

template <int B, bool TRANS>
__global__ void __launch_bounds__(SpmmCfg<B>::THREADS, 1)
    k_spmm_tc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmO,
              const __grid_constant__ CUtensorMap tmW, const SpmmArgs args)
{
    using Cfg = SpmmCfg<B>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align1024(smem_raw);
    uint8_t *slots = smem;
    uint8_t *outbuf = slots + Cfg::S * Cfg::SLOT_BYTES;
    uint64_t *bars = reinterpret_cast<uint64_t *>(outbuf + Cfg::OUT_BYTES);
    uint64_t *full = bars;                 // the entry's copies landed in the slot
    uint64_t *empty = full + Cfg::S;       // the entry's MMAs finished: the slot is free
    uint64_t *tfull = empty + Cfg::S;      // accumulator complete
    uint64_t *tempty = tfull + Cfg::ACC;   // accumulator read out
    uint64_t *ufull = tempty + Cfg::ACC;   // unit published
    uint64_t *uempty = ufull + Cfg::UR;    // unit read by the MMA issuer and the epilogue
    uint64_t *cfull = uempty + Cfg::UR;    // chunk of entries staged
    uint64_t *cempty = cfull + Cfg::D;     // chunk read by every producer
    uint64_t *drain = cempty + Cfg::D;
    // [S][HDR_V4] MMA runs of the slot's entry, two per 16-byte word: run r is
    // (x, y) = (.x, .y) or (.z, .w) of word r / 2 with x = TMEM column | weight
    // block offset (16-byte units) << 8 | run count (run 0 only) << 24 |
    // overwrite-free flag << 28 and y = the instruction descriptor
    uint4 *hdr = reinterpret_cast<uint4 *>((reinterpret_cast<uintptr_t>(drain + 1) + 15) & ~uintptr_t(15));
    // [UR][2] unit id (-1: none left) and its entry count
    volatile int *uring = reinterpret_cast<volatile int *>(hdr + Cfg::S * Cfg::HDR_V4);
    // [D] staged chunks of up to 32 entries of a unit, CH_BYTES each (ints):
    // [0] entry count (-1: no more units), [1] first output row of the unit,
    // [4 + i] entry i (coordinate | member mask << 24), [36 + i] members
    // written by earlier entries of the unit | (offset of the entry's first
    // block in the chunk's block list << 8), [68 ..] BSR ids of the present
    // members' blocks, entry by entry
    int *chunks = const_cast<int *>(uring + 2 * Cfg::UR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(chunks + Cfg::D * (Cfg::CH_BYTES / 4));
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint64_t tmo = args.timeout_ns;
    dependents_may_launch();

    if (threadIdx.x == 0) {
        for (int s = 0; s < Cfg::S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < Cfg::ACC; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], 128);
        }
        for (int u = 0; u < Cfg::UR; ++u) {
            mbar_init(&ufull[u], 1);
            mbar_init(&uempty[u], 5);  // MMA issuer, 4 epilogue warps
        }
        for (int c = 0; c < Cfg::D; ++c) {
            mbar_init(&cfull[c], 1);
            mbar_init(&cempty[c], Cfg::P);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_barrier_init();
        tma_prefetch_map(&tmA);
        tma_prefetch_map(&tmO);
        tma_prefetch_map(&tmW);
    }
    if (warp == Cfg::W_MMA) {
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
        // The producers walk the entries of the chunks the scheduler staged,
        // in order, and each issues the copies of the entries whose slot it
        // owns.  Before the copies it writes the entry's MMA runs into the
        // slot header, so the issuer only reads them; the expect_tx arrive
        // publishes the header with the data.  Slot reuse waits for the one
        // MMA commit of the slot's previous entry, which this warp also
        // issued, so the parity is unambiguous.
        const int p = warp;
        int e = 0;                  // entries walked so far (all units of this CTA)
        int fills[Cfg::S / Cfg::P]; // fills issued per owned slot
        uint32_t stale[Cfg::S / Cfg::P];  // padded mode: positions of an owned slot that may hold a block
#pragma unroll
        for (int i = 0; i < Cfg::S / Cfg::P; ++i) {
            fills[i] = 0;
            stale[i] = (1u << Cfg::G) - 1;  // shared memory starts with anything in it
        }
        bool ok = true;
        for (int cc = 0; ok; ++cc) {
            const int cs = cc & (Cfg::D - 1);
            if (__any_sync(0xffffffffu, !mbar_wait(&cfull[cs], (cc / Cfg::D) & 1, tmo, abort_flag))) {
                ok = false;
                break;
            }
            const int *ch = chunks + cs * (Cfg::CH_BYTES / 4);
            const int n = ch[0];
            if (n < 0) break;  // no more units
            const int m0 = ch[1];
            const uint32_t el = lane < n ? static_cast<uint32_t>(ch[4 + lane]) : 0u;
            const uint32_t ax = lane < n ? static_cast<uint32_t>(ch[36 + lane]) : 0u;
            const int *ids = ch + 68;
            int good = 1;
            for (int t = (p - e) & (Cfg::P - 1); t < n; t += Cfg::P) {
                const uint32_t ent = __shfl_sync(0xffffffffu, el, t);
                const uint32_t aux = __shfl_sync(0xffffffffu, ax, t);
                const int off = static_cast<int>(aux >> 8);
                const uint32_t sb = aux & 0xFFu;
                // the entry that reuses this slot next: pull its activation tile into L2
                const int tn = t + Cfg::S;
                const uint32_t entn = __shfl_sync(0xffffffffu, el, tn < n ? tn : 0);
                const int ee = e + t;
                const int slot = ee & (Cfg::S - 1);
                const int use = ee >> Cfg::S_LOG;
                const uint32_t mask = ent >> 24;
                const uint32_t k = __popc(mask);
                if (lane == 0 && use > 0 && !mbar_wait(&empty[slot], (use - 1) & 1, tmo, abort_flag)) good = 0;
                if (!__shfl_sync(0xffffffffu, good, 0)) {
                    ok = false;
                    break;
                }
                uint8_t *sp = slots + slot * Cfg::SLOT_BYTES;
                if constexpr (Cfg::PAD) {
                    // member m's block sits at position m; positions of absent
                    // members must read as zeros, so the ones that still hold an
                    // earlier entry's block are cleared (generic-proxy stores, made
                    // visible to the tensor core before the barrier publishes them)
                    uint32_t zero = 0;
#pragma unroll
                    for (int i = 0; i < Cfg::S / Cfg::P; ++i)
                        if (slot == p + i * Cfg::P) {
                            zero = stale[i] & ~mask;
                            stale[i] = mask;
                        }
                    if (zero) {
                        for (uint32_t z = zero; z; z &= z - 1) {
                            uint4 *dst = reinterpret_cast<uint4 *>(sp + Cfg::X_BYTES + (__ffs(z) - 1) * Cfg::W_BYTES);
                            for (int c = lane; c < Cfg::W_BYTES / 16; c += 32) dst[c] = make_uint4(0, 0, 0, 0);
                        }
                        fence_async_smem();
                        __syncwarp();
                    }
                }
                if (lane == 0) {
                    if constexpr (!Cfg::PAD) {
                        // runs: consecutive present members with the same first-write
                        // status; their blocks are consecutive in the slot
                        uint2 *hr = reinterpret_cast<uint2 *>(hdr + slot * Cfg::HDR_V4);
                        int nr = 0, mbr = 0;
                        uint32_t q = 0;
                        while (mbr < Cfg::G) {
                            if (!((mask >> mbr) & 1u)) {
                                ++mbr;
                                continue;
                            }
                            const int first = mbr;
                            const uint32_t q0 = q;
                            const uint32_t st = (sb >> mbr) & 1u;
                            int len = 1;
                            ++mbr;
                            ++q;
                            while (mbr < Cfg::G && ((mask >> mbr) & 1u) && ((sb >> mbr) & 1u) == st) {
                                ++len;
                                ++mbr;
                                ++q;
                            }
                            hr[nr++] = make_uint2(static_cast<uint32_t>(first * B) |
                                                      ((q0 * (Cfg::W_BYTES >> 4)) << 8) | (st << 28),
                                                  make_idesc_bf16(128, len * B, false, TRANS));
                        }
                        hr[0].x |= static_cast<uint32_t>(nr) << 24;
                    }
                    mbar_arrive_expect_tx(&full[slot], Cfg::X_BYTES + k * Cfg::W_BYTES);
                    tma_load_2d(sp, &tmA, &full[slot], static_cast<int>(ent & 0xFFFFFFu) * B, m0);
                    // the present members' blocks, one swizzled tile each, straight
                    // from the packed values (stored once, in BSR order): at the
                    // member's own position (padded) or packed in member order
                    uint32_t mm = mask;
                    for (uint32_t qq = 0; qq < k; ++qq, mm &= mm - 1) {
                        const uint32_t pos = Cfg::PAD ? static_cast<uint32_t>(__ffs(mm) - 1) : qq;
                        tma_load_3d(sp + Cfg::X_BYTES + pos * Cfg::W_BYTES, &tmW, &full[slot], 0, 0, ids[off + qq]);
                    }
                    if (tn < n) tma_prefetch_2d(&tmA, static_cast<int>(entn & 0xFFFFFFu) * B, m0);
#pragma unroll
                    for (int i = 0; i < Cfg::S / Cfg::P; ++i)
                        if (slot == p + i * Cfg::P) fills[i] = use + 1;
                }
            }
            // every lane is done with the chunk (lane 0 read its block ids)
            __syncwarp();
            if (lane == 0) mbar_arrive(&cempty[cs]);
            e += n;
        }
        if (lane == 0) {
            if (!ok) {
                *abort_flag = 1;
                set_status(args.status, BSL_ERR_TIMEOUT);
            }
            // every copy this warp issued lands before the CTA's smem is released
            // (the last fill of a slot is the newest phase of its barrier)
#pragma unroll
            for (int i = 0; i < Cfg::S / Cfg::P; ++i) {
                const int slot = p + i * Cfg::P;
                if (fills[i] > 0 && !mbar_wait(&full[slot], (fills[i] - 1) & 1, tmo, nullptr))
                    set_status(args.status, BSL_ERR_TIMEOUT);
            }
        }
        __syncwarp();
    } else if (warp == Cfg::W_MMA) {
        // ------------------------------------------------------------ MMA issuer
        // The whole warp runs the loop converged (waits, header reads); the
        // MMAs and commits are issued by lane 0 (a predicate).  Per entry: one
        // wait, the header's runs (per 128-row half and 16-wide K step one
        // MMA each), one commit that frees the slot.
        Ring ar;
        int e = 0;
        bool ok = true, any = false;
        const uint32_t lead = lane == 0 ? 1u : 0u;
        const uint32_t sbase = smem_u32(slots);
        const uint64_t xdesc0 = make_sdesc(sbase, 16, Cfg::SBO, Cfg::LAYOUT);
        const uint64_t wdesc0 = TRANS ? make_sdesc(sbase + Cfg::X_BYTES, Cfg::W_BYTES, Cfg::SBO, Cfg::LAYOUT)
                                      : make_sdesc(sbase + Cfg::X_BYTES, 16, Cfg::SBO, Cfg::LAYOUT);
        const uint32_t xlo0 = static_cast<uint32_t>(xdesc0), xhi = static_cast<uint32_t>(xdesc0 >> 32);
        const uint32_t wlo0 = static_cast<uint32_t>(wdesc0), whi = static_cast<uint32_t>(wdesc0 >> 32);
        // descriptor address units (16 bytes) per 16-wide K step of the weight operand
        constexpr uint32_t KSTEP_W = TRANS ? (16 * Cfg::ROW_BYTES) >> 4 : 2;
        constexpr uint32_t SUB_LO = Cfg::SUB_BYTES >> 4;
        for (int j = 0;; ++j) {
            int uid = -1, nent = 0, good = 1;
            if (lane == 0) good = unit_take<Cfg::UR>(ufull, uempty, uring, j, &uid, &nent, tmo, abort_flag);
            good = __shfl_sync(0xffffffffu, good, 0);
            uid = __shfl_sync(0xffffffffu, uid, 0);
            nent = __shfl_sync(0xffffffffu, nent, 0);
            if (!good) {
                ok = false;
                break;
            }
            if (uid < 0) break;
            int mt, g;
            decode_unit(args, uid, &mt, &g);
            const bool two = args.M - mt * Cfg::MT > Cfg::BM;  // second 128-row half in range
            if (__any_sync(0xffffffffu, !mbar_wait(&tempty[ar.slot], ar.phase ^ 1, tmo, abort_flag))) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t d0 = tmem_base + ar.slot * Cfg::ACC_COLS;
            for (int t = 0; t < nent; ++t, ++e) {
                const int slot = e & (Cfg::S - 1);
                // the copies are ordered before the MMAs by the barrier itself (both
                // are async-proxy accesses), so no tcgen05 fence is needed here
                if (__any_sync(0xffffffffu, !mbar_wait(&full[slot], (e >> Cfg::S_LOG) & 1, tmo, abort_flag))) {
                    ok = false;
                    break;
                }
                const uint32_t soff = static_cast<uint32_t>(slot) * (Cfg::SLOT_BYTES >> 4);
                const uint32_t xlo = xlo0 + soff, wlo = wlo0 + soff;
                if constexpr (Cfg::PAD) {
                    // one run of all members; the unit's first entry overwrites
                    // the whole accumulator, later ones add to it
                    const uint32_t st = t > 0 ? 1u : 0u;
                    const uint32_t y = make_idesc_bf16(128, Cfg::G * B, false, TRANS);
#pragma unroll
                    for (int kk = 0; kk < B / 16; ++kk)
                        umma_bf16_lo_lead(lead, d0, xlo + kk * 2, xhi, wlo + kk * KSTEP_W, whi, y, kk ? 1u : st);
                    if (two) {
#pragma unroll
                        for (int kk = 0; kk < B / 16; ++kk)
                            umma_bf16_lo_lead(lead, d0 + Cfg::HALF_COLS, xlo + SUB_LO + kk * 2, xhi,
                                               wlo + kk * KSTEP_W, whi, y, kk ? 1u : st);
                    }
                } else {
                    const uint4 *hs = hdr + slot * Cfg::HDR_V4;
                    const uint4 h0 = hs[0];
                    const int nr = static_cast<int>((h0.x >> 24) & 0xFu);
                    auto issue_run = [&](uint32_t x, uint32_t y) {
                        const uint32_t dcol = d0 + (x & 0xFFu);
                        const uint32_t blo = wlo + ((x >> 8) & 0xFFFFu);
                        const uint32_t st = x >> 28;
#pragma unroll
                        for (int kk = 0; kk < B / 16; ++kk)
                            umma_bf16_lo_lead(lead, dcol, xlo + kk * 2, xhi, blo + kk * KSTEP_W, whi, y, kk ? 1u : st);
                        if (two) {
#pragma unroll
                            for (int kk = 0; kk < B / 16; ++kk)
                                umma_bf16_lo_lead(lead, dcol + Cfg::HALF_COLS, xlo + SUB_LO + kk * 2, xhi,
                                                   blo + kk * KSTEP_W, whi, y, kk ? 1u : st);
                        }
                    };
                    issue_run(h0.x, h0.y);
                    if (nr > 1) issue_run(h0.z, h0.w);
                    if constexpr (Cfg::HDR_V4 > 1) {
                        if (nr > 2) {
                            const uint4 h1 = hs[1];
                            issue_run(h1.x, h1.y);
                            if (nr > 3) issue_run(h1.z, h1.w);
                        }
                    }
                }
                // the slot is free once these MMAs finish
                umma_commit_lead(lead, &empty[slot]);
                any = true;
            }
            if (!ok) break;
            if (nent > 0) umma_commit_lead(lead, &tfull[ar.slot]);
            else if (lane == 0) mbar_arrive(&tfull[ar.slot]);
            __syncwarp();
            ar.next(Cfg::ACC);
        }
        if (lane == 0 && !ok) {
            *abort_flag = 1;
            set_status(args.status, BSL_ERR_TIMEOUT);
        }
        if (any) {  // all MMAs of lane 0 complete before TMEM is freed
            umma_commit_lead(lead, drain);
            if (lane == 0 && !mbar_wait(drain, 0, tmo, nullptr)) set_status(args.status, BSL_ERR_TIMEOUT);
        }
        __syncwarp();
    } else if (warp == Cfg::W_SCHED) {
        // ------------------------------------------------------------ scheduler
        // Takes the units of this CTA from the per-weight counter and stages
        // each unit's entries, 32 at a time, for the producers: coordinate and
        // member mask, the members written by earlier entries of the unit
        // (their MMAs accumulate, the others overwrite), the offset of the
        // entry's blocks in the chunk and the BSR ids of those blocks.  The
        // dependent global loads of the plan thus run ahead of the copies.  A
        // new unit is taken only once a chunk slot is free, so the CTA holds at
        // most one unit beyond the one its producers are issuing.
        bool ok = true, drained = false;  // drained: this CTA's take past the last unit is done
        const bool fixed = args.units <= static_cast<int>(gridDim.x);
        int cc = 0;                       // chunks staged
        for (int j = 0; ok; ++j) {
            int good = 1;
            if (lane == 0 && cc >= Cfg::D)
                good = mbar_wait(&cempty[cc & (Cfg::D - 1)], ((cc / Cfg::D) - 1) & 1, tmo, abort_flag);
            if (!__shfl_sync(0xffffffffu, good, 0)) {
                ok = false;
                break;
            }
            int ord = -1;
            if (lane == 0) {
                // every CTA's first unit is unit blockIdx.x (grid <= units); the
                // counter hands out the rest, and is not used when there is no rest
                if (j == 0) ord = static_cast<int>(blockIdx.x);
                else ord = fixed ? -1 : take_unit(args.sched, args.units);
                drained = ord < 0;
            }
            ord = __shfl_sync(0xffffffffu, ord, 0);
            int mt = 0, g = 0, z = 0, zend = 0, bcur = 0;
            if (ord >= 0) {
                decode_unit(args, ord, &mt, &g);
                z = args.grp_ptr[g];
                zend = args.grp_ptr[g + 1];
                bcur = args.grp_bptr[g];
            }
            if (lane == 0) {
                const int s = j % Cfg::UR;
                if (j >= Cfg::UR && !mbar_wait(&uempty[s], ((j / Cfg::UR) - 1) & 1, tmo, abort_flag)) {
                    good = 0;
                } else {
                    uring[2 * s] = ord;
                    uring[2 * s + 1] = zend - z;
                    mbar_arrive(&ufull[s]);
                }
            }
            if (!__shfl_sync(0xffffffffu, good, 0)) {
                ok = false;
                break;
            }
            if (ord < 0) break;
            const int m0 = mt * Cfg::MT;
            uint32_t seen_carry = 0;  // members present in earlier chunks of this unit
            for (int eb = z; eb < zend; eb += 32) {
                const int n = min(32, zend - eb);
                const uint32_t el = lane < n ? static_cast<uint32_t>(args.grp_ent[eb + lane]) : 0u;
                const uint32_t ml = el >> 24;
                const int kl = __popc(ml);
                int incl = kl;      // inclusive prefix of block counts over the chunk
                uint32_t orl = ml;  // inclusive prefix OR of member masks
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int v = __shfl_up_sync(0xffffffffu, incl, o);
                    const uint32_t w = __shfl_up_sync(0xffffffffu, orl, o);
                    if (lane >= o) {
                        incl += v;
                        orl |= w;
                    }
                }
                uint32_t seen_ex = __shfl_up_sync(0xffffffffu, orl, 1);
                seen_ex = (lane == 0 ? 0u : seen_ex) | seen_carry;
                const int total = __shfl_sync(0xffffffffu, incl, 31);
                const uint32_t all_or = __shfl_sync(0xffffffffu, orl, 31);
                const int cs = cc & (Cfg::D - 1);
                if (lane == 0 && cc >= Cfg::D && eb > z)
                    good = mbar_wait(&cempty[cs], ((cc / Cfg::D) - 1) & 1, tmo, abort_flag);
                if (!__shfl_sync(0xffffffffu, good, 0)) {
                    ok = false;
                    break;
                }
                int *ch = chunks + cs * (Cfg::CH_BYTES / 4);
                if (lane == 0) {
                    ch[0] = n;
                    ch[1] = m0;
                }
                ch[4 + lane] = static_cast<int>(el);
                ch[36 + lane] = static_cast<int>(seen_ex | static_cast<uint32_t>(incl - kl) << 8);
                for (int i = lane; i < total; i += 32) ch[68 + i] = args.grp_blk[bcur + i];
                __syncwarp();
                if (lane == 0) mbar_arrive(&cfull[cs]);
                bcur += total;
                seen_carry |= all_or;
                ++cc;
            }
        }
        if (ok) {  // tell the producers that no unit is left
            int good = 1;
            const int cs = cc & (Cfg::D - 1);
            if (lane == 0) {
                if (cc >= Cfg::D && !mbar_wait(&cempty[cs], ((cc / Cfg::D) - 1) & 1, tmo, abort_flag)) {
                    good = 0;
                } else {
                    chunks[cs * (Cfg::CH_BYTES / 4)] = -1;
                    mbar_arrive(&cfull[cs]);
                }
            }
            ok = __shfl_sync(0xffffffffu, good, 0) != 0;
        }
        if (lane == 0 && !ok) {
            *abort_flag = 1;
            set_status(args.status, BSL_ERR_TIMEOUT);
            // take the remaining units too (they are left undone: the status
            // reports the timeout), so that the counter still returns to zero
            if (!drained && !fixed)
                while (take_unit(args.sched, args.units) >= 0) {
                }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue
        // Each warp drains its own 32 TMEM lanes (tile rows) of every chunk
        // and writes them with its own TMA stores (two staging chunks per
        // warp), so the four epilogue warps never wait on one another.
        const int q = warp & 3;  // TMEM lane quarter this warp may access
        uint8_t *wbuf = outbuf + q * 2 * Cfg::WARP_OUT;
        Ring ar;
        uint32_t ob = 0;
        bool ok = true;
        for (int j = 0;; ++j) {
            int uid = -1, nent = 0, go = 1;
            if (lane == 0) {
                go = unit_take<Cfg::UR>(ufull, uempty, uring, j, &uid, &nent, tmo, abort_flag);
                if (go && uid >= 0) go = mbar_wait(&tfull[ar.slot], ar.phase, tmo, abort_flag);
            }
            go = __shfl_sync(0xffffffffu, go, 0);
            uid = __shfl_sync(0xffffffffu, uid, 0);
            if (!go) {
                ok = false;
                break;
            }
            if (uid < 0) break;
            tc_fence_after();
            int mt, g;
            decode_unit(args, uid, &mt, &g);
            const int m0 = mt * Cfg::MT;
            const int nsub = args.M - m0 > Cfg::BM ? 2 : 1;
            // members of the group and whether they hold any block (lane i < G)
            const int mi = g * Cfg::G + lane;
            int mseg = -1, mnz = 0;
            if (lane < Cfg::G && mi < args.nseg) {
                mseg = args.seg_order[mi];
                mnz = args.seg_ptr[mseg + 1] > args.seg_ptr[mseg];
            }
            for (int s = 0; s < nsub; ++s) {
                const int r0 = m0 + s * Cfg::BM + q * 32;  // first output row of this warp
                if (r0 >= args.M) continue;
                for (int mbr = 0; mbr < Cfg::G; ++mbr) {
                    const int seg = __shfl_sync(0xffffffffu, mseg, mbr);
                    const int nz = __shfl_sync(0xffffffffu, mnz, mbr);
                    if (seg < 0) break;
                    uint32_t v[B];
                    // the bias of the member's b output columns (the same for every row)
                    float bv[B];
                    if (args.bias) {
                        const uint4 *bp = reinterpret_cast<const uint4 *>(args.bias + static_cast<int64_t>(seg) * B);
#pragma unroll
                        for (int c = 0; c < B / 8; ++c) {
                            const uint4 u = __ldg(bp + c);
                            const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                            for (int h = 0; h < 4; ++h) {
                                bv[8 * c + 2 * h] = __uint_as_float(w4[h] << 16);
                                bv[8 * c + 2 * h + 1] = __uint_as_float(w4[h] & 0xFFFF0000u);
                            }
                        }
                    }
                    if (nz) {
                        const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                                               ar.slot * Cfg::ACC_COLS + s * Cfg::HALF_COLS + mbr * B;
#pragma unroll
                        for (int c = 0; c < B / 16; ++c)
                            tmem_ld16(taddr + c * 16, *reinterpret_cast<uint32_t(*)[16]>(&v[c * 16]));
                        tmem_wait_ld();
                    } else {
#pragma unroll
                        for (int c = 0; c < B; ++c) v[c] = 0u;
                    }
                    if (args.bias) {
#pragma unroll
                        for (int c = 0; c < B; ++c) v[c] = __float_as_uint(__uint_as_float(v[c]) + bv[c]);
                    }
                    if (lane == 0) bulk_wait_group_read<1>();  // staging chunk `ob` was read out
                    __syncwarp();
                    uint8_t *dst = wbuf + ob * Cfg::WARP_OUT + lane * Cfg::ROW_BYTES;
#pragma unroll
                    for (int c = 0; c < B / 8; ++c) {
                        uint4 pk;
                        pk.x = pack_bf16x2(__uint_as_float(v[8 * c + 0]), __uint_as_float(v[8 * c + 1]));
                        pk.y = pack_bf16x2(__uint_as_float(v[8 * c + 2]), __uint_as_float(v[8 * c + 3]));
                        pk.z = pack_bf16x2(__uint_as_float(v[8 * c + 4]), __uint_as_float(v[8 * c + 5]));
                        pk.w = pack_bf16x2(__uint_as_float(v[8 * c + 6]), __uint_as_float(v[8 * c + 7]));
                        *reinterpret_cast<uint4 *>(dst + swz_chunk<B>(c, lane) * 16) = pk;
                    }
                    fence_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        tma_store_2d(&tmO, wbuf + ob * Cfg::WARP_OUT, seg * B, r0);
                        bulk_commit_group();
                    }
                    ob ^= 1;
                }
            }
            // every TMEM read of this accumulator is complete (each was waited)
            tc_fence_before();
            mbar_arrive(&tempty[ar.slot]);
            ar.next(Cfg::ACC);
        }
        if (lane == 0) {
            if (!ok) {
                *abort_flag = 1;
                set_status(args.status, BSL_ERR_TIMEOUT);
            }
            bulk_wait_group<0>();
        }
        __syncwarp();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == Cfg::W_MMA) {
        tc_fence_after();
        tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
    }
}

template <int B, bool TRANS>
bsl_status run(const CUtensorMap &a, const CUtensorMap &o, const CUtensorMap &w, const SpmmArgs &args,
               cudaStream_t s)
{
    using Cfg = SpmmCfg<B>;
    auto kern = k_spmm_tc<B, TRANS>;
    const bsl_status sa = set_smem_once(reinterpret_cast<const void *>(kern), Cfg::SMEM_BYTES);
    if (sa != BSL_OK) return sa;
    // the work counter is zero here: the pack zeroed it and every launch,
    // one that ran out of time included, sets it back to zero at its end
    const int grid = args.units < num_sms() ? args.units : num_sms();
    return cuda_status(launch_dependent(kern, grid, Cfg::THREADS, Cfg::SMEM_BYTES, s, a, o, w, args));
}

}  // namespace

bsl_status launch_spmm_tc(const void *A, int32_t M, int32_t a_cols, const bsl_bsr *W, bool transposed,
                          const void *bias, void *out, int32_t out_cols, cudaStream_t s)
{
    const int B = W->b;
    if (W->nnz == 0 && (transposed || !bias))
        return cuda_status(cudaMemsetAsync(out, 0, static_cast<size_t>(M) * out_cols * 2, s));
    CUtensorMap ma, mo, mw;
    if (!make_map_2d(&ma, A, a_cols, M, static_cast<uint64_t>(a_cols) * 2, B, 256, 2 * B) ||
        !make_map_2d(&mo, out, out_cols, M, static_cast<uint64_t>(out_cols) * 2, B, 32, 2 * B) ||
        (W->nnz > 0 && !make_block_map(&mw, W->values, B, W->nnz, B)))
        return BSL_ERR_CUDA;
    if (W->nnz == 0) mw = ma;  // no weight block is ever loaded
    const int G = 128 / B;
    SpmmArgs args;
    args.M = M;
    args.mtiles = (M + 255) / 256;
    args.nseg = transposed ? W->K / B : W->N / B;
    args.ngroups = (args.nseg + G - 1) / G;
    args.units = args.ngroups * args.mtiles;
    args.seg_ptr = transposed ? W->col_ptr : W->row_ptr;
    args.seg_order = transposed ? W->col_order : W->row_order;
    args.grp_ptr = transposed ? W->cgrp_ptr : W->rgrp_ptr;
    args.grp_bptr = transposed ? W->cgrp_bptr : W->rgrp_bptr;
    args.grp_ent = transposed ? W->cgrp_ent : W->rgrp_ent;
    args.grp_blk = transposed ? W->cgrp_blk : W->rgrp_blk;
    args.sched = W->sched + (transposed ? 2 : 0);
    args.bias = transposed ? nullptr : static_cast<const __nv_bfloat16 *>(bias);
    args.status = W->status;
    args.timeout_ns = wait_timeout_ns();
    if (B == 64) return transposed ? run<64, true>(ma, mo, mw, args, s) : run<64, false>(ma, mo, mw, args, s);
    return transposed ? run<32, true>(ma, mo, mw, args, s) : run<32, false>(ma, mo, mw, args, s);
}

}  // namespace bsl

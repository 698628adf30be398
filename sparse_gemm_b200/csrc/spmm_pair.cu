// spmm_pair.cu -- block-sparse forward on pairs of SMs (tcgen05 cta_group::2).
//
//   Y [M,N] = X [M,K] . W~^T (+ bias)       (Hugging Face pytorch_block_sparse
//   release note, "Block-Sparse Implementation and Usage": only the nonzero
//   b x b blocks of W are kept and multiplied; torchao sparsity README,
//   Table 4.1: the BSR index lists them per block row.)
//
// Why pairs.  At low density each stored block needs its own activation tile
// X[256 rows, c-block], and moving those tiles from L2 into shared memory,
// not tensor-core arithmetic, sets the pace.  Activation tiles are shared by
// the block rows of a group (G = 256/b rows taken longest first; the pack
// merged their block columns into ascending "entries" with a member mask),
// so bigger groups mean fewer tile copies.  A group's accumulator for 256
// rows of M is 256 x G*b = 256 x 256 fp32, which is the whole tensor memory
// of one SM, but only half of it on each SM of a pair: the two CTAs of a
// cluster run one tcgen05.mma.cta_group::2 of M = 256, each SM holding 128
// rows of the activation tile (operand A) and of the accumulator, and half of
// the weight rows of the MMA (operand B: the hardware lets both SMs read
// both halves).  So each SM keeps two accumulators (512 TMEM columns) and the
// epilogue of one unit overlaps the MMAs of the next, every weight block is
// fetched once per 256 rows, and an M = 256 instruction does twice the work
// of one M = 128 instruction for less shared-memory operand traffic per SM.
//
// Unit = (256-row tile of M, group).  Per entry (one block column of the
// group's union): each CTA copies its 128-row half of the activation tile
// into an X slot and its half of the present members' weight rows into
// consecutive slots of a weight ring (half-blocks of b/2 rows; for a run of
// L consecutive members, CTA h holds half-blocks h*L .. h*L+L-1 of the run's
// 2L).  All copies of both CTAs complete on the leader CTA's barrier
// (.cta_group::2 copies), the leader's single MMA thread issues the run
// MMAs (N = L*b), and one commit multicast to both CTAs frees the entry's
// slots.  The weight ring is separate from the X slots because most entries
// carry one or two of the G possible blocks: a slot sized for G blocks would
// hold mostly empty space.
//
// Roles per CTA (one CTA per SM, clusters of two):
//   warps 0..3  producers: entry e is issued by warp e % 4 of each CTA
//   warp 4      TMEM owner (both CTAs); in the leader CTA the MMA issuer
//   warps 5..8  epilogue: TMEM -> registers (+ bias) -> bf16 (RNE) ->
//               swizzled smem -> TMA store of the CTA's own 128 rows
// The leader's first producer takes units from the weight's work counter
// (zeroed in stream order before each launch) and publishes each id to both
// CTAs.  Every wait is bounded in time; on expiry the kernel records
// BSL_ERR_TIMEOUT, raises the abort flag of both CTAs, drains and exits.
#include "common.cuh"
#include "internal.h"

namespace bsl {
namespace {

// ---------------------------------------------------------------- cluster helpers

__device__ __forceinline__ uint32_t cluster_rank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// shared::cluster address of the same smem offset in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t map_to(uint32_t saddr, uint32_t rank)
{
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
    return r;
}

__device__ __forceinline__ void cluster_sync_all()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ void remote_arrive(uint32_t cluster_addr)
{
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

__device__ __forceinline__ void st_cluster_u32(uint32_t cluster_addr, uint32_t v)
{
    asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(cluster_addr), "r"(v) : "memory");
}

// try_wait with cluster-scope acquire (the barrier receives arrivals from the
// other CTA of the pair that publish data the waiter then reads)
__device__ __forceinline__ bool mbar_try_wait_cl(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ bool mbar_wait_cl(uint64_t *bar, uint32_t parity, uint64_t timeout_ns,
                                             const volatile int *abort)
{
    const uint32_t a = smem_u32(bar);
    if (mbar_try_wait_cl(a, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
#pragma unroll 1
        for (int i = 0; i < 64; ++i)
            if (mbar_try_wait_cl(a, parity)) return true;
        if (abort && *abort) return false;
        if (globaltimer_ns() - t0 > timeout_ns) return false;
    }
}

// 2-D / 3-D tiled loads into this CTA's shared memory whose completion is
// signalled on a barrier of either CTA of the pair (`bar` is a
// shared::cluster address).
__device__ __forceinline__ void tma_load_2d_pair(void *dst, const CUtensorMap *map, uint32_t bar, int32_t x,
                                                 int32_t y)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y)
        : "memory");
}

__device__ __forceinline__ void tma_load_3d_pair(void *dst, const CUtensorMap *map, uint32_t bar, int32_t x,
                                                 int32_t y, int32_t z)
{
    asm volatile(
        "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y), "r"(z)
        : "memory");
}

__device__ __forceinline__ void tmem_alloc2(uint32_t *dst_smem, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tmem_relinquish2()
{
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc2(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// M = 256 MMA over the pair, issued by one thread of the leader CTA
// (predicated on `leader` so the issuing warp stays converged).
__device__ __forceinline__ void umma2_lead(uint32_t leader, uint32_t d_tmem, uint32_t a_lo, uint32_t a_hi,
                                           uint32_t b_lo, uint32_t b_hi, uint32_t idesc, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p, e;\n\t.reg .b64 ad, bd;\n\t"
        "setp.ne.b32 e, %7, 0;\n\t"
        "mov.b64 ad, {%1, %2};\n\t"
        "mov.b64 bd, {%3, %4};\n\t"
        "setp.ne.b32 p, %6, 0;\n\t"
        "@e tcgen05.mma.cta_group::2.kind::f16 [%0], ad, bd, %5, p;\n\t}" ::"r"(d_tmem),
        "r"(a_lo), "r"(a_hi), "r"(b_lo), "r"(b_hi), "r"(idesc), "r"(accumulate), "r"(leader)
        : "memory");
}

// Arrive on the barrier at this smem offset in both CTAs once every MMA the
// thread issued so far is done.
__device__ __forceinline__ void umma2_commit_both(uint32_t leader, uint64_t *bar)
{
    asm volatile(
        "{\n\t.reg .pred e;\n\t"
        "setp.ne.b32 e, %1, 0;\n\t"
        "@e tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %2;\n\t}" ::"r"(
            smem_u32(bar)),
        "r"(leader), "h"(static_cast<uint16_t>(3))
        : "memory");
}

// ---------------------------------------------------------------- configuration

template <int B>
struct PairCfg {
    static constexpr int G = 256 / B;                   // members per group
    static constexpr int ROW_BYTES = B * 2;             // 128 B (b = 64) or 64 B (b = 32)
    static constexpr int XH_BYTES = 128 * ROW_BYTES;    // this CTA's half of an activation tile
    static constexpr int HB_ROWS = B / 2;               // rows of a half-block
    static constexpr int HB_BYTES = HB_ROWS * ROW_BYTES;
    // One ring of units of a half-block's size holds the entries in flight:
    // an entry takes XU units for its activation half-tile and one per
    // present member, contiguous (it starts over at unit 0 when it would run
    // past the end), so light entries leave room for more of them.
    static constexpr int UB = HB_BYTES;                 // ring unit: 4 KB (b = 64), 1 KB (b = 32)
    static constexpr int XU = XH_BYTES / UB;            // units of an activation half-tile: 4 or 8
    static constexpr int RU = B == 64 ? 46 : 192;       // ring units (184 KB or 192 KB)
    static constexpr int UPL = (RU + 31) / 32;          // ring units tracked per lane
    static constexpr int SE = 16;                       // entries in flight at most (barriers, headers)
    static constexpr int W = 16 / G;                    // entries the MMA issuer interleaves
    static constexpr int P = 4;                         // producer warps
    static constexpr int UR = 16;                       // unit-id ring
    static constexpr int W_MMA = P;
    static constexpr int THREADS = (P + 5) * 32;
    static constexpr int ROLES = P + 5;                 // warps of a CTA that read unit ids
    static constexpr int WARP_OUT = 32 * ROW_BYTES;     // one epilogue staging chunk (32 rows)
    static constexpr int OUT_BYTES = 4 * 2 * WARP_OUT;
    static constexpr int ACC = 2;
    static constexpr int ACC_COLS = G * B;              // 256
    static constexpr int TMEM_COLS = ACC * ACC_COLS;    // 512
    static constexpr uint32_t LAYOUT = B == 64 ? kLayoutSw128 : kLayoutSw64;
    static constexpr uint32_t SBO = 8 * ROW_BYTES;
    static constexpr int NUM_BARS = 2 * SE + 2 * ACC + 2 * UR + 1;
    static constexpr int HDR_V4 = 1 + G / 2;            // per entry: {first unit, run count}, then two runs per word
    static constexpr int BLK_IDS = 32 * G;
    static constexpr int SMEM_BYTES = RU * UB + OUT_BYTES + NUM_BARS * 8 + SE * HDR_V4 * 16 + UR * 4 +
                                      P * BLK_IDS * 4 + 64 + 1024;
    static_assert(ACC_COLS == 256 && TMEM_COLS == 512, "TMEM layout");
    static_assert(SE % P == 0 && G <= 8 && G % 2 == 0, "entry slots / members");
    static_assert(RU >= 2 * (XU + G) && RU <= 255 && UB % 1024 == 0, "ring: two largest entries, 8-bit unit index");
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

struct PairArgs {
    int32_t M, nseg, ngroups, mtiles, units;
    const int32_t *seg_ptr;    // [nseg+1] blocks per block row (empty rows give bias / zeros)
    const int32_t *seg_order;  // [nseg] longest first; group g = seg_order[g*G .. g*G+G-1]
    const int32_t *grp_ptr;    // [ngroups+1] entry range per group
    const int32_t *grp_bptr;   // [ngroups+1] block range per group
    const int32_t *grp_ent;    // entries: block column | (member mask << 24)
    const int32_t *grp_blk;    // BSR block of every present member, entry by entry
    int32_t *sched;            // [1] next unit (zeroed before every launch)
    const __nv_bfloat16 *bias; // [N] or null
    int32_t *status;
    uint64_t timeout_ns;
};

__device__ __forceinline__ uint8_t *align1024(uint8_t *p)
{
    return reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

template <int B>
__device__ __forceinline__ int swz_chunk(int chunk, int row)
{
    if constexpr (B == 64) return chunk ^ (row & 7);
    else return chunk ^ ((row >> 1) & 3);
}

// Work order: m-tiles in chunks of CHUNK (their activation rows stay in L2),
// group-major inside a chunk, groups longest first.
constexpr int CHUNK = 8;
__device__ __forceinline__ void decode_unit(const PairArgs &a, int ord, int *mt, int *g)
{
    const int per_chunk = CHUNK * a.ngroups;
    const int ch = ord / per_chunk;
    const int mt0 = ch * CHUNK;
    const int nmt = min(CHUNK, a.mtiles - mt0);
    const int r = ord - ch * per_chunk;
    *g = r / nmt;
    *mt = mt0 + (r - *g * nmt);
}

// Raise the abort flag of both CTAs (the other role of either CTA stops at
// its next bounded wait).
__device__ __forceinline__ void raise_abort(volatile int *abort_flag, uint32_t peer)
{
    *abort_flag = 1;
    st_cluster_u32(map_to(smem_u32(const_cast<int *>(abort_flag)), peer), 1u);
}

template <int B>
__global__ void __launch_bounds__(PairCfg<B>::THREADS, 1)
    k_spmm_pair(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmY,
                const __grid_constant__ CUtensorMap tmW, const PairArgs args)
{
    using Cfg = PairCfg<B>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align1024(smem_raw);
    uint8_t *ring = smem;
    uint8_t *outbuf = ring + Cfg::RU * Cfg::UB;
    uint64_t *bars = reinterpret_cast<uint64_t *>(outbuf + Cfg::OUT_BYTES);
    uint64_t *full = bars;                 // [SE] leader: both CTAs' copies of the entry landed
    uint64_t *empty = full + Cfg::SE;      // [SE] both CTAs: the entry's MMAs are done
    uint64_t *tfull = empty + Cfg::SE;     // both CTAs: accumulator complete
    uint64_t *tempty = tfull + Cfg::ACC;   // leader: both CTAs read the accumulator out
    uint64_t *ufull = tempty + Cfg::ACC;   // both CTAs: unit id published
    uint64_t *uempty = ufull + Cfg::UR;    // leader: unit id read by every role of both CTAs
    uint64_t *drain = uempty + Cfg::UR;
    // [SE][HDR_V4] per entry slot: word 0 = {first ring unit, run count}; then the
    // MMA runs, two per 16-byte word: x = TMEM column | ring unit of the run's
    // first half-block << 8 | overwrite-free flag << 28; y = instruction descriptor
    uint4 *hdr = reinterpret_cast<uint4 *>((reinterpret_cast<uintptr_t>(drain + 1) + 15) & ~uintptr_t(15));
    volatile int *uring = reinterpret_cast<volatile int *>(hdr + Cfg::SE * Cfg::HDR_V4);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(const_cast<int *>(uring + Cfg::UR));
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    int32_t *blk_ids = reinterpret_cast<int32_t *>(tmem_slot + 4);  // [P][BLK_IDS]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const uint32_t peer = rank ^ 1u;
    const bool is_leader = rank == 0;
    const uint64_t tmo = args.timeout_ns;

    if (threadIdx.x == 0) {
        for (int s = 0; s < Cfg::SE; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < Cfg::ACC; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], 8);  // one arrival per epilogue warp of either CTA
        }
        for (int u = 0; u < Cfg::UR; ++u) {
            mbar_init(&ufull[u], 1);
            mbar_init(&uempty[u], 2 * Cfg::ROLES);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_barrier_init();
        tma_prefetch_map(&tmX);
        tma_prefetch_map(&tmY);
        tma_prefetch_map(&tmW);
    }
    if (warp == Cfg::W_MMA) {
        tmem_alloc2(tmem_slot, Cfg::TMEM_COLS);
        tmem_relinquish2();
    }
    tc_fence_before();
    cluster_sync_all();  // both CTAs' barriers initialised and TMEM allocated
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const uint32_t full_leader0 = map_to(smem_u32(&full[0]), 0);  // full[s] of the leader: + 8 s

    // unit id j of this CTA (-1: no more units); false if the wait ran out
    auto unit_take = [&](int j, int *uid) -> bool {
        const int s = j % Cfg::UR;
        if (!mbar_wait_cl(&ufull[s], (j / Cfg::UR) & 1, tmo, abort_flag)) return false;
        *uid = uring[s];
        const uint32_t ue = smem_u32(&uempty[s]);
        if (is_leader) mbar_arrive(&uempty[s]);
        else remote_arrive(map_to(ue, 0));
        return true;
    };

    if (warp < Cfg::P) {
        // ------------------------------------------------------------ producers
        // Every producer warp of both CTAs walks all entries of every unit and
        // computes the same ring allocation; entry e is issued by warp e % P
        // into entry slot e % SE.  Before an entry slot is reused, the MMAs of
        // its previous entry must be done (empty barrier); before ring units
        // are refilled, so must the MMAs of the last entry that used them
        // (MMAs complete in entry order, so the latest such entry suffices).
        const int p = warp;
        int e = 0;                   // entries walked so far (all units of this CTA)
        int upos = 0;                // next free ring unit
        int lastuse[Cfg::UPL];       // lane l: last entry that used ring unit l * UPL + i
#pragma unroll
        for (int i = 0; i < Cfg::UPL; ++i) lastuse[i] = -1;
        bool ok = true;
        for (int j = 0; ok; ++j) {
            int uid = -1, good = 1;
            if (lane == 0) {
                if (p == 0 && is_leader) {
                    // take the next unit only now that this warp starts it
                    const int s = j % Cfg::UR;
                    if (j >= Cfg::UR && !mbar_wait_cl(&uempty[s], ((j / Cfg::UR) - 1) & 1, tmo, abort_flag)) {
                        good = 0;
                    } else {
                        int ord = atomicAdd(args.sched, 1);
                        if (ord >= args.units) ord = -1;
                        uring[s] = ord;
                        st_cluster_u32(map_to(smem_u32(const_cast<int *>(&uring[s])), 1), static_cast<uint32_t>(ord));
                        mbar_arrive(&ufull[s]);
                        remote_arrive(map_to(smem_u32(&ufull[s]), 1));
                    }
                }
                if (good) good = unit_take(j, &uid);
            }
            good = __shfl_sync(0xffffffffu, good, 0);
            uid = __shfl_sync(0xffffffffu, uid, 0);
            if (!good) {
                ok = false;
                break;
            }
            if (uid < 0) break;
            int mt, g;
            decode_unit(args, uid, &mt, &g);
            const int m0 = mt * 256 + static_cast<int>(rank) * 128;
            const int z = args.grp_ptr[g], zend = args.grp_ptr[g + 1];
            int bcur = args.grp_bptr[g];
            uint32_t seen_carry = 0;  // members present in earlier chunks of this unit
            for (int eb = z; eb < zend && ok; eb += 32) {
                const int n = min(32, zend - eb);
                const int el = lane < n ? args.grp_ent[eb + lane] : 0;
                const uint32_t ml = static_cast<uint32_t>(el) >> 24;
                const int kl = __popc(ml);
                int incl = kl;       // inclusive prefix of block counts over the chunk
                uint32_t orl = ml;   // inclusive prefix OR of member masks
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int v = __shfl_up_sync(0xffffffffu, incl, o);
                    const uint32_t w = __shfl_up_sync(0xffffffffu, orl, o);
                    if (lane >= o) {
                        incl += v;
                        orl |= w;
                    }
                }
                const int excl = incl - kl;
                uint32_t seen_ex = __shfl_up_sync(0xffffffffu, orl, 1);
                seen_ex = (lane == 0 ? 0u : seen_ex) | seen_carry;
                const int total = __shfl_sync(0xffffffffu, incl, 31);
                const uint32_t all_or = __shfl_sync(0xffffffffu, orl, 31);
                int32_t *ids = blk_ids + p * Cfg::BLK_IDS;
                __syncwarp();  // lane 0 has finished reading the previous chunk's ids
                for (int i = lane; i < total; i += 32) ids[i] = args.grp_blk[bcur + i];
                __syncwarp();
                for (int t = 0; t < n; ++t) {
                    const uint32_t ent = static_cast<uint32_t>(__shfl_sync(0xffffffffu, el, t));
                    const uint32_t mask = ent >> 24;
                    const int k = __popc(mask);
                    // ring units of this entry: XU + k consecutive, from upos (or 0 on wrap)
                    const int size = Cfg::XU + k;
                    int u0 = upos;
                    if (u0 + size > Cfg::RU) u0 = 0;
                    upos = u0 + size;
                    int need = -1;  // latest entry that used any of these units
#pragma unroll
                    for (int i = 0; i < Cfg::UPL; ++i) {
                        const int u = lane * Cfg::UPL + i;
                        if (u >= u0 && u < u0 + size) {
                            need = max(need, lastuse[i]);
                            lastuse[i] = e;
                        }
                    }
#pragma unroll
                    for (int o = 16; o; o >>= 1) need = max(need, __shfl_xor_sync(0xffffffffu, need, o));
                    if ((e & (Cfg::P - 1)) == p) {
                        const int off = __shfl_sync(0xffffffffu, excl, t);
                        const uint32_t sb = __shfl_sync(0xffffffffu, seen_ex, t);
                        if (lane == 0) {
                            const int slot = e % Cfg::SE;
                            if (e >= Cfg::SE && !mbar_wait(&empty[slot], ((e / Cfg::SE) - 1) & 1, tmo, abort_flag))
                                good = 0;
                            if (good && need > e - Cfg::SE && need >= 0 &&
                                !mbar_wait(&empty[need % Cfg::SE], (need / Cfg::SE) & 1, tmo, abort_flag))
                                good = 0;
                            if (good) {
                                // runs: consecutive present members with the same first-write
                                // status; their half-blocks follow the activation half-tile
                                uint4 *hs = hdr + slot * Cfg::HDR_V4;
                                uint2 *hr = reinterpret_cast<uint2 *>(hs + 1);
                                int nr = 0, mbr = 0, q = 0;
                                const int wu0 = u0 + Cfg::XU;  // ring unit of the first half-block
                                const uint32_t fb = full_leader0 + 8u * static_cast<uint32_t>(slot);
                                while (mbr < Cfg::G) {
                                    if (!((mask >> mbr) & 1u)) {
                                        ++mbr;
                                        continue;
                                    }
                                    const int first = mbr, q0 = q;
                                    const uint32_t st = (sb >> mbr) & 1u;
                                    int len = 1;
                                    ++mbr;
                                    while (mbr < Cfg::G && ((mask >> mbr) & 1u) && ((sb >> mbr) & 1u) == st) {
                                        ++len;
                                        ++mbr;
                                    }
                                    q += len;
                                    hr[nr++] = make_uint2(static_cast<uint32_t>(first * B) |
                                                              (static_cast<uint32_t>(wu0 + q0) << 8) | (st << 28),
                                                          make_idesc_bf16(256, len * B, false, false));
                                    // this CTA's half-blocks of the run: h*len .. h*len+len-1
                                    for (int i = 0; i < len; ++i) {
                                        const int hb = static_cast<int>(rank) * len + i;
                                        tma_load_3d_pair(ring + (wu0 + q0 + i) * Cfg::UB, &tmW, fb, 0,
                                                         (hb & 1) * Cfg::HB_ROWS, ids[off + q0 + (hb >> 1)]);
                                    }
                                }
                                hs[0] = make_uint4(static_cast<uint32_t>(u0), static_cast<uint32_t>(nr), 0u, 0u);
                                if (is_leader)
                                    mbar_arrive_expect_tx(&full[slot], 2u * (Cfg::XH_BYTES + k * Cfg::HB_BYTES));
                                tma_load_2d_pair(ring + u0 * Cfg::UB, &tmX, fb, static_cast<int>(ent & 0xFFFFFFu) * B,
                                                 m0);
                            }
                        }
                        if (!__shfl_sync(0xffffffffu, good, 0)) {
                            ok = false;
                            break;
                        }
                    }
                    ++e;
                }
                bcur += total;
                seen_carry |= all_or;
            }
        }
        if (lane == 0) {
            if (!ok) {
                raise_abort(abort_flag, peer);
                set_status(args.status, BSL_ERR_TIMEOUT);
                // the other CTA's copies of entries this CTA's leader never armed can only
                // be waited out: give them time to land before shared memory is released
                if (!is_leader) {
                    const uint64_t t0 = globaltimer_ns();
                    while (globaltimer_ns() - t0 < 50000u) __nanosleep(1000);
                }
            }
            // before this CTA's shared memory can go away: the copies of this
            // warp's last entries (both CTAs' bytes, on the leader's barriers)
            // landed, and in both CTAs their MMAs (whose commits arrive here)
            // are done; these are the newest phases of their entry slots
            for (int le = e > Cfg::SE ? e - Cfg::SE : 0; le < e; ++le) {
                if ((le & (Cfg::P - 1)) != p) continue;
                const int slot = le % Cfg::SE;
                if (is_leader && !mbar_wait(&full[slot], (le / Cfg::SE) & 1, tmo, nullptr))
                    set_status(args.status, BSL_ERR_TIMEOUT);
                if (ok && !mbar_wait(&empty[slot], (le / Cfg::SE) & 1, tmo, nullptr))
                    set_status(args.status, BSL_ERR_TIMEOUT);
            }
        }
        __syncwarp();
    } else if (warp == Cfg::W_MMA) {
        // ------------------------------------------------------------ MMA issuer (leader)
        // The whole warp runs the loop converged; lane 0 issues the MMAs and
        // commits.  The other CTA's TMEM owner only takes unit ids.
        uint32_t acc = 0, acc_phase = 0;
        int e = 0;
        bool ok = true, any = false;
        const uint32_t lead = (lane == 0 && is_leader) ? 1u : 0u;
        const uint64_t rdesc0 = make_sdesc(smem_u32(ring), 16, Cfg::SBO, Cfg::LAYOUT);
        const uint32_t rlo0 = static_cast<uint32_t>(rdesc0), rhi = static_cast<uint32_t>(rdesc0 >> 32);
        constexpr uint32_t U_LO = Cfg::UB >> 4;  // descriptor address units (16 bytes) per ring unit
        for (int j = 0;; ++j) {
            int uid = -1, good = 1;
            if (lane == 0) good = unit_take(j, &uid);
            good = __shfl_sync(0xffffffffu, good, 0);
            uid = __shfl_sync(0xffffffffu, uid, 0);
            if (!good) {
                ok = false;
                break;
            }
            if (uid < 0) break;
            if (!is_leader) continue;
            int mt, g;
            decode_unit(args, uid, &mt, &g);
            const int z = args.grp_ptr[g], zend = args.grp_ptr[g + 1];
            if (__any_sync(0xffffffffu, !mbar_wait_cl(&tempty[acc], acc_phase ^ 1, tmo, abort_flag))) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t d0 = tmem_base + acc * Cfg::ACC_COLS;
            // Entries are issued a window of W at a time, K-step major over all
            // the window's runs: consecutive MMAs then accumulate into different
            // TMEM columns (other members, other runs), so the tensor pipe does not
            // wait for one MMA's result before starting the next.  MMAs that do
            // share a member keep their order within each K step, so the first
            // (overwriting) MMA of a member still comes first.
            for (int t = z; t < zend;) {
                const int nw = min(Cfg::W, zend - t);
                bool bad = false;
                for (int i = 0; i < nw; ++i)
                    bad |= !mbar_wait(&full[(e + i) % Cfg::SE], ((e + i) / Cfg::SE) & 1, tmo, abort_flag);
                if (__any_sync(0xffffffffu, bad)) {
                    ok = false;
                    break;
                }
                // runs of the window: x = TMEM column | ring unit of the run's first
                // half-block << 8 | ring unit of its activation half-tile << 16 |
                // overwrite-free flag << 28; y = instruction descriptor (0: no run)
                uint32_t rx[Cfg::W * Cfg::G], ry[Cfg::W * Cfg::G];
#pragma unroll
                for (int i = 0; i < Cfg::W; ++i) {
                    const uint4 *hs = hdr + ((e + i) % Cfg::SE) * Cfg::HDR_V4;
                    const uint4 h0 = i < nw ? hs[0] : make_uint4(0, 0, 0, 0);
                    const int nr = static_cast<int>(h0.y);
#pragma unroll
                    for (int wv = 1; wv < Cfg::HDR_V4; ++wv) {
                        const uint4 h1 = nr > 2 * (wv - 1) ? hs[wv] : make_uint4(0, 0, 0, 0);
                        const int r0 = i * Cfg::G + 2 * (wv - 1);
                        rx[r0] = h1.x | (h0.x << 16);
                        ry[r0] = nr > 2 * (wv - 1) ? h1.y : 0u;
                        rx[r0 + 1] = h1.z | (h0.x << 16);
                        ry[r0 + 1] = nr > 2 * (wv - 1) + 1 ? h1.w : 0u;
                    }
                }
#pragma unroll
                for (int kk = 0; kk < B / 16; ++kk)
#pragma unroll
                    for (int r = 0; r < Cfg::W * Cfg::G; ++r)
                        if (ry[r])
                            umma2_lead(lead, d0 + (rx[r] & 0xFFu), rlo0 + ((rx[r] >> 16) & 0xFFu) * U_LO + kk * 2,
                                       rhi, rlo0 + ((rx[r] >> 8) & 0xFFu) * U_LO + kk * 2, rhi, ry[r],
                                       kk ? 1u : ((rx[r] >> 28) & 1u));
                for (int i = 0; i < nw; ++i)
                    umma2_commit_both(lead, &empty[(e + i) % Cfg::SE]);  // the entry's slots are free in both CTAs
                any = true;
                e += nw;
                t += nw;
            }
            if (!ok) break;
            if (zend > z) {
                umma2_commit_both(lead, &tfull[acc]);
            } else if (lane == 0) {  // no entry: nothing to wait for, the accumulator is "complete"
                mbar_arrive(&tfull[acc]);
                remote_arrive(map_to(smem_u32(&tfull[acc]), 1));
            }
            __syncwarp();
            if (++acc == Cfg::ACC) {
                acc = 0;
                acc_phase ^= 1;
            }
        }
        if (lane == 0 && !ok) {
            raise_abort(abort_flag, peer);
            set_status(args.status, BSL_ERR_TIMEOUT);
        }
        if (is_leader && any) {  // every MMA is complete before TMEM is freed
            // commit to this CTA's barrier only (no arrival may be left in flight to the other)
            if (lead)
                asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                                 smem_u32(drain))
                             : "memory");
            if (lane == 0 && !mbar_wait(drain, 0, tmo, nullptr)) set_status(args.status, BSL_ERR_TIMEOUT);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;  // TMEM lane quarter this warp may access
        uint8_t *wbuf = outbuf + q * 2 * Cfg::WARP_OUT;
        uint32_t acc = 0, acc_phase = 0, ob = 0;
        bool ok = true;
        const uint32_t te_leader0 = map_to(smem_u32(&tempty[0]), 0);
        for (int j = 0;; ++j) {
            int uid = -1, go = 1;
            if (lane == 0) {
                go = unit_take(j, &uid);
                if (go && uid >= 0) go = mbar_wait(&tfull[acc], acc_phase, tmo, abort_flag);
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
            const int r0 = mt * 256 + static_cast<int>(rank) * 128 + q * 32;  // first output row of this warp
            const int mi = g * Cfg::G + lane;
            int mseg = -1, mnz = 0;
            if (lane < Cfg::G && mi < args.nseg) {
                mseg = args.seg_order[mi];
                mnz = args.seg_ptr[mseg + 1] > args.seg_ptr[mseg];
            }
            for (int mbr = 0; mbr < Cfg::G; ++mbr) {
                const int seg = __shfl_sync(0xffffffffu, mseg, mbr);
                const int nz = __shfl_sync(0xffffffffu, mnz, mbr);
                if (seg < 0) break;
                uint32_t v[B];
                if (nz) {
                    const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * Cfg::ACC_COLS +
                                           mbr * B;
#pragma unroll
                    for (int c = 0; c < B / 16; ++c)
                        tmem_ld16(taddr + c * 16, *reinterpret_cast<uint32_t(*)[16]>(&v[c * 16]));
                    tmem_wait_ld();
                } else {
#pragma unroll
                    for (int c = 0; c < B; ++c) v[c] = 0u;
                }
                if (r0 >= args.M) continue;  // rows past M: nothing to store (TMEM was read anyway)
                if (args.bias) {
                    const uint4 *bp = reinterpret_cast<const uint4 *>(args.bias + static_cast<int64_t>(seg) * B);
#pragma unroll
                    for (int c = 0; c < B / 8; ++c) {
                        const uint4 u = __ldg(bp + c);
                        const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                        for (int h = 0; h < 4; ++h) {
                            v[8 * c + 2 * h] = __float_as_uint(__uint_as_float(v[8 * c + 2 * h]) +
                                                               __uint_as_float(w4[h] << 16));
                            v[8 * c + 2 * h + 1] = __float_as_uint(__uint_as_float(v[8 * c + 2 * h + 1]) +
                                                                   __uint_as_float(w4[h] & 0xFFFF0000u));
                        }
                    }
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
                    tma_store_2d(&tmY, wbuf + ob * Cfg::WARP_OUT, seg * B, r0);
                    bulk_commit_group();
                }
                ob ^= 1;
            }
            // every TMEM read of this accumulator is complete (each was waited)
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if (is_leader) mbar_arrive(&tempty[acc]);
                else remote_arrive(te_leader0 + 8u * acc);
            }
            if (++acc == Cfg::ACC) {
                acc = 0;
                acc_phase ^= 1;
            }
        }
        if (lane == 0) {
            if (!ok) {
                raise_abort(abort_flag, peer);
                set_status(args.status, BSL_ERR_TIMEOUT);
            }
            bulk_wait_group<0>();
        }
        __syncwarp();
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync_all();  // no copy, commit or arrival of the pair targets this CTA any more
    tc_fence_after();
    if (warp == Cfg::W_MMA) tmem_dealloc2(tmem_base, Cfg::TMEM_COLS);
}

template <int B>
bsl_status run(const CUtensorMap &x, const CUtensorMap &y, const CUtensorMap &w, const PairArgs &args,
               cudaStream_t s)
{
    using Cfg = PairCfg<B>;
    auto kern = k_spmm_pair<B>;
    const bsl_status sa = set_smem_once(reinterpret_cast<const void *>(kern), Cfg::SMEM_BYTES);
    if (sa != BSL_OK) return sa;
    cudaError_t e;
    e = cudaMemsetAsync(args.sched, 0, sizeof(int32_t), s);
    if (e != cudaSuccess) return cuda_status(e);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2);
    cfg.blockDim = dim3(Cfg::THREADS);
    cfg.dynamicSmemBytes = Cfg::SMEM_BYTES;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    // one pair per two SMs that can host one at the same time (per device, cached)
    static int pairs_cache[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    int pairs_max = dev < 64 ? pairs_cache[dev] : 0;
    if (pairs_max <= 0) {
        cfg.gridDim = dim3(num_sms() & ~1);
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n <= 0) {
            cudaGetLastError();
            n = num_sms() / 2;
        }
        pairs_max = n < num_sms() / 2 ? n : num_sms() / 2;
        if (dev < 64) pairs_cache[dev] = pairs_max;
    }
    const int pairs = args.units < pairs_max ? args.units : pairs_max;
    cfg.gridDim = dim3(2 * (pairs > 0 ? pairs : 1));
    return cuda_status(cudaLaunchKernelEx(&cfg, kern, x, y, w, args));
}

}  // namespace

bsl_status launch_spmm_pair(const void *X, int32_t M, const bsl_bsr *W, const void *bias, void *Y, cudaStream_t s)
{
    const int B = W->b;
    CUtensorMap mx, my, mw;
    if (!make_map_2d(&mx, X, W->K, M, static_cast<uint64_t>(W->K) * 2, B, 128, 2 * B) ||
        !make_map_2d(&my, Y, W->N, M, static_cast<uint64_t>(W->N) * 2, B, 32, 2 * B) ||
        (W->nnz > 0 && !make_block_map(&mw, W->values, B, W->nnz, B / 2)))
        return BSL_ERR_CUDA;
    if (W->nnz == 0) mw = mx;  // no weight block is ever loaded
    const int G = 256 / B;
    PairArgs args;
    args.M = M;
    args.mtiles = (M + 255) / 256;
    args.nseg = W->N / B;
    args.ngroups = (args.nseg + G - 1) / G;
    args.units = args.ngroups * args.mtiles;
    args.seg_ptr = W->row_ptr;
    args.seg_order = W->row_order;
    args.grp_ptr = W->rgrp_ptr;
    args.grp_bptr = W->rgrp_bptr;
    args.grp_ent = W->rgrp_ent;
    args.grp_blk = W->rgrp_blk;
    args.sched = W->sched;
    args.bias = static_cast<const __nv_bfloat16 *>(bias);
    args.status = W->status;
    args.timeout_ns = wait_timeout_ns();
    return B == 64 ? run<64>(mx, my, mw, args, s) : run<32>(mx, my, mw, args, s);
}

}  // namespace bsl

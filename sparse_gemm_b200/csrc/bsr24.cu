// bsr24.cu -- block-sparse weight with the 2:4 pattern inside its blocks, on sm_100a.
//
// The weight keeps only its nonzero b x b blocks (Hugging Face
// pytorch_block_sparse release note, "Block-Sparse Implementation and
// Usage"), and inside every kept block two of every four consecutive
// elements along K are zero: the "50% sparse pattern within blocks" of the
// release note's "Future Development Roadmap" and the "blocks of 2:4" of the
// "Lecture 11: Sparsity" summary (43:51).  Each kept block is stored in the
// compressed form of the torchao sparsity README, Table 4.1 ("NVIDIA 2:4
// compressed representation"): b rows of b/2 kept values plus b/16 16-bit
// position words per row (the layout of bsl_semi24, one block at a time).
//
// k_bsr24_fwd: Y [M][N] = X [M][K] . W^T on the sparse tensor-core MMA, the
// weight as the compressed A operand, driven by the packed weight's row-group
// plan (groups of G = 128/b block rows in longest-first order; one entry per
// block column any member holds, with a member mask).  A tile is one group
// (the 128 TMEM lanes: member m's block rows on lanes m*b .. m*b+b-1) times
// 224 tokens.  Per entry one stage holds the members' compressed blocks (a
// zero block for absent members), the activation tile X[t0:t0+224, c*b:(c+1)*b]
// and the present members' position words, all by TMA.  b = 64: 2 members,
// two K = 32 MMAs of N = 224 per entry, 64-byte weight rows; b = 32: 4
// members, one MMA per entry, 32-byte weight rows (32-byte swizzle).
// Persistent, one CTA per SM; tiles token-tile major, every group (heaviest
// first) inside, taken round robin.
// Roles (16 warps):
//   warp 2      plan: reads each tile's plan 32 entries at a time (lane i
//               entry i: column, member mask, block ids by a warp prefix sum
//               of the member counts) into a 4-chunk shared-memory ring;
//   warps 0, 3  producers (lane 0 each, alternate stages): issue each staged
//               entry's copies into a 5-stage (b = 64) or 8-stage (b = 32)
//               ring and write the entry's member mask in the stage;
//   warp 1      MMA issuer (lane 0), TMEM owner;
//   warps 4-7   metadata: per stage, their 32 TMEM lanes' position words from
//               shared memory into the lane layout of the sparse MMA, written
//               to an 8-stage TMEM ring (one 4-column-aligned column per MMA);
//   warps 8-15  epilogue, two per lane quarter taking alternate 32-token
//               chunks: TMEM -> registers (+ bias) -> bf16, transposed through
//               a 2 KB staging chunk per warp, TMA store at the member's rows.
// TMEM: two 128 x 224 fp32 accumulators (columns 0..447), so a tile's epilogue
// overlaps the next tile's MMAs; the metadata ring from column 448 (8 or 4
// columns per stage for b = 64 or 32).
// Sparse-MMA metadata layout in TMEM (measured on B200, selector 0): for rows
// 16q .. 16q+15, lane 16q + 8kh + i holds the positions of K half kh: bits
// 0-15 for row 16q + i, bits 16-31 for row 16q + 8 + i.
//
// Every wait is bounded (BSL_ERR_TIMEOUT in the status word, then all roles
// leave through an abort flag).
#include "common.cuh"
#include "internal.h"

namespace bsl {
namespace {

__device__ __forceinline__ uint8_t *align1024(uint8_t *p)
{
    return reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

constexpr int kBsr24Tokens = 224;  // tokens per tile (MMA N)

// Shared-memory descriptor layout code of the 32-byte swizzle (the b = 32
// compressed rows are 32 bytes); 64- and 128-byte are kLayoutSw64 / kLayoutSw128.
constexpr uint32_t kLayoutSw32 = 6;

template <int B_>
struct Bsr24Cfg {
    static constexpr int B = B_;                     // block size: 64 or 32
    static constexpr int G = 128 / B;                // block rows per group
    static constexpr int KSTEPS = B / 32;            // K = 32 sparse MMAs per entry
    static constexpr int BT = kBsr24Tokens;
    static constexpr int S = B == 64 ? 5 : 8;        // copy stages, one entry each
    static constexpr int A_ROW = B;                  // bytes of a compressed block row (B/2 bf16)
    static constexpr uint32_t A_LAYOUT = B == 64 ? kLayoutSw64 : kLayoutSw32;
    static constexpr uint32_t X_LAYOUT = B == 64 ? kLayoutSw128 : kLayoutSw64;
    static constexpr int A_BLOCK = B * A_ROW;        // one compressed block
    static constexpr int A_BYTES = G * A_BLOCK;      // 128 rows
    static constexpr int B_BYTES = BT * B * 2;       // 224 rows of B activations
    static constexpr int META_BLOCK = B * (B / 16) * 2;  // one block's position words
    static constexpr int META_OFF = A_BYTES + B_BYTES;
    static constexpr int HDR_OFF = META_OFF + G * META_BLOCK;
    static constexpr int STAGE_BYTES = (HDR_OFF + 16 + 1023) / 1024 * 1024;
    static constexpr int MS = 8;                     // metadata ring stages (TMEM)
    static constexpr int MCOLS = 4 * KSTEPS;         // TMEM columns per metadata stage
    static constexpr int ACC = 2;                    // accumulator buffers
    static constexpr int META_COL = ACC * BT;
    static constexpr int TMEM_COLS = 512;
    static constexpr int EPI_WARPS = 8;
    static constexpr int OUT_CHUNK = 32 * 32 * 2;    // 32 tokens x 32 features bf16
    static constexpr int OUT_BYTES = EPI_WARPS * 2 * OUT_CHUNK;
    static constexpr int W_PROD = 0, W_MMA = 1, W_PLAN = 2, W_PROD2 = 3, W_META = 4, W_EPI = 8;
    static constexpr int P = 2;                      // producer warps (0 and 3), stage g by warp g % P
    static constexpr int THREADS = 16 * 32;
    static constexpr int D = 4;                      // plan chunk ring
    // chunk (ints): [0] entries (-1: no more tiles), [1] first token of the
    // tile, [2 + i] block column of entry i, [34 + i] member mask, [66 + 32m + i]
    // block of member m (nnz: the zero block)
    static constexpr int CHUNK_INTS = 2 + 32 * (2 + G);
    static constexpr int CHUNK_BYTES = (CHUNK_INTS * 4 + 15) / 16 * 16;
    static constexpr int BAR_BYTES = 1024;
    static constexpr int SMEM_BYTES = 1024 + S * STAGE_BYTES + OUT_BYTES + D * CHUNK_BYTES + BAR_BYTES;
    static_assert(META_COL + MCOLS * MS <= TMEM_COLS, "TMEM columns");
    static_assert((2 * S + 2 * MS + 2 * ACC + 2 * D + 1) * 8 + 8 <= BAR_BYTES, "barrier area");
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
    static_assert(B == 64 || B == 32, "block size");
};

struct Bsr24Args {
    int32_t M, R, nnz;
    int32_t ntt;      // token tiles
    int32_t ngroups;  // row groups
    int32_t tiles;    // groups x token tiles
    const int32_t *row_order, *grp_ptr, *grp_bptr, *grp_ent, *grp_blk;
    const __nv_bfloat16 *bias;
    int32_t *status;
    uint64_t timeout_ns;
};

__device__ __forceinline__ void umma_sp_lead(uint32_t leader, uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                             uint32_t meta_tmem, uint32_t idesc, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p, e;\n\t"
        "setp.ne.b32 e, %6, 0;\n\t"
        "setp.ne.b32 p, %5, 0;\n\t"
        "@e tcgen05.mma.sp.cta_group::1.kind::f16 [%0], %1, %2, [%3], %4, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(meta_tmem), "r"(idesc), "r"(accumulate), "r"(leader)
        : "memory");
}

__device__ __forceinline__ void tmem_st1(uint32_t taddr, uint32_t w)
{
    asm volatile("tcgen05.st.sync.aligned.32x32b.x1.b32 [%0], {%1};" ::"r"(taddr), "r"(w) : "memory");
}

__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
}

// Tile t of the launch: token tile t / ngroups, group t % ngroups.  The CTAs
// running at one time work on one or two token tiles across every group, so
// the activations they read (a few MB) and the compressed weight stay in L2.
__device__ __forceinline__ int tile_group(int t, const Bsr24Args &a) { return t % a.ngroups; }
__device__ __forceinline__ int tile_token0(int t, const Bsr24Args &a) { return (t / a.ngroups) * kBsr24Tokens; }

// Entries of tile t's group (0 past the last tile).
__device__ __forceinline__ int tile_entries(int t, const Bsr24Args &a)
{
    if (t >= a.tiles) return 0;
    const int grp = tile_group(t, a);
    return __ldg(a.grp_ptr + grp + 1) - __ldg(a.grp_ptr + grp);
}

// Block row of member m of tile t's group (G members), or -1 (no such member or tile).
__device__ __forceinline__ int tile_block_row(int t, int m, int G, const Bsr24Args &a)
{
    if (t >= a.tiles) return -1;
    const int gi = tile_group(t, a) * G + m;
    return gi < a.R ? __ldg(a.row_order + gi) : -1;
}

template <int B>
__global__ void __launch_bounds__(Bsr24Cfg<B>::THREADS, 1)
    k_bsr24_fwd(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmX,
                const __grid_constant__ CUtensorMap tmY, const uint8_t *__restrict__ meta, const Bsr24Args args)
{
    using C = Bsr24Cfg<B>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *stages = align1024(smem_raw);
    uint8_t *outbuf = stages + C::S * C::STAGE_BYTES;
    int *chunks = reinterpret_cast<int *>(outbuf + C::OUT_BYTES);
    uint64_t *bars = reinterpret_cast<uint64_t *>(reinterpret_cast<uint8_t *>(chunks) + C::D * C::CHUNK_BYTES);
    uint64_t *full = bars;               // stage copies landed
    uint64_t *empty = full + C::S;       // stage MMAs finished
    uint64_t *mfull = empty + C::S;      // metadata of a stage written to TMEM (4 warps)
    uint64_t *mempty = mfull + C::MS;    // metadata read by the stage's MMAs
    uint64_t *afull = mempty + C::MS;    // [ACC] accumulator complete
    uint64_t *aempty = afull + C::ACC;   // [ACC] accumulator read out (8 warps)
    uint64_t *cfull = aempty + C::ACC;   // [D] plan chunk staged
    uint64_t *cempty = cfull + C::D;     // [D] plan chunk issued by the producer
    uint64_t *drain = cempty + C::D;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint64_t tmo = args.timeout_ns;
    dependents_may_launch();

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int s = 0; s < C::MS; ++s) {
            mbar_init(&mfull[s], 4);
            mbar_init(&mempty[s], 1);
        }
        for (int a = 0; a < C::ACC; ++a) {
            mbar_init(&afull[a], 1);
            mbar_init(&aempty[a], C::EPI_WARPS);
        }
        for (int c = 0; c < C::D; ++c) {
            mbar_init(&cfull[c], 1);
            mbar_init(&cempty[c], C::P);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_barrier_init();
        tma_prefetch_map(&tmA);
        tma_prefetch_map(&tmX);
        tma_prefetch_map(&tmY);
    }
    if (warp == C::W_MMA) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    wait_for_prior_grid();  // set-up above touched no global memory

    if (warp == C::W_PLAN) {
        // ------------------------------------------------------------ plan
        // Stages each tile's entries, 32 at a time, for the producer: lane i
        // reads entry e0 + i (column and member mask), a warp prefix sum of
        // the member counts gives its first block's position in grp_blk, and
        // it reads its members' block ids.  The next tile's plan range is
        // read one tile ahead.  Runs up to D chunks ahead of the producer.
        bool ok = true;
        int cc = 0;  // chunks staged
        auto stage_chunk = [&](int n, int t0, int col, uint32_t mask, const int (&blk)[C::G]) {
            const int cs = cc % C::D;
            int good = 1;
            if (lane == 0 && cc >= C::D && !mbar_wait(&cempty[cs], ((cc / C::D) - 1) & 1, tmo, abort_flag))
                good = 0;
            if (!__shfl_sync(0xffffffffu, good, 0)) return false;
            int *ch = chunks + cs * (C::CHUNK_BYTES / 4);
            if (lane == 0) {
                ch[0] = n;
                ch[1] = t0;
            }
            ch[2 + lane] = col;
            ch[34 + lane] = static_cast<int>(mask);
#pragma unroll
            for (int m = 0; m < C::G; ++m) ch[66 + 32 * m + lane] = blk[m];
            __syncwarp();
            if (lane == 0) mbar_arrive(&cfull[cs]);
            ++cc;
            return true;
        };
        int t = blockIdx.x;
        int nb = 0, ne = 0, nbb = 0;  // plan range of tile t
        if (t < args.tiles) {
            const int grp = tile_group(t, args);
            nb = __ldg(args.grp_ptr + grp);
            ne = __ldg(args.grp_ptr + grp + 1);
            nbb = __ldg(args.grp_bptr + grp);
        }
        for (; ok && t < args.tiles; t += gridDim.x) {
            const int t0 = tile_token0(t, args);
            const int e_beg = nb, e_end = ne;
            int bbase = nbb;
            const int tn = t + static_cast<int>(gridDim.x);
            if (tn < args.tiles) {  // the next tile's range, used one tile later
                const int grp = tile_group(tn, args);
                nb = __ldg(args.grp_ptr + grp);
                ne = __ldg(args.grp_ptr + grp + 1);
                nbb = __ldg(args.grp_bptr + grp);
            }
            for (int e0 = e_beg; ok && e0 < e_end; e0 += 32) {
                const int e = e0 + lane;
                int col = 0;
                uint32_t mask = 0;
                if (e < e_end) {
                    const int ent = __ldg(args.grp_ent + e);
                    col = ent & 0xFFFFFF;
                    mask = static_cast<uint32_t>(ent) >> 24;
                }
                const int cnt = __popc(mask);
                int incl = cnt;
#pragma unroll
                for (int d = 1; d < 32; d <<= 1) {
                    const int v = __shfl_up_sync(0xffffffffu, incl, d);
                    if (lane >= d) incl += v;
                }
                const int first = bbase + incl - cnt;  // grp_blk position of the entry's first block
                bbase += __shfl_sync(0xffffffffu, incl, 31);
                int blk[C::G];
#pragma unroll
                for (int m = 0; m < C::G; ++m)
                    blk[m] = ((mask >> m) & 1u) ? __ldg(args.grp_blk + first + __popc(mask & ((1u << m) - 1u)))
                                                : args.nnz;  // the zero block
                const int n = e_end - e0 < 32 ? e_end - e0 : 32;
                if (!stage_chunk(n, t0, col, mask, blk)) ok = false;
            }
        }
        if (ok) {
            int none[C::G];
#pragma unroll
            for (int m = 0; m < C::G; ++m) none[m] = 0;
            if (!stage_chunk(-1, 0, 0, 0u, none)) ok = false;
        }
        if (lane == 0 && !ok) {
            *abort_flag = 1;
            set_status(args.status, BSL_ERR_TIMEOUT);
        }
        __syncwarp();
    } else if (warp == C::W_PROD || warp == C::W_PROD2) {
        // ------------------------------------------------------------ producers
        // Two warps walk the staged entries; lane 0 of warp p issues the
        // copies of the stages g with g % P == p (one thread issues only so
        // many copies per microsecond): the members' compressed blocks, the
        // activation tile and the present members' position words, and the
        // member mask into the stage.
        const int p = warp == C::W_PROD ? 0 : 1;
        if (lane == 0) {
            bool ok = true;
            int g = 0;  // stages issued
            for (int cc = 0; ok; ++cc) {
                const int cs = cc % C::D;
                if (!mbar_wait(&cfull[cs], (cc / C::D) & 1, tmo, abort_flag)) {
                    ok = false;
                    break;
                }
                const volatile int *ch = chunks + cs * (C::CHUNK_BYTES / 4);
                const int n = ch[0];
                if (n < 0) break;
                const int t0 = ch[1];
                for (int j = 0; j < n; ++j, ++g) {
                    if (g % C::P != p) continue;
                    const int cj = ch[2 + j];
                    const uint32_t mj = static_cast<uint32_t>(ch[34 + j]);
                    const int slot = g % C::S;
                    if (g >= C::S && !mbar_wait(&empty[slot], ((g / C::S) - 1) & 1, tmo, abort_flag)) {
                        ok = false;
                        break;
                    }
                    uint8_t *st = stages + slot * C::STAGE_BYTES;
                    *reinterpret_cast<volatile uint32_t *>(st + C::HDR_OFF) = mj;
                    mbar_arrive_expect_tx(&full[slot], C::A_BYTES + C::B_BYTES + __popc(mj) * C::META_BLOCK);
#pragma unroll
                    for (int m = 0; m < C::G; ++m) {
                        const int bj = ch[66 + 32 * m + j];
                        tma_load_3d(st + m * C::A_BLOCK, &tmA, &full[slot], 0, 0, bj);
                        if ((mj >> m) & 1u)
                            bulk_load(st + C::META_OFF + m * C::META_BLOCK,
                                      meta + static_cast<size_t>(bj) * C::META_BLOCK, C::META_BLOCK, &full[slot]);
                    }
                    tma_load_2d(st + C::A_BYTES, &tmX, &full[slot], cj * C::B, t0);
                }
                mbar_arrive(&cempty[cs]);  // the chunk is read
            }
            if (!ok) {
                *abort_flag = 1;
                set_status(args.status, BSL_ERR_TIMEOUT);
            }
            // every copy lands before the CTA's shared memory is released (the
            // last fill of a slot, by either warp, is the newest phase of its
            // barrier; an aborted run may wait on an older phase, which the
            // bounded wait ends)
            for (int s = 0; s < C::S && s < g; ++s) {
                const int fills = (g - s + C::S - 1) / C::S;
                if (!mbar_wait(&full[s], (fills - 1) & 1, tmo, nullptr)) set_status(args.status, BSL_ERR_TIMEOUT);
            }
        }
        __syncwarp();
    } else if (warp == C::W_MMA) {
        // ------------------------------------------------------------ MMA issuer
        const uint32_t idesc = make_idesc_bf16(128, C::BT, false, false) | (1u << 2);  // bit 2: sparse
        const uint32_t lead = lane == 0;
        bool ok = true, any = false;
        int g = 0, it = 0;
        int nent_next = tile_entries(blockIdx.x, args);
        for (int t = blockIdx.x; ok && t < args.tiles; t += gridDim.x, ++it) {
            const int nent = nent_next;
            nent_next = tile_entries(t + gridDim.x, args);  // used one tile later
            const int acc = it & 1;
            if (it >= C::ACC &&
                __any_sync(0xffffffffu, !mbar_wait(&aempty[acc], ((it / C::ACC) - 1) & 1, tmo, abort_flag))) {
                ok = false;
                break;
            }
            tc_fence_after();
            for (int k = 0; k < nent; ++k, ++g) {
                const int slot = g % C::S, ms = g % C::MS;
                if (__any_sync(0xffffffffu, !mbar_wait(&full[slot], (g / C::S) & 1, tmo, abort_flag) ||
                                                !mbar_wait(&mfull[ms], (g / C::MS) & 1, tmo, abort_flag))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t a_base = smem_u32(stages + slot * C::STAGE_BYTES);
                const uint32_t b_base = a_base + C::A_BYTES;
#pragma unroll
                for (int j = 0; j < C::KSTEPS; ++j) {
                    const uint64_t ad = make_sdesc(a_base + j * 32, 16, 8 * C::A_ROW, C::A_LAYOUT);
                    const uint64_t bd = make_sdesc(b_base + j * 64, 16, 8 * 2 * C::B, C::X_LAYOUT);
                    umma_sp_lead(lead, tmem + acc * C::BT, ad, bd, tmem + C::META_COL + ms * C::MCOLS + j * 4,
                                 idesc, (k | j) != 0);
                }
                umma_commit_lead(lead, &empty[slot]);
                umma_commit_lead(lead, &mempty[ms]);
                any = true;
                __syncwarp();
            }
            if (!ok) break;
            if (nent > 0) umma_commit_lead(lead, &afull[acc]);
            else if (lane == 0) mbar_arrive(&afull[acc]);  // nothing to wait for: the tile is zeros
            __syncwarp();
        }
        if (lane == 0 && !ok) {
            *abort_flag = 1;
            set_status(args.status, BSL_ERR_TIMEOUT);
        }
        if (any) {  // every MMA is complete before TMEM is freed
            umma_commit_lead(lead, drain);
            if (lane == 0 && !mbar_wait(drain, 0, tmo, nullptr)) set_status(args.status, BSL_ERR_TIMEOUT);
        }
        __syncwarp();
    } else if (warp >= C::W_META && warp < C::W_META + 4) {
        // ------------------------------------------------------------ metadata
        // Warp q covers TMEM lanes 32q .. 32q+31: member m = 32q / b, rows
        // 32q % b .. +31 of its block.  Lane l reads its row's b/8 bytes of
        // position words (one 32-bit word per K = 32 step of the entry), then
        // takes the 16-bit halves its TMEM lane holds from lanes src_lo / src_hi.
        const int q = warp & 3, m = (32 * q) / B;
        const int row = (32 * q) % B + lane;
        const int src_lo = (lane & 16) | (lane & 7), src_hi = src_lo + 8;
        const bool upper = (lane >> 3) & 1;
        constexpr uint32_t pad = 0x44444444u;  // absent member: pairs (0, 1) over zeros
        bool ok = true;
        int g = 0;
        int nent_next = tile_entries(blockIdx.x, args);
        for (int t = blockIdx.x; ok && t < args.tiles; t += gridDim.x) {
            const int nent = nent_next;
            nent_next = tile_entries(t + gridDim.x, args);
            for (int k = 0; k < nent; ++k, ++g) {
                const int slot = g % C::S, ms = g % C::MS;
                if (__any_sync(0xffffffffu, !mbar_wait(&full[slot], (g / C::S) & 1, tmo, abort_flag))) {
                    ok = false;
                    break;
                }
                const uint8_t *st = stages + slot * C::STAGE_BYTES;
                const uint32_t mj = *reinterpret_cast<const volatile uint32_t *>(st + C::HDR_OFF);
                const uint32_t *src =
                    reinterpret_cast<const uint32_t *>(st + C::META_OFF + m * C::META_BLOCK + row * (B / 8));
                const bool present = (mj >> m) & 1u;
                uint32_t w[C::KSTEPS];
#pragma unroll
                for (int j = 0; j < C::KSTEPS; ++j) {
                    const uint32_t x = present ? src[j] : pad;
                    const uint32_t lo = __shfl_sync(0xffffffffu, x, src_lo);
                    const uint32_t hi = __shfl_sync(0xffffffffu, x, src_hi);
                    w[j] = (upper ? lo >> 16 : lo & 0xFFFFu) | (upper ? hi & 0xFFFF0000u : hi << 16);
                }
                if (g >= C::MS &&
                    __any_sync(0xffffffffu, !mbar_wait(&mempty[ms], ((g / C::MS) - 1) & 1, tmo, abort_flag))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t taddr = tmem + (static_cast<uint32_t>(32 * q) << 16) + C::META_COL + ms * C::MCOLS;
#pragma unroll
                for (int j = 0; j < C::KSTEPS; ++j) tmem_st1(taddr + 4 * j, w[j]);
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&mfull[ms]);
            }
        }
        if (lane == 0 && !ok) {
            *abort_flag = 1;
            set_status(args.status, BSL_ERR_TIMEOUT);
        }
        __syncwarp();
    } else if (warp >= C::W_EPI) {
        // ------------------------------------------------------------ epilogue
        // Warp e reads TMEM lanes 32q .. 32q+31 (member q / 2, block rows
        // 32(q % 2) ..), 32-token chunks c = e / 4, e / 4 + 2, ...; neighbouring
        // lanes swap values so each writes one 32-bit word (two features of
        // one token) into its [32 tokens][32 features] staging chunk.
        const int e = warp - C::W_EPI, q = warp & 3, half = e >> 2;
        uint8_t *wbuf = outbuf + e * 2 * C::OUT_CHUNK;
        const bool odd = lane & 1;
        bool ok = true;
        int it = 0, ob = 0;
        int nent_next = tile_entries(blockIdx.x, args);
        int row_next = tile_block_row(blockIdx.x, (32 * q) / B, C::G, args);
        for (int t = blockIdx.x; ok && t < args.tiles; t += gridDim.x, ++it) {
            const int t0 = tile_token0(t, args);
            const int nent = nent_next, brow = row_next;
            nent_next = tile_entries(t + gridDim.x, args);  // used one tile later
            row_next = tile_block_row(t + gridDim.x, (32 * q) / B, C::G, args);
            const int acc = it & 1;
            const bool member = brow >= 0;
            const int f0 = member ? brow * C::B + (32 * q) % B : 0;
            const float bv = (args.bias && member) ? __bfloat162float(args.bias[f0 + lane]) : 0.f;
            const int left = args.M - t0;
            const int nch = left >= C::BT ? C::BT / 32 : (left + 31) / 32;
            if (__any_sync(0xffffffffu, !mbar_wait(&afull[acc], (it / C::ACC) & 1, tmo, abort_flag))) {
                ok = false;
                break;
            }
            tc_fence_after();
            int last = -1;  // this warp's last chunk
            for (int c = half; c < nch; c += 2) last = c;
            if (last < 0) {  // no chunk for this warp: release at once
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&aempty[acc]);
            }
            for (int c = half; c < nch; c += 2) {
                uint32_t v[32];
                if (nent > 0) {
                    tmem_ld32(tmem + (static_cast<uint32_t>(32 * q) << 16) + acc * C::BT + c * 32, v);
                    tmem_wait_ld();
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) v[i] = 0u;
                }
                if (c == last) {  // this warp's last TMEM read of the tile
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&aempty[acc]);
                }
                if (!member) continue;
                if (lane == 0) bulk_wait_group_read<1>();  // staging chunk `ob` was read out
                __syncwarp();
                uint8_t *dst = wbuf + ob * C::OUT_CHUNK;
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                    const float a = __uint_as_float(v[2 * u]) + bv, b = __uint_as_float(v[2 * u + 1]) + bv;
                    const float other = __shfl_xor_sync(0xffffffffu, odd ? a : b, 1);
                    const uint32_t word = odd ? pack_bf16x2(other, b) : pack_bf16x2(a, other);
                    *reinterpret_cast<uint32_t *>(dst + (2 * u + odd) * 64 + (lane & ~1) * 2) = word;
                }
                fence_async_smem();
                __syncwarp();
                if (lane == 0) {
                    tma_store_2d(&tmY, dst, f0, t0 + 32 * c);
                    bulk_commit_group();
                }
                ob ^= 1;
            }
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
    if (warp == C::W_MMA) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

// Compressed blocks [nnz + 1][b][b/2] bf16 (the last one zero) as a 3-D map:
// x = kept value in a row, y = row in the block, z = block; the rows are b
// bytes, swizzled over b bytes.
bool make_block24_map(CUtensorMap *map, const void *values, int32_t b, int32_t nblocks)
{
    return make_map_3d(map, values, static_cast<uint64_t>(b) / 2, static_cast<uint64_t>(b),
                       static_cast<uint64_t>(nblocks), static_cast<uint64_t>(b),
                       static_cast<uint64_t>(b) * b, static_cast<uint32_t>(b) / 2, static_cast<uint32_t>(b), b);
}

}  // namespace

bsl_status launch_bsr24_compress(const bsl_bsr *W, void *values24, uint16_t *meta24, cudaStream_t s)
{
    // the kept blocks, viewed as nnz*b rows of b elements, compressed like a
    // 2:4 weight of K = b; then one zero block after them
    const size_t block_bytes = static_cast<size_t>(W->b) * (W->b / 2) * 2;
    if (W->nnz > 0) {
        bsl_semi24 view;
        view.N = W->nnz * W->b;
        view.K = W->b;
        view.values = values24;
        view.meta = meta24;
        view.status = W->status;
        const bsl_status st = launch_compress24(W->values, &view, s);
        if (st != BSL_OK) return st;
    }
    return cuda_status(cudaMemsetAsync(static_cast<uint8_t *>(values24) + W->nnz * block_bytes, 0, block_bytes, s));
}

namespace {

template <int B>
bsl_status run_bsr24(const void *X, int32_t M, const bsl_bsr *W, const void *values24, const uint16_t *meta24,
                     const void *bias, void *Y, cudaStream_t s)
{
    using C = Bsr24Cfg<B>;
    CUtensorMap ma, mx, my;
    if (!make_block24_map(&ma, values24, B, W->nnz + 1) ||
        !make_map_2d(&mx, X, W->K, M, static_cast<uint64_t>(W->K) * 2, B, C::BT, 2 * B) ||
        !make_map_2d(&my, Y, W->N, M, static_cast<uint64_t>(W->N) * 2, 32, 32, 0))
        return BSL_ERR_CUDA;
    Bsr24Args args;
    args.M = M;
    args.R = W->N / B;
    args.nnz = W->nnz;
    args.ntt = (M + C::BT - 1) / C::BT;
    args.ngroups = (args.R + C::G - 1) / C::G;
    const int64_t tiles = static_cast<int64_t>(args.ngroups) * args.ntt;
    if (tiles > 0x7FFFFFFF) return BSL_ERR_UNSUPPORTED;
    args.tiles = static_cast<int32_t>(tiles);
    args.row_order = W->row_order;
    args.grp_ptr = W->rgrp_ptr;
    args.grp_bptr = W->rgrp_bptr;
    args.grp_ent = W->rgrp_ent;
    args.grp_blk = W->rgrp_blk;
    args.bias = static_cast<const __nv_bfloat16 *>(bias);
    args.status = W->status;
    args.timeout_ns = wait_timeout_ns();
    auto kern = k_bsr24_fwd<B>;
    const bsl_status sa = set_smem_once(reinterpret_cast<const void *>(kern), C::SMEM_BYTES);
    if (sa != BSL_OK) return sa;
    const int grid = args.tiles < num_sms() ? args.tiles : num_sms();
    return cuda_status(launch_dependent(kern, grid, C::THREADS, C::SMEM_BYTES, s, ma, mx, my,
                                        reinterpret_cast<const uint8_t *>(meta24), args));
}

}  // namespace

bsl_status launch_bsr24_fwd(const void *X, int32_t M, const bsl_bsr *W, const void *values24,
                            const uint16_t *meta24, const void *bias, void *Y, cudaStream_t s)
{
    if (W->b == 64) return run_bsr24<64>(X, M, W, values24, meta24, bias, Y, s);
    if (W->b == 32) return run_bsr24<32>(X, M, W, values24, meta24, bias, Y, s);
    return BSL_ERR_UNSUPPORTED;
}

}  // namespace bsl

// stream_fwd.cu -- small-M forward by streaming the packed weight once.
//
// For a handful of tokens the forward is bound by reading the weight, not by
// arithmetic.  The lecture summary "Lecture 11: Sparsity" (48:12, "load and
// sparse expand") describes the remedy: read the compressed form, expand it
// on chip, multiply densely.  Here the compressed form is the packed BSR
// blocks, which are already dense b x b tiles, so "expanding" is placing them
// in shared memory next to the activation slice they multiply.
//
// Decomposition: the BSR block list [0, nnz) is cut into contiguous ranges,
// one per CTA of a one-CTA-per-SM grid: equal shares, each moved to a
// nearby block-row start where there is one, the starts chosen to make the
// largest range as small as they can (the pack computes these bounds), so
// block rows of up to a CTA's share never straddle two CTAs and only longer
// ones do.  Each CTA's range is cut into equal shares for its 8
// warps (block counts, not block rows, are balanced).
// Each warp streams its share through its own ring of slots; a slot holds one
// weight block and the activation slice X[0:MP, c*b:(c+1)*b] it multiplies,
// both brought in by TMA (swizzled rows, rows past M read as zeros).  The
// weight copies, which depend on nothing, leave first; each slot is refilled
// as soon as it is read, with a few slots per warp (enough to keep DRAM
// busy).  The operands go to registers with ldmatrix; mma.sync m16n8k16
// (bf16 in, fp32 accumulate) forms Y^T[n][m] = W_blk[n][:] . X[m][:], and
// the sum of the current block row stays in registers:
//   - a block row entirely inside the warp's share is finished there: bias
//     added, rounded to bf16, staged in shared memory, written to Y with
//     16-byte stores;
//   - a block row cut by share boundaries leaves an fp32 partial.  After all
//     warps of the CTA are done, the partials sit in their rings and the
//     CTA's first contributor to each cut row adds them in warp order.  A row
//     that lies inside the CTA's range is then written; a (long) row that
//     reaches into other CTAs' ranges leaves the CTA's sum in the workspace,
//     and the last CTA to count itself in on the row's counter adds the CTAs'
//     sums in CTA order and writes the row.
// Every sum has a fixed order (the same whoever arrives last), so results
// are identical run to run.  Block rows without blocks are written (bias or
// zeros) at the end.  The last CTA to count itself in on a row's counter
// sets it back to zero, and a warp that gave up waiting still counts itself
// in, so every call leaves the counters at zero: the workspace is zeroed once
// when it is allocated and no memset precedes the kernel.
#include "common.cuh"
#include "internal.h"

namespace bsl {
namespace {

constexpr int kStreamWarps = 8;
// Copy bytes a warp keeps in flight, at most (two slots at least): 96 KB per
// SM already covers the DRAM bandwidth-delay product (~6.5 TB/s x ~2 us over
// 148 SMs); more only queues in the memory system and takes shared memory
// from L1 (decode forward, 3 KB slots: 8 per warp 12.7 us, 4 per warp 11.0 us).
constexpr int kWarpInFlight = 12 * 1024;

template <int B, int MP>
struct StreamCfg {
    static constexpr int ROW_BYTES = B * 2;
    static constexpr int W_BLK = B * ROW_BYTES;        // one weight block
    static constexpr int X_BLK = MP * ROW_BYTES;       // its activation slice (MP x b)
    static constexpr int SLOT = W_BLK + X_BLK;
    static constexpr int NSLOT = kWarpInFlight / SLOT > 2 ? kWarpInFlight / SLOT : 2;
    static constexpr int WARP_BYTES = NSLOT * SLOT;
    static constexpr int OUT_BYTES = MP * ROW_BYTES;   // per-warp bf16 staging of one block row
    static constexpr int PART = B * MP;                // floats of one partial
    static constexpr int SMEM_BYTES =
        kStreamWarps * (WARP_BYTES + OUT_BYTES) + kStreamWarps * NSLOT * 8 + 1024;
    static_assert(NSLOT >= 2, "ring too small");
    static_assert(SLOT % 1024 == 0 && W_BLK % 1024 == 0, "slot alignment for the swizzled copies");
    static_assert(2 * PART * 4 <= WARP_BYTES, "a warp's two partials fit in its ring");
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

struct StreamArgs {
    __nv_bfloat16 *Y;
    float *ws;                  // [CTAs][2][b*MP] partial sums of rows cut between CTAs
    int32_t *cnt;               // [CTAs] arrival counters (zero between calls)
    const int32_t *row_ptr, *col_idx;
    const int32_t *sbounds;     // CTA ranges made by the pack ([0] = their CTA count)
    const __nv_bfloat16 *bias;  // [N] added to every output row (null: none)
    int32_t M, N, K, R, C, nnz;
    int32_t *status;
    uint64_t timeout_ns;
};

__device__ __forceinline__ uint8_t *align1024(uint8_t *p)
{
    return reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// first block of share u when nnz blocks are split over U shares
// floor(x / d) for 0 <= x < 2^63, 0 < d < 2^31, in 32-bit arithmetic when x
// fits (the usual case: a 64-bit division is a long emulated sequence)
__device__ __forceinline__ int floor_div(uint64_t x, int d)
{
    if (x <= 0xFFFFFFFFull) return static_cast<int>(static_cast<uint32_t>(x) / static_cast<uint32_t>(d));
    return static_cast<int>(x / static_cast<uint64_t>(d));
}

__device__ __forceinline__ int share_begin(int u, int U, int nnz)
{
    return floor_div(static_cast<uint64_t>(u) * static_cast<uint32_t>(nnz), U);
}

// Count the caller in and return the new count.  Release: the caller's
// earlier writes are visible before the new count; acquire: the caller's
// later reads see what the earlier arrivers released.
__device__ __forceinline__ int arrive_count(int32_t *p)
{
    int old;
    asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], 1;" : "=r"(old) : "l"(p) : "memory");
    return old + 1;
}

// the share that holds block p (the last u with share_begin(u) <= p);
// share_begin(u) = floor(u * nnz / U), so u is within one of floor(p * U / nnz)
__device__ __forceinline__ int share_of(int p, int U, int nnz)
{
    int u = floor_div(static_cast<uint64_t>(p) * static_cast<uint32_t>(U), nnz);
    u = u < 0 ? 0 : (u > U - 1 ? U - 1 : u);
    while (u > 0 && share_begin(u, U, nnz) > p) --u;
    while (u + 1 < U && share_begin(u + 1, U, nnz) <= p) ++u;
    return u;
}

// The block row holding block p (0 <= p < nnz): the last r with
// row_ptr[r] <= p, by a warp-parallel search (two or three rounds of one
// load per lane).
__device__ __forceinline__ int row_holding(const StreamArgs &a, int p, int lane)
{
    int lo = 0, hi = a.R;  // row_ptr[lo] <= p < row_ptr[hi]
    while (hi - lo > 1) {
        const int step = (hi - lo + 31) / 32;
        const int probe = lo + lane * step;
        const bool le = probe < hi && a.row_ptr[probe] <= p;
        const int last = 31 - __clz(__ballot_sync(0xffffffffu, le));  // lane 0 always qualifies
        lo = lo + last * step;
        hi = min(hi, lo + step);
    }
    return lo;
}

// First block of CTA c (0 <= c <= U): the pack's bounds when they were made
// for this grid size, else the equal share.
__device__ __forceinline__ int cta_bound(const StreamArgs &a, bool snapped, int c, int U)
{
    return snapped ? __ldg(a.sbounds + 1 + c) : share_begin(c, U, a.nnz);
}

// First block of warp w (0 <= w <= kStreamWarps) of a CTA whose range starts
// at cq0 and holds n blocks.
__device__ __forceinline__ int warp_bound(int w, int cq0, int n)
{
    return cq0 + static_cast<int>((static_cast<int64_t>(w) * n) / kStreamWarps);
}

// The warp of the CTA whose share holds block p (cq0 <= p < cq0 + n).
__device__ __forceinline__ int warp_of(int p, int cq0, int n)
{
    int u = floor_div(static_cast<uint64_t>(p - cq0) * kStreamWarps, n);
    u = u > kStreamWarps - 1 ? kStreamWarps - 1 : u;
    while (u > 0 && warp_bound(u, cq0, n) > p) --u;
    while (u + 1 < kStreamWarps && warp_bound(u + 1, cq0, n) <= p) ++u;
    return u;
}

// The CTA whose range holds block p (0 <= p < nnz); warp-collective.  A
// bound made by the pack lies within q = floor(nnz / (2U)) blocks of its equal
// share and equal shares are at least 2q apart (more than q between a share's
// bound and the next share's), so the CTA is the equal share's CTA or one of
// its two neighbours: lanes 0..3 look at the bounds of those three in one
// round of loads.
__device__ __forceinline__ int cta_of(const StreamArgs &a, bool snapped, int p, int U, int lane)
{
    const int c = share_of(p, U, a.nnz);
    if (!snapped) return c;
    const int k = c - 1 + lane;
    const int v = lane < 4 && k >= 0 && k <= U ? __ldg(a.sbounds + 1 + k) : 0;
    const int vn = __shfl_down_sync(0xffffffffu, v, 1);
    const unsigned m = __ballot_sync(0xffffffffu, lane < 3 && k >= 0 && k < U && v <= p && p < vn);
    return m ? c - 1 + (__ffs(m) - 1) : c;
}

template <int B>
__device__ __forceinline__ int swz_chunk(int chunk, int row)
{
    if constexpr (B == 64) return chunk ^ (row & 7);
    else return chunk ^ ((row >> 1) & 3);
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

template <int B, int MP>
struct RowAcc {
    static constexpr int MT = B / 16;   // 16-row tiles of the block (output features)
    static constexpr int NT = MP / 8;   // 8-token tiles
    float d[MT][NT][4];
    __device__ __forceinline__ void zero()
    {
#pragma unroll
        for (int i = 0; i < MT; ++i)
#pragma unroll
            for (int j = 0; j < NT; ++j)
#pragma unroll
                for (int e = 0; e < 4; ++e) d[i][j][e] = 0.f;
    }
    // add a block row stored as floats by store() (element (n, m) at n * MP + m);
    // cg: read through L2 only (another CTA wrote it)
    template <bool CG = false>
    __device__ __forceinline__ void add(const float *src, int lane)
    {
        const int g = lane >> 2, c2 = (lane & 3) * 2;
#pragma unroll
        for (int i = 0; i < MT; ++i)
#pragma unroll
            for (int j = 0; j < NT; ++j)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const float2 *p = reinterpret_cast<const float2 *>(src + (i * 16 + g + h * 8) * MP + j * 8 + c2);
                    const float2 v = CG ? __ldcg(p) : *p;
                    d[i][j][2 * h] += v.x;
                    d[i][j][2 * h + 1] += v.y;
                }
    }
    // store as floats, element (feature n, token m) at n * MP + m
    __device__ __forceinline__ void store(float *dst, int lane) const
    {
        const int g = lane >> 2, c2 = (lane & 3) * 2;
#pragma unroll
        for (int i = 0; i < MT; ++i)
#pragma unroll
            for (int j = 0; j < NT; ++j)
#pragma unroll
                for (int h = 0; h < 2; ++h)
                    *reinterpret_cast<float2 *>(dst + (i * 16 + g + h * 8) * MP + j * 8 + c2) =
                        make_float2(d[i][j][2 * h], d[i][j][2 * h + 1]);
    }
};

__device__ __forceinline__ float bias_of(const StreamArgs &a, int64_t col)
{
    return a.bias ? __bfloat162float(a.bias[col]) : 0.f;
}

// Write M rows of block row r from the warp's bf16 staging ([MP][b]) with
// 16-byte stores.
template <int B, int MP>
__device__ __forceinline__ void store_staged(const StreamArgs &a, const uint8_t *stage, int r, int lane)
{
    constexpr int CPR = B / 8;  // 16-byte chunks per row
    __syncwarp();
    for (int idx = lane; idx < a.M * CPR; idx += 32) {
        const int m = idx / CPR, ch = idx - m * CPR;
        const uint4 v = *reinterpret_cast<const uint4 *>(stage + m * (2 * B) + ch * 16);
        *reinterpret_cast<uint4 *>(a.Y + static_cast<int64_t>(m) * a.N + static_cast<int64_t>(r) * B + ch * 8) = v;
    }
    __syncwarp();
}

// A whole block row held in registers: bias, bf16, staged, stored.
template <int B, int MP>
__device__ __forceinline__ void write_row(const RowAcc<B, MP> &acc, const StreamArgs &a, int r, uint8_t *stage,
                                          int lane)
{
    const int g = lane >> 2, c2 = (lane & 3) * 2;
    __nv_bfloat16 *s = reinterpret_cast<__nv_bfloat16 *>(stage);
#pragma unroll
    for (int i = 0; i < RowAcc<B, MP>::MT; ++i)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int n = i * 16 + g + h * 8;
            const float bb = bias_of(a, static_cast<int64_t>(r) * B + n);
#pragma unroll
            for (int j = 0; j < RowAcc<B, MP>::NT; ++j) {
                const int m = j * 8 + c2;
                s[m * B + n] = __float2bfloat16_rn(acc.d[i][j][2 * h] + bb);
                s[(m + 1) * B + n] = __float2bfloat16_rn(acc.d[i][j][2 * h + 1] + bb);
            }
        }
    store_staged<B, MP>(a, stage, r, lane);
}

template <int B, int MP>
__global__ void __launch_bounds__(kStreamWarps * 32, 1)
    k_stream_fwd(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                 const StreamArgs a)
{
    using Cfg = StreamCfg<B, MP>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align1024(smem_raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint8_t *ring = smem + warp * Cfg::WARP_BYTES;
    uint8_t *stage = smem + kStreamWarps * Cfg::WARP_BYTES + warp * Cfg::OUT_BYTES;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kStreamWarps * (Cfg::WARP_BYTES + Cfg::OUT_BYTES)) +
                     warp * Cfg::NSLOT;

    dependents_may_launch();
    wait_for_prior_grid();  // every step below reads or writes global memory
    const int U = gridDim.x;
    const int GW = U * kStreamWarps;
    const int gw = blockIdx.x * kStreamWarps + warp;
    // whether block row gw is empty (written at the end, bias or zeros): the
    // load leaves now rather than after the share is streamed
    const bool gw_empty = gw < a.R && a.row_ptr[gw + 1] == a.row_ptr[gw];
    // this CTA's blocks [cq0, cq1): the pack's bounds made for this grid size
    // (the three loads go out together), else equal shares
    bool snapped = false;
    int cq0, cq1;
    {
        const bool fits = U <= BSL_SBOUNDS_LEN - 2;
        const int s0 = fits ? __ldg(a.sbounds) : 0;
        const int b0 = fits ? __ldg(a.sbounds + 1 + blockIdx.x) : 0;
        const int b1 = fits ? __ldg(a.sbounds + 2 + blockIdx.x) : 0;
        snapped = s0 == U;
        cq0 = snapped ? b0 : share_begin(blockIdx.x, U, a.nnz);
        cq1 = snapped ? b1 : share_begin(blockIdx.x + 1, U, a.nnz);
    }
    const int cn = cq1 - cq0;
    const int q0 = warp_bound(warp, cq0, cn), q1 = warp_bound(warp + 1, cq0, cn);
    const int nblk = q1 > q0 ? q1 - q0 : 0;
    const int nfirst = nblk < Cfg::NSLOT ? nblk : Cfg::NSLOT;
    if (threadIdx.x == 0) {
        tma_prefetch_map(&tmW);
        tma_prefetch_map(&tmX);
    }
    // block columns of the share's first 32 blocks, one per lane: the load is
    // in flight while the weight copies are issued
    int cidx = q0 + lane < q1 ? a.col_idx[q0 + lane] : 0;

    // the weight blocks depend on nothing: their copies go out first, each
    // slot armed for its block and activation slice together
    if (lane == 0 && nblk > 0) {
        for (int s = 0; s < Cfg::NSLOT; ++s) mbar_init(&bars[s], 1);
        fence_barrier_init();
        for (int t = 0; t < nfirst; ++t) {
            mbar_arrive_expect_tx(&bars[t], Cfg::SLOT);
            tma_load_2d(ring + t * Cfg::SLOT, &tmW, &bars[t], 0, (q0 + t) * B);
        }
    }
    __syncwarp();

    RowAcc<B, MP> acc, part0;  // the current row; the share's first row when it is cut
    acc.zero();
    part0.zero();
    int first_row = 0, last_row = -1;  // rows of blocks q0 and q1 - 1
    int fr_beg = 0, fr_end = 0, lr_beg = 0, lr_end = 0;  // their block ranges
    bool cut_first = false, cut_last = false, ok = true;
    int issued = nfirst;

    if (nblk > 0) {
        // block columns of 32 consecutive blocks of the share, one per lane
        int cbase = q0;
        auto col_of = [&](int p) {  // warp-uniform p; refreshes the lane cache when p leaves it
            if (p >= cbase + 32) {
                cbase = p;
                cidx = p + lane < q1 ? a.col_idx[p + lane] : 0;
            }
            const int c = __shfl_sync(0xffffffffu, cidx, p - cbase);
            return c >= 0 && c < a.C ? c : 0;  // a column outside the weight (bad index) reads column 0
        };
        // the activation slices of the first blocks, once their columns are known
        for (int t = 0; t < nfirst; ++t) {
            const int c = col_of(q0 + t);
            if (lane == 0) tma_load_2d(ring + t * Cfg::SLOT + Cfg::W_BLK, &tmX, &bars[t], c * B, 0);
        }

        first_row = row_holding(a, q0, lane);
        int r = first_row;
        int rbase = r;
        int rp = rbase + 1 + lane <= a.R ? a.row_ptr[rbase + 1 + lane] : 0x7fffffff;
        int row_end = __shfl_sync(0xffffffffu, rp, 0);
        int row_beg = a.row_ptr[first_row];
        fr_beg = row_beg;
        fr_end = row_end;
        cut_first = row_beg < q0;
        bool have = false;
        constexpr int KK = B / 16;

        for (int t = 0; t < nblk; ++t) {
            const int p = q0 + t;
            while (p >= row_end) {  // leaving block row r (which ended inside the share)
                if (have) {
                    if (r == first_row && cut_first) part0 = acc;
                    else write_row<B, MP>(acc, a, r, stage, lane);
                    acc.zero();
                    have = false;
                }
                ++r;
                row_beg = row_end;
                if (r - rbase >= 32) {  // refresh the lane cache of row ends
                    rbase = r;
                    rp = rbase + 1 + lane <= a.R ? a.row_ptr[rbase + 1 + lane] : 0x7fffffff;
                }
                row_end = __shfl_sync(0xffffffffu, rp, r - rbase);
            }
            const int s = t % Cfg::NSLOT;
            const bool landed = mbar_wait(&bars[s], (t / Cfg::NSLOT) & 1, a.timeout_ns, nullptr);
            if (!__all_sync(0xffffffffu, landed)) {  // uniform decision across the warp
                ok = false;
                break;
            }
            have = true;
            const uint32_t wbase = smem_u32(ring + s * Cfg::SLOT);
            const uint32_t xbase = wbase + Cfg::W_BLK;
#pragma unroll
            for (int kk = 0; kk < KK; ++kk) {
                // activation fragments of this k step: two 8-token tiles per ldmatrix.x4
                uint32_t xb[RowAcc<B, MP>::NT][2];
#pragma unroll
                for (int j = 0; j < RowAcc<B, MP>::NT; j += 2) {
                    const int tok = (j + (lane >> 4)) * 8 + (lane & 7);
                    const int chunk = kk * 2 + ((lane >> 3) & 1);
                    ldmatrix_x4(xbase + tok * Cfg::ROW_BYTES + swz_chunk<B>(chunk, tok) * 16, xb[j][0], xb[j][1],
                                xb[j + 1][0], xb[j + 1][1]);
                }
#pragma unroll
                for (int i = 0; i < RowAcc<B, MP>::MT; ++i) {
                    const int row = i * 16 + (lane & 15);  // weight row inside the block
                    const int chunk = kk * 2 + (lane >> 4);
                    uint32_t a0, a1, a2, a3;
                    ldmatrix_x4(wbase + row * Cfg::ROW_BYTES + swz_chunk<B>(chunk, row) * 16, a0, a1, a2, a3);
#pragma unroll
                    for (int j = 0; j < RowAcc<B, MP>::NT; ++j)
                        mma_bf16_16816(acc.d[i][j], a0, a1, a2, a3, xb[j][0], xb[j][1]);
                }
            }
            // the slot is read: refill it with the block NSLOT ahead
            const int tn = t + Cfg::NSLOT;
            if (tn < nblk) {
                const int c = col_of(q0 + tn);
                __syncwarp();
                if (lane == 0) {
                    fence_async_smem();  // ldmatrix reads of this slot precede the next TMA write
                    mbar_arrive_expect_tx(&bars[s], Cfg::SLOT);
                    tma_load_2d(ring + s * Cfg::SLOT, &tmW, &bars[s], 0, (q0 + tn) * B);
                    tma_load_2d(ring + s * Cfg::SLOT + Cfg::W_BLK, &tmX, &bars[s], c * B, 0);
                }
                issued = tn + 1;
            }
        }
        if (ok) {
            last_row = r;
            lr_beg = row_beg;
            lr_end = row_end;
            cut_last = row_end > q1;
            if (last_row == first_row && cut_first) {
                part0 = acc;  // the share lies inside one row cut at its start: one partial
                cut_last = false;
            } else if (!cut_last) {
                write_row<B, MP>(acc, a, last_row, stage, lane);
            }
        }
    }
    if (!ok) {
        if (lane == 0) {
            set_status(a.status, BSL_ERR_TIMEOUT);
            // let this warp's copies land before its shared memory goes away
            for (int s = 0; s < Cfg::NSLOT && s < issued; ++s) {
                const int lastt = s + ((issued - 1 - s) / Cfg::NSLOT) * Cfg::NSLOT;  // last fill of slot s
                mbar_wait(&bars[s], (lastt / Cfg::NSLOT) & 1, a.timeout_ns, nullptr);
            }
        }
        if (nblk > 0) {
            // the row of the share's last block from the index alone, so that
            // this warp still counts itself in on every row it shares with
            // other CTAs and the counters return to zero (its sums are
            // incomplete; the status word reports the timeout)
            last_row = row_holding(a, q1 - 1, lane);
            lr_beg = a.row_ptr[last_row];
            lr_end = a.row_ptr[last_row + 1];
            cut_last = lr_end > q1 && !(last_row == first_row && cut_first);
        }
    }
    // the ring is read out: it now holds the warp's partials, [0] = first row
    // cut at the share's start, [1] = last row cut at its end
    float *myparts = reinterpret_cast<float *>(ring);
    __syncwarp();
    if (cut_first) part0.store(myparts, lane);
    if (cut_last) acc.store(myparts + Cfg::PART, lane);
    __syncthreads();

    // Cut rows.  The CTA's first contributor to a row (the warp whose share
    // holds the row's first block inside this CTA) adds the CTA's partials of
    // that row in warp order.
    for (int which = 0; which < 2; ++which) {
        const bool mine = which == 0 ? cut_first : cut_last;
        if (!mine) continue;
        const int r = which == 0 ? first_row : last_row;
        const int beg = which == 0 ? fr_beg : lr_beg, end = which == 0 ? fr_end : lr_end;
        const int lead = warp_of(beg > cq0 ? beg : cq0, cq0, cn);
        if (lead != warp) continue;
        RowAcc<B, MP> sum;  // the partials added in warp (then CTA) order, from zero
        sum.zero();
        const int wl = warp_of(end - 1 < cq1 - 1 ? end - 1 : cq1 - 1, cq0, cn);
        for (int w = warp; w <= wl; ++w) {
            const int sb = warp_bound(w, cq0, cn);
            if (warp_bound(w + 1, cq0, cn) == sb) continue;  // empty share: no partial
            // slot 0 holds a row that began before the warp's share, slot 1 the rest
            const float *src = reinterpret_cast<const float *>(smem + w * Cfg::WARP_BYTES) +
                               (sb > beg ? 0 : Cfg::PART);
            sum.add(src, lane);
        }
        if (beg >= cq0 && end <= cq1) {  // the whole row lies in this CTA's share
            write_row<B, MP>(sum, a, r, stage, lane);
            continue;
        }
        // the row reaches into other CTAs: this CTA's sum goes to the workspace;
        // the last CTA to arrive adds all of them in CTA order
        float *mine_ws = a.ws + (static_cast<int64_t>(blockIdx.x) * 2 + (cq0 >= beg ? 0 : 1)) * Cfg::PART;
        sum.store(mine_ws, lane);
        // CTAs holding the row's first and last block, and how many of the
        // CTAs between them hold any block (31 bounds per round of loads)
        const int c0 = cta_of(a, snapped, beg, U, lane);
        const int c1 = cta_of(a, snapped, end - 1, U, lane);
        int contributors = 0;
        for (int base = c0; base <= c1; base += 31) {
            const int c = base + lane;
            const int bc = cta_bound(a, snapped, c < U ? c : U, U);
            const int bn = __shfl_down_sync(0xffffffffu, bc, 1);
            contributors += __popc(__ballot_sync(0xffffffffu, lane < 31 && c <= c1 && bn > bc));
        }
        // every lane's stores happen before lane 0's release of the count; the
        // last arriver's acquire orders its reads of the other sums after it
        __syncwarp();
        int last = 0;
        if (lane == 0) last = arrive_count(a.cnt + c0) == contributors;
        last = __shfl_sync(0xffffffffu, last, 0);
        __syncwarp();
        if (!last) continue;
        sum.zero();
        for (int base = c0; base <= c1; base += 31) {
            const int c = base + lane;
            const int bc = cta_bound(a, snapped, c < U ? c : U, U);
            const int bn = __shfl_down_sync(0xffffffffu, bc, 1);
            const unsigned held = __ballot_sync(0xffffffffu, lane < 31 && c <= c1 && bn > bc);
            // slot 0 of a CTA holds the row when its range starts inside the row
            const unsigned first = __ballot_sync(0xffffffffu, bc >= beg);
            for (unsigned m = held; m; m &= m - 1) {
                const int j = __ffs(m) - 1;
                const float *src =
                    a.ws + (static_cast<int64_t>(base + j) * 2 + ((first >> j) & 1u ? 0 : 1)) * Cfg::PART;
                sum.template add<true>(src, lane);
            }
        }
        if (lane == 0) a.cnt[c0] = 0;  // every contributor is in: ready for the next call
        write_row<B, MP>(sum, a, r, stage, lane);
    }

    // block rows without blocks: bias (or zeros), rows r = gw, gw + GW, ...
    for (int r = gw; r < a.R; r += GW) {
        if (r == gw ? !gw_empty : a.row_ptr[r + 1] != a.row_ptr[r]) continue;
        __nv_bfloat16 *s = reinterpret_cast<__nv_bfloat16 *>(stage);
        for (int idx = lane; idx < MP * B; idx += 32)
            s[idx] = __float2bfloat16_rn(bias_of(a, static_cast<int64_t>(r) * B + (idx % B)));
        store_staged<B, MP>(a, stage, r, lane);
    }
}

template <int B, int MP>
bsl_status run(const void *X, const void *values, StreamArgs a, cudaStream_t s)
{
    using Cfg = StreamCfg<B, MP>;
    const int grid = num_sms();
    CUtensorMap mw, mx;
    if (!make_map_2d(&mw, a.nnz > 0 ? values : X, B, static_cast<uint64_t>(a.nnz > 0 ? a.nnz : 1) * B, 2 * B, B, B,
                     2 * B) ||
        !make_map_2d(&mx, X, a.K, a.M, static_cast<uint64_t>(a.K) * 2, B, MP, 2 * B))
        return BSL_ERR_CUDA;
    auto kern = k_stream_fwd<B, MP>;
    const bsl_status sa = set_smem_once(reinterpret_cast<const void *>(kern), Cfg::SMEM_BYTES);
    if (sa != BSL_OK) return sa;
    return cuda_status(launch_dependent(kern, grid, kStreamWarps * 32, Cfg::SMEM_BYTES, s, mw, mx, a));
}

size_t partials_bytes(int32_t M, int32_t b)
{
    const int MP = M <= 16 ? 16 : 32;
    return static_cast<size_t>(num_sms()) * 2 * b * MP * sizeof(float);
}

}  // namespace

// workspace: [CTAs] counters first (their place does not depend on M), then
// the partial sums
static size_t counters_bytes() { return (static_cast<size_t>(num_sms()) * 4 + 15) & ~size_t(15); }

size_t stream_workspace_bytes(int32_t M, const bsl_bsr *W)
{
    return counters_bytes() + partials_bytes(M, W->b);
}

bsl_status launch_stream_fwd(const void *X, int32_t M, const bsl_bsr *W, const void *bias, void *Y, void *ws,
                             cudaStream_t s)
{
    const int B = W->b;
    StreamArgs a;
    a.Y = static_cast<__nv_bfloat16 *>(Y);
    a.cnt = static_cast<int32_t *>(ws);
    a.ws = reinterpret_cast<float *>(static_cast<uint8_t *>(ws) + counters_bytes());
    a.row_ptr = W->row_ptr;
    a.sbounds = W->sbounds;
    a.col_idx = W->col_idx;
    a.bias = static_cast<const __nv_bfloat16 *>(bias);
    a.M = M;
    a.N = W->N;
    a.K = W->K;
    a.R = W->N / B;
    a.C = W->K / B;
    a.nnz = W->nnz;
    a.status = W->status;
    a.timeout_ns = wait_timeout_ns();
    if (B == 64) return M <= 16 ? run<64, 16>(X, W->values, a, s) : run<64, 32>(X, W->values, a, s);
    return M <= 16 ? run<32, 16>(X, W->values, a, s) : run<32, 32>(X, W->values, a, s);
}

}  // namespace bsl

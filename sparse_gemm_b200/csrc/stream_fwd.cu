// stream_fwd.cu -- small-M forward by streaming the packed weight once.
//
// For a handful of tokens the forward is bound by reading the weight, not by
// arithmetic.  The lecture summary "Lecture 11: Sparsity" (48:12, "load and
// sparse expand") describes the remedy: read the compressed form, expand it
// on chip, multiply densely.  Here the compressed form is the packed BSR
// blocks, which are already dense b x b tiles, so "expanding" is placing them
// in shared memory next to the activation slice they multiply.
//
// Decomposition: the BSR block list [0, nnz) is cut into equal contiguous
// shares, one per warp of a one-CTA-per-SM grid (block counts, not block
// rows, are balanced; the 8 warps of a CTA hold consecutive shares).  Each
// warp streams its share through its own ring of slots; a slot holds one
// weight block and the activation slice X[0:MP, c*b:(c+1)*b] it multiplies,
// both brought in by TMA (swizzled rows, rows past M read as zeros).  The
// weight copies, which depend on nothing, leave first; a ring usually holds
// the warp's whole share.  The operands go to registers with ldmatrix;
// mma.sync m16n8k16 (bf16 in, fp32 accumulate) forms
// Y^T[n][m] = W_blk[n][:] . X[m][:], and the sum of the current block row
// stays in registers:
//   - a block row entirely inside the warp's share is finished there: bias
//     added, rounded to bf16, staged in shared memory, written to Y with
//     16-byte stores;
//   - a block row cut by share boundaries leaves an fp32 partial.  After all
//     warps of the CTA are done, the partials sit in their rings and the
//     CTA's first contributor to each cut row adds them in warp order.  A row
//     that lies inside the CTA's share is then written; a row that reaches
//     into other CTAs' shares leaves the CTA's sum in the workspace, and the
//     last CTA to count itself in on the row's counter adds the CTAs' sums in
//     CTA order and writes the row.
// Every sum has a fixed order (the same whoever arrives last), so results
// are identical run to run.  Block rows without blocks are written (bias or
// zeros) at the end.  The counters are zeroed on the stream before every
// launch, so nothing in the workspace has to survive from one call to the
// next.
#include "common.cuh"
#include "internal.h"

namespace bsl {
namespace {

constexpr int kStreamWarps = 8;
constexpr int kWarpSmem = 24 * 1024;  // ring bytes per warp

template <int B, int MP>
struct StreamCfg {
    static constexpr int ROW_BYTES = B * 2;
    static constexpr int W_BLK = B * ROW_BYTES;        // one weight block
    static constexpr int X_BLK = MP * ROW_BYTES;       // its activation slice (MP x b)
    static constexpr int SLOT = W_BLK + X_BLK;
    static constexpr int NSLOT = kWarpSmem / SLOT;
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
    int32_t *cnt;               // [CTAs] arrival counters (zero at launch)
    const int32_t *row_ptr, *col_idx;
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
__device__ __forceinline__ int share_begin(int u, int U, int nnz)
{
    return static_cast<int>((static_cast<int64_t>(u) * nnz) / U);
}

// the share that holds block p (the last u with share_begin(u) <= p);
// share_begin(u) = floor(u * nnz / U), so u is within one of floor(p * U / nnz)
__device__ __forceinline__ int share_of(int p, int U, int nnz)
{
    int u = static_cast<int>((static_cast<int64_t>(p) * U) / nnz);
    u = u < 0 ? 0 : (u > U - 1 ? U - 1 : u);
    while (u > 0 && share_begin(u, U, nnz) > p) --u;
    while (u + 1 < U && share_begin(u + 1, U, nnz) <= p) ++u;
    return u;
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

// A block row held as floats (n * MP + m, PER = b*MP/32 per lane): bias,
// bf16, staged, stored.
template <int B, int MP>
__device__ __forceinline__ void write_row_flat(const float (&sum)[B * MP / 32], const StreamArgs &a, int r,
                                               uint8_t *stage, int lane)
{
    __nv_bfloat16 *s = reinterpret_cast<__nv_bfloat16 *>(stage);
#pragma unroll
    for (int e = 0; e < B * MP / 32; ++e) {
        const int idx = e * 32 + lane;
        const int n = idx / MP, m = idx % MP;
        s[m * B + n] = __float2bfloat16_rn(sum[e] + bias_of(a, static_cast<int64_t>(r) * B + n));
    }
    store_staged<B, MP>(a, stage, r, lane);
}

template <int B, int MP>
__global__ void __launch_bounds__(kStreamWarps * 32, 1)
    k_stream_fwd(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                 const StreamArgs a)
{
    using Cfg = StreamCfg<B, MP>;
    constexpr int PER = Cfg::PART / 32;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align1024(smem_raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint8_t *ring = smem + warp * Cfg::WARP_BYTES;
    uint8_t *stage = smem + kStreamWarps * Cfg::WARP_BYTES + warp * Cfg::OUT_BYTES;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kStreamWarps * (Cfg::WARP_BYTES + Cfg::OUT_BYTES)) +
                     warp * Cfg::NSLOT;

    const int GW = gridDim.x * kStreamWarps;
    const int gw = blockIdx.x * kStreamWarps + warp;
    const int q0 = share_begin(gw, GW, a.nnz), q1 = share_begin(gw + 1, GW, a.nnz);
    const int cq0 = share_begin(blockIdx.x * kStreamWarps, GW, a.nnz);          // this CTA's blocks
    const int cq1 = share_begin((blockIdx.x + 1) * kStreamWarps, GW, a.nnz);
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

        // first block row of the share: last r with row_ptr[r] <= q0, by a
        // warp-parallel search (two or three rounds of one load per lane)
        int lo = 0, hi = a.R;  // row_ptr[lo] <= q0 < row_ptr[hi]
        while (hi - lo > 1) {
            const int step = (hi - lo + 31) / 32;
            const int probe = lo + lane * step;
            const bool le = probe < hi && a.row_ptr[probe] <= q0;
            const int last = 31 - __clz(__ballot_sync(0xffffffffu, le));  // lane 0 always qualifies
            lo = lo + last * step;
            hi = min(hi, lo + step);
        }
        first_row = lo;
        int r = lo;
        int rbase = r;
        int rp = rbase + 1 + lane <= a.R ? a.row_ptr[rbase + 1 + lane] : 0x7fffffff;
        int row_end = __shfl_sync(0xffffffffu, rp, 0);
        cut_first = a.row_ptr[first_row] < q0;
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
        cut_first = cut_last = false;  // nothing of this warp is combined
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
    const int w_lo = blockIdx.x * kStreamWarps;
    for (int which = 0; which < 2; ++which) {
        const bool mine = which == 0 ? cut_first : cut_last;
        if (!mine) continue;
        const int r = which == 0 ? first_row : last_row;
        const int beg = a.row_ptr[r], end = a.row_ptr[r + 1];
        const int lead = share_of(beg > cq0 ? beg : cq0, GW, a.nnz);
        if (lead != gw) continue;
        float sum[PER];
#pragma unroll
        for (int e = 0; e < PER; ++e) sum[e] = 0.f;
        const int wl = share_of(end - 1 < cq1 - 1 ? end - 1 : cq1 - 1, GW, a.nnz);
        for (int w = gw; w <= wl; ++w) {
            const int sb = share_begin(w, GW, a.nnz);
            if (share_begin(w + 1, GW, a.nnz) == sb) continue;  // empty share: no partial
            // slot 0 holds a row that began before the warp's share, slot 1 the rest
            const float *src = reinterpret_cast<const float *>(smem + (w - w_lo) * Cfg::WARP_BYTES) +
                               (sb > beg ? 0 : Cfg::PART);
#pragma unroll
            for (int e = 0; e < PER; ++e) sum[e] += src[e * 32 + lane];
        }
        if (beg >= cq0 && end <= cq1) {  // the whole row lies in this CTA's share
            write_row_flat<B, MP>(sum, a, r, stage, lane);
            continue;
        }
        // the row reaches into other CTAs: this CTA's sum goes to the workspace;
        // the last CTA to arrive adds all of them in CTA order
        float *mine_ws = a.ws + (static_cast<int64_t>(blockIdx.x) * 2 + (cq0 >= beg ? 0 : 1)) * Cfg::PART;
#pragma unroll
        for (int e = 0; e < PER; ++e) __stcg(mine_ws + e * 32 + lane, sum[e]);
        // CTAs holding the row's first and last block (CTA c owns warps 8c .. 8c+7)
        const int c0 = share_of(beg, GW, a.nnz) / kStreamWarps;
        const int c1 = share_of(end - 1, GW, a.nnz) / kStreamWarps;
        int contributors = 0;
        for (int c = c0; c <= c1; ++c)
            contributors += share_begin((c + 1) * kStreamWarps, GW, a.nnz) > share_begin(c * kStreamWarps, GW, a.nnz);
        __threadfence();  // every lane's part of the sum is visible before the count says so
        __syncwarp();
        int last = 0;
        if (lane == 0) last = atomicAdd(a.cnt + c0, 1) == contributors - 1;
        if (!__shfl_sync(0xffffffffu, last, 0)) continue;
        __threadfence();  // the other CTAs' sums are read after their counts
#pragma unroll
        for (int e = 0; e < PER; ++e) sum[e] = 0.f;
        for (int c = c0; c <= c1; ++c) {
            const int cb = share_begin(c * kStreamWarps, GW, a.nnz);
            if (share_begin((c + 1) * kStreamWarps, GW, a.nnz) == cb) continue;  // empty CTA share
            const float *src = a.ws + (static_cast<int64_t>(c) * 2 + (cb >= beg ? 0 : 1)) * Cfg::PART;
#pragma unroll
            for (int e = 0; e < PER; ++e) sum[e] += __ldcg(src + e * 32 + lane);
        }
        write_row_flat<B, MP>(sum, a, r, stage, lane);
    }

    // block rows without blocks: bias (or zeros), rows r = gw, gw + GW, ...
    for (int r = gw; r < a.R; r += GW) {
        if (a.row_ptr[r + 1] != a.row_ptr[r]) continue;
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
    // counters start at zero on every launch (stream order)
    cudaError_t e = cudaMemsetAsync(a.cnt, 0, static_cast<size_t>(grid) * sizeof(int32_t), s);
    if (e != cudaSuccess) return cuda_status(e);
    CUtensorMap mw, mx;
    if (!make_map_2d(&mw, a.nnz > 0 ? values : X, B, static_cast<uint64_t>(a.nnz > 0 ? a.nnz : 1) * B, 2 * B, B, B,
                     2 * B) ||
        !make_map_2d(&mx, X, a.K, a.M, static_cast<uint64_t>(a.K) * 2, B, MP, 2 * B))
        return BSL_ERR_CUDA;
    auto kern = k_stream_fwd<B, MP>;
    const bsl_status sa = set_smem_once(reinterpret_cast<const void *>(kern), Cfg::SMEM_BYTES);
    if (sa != BSL_OK) return sa;
    kern<<<grid, kStreamWarps * 32, Cfg::SMEM_BYTES, s>>>(mw, mx, a);
    return cuda_status(cudaGetLastError());
}

size_t partials_bytes(int32_t M, int32_t b)
{
    const int MP = M <= 16 ? 16 : 32;
    return static_cast<size_t>(num_sms()) * 2 * b * MP * sizeof(float);
}

}  // namespace

size_t stream_workspace_bytes(int32_t M, const bsl_bsr *W)
{
    return partials_bytes(M, W->b) + static_cast<size_t>(num_sms()) * sizeof(int32_t);
}

bsl_status launch_stream_fwd(const void *X, int32_t M, const bsl_bsr *W, const void *bias, void *Y, void *ws,
                             cudaStream_t s)
{
    const int B = W->b;
    StreamArgs a;
    a.Y = static_cast<__nv_bfloat16 *>(Y);
    a.ws = static_cast<float *>(ws);
    a.cnt = reinterpret_cast<int32_t *>(static_cast<uint8_t *>(ws) + partials_bytes(M, B));
    a.row_ptr = W->row_ptr;
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

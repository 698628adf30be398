// pack.cu -- dense weight + block mask -> packed block-sparse weight.
//
// Stored form (torchao sparsity README, Table 4.1, BSR and CSR/CSC rows):
// the kept b x b blocks as data, a block-row pointer and block-column index
// (BSR), and the transposed index over the same blocks (CSC) with a map from
// each CSC entry to its BSR block, so the values exist once.  The input is
// the hand-off form of the torchao README introduction: a dense weight with
// zeros in place, here with an explicit block mask.  Everything is integer
// or bit-copy work and deterministic: no atomics decide any output order.
//
// Kernels, in launch order:
//   k_counts     one warp per block row / block column: popcount of the mask
//   k_scan       one CTA: exclusive scans -> row_ptr, col_ptr; nnz check
//   k_fill_rows  one warp per block row: col_idx (ascending) by ballot prefix
//   k_fill_cols  one warp per block column: row_idx, csc_to_bsr
//   k_gather     16-byte vector copy of every kept block into `values`
//   k_order      rank of each row / column in the longest-first order
//   k_group_plan one warp per group of G = 128/b rows (columns) in that order:
//                merges the members' sorted block coordinates into the
//                entry list of the tensor-core kernels (count pass, scan,
//                fill pass); the kernels read the values themselves from
//                `values` (stored once) through this list
//   k_stream_bounds one CTA: the weight-streaming forward's CTA ranges, each
//                bound on a block-row start near its equal share (short rows
//                are never split between CTAs), chosen to minimise the
//                largest range
#include "common.cuh"
#include "internal.h"

namespace bsl {
namespace {

constexpr int kWarps = 8;  // warps per CTA in the per-row / per-column kernels

// counts[0..R) -> row_ptr[1..R], counts of columns -> col_ptr[1..C]
__global__ void k_counts(const uint8_t *__restrict__ mask, int32_t R, int32_t C, int32_t *__restrict__ row_ptr,
                         int32_t *__restrict__ col_ptr)
{
    const int lane = threadIdx.x & 31;
    const int w = blockIdx.x * kWarps + (threadIdx.x >> 5);
    if (w < R) {
        const uint8_t *row = mask + static_cast<int64_t>(w) * C;
        int cnt = 0;
        for (int c = lane; c < C; c += 32) cnt += row[c] != 0;
#pragma unroll
        for (int o = 16; o; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
        if (lane == 0) row_ptr[w + 1] = cnt;
    } else if (col_ptr && w < R + C) {
        const int c = w - R;
        int cnt = 0;
        for (int r = lane; r < R; r += 32) cnt += mask[static_cast<int64_t>(r) * C + c] != 0;
#pragma unroll
        for (int o = 16; o; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
        if (lane == 0) col_ptr[c + 1] = cnt;
    }
}

// Block-wide inclusive scan helper over 1024 threads.
__device__ int block_scan_incl(int v, int *sm)
{
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int t = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += t;
    }
    if (lane == 31) sm[wid] = v;
    __syncthreads();
    if (wid == 0) {
        int s = (lane < (int)(blockDim.x >> 5)) ? sm[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int t = __shfl_up_sync(0xffffffffu, s, o);
            if (lane >= o) s += t;
        }
        sm[lane] = s;
    }
    __syncthreads();
    if (wid > 0) v += sm[wid - 1];
    __syncthreads();
    return v;
}

// In-place: ptr[1..n] holds counts; turns ptr[0..n] into the exclusive prefix.
__device__ void scan_counts(int32_t *ptr, int32_t n, int *sm)
{
    int carry = 0;
    if (threadIdx.x == 0) ptr[0] = 0;
    for (int base = 0; base < n; base += blockDim.x) {
        const int i = base + threadIdx.x;
        const int cnt = i < n ? ptr[i + 1] : 0;
        const int incl = block_scan_incl(cnt, sm) + carry;
        if (i < n) ptr[i + 1] = incl;
        // the last thread of the chunk holds the running total
        __shared__ int tot;
        if (threadIdx.x == blockDim.x - 1) tot = incl;
        __syncthreads();
        carry = tot;
        __syncthreads();
    }
}

__global__ void __launch_bounds__(1024) k_scan(int32_t *row_ptr, int32_t R, int32_t *col_ptr, int32_t C,
                                               int32_t nnz, int32_t *status)
{
    __shared__ int sm[32];
    scan_counts(row_ptr, R, sm);
    if (col_ptr) scan_counts(col_ptr, C, sm);
    if (threadIdx.x == 0 && status && nnz >= 0 && row_ptr[R] != nnz) set_status(status, BSL_ERR_NNZ_MISMATCH);
}

__global__ void k_fill_rows(const uint8_t *__restrict__ mask, int32_t R, int32_t C,
                            const int32_t *__restrict__ row_ptr, int32_t *__restrict__ col_idx, int32_t nnz)
{
    const int lane = threadIdx.x & 31;
    const int r = blockIdx.x * kWarps + (threadIdx.x >> 5);
    if (r >= R) return;
    const uint8_t *row = mask + static_cast<int64_t>(r) * C;
    int pos = row_ptr[r];
    for (int c0 = 0; c0 < C; c0 += 32) {
        const int c = c0 + lane;
        const bool set = c < C && row[c] != 0;
        const uint32_t bal = __ballot_sync(0xffffffffu, set);
        const int p = pos + __popc(bal & ((1u << lane) - 1u));
        if (set && p < nnz) col_idx[p] = c;
        pos += __popc(bal);
    }
}

__global__ void k_fill_cols(const uint8_t *__restrict__ mask, int32_t R, int32_t C,
                            const int32_t *__restrict__ row_ptr, const int32_t *__restrict__ col_idx,
                            const int32_t *__restrict__ col_ptr, int32_t *__restrict__ row_idx,
                            int32_t *__restrict__ csc_to_bsr, int32_t nnz)
{
    const int lane = threadIdx.x & 31;
    const int c = blockIdx.x * kWarps + (threadIdx.x >> 5);
    if (c >= C) return;
    int pos = col_ptr[c];
    for (int r0 = 0; r0 < R; r0 += 32) {
        const int r = r0 + lane;
        const bool set = r < R && mask[static_cast<int64_t>(r) * C + c] != 0;
        const uint32_t bal = __ballot_sync(0xffffffffu, set);
        const int j = pos + __popc(bal & ((1u << lane) - 1u));
        if (set && j < nnz) {
            // BSR position of (r, c): binary search of c in row r's sorted columns
            int lo = row_ptr[r], hi = row_ptr[r + 1];
            lo = lo < 0 ? 0 : lo;
            hi = hi > nnz ? nnz : hi;
            while (lo < hi) {
                const int mid = (lo + hi) >> 1;
                if (col_idx[mid] < c) lo = mid + 1;
                else hi = mid;
            }
            row_idx[j] = r;
            csc_to_bsr[j] = lo < nnz ? lo : nnz - 1;
        }
        pos += __popc(bal);
    }
}

// values[p][i][:] = W[r*b + i][c*b : c*b + b], 16 bytes per thread per step.
__global__ void k_gather(const uint4 *__restrict__ W, int32_t K, int32_t b, int32_t R,
                         const int32_t *__restrict__ row_ptr, const int32_t *__restrict__ col_idx,
                         uint4 *__restrict__ values, int32_t nnz)
{
    const int vpr = b / 8;                  // 16-byte vectors per block row
    const int64_t per_block = static_cast<int64_t>(b) * vpr;
    // never read past the blocks the mask really has (nnz may disagree with it)
    const int64_t kept = row_ptr[R] < nnz ? row_ptr[R] : nnz;
    const int64_t total = per_block * kept;
    const int64_t wvpr = K / 8;             // 16-byte vectors per W row
    for (int64_t t = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; t < total;
         t += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int p = static_cast<int>(t / per_block);
        const int rem = static_cast<int>(t - static_cast<int64_t>(p) * per_block);
        const int i = rem / vpr, v = rem - i * vpr;
        // block row of p: last r with row_ptr[r] <= p
        int lo = 0, hi = R;
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (row_ptr[mid] <= p) lo = mid;
            else hi = mid;
        }
        const int c = col_idx[p];
        const int64_t src = (static_cast<int64_t>(lo) * b + i) * wvpr + static_cast<int64_t>(c) * vpr + v;
        values[t] = __ldg(W + src);
    }
}

// order[rank] = id, ranking by count (descending) then id (ascending).
__global__ void k_order(const int32_t *__restrict__ ptr, int32_t n, int32_t *__restrict__ order)
{
    extern __shared__ int32_t cnt_sm[];
    const int id = blockIdx.x * blockDim.x + threadIdx.x;
    const int my = id < n ? ptr[id + 1] - ptr[id] : 0;
    int rank = 0;
    for (int base = 0; base < n; base += blockDim.x) {
        const int j = base + threadIdx.x;
        cnt_sm[threadIdx.x] = j < n ? ptr[j + 1] - ptr[j] : -1;
        __syncthreads();
        const int lim = min(static_cast<int>(blockDim.x), n - base);
        for (int q = 0; q < lim; ++q) {
            const int o = cnt_sm[q];
            rank += (o > my) || (o == my && base + q < id);
        }
        __syncthreads();
    }
    if (id < n) order[rank] = id;
}

// One warp per group of G segments, consecutive in `order`: merges the
// members' ascending coordinate lists (a warp-wide minimum per step).  The
// count pass writes the group's entry and block counts to gptr[g+1] and
// bptr[g+1]; after the scan turns them into offsets, the fill pass writes
// entry = coordinate | (member mask << 24) and the BSR block of every
// present member (`blkmap` maps a segment position to its BSR block; null:
// the position itself).
template <int G>
__global__ void k_group_plan(const int32_t *__restrict__ seg_ptr, const int32_t *__restrict__ seg_idx,
                             const int32_t *__restrict__ blkmap, const int32_t *__restrict__ order, int32_t nseg,
                             int32_t ngroups, int32_t *__restrict__ gptr, int32_t *__restrict__ bptr,
                             int32_t *__restrict__ ent, int32_t *__restrict__ blk, int32_t nnz, int fill)
{
    static_assert(G <= 8, "member mask is 8 bits");
    const int lane = threadIdx.x & 31;
    const int g = blockIdx.x * kWarps + (threadIdx.x >> 5);
    if (g >= ngroups) return;
    const int mi = g * G + lane;
    int cur = 0, end = 0;
    if (lane < G && mi < nseg) {
        const int sgm = order[mi];
        cur = max(0, seg_ptr[sgm]);
        end = min(nnz, seg_ptr[sgm + 1]);
    }
    const int e0 = fill ? gptr[g] : 0;
    const int q0 = fill ? bptr[g] : 0;
    int count = 0, nb = 0;
    while (true) {
        const int v = cur < end ? seg_idx[cur] : 0x7fffffff;
        const int m = __reduce_min_sync(0xffffffffu, v);
        if (m == 0x7fffffff) break;
        const bool present = v == m;
        const uint32_t mask = __ballot_sync(0xffffffffu, present);
        if (fill) {
            if (lane == 0 && e0 + count < nnz) ent[e0 + count] = m | static_cast<int32_t>(mask << 24);
            const int pos = q0 + nb + __popc(mask & ((1u << lane) - 1u));
            if (present && pos < nnz) blk[pos] = blkmap ? blkmap[cur] : cur;
        }
        nb += __popc(mask);
        ++count;
        if (present) ++cur;
    }
    if (!fill && lane == 0) {
        gptr[g + 1] = count;
        bptr[g + 1] = nb;
    }
}

__global__ void __launch_bounds__(1024) k_scan_groups(int32_t *a, int32_t na, int32_t *b, int32_t nb_,
                                                      int32_t *c, int32_t nc, int32_t *d, int32_t nd)
{
    __shared__ int sm[32];
    scan_counts(a, na, sm);
    scan_counts(b, nb_, sm);
    scan_counts(c, nc, sm);
    scan_counts(d, nd, sm);
}

template <int G>
void launch_group_plans(const bsl_bsr *o, cudaStream_t s)
{
    const int32_t R = o->N / o->b, C = o->K / o->b, nnz = o->nnz;
    const int nrg = (R + G - 1) / G, ncg = (C + G - 1) / G;
    const int rb = (nrg + kWarps - 1) / kWarps, cbk = (ncg + kWarps - 1) / kWarps;
    for (int fill = 0; fill < 2; ++fill) {
        k_group_plan<G><<<rb, kWarps * 32, 0, s>>>(o->row_ptr, o->col_idx, nullptr, o->row_order, R, nrg,
                                                   o->rgrp_ptr, o->rgrp_bptr, o->rgrp_ent, o->rgrp_blk, nnz,
                                                   fill);
        k_group_plan<G><<<cbk, kWarps * 32, 0, s>>>(o->col_ptr, o->row_idx, o->csc_to_bsr, o->col_order, C, ncg,
                                                    o->cgrp_ptr, o->cgrp_bptr, o->cgrp_ent, o->cgrp_blk, nnz,
                                                    fill);
        if (!fill)
            k_scan_groups<<<1, 1024, 0, s>>>(o->rgrp_ptr, nrg, o->rgrp_bptr, nrg, o->cgrp_ptr, ncg, o->cgrp_bptr,
                                             ncg);
    }
}

// Block ranges of the U CTAs of the weight-streaming forward, sb[0] = U (the
// grid size they were made for), sb[1 + c] = first block of CTA c.  Bound c
// lies within q = floor(nnz / (2U)) blocks of its equal share
// t = floor(c * nnz / U) (the kernel finds a block's CTA from that), on a
// block-row start when the window [t - q, t + q] holds one, else at t; equal
// shares are at least 2q apart, so windows are ordered and no row of up to
// 2q + 1 blocks is ever split.  Among those choices the bounds minimise the
// largest CTA range: the smallest L for which choosing, CTA by CTA, the
// largest allowed bound at most L past the previous one reaches the end
// (larger bounds only relax what follows, so that choice succeeds whenever
// any does).  With q = 0 the bounds are the equal shares.

// index of the last row start <= x among rp[lo..hi], given rp[lo] <= x (rp
// non-decreasing; shared or global memory)
__device__ int last_start_le(const int32_t *rp, int lo, int hi, int64_t x)
{
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (rp[mid] <= x) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

struct BoundsCtx {
    const int32_t *rp;  // row_ptr (a shared-memory copy when it fits)
    int64_t nnz, q;
    int U;
    const int *wlo, *whi;  // [U] row-index range of the row starts inside CTA c's window (wlo > whi: none)
    const int *t;          // [U] equal shares floor(c * nnz / U)
};

// the largest allowed bound of CTA c that is <= x, or -1
__device__ int64_t largest_bound(const BoundsCtx &k, int c, int64_t x)
{
    const int64_t t = k.t[c];
    const int lo = k.wlo[c], hi = k.whi[c];
    if (lo > hi) return t <= x ? t : -1;  // no row start in the window
    if (k.rp[lo] > x) return -1;
    return k.rp[last_start_le(k.rp, lo, hi, x)];
}

// the bounds for the largest range L (written to sb when given); false if
// they cannot reach nnz
__device__ bool bounds_for(const BoundsCtx &k, int64_t L, int32_t *sb)
{
    int64_t prev = 0;
    if (sb) sb[1] = 0;
    for (int c = 1; c < k.U; ++c) {
        const int64_t v = largest_bound(k, c, prev + L);
        if (v < prev) return false;
        prev = v;
        if (sb) sb[1 + c] = static_cast<int32_t>(v);
    }
    if (sb) sb[1 + k.U] = static_cast<int32_t>(k.nnz);
    return k.nnz - prev <= L;
}

// one allowed bound of CTA c: the window's last row start, else t (0 <= c <= U)
__device__ int64_t some_bound(const BoundsCtx &k, int c)
{
    if (c == 0) return 0;
    if (c == k.U) return k.nnz;
    return k.wlo[c] > k.whi[c] ? k.t[c] : k.rp[k.whi[c]];
}

constexpr int kBoundsRowsInSmem = 8192;  // row_ptr entries copied to shared memory, at most

// One CTA (U <= 1024): each CTA's window located once; the largest range of
// one allowed choice is a feasible L to start from; then the smallest feasible L by
// rounds of parallel probes (each round tests evenly spaced values below the
// smallest L known to work), and thread 0 writes the bounds.
__global__ void __launch_bounds__(1024) k_stream_bounds(const int32_t *__restrict__ row_ptr, int32_t R,
                                                        int32_t nnz, int32_t U, int32_t *__restrict__ sb)
{
    __shared__ int32_t srp[kBoundsRowsInSmem];
    __shared__ int wlo[1024], whi[1024], tt[1024];
    __shared__ unsigned long long best;
    const int64_t q = nnz / (2LL * U);
    if (threadIdx.x == 0) sb[0] = U;
    if (q == 0) {
        for (int c = threadIdx.x; c <= U; c += blockDim.x)
            sb[1 + c] = static_cast<int32_t>(static_cast<int64_t>(c) * nnz / U);
        return;
    }
    const bool in_smem = R + 1 <= kBoundsRowsInSmem;
    if (in_smem)
        for (int i = threadIdx.x; i <= R; i += blockDim.x) srp[i] = row_ptr[i];
    if (threadIdx.x == 0) best = 0;
    __syncthreads();
    const int32_t *rp = in_smem ? srp : row_ptr;
    for (int c = threadIdx.x; c < U; c += blockDim.x) {
        const int64_t t = static_cast<int64_t>(c) * nnz / U;
        const int hi = last_start_le(rp, 0, R, t + q);  // rp[0] = 0 <= t + q
        int lo = hi + 1;                                // none inside the window
        if (rp[hi] >= t - q) {
            int a = 0, b = hi;  // the first index in [a, b] with rp >= t - q (b qualifies)
            while (a < b) {
                const int mid = (a + b) >> 1;
                if (rp[mid] >= t - q) b = mid;
                else a = mid + 1;
            }
            lo = a;
        }
        wlo[c] = lo;
        whi[c] = hi;
        tt[c] = static_cast<int>(t);
    }
    __syncthreads();
    const BoundsCtx k{rp, nnz, q, U, wlo, whi, tt};
    // the largest range of one allowed choice (some_bound) is an L that works,
    // and a close one
    for (int c = threadIdx.x; c < U; c += blockDim.x)
        atomicMax(&best, static_cast<unsigned long long>(some_bound(k, c + 1) - some_bound(k, c)));
    __syncthreads();
    int64_t lo = (static_cast<int64_t>(nnz) + U - 1) / U, hi = static_cast<int64_t>(best);
    hi = hi < lo ? lo : (hi > nnz ? nnz : hi);
    __syncthreads();
    while (lo < hi) {
        const int64_t step = (hi - lo + blockDim.x - 1) / blockDim.x;
        if (threadIdx.x == 0) best = static_cast<unsigned long long>(hi);
        __syncthreads();
        const int64_t L = lo + static_cast<int64_t>(threadIdx.x) * step;
        if (L < hi && bounds_for(k, L, nullptr)) atomicMin(&best, static_cast<unsigned long long>(L));
        __syncthreads();
        const int64_t b = static_cast<int64_t>(best);
        // b is the smallest working probe (or hi); the probe a step below it failed
        lo = b - step + 1 > lo ? b - step + 1 : lo;
        hi = b;
        __syncthreads();
    }
    if (threadIdx.x == 0 && !bounds_for(k, lo, sb)) {
        // only with a row_ptr that is not non-decreasing: the allowed choice instead
        for (int c = 0; c <= U; ++c) sb[1 + c] = static_cast<int32_t>(some_bound(k, c));
    }
}

}  // namespace

bsl_status launch_pack_count(const uint8_t *mask, int32_t R, int32_t C, int32_t *row_ptr, cudaStream_t s)
{
    k_counts<<<(R + kWarps - 1) / kWarps, kWarps * 32, 0, s>>>(mask, R, C, row_ptr, nullptr);
    k_scan<<<1, 1024, 0, s>>>(row_ptr, R, nullptr, 0, -1, nullptr);
    return cuda_status(cudaGetLastError());
}

bsl_status launch_pack(const void *W, const uint8_t *mask, const bsl_bsr *o, cudaStream_t s)
{
    const int32_t R = o->N / o->b, C = o->K / o->b, nnz = o->nnz;
    // index arrays start as valid indices (0) even if the mask disagrees with nnz
    if (nnz > 0) {
        cudaMemsetAsync(o->col_idx, 0, sizeof(int32_t) * nnz, s);
        cudaMemsetAsync(o->row_idx, 0, sizeof(int32_t) * nnz, s);
        cudaMemsetAsync(o->csc_to_bsr, 0, sizeof(int32_t) * nnz, s);
    }
    k_counts<<<(R + C + kWarps - 1) / kWarps, kWarps * 32, 0, s>>>(mask, R, C, o->row_ptr, o->col_ptr);
    k_scan<<<1, 1024, 0, s>>>(o->row_ptr, R, o->col_ptr, C, nnz, o->status);
    k_fill_rows<<<(R + kWarps - 1) / kWarps, kWarps * 32, 0, s>>>(mask, R, C, o->row_ptr, o->col_idx, nnz);
    k_fill_cols<<<(C + kWarps - 1) / kWarps, kWarps * 32, 0, s>>>(mask, R, C, o->row_ptr, o->col_idx,
                                                                  o->col_ptr, o->row_idx, o->csc_to_bsr, nnz);
    if (nnz > 0) {
        const int64_t total = static_cast<int64_t>(nnz) * o->b * (o->b / 8);
        const int64_t want = (total + 255) / 256;
        const int grid = static_cast<int>(want < 8L * num_sms() ? want : 8L * num_sms());
        k_gather<<<grid, 256, 0, s>>>(static_cast<const uint4 *>(W), o->K, o->b, R, o->row_ptr, o->col_idx,
                                      static_cast<uint4 *>(o->values), nnz);
    }
    {
        const int U = num_sms();
        if (U <= BSL_SBOUNDS_LEN - 2) {
            k_stream_bounds<<<1, 1024, 0, s>>>(o->row_ptr, R, nnz, U, o->sbounds);
        } else {  // no room for this grid: the kernel falls back to equal shares
            cudaMemsetAsync(o->sbounds, 0, sizeof(int32_t), s);
        }
    }
    k_order<<<(R + 255) / 256, 256, 256 * sizeof(int32_t), s>>>(o->row_ptr, R, o->row_order);
    k_order<<<(C + 255) / 256, 256, 256 * sizeof(int32_t), s>>>(o->col_ptr, C, o->col_order);
    if (nnz > 0) {
        cudaMemsetAsync(o->rgrp_ent, 0, sizeof(int32_t) * nnz, s);
        cudaMemsetAsync(o->rgrp_blk, 0, sizeof(int32_t) * nnz, s);
        cudaMemsetAsync(o->cgrp_ent, 0, sizeof(int32_t) * nnz, s);
        cudaMemsetAsync(o->cgrp_blk, 0, sizeof(int32_t) * nnz, s);
    }
    if (o->b == 64) launch_group_plans<2>(o, s);
    else launch_group_plans<4>(o, s);
    cudaMemsetAsync(o->sched, 0, 8 * sizeof(int32_t), s);
    return cuda_status(cudaGetLastError());
}

}  // namespace bsl

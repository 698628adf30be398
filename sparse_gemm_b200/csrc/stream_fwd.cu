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
// rows, are balanced).  Each warp streams its share through its own ring of
// slots; a slot holds one weight block and the activation slice
// X[0:MP, c*b:(c+1)*b] it multiplies, both brought in by TMA (swizzled rows,
// rows past M read as zeros).  Every warp issues its own copies (one thread
// starts only a few copies per microsecond), and a ring usually holds the
// warp's whole share, so all its loads are in flight from the start.  The
// operands go to registers with ldmatrix; mma.sync m16n8k16 (bf16 in, fp32
// accumulate) forms Y^T[n][m] = W_blk[n][:] . X[m][:], and the partial sum
// of the current block row stays in registers:
//   - a block row entirely inside the warp's share is finished there: bias
//     added, rounded to bf16, staged in shared memory and written to Y with
//     16-byte stores;
//   - a block row cut by share boundaries leaves an fp32 partial in the
//     workspace (slot 0 if it is the share's first row, else slot 1); each
//     contributor then counts itself in on the row's counter, and the last to
//     arrive sums the partials of all contributors in warp order and writes
//     the row.  The sum order does not depend on who arrives last, so
//     results are identical run to run.
// Block rows without blocks are written (bias or zeros) by warp r % warps.
// The counters are zeroed on the stream before every launch, so nothing in
// the workspace has to survive from one call to the next.
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
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

struct StreamArgs {
    __nv_bfloat16 *Y;
    float *ws;                  // [GW][2][b*MP] partials
    int32_t *cnt;               // [GW] arrival counters (zero at launch)
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

// first block of warp share gw when nnz blocks are split over GW warps
__device__ __forceinline__ int share_begin(int gw, int GW, int nnz)
{
    return static_cast<int>((static_cast<int64_t>(gw) * nnz) / GW);
}

// the warp whose share holds block p (the last gw with share_begin(gw) <= p);
// share_begin(gw) = floor(gw * nnz / GW), so gw is within one of
// floor(p * GW / nnz)
__device__ __forceinline__ int warp_of(int p, int GW, int nnz)
{
    int w = static_cast<int>((static_cast<int64_t>(p) * GW) / nnz);
    w = w < 0 ? 0 : (w > GW - 1 ? GW - 1 : w);
    while (w > 0 && share_begin(w, GW, nnz) > p) --w;
    while (w + 1 < GW && share_begin(w + 1, GW, nnz) <= p) ++w;
    return w;
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
};

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

__device__ __forceinline__ float bias_of(const StreamArgs &a, int64_t col)
{
    return a.bias ? __bfloat162float(a.bias[col]) : 0.f;
}

// A finished block row: either the whole row (written to Y) or this warp's
// part of a row shared with other warps (fp32 partial, then the last of the
// row's contributors writes the row).
template <int B, int MP>
__device__ void finish_row(const RowAcc<B, MP> &acc, const StreamArgs &a, int r, int gw, int GW, int q0,
                           uint8_t *stage, int lane)
{
    const int g = lane >> 2, c2 = (lane & 3) * 2;
    const int beg = a.row_ptr[r], end = a.row_ptr[r + 1];
    const int q1 = share_begin(gw + 1, GW, a.nnz);
    if (beg >= q0 && end <= q1) {  // whole row in this share
#pragma unroll
        for (int i = 0; i < RowAcc<B, MP>::MT; ++i)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int n = i * 16 + g + h * 8;
                const float bb = bias_of(a, static_cast<int64_t>(r) * B + n);
#pragma unroll
                for (int j = 0; j < RowAcc<B, MP>::NT; ++j) {
                    const int m = j * 8 + c2;
                    __nv_bfloat16 *s = reinterpret_cast<__nv_bfloat16 *>(stage);
                    s[m * B + n] = __float2bfloat16_rn(acc.d[i][j][2 * h] + bb);
                    s[(m + 1) * B + n] = __float2bfloat16_rn(acc.d[i][j][2 * h + 1] + bb);
                }
            }
        store_staged<B, MP>(a, stage, r, lane);
        return;
    }
    // partial: slot 0 if the row is this share's first row, else slot 1
    constexpr int PART = StreamCfg<B, MP>::PART;
    float *mine = a.ws + (static_cast<int64_t>(gw) * 2 + (q0 >= beg ? 0 : 1)) * PART;
#pragma unroll
    for (int i = 0; i < RowAcc<B, MP>::MT; ++i)
#pragma unroll
        for (int j = 0; j < RowAcc<B, MP>::NT; ++j)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int n = i * 16 + g + h * 8, m = j * 8 + c2;
                __stcg(reinterpret_cast<float2 *>(mine + n * MP + m),
                       make_float2(acc.d[i][j][2 * h], acc.d[i][j][2 * h + 1]));
            }
    const int w0 = warp_of(beg, GW, a.nnz), w1 = warp_of(end - 1, GW, a.nnz);
    int contributors = 0;
    for (int w = w0; w <= w1; ++w) contributors += share_begin(w + 1, GW, a.nnz) > share_begin(w, GW, a.nnz);
    __threadfence();  // every lane's part of the partial is visible before the count says so
    __syncwarp();
    int last = 0;
    if (lane == 0) last = atomicAdd(a.cnt + w0, 1) == contributors - 1;
    if (!__shfl_sync(0xffffffffu, last, 0)) return;
    __threadfence();  // the other contributors' partials are read after their counts
    // last contributor: sum every contributor's partial in warp order
    constexpr int PER = PART / 32;
    float sum[PER];
#pragma unroll
    for (int e = 0; e < PER; ++e) sum[e] = 0.f;
    for (int w = w0; w <= w1; ++w) {
        const int sb = share_begin(w, GW, a.nnz);
        if (share_begin(w + 1, GW, a.nnz) == sb) continue;  // empty share wrote nothing
        const float *src = a.ws + (static_cast<int64_t>(w) * 2 + (sb >= beg ? 0 : 1)) * PART;
#pragma unroll
        for (int e = 0; e < PER; ++e) sum[e] += __ldcg(src + e * 32 + lane);
    }
    __nv_bfloat16 *s = reinterpret_cast<__nv_bfloat16 *>(stage);
#pragma unroll
    for (int e = 0; e < PER; ++e) {
        const int idx = e * 32 + lane;  // = n * MP + m
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
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align1024(smem_raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint8_t *ring = smem + warp * Cfg::WARP_BYTES;
    uint8_t *stage = smem + kStreamWarps * Cfg::WARP_BYTES + warp * Cfg::OUT_BYTES;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kStreamWarps * (Cfg::WARP_BYTES + Cfg::OUT_BYTES)) +
                     warp * Cfg::NSLOT;

    const int GW = gridDim.x * kStreamWarps;
    const int gw = blockIdx.x * kStreamWarps + warp;

    // block rows without blocks: bias (or zeros), rows r = gw, gw + GW, ...
    for (int r = gw; r < a.R; r += GW) {
        if (a.row_ptr[r + 1] != a.row_ptr[r]) continue;
        __nv_bfloat16 *s = reinterpret_cast<__nv_bfloat16 *>(stage);
        for (int idx = lane; idx < MP * B; idx += 32)
            s[idx] = __float2bfloat16_rn(bias_of(a, static_cast<int64_t>(r) * B + (idx % B)));
        store_staged<B, MP>(a, stage, r, lane);
    }

    const int q0 = share_begin(gw, GW, a.nnz), q1 = share_begin(gw + 1, GW, a.nnz);
    if (q0 >= q1) return;  // no block for this warp (no block-wide sync follows)
    const int nblk = q1 - q0;

    // block columns of 32 consecutive blocks of the share, one per lane
    int cbase = q0;
    int cidx = q0 + lane < q1 ? a.col_idx[q0 + lane] : 0;
    auto col_of = [&](int p) {  // warp-uniform p; refreshes the lane cache when p leaves it
        if (p >= cbase + 32) {
            cbase = p;
            cidx = p + lane < q1 ? a.col_idx[p + lane] : 0;
        }
        const int c = __shfl_sync(0xffffffffu, cidx, p - cbase);
        return c >= 0 && c < a.C ? c : 0;  // a column outside the weight (bad index) reads column 0
    };
    auto issue = [&](int t, int c) {  // lane 0: block q0 + t and its activation slice into slot t % NSLOT
        const int s = t % Cfg::NSLOT;
        uint8_t *dst = ring + s * Cfg::SLOT;
        mbar_arrive_expect_tx(&bars[s], Cfg::SLOT);
        tma_load_2d(dst, &tmW, &bars[s], 0, (q0 + t) * B);
        tma_load_2d(dst + Cfg::W_BLK, &tmX, &bars[s], c * B, 0);
    };
    if (lane == 0) {
        for (int s = 0; s < Cfg::NSLOT; ++s) mbar_init(&bars[s], 1);
        fence_barrier_init();
    }
    __syncwarp();
    const int nfirst = nblk < Cfg::NSLOT ? nblk : Cfg::NSLOT;
    for (int t = 0; t < nfirst; ++t) {
        const int c = col_of(q0 + t);
        if (lane == 0) issue(t, c);
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
    int r = lo;
    int rbase = r;
    int rp = rbase + 1 + lane <= a.R ? a.row_ptr[rbase + 1 + lane] : 0x7fffffff;
    int row_end = __shfl_sync(0xffffffffu, rp, 0);

    RowAcc<B, MP> acc;
    acc.zero();
    bool have = false, ok = true;
    int issued = nfirst;
    constexpr int KK = B / 16;

    for (int t = 0; t < nblk; ++t) {
        const int p = q0 + t;
        while (p >= row_end) {  // leaving block row r
            if (have) {
                finish_row<B, MP>(acc, a, r, gw, GW, q0, stage, lane);
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
                issue(tn, c);
            }
            issued = tn + 1;
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
        __syncwarp();
        return;
    }
    if (have) finish_row<B, MP>(acc, a, r, gw, GW, q0, stage, lane);
}

template <int B, int MP>
bsl_status run(const void *X, const void *values, StreamArgs a, cudaStream_t s)
{
    using Cfg = StreamCfg<B, MP>;
    const int grid = num_sms();
    const int GW = grid * kStreamWarps;
    // counters start at zero on every launch (stream order)
    cudaError_t e = cudaMemsetAsync(a.cnt, 0, static_cast<size_t>(GW) * sizeof(int32_t), s);
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
    return static_cast<size_t>(num_sms()) * kStreamWarps * 2 * b * MP * sizeof(float);
}

}  // namespace

size_t stream_workspace_bytes(int32_t M, const bsl_bsr *W)
{
    return partials_bytes(M, W->b) + static_cast<size_t>(num_sms()) * kStreamWarps * sizeof(int32_t);
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

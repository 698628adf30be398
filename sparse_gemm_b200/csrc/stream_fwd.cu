// stream_fwd.cu -- small-M forward by streaming the packed weight once.
//
// For a handful of tokens the forward is bound by reading the weight, not by
// arithmetic.  The lecture summary "Lecture 11: Sparsity" (48:12, "load and
// sparse expand") describes the remedy: read the compressed form, expand it
// on chip, multiply densely.  Here the compressed form is the packed BSR
// blocks, which are already dense b x b tiles, so "expanding" is placing them
// in shared memory for the tensor cores.
//
// Decomposition: the BSR block list [0, nnz) is cut into equal contiguous
// shares, one per warp of a one-CTA-per-SM grid (block counts, not block
// rows, are balanced).  Each warp streams its share through its own ring of
// stages, a stage holding CH consecutive weight blocks (one 2-D TMA copy,
// rows swizzled; every warp issues its own copies, since one thread can
// start only a few copies per microsecond).  The activation slice
// X[0:MP, c*b:(c+1)*b] of a block is small and stays in L2: its mma.sync
// fragments are read straight into registers, a whole stage of blocks ahead
// of use (the L2 latency is paid once per stage, not per block).  The
// weight block goes to registers with ldmatrix; mma.sync m16n8k16 (bf16 in,
// fp32 accumulate) forms Y^T[n][m] = W_blk[n][:] . X[m][:], and the partial
// sum of the current block row stays in registers:
//   - a block row entirely inside the warp's share is rounded to bf16 and
//     written to Y directly;
//   - a block row cut by a share boundary leaves an fp32 partial in the
//     workspace, slot 0 if it is the share's first row, else slot 1;
// k_stream_fixup (launched as a programmatic dependent of the main kernel,
// so its launch overlaps the main kernel) then sums, for every cut row, the
// partials of the warps covering it in warp order, and writes zeros for
// block rows without blocks.  Every sum has a fixed order, so results are
// identical run to run.
#include "common.cuh"
#include "internal.h"

namespace bsl {
namespace {

constexpr int kStreamWarps = 8;
constexpr int kWarpSmem = 24 * 1024;  // ring bytes per warp

template <int B, int MP>
struct StreamCfg {
    static constexpr int ROW_BYTES = B * 2;
    static constexpr int CH = B == 32 ? 4 : 1;          // weight blocks per stage (8 KB)
    static constexpr int W_BLK = B * ROW_BYTES;         // one weight block
    static constexpr int STAGE_BYTES = CH * W_BLK;
    static constexpr int STAGES = kWarpSmem / STAGE_BYTES;
    static constexpr int WARP_BYTES = STAGES * STAGE_BYTES;
    static constexpr int SMEM_BYTES = kStreamWarps * WARP_BYTES + kStreamWarps * STAGES * 8 + 1024;
    static_assert(STAGES >= 2, "ring too small");
    static_assert(STAGE_BYTES % 1024 == 0, "stage alignment for the swizzled copies");
};

struct StreamArgs {
    const __nv_bfloat16 *X;
    __nv_bfloat16 *Y;
    float *ws;
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

// Write a finished block row r: bf16 into Y (direct) or fp32 into a workspace slot.
template <int B, int MP>
__device__ __forceinline__ void flush_row(const RowAcc<B, MP> &acc, const StreamArgs &a, int r, bool direct,
                                          float *slot, int lane)
{
    const int g = lane >> 2, c2 = (lane & 3) * 2;
#pragma unroll
    for (int i = 0; i < RowAcc<B, MP>::MT; ++i)
#pragma unroll
        for (int j = 0; j < RowAcc<B, MP>::NT; ++j)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int n = i * 16 + g + h * 8;   // feature inside the block row
                const int m = j * 8 + c2;           // token
                const float v0 = acc.d[i][j][2 * h], v1 = acc.d[i][j][2 * h + 1];
                if (direct) {
                    const float bb = a.bias ? __bfloat162float(a.bias[static_cast<int64_t>(r) * B + n]) : 0.f;
                    __nv_bfloat16 *y = a.Y + static_cast<int64_t>(m) * a.N + static_cast<int64_t>(r) * B + n;
                    if (m < a.M) y[0] = __float2bfloat16_rn(a.bias ? v0 + bb : v0);
                    if (m + 1 < a.M) y[a.N] = __float2bfloat16_rn(a.bias ? v1 + bb : v1);
                } else {
                    *reinterpret_cast<float2 *>(slot + n * MP + m) = make_float2(v0, v1);
                }
            }
}

template <int B, int MP>
__global__ void __launch_bounds__(kStreamWarps * 32, 1)
    k_stream_fwd(const __grid_constant__ CUtensorMap tmW, const StreamArgs a)
{
    using Cfg = StreamCfg<B, MP>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align1024(smem_raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint8_t *ring = smem + warp * Cfg::WARP_BYTES;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kStreamWarps * Cfg::WARP_BYTES) + warp * Cfg::STAGES;

    // let the fix-up grid launch now; it waits for this grid before reading
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    const int GW = gridDim.x * kStreamWarps;
    const int gw = blockIdx.x * kStreamWarps + warp;
    const int q0 = share_begin(gw, GW, a.nnz), q1 = share_begin(gw + 1, GW, a.nnz);
    if (q0 >= q1) return;  // no block for this warp (no block-wide sync follows)
    const int nchunks = (q1 - q0 + Cfg::CH - 1) / Cfg::CH;
    const int nfirst = nchunks < Cfg::STAGES ? nchunks : Cfg::STAGES;

    // weight copies first: they depend on nothing
    if (lane == 0) {
        for (int s = 0; s < Cfg::STAGES; ++s) mbar_init(&bars[s], 1);
        fence_barrier_init();
        for (int t = 0; t < nfirst; ++t) {
            mbar_arrive_expect_tx(&bars[t], Cfg::STAGE_BYTES);
            tma_load_2d(ring + t * Cfg::STAGE_BYTES, &tmW, &bars[t], 0, (q0 + t * Cfg::CH) * B);
        }
    }
    __syncwarp();  // barrier initialisation visible to the whole warp
    // block columns of 32 consecutive blocks of the share, one per lane
    int cbase = q0;
    int cidx = q0 + lane < q1 ? a.col_idx[q0 + lane] : 0;
    auto col_of = [&](int p) {  // warp-uniform p; refreshes the lane cache when p leaves it
        if (p >= cbase + 32) {
            cbase = p;
            cidx = p + lane < q1 ? a.col_idx[p + lane] : 0;
        }
        const int c = __shfl_sync(0xffffffffu, cidx, p - cbase);
        return c >= 0 && c < a.C ? c : -1;
    };
    // mma.sync B fragments of block column c: X[j*8 + lane/4][c*b + kk*16 + 2*(lane%4) (+8)]
    constexpr int KK = B / 16, NT = MP / 8;
    const int g = lane >> 2, c2 = (lane & 3) * 2;
    auto load_x = [&](int c, uint32_t (&f)[KK][NT][2]) {
#pragma unroll
        for (int kk = 0; kk < KK; ++kk)
#pragma unroll
            for (int j = 0; j < NT; ++j) {
                const int m = j * 8 + g;
                if (c >= 0 && m < a.M) {
                    const __nv_bfloat16 *xp =
                        a.X + static_cast<int64_t>(m) * a.K + static_cast<int64_t>(c) * B + kk * 16 + c2;
                    f[kk][j][0] = __ldg(reinterpret_cast<const uint32_t *>(xp));
                    f[kk][j][1] = __ldg(reinterpret_cast<const uint32_t *>(xp + 8));
                } else {
                    f[kk][j][0] = 0u;
                    f[kk][j][1] = 0u;
                }
            }
    };
    // fragments of a whole stage are loaded one stage ahead (CH blocks in
    // flight), so the L2 latency is paid once per stage, not once per block
    uint32_t xf[Cfg::CH][KK][NT][2];
#pragma unroll
    for (int cb = 0; cb < Cfg::CH; ++cb) load_x(q0 + cb < q1 ? col_of(q0 + cb) : -1, xf[cb]);

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
    const int first_row = lo;
    int rbase = first_row;
    int rp = rbase + 1 + lane <= a.R ? a.row_ptr[rbase + 1 + lane] : 0x7fffffff;
    int r = first_row;
    int row_end = __shfl_sync(0xffffffffu, rp, 0);

    RowAcc<B, MP> acc;
    acc.zero();
    bool have = false, ok = true;
    float *ws_warp = a.ws + static_cast<int64_t>(gw) * 2 * B * MP;
    int issued = nfirst;

    for (int t = 0; t < nchunks; ++t) {
        const int s = t % Cfg::STAGES;
        const bool landed = mbar_wait(&bars[s], (t / Cfg::STAGES) & 1, a.timeout_ns, nullptr);
        if (!__all_sync(0xffffffffu, landed)) {  // uniform decision across the warp
            ok = false;
            break;
        }
        const uint32_t stage_addr = smem_u32(ring + s * Cfg::STAGE_BYTES);
        uint32_t xn[Cfg::CH][KK][NT][2];  // the next stage's fragments
#pragma unroll
        for (int cb = 0; cb < Cfg::CH; ++cb) {
            const int pn = q0 + (t + 1) * Cfg::CH + cb;
            load_x(pn < q1 ? col_of(pn) : -1, xn[cb]);
        }
#pragma unroll
        for (int cb = 0; cb < Cfg::CH; ++cb) {
            const int p = q0 + t * Cfg::CH + cb;
            if (p >= q1) break;
            while (p >= row_end) {  // leaving block row r
                if (have) {
                    const bool direct = a.row_ptr[r] >= q0;  // row began inside the share too
                    flush_row<B, MP>(acc, a, r, direct, ws_warp + (r == first_row ? 0 : B * MP), lane);
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
            have = true;
#pragma unroll
            for (int kk = 0; kk < KK; ++kk) {
#pragma unroll
                for (int i = 0; i < RowAcc<B, MP>::MT; ++i) {
                    const int row = cb * B + i * 16 + (lane & 15);  // weight row inside the stage
                    const int chunk = kk * 2 + (lane >> 4);
                    uint32_t a0, a1, a2, a3;
                    ldmatrix_x4(stage_addr + row * Cfg::ROW_BYTES + swz_chunk<B>(chunk, row) * 16, a0, a1, a2, a3);
#pragma unroll
                    for (int j = 0; j < NT; ++j)
                        mma_bf16_16816(acc.d[i][j], a0, a1, a2, a3, xf[cb][kk][j][0], xf[cb][kk][j][1]);
                }
            }
        }
#pragma unroll
        for (int cb = 0; cb < Cfg::CH; ++cb)
#pragma unroll
            for (int kk = 0; kk < KK; ++kk)
#pragma unroll
                for (int j = 0; j < NT; ++j) {
                    xf[cb][kk][j][0] = xn[cb][kk][j][0];
                    xf[cb][kk][j][1] = xn[cb][kk][j][1];
                }
        __syncwarp();
        const int tn = t + Cfg::STAGES;
        if (tn < nchunks) {
            if (lane == 0) {
                fence_async_smem();  // ldmatrix reads of this stage precede the next TMA write
                mbar_arrive_expect_tx(&bars[s], Cfg::STAGE_BYTES);
                tma_load_2d(ring + s * Cfg::STAGE_BYTES, &tmW, &bars[s], 0, (q0 + tn * Cfg::CH) * B);
            }
            issued = tn + 1;
        }
    }
    if (!ok) {
        if (lane == 0) {
            set_status(a.status, BSL_ERR_TIMEOUT);
            // let this warp's copies land before its shared memory goes away
            for (int t = 0; t < Cfg::STAGES && t < issued; ++t) {
                const int last = t + ((issued - 1 - t) / Cfg::STAGES) * Cfg::STAGES;  // last chunk on stage t
                mbar_wait(&bars[t], (last / Cfg::STAGES) & 1, a.timeout_ns, nullptr);
            }
        }
        __syncwarp();
        return;
    }
    if (have) {
        const bool direct = a.row_ptr[r] >= q0 && row_end <= q1;
        flush_row<B, MP>(acc, a, r, direct, ws_warp + (r == first_row ? 0 : B * MP), lane);
    }
}

// One warp per block row: zeros (or the bias) for rows without blocks; for
// rows cut between warp shares, the sum of the shares' partials in warp order
// (plus the bias).
template <int B, int MP>
__global__ void k_stream_fixup(const StreamArgs a, int GW)
{
    // wait until the main grid has finished and its writes are visible
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int lane = threadIdx.x & 31;
    const int r = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (r >= a.R) return;
    const int beg = a.row_ptr[r], end = a.row_ptr[r + 1];
    constexpr int PER = B * MP / 32;  // elements per lane
    float sum[PER];
#pragma unroll
    for (int e = 0; e < PER; ++e) sum[e] = 0.f;
    if (end > beg) {
        // warp share holding block p: the last gw with share_begin(gw) <= p.
        // share_begin(gw) = floor(gw * nnz / GW), so gw is within one of
        // floor(p * GW / nnz); step to the exact one.
        auto warp_of = [&](int p) {
            int w = static_cast<int>((static_cast<int64_t>(p) * GW) / a.nnz);
            w = w < 0 ? 0 : (w > GW - 1 ? GW - 1 : w);
            while (w > 0 && share_begin(w, GW, a.nnz) > p) --w;
            while (w + 1 < GW && share_begin(w + 1, GW, a.nnz) <= p) ++w;
            return w;
        };
        const int w0 = warp_of(beg), w1 = warp_of(end - 1);
        if (w0 == w1) return;  // written directly by its warp
        for (int w = w0; w <= w1; ++w) {
            const int sb = share_begin(w, GW, a.nnz);
            if (share_begin(w + 1, GW, a.nnz) == sb) continue;  // empty share wrote nothing
            const int slot = sb >= beg ? 0 : 1;
            const float *src = a.ws + (static_cast<int64_t>(w) * 2 + slot) * B * MP;
#pragma unroll
            for (int e = 0; e < PER; ++e) sum[e] += src[e * 32 + lane];
        }
    }
#pragma unroll
    for (int e = 0; e < PER; ++e) {
        const int idx = e * 32 + lane;  // = n * MP + m
        const int n = idx / MP, m = idx % MP;
        const float v = a.bias ? sum[e] + __bfloat162float(a.bias[static_cast<int64_t>(r) * B + n]) : sum[e];
        if (m < a.M)
            a.Y[static_cast<int64_t>(m) * a.N + static_cast<int64_t>(r) * B + n] = __float2bfloat16_rn(v);
    }
}

template <int B, int MP>
bsl_status run(const void *X, const void *values, int32_t K, const StreamArgs &a, cudaStream_t s)
{
    using Cfg = StreamCfg<B, MP>;
    const int grid = num_sms();
    if (a.nnz > 0) {
        CUtensorMap mw;
        if (!make_map_2d(&mw, values, B, static_cast<uint64_t>(a.nnz) * B, 2 * B, B, Cfg::CH * B, 2 * B))
            return BSL_ERR_CUDA;
        auto kern = k_stream_fwd<B, MP>;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM_BYTES);
        if (e != cudaSuccess) return cuda_status(e);
        kern<<<grid, kStreamWarps * 32, Cfg::SMEM_BYTES, s>>>(mw, a);
        if ((e = cudaGetLastError()) != cudaSuccess) return cuda_status(e);
    }
    // same shared-memory carveout as the main kernel: no reconfiguration between the two
    cudaFuncSetAttribute(k_stream_fixup<B, MP>, cudaFuncAttributePreferredSharedMemoryCarveout,
                         cudaSharedmemCarveoutMaxShared);
    const int rows_per_cta = 8;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((a.R + rows_per_cta - 1) / rows_per_cta);
    cfg.blockDim = dim3(rows_per_cta * 32);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cuda_status(cudaLaunchKernelEx(&cfg, k_stream_fixup<B, MP>, a, grid * kStreamWarps));
}

}  // namespace

size_t stream_workspace_bytes(int32_t M, const bsl_bsr *W)
{
    const int MP = M <= 16 ? 16 : 32;
    return static_cast<size_t>(num_sms()) * kStreamWarps * 2 * W->b * MP * sizeof(float);
}

bsl_status launch_stream_fwd(const void *X, int32_t M, const bsl_bsr *W, const void *bias, void *Y, void *ws,
                             cudaStream_t s)
{
    const int B = W->b;
    StreamArgs a;
    a.X = static_cast<const __nv_bfloat16 *>(X);
    a.Y = static_cast<__nv_bfloat16 *>(Y);
    a.ws = static_cast<float *>(ws);
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
    if (B == 64)
        return M <= 16 ? run<64, 16>(X, W->values, W->K, a, s) : run<64, 32>(X, W->values, W->K, a, s);
    return M <= 16 ? run<32, 16>(X, W->values, W->K, a, s) : run<32, 32>(X, W->values, W->K, a, s);
}

}  // namespace bsl

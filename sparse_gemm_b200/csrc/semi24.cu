// semi24.cu -- 2:4 semi-structured linear layer on sm_100a.
//
// The weight is kept in the compressed form of the torchao sparsity README,
// Table 4.1, row "NVIDIA 2:4 compressed representation": a dense matrix of
// half the width holding the unpruned elements of every group of four, plus
// 2-bit positions (include/bsl.h, bsl_semi24, gives the exact layout).
//
// k_compress24: one thread per 16 elements of a row (four groups) reads the
// dense weight with zeros in place and writes the two kept elements of each
// group and their positions.
//
// k_semi24_fwd: Y [M][N] = X [M][K] . W^T on the sparse tensor-core MMA
// (tcgen05.mma.sp, kind::f16).  The compressed weight is the MMA's A operand
// (the operand the instruction takes compressed), so the accumulator holds
// Y^T: TMEM lane = output feature, column = token.  Persistent, one CTA per
// SM, tiles of 256 features x 224 tokens (two M = 128 MMA blocks sharing the
// token tile), 64 dense K per stage (two K = 32 sparse MMAs per block).
// Roles (16 warps):
//   warp 0      TMA producer: per stage the compressed weight tile
//               (256 rows x 64 B, 64-byte swizzle) and the activation tile
//               (224 rows x 128 B, 128-byte swizzle) into a 4-stage ring;
//   warp 1      MMA issuer (lane 0), TMEM owner;
//   warps 4-7   metadata: per stage, the positions of their 32 TMEM lanes
//               loaded from global memory, rearranged into the lane layout
//               the sparse MMA reads (below) and written into a 4-stage
//               TMEM ring with tcgen05.st (the loads run 8 stages ahead);
//   warps 8-15  epilogue: TMEM -> registers (+ bias) -> bf16, transposed
//               through a 2 KB staging chunk per warp, TMA store of
//               32 tokens x 32 features.
// TMEM: columns 0..447 the two 128 x 224 fp32 accumulators (one buffer),
// 448..511 the metadata ring, 16 columns per stage: the metadata of block h,
// K step j at column 4(2h + j) of the stage (a sparse MMA's metadata address
// must be a multiple of 4 columns: an odd one raised a misaligned-address
// error on B200, and CUTLASS's sparse-MMA metadata fragments assume the same
// alignment).
//
// Sparse-MMA metadata layout in TMEM (measured on B200 with an in-bounds
// probe, sparsity selector 0): for rows 16q .. 16q+15 of the A block, TMEM
// lane 16q + 8kh + i holds the positions of K half kh (dense K 16kh ..
// 16kh+15 of the K = 32 step): bits 0-15 for row 16q + i, bits 16-31 for row
// 16q + 8 + i, four bits per group of four as in the compressed form.
//
// Every wait is bounded (BSL_ERR_TIMEOUT in the status word, then all roles
// leave through an abort flag); no wait is left on the way out.
#include "common.cuh"
#include "internal.h"

namespace bsl {
namespace {

__device__ __forceinline__ uint8_t *align1024(uint8_t *p)
{
    return reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// ------------------------------------------------------------ compress

__device__ __forceinline__ uint32_t pick4(uint32_t e0, uint32_t e1, uint32_t e2, uint32_t e3, int p)
{
    return p == 0 ? e0 : p == 1 ? e1 : p == 2 ? e2 : e3;
}

// Chunk i covers elements 16i .. 16i+15 of the row-major weight (rows hold
// K/16 whole chunks), values 8i .. 8i+7 and metadata entry i.
__global__ void k_compress24(const uint4 *__restrict__ W, int64_t chunks, uint4 *__restrict__ values,
                             uint16_t *__restrict__ meta, int32_t *status)
{
    const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i >= chunks) return;
    const uint4 a = __ldg(W + 2 * i), b = __ldg(W + 2 * i + 1);
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    uint32_t out[4];
    uint32_t code = 0;
    bool bad = false;
#pragma unroll
    for (int g = 0; g < 4; ++g) {
        const uint32_t e0 = w[2 * g] & 0xFFFFu, e1 = w[2 * g] >> 16;
        const uint32_t e2 = w[2 * g + 1] & 0xFFFFu, e3 = w[2 * g + 1] >> 16;
        const bool nz[4] = {(e0 & 0x7FFFu) != 0, (e1 & 0x7FFFu) != 0, (e2 & 0x7FFFu) != 0, (e3 & 0x7FFFu) != 0};
        const int cnt = nz[0] + nz[1] + nz[2] + nz[3];
        bad |= cnt > 2;
        // the nonzeros, completed by the lowest-indexed zeros
        int zeros = 0, p0 = -1, p1 = -1;
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            const bool keep = nz[p] || zeros < 2 - cnt;
            zeros += !nz[p];
            if (keep) {
                if (p0 < 0) p0 = p;
                else if (p1 < 0) p1 = p;
            }
        }
        out[g] = pick4(e0, e1, e2, e3, p0) | pick4(e0, e1, e2, e3, p1) << 16;
        code |= static_cast<uint32_t>(p0 | p1 << 2) << (4 * g);
    }
    values[i] = make_uint4(out[0], out[1], out[2], out[3]);
    meta[i] = static_cast<uint16_t>(code);
    if (bad) set_status(status, BSL_ERR_NOT_2_4);
}

// ------------------------------------------------------------ forward

struct Semi24Cfg {
    static constexpr int BF = 256;                    // features per tile (two M = 128 blocks)
    static constexpr int BT = 224;                    // tokens per tile (MMA N)
    static constexpr int BK = 64;                     // dense K per stage
    static constexpr int S = 4;                       // copy stages
    static constexpr int A_BYTES = BF * BK;           // 256 rows x 32 kept bf16
    static constexpr int B_BYTES = BT * BK * 2;       // 224 rows x 64 bf16
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int MS = 4;                      // metadata ring stages (TMEM)
    static constexpr int MCOLS = 16;                  // TMEM columns per metadata stage
    static constexpr int META_COL = 2 * BT;           // first metadata column
    static constexpr int TMEM_COLS = 512;
    static constexpr int EPI_WARPS = 8;
    static constexpr int OUT_CHUNK = 32 * 32 * 2;     // 32 tokens x 32 features bf16
    static constexpr int OUT_BYTES = EPI_WARPS * 2 * OUT_CHUNK;
    static constexpr int W_PROD = 0, W_MMA = 1, W_META = 4, W_EPI = 8;
    static constexpr int BAND = 16;                   // token tiles per band of the tile order
    static constexpr int THREADS = 16 * 32;
    static constexpr int BAR_BYTES = 1024;
    static constexpr int SMEM_BYTES = 1024 + S * STAGE_BYTES + OUT_BYTES + BAR_BYTES;
    static_assert(META_COL + MCOLS * MS <= TMEM_COLS, "TMEM columns");
    static_assert((2 * S + 2 * MS + 3) * 8 + 8 <= BAR_BYTES, "barrier area");
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
};

struct Semi24Args {
    int32_t M, N, K;
    int32_t ntf;    // feature tiles
    int32_t ntt;    // token tiles
    int32_t tiles;  // feature tiles x token tiles
    int32_t ks;     // stages per tile (K / 64)
    const uint16_t *meta;
    const __nv_bfloat16 *bias;
    int32_t *status;
    uint64_t timeout_ns;
};

// Tile t of the launch: bands of BAND token tiles in order, and inside a band
// every feature tile, feature tile major, so the CTAs working at one time
// share the weight slices of a few feature tiles and the activations of one
// band, which stay in L2 while the band is processed.
__device__ __forceinline__ void tile_origin(int t, const Semi24Args &a, int &f0, int &t0)
{
    using C = Semi24Cfg;
    const int band = t / (C::BAND * a.ntf);
    const int idx = t - band * C::BAND * a.ntf;
    const int first = band * C::BAND;
    const int width = a.ntt - first < C::BAND ? a.ntt - first : C::BAND;
    f0 = (idx / width) * C::BF;
    t0 = (first + idx % width) * C::BT;
}

// tcgen05.mma.sp (A compressed, metadata in TMEM), issued by the leader lane
// of a converged warp.
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

// 32 lanes x 32 bit, one column per thread.
__device__ __forceinline__ void tmem_st1(uint32_t taddr, uint32_t w)
{
    asm volatile("tcgen05.st.sync.aligned.32x32b.x1.b32 [%0], {%1};" ::"r"(taddr), "r"(w) : "memory");
}

__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__global__ void __launch_bounds__(Semi24Cfg::THREADS, 1)
    k_semi24_fwd(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmX,
                 const __grid_constant__ CUtensorMap tmY, const Semi24Args args)
{
    using C = Semi24Cfg;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *stages = align1024(smem_raw);
    uint8_t *outbuf = stages + C::S * C::STAGE_BYTES;
    uint64_t *bars = reinterpret_cast<uint64_t *>(outbuf + C::OUT_BYTES);
    uint64_t *full = bars;            // stage copies landed
    uint64_t *empty = full + C::S;    // stage MMAs finished
    uint64_t *mfull = empty + C::S;   // metadata of a stage written to TMEM (4 warps)
    uint64_t *mempty = mfull + C::MS; // metadata read by the stage's MMAs
    uint64_t *afull = mempty + C::MS; // accumulators complete
    uint64_t *aempty = afull + 1;     // accumulators read out (8 warps)
    uint64_t *drain = aempty + 1;
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
        mbar_init(afull, 1);
        mbar_init(aempty, C::EPI_WARPS);
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

    if (warp == C::W_PROD) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            bool ok = true;
            int g = 0;  // stages issued
            for (int t = blockIdx.x; ok && t < args.tiles; t += gridDim.x) {
                int f0, t0;
                tile_origin(t, args, f0, t0);
                for (int k = 0; k < args.ks; ++k, ++g) {
                    const int slot = g % C::S;
                    if (g >= C::S && !mbar_wait(&empty[slot], ((g / C::S) - 1) & 1, tmo, abort_flag)) {
                        ok = false;
                        break;
                    }
                    uint8_t *st = stages + slot * C::STAGE_BYTES;
                    mbar_arrive_expect_tx(&full[slot], C::STAGE_BYTES);
                    tma_load_2d(st, &tmA, &full[slot], k * (C::BK / 2), f0);
                    tma_load_2d(st + C::A_BYTES, &tmX, &full[slot], k * C::BK, t0);
                }
            }
            if (!ok) {
                *abort_flag = 1;
                set_status(args.status, BSL_ERR_TIMEOUT);
            }
            // every copy lands before the CTA's shared memory is released: the
            // last fill of each slot is the newest phase of its barrier
            for (int s = 0; s < C::S && s < g; ++s) {
                const int fills = (g - s + C::S - 1) / C::S;
                if (!mbar_wait(&full[s], (fills - 1) & 1, tmo, nullptr)) set_status(args.status, BSL_ERR_TIMEOUT);
            }
        }
        __syncwarp();
    } else if (warp == C::W_MMA) {
        // ------------------------------------------------------------ MMA issuer
        // Per stage: K step j outer, block h inner, so consecutive MMAs go to
        // different accumulators.  One commit frees the copy stage, one the
        // metadata stage; one per tile publishes the accumulators.
        const uint32_t idesc = make_idesc_bf16(128, C::BT, false, false) | (1u << 2);  // bit 2: sparse
        const uint32_t lead = lane == 0;
        bool ok = true, any = false;
        int g = 0, it = 0;
        for (int t = blockIdx.x; ok && t < args.tiles; t += gridDim.x, ++it) {
            if (it > 0 && __any_sync(0xffffffffu, !mbar_wait(aempty, (it - 1) & 1, tmo, abort_flag))) {
                ok = false;
                break;
            }
            tc_fence_after();
            for (int k = 0; k < args.ks; ++k, ++g) {
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
                for (int j = 0; j < 2; ++j) {
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const uint64_t ad = make_sdesc(a_base + h * (C::A_BYTES / 2) + j * 32, 16, 512, kLayoutSw64);
                        const uint64_t bd = make_sdesc(b_base + j * 64, 16, 1024, kLayoutSw128);
                        umma_sp_lead(lead, tmem + h * C::BT, ad, bd,
                                     tmem + C::META_COL + ms * C::MCOLS + (2 * h + j) * 4, idesc, (k | j) != 0);
                    }
                }
                umma_commit_lead(lead, &empty[slot]);
                umma_commit_lead(lead, &mempty[ms]);
                any = true;
                __syncwarp();
            }
            if (!ok) break;
            umma_commit_lead(lead, afull);
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
        // Lane l loads the 8 bytes of positions (dense K 64k .. 64k+63) of
        // block row 32q + l of each block, then takes from lanes src_lo /
        // src_hi the 16-bit halves that its TMEM lane 32q + l holds (layout in
        // the file header).
        const int q = warp & 3;
        const int src_lo = (lane & 16) | (lane & 7), src_hi = src_lo + 8;
        const bool upper = (lane >> 3) & 1;  // K half kh of the lane
        const size_t row_words = static_cast<size_t>(args.K) / 64;  // 8-byte words per row
        const uint2 *meta = reinterpret_cast<const uint2 *>(args.meta);
        const uint2 pad = make_uint2(0x44444444u, 0x44444444u);  // rows past N: pairs (0, 1) over zeros
        // stages of this CTA, all tiles in order: stage g is step g % ks of the
        // CTA's tile g / ks; the loads run P stages ahead of their use
        constexpr int P = 8;
        const int G = (args.tiles - static_cast<int>(blockIdx.x) + static_cast<int>(gridDim.x) - 1) /
                      static_cast<int>(gridDim.x) * args.ks;
        auto load = [&](int g, uint2 &m0, uint2 &m1) {
            m0 = pad;
            m1 = pad;
            if (g >= G) return;
            const int i = g / args.ks, k = g - i * args.ks;
            const int t = static_cast<int>(blockIdx.x) + i * static_cast<int>(gridDim.x);
            int f0, t0;
            tile_origin(t, args, f0, t0);
            const int r0 = f0 + 32 * q + lane;
            if (r0 < args.N) m0 = __ldg(meta + static_cast<size_t>(r0) * row_words + k);
            if (r0 + 128 < args.N) m1 = __ldg(meta + static_cast<size_t>(r0 + 128) * row_words + k);
        };
        uint2 b0[P], b1[P];
#pragma unroll
        for (int p = 0; p < P; ++p) load(p, b0[p], b1[p]);
        bool ok = true;
        for (int g0 = 0; ok && g0 < G; g0 += P) {
#pragma unroll
            for (int p = 0; p < P; ++p) {
                const int g = g0 + p;
                if (g >= G) break;
                const int ms = g % C::MS;
                uint32_t w[4];
#pragma unroll
                for (int h = 0; h < 2; ++h) {
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        const uint32_t x = h ? (j ? b1[p].y : b1[p].x) : (j ? b0[p].y : b0[p].x);
                        const uint32_t lo = __shfl_sync(0xffffffffu, x, src_lo);
                        const uint32_t hi = __shfl_sync(0xffffffffu, x, src_hi);
                        w[2 * h + j] = (upper ? lo >> 16 : lo & 0xFFFFu) | (upper ? hi & 0xFFFF0000u : hi << 16);
                    }
                }
                load(g + P, b0[p], b1[p]);
                if (g >= C::MS &&
                    __any_sync(0xffffffffu, !mbar_wait(&mempty[ms], ((g / C::MS) - 1) & 1, tmo, abort_flag))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t taddr = tmem + (static_cast<uint32_t>(32 * q) << 16) + C::META_COL + ms * C::MCOLS;
#pragma unroll
                for (int c = 0; c < 4; ++c) tmem_st1(taddr + 4 * c, w[c]);
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
        // Warp e reads block h = e / 4, TMEM lanes 32q .. 32q+31 (features),
        // 32 token columns at a time.  Neighbouring lanes swap values so each
        // writes one 32-bit word (two features of one token) into the
        // [32 tokens][32 features] staging chunk, stored by TMA.
        const int e = warp - C::W_EPI, q = warp & 3, h = e >> 2;
        uint8_t *wbuf = outbuf + e * 2 * C::OUT_CHUNK;
        const bool odd = lane & 1;
        bool ok = true;
        int it = 0, ob = 0;
        for (int t = blockIdx.x; ok && t < args.tiles; t += gridDim.x, ++it) {
            int f0, t0;
            tile_origin(t, args, f0, t0);
            f0 += h * 128 + 32 * q;
            const float bv = (args.bias && f0 + lane < args.N) ? __bfloat162float(args.bias[f0 + lane]) : 0.f;
            const int left = args.M - t0;
            const int nch = left >= C::BT ? C::BT / 32 : (left + 31) / 32;
            if (__any_sync(0xffffffffu, !mbar_wait(afull, it & 1, tmo, abort_flag))) {
                ok = false;
                break;
            }
            tc_fence_after();
            for (int c = 0; c < nch; ++c) {
                uint32_t v[32];
                tmem_ld32(tmem + (static_cast<uint32_t>(32 * q) << 16) + h * C::BT + c * 32, v);
                tmem_wait_ld();
                if (c == nch - 1) {  // this warp's last TMEM read of the tile
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(aempty);
                }
                if (f0 >= args.N) continue;  // no feature of this warp exists
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

}  // namespace

bsl_status launch_compress24(const void *W, const bsl_semi24 *out, cudaStream_t s)
{
    const int64_t chunks = static_cast<int64_t>(out->N) * (out->K / 16);
    const int64_t blocks = (chunks + 255) / 256;
    if (blocks > 0x7FFFFFFF) return BSL_ERR_UNSUPPORTED;
    k_compress24<<<static_cast<unsigned>(blocks), 256, 0, s>>>(
        static_cast<const uint4 *>(W), chunks, static_cast<uint4 *>(out->values), out->meta, out->status);
    return cuda_status(cudaGetLastError());
}

bsl_status launch_semi24_fwd(const void *X, int32_t M, const bsl_semi24 *W, const void *bias, void *Y,
                             cudaStream_t s)
{
    using C = Semi24Cfg;
    CUtensorMap ma, mx, my;
    if (!make_map_2d(&ma, W->values, W->K / 2, W->N, static_cast<uint64_t>(W->K), C::BK / 2, C::BF, 64) ||
        !make_map_2d(&mx, X, W->K, M, static_cast<uint64_t>(W->K) * 2, C::BK, C::BT, 128) ||
        !make_map_2d(&my, Y, W->N, M, static_cast<uint64_t>(W->N) * 2, 32, 32, 0))
        return BSL_ERR_CUDA;
    Semi24Args args;
    args.M = M;
    args.N = W->N;
    args.K = W->K;
    args.ntf = (W->N + C::BF - 1) / C::BF;
    args.ntt = (M + C::BT - 1) / C::BT;
    const int64_t tiles = static_cast<int64_t>(args.ntf) * args.ntt;
    if (tiles > 0x7FFFFFFF) return BSL_ERR_UNSUPPORTED;
    args.tiles = static_cast<int32_t>(tiles);
    args.ks = W->K / C::BK;
    args.meta = W->meta;
    args.bias = static_cast<const __nv_bfloat16 *>(bias);
    args.status = W->status;
    args.timeout_ns = wait_timeout_ns();
    const bsl_status sa = set_smem_once(reinterpret_cast<const void *>(k_semi24_fwd), C::SMEM_BYTES);
    if (sa != BSL_OK) return sa;
    const int grid = args.tiles < num_sms() ? args.tiles : num_sms();
    return cuda_status(launch_dependent(k_semi24_fwd, grid, C::THREADS, C::SMEM_BYTES, s, ma, mx, my, args));
}

}  // namespace bsl

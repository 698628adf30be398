// bias.cu -- gradient of the layer's bias.
//
// BlockSparseLinear is a drop-in for nn.Linear (Hugging Face
// pytorch_block_sparse release note, "Block-Sparse Implementation and
// Usage"), whose forward adds a bias per output column: Y = X W~^T + bias.
// Its gradient is the column sum of the upstream gradient,
//     dbias[n] = sum_m dY[m][n],
// accumulated in fp32 and rounded once to bf16.
//
// One CTA per 64-column tile of dY reads every row of its tile (128 bytes
// per row, a whole cache line per warp request); its 8 warps take rows
// w, w + 8, ... with four loads in flight each, and their partial sums are
// added in warp order through shared memory.  Every sum has a fixed order,
// so the result is identical run to run, and the kernel needs no scratch.
#include "common.cuh"
#include "internal.h"

namespace bsl {
namespace {

constexpr int kBiasWarps = 8;
constexpr int kBiasCols = 64;  // columns per CTA: 2 per lane

__global__ void __launch_bounds__(kBiasWarps * 32)
    k_bias_grad(const __nv_bfloat16 *__restrict__ dY, int32_t M, int32_t N, __nv_bfloat16 *__restrict__ dbias)
{
    __shared__ float2 part[kBiasWarps][32];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int col = blockIdx.x * kBiasCols + 2 * lane;  // N is a multiple of 32: col, col + 1 both valid or not
    const bool valid = col < N;
    float2 acc = make_float2(0.f, 0.f);
    if (valid) {
        const __nv_bfloat162 *base = reinterpret_cast<const __nv_bfloat162 *>(dY + col);
        const int64_t stride = N / 2;  // bf16x2 per row
        int m = warp;
        for (; m + 3 * kBiasWarps < M; m += 4 * kBiasWarps) {
            __nv_bfloat162 v[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) v[u] = base[static_cast<int64_t>(m + u * kBiasWarps) * stride];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const float2 f = __bfloat1622float2(v[u]);
                acc.x += f.x;
                acc.y += f.y;
            }
        }
        for (; m < M; m += kBiasWarps) {
            const float2 f = __bfloat1622float2(base[static_cast<int64_t>(m) * stride]);
            acc.x += f.x;
            acc.y += f.y;
        }
    }
    part[warp][lane] = acc;
    __syncthreads();
    if (warp == 0 && valid) {
        float2 s = part[0][lane];
#pragma unroll
        for (int w = 1; w < kBiasWarps; ++w) {
            s.x += part[w][lane].x;
            s.y += part[w][lane].y;
        }
        reinterpret_cast<__nv_bfloat162 *>(dbias + col)[0] = __floats2bfloat162_rn(s.x, s.y);
    }
}

}  // namespace

bsl_status launch_bias_grad(const void *dY, int32_t M, int32_t N, void *dbias, cudaStream_t s)
{
    const int grid = (N + kBiasCols - 1) / kBiasCols;
    k_bias_grad<<<grid, kBiasWarps * 32, 0, s>>>(static_cast<const __nv_bfloat16 *>(dY), M, N,
                                                  static_cast<__nv_bfloat16 *>(dbias));
    return cuda_status(cudaGetLastError());
}

}  // namespace bsl

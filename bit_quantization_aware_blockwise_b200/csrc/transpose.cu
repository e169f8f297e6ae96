// bf16 matrix transpose, dst[c][r] = src[r][c]: lays a dequantised weight
// w_hat [N, K] out as [K, N], the K-major operand of the fused input-gradient
// product (quest_trust_bwd_linear). 32 x 32 tiles through shared memory (one
// padding column against bank conflicts), persistent over the tiles.
#include <cuda_runtime.h>
#include <stdint.h>

#include "quest_internal.h"

namespace quest {
namespace {

constexpr int kT = 32, kRowsPerPass = 8;

__global__ void __launch_bounds__(kT * kRowsPerPass) transpose_bf16_kernel(const uint16_t* __restrict__ src,
                                                                          int64_t rows, int64_t cols,
                                                                          uint16_t* __restrict__ dst) {
    __shared__ uint16_t tile[kT][kT + 1];
    const int64_t tr = (rows + kT - 1) / kT, tc = (cols + kT - 1) / kT;
    const int tx = threadIdx.x, ty = threadIdx.y;
    for (int64_t t = blockIdx.x; t < tr * tc; t += gridDim.x) {
        const int64_t r0 = (t / tc) * kT, c0 = (t % tc) * kT;
#pragma unroll
        for (int j = 0; j < kT; j += kRowsPerPass) {
            const int64_t r = r0 + ty + j, c = c0 + tx;
            if (r < rows && c < cols) tile[ty + j][tx] = src[r * cols + c];
        }
        __syncthreads();
#pragma unroll
        for (int j = 0; j < kT; j += kRowsPerPass) {
            const int64_t c = c0 + ty + j, r = r0 + tx;
            if (c < cols && r < rows) dst[c * rows + r] = tile[tx][ty + j];
        }
        __syncthreads();
    }
}

}  // namespace

cudaError_t launch_transpose_bf16(const uint16_t* src, int64_t rows, int64_t cols, uint16_t* dst,
                                  cudaStream_t stream) {
    if (rows == 0 || cols == 0) return cudaSuccess;
    const int64_t tiles = ((rows + kT - 1) / kT) * ((cols + kT - 1) / kT);
    const int64_t cap = int64_t(sm_count()) * 8;
    transpose_bf16_kernel<<<(int)(tiles < cap ? tiles : cap), dim3(kT, kRowsPerPass), 0, stream>>>(src, rows, cols,
                                                                                                 dst);
    return cudaGetLastError();
}

}  // namespace quest

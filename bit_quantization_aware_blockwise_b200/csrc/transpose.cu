// bf16 matrix transpose, dst[c][r] = src[r][c]: lays a dequantised weight
// w_hat [N, K] out as [K, N], the K-major operand of the fused input-gradient
// product (quest_trust_bwd_linear). Tiles through shared memory (padding columns
// against bank conflicts), persistent over the tiles; bf16 pairs when both sizes
// are even, single elements otherwise.
#include <cuda_runtime.h>
#include <stdint.h>

#include "quest_internal.h"

namespace quest {
namespace {

constexpr int kT = 32, kRowsPerPass = 8;

__global__ void __launch_bounds__(kT * kRowsPerPass) transpose_bf16_kernel(const uint16_t* __restrict__ src,
                                                                          int64_t rows, int64_t cols,
                                                                          uint16_t* __restrict__ dst) {
    pdl_wait();      // the previous kernel on the stream has completed
    pdl_trigger();   // the next one may be scheduled as CTAs of this one leave
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

// Even sizes and 4-byte aligned pointers: 64 x 64 tiles moved as bf16 pairs, so
// each warp reads and writes 128 contiguous bytes per row (half the instructions
// of the element-wise version).
constexpr int kT2 = 64;

__global__ void __launch_bounds__(32 * kRowsPerPass) transpose_bf16x2_kernel(const uint32_t* __restrict__ src,
                                                                            int64_t rows, int64_t cols,
                                                                            uint32_t* __restrict__ dst) {
    pdl_wait();      // the previous kernel on the stream has completed
    pdl_trigger();   // the next one may be scheduled as CTAs of this one leave
    __shared__ uint16_t tile[kT2][kT2 + 2];
    const int64_t tr = (rows + kT2 - 1) / kT2, tc = (cols + kT2 - 1) / kT2;
    const int tx = threadIdx.x, ty = threadIdx.y;
    const int64_t cols2 = cols / 2, rows2 = rows / 2;
    for (int64_t t = blockIdx.x; t < tr * tc; t += gridDim.x) {
        const int64_t r0 = (t / tc) * kT2, c0 = (t % tc) * kT2;
#pragma unroll
        for (int j = 0; j < kT2; j += kRowsPerPass) {
            const int64_t r = r0 + ty + j, c = c0 + 2 * tx;
            if (r < rows && c < cols) {
                const uint32_t v = src[r * cols2 + c / 2];
                tile[ty + j][2 * tx] = uint16_t(v & 0xFFFFu);
                tile[ty + j][2 * tx + 1] = uint16_t(v >> 16);
            }
        }
        __syncthreads();
#pragma unroll
        for (int j = 0; j < kT2; j += kRowsPerPass) {
            const int64_t c = c0 + ty + j, r = r0 + 2 * tx;
            if (c < cols && r < rows)
                dst[c * rows2 + r / 2] = uint32_t(tile[2 * tx][ty + j]) | (uint32_t(tile[2 * tx + 1][ty + j]) << 16);
        }
        __syncthreads();
    }
}

}  // namespace

cudaError_t launch_transpose_bf16(const uint16_t* src, int64_t rows, int64_t cols, uint16_t* dst,
                                  cudaStream_t stream) {
    if (rows == 0 || cols == 0) return cudaSuccess;
    const int64_t cap = int64_t(sm_count()) * 8;
    if (rows % 2 == 0 && cols % 2 == 0 && (reinterpret_cast<uintptr_t>(src) & 3) == 0 &&
        (reinterpret_cast<uintptr_t>(dst) & 3) == 0) {
        const int64_t tiles = ((rows + kT2 - 1) / kT2) * ((cols + kT2 - 1) / kT2);
        return launch_pdl(transpose_bf16x2_kernel, dim3((unsigned)(tiles < cap ? tiles : cap)), dim3(32, kRowsPerPass),
                          0, stream, reinterpret_cast<const uint32_t*>(src), rows, cols,
                          reinterpret_cast<uint32_t*>(dst));
    }
    const int64_t tiles = ((rows + kT - 1) / kT) * ((cols + kT - 1) / kT);
    return launch_pdl(transpose_bf16_kernel, dim3((unsigned)(tiles < cap ? tiles : cap)), dim3(kT, kRowsPerPass), 0,
                      stream, src, rows, cols, dst);
}

}  // namespace quest

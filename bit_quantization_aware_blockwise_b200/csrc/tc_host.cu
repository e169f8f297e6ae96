// Host helpers of the tcgen05 kernels: tensor-map encoding through the driver
// entry point (no libcuda link), the co-resident CTA-pair count of a cluster
// kernel, and the zero fill of an empty reduction.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "quest_internal.h"

namespace quest {
namespace {

// Writes zeros (K == 0: the empty sum).
__global__ void zero_fill_kernel(uint16_t* y, int32_t* acc, int64_t n) {
    pdl_wait();      // the previous kernel on the stream has completed
    pdl_trigger();   // the next one may be scheduled as CTAs of this one leave
    for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
         i += int64_t(gridDim.x) * blockDim.x) {
        y[i] = 0;
        if (acc) acc[i] = 0;
    }
}

}  // namespace

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

bool make_map_2d(CUtensorMap* map, CUtensorMapDataType dt, const void* base, uint64_t inner,
                 uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
                 CUtensorMapSwizzle swz) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {row_bytes};
    const cuuint32_t box[2] = {box_inner, box_outer};
    const cuuint32_t estr[2] = {1, 1};
    return fn(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Co-resident CTA pairs of a cluster kernel on the current device (cached per
// kernel; the kernel's shared-memory attribute must already be set).
int pair_clusters(int dev, const void* kernel, int threads, uint32_t smem) {
    constexpr int kSlots = 4;
    static int cached_dev[kSlots] = {-1, -1, -1, -1}, cached[kSlots] = {0, 0, 0, 0};
    static const void* cached_fn[kSlots] = {nullptr, nullptr, nullptr, nullptr};
    static int next_slot = 0;
    static std::mutex mu;
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < kSlots; ++i)
        if (cached_fn[i] == kernel && cached_dev[i] == dev) return cached[i];
    int n = 0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * (sm_count() / 2), 1, 1);
    cfg.blockDim = dim3(threads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) != cudaSuccess || n <= 0) {
        cudaGetLastError();
        n = sm_count() / 2;
    }
    const int slot = next_slot;
    next_slot = (next_slot + 1) % kSlots;
    cached_fn[slot] = kernel;
    cached_dev[slot] = dev;
    cached[slot] = n;
    return n;
}

cudaError_t launch_zero_fill(uint16_t* y, int32_t* acc, int64_t n, cudaStream_t stream) {
    int64_t blocks = (n + 255) / 256;
    if (blocks > 4096) blocks = 4096;
    if (blocks < 1) return cudaSuccess;
    return launch_pdl(zero_fill_kernel, dim3((unsigned)blocks), dim3(256), 0, stream, y, acc, n);
}

}  // namespace quest

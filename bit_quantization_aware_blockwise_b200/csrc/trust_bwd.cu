// QuEST trust-estimator backward (sm_100a).
//
// The gradient with respect to the dequantised, Hadamard-domain value is
// multiplied by the trust mask and taken back through the (self-inverse)
// normalised Hadamard transform (pith.science review of QuEST, "What carries
// the argument"; Figure 2 caption: inverse Hadamard transforms on the backward
// pass):  grad_in_block = H (m . grad_out_block) / sqrt(n).
//
// HBM-bound: 2 bytes in, 1/8 byte of mask in, 2 bytes out per element. Same
// team layout as the forward quantizer (quest_device.cuh); the mask byte of a
// chunk covers exactly its 8 elements.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "quest_device.cuh"
#include "quest_internal.h"

namespace quest {
namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ uint32_t ld_mask_byte(const uint8_t* p) {
    uint16_t v;
    asm volatile("ld.global.nc.L1::no_allocate.u8 %0, [%1];" : "=h"(v) : "l"(p));
    return v;
}

__device__ __forceinline__ uint32_t ld_mask_bytes8(const uint8_t* p) {
    // eight 0/1 bytes -> 8-bit mask
    uint2 w;
    asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];"
                 : "=r"(w.x), "=r"(w.y)
                 : "l"(p));
    uint32_t m = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        m |= ((w.x >> (8 * i)) & 1u) << i;
        m |= ((w.y >> (8 * i)) & 1u) << (4 + i);
    }
    return m;
}

template <int HB>
__global__ void __launch_bounds__(kThreads) trust_bwd_kernel(const TrustArgs a) {
    pdl_wait();      // the previous kernel on the stream has completed
    pdl_trigger();   // the next one may be scheduled as CTAs of this one leave
    using S = TeamShape<HB>;
    constexpr int K = S::K, LPB = S::LPB, TPW = 32 / LPB;
    const int lane = threadIdx.x & 31, sub = lane % LPB;
    const int64_t total = a.rows * (a.cols / HB);
    const int64_t warp0 = (int64_t(blockIdx.x) * kThreads + threadIdx.x) >> 5;
    const int64_t wstride = int64_t(gridDim.x) * (kThreads / 32);

    for (int64_t wb = warp0 * TPW; wb < total; wb += wstride * TPW) {
        const int64_t blk = wb + lane / LPB;
        const bool valid = blk < total;
        const int64_t e = blk * HB;  // dense [rows, cols]: flat element offset
        float v[K][8];
        if (valid) {
#pragma unroll
            for (int j = 0; j < K; ++j) {
                const int64_t c0 = e + (sub + LPB * j) * 8;
                ChunkIO<__nv_bfloat16>::load(a.g + c0, v[j]);
                const uint32_t m = a.mask_mode == 0 ? ld_mask_byte(a.mask + c0 / 8)
                                                    : ld_mask_bytes8(a.mask + c0);
#pragma unroll
                for (int i = 0; i < 8; ++i) v[j][i] = ((m >> i) & 1u) ? v[j][i] : 0.0f;
            }
        } else {
#pragma unroll
            for (int j = 0; j < K; ++j)
#pragma unroll
                for (int i = 0; i < 8; ++i) v[j][i] = 0.0f;
        }
        fwht_team<K, LPB>(v, lane);
        if (valid) {
#pragma unroll
            for (int j = 0; j < K; ++j) {
#pragma unroll
                for (int i = 0; i < 8; ++i) v[j][i] *= a.inv_sqrt_hb;
                ChunkIO<__nv_bfloat16>::store(a.out + e + (sub + LPB * j) * 8, v[j]);
            }
        }
    }
}

template <int HB>
cudaError_t launch_hb(const TrustArgs& a, cudaStream_t stream) {
    using S = TeamShape<HB>;
    constexpr int TPW = 32 / S::LPB;
    const int64_t total = a.rows * (a.cols / HB);
    const int64_t warps = (total + TPW - 1) / TPW;
    const int64_t want = (warps + (kThreads / 32) - 1) / (kThreads / 32);
    auto fn = trust_bwd_kernel<HB>;
    const int64_t cap = int64_t(sm_count()) * max_ctas_per_sm((const void*)fn, kThreads, 0);
    const int grid = (int)(want < cap ? want : cap);
    return launch_pdl(fn, dim3((unsigned)grid), dim3(kThreads), 0, stream, a);
}

}  // namespace

// Rows of whole 128-value slabs take the tensor-core kernel (trust_tc.cu); this
// CUDA-core kernel covers the rest (any cols that are a multiple of the block).
cudaError_t launch_trust_bwd(const TrustArgs& a, int had_block, cudaStream_t stream) {
    if (trust_tc_ok(a, had_block)) return launch_trust_tc(a, had_block, stream);
    switch (had_block) {
        case 16: return launch_hb<16>(a, stream);
        case 32: return launch_hb<32>(a, stream);
        case 64: return launch_hb<64>(a, stream);
        case 128: return launch_hb<128>(a, stream);
        case 256: return launch_hb<256>(a, stream);
    }
    return cudaErrorInvalidValue;
}

}  // namespace quest

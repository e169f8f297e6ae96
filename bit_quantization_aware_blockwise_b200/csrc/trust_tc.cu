// QuEST trust-estimator backward with the tensor-core Hadamard factor (sm_100a).
//
// grad_in_block = H (m . grad_out_block) / sqrt(n): the gradient is masked by the
// trust mask in the Hadamard domain and taken back through the self-inverse
// normalised transform (pith.science review of QuEST, "What carries the
// argument"; Figure 2 caption: inverse Hadamard transforms on the backward pass).
//
// The mask is applied to the bf16 words as loaded (an AND with 0x0000 / 0xFFFF
// halves), so the masked words are still the A operand of the MMA in
// quest_tc.cuh; three index bits remain as register butterflies. Per element
// this is about a third of the instructions of the CUDA-core kernel in
// trust_bwd.cu, which stays for shapes this layout does not cover.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "quest_device.cuh"
#include "quest_internal.h"
#include "quest_tc.cuh"

namespace quest {
namespace tc {

__device__ __forceinline__ uint32_t ld_nc_u32(const void* p) {
    uint32_t v;
    asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}

__device__ __forceinline__ uint2 ld_nc_u2(const void* p) {
    uint2 v;
    asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
    return v;
}

// Eight 0/1 mask bytes (bit 0 of each byte counts) -> 8-bit mask, bit i = byte i.
__device__ __forceinline__ uint32_t bytes_to_bits(uint2 w) {
    const uint32_t lo = ((w.x & 0x01010101u) * 0x01020408u) >> 24;
    const uint32_t hi = ((w.y & 0x01010101u) * 0x01020408u) >> 24;
    return (lo & 0xFu) | ((hi & 0xFu) << 4);
}

// Mask state of one slab for this lane: byte f = mask bits of chunk t + 4f.
struct SlabIn {
    uint4 raw[4];
    uint32_t m;   // bits: the raw 32-bit word (chunks 4t .. 4t+3); bytes: already per chunk
};

__device__ __forceinline__ void load_in(const TrustArgs& a, int64_t slab, int t, SlabIn& in) {
    load_slab(reinterpret_cast<const char*>(a.g) + slab * 256, t, in.raw);
    if (a.mask_mode == 0) {
        in.m = ld_nc_u32(a.mask + slab * 16 + 4 * t);
    } else {
        uint32_t m = 0;
#pragma unroll
        for (int f = 0; f < 4; ++f) m |= bytes_to_bits(ld_nc_u2(a.mask + slab * 128 + 8 * (t + 4 * f))) << (8 * f);
        in.m = m;
    }
}

__device__ __forceinline__ void zero_in(SlabIn& in) {
    zero4(in.raw);
    in.m = 0;
}

// Zero the masked bf16 values of one chunk: bit i of `m` keeps value i, which
// is the low (i even) or high half of word i / 2.
__device__ __forceinline__ void mask_chunk(uint4& w, uint32_t m) {
    // byte k of s has its top bit = bit k of m (k < 4); of s2 = bit 4 + k
    const uint32_t s = (m & 0xFu) * 0x10204080u, s2 = ((m >> 4) & 0xFu) * 0x10204080u;
    w.x &= prmt(s, 0u, 0x9988u);    // halves <- sign of bytes 0, 1
    w.y &= prmt(s, 0u, 0xBBAAu);    // bytes 2, 3
    w.z &= prmt(s2, 0u, 0x9988u);
    w.w &= prmt(s2, 0u, 0xBBAAu);
}

template <int HB>
__global__ void __launch_bounds__(kThreads) trust_tc_kernel(const TrustArgs a) {
    pdl_wait();      // the previous kernel on the stream (the mask's producer) has completed
    pdl_trigger();   // the next one may be scheduled as CTAs of this one leave
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    const int64_t total = a.rows * (a.cols / 128);
    const int64_t warp0 = (int64_t(blockIdx.x) * kThreads + threadIdx.x) >> 5;
    const int64_t step = int64_t(gridDim.x) * (kThreads / 32) * 8;
    const BFrag B = make_bfrag(lane, tmask_of<HB>());
    const float2 sc = make_float2(a.inv_sqrt_hb, a.inv_sqrt_hb);

    SlabIn in;
    if (warp0 * 8 + g < total) load_in(a, warp0 * 8 + g, t, in);
    else zero_in(in);
    for (int64_t s0 = warp0 * 8; s0 < total; s0 += step) {
        const int64_t slab = s0 + g;
        const bool valid = slab < total;
        // bits mode: word of chunks 4t..4t+3 -> byte f = chunk t + 4f (every lane shuffles)
        const uint32_t m = a.mask_mode == 0 ? quad_transpose_bytes(in.m, t) : in.m;
#pragma unroll
        for (int f = 0; f < 4; ++f) mask_chunk(in.raw[f], (m >> (8 * f)) & 0xFFu);
        float2 P[16];
        mma_stage(in.raw, B, P);
        if (slab + step < total) load_in(a, slab + step, t, in);
        else zero_in(in);
        reg_stages<HB>(P, lane);
        if (valid) {
            char* out = reinterpret_cast<char*>(a.out) + slab * 256;
#pragma unroll
            for (int f = 0; f < 4; ++f) {
                uint32_t w[4];
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                    const float2 y = __fmul2_rn(P[4 * f + p], sc);
                    w[p] = pack_bf16x2(y.x, y.y);
                }
                *reinterpret_cast<uint4*>(out + 16 * (t + 4 * f)) = make_uint4(w[0], w[1], w[2], w[3]);
            }
        }
    }
}

template <int HB>
cudaError_t launch_hb(const TrustArgs& a, cudaStream_t stream) {
    const int64_t slabs = a.rows * (a.cols / 128);
    const int64_t warps = (slabs + 7) / 8;
    auto fn = trust_tc_kernel<HB>;
    const int64_t cap = int64_t(sm_count()) * max_ctas_per_sm((const void*)fn, kThreads, 0);
    const int64_t want = (warps + kThreads / 32 - 1) / (kThreads / 32);
    return launch_pdl(fn, dim3((unsigned)(want < cap ? want : cap)), dim3(kThreads), 0, stream, a);
}

}  // namespace tc

bool trust_tc_ok(const TrustArgs& a, int had_block) {
    if (a.cols % 128 != 0 || (had_block == 256 && a.cols % 256 != 0)) return false;
    if ((reinterpret_cast<uintptr_t>(a.g) & 15) != 0 || (reinterpret_cast<uintptr_t>(a.out) & 15) != 0) return false;
    const uintptr_t malign = a.mask_mode == 0 ? 4 : 8;
    return (reinterpret_cast<uintptr_t>(a.mask) % malign) == 0;
}

cudaError_t launch_trust_tc(const TrustArgs& a, int had_block, cudaStream_t stream) {
    switch (had_block) {
        case 16: return tc::launch_hb<16>(a, stream);
        case 32: return tc::launch_hb<32>(a, stream);
        case 64: return tc::launch_hb<64>(a, stream);
        case 128: return tc::launch_hb<128>(a, stream);
        case 256: return tc::launch_hb<256>(a, stream);
    }
    return cudaErrorInvalidValue;
}

}  // namespace quest

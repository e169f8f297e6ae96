// Tensor-core Hadamard factor shared by the bf16 quantizer and the trust
// backward (sm_100a).
//
// The Sylvester matrix factors over the bits of the element index, H_128 =
// H_2 (x) ... (x) H_2, so any four of the seven bits can be transformed at once by
// a 16 x 16 matrix product. Each lane's 16-byte load of 8 bf16 values is,
// unchanged, its part of the A operand of an m16n8k16 bf16 MMA (fp32
// accumulation; products of inputs with +-1 are exact), the result lands on the
// same lane in the same element order, and the remaining index bits are
// butterflies in registers.
//
// Layout. A warp step covers 8 slabs of 128 values. Lane = 4 g + t: slab g,
// chunks c = t + 4 f (f = 0..3) of 8 values each. With element index bits
// b0..b6 within the slab: b0 = position in a 32-bit word, (b1, b2) = word of the
// chunk, (b3, b4) = t, (b5, b6) = f. MMA f transforms bits (b0, b3, b4, b2) as
// its k bits; b1 is the row half of the fragment; b1, b5, b6 (and the slab bit
// for 256-blocks) are done in registers / by one shuffle.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "quest_device.cuh"

namespace quest {
namespace tc {

constexpr int kThreads = 128;

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

// 16 x 16 transform matrix on the MMA's k / n bits: entry (k, n) is the product
// over the 4 bits of H_2 (bit in `tmask`) or I_2 (bit not in the block).
__device__ __forceinline__ float mat_entry(int k, int n, int tmask) {
    int neg = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int ki = (k >> i) & 1, ni = (n >> i) & 1;
        if ((tmask >> i) & 1) neg ^= ki & ni;
        else if (ki != ni) return 0.0f;
    }
    return neg ? -1.0f : 1.0f;
}

__device__ __forceinline__ uint32_t bf16x2_bits(float lo, float hi) {
    const uint32_t l = __bfloat16_as_ushort(__float2bfloat16_rn(lo));
    const uint32_t h = __bfloat16_as_ushort(__float2bfloat16_rn(hi));
    return l | (h << 16);
}

// B fragments (k = 2t, 2t+1 and 2t+8, 2t+9; n = g + 8 tile) of the transform matrix.
struct BFrag {
    uint32_t b[2][2];   // [n tile][register]
};

__device__ __forceinline__ BFrag make_bfrag(int lane, int tmask) {
    const int g = lane >> 2, t = lane & 3;
    BFrag f;
#pragma unroll
    for (int tile = 0; tile < 2; ++tile) {
        const int n = g + 8 * tile;
        f.b[tile][0] = bf16x2_bits(mat_entry(2 * t, n, tmask), mat_entry(2 * t + 1, n, tmask));
        f.b[tile][1] = bf16x2_bits(mat_entry(2 * t + 8, n, tmask), mat_entry(2 * t + 9, n, tmask));
    }
    return f;
}

__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%10,%10,%10,%10};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(0.0f));
}

// The 4 chunks (16 bytes each) this lane loads from a slab at `src`.
__device__ __forceinline__ void load_slab(const char* src, int t, uint4 (&r)[4]) {
#pragma unroll
    for (int f = 0; f < 4; ++f) r[f] = ld_stream_v4(src + (t + 4 * f) * 16);
}

__device__ __forceinline__ void zero4(uint4 (&r)[4]) {
#pragma unroll
    for (int f = 0; f < 4; ++f) r[f] = make_uint4(0u, 0u, 0u, 0u);
}

// Transform bits (b0, b3, b4, b2) by MMA: P[4f + w] = values 2w, 2w+1 of chunk f.
// The loaded words go to the A registers in load order (an aligned quad, no
// moves): word 1 (b1 = 1) is the fragment's row half, word 2 (b2 = 1) its k3 half.
__device__ __forceinline__ void mma_stage(const uint4 (&r)[4], const BFrag& B, float2 (&P)[16]) {
#pragma unroll
    for (int f = 0; f < 4; ++f) {
        float d0[4], d1[4];
        mma16816(d0, r[f].x, r[f].y, r[f].z, r[f].w, B.b[0][0], B.b[0][1]);
        mma16816(d1, r[f].x, r[f].y, r[f].z, r[f].w, B.b[1][0], B.b[1][1]);
        P[4 * f + 0] = make_float2(d0[0], d0[1]);   // word 0: b1 = 0, b2 = 0
        P[4 * f + 1] = make_float2(d0[2], d0[3]);   // word 1: b1 = 1, b2 = 0
        P[4 * f + 2] = make_float2(d1[0], d1[1]);   // word 2: b1 = 0, b2 = 1
        P[4 * f + 3] = make_float2(d1[2], d1[3]);   // word 3: b1 = 1, b2 = 1
    }
}

__device__ __forceinline__ void bfly(float2& a, float2& b) {
    const float2 s = __fadd2_rn(a, b);
    b = f2_sub(a, b);
    a = s;
}

// Remaining in-register bits: b1 (index stride 1), b5 (stride 4), b6 (stride 8);
// for 256-blocks also the slab bit (lane ^ 4).
template <int HB>
__device__ __forceinline__ void reg_stages(float2 (&P)[16], int lane) {
#pragma unroll
    for (int j = 0; j < 16; j += 2) bfly(P[j], P[j + 1]);
    if constexpr (HB >= 64) {
#pragma unroll
        for (int j = 0; j < 16; ++j)
            if ((j & 4) == 0) bfly(P[j], P[j + 4]);
    }
    if constexpr (HB >= 128) {
#pragma unroll
        for (int j = 0; j < 8; ++j) bfly(P[j], P[j + 8]);
    }
    if constexpr (HB == 256) {
        const float sgn = (lane & 4) ? -1.0f : 1.0f;   // odd slab of the pair takes a - b
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const float2 o = make_float2(__shfl_xor_sync(0xFFFFFFFFu, P[j].x, 4),
                                         __shfl_xor_sync(0xFFFFFFFFu, P[j].y, 4));
            P[j] = __ffma2_rn(P[j], make_float2(sgn, sgn), o);
        }
    }
}

// Byte transpose across a lane quad: lane t holds byte f = value of chunk t + 4f;
// returns the word of chunks 4t .. 4t+3 (byte j = chunk 4t + j).
__device__ __forceinline__ uint32_t quad_transpose_bytes(uint32_t x, int t) {
    const uint32_t p1 = __shfl_xor_sync(0xFFFFFFFFu, x, 1);
    const uint32_t z = prmt(x, p1, (t & 1) ? 0x3715u : 0x6240u);
    const uint32_t p2 = __shfl_xor_sync(0xFFFFFFFFu, z, 2);
    return prmt(z, p2, (t & 2) ? 0x3276u : 0x5410u);
}

// Transform bits of a block size: HB = 16 leaves b4 (k bit 2) to the identity.
template <int HB>
constexpr int tmask_of() { return HB == 16 ? 0xB : 0xF; }   // HB = 16 leaves b4 alone

}  // namespace tc
}  // namespace quest

// Device helpers shared by the quantizer and trust-backward kernels:
// vector loads/stores, bf16 unpacking and the register/shuffle fast
// Walsh-Hadamard transform.
//
// Data layout used by both kernels ("team" layout): one Hadamard block of HB
// elements is owned by a team of LPB = HB / (8 K) consecutive lanes. Lane s of
// the team holds K chunks of 8 consecutive elements, chunk j being block chunk
// s + LPB * j. An element's index e inside the block therefore splits as
//   bits 0..2                 position inside the chunk   (in registers)
//   next log2(LPB) bits       lane inside the team        (across lanes)
//   top log2(K) bits          chunk slot j                (in registers)
// Every warp-wide 16-byte load of chunk slot j covers whole 32-byte sectors.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace quest {

// 1.5 * 2^23: fp32 values in [2^23, 2^24) are spaced exactly 1 apart, so
// fma_rd(y, inv, kMagic) == kMagic + floor(y * inv) for |y * inv| < 2^22, and
// the integer sits in the low mantissa bits of the result.
constexpr float kMagic = 12582912.0f;
constexpr uint32_t kMagicBits = 0x4B400000u;

__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ void st_v4(void* p, uint4 v) {
    asm volatile("st.global.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y),
                 "r"(v.z), "r"(v.w)
                 : "memory");
}

__device__ __forceinline__ float bf16lo_to_f32(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi_to_f32(uint32_t w) {
    return __uint_as_float(w & 0xFFFF0000u);
}

// Two fp32 -> bf16x2 (round to nearest even), `lo` in the low half.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}

// Load chunk (8 elements) of T = bf16 or fp32 into fp32 registers.
template <typename T>
struct ChunkIO;

template <>
struct ChunkIO<__nv_bfloat16> {
    static constexpr int kBytes = 16;
    __device__ __forceinline__ static void load(const void* p, float v[8]) {
        uint4 w = ld_stream_v4(p);
        v[0] = bf16lo_to_f32(w.x); v[1] = bf16hi_to_f32(w.x);
        v[2] = bf16lo_to_f32(w.y); v[3] = bf16hi_to_f32(w.y);
        v[4] = bf16lo_to_f32(w.z); v[5] = bf16hi_to_f32(w.z);
        v[6] = bf16lo_to_f32(w.w); v[7] = bf16hi_to_f32(w.w);
    }
    __device__ __forceinline__ static void store(void* p, const float v[8]) {
        uint4 w;
        w.x = pack_bf16x2(v[0], v[1]); w.y = pack_bf16x2(v[2], v[3]);
        w.z = pack_bf16x2(v[4], v[5]); w.w = pack_bf16x2(v[6], v[7]);
        st_v4(p, w);
    }
};

template <>
struct ChunkIO<float> {
    static constexpr int kBytes = 32;
    __device__ __forceinline__ static void load(const void* p, float v[8]) {
        uint4 a = ld_stream_v4(p);
        uint4 b = ld_stream_v4(static_cast<const char*>(p) + 16);
        v[0] = __uint_as_float(a.x); v[1] = __uint_as_float(a.y);
        v[2] = __uint_as_float(a.z); v[3] = __uint_as_float(a.w);
        v[4] = __uint_as_float(b.x); v[5] = __uint_as_float(b.y);
        v[6] = __uint_as_float(b.z); v[7] = __uint_as_float(b.w);
    }
    __device__ __forceinline__ static void store(void* p, const float v[8]) {
        st_v4(p, make_uint4(__float_as_uint(v[0]), __float_as_uint(v[1]),
                            __float_as_uint(v[2]), __float_as_uint(v[3])));
        st_v4(static_cast<char*>(p) + 16,
              make_uint4(__float_as_uint(v[4]), __float_as_uint(v[5]),
                         __float_as_uint(v[6]), __float_as_uint(v[7])));
    }
};

// Unnormalised Walsh-Hadamard butterflies over the team layout described at
// the top of this file: v[j][i] is element (s + LPB*j)*8 + i of the block,
// s = lane % LPB. After the call v holds (H x) at the same positions, with
// H_ek = (-1)^popcount(e & k) (Sylvester order, no 1/sqrt(n) factor).
template <int K, int LPB>
__device__ __forceinline__ void fwht_team(float (&v)[K][8], int lane) {
    // bits 0..2: inside each chunk
#pragma unroll
    for (int j = 0; j < K; ++j) {
#pragma unroll
        for (int h = 1; h < 8; h <<= 1) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                if ((i & h) == 0) {
                    float a = v[j][i], b = v[j][i + h];
                    v[j][i] = a + b;
                    v[j][i + h] = a - b;
                }
            }
        }
    }
    // lane bits: partner lane differs in one bit; the lane holding the set bit
    // takes (partner - self), the other (self + partner).
#pragma unroll
    for (int s = 1; s < LPB; s <<= 1) {
        const float sgn = (lane & s) ? -1.0f : 1.0f;
#pragma unroll
        for (int j = 0; j < K; ++j) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                float other = __shfl_xor_sync(0xFFFFFFFFu, v[j][i], s);
                v[j][i] = fmaf(sgn, v[j][i], other);
            }
        }
    }
    // chunk-slot bits: butterflies between chunk slots j and j + h
#pragma unroll
    for (int h = 1; h < K; h <<= 1) {
#pragma unroll
        for (int j = 0; j < K; ++j) {
            if ((j & h) == 0) {
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    float a = v[j][i], b = v[j + h][i];
                    v[j][i] = a + b;
                    v[j + h][i] = a - b;
                }
            }
        }
    }
}

// Sum over the LPB lanes of a team.
template <int LPB>
__device__ __forceinline__ float team_sum(float x) {
#pragma unroll
    for (int s = 1; s < LPB; s <<= 1) x += __shfl_xor_sync(0xFFFFFFFFu, x, s);
    return x;
}

// Team shape for a Hadamard block size: K chunks of 8 per lane, LPB lanes.
template <int HB>
struct TeamShape {
    static_assert(HB >= 16 && HB <= 256 && (HB & (HB - 1)) == 0, "HB must be 16..256, pow2");
    static constexpr int kChunks = HB / 8;
    static constexpr int K = kChunks >= 4 ? 4 : kChunks;
    static constexpr int LPB = kChunks / K;
    static_assert(LPB >= 1 && LPB <= 32, "team does not fit a warp");
};

}  // namespace quest

// ---------------------------------------------------------------------------
// Half-slab layout (TMA-staged kernels). A slab is 128 consecutive elements of
// a row, held by two adjacent lanes: lane half h (= lane & 1) holds elements
// h*64 + k, k = 0..63, as 32 packed pairs P[j] = (element 2j, element 2j+1).
// Index bits of an element inside a Hadamard block:
//   bit 0        inside a pair      (scalar add/sub)
//   bits 1..5    pair index j       (packed fp32x2 butterflies)
//   bit 6        lane ^ 1           (HB >= 128, shuffle)
//   bit 7        lane ^ 2           (HB == 256, shuffle)
// ---------------------------------------------------------------------------
namespace quest {

__device__ __forceinline__ float2 f2_sub(float2 a, float2 b) {
    return __ffma2_rn(b, make_float2(-1.0f, -1.0f), a);  // a - b, one rounding
}

}  // namespace quest

// ---------------------------------------------------------------------------
// Interleaved half-slab layout (direct-load kernels). Lane h (= lane & 1) of a
// pair holds chunks 2k + h, k = 0..7, of a 128-element slab (8 elements per
// chunk), so the two lanes' 16-byte loads of chunk slot k cover one 32-byte
// sector. Pair P[4k + p] = (element 2p, element 2p + 1) of chunk 2k + h.
// Element index bits inside a block:
//   bit 0            inside a pair                  (scalar add/sub)
//   bits 1, 2        pair bits 0, 1                 (packed butterflies)
//   bit 3            lane ^ 1                       (shuffle)
//   bits 4, 5, 6     pair bits 2, 3, 4              (packed, for HB >= 32/64/128)
//   bit 7            lane ^ 2 (the next slab)       (shuffle, HB == 256)
// A lane holds the pairs of block b in [b*PPB, (b+1)*PPB), PPB = min(HB, 128)/4.
// ---------------------------------------------------------------------------
namespace quest {

template <int HB>
__device__ __forceinline__ void fwht_interleaved(float2 (&P)[32], int lane) {
    static_assert(HB >= 16 && HB <= 256 && (HB & (HB - 1)) == 0, "HB");
#pragma unroll
    for (int j = 0; j < 32; ++j) {
        const float a = P[j].x, b = P[j].y;
        P[j] = make_float2(a + b, a - b);
    }
    // pair-index bit t is element bit t+1 (t < 2) or t+2 (t >= 2)
#pragma unroll
    for (int t = 0; t < 5; ++t) {
        const int elem_bit = t < 2 ? t + 1 : t + 2;
        if ((1 << elem_bit) < HB) {
            const int h = 1 << t;
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                if ((j & h) == 0) {
                    const float2 a = P[j], b = P[j + h];
                    P[j] = __fadd2_rn(a, b);
                    P[j + h] = f2_sub(a, b);
                }
            }
        }
    }
#pragma unroll
    for (int s = 1; s <= 2; s <<= 1) {
        if ((s == 1 && HB >= 16) || (s == 2 && HB >= 256)) {
            const float sg = (lane & s) ? -1.0f : 1.0f;
            const float2 sg2 = make_float2(sg, sg);
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                float2 o;
                o.x = __shfl_xor_sync(0xFFFFFFFFu, P[j].x, s);
                o.y = __shfl_xor_sync(0xFFFFFFFFu, P[j].y, s);
                P[j] = __ffma2_rn(P[j], sg2, o);
            }
        }
    }
}

}  // namespace quest

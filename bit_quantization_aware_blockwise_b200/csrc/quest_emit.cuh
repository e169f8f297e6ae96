// Per-element decision path shared by the half-slab quantizer kernels.
//
// Codes are produced biased, s = 1.5*2^23 + q_b with q_b = q + 2^(b-1) in
// [0, 2^b - 1], so that one integer multiply-add per element packs them (see
// the packing constants in quest_api.cu).
#pragma once

#include <cuda_fp16.h>
#include <cuda_fp4.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "quest_device.cuh"
#include "quest_internal.h"

namespace quest {

// Per-group constants of the decision path.
struct GroupK {
    float delta;   // Delta
    float a, c;    // u = sat(y_u * a + c)      (saturating path)
    float inv;     // t = y_u * inv             (exact path, general mask)
    float thr2;    // (edge * sqrt(HB) * Delta)^2
    float ch;      // yhat = q_b * Delta + ch
};

// From the sum of squares ss of a group's unnormalised transformed values:
// r = sqrt(ss / count), Delta = c_delta r, t = y / Delta. One approximate
// reciprocal square root (relative error a few 1e-7) serves all of them; a
// decision that this moves lies within 1e-6 relative of a cell boundary.
__device__ __forceinline__ GroupK make_group(const QuantConsts& k, float ss) {
    GroupK g;
    if (ss > 0.0f) {
        const float rs = rsqrtf(ss);
        g.delta = ss * rs * k.delta_k;
        g.inv = rs * k.inv_k;
        g.a = rs * k.a_k;
        g.c = 0.5f;
        g.thr2 = ss * k.thr2_k;
    } else {
        g.delta = 0.0f;
        g.inv = 0.0f;
        g.a = 0.0f;
        g.c = 0.5f + 0.5f * k.inv_levels;   // lands in the cell of q = 0
        g.thr2 = __int_as_float(0x7F800000);
    }
    g.ch = (0.5f - k.half_levels) * g.delta;
    return g;
}

// Biased code s = kMagic + q_b of a pair of transformed values.
template <bool SAT>
__device__ __forceinline__ float2 decide(float2 y, const GroupK& g, const QuantConsts& k) {
    if constexpr (SAT) {
        const float2 u = make_float2(__saturatef(__fmaf_rn(y.x, g.a, g.c)),
                                     __saturatef(__fmaf_rn(y.y, g.a, g.c)));
        return __ffma2_rd(u, make_float2(k.sat_k, k.sat_k), make_float2(kMagic, kMagic));
    } else {
        const float2 t = __ffma2_rd(y, make_float2(g.inv, g.inv), make_float2(k.s_mid, k.s_mid));
        return make_float2(fminf(fmaxf(t.x, kMagic), k.s_top), fminf(fmaxf(t.y, kMagic), k.s_top));
    }
}

// Trust-mask byte of the 8 elements in pairs [4*byte, 4*byte + 4): bit i = element i.
// For T >= 1: m = [y^2 <= thr^2], read off the sign of y^2 - thr^2.
template <int PPB, int N>
__device__ __forceinline__ uint32_t mask_byte_edge(const float2 (&P)[N], const GroupK* G, int byte) {
    uint32_t acc = 0;
#pragma unroll
    for (int j = 4 * byte + 3; j >= 4 * byte; --j) {
        const float t2 = G[j / PPB].thr2;
        const float2 d = __ffma2_rn(P[j], P[j], make_float2(-t2, -t2));
        acc = __funnelshift_l(__float_as_uint(d.y), acc, 1);
        acc = __funnelshift_l(__float_as_uint(d.x), acc, 1);
    }
    return acc;
}

// General T: m = [|t - (q + 1/2)| <= T/2] with q from the exact floor of t.
template <int PPB, int N>
__device__ __forceinline__ uint32_t mask_byte_cell(const float2 (&P)[N], const GroupK* G, int byte,
                                                   const QuantConsts& k) {
    uint32_t acc = 0;
#pragma unroll
    for (int j = 4 * byte + 3; j >= 4 * byte; --j) {
        const GroupK& g = G[j / PPB];
        // q + 1/2 = q_b + cell_center, q_b from the exact floor of t
        const float2 t = __fmul2_rn(P[j], make_float2(g.inv, g.inv));
        float2 sf = __ffma2_rd(P[j], make_float2(g.inv, g.inv), make_float2(k.s_mid, k.s_mid));
        sf = make_float2(fminf(fmaxf(sf.x, kMagic), k.s_top), fminf(fmaxf(sf.y, kMagic), k.s_top));
        const float ex = fabsf(t.x - ((sf.x - kMagic) + k.cell_center)) - k.half_trust;
        const float ey = fabsf(t.y - ((sf.y - kMagic) + k.cell_center)) - k.half_trust;
        const bool zero_group = !(g.delta > 0.0f);
        acc = __funnelshift_l(__float_as_uint(zero_group ? -1.0f : ey), acc, 1);
        acc = __funnelshift_l(__float_as_uint(zero_group ? -1.0f : ex), acc, 1);
    }
    return acc;
}

template <int PPB, int N>
__device__ __forceinline__ uint32_t mask_byte(const float2 (&P)[N], const GroupK* G, int byte,
                                              const QuantConsts& k) {
    return k.trust_ge1 ? mask_byte_edge<PPB>(P, G, byte) : mask_byte_cell<PPB>(P, G, byte, k);
}

// Biased codes of the 8 elements of one chunk (pairs 4c .. 4c+3 of a lane).
template <bool SAT, int PPB, int N>
__device__ __forceinline__ void chunk_decide(const float2 (&P)[N], const GroupK* G, int c,
                                             const QuantConsts& k, float2 (&s)[4]) {
#pragma unroll
    for (int p = 0; p < 4; ++p) s[p] = decide<SAT>(P[4 * c + p], G[(4 * c + p) / PPB], k);
}

// The 8 codes of a chunk in the low 8*CB bits (CB <= 4), with the constants of
// an 8-field word (pack8_add / pack8_xor).
template <int CB>
__device__ __forceinline__ uint32_t chunk_pack(const float2 (&s)[4], const QuantConsts& k) {
    static_assert(CB <= 4, "8-bit codes take chunk_pack_i8");
    uint32_t acc = 0;
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        acc += __float_as_uint(s[p].x) << (CB * 2 * p);
        acc += __float_as_uint(s[p].y) << (CB * (2 * p + 1));
    }
    return ((acc + k.pack8_add) ^ k.pack8_xor) & (CB == 4 ? 0xFFFFFFFFu : ((1u << (8 * CB)) - 1u));
}

// The 8 one-byte codes of a chunk as two 32-bit words. FMT 0: q and 1: c = 2q + 1
// as int8 (pack2_* constants); FMT 2: c as FP8 E4M3 (exact for |c| <= 15).
template <int FMT>
__device__ __forceinline__ uint2 chunk_pack_i8(const float2 (&s)[4], const QuantConsts& k) {
    uint32_t w[2];
    if constexpr (FMT == 2) {
        uint32_t h[4];
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            // q_b = s - 1.5*2^23 exactly; c = 2 (q_b + 1/2 - 2^(b-1))
            const float2 qb = __fadd2_rn(s[p], make_float2(-kMagic, -kMagic));
            const float2 c = __ffma2_rn(qb, make_float2(2.0f, 2.0f),
                                        make_float2(2.0f * k.cell_center, 2.0f * k.cell_center));
            h[p] = __nv_cvt_float2_to_fp8x2(c, __NV_SATFINITE, __NV_E4M3);
        }
        w[0] = h[0] | (h[1] << 16);
        w[1] = h[2] | (h[3] << 16);
    } else {
        constexpr uint32_t m = FMT == 1 ? 2u : 1u;
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const uint32_t acc = __float_as_uint(s[2 * u].x) * m + __float_as_uint(s[2 * u].y) * (m << 8) +
                                 __float_as_uint(s[2 * u + 1].x) * (m << 16) +
                                 __float_as_uint(s[2 * u + 1].y) * (m << 24);
            w[u] = (acc + k.pack2_add) ^ k.pack2_xor;
        }
    }
    return make_uint2(w[0], w[1]);
}

// ---------------------------------------------------------------------------
// FP4 (E2M1) grid. A chunk's 8 codes form one 32-bit word, element j of the
// chunk in nibble j; t = y_u * inv is rounded onto the grid by the hardware
// conversion (nearest, ties to the even mantissa, saturating at +-6, the sign
// of t kept, so a small negative t gives -0).
// ---------------------------------------------------------------------------
template <int PPB, int N>
__device__ __forceinline__ uint32_t chunk_fp4(const float2 (&P)[N], const GroupK* G, int c) {
    uint32_t w = 0;
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        const GroupK& g = G[(4 * c + p) / PPB];
        const float2 t = __fmul2_rn(P[4 * c + p], make_float2(g.inv, g.inv));
        w |= uint32_t(__nv_cvt_float2_to_fp4x2(t, __NV_E2M1, cudaRoundNearest)) << (8 * p);
    }
    return w;
}

// The grid values of a pair of codes (byte p of a chunk word) as fp32.
__device__ __forceinline__ float2 fp4_pair_value(uint32_t w, int p) {
    const __half2_raw h = __nv_cvt_fp4x2_to_halfraw2((__nv_fp4x2_storage_t)((w >> (8 * p)) & 0xFFu), __NV_E2M1);
    return __half22float2(*reinterpret_cast<const __half2*>(&h));
}

// int8 c = 2 Q of a chunk word. Each pair of grid values is decoded to an f16
// pair (exact), then 2 Q + 1152 (exact: f16 holds the integers of [1024, 2048)
// with unit spacing) leaves c + 128 in the low byte of each half; one byte
// permutation gathers four of them and an XOR with 0x80 removes the bias.
__device__ __forceinline__ uint32_t fp4_prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}
__device__ __forceinline__ uint2 fp4_operand_i8(uint32_t w) {
    uint32_t h[4];
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        const __half2_raw r = __nv_cvt_fp4x2_to_halfraw2((__nv_fp4x2_storage_t)((w >> (8 * p)) & 0xFFu), __NV_E2M1);
        const __half2 u = __hfma2(*reinterpret_cast<const __half2*>(&r), __floats2half2_rn(2.0f, 2.0f),
                                  __floats2half2_rn(1152.0f, 1152.0f));
        h[p] = *reinterpret_cast<const uint32_t*>(&u);
    }
    return make_uint2(fp4_prmt(h[0], h[1], 0x6420u) ^ 0x80808080u, fp4_prmt(h[2], h[3], 0x6420u) ^ 0x80808080u);
}

// yhat = Q Delta for the 4 pairs of chunk c.
template <int PPB>
__device__ __forceinline__ void fp4_dequant(uint32_t w, const GroupK* G, int c, float2 (&y)[4]) {
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        const float d = G[(4 * c + p) / PPB].delta;
        y[p] = __fmul2_rn(fp4_pair_value(w, p), make_float2(d, d));
    }
}

// General-T trust mask byte of chunk c on the FP4 grid: m = [|t - Q| <= (T/2) w],
// w the width of the grid interval that holds |t| (0.5 below 2, 1 below 4, else 2).
template <int PPB, int N>
__device__ __forceinline__ uint32_t mask_byte_fp4_cell(const float2 (&P)[N], const GroupK* G, int c,
                                                       uint32_t w, const QuantConsts& k) {
    uint32_t acc = 0;
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        const GroupK& g = G[(4 * c + p) / PPB];
        const float2 t = __fmul2_rn(P[4 * c + p], make_float2(g.inv, g.inv));
        const float2 q = fp4_pair_value(w, p);
        const float ax = fabsf(t.x), ay = fabsf(t.y);
        const float wx = ax < 2.0f ? 0.5f : (ax < 4.0f ? 1.0f : 2.0f);
        const float wy = ay < 2.0f ? 0.5f : (ay < 4.0f ? 1.0f : 2.0f);
        acc |= uint32_t(fabsf(t.x - q.x) <= k.half_trust * wx) << (2 * p);
        acc |= uint32_t(fabsf(t.y - q.y) <= k.half_trust * wy) << (2 * p + 1);
    }
    return acc;
}

}  // namespace quest

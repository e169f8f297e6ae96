// QuEST quantizer for bf16 input with a tensor-core Hadamard factor (sm_100a).
//
// Same method as quantize_hs.cu (pith.science review of QuEST, "What carries
// the argument"; atlas.scime.ai summary, "Approach"): per Hadamard block
// y = H x / sqrt(n); per RMS group Delta = alpha_b r / 2^(b-1); q = clamp(floor(y /
// Delta)); trust mask m = [|t - (q+1/2)| <= T/2].
//
// Why. On B200 the CUDA-core quantizer is bound by instruction issue, not by
// HBM: its butterflies, bf16 unpacking and cross-lane shuffles are about a third
// of ~14.5 instructions per element. The Sylvester matrix factors over the bits
// of the element index, H_128 = H_2 (x) ... (x) H_2, so any four of the seven
// bits can be transformed at once by a 16 x 16 matrix product. Here each lane's
// 16-byte load of 8 bf16 values is, unchanged, its part of the A operand of an
// m16n8k16 bf16 MMA (fp32 accumulation, exact products of inputs with +-1), the
// result lands on the same lane in the same element order, and only the three
// remaining index bits are butterflies in registers.
//
// Layout. A warp step covers 8 slabs of 128 values. Lane = 4 g + t: slab g,
// chunks c = t + 4 f (f = 0..3) of 8 values each. With element index bits
// b0..b6 within the slab: b0 = position in a 32-bit word, (b1, b2) = word of the
// chunk, (b3, b4) = t, (b5, b6) = f. MMA f transforms bits (b0, b3, b4, b1) as
// its k bits; b2 is the row half of the fragment; b2, b5, b6 (and the slab bit
// for 256-blocks) are done in registers / by one shuffle.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "quest_device.cuh"
#include "quest_emit.cuh"
#include "quest_internal.h"

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

// Transform bits (b0, b1, b3, b4) by MMA: P[4f + w] = values 2w, 2w+1 of chunk f.
__device__ __forceinline__ void mma_stage(const uint4 (&r)[4], const BFrag& B, float2 (&P)[16]) {
#pragma unroll
    for (int f = 0; f < 4; ++f) {
        // A registers: (row g, k3 = 0) = word 0, (row g+8, k3 = 0) = word 2,
        //              (row g, k3 = 1) = word 1, (row g+8, k3 = 1) = word 3
        float d0[4], d1[4];
        mma16816(d0, r[f].x, r[f].z, r[f].y, r[f].w, B.b[0][0], B.b[0][1]);
        mma16816(d1, r[f].x, r[f].z, r[f].y, r[f].w, B.b[1][0], B.b[1][1]);
        P[4 * f + 0] = make_float2(d0[0], d0[1]);   // word 0: b1 = 0, b2 = 0
        P[4 * f + 1] = make_float2(d1[0], d1[1]);   // word 1: b1 = 1, b2 = 0
        P[4 * f + 2] = make_float2(d0[2], d0[3]);   // word 2: b1 = 0, b2 = 1
        P[4 * f + 3] = make_float2(d1[2], d1[3]);   // word 3: b1 = 1, b2 = 1
    }
}

__device__ __forceinline__ void bfly(float2& a, float2& b) {
    const float2 s = __fadd2_rn(a, b);
    b = f2_sub(a, b);
    a = s;
}

// Remaining in-register bits: b2 (index stride 2), b5 (stride 4), b6 (stride 8);
// for 256-blocks also the slab bit (lane ^ 4).
template <int HB>
__device__ __forceinline__ void reg_stages(float2 (&P)[16], int lane) {
#pragma unroll
    for (int j = 0; j < 16; ++j)
        if ((j & 2) == 0) bfly(P[j], P[j + 2]);
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

// Blocks per lane and pairs of one block in a lane.
template <int HB>
struct Blk {
    static constexpr int NBL = HB <= 32 ? 4 : (HB == 64 ? 2 : 1);
    static constexpr int PPB = 16 / NBL;
};

template <int HB>
__device__ __forceinline__ void lane_sums(const float2 (&P)[16], float (&ss)[Blk<HB>::NBL]) {
    constexpr int NBL = Blk<HB>::NBL, PPB = Blk<HB>::PPB;
#pragma unroll
    for (int b = 0; b < NBL; ++b) {
        float2 acc0 = make_float2(0.0f, 0.0f), acc1 = acc0;
#pragma unroll
        for (int j = b * PPB; j < (b + 1) * PPB; j += 2) {
            acc0 = __ffma2_rn(P[j], P[j], acc0);
            acc1 = __ffma2_rn(P[j + 1], P[j + 1], acc1);
        }
        const float2 a = __fadd2_rn(acc0, acc1);
        ss[b] = a.x + a.y;
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

// Quantise and store this lane's 32 values: chunks c = t + 4f of the slab whose
// first element is `e_slab` in row `row`.
template <int PPB, int CB, bool MULT2, bool SAT>
__device__ __forceinline__ void emit(const QuantArgs& A, const float2 (&P)[16], const GroupK* G, int64_t row,
                                     int64_t e_slab, int t, bool valid) {
    const QuantConsts& k = A.c;
    uint8_t* codes = A.codes + row * A.codes_row_bytes + e_slab * CB / 8;
    const bool do_mask = k.mask_mode >= 0, do_deq = valid && k.deq_mode >= 0;
    uint32_t cbytes = 0, mbytes = 0;
#pragma unroll
    for (int f = 0; f < 4; ++f) {
        const int c = t + 4 * f;
        float2 s[4];
        chunk_decide<SAT, PPB>(P, G, f, k, s);
        if constexpr (CB == 8) {
            if (valid) *reinterpret_cast<uint2*>(codes + 8 * c) = chunk_pack_i8<MULT2>(s, k);
        } else if constexpr (CB == 4) {
            if (valid) *reinterpret_cast<uint32_t*>(codes + 4 * c) = chunk_pack<4>(s, k);
        } else if constexpr (CB == 2) {
            if (valid) *reinterpret_cast<uint16_t*>(codes + 2 * c) = (uint16_t)chunk_pack<2>(s, k);
        } else {
            cbytes |= chunk_pack<1>(s, k) << (8 * f);
        }
        if (do_mask) mbytes |= mask_byte<PPB>(P, G, f, k) << (8 * f);
        if (do_deq) {
            // yhat = q_b Delta + (1/2 - 2^(b-1)) Delta
            float2 y[4];
#pragma unroll
            for (int p = 0; p < 4; ++p) {
                const GroupK& g = G[(4 * f + p) / PPB];
                const float2 qb = __fadd2_rn(s[p], make_float2(-kMagic, -kMagic));
                y[p] = __ffma2_rn(qb, make_float2(g.delta, g.delta), make_float2(g.ch, g.ch));
            }
            const int64_t e = e_slab + 8 * c;
            if (k.deq_mode == 0) {
                *reinterpret_cast<uint4*>(A.deq + row * A.deq_row_bytes + 2 * e) =
                    make_uint4(pack_bf16x2(y[0].x, y[0].y), pack_bf16x2(y[1].x, y[1].y),
                               pack_bf16x2(y[2].x, y[2].y), pack_bf16x2(y[3].x, y[3].y));
            } else {
                uint8_t* dst = A.deq + row * A.deq_row_bytes + 4 * e;
                *reinterpret_cast<uint4*>(dst) = make_uint4(__float_as_uint(y[0].x), __float_as_uint(y[0].y),
                                                            __float_as_uint(y[1].x), __float_as_uint(y[1].y));
                *reinterpret_cast<uint4*>(dst + 16) = make_uint4(__float_as_uint(y[2].x), __float_as_uint(y[2].y),
                                                                 __float_as_uint(y[3].x), __float_as_uint(y[3].y));
            }
        }
    }
    if constexpr (CB == 1) {
        const uint32_t w = quad_transpose_bytes(cbytes, t);   // runs on every lane: it shuffles
        if (valid) *reinterpret_cast<uint32_t*>(codes + 4 * t) = w;
    }
    if (do_mask) {
        if (k.mask_mode == 0) {
            const uint32_t w = quad_transpose_bytes(mbytes, t);
            if (valid) *reinterpret_cast<uint32_t*>(A.mask + row * A.mask_row_bytes + e_slab / 8 + 4 * t) = w;
        } else if (valid) {
            uint8_t* dst = A.mask + row * A.mask_row_bytes + e_slab;
#pragma unroll
            for (int f = 0; f < 4; ++f) {
                const uint32_t bits = (mbytes >> (8 * f)) & 0xFFu;
                uint2 b;
                b.x = (bits & 1u) | ((bits >> 1) & 1u) << 8 | ((bits >> 2) & 1u) << 16 | ((bits >> 3) & 1u) << 24;
                b.y = ((bits >> 4) & 1u) | ((bits >> 5) & 1u) << 8 | ((bits >> 6) & 1u) << 16 | ((bits >> 7) & 1u) << 24;
                *reinterpret_cast<uint2*>(dst + 8 * (t + 4 * f)) = b;
            }
        }
    }
}

template <int HB>
constexpr int tmask_of() { return HB == 16 ? 0xB : 0xF; }   // HB = 16 leaves b4 alone

template <int HB, int CB, bool MULT2, bool SAT>
__global__ void __launch_bounds__(kThreads) quantize_tc_groups(const QuantArgs A) {
    constexpr int NBL = Blk<HB>::NBL, PPB = Blk<HB>::PPB;
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    const int64_t spr = A.cols / 128;
    const int64_t total = A.rows * spr;
    const int64_t warp0 = (int64_t(blockIdx.x) * kThreads + threadIdx.x) >> 5;
    const int64_t step = int64_t(gridDim.x) * (kThreads / 32) * 8;
    const BFrag B = make_bfrag(lane, tmask_of<HB>());
    auto src_of = [&](int64_t slab) -> const char* {
        if (A.dense) return A.x + slab * 256;
        const int64_t row = slab / spr, sc = slab - row * spr;
        return A.x + row * A.ld_x_bytes + sc * 256;
    };

    uint4 raw[4];
    if (warp0 * 8 + g < total) load_slab(src_of(warp0 * 8 + g), t, raw);
    else zero4(raw);
    for (int64_t s0 = warp0 * 8; s0 < total; s0 += step) {
        const int64_t slab = s0 + g;
        const bool valid = slab < total;
        float2 P[16];
        mma_stage(raw, B, P);
        if (slab + step < total) load_slab(src_of(slab + step), t, raw);
        else zero4(raw);
        reg_stages<HB>(P, lane);
        float ss[NBL];
        lane_sums<HB>(P, ss);
        GroupK G[NBL];
#pragma unroll
        for (int b = 0; b < NBL; ++b) {
            float v = ss[b] + __shfl_xor_sync(0xFFFFFFFFu, ss[b], 1);
            if constexpr (HB >= 32) v += __shfl_xor_sync(0xFFFFFFFFu, v, 2);
            if constexpr (HB == 256) v += __shfl_xor_sync(0xFFFFFFFFu, v, 4);
            G[b] = make_group(A.c, v);
        }
        const int64_t E = slab * 128;   // dense outputs: row 0 with a flat offset
        emit<PPB, CB, MULT2, SAT>(A, P, G, 0, E, t, valid);
        if (valid) {
            float* sp = A.scales + E / HB;
            if constexpr (HB == 256) {
                if ((g & 1) == 0 && t == 0) sp[0] = G[0].delta;
            } else if constexpr (HB == 128) {
                if (t == 0) sp[0] = G[0].delta;
            } else if constexpr (HB == 64) {
                if (t < 2) sp[t] = t ? G[1].delta : G[0].delta;   // block = b6
            } else if constexpr (HB == 32) {
                sp[t] = t == 0 ? G[0].delta : t == 1 ? G[1].delta : t == 2 ? G[2].delta : G[3].delta;   // block = f
            } else {
                // 16-blocks: index b4 + 2 (b5 + 2 b6) = (t >> 1) + 2 f; lanes t and t ^ 1 agree
                const int t1 = t >> 1, lo = (t & 1) ? 2 : 0;
                sp[t1 + 2 * lo] = (t & 1) ? G[2].delta : G[0].delta;
                sp[t1 + 2 * (lo + 1)] = (t & 1) ? G[3].delta : G[1].delta;
            }
        }
    }
}

// One RMS over each row of spr slabs. SUB = slabs per lane group (spr / 8 when
// spr >= 8, so a warp holds a whole row); for spr < 8 a warp step covers 8 / spr rows.
template <int HB, int CB, bool MULT2, bool SAT, int SUB>
__global__ void __launch_bounds__(kThreads) quantize_tc_rows(const QuantArgs A, int spr) {
    constexpr int NBL = Blk<HB>::NBL, PPB = Blk<HB>::PPB;
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    const int rps = SUB > 1 ? 1 : 8 / spr;          // rows per warp step
    const int r_in = SUB > 1 ? 0 : g / spr, sc0 = SUB > 1 ? g : g % spr;
    const int64_t warp0 = (int64_t(blockIdx.x) * kThreads + threadIdx.x) >> 5;
    const int64_t step = int64_t(gridDim.x) * (kThreads / 32) * rps;
    const BFrag B = make_bfrag(lane, tmask_of<HB>());
    auto src_of = [&](int64_t row, int u) -> const char* {
        return A.x + row * A.ld_x_bytes + int64_t(sc0 + 8 * u) * 256;
    };

    for (int64_t r0 = warp0 * rps; r0 < A.rows; r0 += step) {
        const int64_t row = r0 + r_in;
        const bool valid = row < A.rows;
        uint4 raw[SUB][4];
#pragma unroll
        for (int u = 0; u < SUB; ++u) {
            if (valid) load_slab(src_of(row, u), t, raw[u]);
            else zero4(raw[u]);
        }
        float2 P[SUB][16];
        float v = 0.0f;
#pragma unroll
        for (int u = 0; u < SUB; ++u) {
            mma_stage(raw[u], B, P[u]);
            reg_stages<HB>(P[u], lane);
            float ss[NBL];
            lane_sums<HB>(P[u], ss);
#pragma unroll
            for (int b = 0; b < NBL; ++b) v += ss[b];
        }
        // lanes of one row: the quad, and for spr > 1 the groups g of that row
        v += __shfl_xor_sync(0xFFFFFFFFu, v, 1);
        v += __shfl_xor_sync(0xFFFFFFFFu, v, 2);
        const int gspan = SUB > 1 ? 8 : spr;
        for (int s = 4; s < 4 * gspan; s <<= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, s);
        GroupK G[NBL];
        G[0] = make_group(A.c, v);
#pragma unroll
        for (int b = 1; b < NBL; ++b) G[b] = G[0];
#pragma unroll
        for (int u = 0; u < SUB; ++u)
            emit<PPB, CB, MULT2, SAT>(A, P[u], G, row, int64_t(sc0 + 8 * u) * 128, t, valid);
        if (valid && sc0 == 0 && t == 0) A.scales[row] = G[0].delta;
    }
}

template <int HB, int CB, bool MULT2, bool SAT>
cudaError_t launch_t(const QuantArgs& a, bool row_mode, cudaStream_t s) {
    const int sms = sm_count();
    if (row_mode) {
        const int spr = (int)(a.cols / 128);
        auto go = [&](auto fn, int64_t rows_per_warp) {
            const int64_t warps = (a.rows + rows_per_warp - 1) / rows_per_warp;
            const int64_t cap = int64_t(sms) * max_ctas_per_sm((const void*)fn, kThreads, 0);
            const int64_t want = (warps + kThreads / 32 - 1) / (kThreads / 32);
            fn<<<(int)(want < cap ? want : cap), kThreads, 0, s>>>(a, spr);
        };
        if (spr == 16) go(quantize_tc_rows<HB, CB, MULT2, SAT, 2>, 1);
        else if (spr == 8) go(quantize_tc_rows<HB, CB, MULT2, SAT, 1>, 1);
        else go(quantize_tc_rows<HB, CB, MULT2, SAT, 1>, 8 / spr);
    } else {
        const int64_t slabs = a.rows * (a.cols / 128);
        const int64_t warps = (slabs + 7) / 8;
        auto fn = quantize_tc_groups<HB, CB, MULT2, SAT>;
        const int64_t cap = int64_t(sms) * max_ctas_per_sm((const void*)fn, kThreads, 0);
        const int64_t want = (warps + kThreads / 32 - 1) / (kThreads / 32);
        fn<<<(int)(want < cap ? want : cap), kThreads, 0, s>>>(a);
    }
    return cudaGetLastError();
}

template <int HB, int CB, bool MULT2>
cudaError_t launch_sat(const QuantArgs& a, int bits, bool row, cudaStream_t s) {
    return bits <= 6 ? launch_t<HB, CB, MULT2, true>(a, row, s) : launch_t<HB, CB, MULT2, false>(a, row, s);
}

template <int HB>
cudaError_t launch_hb(const QuantArgs& a, int bits, int cb, bool row, cudaStream_t s) {
    switch (cb) {
        case 1: return launch_sat<HB, 1, false>(a, bits, row, s);
        case 2: return launch_sat<HB, 2, false>(a, bits, row, s);
        case 4: return launch_sat<HB, 4, false>(a, bits, row, s);
        case 8: return a.c.pack2_mult == 2 ? launch_sat<HB, 8, true>(a, bits, row, s)
                                           : launch_sat<HB, 8, false>(a, bits, row, s);
    }
    return cudaErrorInvalidValue;
}

}  // namespace tc

bool tc_path_ok(const QuantArgs& a, quest_dtype x_dtype, int had_block, int cbits, bool row_mode) {
    if (x_dtype != QUEST_BF16) return false;
    if (a.cols % 128 != 0 || (a.ld_x_bytes % 16) != 0 || (reinterpret_cast<uintptr_t>(a.x) & 15) != 0)
        return false;
    if (had_block == 256 && a.cols % 256 != 0) return false;
    // per-lane stores: codes 8 / 4 / 2 bytes per chunk (4-byte words for 1-bit), mask bits 4 bytes
    const uintptr_t code_align = cbits == 8 ? 8 : 4;
    if ((reinterpret_cast<uintptr_t>(a.codes) % (cbits == 2 ? 2 : code_align)) != 0) return false;
    if (a.mask && (reinterpret_cast<uintptr_t>(a.mask) % 4) != 0) return false;
    if (row_mode) {
        const int64_t spr = a.cols / 128;
        if (!(spr == 1 || spr == 2 || spr == 4 || spr == 8 || spr == 16)) return false;
        if (had_block == 256 && spr < 2) return false;
    }
    return true;
}

cudaError_t launch_quantize_tc(const QuantArgs& a, int had_block, int cbits, int bits, bool row_mode,
                               cudaStream_t stream) {
    switch (had_block) {
        case 16: return tc::launch_hb<16>(a, bits, cbits, row_mode, stream);
        case 32: return tc::launch_hb<32>(a, bits, cbits, row_mode, stream);
        case 64: return tc::launch_hb<64>(a, bits, cbits, row_mode, stream);
        case 128: return tc::launch_hb<128>(a, bits, cbits, row_mode, stream);
        case 256: return tc::launch_hb<256>(a, bits, cbits, row_mode, stream);
    }
    return cudaErrorInvalidValue;
}

}  // namespace quest

// QuEST quantizer for bf16 input with a tensor-core Hadamard factor (sm_100a).
//
// Same method as quantize_hs.cu (pith.science review of QuEST, "What carries
// the argument"; atlas.scime.ai summary, "Approach"): per Hadamard block
// y = H x / sqrt(n); per RMS group Delta = alpha_b r / 2^(b-1); q = clamp(floor(y /
// Delta)); trust mask m = [|t - (q+1/2)| <= T/2].
//
// Why. On B200 the CUDA-core quantizer is bound by instruction issue, not by
// HBM: its butterflies, bf16 unpacking and cross-lane shuffles are about a third
// of ~14.5 instructions per element. Here four of the seven index bits go through
// a 16 x 16 tensor-core product (quest_tc.cuh, which also gives the data layout).
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "quest_device.cuh"
#include "quest_emit.cuh"
#include "quest_internal.h"
#include "quest_tc.cuh"

namespace quest {
namespace tc {

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

// Quantise and store this lane's 32 values: chunks c = t + 4f of the slab whose
// first element is `e_slab` in row `row`.
// OUT selects the outputs at compile time for the common calls, so that the
// unrolled chunk loop is one straight block: 0 = as the call's flags say (mask,
// dequant and the trust form read at run time), 1 = codes + mask bits with T >= 1,
// no dequant, 2 = codes only.
template <int PPB, int CB, int FMT, bool SAT, int OUT>
__device__ __forceinline__ void emit(const QuantArgs& A, const float2 (&P)[16], const GroupK* G, int64_t row,
                                     int64_t e_slab, int t, bool valid) {
    const QuantConsts& k = A.c;
    uint8_t* codes = A.codes + row * A.codes_row_bytes + e_slab * CB / 8;
    const bool do_mask = OUT == 1 ? true : (OUT == 2 ? false : k.mask_mode >= 0);
    const bool do_deq = OUT != 0 ? false : (valid && k.deq_mode >= 0);
    const bool trust_ge1 = OUT == 1 ? true : k.trust_ge1 != 0;
    const bool mask_bits = OUT == 1 ? true : k.mask_mode == 0;
    uint32_t cbytes = 0, mbytes = 0;
#pragma unroll
    for (int f = 0; f < 4; ++f) {
        const int c = t + 4 * f;
        float2 y[4];   // dequantised values of the chunk (when requested)
        if constexpr (FMT >= 3) {
            // FP4 grid: FMT 3 packed E2M1 codes, FMT 4 int8 c = 2Q
            const uint32_t w4 = chunk_fp4<PPB>(P, G, f);
            if constexpr (FMT == 3) {
                if (valid) *reinterpret_cast<uint32_t*>(codes + 4 * c) = w4;
            } else {
                if (valid) *reinterpret_cast<uint2*>(codes + 8 * c) = fp4_operand_i8(w4);
            }
            if (do_mask && !trust_ge1) mbytes |= mask_byte_fp4_cell<PPB>(P, G, f, w4, k) << (8 * f);
            if (do_deq) fp4_dequant<PPB>(w4, G, f, y);
        } else {
            float2 s[4];
            chunk_decide<SAT, PPB>(P, G, f, k, s);
            if constexpr (CB == 8) {
                if (valid) *reinterpret_cast<uint2*>(codes + 8 * c) = chunk_pack_i8<FMT>(s, k);
            } else if constexpr (CB == 4) {
                if (valid) *reinterpret_cast<uint32_t*>(codes + 4 * c) = chunk_pack<4>(s, k);
            } else if constexpr (CB == 2) {
                if (valid) *reinterpret_cast<uint16_t*>(codes + 2 * c) = (uint16_t)chunk_pack<2>(s, k);
            } else {
                cbytes |= chunk_pack<1>(s, k) << (8 * f);
            }
            if (do_deq) {
                // yhat = q_b Delta + (1/2 - 2^(b-1)) Delta
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                    const GroupK& g = G[(4 * f + p) / PPB];
                    const float2 qb = __fadd2_rn(s[p], make_float2(-kMagic, -kMagic));
                    y[p] = __ffma2_rn(qb, make_float2(g.delta, g.delta), make_float2(g.ch, g.ch));
                }
            }
        }
        if (do_deq) {
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
    // trust mask bytes: one loop per form of the test, so that neither is predicated
    // into the other's path (the FP4 grid's general form was taken with its codes)
    if (do_mask) {
        if (trust_ge1) {
#pragma unroll
            for (int f = 0; f < 4; ++f) mbytes |= mask_byte_edge<PPB>(P, G, f) << (8 * f);
        } else if constexpr (FMT < 3) {
#pragma unroll
            for (int f = 0; f < 4; ++f) mbytes |= mask_byte_cell<PPB>(P, G, f, k) << (8 * f);
        }
    }
    if constexpr (CB == 1) {
        const uint32_t w = quad_transpose_bytes(cbytes, t);   // runs on every lane: it shuffles
        if (valid) *reinterpret_cast<uint32_t*>(codes + 4 * t) = w;
    }
    if (do_mask) {
        if (mask_bits) {
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


// Everything after the MMA for one slab of the group-RMS kernel.
template <int HB, int CB, int FMT, bool SAT, int OUT>
__device__ __forceinline__ void group_slab(const QuantArgs& A, float2 (&P)[16], int64_t slab, bool valid,
                                           int lane) {
    constexpr int NBL = Blk<HB>::NBL, PPB = Blk<HB>::PPB;
    const int g = lane >> 2, t = lane & 3;
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
    emit<PPB, CB, FMT, SAT, OUT>(A, P, G, 0, E, t, valid);
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

// Loads run kDepth warp steps ahead of the arithmetic (on B200 a second step in
// flight costs more in registers, and so in resident warps, than it hides).
constexpr int kDepth = 1;

template <int HB, int CB, int FMT, bool SAT, int OUT>
__global__ void __launch_bounds__(kThreads) quantize_tc_groups(const QuantArgs A) {
    pdl_wait();      // the previous kernel on the stream has completed
    pdl_trigger();   // the next one may be scheduled as CTAs of this one leave
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

    uint4 raw[kDepth][4];
#pragma unroll
    for (int d = 0; d < kDepth; ++d) {
        const int64_t slab = warp0 * 8 + g + d * step;
        if (slab < total) load_slab(src_of(slab), t, raw[d]);
        else zero4(raw[d]);
    }
    for (int64_t s0 = warp0 * 8; s0 < total; s0 += kDepth * step) {
#pragma unroll
        for (int d = 0; d < kDepth; ++d) {
            const int64_t base = s0 + d * step;
            if (base >= total) break;   // warp-uniform
            const int64_t slab = base + g;
            float2 P[16];
            mma_stage(raw[d], B, P);
            const int64_t next = slab + kDepth * step;
            if (next < total) load_slab(src_of(next), t, raw[d]);
            else zero4(raw[d]);
            group_slab<HB, CB, FMT, SAT, OUT>(A, P, slab, slab < total, lane);
        }
    }
}

// One RMS over each row of spr slabs. SUB = slabs per lane group (spr / 8 when
// spr >= 8, so a warp holds a whole row); for spr < 8 a warp step covers 8 / spr rows.
// As in the group kernel, the loads of a warp's next row are issued as soon as the
// MMA has consumed the current row's registers, so they land during its arithmetic.
// The rows of a second tensor (A.rows2 > 0, the other operand of a linear layer)
// follow those of the first in one virtual row space, so both take one launch.
template <int HB, int CB, int FMT, bool SAT, int SUB, int OUT>
__global__ void __launch_bounds__(kThreads, 3) quantize_tc_rows(const QuantArgs A, int spr) {
    pdl_wait();      // the previous kernel on the stream has completed
    pdl_trigger();   // the next one may be scheduled as CTAs of this one leave
    constexpr int NBL = Blk<HB>::NBL, PPB = Blk<HB>::PPB;
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    const int rps = SUB > 1 ? 1 : 8 / spr;          // rows per warp step
    const int r_in = SUB > 1 ? 0 : g / spr, sc0 = SUB > 1 ? g : g % spr;
    const int64_t warp0 = (int64_t(blockIdx.x) * kThreads + threadIdx.x) >> 5;
    const int64_t step = int64_t(gridDim.x) * (kThreads / 32) * rps;
    const int64_t total = A.rows + A.rows2;
    const BFrag B = make_bfrag(lane, tmask_of<HB>());
    auto load_row = [&](int64_t vrow, uint4 (&raw)[SUB][4]) {
        const char* src = vrow < A.rows ? A.x + vrow * A.ld_x_bytes : A.x2 + (vrow - A.rows) * A.ld_x_bytes;
#pragma unroll
        for (int u = 0; u < SUB; ++u) {
            if (vrow < total) load_slab(src + int64_t(sc0 + 8 * u) * 256, t, raw[u]);
            else zero4(raw[u]);
        }
    };

    uint4 raw[SUB][4];
    load_row(warp0 * rps + r_in, raw);
    for (int64_t r0 = warp0 * rps; r0 < total; r0 += step) {
        const int64_t vrow = r0 + r_in;
        const bool valid = vrow < total;
        float2 P[SUB][16];
#pragma unroll
        for (int u = 0; u < SUB; ++u) mma_stage(raw[u], B, P[u]);
        load_row(vrow + step, raw);
        float v = 0.0f;
#pragma unroll
        for (int u = 0; u < SUB; ++u) {
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
        // the tensor this row belongs to
        QuantArgs T = A;
        int64_t row = vrow;
        if (vrow >= A.rows) {
            T.codes = A.codes2;
            T.scales = A.scales2;
            row = vrow - A.rows;
        }
#pragma unroll
        for (int u = 0; u < SUB; ++u)
            emit<PPB, CB, FMT, SAT, OUT>(T, P[u], G, row, int64_t(sc0 + 8 * u) * 128, t, valid);
        if (valid && sc0 == 0 && t == 0) T.scales[row] = G[0].delta;
    }
}

template <int HB, int CB, int FMT, bool SAT, int OUT>
cudaError_t launch_out(const QuantArgs& a, bool row_mode, cudaStream_t s) {
    const int sms = sm_count();
    // grids never exceed the resident capacity (persistent, grid-stride)
    if (row_mode) {
        const int spr = (int)(a.cols / 128);
        auto go = [&](auto fn, int64_t rows_per_warp) {
            const int64_t warps = (a.rows + a.rows2 + rows_per_warp - 1) / rows_per_warp;
            const int64_t cap = int64_t(sms) * max_ctas_per_sm((const void*)fn, kThreads, 0);
            const int64_t want = (warps + kThreads / 32 - 1) / (kThreads / 32);
            return launch_pdl(fn, dim3((unsigned)(want < cap ? want : cap)), dim3(kThreads), 0, s, a, spr);
        };
        if (spr == 16) return go(quantize_tc_rows<HB, CB, FMT, SAT, 2, OUT>, 1);
        if (spr == 8) return go(quantize_tc_rows<HB, CB, FMT, SAT, 1, OUT>, 1);
        return go(quantize_tc_rows<HB, CB, FMT, SAT, 1, OUT>, 8 / spr);
    }
    const int64_t slabs = a.rows * (a.cols / 128);
    const int64_t warps = (slabs + 7) / 8;
    auto fn = quantize_tc_groups<HB, CB, FMT, SAT, OUT>;
    const int64_t cap = int64_t(sms) * max_ctas_per_sm((const void*)fn, kThreads, 0);
    const int64_t want = (warps + kThreads / 32 - 1) / (kThreads / 32);
    return launch_pdl(fn, dim3((unsigned)(want < cap ? want : cap)), dim3(kThreads), 0, s, a);
}

// The compile-time output sets (OUT 1, 2) for Hadamard block 128; everything else
// reads its flags at run time (OUT 0).
template <int HB, int CB, int FMT, bool SAT>
cudaError_t launch_t(const QuantArgs& a, bool row_mode, cudaStream_t s) {
    if constexpr (HB == 128 && FMT < 3) {
        const QuantConsts& k = a.c;
        if (k.deq_mode < 0 && k.mask_mode == 0 && k.trust_ge1) return launch_out<HB, CB, FMT, SAT, 1>(a, row_mode, s);
        if (k.deq_mode < 0 && k.mask_mode < 0) return launch_out<HB, CB, FMT, SAT, 2>(a, row_mode, s);
    }
    return launch_out<HB, CB, FMT, SAT, 0>(a, row_mode, s);
}

template <int HB, int CB, int FMT>
cudaError_t launch_sat(const QuantArgs& a, int bits, bool row, cudaStream_t s) {
    // E4M3 codes (b <= 4) and the FP4 grid (no integer decision path)
    if constexpr (FMT >= 2) return launch_t<HB, CB, FMT, true>(a, row, s);
    else return bits <= 6 ? launch_t<HB, CB, FMT, true>(a, row, s) : launch_t<HB, CB, FMT, false>(a, row, s);
}

template <int HB>
cudaError_t launch_hb(const QuantArgs& a, int bits, int cb, bool row, cudaStream_t s) {
    switch (cb) {
        case 1: return launch_sat<HB, 1, 0>(a, bits, row, s);
        case 2: return launch_sat<HB, 2, 0>(a, bits, row, s);
        case 4: return a.c.grid_fp4 ? launch_sat<HB, 4, 3>(a, bits, row, s) : launch_sat<HB, 4, 0>(a, bits, row, s);
        case 8: return a.c.grid_fp4 ? launch_sat<HB, 8, 4>(a, bits, row, s)
                : a.c.code_fp8 ? launch_sat<HB, 8, 2>(a, bits, row, s)
                                    : a.c.pack2_mult == 2 ? launch_sat<HB, 8, 1>(a, bits, row, s)
                                                          : launch_sat<HB, 8, 0>(a, bits, row, s);
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

// Direct-load QuEST quantizer on the interleaved half-slab layout (sm_100a).
//
// Same method as quantize_fwd.cu (pith.science review of QuEST, "What carries
// the argument"; atlas.scime.ai summary, "Approach"): per Hadamard block
// y = H x / sqrt(n); per RMS group r = sqrt(mean(y^2)), Delta = alpha_b r /
// 2^(b-1); q = clamp(floor(y/Delta)); trust mask m = [|t - (q+1/2)| <= T/2].
//
// Why this layout. On B200 a streaming pass over a ~64 MB tensor is limited by
// the bytes in flight from the first microsecond: plain 16-byte loads where each
// lane pair reads whole 32-byte sectors beat TMA or bulk staging into shared
// memory, which top out near 3.4 TB/s at this size. Each lane therefore loads
// its 8 chunks (16 bytes of bf16 each) straight into registers, in the
// interleaved half-slab layout of quest_device.cuh, and the transform runs with
// packed fp32x2 butterflies and one shuffle stage. Codes and mask bits are
// exchanged between the two lanes of a slab so that every store covers whole
// sectors.
//
//   quantize_hs_groups   one RMS per Hadamard block; each warp takes 16
//                        consecutive slabs per step (grid-stride loop).
//   quantize_hs_rows     one RMS per row for rows of 128 * {1, 2, 4, 8, 16}
//                        columns: a row is a segment of 2 * slabs lanes, so the
//                        row sum is a segmented shuffle reduction.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "quest_device.cuh"
#include "quest_emit.cuh"
#include "quest_internal.h"

namespace quest {
namespace hs {

constexpr int kThreads = 128;

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

// Raw 16-byte chunks of this lane's half-slab (chunk 2k + h of a slab): 8 for
// bf16 input, 16 for fp32.
template <typename Tin>
struct Raw {
    static constexpr int N = sizeof(Tin) == 2 ? 8 : 16;
    uint4 v[N];
};

template <typename Tin>
__device__ __forceinline__ void issue_loads(const char* src, int h, Raw<Tin>& r) {
    constexpr int kChunkBytes = 8 * sizeof(Tin);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const char* p = src + (2 * k + h) * kChunkBytes;
        if constexpr (sizeof(Tin) == 2) {
            r.v[k] = ld_stream_v4(p);
        } else {
            r.v[2 * k] = ld_stream_v4(p);
            r.v[2 * k + 1] = ld_stream_v4(p + 16);
        }
    }
}

template <typename Tin>
__device__ __forceinline__ void zero_raw(Raw<Tin>& r) {
#pragma unroll
    for (int k = 0; k < Raw<Tin>::N; ++k) r.v[k] = make_uint4(0u, 0u, 0u, 0u);
}

template <typename Tin>
__device__ __forceinline__ void unpack(const Raw<Tin>& r, float2 (&P)[32]) {
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        if constexpr (sizeof(Tin) == 2) {
            const uint4 v = r.v[k];
            P[4 * k + 0] = make_float2(bf16lo_to_f32(v.x), bf16hi_to_f32(v.x));
            P[4 * k + 1] = make_float2(bf16lo_to_f32(v.y), bf16hi_to_f32(v.y));
            P[4 * k + 2] = make_float2(bf16lo_to_f32(v.z), bf16hi_to_f32(v.z));
            P[4 * k + 3] = make_float2(bf16lo_to_f32(v.w), bf16hi_to_f32(v.w));
        } else {
            const uint4 a = r.v[2 * k], b = r.v[2 * k + 1];
            P[4 * k + 0] = make_float2(__uint_as_float(a.x), __uint_as_float(a.y));
            P[4 * k + 1] = make_float2(__uint_as_float(a.z), __uint_as_float(a.w));
            P[4 * k + 2] = make_float2(__uint_as_float(b.x), __uint_as_float(b.y));
            P[4 * k + 3] = make_float2(__uint_as_float(b.z), __uint_as_float(b.w));
        }
    }
}

// bf16 input is software-pipelined: the next step's 8 chunks (32 registers) are
// in flight while the current step computes. fp32 input would need 64 more
// registers for that and loads at the top of each step instead.
template <typename Tin>
struct Pipe {
    static constexpr bool kOn = sizeof(Tin) == 2;
    static constexpr int kMinBlocks = kOn ? 3 : 4;   // 128-thread blocks per SM
};

// Interleave 8 per-chunk bytes of the two lanes of a slab (lane h holds chunks
// 2k + h in byte k of (lo, hi)) into the 8 bytes this lane stores: chunks 0..7
// for h = 0, chunks 8..15 for h = 1.
__device__ __forceinline__ uint2 exchange_bytes(uint32_t lo, uint32_t hi, int h) {
    const uint32_t send = h ? lo : hi;
    const uint32_t r = __shfl_xor_sync(0xFFFFFFFFu, send, 1);
    const uint32_t own = h ? hi : lo;
    const uint32_t first = h ? r : own, second = h ? own : r;
    return make_uint2(prmt(first, second, 0x5140u), prmt(first, second, 0x7362u));
}

// Same for 16-bit fields: lane h holds chunks 2k + h in halfword k of (w0..w3);
// returns the 16 bytes this lane stores (chunks 0..7 or 8..15).
__device__ __forceinline__ uint4 exchange_halves(const uint32_t (&w)[4], int h) {
    const uint32_t s0 = h ? w[0] : w[2], s1 = h ? w[1] : w[3];
    const uint32_t r0 = __shfl_xor_sync(0xFFFFFFFFu, s0, 1);
    const uint32_t r1 = __shfl_xor_sync(0xFFFFFFFFu, s1, 1);
    const uint32_t o0 = h ? w[2] : w[0], o1 = h ? w[3] : w[1];
    const uint32_t f0 = h ? r0 : o0, g0 = h ? o0 : r0;
    const uint32_t f1 = h ? r1 : o1, g1 = h ? o1 : r1;
    return make_uint4(prmt(f0, g0, 0x5410u), prmt(f0, g0, 0x7632u), prmt(f1, g1, 0x5410u),
                      prmt(f1, g1, 0x7632u));
}

// Quantise and store the 64 values of this lane's half-slab. `e_slab` is the
// element index (within its row) of the slab's first element. One pass over
// the 8 chunks computes each chunk's decisions once and uses them for its
// codes, mask byte and dequantised values, so a chunk's registers die early.
template <int PPB, int CB, int FMT, bool SAT>
__device__ __forceinline__ void emit(const QuantArgs& A, const float2 (&P)[32], const GroupK* G,
                                     int64_t row, int64_t e_slab, int h, bool valid) {
    const QuantConsts& k = A.c;
    uint8_t* codes = A.codes + row * A.codes_row_bytes + e_slab * CB / 8;   // slab's codes
    const bool do_mask = k.mask_mode >= 0, do_deq = valid && k.deq_mode >= 0;
    uint32_t W[8];
    uint32_t mlo = 0, mhi = 0;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        float2 y[4];   // dequantised values of the chunk (when requested)
        uint32_t m = 0;
        if constexpr (FMT >= 3) {
            // FP4 grid: FMT 3 packed E2M1 codes, FMT 4 int8 c = 2Q
            const uint32_t w4 = chunk_fp4<PPB>(P, G, c);
            if constexpr (FMT == 3) {
                W[c] = w4;
            } else {
                if (valid) *reinterpret_cast<uint2*>(codes + (2 * c + h) * 8) = fp4_operand_i8(w4);
            }
            if (do_mask)
                m = k.trust_ge1 ? mask_byte_edge<PPB>(P, G, c) : mask_byte_fp4_cell<PPB>(P, G, c, w4, k);
            if (do_deq) fp4_dequant<PPB>(w4, G, c, y);
        } else {
            float2 s[4];
            chunk_decide<SAT, PPB>(P, G, c, k, s);
            if constexpr (CB == 8) {
                if (valid) *reinterpret_cast<uint2*>(codes + (2 * c + h) * 8) = chunk_pack_i8<FMT>(s, k);
            } else {
                W[c] = chunk_pack<CB>(s, k);
            }
            if (do_mask) m = mask_byte<PPB>(P, G, c, k);
            if (do_deq) {
                // yhat = q_b Delta + (1/2 - 2^(b-1)) Delta
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                    const GroupK& g = G[(4 * c + p) / PPB];
                    const float2 qb = __fadd2_rn(s[p], make_float2(-kMagic, -kMagic));
                    y[p] = __ffma2_rn(qb, make_float2(g.delta, g.delta), make_float2(g.ch, g.ch));
                }
            }
        }
        if (do_mask) {
            if (c < 4) mlo |= m << (8 * c);
            else mhi |= m << (8 * (c - 4));
        }
        if (do_deq) {
            const int64_t e = e_slab + (2 * c + h) * 8;
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

    // ---- codes: the two lanes of a slab trade fields so each store covers whole
    // sectors (the exchanges run on every lane: they shuffle)
    if constexpr (CB == 4) {
        // h = 0 stores bytes [0,16) and [32,48) of the slab's codes, h = 1 the others
        uint32_t recv[4];
        const int give0[4] = {2, 3, 6, 7}, give1[4] = {0, 1, 4, 5};
#pragma unroll
        for (int i = 0; i < 4; ++i) recv[i] = __shfl_xor_sync(0xFFFFFFFFu, h ? W[give1[i]] : W[give0[i]], 1);
        // h = 0: [W0 r0 W1 r1] [W4 r2 W5 r3]; h = 1: [r0 W2 r1 W3] [r2 W6 r3 W7]
        const uint4 a = h ? make_uint4(recv[0], W[2], recv[1], W[3]) : make_uint4(W[0], recv[0], W[1], recv[1]);
        const uint4 b = h ? make_uint4(recv[2], W[6], recv[3], W[7]) : make_uint4(W[4], recv[2], W[5], recv[3]);
        if (valid) {
            *reinterpret_cast<uint4*>(codes + 16 * h) = a;
            *reinterpret_cast<uint4*>(codes + 32 + 16 * h) = b;
        }
    } else if constexpr (CB == 2) {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) w[i] = W[2 * i] | (W[2 * i + 1] << 16);
        const uint4 o = exchange_halves(w, h);
        if (valid) *reinterpret_cast<uint4*>(codes + 16 * h) = o;
    } else if constexpr (CB == 1) {
        const uint32_t lo = W[0] | (W[1] << 8) | (W[2] << 16) | (W[3] << 24);
        const uint32_t hi = W[4] | (W[5] << 8) | (W[6] << 16) | (W[7] << 24);
        const uint2 o = exchange_bytes(lo, hi, h);
        if (valid) *reinterpret_cast<uint2*>(codes + 8 * h) = o;
    }

    // ---- trust mask (1 = kept): 8 mask bytes = chunks 8h .. 8h+7 after the exchange
    if (do_mask) {
        const uint2 m = exchange_bytes(mlo, mhi, h);
        if (valid) {
            if (k.mask_mode == 0) {
                *reinterpret_cast<uint2*>(A.mask + row * A.mask_row_bytes + e_slab / 8 + 8 * h) = m;
            } else {
                uint8_t* dst = A.mask + row * A.mask_row_bytes + e_slab + 64 * h;
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const uint32_t bits = ((q < 4 ? m.x : m.y) >> (8 * (q & 3))) & 0xFFu;
                    uint2 b;
                    b.x = (bits & 1u) | ((bits >> 1) & 1u) << 8 | ((bits >> 2) & 1u) << 16 | ((bits >> 3) & 1u) << 24;
                    b.y = ((bits >> 4) & 1u) | ((bits >> 5) & 1u) << 8 | ((bits >> 6) & 1u) << 16 | ((bits >> 7) & 1u) << 24;
                    *reinterpret_cast<uint2*>(dst + 8 * q) = b;
                }
            }
        }
    }
}

// Sum of squares of the pairs of each block this lane holds (4 partial sums).
template <int PPB>
__device__ __forceinline__ void block_sums(const float2 (&P)[32], float (&ss)[32 / PPB]) {
    constexpr int BPL = 32 / PPB;
#pragma unroll
    for (int b = 0; b < BPL; ++b) {
        constexpr int NA = PPB >= 4 ? 4 : PPB;
        float2 acc[NA];
#pragma unroll
        for (int u = 0; u < NA; ++u) acc[u] = make_float2(0.0f, 0.0f);
#pragma unroll
        for (int j = b * PPB; j < (b + 1) * PPB; ++j) acc[j % NA] = __ffma2_rn(P[j], P[j], acc[j % NA]);
#pragma unroll
        for (int u = 1; u < NA; ++u) acc[0] = __fadd2_rn(acc[0], acc[u]);
        ss[b] = acc[0].x + acc[0].y;
    }
}

template <typename Tin, int HB, int CB, int FMT, bool SAT>
__global__ void __launch_bounds__(kThreads, Pipe<Tin>::kMinBlocks) quantize_hs_groups(const QuantArgs A) {
    pdl_wait();      // the previous kernel on the stream has completed
    pdl_trigger();   // the next one may be scheduled as CTAs of this one leave
    constexpr int PPB = (HB >= 128 ? 128 : HB) / 4;   // pairs of one block in this lane
    constexpr int BPL = 32 / PPB;
    const int lane = threadIdx.x & 31, h = lane & 1, pw = lane >> 1;
    const int64_t spr = A.cols / 128;
    const int64_t total = A.rows * spr;
    const int64_t warp0 = (int64_t(blockIdx.x) * kThreads + threadIdx.x) >> 5;
    const int64_t step = int64_t(gridDim.x) * (kThreads / 32) * 16;
    auto src_of = [&](int64_t slab) -> const char* {
        if (A.dense) return A.x + slab * 128 * int64_t(sizeof(Tin));
        const int64_t row = slab / spr, sc = slab - row * spr;
        return A.x + row * A.ld_x_bytes + sc * 128 * int64_t(sizeof(Tin));
    };

    Raw<Tin> raw;
    if constexpr (Pipe<Tin>::kOn) {
        if (warp0 * 16 + pw < total) issue_loads<Tin>(src_of(warp0 * 16 + pw), h, raw);
        else zero_raw<Tin>(raw);
    }
    for (int64_t s0 = warp0 * 16; s0 < total; s0 += step) {
        const int64_t slab = s0 + pw;
        const bool valid = slab < total;
        const int64_t E = slab * 128;        // flat element offset: the outputs are dense
        float2 P[32];
        if constexpr (Pipe<Tin>::kOn) {
            unpack<Tin>(raw, P);
            if (slab + step < total) issue_loads<Tin>(src_of(slab + step), h, raw);
            else zero_raw<Tin>(raw);
        } else {
            if (valid) issue_loads<Tin>(src_of(slab), h, raw);
            else zero_raw<Tin>(raw);
            unpack<Tin>(raw, P);
        }
        fwht_interleaved<HB>(P, lane);
        float ss[BPL];
        block_sums<PPB>(P, ss);
        GroupK G[BPL];
#pragma unroll
        for (int b = 0; b < BPL; ++b) {
            float v = ss[b] + __shfl_xor_sync(0xFFFFFFFFu, ss[b], 1);
            if constexpr (HB >= 256) v += __shfl_xor_sync(0xFFFFFFFFu, v, 2);
            G[b] = make_group(A.c, v);
        }
        // row 0 with a flat offset addresses every dense output
        emit<PPB, CB, FMT, SAT>(A, P, G, 0, E, h, valid);
        if (valid) {
            float* sp = A.scales + E / HB;   // scales are dense [rows, cols / HB]
            if constexpr (HB == 256) {
                if ((pw & 1) == 0 && h == 0) sp[0] = G[0].delta;
            } else if constexpr (HB == 128) {
                if (h == 0) sp[0] = G[0].delta;
            } else {
                // this slab holds 128/HB blocks; lane h writes half of them
                constexpr int NB = 128 / HB, MINE = NB / 2;
#pragma unroll
                for (int i = 0; i < MINE; ++i) sp[MINE * h + i] = h ? G[MINE + i].delta : G[i].delta;
            }
        }
    }
}

template <typename Tin, int HB, int CB, int FMT, bool SAT>
__global__ void __launch_bounds__(kThreads, Pipe<Tin>::kMinBlocks) quantize_hs_rows(const QuantArgs A, int spr) {
    pdl_wait();      // the previous kernel on the stream has completed
    pdl_trigger();   // the next one may be scheduled as CTAs of this one leave
    constexpr int PPB = (HB >= 128 ? 128 : HB) / 4;
    constexpr int BPL = 32 / PPB;
    const int lane = threadIdx.x & 31, h = lane & 1;
    const int lpr = 2 * spr;                 // lanes per row, a power of two <= 32
    const int rpw = 32 / lpr;                // rows per warp
    const int r_in_w = lane / lpr, sc = (lane % lpr) >> 1;
    const int64_t warp0 = (int64_t(blockIdx.x) * kThreads + threadIdx.x) >> 5;
    const int64_t step = int64_t(gridDim.x) * (kThreads / 32) * rpw;
    auto src_of = [&](int64_t row) -> const char* {
        return A.x + row * A.ld_x_bytes + int64_t(sc) * 128 * int64_t(sizeof(Tin));
    };

    Raw<Tin> raw;
    if constexpr (Pipe<Tin>::kOn) {
        if (warp0 * rpw + r_in_w < A.rows) issue_loads<Tin>(src_of(warp0 * rpw + r_in_w), h, raw);
        else zero_raw<Tin>(raw);
    }
    for (int64_t r0 = warp0 * rpw; r0 < A.rows; r0 += step) {
        const int64_t row = r0 + r_in_w;
        const bool valid = row < A.rows;
        float2 P[32];
        if constexpr (Pipe<Tin>::kOn) {
            unpack<Tin>(raw, P);
            if (row + step < A.rows) issue_loads<Tin>(src_of(row + step), h, raw);
            else zero_raw<Tin>(raw);
        } else {
            if (valid) issue_loads<Tin>(src_of(row), h, raw);
            else zero_raw<Tin>(raw);
            unpack<Tin>(raw, P);
        }
        fwht_interleaved<HB>(P, lane);
        float ss[BPL];
        block_sums<PPB>(P, ss);
        float v = 0.0f;
#pragma unroll
        for (int b = 0; b < BPL; ++b) v += ss[b];
        for (int s = 1; s < lpr; s <<= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, s);
        GroupK G[BPL];
        G[0] = make_group(A.c, v);
#pragma unroll
        for (int b = 1; b < BPL; ++b) G[b] = G[0];
        emit<PPB, CB, FMT, SAT>(A, P, G, row, int64_t(sc) * 128, h, valid);
        if (valid && sc == 0 && h == 0) A.scales[row] = G[0].delta;
    }
}

template <typename Tin, int HB, int CB, int FMT, bool SAT>
cudaError_t launch_t(const QuantArgs& a, bool row_mode, cudaStream_t s) {
    const int sms = sm_count();
    if (row_mode) {
        const int spr = (int)(a.cols / 128);
        const int rpw = 16 / spr;
        const int64_t warps = (a.rows + rpw - 1) / rpw;
        auto fn = quantize_hs_rows<Tin, HB, CB, FMT, SAT>;
        const int64_t cap = int64_t(sms) * max_ctas_per_sm((const void*)fn, kThreads, 0);
        const int64_t want = (warps + kThreads / 32 - 1) / (kThreads / 32);
        return launch_pdl(fn, dim3((unsigned)(want < cap ? want : cap)), dim3(kThreads), 0, s, a, spr);
    } else {
        const int64_t slabs = a.rows * (a.cols / 128);
        const int64_t warps = (slabs + 15) / 16;
        auto fn = quantize_hs_groups<Tin, HB, CB, FMT, SAT>;
        const int64_t cap = int64_t(sms) * max_ctas_per_sm((const void*)fn, kThreads, 0);
        const int64_t want = (warps + kThreads / 32 - 1) / (kThreads / 32);
        return launch_pdl(fn, dim3((unsigned)(want < cap ? want : cap)), dim3(kThreads), 0, s, a);
    }
}

template <typename Tin, int HB, int CB, int FMT>
cudaError_t launch_sat(const QuantArgs& a, int bits, bool row, cudaStream_t s) {
    // E4M3 codes (b <= 4) and the FP4 grid (no integer decision path)
    if constexpr (FMT >= 2) return launch_t<Tin, HB, CB, FMT, true>(a, row, s);
    else return bits <= 6 ? launch_t<Tin, HB, CB, FMT, true>(a, row, s)
                          : launch_t<Tin, HB, CB, FMT, false>(a, row, s);
}

template <typename Tin, int HB>
cudaError_t launch_hb(const QuantArgs& a, int bits, int cb, bool row, cudaStream_t s) {
    switch (cb) {
        case 1: return launch_sat<Tin, HB, 1, 0>(a, bits, row, s);
        case 2: return launch_sat<Tin, HB, 2, 0>(a, bits, row, s);
        case 4: return a.c.grid_fp4 ? launch_sat<Tin, HB, 4, 3>(a, bits, row, s)
                                    : launch_sat<Tin, HB, 4, 0>(a, bits, row, s);
        case 8: return a.c.grid_fp4 ? launch_sat<Tin, HB, 8, 4>(a, bits, row, s)
                : a.c.code_fp8 ? launch_sat<Tin, HB, 8, 2>(a, bits, row, s)
                                    : a.c.pack2_mult == 2 ? launch_sat<Tin, HB, 8, 1>(a, bits, row, s)
                                                          : launch_sat<Tin, HB, 8, 0>(a, bits, row, s);
    }
    return cudaErrorInvalidValue;
}

template <typename Tin>
cudaError_t launch_dtype(const QuantArgs& a, int bits, int hb, int cb, bool row, cudaStream_t s) {
    switch (hb) {
        case 16: return launch_hb<Tin, 16>(a, bits, cb, row, s);
        case 32: return launch_hb<Tin, 32>(a, bits, cb, row, s);
        case 64: return launch_hb<Tin, 64>(a, bits, cb, row, s);
        case 128: return launch_hb<Tin, 128>(a, bits, cb, row, s);
        case 256: return launch_hb<Tin, 256>(a, bits, cb, row, s);
    }
    return cudaErrorInvalidValue;
}

}  // namespace hs

bool hs_path_ok(const QuantArgs& a, int had_block, int cbits, bool row_mode) {
    if (a.cols % 128 != 0 || (a.ld_x_bytes % 16) != 0 || (reinterpret_cast<uintptr_t>(a.x) & 15) != 0)
        return false;
    if (had_block == 256 && a.cols % 256 != 0) return false;
    // vector stores: codes 16 bytes (8 for 1-bit and for 8-bit chunks), mask 8 bytes
    const uintptr_t code_align = (cbits == 1 || cbits == 8) ? 8 : 16;
    if ((reinterpret_cast<uintptr_t>(a.codes) % code_align) != 0) return false;
    if (a.mask && (reinterpret_cast<uintptr_t>(a.mask) % 8) != 0) return false;
    if (row_mode) {
        const int64_t spr = a.cols / 128;
        if (spr > 16 || (spr & (spr - 1)) != 0) return false;
        if (had_block == 256 && spr < 2) return false;
    }
    return true;
}

cudaError_t launch_quantize_hs(const QuantArgs& a, quest_dtype x_dtype, int had_block, int cbits,
                               int bits, bool row_mode, cudaStream_t stream) {
    if (x_dtype == QUEST_BF16) return hs::launch_dtype<__nv_bfloat16>(a, bits, had_block, cbits, row_mode, stream);
    return hs::launch_dtype<float>(a, bits, had_block, cbits, row_mode, stream);
}

}  // namespace quest

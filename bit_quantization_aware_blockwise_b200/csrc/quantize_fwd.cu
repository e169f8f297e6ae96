// QuEST forward quantizer kernels (sm_100a).
//
// Method (pith.science review of QuEST, "What carries the argument";
// atlas.scime.ai summary, "Approach"): per Hadamard block, y = H x / sqrt(n);
// per RMS group, r = sqrt(mean(y^2)); Delta = alpha_b r / 2^(b-1);
// q = clamp(floor(y / Delta)); yhat = (q + 1/2) Delta; trust mask
// m = [|y/Delta - (q + 1/2)| <= T/2].
//
// The pass is bound by HBM bandwidth and by instruction issue (about 2.7
// bytes move per element at b = 4, so every instruction per element counts).
// The kernels therefore:
//   * keep one Hadamard block in the registers of a team of lanes
//     (quest_device.cuh) and transform it with in-register butterflies plus
//     two shuffle stages; the 1/sqrt(n) factor is folded into the group
//     constants, never applied per element;
//   * compute floor(y * inv) + 2^23*1.5 with one round-down FMA, clamp it with
//     two min/max, and pack codes with one integer multiply-add per element:
//     the packed word is sum_i bits(s_i) * mult * 2^(cb*i) + const (mod 2^32)
//     followed by an XOR that turns the biased fields into two's complement;
//   * for T >= 1 take the mask as the sign of |y_u| - thr (m = [|t| <= edge],
//     equivalent to the half-interval rule whenever T >= 1), accumulated into a
//     bit word with one funnel shift per element.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "quest_device.cuh"
#include "quest_internal.h"
#include "quest_sync.cuh"
#include "quest_emit.cuh"

namespace quest {
namespace {

constexpr int kThreads = 256;

// Quantise, pack and store one team's share (K chunks) of one Hadamard block.
//   v      transformed values y_u (unnormalised), team layout
//   delta  Delta of the block's RMS group; inv_u = 1/(sqrt(HB) Delta) or 0
//   thr_u  edge * sqrt(HB) * Delta (or +inf for an all-zero group)
//   codes/mask/deq   pointers to the block's first element in each output
template <int CB, int K, int LPB>
__device__ __forceinline__ void emit_block(const QuantConsts& c, const float (&v)[K][8],
                                           float delta, float inv_u, float thr_u, int sub,
                                           uint8_t* codes, uint8_t* mask, uint8_t* deq) {
#pragma unroll
    for (int j = 0; j < K; ++j) {
        const int e0 = (sub + LPB * j) * 8;  // first element of this chunk in the block
        float s[8];
#pragma unroll
        for (int i = 0; i < 8; ++i)
            s[i] = fminf(fmaxf(__fmaf_rd(v[j][i], inv_u, kMagic), c.s_lo), c.s_hi);

        // ---- codes
        if constexpr (CB == 8) {
            uint32_t w0 = c.pack_add, w1 = c.pack_add;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                w0 += __float_as_uint(s[i]) * (c.pack_mult << (8 * i));
                w1 += __float_as_uint(s[4 + i]) * (c.pack_mult << (8 * i));
            }
            uint2 w = make_uint2(w0 ^ c.pack_xor, w1 ^ c.pack_xor);
            *reinterpret_cast<uint2*>(codes + e0) = w;
        } else {
            uint32_t w = c.pack_add;
#pragma unroll
            for (int i = 0; i < 8; ++i) w += __float_as_uint(s[i]) * (c.pack_mult << (CB * i));
            w ^= c.pack_xor;
            if constexpr (CB == 4) *reinterpret_cast<uint32_t*>(codes + e0 / 2) = w;
            if constexpr (CB == 2) *reinterpret_cast<uint16_t*>(codes + e0 / 4) = (uint16_t)w;
            if constexpr (CB == 1) codes[e0 / 8] = (uint8_t)w;
        }

        // ---- trust mask (bit i of m = element e0 + i; 1 = trusted)
        if (c.mask_mode >= 0) {
            uint32_t m = 0;
            if (c.trust_ge1) {
#pragma unroll
                for (int i = 7; i >= 0; --i)
                    m = __funnelshift_l(__float_as_uint(fabsf(v[j][i]) - thr_u), m, 1);
            } else if (inv_u == 0.0f) {
                m = 0xFFu;  // all-zero group: every entry trusted
            } else {
#pragma unroll
                for (int i = 7; i >= 0; --i) {
                    float t = v[j][i] * inv_u;
                    float e = (t - (s[i] - kMagic)) - 0.5f;
                    m = __funnelshift_l(__float_as_uint(fabsf(e) - c.half_trust), m, 1);
                }
            }
            if (c.mask_mode == 0) {
                mask[e0 / 8] = (uint8_t)m;
            } else {
                uint2 b;
                b.x = (m & 1u) | ((m >> 1) & 1u) << 8 | ((m >> 2) & 1u) << 16 | ((m >> 3) & 1u) << 24;
                b.y = ((m >> 4) & 1u) | ((m >> 5) & 1u) << 8 | ((m >> 6) & 1u) << 16 |
                      ((m >> 7) & 1u) << 24;
                *reinterpret_cast<uint2*>(mask + e0) = b;
            }
        }

        // ---- dequantised value yhat = (q + 1/2) Delta, Hadamard domain
        if (c.deq_mode >= 0) {
            float yh[8];
            const float half_d = 0.5f * delta;
#pragma unroll
            for (int i = 0; i < 8; ++i) yh[i] = fmaf(s[i] - kMagic, delta, half_d);
            if (c.deq_mode == 0)
                ChunkIO<__nv_bfloat16>::store(deq + 2 * e0, yh);
            else
                ChunkIO<float>::store(deq + 4 * e0, yh);
        }
    }
}

// Group constants from the block's (or row's) sum of y_u^2.
__device__ __forceinline__ void group_consts(const QuantConsts& c, float ss, float& delta,
                                             float& inv_u, float& thr_u) {
    const float r = sqrtf(ss * c.inv_count);
    delta = c.c_delta * r;
    if (delta > 0.0f) {
        const float sd = c.sqrt_hb * delta;
        inv_u = __frcp_rn(sd);
        thr_u = c.edge * sd;
    } else {
        inv_u = 0.0f;
        thr_u = __int_as_float(0x7F800000);  // +inf: every |y| - thr < 0
    }
}

// One RMS group per Hadamard block. Each warp handles TPW = 32/LPB consecutive
// blocks per step (flattened over rows), a grid-stride loop over warps; loop
// bounds are warp-uniform so every shuffle has all 32 lanes.
template <typename Tin, int HB, int CB>
__global__ void __launch_bounds__(kThreads) quantize_groups_kernel(const QuantArgs a) {
    using S = TeamShape<HB>;
    constexpr int K = S::K, LPB = S::LPB, TPW = 32 / LPB;
    constexpr int kElem = sizeof(Tin);
    const int lane = threadIdx.x & 31, sub = lane % LPB;
    const int64_t bpr = a.cols / HB;
    const int64_t total = a.rows * bpr;
    const int64_t warp0 = (int64_t(blockIdx.x) * kThreads + threadIdx.x) >> 5;
    const int64_t wstride = int64_t(gridDim.x) * (kThreads / 32);

    for (int64_t wb = warp0 * TPW; wb < total; wb += wstride * TPW) {
        const int64_t blk = wb + lane / LPB;
        const bool valid = blk < total;
        float v[K][8];
        if (valid) {
            const char* xb;
            if (a.dense) {
                xb = a.x + blk * HB * kElem;
            } else {
                const int64_t row = blk / bpr, bc = blk - row * bpr;
                xb = a.x + row * a.ld_x_bytes + bc * HB * kElem;
            }
#pragma unroll
            for (int j = 0; j < K; ++j) ChunkIO<Tin>::load(xb + (sub + LPB * j) * 8 * kElem, v[j]);
        } else {
#pragma unroll
            for (int j = 0; j < K; ++j)
#pragma unroll
                for (int i = 0; i < 8; ++i) v[j][i] = 0.0f;
        }
        fwht_team<K, LPB>(v, lane);
        float ss = 0.0f;
#pragma unroll
        for (int j = 0; j < K; ++j)
#pragma unroll
            for (int i = 0; i < 8; ++i) ss = fmaf(v[j][i], v[j][i], ss);
        ss = team_sum<LPB>(ss);
        float delta, inv_u, thr_u;
        group_consts(a.c, ss, delta, inv_u, thr_u);
        if (valid) {
            // outputs are dense [rows, cols]: the flat block index addresses them
            const int64_t e = blk * HB;
            emit_block<CB, K, LPB>(a.c, v, delta, inv_u, thr_u, sub, a.codes + e * CB / 8,
                                   a.mask ? a.mask + (a.c.mask_mode == 0 ? e / 8 : e) : nullptr,
                                   a.deq ? a.deq + e * (a.c.deq_mode == 0 ? 2 : 4) : nullptr);
            if (sub == 0) a.scales[blk] = delta;
        }
    }
}

// One RMS group per row (rms_group == cols). A CTA of 8 warps handles 8/WPR
// rows; WPR warps share a row, each holding P passes of TPW blocks in
// registers, so that the whole row is read once. Row sums meet in shared memory.
template <typename Tin, int HB, int CB, int P>
__global__ void __launch_bounds__(kThreads) quantize_rows_kernel(const QuantArgs a, int wpr) {
    using S = TeamShape<HB>;
    constexpr int K = S::K, LPB = S::LPB, TPW = 32 / LPB;
    constexpr int kElem = sizeof(Tin);
    __shared__ float partial[2][kThreads / 32];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int sub = lane % LPB, team = lane / LPB;
    const int rows_per_cta = (kThreads / 32) / wpr;
    const int row_in_cta = warp / wpr, w_in_row = warp % wpr;
    const int64_t bpr = a.cols / HB;
    int buf = 0;

    for (int64_t row0 = int64_t(blockIdx.x) * rows_per_cta; row0 < a.rows;
         row0 += int64_t(gridDim.x) * rows_per_cta, buf ^= 1) {
        const int64_t row = row0 + row_in_cta;
        const bool row_ok = row < a.rows;
        float v[P][K][8];
        float ss = 0.0f;
#pragma unroll
        for (int p = 0; p < P; ++p) {
            const int64_t bc = int64_t(w_in_row * TPW + team) + int64_t(p) * wpr * TPW;
            if (row_ok && bc < bpr) {
                const char* xb = a.x + row * a.ld_x_bytes + bc * HB * kElem;
#pragma unroll
                for (int j = 0; j < K; ++j)
                    ChunkIO<Tin>::load(xb + (sub + LPB * j) * 8 * kElem, v[p][j]);
            } else {
#pragma unroll
                for (int j = 0; j < K; ++j)
#pragma unroll
                    for (int i = 0; i < 8; ++i) v[p][j][i] = 0.0f;
            }
            fwht_team<K, LPB>(v[p], lane);
#pragma unroll
            for (int j = 0; j < K; ++j)
#pragma unroll
                for (int i = 0; i < 8; ++i) ss = fmaf(v[p][j][i], v[p][j][i], ss);
        }
#pragma unroll
        for (int s = 1; s < 32; s <<= 1) ss += __shfl_xor_sync(0xFFFFFFFFu, ss, s);
        if (lane == 0) partial[buf][warp] = ss;
        __syncthreads();
        float tot = 0.0f;
        for (int w = 0; w < wpr; ++w) tot += partial[buf][row_in_cta * wpr + w];
        // (the other buffer is written next iteration, after this barrier)
        float delta, inv_u, thr_u;
        group_consts(a.c, tot, delta, inv_u, thr_u);
        if (row_ok) {
#pragma unroll
            for (int p = 0; p < P; ++p) {
                const int64_t bc = int64_t(w_in_row * TPW + team) + int64_t(p) * wpr * TPW;
                if (bc < bpr) {
                    const int64_t e = bc * HB;
                    emit_block<CB, K, LPB>(
                        a.c, v[p], delta, inv_u, thr_u, sub,
                        a.codes + row * a.codes_row_bytes + e * CB / 8,
                        a.mask ? a.mask + row * a.mask_row_bytes + (a.c.mask_mode == 0 ? e / 8 : e)
                               : nullptr,
                        a.deq ? a.deq + row * a.deq_row_bytes + e * (a.c.deq_mode == 0 ? 2 : 4)
                              : nullptr);
                }
            }
            if (w_in_row == 0 && lane == 0) a.scales[row] = delta;
        }
    }
}

template <typename Tin, int HB, int CB>
cudaError_t launch_groups(const QuantArgs& a, cudaStream_t stream) {
    using S = TeamShape<HB>;
    constexpr int TPW = 32 / S::LPB;
    const int64_t total = a.rows * (a.cols / HB);
    const int64_t warps = (total + TPW - 1) / TPW;
    const int64_t want = (warps + (kThreads / 32) - 1) / (kThreads / 32);
    auto fn = quantize_groups_kernel<Tin, HB, CB>;
    const int64_t cap = int64_t(sm_count()) * max_ctas_per_sm((const void*)fn, kThreads, 0);
    const int grid = (int)(want < cap ? want : cap);
    fn<<<grid, kThreads, 0, stream>>>(a);
    return cudaGetLastError();
}

template <typename Tin, int HB, int CB>
cudaError_t launch_rows(const QuantArgs& a, cudaStream_t stream) {
    using S = TeamShape<HB>;
    constexpr int TPW = 32 / S::LPB;
    const int64_t bpr = a.cols / HB;
    // smallest warps-per-row with at most 2 passes of TPW blocks per warp
    int wpr = 1;
    while (wpr < 8 && int64_t(2) * wpr * TPW < bpr) wpr *= 2;
    const bool one_pass = int64_t(wpr) * TPW >= bpr;
    const int rows_per_cta = 8 / wpr;
    const int64_t want = (a.rows + rows_per_cta - 1) / rows_per_cta;
    const void* fnp = one_pass ? (const void*)quantize_rows_kernel<Tin, HB, CB, 1>
                               : (const void*)quantize_rows_kernel<Tin, HB, CB, 2>;
    const int64_t cap = int64_t(sm_count()) * max_ctas_per_sm(fnp, kThreads, 0);
    const int grid = (int)(want < cap ? want : cap);
    if (one_pass)
        quantize_rows_kernel<Tin, HB, CB, 1><<<grid, kThreads, 0, stream>>>(a, wpr);
    else
        quantize_rows_kernel<Tin, HB, CB, 2><<<grid, kThreads, 0, stream>>>(a, wpr);
    return cudaGetLastError();
}

template <typename Tin, int HB>
cudaError_t launch_hb(const QuantArgs& a, int cbits, bool row_mode, cudaStream_t s) {
    switch (cbits) {
        case 1: return row_mode ? launch_rows<Tin, HB, 1>(a, s) : launch_groups<Tin, HB, 1>(a, s);
        case 2: return row_mode ? launch_rows<Tin, HB, 2>(a, s) : launch_groups<Tin, HB, 2>(a, s);
        case 4: return row_mode ? launch_rows<Tin, HB, 4>(a, s) : launch_groups<Tin, HB, 4>(a, s);
        case 8: return row_mode ? launch_rows<Tin, HB, 8>(a, s) : launch_groups<Tin, HB, 8>(a, s);
    }
    return cudaErrorInvalidValue;
}

template <typename Tin>
cudaError_t launch_dtype(const QuantArgs& a, int hb, int cbits, bool row_mode, cudaStream_t s) {
    switch (hb) {
        case 16: return launch_hb<Tin, 16>(a, cbits, row_mode, s);
        case 32: return launch_hb<Tin, 32>(a, cbits, row_mode, s);
        case 64: return launch_hb<Tin, 64>(a, cbits, row_mode, s);
        case 128: return launch_hb<Tin, 128>(a, cbits, row_mode, s);
        case 256: return launch_hb<Tin, 256>(a, cbits, row_mode, s);
    }
    return cudaErrorInvalidValue;
}

}  // namespace
// ===========================================================================
// TMA-staged quantizer, one RMS group per Hadamard block (rows whose length is
// a multiple of 128).
//
// One persistent CTA per SM: warp 0 streams tiles of whole 128-element slabs
// into a ring of shared-memory stages with 3-D TMA copies (128-byte swizzle);
// 11 consumer warps (8 for fp32 input) take each stage, two lanes per slab
// (half-slab layout, quest_device.cuh), transform with packed fp32x2
// butterflies and write codes, mask bits, scales and (optionally) dequantised
// values to global memory with 8- and 16-byte vector stores. A stage is
// released as soon as its consumers have its data in registers.
//
// Per element, the decision path is: u = sat(y_u * a + c) (one FMA that also
// clamps), s = fma_rd(u, 2^b (1 - 2^-23), 1.5*2^23) (packed: the biased code
// q + 2^(b-1) in the low mantissa bits), one integer multiply-add to pack, and
// for the mask one packed FMA y_u^2 - thr^2 whose sign is the trust bit. The
// saturating form moves a decision boundary by at most 2^(b-23) (plus one
// rounding of u), far inside the 1e-5 band, so it is used for b <= 6; b = 7, 8
// take the exact floor-then-clamp form.
// ===========================================================================
namespace tma {

constexpr int kStageBudget = 192 * 1024;

// Shape of the CTA and its stage ring: bf16 inputs run 11 consumer warps (176
// slabs, 44 KB per stage, 4 stages), fp32 inputs 8 (128 slabs, 64 KB, 3 stages).
// One CTA per SM. The transform keeps 64 values per lane in registers; with
// the producer warp the CTA is 12 (or 9) warps, which leaves ~168 registers per
// thread (the allocation rounds a CTA up to whole groups of four warps).
template <typename Tin>
struct Geo {
    static constexpr int kEsize = sizeof(Tin);
    static constexpr int kConsumerWarps = kEsize == 2 ? 11 : 8;
    static constexpr int kConsumerThreads = 32 * kConsumerWarps;
    static constexpr int kThreads = kConsumerThreads + 32;     // + producer warp
    static constexpr int kSlabsPerStage = kConsumerThreads / 2;
    static constexpr int kRowElems = 128 / kEsize;             // elements per 128-byte smem row
    static constexpr int kRowsPerHalf = 64 / kRowElems;        // smem rows per half-slab: 1 or 2
    static constexpr int kStageBytes = kSlabsPerStage * 128 * kEsize;
    static constexpr int kStages = kStageBudget / kStageBytes; // 4 (bf16) or 3 (fp32)
    static constexpr int kMaxSlabCols = 256 / (2 * kRowsPerHalf);  // box dim 1 <= 256
    static constexpr int kBarOffset = kStages * kStageBytes;
    // bars: full[kStages], empty[kStages]; then the abort flag
    static constexpr int kAbortOffset = kBarOffset + 16 * kStages;
    static constexpr int kSmemUsed = kAbortOffset + 16;
    static constexpr int kSmemTotal = kSmemUsed + 1024;
};

struct TileGeo {
    int S_c;         // slabs of a tile along the row
    int R_t;         // rows of a tile
    int tiles_c;     // tiles along the row
    int num_tiles;
    int spr;         // slabs per tensor row
    uint32_t box_bytes;
};

__device__ int g_quant_status = 0;

// Unpack 64 bf16 (32 words) or read 64 fp32 of this lane's half-slab from a stage.
template <typename Tin>
__device__ __forceinline__ void read_half_slab(uint32_t stage_base, uint32_t row0, float2 (&P)[32]) {
    if constexpr (sizeof(Tin) == 2) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const uint4 v = sync::lds128(stage_base + row0 * 128 + ((j ^ (row0 & 7)) << 4));
            P[4 * j + 0] = make_float2(bf16lo_to_f32(v.x), bf16hi_to_f32(v.x));
            P[4 * j + 1] = make_float2(bf16lo_to_f32(v.y), bf16hi_to_f32(v.y));
            P[4 * j + 2] = make_float2(bf16lo_to_f32(v.z), bf16hi_to_f32(v.z));
            P[4 * j + 3] = make_float2(bf16lo_to_f32(v.w), bf16hi_to_f32(v.w));
        }
    } else {
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const uint32_t row = row0 + r;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const uint4 v = sync::lds128(stage_base + row * 128 + ((j ^ (row & 7)) << 4));
                P[16 * r + 2 * j] = make_float2(__uint_as_float(v.x), __uint_as_float(v.y));
                P[16 * r + 2 * j + 1] = make_float2(__uint_as_float(v.z), __uint_as_float(v.w));
            }
        }
    }
}

// Quantise, pack and store the 64 values of one half-slab. `e0` is the index
// of its first element within its row; outputs are dense [rows, cols].
template <int HB, int CB, bool MULT2, bool SAT>
__device__ __forceinline__ void emit_half(const QuantArgs& A, const float2 (&P)[32],
                                          const GroupK* G, int64_t row, int64_t e0) {
    constexpr int PPB = 32 / ((HB >= 64) ? 1 : 64 / HB);
    const QuantConsts& k = A.c;

    // ---- codes: 64*CB/8 bytes, written 16 (or 8) bytes at a time
    {
        constexpr int NW = 2 * CB;   // 32-bit words per half-slab
        uint8_t* dst = A.codes + row * A.codes_row_bytes + e0 * CB / 8;
        if constexpr (NW == 2) {
            *reinterpret_cast<uint2*>(dst) =
                make_uint2(code_word<32 / ((HB >= 64) ? 1 : 64 / HB), CB, MULT2, SAT>(P, G, 0, k), code_word<32 / ((HB >= 64) ? 1 : 64 / HB), CB, MULT2, SAT>(P, G, 1, k));
        } else {
#pragma unroll
            for (int w = 0; w < NW; w += 4)
                *reinterpret_cast<uint4*>(dst + 4 * w) = make_uint4(
                    code_word<32 / ((HB >= 64) ? 1 : 64 / HB), CB, MULT2, SAT>(P, G, w, k), code_word<32 / ((HB >= 64) ? 1 : 64 / HB), CB, MULT2, SAT>(P, G, w + 1, k),
                    code_word<32 / ((HB >= 64) ? 1 : 64 / HB), CB, MULT2, SAT>(P, G, w + 2, k), code_word<32 / ((HB >= 64) ? 1 : 64 / HB), CB, MULT2, SAT>(P, G, w + 3, k));
        }
    }

    // ---- trust mask (1 = kept)
    if (k.mask_mode >= 0) {
        uint32_t by[8];
#pragma unroll
        for (int b = 0; b < 8; ++b) by[b] = mask_byte<32 / ((HB >= 64) ? 1 : 64 / HB)>(P, G, b, k);
        if (k.mask_mode == 0) {
            const uint32_t m0 = by[0] | (by[1] << 8) | (by[2] << 16) | (by[3] << 24);
            const uint32_t m1 = by[4] | (by[5] << 8) | (by[6] << 16) | (by[7] << 24);
            *reinterpret_cast<uint2*>(A.mask + row * A.mask_row_bytes + e0 / 8) = make_uint2(m0, m1);
        } else {
            uint8_t* dst = A.mask + row * A.mask_row_bytes + e0;
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const uint32_t bits = by[q];
                uint2 b;
                b.x = (bits & 1u) | ((bits >> 1) & 1u) << 8 | ((bits >> 2) & 1u) << 16 | ((bits >> 3) & 1u) << 24;
                b.y = ((bits >> 4) & 1u) | ((bits >> 5) & 1u) << 8 | ((bits >> 6) & 1u) << 16 | ((bits >> 7) & 1u) << 24;
                *reinterpret_cast<uint2*>(dst + 8 * q) = b;
            }
        }
    }

    // ---- dequantised values yhat = q_b Delta + (1/2 - 2^(b-1)) Delta
    if (k.deq_mode >= 0) {
        if (k.deq_mode == 0) {
            uint8_t* dst = A.deq + row * A.deq_row_bytes + e0 * 2;
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                uint32_t o[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int j = 4 * q + i;
                    const GroupK& g = G[j / PPB];
                    const float2 qb = __fadd2_rn(decide<SAT>(P[j], g, k), make_float2(-kMagic, -kMagic));
                    const float2 yh = __ffma2_rn(qb, make_float2(g.delta, g.delta), make_float2(g.ch, g.ch));
                    o[i] = pack_bf16x2(yh.x, yh.y);
                }
                *reinterpret_cast<uint4*>(dst + 16 * q) = make_uint4(o[0], o[1], o[2], o[3]);
            }
        } else {
            uint8_t* dst = A.deq + row * A.deq_row_bytes + e0 * 4;
#pragma unroll
            for (int j = 0; j < 32; j += 2) {
                const GroupK& g0 = G[j / PPB];
                const GroupK& g1 = G[(j + 1) / PPB];
                const float2 q0 = __fadd2_rn(decide<SAT>(P[j], g0, k), make_float2(-kMagic, -kMagic));
                const float2 q1 = __fadd2_rn(decide<SAT>(P[j + 1], g1, k), make_float2(-kMagic, -kMagic));
                const float2 y0 = __ffma2_rn(q0, make_float2(g0.delta, g0.delta), make_float2(g0.ch, g0.ch));
                const float2 y1 = __ffma2_rn(q1, make_float2(g1.delta, g1.delta), make_float2(g1.ch, g1.ch));
                *reinterpret_cast<uint4*>(dst + 8 * j) = make_uint4(__float_as_uint(y0.x), __float_as_uint(y0.y),
                                                                    __float_as_uint(y1.x), __float_as_uint(y1.y));
            }
        }
    }
}

template <typename Tin, int HB, int CB, bool MULT2, bool SAT>
__global__ void __launch_bounds__(Geo<Tin>::kThreads, 1)
quantize_tma_kernel(const __grid_constant__ CUtensorMap map_x, const QuantArgs A, const TileGeo g) {
    using Gm = Geo<Tin>;
    constexpr int BPL = (HB >= 64) ? 1 : 64 / HB;
    constexpr int PPB = 32 / BPL;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = sync::smem_u32(smem);
    const uint32_t bar_full = sbase + Gm::kBarOffset;
    const uint32_t bar_empty = bar_full + 8 * Gm::kStages;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Gm::kAbortOffset);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < Gm::kStages; ++s) {
            sync::mbar_init(bar_full + 8 * s, 1);
            sync::mbar_init(bar_empty + 8 * s, Gm::kConsumerThreads);
        }
        *abort_flag = 0;
        sync::fence_mbar_init();
        sync::prefetch_tensormap(&map_x);
    }
    __syncthreads();

    if (warp == 0) {
        // ---------------------------------------------------------------- producer
        if (lane == 0) {
            uint32_t it = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < g.num_tiles; tile += gridDim.x, ++it) {
                const uint32_t st = it % Gm::kStages, ph = (it / Gm::kStages) & 1;
                if (!sync::mbar_wait(bar_empty + 8 * st, ph ^ 1, abort_flag, &g_quant_status,
                                     (int)QUEST_ETIMEOUT)) {
                    ok = false;
                    break;
                }
                const int tr = tile / g.tiles_c, tc = tile - tr * g.tiles_c;
                sync::mbar_arrive_expect_tx(bar_full + 8 * st, g.box_bytes);
                sync::tma_load_3d(sbase + st * Gm::kStageBytes, &map_x, 0,
                                  tc * g.S_c * 2 * Gm::kRowsPerHalf, tr * g.R_t, bar_full + 8 * st);
            }
            if (!ok) {  // loads still landing in the last stages
                const uint32_t n = it < (uint32_t)Gm::kStages ? it : Gm::kStages;
                for (uint32_t i = it - n; i < it; ++i)
                    sync::mbar_drain(bar_full + 8 * (i % Gm::kStages), (i / Gm::kStages) & 1);
            }
        }
        return;
    }

    // -------------------------------------------------------------------- consumers
    const int L = threadIdx.x - 32;                 // 0..255
    const int slab = L >> 1, half = L & 1;
    const int sr = slab / g.S_c, sc = slab - sr * g.S_c;
    const bool slot_ok = sr < g.R_t;
    const uint32_t row0 = uint32_t(2 * slab + half) * Gm::kRowsPerHalf;
    uint32_t it = 0;
    for (int tile = blockIdx.x; tile < g.num_tiles; tile += gridDim.x, ++it) {
        const uint32_t st = it % Gm::kStages, ph = (it / Gm::kStages) & 1;
        const bool got = sync::mbar_wait(bar_full + 8 * st, ph, abort_flag, &g_quant_status,
                                         (int)QUEST_ETIMEOUT);
        if (__any_sync(0xFFFFFFFFu, !got)) break;   // on a timeout the warp leaves together
        float2 P[32];
        read_half_slab<Tin>(sbase + st * Gm::kStageBytes, row0, P);
        sync::mbar_arrive(bar_empty + 8 * st);

        const int trow = tile / g.tiles_c, tcol = tile - trow * g.tiles_c;
        const int64_t row = int64_t(trow) * g.R_t + sr;
        const int scol = tcol * g.S_c + sc;
        const bool valid = slot_ok && row < A.rows && scol < g.spr;

        fwht_halfslab<HB>(P, lane);

        // sums of squares, per block held (or shared) by this lane
        float ssb[BPL];
#pragma unroll
        for (int b = 0; b < BPL; ++b) {
            constexpr int NA = PPB >= 4 ? 4 : PPB;   // independent partial sums
            float2 acc[NA];
#pragma unroll
            for (int u = 0; u < NA; ++u) acc[u] = make_float2(0.0f, 0.0f);
#pragma unroll
            for (int j = b * PPB; j < (b + 1) * PPB; ++j) acc[j % NA] = __ffma2_rn(P[j], P[j], acc[j % NA]);
#pragma unroll
            for (int u = 1; u < NA; ++u) acc[0] = __fadd2_rn(acc[0], acc[u]);
            ssb[b] = slot_ok ? acc[0].x + acc[0].y : 0.0f;
        }
        GroupK G[BPL];
#pragma unroll
        for (int b = 0; b < BPL; ++b) {
            float v = ssb[b];
            if constexpr (HB >= 128) v += __shfl_xor_sync(0xFFFFFFFFu, v, 1);
            if constexpr (HB >= 256) v += __shfl_xor_sync(0xFFFFFFFFu, v, 2);
            G[b] = make_group(A.c, v);
        }
        if (valid) {
            const int64_t e0 = int64_t(scol) * 128 + half * 64;
            emit_half<HB, CB, MULT2, SAT>(A, P, G, row, e0);
            const int64_t gpr = A.cols / HB;   // groups per row
            if constexpr (HB >= 128) {
                if ((L & (HB / 64 - 1)) == 0) A.scales[row * gpr + e0 / HB] = G[0].delta;
            } else {
#pragma unroll
                for (int b = 0; b < BPL; ++b) A.scales[row * gpr + e0 / HB + b] = G[b].delta;
            }
        }
    }
}

template <typename Tin, int HB, int CB, bool MULT2, bool SAT>
cudaError_t launch_tma_t(const QuantArgs& a, const TileGeo& g, const CUtensorMap& map, cudaStream_t s) {
    using Gm = Geo<Tin>;
    auto fn = quantize_tma_kernel<Tin, HB, CB, MULT2, SAT>;
    static thread_local int attr_dev = -1;
    int dev = 0;
    cudaGetDevice(&dev);
    if (attr_dev != dev) {
        cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, Gm::kSmemTotal);
        if (e != cudaSuccess) return e;
        attr_dev = dev;
    }
    const int sms = sm_count();
    const int grid = g.num_tiles < sms ? g.num_tiles : sms;
    fn<<<grid, Gm::kThreads, Gm::kSmemTotal, s>>>(map, a, g);
    return cudaGetLastError();
}

template <typename Tin, int HB, int CB, bool MULT2>
cudaError_t launch_tma_cb(const QuantArgs& a, int bits, const TileGeo& g, const CUtensorMap& map,
                          cudaStream_t s) {
    return bits <= 6 ? launch_tma_t<Tin, HB, CB, MULT2, true>(a, g, map, s)
                     : launch_tma_t<Tin, HB, CB, MULT2, false>(a, g, map, s);
}

template <typename Tin, int HB>
cudaError_t launch_tma_hb(const QuantArgs& a, int bits, int cb, const TileGeo& g,
                          const CUtensorMap& map, cudaStream_t s) {
    switch (cb) {
        case 1: return launch_tma_cb<Tin, HB, 1, false>(a, bits, g, map, s);
        case 2: return launch_tma_cb<Tin, HB, 2, false>(a, bits, g, map, s);
        case 4: return launch_tma_cb<Tin, HB, 4, false>(a, bits, g, map, s);
        case 8: return a.c.pack2_mult == 2 ? launch_tma_cb<Tin, HB, 8, true>(a, bits, g, map, s)
                                           : launch_tma_cb<Tin, HB, 8, false>(a, bits, g, map, s);
    }
    return cudaErrorInvalidValue;
}

template <typename Tin>
cudaError_t launch_tma(const QuantArgs& a, int bits, int hb, int cb, cudaStream_t s) {
    using Gm = Geo<Tin>;
    TileGeo g;
    g.spr = (int)(a.cols / 128);
    g.S_c = g.spr < Gm::kMaxSlabCols ? g.spr : Gm::kMaxSlabCols;
    if (g.S_c > Gm::kSlabsPerStage) g.S_c = Gm::kSlabsPerStage;
    g.R_t = Gm::kSlabsPerStage / g.S_c;
    // keep at least ~4 tiles per SM on small tensors
    const int64_t want_tiles = 4LL * sm_count();
    while (g.R_t > 1 && ((a.rows + g.R_t - 1) / g.R_t) * ((g.spr + g.S_c - 1) / g.S_c) < want_tiles)
        g.R_t = (g.R_t + 1) / 2;
    g.tiles_c = (g.spr + g.S_c - 1) / g.S_c;
    const int64_t tiles_r = (a.rows + g.R_t - 1) / g.R_t;
    if (tiles_r * g.tiles_c > 0x7FFFFFFF) return cudaErrorInvalidValue;
    g.num_tiles = (int)(tiles_r * g.tiles_c);
    g.box_bytes = (uint32_t)g.R_t * g.S_c * 128 * Gm::kEsize;
    CUtensorMap map;
    const uint64_t dims[3] = {(uint64_t)Gm::kRowElems, (uint64_t)(a.cols / Gm::kRowElems), (uint64_t)a.rows};
    const uint64_t strides[2] = {128, (uint64_t)a.ld_x_bytes};
    const uint32_t box[3] = {(uint32_t)Gm::kRowElems, (uint32_t)(g.S_c * 2 * Gm::kRowsPerHalf), (uint32_t)g.R_t};
    if (!encode_tensor_map(&map, sizeof(Tin) == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                           3, a.x, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    switch (hb) {
        case 16: return launch_tma_hb<Tin, 16>(a, bits, cb, g, map, s);
        case 32: return launch_tma_hb<Tin, 32>(a, bits, cb, g, map, s);
        case 64: return launch_tma_hb<Tin, 64>(a, bits, cb, g, map, s);
        case 128: return launch_tma_hb<Tin, 128>(a, bits, cb, g, map, s);
        case 256: return launch_tma_hb<Tin, 256>(a, bits, cb, g, map, s);
    }
    return cudaErrorInvalidValue;
}

}  // namespace tma

// Whether the TMA-staged kernel handles this request (otherwise the direct one does).
// Path choice, from measurements on B200 at the 16384 x 2048 activation shape:
// the staged kernel wins for one RMS per block (b = 4: 32.8 vs 37.9 us), the
// direct kernel for one RMS per row (36.9 vs 37.9 us; 18.5 vs 20.5 us for the
// 5632 x 2048 weights). Staged streaming tops out near 4.7 TB/s on this part,
// below plain 16-byte loads, so the direct kernel keeps the rows it wins.
bool tma_path_ok(const QuantArgs& a, quest_dtype x_dtype, int cbits, bool row_mode) {
    if (row_mode) return false;
    if (a.cols % 128 != 0) return false;
    const int esize = x_dtype == QUEST_BF16 ? 2 : 4;
    if (a.ld_x_bytes % 16 != 0 || (reinterpret_cast<uintptr_t>(a.x) & 15) != 0) return false;
    // vector stores of a half-slab: codes 8 (1-bit) or 16 bytes, mask bits 8 bytes
    const uintptr_t code_align = cbits == 1 ? 8 : 16;
    if ((reinterpret_cast<uintptr_t>(a.codes) % code_align) != 0) return false;
    if (a.mask && (reinterpret_cast<uintptr_t>(a.mask) % 8) != 0) return false;
    const int max_slab_cols = esize == 2 ? 128 : 64;
    if (row_mode && a.cols / 128 > max_slab_cols) return false;
    return true;
}

cudaError_t launch_quantize(const QuantArgs& a, quest_dtype x_dtype, int had_block, int cbits,
                            int bits, bool row_mode, cudaStream_t stream) {
    if (tc_path_ok(a, x_dtype, had_block, cbits, row_mode))
        return launch_quantize_tc(a, had_block, cbits, bits, row_mode, stream);
    if (hs_path_ok(a, had_block, cbits, row_mode))
        return launch_quantize_hs(a, x_dtype, had_block, cbits, bits, row_mode, stream);
    if (a.c.code_fp8) return cudaErrorNotSupported;   // E4M3 codes only on the two layouts above
    if (tma_path_ok(a, x_dtype, cbits, row_mode)) {
        if (x_dtype == QUEST_BF16) return tma::launch_tma<__nv_bfloat16>(a, bits, had_block, cbits, stream);
        return tma::launch_tma<float>(a, bits, had_block, cbits, stream);
    }
    if (x_dtype == QUEST_BF16) return launch_dtype<__nv_bfloat16>(a, had_block, cbits, row_mode, stream);
    return launch_dtype<float>(a, had_block, cbits, row_mode, stream);
}

int read_and_clear_quant_status(cudaStream_t stream, cudaError_t* err) {
    int v = 0, zero = 0;
    cudaError_t e = cudaMemcpyFromSymbolAsync(&v, tma::g_quant_status, sizeof(int), 0,
                                              cudaMemcpyDeviceToHost, stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    if (e == cudaSuccess && v != 0)
        e = cudaMemcpyToSymbolAsync(tma::g_quant_status, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    *err = e;
    return v;
}

}  // namespace quest

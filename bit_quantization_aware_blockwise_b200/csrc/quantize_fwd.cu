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
    pdl_wait();      // the previous kernel on the stream has completed
    pdl_trigger();   // the next one may be scheduled as CTAs of this one leave
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
    pdl_wait();      // the previous kernel on the stream has completed
    pdl_trigger();   // the next one may be scheduled as CTAs of this one leave
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
    return launch_pdl(fn, dim3((unsigned)grid), dim3(kThreads), 0, stream, a);
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
        return launch_pdl(quantize_rows_kernel<Tin, HB, CB, 1>, dim3((unsigned)grid), dim3(kThreads), 0, stream, a,
                          wpr);
    return launch_pdl(quantize_rows_kernel<Tin, HB, CB, 2>, dim3((unsigned)grid), dim3(kThreads), 0, stream, a, wpr);
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
cudaError_t launch_quantize(const QuantArgs& a, quest_dtype x_dtype, int had_block, int cbits,
                            int bits, bool row_mode, cudaStream_t stream) {
    if (tc_path_ok(a, x_dtype, had_block, cbits, row_mode))
        return launch_quantize_tc(a, had_block, cbits, bits, row_mode, stream);
    if (hs_path_ok(a, had_block, cbits, row_mode))
        return launch_quantize_hs(a, x_dtype, had_block, cbits, bits, row_mode, stream);
    // E4M3 operand codes and the FP4 grid only on the two layouts above
    if (a.c.code_fp8 || a.c.grid_fp4) return cudaErrorNotSupported;
    if (x_dtype == QUEST_BF16) return launch_dtype<__nv_bfloat16>(a, had_block, cbits, row_mode, stream);
    return launch_dtype<float>(a, had_block, cbits, row_mode, stream);
}

}  // namespace quest

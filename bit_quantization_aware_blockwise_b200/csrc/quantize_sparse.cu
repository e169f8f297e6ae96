// QuEST quantizer, 2:4-sparse INT variant, for bf16 input (sm_100a).
//
// The pages evaluate QuEST on a 2:4-sparse INT4 format (atlas.scime.ai summary
// of QuEST, ablation table; pith.science review, results list and Figure 4a)
// without spelling it out. This library reads it as: the Hadamard transform and
// RMS of the dense quantizer (quantize_tc.cu); in every run of four consecutive
// transformed values the two of largest magnitude survive (on equal magnitudes
// the lower index wins); survivors go onto the b-bit midrise grid whose step
// minimises the MSE of the surviving values of an N(0,1) input
// (quest_alpha_sparse24); the trust mask applies the half-interval rule to every
// value's total error, so a pruned value (rebuilt as 0) keeps its gradient iff
// |t| <= T/2.
//
// Layout: the tensor-core layout of quest_tc.cuh. A lane's chunk of 8
// consecutive values holds two whole runs of four (pairs P[4f], P[4f+1] and
// P[4f+2], P[4f+3]), so the pruning, the compaction of the kept codes and the
// metadata stay in registers. Outputs per chunk: 4 code bytes (the kept values
// of each run in index order, c = 2q + 1 as int8: the compressed operand of a
// sparse tensor-core product), one metadata byte (per run a nibble, the lower
// kept index in bits 0-1, the higher in bits 2-3; the first run in the low
// nibble) and one mask byte.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "quest_device.cuh"
#include "quest_emit.cuh"
#include "quest_internal.h"
#include "quest_tc.cuh"

namespace quest {
namespace sp {

using tc::kThreads;

// Kept flags of a run of four values (bit i = value i survives): value i
// survives when fewer than two others beat it, value j beating value i when
// |v_j| > |v_i|, or |v_j| == |v_i| and j < i.
__device__ __forceinline__ uint32_t kept_of_run(float v0, float v1, float v2, float v3) {
    const float a0 = fabsf(v0), a1 = fabsf(v1), a2 = fabsf(v2), a3 = fabsf(v3);
    const int w01 = a0 >= a1, w02 = a0 >= a2, w03 = a0 >= a3;   // the lower index wins a tie
    const int w12 = a1 >= a2, w13 = a1 >= a3, w23 = a2 >= a3;
    const int l0 = 3 - w01 - w02 - w03;
    const int l1 = w01 + 2 - w12 - w13;
    const int l2 = w02 + w12 + 1 - w23;
    const int l3 = w03 + w13 + w23;
    return uint32_t(l0 < 2) | uint32_t(l1 < 2) << 1 | uint32_t(l2 < 2) << 2 | uint32_t(l3 < 2) << 3;
}

// Trust-mask byte of chunk f for the threshold thr2 on the unnormalised y^2.
__device__ __forceinline__ uint32_t mask_byte_thr(const float2 (&P)[16], int f, float thr2) {
    uint32_t acc = 0;
#pragma unroll
    for (int j = 4 * f + 3; j >= 4 * f; --j) {
        const float2 d = __ffma2_rn(P[j], P[j], make_float2(-thr2, -thr2));
        acc = __funnelshift_l(__float_as_uint(d.y), acc, 1);
        acc = __funnelshift_l(__float_as_uint(d.x), acc, 1);
    }
    return acc;
}

// Quantise, prune and store this lane's 32 values (chunks c = t + 4f of the slab
// whose first element is e_slab in row `row`). OUT = 0 reads the optional outputs
// (mask, dequant) from the arguments; OUT = 1 writes codes and metadata only, the
// set the sparse layer consumes, with the optional paths compiled out.
template <bool SAT, int OUT>
__device__ __forceinline__ void emit_sparse(const SparseArgs& S, const float2 (&P)[16], const GroupK& G,
                                            int64_t row, int64_t e_slab, int t, bool valid) {
    const QuantArgs& A = S.q;
    const QuantConsts& k = A.c;
    uint8_t* codes = A.codes + row * A.codes_row_bytes + e_slab / 2;
    const int coff = 1 - (1 << S.bits);   // c = 2 q_b + 1 - 2^b
    const float thr2p = G.thr2 * S.prune_ratio;
    const bool do_mask = OUT == 0 && k.mask_mode >= 0, do_deq = OUT == 0 && valid && k.deq_mode >= 0;
    uint32_t mbytes = 0, metab = 0;
#pragma unroll
    for (int f = 0; f < 4; ++f) {
        const int c = t + 4 * f;
        float2 s[4];
        chunk_decide<SAT, 16>(P, &G, f, k, s);
        uint32_t word = 0, kept8 = 0, nib = 0;
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const float2 p0 = P[4 * f + 2 * r], p1 = P[4 * f + 2 * r + 1];
            const uint32_t km = kept_of_run(p0.x, p0.y, p1.x, p1.y);
            const int c0 = 2 * int(__float_as_uint(s[2 * r].x) - kMagicBits) + coff;
            const int c1 = 2 * int(__float_as_uint(s[2 * r].y) - kMagicBits) + coff;
            const int c2 = 2 * int(__float_as_uint(s[2 * r + 1].x) - kMagicBits) + coff;
            const int c3 = 2 * int(__float_as_uint(s[2 * r + 1].y) - kMagicBits) + coff;
            const int lo = (km & 1u) ? c0 : ((km & 2u) ? c1 : c2);
            const int hi = (km & 8u) ? c3 : ((km & 4u) ? c2 : c1);
            word |= (uint32_t(lo) & 0xFFu) << (16 * r) | (uint32_t(hi) & 0xFFu) << (16 * r + 8);
            kept8 |= km << (4 * r);
            const uint32_t i0 = __ffs(km) - 1, i1 = 31 - __clz(km);
            nib |= (i0 | (i1 << 2)) << (4 * r);
        }
        if (valid) *reinterpret_cast<uint32_t*>(codes + 4 * c) = word;
        metab |= nib << (8 * f);
        if (do_mask) {
            const uint32_t mk = k.trust_ge1 ? mask_byte_edge<16>(P, &G, f) : mask_byte_cell<16>(P, &G, f, k);
            const uint32_t mp = mask_byte_thr(P, f, thr2p);
            mbytes |= (((kept8 & mk) | (~kept8 & mp)) & 0xFFu) << (8 * f);
        }
        if (do_deq) {
            // yhat = q_b Delta + (1/2 - 2^(b-1)) Delta for kept values, 0 for pruned ones
            uint32_t w[4];
#pragma unroll
            for (int p = 0; p < 4; ++p) {
                const float2 qb = __fadd2_rn(s[p], make_float2(-kMagic, -kMagic));
                float2 y = __ffma2_rn(qb, make_float2(G.delta, G.delta), make_float2(G.ch, G.ch));
                if (!((kept8 >> (2 * p)) & 1u)) y.x = 0.0f;
                if (!((kept8 >> (2 * p + 1)) & 1u)) y.y = 0.0f;
                w[p] = pack_bf16x2(y.x, y.y);
            }
            const int64_t e = e_slab + 8 * c;
            *reinterpret_cast<uint4*>(A.deq + row * A.deq_row_bytes + 2 * e) = make_uint4(w[0], w[1], w[2], w[3]);
        }
    }
    // byte f of a lane holds chunk t + 4f; after the transpose lane t holds chunks 4t .. 4t+3
    const uint32_t mw = tc::quad_transpose_bytes(metab, t);   // every lane: it shuffles
    if (valid) *reinterpret_cast<uint32_t*>(S.meta + row * S.meta_row_bytes + e_slab / 8 + 4 * t) = mw;
    if (do_mask) {
        const uint32_t w = tc::quad_transpose_bytes(mbytes, t);
        if (valid) *reinterpret_cast<uint32_t*>(A.mask + row * A.mask_row_bytes + e_slab / 8 + 4 * t) = w;
    }
}

__device__ __forceinline__ float lane_sum_sq(const float2 (&P)[16]) {
    float2 acc0 = make_float2(0.0f, 0.0f), acc1 = acc0;
#pragma unroll
    for (int j = 0; j < 16; j += 2) {
        acc0 = __ffma2_rn(P[j], P[j], acc0);
        acc1 = __ffma2_rn(P[j + 1], P[j + 1], acc1);
    }
    const float2 a = __fadd2_rn(acc0, acc1);
    return a.x + a.y;
}

// One RMS per 128-value slab (Hadamard block 128): a warp step covers 8 slabs.
template <bool SAT, int OUT>
__global__ void __launch_bounds__(kThreads) quantize_sparse_groups(const SparseArgs S) {
    pdl_wait();
    pdl_trigger();
    const QuantArgs& A = S.q;
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    const int64_t spr = A.cols / 128;
    const int64_t total = A.rows * spr;
    const int64_t warp0 = (int64_t(blockIdx.x) * kThreads + threadIdx.x) >> 5;
    const int64_t step = int64_t(gridDim.x) * (kThreads / 32) * 8;
    const tc::BFrag B = tc::make_bfrag(lane, tc::tmask_of<128>());
    uint4 raw[4];
    {
        const int64_t slab = warp0 * 8 + g;
        if (slab < total) tc::load_slab(A.x + slab * 256, t, raw);
        else tc::zero4(raw);
    }
    for (int64_t s0 = warp0 * 8; s0 < total; s0 += step) {
        const int64_t slab = s0 + g, next = slab + step;
        float2 P[16];
        tc::mma_stage(raw, B, P);
        if (next < total) tc::load_slab(A.x + next * 256, t, raw);
        else tc::zero4(raw);
        tc::reg_stages<128>(P, lane);
        float v = lane_sum_sq(P);
        v += __shfl_xor_sync(0xFFFFFFFFu, v, 1);
        v += __shfl_xor_sync(0xFFFFFFFFu, v, 2);
        const GroupK G = make_group(A.c, v);
        const bool valid = slab < total;
        const int64_t row = valid ? slab / spr : 0, e_slab = (slab - row * spr) * 128;
        emit_sparse<SAT, OUT>(S, P, G, row, e_slab, t, valid);
        if (valid && t == 0) A.scales[slab] = G.delta;
    }
}

// One RMS per row of spr = cols / 128 slabs (spr in 1, 2, 4, 8, 16). SUB slabs per
// lane group (spr / 8 when spr >= 8: a warp holds a row); for spr < 8 a warp step
// covers 8 / spr rows.
// Four CTAs per SM for the codes-and-metadata set (124 registers at SUB = 2, no spill);
// three with the optional outputs.
template <bool SAT, int SUB, int OUT>
__global__ void __launch_bounds__(kThreads, OUT == 1 ? 4 : 3) quantize_sparse_rows(const SparseArgs S, int spr) {
    pdl_wait();
    pdl_trigger();
    const QuantArgs& A = S.q;
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    const int rps = SUB > 1 ? 1 : (spr >= 8 ? 1 : 8 / spr);   // rows per warp step
    const int r_in = rps > 1 ? g / spr : 0, sc0 = rps > 1 ? g % spr : g;
    const int gspan = rps > 1 ? spr : 8;                        // lane groups of one row
    const int64_t warp0 = (int64_t(blockIdx.x) * kThreads + threadIdx.x) >> 5;
    const int64_t step = int64_t(gridDim.x) * (kThreads / 32) * rps;
    const tc::BFrag B = tc::make_bfrag(lane, tc::tmask_of<128>());
    auto load_row = [&](int64_t row, uint4 (&raw)[SUB][4]) {
#pragma unroll
        for (int u = 0; u < SUB; ++u) {
            if (row < A.rows) tc::load_slab(A.x + row * A.ld_x_bytes + int64_t(sc0 + 8 * u) * 256, t, raw[u]);
            else tc::zero4(raw[u]);
        }
    };
    uint4 raw[SUB][4];
    load_row(warp0 * rps + r_in, raw);
    for (int64_t r0 = warp0 * rps; r0 < A.rows; r0 += step) {
        const int64_t row = r0 + r_in;
        const bool valid = row < A.rows;
        float2 P[SUB][16];
#pragma unroll
        for (int u = 0; u < SUB; ++u) tc::mma_stage(raw[u], B, P[u]);
        load_row(row + step, raw);
        float v = 0.0f;
#pragma unroll
        for (int u = 0; u < SUB; ++u) {
            tc::reg_stages<128>(P[u], lane);
            v += lane_sum_sq(P[u]);
        }
        v += __shfl_xor_sync(0xFFFFFFFFu, v, 1);
        v += __shfl_xor_sync(0xFFFFFFFFu, v, 2);
        for (int sh = 4; sh < 4 * gspan; sh <<= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, sh);
        const GroupK G = make_group(A.c, v);
#pragma unroll
        for (int u = 0; u < SUB; ++u)
            emit_sparse<SAT, OUT>(S, P[u], G, valid ? row : 0, int64_t(sc0 + 8 * u) * 128, t, valid);
        if (valid && sc0 == 0 && t == 0) A.scales[row] = G.delta;
    }
}

template <bool SAT, int OUT>
cudaError_t launch_out(const SparseArgs& s, bool row_mode, cudaStream_t stream) {
    const QuantArgs& a = s.q;
    const int sms = sm_count();
    if (row_mode) {
        const int spr = (int)(a.cols / 128);
        auto go = [&](auto fn, int64_t rows_per_warp) {
            const int64_t warps = (a.rows + rows_per_warp - 1) / rows_per_warp;
            const int64_t cap = int64_t(sms) * max_ctas_per_sm((const void*)fn, kThreads, 0);
            const int64_t want = (warps + kThreads / 32 - 1) / (kThreads / 32);
            return launch_pdl(fn, dim3((unsigned)(want < cap ? want : cap)), dim3(kThreads), 0, stream, s, spr);
        };
        if (spr == 16) return go(quantize_sparse_rows<SAT, 2, OUT>, 1);
        if (spr == 8) return go(quantize_sparse_rows<SAT, 1, OUT>, 1);
        return go(quantize_sparse_rows<SAT, 1, OUT>, 8 / spr);
    }
    const int64_t warps = (a.rows * (a.cols / 128) + 7) / 8;
    auto fn = quantize_sparse_groups<SAT, OUT>;
    const int64_t cap = int64_t(sms) * max_ctas_per_sm((const void*)fn, kThreads, 0);
    const int64_t want = (warps + kThreads / 32 - 1) / (kThreads / 32);
    return launch_pdl(fn, dim3((unsigned)(want < cap ? want : cap)), dim3(kThreads), 0, stream, s);
}

}  // namespace sp

cudaError_t launch_quantize_sparse24(const SparseArgs& s, bool row_mode, cudaStream_t stream) {
    // codes and metadata only (no mask, no dequant): the output set compiled in
    const bool lean = s.q.c.mask_mode < 0 && s.q.c.deq_mode < 0;
    if (s.bits <= 6)
        return lean ? sp::launch_out<true, 1>(s, row_mode, stream) : sp::launch_out<true, 0>(s, row_mode, stream);
    return lean ? sp::launch_out<false, 1>(s, row_mode, stream) : sp::launch_out<false, 0>(s, row_mode, stream);
}

}  // namespace quest

// CTA-pair tcgen05 bf16 products: the input gradient of the quantized linear layer
// with the trust backward fused into the epilogue, and the linear layer on bf16
// dequantised operands (see the kernel's comment).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace quest {
namespace {
// Device-side status word of this file's kernels (0 = fine). Written only when a
// bounded wait gives up; read and cleared by quest_device_status().
__device__ int g_tc_status = 0;
}  // namespace
}  // namespace quest

#include "tc_common.cuh"

namespace quest {
namespace {

// ---------------------------------------------------------------------------
// Input gradient of the quantized linear layer with the trust backward fused
// into the epilogue (pith.science review, "What carries the argument": the
// gradient is masked in the Hadamard domain; Figure 2 caption: the inverse
// transforms run on the backward pass):
//   G[m][k]   = sum_n gy[m][n] wt[k][n]                (bf16 x bf16 -> fp32, kind::f16)
//   gx[m][b]  = H (mask[m][b] * G[m][b]) / sqrt(128)   per 128-column block b of a row
// CTA pairs as in the integer layer: M = 256, N = 256 per MMA and K = 16 bf16
// (32 bytes) per MMA, so a 128-byte stage row holds four K steps as there and the
// shared-memory ring, barriers and TMEM accumulators are the same. The epilogue
// thread that owns an accumulator row (one TMEM lane) holds a whole 128-column
// block in registers: the mask and the 128-point transform are register work with
// no exchange, and G never reaches HBM. The same kernel without the mask and the
// transform is the linear layer on bf16 dequantised operands, y = x_hat w_hat^T
// (yhat = (q + 1/2) Delta rounded to bf16, any RMS grouping). Tiles run output-column-fastest: the pairs in
// flight share a few 256-row blocks of grad_y (which, at 16384 x 5632 bf16, is larger
// than L2) and all of w_hat_t, so grad_y streams from HBM about once.
constexpr uint32_t kIdescBf16Pair = (1u << 4)     // D: fp32
                                  | (1u << 7)     // A: bf16
                                  | (1u << 10)    // B: bf16
                                  | (uint32_t(BN >> 3) << 17) | (uint32_t(256 >> 4) << 24);

__device__ __forceinline__ void tc_mma_bf16_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                                 uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(kIdescBf16Pair), "r"(accumulate)
        : "memory");
}

struct TrustLinearParams {
    const uint8_t* mask;        // trust mask bits [M, K / 8]
    float scale;                // 1 / sqrt(128)
    int M, N, K;                // G is [M, K]; the reduction runs over N
    int num_m2, num_n, num_k;   // 256-row tiles, 256-column output tiles, 64-element steps of N
};

// Unnormalised 128-point Walsh-Hadamard transform (Sylvester order) of one
// thread's registers: the first stage inside each pair, the other six as packed
// fp32x2 butterflies (a - b as one fused b * -1 + a, a single rounding).
__device__ __forceinline__ void fwht128_regs(float2 (&w)[64]) {
#pragma unroll
    for (int j = 0; j < 64; ++j) w[j] = make_float2(w[j].x + w[j].y, w[j].x - w[j].y);
#pragma unroll
    for (int h = 1; h < 64; h <<= 1) {
#pragma unroll
        for (int j = 0; j < 64; ++j) {
            if ((j & h) == 0) {
                const float2 a = w[j], b = w[j + h];
                w[j] = __fadd2_rn(a, b);
                w[j + h] = __ffma2_rn(b, make_float2(-1.0f, -1.0f), a);
            }
        }
    }
}

// TRUST: the epilogue masks and transforms each 128-column block (the input gradient);
// otherwise it stores the product as it is (the linear layer on bf16 yhat operands).
template <bool TRUST>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
bf16_pair_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                 const __grid_constant__ CUtensorMap map_y, const TrustLinearParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar_full = sbase + kPSmemBar;                 // [kPStages], used in the even CTA
    const uint32_t bar_empty = bar_full + 8 * kPStages;          // [kPStages]
    const uint32_t bar_tfull = bar_empty + 8 * kPStages;         // [2]
    const uint32_t bar_tempty = bar_tfull + 16;                  // [2], used in the even CTA
    const uint32_t bar_drain = bar_tempty + 16;                  // [1]
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kPSmemAbort);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kPSmemTmemSlot);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const bool even = rank == 0;
    const int pair = blockIdx.x >> 1, num_pairs = gridDim.x >> 1;
    const int num_tiles = p.num_m2 * p.num_n;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kPStages; ++s) {
            mbar_init(bar_full + 8 * s, 1);
            mbar_init(bar_empty + 8 * s, 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar_tfull + 8 * b, 1);
            mbar_init(bar_tempty + 8 * b, 2);
        }
        mbar_init(bar_drain, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_a)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_b)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_y)) : "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_slot)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    cluster_sync();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    // the prologue above touched no global memory: wait here for the previous
    // kernel on the stream, then let the next kernel be scheduled
    pdl_wait();
    pdl_trigger();

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer (both CTAs)
        if (lane == 0) {
            const uint32_t full_even = map_to_rank(bar_full, 0);
            uint32_t stage = 0, phase = 0;
            uint64_t issued = 0;
            bool ok = true;
            for (int tile = pair; tile < num_tiles && ok; tile += num_pairs) {
                const int m0 = (tile / p.num_n) * 256 + 128 * int(rank);
                const int k0 = (tile % p.num_n) * BN + 128 * int(rank);
                for (int kb = 0; kb < p.num_k; ++kb) {
                    if (!mbar_wait(bar_empty + 8 * stage, phase ^ 1, abort_flag, kWaitLimitNs, kSuspendProducerNs)) {
                        ok = false;
                        break;
                    }
                    if (even) mbar_arrive_expect_tx(bar_full + 8 * stage, kPTxBytes);
                    const uint32_t fb = full_even + 8 * stage;
                    tma_load_2d_pair(sbase + kPSmemA + stage * kPStageA, &map_a, kb * 64, m0, fb);
                    tma_load_2d_pair(sbase + kPSmemB + stage * kPStageB, &map_b, kb * 64, k0, fb);
                    ++issued;
                    if (++stage == kPStages) { stage = 0; phase ^= 1; }
                }
            }
            if (!ok && even) {
                const uint64_t n = issued < kPStages ? issued : kPStages;
                for (uint64_t i = issued - n; i < issued; ++i) {
                    const uint32_t st = uint32_t(i % kPStages), ph = uint32_t((i / kPStages) & 1);
                    const uint64_t t0 = global_timer_ns();
                    while (!mbar_try_wait(bar_full + 8 * st, ph) && global_timer_ns() - t0 < kWaitLimitNs) {
                    }
                }
            } else if (!ok) {
                const uint64_t t0 = global_timer_ns();
                while (global_timer_ns() - t0 < 10000000ull) {
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer (even CTA)
        if (even && lane == 0) {
            uint32_t stage = 0, phase = 0;
            bool ok = true;
            int local = 0;
            for (int tile = pair; tile < num_tiles && ok; tile += num_pairs, ++local) {
                const uint32_t buf = local & 1, bphase = (local >> 1) & 1;
                if (!mbar_wait(bar_tempty + 8 * buf, bphase ^ 1, abort_flag, kWaitLimitNs, kSuspendMmaNs)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + buf * BN;
                for (int kb = 0; kb < p.num_k; ++kb) {
                    if (!mbar_wait(bar_full + 8 * stage, phase, abort_flag, kWaitLimitNs, kSuspendMmaNs)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_addr = sbase + kPSmemA + stage * kPStageA;
                    const uint32_t b_addr = sbase + kPSmemB + stage * kPStageB;
#pragma unroll
                    for (int kk = 0; kk < BK / kUmmaK; ++kk) {
                        tc_mma_bf16_pair(d_tmem, smem_desc_k128(a_addr + kk * kUmmaK),
                                         smem_desc_k128(b_addr + kk * kUmmaK), (kb | kk) != 0);
                    }
                    tc_commit_pair_mc(bar_empty + 8 * stage);
                    if (++stage == kPStages) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
                tc_commit_pair_mc(bar_tfull + 8 * buf);
            }
            tc_commit_pair(bar_drain);
            const uint64_t t0 = global_timer_ns();
            while (!mbar_try_wait(bar_drain, 0) && global_timer_ns() - t0 < kWaitLimitNs) {
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue (warps 2..5, both CTAs)
        const int et = threadIdx.x - 64;
        const int quarter = warp & 3;
        const int row_in_tile = quarter * 32 + lane;
        const uint32_t lane_addr = uint32_t(quarter * 32) << 16;
        const uint32_t tempty_even = map_to_rank(bar_tempty, 0);
        const int64_t mask_row_bytes = p.K / 8;
        int local = 0;
        int cbuf = 0;
        for (int tile = pair; tile < num_tiles; tile += num_pairs, ++local) {
            const int m0 = (tile / p.num_n) * 256 + 128 * int(rank), k0 = (tile % p.num_n) * BN;
            const uint32_t buf = local & 1, bphase = (local >> 1) & 1;
            const int m = m0 + row_in_tile;
            // this row's mask bits for the tile's two blocks, fetched before the wait
            uint4 mw[2] = {make_uint4(0u, 0u, 0u, 0u), make_uint4(0u, 0u, 0u, 0u)};
            if constexpr (TRUST) {
#pragma unroll
                for (int b = 0; b < 2; ++b) {
                    const int kb0 = k0 + 128 * b;
                    if (m < p.M && kb0 < p.K)
                        mw[b] = *reinterpret_cast<const uint4*>(p.mask + int64_t(m) * mask_row_bytes + kb0 / 8);
                }
            }
            const bool got = mbar_wait(bar_tfull + 8 * buf, bphase, abort_flag, kWaitLimitNs, kSuspendEpilogueNs);
            if (epi_any(!got)) break;
            tc_fence_after();
            const uint32_t t_acc = tmem_base + lane_addr + buf * BN;
#pragma unroll 1
            for (int b = 0; b < 2; ++b) {
                if (k0 + 128 * b >= p.K) break;   // tile-uniform: the ragged last column tile
                const uint4 mb = b == 0 ? mw[0] : mw[1];
                float2 w[64];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint32_t r[32];
                    QUEST_TMEM_LD32(t_acc + 128 * b + 32 * c, r);
                    tmem_wait_ld();
                    const uint32_t bits = c == 0 ? mb.x : c == 1 ? mb.y : c == 2 ? mb.z : mb.w;
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        if constexpr (TRUST) {
                            // keep G where the mask bit is 1 (bit j of the word = column 32c + j)
                            const uint32_t k0m = 0u - ((bits >> (2 * i)) & 1u);
                            const uint32_t k1m = 0u - ((bits >> (2 * i + 1)) & 1u);
                            w[16 * c + i] =
                                make_float2(__uint_as_float(r[2 * i] & k0m), __uint_as_float(r[2 * i + 1] & k1m));
                        } else {
                            w[16 * c + i] = make_float2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
                        }
                    }
                }
                if constexpr (TRUST) fwht128_regs(w);
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const uint32_t stg = sbase + kPSmemC + cbuf * kCBytes + row_in_tile * (kChunkCols * 2);
                    const uint32_t swz = (row_in_tile >> 1) & 3;
#pragma unroll
                    for (int q16 = 0; q16 < 4; ++q16) {
                        uint32_t o[4];
#pragma unroll
                        for (int h = 0; h < 4; ++h) {
                            const float2 v = w[16 * c + 4 * q16 + h];
                            __nv_bfloat162 hb = TRUST ? __floats2bfloat162_rn(v.x * p.scale, v.y * p.scale)
                                                      : __floats2bfloat162_rn(v.x, v.y);
                            o[h] = *reinterpret_cast<uint32_t*>(&hb);
                        }
                        asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(stg + ((q16 ^ swz) << 4)),
                                     "r"(o[0]), "r"(o[1]), "r"(o[2]), "r"(o[3])
                                     : "memory");
                    }
                    fence_proxy_async_smem();
                    epi_bar();
                    if (et == 0) {
                        tma_store_2d(&map_y, sbase + kPSmemC + cbuf * kCBytes, k0 + 128 * b + c * kChunkCols, m0);
                        bulk_commit();
                        bulk_wait_read_le1();
                    }
                    epi_bar();
                    cbuf ^= 1;
                }
            }
            tc_fence_before();
            epi_bar();
            if (et == 0) mbar_arrive_remote(tempty_even + 8 * buf);
        }
        if (et == 0) bulk_wait_all();
    }

    tc_fence_before();
    cluster_sync();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTmemCols)
                     : "memory");
    }
}

// out [M, K] = a [M, N] b [K, N]^T (both N-contiguous), with the trust epilogue when
// TRUST (mask bits [M, K / 8]).
template <bool TRUST>
cudaError_t launch_bf16_pair(const uint16_t* gy, const uint16_t* wt, const uint8_t* mask, int64_t M, int64_t N,
                             int64_t K, uint16_t* gx, cudaStream_t stream) {
    CUtensorMap ma, mb, my;
    if (!make_map_2d(&ma, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, gy, N, M, N * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map_2d(&mb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, wt, N, K, N * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map_2d(&my, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, gx, K, M, K * 2, kChunkCols, 128,
                     CU_TENSOR_MAP_SWIZZLE_64B))
        return cudaErrorInvalidValue;
    TrustLinearParams p;
    p.mask = mask;
    p.scale = TRUST ? 0.08838834764831845f : 1.0f;   // 1 / sqrt(128) for the inverse transform
    p.M = (int)M; p.N = (int)N; p.K = (int)K;
    p.num_m2 = (int)((M + 255) / 256);
    p.num_n = (int)((K + BN - 1) / BN);
    p.num_k = (int)((N + 63) / 64);
    static thread_local int attr_dev = -1;
    int dev = 0;
    cudaGetDevice(&dev);
    if (attr_dev != dev) {
        cudaError_t e = cudaFuncSetAttribute(bf16_pair_kernel<TRUST>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, kPSmemTotal);
        if (e != cudaSuccess) return e;
        attr_dev = dev;
    }
    const int tiles = p.num_m2 * p.num_n;
    const int pairs = pair_clusters(dev, (const void*)bf16_pair_kernel<TRUST>, kThreads, kPSmemTotal);
    const int grid_pairs = tiles < pairs ? tiles : pairs;
    return launch_pdl(bf16_pair_kernel<TRUST>, dim3(2 * grid_pairs), dim3(kThreads), kPSmemTotal, stream, ma, mb,
                      my, p);
}

}  // namespace

cudaError_t launch_trust_linear(const uint16_t* gy, const uint16_t* wt, const uint8_t* mask, int64_t M,
                                int64_t N, int64_t K, uint16_t* gx, cudaStream_t stream) {
    if (M == 0 || K == 0) return cudaSuccess;
    if (N == 0) {   // the empty sum: G = 0, so the gradient is 0
        return launch_zero_fill(gx, nullptr, M * K, stream);
    }
    return launch_bf16_pair<true>(gy, wt, mask, M, N, K, gx, stream);
}

cudaError_t launch_linear_bf16(const uint16_t* x_hat, const uint16_t* w_hat, int64_t M, int64_t N, int64_t K,
                               uint16_t* y, cudaStream_t stream) {
    if (M == 0 || N == 0) return cudaSuccess;
    if (K == 0) return launch_zero_fill(y, nullptr, M * N, stream);   // the empty sum
    // the pair kernel's product runs over its second dimension: y [M, N] = x_hat [M, K] w_hat [N, K]^T
    return launch_bf16_pair<false>(x_hat, w_hat, nullptr, M, K, N, y, stream);
}

int read_and_clear_trust_linear_status(cudaStream_t stream, cudaError_t* err) {
    int v = 0, zero = 0;
    cudaError_t e = cudaMemcpyFromSymbolAsync(&v, g_tc_status, sizeof(int), 0, cudaMemcpyDeviceToHost, stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    if (e == cudaSuccess && v != 0)
        e = cudaMemcpyToSymbolAsync(g_tc_status, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    *err = e;
    return v;
}

}  // namespace quest

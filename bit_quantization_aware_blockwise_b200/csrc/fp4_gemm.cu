// Linear layer on FP4 (E2M1) QuEST codes on the block-scaled FP4 tensor cores
// (sm_100a):
//
//   acc[m][n] = sum_k Q_A[m][k] * Q_B[n][k]     (E2M1 x E2M1, fp32 accumulation)
//   y[m][n]   = bf16_rne(acc * sa[m] * sb[n])
//
// with Q the grid values of the FP4 variant of the quantizer (codes packed two
// per byte, element 2j in the low nibble) and sa, sb its per-row steps Delta
// (the quantized value is Q * Delta). Every product of two E2M1 values is a
// multiple of 1/4 of magnitude at most 36, so at K <= 2^14 every partial sum is
// a multiple of 1/4 below 2^20 and the fp32 accumulation is exact.
//
// The pages evaluate an FP4 grid for QuEST (pith.science review, Figure 4a and
// "Assumptions & free parameters"); the block-scaled MMA kind (kind::mxf4, one
// UE8M0 scale per 32 K values) runs at twice the rate of the int8 kind. The
// block scales are all 1.0: a 32-column TMEM region holding the byte 0x7F
// (2^0 in UE8M0) in every lane is written once per CTA, and every MMA points its
// A and B scale operands into it, so no scale ever leaves the chip.
//
// Structure: CTA pairs (cluster of 2, cta_group::2), M = 256 x N = 240 pair
// tiles; per CTA a 6-stage ring of A [128 x 128 B] and B [120 x 128 B] tiles
// (256 FP4 values per row per stage); four tcgen05.mma (K = 64 each) per stage;
// two 240-column fp32 accumulators (TMEM columns 0 and 240) alternate so the
// epilogue of one tile overlaps the mainloop of the next; TMEM columns 480-511
// hold the scale bytes. N = 240 is the widest tile two accumulators and the
// scale columns leave room for, and it divides N = 5632 into 23.5 tiles (224
// gave 25.1, so every pair ran a mostly empty 26th column of tiles). Epilogue:
// eight warps, two per TMEM lane quarter, each taking half of the tile's columns
// of its 32 accumulator rows, 32 columns at a time (the last 16 with a
// 16-column load and store): scale, round to bf16, store through its own staging
// buffers and TMA stores (warp-level syncs only). At the FP4 rate a tile's
// mainloop is short (about 3.8K cycles), and with one warp per lane quarter the
// epilogue did not fit in it (16384 x 5632 x 2048: 94.7 us, against 75.8 us with
// the epilogue skipped). Every
// mbarrier wait is bounded; a timeout records QUEST_ETIMEOUT in the device
// status word and the CTA drains its copies, frees TMEM and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace quest {
namespace {
// Device-side status word of this file's kernel (0 = fine). Written only when a
// bounded wait gives up; read and cleared by quest_device_status().
__device__ int g_tc_status = 0;
}  // namespace
}  // namespace quest

#include "tc_common.cuh"

namespace quest {
namespace {

constexpr int kFBN = 240;                                   // output columns per pair tile
constexpr int kFThreads = 320;                              // producer, MMA, 8 epilogue warps
constexpr int kFEpiThreads = 256;
constexpr int kFChunks = kFBN / kChunkCols;                 // 7 whole 32-column chunks and a 16-column tail
constexpr int kFTailCols = kFBN - kFChunks * kChunkCols;    // 16
constexpr int kFHalfChunks = 4;                             // half 0: chunks 0-3; half 1: 4-6 and the tail
constexpr int kFStages = 6;
constexpr uint32_t kFStageA = 128 * BK;                     // 128 rows x 128 bytes (256 FP4 values)
constexpr uint32_t kFStageB = (kFBN / 2) * BK;              // 120 rows x 128 bytes
constexpr uint32_t kFTxBytes = 2 * (kFStageA + kFStageB);   // both CTAs land on the even CTA's barrier
constexpr uint32_t kFSmemA = 0;
constexpr uint32_t kFSmemB = kFSmemA + kFStages * kFStageA;
constexpr uint32_t kFSmemC = kFSmemB + kFStages * kFStageB;
constexpr uint32_t kFWarpCBytes = 32 * kChunkCols * 2;      // one warp's 32 x 32 bf16 staging chunk
constexpr uint32_t kFSmemScale = kFSmemC + 8 * 2 * kFWarpCBytes;   // float[kFBN]
constexpr uint32_t kFSmemBar = kFSmemScale + kFBN * 4;
constexpr uint32_t kFNumBars = 2 * kFStages + 4 + 1;
constexpr uint32_t kFSmemTmemSlot = kFSmemBar + kFNumBars * 8;
constexpr uint32_t kFSmemAbort = kFSmemTmemSlot + 4;
constexpr uint32_t kFSmemUsed = kFSmemAbort + 4;
constexpr uint32_t kFSmemTotal = kFSmemUsed + 1024;
static_assert(kFStageB % 1024 == 0, "128-byte-swizzled stages start on 1 KB boundaries");
static_assert(kFSmemTotal <= 227 * 1024, "FP4 pair kernel shared memory");
constexpr uint32_t kFAccStride = kFBN;                      // accumulator buffers at TMEM columns 0 and 240
constexpr uint32_t kFScaleCol = 480;                        // 32 columns of 0x7F bytes: A scales at 480, B at 496
static_assert(kFAccStride + kFBN <= kFScaleCol && kFScaleCol + 32 <= kTmemCols, "TMEM columns");
static_assert(kFTailCols == 16, "one 16-column tail chunk");

// Block-scaled instruction descriptor: A and B E2M1 (format 1 of the FP4 kind),
// K-major, N = 240, UE8M0 scales (bit 23), M = 256, scale-factor ids 0, K = 64.
constexpr uint32_t kIdescFp4 = (1u << 7) | (1u << 10) | (uint32_t(kFBN >> 3) << 17) | (1u << 23) |
                               (uint32_t(256 >> 4) << 24);

__device__ __forceinline__ void tc_mma_fp4_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                                uint32_t accumulate, uint32_t sfa, uint32_t sfb) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
            d_tmem),
        "l"(adesc), "l"(bdesc), "r"(kIdescFp4), "r"(accumulate), "r"(sfa), "r"(sfb)
        : "memory");
}

// Named barrier 1 over the 256 epilogue threads, and an OR-vote on it.
__device__ __forceinline__ void fepi_bar() { asm volatile("bar.sync 1, %0;" ::"n"(kFEpiThreads) : "memory"); }
__device__ __forceinline__ bool fepi_any(bool pred) {
    uint32_t out;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, 1, %2, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(out)
        : "r"((uint32_t)pred), "n"(kFEpiThreads)
        : "memory");
    return out != 0;
}

// 32 consecutive TMEM columns of this warp's 32 lanes <- the same 32-bit word.
__device__ __forceinline__ void tmem_fill32(uint32_t taddr, uint32_t v) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,"
        "%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1};" ::"r"(taddr),
        "r"(v)
        : "memory");
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

struct Fp4Params {
    const float* sa;    // [M]
    const float* sb;    // [N]
    float* acc;         // optional fp32 [M, N] copy of the accumulator
    int M, N, K;
    int num_m2, num_n, num_k;   // 256-row pair tiles, 240-column tiles, 256-value K steps
};

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kFThreads, 1)
fp4_gemm_pair_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                     const __grid_constant__ CUtensorMap map_y, const __grid_constant__ CUtensorMap map_y16,
                     const Fp4Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar_full = sbase + kFSmemBar;                 // [kFStages], used in the even CTA
    const uint32_t bar_empty = bar_full + 8 * kFStages;          // [kFStages]
    const uint32_t bar_tfull = bar_empty + 8 * kFStages;         // [2]
    const uint32_t bar_tempty = bar_tfull + 16;                  // [2], used in the even CTA
    const uint32_t bar_drain = bar_tempty + 16;                  // [1]
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kFSmemAbort);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kFSmemTmemSlot);
    float* s_scale = reinterpret_cast<float*>(smem + kFSmemScale);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const bool even = rank == 0;
    const int pair = blockIdx.x >> 1, num_pairs = gridDim.x >> 1;
    const int num_tiles = p.num_m2 * p.num_n;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kFStages; ++s) {
            mbar_init(bar_full + 8 * s, 1);
            mbar_init(bar_empty + 8 * s, 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar_tfull + 8 * b, 1);
            mbar_init(bar_tempty + 8 * b, 16);   // one arrival from each epilogue warp of both CTAs
        }
        mbar_init(bar_drain, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_a)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_b)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_y)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_y16)) : "memory");
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
    if (warp >= 2) {
        // the block scales: byte 0x7F (1.0) in every lane of columns 480-511, written
        // by each epilogue warp into its own lane quarter, in both CTAs
        tmem_fill32(tmem_base + (uint32_t((warp & 3) * 32) << 16) + kFScaleCol, 0x7F7F7F7Fu);
    }
    tc_fence_before();
    cluster_sync();   // the scale columns of both CTAs are written before the first MMA
    tc_fence_after();
    // nothing above touched global memory: wait for the kernel that wrote the codes,
    // then let the next kernel be scheduled
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
                const int m0 = (tile % p.num_m2) * 256 + 128 * int(rank);
                const int n0 = (tile / p.num_m2) * kFBN + (kFBN / 2) * int(rank);
                for (int kb = 0; kb < p.num_k; ++kb) {
                    if (!mbar_wait(bar_empty + 8 * stage, phase ^ 1, abort_flag, kWaitLimitNs, kSuspendProducerNs)) {
                        ok = false;
                        break;
                    }
                    if (even) mbar_arrive_expect_tx(bar_full + 8 * stage, kFTxBytes);
                    const uint32_t fb = full_even + 8 * stage;
                    tma_load_2d_pair(sbase + kFSmemA + stage * kFStageA, &map_a, kb * BK, m0, fb);
                    tma_load_2d_pair(sbase + kFSmemB + stage * kFStageB, &map_b, kb * BK, n0, fb);
                    ++issued;
                    if (++stage == kFStages) { stage = 0; phase ^= 1; }
                }
            }
            if (!ok && even) {
                const uint64_t n = issued < kFStages ? issued : kFStages;
                for (uint64_t i = issued - n; i < issued; ++i) {
                    const uint32_t st = uint32_t(i % kFStages), ph = uint32_t((i / kFStages) & 1);
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
            const uint32_t sfa = tmem_base + kFScaleCol, sfb = tmem_base + kFScaleCol + 16;
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
                const uint32_t d_tmem = tmem_base + buf * kFAccStride;
                for (int kb = 0; kb < p.num_k; ++kb) {
                    if (!mbar_wait(bar_full + 8 * stage, phase, abort_flag, kWaitLimitNs, kSuspendMmaNs)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_addr = sbase + kFSmemA + stage * kFStageA;
                    const uint32_t b_addr = sbase + kFSmemB + stage * kFStageB;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {   // 64 FP4 values = 32 bytes per MMA
                        tc_mma_fp4_pair(d_tmem, smem_desc_k128(a_addr + kk * 32), smem_desc_k128(b_addr + kk * 32),
                                        (kb | kk) != 0, sfa, sfb);
                    }
                    tc_commit_pair_mc(bar_empty + 8 * stage);
                    if (++stage == kFStages) { stage = 0; phase ^= 1; }
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
        // ------------------------------------------------------------ epilogue (warps 2..9, both CTAs)
        const int et = threadIdx.x - 64;             // 0..255
        const int quarter = warp & 3;                // TMEM lanes 32*quarter .. +31
        const int half = (warp - 2) >> 2;            // column chunks [0, 4) or [4, 7)
        const int c_lo = half * kFHalfChunks, c_hi = half ? kFChunks + 1 : kFHalfChunks;   // chunk 7: the tail
        const int row_in_tile = quarter * 32 + lane;
        const uint32_t lane_addr = uint32_t(quarter * 32) << 16;
        const uint32_t tempty_even = map_to_rank(bar_tempty, 0);
        int local = 0;
        int cbuf = 0;
        for (int tile = pair; tile < num_tiles; tile += num_pairs, ++local) {
            const int m0 = (tile % p.num_m2) * 256 + 128 * int(rank), n0 = (tile / p.num_m2) * kFBN;
            const uint32_t buf = local & 1, bphase = (local >> 1) & 1;
            fepi_bar();   // everyone is done with the previous tile's column scales
            for (int c = et; c < kFBN; c += kFEpiThreads) {
                const int n = n0 + c;
                s_scale[c] = n < p.N ? p.sb[n] : 0.0f;
            }
            const int m = m0 + row_in_tile;
            const float sa_m = m < p.M ? p.sa[m] : 0.0f;
            const bool got = mbar_wait(bar_tfull + 8 * buf, bphase, abort_flag, kWaitLimitNs, kSuspendEpilogueNs);
            if (fepi_any(!got)) break;
            tc_fence_after();
            const uint32_t t_acc = tmem_base + lane_addr + buf * kFAccStride;
            // each warp stores its own 32 rows: 32 x 32 bf16 chunks through two staging
            // buffers of its own, so no chunk waits on the other warps
            const uint32_t stg_w = sbase + kFSmemC + uint32_t(warp - 2) * 2 * kFWarpCBytes;
            const uint32_t swz = (lane >> 1) & 3;
#pragma unroll 1
            for (int c = c_lo; c < c_hi; ++c) {
                uint32_t r[32];
                if (c == kFChunks) {
                    // the last 16 columns: a 16-column load (nothing past the tile is read)
                    QUEST_TMEM_LD16(t_acc + c * kChunkCols, r);
                } else {
                    QUEST_TMEM_LD32(t_acc + c * kChunkCols, r);
                }
                tmem_wait_ld();
                if (c == c_hi - 1) {
                    // this warp's part of the accumulator is read: hand it back to the MMA
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive_remote(tempty_even + 8 * buf);
                }
                const float* sc = s_scale + c * kChunkCols;
                if (lane == 0) bulk_wait_read_le1();   // the buffer used two chunks ago is free
                __syncwarp();
                if (c == kFChunks) {
                    // tail: 32 rows x 16 bf16, unswizzled, one 16-column TMA box
                    const uint32_t stg = stg_w + cbuf * kFWarpCBytes + lane * (kFTailCols * 2);
#pragma unroll
                    for (int q16 = 0; q16 < 2; ++q16) {
                        uint32_t w[4];
#pragma unroll
                        for (int h = 0; h < 4; ++h) {
                            const int i = q16 * 8 + h * 2;
                            const float2 y = __fmul2_rn(
                                __fmul2_rn(make_float2(__uint_as_float(r[i]), __uint_as_float(r[i + 1])),
                                           make_float2(sa_m, sa_m)),
                                *reinterpret_cast<const float2*>(sc + i));
                            __nv_bfloat162 hb = __floats2bfloat162_rn(y.x, y.y);
                            w[h] = *reinterpret_cast<uint32_t*>(&hb);
                        }
                        asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(stg + (q16 << 4)), "r"(w[0]),
                                     "r"(w[1]), "r"(w[2]), "r"(w[3])
                                     : "memory");
                    }
                    if (p.acc != nullptr && m < p.M) {
                        float* arow = p.acc + int64_t(m) * p.N;
#pragma unroll
                        for (int i = 0; i < kFTailCols; ++i) {
                            const int n = n0 + c * kChunkCols + i;
                            if (n < p.N) arow[n] = __uint_as_float(r[i]);
                        }
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        tma_store_2d(&map_y16, stg_w + cbuf * kFWarpCBytes, n0 + c * kChunkCols, m0 + 32 * quarter);
                        bulk_commit();
                    }
                    cbuf ^= 1;
                    continue;
                }
                const uint32_t stg = stg_w + cbuf * kFWarpCBytes + lane * (kChunkCols * 2);
#pragma unroll
                for (int q16 = 0; q16 < 4; ++q16) {
                    uint32_t w[4];
#pragma unroll
                    for (int h = 0; h < 4; ++h) {
                        const int i = q16 * 8 + h * 2;
                        const float2 y = __fmul2_rn(
                            __fmul2_rn(make_float2(__uint_as_float(r[i]), __uint_as_float(r[i + 1])),
                                       make_float2(sa_m, sa_m)),
                            *reinterpret_cast<const float2*>(sc + i));
                        __nv_bfloat162 hb = __floats2bfloat162_rn(y.x, y.y);
                        w[h] = *reinterpret_cast<uint32_t*>(&hb);
                    }
                    asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(stg + ((q16 ^ swz) << 4)),
                                 "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3])
                                 : "memory");
                }
                if (p.acc != nullptr && m < p.M) {
                    float* arow = p.acc + int64_t(m) * p.N;
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const int n = n0 + c * kChunkCols + i;
                        if (n < p.N) arow[n] = __uint_as_float(r[i]);
                    }
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    tma_store_2d(&map_y, stg_w + cbuf * kFWarpCBytes, n0 + c * kChunkCols, m0 + 32 * quarter);
                    bulk_commit();
                }
                cbuf ^= 1;
            }
        }
        if (lane == 0) bulk_wait_all();
    }

    tc_fence_before();
    cluster_sync();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTmemCols)
                     : "memory");
    }
}

}  // namespace

cudaError_t launch_fp4_linear(const uint8_t* A, const float* sa, const uint8_t* B, const float* sb, int64_t M,
                              int64_t N, int64_t K, uint16_t* y, float* acc, cudaStream_t stream) {
    if (M == 0 || N == 0) return cudaSuccess;
    if (K == 0) {
        if (acc) cudaMemsetAsync(acc, 0, size_t(M * N) * sizeof(float), stream);
        return launch_zero_fill(y, nullptr, M * N, stream);
    }
    const int64_t kb = K / 2;   // bytes per row of packed codes
    CUtensorMap ma, mb, my, my16;
    if (!make_map_2d(&ma, CU_TENSOR_MAP_DATA_TYPE_UINT8, A, kb, M, kb, BK, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map_2d(&mb, CU_TENSOR_MAP_DATA_TYPE_UINT8, B, kb, N, kb, BK, kFBN / 2, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map_2d(&my, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, y, N, M, N * 2, kChunkCols, 32,
                     CU_TENSOR_MAP_SWIZZLE_64B) ||
        !make_map_2d(&my16, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, y, N, M, N * 2, kFTailCols, 32,
                     CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    Fp4Params p;
    p.sa = sa; p.sb = sb; p.acc = acc;
    p.M = (int)M; p.N = (int)N; p.K = (int)K;
    p.num_m2 = (int)((M + 255) / 256);
    p.num_n = (int)((N + kFBN - 1) / kFBN);
    p.num_k = (int)((kb + BK - 1) / BK);
    static thread_local int attr_dev = -1;
    int dev = 0;
    cudaGetDevice(&dev);
    if (attr_dev != dev) {
        cudaError_t e = cudaFuncSetAttribute(fp4_gemm_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             kFSmemTotal);
        if (e != cudaSuccess) return e;
        attr_dev = dev;
    }
    const int tiles = p.num_m2 * p.num_n;
    const int pairs = pair_clusters(dev, (const void*)fp4_gemm_pair_kernel, kFThreads, kFSmemTotal);
    const int grid_pairs = tiles < pairs ? tiles : pairs;
    return launch_pdl(fp4_gemm_pair_kernel, dim3(2 * grid_pairs), dim3(kFThreads), kFSmemTotal, stream, ma, mb, my,
                      my16, p);
}

int read_and_clear_fp4_status(cudaStream_t stream, cudaError_t* err) {
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

// Integer linear layer on QuEST codes: tcgen05 kind::i8 GEMM with TMEM
// accumulators and a fused dequantisation epilogue (sm_100a).
//
//   acc[m][n] = sum_k A[m][k] * B[n][k]        (int8 x int8 -> int32, exact)
//   y[m][n]   = bf16_rne(acc * (sa[m]/2) * (sb[n]/2))
//
// The pages run the QuEST linear layers as INT4 kernels on the integer codes
// (atlas.scime.ai summary of QuEST, "Key results"; pith.science review,
// Figure 5). On sm_100a the codes travel as int8 (c = 2q + 1, |c| <= 15 at
// b = 4), which makes the int8 tensor-core product exact.
//
// Structure (one persistent CTA per SM, 192 threads):
//   warp 0     TMA producer: A [128 x 128] and B [256 x 128] int8 tiles,
//              128-byte swizzle, kStages-deep smem ring guarded by mbarriers.
//   warp 1     TMEM allocator and MMA issuer: one thread issues four
//              tcgen05.mma (K = 32 each) per stage into a 128 x 256 int32
//              accumulator; two accumulators (512 TMEM columns) alternate so
//              the epilogue of tile i overlaps the mainloop of tile i + 1.
//   warps 2-5  epilogue: tcgen05.ld 32 columns at a time, scale, round to
//              bf16, stage in 64-byte-swizzled smem, TMA store.
// No cluster, no multicast. Every mbarrier wait is bounded in time; on
// timeout the CTA records QUEST_ETIMEOUT in a device status word, drains its
// in-flight copies and MMAs, frees TMEM and returns.
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

// Wait bound of a launch that carries the injected timeout fault.
constexpr uint64_t kInjectedWaitLimitNs = 1000000ull;   // 1 ms

// Shared-memory layout of the single-CTA kernel.
constexpr int kStages = 4;
constexpr uint32_t kStageA = BM * BK, kStageB = BN * BK, kStageBytes = kStageA + kStageB;
constexpr uint32_t kSmemA = 0;
constexpr uint32_t kSmemB = kSmemA + kStages * kStageA;
constexpr uint32_t kSmemC = kSmemB + kStages * kStageB;
constexpr uint32_t kSmemScale = kSmemC + 2 * kCBytes;       // float[BN]
constexpr uint32_t kSmemBar = kSmemScale + BN * 4;
constexpr uint32_t kNumBars = 2 * kStages + 4 + 1;
constexpr uint32_t kSmemTmemSlot = kSmemBar + kNumBars * 8;
constexpr uint32_t kSmemAbort = kSmemTmemSlot + 4;
constexpr uint32_t kSmemUsed = kSmemAbort + 4;
constexpr uint32_t kSmemTotal = kSmemUsed + 1024;           // slack for 1 KB alignment

// Instruction descriptor of tcgen05.mma kind::i8: D int32, A and B signed
// int8, both K-major, M = 128, N = 256.
constexpr uint32_t kIdesc = (2u << 4)           // D format: s32
                            | (1u << 7)         // A: signed 8-bit
                            | (1u << 10)        // B: signed 8-bit
                            | (uint32_t(BN >> 3) << 17) | (uint32_t(BM >> 4) << 24);
__device__ __forceinline__ void tc_mma_i8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(kIdesc), "r"(accumulate)
        : "memory");
}

struct GemmParams {
    const float* sa;
    const float* sb;
    int32_t* acc;       // optional int32 copy of the accumulator
    int M, N, K;
    int num_m, num_n, num_k;
    // Injected fault (tests of the timeout path): the producer issues no copies,
    // so nothing is ever in flight and the pipeline waits run out after limit_ns.
    int withhold;
    uint64_t limit_ns;  // bound of each pipeline wait (kWaitLimitNs normally)
};

__global__ void __launch_bounds__(kThreads, 1)
w4a4_gemm_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                 const __grid_constant__ CUtensorMap map_y, const GemmParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar_full = sbase + kSmemBar;                  // [kStages]
    const uint32_t bar_empty = bar_full + 8 * kStages;           // [kStages]
    const uint32_t bar_tfull = bar_empty + 8 * kStages;          // [2]
    const uint32_t bar_tempty = bar_tfull + 16;                  // [2]
    const uint32_t bar_drain = bar_tempty + 16;                  // [1] MMA drain on abort
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kSmemAbort);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kSmemTmemSlot);
    float* s_scale = reinterpret_cast<float*>(smem + kSmemScale);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int num_tiles = p.num_m * p.num_n;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(bar_full + 8 * s, 1);
            mbar_init(bar_empty + 8 * s, 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar_tfull + 8 * b, 1);
            mbar_init(bar_tempty + 8 * b, kEpiThreads);
        }
        mbar_init(bar_drain, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_a)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_b)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_y)) : "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_slot)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    // the prologue above touched no global memory: wait here for the previous
    // kernel on the stream, then let the next kernel be scheduled
    pdl_wait();
    pdl_trigger();

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            uint32_t stage = 0, phase = 0;
            uint64_t issued = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < num_tiles && ok && !p.withhold; tile += gridDim.x) {
                const int m0 = (tile % p.num_m) * BM, n0 = (tile / p.num_m) * BN;
                for (int kb = 0; kb < p.num_k; ++kb) {
                    if (!mbar_wait(bar_empty + 8 * stage, phase ^ 1, abort_flag, p.limit_ns, kSuspendProducerNs)) {
                        ok = false;
                        break;
                    }
                    const uint32_t fb = bar_full + 8 * stage;
                    mbar_arrive_expect_tx(fb, kStageBytes);
                    tma_load_2d(sbase + kSmemA + stage * kStageA, &map_a, kb * BK, m0, fb);
                    tma_load_2d(sbase + kSmemB + stage * kStageB, &map_b, kb * BK, n0, fb);
                    ++issued;
                    if (++stage == kStages) { stage = 0; phase ^= 1; }
                }
            }
            if (!ok) {
                // drain: the last min(issued, kStages) loads may still be landing
                const uint64_t n = issued < kStages ? issued : kStages;
                for (uint64_t i = issued - n; i < issued; ++i) {
                    const uint32_t st = uint32_t(i % kStages), ph = uint32_t((i / kStages) & 1);
                    const uint64_t t0 = global_timer_ns();
                    while (!mbar_try_wait(bar_full + 8 * st, ph) && global_timer_ns() - t0 < kWaitLimitNs) {
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            uint32_t stage = 0, phase = 0;
            bool ok = true;
            int local = 0;
            for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++local) {
                const uint32_t buf = local & 1, bphase = (local >> 1) & 1;
                if (!mbar_wait(bar_tempty + 8 * buf, bphase ^ 1, abort_flag, p.limit_ns, kSuspendMmaNs)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + buf * BN;
                for (int kb = 0; kb < p.num_k; ++kb) {
                    if (!mbar_wait(bar_full + 8 * stage, phase, abort_flag, p.limit_ns, kSuspendMmaNs)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_addr = sbase + kSmemA + stage * kStageA;
                    const uint32_t b_addr = sbase + kSmemB + stage * kStageB;
#pragma unroll
                    for (int kk = 0; kk < BK / kUmmaK; ++kk) {
                        tc_mma_i8(d_tmem, smem_desc_k128(a_addr + kk * kUmmaK),
                                  smem_desc_k128(b_addr + kk * kUmmaK), (kb | kk) != 0);
                    }
                    tc_commit(bar_empty + 8 * stage);  // frees the smem stage when these MMAs finish
                    if (++stage == kStages) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
                tc_commit(bar_tfull + 8 * buf);        // accumulator ready for the epilogue
            }
            // make sure every issued MMA has finished before TMEM is released
            tc_commit(bar_drain);
            const uint64_t t0 = global_timer_ns();
            while (!mbar_try_wait(bar_drain, 0) && global_timer_ns() - t0 < kWaitLimitNs) {
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue (warps 2..5)
        const int et = threadIdx.x - 64;             // 0..127
        const int quarter = warp & 3;                // this warp may read TMEM lanes 32*quarter..+31
        const int row_in_tile = quarter * 32 + lane; // accumulator row = TMEM lane
        const uint32_t lane_addr = uint32_t(quarter * 32) << 16;
        int local = 0;
        int cbuf = 0;
        for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++local) {
            const int m0 = (tile % p.num_m) * BM, n0 = (tile / p.num_m) * BN;
            const uint32_t buf = local & 1, bphase = (local >> 1) & 1;
            epi_bar();  // everyone is done with the previous tile's column scales
            for (int c = et; c < BN; c += kEpiThreads) {
                const int n = n0 + c;
                s_scale[c] = n < p.N ? p.sb[n] * 0.5f : 0.0f;
            }
            const int m = m0 + row_in_tile;
            const float sa_half = m < p.M ? p.sa[m] * 0.5f : 0.0f;
            const bool got = mbar_wait(bar_tfull + 8 * buf, bphase, abort_flag, p.limit_ns, kSuspendEpilogueNs);
            if (epi_any(!got)) break;  // all 128 threads leave together
            tc_fence_after();
            const uint32_t t_acc = tmem_base + lane_addr + buf * BN;
#pragma unroll 1
            for (int c = 0; c < BN / kChunkCols; ++c) {
                uint32_t r[32];
                QUEST_TMEM_LD32(t_acc + c * kChunkCols, r);
                tmem_wait_ld();
                const float* sc = s_scale + c * kChunkCols;
                const uint32_t stg = sbase + kSmemC + cbuf * kCBytes + row_in_tile * (kChunkCols * 2);
                const uint32_t swz = (row_in_tile >> 1) & 3;
#pragma unroll
                for (int q16 = 0; q16 < 4; ++q16) {
                    uint32_t w[4];
#pragma unroll
                    for (int h = 0; h < 4; ++h) {
                        const int i = q16 * 8 + h * 2;
                        // (acc * sa/2) * sb/2 per column, two columns per packed multiply
                        const float2 s01 = *reinterpret_cast<const float2*>(sc + i);
                        const float2 y = __fmul2_rn(
                            __fmul2_rn(make_float2((float)(int32_t)r[i], (float)(int32_t)r[i + 1]),
                                       make_float2(sa_half, sa_half)),
                            s01);
                        __nv_bfloat162 hb = __floats2bfloat162_rn(y.x, y.y);
                        w[h] = *reinterpret_cast<uint32_t*>(&hb);
                    }
                    const uint32_t dst = stg + ((q16 ^ swz) << 4);
                    asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(dst), "r"(w[0]),
                                 "r"(w[1]), "r"(w[2]), "r"(w[3])
                                 : "memory");
                }
                if (p.acc != nullptr && m < p.M) {
                    int32_t* arow = p.acc + int64_t(m) * p.N;
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const int n = n0 + c * kChunkCols + i;
                        if (n < p.N) arow[n] = (int32_t)r[i];
                    }
                }
                fence_proxy_async_smem();
                epi_bar();
                if (et == 0) {
                    tma_store_2d(&map_y, sbase + kSmemC + cbuf * kCBytes, n0 + c * kChunkCols, m0);
                    bulk_commit();
                    bulk_wait_read_le1();  // the other staging buffer is free again
                }
                epi_bar();
                cbuf ^= 1;
            }
            tc_fence_before();
            mbar_arrive(bar_tempty + 8 * buf);
        }
        if (et == 0) bulk_wait_all();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                     "r"(kTmemCols)
                     : "memory");
    }
}

// ---------------------------------------------------------------------------
// CTA-pair variant (cluster of 2, tcgen05 cta_group::2): one MMA of M = 256,
// N = 256 per K step, issued by the even CTA, reading A rows 0-127 and B rows
// (output columns) 0-127 from its own shared memory and A rows 128-255 and B
// rows 128-255 from its peer's. Each CTA therefore stages 32 KB per K step
// instead of 48 KB for the same tensor-core work, and six stages fit where the
// single-CTA kernel holds four: on B200 the single-CTA MMA thread waits for
// operand tiles about a fifth of the time (L2 latency with 192 KB in flight).
// Loads carry no multicast: each CTA fetches its own halves, and both signal
// the even CTA's full barrier. The even CTA's tcgen05.commit (multicast to both
// CTAs of the pair) frees a stage in both rings and hands each CTA its half of
// the accumulator (rows 0-127 land in the even CTA's TMEM, 128-255 in the odd's).

// kind::i8, s32 accumulator, signed A and B, K-major, M = 256, N = 256.
constexpr uint32_t kIdescPair = (2u << 4) | (1u << 7) | (1u << 10) | (uint32_t(BN >> 3) << 17) |
                                (uint32_t(256 >> 4) << 24);
__device__ __forceinline__ void tc_mma_i8_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                               uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(kIdescPair), "r"(accumulate)
        : "memory");
}

struct PairParams {
    const float* sa;
    const float* sb;
    int32_t* acc;
    int M, N, K;
    int num_m2, num_n, num_k;   // 256-row pair tiles, 256-column tiles, K steps
};

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
w4a4_gemm_pair_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                      const __grid_constant__ CUtensorMap map_y, const PairParams p) {
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
    float* s_scale = reinterpret_cast<float*>(smem + kPSmemScale);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const bool even = rank == 0;
    const int pair = blockIdx.x >> 1, num_pairs = gridDim.x >> 1;
    const int num_tiles = p.num_m2 * p.num_n;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kPStages; ++s) {
            mbar_init(bar_full + 8 * s, 1);     // the even CTA's producer arms it for both CTAs' bytes
            mbar_init(bar_empty + 8 * s, 1);    // one multicast commit per use
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar_tfull + 8 * b, 1);
            mbar_init(bar_tempty + 8 * b, 2);   // one arrival from each CTA's epilogue
        }
        mbar_init(bar_drain, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_a)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_b)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_y)) : "memory");
    }
    if (warp == 1) {
        // both CTAs allocate together (same warp, same slot offset)
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_slot)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    cluster_sync();   // barrier initialisation and the TMEM address are visible across the pair
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    // the prologue above touched no global memory: wait here for the kernel that
    // produced the operand codes, then let the next kernel be scheduled
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
                const int n0 = (tile / p.num_m2) * BN + 128 * int(rank);
                for (int kb = 0; kb < p.num_k; ++kb) {
                    if (!mbar_wait(bar_empty + 8 * stage, phase ^ 1, abort_flag, kWaitLimitNs, kSuspendProducerNs)) {
                        ok = false;
                        break;
                    }
                    if (even) mbar_arrive_expect_tx(bar_full + 8 * stage, kPTxBytes);
                    const uint32_t fb = full_even + 8 * stage;
                    tma_load_2d_pair(sbase + kPSmemA + stage * kPStageA, &map_a, kb * BK, m0, fb);
                    tma_load_2d_pair(sbase + kPSmemB + stage * kPStageB, &map_b, kb * BK, n0, fb);
                    ++issued;
                    if (++stage == kPStages) { stage = 0; phase ^= 1; }
                }
            }
            if (!ok && even) {
                // drain: the last min(issued, kPStages) stages may still be landing
                const uint64_t n = issued < kPStages ? issued : kPStages;
                for (uint64_t i = issued - n; i < issued; ++i) {
                    const uint32_t st = uint32_t(i % kPStages), ph = uint32_t((i / kPStages) & 1);
                    const uint64_t t0 = global_timer_ns();
                    while (!mbar_try_wait(bar_full + 8 * st, ph) && global_timer_ns() - t0 < kWaitLimitNs) {
                    }
                }
            } else if (!ok) {
                // the odd CTA cannot observe the even CTA's barrier: give its copies time to land
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
                        tc_mma_i8_pair(d_tmem, smem_desc_k128(a_addr + kk * kUmmaK),
                                       smem_desc_k128(b_addr + kk * kUmmaK), (kb | kk) != 0);
                    }
                    tc_commit_pair_mc(bar_empty + 8 * stage);   // frees the stage in both CTAs
                    if (++stage == kPStages) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
                tc_commit_pair_mc(bar_tfull + 8 * buf);         // both halves of the accumulator ready
            }
            tc_commit_pair(bar_drain);
            const uint64_t t0 = global_timer_ns();
            while (!mbar_try_wait(bar_drain, 0) && global_timer_ns() - t0 < kWaitLimitNs) {
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue (warps 2..5, both CTAs)
        const int et = threadIdx.x - 64;             // 0..127
        const int quarter = warp & 3;                // this warp may read TMEM lanes 32*quarter..+31
        const int row_in_tile = quarter * 32 + lane; // accumulator row = TMEM lane
        const uint32_t lane_addr = uint32_t(quarter * 32) << 16;
        const uint32_t tempty_even = map_to_rank(bar_tempty, 0);
        int local = 0;
        int cbuf = 0;
        for (int tile = pair; tile < num_tiles; tile += num_pairs, ++local) {
            const int m0 = (tile % p.num_m2) * 256 + 128 * int(rank), n0 = (tile / p.num_m2) * BN;
            const uint32_t buf = local & 1, bphase = (local >> 1) & 1;
            epi_bar();  // everyone is done with the previous tile's column scales
            for (int c = et; c < BN; c += kEpiThreads) {
                const int n = n0 + c;
                s_scale[c] = n < p.N ? p.sb[n] * 0.5f : 0.0f;
            }
            const int m = m0 + row_in_tile;
            const float sa_half = m < p.M ? p.sa[m] * 0.5f : 0.0f;
            const bool got = mbar_wait(bar_tfull + 8 * buf, bphase, abort_flag, kWaitLimitNs, kSuspendEpilogueNs);
            if (epi_any(!got)) break;  // all 128 threads leave together
            tc_fence_after();
            const uint32_t t_acc = tmem_base + lane_addr + buf * BN;
#pragma unroll 1
            for (int c = 0; c < BN / kChunkCols; ++c) {
                uint32_t r[32];
                QUEST_TMEM_LD32(t_acc + c * kChunkCols, r);
                tmem_wait_ld();
                const float* sc = s_scale + c * kChunkCols;
                const uint32_t stg = sbase + kPSmemC + cbuf * kCBytes + row_in_tile * (kChunkCols * 2);
                const uint32_t swz = (row_in_tile >> 1) & 3;
#pragma unroll
                for (int q16 = 0; q16 < 4; ++q16) {
                    uint32_t w[4];
#pragma unroll
                    for (int h = 0; h < 4; ++h) {
                        const int i = q16 * 8 + h * 2;
                        // (acc * sa/2) * sb/2 per column, two columns per packed multiply
                        const float2 s01 = *reinterpret_cast<const float2*>(sc + i);
                        const float2 y = __fmul2_rn(
                            __fmul2_rn(make_float2((float)(int32_t)r[i], (float)(int32_t)r[i + 1]),
                                       make_float2(sa_half, sa_half)),
                            s01);
                        __nv_bfloat162 hb = __floats2bfloat162_rn(y.x, y.y);
                        w[h] = *reinterpret_cast<uint32_t*>(&hb);
                    }
                    const uint32_t dst = stg + ((q16 ^ swz) << 4);
                    asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(dst), "r"(w[0]),
                                 "r"(w[1]), "r"(w[2]), "r"(w[3])
                                 : "memory");
                }
                if (p.acc != nullptr && m < p.M) {
                    int32_t* arow = p.acc + int64_t(m) * p.N;
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const int n = n0 + c * kChunkCols + i;
                        if (n < p.N) arow[n] = (int32_t)r[i];
                    }
                }
                fence_proxy_async_smem();
                epi_bar();
                if (et == 0) {
                    tma_store_2d(&map_y, sbase + kPSmemC + cbuf * kCBytes, n0 + c * kChunkCols, m0);
                    bulk_commit();
                    bulk_wait_read_le1();  // the other staging buffer is free again
                }
                epi_bar();
                cbuf ^= 1;
            }
            // every thread's TMEM loads of this buffer are complete (wait::ld above)
            tc_fence_before();
            epi_bar();
            if (et == 0) mbar_arrive_remote(tempty_even + 8 * buf);
        }
        if (et == 0) bulk_wait_all();
    }

    tc_fence_before();
    cluster_sync();   // neither CTA leaves while the pair's MMAs or copies may touch its memory
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTmemCols)
                     : "memory");
    }
}

cudaError_t launch_pair(const int8_t* A, const float* sa, const int8_t* B, const float* sb, int64_t M,
                        int64_t N, int64_t K, uint16_t* y, int32_t* acc, cudaStream_t stream) {
    CUtensorMap ma, mb, my;
    if (!make_map_2d(&ma, CU_TENSOR_MAP_DATA_TYPE_UINT8, A, K, M, K, BK, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map_2d(&mb, CU_TENSOR_MAP_DATA_TYPE_UINT8, B, K, N, K, BK, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map_2d(&my, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, y, N, M, N * 2, kChunkCols, 128,
                     CU_TENSOR_MAP_SWIZZLE_64B))
        return cudaErrorInvalidValue;
    PairParams p;
    p.sa = sa; p.sb = sb; p.acc = acc;
    p.M = (int)M; p.N = (int)N; p.K = (int)K;
    p.num_m2 = (int)((M + 255) / 256);
    p.num_n = (int)((N + BN - 1) / BN);
    p.num_k = (int)((K + BK - 1) / BK);
    static thread_local int attr_dev = -1;
    int dev = 0;
    cudaGetDevice(&dev);
    if (attr_dev != dev) {
        cudaError_t e = cudaFuncSetAttribute(w4a4_gemm_pair_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, kPSmemTotal);
        if (e != cudaSuccess) return e;
        attr_dev = dev;
    }
    const int tiles = p.num_m2 * p.num_n;
    const int pairs = pair_clusters(dev, (const void*)w4a4_gemm_pair_kernel, kThreads, kPSmemTotal);
    const int grid_pairs = tiles < pairs ? tiles : pairs;
    return launch_pdl(w4a4_gemm_pair_kernel, dim3(2 * grid_pairs), dim3(kThreads), kPSmemTotal, stream, ma, mb, my,
                      p);
}

}  // namespace

cudaError_t launch_w4a4(const int8_t* A, const float* sa, const int8_t* B, const float* sb,
                        int64_t M, int64_t N, int64_t K, uint16_t* y, int32_t* acc,
                        cudaStream_t stream, bool inject_timeout) {
    if (M == 0 || N == 0) return cudaSuccess;
    if (K == 0) {
        return launch_zero_fill(y, acc, M * N, stream);
    }
    // more than one 128-row block: CTA pairs (M = 256 tiles); otherwise one CTA per
    // tile (which also handles any M, and carries the injected timeout)
    if (M > BM && !inject_timeout) return launch_pair(A, sa, B, sb, M, N, K, y, acc, stream);
    CUtensorMap ma, mb, my;
    if (!make_map_2d(&ma, CU_TENSOR_MAP_DATA_TYPE_UINT8, A, K, M, K, BK, BM, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map_2d(&mb, CU_TENSOR_MAP_DATA_TYPE_UINT8, B, K, N, K, BK, BN, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map_2d(&my, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, y, N, M, N * 2, kChunkCols, BM,
                     CU_TENSOR_MAP_SWIZZLE_64B))
        return cudaErrorInvalidValue;
    GemmParams p;
    p.sa = sa; p.sb = sb; p.acc = acc;
    p.M = (int)M; p.N = (int)N; p.K = (int)K;
    p.num_m = (int)((M + BM - 1) / BM);
    p.num_n = (int)((N + BN - 1) / BN);
    p.num_k = (int)((K + BK - 1) / BK);
    p.withhold = inject_timeout ? 1 : 0;
    p.limit_ns = inject_timeout ? kInjectedWaitLimitNs : kWaitLimitNs;
    static thread_local int attr_dev = -1;
    int dev = 0;
    cudaGetDevice(&dev);
    if (attr_dev != dev) {
        cudaError_t e = cudaFuncSetAttribute(w4a4_gemm_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemTotal);
        if (e != cudaSuccess) return e;
        attr_dev = dev;
    }
    const int tiles = p.num_m * p.num_n;
    const int sms = sm_count();
    const int grid = tiles < sms ? tiles : sms;
    return launch_pdl(w4a4_gemm_kernel, dim3(grid), dim3(kThreads), kSmemTotal, stream, ma, mb, my, p);
}

int read_and_clear_gemm_status(cudaStream_t stream, cudaError_t* err) {
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

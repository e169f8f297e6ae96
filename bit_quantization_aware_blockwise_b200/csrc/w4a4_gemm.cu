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

#include <mutex>

#include "quest_internal.h"

namespace quest {

// Device-side status word of the integer linear layer (0 = fine). Written only
// when a bounded wait gives up; read and cleared by quest_device_status().
__device__ int g_gemm_status = 0;

namespace {

constexpr int BM = 128, BN = 256, BK = 128;   // BK in int8 elements (= bytes)
constexpr int kStages = 4;
constexpr int kUmmaK = 32;                    // K of one kind::i8 MMA
constexpr int kThreads = 192;
constexpr int kEpiThreads = 128;
constexpr int kChunkCols = 32;                // epilogue columns per TMEM load / TMA store
constexpr uint32_t kTmemCols = 512;           // two 256-column accumulators
constexpr uint32_t kStageA = BM * BK, kStageB = BN * BK, kStageBytes = kStageA + kStageB;
constexpr uint32_t kCBytes = BM * kChunkCols * 2;  // one bf16 staging chunk (8 KB)
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
constexpr uint64_t kWaitLimitNs = 2000000000ull;            // 2 s per wait

// Instruction descriptor of tcgen05.mma kind::i8: D int32, A and B signed
// int8, both K-major, M = 128, N = 256.
constexpr uint32_t kIdesc = (2u << 4)           // D format: s32
                            | (1u << 7)         // A: signed 8-bit
                            | (1u << 10)        // B: signed 8-bit
                            | (uint32_t(BN >> 3) << 17) | (uint32_t(BM >> 4) << 24);

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Bounded wait for the phase of `bar` with parity `parity`. Returns false when
// the CTA is aborting (another role timed out) or this wait timed out.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          uint64_t limit_ns = kWaitLimitNs) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 63u) == 0) {
            if (*abort_flag) return false;
            if (global_timer_ns() - t0 > limit_ns) {
                *abort_flag = 1;
                atomicExch(&g_gemm_status, (int)QUEST_ETIMEOUT);
                return false;
            }
        }
    }
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int c0, int c1,
                                            uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(bar)
        : "memory");
}
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, uint32_t src, int c0, int c1) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(c0), "r"(c1), "r"(src)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read_le1() {
    asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 1, %0;" ::"n"(kEpiThreads) : "memory"); }
// OR-vote over the 128 epilogue threads (named barrier 1).
__device__ __forceinline__ bool epi_any(bool pred) {
    uint32_t out;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, 1, %2, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(out)
        : "r"((uint32_t)pred), "n"(kEpiThreads)
        : "memory");
    return out != 0;
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}
__device__ __forceinline__ void tc_mma_i8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(kIdesc), "r"(accumulate)
        : "memory");
}

// Shared-memory matrix descriptor of a K-major tile with 128-byte rows and the
// 128-byte swizzle written by TMA: 8-row core groups 1024 bytes apart.
__device__ __forceinline__ uint64_t smem_desc_k128(uint32_t addr) {
    uint64_t d = 0;
    d |= uint64_t((addr >> 4) & 0x3FFFu);          // start address
    d |= uint64_t(1) << 16;                        // leading byte offset (unused for swizzled K-major)
    d |= uint64_t(1024 >> 4) << 32;                // stride byte offset: 8 rows x 128 B
    d |= uint64_t(1) << 46;                        // descriptor version (sm_100)
    d |= uint64_t(2) << 61;                        // layout: 128-byte swizzle
    return d;
}

#define QUEST_TMEM_LD32(taddr, r)                                                              \
    asm volatile(                                                                              \
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "                                             \
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"                              \
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"             \
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), \
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),          \
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),       \
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),       \
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),       \
          "=r"(r[31])                                                                          \
        : "r"(taddr))

#define QUEST_TMEM_LD16(taddr, r)                                                              \
    asm volatile(                                                                              \
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "                                             \
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"                      \
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), \
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),          \
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])                                                \
        : "r"(taddr))

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

struct GemmParams {
    const float* sa;
    const float* sb;
    int32_t* acc;       // optional int32 copy of the accumulator
    int M, N, K;
    int num_m, num_n, num_k;
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

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            uint32_t stage = 0, phase = 0;
            uint64_t issued = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
                const int m0 = (tile % p.num_m) * BM, n0 = (tile / p.num_m) * BN;
                for (int kb = 0; kb < p.num_k; ++kb) {
                    if (!mbar_wait(bar_empty + 8 * stage, phase ^ 1, abort_flag)) { ok = false; break; }
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
                if (!mbar_wait(bar_tempty + 8 * buf, bphase ^ 1, abort_flag)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + buf * BN;
                for (int kb = 0; kb < p.num_k; ++kb) {
                    if (!mbar_wait(bar_full + 8 * stage, phase, abort_flag)) { ok = false; break; }
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
            const bool got = mbar_wait(bar_tfull + 8 * buf, bphase, abort_flag);
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
                        const float y0 = (float)(int32_t)r[i] * sa_half * sc[i];
                        const float y1 = (float)(int32_t)r[i + 1] * sa_half * sc[i + 1];
                        __nv_bfloat162 hb = __floats2bfloat162_rn(y0, y1);
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

constexpr int kPStages = 6;
constexpr uint32_t kPStageA = 128 * BK, kPStageB = 128 * BK;      // per CTA
constexpr uint32_t kPTxBytes = 2 * (kPStageA + kPStageB);         // both CTAs land on one barrier
constexpr uint32_t kPSmemA = 0;
constexpr uint32_t kPSmemB = kPSmemA + kPStages * kPStageA;
constexpr uint32_t kPSmemC = kPSmemB + kPStages * kPStageB;
constexpr uint32_t kPSmemScale = kPSmemC + 2 * kCBytes;
constexpr uint32_t kPSmemBar = kPSmemScale + BN * 4;
constexpr uint32_t kPNumBars = 2 * kPStages + 4 + 1;
constexpr uint32_t kPSmemTmemSlot = kPSmemBar + kPNumBars * 8;
constexpr uint32_t kPSmemAbort = kPSmemTmemSlot + 4;
constexpr uint32_t kPSmemUsed = kPSmemAbort + 4;
constexpr uint32_t kPSmemTotal = kPSmemUsed + 1024;
static_assert(kPSmemTotal <= 227 * 1024, "pair kernel shared memory");

// kind::i8, s32 accumulator, signed A and B, K-major, M = 256, N = 256.
constexpr uint32_t kIdescPair = (2u << 4) | (1u << 7) | (1u << 10) | (uint32_t(BN >> 3) << 17) |
                                (uint32_t(256 >> 4) << 24);

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// Shared::cluster address of the same shared-memory offset in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t map_to_rank(uint32_t addr, uint32_t rank) {
    uint32_t d;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(d) : "r"(addr), "r"(rank));
    return d;
}
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Arrive on a barrier that may live in the peer CTA (default .release.cta
// semantics: the caller orders its TMEM reads with tcgen05.fence::before_thread_sync;
// a cluster-scope release would wait for the whole CTA's memory traffic).
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
// TMA load into this CTA's shared memory whose completion is counted on a
// barrier that may live in the peer CTA (`bar` is a shared::cluster address).
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map, int c0, int c1,
                                                 uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(bar)
        : "memory");
}
__device__ __forceinline__ void tc_commit_pair_mc(uint32_t bar) {
    // arrive once on `bar` (same offset) in both CTAs of the pair
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
            bar),
        "h"((uint16_t)0x3)
        : "memory");
}
__device__ __forceinline__ void tc_commit_pair(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}
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
                    if (!mbar_wait(bar_empty + 8 * stage, phase ^ 1, abort_flag)) { ok = false; break; }
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
                if (!mbar_wait(bar_tempty + 8 * buf, bphase ^ 1, abort_flag)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + buf * BN;
                for (int kb = 0; kb < p.num_k; ++kb) {
                    if (!mbar_wait(bar_full + 8 * stage, phase, abort_flag)) { ok = false; break; }
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
            const bool got = mbar_wait(bar_tfull + 8 * buf, bphase, abort_flag);
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
                        const float y0 = (float)(int32_t)r[i] * sa_half * sc[i];
                        const float y1 = (float)(int32_t)r[i + 1] * sa_half * sc[i + 1];
                        __nv_bfloat162 hb = __floats2bfloat162_rn(y0, y1);
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

// ---------------------------------------------------------------------------
// Per-group scales along K (one scale per row and per 128-wide K group on both
// operands): Y[m][n] = sum_g (sa[m][g]/2)(sb[n][g]/2) * P_g[m][n], P_g the
// product of group g's codes. The codes come as FP8 E4M3 (c = 2q + 1, odd,
// |c| <= 15, exact in E4M3), so tcgen05 kind::f8f6f4 with fp32 accumulation
// gives every P_g exactly (integers below 2^24) with no int -> float step.
// CTA pairs as above, tiles of 256 x 128, one stage per group; the MMA cycles
// four 128-column TMEM slots, one group each, and eight epilogue warps (two per
// TMEM lane quarter, 64 columns each) fold every group into fp32 accumulators
// held in registers: acc += P_g * (sa/2)(sb/2), two packed FMA-class
// instructions per pair of outputs per group. A group's completion is read off
// its stage's empty barrier (one commit per group). This layer is bounded by the
// TMEM round trip, not the tensor cores: four slots hold about 1000 cycles of
// MMA work per SM, while a slot takes about 3000 cycles from the commit to its
// release by both CTAs' epilogues (clock64 counters on B200).

constexpr int kGThreads = 320;               // producer, MMA, 8 epilogue warps
constexpr int kGEpiThreads = 256;
constexpr int kGBN = 128;                    // output columns per pair tile
constexpr int kGStages = 6;
constexpr int kGSlots = 4;                   // TMEM slots of kGBN columns
constexpr int kGroup = 128;                  // K group = one stage
constexpr int kGScaleBlock = 16;             // groups of scales staged at a time
constexpr uint32_t kGStageA = 128 * BK, kGStageB = (kGBN / 2) * BK;   // per CTA
constexpr uint32_t kGTxBytes = 2 * (kGStageA + kGStageB);
constexpr uint32_t kGSmemA = 0;
constexpr uint32_t kGSmemB = kGSmemA + kGStages * kGStageA;
constexpr uint32_t kGScaleBytes = kGScaleBlock * (kGBN + 128) * 4;    // one block: sb [16][128], sa [16][128]
constexpr uint32_t kGSmemS = kGSmemB + kGStages * kGStageB;           // two blocks (double buffer)
constexpr uint32_t kGSmemC = kGSmemS + 2 * kGScaleBytes;              // 8 warps x 2 x 2 KB
constexpr uint32_t kGCBytes = 32 * 32 * 2;                            // 32 rows x 32 bf16
constexpr uint32_t kGSmemBar = kGSmemC + 8 * 2 * kGCBytes;
constexpr uint32_t kGNumBars = 2 * kGStages + kGSlots + 1;
constexpr uint32_t kGSmemTmemSlot = kGSmemBar + kGNumBars * 8;
constexpr uint32_t kGSmemAbort = kGSmemTmemSlot + 4;
constexpr uint32_t kGSmemUsed = kGSmemAbort + 4;
constexpr uint32_t kGSmemTotal = kGSmemUsed + 1024;
static_assert(kGSmemTotal <= 227 * 1024, "grouped kernel shared memory");
static_assert(kGSlots * kGBN == kTmemCols, "TMEM slots");
static_assert(kGSlots < kGStages, "the epilogue reads group completion off the stage barriers");

// kind::f8f6f4, f32 accumulator, A and B E4M3, K-major, M = 256, N = 128.
constexpr uint32_t kIdescGrouped = (1u << 4) | (0u << 7) | (0u << 10) | (uint32_t(kGBN >> 3) << 17) |
                                   (uint32_t(256 >> 4) << 24);

__device__ __forceinline__ void tc_mma_f8_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                               uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(kIdescGrouped), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void gepi_bar() {
    asm volatile("bar.sync 1, %0;" ::"n"(kGEpiThreads) : "memory");
}
__device__ __forceinline__ bool gepi_any(bool pred) {
    uint32_t out;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, 1, %2, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(out)
        : "r"((uint32_t)pred), "n"(kGEpiThreads)
        : "memory");
    return out != 0;
}

__device__ __forceinline__ void cp_async4(uint32_t dst, const float* src, bool valid) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src), "r"(valid ? 4 : 0)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

struct GroupedParams {
    const float* sa;    // [M, K / 128]
    const float* sb;    // [N, K / 128]
    float* y32;         // optional fp32 copy of Y [M, N]
    int M, N, K;
    int num_m2, num_n, num_k;   // 256-row pair tiles, 128-column tiles, K groups
};

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGThreads, 1)
w4a4_gemm_grouped_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                         const __grid_constant__ CUtensorMap map_y, const GroupedParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar_full = sbase + kGSmemBar;                 // [kGStages], used in the even CTA
    const uint32_t bar_empty = bar_full + 8 * kGStages;          // [kGStages]
    const uint32_t bar_tempty = bar_empty + 8 * kGStages;        // [kGSlots], used in the even CTA
    const uint32_t bar_drain = bar_tempty + 8 * kGSlots;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kGSmemAbort);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kGSmemTmemSlot);
    // scale blocks (double buffer): [16][128] sb[n0 + n][g0 + gg], then [16][128] sa[m0 + r][g0 + gg]
    float* s_sc = reinterpret_cast<float*>(smem + kGSmemS);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const bool even = rank == 0;
    const int pair = blockIdx.x >> 1, num_pairs = gridDim.x >> 1;
    const int num_tiles = p.num_m2 * p.num_n;
    const int G = p.num_k;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kGStages; ++s) {
            mbar_init(bar_full + 8 * s, 1);
            mbar_init(bar_empty + 8 * s, 1);
        }
        for (int b = 0; b < kGSlots; ++b) mbar_init(bar_tempty + 8 * b, 16);   // 8 epilogue warps x 2 CTAs
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

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer (both CTAs)
        if (lane == 0) {
            const uint32_t full_even = map_to_rank(bar_full, 0);
            uint32_t stage = 0, phase = 0;
            uint64_t issued = 0;
            bool ok = true;
            for (int tile = pair; tile < num_tiles && ok; tile += num_pairs) {
                const int m0 = (tile % p.num_m2) * 256 + 128 * int(rank);
                const int n0 = (tile / p.num_m2) * kGBN + (kGBN / 2) * int(rank);
                for (int kb = 0; kb < G; ++kb) {
                    if (!mbar_wait(bar_empty + 8 * stage, phase ^ 1, abort_flag)) { ok = false; break; }
                    if (even) mbar_arrive_expect_tx(bar_full + 8 * stage, kGTxBytes);
                    const uint32_t fb = full_even + 8 * stage;
                    tma_load_2d_pair(sbase + kGSmemA + stage * kGStageA, &map_a, kb * BK, m0, fb);
                    tma_load_2d_pair(sbase + kGSmemB + stage * kGStageB, &map_b, kb * BK, n0, fb);
                    ++issued;
                    if (++stage == kGStages) { stage = 0; phase ^= 1; }
                }
            }
            if (!ok && even) {
                const uint64_t n = issued < kGStages ? issued : kGStages;
                for (uint64_t i = issued - n; i < issued; ++i) {
                    const uint32_t st = uint32_t(i % kGStages), ph = uint32_t((i / kGStages) & 1);
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
            uint32_t gcount = 0;   // groups issued so far: TMEM slot = gcount % kGSlots
            bool ok = true;
            for (int tile = pair; tile < num_tiles && ok; tile += num_pairs) {
                for (int kb = 0; kb < G; ++kb, ++gcount) {
                    const uint32_t slot = gcount % kGSlots, sphase = (gcount / kGSlots) & 1;
                    if (!mbar_wait(bar_tempty + 8 * slot, sphase ^ 1, abort_flag)) { ok = false; break; }
                    if (!mbar_wait(bar_full + 8 * stage, phase, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t d_tmem = tmem_base + slot * kGBN;
                    const uint32_t a_addr = sbase + kGSmemA + stage * kGStageA;
                    const uint32_t b_addr = sbase + kGSmemB + stage * kGStageB;
#pragma unroll
                    for (int kk = 0; kk < BK / kUmmaK; ++kk) {
                        tc_mma_f8_pair(d_tmem, smem_desc_k128(a_addr + kk * kUmmaK),
                                       smem_desc_k128(b_addr + kk * kUmmaK), kk != 0);
                    }
                    // frees the stage in both CTAs and, the same event, marks this group's
                    // partials ready for the epilogue (which waits on this stage's barrier)
                    tc_commit_pair_mc(bar_empty + 8 * stage);
                    if (++stage == kGStages) { stage = 0; phase ^= 1; }
                }
            }
            tc_commit_pair(bar_drain);
            const uint64_t t0 = global_timer_ns();
            while (!mbar_try_wait(bar_drain, 0) && global_timer_ns() - t0 < kWaitLimitNs) {
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue (warps 2..9, both CTAs)
        const int et = threadIdx.x - 64;                   // 0..255
        const int ew = et >> 5;                            // epilogue warp 0..7
        const int quarter = warp & 3;                      // TMEM lanes 32*quarter .. +31
        const int half = ew >> 2;                          // columns 64*half .. +63 of the tile
        const int row_in_tile = quarter * 32 + lane;
        const uint32_t lane_addr = uint32_t(quarter * 32) << 16;
        const uint32_t tempty_even = map_to_rank(bar_tempty, 0);
        const uint32_t stg0 = sbase + kGSmemC + uint32_t(ew) * 2 * kGCBytes;
        const int Gs = p.K / kGroup;                       // scale columns per row
        // issue the copies of scale block (tile, g0) into buffer b: transposed to [group][column]
        auto prefetch = [&](int tile, int g0, int b) {
            if (tile < num_tiles) {
                const int pm0 = (tile % p.num_m2) * 256 + 128 * int(rank), pn0 = (tile / p.num_m2) * kGBN;
                const int nb = (G - g0) < kGScaleBlock ? (G - g0) : kGScaleBlock;
                const uint32_t base = sbase + kGSmemS + uint32_t(b) * kGScaleBytes;
#pragma unroll
                for (int k = 0; k < kGScaleBlock * kGBN / kGEpiThreads; ++k) {
                    const int i = et + k * kGEpiThreads, n = i / kGScaleBlock, gg = i % kGScaleBlock;
                    const bool v = gg < nb && pn0 + n < p.N;
                    cp_async4(base + 4 * (gg * kGBN + n), p.sb + (v ? int64_t(pn0 + n) * Gs + g0 + gg : 0), v);
                }
#pragma unroll
                for (int k = 0; k < kGScaleBlock * 128 / kGEpiThreads; ++k) {
                    const int i = et + k * kGEpiThreads, r = i / kGScaleBlock, gg = i % kGScaleBlock;
                    const bool v = gg < nb && pm0 + r < p.M;
                    cp_async4(base + 4 * (kGScaleBlock * kGBN + gg * 128 + r),
                              p.sa + (v ? int64_t(pm0 + r) * Gs + g0 + gg : 0), v);
                }
            }
            cp_async_commit();
        };
        uint32_t gcount = 0;
        int cbuf = 0, sbuf = 0;
        bool aborted = false;
        prefetch(pair, 0, 0);
        for (int tile = pair; tile < num_tiles && !aborted; tile += num_pairs) {
            const int m0 = (tile % p.num_m2) * 256 + 128 * int(rank), n0 = (tile / p.num_m2) * kGBN;
            float2 acc[32];   // columns 64*half + 2j, +1
#pragma unroll
            for (int j = 0; j < 32; ++j) acc[j] = make_float2(0.0f, 0.0f);
            for (int g = 0; g < G; ++g, ++gcount) {
                if ((g % kGScaleBlock) == 0) {
                    // a thread whose wait gave up stops the whole epilogue here (uniform exit)
                    if (gepi_any(aborted)) break;
                    // this block's scales have landed, and every thread is done with the other
                    // buffer: start copying the next block into it (one tile ahead at most)
                    cp_async_wait_all();
                    gepi_bar();
                    if (g + kGScaleBlock < G) prefetch(tile, g + kGScaleBlock, sbuf ^ 1);
                    else prefetch(tile + num_pairs, 0, sbuf ^ 1);
                }
                // group gcount's MMAs are complete when its stage's empty barrier completes
                // that use; the epilogue trails the MMA by at most kGSlots < kGStages groups,
                // so the parity cannot alias
                const uint32_t slot = gcount % kGSlots;
                const uint32_t gst = gcount % kGStages, gph = (gcount / kGStages) & 1;
                if (!mbar_wait(bar_empty + 8 * gst, gph, abort_flag)) aborted = true;
                if (aborted) continue;   // later waits return at once (abort flag); exit at the next check
                tc_fence_after();
                const uint32_t t_grp = tmem_base + lane_addr + slot * kGBN + 64 * half;
                uint32_t r0[32], r1[32];
                QUEST_TMEM_LD32(t_grp, r0);
                QUEST_TMEM_LD32(t_grp + 32, r1);
                tmem_wait_ld();
                // the group's partials are in registers: hand the slot back
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_remote(tempty_even + 8 * slot);
                // (sa/2)(sb/2): the factor 1/4 rides on the row scale
                const float* sblk = s_sc + sbuf * (kGScaleBytes / 4);
                const float sx = 0.25f * sblk[kGScaleBlock * kGBN + (g % kGScaleBlock) * 128 + row_in_tile];
                const float4* sw4 = reinterpret_cast<const float4*>(sblk + (g % kGScaleBlock) * kGBN + 64 * half);
                if ((g % kGScaleBlock) == kGScaleBlock - 1 || g == G - 1) sbuf ^= 1;   // next block, other buffer
#pragma unroll
                for (int q4 = 0; q4 < 16; ++q4) {
                    const float4 w4 = sw4[q4];
                    const uint32_t* r = q4 < 8 ? r0 : r1;
                    const int i = (q4 & 7) * 4;
                    const float2 w01 = __fmul2_rn(make_float2(sx, sx), make_float2(w4.x, w4.y));
                    const float2 w23 = __fmul2_rn(make_float2(sx, sx), make_float2(w4.z, w4.w));
                    acc[2 * q4] = __ffma2_rn(make_float2(__uint_as_float(r[i]), __uint_as_float(r[i + 1])), w01,
                                             acc[2 * q4]);
                    acc[2 * q4 + 1] = __ffma2_rn(make_float2(__uint_as_float(r[i + 2]), __uint_as_float(r[i + 3])),
                                                 w23, acc[2 * q4 + 1]);
                }
            }
            if (gepi_any(aborted)) { aborted = true; break; }
            // ---- output: this warp's 32 rows x 64 columns, in 2 chunks of 32 columns
            const int m = m0 + row_in_tile;
            if (p.y32 != nullptr && m < p.M) {
                float* yrow = p.y32 + int64_t(m) * p.N + n0 + 64 * half;
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int n = n0 + 64 * half + 2 * j;
                    if (n < p.N) yrow[2 * j] = acc[j].x;
                    if (n + 1 < p.N) yrow[2 * j + 1] = acc[j].y;
                }
            }
            const uint32_t swz = (lane >> 1) & 3;
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                if (lane == 0) bulk_wait_read_le1();   // the buffer used two chunks ago is free
                __syncwarp();
                const uint32_t stg = stg0 + cbuf * kGCBytes + lane * 64;
#pragma unroll
                for (int q16 = 0; q16 < 4; ++q16) {
                    uint32_t w[4];
#pragma unroll
                    for (int h = 0; h < 4; ++h) {
                        const float2 v = acc[c * 16 + q16 * 4 + h];
                        __nv_bfloat162 hb = __floats2bfloat162_rn(v.x, v.y);
                        w[h] = *reinterpret_cast<uint32_t*>(&hb);
                    }
                    asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(stg + ((q16 ^ swz) << 4)),
                                 "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3])
                                 : "memory");
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    tma_store_2d(&map_y, stg0 + cbuf * kGCBytes, n0 + 64 * half + c * kChunkCols, m0 + 32 * quarter);
                    bulk_commit();
                }
                cbuf ^= 1;
            }
        }
        cp_async_wait_all();   // no copy may still target shared memory at exit
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
// no exchange, and G never reaches HBM.
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

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
trust_linear_pair_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
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

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer (both CTAs)
        if (lane == 0) {
            const uint32_t full_even = map_to_rank(bar_full, 0);
            uint32_t stage = 0, phase = 0;
            uint64_t issued = 0;
            bool ok = true;
            for (int tile = pair; tile < num_tiles && ok; tile += num_pairs) {
                const int m0 = (tile % p.num_m2) * 256 + 128 * int(rank);
                const int k0 = (tile / p.num_m2) * BN + 128 * int(rank);
                for (int kb = 0; kb < p.num_k; ++kb) {
                    if (!mbar_wait(bar_empty + 8 * stage, phase ^ 1, abort_flag)) { ok = false; break; }
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
                if (!mbar_wait(bar_tempty + 8 * buf, bphase ^ 1, abort_flag)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + buf * BN;
                for (int kb = 0; kb < p.num_k; ++kb) {
                    if (!mbar_wait(bar_full + 8 * stage, phase, abort_flag)) { ok = false; break; }
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
            const int m0 = (tile % p.num_m2) * 256 + 128 * int(rank), k0 = (tile / p.num_m2) * BN;
            const uint32_t buf = local & 1, bphase = (local >> 1) & 1;
            const int m = m0 + row_in_tile;
            // this row's mask bits for the tile's two blocks, fetched before the wait
            uint4 mw[2];
#pragma unroll
            for (int b = 0; b < 2; ++b) {
                const int kb0 = k0 + 128 * b;
                mw[b] = (m < p.M && kb0 < p.K)
                            ? *reinterpret_cast<const uint4*>(p.mask + int64_t(m) * mask_row_bytes + kb0 / 8)
                            : make_uint4(0u, 0u, 0u, 0u);
            }
            const bool got = mbar_wait(bar_tfull + 8 * buf, bphase, abort_flag);
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
                        // keep G where the mask bit is 1 (bit j of the word = column 32c + j)
                        const uint32_t k0m = 0u - ((bits >> (2 * i)) & 1u);
                        const uint32_t k1m = 0u - ((bits >> (2 * i + 1)) & 1u);
                        w[16 * c + i] = make_float2(__uint_as_float(r[2 * i] & k0m), __uint_as_float(r[2 * i + 1] & k1m));
                    }
                }
                fwht128_regs(w);
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
                            __nv_bfloat162 hb = __floats2bfloat162_rn(v.x * p.scale, v.y * p.scale);
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

// Writes zeros (K == 0: the empty sum).
__global__ void zero_fill_kernel(uint16_t* y, int32_t* acc, int64_t n) {
    for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
         i += int64_t(gridDim.x) * blockDim.x) {
        y[i] = 0;
        if (acc) acc[i] = 0;
    }
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

bool make_map_2d(CUtensorMap* map, CUtensorMapDataType dt, const void* base, uint64_t inner,
                 uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
                 CUtensorMapSwizzle swz) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {row_bytes};
    const cuuint32_t box[2] = {box_inner, box_outer};
    const cuuint32_t estr[2] = {1, 1};
    return fn(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Co-resident CTA pairs of a cluster kernel on the current device (cached per
// kernel; the kernel's shared-memory attribute must already be set).
int pair_clusters(int dev, const void* kernel, int threads, uint32_t smem) {
    constexpr int kSlots = 4;
    static int cached_dev[kSlots] = {-1, -1, -1, -1}, cached[kSlots] = {0, 0, 0, 0};
    static const void* cached_fn[kSlots] = {nullptr, nullptr, nullptr, nullptr};
    static int next_slot = 0;
    static std::mutex mu;
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < kSlots; ++i)
        if (cached_fn[i] == kernel && cached_dev[i] == dev) return cached[i];
    int n = 0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * (sm_count() / 2), 1, 1);
    cfg.blockDim = dim3(threads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) != cudaSuccess || n <= 0) {
        cudaGetLastError();
        n = sm_count() / 2;
    }
    const int slot = next_slot;
    next_slot = (next_slot + 1) % kSlots;
    cached_fn[slot] = kernel;
    cached_dev[slot] = dev;
    cached[slot] = n;
    return n;
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
    w4a4_gemm_pair_kernel<<<2 * grid_pairs, kThreads, kPSmemTotal, stream>>>(ma, mb, my, p);
    return cudaGetLastError();
}

cudaError_t launch_grouped(const int8_t* A, const float* sa, const int8_t* B, const float* sb, int64_t M,
                           int64_t N, int64_t K, uint16_t* y, float* y32, cudaStream_t stream) {
    CUtensorMap ma, mb, my;
    if (!make_map_2d(&ma, CU_TENSOR_MAP_DATA_TYPE_UINT8, A, K, M, K, BK, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map_2d(&mb, CU_TENSOR_MAP_DATA_TYPE_UINT8, B, K, N, K, BK, kGBN / 2, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map_2d(&my, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, y, N, M, N * 2, kChunkCols, 32,
                     CU_TENSOR_MAP_SWIZZLE_64B))
        return cudaErrorInvalidValue;
    GroupedParams p;
    p.sa = sa; p.sb = sb; p.y32 = y32;
    p.M = (int)M; p.N = (int)N; p.K = (int)K;
    p.num_m2 = (int)((M + 255) / 256);
    p.num_n = (int)((N + kGBN - 1) / kGBN);
    p.num_k = (int)(K / kGroup);
    static thread_local int attr_dev = -1;
    int dev = 0;
    cudaGetDevice(&dev);
    if (attr_dev != dev) {
        cudaError_t e = cudaFuncSetAttribute(w4a4_gemm_grouped_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, kGSmemTotal);
        if (e != cudaSuccess) return e;
        attr_dev = dev;
    }
    const int tiles = p.num_m2 * p.num_n;
    const int pairs = pair_clusters(dev, (const void*)w4a4_gemm_grouped_kernel, kGThreads, kGSmemTotal);
    const int grid_pairs = tiles < pairs ? tiles : pairs;
    w4a4_gemm_grouped_kernel<<<2 * grid_pairs, kGThreads, kGSmemTotal, stream>>>(ma, mb, my, p);
    return cudaGetLastError();
}

cudaError_t launch_trust_linear_pair(const uint16_t* gy, const uint16_t* wt, const uint8_t* mask, int64_t M,
                                     int64_t N, int64_t K, uint16_t* gx, cudaStream_t stream) {
    CUtensorMap ma, mb, my;
    if (!make_map_2d(&ma, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, gy, N, M, N * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map_2d(&mb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, wt, N, K, N * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map_2d(&my, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, gx, K, M, K * 2, kChunkCols, 128,
                     CU_TENSOR_MAP_SWIZZLE_64B))
        return cudaErrorInvalidValue;
    TrustLinearParams p;
    p.mask = mask;
    p.scale = 0.08838834764831845f;   // 1 / sqrt(128)
    p.M = (int)M; p.N = (int)N; p.K = (int)K;
    p.num_m2 = (int)((M + 255) / 256);
    p.num_n = (int)((K + BN - 1) / BN);
    p.num_k = (int)((N + 63) / 64);
    static thread_local int attr_dev = -1;
    int dev = 0;
    cudaGetDevice(&dev);
    if (attr_dev != dev) {
        cudaError_t e = cudaFuncSetAttribute(trust_linear_pair_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, kPSmemTotal);
        if (e != cudaSuccess) return e;
        attr_dev = dev;
    }
    const int tiles = p.num_m2 * p.num_n;
    const int pairs = pair_clusters(dev, (const void*)trust_linear_pair_kernel, kThreads, kPSmemTotal);
    const int grid_pairs = tiles < pairs ? tiles : pairs;
    trust_linear_pair_kernel<<<2 * grid_pairs, kThreads, kPSmemTotal, stream>>>(ma, mb, my, p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_trust_linear(const uint16_t* gy, const uint16_t* wt, const uint8_t* mask, int64_t M,
                                int64_t N, int64_t K, uint16_t* gx, cudaStream_t stream) {
    if (M == 0 || K == 0) return cudaSuccess;
    if (N == 0) {   // the empty sum: G = 0, so the gradient is 0
        const int64_t n = M * K;
        int64_t blocks = (n + 255) / 256;
        if (blocks > 4096) blocks = 4096;
        zero_fill_kernel<<<(int)blocks, 256, 0, stream>>>(gx, nullptr, n);
        return cudaGetLastError();
    }
    return launch_trust_linear_pair(gy, wt, mask, M, N, K, gx, stream);
}

cudaError_t launch_w4a4_grouped(const int8_t* A, const float* sa, const int8_t* B, const float* sb,
                                int64_t M, int64_t N, int64_t K, uint16_t* y, float* y32,
                                cudaStream_t stream) {
    if (M == 0 || N == 0) return cudaSuccess;
    if (K == 0) {
        const int64_t n = M * N;
        int64_t blocks = (n + 255) / 256;
        if (blocks > 4096) blocks = 4096;
        zero_fill_kernel<<<(int)blocks, 256, 0, stream>>>(y, nullptr, n);
        if (y32) cudaMemsetAsync(y32, 0, size_t(n) * sizeof(float), stream);
        return cudaGetLastError();
    }
    return launch_grouped(A, sa, B, sb, M, N, K, y, y32, stream);
}

cudaError_t launch_w4a4(const int8_t* A, const float* sa, const int8_t* B, const float* sb,
                        int64_t M, int64_t N, int64_t K, uint16_t* y, int32_t* acc,
                        cudaStream_t stream) {
    if (M == 0 || N == 0) return cudaSuccess;
    if (K == 0) {
        const int64_t n = M * N;
        int64_t blocks = (n + 255) / 256;
        if (blocks > 4096) blocks = 4096;
        zero_fill_kernel<<<(int)blocks, 256, 0, stream>>>(y, acc, n);
        return cudaGetLastError();
    }
    // more than one 128-row block: CTA pairs (M = 256 tiles); otherwise one CTA per tile
    if (M > BM) return launch_pair(A, sa, B, sb, M, N, K, y, acc, stream);
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
    w4a4_gemm_kernel<<<grid, kThreads, kSmemTotal, stream>>>(ma, mb, my, p);
    return cudaGetLastError();
}

int read_and_clear_gemm_status(cudaStream_t stream, cudaError_t* err) {
    int v = 0, zero = 0;
    cudaError_t e = cudaMemcpyFromSymbolAsync(&v, g_gemm_status, sizeof(int), 0,
                                              cudaMemcpyDeviceToHost, stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    if (e == cudaSuccess && v != 0)
        e = cudaMemcpyToSymbolAsync(g_gemm_status, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    *err = e;
    return v;
}

}  // namespace quest

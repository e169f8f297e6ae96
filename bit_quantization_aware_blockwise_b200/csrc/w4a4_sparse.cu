// Linear layer on 2:4-sparse QuEST weight codes: tcgen05.mma.sp kind::i8 with
// the weights as the sparse operand (sm_100a).
//
//   acc[m][n] = sum_k X[m][k] * W[n][k]      (W 2:4-sparse along k; int8 -> int32, exact)
//   y[m][n]   = bf16_rne(acc * (sx[m]/2) * (sw[n]/2))
//
// The pages evaluate QuEST with 2:4 sparsity added to INT4 (atlas.scime.ai summary
// of QuEST, ablation table; pith.science review, Figure 4a). The sparse tensor
// cores take the sparse operand as A (the M side of the MMA), so the product runs
// transposed: A = the compressed weight codes (128 weight rows per tile), B = the
// activation codes (224 tokens per tile), D[n][m] in TMEM, and the epilogue writes
// y[m][n] through a transposed shared-memory stage.
//
// Operands per stage (128 logical K values):
//   A  compressed weights, 128 rows x 64 bytes (the two survivors of each run of
//      four), 64-byte swizzle;
//   B  activation codes, 224 rows x 128 bytes, 128-byte swizzle;
//   E  metadata, 128 rows x 16 bytes (a nibble per run: the lower survivor's index
//      in bits 0-1, the higher one's in bits 2-3), no swizzle, copied into TMEM
//      (tcgen05.cp 128x128b: lane = weight row, four 32-bit columns).
// Each stage is two sparse MMAs (M = 128, N = 224, K = 64 logical); MMA j reads
// its metadata from columns 2j, 2j+1 of the stage's slot.
//
// Two kernels. With at most 128 weight rows (N <= 128), one persistent CTA per SM
// (192 threads: warp 0 TMA producer, warp 1 TMEM allocator, metadata copies and
// MMA issuer, warps 2-5 epilogue), the structure above. Otherwise CTA pairs
// (cluster of two, cta_group::2, M = 256 weight rows per MMA; see below). In both,
// two 224-column accumulators alternate (the epilogue of tile i overlaps the
// mainloop of tile i + 1) and the metadata columns sit after them; each epilogue
// warp stores its own 32 weight rows through staging buffers of its own. No TMA
// multicast. Every wait is bounded in time; on timeout the CTA records
// QUEST_ETIMEOUT, drains its copies and MMAs, frees TMEM and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace quest {
namespace {
// Device-side status word of this file's kernel (0 = fine); read and cleared by
// quest_device_status().
__device__ int g_tc_status = 0;
}  // namespace
}  // namespace quest

#include "tc_common.cuh"

namespace quest {
namespace {

constexpr int SBM = 128;                 // weight rows per tile (MMA M)
constexpr int SBN = 224;                 // tokens per tile (MMA N)
constexpr int SBK = 128;                 // logical K per stage
constexpr int kSStages = 5;
constexpr uint32_t kSStageA = SBM * SBK / 2;        // 8 KB: compressed weights
constexpr uint32_t kSStageB = SBN * SBK;            // 28 KB: activation codes
constexpr uint32_t kSStageE = SBM * SBK / 8;        // 2 KB: metadata
constexpr uint32_t kSTx = kSStageA + kSStageB + kSStageE;
constexpr uint32_t kSSmemA = 0;
constexpr uint32_t kSSmemB = kSSmemA + kSStages * kSStageA;
constexpr uint32_t kSSmemE = kSSmemB + kSStages * kSStageB;
// Transposed output stage: every epilogue warp owns kStgBufs buffers of 32 tokens x its 32
// weight rows (bf16, 2 KB), each written back by the warp's own TMA store.
constexpr int kStgBufs = 4;
constexpr uint32_t kStgBytes = 32 * 32 * 2;
constexpr uint32_t kSCBytes = 4 * kStgBufs * kStgBytes;   // 32 KB per CTA
constexpr uint32_t kSSmemC = kSSmemE + kSStages * kSStageE;
constexpr uint32_t kSSmemScale = kSSmemC + kSCBytes;       // float[SBN]: the tokens' scales
static_assert(kSSmemScale % 16 == 0, "16-byte scale loads");
constexpr uint32_t kSSmemBar = kSSmemScale + SBN * 4;
constexpr uint32_t kSNumBars = 2 * kSStages + 4 + 1;
constexpr uint32_t kSSmemTmemSlot = kSSmemBar + kSNumBars * 8;
constexpr uint32_t kSSmemAbort = kSSmemTmemSlot + 4;
constexpr uint32_t kSSmemUsed = kSSmemAbort + 4;
constexpr uint32_t kSSmemTotal = kSSmemUsed + 1024;
static_assert(kSSmemTotal <= 227 * 1024, "sparse kernel shared memory");
static_assert(kSStageA % 1024 == 0 && kSStageB % 1024 == 0 && kSStageE % 1024 == 0, "stage alignment");
constexpr uint32_t kSAccCols = SBN;                  // accumulator buffers at columns 0 and SBN
constexpr uint32_t kSMetaCol = 2 * SBN;              // metadata slots: 4 columns per stage
static_assert(kSMetaCol + 4 * kSStages <= kTmemCols, "TMEM columns");

// tcgen05 kind::i8 with sparse A: D int32, A and B signed int8, K-major,
// M = 128, N = 224, sparsity flag (bit 2).
constexpr uint32_t kIdescSp = (1u << 2) | (2u << 4) | (1u << 7) | (1u << 10) | (uint32_t(SBN >> 3) << 17) |
                              (uint32_t(SBM >> 4) << 24);

__device__ __forceinline__ void tc_mma_sp_i8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t e_tmem,
                                             uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %5, 0;\n\t"
        "tcgen05.mma.sp.cta_group::1.kind::i8 [%0], %1, %2, [%3], %4, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(e_tmem), "r"(kIdescSp), "r"(accumulate)
        : "memory");
}

// K-major operand with 64-byte rows and the 64-byte swizzle written by TMA:
// 8-row core groups 512 bytes apart.
__device__ __forceinline__ uint64_t smem_desc_k64(uint32_t addr) {
    uint64_t d = 0;
    d |= uint64_t((addr >> 4) & 0x3FFFu);   // start address
    d |= uint64_t(1) << 16;                 // leading byte offset (unused for swizzled K-major)
    d |= uint64_t(512 >> 4) << 32;          // stride byte offset: 8 rows x 64 B
    d |= uint64_t(1) << 46;                 // descriptor version (sm_100)
    d |= uint64_t(4) << 61;                 // layout: 64-byte swizzle
    return d;
}
// The metadata stage: 128 rows of 16 bytes, no swizzle: 8-row core matrices of
// 128 contiguous bytes, 128 bytes apart.
__device__ __forceinline__ uint64_t smem_desc_meta(uint32_t addr) {
    uint64_t d = 0;
    d |= uint64_t((addr >> 4) & 0x3FFFu);
    d |= uint64_t(kSStageE >> 4) << 16;     // leading byte offset (a second 16-byte column; unused)
    d |= uint64_t(128 >> 4) << 32;          // stride byte offset: 8 rows x 16 B
    d |= uint64_t(1) << 46;
    return d;                               // layout 0: no swizzle
}
__device__ __forceinline__ void tc_cp_meta(uint32_t taddr, uint64_t sdesc) {
    asm volatile("tcgen05.cp.cta_group::1.128x128b [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

__device__ __forceinline__ void bulk_wait_read_stg() {
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(kStgBufs - 1) : "memory");
}

// 16 TMEM lanes x 32 columns in the 16x256b pattern: thread t receives, for k = 0..3,
// r[4k], r[4k+1] = lane t/4, columns 8k + 2(t%4), 8k + 2(t%4) + 1 and r[4k+2], r[4k+3] =
// lane t/4 + 8, the same columns (the fragment layout of an 8 x 8 matrix pair).
#define QUEST_TMEM_LD16X256_X4(taddr, r)                                                       \
    asm volatile(                                                                              \
        "tcgen05.ld.sync.aligned.16x256b.x4.b32 "                                             \
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"                      \
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), \
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),          \
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])                                                \
        : "r"(taddr))

// Four 8 x 8 bf16 matrices, each stored transposed (rows of the fragment become columns).
__device__ __forceinline__ void stmatrix_x4_trans(uint32_t addr, uint32_t r0, uint32_t r1, uint32_t r2,
                                                  uint32_t r3) {
    asm volatile("stmatrix.sync.aligned.m8n8.x4.trans.shared.b16 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(r0),
                 "r"(r1), "r"(r2), "r"(r3)
                 : "memory");
}

// This warp's 32 weight rows x SBN tokens of a finished accumulator out to y[m][n]. The
// accumulator holds D[n][m] (lane = weight row), y wants rows of tokens, so each 32-token
// chunk is read in the 16x256b pattern, in which a thread holds two adjacent tokens of two
// weight rows: scaled, rounded to bf16 pairs, these are the fragments of 8 x 8 matrices that
// stmatrix.trans writes transposed into a staging buffer laid out as y's rows ([token][32
// weight rows], 64-byte swizzle); the warp's own TMA store writes the 32 x 32 box. Four
// stmatrix per chunk replace 32 16-bit stores of a thread-per-row layout. The buffer is
// reused once at most kStgBufs - 1 of the warp's stores are still reading. n_w: the warp's
// first weight row; sw_half: the scale of weight row n_w + lane. Lane 0 issues the stores.
__device__ __forceinline__ void store_tile_transposed(const CUtensorMap& map_y, uint32_t t_acc, uint32_t stg_addr,
                                                      int& cbuf, int lane, int n_w, int m0, float sw_half,
                                                      const float* s_scale, int32_t* acc, int M, int N) {
    const int g = lane >> 2, t = lane & 3, q = lane >> 3, rr = lane & 7;
    // scales of the weight rows this thread holds: n_w + 16h + 8rb + g
    float swr[2][2];
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int rb = 0; rb < 2; ++rb) swr[h][rb] = __shfl_sync(0xFFFFFFFFu, sw_half, 16 * h + 8 * rb + g);
#pragma unroll 1
    for (int c = 0; c < SBN / 32; ++c) {
        uint32_t ra[2][16];   // lanes 0-15 and 16-31 of the warp's quarter
        QUEST_TMEM_LD16X256_X4(t_acc + c * 32, ra[0]);
        QUEST_TMEM_LD16X256_X4(t_acc + (16u << 16) + c * 32, ra[1]);
        tmem_wait_ld();
        if (lane == 0) bulk_wait_read_stg();
        __syncwarp();
        const uint32_t base = stg_addr + cbuf * kStgBytes;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            uint32_t P[4][2];   // [8-token block k][weight-row block rb]: a bf16 pair
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float2 s = *reinterpret_cast<const float2*>(s_scale + c * 32 + 8 * k + 2 * t);
#pragma unroll
                for (int rb = 0; rb < 2; ++rb) {
                    // (acc * sw/2) * sx/2 per token, two tokens per packed multiply
                    const float2 v = __fmul2_rn(__fmul2_rn(make_float2((float)(int32_t)ra[h][4 * k + 2 * rb],
                                                                       (float)(int32_t)ra[h][4 * k + 2 * rb + 1]),
                                                           make_float2(swr[h][rb], swr[h][rb])),
                                                s);
                    __nv_bfloat162 hb = __floats2bfloat162_rn(v.x, v.y);
                    P[k][rb] = *reinterpret_cast<uint32_t*>(&hb);
                }
            }
            // matrix j of an x4 takes its row addresses from threads 8j .. 8j + 7: token
            // 8k + rr of the chunk, weight-row block nb (16 bytes), 64-byte swizzle
#pragma unroll
            for (int kp = 0; kp < 2; ++kp) {
                const int k = 2 * kp + (q >> 1), nb = 2 * h + (q & 1), m = 8 * k + rr;
                const uint32_t addr = base + uint32_t(m) * 64u + (uint32_t(nb ^ ((m >> 1) & 3)) << 4);
                stmatrix_x4_trans(addr, P[2 * kp][0], P[2 * kp][1], P[2 * kp + 1][0], P[2 * kp + 1][1]);
            }
            if (acc != nullptr) {
#pragma unroll
                for (int k = 0; k < 4; ++k)
#pragma unroll
                    for (int rb = 0; rb < 2; ++rb)
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            const int n = n_w + 16 * h + 8 * rb + g, m = m0 + c * 32 + 8 * k + 2 * t + e;
                            if (n < N && m < M) acc[int64_t(m) * N + n] = (int32_t)ra[h][4 * k + 2 * rb + e];
                        }
            }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
            tma_store_2d(&map_y, base, n_w, m0 + c * 32);
            bulk_commit();
        }
        cbuf = cbuf + 1 == kStgBufs ? 0 : cbuf + 1;
    }
}

struct SparseParams {
    const float* sx;    // token scales [M]
    const float* sw;    // weight row scales [N]
    int32_t* acc;       // optional int32 copy of the accumulator [M][N]
    int M, N, K;
    int num_n, num_m, num_k;   // weight-row tiles (128), token tiles (224), K stages (128)
};

__global__ void __launch_bounds__(kThreads, 1)
w4a4_sparse_kernel(const __grid_constant__ CUtensorMap map_w, const __grid_constant__ CUtensorMap map_x,
                   const __grid_constant__ CUtensorMap map_e, const __grid_constant__ CUtensorMap map_y,
                   const SparseParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar_full = sbase + kSSmemBar;             // [kSStages]
    const uint32_t bar_empty = bar_full + 8 * kSStages;      // [kSStages]
    const uint32_t bar_tfull = bar_empty + 8 * kSStages;     // [2]
    const uint32_t bar_tempty = bar_tfull + 16;              // [2]
    const uint32_t bar_drain = bar_tempty + 16;              // [1]
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kSSmemAbort);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kSSmemTmemSlot);
    float* s_scale = reinterpret_cast<float*>(smem + kSSmemScale);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int num_tiles = p.num_n * p.num_m;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kSStages; ++s) {
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
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_w)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_x)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_e)) : "memory");
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
    pdl_wait();
    pdl_trigger();

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            uint32_t stage = 0, phase = 0;
            uint64_t issued = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
                const int n0 = (tile % p.num_n) * SBM, m0 = (tile / p.num_n) * SBN;
                for (int kb = 0; kb < p.num_k; ++kb) {
                    if (!mbar_wait(bar_empty + 8 * stage, phase ^ 1, abort_flag, kWaitLimitNs, kSuspendProducerNs)) {
                        ok = false;
                        break;
                    }
                    const uint32_t fb = bar_full + 8 * stage;
                    mbar_arrive_expect_tx(fb, kSTx);
                    tma_load_2d(sbase + kSSmemA + stage * kSStageA, &map_w, kb * (SBK / 2), n0, fb);
                    tma_load_2d(sbase + kSSmemB + stage * kSStageB, &map_x, kb * SBK, m0, fb);
                    tma_load_2d(sbase + kSSmemE + stage * kSStageE, &map_e, kb * (SBK / 8), n0, fb);
                    ++issued;
                    if (++stage == kSStages) { stage = 0; phase ^= 1; }
                }
            }
            if (!ok) {
                const uint64_t n = issued < kSStages ? issued : kSStages;
                for (uint64_t i = issued - n; i < issued; ++i) {
                    const uint32_t st = uint32_t(i % kSStages), ph = uint32_t((i / kSStages) & 1);
                    const uint64_t t0 = global_timer_ns();
                    while (!mbar_try_wait(bar_full + 8 * st, ph) && global_timer_ns() - t0 < kWaitLimitNs) {
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ metadata copies and MMAs
        if (lane == 0) {
            uint32_t stage = 0, phase = 0;
            bool ok = true;
            int local = 0;
            for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++local) {
                const uint32_t buf = local & 1, bphase = (local >> 1) & 1;
                if (!mbar_wait(bar_tempty + 8 * buf, bphase ^ 1, abort_flag, kWaitLimitNs, kSuspendMmaNs)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + buf * kSAccCols;
                for (int kb = 0; kb < p.num_k; ++kb) {
                    if (!mbar_wait(bar_full + 8 * stage, phase, abort_flag, kWaitLimitNs, kSuspendMmaNs)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_addr = sbase + kSSmemA + stage * kSStageA;
                    const uint32_t b_addr = sbase + kSSmemB + stage * kSStageB;
                    const uint32_t e_tmem = tmem_base + kSMetaCol + 4 * stage;
                    // the copy and the MMAs after it run in issue order
                    tc_cp_meta(e_tmem, smem_desc_meta(sbase + kSSmemE + stage * kSStageE));
#pragma unroll
                    for (int kk = 0; kk < SBK / 64; ++kk) {
                        tc_mma_sp_i8(d_tmem, smem_desc_k64(a_addr + kk * 32), smem_desc_k128(b_addr + kk * 64),
                                     e_tmem + 2 * kk, (kb | kk) != 0);
                    }
                    tc_commit(bar_empty + 8 * stage);   // frees the stage (and its metadata slot)
                    if (++stage == kSStages) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
                tc_commit(bar_tfull + 8 * buf);
            }
            tc_commit(bar_drain);
            const uint64_t t0 = global_timer_ns();
            while (!mbar_try_wait(bar_drain, 0) && global_timer_ns() - t0 < kWaitLimitNs) {
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue (warps 2..5)
        const int et = threadIdx.x - 64;              // 0..127
        const int quarter = warp & 3;                 // TMEM lanes 32*quarter .. +31
        const int row = quarter * 32 + lane;          // weight row within the tile = TMEM lane
        const uint32_t lane_addr = uint32_t(quarter * 32) << 16;
        const uint32_t stg_w_addr = sbase + kSSmemC + (warp - 2) * kStgBufs * kStgBytes;
        int local = 0, cbuf = 0;
        for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++local) {
            const int n0 = (tile % p.num_n) * SBM, m0 = (tile / p.num_n) * SBN;
            const uint32_t buf = local & 1, bphase = (local >> 1) & 1;
            epi_bar();   // everyone is done with the previous tile's token scales
            for (int c = et; c < SBN; c += kEpiThreads) {
                const int m = m0 + c;
                s_scale[c] = m < p.M ? p.sx[m] * 0.5f : 0.0f;
            }
            const int n = n0 + row;
            const float sw_half = n < p.N ? p.sw[n] * 0.5f : 0.0f;
            const bool got = mbar_wait(bar_tfull + 8 * buf, bphase, abort_flag, kWaitLimitNs, kSuspendEpilogueNs);
            if (epi_any(!got)) break;   // also orders the token scales above (bar.red)
            tc_fence_after();
            const uint32_t t_acc = tmem_base + lane_addr + buf * kSAccCols;
            store_tile_transposed(map_y, t_acc, stg_w_addr, cbuf, lane, n0 + 32 * quarter, m0, sw_half, s_scale,
                                  p.acc, p.M, p.N);
            tc_fence_before();
            mbar_arrive(bar_tempty + 8 * buf);
        }
        if (lane == 0) bulk_wait_all();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTmemCols)
                     : "memory");
    }
}

// ---------------------------------------------------------------------------
// CTA-pair variant (cluster of 2, tcgen05 cta_group::2): one sparse MMA of
// M = 256 weight rows (128 per CTA, each CTA's own compressed rows and metadata),
// N = 224 tokens (112 rows of B per CTA), K = 64 logical per instruction, issued by
// the even CTA. A stage stages 24 KB per CTA instead of 38 KB for the same tensor
// work per SM: the activation tile is split between the two CTAs. The metadata copy
// (tcgen05.cp cta_group::2, issued by the even CTA) fills each CTA's TMEM slot from
// its own shared memory. Barriers as the dense CTA-pair layer: both producers
// signal the even CTA's full barrier, the even CTA's commits (multicast to both
// CTAs) free stages and hand each CTA its half of the accumulator, each epilogue
// returns its buffer with one arrival on the even CTA's barrier.
//
// Metadata, two forms. Staged (any K): a 2 KB slab rides in every stage of the
// ring and one tcgen05.cp per stage moves it into a rotating 4-column slot just
// before the stage's two MMAs. Resident (K <= 2048): the 64 TMEM columns after
// the two accumulators hold the metadata of the whole reduction for this CTA's
// 128 weight rows; the pair walks its tiles in weight-major order, so the block
// (K/8 bytes per row) is loaded and copied into TMEM once per weight tile, and
// the ring carries only operand codes. Before overwriting the columns for the
// next weight tile the issuer waits for the previous tile's accumulator commit
// (its MMAs have read the old metadata); the copies' own commit frees the
// shared-memory block for the producer.
constexpr int kPSStages = 7;
constexpr int PBN = SBN / 2;                             // B rows per CTA
constexpr uint32_t kPSStageB = PBN * SBK;                // 14 KB
// Shared memory of the pair kernel. Staged metadata: a 2 KB slab per stage in the
// ring. Resident metadata (K <= kResidentMaxK): no metadata in the ring, one slab
// per 128-value K stage of the whole reduction, loaded once per weight tile.
constexpr int kResidentMaxK = (kTmemCols - kSMetaCol) / 4 * SBK;   // 16 stages of 4 columns: K <= 2048
template <bool R>
struct PairLayout {
    static constexpr uint32_t kStageE = R ? 0u : kSStageE;
    static constexpr uint32_t kTx = 2 * (kSStageA + kPSStageB + kStageE);   // both CTAs land on one barrier
    static constexpr uint32_t kA = 0;
    static constexpr uint32_t kB = kA + kPSStages * kSStageA;
    static constexpr uint32_t kE = kB + kPSStages * kPSStageB;     // staged slabs, or the resident block
    static constexpr uint32_t kEBytes = R ? uint32_t(kResidentMaxK / SBK) * kSStageE : kPSStages * kSStageE;
    static constexpr uint32_t kC = kE + kEBytes;
    static constexpr uint32_t kScale = kC + kSCBytes;
    static constexpr uint32_t kBar = kScale + SBN * 4;
    static constexpr uint32_t kNumBars = 2 * kPSStages + 4 + 1 + 2;   // + metadata full / empty
    static constexpr uint32_t kTmemSlot = kBar + kNumBars * 8;
    static constexpr uint32_t kAbort = kTmemSlot + 4;
    static constexpr uint32_t kTotal = kAbort + 4 + 1024;
    static_assert(kTotal <= 227 * 1024, "sparse pair kernel shared memory");
    static_assert(kScale % 16 == 0, "16-byte scale loads");
};
static_assert(kPSStageB % 1024 == 0, "stage alignment");
static_assert(kSMetaCol + 4 * kPSStages <= kTmemCols, "TMEM columns");
static_assert(kResidentMaxK >= SBK, "resident metadata");

constexpr uint32_t kIdescSpPair = (1u << 2) | (2u << 4) | (1u << 7) | (1u << 10) | (uint32_t(SBN >> 3) << 17) |
                                  (uint32_t(256 >> 4) << 24);

__device__ __forceinline__ void tc_mma_sp_i8_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t e_tmem,
                                                  uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %5, 0;\n\t"
        "tcgen05.mma.sp.cta_group::2.kind::i8 [%0], %1, %2, [%3], %4, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(e_tmem), "r"(kIdescSpPair), "r"(accumulate)
        : "memory");
}
__device__ __forceinline__ void tc_cp_meta_pair(uint32_t taddr, uint64_t sdesc) {
    asm volatile("tcgen05.cp.cta_group::2.128x128b [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

struct SparsePairParams {
    const float* sx;
    const float* sw;
    int32_t* acc;
    int M, N, K;
    int num_n2, num_m, num_k;   // 256-row weight pair tiles, token tiles (224), K stages (128)
};

template <bool kResident>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
w4a4_sparse_pair_kernel(const __grid_constant__ CUtensorMap map_w, const __grid_constant__ CUtensorMap map_x,
                        const __grid_constant__ CUtensorMap map_e, const __grid_constant__ CUtensorMap map_y,
                        const SparsePairParams p) {
    using L = PairLayout<kResident>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar_full = sbase + L::kBar;               // [kPSStages], used in the even CTA
    const uint32_t bar_empty = bar_full + 8 * kPSStages;     // [kPSStages]
    const uint32_t bar_tfull = bar_empty + 8 * kPSStages;    // [2]
    const uint32_t bar_tempty = bar_tfull + 16;              // [2], used in the even CTA
    const uint32_t bar_drain = bar_tempty + 16;              // [1]
    const uint32_t bar_mfull = bar_drain + 8;                // resident metadata landed (even CTA)
    const uint32_t bar_mempty = bar_mfull + 8;               // resident metadata copied into TMEM
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kAbort);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kTmemSlot);
    float* s_scale = reinterpret_cast<float*>(smem + L::kScale);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const bool even = rank == 0;
    const int pair = blockIdx.x >> 1, num_pairs = gridDim.x >> 1;
    const int num_tiles = p.num_n2 * p.num_m;
    // Tiles of this pair. Staged metadata: every num_pairs-th tile, token tiles
    // fastest within a weight tile's column of the grid (tile = n2 + num_n2 * mt).
    // Resident metadata: a contiguous run of tiles in weight-major order
    // (tile = mt + num_m * n2), so a pair meets one or two weight tiles and
    // copies each one's metadata into TMEM once.
    const int t_begin = kResident ? int((int64_t(pair) * num_tiles) / num_pairs) : pair;
    const int t_end = kResident ? int((int64_t(pair + 1) * num_tiles) / num_pairs) : num_tiles;
    const int t_step = kResident ? 1 : num_pairs;
    auto tile_n2 = [&](int tile) { return kResident ? tile / p.num_m : tile % p.num_n2; };
    auto tile_mt = [&](int tile) { return kResident ? tile % p.num_m : tile / p.num_n2; };

    if (threadIdx.x == 0) {
        for (int s = 0; s < kPSStages; ++s) {
            mbar_init(bar_full + 8 * s, 1);
            mbar_init(bar_empty + 8 * s, 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar_tfull + 8 * b, 1);
            mbar_init(bar_tempty + 8 * b, 2);
        }
        mbar_init(bar_drain, 1);
        mbar_init(bar_mfull, 1);
        mbar_init(bar_mempty, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_w)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_x)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_e)) : "memory");
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
    pdl_wait();
    pdl_trigger();

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer (both CTAs)
        if (lane == 0) {
            const uint32_t full_even = map_to_rank(bar_full, 0);
            uint32_t stage = 0, phase = 0, mphase = 0;
            uint64_t issued = 0;
            bool ok = true, mphase_issued = false;
            int cur_n2 = -1;
            for (int tile = t_begin; tile < t_end && ok; tile += t_step) {
                const int n0 = tile_n2(tile) * 256 + 128 * int(rank);
                const int m0 = tile_mt(tile) * SBN + PBN * int(rank);
                if (kResident && tile_n2(tile) != cur_n2) {
                    // the whole reduction's metadata of this CTA's 128 weight rows, once
                    // the previous weight tile's block has been copied into TMEM
                    if (!mbar_wait(bar_mempty, mphase ^ 1, abort_flag, kWaitLimitNs, kSuspendProducerNs)) {
                        ok = false;
                        break;
                    }
                    if (even) mbar_arrive_expect_tx(bar_mfull, 2u * uint32_t(p.num_k) * kSStageE);
                    const uint32_t mb = map_to_rank(bar_mfull, 0);
                    for (int kb = 0; kb < p.num_k; ++kb)
                        tma_load_2d_pair(sbase + L::kE + kb * kSStageE, &map_e, kb * (SBK / 8), n0, mb);
                    mphase ^= 1;
                    mphase_issued = true;
                    cur_n2 = tile_n2(tile);
                }
                for (int kb = 0; kb < p.num_k; ++kb) {
                    if (!mbar_wait(bar_empty + 8 * stage, phase ^ 1, abort_flag, kWaitLimitNs, kSuspendProducerNs)) {
                        ok = false;
                        break;
                    }
                    if (even) mbar_arrive_expect_tx(bar_full + 8 * stage, L::kTx);
                    const uint32_t fb = full_even + 8 * stage;
                    tma_load_2d_pair(sbase + L::kA + stage * kSStageA, &map_w, kb * (SBK / 2), n0, fb);
                    tma_load_2d_pair(sbase + L::kB + stage * kPSStageB, &map_x, kb * SBK, m0, fb);
                    if (!kResident)
                        tma_load_2d_pair(sbase + L::kE + stage * kSStageE, &map_e, kb * (SBK / 8), n0, fb);
                    ++issued;
                    if (++stage == kPSStages) { stage = 0; phase ^= 1; }
                }
            }
            if (!ok && even && kResident && mphase_issued) {
                // the last metadata block may still be landing
                const uint64_t t0 = global_timer_ns();
                while (!mbar_try_wait(bar_mfull, mphase ^ 1) && global_timer_ns() - t0 < kWaitLimitNs) {
                }
            }
            if (!ok && even) {
                const uint64_t n = issued < kPSStages ? issued : kPSStages;
                for (uint64_t i = issued - n; i < issued; ++i) {
                    const uint32_t st = uint32_t(i % kPSStages), ph = uint32_t((i / kPSStages) & 1);
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
        // ------------------------------------------------------------ metadata copies and MMAs (even CTA)
        if (even && lane == 0) {
            uint32_t stage = 0, phase = 0, mphase = 0;
            bool ok = true;
            int local = 0, cur_n2 = -1;
            for (int tile = t_begin; tile < t_end && ok; tile += t_step, ++local) {
                const uint32_t buf = local & 1, bphase = (local >> 1) & 1;
                if (!mbar_wait(bar_tempty + 8 * buf, bphase ^ 1, abort_flag, kWaitLimitNs, kSuspendMmaNs)) {
                    ok = false;
                    break;
                }
                if (kResident && tile_n2(tile) != cur_n2) {
                    if (cur_n2 >= 0) {
                        // the previous tile's MMAs (its accumulator commit) must have read
                        // the old metadata before the copies overwrite those columns
                        const uint32_t pb = (local - 1) & 1, pph = ((local - 1) >> 1) & 1;
                        if (!mbar_wait(bar_tfull + 8 * pb, pph, abort_flag, kWaitLimitNs, kSuspendMmaNs)) {
                            ok = false;
                            break;
                        }
                    }
                    if (!mbar_wait(bar_mfull, mphase, abort_flag, kWaitLimitNs, kSuspendMmaNs)) { ok = false; break; }
                    tc_fence_after();
                    for (int kb = 0; kb < p.num_k; ++kb)
                        tc_cp_meta_pair(tmem_base + kSMetaCol + 4 * kb, smem_desc_meta(sbase + L::kE + kb * kSStageE));
                    tc_commit_pair_mc(bar_mempty);   // both CTAs' blocks are free once copied
                    mphase ^= 1;
                    cur_n2 = tile_n2(tile);
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + buf * kSAccCols;
                for (int kb = 0; kb < p.num_k; ++kb) {
                    if (!mbar_wait(bar_full + 8 * stage, phase, abort_flag, kWaitLimitNs, kSuspendMmaNs)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_addr = sbase + L::kA + stage * kSStageA;
                    const uint32_t b_addr = sbase + L::kB + stage * kPSStageB;
                    const uint32_t e_tmem = tmem_base + kSMetaCol + 4 * (kResident ? uint32_t(kb) : stage);
                    if (!kResident) tc_cp_meta_pair(e_tmem, smem_desc_meta(sbase + L::kE + stage * kSStageE));
#pragma unroll
                    for (int kk = 0; kk < SBK / 64; ++kk) {
                        tc_mma_sp_i8_pair(d_tmem, smem_desc_k64(a_addr + kk * 32), smem_desc_k128(b_addr + kk * 64),
                                          e_tmem + 2 * kk, (kb | kk) != 0);
                    }
                    tc_commit_pair_mc(bar_empty + 8 * stage);
                    if (++stage == kPSStages) { stage = 0; phase ^= 1; }
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
        const int row = quarter * 32 + lane;          // weight row within this CTA's half = TMEM lane
        const uint32_t lane_addr = uint32_t(quarter * 32) << 16;
        const uint32_t tempty_even = map_to_rank(bar_tempty, 0);
        const uint32_t stg_w_addr = sbase + L::kC + (warp - 2) * kStgBufs * kStgBytes;
        int local = 0, cbuf = 0;
        for (int tile = t_begin; tile < t_end; tile += t_step, ++local) {
            const int n0 = tile_n2(tile) * 256 + 128 * int(rank), m0 = tile_mt(tile) * SBN;
            const uint32_t buf = local & 1, bphase = (local >> 1) & 1;
            epi_bar();
            for (int c = et; c < SBN; c += kEpiThreads) {
                const int m = m0 + c;
                s_scale[c] = m < p.M ? p.sx[m] * 0.5f : 0.0f;
            }
            const int n = n0 + row;
            const float sw_half = n < p.N ? p.sw[n] * 0.5f : 0.0f;
            const bool got = mbar_wait(bar_tfull + 8 * buf, bphase, abort_flag, kWaitLimitNs, kSuspendEpilogueNs);
            if (epi_any(!got)) break;   // also orders the token scales above (bar.red)
            tc_fence_after();
            const uint32_t t_acc = tmem_base + lane_addr + buf * kSAccCols;
            store_tile_transposed(map_y, t_acc, stg_w_addr, cbuf, lane, n0 + 32 * quarter, m0, sw_half, s_scale,
                                  p.acc, p.M, p.N);
            tc_fence_before();
            epi_bar();
            if (et == 0) mbar_arrive_remote(tempty_even + 8 * buf);
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

template <bool kResident>
cudaError_t launch_sparse_pair(const CUtensorMap& mw, const CUtensorMap& mx, const CUtensorMap& me,
                               const CUtensorMap& my, const SparsePairParams& pp, cudaStream_t stream) {
    constexpr uint32_t smem = PairLayout<kResident>::kTotal;
    static thread_local int attr_dev = -1;
    int dev = 0;
    cudaGetDevice(&dev);
    if (attr_dev != dev) {
        cudaError_t e = cudaFuncSetAttribute(w4a4_sparse_pair_kernel<kResident>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        attr_dev = dev;
    }
    const int tiles = pp.num_n2 * pp.num_m;
    const int npairs = pair_clusters(dev, (const void*)w4a4_sparse_pair_kernel<kResident>, kThreads, smem);
    const int grid_pairs = tiles < npairs ? tiles : npairs;
    return launch_pdl(w4a4_sparse_pair_kernel<kResident>, dim3(2 * grid_pairs), dim3(kThreads), smem, stream, mw, mx,
                      me, my, pp);
}

}  // namespace

cudaError_t launch_w4a4_sparse24(const int8_t* X, const float* sx, const int8_t* W, const uint8_t* E,
                                 const float* sw, int64_t M, int64_t N, int64_t K, uint16_t* y, int32_t* acc,
                                 cudaStream_t stream) {
    if (M == 0 || N == 0) return cudaSuccess;
    if (K == 0) return launch_zero_fill(y, acc, M * N, stream);
    CUtensorMap mw, mx, me, my;
    // more than one 128-row block of weights: CTA pairs (M = 256 weight rows per MMA)
    const bool pairs = N > SBM;
    if (!make_map_2d(&mw, CU_TENSOR_MAP_DATA_TYPE_UINT8, W, K / 2, N, K / 2, SBK / 2, SBM,
                     CU_TENSOR_MAP_SWIZZLE_64B) ||
        !make_map_2d(&mx, CU_TENSOR_MAP_DATA_TYPE_UINT8, X, K, M, K, SBK, pairs ? PBN : SBN,
                     CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map_2d(&me, CU_TENSOR_MAP_DATA_TYPE_UINT8, E, K / 8, N, K / 8, SBK / 8, SBM,
                     CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !make_map_2d(&my, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, y, N, M, N * 2, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B))
        return cudaErrorInvalidValue;
    if (pairs) {
        SparsePairParams pp;
        pp.sx = sx; pp.sw = sw; pp.acc = acc;
        pp.M = (int)M; pp.N = (int)N; pp.K = (int)K;
        pp.num_n2 = (int)((N + 255) / 256);
        pp.num_m = (int)((M + SBN - 1) / SBN);
        pp.num_k = (int)((K + SBK - 1) / SBK);
        return K <= kResidentMaxK ? launch_sparse_pair<true>(mw, mx, me, my, pp, stream)
                                  : launch_sparse_pair<false>(mw, mx, me, my, pp, stream);
    }
    SparseParams p;
    p.sx = sx; p.sw = sw; p.acc = acc;
    p.M = (int)M; p.N = (int)N; p.K = (int)K;
    p.num_n = (int)((N + SBM - 1) / SBM);
    p.num_m = (int)((M + SBN - 1) / SBN);
    p.num_k = (int)((K + SBK - 1) / SBK);
    static thread_local int attr_dev = -1;
    int dev = 0;
    cudaGetDevice(&dev);
    if (attr_dev != dev) {
        cudaError_t e = cudaFuncSetAttribute(w4a4_sparse_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             kSSmemTotal);
        if (e != cudaSuccess) return e;
        attr_dev = dev;
    }
    const int tiles = p.num_n * p.num_m;
    const int sms = sm_count();
    const int grid = tiles < sms ? tiles : sms;
    return launch_pdl(w4a4_sparse_kernel, dim3(grid), dim3(kThreads), kSSmemTotal, stream, mw, mx, me, my, p);
}

int read_and_clear_sparse_status(cudaStream_t stream, cudaError_t* err) {
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

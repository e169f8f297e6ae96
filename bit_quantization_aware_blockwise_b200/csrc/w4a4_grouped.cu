// Linear layer on QuEST codes with per-group scales along K (one scale per row and
// per 128-wide K group on both operands): CTA-pair tcgen05 kind::f8f6f4 kernel on
// E4M3 codes with a per-group TMEM round trip into two ping-pong epilogue teams
// (see the kernel's comment).
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
// Per-group scales along K (one scale per row and per 128-wide K group on both
// operands): Y[m][n] = sum_g (sa[m][g]/2)(sb[n][g]/2) * P_g[m][n], P_g the
// product of group g's codes. The codes come as FP8 E4M3 (c = 2q + 1, odd,
// |c| <= 15, exact in E4M3), so tcgen05 kind::f8f6f4 with fp32 accumulation
// gives every P_g exactly (integers below 2^24) with no int -> float step.
//
// Every group's product makes a round trip through TMEM to registers, where it
// is scaled and added: acc += P_g * (sa/2)(sb/2), two packed FP instructions per
// pair of outputs per group. A pair tile is 256 rows x 256 columns, computed as two
// 128-column halves: every operand stage holds one group of the tile's A rows and
// of the B rows of both halves, and the MMA issuer runs both halves' MMAs off it
// (half 0 into one TMEM slot, half 1 into another), so A crosses from L2 once per
// group for both. The epilogue runs as two teams of four warps (one warp per TMEM
// lane quarter on each team), team h owning the 128 x 128 accumulator of half h in
// registers; the two warps on a scheduler read alternate slots. Each team has two
// of the four 128-column TMEM slots (groups alternate between them); a slot's full
// barrier (committed by the MMA issuer in both CTAs) says that its group's product
// is complete, its empty barrier (8 warp arrivals) that the team has read it. A slot
// is never reissued before its team has read it, so its full barrier is at most one
// phase ahead of the team's wait. An epilogue thread holds its row of the
// accumulator (128 registers) and two 16-column TMEM load buffers, so the load of
// the next 16 columns overlaps the arithmetic on the current ones.
//
// What bounds it (16384 x 5632 x 2048, scratch variants of the earlier layout,
// in which the two teams took two different 256 x 128 tiles and every stage held
// one tile's group, timed on B200): 400 us as built; 393 us with half the MMAs;
// 330 us with the FP work removed; 254 us with neither MMAs nor FP work, the
// operand feed of 48 KB per 256 x 128 x 128 group (2.16 GB in 254 us, 8.5 TB/s
// of TMA loads). Sharing A between the two halves cuts that feed by a third
// (64 KB per 256 x 256 x 128 group), yet the layer gained only 1-2 % (387 us
// against 390 us in an interleaved A/B, outputs identical): the hand-off of the
// TMEM slots (the MMA's commit, the team's reads, the arrivals from both CTAs,
// the polling on both sides) sets the pace, not the feed. TMEM reads are not the
// limit (a probe of back-to-back tcgen05.ld reads 460-935 B per clock per SM;
// this layer moves about 50). A lockstep layout (eight warps on the same group,
// 64 columns each, two 32-column loads per wait) measured the same 403 us.

// Every wait of this kernel polls: the hand-off of its TMEM slots is a latency chain,
// and parking the waiting threads (the other tensor-core layers' setting) cost 1 %.
constexpr uint32_t kGPollNs = 0;
constexpr int kGThreads = 384;               // warpgroup 0: producer, MMA (2 warps idle); 1, 2: the teams
constexpr int kGTeamThreads = 128;
constexpr int kGBN = 128;                    // output columns per team (one half of a pair tile)
constexpr int kGWide = 2 * kGBN;             // output columns per pair tile
constexpr int kGStages = 5;
constexpr int kGSlots = 4;                   // TMEM slots of kGBN columns, two per team
constexpr int kGroup = 128;                  // K group = one stage
constexpr int kGScaleBlock = 8;              // groups of scales staged at a time
// per CTA and stage: 128 A rows; the B rows of half 0, then of half 1 (kGBN / 2 each)
constexpr uint32_t kGStageA = 128 * BK, kGStageBHalf = (kGBN / 2) * BK, kGStageB = 2 * kGStageBHalf;
constexpr uint32_t kGTxBytes = 2 * (kGStageA + kGStageB);
constexpr uint32_t kGSmemA = 0;
constexpr uint32_t kGSmemB = kGSmemA + kGStages * kGStageA;
constexpr uint32_t kGScaleBytes = kGScaleBlock * (kGBN + 128) * 4;    // one block: sb [8][128], sa [8][128]
constexpr uint32_t kGSmemS = kGSmemB + kGStages * kGStageB;           // 2 teams x 2 blocks (double buffer)
constexpr uint32_t kGSmemC = kGSmemS + 4 * kGScaleBytes;              // 8 warps x 2 x 2 KB
constexpr uint32_t kGCBytes = 32 * 32 * 2;                            // 32 rows x 32 bf16
constexpr uint32_t kGSmemBar = kGSmemC + 8 * 2 * kGCBytes;
constexpr uint32_t kGNumBars = 2 * kGStages + 2 * kGSlots + 1;
constexpr uint32_t kGSmemTmemSlot = kGSmemBar + kGNumBars * 8;
constexpr uint32_t kGSmemAbort = kGSmemTmemSlot + 4;
constexpr uint32_t kGSmemUsed = kGSmemAbort + 4;
constexpr uint32_t kGSmemTotal = kGSmemUsed + 1024;
static_assert(kGSmemTotal <= 227 * 1024, "grouped kernel shared memory");
static_assert(kGSlots * kGBN == kTmemCols, "TMEM slots");

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

// Named barrier 1 + team over the team's 128 threads, and an OR-vote on it.
__device__ __forceinline__ void team_bar(int team) {
    asm volatile("bar.sync %0, %1;" ::"r"(1 + team), "n"(kGTeamThreads) : "memory");
}
__device__ __forceinline__ bool team_any(int team, bool pred) {
    uint32_t out;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(out)
        : "r"((uint32_t)pred), "r"(1 + team), "n"(kGTeamThreads)
        : "memory");
    return out != 0;
}

// tcgen05.wait::ld that names the loaded registers as read-write operands, so no
// use of them can be scheduled above the wait.
#define QUEST_TMEM_WAIT16(r)                                                                   \
    asm volatile("tcgen05.wait::ld.sync.aligned;"                                             \
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]),     \
                   "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]),   \
                   "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15])                          \
                 :                                                                             \
                 : "memory")

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
    int num_m2, num_n, num_k;   // 256-row and 256-column pair tiles, K groups
};

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGThreads, 1)
w4a4_gemm_grouped_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                         const __grid_constant__ CUtensorMap map_y, const GroupedParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar_full = sbase + kGSmemBar;                 // [kGStages], used in the even CTA
    const uint32_t bar_empty = bar_full + 8 * kGStages;          // [kGStages]
    const uint32_t bar_tfull = bar_empty + 8 * kGStages;         // [kGSlots]
    const uint32_t bar_tempty = bar_tfull + 8 * kGSlots;         // [kGSlots], used in the even CTA
    const uint32_t bar_drain = bar_tempty + 8 * kGSlots;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kGSmemAbort);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kGSmemTmemSlot);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const bool even = rank == 0;
    const int pair = blockIdx.x >> 1, num_pairs = gridDim.x >> 1;
    const int num_tiles = p.num_m2 * p.num_n;
    const int G = p.num_k;
    // this pair's tiles: pair + i * num_pairs for i < ntl
    const int ntl = (num_tiles - pair + num_pairs - 1) / num_pairs;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kGStages; ++s) {
            mbar_init(bar_full + 8 * s, 1);
            mbar_init(bar_empty + 8 * s, 1);
        }
        for (int b = 0; b < kGSlots; ++b) {
            mbar_init(bar_tfull + 8 * b, 1);
            mbar_init(bar_tempty + 8 * b, 8);   // 4 team warps x 2 CTAs
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
            for (int i = 0; i < ntl && ok; ++i) {
                const int tile = pair + i * num_pairs;
                const int m0 = (tile % p.num_m2) * 256 + 128 * int(rank);
                // half h's B rows: n0 + h * kGBN .. + kGBN / 2 - 1 in this CTA
                const int n0 = (tile / p.num_m2) * kGWide + (kGBN / 2) * int(rank);
                for (int kb = 0; kb < G && ok; ++kb) {
                    if (!mbar_wait(bar_empty + 8 * stage, phase ^ 1, abort_flag, kWaitLimitNs, kGPollNs)) {
                        ok = false;
                        break;
                    }
                    if (even) mbar_arrive_expect_tx(bar_full + 8 * stage, kGTxBytes);
                    const uint32_t fb = full_even + 8 * stage;
                    const uint32_t b_st = sbase + kGSmemB + stage * kGStageB;
                    tma_load_2d_pair(sbase + kGSmemA + stage * kGStageA, &map_a, kb * BK, m0, fb);
                    tma_load_2d_pair(b_st, &map_b, kb * BK, n0, fb);
                    tma_load_2d_pair(b_st + kGStageBHalf, &map_b, kb * BK, n0 + kGBN, fb);
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
            uint32_t gc = 0;   // groups issued (the same for both halves): half h's slot is 2 h + (gc & 1)
            bool ok = true;
            for (int i = 0; i < ntl && ok; ++i) {
                for (int kb = 0; kb < G && ok; ++kb) {
                    if (!mbar_wait(bar_full + 8 * stage, phase, abort_flag, kWaitLimitNs, kGPollNs)) {
                        ok = false;
                        break;
                    }
                    const uint32_t a_addr = sbase + kGSmemA + stage * kGStageA;
                    const uint32_t b_st = sbase + kGSmemB + stage * kGStageB;
                    const uint32_t sphase = (gc >> 1) & 1;
#pragma unroll 1
                    for (int h = 0; h < 2; ++h) {
                        const uint32_t slot = 2 * h + (gc & 1);
                        if (!mbar_wait(bar_tempty + 8 * slot, sphase ^ 1, abort_flag, kWaitLimitNs, kGPollNs)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t d_tmem = tmem_base + slot * kGBN;
                        const uint32_t b_addr = b_st + h * kGStageBHalf;
#pragma unroll
                        for (int kk = 0; kk < BK / kUmmaK; ++kk) {
                            tc_mma_f8_pair(d_tmem, smem_desc_k128(a_addr + kk * kUmmaK),
                                           smem_desc_k128(b_addr + kk * kUmmaK), kk != 0);
                        }
                        if (h == 1) tc_commit_pair_mc(bar_empty + 8 * stage);   // frees the stage in both CTAs
                        tc_commit_pair_mc(bar_tfull + 8 * slot);                 // the half's product is ready
                    }
                    ++gc;
                    if (++stage == kGStages) { stage = 0; phase ^= 1; }
                }
            }
            tc_commit_pair(bar_drain);
            const uint64_t t0 = global_timer_ns();
            while (!mbar_try_wait(bar_drain, 0) && global_timer_ns() - t0 < kWaitLimitNs) {
            }
        }
    } else if (warp >= 4) {
        // ------------------------------------------------------------ epilogue (warps 4..11, both CTAs)
        const int ew = warp - 4;                           // epilogue warp 0..7
        const int team = ew >> 2;                          // half of every tile: columns kGBN * team ..
        const int tt = (ew & 3) * 32 + lane;               // thread in team 0..127
        const int quarter = warp & 3;                      // TMEM lanes 32*quarter .. +31
        const int row_in_tile = quarter * 32 + lane;
        const uint32_t lane_addr = uint32_t(quarter * 32) << 16;
        const uint32_t tempty_even = map_to_rank(bar_tempty, 0);
        const uint32_t stg0 = sbase + kGSmemC + uint32_t(ew) * 2 * kGCBytes;
        const uint32_t sc_base = kGSmemS + uint32_t(team) * 2 * kGScaleBytes;   // this team's two blocks
        const int Gs = p.K / kGroup;                       // scale columns per row
        // issue the copies of the scales of groups g0 .. g0+7 of local tile i into buffer b,
        // transposed to [group][column] and [group][row]
        auto prefetch = [&](int i, int g0, int b) {
            if (i < ntl) {
                const int tile = pair + i * num_pairs;
                const int pm0 = (tile % p.num_m2) * 256 + 128 * int(rank);
                const int pn0 = (tile / p.num_m2) * kGWide + kGBN * team;
                const int nb = (G - g0) < kGScaleBlock ? (G - g0) : kGScaleBlock;
                const uint32_t base = sbase + sc_base + uint32_t(b) * kGScaleBytes;
#pragma unroll
                for (int k = 0; k < kGScaleBlock * kGBN / kGTeamThreads; ++k) {
                    const int e = tt + k * kGTeamThreads, n = e / kGScaleBlock, gg = e % kGScaleBlock;
                    const bool v = gg < nb && pn0 + n < p.N;
                    cp_async4(base + 4 * (gg * kGBN + n), p.sb + (v ? int64_t(pn0 + n) * Gs + g0 + gg : 0), v);
                }
#pragma unroll
                for (int k = 0; k < kGScaleBlock * 128 / kGTeamThreads; ++k) {
                    const int e = tt + k * kGTeamThreads, r = e / kGScaleBlock, gg = e % kGScaleBlock;
                    const bool v = gg < nb && pm0 + r < p.M;
                    cp_async4(base + 4 * (kGScaleBlock * kGBN + gg * 128 + r),
                              p.sa + (v ? int64_t(pm0 + r) * Gs + g0 + gg : 0), v);
                }
            }
            cp_async_commit();
        };
        int cbuf = 0, sbuf = 0;
        bool aborted = false;
        prefetch(0, 0, 0);
        for (int i = 0; i < ntl && !aborted; ++i) {
            const int tile = pair + i * num_pairs;
            const int m0 = (tile % p.num_m2) * 256 + 128 * int(rank);
            const int n0 = (tile / p.num_m2) * kGWide + kGBN * team;
            float2 acc[64];   // columns 2j, 2j + 1 of the tile
#pragma unroll
            for (int j = 0; j < 64; ++j) acc[j] = make_float2(0.0f, 0.0f);
            for (int g = 0; g < G; ++g) {
                if ((g % kGScaleBlock) == 0) {
                    // a thread whose wait gave up stops the whole team here (uniform exit)
                    if (team_any(team, aborted)) break;
                    // this block's scales have landed, and every thread of the team is done
                    // with the other buffer: start copying the next block into it
                    cp_async_wait_all();
                    team_bar(team);
                    if (g + kGScaleBlock < G) prefetch(i, g + kGScaleBlock, sbuf ^ 1);
                    else prefetch(i + 1, 0, sbuf ^ 1);
                }
                // G groups in every tile before i
                const uint32_t ga = uint32_t(G) * uint32_t(i) + uint32_t(g);   // the team's group count
                const uint32_t slot = 2 * team + (ga & 1);
                // the warp decides together: the TMEM loads below are warp-collective
                const bool got = mbar_wait(bar_tfull + 8 * slot, (ga >> 1) & 1, abort_flag, kWaitLimitNs, kGPollNs);
                if (!__all_sync(0xFFFFFFFFu, got)) aborted = true;
                if (aborted) continue;   // later waits return at once (abort flag); exit at the next check
                tc_fence_after();
                const uint32_t t_grp = tmem_base + lane_addr + slot * kGBN;
                // (sa/2)(sb/2): the factor 1/4 rides on the row scale
                const float* sblk = reinterpret_cast<const float*>(smem + sc_base) + sbuf * (kGScaleBytes / 4);
                const float sx = 0.25f * sblk[kGScaleBlock * kGBN + (g % kGScaleBlock) * 128 + row_in_tile];
                const float4* sw4 = reinterpret_cast<const float4*>(sblk + (g % kGScaleBlock) * kGBN);
                if ((g % kGScaleBlock) == kGScaleBlock - 1 || g == G - 1) sbuf ^= 1;   // next block, other buffer
                // 16 columns per TMEM load, two buffers: the load of columns 16 (q + 1) ..
                // is in flight while columns 16 q .. are scaled and added
                uint32_t rbuf[2][16];
                QUEST_TMEM_LD16(t_grp, rbuf[0]);
                QUEST_TMEM_WAIT16(rbuf[0]);
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    uint32_t (&r)[16] = rbuf[q & 1];
                    if (q < 7) QUEST_TMEM_LD16(t_grp + 16 * (q + 1), rbuf[(q + 1) & 1]);
                    if (q == 7) {
                        // the group's partials are all in registers: hand the slot back
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive_remote(tempty_even + 8 * slot);
                    }
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        const float4 w4 = sw4[4 * q + v];
                        const float2 w01 = __fmul2_rn(make_float2(sx, sx), make_float2(w4.x, w4.y));
                        const float2 w23 = __fmul2_rn(make_float2(sx, sx), make_float2(w4.z, w4.w));
                        float2& a0 = acc[8 * q + 2 * v];
                        float2& a1 = acc[8 * q + 2 * v + 1];
                        a0 = __ffma2_rn(make_float2(__uint_as_float(r[4 * v]), __uint_as_float(r[4 * v + 1])), w01,
                                        a0);
                        a1 = __ffma2_rn(make_float2(__uint_as_float(r[4 * v + 2]), __uint_as_float(r[4 * v + 3])),
                                        w23, a1);
                    }
                    if (q < 7) QUEST_TMEM_WAIT16(rbuf[(q + 1) & 1]);
                }
            }
            if (team_any(team, aborted)) { aborted = true; break; }
            // ---- output: this warp's 32 rows x 128 columns, in 4 chunks of 32 columns
            const int m = m0 + row_in_tile;
            if (p.y32 != nullptr && m < p.M) {
                float* yrow = p.y32 + int64_t(m) * p.N + n0;
#pragma unroll
                for (int j = 0; j < 64; ++j) {
                    const int n = n0 + 2 * j;
                    if (n < p.N) yrow[2 * j] = acc[j].x;
                    if (n + 1 < p.N) yrow[2 * j + 1] = acc[j].y;
                }
            }
            const uint32_t swz = (lane >> 1) & 3;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                if (lane == 0) bulk_wait_read_le1();   // the buffer used two chunks ago is free
                __syncwarp();
                const uint32_t stg = stg0 + cbuf * kGCBytes + lane * 64;
#pragma unroll
                for (int q16 = 0; q16 < 4; ++q16) {
                    uint32_t w[4];
#pragma unroll
                    for (int h = 0; h < 4; ++h) {
                        const float2 v = acc[q * 16 + q16 * 4 + h];
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
                    tma_store_2d(&map_y, stg0 + cbuf * kGCBytes, n0 + q * kChunkCols, m0 + 32 * quarter);
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
    p.num_n = (int)((N + kGWide - 1) / kGWide);
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
    return launch_pdl(w4a4_gemm_grouped_kernel, dim3(2 * grid_pairs), dim3(kGThreads), kGSmemTotal, stream, ma, mb,
                      my, p);
}

}  // namespace

cudaError_t launch_w4a4_grouped(const int8_t* A, const float* sa, const int8_t* B, const float* sb,
                                int64_t M, int64_t N, int64_t K, uint16_t* y, float* y32,
                                cudaStream_t stream) {
    if (M == 0 || N == 0) return cudaSuccess;
    if (K == 0) {
        const int64_t n = M * N;
        if (y32) cudaMemsetAsync(y32, 0, size_t(n) * sizeof(float), stream);
        return launch_zero_fill(y, nullptr, n, stream);
    }
    return launch_grouped(A, sa, B, sb, M, N, K, y, y32, stream);
}

int read_and_clear_grouped_status(cudaStream_t stream, cudaError_t* err) {
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

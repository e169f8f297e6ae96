// Building blocks shared by the tcgen05 kernels (w4a4_gemm.cu, w4a4_grouped.cu,
// trust_linear.cu): mbarrier, TMA and bulk-copy wrappers, tcgen05 fences,
// commits and TMEM loads, the K-major 128-byte-swizzle shared-memory descriptor,
// the cluster (CTA pair) helpers, and the shared-memory layout of the CTA-pair
// pipeline used by the integer layer and the fused input gradient.
//
// Every bounded wait records a timeout in the device status word `g_tc_status`,
// which each including file defines (one per file, read and cleared by its own
// read_and_clear_*_status) in namespace quest's unnamed namespace before it
// includes this header.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "quest_internal.h"

namespace quest {

// Host helpers (tc_host.cu).
// A 2-D tensor map over a row-major matrix of `outer` rows of `inner` elements.
bool make_map_2d(CUtensorMap* map, CUtensorMapDataType dt, const void* base, uint64_t inner,
                 uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
                 CUtensorMapSwizzle swz);
// Co-resident CTA pairs of a cluster kernel on device `dev` (the kernel's
// shared-memory attribute must already be set); cached per kernel.
int pair_clusters(int dev, const void* kernel, int threads, uint32_t smem);
// y[0..n) = 0 (bf16) and, when acc is given, acc[0..n) = 0: the empty sum (K == 0).
cudaError_t launch_zero_fill(uint16_t* y, int32_t* acc, int64_t n, cudaStream_t stream);

namespace {

constexpr int BM = 128, BN = 256, BK = 128;   // BK in int8 elements (= bytes)
constexpr int kUmmaK = 32;                    // K of one kind::i8 MMA
constexpr int kThreads = 192;
constexpr int kEpiThreads = 128;
constexpr int kChunkCols = 32;                // epilogue columns per TMEM load / TMA store
constexpr uint32_t kTmemCols = 512;           // two 256-column accumulators
constexpr uint32_t kCBytes = BM * kChunkCols * 2;  // one bf16 staging chunk (8 KB)
constexpr uint64_t kWaitLimitNs = 2000000000ull;            // 2 s per wait
// Suspend-time hints (ns) of the bounded waits by role; 0 polls. With the MMA
// issuer polling its full barrier (it waits on the operand feed most of the time)
// the integer, FP4, 2:4-sparse and bf16 pair layers ran 4-8 % slower than with
// every role parked (hints on the producer and epilogue alone changed nothing);
// the grouped layer, whose per-group TMEM hand-off is latency-bound, polls.
constexpr uint32_t kSuspendProducerNs = 2000;
constexpr uint32_t kSuspendMmaNs = 2000;
constexpr uint32_t kSuspendEpilogueNs = 2000;

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
// The same test with a suspend-time hint: while the phase is incomplete the thread
// is parked, up to hint_ns, and woken when the phase completes, instead of returning
// at once. A polling warp issues a few instructions per try on a scheduler it shares
// with warps doing the work (and draws power under the cap).
__device__ __forceinline__ bool mbar_try_wait_hint(uint32_t bar, uint32_t parity, uint32_t hint_ns) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(hint_ns)
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
// suspend_ns > 0: each try parks the thread up to suspend_ns (see mbar_try_wait_hint).
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          uint64_t limit_ns = kWaitLimitNs, uint32_t suspend_ns = 0) {
    auto test = [&]() { return suspend_ns ? mbar_try_wait_hint(bar, parity, suspend_ns) : mbar_try_wait(bar, parity); };
    if (test()) return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t it = 1;; ++it) {
        if (test()) return true;
        if ((it & 63u) == 0) {
            if (*abort_flag) return false;
            if (global_timer_ns() - t0 > limit_ns) {
                *abort_flag = 1;
                atomicExch(&g_tc_status, (int)QUEST_ETIMEOUT);
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

// ---------------------------------------------------------------------------
// Shared-memory layout of the CTA-pair pipeline (per CTA): a ring of stages of
// A (128 rows x 128 bytes) and B (128 rows x 128 bytes), two bf16 staging chunks
// for the epilogue's TMA stores, one float per output column, the barriers.
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
}  // namespace
}  // namespace quest

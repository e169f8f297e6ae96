// Tensor-core peak probe: back-to-back tcgen05.mma kind::i8 (M = 128, N = 256,
// K = 32, the integer linear layer's instruction shape) from shared-memory
// operands into one TMEM accumulator, one CTA per SM, no loads and no epilogue.
// The caller times a launch; 2 * 128 * 256 * 32 * iters * SMs / time is the
// int8 MMA rate this part sustains at its current clocks, the denominator the
// GEMM's tensor-core fraction can be read against besides the nominal figure.
// The same kernel with kind::f16 (bf16 operands, K = 16) gives the bf16 rate
// measured the same way, against which a library bf16 GEMM can be read.
//
// Built into its own library (libquest_probe.so) for the benchmark: it is a
// measurement aid, not part of the QuEST path, so the product library does not
// export it.
#include <cuda_runtime.h>
#include <stdint.h>

#include "quest.h"
#include "quest_probe.h"

namespace quest {

__device__ int g_probe_status = 0;

namespace {

// At most 2^16 MMAs per CTA: a few milliseconds at any clock, far inside the
// kernel's 2 s completion wait, so that wait never gives up (and never frees
// TMEM) while MMAs are still in flight. The benchmark runs 20000; a scratch
// variant of the pair probe run with 200000 ended in an illegal-address error
// whose cause reading the code did not show, so runs stay in the range that has
// been exercised.
constexpr int kMaxIters = 1 << 16;

int probe_sm_count() {
    int dev = 0, n = 0;
    cudaGetDevice(&dev);
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 1;
    return n;
}

constexpr int kProbeThreads = 128;
constexpr uint32_t kProbeSmem = 120 * 1024;   // more than half an SM: one CTA per SM
constexpr uint32_t kA = 0, kB = 128 * 128;     // A 128 x 128 B, B 256 x 128 B (swizzled rows)
constexpr uint32_t kBar = kB + 256 * 128;
constexpr uint32_t kSlot = kBar + 8;
constexpr uint32_t kIdescProbe = (2u << 4) | (1u << 7) | (1u << 10) | (uint32_t(256 >> 3) << 17) |
                                 (uint32_t(128 >> 4) << 24);

__device__ __forceinline__ uint64_t probe_desc(uint32_t addr) {
    uint64_t d = 0;
    d |= uint64_t((addr >> 4) & 0x3FFFu);
    d |= uint64_t(1) << 16;
    d |= uint64_t(1024 >> 4) << 32;
    d |= uint64_t(1) << 46;
    d |= uint64_t(2) << 61;
    return d;
}

// kind::f16 with bf16 A and B, fp32 accumulator (M = 128, N = 256, K = 16: the
// same 32 bytes per operand row as the int8 instruction), for the bf16 layers.
constexpr uint32_t kIdescProbeBf16 = (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(256 >> 3) << 17) |
                                     (uint32_t(128 >> 4) << 24);

template <bool kBf16>
__global__ void __launch_bounds__(kProbeThreads, 1) probe_mma_dense_kernel(int iters) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
    for (uint32_t i = threadIdx.x * 16; i < kBar; i += kProbeThreads * 16)
        *reinterpret_cast<uint4*>(smem + i) = make_uint4(0x01010101u, 0x01010101u, 0x01010101u, 0x01010101u);
    const uint32_t bar = sbase + kBar;
    if (threadIdx.x == 0) {
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar) : "memory");
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    const int warp = threadIdx.x >> 5;
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 256;" ::"r"(sbase + kSlot)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // operand writes -> tensor core
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + kSlot);

    if (threadIdx.x == 0) {
        const uint64_t a = probe_desc(sbase + kA), b = probe_desc(sbase + kB);
        for (int i = 0; i < iters; ++i) {
            if (kBf16)
                asm volatile(
                    "{\n\t.reg .pred p;\n\t"
                    "setp.ne.b32 p, %4, 0;\n\t"
                    "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem),
                    "l"(a), "l"(b), "r"(kIdescProbeBf16), "r"(i)
                    : "memory");
            else
                asm volatile(
                    "{\n\t.reg .pred p;\n\t"
                    "setp.ne.b32 p, %4, 0;\n\t"
                    "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem),
                    "l"(a), "l"(b), "r"(kIdescProbe), "r"(i)
                    : "memory");
        }
        asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                     : "memory");
        // bounded wait for the MMAs to finish (2 s)
        uint64_t t0, t;
        asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
        for (;;) {
            uint32_t ok;
            asm volatile(
                "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], 0;\n\t"
                "selp.u32 %0, 1, 0, p;\n\t}"
                : "=r"(ok)
                : "r"(bar)
                : "memory");
            if (ok) break;
            asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
            if (t - t0 > 2000000000ull) {
                atomicExch(&g_probe_status, (int)QUEST_ETIMEOUT);
                break;
            }
        }
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (warp == 0) {
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 256;" ::"r"(tmem) : "memory");
    }
}

// The same probe for the block-scaled FP4 kind: tcgen05.mma kind::mxf4 (M = 128,
// N = 256, K = 64) with unit UE8M0 block scales (byte 0x7F) held in TMEM columns
// 480-511, the scale arrangement of the FP4 linear layer.
constexpr uint32_t kIdescProbeFp4 = (1u << 7) | (1u << 10) | (uint32_t(256 >> 3) << 17) | (1u << 23) |
                                    (uint32_t(128 >> 4) << 24);

__global__ void __launch_bounds__(kProbeThreads, 1) probe_mma_fp4_kernel(int iters) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
    for (uint32_t i = threadIdx.x * 16; i < kBar; i += kProbeThreads * 16)
        *reinterpret_cast<uint4*>(smem + i) = make_uint4(0x22222222u, 0x22222222u, 0x22222222u, 0x22222222u);
    const uint32_t bar = sbase + kBar;
    if (threadIdx.x == 0) {
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar) : "memory");
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    const int warp = threadIdx.x >> 5;
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(sbase + kSlot)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + kSlot);
    {
        // unit block scales in this warp's lane quarter, columns 480-511
        const uint32_t v = 0x7F7F7F7Fu, taddr = tmem + (uint32_t(warp * 32) << 16) + 480;
        asm volatile(
            "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
            "{%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,"
            "%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1};" ::"r"(taddr),
            "r"(v)
            : "memory");
        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");

    if (threadIdx.x == 0) {
        const uint64_t a = probe_desc(sbase + kA), b = probe_desc(sbase + kB);
        const uint32_t sfa = tmem + 480, sfb = tmem + 496;
        for (int i = 0; i < iters; ++i) {
            asm volatile(
                "{\n\t.reg .pred p;\n\t"
                "setp.ne.b32 p, %4, 0;\n\t"
                "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
                    tmem),
                "l"(a), "l"(b), "r"(kIdescProbeFp4), "r"(i), "r"(sfa), "r"(sfb)
                : "memory");
        }
        asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                     : "memory");
        uint64_t t0, t;
        asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
        for (;;) {
            uint32_t ok;
            asm volatile(
                "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], 0;\n\t"
                "selp.u32 %0, 1, 0, p;\n\t}"
                : "=r"(ok)
                : "r"(bar)
                : "memory");
            if (ok) break;
            asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
            if (t - t0 > 2000000000ull) {
                atomicExch(&g_probe_status, (int)QUEST_ETIMEOUT);
                break;
            }
        }
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (warp == 0) {
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem) : "memory");
    }
}

// The same for the 2:4-sparse integer kind of the sparse linear layer:
// tcgen05.mma.sp kind::i8 (M = 128, N = 256, K = 64 logical, 32 bytes of the
// compressed A per row), metadata in TMEM (byte 0x44: every run keeps indices
// 0 and 1). With cp_every = c > 0, a tcgen05.cp (128x128b, four columns of
// metadata from shared memory) precedes every c-th MMA and that MMA and the
// next c - 1 read the copied columns, the pattern of a layer that stages its
// metadata through shared memory with its operands (c = 2 per 128-value stage).
constexpr uint32_t kIdescProbeSp = (1u << 2) | (2u << 4) | (1u << 7) | (1u << 10) | (uint32_t(256 >> 3) << 17) |
                                   (uint32_t(128 >> 4) << 24);
constexpr uint32_t kMetaSmem = kSlot + 1024 - (kSlot % 1024);   // 2 KB: 128 rows x 16 bytes
constexpr int kMetaSlots = 8;                                    // rotating 4-column slots from column 288
static_assert(kMetaSmem + 2048 <= kProbeSmem, "probe shared memory");

__global__ void __launch_bounds__(kProbeThreads, 1) probe_mma_sp_i8_kernel(int iters, int cp_every) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
    for (uint32_t i = threadIdx.x * 16; i < kBar; i += kProbeThreads * 16)
        *reinterpret_cast<uint4*>(smem + i) = make_uint4(0x01010101u, 0x01010101u, 0x01010101u, 0x01010101u);
    for (uint32_t i = threadIdx.x * 16; i < 2048; i += kProbeThreads * 16)
        *reinterpret_cast<uint4*>(smem + kMetaSmem + i) = make_uint4(0x44444444u, 0x44444444u, 0x44444444u,
                                                                     0x44444444u);
    const uint32_t bar = sbase + kBar;
    if (threadIdx.x == 0) {
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar) : "memory");
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    const int warp = threadIdx.x >> 5;
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(sbase + kSlot)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + kSlot);
    {
        // metadata 0x44 in this warp's lane quarter, columns 256-287 (the resident set)
        // and 288-319 (the copy slots, so the first reads before any copy are valid too)
        const uint32_t v = 0x44444444u;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const uint32_t taddr = tmem + (uint32_t(warp * 32) << 16) + 256 + 32 * h;
            asm volatile(
                "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
                "{%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,"
                "%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1};" ::"r"(taddr),
                "r"(v)
                : "memory");
        }
        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");

    if (threadIdx.x == 0) {
        const uint64_t a = probe_desc(sbase + kA), b = probe_desc(sbase + kB);
        uint64_t md = 0;
        md |= uint64_t(((sbase + kMetaSmem) >> 4) & 0x3FFFu);
        md |= uint64_t(2048 >> 4) << 16;
        md |= uint64_t(128 >> 4) << 32;
        md |= uint64_t(1) << 46;
        uint32_t e = tmem + 256;
        for (int i = 0; i < iters; ++i) {
            if (cp_every > 0 && i % cp_every == 0) {
                e = tmem + 288 + 4 * uint32_t((i / cp_every) % kMetaSlots);
                asm volatile("tcgen05.cp.cta_group::1.128x128b [%0], %1;" ::"r"(e), "l"(md) : "memory");
            }
            const uint32_t ei = cp_every > 0 ? e + 2 * uint32_t((i % cp_every) & 1) : e;
            asm volatile(
                "{\n\t.reg .pred p;\n\t"
                "setp.ne.b32 p, %5, 0;\n\t"
                "tcgen05.mma.sp.cta_group::1.kind::i8 [%0], %1, %2, [%3], %4, p;\n\t}" ::"r"(tmem),
                "l"(a), "l"(b), "r"(ei), "r"(kIdescProbeSp), "r"(i)
                : "memory");
        }
        asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                     : "memory");
        uint64_t t0, t;
        asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
        for (;;) {
            uint32_t ok;
            asm volatile(
                "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], 0;\n\t"
                "selp.u32 %0, 1, 0, p;\n\t}"
                : "=r"(ok)
                : "r"(bar)
                : "memory");
            if (ok) break;
            asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
            if (t - t0 > 2000000000ull) {
                atomicExch(&g_probe_status, (int)QUEST_ETIMEOUT);
                break;
            }
        }
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (warp == 0) {
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem) : "memory");
    }
}

}  // namespace
}  // namespace quest

extern "C" quest_status quest_probe_mma_fp4(int iters, int* ctas, void* stream) {
    using namespace quest;
    if (iters < 1 || iters > kMaxIters || ctas == nullptr) return QUEST_EINVAL;
    static thread_local int attr_dev = -1;
    int dev = 0;
    cudaGetDevice(&dev);
    if (attr_dev != dev) {
        if (cudaFuncSetAttribute(probe_mma_fp4_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kProbeSmem + 1024) != cudaSuccess)
            return QUEST_ECUDA;
        attr_dev = dev;
    }
    *ctas = probe_sm_count();
    probe_mma_fp4_kernel<<<*ctas, kProbeThreads, kProbeSmem + 1024, static_cast<cudaStream_t>(stream)>>>(iters);
    return cudaGetLastError() == cudaSuccess ? QUEST_OK : QUEST_ECUDA;
}

namespace quest {
namespace {

// The int8 kind as the linear layer issues it: CTA pairs (cluster of two,
// tcgen05.mma.cta_group::2.kind::i8, M = 256 across the pair, N = 256, K = 32), each
// CTA holding its 128 rows of A and 128 rows of B in shared memory; the even CTA
// issues, one multicast commit ends the run in both CTAs.
constexpr uint32_t kIdescProbePair = (2u << 4) | (1u << 7) | (1u << 10) | (uint32_t(256 >> 3) << 17) |
                                     (uint32_t(256 >> 4) << 24);

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kProbeThreads, 1) probe_mma_i8_pair_kernel(int iters) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
    const uint32_t bar = sbase, slot = sbase + 16, a_addr = sbase + 1024, b_addr = a_addr + 128 * 128;
    for (uint32_t i = threadIdx.x * 16; i < 2 * 128 * 128; i += kProbeThreads * 16)
        *reinterpret_cast<uint4*>(smem + 1024 + i) = make_uint4(0x01010101u, 0x01010101u, 0x01010101u, 0x01010101u);
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    uint32_t rank;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(rank));
    if (threadIdx.x == 0) {
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar) : "memory");
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    const int warp = threadIdx.x >> 5;
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(slot) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + 16);
    if (rank == 0 && threadIdx.x == 0) {
        for (int i = 0; i < iters; ++i) {
            const uint32_t kk = uint32_t(i & 3) * 32;   // the four 32-byte K steps of a 128-byte row
            asm volatile(
                "{\n\t.reg .pred p;\n\t"
                "setp.ne.b32 p, %4, 0;\n\t"
                "tcgen05.mma.cta_group::2.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem),
                "l"(probe_desc(a_addr + kk)), "l"(probe_desc(b_addr + kk)), "r"(kIdescProbePair), "r"(i)
                : "memory");
        }
        asm volatile(
            "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
                bar),
            "h"((uint16_t)0x3)
            : "memory");
    }
    if (threadIdx.x == 0) {
        // bounded wait for the pair's MMAs (2 s; iters <= 2^16 take a few milliseconds)
        uint64_t t0, t;
        asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
        for (;;) {
            uint32_t ok;
            asm volatile(
                "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], 0;\n\t"
                "selp.u32 %0, 1, 0, p;\n\t}"
                : "=r"(ok)
                : "r"(bar)
                : "memory");
            if (ok) break;
            asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
            if (t - t0 > 2000000000ull) {
                atomicExch(&g_probe_status, (int)QUEST_ETIMEOUT);
                break;
            }
        }
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
    if (warp == 0) {
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, 512;" ::"r"(tmem) : "memory");
    }
}

template <bool kBf16>
quest_status launch_probe_dense(int iters, int* ctas, void* stream) {
    if (iters < 1 || iters > kMaxIters || ctas == nullptr) return QUEST_EINVAL;
    static thread_local int attr_dev = -1;
    int dev = 0;
    cudaGetDevice(&dev);
    if (attr_dev != dev) {
        if (cudaFuncSetAttribute(probe_mma_dense_kernel<kBf16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kProbeSmem + 1024) != cudaSuccess)
            return QUEST_ECUDA;
        attr_dev = dev;
    }
    *ctas = probe_sm_count();
    probe_mma_dense_kernel<kBf16>
        <<<*ctas, kProbeThreads, kProbeSmem + 1024, static_cast<cudaStream_t>(stream)>>>(iters);
    return cudaGetLastError() == cudaSuccess ? QUEST_OK : QUEST_ECUDA;
}

}  // namespace
}  // namespace quest

extern "C" quest_status quest_probe_mma_i8(int iters, int* ctas, void* stream) {
    return quest::launch_probe_dense<false>(iters, ctas, stream);
}

extern "C" quest_status quest_probe_mma_bf16(int iters, int* ctas, void* stream) {
    return quest::launch_probe_dense<true>(iters, ctas, stream);
}

extern "C" quest_status quest_probe_status(void* stream) {
    int v = 0, zero = 0;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaMemcpyFromSymbolAsync(&v, quest::g_probe_status, sizeof(int), 0, cudaMemcpyDeviceToHost, s) !=
            cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return QUEST_ECUDA;
    if (v != 0) {
        cudaMemcpyToSymbolAsync(quest::g_probe_status, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, s);
        cudaStreamSynchronize(s);
    }
    return static_cast<quest_status>(v);
}

extern "C" quest_status quest_probe_mma_sp_i8(int iters, int cp_every, int* ctas, void* stream) {
    using namespace quest;
    if (iters < 1 || iters > kMaxIters || cp_every < 0 || cp_every > 64 || ctas == nullptr) return QUEST_EINVAL;
    static thread_local int attr_dev = -1;
    int dev = 0;
    cudaGetDevice(&dev);
    if (attr_dev != dev) {
        if (cudaFuncSetAttribute(probe_mma_sp_i8_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kProbeSmem + 1024) != cudaSuccess)
            return QUEST_ECUDA;
        attr_dev = dev;
    }
    *ctas = probe_sm_count();
    probe_mma_sp_i8_kernel<<<*ctas, kProbeThreads, kProbeSmem + 1024, static_cast<cudaStream_t>(stream)>>>(iters,
                                                                                                       cp_every);
    return cudaGetLastError() == cudaSuccess ? QUEST_OK : QUEST_ECUDA;
}

extern "C" quest_status quest_probe_mma_i8_pair(int iters, int* ctas, void* stream) {
    using namespace quest;
    if (iters < 1 || iters > kMaxIters || ctas == nullptr) return QUEST_EINVAL;
    static thread_local int attr_dev = -1;
    int dev = 0;
    cudaGetDevice(&dev);
    if (attr_dev != dev) {
        if (cudaFuncSetAttribute(probe_mma_i8_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kProbeSmem + 1024) != cudaSuccess)
            return QUEST_ECUDA;
        attr_dev = dev;
    }
    *ctas = probe_sm_count() & ~1;   // whole pairs, one CTA per SM
    probe_mma_i8_pair_kernel<<<*ctas, kProbeThreads, kProbeSmem + 1024, static_cast<cudaStream_t>(stream)>>>(iters);
    return cudaGetLastError() == cudaSuccess ? QUEST_OK : QUEST_ECUDA;
}

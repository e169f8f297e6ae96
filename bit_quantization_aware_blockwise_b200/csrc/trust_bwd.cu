// QuEST trust-estimator backward (sm_100a).
//
// The gradient with respect to the dequantised, Hadamard-domain value is
// multiplied by the trust mask and taken back through the (self-inverse)
// normalised Hadamard transform (pith.science review of QuEST, "What carries
// the argument"; Figure 2 caption: inverse Hadamard transforms on the backward
// pass):  grad_in_block = H (m . grad_out_block) / sqrt(n).
//
// HBM-bound: 2 bytes in, 1/8 byte of mask in, 2 bytes out per element. Same
// team layout as the forward quantizer (quest_device.cuh); the mask byte of a
// chunk covers exactly its 8 elements.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "quest_device.cuh"
#include "quest_internal.h"
#include "quest_sync.cuh"

namespace quest {
namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ uint32_t ld_mask_byte(const uint8_t* p) {
    uint16_t v;
    asm volatile("ld.global.nc.L1::no_allocate.u8 %0, [%1];" : "=h"(v) : "l"(p));
    return v;
}

__device__ __forceinline__ uint32_t ld_mask_bytes8(const uint8_t* p) {
    // eight 0/1 bytes -> 8-bit mask
    uint2 w;
    asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];"
                 : "=r"(w.x), "=r"(w.y)
                 : "l"(p));
    uint32_t m = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        m |= ((w.x >> (8 * i)) & 1u) << i;
        m |= ((w.y >> (8 * i)) & 1u) << (4 + i);
    }
    return m;
}

template <int HB>
__global__ void __launch_bounds__(kThreads) trust_bwd_kernel(const TrustArgs a) {
    using S = TeamShape<HB>;
    constexpr int K = S::K, LPB = S::LPB, TPW = 32 / LPB;
    const int lane = threadIdx.x & 31, sub = lane % LPB;
    const int64_t total = a.rows * (a.cols / HB);
    const int64_t warp0 = (int64_t(blockIdx.x) * kThreads + threadIdx.x) >> 5;
    const int64_t wstride = int64_t(gridDim.x) * (kThreads / 32);

    for (int64_t wb = warp0 * TPW; wb < total; wb += wstride * TPW) {
        const int64_t blk = wb + lane / LPB;
        const bool valid = blk < total;
        const int64_t e = blk * HB;  // dense [rows, cols]: flat element offset
        float v[K][8];
        if (valid) {
#pragma unroll
            for (int j = 0; j < K; ++j) {
                const int64_t c0 = e + (sub + LPB * j) * 8;
                ChunkIO<__nv_bfloat16>::load(a.g + c0, v[j]);
                const uint32_t m = a.mask_mode == 0 ? ld_mask_byte(a.mask + c0 / 8)
                                                    : ld_mask_bytes8(a.mask + c0);
#pragma unroll
                for (int i = 0; i < 8; ++i) v[j][i] = ((m >> i) & 1u) ? v[j][i] : 0.0f;
            }
        } else {
#pragma unroll
            for (int j = 0; j < K; ++j)
#pragma unroll
                for (int i = 0; i < 8; ++i) v[j][i] = 0.0f;
        }
        fwht_team<K, LPB>(v, lane);
        if (valid) {
#pragma unroll
            for (int j = 0; j < K; ++j) {
#pragma unroll
                for (int i = 0; i < 8; ++i) v[j][i] *= a.inv_sqrt_hb;
                ChunkIO<__nv_bfloat16>::store(a.out + e + (sub + LPB * j) * 8, v[j]);
            }
        }
    }
}

template <int HB>
cudaError_t launch_hb(const TrustArgs& a, cudaStream_t stream) {
    using S = TeamShape<HB>;
    constexpr int TPW = 32 / S::LPB;
    const int64_t total = a.rows * (a.cols / HB);
    const int64_t warps = (total + TPW - 1) / TPW;
    const int64_t want = (warps + (kThreads / 32) - 1) / (kThreads / 32);
    auto fn = trust_bwd_kernel<HB>;
    const int64_t cap = int64_t(sm_count()) * max_ctas_per_sm((const void*)fn, kThreads, 0);
    const int grid = (int)(want < cap ? want : cap);
    fn<<<grid, kThreads, 0, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace

// ===========================================================================
// TMA-staged trust backward (rows of a multiple of 128 elements): the same
// producer / consumer ring as the TMA-staged quantizer, half-slab layout (two
// lanes per 128-element slab), packed fp32x2 butterflies, 1/sqrt(n) applied
// with one packed multiply. Each lane fetches its 64 mask bits (or bytes) from
// global memory before waiting for its stage so the two latencies overlap.
// ===========================================================================
namespace tma_trust {

constexpr int kConsumerWarps = 11;   // + producer = 12 warps: ~168 registers per thread
constexpr int kConsumerThreads = 32 * kConsumerWarps;
constexpr int kThreadsTma = kConsumerThreads + 32;
constexpr int kSlabsPerStage = kConsumerThreads / 2;
constexpr int kStageBytes = kSlabsPerStage * 256;           // bf16, 44 KB
constexpr int kStages = 4;
constexpr int kBarOffset = kStages * kStageBytes;
constexpr int kAbortOffset = kBarOffset + 16 * kStages;
constexpr int kSmemTotal = kAbortOffset + 16 + 1024;

__device__ int g_trust_status = 0;

struct Geo {
    int R_t;          // rows per tile (tiles are whole rows when they fit)
    int S_c;          // slabs per tile along a row
    int tiles_c, num_tiles, spr;
    uint32_t box_bytes;
};

// 64 mask bits of the half-slab starting at element e0 (dense layout).
__device__ __forceinline__ uint2 load_mask64(const TrustArgs& a, int64_t e0) {
    if (a.mask_mode == 0) return *reinterpret_cast<const uint2*>(a.mask + e0 / 8);
    uint32_t m0 = 0, m1 = 0;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        const uint2 w = *reinterpret_cast<const uint2*>(a.mask + e0 + 8 * q);
        uint32_t bits = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            bits |= ((w.x >> (8 * i)) & 1u) << i;
            bits |= ((w.y >> (8 * i)) & 1u) << (4 + i);
        }
        if (q < 4) m0 |= bits << (8 * q); else m1 |= bits << (8 * (q - 4));
    }
    return make_uint2(m0, m1);
}

template <int HB>
__global__ void __launch_bounds__(kThreadsTma, 1)
trust_tma_kernel(const __grid_constant__ CUtensorMap map_g, const TrustArgs a, const Geo g) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = sync::smem_u32(smem);
    const uint32_t bar_full = sbase + kBarOffset;
    const uint32_t bar_empty = bar_full + 8 * kStages;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kAbortOffset);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            sync::mbar_init(bar_full + 8 * s, 1);
            sync::mbar_init(bar_empty + 8 * s, kConsumerThreads);
        }
        *abort_flag = 0;
        sync::fence_mbar_init();
        sync::prefetch_tensormap(&map_g);
    }
    __syncthreads();

    if (warp == 0) {
        if (lane == 0) {
            uint32_t it = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < g.num_tiles; tile += gridDim.x, ++it) {
                const uint32_t st = it % kStages, ph = (it / kStages) & 1;
                if (!sync::mbar_wait(bar_empty + 8 * st, ph ^ 1, abort_flag, &g_trust_status,
                                     (int)QUEST_ETIMEOUT)) {
                    ok = false;
                    break;
                }
                const int tr = tile / g.tiles_c, tc = tile - tr * g.tiles_c;
                sync::mbar_arrive_expect_tx(bar_full + 8 * st, g.box_bytes);
                sync::tma_load_3d(sbase + st * kStageBytes, &map_g, 0, tc * g.S_c * 2, tr * g.R_t,
                                  bar_full + 8 * st);
            }
            if (!ok) {
                const uint32_t n = it < (uint32_t)kStages ? it : kStages;
                for (uint32_t i = it - n; i < it; ++i)
                    sync::mbar_drain(bar_full + 8 * (i % kStages), (i / kStages) & 1);
            }
        }
        return;
    }

    const int L = threadIdx.x - 32;
    const int slab = L >> 1, half = L & 1;
    const int sr = slab / g.S_c, sc = slab - sr * g.S_c;
    const bool slot_ok = sr < g.R_t;
    const uint32_t row0 = uint32_t(2 * slab + half);
    const float2 scale2 = make_float2(a.inv_sqrt_hb, a.inv_sqrt_hb);
    // where this lane's half-slab of `tile` lives; false if it is padding
    auto locate = [&](int tile, int64_t& e0) -> bool {
        const int trow = tile / g.tiles_c, tcol = tile - trow * g.tiles_c;
        const int64_t row = int64_t(trow) * g.R_t + sr;
        const int scol = tcol * g.S_c + sc;
        e0 = row * a.cols + int64_t(scol) * 128 + half * 64;   // dense [rows, cols]
        return slot_ok && row < a.rows && scol < g.spr;
    };
    // the mask of the next tile is requested one tile ahead, so its latency
    // hides behind the current tile
    int64_t e_cur = 0;
    bool v_cur = blockIdx.x < g.num_tiles && locate(blockIdx.x, e_cur);
    uint2 m_cur = v_cur ? load_mask64(a, e_cur) : make_uint2(0u, 0u);
    uint32_t it = 0;
    for (int tile = blockIdx.x; tile < g.num_tiles; tile += gridDim.x, ++it) {
        const uint32_t st = it % kStages, ph = (it / kStages) & 1;
        const int nxt = tile + gridDim.x;
        int64_t e_nxt = 0;
        const bool v_nxt = nxt < g.num_tiles && locate(nxt, e_nxt);
        const uint2 m_nxt = v_nxt ? load_mask64(a, e_nxt) : make_uint2(0u, 0u);

        const bool got = sync::mbar_wait(bar_full + 8 * st, ph, abort_flag, &g_trust_status,
                                         (int)QUEST_ETIMEOUT);
        if (__any_sync(0xFFFFFFFFu, !got)) break;   // the warp leaves together on a timeout
        float2 P[32];
        const uint32_t base = sbase + st * kStageBytes;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const uint4 v = sync::lds128(base + row0 * 128 + ((j ^ (row0 & 7)) << 4));
            const uint32_t mw = (j < 4) ? m_cur.x : m_cur.y;
            const int sh = 8 * (j & 3);
            const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const uint32_t b2 = mw >> (sh + 2 * q);
                P[4 * j + q] = make_float2((b2 & 1u) ? bf16lo_to_f32(w4[q]) : 0.0f,
                                           (b2 & 2u) ? bf16hi_to_f32(w4[q]) : 0.0f);
            }
        }
        sync::mbar_arrive(bar_empty + 8 * st);
        fwht_halfslab<HB>(P, lane);
        if (v_cur) {
            uint8_t* dst = reinterpret_cast<uint8_t*>(a.out + e_cur);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                uint32_t o[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float2 y = __fmul2_rn(P[4 * q + i], scale2);
                    o[i] = pack_bf16x2(y.x, y.y);
                }
                *reinterpret_cast<uint4*>(dst + 16 * q) = make_uint4(o[0], o[1], o[2], o[3]);
            }
        }
        e_cur = e_nxt;
        v_cur = v_nxt;
        m_cur = m_nxt;
    }
}

template <int HB>
cudaError_t launch_t(const TrustArgs& a, const Geo& g, const CUtensorMap& map, cudaStream_t s) {
    auto fn = trust_tma_kernel<HB>;
    static thread_local int attr_dev = -1;
    int dev = 0;
    cudaGetDevice(&dev);
    if (attr_dev != dev) {
        cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemTotal);
        if (e != cudaSuccess) return e;
        attr_dev = dev;
    }
    const int sms = sm_count();
    const int grid = g.num_tiles < sms ? g.num_tiles : sms;
    fn<<<grid, kThreadsTma, kSmemTotal, s>>>(map, a, g);
    return cudaGetLastError();
}

cudaError_t launch(const TrustArgs& a, int hb, cudaStream_t s) {
    Geo g;
    g.spr = (int)(a.cols / 128);
    g.S_c = g.spr < 128 ? g.spr : 128;   // box dim 1 = 2 * S_c <= 256
    g.R_t = kSlabsPerStage / g.S_c;
    const int64_t want_tiles = 4LL * sm_count();
    while (g.R_t > 1 && ((a.rows + g.R_t - 1) / g.R_t) * ((g.spr + g.S_c - 1) / g.S_c) < want_tiles)
        g.R_t = (g.R_t + 1) / 2;
    g.tiles_c = (g.spr + g.S_c - 1) / g.S_c;
    const int64_t tiles_r = (a.rows + g.R_t - 1) / g.R_t;
    if (tiles_r * g.tiles_c > 0x7FFFFFFF) return cudaErrorInvalidValue;
    g.num_tiles = (int)(tiles_r * g.tiles_c);
    g.box_bytes = (uint32_t)g.R_t * g.S_c * 256;
    CUtensorMap map;
    const uint64_t dims[3] = {64, (uint64_t)(a.cols / 64), (uint64_t)a.rows};
    const uint64_t strides[2] = {128, (uint64_t)a.cols * 2};
    const uint32_t box[3] = {64, (uint32_t)(g.S_c * 2), (uint32_t)g.R_t};
    if (!encode_tensor_map(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, a.g, dims, strides, box,
                           CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    switch (hb) {
        case 16: return launch_t<16>(a, g, map, s);
        case 32: return launch_t<32>(a, g, map, s);
        case 64: return launch_t<64>(a, g, map, s);
        case 128: return launch_t<128>(a, g, map, s);
        case 256: return launch_t<256>(a, g, map, s);
    }
    return cudaErrorInvalidValue;
}

}  // namespace tma_trust

cudaError_t launch_trust_bwd(const TrustArgs& a, int had_block, cudaStream_t stream) {
    if (a.cols % 128 == 0 && (reinterpret_cast<uintptr_t>(a.g) & 15) == 0 &&
        (reinterpret_cast<uintptr_t>(a.mask) & 7) == 0)
        return tma_trust::launch(a, had_block, stream);
    switch (had_block) {
        case 16: return launch_hb<16>(a, stream);
        case 32: return launch_hb<32>(a, stream);
        case 64: return launch_hb<64>(a, stream);
        case 128: return launch_hb<128>(a, stream);
        case 256: return launch_hb<256>(a, stream);
    }
    return cudaErrorInvalidValue;
}

int read_and_clear_trust_status(cudaStream_t stream, cudaError_t* err) {
    int v = 0, zero = 0;
    cudaError_t e = cudaMemcpyFromSymbolAsync(&v, tma_trust::g_trust_status, sizeof(int), 0,
                                              cudaMemcpyDeviceToHost, stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    if (e == cudaSuccess && v != 0)
        e = cudaMemcpyToSymbolAsync(tma_trust::g_trust_status, &zero, sizeof(int), 0,
                                    cudaMemcpyHostToDevice, stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    *err = e;
    return v;
}

}  // namespace quest

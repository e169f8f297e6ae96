// Internal (non-ABI) declarations shared by the host entry points and the
// kernel launchers.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "quest.h"

namespace quest {

// Per-call constants of the forward quantizer (host-computed, passed by value).
struct QuantConsts {
    float c_delta;      // alpha_b / 2^(b-1): Delta = c_delta * r
    float inv_count;    // 1 / (HB * G): mean of the normalised y^2 = sum(y_u^2) * inv_count
    float sqrt_hb;      // sqrt(HB): y = y_u / sqrt(HB)
    float edge;         // 2^(b-1) + (T-1)/2: for T >= 1, m = [|t| <= edge]
    float half_trust;   // T / 2 (general mask rule)
    float s_lo, s_hi;   // kMagic + lo, kMagic + hi (clamp bounds of the biased code)
    uint32_t pack_mult; // 1, or 2 for the c = 2q+1 operand form
    uint32_t pack_add;  // additive constant of the modular packing (see quantize_fwd.cu)
    uint32_t pack_xor;  // un-biasing mask of the packed word
    // half-slab (TMA-staged) decision path, codes biased as q_b = q + 2^(b-1)
    float inv_levels;   // 2^-b
    // Per-group constants from rs = rsqrt(sum of y_u^2) (one MUFU op per group):
    float delta_k;      // Delta = ss * rs * delta_k          (c_delta * sqrt(inv_count))
    float inv_k;        // 1 / (sqrt(HB) Delta) = rs * inv_k
    float a_k;          // inv * 2^-b = rs * a_k
    float thr2_k;       // (edge sqrt(HB) Delta)^2 = ss * thr2_k
    float half_levels;  // 2^(b-1)
    float sat_k;        // 2^b (1 - 2^-23)
    float s_mid;        // kMagic + 2^(b-1)
    float s_top;        // kMagic + 2^b - 1
    float cell_center;  // 1/2 - 2^(b-1): q + 1/2 = q_b + cell_center
    uint32_t pack2_mult, pack2_add, pack2_xor;   // 32-bit words of 32/cb fields
    uint32_t pack8_add, pack8_xor;                // words of 8 fields (cb <= 4)
    int trust_ge1;      // 1: use m = [|t| <= edge]
    int code_fp8;       // operand codes c = 2q + 1 stored as FP8 E4M3
    int grid_fp4;       // 0 integer grid; 1 FP4 grid, packed E2M1 codes; 2 FP4 grid, int8 c = 2Q
    int mask_mode;      // -1 none, 0 bits, 1 bytes
    int deq_mode;       // -1 none, 0 bf16, 1 fp32
};

struct QuantArgs {
    const char* x;
    int64_t ld_x_bytes;      // row pitch of x in bytes
    int64_t rows, cols;
    int dense;               // 1 when x rows are contiguous (ld == cols)
    uint8_t* codes;
    int64_t codes_row_bytes;
    float* scales;
    uint8_t* mask;
    int64_t mask_row_bytes;
    uint8_t* deq;
    int64_t deq_row_bytes;
    QuantConsts c;
    // Optional second tensor of the same width and constants, quantized by the
    // same row-RMS launch after the first (rows2 == 0: none): its rows follow
    // those of x in one virtual row space. No mask or dequant for it.
    const char* x2;
    uint8_t* codes2;
    float* scales2;
    int64_t rows2;
};

// 2:4-sparse quantizer (quantize_sparse.cu): the dense quantizer's arguments with
// the compressed code rows (cols / 2 bytes), the metadata and the pruned mask rule.
struct SparseArgs {
    QuantArgs q;
    uint8_t* meta;           // [rows, cols / 8]: per run of four a nibble of the two kept indices
    int64_t meta_row_bytes;
    float prune_ratio;       // (T/2)^2 / edge^2: a pruned value's threshold on y^2, relative to thr2
    int bits;
};

struct TrustArgs {
    const uint16_t* g;       // bf16 [rows, cols]
    const uint8_t* mask;     // bits or bytes
    int mask_mode;           // 0 bits, 1 bytes
    int64_t rows, cols;
    uint16_t* out;           // bf16 [rows, cols]
    float inv_sqrt_hb;
};

// Launchers (return cudaSuccess or the launch error).
cudaError_t launch_quantize(const QuantArgs& a, quest_dtype x_dtype, int had_block, int cbits,
                            int bits, bool row_mode, cudaStream_t stream);
// Direct-load interleaved half-slab quantizer (quantize_hs.cu).
bool hs_path_ok(const QuantArgs& a, int had_block, int cbits, bool row_mode);
cudaError_t launch_quantize_hs(const QuantArgs& a, quest_dtype x_dtype, int had_block, int cbits,
                               int bits, bool row_mode, cudaStream_t stream);
// bf16 quantizer with the 16-point Hadamard factor on tensor cores (quantize_tc.cu).
bool tc_path_ok(const QuantArgs& a, quest_dtype x_dtype, int had_block, int cbits, bool row_mode);
cudaError_t launch_quantize_tc(const QuantArgs& a, int had_block, int cbits, int bits, bool row_mode,
                               cudaStream_t stream);
cudaError_t launch_trust_bwd(const TrustArgs& a, int had_block, cudaStream_t stream);
cudaError_t launch_quantize_sparse24(const SparseArgs& s, bool row_mode, cudaStream_t stream);
// Trust backward with the tensor-core Hadamard factor (trust_tc.cu).
bool trust_tc_ok(const TrustArgs& a, int had_block);
cudaError_t launch_trust_tc(const TrustArgs& a, int had_block, cudaStream_t stream);
// inject_timeout: the launch withholds its operand loads and bounds its waits at
// 1 ms (quest_debug_inject_fault, QUEST_FAULT_WAIT_TIMEOUT); false on every normal call.
cudaError_t launch_w4a4(const int8_t* A, const float* sa, const int8_t* B, const float* sb,
                        int64_t M, int64_t N, int64_t K, uint16_t* y, int32_t* acc,
                        cudaStream_t stream, bool inject_timeout = false);

// Read (synchronising `stream`) and clear the device status word of the integer
// linear layer (w4a4_gemm.cu), the grouped layer (w4a4_grouped.cu), the fused
// input gradient (trust_linear.cu) and the FP4 layer (fp4_gemm.cu); each returns
// its value (0 or a quest_status).
cudaError_t launch_w4a4_sparse24(const int8_t* X, const float* sx, const int8_t* W, const uint8_t* E,
                                 const float* sw, int64_t M, int64_t N, int64_t K, uint16_t* y, int32_t* acc,
                                 cudaStream_t stream);
int read_and_clear_gemm_status(cudaStream_t stream, cudaError_t* err);
int read_and_clear_sparse_status(cudaStream_t stream, cudaError_t* err);
int read_and_clear_grouped_status(cudaStream_t stream, cudaError_t* err);
int read_and_clear_trust_linear_status(cudaStream_t stream, cudaError_t* err);
int read_and_clear_fp4_status(cudaStream_t stream, cudaError_t* err);
// dst[c][r] = src[r][c] for bf16 [rows, cols] (transpose.cu).
cudaError_t launch_transpose_bf16(const uint16_t* src, int64_t rows, int64_t cols, uint16_t* dst,
                                  cudaStream_t stream);
// Input gradient of the quantized linear layer with the trust backward fused in:
// gx = H (mask * (gy wt^T)) / sqrt(128) per 128-column block (trust_linear.cu).
cudaError_t launch_trust_linear(const uint16_t* gy, const uint16_t* wt, const uint8_t* mask, int64_t M,
                                int64_t N, int64_t K, uint16_t* gx, cudaStream_t stream);
// y [M, N] = x_hat [M, K] w_hat [N, K]^T on bf16 operands, fp32 accumulation (trust_linear.cu).
cudaError_t launch_linear_bf16(const uint16_t* x_hat, const uint16_t* w_hat, int64_t M, int64_t N, int64_t K,
                               uint16_t* y, cudaStream_t stream);
// y [M, N] = (sum_k Q_a Q_w) sa[m] sb[n] on packed E2M1 codes, block-scaled FP4 MMA (fp4_gemm.cu).
cudaError_t launch_fp4_linear(const uint8_t* A, const float* sa, const uint8_t* B, const float* sb, int64_t M,
                              int64_t N, int64_t K, uint16_t* y, float* acc, cudaStream_t stream);
cudaError_t launch_w4a4_grouped(const int8_t* A, const float* sa, const int8_t* B, const float* sb,
                                int64_t M, int64_t N, int64_t K, uint16_t* y, float* y32,
                                cudaStream_t stream);

// Number of SMs and max resident CTAs of `func` per SM on the current device.
int sm_count();
int max_ctas_per_sm(const void* func, int threads, size_t smem);

// Programmatic dependent launch. A kernel launched by launch_pdl may be scheduled
// while the kernel before it on the stream is still finishing (once every CTA of
// that kernel has called pdl_trigger() or exited); it must call pdl_wait() before
// it reads or writes global memory: pdl_wait() returns once the previous kernel
// has completed and its writes are visible. The kernels of the hot path call
// pdl_wait() and then pdl_trigger() before their first global access, so the
// launch and prologue of the next kernel overlap the tail of the current one.
#ifdef __CUDACC__
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
#endif

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                              Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

}  // namespace quest

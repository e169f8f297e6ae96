/*
 * quest.h -- C ABI of the QuEST quantizer hot path for NVIDIA B200 (sm_100a).
 *
 * Method: "QuEST: Stable Training of LLMs with 1-Bit Weights and Activations"
 * (Panferov, Chen, Tabesh, Castro, Nikdan, Alistarh; arXiv 2502.05003), as
 * described on the pith.science review page ("What carries the argument",
 * "Assumptions & free parameters", Figures 2 and 5) and the atlas.scime.ai
 * summary ("Approach", "Key results").
 *
 * General conventions
 *   - Every tensor argument is a DEVICE pointer to memory the caller owns
 *     (allocated by the caller, e.g. through PyTorch). The library allocates no
 *     device memory, keeps no per-call state and never synchronises: every
 *     entry point validates its arguments on the host, enqueues its kernel(s) on
 *     `stream` and returns.
 *   - `stream` is a cudaStream_t passed as void*; NULL means the legacy default
 *     stream. The current CUDA device must be the device owning the pointers.
 *   - Matrices are row-major. "rows" is the number of independent vectors, "cols"
 *     the length along which the Hadamard transform and the RMS groups run (the
 *     reduction dimension of the linear layer that consumes the codes).
 *   - bf16 means IEEE bfloat16 (1-8-7), stored as 16-bit little-endian words.
 *   - Errors: a non-zero quest_status. Argument errors are detected before any
 *     launch and leave every output untouched; QUEST_ECUDA reports a launch or
 *     driver error (the CUDA error string is available from
 *     quest_last_error_message()). Nothing in the library traps or asserts on
 *     the device.
 *   - Thread safety: all entry points may be called concurrently from several
 *     host threads (the per-thread error message is thread-local).
 */
#ifndef QUEST_B200_H
#define QUEST_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum quest_status {
    QUEST_OK = 0,
    QUEST_EINVAL = 1,         /* an argument is out of range, NULL or misaligned */
    QUEST_EUNSUPPORTED = 2,   /* a valid request the library does not implement */
    QUEST_ECUDA = 3,          /* CUDA launch / driver error */
    QUEST_ETIMEOUT = 4        /* a bounded device-side wait gave up */
} quest_status;

typedef enum quest_dtype {
    QUEST_BF16 = 0,
    QUEST_FP32 = 1
} quest_dtype;

/* How integer codes are stored.
 *   QUEST_CODES_PACKED        two's-complement code q in a container of
 *                             1/2/4/4/8/8/8/8 bits for b = 1..8, packed little-
 *                             endian inside each byte (element 2j in the low
 *                             nibble at 4-bit, element 8j in bit 0 at 1-bit).
 *                             Row stride: cols * container_bits / 8 bytes.
 *   QUEST_CODES_INT8          one int8 per element holding q.
 *   QUEST_CODES_GEMM_OPERAND  one int8 per element holding c = 2q + 1 (odd,
 *                             |c| <= 2^b - 1), the exact integer form of the
 *                             midrise level (q + 1/2); requires b <= 7.
 *   QUEST_CODES_GEMM_OPERAND_E4M3
 *                             one byte per element holding the same c in the
 *                             OCP FP8 E4M3 format (sign, 4-bit exponent with
 *                             bias 7, 3-bit mantissa), exact for |c| <= 15:
 *                             requires b <= 4. It is the operand of
 *                             quest_w4a4_linear_grouped. Supported where the
 *                             rows are whole 128-value slabs with 8-byte aligned
 *                             codes and at most 16 slabs per row in row-RMS mode
 *                             (QUEST_EUNSUPPORTED otherwise).
 * The FP4 grid (bits must be 4; see quest_quantize_fwd for the grid, scale and
 * mask of this variant):
 *   QUEST_CODES_FP4_PACKED    4-bit OCP E2M1 codes (bit 3 sign, bits 2..1
 *                             exponent with bias 1, bit 0 mantissa), two per
 *                             byte, element 2j in the low nibble. Row stride
 *                             cols / 2 bytes; codes 4-byte aligned.
 *   QUEST_CODES_FP4_OPERAND   one int8 per element holding c = 2 Q, twice the
 *                             grid value Q (c in {0, +-1, +-2, +-3, +-4, +-6,
 *                             +-8, +-12}): the exact integer operand of
 *                             quest_w4a4_linear, whose Y = acc (Delta_x / 2)
 *                             (Delta_w / 2) then equals sum Q_x Q_w Delta_x Delta_w.
 * Both FP4 forms are supported where the rows are whole 128-value slabs with
 * aligned codes and at most 16 slabs per row in row-RMS mode (QUEST_EUNSUPPORTED
 * otherwise). */
typedef enum quest_code_mode {
    QUEST_CODES_PACKED = 0,
    QUEST_CODES_INT8 = 1,
    QUEST_CODES_GEMM_OPERAND = 2,
    QUEST_CODES_GEMM_OPERAND_E4M3 = 3,
    QUEST_CODES_FP4_PACKED = 4,
    QUEST_CODES_FP4_OPERAND = 5
} quest_code_mode;

/* How the trust mask is stored (1 = gradient kept, 0 = gradient zeroed).
 *   QUEST_MASK_BITS   uint32 words [rows, cols/32]; bit j of word w is column
 *                     32w + j (equivalently bytes [rows, cols/8], bit j of byte
 *                     i is column 8i + j).
 *   QUEST_MASK_BYTES  uint8 [rows, cols], one 0/1 byte per element. */
typedef enum quest_mask_mode {
    QUEST_MASK_BITS = 0,
    QUEST_MASK_BYTES = 1
} quest_mask_mode;

/*
 * quest_quantize_fwd -- QuEST forward quantizer with trust mask.
 *
 * Follows pith.science review, "What carries the argument" (Hadamard transform,
 * then projection onto a uniform grid whose scale minimises the L2 error
 * against a standard Gaussian; the mask zeroes entries whose quantization error
 * exceeds half a quantization interval), atlas.scime.ai summary, "Approach"
 * (Hadamard transform with RMS normalisation, MSE-optimal Gaussian clipping,
 * trust threshold) and pith.science review, "Assumptions & free parameters"
 * (alpha fixed from an N(0,1) target). For every row and every Hadamard block
 * of `had_block` consecutive columns:
 *     y     = H x_block / sqrt(had_block)      (Sylvester order, H_ij = (-1)^popcount(i&j))
 *     r     = sqrt(mean(y^2))   over the rms group (`rms_group` consecutive columns)
 *     Delta = alpha_b * r / 2^(b-1)            (alpha_b = quest_alpha(bits))
 *     t     = y / Delta
 *     q     = clamp(floor(t), -2^(b-1), 2^(b-1) - 1)
 *     yhat  = (q + 1/2) * Delta                (stays in the Hadamard domain)
 *     m     = [ |t - (q + 1/2)| <= trust / 2 ]
 * A group with r == 0 yields Delta = 0, q = 0, yhat = 0, m = 1. Inputs holding
 * NaN or Inf propagate into that group's outputs (codes become unspecified but
 * in range); they are not checked.
 *
 * FP4 grid (code_mode QUEST_CODES_FP4_*, bits = 4). The pages report QuEST on an
 * FP4 grid too and that it trails INT4 through a higher Gaussian MSE once
 * clipping is allowed (pith.science review, "What carries the argument" and its
 * results list); they do not spell the variant out. This library reads it as the
 * same transform and RMS with the grid and mask replaced:
 *     Delta = s* r                             (s* = quest_alpha_fp4(), the scale
 *                                               of the E2M1 grid minimising the
 *                                               MSE on N(0,1))
 *     Q     = the E2M1 value nearest to t = y / Delta (ties to the even mantissa,
 *             saturating at +-6; the code of a small negative t is -0)
 *     yhat  = Q * Delta
 *     m     = [ |t - Q| <= trust / 2 * w(t) ],  w = the width of the grid
 *             interval that holds |t| (0.5 below 2, 1 below 4, 2 above; beyond 6
 *             the last interval [4, 6] counts), so for trust >= 1:
 *             m = [ |t| <= 6 + trust ].
 *
 * Arguments
 *   x          device, x_dtype [rows, ld_x] (only the first `cols` columns read);
 *              16-byte aligned; ld_x * sizeof(x_dtype) a multiple of 16 bytes.
 *   rows       >= 0 (0 is a no-op).   cols > 0, a multiple of had_block.
 *   bits       1..8.   had_block: 16, 32, 64, 128 or 256.
 *   rms_group  had_block (one RMS per Hadamard block) or cols (one RMS per row,
 *              the per-row scale form used by the integer linear layer; then
 *              cols <= 16384).
 *   trust      trust factor T > 0 (1.0 = half an interval; the 1-bit runs of the
 *              pages widen the outer trust region with s* = 1.30).
 *   code_mode  storage of `codes` (see quest_code_mode); codes must be aligned to
 *              8 bytes (4 for 4-bit packed, 2 for 2-bit, 1 for 1-bit).
 *   codes      device, required: quest_codes_bytes(rows, cols, bits, code_mode) bytes.
 *   scales     device, required: fp32 [rows, cols / rms_group], Delta per group.
 *   mask_mode, mask   device, optional (NULL = not written): quest_mask_bytes() bytes.
 *   dequant    device, optional (NULL = not written): dequant_dtype [rows, cols],
 *              16-byte aligned, yhat.
 * Returns QUEST_OK, QUEST_EINVAL (bad argument), QUEST_EUNSUPPORTED, QUEST_ECUDA.
 */
quest_status quest_quantize_fwd(const void* x, quest_dtype x_dtype, int64_t rows, int64_t cols,
                                int64_t ld_x, int bits, int had_block, int64_t rms_group,
                                float trust, quest_code_mode code_mode, void* codes,
                                float* scales, quest_mask_mode mask_mode, void* mask,
                                void* dequant, quest_dtype dequant_dtype, void* stream);

/*
 * quest_quantize_operands -- both operands of a QuEST linear layer in one call:
 * quest_quantize_fwd with rms_group = K (one RMS per row), no mask and no dequant,
 * on x [M, K] and on w [N, K], both dense (row pitch K elements) and of one dtype.
 * Where both tensors take the tensor-core row layout (bf16, rows of whole 128-value
 * slabs, at most 16 slabs per row, aligned codes) the library quantizes them in a
 * single launch, w's rows after x's; otherwise it issues the two quantizations one
 * after the other. Outputs and errors as quest_quantize_fwd (codes in code_mode,
 * scales fp32 [M] and [N], Delta per row); M == 0 or N == 0 skips that tensor.
 */
quest_status quest_quantize_operands(const void* x, int64_t M, const void* w, int64_t N, int64_t K,
                                     quest_dtype dtype, int bits, int had_block, quest_code_mode code_mode,
                                     void* x_codes, float* x_scales, void* w_codes, float* w_scales,
                                     void* stream);

/*
 * quest_quantize_sparse24 -- the 2:4-sparse INT variant of the QuEST quantizer.
 *
 * The pages evaluate QuEST on a 2:4-sparse INT4 format and report that adding 2:4
 * sparsity to QuEST INT4 costs accuracy (atlas.scime.ai summary, ablation table;
 * pith.science review, results list and Figure 4a: INT, FP and INT+sparse formats
 * at 4 bits), without spelling the format out. This library reads it as the
 * transform and RMS of quest_quantize_fwd (Hadamard block 128, r over every value
 * of the rms group), then, in every run of four consecutive transformed values:
 *     keep the two values of largest |y| (on equal magnitudes the lower index wins),
 *     Delta = quest_alpha_sparse24(bits) * r / 2^(b-1),  t = y / Delta,
 *     kept:   q = clamp(floor(t), -2^(b-1), 2^(b-1)-1), yhat = (q + 1/2) Delta,
 *             m = [ |t - (q + 1/2)| <= trust / 2 ]
 *     pruned: yhat = 0, m = [ |t| <= trust / 2 ]   (the half-interval rule on the
 *             value's total error)
 * A group with r == 0 keeps the lower two indices of each run with q = 0, m = 1.
 *
 * Arguments
 *   x          device bf16 [rows, cols], dense (row pitch cols), 16-byte aligned.
 *   rows >= 0; cols a positive multiple of 128.   bits 1..7.
 *   had_block  must be 128 (QUEST_EUNSUPPORTED otherwise).
 *   rms_group  128, or cols (one RMS per row; then cols in 128, 256, 512, 1024, 2048).
 *   trust      T > 0.
 *   codes      device int8 [rows, cols / 2], 8-byte aligned: per run of four the two
 *              kept values' c = 2q + 1 in index order (the compressed operand of
 *              quest_w4a4_linear_sparse24).
 *   meta       device uint8 [rows, cols / 8], 4-byte aligned: per run a nibble with
 *              the lower kept index in bits 0-1 and the higher in bits 2-3; byte j
 *              holds runs 2j (low nibble) and 2j + 1.
 *   scales     device fp32 [rows, cols / rms_group], Delta per group.
 *   mask       device, optional: uint32 mask words [rows, cols / 32] as QUEST_MASK_BITS.
 *   dequant    device, optional: bf16 [rows, cols] yhat (0 where pruned), 16-byte aligned.
 * Returns QUEST_OK, QUEST_EINVAL, QUEST_EUNSUPPORTED or QUEST_ECUDA.
 */
quest_status quest_quantize_sparse24(const void* x, int64_t rows, int64_t cols, int bits, int had_block,
                                     int64_t rms_group, float trust, void* codes, void* meta, float* scales,
                                     void* mask, void* dequant, void* stream);

/*
 * quest_trust_bwd -- trust-estimator backward.
 *
 * Follows pith.science review, "What carries the argument" (the gradient is
 * multiplied in the Hadamard domain by the binary mask) and Figure 2's caption
 * (two inverse Hadamard transforms on the backward pass, one per operand). For
 * every row and block:
 *     grad_in_block = H^T (m . grad_out_block) / sqrt(had_block)
 * (H is symmetric, so the inverse of the normalised transform is itself). No
 * gradient flows through the RMS scale.
 *
 * Arguments
 *   grad_out   device, bf16 [rows, cols], dL/dyhat in the Hadamard domain; 16-byte aligned.
 *   mask       device, the mask written by quest_quantize_fwd in `mask_mode`.
 *   rows >= 0; cols > 0, a multiple of had_block.
 *   had_block  16, 32, 64, 128 or 256 (the value used in the forward pass).
 *   grad_in    device, bf16 [rows, cols], dL/dx; 16-byte aligned; may not alias grad_out.
 */
quest_status quest_trust_bwd(const void* grad_out, const void* mask, quest_mask_mode mask_mode,
                             int64_t rows, int64_t cols, int had_block, void* grad_in,
                             void* stream);

/*
 * quest_w4a4_linear -- integer linear layer on QuEST codes.
 *
 * The pages' GPU kernels run the linear layers of a QuEST INT4 model on the
 * integer codes, with quantization, dequantization and Hadamard costs included
 * (atlas.scime.ai summary, "Key results"; pith.science review, Figure 5). Because
 * the Hadamard matrix is orthogonal, transforming both operands leaves the
 * product unchanged (pith.science review, "Assumptions & free parameters"), so
 * the product of the two Hadamard-domain operands is the layer output:
 *     acc[m][n] = sum_k a_codes[m][k] * w_codes[n][k]          (exact, int32)
 *     y[m][n]   = bf16_rne( acc[m][n] * (a_scales[m] / 2) * (w_scales[n] / 2) )
 * With codes in GEMM-operand form (c = 2q + 1) and per-row scales Delta
 * (rms_group = cols), y equals yhat_a . yhat_w^T.
 *
 * Arguments
 *   a_codes    device, int8 [M, K] row-major (K contiguous); 16-byte aligned.
 *   a_scales   device, fp32 [M].
 *   w_codes    device, int8 [N, K] row-major (the nn.Linear weight layout).
 *   w_scales   device, fp32 [N].
 *   M >= 0, N >= 0 (0 = no-op); N a multiple of 8; K >= 0, a multiple of 16,
 *   K < 131072 (so that any int8 products fit the int32 accumulator).
 *   y          device, bf16 [M, N]; 16-byte aligned.
 *   acc        device, optional int32 [M, N] copy of the accumulator (NULL = not
 *              written); meant for exactness checks.
 */
quest_status quest_w4a4_linear(const int8_t* a_codes, const float* a_scales,
                               const int8_t* w_codes, const float* w_scales, int64_t M,
                               int64_t N, int64_t K, void* y, int32_t* acc, void* stream);

/*
 * quest_w4a4_linear_grouped -- linear layer on QuEST codes with one scale per
 * row and per group of 128 consecutive K indices on both operands (the codes of
 * a quantize_fwd call with rms_group = had_block = 128 in the
 * QUEST_CODES_GEMM_OPERAND_E4M3 form).
 *
 * Same layer as quest_w4a4_linear (pith.science review, "Assumptions & free
 * parameters": a Hadamard transform applied to both operands leaves the product
 * unchanged), with the scales varying along K, so each group's exact integer
 * product is scaled on its own:
 *     acc_g[m][n] = sum over k in group g of a_codes[m][k] * w_codes[n][k]
 *     y[m][n]     = bf16_rne( sum_g (a_scales[m][g]/2) (w_scales[n][g]/2) acc_g[m][n] )
 * acc_g is exact (FP8 E4M3 tensor-core products accumulated in fp32) whenever
 * every partial sum is an integer below 2^24 in magnitude, which holds for
 * codes c = 2q + 1 with |c| <= 15; the group sum runs in fp32 (its rounding
 * error is below 1e-6 of sum_g |term_g|); the pages do not fix this precision.
 *
 * Arguments
 *   a_codes    device, FP8 E4M3 bytes [M, K] row-major; 16-byte aligned.
 *   a_scales   device, fp32 [M, K / group] row-major.
 *   w_codes    device, FP8 E4M3 bytes [N, K] row-major; 16-byte aligned.
 *   w_scales   device, fp32 [N, K / group] row-major.
 *   M >= 0, N >= 0 (0 = no-op); N a multiple of 8; K >= 0, a multiple of
 *   `group`, K < 2^24.
 *   group      must be 128 (QUEST_EUNSUPPORTED otherwise).
 *   y          device, bf16 [M, N]; 16-byte aligned.
 *   y_f32      device, optional fp32 [M, N] copy of y before the bf16 rounding
 *              (NULL = not written); meant for exactness checks.
 */
quest_status quest_w4a4_linear_grouped(const uint8_t* a_codes, const float* a_scales,
                                       const uint8_t* w_codes, const float* w_scales, int64_t M,
                                       int64_t N, int64_t K, int64_t group, void* y, float* y_f32,
                                       void* stream);

/*
 * quest_w4a4_linear_sparse24 -- integer linear layer with 2:4-sparse weight codes
 * on the sparse tensor cores.
 *
 * The layer of quest_w4a4_linear (pith.science review, Figure 5; "Assumptions &
 * free parameters": a transform on both operands leaves the product unchanged)
 * with the weights in the 2:4-sparse format the pages evaluate (atlas.scime.ai
 * summary, ablation table; pith.science review, Figure 4a), as
 * quest_quantize_sparse24 writes them with rms_group = K (one step per row):
 *     acc[m][n] = sum_k x_codes[m][k] * w[n][k]    (w = the weight codes with the
 *                                                   pruned values zero; exact, int32)
 *     y[m][n]   = bf16_rne( acc[m][n] * (x_scales[m] / 2) * (w_scales[n] / 2) )
 * The weights are the sparse operand of tcgen05.mma.sp (kind::i8): each run of four
 * K values contributes its two survivors.
 *
 * Arguments
 *   x_codes    device int8 [M, K] (c = 2q + 1, as quest_quantize_operands writes), 16-byte aligned.
 *   x_scales   device fp32 [M].
 *   w_codes    device int8 [N, K / 2]: the survivors' codes, 16-byte aligned.
 *   w_meta     device uint8 [N, K / 8]: the survivors' indices (quest_quantize_sparse24's
 *              meta), 16-byte aligned.
 *   w_scales   device fp32 [N].
 *   M, N >= 0 (0 = no-op); N a multiple of 8; K a multiple of 128, K < 131072.
 *   y          device bf16 [M, N], 16-byte aligned.
 *   acc        device, optional int32 [M, N] copy of the accumulator (NULL = not written).
 * Returns QUEST_OK, QUEST_EINVAL or QUEST_ECUDA; a bounded device-side wait that gives
 * up is reported by quest_device_status as QUEST_ETIMEOUT.
 */
quest_status quest_w4a4_linear_sparse24(const int8_t* x_codes, const float* x_scales, const int8_t* w_codes,
                                        const uint8_t* w_meta, const float* w_scales, int64_t M, int64_t N, int64_t K,
                                        void* y, int32_t* acc, void* stream);

/*
 * quest_fp4_linear -- linear layer on FP4 (E2M1) QuEST codes on the block-scaled
 * FP4 tensor cores.
 *
 * The FP4-grid variant of the quantizer (pith.science review, Figure 4a and
 * "Assumptions & free parameters"; the codes of a quantize_fwd call with
 * code_mode QUEST_CODES_FP4_PACKED and rms_group = cols, so one step Delta per
 * row) feeds the layer directly:
 *     acc[m][n] = sum_k Q_a[m][k] * Q_w[n][k]     (Q the E2M1 grid values)
 *     y[m][n]   = bf16_rne( acc[m][n] * a_scales[m] * w_scales[n] )
 * Every product of two E2M1 values is a multiple of 1/4 of magnitude <= 36, so
 * for K <= 16384 every partial sum is a multiple of 1/4 below 2^20 and the fp32
 * accumulation is exact. Same result as quest_w4a4_linear on the operand form
 * c = 2Q (QUEST_CODES_FP4_OPERAND), at twice its tensor-core rate and half its
 * operand bytes.
 *
 * Arguments
 *   a_codes    device, packed E2M1 [M, K/2] bytes (element 2j in the low nibble
 *              of byte j); 16-byte aligned.
 *   a_scales   device, fp32 [M] (Delta of each row).
 *   w_codes    device, packed E2M1 [N, K/2] bytes; 16-byte aligned.
 *   w_scales   device, fp32 [N].
 *   M >= 0, N >= 0 (0 = no-op); N a multiple of 8; K >= 0, a multiple of 32,
 *   K <= 16384.
 *   y          device, bf16 [M, N]; 16-byte aligned.
 *   acc        device, optional fp32 [M, N] copy of the accumulator (NULL = not
 *              written); meant for exactness checks.
 * Errors: QUEST_EINVAL on bad sizes, NULL or misaligned pointers (checked before
 * any launch); QUEST_ECUDA on a launch failure. A bounded device-side wait that
 * gives up is reported by quest_device_status as QUEST_ETIMEOUT.
 */
quest_status quest_fp4_linear(const uint8_t* a_codes, const float* a_scales, const uint8_t* w_codes,
                              const float* w_scales, int64_t M, int64_t N, int64_t K, void* y, float* acc,
                              void* stream);

/*
 * quest_trust_bwd_linear -- input gradient of a QuEST linear layer with the
 * trust backward fused into the product.
 *
 * Backward pass of y = x_hat w_hat^T, where x_hat is the quantized input in the
 * Hadamard domain carrying trust mask m (pith.science review, "What carries the
 * argument": the gradient is masked in the Hadamard domain; Figure 2 caption:
 * the inverse transforms run on the backward pass):
 *     G      = grad_y w_hat                              [M, K]  (fp32 accumulation)
 *     grad_x = H (m * G) / sqrt(128) per 128-column block          (bf16, RNE)
 * which equals quest_trust_bwd applied to G, with G kept on chip.
 *
 * Arguments
 *   grad_y   device bf16 [M, N], the gradient of the layer output, row-major.
 *   w_hat_t  device bf16 [K, N]: the dequantised weights w_hat [N, K] (Hadamard
 *            domain, e.g. quest_quantize_fwd's `dequant` of the weight)
 *            transposed, so that both operands run along N (see quest_transpose_bf16).
 *   mask     device, the trust mask bits of x_hat [M, K] (QUEST_MASK_BITS layout).
 *   M, N, K  >= 0; N a multiple of 8, K a multiple of 128; M, K < 2^31.
 *   had_block  128 (QUEST_EUNSUPPORTED otherwise).
 *   grad_x   device bf16 [M, K].
 * grad_y, w_hat_t, mask and grad_x 16-byte aligned. N == 0 writes zeros.
 * Returns QUEST_OK, QUEST_EINVAL, QUEST_EUNSUPPORTED or QUEST_ECUDA; a bounded wait
 * that gives up is reported by quest_device_status as QUEST_ETIMEOUT.
 */
quest_status quest_trust_bwd_linear(const void* grad_y, const void* w_hat_t, const void* mask, int64_t M,
                                    int64_t N, int64_t K, int had_block, void* grad_x, void* stream);

/*
 * quest_linear_bf16 -- the linear layer of QuEST training on dequantised operands.
 *
 * The forward pass multiplies the quantized operands in the Hadamard domain
 * (pith.science review, "Assumptions & free parameters": the transform applied to
 * both operands leaves the product unchanged; Figure 2 caption: two Hadamard
 * transforms on the forward pass):
 *     y = x_hat w_hat^T        x_hat [M, K], w_hat [N, K] bf16 (e.g. quest_quantize_fwd's
 *                              bf16 `dequant` of each operand, any RMS grouping),
 *                              fp32 accumulation, y bf16 [M, N] (RNE).
 * With per-128-group scales this is the layer of quest_w4a4_linear_grouped computed on
 * yhat rounded to bf16 instead of on the exact codes.
 *
 * Arguments: M, N, K >= 0, K and N multiples of 8, M, N, K < 2^31; x_hat, w_hat and y
 * device pointers, 16-byte aligned, y not overlapping the operands. K == 0 writes zeros.
 * Returns QUEST_OK, QUEST_EINVAL or QUEST_ECUDA (a bounded wait that gives up is
 * reported by quest_device_status, like quest_trust_bwd_linear's).
 */
quest_status quest_linear_bf16(const void* x_hat, const void* w_hat, int64_t M, int64_t N, int64_t K, void* y,
                               void* stream);

/*
 * quest_transpose_bf16 -- dst[c][r] = src[r][c] for a bf16 [rows, cols] matrix
 * (row-major, dense); dst is [cols, rows]. Produces the w_hat_t operand of
 * quest_trust_bwd_linear from a dequantised weight. src and dst must not overlap.
 * Returns QUEST_OK, QUEST_EINVAL or QUEST_ECUDA.
 */
quest_status quest_transpose_bf16(const void* src, int64_t rows, int64_t cols, void* dst, void* stream);

/*
 * quest_device_status -- synchronises `stream`, then reports (and clears) the
 * device-side status of the integer linear layer on the current device:
 * QUEST_ETIMEOUT if one of its bounded pipeline waits gave up since the last
 * call (its output is then incomplete), QUEST_OK otherwise, QUEST_ECUDA on a
 * CUDA error. The quantizer and trust kernels have no waits and never set it;
 * quest_trust_bwd_linear shares the linear layer's status word.
 */
quest_status quest_device_status(void* stream);

/* alpha_b, the clip edge of the b-bit grid (2^(b-1) times the step that minimises
 * the MSE of the midrise uniform quantizer for X ~ N(0,1)); bits 1..8. Follows
 * pith.science review, "What carries the argument" (the grid's scale minimises the
 * L2 error against a standard Gaussian) and "Assumptions & free parameters" (alpha
 * is fixed from an N(0,1) target, not fitted to data). Computed on the host at
 * first use. Returns NaN for an invalid bit-width. */
double quest_alpha(int bits);

/* s*, the scale of the OCP E2M1 (FP4) grid {0, +-0.5, +-1, +-1.5, +-2, +-3, +-4, +-6}
 * that minimises E[(X - s Q(X / s))^2] for X ~ N(0,1), Q round-to-nearest onto the
 * grid (the FP4 code modes use Delta = s* r). The same Gaussian-MSE fit as alpha_b
 * (pith.science review, "What carries the argument"; "Assumptions & free
 * parameters") applied to the FP4 grid the review's results list and Figure 4a
 * compare against INT4. Computed on the host at first use. */
double quest_alpha_fp4(void);

/* alpha_b of the 2:4-sparse format (quest_quantize_sparse24): 2^(b-1) times the step
 * of the midrise grid that minimises the MSE of the values surviving 2:4 pruning of
 * an N(0,1) input (of four values, the two of largest magnitude). The Gaussian fit of
 * pith.science review, "What carries the argument" and "Assumptions & free
 * parameters", taken on the sparse format the ablation table of the atlas.scime.ai
 * summary evaluates. bits 1..8; NaN otherwise. Computed on the host at first use. */
double quest_alpha_sparse24(int bits);

/* Bits of the storage container of a b-bit packed code: 1, 2, 4, 4, 8, 8, 8, 8. 0 if invalid. */
int quest_container_bits(int bits);

/* Bytes needed for `codes` / `mask` of a rows x cols tensor; 0 for invalid arguments. */
size_t quest_codes_bytes(int64_t rows, int64_t cols, int bits, quest_code_mode mode);
size_t quest_mask_bytes(int64_t rows, int64_t cols, quest_mask_mode mode);

/* Static description of a status code. */
const char* quest_status_string(quest_status s);

/* Detail of the last error on the calling host thread ("" if none). */
const char* quest_last_error_message(void);

/* ABI version (major * 10000 + minor * 100 + patch). */
int quest_version(void);

#ifdef __cplusplus
}
#endif

#endif /* QUEST_B200_H */

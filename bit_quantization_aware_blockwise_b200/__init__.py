"""QuEST quantizer hot path on B200 (sm_100a).

The product is the C-ABI library ``libquest_b200.so`` (declared in
``include/quest.h``); this package is its thin Python binding. Importing the
package loads nothing: the library is loaded on first use, and every call fails
loudly (``QuestError``) when it is missing or no CUDA device is present. There
is no CPU fallback.
"""
from ._binding import (  # noqa: F401
    QuestError,
    CODES_PACKED,
    CODES_INT8,
    CODES_GEMM_OPERAND,
    CODES_GEMM_OPERAND_E4M3,
    CODES_FP4_PACKED,
    CODES_FP4_OPERAND,
    MASK_BITS,
    MASK_BYTES,
    BF16,
    FP32,
    library_path,
    load_library,
    alpha,
    alpha_fp4,
    codes_bytes,
    mask_bytes,
    container_bits,
    quantize_fwd,
    quantize_operands,
    quantize_operands_raw,
    trust_bwd,
    w4a4_linear,
    quantize_fwd_raw,
    trust_bwd_raw,
    w4a4_linear_raw,
    w4a4_linear_grouped,
    w4a4_linear_grouped_raw,
    trust_bwd_linear,
    trust_bwd_linear_raw,
    transpose_bf16,
    transpose_bf16_raw,
    linear_bf16,
    linear_bf16_raw,
    fp4_linear,
    fp4_linear_raw,
    device_status,
    probe_mma_i8,
    probe_mma_fp4,
    probe_status,
    debug_inject_fault,
    FAULT_NONE,
    FAULT_LAUNCH,
    FAULT_WAIT_TIMEOUT,
)

__all__ = [
    "QuestError", "CODES_PACKED", "CODES_INT8", "CODES_GEMM_OPERAND", "CODES_GEMM_OPERAND_E4M3", "CODES_FP4_PACKED",
    "CODES_FP4_OPERAND", "MASK_BITS",
    "MASK_BYTES", "BF16", "FP32", "library_path", "load_library", "alpha", "alpha_fp4", "codes_bytes", "mask_bytes",
    "container_bits", "quantize_fwd", "quantize_operands", "quantize_operands_raw", "trust_bwd", "w4a4_linear", "quantize_fwd_raw",
    "trust_bwd_raw", "w4a4_linear_raw", "w4a4_linear_grouped", "w4a4_linear_grouped_raw",
    "trust_bwd_linear", "trust_bwd_linear_raw", "transpose_bf16", "transpose_bf16_raw",
    "linear_bf16", "linear_bf16_raw", "fp4_linear", "fp4_linear_raw", "device_status", "probe_mma_i8", "probe_mma_fp4", "probe_status",
    "debug_inject_fault", "FAULT_NONE", "FAULT_LAUNCH", "FAULT_WAIT_TIMEOUT",
]

"""ctypes binding of ``libquest_b200.so`` (see ``include/quest.h``).

Argument marshalling only: every step of the quantizer, trust backward and
integer linear layer runs in the library's CUDA kernels. PyTorch supplies
device memory and the current stream. The library is loaded on first use; if
it is missing, or a call fails, ``QuestError`` is raised. There is no fallback.
"""
from __future__ import annotations

import ctypes
import os
import threading

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_NAME = "libquest_b200.so"

CODES_PACKED, CODES_INT8, CODES_GEMM_OPERAND, CODES_GEMM_OPERAND_E4M3 = 0, 1, 2, 3
CODES_FP4_PACKED, CODES_FP4_OPERAND = 4, 5   # FP4 (E2M1) grid, bits = 4
MASK_BITS, MASK_BYTES = 0, 1
BF16, FP32 = 0, 1
_STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported", 3: "CUDA error", 4: "device wait timed out"}

# Every symbol the header declares, with (restype, argtypes).
_p, _i64, _int, _f32, _f64, _sz = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float,
                                   ctypes.c_double, ctypes.c_size_t)
SIGNATURES = {
    "quest_quantize_fwd": (_int, [_p, _int, _i64, _i64, _i64, _int, _int, _i64, _f32, _int, _p, _p,
                                  _int, _p, _p, _int, _p]),
    "quest_trust_bwd": (_int, [_p, _p, _int, _i64, _i64, _int, _p, _p]),
    "quest_quantize_operands": (_int, [_p, _i64, _p, _i64, _i64, _int, _int, _int, _int, _p, _p, _p, _p, _p]),
    "quest_w4a4_linear": (_int, [_p, _p, _p, _p, _i64, _i64, _i64, _p, _p, _p]),
    "quest_w4a4_linear_grouped": (_int, [_p, _p, _p, _p, _i64, _i64, _i64, _i64, _p, _p, _p]),
    "quest_trust_bwd_linear": (_int, [_p, _p, _p, _i64, _i64, _i64, _int, _p, _p]),
    "quest_transpose_bf16": (_int, [_p, _i64, _i64, _p, _p]),
    "quest_linear_bf16": (_int, [_p, _p, _i64, _i64, _i64, _p, _p]),
    "quest_fp4_linear": (_int, [_p, _p, _p, _p, _i64, _i64, _i64, _p, _p, _p]),
    "quest_device_status": (_int, [_p]),
    "quest_alpha": (_f64, [_int]),
    "quest_alpha_fp4": (_f64, []),
    "quest_container_bits": (_int, [_int]),
    "quest_codes_bytes": (_sz, [_i64, _i64, _int, _int]),
    "quest_mask_bytes": (_sz, [_i64, _i64, _int]),
    "quest_status_string": (ctypes.c_char_p, [_int]),
    "quest_last_error_message": (ctypes.c_char_p, []),
    "quest_version": (_int, []),
    "quest_debug_inject_fault": (_int, [_int]),
    "quest_quantize_sparse24": (_int, [_p, _i64, _i64, _int, _int, _i64, _f32, _p, _p, _p, _p, _p, _p]),
    "quest_alpha_sparse24": (_f64, [_int]),
    "quest_w4a4_linear_sparse24": (_int, [_p, _p, _p, _p, _p, _i64, _i64, _i64, _p, _p, _p]),
}

# The benchmark's tensor-core rate probes (include/quest_probe.h), in their own library.
_PROBE_LIB_NAME = "libquest_probe.so"
PROBE_SIGNATURES = {
    "quest_probe_mma_i8": (_int, [_int, _p, _p]),
    "quest_probe_mma_fp4": (_int, [_int, _p, _p]),
    "quest_probe_mma_bf16": (_int, [_int, _p, _p]),
    "quest_probe_mma_i8_pair": (_int, [_int, _p, _p]),
    "quest_probe_mma_sp_i8": (_int, [_int, _int, _p, _p]),
    "quest_probe_status": (_int, [_p]),
}

FAULT_NONE, FAULT_LAUNCH, FAULT_WAIT_TIMEOUT = 0, 1, 2   # include/quest_debug.h

_lock = threading.Lock()
_lib = None
_probe_lib = None


class QuestError(RuntimeError):
    """A quest_* call failed (or the library could not be loaded)."""

    def __init__(self, msg, status=None):
        super().__init__(msg)
        self.status = status


def library_path() -> str:
    return os.environ.get("QUEST_B200_LIB", os.path.join(_HERE, _LIB_NAME))


def load_library():
    """Load the library (once). Raises QuestError if it is not built."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        path = library_path()
        if not os.path.exists(path):
            raise QuestError(f"{path} not found: build it with "
                             "`python -m bit_quantization_aware_blockwise_b200.build`")
        try:
            lib = ctypes.CDLL(path)
        except OSError as e:
            raise QuestError(f"cannot load {path}: {e}") from e
        for name, (res, args) in SIGNATURES.items():
            f = getattr(lib, name)
            f.restype = res
            f.argtypes = args
        _lib = lib
        return lib


def load_probe_library():
    """Load the benchmark's probe library (once). Raises QuestError if it is not built."""
    global _probe_lib
    load_library()
    with _lock:
        if _probe_lib is not None:
            return _probe_lib
        path = os.path.join(os.path.dirname(library_path()), _PROBE_LIB_NAME)
        if not os.path.exists(path):
            raise QuestError(f"{path} not found: build it with "
                             "`python -m bit_quantization_aware_blockwise_b200.build`")
        try:
            lib = ctypes.CDLL(path)
        except OSError as e:
            raise QuestError(f"cannot load {path}: {e}") from e
        for name, (res, args) in PROBE_SIGNATURES.items():
            f = getattr(lib, name)
            f.restype = res
            f.argtypes = args
        _probe_lib = lib
        return lib


def _check(status: int, what: str):
    if status != 0:
        detail = load_library().quest_last_error_message().decode(errors="replace")
        raise QuestError(f"{what}: {_STATUS.get(status, status)}: {detail}", status)


# ---------------------------------------------------------------------------
# Raw entry points (integer device pointers and stream handle)
# ---------------------------------------------------------------------------

def quantize_fwd_raw(x, x_dtype, rows, cols, ld_x, bits, had_block, rms_group, trust, code_mode,
                     codes, scales, mask_mode, mask, dequant, dequant_dtype, stream=0):
    _check(load_library().quest_quantize_fwd(x, x_dtype, rows, cols, ld_x, bits, had_block,
                                             rms_group, trust, code_mode, codes, scales,
                                             mask_mode, mask, dequant, dequant_dtype, stream),
           "quest_quantize_fwd")


def quantize_operands_raw(x, M, w, N, K, dtype, bits, had_block, code_mode, x_codes, x_scales, w_codes,
                          w_scales, stream=0):
    _check(load_library().quest_quantize_operands(x, M, w, N, K, dtype, bits, had_block, code_mode, x_codes,
                                                  x_scales, w_codes, w_scales, stream), "quest_quantize_operands")


def trust_bwd_raw(grad_out, mask, mask_mode, rows, cols, had_block, grad_in, stream=0):
    _check(load_library().quest_trust_bwd(grad_out, mask, mask_mode, rows, cols, had_block,
                                          grad_in, stream), "quest_trust_bwd")


def w4a4_linear_raw(a_codes, a_scales, w_codes, w_scales, M, N, K, y, acc=None, stream=0):
    _check(load_library().quest_w4a4_linear(a_codes, a_scales, w_codes, w_scales, M, N, K, y, acc,
                                            stream), "quest_w4a4_linear")


def trust_bwd_linear_raw(grad_y, w_hat_t, mask, M, N, K, had_block, grad_x, stream=0):
    _check(load_library().quest_trust_bwd_linear(grad_y, w_hat_t, mask, M, N, K, had_block, grad_x, stream),
           "quest_trust_bwd_linear")


def linear_bf16_raw(x_hat, w_hat, M, N, K, y, stream=0):
    _check(load_library().quest_linear_bf16(x_hat, w_hat, M, N, K, y, stream), "quest_linear_bf16")


def fp4_linear_raw(a_codes, a_scales, w_codes, w_scales, M, N, K, y, acc=None, stream=0):
    _check(load_library().quest_fp4_linear(a_codes, a_scales, w_codes, w_scales, M, N, K, y, acc, stream),
           "quest_fp4_linear")


def transpose_bf16_raw(src, rows, cols, dst, stream=0):
    _check(load_library().quest_transpose_bf16(src, rows, cols, dst, stream), "quest_transpose_bf16")


def w4a4_linear_grouped_raw(a_codes, a_scales, w_codes, w_scales, M, N, K, group, y, y_f32=None, stream=0):
    _check(load_library().quest_w4a4_linear_grouped(a_codes, a_scales, w_codes, w_scales, M, N, K, group, y,
                                                    y_f32, stream), "quest_w4a4_linear_grouped")


def device_status(stream=0):
    """Synchronise ``stream`` and raise QuestError if a bounded device wait gave up."""
    _check(load_library().quest_device_status(stream), "quest_device_status")


def alpha(bits: int) -> float:
    return float(load_library().quest_alpha(bits))


def alpha_fp4() -> float:
    """s*, the Gaussian-MSE-optimal scale of the E2M1 grid (Delta = s* r)."""
    return float(load_library().quest_alpha_fp4())


def container_bits(bits: int) -> int:
    return int(load_library().quest_container_bits(bits))


def codes_bytes(rows: int, cols: int, bits: int, code_mode: int = CODES_PACKED) -> int:
    return int(load_library().quest_codes_bytes(rows, cols, bits, code_mode))


def mask_bytes(rows: int, cols: int, mask_mode: int = MASK_BITS) -> int:
    return int(load_library().quest_mask_bytes(rows, cols, mask_mode))


# ---------------------------------------------------------------------------
# torch-tensor wrappers (allocate outputs with torch, pass pointers)
# ---------------------------------------------------------------------------

def _torch():
    import torch
    return torch


def _stream_handle(stream, device):
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return s.cuda_stream


def _require_cuda(t, name):
    if not t.is_cuda:
        raise QuestError(f"{name} must be a CUDA tensor (there is no CPU path)")


def quantize_fwd(x, bits: int, had_block: int = 128, rms_group: int | None = None,
                 trust: float = 1.0, code_mode: int = CODES_PACKED, mask_mode: int | None = MASK_BITS,
                 dequant: str | None = None, out: dict | None = None, stream=None) -> dict:
    """Quantize the rows of a 2-D CUDA tensor ``x`` (bf16 or fp32, unit stride along
    columns). Returns ``{"codes", "scales", "mask", "dequant"}`` (mask/dequant None
    when not requested). ``rms_group`` defaults to ``had_block``; pass ``x.shape[1]``
    for one RMS per row. Outputs may be supplied in ``out`` to avoid allocation."""
    torch = _torch()
    _require_cuda(x, "x")
    if x.dim() != 2 or x.stride(1) != 1:
        raise QuestError("x must be 2-D with unit column stride")
    if x.dtype == torch.bfloat16:
        xd = BF16
    elif x.dtype == torch.float32:
        xd = FP32
    else:
        raise QuestError("x must be bfloat16 or float32")
    rows, cols = x.shape
    rms_group = had_block if rms_group is None else int(rms_group)
    out = {} if out is None else out
    dev = x.device
    codes = out.get("codes")
    if codes is None:
        codes = torch.empty(max(codes_bytes(rows, cols, bits, code_mode), 1), dtype=torch.uint8, device=dev)
    scales = out.get("scales")
    if scales is None:
        scales = torch.empty((rows, cols // rms_group if rms_group else 0), dtype=torch.float32, device=dev)
    mask = out.get("mask")
    if mask is None and mask_mode is not None:
        mask = torch.empty(max(mask_bytes(rows, cols, mask_mode), 1), dtype=torch.uint8, device=dev)
    deq = out.get("dequant")
    deq_dtype = BF16
    if dequant is not None:
        deq_dtype = BF16 if dequant == "bf16" else FP32
        if deq is None:
            deq = torch.empty((rows, cols), dtype=torch.bfloat16 if deq_dtype == BF16 else torch.float32,
                              device=dev)
    quantize_fwd_raw(x.data_ptr(), xd, rows, cols, x.stride(0) if rows > 1 else cols, bits,
                     had_block, rms_group, float(trust), code_mode, codes.data_ptr(),
                     scales.data_ptr(), MASK_BITS if mask_mode is None else mask_mode,
                     mask.data_ptr() if mask is not None else None,
                     deq.data_ptr() if deq is not None else None, deq_dtype,
                     _stream_handle(stream, dev))
    return {"codes": codes, "scales": scales, "mask": mask, "dequant": deq}


def quantize_sparse24_raw(x, rows, cols, bits, had_block, rms_group, trust, codes, meta, scales, mask=None,
                          dequant=None, stream=0):
    _check(load_library().quest_quantize_sparse24(x, rows, cols, bits, had_block, rms_group, trust, codes, meta,
                                                  scales, mask, dequant, stream), "quest_quantize_sparse24")


def quantize_sparse24(x, bits: int = 4, rms_group: int | None = None, trust: float = 1.0, mask: bool = True,
                      dequant: bool = False, stream=None) -> dict:
    """2:4-sparse quantizer of the rows of a dense bf16 CUDA tensor ``x`` (Hadamard block
    128). Returns ``{"codes": int8 [rows, cols/2], "meta": uint8 [rows, cols/8],
    "scales": fp32 [rows, cols/rms_group], "mask": uint32 [rows, cols/32] or None,
    "dequant": bf16 [rows, cols] or None}`` (see include/quest.h)."""
    torch = _torch()
    _require_cuda(x, "x")
    if x.dim() != 2 or x.dtype != torch.bfloat16 or not x.is_contiguous():
        raise QuestError("x must be a contiguous 2-D bf16 tensor")
    rows, cols = x.shape
    rg = 128 if rms_group is None else int(rms_group)
    dev = x.device
    codes = torch.empty((rows, cols // 2), dtype=torch.int8, device=dev)
    meta = torch.empty((rows, cols // 8), dtype=torch.uint8, device=dev)
    scales = torch.empty((rows, cols // rg if rg else 0), dtype=torch.float32, device=dev)
    m = torch.empty((rows, cols // 32), dtype=torch.int32, device=dev) if mask else None
    deq = torch.empty((rows, cols), dtype=torch.bfloat16, device=dev) if dequant else None
    quantize_sparse24_raw(x.data_ptr(), rows, cols, bits, 128, rg, trust, codes.data_ptr(), meta.data_ptr(),
                          scales.data_ptr(), m.data_ptr() if m is not None else None,
                          deq.data_ptr() if deq is not None else None, _stream_handle(stream, dev))
    return {"codes": codes, "meta": meta, "scales": scales, "mask": m, "dequant": deq}


def w4a4_linear_sparse24_raw(x_codes, x_scales, w_codes, w_meta, w_scales, M, N, K, y, acc=None, stream=0):
    _check(load_library().quest_w4a4_linear_sparse24(x_codes, x_scales, w_codes, w_meta, w_scales, M, N, K, y, acc,
                                                     stream), "quest_w4a4_linear_sparse24")


def w4a4_linear_sparse24(x_codes, x_scales, w_codes, w_meta, w_scales, out=None, acc: bool = False, stream=None):
    """y [M, N] bf16 = (x_codes @ w^T) * (x_scales/2)[:, None] * (w_scales/2)[None, :] with w the
    2:4-sparse weight codes given compressed (w_codes [N, K/2], w_meta [N, K/8]). Returns y, or
    (y, acc int32) with ``acc=True``."""
    torch = _torch()
    for t, name in ((x_codes, "x_codes"), (w_codes, "w_codes"), (w_meta, "w_meta"), (x_scales, "x_scales"),
                    (w_scales, "w_scales")):
        _require_cuda(t, name)
        if not t.is_contiguous():
            raise QuestError(f"{name} must be contiguous")
    M, K = x_codes.shape
    N = w_codes.shape[0]
    if w_codes.shape[1] * 2 != K or w_meta.shape != (N, K // 8):
        raise QuestError("w_codes must be [N, K/2] and w_meta [N, K/8]")
    dev = x_codes.device
    y = out if out is not None else torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    a = torch.empty((M, N), dtype=torch.int32, device=dev) if acc else None
    w4a4_linear_sparse24_raw(x_codes.data_ptr(), x_scales.data_ptr(), w_codes.data_ptr(), w_meta.data_ptr(),
                             w_scales.data_ptr(), M, N, K, y.data_ptr(), a.data_ptr() if a is not None else None,
                             _stream_handle(stream, dev))
    return (y, a) if acc else y


def alpha_sparse24(bits: int) -> float:
    return float(load_library().quest_alpha_sparse24(bits))


def quantize_operands(x, w, bits: int = 4, had_block: int = 128, code_mode: int = CODES_GEMM_OPERAND,
                      stream=None):
    """Operand codes of a linear layer, one RMS per row: x [M, K] and w [N, K] (same dtype,
    contiguous) in one call. Returns ({"codes", "scales"} for x, the same for w)."""
    torch = _torch()
    _require_cuda(x, "x")
    _require_cuda(w, "w")
    if x.dim() != 2 or w.dim() != 2 or x.shape[1] != w.shape[1] or x.dtype != w.dtype:
        raise QuestError("x [M, K] and w [N, K] of one dtype expected")
    if not (x.is_contiguous() and w.is_contiguous()):
        raise QuestError("x and w must be contiguous")
    if x.dtype == torch.bfloat16:
        dt = BF16
    elif x.dtype == torch.float32:
        dt = FP32
    else:
        raise QuestError("x and w must be bfloat16 or float32")
    (M, K), N = x.shape, w.shape[0]
    dev = x.device
    cx = torch.empty(max(codes_bytes(M, K, bits, code_mode), 1), dtype=torch.uint8, device=dev)
    cw = torch.empty(max(codes_bytes(N, K, bits, code_mode), 1), dtype=torch.uint8, device=dev)
    sx = torch.empty(max(M, 1), dtype=torch.float32, device=dev)
    sw = torch.empty(max(N, 1), dtype=torch.float32, device=dev)
    quantize_operands_raw(x.data_ptr(), M, w.data_ptr(), N, K, dt, bits, had_block, code_mode, cx.data_ptr(),
                          sx.data_ptr(), cw.data_ptr(), sw.data_ptr(), _stream_handle(stream, dev))
    return {"codes": cx, "scales": sx[:M]}, {"codes": cw, "scales": sw[:N]}


def trust_bwd(grad_out, mask, had_block: int = 128, mask_mode: int = MASK_BITS, out=None,
              stream=None):
    """grad_in = H (m * grad_out) / sqrt(n) per block; bf16 in and out."""
    torch = _torch()
    _require_cuda(grad_out, "grad_out")
    _require_cuda(mask, "mask")
    if grad_out.dtype != torch.bfloat16 or grad_out.dim() != 2 or not grad_out.is_contiguous():
        raise QuestError("grad_out must be a contiguous 2-D bfloat16 tensor")
    rows, cols = grad_out.shape
    if out is None:
        out = torch.empty_like(grad_out)
    trust_bwd_raw(grad_out.data_ptr(), mask.data_ptr(), mask_mode, rows, cols, had_block,
                  out.data_ptr(), _stream_handle(stream, grad_out.device))
    return out


def trust_bwd_linear(grad_y, w_hat_t, mask, had_block: int = 128, out=None, stream=None):
    """grad_x = H (m * (grad_y @ w_hat_t^T)) / sqrt(128) per 128-column block: the input
    gradient of a quantized linear layer. grad_y bf16 [M, N], w_hat_t bf16 [K, N] (the
    dequantised weight, transposed), mask = the input's trust mask bits [M, K/8]."""
    torch = _torch()
    for t, n in ((grad_y, "grad_y"), (w_hat_t, "w_hat_t"), (mask, "mask")):
        _require_cuda(t, n)
    if grad_y.dtype != torch.bfloat16 or w_hat_t.dtype != torch.bfloat16:
        raise QuestError("grad_y and w_hat_t must be bfloat16")
    if grad_y.dim() != 2 or w_hat_t.dim() != 2 or not (grad_y.is_contiguous() and w_hat_t.is_contiguous()):
        raise QuestError("grad_y and w_hat_t must be contiguous 2-D tensors")
    M, N = grad_y.shape
    K = w_hat_t.shape[0]
    if w_hat_t.shape[1] != N:
        raise QuestError("w_hat_t must be [K, N] with grad_y [M, N]")
    if out is None:
        out = torch.empty((M, K), dtype=torch.bfloat16, device=grad_y.device)
    trust_bwd_linear_raw(grad_y.data_ptr(), w_hat_t.data_ptr(), mask.data_ptr(), M, N, K, had_block,
                         out.data_ptr(), _stream_handle(stream, grad_y.device))
    return out


def linear_bf16(x_hat, w_hat, out=None, stream=None):
    """y = x_hat @ w_hat^T on bf16 operands [M, K] and [N, K] (fp32 accumulation, bf16 out)."""
    torch = _torch()
    _require_cuda(x_hat, "x_hat")
    _require_cuda(w_hat, "w_hat")
    if x_hat.dtype != torch.bfloat16 or w_hat.dtype != torch.bfloat16:
        raise QuestError("x_hat and w_hat must be bfloat16")
    if x_hat.dim() != 2 or w_hat.dim() != 2 or x_hat.shape[1] != w_hat.shape[1]:
        raise QuestError("x_hat [M, K] and w_hat [N, K] expected")
    if not (x_hat.is_contiguous() and w_hat.is_contiguous()):
        raise QuestError("x_hat and w_hat must be contiguous")
    (M, K), N = x_hat.shape, w_hat.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=x_hat.device)
    linear_bf16_raw(x_hat.data_ptr(), w_hat.data_ptr(), M, N, K, out.data_ptr(), _stream_handle(stream, x_hat.device))
    return out


def transpose_bf16(src, out=None, stream=None):
    """[rows, cols] bf16 -> [cols, rows] (a library kernel)."""
    torch = _torch()
    _require_cuda(src, "src")
    if src.dtype != torch.bfloat16 or src.dim() != 2 or not src.is_contiguous():
        raise QuestError("src must be a contiguous 2-D bfloat16 tensor")
    rows, cols = src.shape
    if out is None:
        out = torch.empty((cols, rows), dtype=torch.bfloat16, device=src.device)
    transpose_bf16_raw(src.data_ptr(), rows, cols, out.data_ptr(), _stream_handle(stream, src.device))
    return out


def w4a4_linear(a_codes, a_scales, w_codes, w_scales, out=None, acc: bool = False, stream=None):
    """y = bf16((a_codes @ w_codes^T) * (a_scales/2)[:, None] * (w_scales/2)[None, :]).
    Codes are int8 [M, K] and [N, K]; returns y (and the int32 accumulator if acc)."""
    torch = _torch()
    for t, n in ((a_codes, "a_codes"), (w_codes, "w_codes"), (a_scales, "a_scales"), (w_scales, "w_scales")):
        _require_cuda(t, n)
    if a_codes.dtype not in (torch.int8, torch.uint8) or w_codes.dtype not in (torch.int8, torch.uint8):
        raise QuestError("codes must be int8")
    if not (a_codes.is_contiguous() and w_codes.is_contiguous()):
        raise QuestError("codes must be contiguous")
    M, K = a_codes.shape
    N, K2 = w_codes.shape
    if K != K2:
        raise QuestError("a_codes and w_codes disagree on K")
    dev = a_codes.device
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    acc_t = torch.empty((M, N), dtype=torch.int32, device=dev) if acc else None
    w4a4_linear_raw(a_codes.data_ptr(), a_scales.data_ptr(), w_codes.data_ptr(), w_scales.data_ptr(),
                    M, N, K, out.data_ptr(), acc_t.data_ptr() if acc_t is not None else None,
                    _stream_handle(stream, dev))
    return (out, acc_t) if acc else out


def fp4_linear(a_codes, a_scales, w_codes, w_scales, K: int, out=None, acc: bool = False, stream=None):
    """y = bf16((Q_a @ Q_w^T) * a_scales[:, None] * w_scales[None, :]) on packed E2M1 codes
    (uint8 [M, K/2] and [N, K/2], the CODES_FP4_PACKED form with one scale per row).
    Returns y (and the fp32 accumulator sum_k Q_a Q_w if acc)."""
    torch = _torch()
    for t, n in ((a_codes, "a_codes"), (w_codes, "w_codes"), (a_scales, "a_scales"), (w_scales, "w_scales")):
        _require_cuda(t, n)
    if a_codes.dtype not in (torch.int8, torch.uint8) or w_codes.dtype not in (torch.int8, torch.uint8):
        raise QuestError("packed codes must be uint8")
    if not (a_codes.is_contiguous() and w_codes.is_contiguous()):
        raise QuestError("codes must be contiguous")
    M, N = a_scales.numel(), w_scales.numel()   # one scale per row
    if a_codes.numel() < M * (K // 2) or w_codes.numel() < N * (K // 2):
        raise QuestError("codes must hold K/2 bytes per row")
    dev = a_codes.device
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    acc_t = torch.empty((M, N), dtype=torch.float32, device=dev) if acc else None
    fp4_linear_raw(a_codes.data_ptr(), a_scales.data_ptr(), w_codes.data_ptr(), w_scales.data_ptr(), M, N, K,
                   out.data_ptr(), acc_t.data_ptr() if acc_t is not None else None, _stream_handle(stream, dev))
    return (out, acc_t) if acc else out


def w4a4_linear_grouped(a_codes, a_scales, w_codes, w_scales, out=None, y_f32: bool = False,
                        group: int = 128, stream=None):
    """y = bf16(sum_g (a_scales[:, g]/2)(w_scales[:, g]/2) * (A_g @ W_g^T)), A_g / W_g the
    codes of K-group g. Codes are FP8 E4M3 bytes [M, K] / [N, K] (float8_e4m3fn or uint8:
    the CODES_GEMM_OPERAND_E4M3 form); scales fp32 [M, K/group] / [N, K/group].
    Returns y (and the fp32 result before rounding if y_f32)."""
    torch = _torch()
    for t, n in ((a_codes, "a_codes"), (w_codes, "w_codes"), (a_scales, "a_scales"), (w_scales, "w_scales")):
        _require_cuda(t, n)
    ok = (torch.uint8, torch.float8_e4m3fn)
    if a_codes.dtype not in ok or w_codes.dtype not in ok:
        raise QuestError("codes must be FP8 E4M3 (float8_e4m3fn or uint8 bytes)")
    if not (a_codes.is_contiguous() and w_codes.is_contiguous() and a_scales.is_contiguous()
            and w_scales.is_contiguous()):
        raise QuestError("codes and scales must be contiguous")
    M, K = a_codes.shape
    N, K2 = w_codes.shape
    if K != K2:
        raise QuestError("a_codes and w_codes disagree on K")
    if group <= 0 or K % group != 0 or a_scales.numel() != M * (K // group) or w_scales.numel() != N * (K // group):
        raise QuestError("scales must be [M, K/group] and [N, K/group]")
    dev = a_codes.device
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    y32 = torch.empty((M, N), dtype=torch.float32, device=dev) if y_f32 else None
    w4a4_linear_grouped_raw(a_codes.data_ptr(), a_scales.data_ptr(), w_codes.data_ptr(), w_scales.data_ptr(),
                            M, N, K, group, out.data_ptr(), y32.data_ptr() if y32 is not None else None,
                            _stream_handle(stream, dev))
    return (out, y32) if y_f32 else out


def _check_probe(status: int, what: str):
    if status != 0:
        raise QuestError(f"{what}: {_STATUS.get(status, status)}", status)


def probe_mma_i8(iters, stream=0):
    """Enqueue the int8 tensor-core peak probe; returns the number of CTAs launched."""
    ctas = ctypes.c_int(0)
    _check_probe(load_probe_library().quest_probe_mma_i8(iters, ctypes.byref(ctas), stream), "quest_probe_mma_i8")
    return ctas.value


def probe_mma_fp4(iters, stream=0):
    """Enqueue the FP4 (kind::mxf4) tensor-core peak probe; returns the number of CTAs launched."""
    ctas = ctypes.c_int(0)
    _check_probe(load_probe_library().quest_probe_mma_fp4(iters, ctypes.byref(ctas), stream), "quest_probe_mma_fp4")
    return ctas.value


def probe_mma_i8_pair(iters, stream=0):
    """Enqueue the CTA-pair int8 probe (cta_group::2, M = 256); returns the number of CTAs."""
    ctas = ctypes.c_int(0)
    _check_probe(load_probe_library().quest_probe_mma_i8_pair(iters, ctypes.byref(ctas), stream),
                 "quest_probe_mma_i8_pair")
    return ctas.value


def probe_mma_bf16(iters, stream=0):
    """Enqueue the bf16 (kind::f16) tensor-core probe; returns the number of CTAs launched."""
    ctas = ctypes.c_int(0)
    _check_probe(load_probe_library().quest_probe_mma_bf16(iters, ctypes.byref(ctas), stream), "quest_probe_mma_bf16")
    return ctas.value


def probe_mma_sp_i8(iters, cp_every=0, stream=0):
    """Enqueue the 2:4-sparse int8 tensor-core probe (metadata copied every `cp_every` MMAs,
    0 = resident); returns the number of CTAs launched."""
    ctas = ctypes.c_int(0)
    _check_probe(load_probe_library().quest_probe_mma_sp_i8(iters, cp_every, ctypes.byref(ctas), stream),
                 "quest_probe_mma_sp_i8")
    return ctas.value


def probe_status(stream=0):
    _check_probe(load_probe_library().quest_probe_status(stream), "quest_probe_status")


def debug_inject_fault(fault):
    """Arm a fault for the next launching call on this thread (include/quest_debug.h)."""
    _check(load_library().quest_debug_inject_fault(fault), "quest_debug_inject_fault")

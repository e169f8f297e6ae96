"""QuEST oracle: plain fp64 CPU reference of the quantizer, trust backward and
integer linear layer (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. The product library never does, and
this package imports nothing from the product.

The arithmetic lives in ``quest_oracle.c`` (plain C, built with gcc on first
use); this module only marshals numpy arrays. See the C file's header for the
passages of the QuEST pages each step follows and the readings taken where the
pages are silent.

Parity status: every function here is pinned by ``tests/test_oracle_pins.py``
against closed forms, library routines (scipy's Hadamard construction, numerical
quadrature, numpy integer matmul, torch's bfloat16 conversion) and brute force.
Agreement with the authors' own numerics (their RMS granularity, grid
parametrisation and Hadamard ordering) cannot be pinned: the pages print no
intermediate values.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "quest_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "libquest_oracle.so")
_lock = threading.Lock()
_lib = None

_p = ctypes.c_void_p
_i64 = ctypes.c_int64
_int = ctypes.c_int
_dbl = ctypes.c_double


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no fast-math) into ``oracle/_build``."""
    os.makedirs(_BUILD_DIR, exist_ok=True)
    stale = (not os.path.exists(_LIB_PATH)) or (
        os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)
    )
    if force or stale:
        tmp = _LIB_PATH + f".{os.getpid()}.tmp"
        cmd = ["gcc", "-O2", "-std=c11", "-D_GNU_SOURCE", "-fPIC", "-shared",
               "-fno-fast-math", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        lib = ctypes.CDLL(build())
        lib.oracle_hadamard.argtypes = [_int, _p]
        lib.oracle_hadamard.restype = _int
        lib.oracle_gauss_mse.argtypes = [_int, _dbl]
        lib.oracle_gauss_mse.restype = _dbl
        lib.oracle_alpha.argtypes = [_int, _p, _p, _p]
        lib.oracle_alpha.restype = _int
        lib.oracle_quantize.argtypes = [_p, _i64, _i64, _i64, _int, _i64, _int, _dbl, _dbl,
                                        _p, _p, _p, _p, _p, _p, _p, _p]
        lib.oracle_quantize.restype = _int
        lib.oracle_e2m1_value.argtypes = [_int]
        lib.oracle_e2m1_value.restype = _dbl
        lib.oracle_e2m1_round.argtypes = [_dbl]
        lib.oracle_e2m1_round.restype = _int
        lib.oracle_fp4_gauss_mse.argtypes = [_dbl]
        lib.oracle_fp4_gauss_mse.restype = _dbl
        lib.oracle_fp4_scale.argtypes = [_p, _p]
        lib.oracle_fp4_scale.restype = _int
        lib.oracle_quantize_fp4.argtypes = [_p, _i64, _i64, _i64, _int, _i64, _dbl, _dbl,
                                            _p, _p, _p, _p, _p, _p, _p, _p, _p]
        lib.oracle_quantize_fp4.restype = _int
        lib.oracle_sparse24_mse.argtypes = [_int, _dbl]
        lib.oracle_sparse24_mse.restype = _dbl
        lib.oracle_sparse24_alpha.argtypes = [_int, _p, _p, _p]
        lib.oracle_sparse24_alpha.restype = _int
        lib.oracle_quantize_sparse24.argtypes = [_p, _i64, _i64, _i64, _int, _i64, _int, _dbl, _dbl,
                                                 _p, _p, _p, _p, _p, _p, _p, _p, _p, _p]
        lib.oracle_quantize_sparse24.restype = _int
        lib.oracle_trust_bwd.argtypes = [_p, _p, _i64, _i64, _int, _p]
        lib.oracle_trust_bwd.restype = _int
        lib.oracle_gemm_i8.argtypes = [_p, _p, _i64, _i64, _i64, _p]
        lib.oracle_gemm_i8.restype = _int
        lib.oracle_dequant_linear.argtypes = [_p, _p, _p, _i64, _i64, _p]
        lib.oracle_dequant_linear.restype = _int
        lib.oracle_linear_grouped.argtypes = [_p, _p, _p, _p, _i64, _i64, _i64, _i64, _p, _p]
        lib.oracle_linear_grouped.restype = _int
        lib.oracle_bf16_rne.argtypes = [_dbl]
        lib.oracle_bf16_rne.restype = ctypes.c_uint16
        lib.oracle_bf16_rne_array.argtypes = [_p, _i64, _p]
        lib.oracle_bf16_rne_array.restype = None
        _lib = lib
        return lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _check(rc, what):
    if rc != 0:
        raise ValueError(f"oracle {what}: invalid arguments (rc={rc})")


def hadamard(n: int) -> np.ndarray:
    """Unnormalised Sylvester Hadamard matrix, H[i, j] = (-1)^popcount(i & j)."""
    H = np.empty((n, n), dtype=np.float64)
    _check(_load().oracle_hadamard(n, _ptr(H)), "hadamard")
    return H


def gauss_mse(bits: int, delta: float) -> float:
    """E[(X - Q(X))^2] for X ~ N(0,1) and the 2^bits-level midrise grid of step delta."""
    return float(_load().oracle_gauss_mse(bits, delta))


def alpha(bits: int):
    """(alpha_b, optimal step Delta*, minimal Gaussian MSE) for ``bits``."""
    a, d, m = _dbl(), _dbl(), _dbl()
    _check(_load().oracle_alpha(bits, ctypes.byref(a), ctypes.byref(d), ctypes.byref(m)), "alpha")
    return a.value, d.value, m.value


def quantize(x, bits: int, had: int = 128, rms_group: int | None = None, trust: float = 1.0):
    """Quantize rows of ``x`` (any real array of shape [rows, cols]; converted to fp64
    exactly for bf16/fp32 inputs). Returns a dict of numpy arrays:
    y, t, q, yhat, mask, scale, d_round, d_mask (see ``quest_oracle.c``)."""
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float64))
    if x.ndim != 2:
        raise ValueError("x must be 2-D")
    rows, cols = x.shape
    rms_group = had if rms_group is None else int(rms_group)
    a, _, _ = alpha(bits)
    out = {
        "y": np.empty((rows, cols)), "t": np.empty((rows, cols)),
        "q": np.empty((rows, cols), dtype=np.int32), "yhat": np.empty((rows, cols)),
        "mask": np.empty((rows, cols), dtype=np.uint8),
        "scale": np.empty((rows, cols // rms_group if rms_group else 0)),
        "d_round": np.empty((rows, cols)), "d_mask": np.empty((rows, cols)),
    }
    rc = _load().oracle_quantize(
        _ptr(x), rows, cols, cols, had, rms_group, bits, float(trust), a,
        _ptr(out["y"]), _ptr(out["t"]), _ptr(out["q"]), _ptr(out["yhat"]),
        _ptr(out["mask"]), _ptr(out["scale"]), _ptr(out["d_round"]), _ptr(out["d_mask"]))
    _check(rc, "quantize")
    return out


def e2m1_value(code: int) -> float:
    """Value of a 4-bit E2M1 code (bit 3 sign, 2 exponent bits with bias 1, 1 mantissa bit)."""
    return float(_load().oracle_e2m1_value(int(code)))


def e2m1_round(t: float) -> int:
    """E2M1 code nearest to t (ties to the even mantissa, saturating at +-6, sign of t kept)."""
    return int(_load().oracle_e2m1_round(float(t)))


def fp4_gauss_mse(s: float) -> float:
    """E[(X - s Q(X/s))^2] for X ~ N(0,1), Q round-to-nearest onto the E2M1 grid."""
    return float(_load().oracle_fp4_gauss_mse(float(s)))


def alpha_fp4():
    """(s*, minimal Gaussian MSE): the scale of the E2M1 grid that minimises the MSE."""
    s, m = _dbl(), _dbl()
    _check(_load().oracle_fp4_scale(ctypes.byref(s), ctypes.byref(m)), "fp4_scale")
    return s.value, m.value


def quantize_fp4(x, had: int = 128, rms_group: int | None = None, trust: float = 1.0):
    """FP4 (E2M1) grid quantizer of the rows of ``x``. Returns a dict of numpy arrays:
    y, t, code (4-bit E2M1), value (grid value Q), yhat, mask, scale, d_round, d_mask."""
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float64))
    if x.ndim != 2:
        raise ValueError("x must be 2-D")
    rows, cols = x.shape
    rms_group = had if rms_group is None else int(rms_group)
    s, _ = alpha_fp4()
    out = {
        "y": np.empty((rows, cols)), "t": np.empty((rows, cols)),
        "code": np.empty((rows, cols), dtype=np.uint8), "value": np.empty((rows, cols)),
        "yhat": np.empty((rows, cols)), "mask": np.empty((rows, cols), dtype=np.uint8),
        "scale": np.empty((rows, cols // rms_group if rms_group else 0)),
        "d_round": np.empty((rows, cols)), "d_mask": np.empty((rows, cols)),
    }
    rc = _load().oracle_quantize_fp4(
        _ptr(x), rows, cols, cols, had, rms_group, float(trust), s,
        _ptr(out["y"]), _ptr(out["t"]), _ptr(out["code"]), _ptr(out["value"]), _ptr(out["yhat"]),
        _ptr(out["mask"]), _ptr(out["scale"]), _ptr(out["d_round"]), _ptr(out["d_mask"]))
    _check(rc, "quantize_fp4")
    return out


def sparse24_mse(bits: int, delta: float) -> float:
    """E[(X - Q(X))^2 | X kept] for the 2:4-sparse format: of four iid N(0,1) values the
    two of largest magnitude are kept; Q the 2^bits-level midrise grid of step delta."""
    return float(_load().oracle_sparse24_mse(bits, delta))


_sparse_alpha_cache = {}


def alpha_sparse24(bits: int):
    """(alpha_b, optimal step, minimal MSE of the kept values) of the 2:4-sparse format."""
    if bits not in _sparse_alpha_cache:
        a, d, m = _dbl(), _dbl(), _dbl()
        _check(_load().oracle_sparse24_alpha(bits, ctypes.byref(a), ctypes.byref(d), ctypes.byref(m)),
               "sparse24_alpha")
        _sparse_alpha_cache[bits] = (a.value, d.value, m.value)
    return _sparse_alpha_cache[bits]


def quantize_sparse24(x, bits: int, had: int = 128, rms_group: int | None = None, trust: float = 1.0):
    """2:4-sparse quantizer of the rows of ``x`` (see ``quest_oracle.c``). Returns a dict of
    numpy arrays: y, t, q (0 where pruned), kept (1 = survives), yhat, mask, scale, d_round,
    d_mask, d_prune."""
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float64))
    if x.ndim != 2:
        raise ValueError("x must be 2-D")
    rows, cols = x.shape
    rms_group = had if rms_group is None else int(rms_group)
    a, _, _ = alpha_sparse24(bits)
    out = {
        "y": np.empty((rows, cols)), "t": np.empty((rows, cols)),
        "q": np.empty((rows, cols), dtype=np.int32), "kept": np.empty((rows, cols), dtype=np.uint8),
        "yhat": np.empty((rows, cols)), "mask": np.empty((rows, cols), dtype=np.uint8),
        "scale": np.empty((rows, cols // rms_group if rms_group else 0)),
        "d_round": np.empty((rows, cols)), "d_mask": np.empty((rows, cols)), "d_prune": np.empty((rows, cols)),
    }
    rc = _load().oracle_quantize_sparse24(
        _ptr(x), rows, cols, cols, had, rms_group, bits, float(trust), a,
        _ptr(out["y"]), _ptr(out["t"]), _ptr(out["q"]), _ptr(out["kept"]), _ptr(out["yhat"]),
        _ptr(out["mask"]), _ptr(out["scale"]), _ptr(out["d_round"]), _ptr(out["d_mask"]), _ptr(out["d_prune"]))
    _check(rc, "quantize_sparse24")
    return out


def trust_bwd(g, mask, had: int = 128) -> np.ndarray:
    """g_x = H^T (m * g) / sqrt(had) per block, fp64."""
    g = np.ascontiguousarray(np.asarray(g, dtype=np.float64))
    m = np.ascontiguousarray(np.asarray(mask, dtype=np.uint8))
    if g.shape != m.shape or g.ndim != 2:
        raise ValueError("g and mask must have the same 2-D shape")
    out = np.empty_like(g)
    _check(_load().oracle_trust_bwd(_ptr(g), _ptr(m), g.shape[0], g.shape[1], had, _ptr(out)),
           "trust_bwd")
    return out


def trust_bwd_linear(g_y, w_hat, mask, had: int = 128) -> np.ndarray:
    """Input gradient of a linear layer y = x_hat w_hat^T whose quantized input carried
    trust mask m (pith.science review, "What carries the argument" and Figure 2
    caption: the gradient is masked in the Hadamard domain, then transformed back):
        G   = g_y @ w_hat            [rows, K]  (fp64; numpy's matmul)
        g_x = H^T (m * G) / sqrt(had) per block (``trust_bwd``)
    g_y [rows, N], w_hat [N, K] (the dequantised weights, Hadamard domain), mask [rows, K]."""
    g_y = np.asarray(g_y, dtype=np.float64)
    w_hat = np.asarray(w_hat, dtype=np.float64)
    if g_y.ndim != 2 or w_hat.ndim != 2 or g_y.shape[1] != w_hat.shape[0]:
        raise ValueError("g_y [rows, N] and w_hat [N, K] expected")
    return trust_bwd(g_y @ w_hat, mask, had)


def linear_bf16(x_hat, w_hat) -> np.ndarray:
    """y = x_hat @ w_hat^T in fp64 (numpy's matmul): the linear layer on dequantised
    operands in the Hadamard domain (pith.science review, "Assumptions & free
    parameters": the transform applied to both operands leaves the product unchanged).
    x_hat [M, K], w_hat [N, K]; bf16 inputs are exact in fp64."""
    x_hat = np.asarray(x_hat, dtype=np.float64)
    w_hat = np.asarray(w_hat, dtype=np.float64)
    if x_hat.ndim != 2 or w_hat.ndim != 2 or x_hat.shape[1] != w_hat.shape[1]:
        raise ValueError("x_hat [M, K] and w_hat [N, K] expected")
    return x_hat @ w_hat.T


def gemm_i8(a, b) -> np.ndarray:
    """acc = A @ B^T in int64 by a triple loop; A [M,K], B [N,K] int8."""
    a = np.ascontiguousarray(np.asarray(a, dtype=np.int8))
    b = np.ascontiguousarray(np.asarray(b, dtype=np.int8))
    if a.ndim != 2 or b.ndim != 2 or a.shape[1] != b.shape[1]:
        raise ValueError("A [M,K] and B [N,K] expected")
    acc = np.empty((a.shape[0], b.shape[0]), dtype=np.int64)
    _check(_load().oracle_gemm_i8(_ptr(a), _ptr(b), a.shape[0], b.shape[0], a.shape[1], _ptr(acc)),
           "gemm_i8")
    return acc


def dequant_linear(acc, delta_a, delta_b) -> np.ndarray:
    """Y = acc * (Delta_a/2)[:, None] * (Delta_b/2)[None, :] in fp64."""
    acc = np.ascontiguousarray(np.asarray(acc, dtype=np.int64))
    da = np.ascontiguousarray(np.asarray(delta_a, dtype=np.float64))
    db = np.ascontiguousarray(np.asarray(delta_b, dtype=np.float64))
    y = np.empty(acc.shape, dtype=np.float64)
    _check(_load().oracle_dequant_linear(_ptr(acc), _ptr(da), _ptr(db), acc.shape[0],
                                         acc.shape[1], _ptr(y)), "dequant_linear")
    return y


def linear_grouped(a, b, delta_a, delta_b, group: int = 128):
    """Y = sum_g (Delta_a[:, g]/2)(Delta_b[:, g]/2) * (A_g @ B_g^T) in fp64, with A_g the
    int8 codes of K-group g; returns (Y, sum_g |term_g|)."""
    a = np.ascontiguousarray(np.asarray(a, dtype=np.int8))
    b = np.ascontiguousarray(np.asarray(b, dtype=np.int8))
    da = np.ascontiguousarray(np.asarray(delta_a, dtype=np.float64))
    db = np.ascontiguousarray(np.asarray(delta_b, dtype=np.float64))
    M, K = a.shape
    N = b.shape[0]
    assert b.shape[1] == K and da.shape == (M, K // group) and db.shape == (N, K // group)
    y = np.empty((M, N), dtype=np.float64)
    mag = np.empty((M, N), dtype=np.float64)
    _check(_load().oracle_linear_grouped(_ptr(a), _ptr(b), _ptr(da), _ptr(db), M, N, K, group,
                                         _ptr(y), _ptr(mag)), "linear_grouped")
    return y, mag


def bf16_rne(v) -> np.ndarray:
    """Round fp64 values to bfloat16 (nearest-even, one rounding); returns uint16 bits."""
    v = np.ascontiguousarray(np.asarray(v, dtype=np.float64))
    out = np.empty(v.shape, dtype=np.uint16)
    _load().oracle_bf16_rne_array(_ptr(v), v.size, _ptr(out))
    return out


def bf16_bits_to_f64(bits) -> np.ndarray:
    """Exact value of bfloat16 bit patterns as fp64."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)

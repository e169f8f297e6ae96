"""Comparison rules between the CUDA library's outputs and the oracle.

Integer outputs (codes, masks, accumulators) must match bit for bit, except a
code or mask bit whose pre-round value t lies within 1e-5 * max(|t|, 1) of its
decision boundary (the two sides compute t in different precision: fp32 on the
GPU, fp64 in the oracle). Floating outputs are compared with the oracle's fp64
value: bf16 outputs must equal its round-to-nearest-even bf16 value or be within
one bf16 ulp of it, or within 2e-3 relative (with a floor for values that cancel).
"""
import numpy as np

import oracle

EXEMPT_REL = 1e-5
FLOAT_REL = 2e-3


def e4m3_decode(raw):
    """Value of OCP FP8 E4M3 bytes by the format's definition: sign, 4-bit exponent
    with bias 7 (0 = subnormal), 3-bit mantissa; 0x7F / 0xFF are NaN."""
    b = np.asarray(raw, dtype=np.uint8).astype(np.int64)
    sign = np.where(b >> 7, -1.0, 1.0)
    e = (b >> 3) & 15
    m = (b & 7).astype(np.float64)
    v = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    v = np.where((e == 15) & ((b & 7) == 7), np.nan, v)
    return sign * v


def e4m3_encode_int(c):
    """E4M3 bytes of integers exactly representable in the format (|c| <= 15 here)."""
    c = np.asarray(c, dtype=np.int64)
    a = np.abs(c)
    assert np.all(a <= 15)
    e = np.where(a > 0, np.floor(np.log2(np.maximum(a, 1))).astype(np.int64), 0)
    m = np.where(a > 0, (a * 8) // (1 << e) - 8, 0)
    byte = np.where(a > 0, ((e + 7) << 3) | m, 0) | np.where(c < 0, 0x80, 0)
    return byte.astype(np.uint8)


def unpack_codes(raw, rows, cols, bits, mode):
    """Decode the library's code buffer into int codes [rows, cols] (q, or c=2q+1 for
    the GEMM operand forms)."""
    raw = np.asarray(raw, dtype=np.uint8).reshape(-1)
    if mode == 3:  # E4M3 operand form
        v = e4m3_decode(raw[: rows * cols]).reshape(rows, cols)
        assert np.all(v == np.round(v)), "E4M3 operand codes must be integers"
        return v.astype(np.int32)
    if mode in (1, 2):  # int8 forms
        return raw[: rows * cols].view(np.int8).reshape(rows, cols).astype(np.int32)
    cb = [0, 1, 2, 4, 4, 8, 8, 8, 8][bits]
    if cb == 8:
        return raw[: rows * cols].view(np.int8).reshape(rows, cols).astype(np.int32)
    per = 8 // cb
    by = raw[: rows * cols // per].reshape(rows, cols // per).astype(np.int32)
    fields = np.stack([(by >> (cb * i)) & ((1 << cb) - 1) for i in range(per)], axis=-1)
    fields = fields.reshape(rows, cols)
    sign = 1 << (cb - 1)
    return np.where(fields >= sign, fields - (1 << cb), fields)


def unpack_mask_bits(raw, rows, cols):
    by = np.asarray(raw, dtype=np.uint8).reshape(-1)[: rows * cols // 8].reshape(rows, cols // 8)
    return np.unpackbits(by, axis=1, bitorder="little")[:, :cols]


def exempt_codes(o):
    return o["d_round"] <= EXEMPT_REL * np.maximum(np.abs(o["t"]), 1.0)


def exempt_mask(o):
    return o["d_mask"] <= EXEMPT_REL * np.maximum(np.abs(o["t"]), 1.0)


def check_codes(q_gpu, o, what="codes"):
    """Exact outside the exemption band; within one step inside it."""
    ex = exempt_codes(o)
    bad = (q_gpu != o["q"]) & ~ex
    assert not bad.any(), f"{what}: {int(bad.sum())} non-exempt mismatches, first at {np.argwhere(bad)[:5].tolist()}"
    assert np.all(np.abs(q_gpu - o["q"])[ex] <= 1)
    return int(ex.sum())


def check_codes_operand(c_gpu, o):
    return check_codes((c_gpu - 1) // 2, o, "operand codes")


# Exempt mask bits allowed, as a fraction of the elements (plus one). The band is
# 2e-5 max(|t|, 1) wide around each flip point of the mask. With T >= 1 the mask
# flips only at the two outer edges, beyond the clip, so the band holds next to
# nothing; with T < 1 every unit of t has two flip points and the band holds about
# 4e-5 E[max(|t|, 1)] of the elements (~1e-4 at b = 4), hence the wider default there.
MASK_EXEMPT_FRAC = 1e-4
MASK_EXEMPT_FRAC_TRUST_BELOW_1 = 5e-4


def check_mask(m_gpu, o, max_frac=MASK_EXEMPT_FRAC):
    """Bit-exact outside the exemption band; returns the exempt count, which must stay
    below max_frac of the elements (a d_mask that exempted everything fails here)."""
    ex = exempt_mask(o)
    bad = (m_gpu != o["mask"]) & ~ex
    assert not bad.any(), f"mask: {int(bad.sum())} non-exempt mismatches, first at {np.argwhere(bad)[:5].tolist()}"
    n_ex = int(ex.sum())
    assert n_ex <= max_frac * ex.size + 1, f"mask: {n_ex} of {ex.size} bits exempt"
    return n_ex


def bf16_ulp(v):
    a = np.abs(v)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, -126)
    return np.exp2(e - 7)


def check_bf16(gpu_bits, ref, floor=None, skip=None, what="bf16"):
    """gpu_bits: uint16 bf16 patterns; ref: fp64 values."""
    gpu_bits = np.asarray(gpu_bits, dtype=np.uint16)
    ref = np.asarray(ref, dtype=np.float64)
    g = oracle.bf16_bits_to_f64(gpu_bits)
    r_rne = oracle.bf16_rne(ref)
    r16 = oracle.bf16_bits_to_f64(r_rne)
    err = np.abs(g - ref)
    denom = np.abs(ref) if floor is None else np.maximum(np.abs(ref), floor)
    ok = (gpu_bits == r_rne) | (np.abs(g - r16) <= bf16_ulp(r16) * (1 + 1e-12)) | (err <= FLOAT_REL * denom)
    if skip is not None:
        ok |= skip
    assert ok.all(), f"{what}: {int((~ok).sum())} mismatches, first at {np.argwhere(~ok)[:5].tolist()}"
    exact = float((gpu_bits == r_rne)[~skip if skip is not None else slice(None)].mean())
    return exact


def check_f32(gpu, ref, rel, floor=None, skip=None, what="fp32"):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    denom = np.abs(ref) if floor is None else np.maximum(np.abs(ref), floor)
    ok = np.abs(gpu - ref) <= rel * denom + 1e-30
    if skip is not None:
        ok |= skip
    assert ok.all(), f"{what}: {int((~ok).sum())} beyond rel {rel}, worst {np.max(np.abs(gpu-ref)[~ok] / denom[~ok])}"

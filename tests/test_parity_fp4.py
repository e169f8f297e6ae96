"""Parity of the FP4 (E2M1) grid of quest_quantize_fwd with the oracle, and of the
linear layer on FP4 operand codes.

Codes: bit-exact (4-bit E2M1 nibbles, or int8 c = 2Q) outside the 1e-5 band
around a decision point (a midpoint between neighbouring grid values, or t = 0
where the sign bit flips); inside it the grid value may differ by one step.
Masks: exact outside the band around a flip point. Scales: 1e-5 relative.
Dequantised values: bf16 within one ulp of the rounded oracle value (fp32 within
1e-5), skipped where the code is exempt.
"""
import numpy as np
import pytest
import torch

import oracle
import bit_quantization_aware_blockwise_b200 as q
from bit_quantization_aware_blockwise_b200 import inputs
from parity import (MASK_EXEMPT_FRAC, MASK_EXEMPT_FRAC_TRUST_BELOW_1, check_bf16, check_f32, check_mask,
                    exempt_codes, unpack_mask_bits)

pytestmark = pytest.mark.gpu

SCALE_REL = 1e-5
E2M1 = np.array([oracle.e2m1_value(c) for c in range(16)])


def unpack_fp4(raw, rows, cols):
    by = np.asarray(raw, dtype=np.uint8).reshape(-1)[: rows * cols // 2].reshape(rows, cols // 2)
    return np.stack([by & 0xF, by >> 4], axis=-1).reshape(rows, cols)


def run_gpu(x_cpu, had=128, rms_group=None, trust=1.0, code_mode=q.CODES_FP4_PACKED,
            mask_mode=q.MASK_BITS, dequant="bf16"):
    rows, cols = x_cpu.shape
    out = q.quantize_fwd(x_cpu.to("cuda"), 4, had_block=had, rms_group=rms_group, trust=trust,
                         code_mode=code_mode, mask_mode=mask_mode, dequant=dequant)
    torch.cuda.synchronize()
    res = {"scales": out["scales"].cpu().numpy()}
    raw = out["codes"].cpu().numpy()
    if code_mode == q.CODES_FP4_PACKED:
        res["code"] = unpack_fp4(raw, rows, cols)
        res["value"] = E2M1[res["code"]]
    else:
        c = raw[: rows * cols].view(np.int8).reshape(rows, cols).astype(np.float64)
        res["value"] = c / 2.0
    if mask_mode == q.MASK_BITS:
        res["mask"] = unpack_mask_bits(out["mask"].cpu().numpy(), rows, cols)
    elif mask_mode == q.MASK_BYTES:
        res["mask"] = out["mask"].cpu().numpy()[: rows * cols].reshape(rows, cols)
    if dequant == "bf16":
        res["deq_bits"] = out["dequant"].cpu().view(torch.int16).numpy().view(np.uint16)
    elif dequant == "fp32":
        res["deq"] = out["dequant"].cpu().numpy().astype(np.float64)
    return res


def neighbours(v, w):
    """True where grid values v and w are equal or adjacent on the signed grid."""
    grid = np.unique(E2M1)
    iv = np.searchsorted(grid, v)
    iw = np.searchsorted(grid, w)
    return np.abs(iv - iw) <= 1


def check_fp4(res, o, trust=1.0):
    ex = exempt_codes(o)
    if "code" in res:
        bad = (res["code"] != o["code"]) & ~ex
    else:
        bad = (res["value"] != o["value"]) & ~ex
    assert not bad.any(), f"codes: {int(bad.sum())} non-exempt mismatches, first at {np.argwhere(bad)[:5].tolist()}"
    assert np.all(neighbours(res["value"][ex], o["value"][ex]))
    check_f32(res["scales"], o["scale"], SCALE_REL, what="scales")
    if "mask" in res:
        check_mask(res["mask"], o, MASK_EXEMPT_FRAC if trust >= 1 else MASK_EXEMPT_FRAC_TRUST_BELOW_1)
    diff = res["value"] != o["value"]
    if "deq_bits" in res:
        check_bf16(res["deq_bits"], o["yhat"], skip=diff, what="dequant bf16")
    if "deq" in res:
        check_f32(res["deq"], o["yhat"], SCALE_REL, floor=1e-30, skip=diff, what="dequant fp32")
    return int(ex.sum())


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("had", [16, 32, 64, 128, 256])
def test_fp4_group_rms_packed(cuda_device, dtype, had):
    # 37 rows x 768: a ragged last warp step in both layouts
    x = inputs.activations(37, 768, seed=had, dtype=dtype)
    o = oracle.quantize_fp4(inputs.to_f64(x), had=had)
    n_ex = check_fp4(run_gpu(x, had=had), o)
    assert n_ex <= 1e-3 * x.numel()


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("spr", [1, 2, 4, 8, 16])
def test_fp4_row_rms_operand(cuda_device, dtype, spr):
    cols = 128 * spr
    x = inputs.activations(27, cols, seed=spr, dtype=dtype)
    o = oracle.quantize_fp4(inputs.to_f64(x), had=128, rms_group=cols)
    check_fp4(run_gpu(x, rms_group=cols, code_mode=q.CODES_FP4_OPERAND), o)


@pytest.mark.parametrize("trust", [0.6, 1.5])
@pytest.mark.parametrize("code_mode", [q.CODES_FP4_PACKED, q.CODES_FP4_OPERAND])
def test_fp4_trust_forms_byte_mask_fp32_dequant(cuda_device, trust, code_mode):
    # T < 1 takes the interval rule per element, T >= 1 the edge |t| <= 6 + T
    x = inputs.activations(21, 1024, seed=int(trust * 10), dtype="bf16")
    o = oracle.quantize_fp4(inputs.to_f64(x), had=64, trust=trust)
    res = run_gpu(x, had=64, trust=trust, code_mode=code_mode, mask_mode=q.MASK_BYTES, dequant="fp32")
    check_fp4(res, o, trust)
    assert 0 < res["mask"].mean() <= 1


def test_fp4_saturation_and_zero_groups(cuda_device):
    g = np.random.default_rng(3)
    x = g.standard_normal((16, 512)).astype(np.float32)
    # a constant offset on a block lands on y_0 alone (row 0 of H is all ones):
    # t_0 = sqrt(128) / s* ~ 23, far beyond 6, saturates and is masked
    x[0, :128] += 50.0
    x[1, 128:256] -= 3e3
    x[2, :128] = 0.0       # a zero group: Delta = 0, codes +0, mask 1, yhat 0
    x[3, 256:384] = 0.0
    xt = torch.from_numpy(x)
    o = oracle.quantize_fp4(x.astype(np.float64), had=128)
    res = run_gpu(xt, dequant="fp32")
    check_fp4(res, o)
    assert np.all(res["code"][2, :128] == 0) and np.all(res["mask"][2, :128] == 1)
    assert res["scales"][2, 0] == 0 and np.all(res["deq"][2, :128] == 0)
    assert res["value"][0, 0] == 6.0 and res["mask"][0, 0] == 0
    assert res["value"][1, 128] == -6.0 and res["mask"][1, 128] == 0


def test_fp4_workload_sampled(cuda_device):
    # the 16384 x 2048 activation workload at full size in the launch configuration
    # the benchmark uses; the oracle recomputes 64 sampled rows
    x = inputs.activation_input()
    rows = np.unique(np.concatenate([[0, x.shape[0] - 1],
                                     np.random.default_rng(9).choice(x.shape[0], 62, replace=False)]))
    res = run_gpu(x, dequant=None)
    o = oracle.quantize_fp4(inputs.to_f64(x[rows]), had=128)
    sub = {k: v[rows] for k, v in res.items()}
    check_fp4(sub, o)


def test_fp4_linear_end_to_end(cuda_device):
    # X and W quantized onto the FP4 grid as int8 operands c = 2Q (one RMS per row),
    # multiplied by the int8 tensor-core layer: Y = acc (Delta_x/2)(Delta_w/2)
    dev = torch.device("cuda:0")
    X = inputs.activation_input(rows=512)
    W = inputs.weight_up(rows=768)
    K = X.shape[1]
    qx = q.quantize_fwd(X.to(dev), 4, rms_group=K, code_mode=q.CODES_FP4_OPERAND, mask_mode=None)
    qw = q.quantize_fwd(W.to(dev), 4, rms_group=K, code_mode=q.CODES_FP4_OPERAND, mask_mode=None)
    cx = qx["codes"].view(torch.int8).reshape(512, K)
    cw = qw["codes"].view(torch.int8).reshape(768, K)
    y, acc_gpu = q.w4a4_linear(cx, qx["scales"].reshape(-1), cw, qw["scales"].reshape(-1), acc=True)
    q.device_status()
    ox = oracle.quantize_fp4(inputs.to_f64(X), had=128, rms_group=K)
    ow = oracle.quantize_fp4(inputs.to_f64(W), had=128, rms_group=K)
    gx = cx.cpu().numpy().astype(np.int64)
    gw = cw.cpu().numpy().astype(np.int64)
    check_fp4({"value": gx / 2.0, "scales": qx["scales"].cpu().numpy()}, ox)
    check_fp4({"value": gw / 2.0, "scales": qw["scales"].cpu().numpy()}, ow)
    ref_cx = np.rint(2 * ox["value"]).astype(np.int8)
    ref_cw = np.rint(2 * ow["value"]).astype(np.int8)
    acc = oracle.gemm_i8(ref_cx, ref_cw)
    ref = oracle.dequant_linear(acc, ox["scale"][:, 0], ow["scale"][:, 0])
    same = np.all(gx == ref_cx, axis=1)[:, None] & np.all(gw == ref_cw, axis=1)[None, :]
    assert same.mean() > 0.9
    assert np.array_equal(acc_gpu.cpu().numpy()[same], acc[same].astype(np.int32))
    yb = y.cpu().view(torch.int16).numpy().view(np.uint16)
    check_bf16(yb, ref, skip=~same, what="y end to end (FP4)")
    # sanity, not parity: the FP4 product tracks X W^T with an error of the order of
    # the grid's Gaussian MSE on both operands
    exact = inputs.to_f64(X) @ inputs.to_f64(W).T
    rel = np.linalg.norm(oracle.bf16_bits_to_f64(yb) - exact) / np.linalg.norm(exact)
    assert rel < 0.3

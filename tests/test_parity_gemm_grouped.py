"""Parity of quest_w4a4_linear_grouped (one scale per row and per 128-wide K
group on both operands, FP8 E4M3 operand codes) with the oracle's per-group
fp64 layer on the same integer codes.

The fp32 result must lie within 1e-6 of sum_g |term_g| of the oracle value (the
kernel sums the exact per-group integer products in fp32); the bf16 output
within one bf16 ulp of the correctly rounded oracle value or that same bound.
"""
import numpy as np
import pytest
import torch

import oracle
import bit_quantization_aware_blockwise_b200 as q
from bit_quantization_aware_blockwise_b200 import inputs
from parity import check_bf16, check_codes_operand, e4m3_encode_int, unpack_codes

pytestmark = pytest.mark.gpu

F32_REL = 1e-6


def _case(M, N, K, seed, lo=-8, hi=8):
    g = np.random.default_rng(seed)
    a = (2 * g.integers(lo, hi, size=(M, K)) + 1).astype(np.int8)
    b = (2 * g.integers(lo, hi, size=(N, K)) + 1).astype(np.int8)
    sa = np.exp(g.uniform(-6, -2, size=(M, K // 128))).astype(np.float32)
    sb = np.exp(g.uniform(-6, -2, size=(N, K // 128))).astype(np.float32)
    return a, b, sa, sb


def fp8(c, dev):
    """Integer codes -> E4M3 bytes on the device (encoded on the host)."""
    return torch.from_numpy(e4m3_encode_int(c)).to(dev)


def run_gpu(a, b, sa, sb):
    dev = torch.device("cuda:0")
    A = fp8(a, dev)
    B = fp8(b, dev)
    SA = torch.from_numpy(np.ascontiguousarray(sa)).to(dev)
    SB = torch.from_numpy(np.ascontiguousarray(sb)).to(dev)
    y, y32 = q.w4a4_linear_grouped(A, SA, B, SB, y_f32=True)
    q.device_status()
    return y.cpu().view(torch.int16).numpy().view(np.uint16), y32.cpu().numpy().astype(np.float64)


def check(a, b, sa, sb):
    y, y32 = run_gpu(a, b, sa, sb)
    ref, mag = oracle.linear_grouped(a, b, sa.astype(np.float64), sb.astype(np.float64))
    err = np.abs(y32 - ref)
    bound = F32_REL * mag + 1e-30
    assert np.all(err <= bound), f"fp32 result off by up to {float(np.max(err / bound)):.3g} x the bound"
    check_bf16(y, ref, floor=mag * 1e-6 / 2e-3, what="y")


@pytest.mark.parametrize("M,N,K", [(256, 256, 128), (256, 512, 2048), (300, 520, 256), (1, 8, 128),
                                   (129, 264, 384), (640, 1280, 1024), (128, 256, 4096), (64, 248, 2176)])
def test_grouped_shapes(cuda_device, M, N, K):
    check(*_case(M, N, K, seed=M + N + K))


@pytest.mark.parametrize("M,N,K", [(2560, 2080, 640), (9400, 1272, 128), (7424, 1016, 384)])
def test_grouped_several_tiles_per_pair(cuda_device, M, N, K):
    # more pair tiles than CTA pairs on the part (148 SMs: 74 pairs): each pair takes
    # 2-3, 5 or 3-4 tiles, two at a time (odd counts leave a last tile alone), with an
    # odd number of K groups (5, 1, 3) and ragged rows or columns
    check(*_case(M, N, K, seed=M + N + K))


def test_grouped_largest_codes(cuda_device):
    # |c| = 15 everywhere: every group's product is +-128 * 225 = +-28800
    M, N, K = 256, 256, 512
    g = np.random.default_rng(3)
    a = np.where(g.random((M, K)) < 0.5, -15, 15).astype(np.int8)
    b = np.where(g.random((N, K)) < 0.5, -15, 15).astype(np.int8)
    a[0, :] = 15
    b[0, :] = 15
    sa = np.exp(g.uniform(-4, 0, size=(M, K // 128))).astype(np.float32)
    sb = np.exp(g.uniform(-4, 0, size=(N, K // 128))).astype(np.float32)
    check(a, b, sa, sb)


def test_grouped_constant_scales_match_the_row_scaled_layer(cuda_device):
    # the grouped kernel with scales constant along K against the row-scaled kernel
    a, b, _, _ = _case(384, 512, 1024, seed=9)
    ra = np.exp(np.random.default_rng(1).uniform(-5, -1, size=384)).astype(np.float32)
    rb = np.exp(np.random.default_rng(2).uniform(-5, -1, size=512)).astype(np.float32)
    dev = torch.device("cuda:0")
    A, B = torch.from_numpy(a).to(dev), torch.from_numpy(b).to(dev)
    y_row = q.w4a4_linear(A, torch.from_numpy(ra).to(dev), B, torch.from_numpy(rb).to(dev))
    y_grp, y32 = q.w4a4_linear_grouped(fp8(a, dev), torch.from_numpy(np.repeat(ra[:, None], 8, axis=1)).to(dev),
                                       fp8(b, dev), torch.from_numpy(np.repeat(rb[:, None], 8, axis=1)).to(dev),
                                       y_f32=True)
    q.device_status()
    ref = oracle.dequant_linear(oracle.gemm_i8(a, b), ra.astype(np.float64), rb.astype(np.float64))
    check_bf16(y_row.cpu().view(torch.int16).numpy().view(np.uint16), ref, what="row-scaled")
    _, mag = oracle.linear_grouped(a, b, np.repeat(ra[:, None], 8, axis=1).astype(np.float64),
                                   np.repeat(rb[:, None], 8, axis=1).astype(np.float64))
    assert np.all(np.abs(y32.cpu().numpy() - ref) <= F32_REL * mag + 1e-30)


def test_grouped_k_zero_and_empty(cuda_device):
    dev = torch.device("cuda:0")
    z = lambda *s: torch.zeros(s, dtype=torch.uint8, device=dev)
    y, y32 = q.w4a4_linear_grouped(z(5, 0), torch.zeros((5, 0), device=dev), z(8, 0),
                                   torch.zeros((8, 0), device=dev), y_f32=True)
    torch.cuda.synchronize()
    assert torch.all(y == 0) and torch.all(y32 == 0)
    y = q.w4a4_linear_grouped(z(0, 128), torch.zeros((0, 1), device=dev), z(8, 128),
                              torch.ones((8, 1), device=dev))
    assert y.numel() == 0


def test_grouped_full_shape_sampled(cuda_device):
    # 16384 x 5632 x 2048 (16 groups): the oracle recomputes a 20 x 20 grid of outputs
    M, N, K = inputs.TOKENS, inputs.MLP_WIDTH, inputs.HIDDEN
    a, b, sa, sb = _case(M, N, K, seed=41)
    y, y32 = run_gpu(a, b, sa, sb)
    g = np.random.default_rng(42)
    rows = np.unique(np.concatenate([[0, M - 1], g.choice(M, 18, replace=False)]))
    cols = np.unique(np.concatenate([[0, N - 1], g.choice(N, 18, replace=False)]))
    ref, mag = oracle.linear_grouped(a[rows], b[cols], sa[rows].astype(np.float64), sb[cols].astype(np.float64))
    assert np.all(np.abs(y32[np.ix_(rows, cols)] - ref) <= F32_REL * mag + 1e-30)
    check_bf16(y[np.ix_(rows, cols)], ref, floor=mag * 1e-6 / 2e-3, what="y (sampled)")


def test_grouped_linear_end_to_end(cuda_device):
    # X and W quantized at b = 4 with one RMS per 128-group (operand codes) on the
    # GPU, then the grouped layer; the oracle runs the same chain in fp64.
    dev = torch.device("cuda:0")
    X = inputs.activation_input(rows=256)
    W = inputs.weight_up(rows=384)
    K = X.shape[1]
    E4M3 = q.CODES_GEMM_OPERAND_E4M3
    qx = q.quantize_fwd(X.to(dev), 4, rms_group=128, code_mode=E4M3, mask_mode=None)
    qw = q.quantize_fwd(W.to(dev), 4, rms_group=128, code_mode=E4M3, mask_mode=None)
    cx = qx["codes"].reshape(256, K)
    cw = qw["codes"].reshape(384, K)
    y = q.w4a4_linear_grouped(cx, qx["scales"].reshape(256, K // 128), cw, qw["scales"].reshape(384, K // 128))
    q.device_status()
    ox = oracle.quantize(inputs.to_f64(X), bits=4, had=128)
    ow = oracle.quantize(inputs.to_f64(W), bits=4, had=128)
    gpu_cx = unpack_codes(cx.cpu().numpy(), 256, K, 4, 3)
    gpu_cw = unpack_codes(cw.cpu().numpy(), 384, K, 4, 3)
    check_codes_operand(gpu_cx, ox)
    check_codes_operand(gpu_cw, ow)
    ref, mag = oracle.linear_grouped((2 * ox["q"] + 1).astype(np.int8), (2 * ow["q"] + 1).astype(np.int8),
                                     ox["scale"], ow["scale"])
    same = np.all(gpu_cx == 2 * ox["q"] + 1, axis=1)[:, None] & np.all(gpu_cw == 2 * ow["q"] + 1, axis=1)[None, :]
    assert same.mean() > 0.95
    # the GPU scales differ from the oracle's by a few fp32 ulp, so each term by a
    # few 1e-7 of itself: 2e-3 relative, with sum_g |term_g| * 5e-4 as the floor
    check_bf16(y.cpu().view(torch.int16).numpy().view(np.uint16), ref, floor=mag * 1e-6 / 2e-3, skip=~same,
               what="y end to end")

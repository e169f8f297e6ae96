"""Parity of quest_w4a4_linear (tcgen05 int8 GEMM, through the C ABI) with the
oracle's triple-loop int64 GEMM and fp64 dequantisation.

The int32 accumulator must match bit for bit; the bf16 output must be within one
bf16 ulp of the correctly rounded fp64 value (the kernel scales in fp32).
"""
import numpy as np
import pytest
import torch

import oracle
import bit_quantization_aware_blockwise_b200 as q
from bit_quantization_aware_blockwise_b200 import inputs
from parity import check_bf16, check_codes_operand, unpack_codes

pytestmark = pytest.mark.gpu


def run_gpu(a, b, sa, sb, acc=True):
    dev = torch.device("cuda:0")
    A = torch.from_numpy(np.ascontiguousarray(a)).to(dev)
    B = torch.from_numpy(np.ascontiguousarray(b)).to(dev)
    SA = torch.from_numpy(np.ascontiguousarray(sa, dtype=np.float32)).to(dev)
    SB = torch.from_numpy(np.ascontiguousarray(sb, dtype=np.float32)).to(dev)
    res = q.w4a4_linear(A, SA, B, SB, acc=acc)
    q.device_status()
    if acc:
        y, ac = res
        return y.cpu().view(torch.int16).numpy().view(np.uint16), ac.cpu().numpy()
    return res.cpu().view(torch.int16).numpy().view(np.uint16), None


def check(a, b, sa, sb):
    y, acc = run_gpu(a, b, sa, sb)
    ref_acc = oracle.gemm_i8(a, b)
    assert np.array_equal(acc.astype(np.int64), ref_acc), \
        f"acc mismatches: {int((acc != ref_acc).sum())}"
    ref_y = oracle.dequant_linear(ref_acc, sa.astype(np.float64), sb.astype(np.float64))
    check_bf16(y, ref_y, what="y")


@pytest.mark.parametrize("M,N,K", [(128, 256, 128), (256, 512, 2048), (128, 256, 4096),
                                   (300, 520, 256), (1, 8, 16), (127, 248, 112), (129, 264, 144),
                                   (640, 1280, 384)])
def test_codes_full_range(cuda_device, M, N, K):
    a = inputs.gemm_codes(M, K, seed=M + K)
    b = inputs.gemm_codes(N, K, seed=N + 3 * K)
    sa = inputs.positive_scales(M, seed=1)
    sb = inputs.positive_scales(N, seed=2)
    check(a, b, sa, sb)


@pytest.mark.parametrize("M,N,K", [
    (2560, 2080, 384),   # 10 x 9 = 90 pair tiles: a full wave of 74, then 16
    (3072, 2560, 128),   # 12 x 10 = 120 pair tiles: a full wave, then 46
])
def test_two_wave_schedules(cuda_device, M, N, K):
    # More tiles than CTA pairs, so pairs take a second tile with the TMEM
    # accumulator and stage rings carried over; the first shape's last column
    # block (N = 2080) is ragged, its second 128-column half wholly past N.
    a = inputs.gemm_codes(M, K, seed=M + 7)
    b = inputs.gemm_codes(N, K, seed=N + 9)
    check(a, b, inputs.positive_scales(M, seed=11), inputs.positive_scales(N, seed=12))


def test_int8_extremes(cuda_device):
    # every int8 value, including -128 * -128 products
    M, N, K = 256, 256, 1024
    g = np.random.default_rng(3)
    a = g.integers(-128, 128, size=(M, K)).astype(np.int8)
    b = g.integers(-128, 128, size=(N, K)).astype(np.int8)
    a[0, :] = -128
    b[0, :] = -128
    check(a, b, np.ones(M, np.float32), np.ones(N, np.float32) * 1e-4)


def test_closed_form_constant_codes(cuda_device):
    K = 2048
    a = np.full((128, K), 15, np.int8)
    b = np.full((256, K), 15, np.int8)
    y, acc = run_gpu(a, b, np.ones(128, np.float32), np.ones(256, np.float32))
    assert np.all(acc == 225 * K)


def test_k_zero_and_empty(cuda_device):
    y, acc = run_gpu(np.zeros((5, 0), np.int8), np.zeros((8, 0), np.int8),
                     np.ones(5, np.float32), np.ones(8, np.float32))
    assert np.all(acc == 0) and np.all(y == 0)
    y, acc = run_gpu(np.zeros((0, 32), np.int8), np.zeros((8, 32), np.int8),
                     np.ones(0, np.float32), np.ones(8, np.float32))
    assert y.size == 0


def test_repeated_calls_are_stable(cuda_device):
    a = inputs.gemm_codes(384, 512, seed=5)
    b = inputs.gemm_codes(768, 512, seed=6)
    sa, sb = inputs.positive_scales(384, 7), inputs.positive_scales(768, 8)
    y0, acc0 = run_gpu(a, b, sa, sb)
    for _ in range(3):
        y1, acc1 = run_gpu(a, b, sa, sb)
        assert np.array_equal(acc0, acc1) and np.array_equal(y0, y1)


def test_full_shape_sampled(cuda_device):
    # 16384 x 5632 x 2048 with seeded b = 4 operand codes: the launch the benchmark
    # times. The oracle recomputes a 24 x 24 grid of sampled outputs.
    M, N, K = inputs.TOKENS, inputs.MLP_WIDTH, inputs.HIDDEN
    a = inputs.gemm_codes(M, K, seed=31)
    b = inputs.gemm_codes(N, K, seed=32)
    sa, sb = inputs.positive_scales(M, 33), inputs.positive_scales(N, 34)
    y, acc = run_gpu(a, b, sa, sb)
    g = np.random.default_rng(35)
    rows = np.unique(np.concatenate([[0, M - 1], g.choice(M, 22, replace=False)]))
    cols = np.unique(np.concatenate([[0, N - 1], g.choice(N, 22, replace=False)]))
    ref_acc = oracle.gemm_i8(a[rows], b[cols])
    assert np.array_equal(acc[np.ix_(rows, cols)].astype(np.int64), ref_acc)
    ref_y = oracle.dequant_linear(ref_acc, sa[rows].astype(np.float64), sb[cols].astype(np.float64))
    check_bf16(y[np.ix_(rows, cols)], ref_y, what="y (sampled)")


def test_quantized_linear_end_to_end(cuda_device):
    # X (heavy-tailed activations) and W (Gaussian weights) quantized to b = 4
    # operand codes with one RMS per row on the GPU, then multiplied. The oracle runs
    # the same chain in fp64; rows whose codes sit on a rounding boundary are
    # compared only through the codes check.
    dev = torch.device("cuda:0")
    X = inputs.activation_input(rows=512)
    W = inputs.weight_up(rows=768)
    K = X.shape[1]
    qx = q.quantize_fwd(X.to(dev), 4, rms_group=K, code_mode=q.CODES_GEMM_OPERAND, mask_mode=None)
    qw = q.quantize_fwd(W.to(dev), 4, rms_group=K, code_mode=q.CODES_GEMM_OPERAND, mask_mode=None)
    cx = qx["codes"].view(torch.int8).reshape(512, K)
    cw = qw["codes"].view(torch.int8).reshape(768, K)
    y = q.w4a4_linear(cx, qx["scales"].reshape(-1), cw, qw["scales"].reshape(-1))
    q.device_status()
    ox = oracle.quantize(inputs.to_f64(X), bits=4, had=128, rms_group=K)
    ow = oracle.quantize(inputs.to_f64(W), bits=4, had=128, rms_group=K)
    check_codes_operand(unpack_codes(cx.cpu().numpy(), 512, K, 4, 2), ox)
    check_codes_operand(unpack_codes(cw.cpu().numpy(), 768, K, 4, 2), ow)
    acc = oracle.gemm_i8((2 * ox["q"] + 1).astype(np.int8), (2 * ow["q"] + 1).astype(np.int8))
    ref = oracle.dequant_linear(acc, ox["scale"][:, 0], ow["scale"][:, 0])
    gpu_cx = unpack_codes(cx.cpu().numpy(), 512, K, 4, 2)
    gpu_cw = unpack_codes(cw.cpu().numpy(), 768, K, 4, 2)
    rows_same = np.all(gpu_cx == 2 * ox["q"] + 1, axis=1)
    cols_same = np.all(gpu_cw == 2 * ow["q"] + 1, axis=1)
    skip = ~(rows_same[:, None] & cols_same[None, :])
    assert skip.mean() < 0.05
    yb = y.cpu().view(torch.int16).numpy().view(np.uint16)
    # scales differ from the oracle's by a few fp32 ulp: allow 2e-3 relative
    check_bf16(yb, ref, skip=skip, what="y end to end")
    # sanity, not parity: the quantized product approximates X W^T (orthogonality
    # of the transform) with the error expected from two 4-bit operands
    exact = inputs.to_f64(X) @ inputs.to_f64(W).T
    rel = np.linalg.norm(oracle.bf16_bits_to_f64(yb) - exact) / np.linalg.norm(exact)
    assert rel < 0.3


def test_w1a1_linear_end_to_end(cuda_device):
    # The 1-bit path: X and W quantized at b = 1 (one RMS per row, operand codes
    # c = 2q + 1 in {-1, +1}) and multiplied by the same int8 tensor-core GEMM.
    dev = torch.device("cuda:0")
    X = inputs.activation_input(rows=384)
    W = inputs.weight_up(rows=512)
    K = X.shape[1]
    qx = q.quantize_fwd(X.to(dev), 1, rms_group=K, code_mode=q.CODES_GEMM_OPERAND, mask_mode=None)
    qw = q.quantize_fwd(W.to(dev), 1, rms_group=K, code_mode=q.CODES_GEMM_OPERAND, mask_mode=None)
    cx = qx["codes"].view(torch.int8).reshape(384, K)
    cw = qw["codes"].view(torch.int8).reshape(512, K)
    y, acc_gpu = q.w4a4_linear(cx, qx["scales"].reshape(-1), cw, qw["scales"].reshape(-1), acc=True)
    q.device_status()
    gpu_cx = unpack_codes(cx.cpu().numpy(), 384, K, 1, 2)
    gpu_cw = unpack_codes(cw.cpu().numpy(), 512, K, 1, 2)
    assert set(np.unique(gpu_cx)) <= {-1, 1} and set(np.unique(gpu_cw)) <= {-1, 1}
    ox = oracle.quantize(inputs.to_f64(X), bits=1, had=128, rms_group=K)
    ow = oracle.quantize(inputs.to_f64(W), bits=1, had=128, rms_group=K)
    check_codes_operand(gpu_cx, ox)
    check_codes_operand(gpu_cw, ow)
    acc = oracle.gemm_i8((2 * ox["q"] + 1).astype(np.int8), (2 * ow["q"] + 1).astype(np.int8))
    ref = oracle.dequant_linear(acc, ox["scale"][:, 0], ow["scale"][:, 0])
    rows_same = np.all(gpu_cx == 2 * ox["q"] + 1, axis=1)
    cols_same = np.all(gpu_cw == 2 * ow["q"] + 1, axis=1)
    same = rows_same[:, None] & cols_same[None, :]
    assert same.mean() > 0.95
    # the accumulator is exact wherever both code rows agree with the oracle's
    assert np.array_equal(acc_gpu.cpu().numpy()[same], acc[same].astype(np.int32))
    yb = y.cpu().view(torch.int16).numpy().view(np.uint16)
    check_bf16(yb, ref, skip=~same, what="y end to end (W1A1)")
    # sanity, not parity: the 1-bit product still tracks X W^T
    exact = inputs.to_f64(X) @ inputs.to_f64(W).T
    yv = oracle.bf16_bits_to_f64(yb)
    corr = np.sum(yv * exact) / (np.linalg.norm(yv) * np.linalg.norm(exact))
    assert corr > 0.5


@pytest.mark.parametrize("M,N,K", [(64, 8, 131056), (200, 16, 65536)])
def test_longest_reduction(cuda_device, M, N, K):
    # K up to the largest the library accepts (< 131072, a multiple of 16), with codes at
    # the b = 4 extremes so |acc| reaches K * 225: the int32 accumulator stays exact
    a = np.full((M, K), 15, np.int8)
    b = np.full((N, K), -15, np.int8)
    a[1::2] = inputs.gemm_codes(M // 2, K, seed=41)
    b[1::2] = inputs.gemm_codes(N // 2, K, seed=42)
    check(a, b, inputs.positive_scales(M, seed=43), inputs.positive_scales(N, seed=44))

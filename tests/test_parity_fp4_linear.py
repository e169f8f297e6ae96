"""Parity of quest_fp4_linear (packed E2M1 codes on the block-scaled FP4 tensor cores,
through the C ABI) with the oracle.

The oracle's product is the integer one on the operand form c = 2Q of the same codes
(Q the E2M1 grid value): sum_k c_a c_w = 4 sum_k Q_a Q_w exactly, so the kernel's fp32
accumulator must equal the oracle's int64 sum / 4 bit for bit (every partial sum is a
multiple of 1/4 below 2^20). y is bf16: equal to the rounded fp64 value
acc * Delta_a * Delta_w, within one bf16 ulp of it, or within 2e-3 of it."""
import numpy as np
import pytest
import torch

import oracle
import bit_quantization_aware_blockwise_b200 as q
from bit_quantization_aware_blockwise_b200 import inputs
from parity import check_bf16

pytestmark = pytest.mark.gpu

E2M1_2Q = np.array([int(round(2 * oracle.e2m1_value(c))) for c in range(16)], dtype=np.int8)


def operand_2q(packed, K):
    """Packed nibbles [rows, K/2] -> int8 c = 2Q [rows, K] (element 2j from the low nibble)."""
    by = np.asarray(packed, dtype=np.uint8).reshape(-1, K // 2)
    nib = np.stack([by & 0xF, by >> 4], axis=-1).reshape(by.shape[0], K)
    return E2M1_2Q[nib]


def run(pa, sa, pw, sw, K):
    dev = torch.device("cuda:0")
    y, acc = q.fp4_linear(torch.from_numpy(pa).to(dev), torch.from_numpy(sa).to(dev),
                          torch.from_numpy(pw).to(dev), torch.from_numpy(sw).to(dev), K, acc=True)
    q.device_status()
    return y.cpu().view(torch.int16).numpy().view(np.uint16), acc.cpu().numpy().astype(np.float64)


def check(pa, sa, pw, sw, K, rows=None):
    y, acc = run(pa, sa, pw, sw, K)
    if rows is not None:
        y, acc, pa, sa = y[rows], acc[rows], pa[rows], sa[rows]
    ref = oracle.gemm_i8(operand_2q(pa, K), operand_2q(pw, K))
    assert np.array_equal(acc * 4.0, ref.astype(np.float64)), \
        f"accumulator differs at {np.argwhere(acc * 4.0 != ref)[:5].tolist()}"
    check_bf16(y, oracle.dequant_linear(ref, sa, sw), what="y")


@pytest.mark.parametrize("M,N,K", [(256, 224, 256), (300, 520, 384), (1, 8, 32), (129, 232, 96),
                                   (2560, 2080, 640), (512, 5632, 2048)])
def test_fp4_linear_matches_oracle(cuda_device, M, N, K):
    # ragged M and N, K below one 256-value stage or not a multiple of it, more pair tiles
    # than CTA pairs (both accumulators in turn), and a row block of the full layer
    check(inputs.fp4_codes(M, K, seed=M), inputs.positive_scales(M, M + 1),
          inputs.fp4_codes(N, K, seed=N + 2), inputs.positive_scales(N, N + 3), K)


def test_fp4_linear_largest_products(cuda_device):
    # all codes +-6 (0x7 / 0xF): |acc| = 36 K at K = 16384, the largest K accepted
    M, N, K = 256, 224, 16384
    g = np.random.default_rng(5)
    pa = np.where(g.random((M, K // 2)) < 0.5, 0x77, 0xFF).astype(np.uint8)
    pa[:128] = 0x77   # rows of +6 only: acc = +-36 K exactly
    pw = np.full((N, K // 2), 0x77, np.uint8)
    pw[N // 2:] = 0xFF
    sa, sw = np.full(M, 0.5, np.float32), np.full(N, 0.25, np.float32)
    check(pa, sa, pw, sw, K)
    _, acc = run(pa, sa, pw, sw, K)
    assert acc[0, 0] == 36.0 * K and acc[0, N - 1] == -36.0 * K


def test_fp4_linear_empty_and_k_zero(cuda_device):
    dev = torch.device("cuda:0")
    y = torch.full((4, 16), 1.0, dtype=torch.bfloat16, device=dev)
    q.fp4_linear(torch.zeros(0, dtype=torch.uint8, device=dev), torch.ones(4, device=dev),
                 torch.zeros(0, dtype=torch.uint8, device=dev), torch.ones(16, device=dev), 0, out=y)
    q.device_status()
    assert not y.float().abs().sum().item()


def test_fp4_linear_full_shape_sampled(cuda_device):
    # 16384 x 5632 x 2048 (the layer's full size, the launch the configs time): the oracle
    # recomputes 24 sampled rows
    M, N, K = inputs.TOKENS, inputs.MLP_WIDTH, inputs.HIDDEN
    pa, sa = inputs.fp4_codes(M, K, seed=21), inputs.positive_scales(M, 22)
    pw, sw = inputs.fp4_codes(N, K, seed=23), inputs.positive_scales(N, 24)
    rows = np.unique(np.concatenate([[0, M - 1], np.random.default_rng(13).choice(M, 22, replace=False)]))
    check(pa, sa, pw, sw, K, rows=rows)


def test_fp4_linear_end_to_end_from_the_quantizer(cuda_device):
    # X and W quantized onto the FP4 grid as packed E2M1 codes with one RMS per row, then
    # multiplied on the FP4 tensor cores; against the oracle's codes and steps, rows whose
    # codes sit on a rounding boundary are compared only through the GPU's own codes
    dev = torch.device("cuda:0")
    X = inputs.activation_input(rows=512)
    W = inputs.weight_up(rows=768)
    K = X.shape[1]
    qx = q.quantize_fwd(X.to(dev), 4, rms_group=K, code_mode=q.CODES_FP4_PACKED, mask_mode=None)
    qw = q.quantize_fwd(W.to(dev), 4, rms_group=K, code_mode=q.CODES_FP4_PACKED, mask_mode=None)
    pa = qx["codes"].cpu().numpy()[: 512 * K // 2].reshape(512, K // 2)
    pw = qw["codes"].cpu().numpy()[: 768 * K // 2].reshape(768, K // 2)
    sa, sw = qx["scales"].cpu().numpy().reshape(-1), qw["scales"].cpu().numpy().reshape(-1)
    check(pa, sa, pw, sw, K)
    ox = oracle.quantize_fp4(inputs.to_f64(X), had=128, rms_group=K)
    ow = oracle.quantize_fp4(inputs.to_f64(W), had=128, rms_group=K)
    same = (np.all(operand_2q(pa, K) == np.rint(2 * ox["value"]), axis=1)[:, None]
            & np.all(operand_2q(pw, K) == np.rint(2 * ow["value"]), axis=1)[None, :])
    assert same.mean() > 0.9
    y, _ = run(pa, sa, pw, sw, K)
    ref = oracle.dequant_linear(oracle.gemm_i8(np.rint(2 * ox["value"]).astype(np.int8),
                                               np.rint(2 * ow["value"]).astype(np.int8)),
                                ox["scale"][:, 0], ow["scale"][:, 0])
    check_bf16(y, ref, skip=~same, what="y end to end (FP4 tensor cores)")

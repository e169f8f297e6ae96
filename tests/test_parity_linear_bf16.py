"""Parity of quest_linear_bf16 (tcgen05 bf16 product of dequantised operands, through
the C ABI) with the oracle, and the QAT forward chain it serves.

y is bf16: it must equal the round-to-nearest-even value of the fp64 product of the
same bf16 inputs, be within one bf16 ulp of it, or within 2e-3 of max(|ref|, floor),
where 2e-3 * floor is the standard bound K * 2^-24 * sum_k |x_k w_k| on the error of
an fp32 sum of K exact products (it matters only where the sum cancels)."""
import numpy as np
import pytest
import torch

import oracle
import bit_quantization_aware_blockwise_b200 as q
from bit_quantization_aware_blockwise_b200 import inputs
from parity import check_bf16

pytestmark = pytest.mark.gpu


def run(xh, wh):
    dev = torch.device("cuda:0")
    y = q.linear_bf16(xh.to(dev), wh.to(dev))
    q.device_status()
    return y.cpu().view(torch.int16).numpy().view(np.uint16)


def fp32_floor(x64, w64):
    """floor whose 2e-3 share is the fp32 accumulation bound K 2^-24 sum |x||w|."""
    K = x64.shape[1]
    return max(K, 1) * 2.0 ** -24 * (np.abs(x64) @ np.abs(w64).T) / 2e-3


def check(xh, wh, what="y"):
    x64, w64 = inputs.to_f64(xh), inputs.to_f64(wh)
    ref = oracle.linear_bf16(x64, w64)
    check_bf16(run(xh, wh), ref, floor=fp32_floor(x64, w64), what=what)


@pytest.mark.parametrize("M,N,K", [(300, 520, 384), (256, 256, 64), (1, 8, 8), (129, 264, 1032),
                                   (2560, 2080, 256), (512, 5632, 2048)])
def test_linear_bf16_matches_oracle(cuda_device, M, N, K):
    check(inputs.gaussian(M, K, seed=M), inputs.gaussian(N, K, seed=N + 1, std=0.02))


def test_linear_bf16_empty(cuda_device):
    dev = torch.device("cuda:0")
    y = torch.full((4, 16), 1.0, dtype=torch.bfloat16, device=dev)
    q.linear_bf16(torch.zeros((4, 0), dtype=torch.bfloat16, device=dev),
                  torch.zeros((16, 0), dtype=torch.bfloat16, device=dev), out=y)
    q.device_status()
    assert not y.float().abs().sum().item()
    y = q.linear_bf16(torch.zeros((0, 64), dtype=torch.bfloat16, device=dev),
                      torch.zeros((16, 64), dtype=torch.bfloat16, device=dev))
    assert y.shape == (0, 16)


def test_linear_bf16_full_shape_sampled(cuda_device):
    # 16384 x 5632 x 2048: the timed launch; the oracle recomputes 24 rows
    M, N, K = inputs.TOKENS, inputs.MLP_WIDTH, inputs.HIDDEN
    xh, wh = inputs.activation_input(), inputs.weight_up()
    y = run(xh, wh)
    rows = np.unique(np.concatenate([[0, M - 1], np.random.default_rng(12).choice(M, 22, replace=False)]))
    x64, w64 = inputs.to_f64(xh[rows]), inputs.to_f64(wh)
    check_bf16(y[rows], oracle.linear_bf16(x64, w64), floor=fp32_floor(x64, w64), what="y (sampled rows)")


@pytest.mark.parametrize("rms", ["group", "row"])
def test_qat_forward_on_dequantised_operands(cuda_device, rms):
    # the QAT forward: both operands quantized (b = 4), dequantised to bf16 yhat, multiplied.
    # Against the GPU's own yhat the product is checked as above; against the exact
    # result on the codes (the grouped or row-scaled layer of the oracle) the difference
    # is the bf16 rounding of yhat, at most 2^-8 of each term's magnitude.
    dev = torch.device("cuda:0")
    X = inputs.activation_input(rows=384)
    W = inputs.weight_up(rows=512)
    K = X.shape[1]
    rg = 128 if rms == "group" else K
    qx = q.quantize_fwd(X.to(dev), 4, rms_group=rg, code_mode=q.CODES_INT8, mask_mode=None, dequant="bf16")
    qw = q.quantize_fwd(W.to(dev), 4, rms_group=rg, code_mode=q.CODES_INT8, mask_mode=None, dequant="bf16")
    xh, wh = qx["dequant"], qw["dequant"]
    y = q.linear_bf16(xh, wh)
    q.device_status()
    yb = y.cpu().view(torch.int16).numpy().view(np.uint16)
    x64, w64 = inputs.to_f64(xh.cpu()), inputs.to_f64(wh.cpu())
    check_bf16(yb, oracle.linear_bf16(x64, w64), floor=fp32_floor(x64, w64), what="y on the GPU's yhat")
    # the exact layer on the oracle's codes and scales
    ox = oracle.quantize(inputs.to_f64(X), bits=4, had=128, rms_group=rg)
    ow = oracle.quantize(inputs.to_f64(W), bits=4, had=128, rms_group=rg)
    exact = oracle.linear_bf16(ox["yhat"], ow["yhat"])
    emag = np.abs(ox["yhat"]) @ np.abs(ow["yhat"]).T
    # rows and columns whose codes sit on a rounding boundary are compared only above
    same = (np.all(qx["codes"].cpu().numpy()[: 384 * K].view(np.int8).reshape(384, K) == ox["q"], axis=1)[:, None]
            & np.all(qw["codes"].cpu().numpy()[: 512 * K].view(np.int8).reshape(512, K) == ow["q"], axis=1)[None, :])
    assert same.mean() > 0.9
    err = np.abs(oracle.bf16_bits_to_f64(yb) - exact)
    assert np.all((err <= 2 ** -7 * emag + np.abs(exact) * 2 ** -8)[same])

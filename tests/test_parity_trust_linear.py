"""Parity of quest_trust_bwd_linear (tcgen05 bf16 product with the trust backward in
its epilogue, through the C ABI) and quest_transpose_bf16 with the oracle.

grad_x is bf16: it must equal the round-to-nearest-even value of the fp64 oracle,
be within one bf16 ulp of it, or within 2e-3 of max(|ref|, the RMS of the ref's
128-block) (the 128-point transform cancels; fp32 accumulation over N and the
transform add about 1e-6 of the block RMS). The transpose is exact.
"""
import numpy as np
import pytest
import torch

import oracle
import bit_quantization_aware_blockwise_b200 as q
from bit_quantization_aware_blockwise_b200 import inputs
from parity import check_bf16, unpack_mask_bits

pytestmark = pytest.mark.gpu


def block_rms(ref, had=128):
    r = np.sqrt((ref.reshape(ref.shape[0], -1, had) ** 2).mean(axis=2))
    return np.repeat(r, had, axis=1)


def run(gy, wt, mask_bits):
    dev = torch.device("cuda:0")
    out = q.trust_bwd_linear(gy.to(dev), wt.to(dev), torch.from_numpy(mask_bits).to(dev))
    q.device_status()
    return out.cpu().view(torch.int16).numpy().view(np.uint16)


def case(M, N, K, seed, keep=0.97):
    gy = inputs.upstream_grad(M, N, seed=seed)
    w = inputs.weights(N, K, seed=seed + 1)           # w_hat [N, K]
    wt = w.t().contiguous()                            # [K, N]
    m01 = inputs.random_mask(M, K, seed=seed + 2, keep_prob=keep)
    return gy, w, wt, m01


@pytest.mark.parametrize("M,N,K", [(300, 520, 384), (256, 64, 256), (1, 8, 128), (129, 1032, 640),
                                   (2560, 2080, 256), (512, 5632, 2048)])
def test_trust_bwd_linear_matches_oracle(cuda_device, M, N, K):
    gy, w, wt, m01 = case(M, N, K, seed=M + N)
    got = run(gy, wt, inputs.pack_mask_bits(m01))
    ref = oracle.trust_bwd_linear(inputs.to_f64(gy), inputs.to_f64(w), m01)
    check_bf16(got, ref, floor=block_rms(ref), what="grad_x")


def test_trust_bwd_linear_mask_extremes(cuda_device):
    M, N, K = 256, 256, 256
    gy, w, wt, _ = case(M, N, K, seed=7)
    ones = np.ones((M, K), np.uint8)
    zeros = np.zeros((M, K), np.uint8)
    got = run(gy, wt, inputs.pack_mask_bits(ones))
    ref = oracle.trust_bwd_linear(inputs.to_f64(gy), inputs.to_f64(w), ones)
    check_bf16(got, ref, floor=block_rms(ref), what="all kept")
    got = run(gy, wt, inputs.pack_mask_bits(zeros))
    assert not got.any()


def test_trust_bwd_linear_empty_reduction_and_rows(cuda_device):
    dev = torch.device("cuda:0")
    gy = torch.zeros((4, 0), dtype=torch.bfloat16, device=dev)
    wt = torch.zeros((256, 0), dtype=torch.bfloat16, device=dev)
    mask = torch.full((4, 32), 0xFF, dtype=torch.uint8, device=dev)
    out = torch.full((4, 256), 1.0, dtype=torch.bfloat16, device=dev)
    q.trust_bwd_linear(gy, wt, mask, out=out)
    q.device_status()
    assert not out.float().abs().sum().item()
    gy = torch.zeros((0, 64), dtype=torch.bfloat16, device=dev)
    out = q.trust_bwd_linear(gy, torch.zeros((128, 64), dtype=torch.bfloat16, device=dev),
                             torch.zeros((1, 16), dtype=torch.uint8, device=dev))
    assert out.shape == (0, 128)


def test_trust_bwd_linear_full_shape_sampled(cuda_device):
    # 16384 x 5632 -> 2048: the launch the benchmark times; the oracle recomputes 24 rows
    M, N, K = inputs.TOKENS, inputs.MLP_WIDTH, inputs.HIDDEN
    gy = inputs.layer_output_grad()
    w = inputs.weight_up()                             # an N(0, 0.02^2) w_hat [N, K]
    wt = w.t().contiguous()                            # [K, N]
    m01 = inputs.random_mask(M, K, seed=6, keep_prob=0.99)
    got = run(gy, wt, inputs.pack_mask_bits(m01))
    rows = np.unique(np.concatenate([[0, M - 1], np.random.default_rng(8).choice(M, 22, replace=False)]))
    ref = oracle.trust_bwd_linear(inputs.to_f64(gy[rows]), inputs.to_f64(w), m01[rows])
    check_bf16(got[rows], ref, floor=block_rms(ref), what="grad_x (sampled rows)")


def test_backward_chain_from_library_outputs(cuda_device):
    # the chain a QAT step runs: X quantized (its trust mask), W quantized with bf16
    # dequant (w_hat, Hadamard domain), w_hat transposed by the library, then the
    # fused input gradient; checked against the oracle on the GPU's own intermediates
    dev = torch.device("cuda:0")
    X = inputs.activation_input(rows=384)
    W = inputs.weight_up(rows=640)                      # [N = 640, K = 2048]
    gy = inputs.upstream_grad(384, 640, seed=11)
    qx = q.quantize_fwd(X.to(dev), 4, mask_mode=q.MASK_BITS)
    qw = q.quantize_fwd(W.to(dev), 4, rms_group=W.shape[1], code_mode=q.CODES_GEMM_OPERAND,
                        mask_mode=None, dequant="bf16")
    wt = q.transpose_bf16(qw["dequant"])
    out = q.trust_bwd_linear(gy.to(dev), wt, qx["mask"])
    q.device_status()
    w_hat = qw["dequant"].cpu().float().numpy().astype(np.float64)
    m01 = unpack_mask_bits(qx["mask"].cpu().numpy(), 384, 2048)
    ref = oracle.trust_bwd_linear(inputs.to_f64(gy), w_hat, m01)
    got = out.cpu().view(torch.int16).numpy().view(np.uint16)
    check_bf16(got, ref, floor=block_rms(ref), what="grad_x (chain)")


@pytest.mark.parametrize("rows,cols", [(1, 1), (31, 33), (64, 64), (5632, 2048), (100, 3000)])
def test_transpose_is_exact(cuda_device, rows, cols):
    src = inputs.gaussian(rows, cols, seed=rows + cols)
    got = q.transpose_bf16(src.to("cuda")).cpu()
    q.device_status()
    assert torch.equal(got.view(torch.int16), src.t().contiguous().view(torch.int16))

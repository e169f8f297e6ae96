"""Parity of quest_trust_bwd (CUDA, through the C ABI) with the fp64 oracle.

Output bf16 values must be within one bf16 ulp of the correctly rounded oracle
value, or within 2e-3 of max(|ref|, RMS of the reference block) (the transform
sums 128 signed terms, so single outputs can cancel far below their block's
scale).
"""
import numpy as np
import pytest
import torch

import oracle
import bit_quantization_aware_blockwise_b200 as q
from bit_quantization_aware_blockwise_b200 import inputs
from parity import check_bf16

pytestmark = pytest.mark.gpu


def _block_rms(ref, had):
    r, c = ref.shape
    b = np.sqrt(np.mean(ref.reshape(r, c // had, had) ** 2, axis=2))
    return np.repeat(b, had, axis=1)


def run_gpu(g_cpu, mask01, had=128, mask_mode=q.MASK_BITS):
    dev = torch.device("cuda:0")
    g = g_cpu.to(dev)
    if mask_mode == q.MASK_BITS:
        m = torch.from_numpy(inputs.pack_mask_bits(mask01).view(np.uint8).reshape(-1)).to(dev)
    else:
        m = torch.from_numpy(np.ascontiguousarray(mask01, dtype=np.uint8).reshape(-1)).to(dev)
    out = q.trust_bwd(g, m, had_block=had, mask_mode=mask_mode)
    torch.cuda.synchronize()
    return out.cpu().view(torch.int16).numpy().view(np.uint16)


def check(g_cpu, mask01, had=128, mask_mode=q.MASK_BITS):
    got = run_gpu(g_cpu, mask01, had, mask_mode)
    ref = oracle.trust_bwd(inputs.to_f64(g_cpu), mask01, had=had)
    return check_bf16(got, ref, floor=_block_rms(ref, had), what="grad_in")


@pytest.mark.parametrize("had", [16, 32, 64, 128, 256])
@pytest.mark.parametrize("mask_mode", [q.MASK_BITS, q.MASK_BYTES])
def test_random_masks(cuda_device, had, mask_mode):
    g = inputs.upstream_grad(96, 1024, seed=had)
    m = inputs.random_mask(96, 1024, seed=had + 1, keep_prob=0.97)
    exact = check(g, m, had, mask_mode)
    assert exact > 0.95


@pytest.mark.parametrize("rows,cols", [(1, 128), (5, 384), (31, 2048), (3, 128 * 44)])
def test_ragged_shapes(cuda_device, rows, cols):
    g = inputs.upstream_grad(rows, cols, seed=rows)
    m = inputs.random_mask(rows, cols, seed=cols, keep_prob=0.9)
    check(g, m)


def test_all_ones_mask_inverts_the_forward_transform(cuda_device):
    # H/sqrt(n) is an involution: feeding the oracle's transformed values (rounded to
    # bf16) through the backward with every entry trusted gives back the input to
    # within the bf16 rounding of the input.
    x = inputs.gaussian(16, 512, seed=2, std=1.0, dtype="fp32")
    y = oracle.quantize(inputs.to_f64(x), bits=4)["y"]
    g = torch.from_numpy(y.astype(np.float32)).to(torch.bfloat16)
    got = run_gpu(g, np.ones((16, 512), dtype=np.uint8))
    back = oracle.bf16_bits_to_f64(got)
    assert np.max(np.abs(back - inputs.to_f64(x))) < 0.02


def test_all_zero_mask(cuda_device):
    g = inputs.upstream_grad(8, 256, seed=1)
    got = run_gpu(g, np.zeros((8, 256), dtype=np.uint8))
    assert np.all((got & 0x7FFF) == 0)


def test_mask_from_the_oracle_quantizer(cuda_device):
    # The trust path as it runs in training: the mask of a b = 4 quantization of
    # heavy-tailed activations, applied to a small Gaussian gradient.
    x = inputs.activation_input(rows=256)
    m = oracle.quantize(inputs.to_f64(x), bits=4)["mask"]
    g = inputs.grad_input(rows=256)
    check(g, m)


def test_full_grad_workload_sampled(cuda_device):
    # 16384 x 2048 gradient; the mask keeps ~98% (the b = 4 masked rate of the
    # activation workload is about 2%). The oracle checks 48 sampled rows.
    g = inputs.grad_input()
    m = inputs.random_mask(g.shape[0], g.shape[1], seed=77, keep_prob=0.98)
    got = run_gpu(g, m)
    rows = np.unique(np.concatenate([[0, g.shape[0] - 1],
                                     np.random.default_rng(5).choice(g.shape[0], 48, replace=False)]))
    ref = oracle.trust_bwd(inputs.to_f64(g[rows]), m[rows], had=128)
    check_bf16(got[rows], ref, floor=_block_rms(ref, 128), what="grad_in (sampled)")


def test_empty(cuda_device):
    g = torch.zeros((0, 256), dtype=torch.bfloat16, device="cuda")
    m = torch.zeros(1, dtype=torch.uint8, device="cuda")
    out = q.trust_bwd(g, m)
    torch.cuda.synchronize()
    assert out.shape == (0, 256)


def test_under_aligned_mask_uses_the_direct_kernel(cuda_device):
    dev = torch.device("cuda:0")
    g = inputs.upstream_grad(24, 512, seed=3)
    m = inputs.random_mask(24, 512, seed=4, keep_prob=0.9)
    bits = torch.from_numpy(inputs.pack_mask_bits(m).view(np.uint8).reshape(-1))
    buf = torch.zeros(bits.numel() + 16, dtype=torch.uint8)
    buf[3:3 + bits.numel()] = bits
    buf = buf.to(dev)
    gd = g.to(dev)
    out = torch.empty_like(gd)
    q.trust_bwd_raw(gd.data_ptr(), buf.data_ptr() + 3, q.MASK_BITS, 24, 512, 128, out.data_ptr(),
                    torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    ref = oracle.trust_bwd(inputs.to_f64(g), m, had=128)
    check_bf16(out.cpu().view(torch.int16).numpy().view(np.uint16), ref, floor=_block_rms(ref, 128))


@pytest.mark.parametrize("had,cols", [(16, 48), (64, 192)])
def test_rows_not_multiple_of_128(cuda_device, had, cols):
    g = inputs.upstream_grad(17, cols, seed=cols)
    m = inputs.random_mask(17, cols, seed=1, keep_prob=0.8)
    check(g, m, had, q.MASK_BYTES)

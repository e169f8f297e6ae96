"""Parity of quest_quantize_operands (both operands of a linear layer, one RMS per row,
in one call) with the oracle, and identity with two quest_quantize_fwd calls.

Where both tensors take the tensor-core row layout the library runs one launch over
the rows of x then w; its codes and scales must equal, bit for bit, those of the two
separate calls, and match the oracle under the usual rules (parity.py)."""
import numpy as np
import pytest
import torch

import oracle
import bit_quantization_aware_blockwise_b200 as q
from bit_quantization_aware_blockwise_b200 import inputs
from parity import check_codes_operand, check_f32, unpack_codes

pytestmark = pytest.mark.gpu


def separate(x, w, bits, mode):
    K = x.shape[1]
    ox = q.quantize_fwd(x, bits, rms_group=K, code_mode=mode, mask_mode=None)
    ow = q.quantize_fwd(w, bits, rms_group=K, code_mode=mode, mask_mode=None)
    return ox, ow


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("M,N,K", [(300, 520, 2048), (37, 129, 1024), (64, 8, 512), (5, 700, 256),
                                   (16, 16, 128)])
@pytest.mark.parametrize("mode", [q.CODES_GEMM_OPERAND, q.CODES_FP4_OPERAND])
def test_operands_match_oracle_and_separate_calls(cuda_device, dtype, M, N, K, mode):
    dev = torch.device("cuda:0")
    x = inputs.activations(M, K, seed=M, dtype=dtype)
    w = inputs.weights(N, K, seed=N, dtype=dtype)
    (cx, sx), (cw, sw) = [(d["codes"], d["scales"]) for d in q.quantize_operands(x.to(dev), w.to(dev), 4, 128, mode)]
    q.device_status()
    ox, ow = separate(x.to(dev), w.to(dev), 4, mode)
    torch.cuda.synchronize()
    assert torch.equal(cx[: M * K], ox["codes"][: M * K]) and torch.equal(cw[: N * K], ow["codes"][: N * K])
    assert torch.equal(sx, ox["scales"].reshape(-1)) and torch.equal(sw, ow["scales"].reshape(-1))
    if mode == q.CODES_GEMM_OPERAND:
        for c, s, t, rows in ((cx, sx, x, M), (cw, sw, w, N)):
            o = oracle.quantize(inputs.to_f64(t), bits=4, had=128, rms_group=K)
            check_codes_operand(unpack_codes(c.cpu().numpy(), rows, K, 4, 2), o)
            check_f32(s.cpu().numpy()[:, None], o["scale"], 1e-5)
    else:
        for c, s, t, rows in ((cx, sx, x, M), (cw, sw, w, N)):
            o = oracle.quantize_fp4(inputs.to_f64(t), had=128, rms_group=K)
            v = c.cpu().numpy()[: rows * K].view(np.int8).reshape(rows, K) / 2.0
            ex = o["d_round"] <= 1e-5 * np.maximum(np.abs(o["t"]), 1.0)
            assert not ((v != o["value"]) & ~ex).any()
            check_f32(s.cpu().numpy()[:, None], o["scale"], 1e-5)


def test_operands_empty_sides(cuda_device):
    dev = torch.device("cuda:0")
    x = inputs.activations(0, 512, seed=1).to(dev)
    w = inputs.weights(40, 512, seed=2).to(dev)
    (dx, dw) = q.quantize_operands(x, w)
    ow = q.quantize_fwd(w, 4, rms_group=512, code_mode=q.CODES_GEMM_OPERAND, mask_mode=None)
    torch.cuda.synchronize()
    assert torch.equal(dw["codes"][: 40 * 512], ow["codes"][: 40 * 512])
    (dx, dw) = q.quantize_operands(w, x)
    torch.cuda.synchronize()
    assert torch.equal(dx["codes"][: 40 * 512], ow["codes"][: 40 * 512])


def test_operands_full_layer_equals_separate_calls(cuda_device):
    # X 16384 x 2048 and W_up 5632 x 2048: the benchmark's launch
    dev = torch.device("cuda:0")
    x = inputs.activation_input().to(dev)
    w = inputs.weight_up().to(dev)
    dx, dw = q.quantize_operands(x, w)
    ox, ow = separate(x, w, 4, q.CODES_GEMM_OPERAND)
    torch.cuda.synchronize()
    assert torch.equal(dx["codes"], ox["codes"]) and torch.equal(dw["codes"], ow["codes"])
    assert torch.equal(dx["scales"], ox["scales"].reshape(-1)) and torch.equal(dw["scales"], ow["scales"].reshape(-1))

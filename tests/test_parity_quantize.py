"""Parity of quest_quantize_fwd (CUDA, through the C ABI) with the fp64 oracle.

Codes and masks: bit-exact outside the 1e-5 boundary band (see parity.py).
Scales: fp32 within 1e-5 relative (fp32 sum of squares, sqrt and one product:
a few ulp), inside the 2e-3 bound. Dequantised values: bf16 within one ulp of
the correctly rounded oracle value; fp32 within 1e-5 relative.
"""
import numpy as np
import pytest
import torch

import oracle
import bit_quantization_aware_blockwise_b200 as q
from bit_quantization_aware_blockwise_b200 import inputs
from parity import (MASK_EXEMPT_FRAC, MASK_EXEMPT_FRAC_TRUST_BELOW_1, check_bf16, check_codes,
                    check_codes_operand, check_f32, check_mask, unpack_codes, unpack_mask_bits)

pytestmark = pytest.mark.gpu

SCALE_REL = 1e-5


def run_gpu(x_cpu, bits, had=128, rms_group=None, trust=1.0, code_mode=q.CODES_PACKED,
            mask_mode=q.MASK_BITS, dequant="bf16", ld=None):
    dev = torch.device("cuda:0")
    rows, cols = x_cpu.shape
    if ld is not None and ld != cols:
        big = torch.zeros((rows, ld), dtype=x_cpu.dtype)
        big[:, :cols] = x_cpu
        x = big.to(dev)[:, :cols]
    else:
        x = x_cpu.to(dev)
    out = q.quantize_fwd(x, bits, had_block=had, rms_group=rms_group, trust=trust,
                         code_mode=code_mode, mask_mode=mask_mode, dequant=dequant)
    torch.cuda.synchronize()
    res = {"scales": out["scales"].cpu().numpy()}
    res["codes"] = unpack_codes(out["codes"].cpu().numpy(), rows, cols, bits, code_mode)
    if mask_mode == q.MASK_BITS:
        res["mask"] = unpack_mask_bits(out["mask"].cpu().numpy(), rows, cols)
    elif mask_mode == q.MASK_BYTES:
        res["mask"] = out["mask"].cpu().numpy()[: rows * cols].reshape(rows, cols)
    if dequant == "bf16":
        res["deq_bits"] = out["dequant"].cpu().view(torch.int16).numpy().view(np.uint16)
    elif dequant == "fp32":
        res["deq"] = out["dequant"].cpu().numpy().astype(np.float64)
    return res


def check_all(res, o, bits, code_mode=q.CODES_PACKED, rms_group=None, trust=1.0):
    if code_mode == q.CODES_GEMM_OPERAND:
        n_ex = check_codes_operand(res["codes"], o)
        exq = (res["codes"] - 1) // 2 != o["q"]
    else:
        n_ex = check_codes(res["codes"], o)
        exq = res["codes"] != o["q"]
    check_f32(res["scales"], o["scale"], SCALE_REL, what="scales")
    if "mask" in res:
        check_mask(res["mask"], o, MASK_EXEMPT_FRAC if trust >= 1 else MASK_EXEMPT_FRAC_TRUST_BELOW_1)
    if "deq_bits" in res:
        check_bf16(res["deq_bits"], o["yhat"], skip=exq, what="dequant bf16")
    if "deq" in res:
        check_f32(res["deq"], o["yhat"], SCALE_REL, skip=exq, what="dequant fp32")
    return n_ex


def test_smoke_config_fp32_256x512(cuda_device):
    # fp32 [256, 512] N(0,1) seed 0; block 128, RMS per 128-group, b = 4, T = 1:
    # int8 codes, fp32 dequant, byte mask.
    x = inputs.smoke_input()
    o = oracle.quantize(inputs.to_f64(x), bits=4, had=128)
    res = run_gpu(x, 4, code_mode=q.CODES_INT8, mask_mode=q.MASK_BYTES, dequant="fp32")
    n_ex = check_all(res, o, 4, q.CODES_INT8)
    # the exempt set is a property of the data: values within 1e-5 of a boundary
    assert n_ex <= 1e-4 * x.numel()


@pytest.mark.parametrize("bits", [1, 2, 3, 4, 5, 6, 7, 8])
def test_activations_all_bits(cuda_device, bits):
    # Student-t(3) activations with outlier channels, 512 x 2048 (a slice of the
    # 16384 x 2048 workload: 8192 blocks, several waves of warps).
    x = inputs.activation_input(rows=512)
    o = oracle.quantize(inputs.to_f64(x), bits=bits, had=128)
    res = run_gpu(x, bits)
    check_all(res, o, bits)


@pytest.mark.parametrize("had", [16, 32, 64, 128, 256])
def test_hadamard_block_sizes(cuda_device, had):
    x = inputs.activations(37, 1024, seed=5)
    for bits in (2, 4):
        o = oracle.quantize(inputs.to_f64(x), bits=bits, had=had)
        check_all(run_gpu(x, bits, had=had), o, bits)


@pytest.mark.parametrize("rows,cols", [(1, 128), (7, 384), (3, 128 * 45), (33, 640), (130, 256)])
def test_ragged_shapes(cuda_device, rows, cols):
    x = inputs.activations(rows, cols, seed=rows + cols)
    o = oracle.quantize(inputs.to_f64(x), bits=4, had=128)
    check_all(run_gpu(x, 4), o, 4)


def test_row_pitch_larger_than_cols(cuda_device):
    x = inputs.activations(20, 512, seed=8)
    o = oracle.quantize(inputs.to_f64(x), bits=3, had=128)
    check_all(run_gpu(x, 3, ld=776), o, 3)
    o = oracle.quantize(inputs.to_f64(x), bits=4, had=128, rms_group=512)
    check_all(run_gpu(x, 4, ld=776, rms_group=512, code_mode=q.CODES_GEMM_OPERAND), o, 4,
              q.CODES_GEMM_OPERAND)


@pytest.mark.parametrize("cols", [128, 256, 1024, 2048, 5632, 8192, 16384])
def test_row_rms_operand_codes(cuda_device, cols):
    # One RMS per row and int8 c = 2q + 1 codes: the operands of the linear layer.
    rows = max(2, min(64, (1 << 20) // cols))
    x = inputs.activations(rows, cols, seed=cols)
    o = oracle.quantize(inputs.to_f64(x), bits=4, had=128, rms_group=cols)
    res = run_gpu(x, 4, rms_group=cols, code_mode=q.CODES_GEMM_OPERAND, dequant="bf16")
    check_all(res, o, 4, q.CODES_GEMM_OPERAND)


@pytest.mark.parametrize("had,cols", [(16, 8192), (32, 2048), (64, 1024), (256, 4096), (16, 1024)])
def test_row_rms_other_blocks(cuda_device, had, cols):
    x = inputs.weights(9, cols, seed=had)
    o = oracle.quantize(inputs.to_f64(x), bits=2, had=had, rms_group=cols)
    check_all(run_gpu(x, 2, had=had, rms_group=cols), o, 2)


@pytest.mark.parametrize("bits,trust", [(1, 1.3), (2, 1.3), (4, 0.5), (3, 0.8), (8, 2.0)])
def test_trust_factors(cuda_device, bits, trust):
    x = inputs.activations(64, 1024, seed=11)
    o = oracle.quantize(inputs.to_f64(x), bits=bits, had=128, trust=trust)
    check_all(run_gpu(x, bits, trust=trust), o, bits, trust=trust)


def test_zero_groups_and_rows(cuda_device):
    x = inputs.activations(8, 512, seed=3).clone()
    x[0] = 0
    x[3, 128:256] = 0
    for trust in (1.0, 0.5):
        o = oracle.quantize(inputs.to_f64(x), bits=4, had=128, trust=trust)
        check_all(run_gpu(x, 4, trust=trust), o, 4, trust=trust)
        o = oracle.quantize(inputs.to_f64(x), bits=4, had=128, rms_group=512, trust=trust)
        check_all(run_gpu(x, 4, rms_group=512, trust=trust), o, 4, trust=trust)


def test_empty_input(cuda_device):
    x = torch.zeros((0, 256), dtype=torch.bfloat16, device="cuda")
    out = q.quantize_fwd(x, 4)
    torch.cuda.synchronize()
    assert out["scales"].numel() == 0


def _sample_rows(n, k, seed):
    g = np.random.default_rng(seed)
    rows = set(g.choice(n, size=k, replace=False).tolist()) | {0, n - 1}
    return np.array(sorted(rows))


@pytest.mark.parametrize("bits", [1, 2, 3, 4, 8])
def test_full_activation_workload_sampled(cuda_device, bits):
    # The full 16384 x 2048 activation tensor in the launch configuration the
    # benchmark uses; the oracle checks 48 sampled rows (plus the first and last).
    x = inputs.activation_input()
    res = run_gpu(x, bits, dequant="bf16" if bits == 4 else None)
    rows = _sample_rows(x.shape[0], 48, bits)
    o = oracle.quantize(inputs.to_f64(x[rows]), bits=bits, had=128)
    sub = {k: v[rows] for k, v in res.items()}
    check_all(sub, o, bits)


@pytest.mark.parametrize("which,bits", [("up", 1), ("up", 4), ("down", 1), ("down", 4)])
def test_full_weight_workloads_sampled(cuda_device, which, bits):
    w = inputs.weight_up() if which == "up" else inputs.weight_down()
    res = run_gpu(w, bits)
    rows = _sample_rows(w.shape[0], 40, bits + 7)
    o = oracle.quantize(inputs.to_f64(w[rows]), bits=bits, had=128)
    check_all({k: v[rows] for k, v in res.items()}, o, bits)


def test_full_operand_quantization_sampled(cuda_device):
    # The linear layer's operands: X 16384 x 2048 and W_up 5632 x 2048, one RMS per row.
    for t in (inputs.activation_input(), inputs.weight_up()):
        res = run_gpu(t, 4, rms_group=t.shape[1], code_mode=q.CODES_GEMM_OPERAND, dequant=None,
                      mask_mode=None)
        rows = _sample_rows(t.shape[0], 40, 99)
        o = oracle.quantize(inputs.to_f64(t[rows]), bits=4, had=128, rms_group=t.shape[1])
        check_all({k: v[rows] for k, v in res.items()}, o, 4, q.CODES_GEMM_OPERAND)


def test_mask_rate_on_gaussian_rows(cuda_device):
    # A property that holds at any size: with one RMS per long N(0,1) row and T = 1
    # the masked fraction is the Gaussian tail mass beyond alpha_b.
    import scipy.stats
    x = inputs.gaussian(256, 16384, seed=21)
    for bits in (1, 4):
        res = run_gpu(x, bits, rms_group=16384, dequant=None)
        rate = 1.0 - res["mask"].mean()
        p = 2 * scipy.stats.norm.sf(q.alpha(bits))
        n = res["mask"].size
        assert abs(rate - p) < 5 * np.sqrt(p * (1 - p) / n) + 2e-4


@pytest.mark.parametrize("had,cols", [(16, 80), (32, 96), (64, 192), (64, 320)])
def test_rows_not_multiple_of_128_use_the_direct_kernel(cuda_device, had, cols):
    x = inputs.activations(29, cols, seed=cols)
    for bits in (1, 4):
        o = oracle.quantize(inputs.to_f64(x), bits=bits, had=had)
        check_all(run_gpu(x, bits, had=had), o, bits)
        o = oracle.quantize(inputs.to_f64(x), bits=bits, had=had, rms_group=cols)
        check_all(run_gpu(x, bits, had=had, rms_group=cols), o, bits)


@pytest.mark.parametrize("bits", [2, 4, 8])
def test_under_aligned_outputs_use_the_direct_kernel(cuda_device, bits):
    # codes (and mask bits) just past an allocation's start: valid for the ABI, too
    # little alignment for the vector stores of the slab-layout kernels.
    dev = torch.device("cuda:0")
    x_cpu = inputs.activations(40, 512, seed=bits)
    x = x_cpu.to(dev)
    nb = q.codes_bytes(40, 512, bits)
    codes = torch.zeros(nb + 64, dtype=torch.uint8, device=dev)
    mask = torch.zeros(40 * 512 // 8 + 64, dtype=torch.uint8, device=dev)
    scales = torch.zeros(40 * 4, dtype=torch.float32, device=dev)
    # the ABI's own minimum alignment for this container, but not 16 bytes
    off = {1: 1, 2: 2, 4: 4, 8: 8}[q.container_bits(bits)]
    q.quantize_fwd_raw(x.data_ptr(), 0, 40, 512, 512, bits, 128, 128, 1.0, q.CODES_PACKED,
                       codes.data_ptr() + off, scales.data_ptr(), q.MASK_BITS, mask.data_ptr() + 1,
                       None, 0, torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    o = oracle.quantize(inputs.to_f64(x_cpu), bits=bits, had=128)
    res = {"codes": unpack_codes(codes.cpu().numpy()[off:off + nb], 40, 512, bits, q.CODES_PACKED),
           "scales": scales.cpu().numpy().reshape(40, 4),
           "mask": unpack_mask_bits(mask.cpu().numpy()[1:1 + 40 * 64], 40, 512)}
    check_all(res, o, bits)


def test_device_status_is_clean_after_the_suite(cuda_device):
    q.device_status()


@pytest.mark.parametrize("rms", ["group", "row"])
def test_one_bit_outer_trust_from_the_pages(cuda_device, rms):
    # the 1-bit runs widen the outer trust region with the factor s* the pages print
    # (tests/golden/pages_parameters.txt), passed as the trust argument
    from test_oracle_pins import _golden
    s_star = _golden("outer_trust_scale_1bit")
    x = inputs.activations(64, 2048, seed=17)
    rg = 128 if rms == "group" else 2048
    o = oracle.quantize(inputs.to_f64(x), bits=1, had=128, rms_group=rg, trust=s_star)
    res = run_gpu(x, 1, rms_group=rg, trust=s_star)
    check_all(res, o, 1)
    assert 0 < 1 - res["mask"].mean() < 0.2

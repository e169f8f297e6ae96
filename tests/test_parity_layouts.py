"""Parity of quest_quantize_fwd with the oracle across every kernel layout.

The library picks a kernel per call: bf16 input takes the tensor-core layout
(8 slabs per warp step, lane quads per slab), fp32 input the register layout
(two lanes per slab). Each has its own index bookkeeping for every Hadamard
block size, every code container, both mask forms, both dequant types and the
row-RMS shapes of 1, 2, 4, 8 and 16 slabs per row; these cases walk all of them
on small inputs the oracle finishes in seconds.
"""
import pytest

import oracle
import bit_quantization_aware_blockwise_b200 as q
from bit_quantization_aware_blockwise_b200 import inputs
from parity import check_codes_operand
from test_parity_quantize import check_all, run_gpu

pytestmark = pytest.mark.gpu

HADS = [16, 32, 64, 128, 256]


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("had", HADS)
@pytest.mark.parametrize("bits", [1, 2, 4, 8])
def test_group_rms_all_containers(cuda_device, dtype, had, bits):
    # 37 rows x 768: 222 slabs, so the last warp step is ragged in both layouts
    x = inputs.activations(37, 768, seed=had + bits, dtype=dtype)
    o = oracle.quantize(inputs.to_f64(x), bits=bits, had=had)
    check_all(run_gpu(x, bits, had=had), o, bits)


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("had", HADS)
def test_group_rms_byte_mask_fp32_dequant(cuda_device, dtype, had):
    x = inputs.activations(21, 512, seed=had, dtype=dtype)
    o = oracle.quantize(inputs.to_f64(x), bits=3, had=had, trust=1.2)
    res = run_gpu(x, 3, had=had, trust=1.2, code_mode=q.CODES_INT8, mask_mode=q.MASK_BYTES,
                  dequant="fp32")
    check_all(res, o, 3, q.CODES_INT8)


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("had", HADS)
@pytest.mark.parametrize("spr", [1, 2, 4, 8, 16])
def test_row_rms_all_slab_counts(cuda_device, dtype, had, spr):
    cols = 128 * spr
    if had > cols:
        pytest.skip("a Hadamard block wider than the row")
    rows = 27
    x = inputs.activations(rows, cols, seed=spr * 7 + had, dtype=dtype)
    o = oracle.quantize(inputs.to_f64(x), bits=4, had=had, rms_group=cols)
    res = run_gpu(x, 4, had=had, rms_group=cols, code_mode=q.CODES_GEMM_OPERAND)
    check_all(res, o, 4, q.CODES_GEMM_OPERAND)
    o = oracle.quantize(inputs.to_f64(x), bits=2, had=had, rms_group=cols, trust=0.7)
    res = run_gpu(x, 2, had=had, rms_group=cols, trust=0.7, mask_mode=q.MASK_BYTES, dequant="fp32")
    check_all(res, o, 2, trust=0.7)


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("bits", [1, 2, 3, 4])
@pytest.mark.parametrize("rms", ["group", "row"])
def test_e4m3_operand_codes(cuda_device, dtype, bits, rms):
    # c = 2q + 1 stored as FP8 E4M3 (the grouped linear layer's operand)
    x = inputs.activations(45, 1024, seed=bits, dtype=dtype)
    rg = 128 if rms == "group" else 1024
    o = oracle.quantize(inputs.to_f64(x), bits=bits, had=128, rms_group=rg)
    res = run_gpu(x, bits, rms_group=rg, code_mode=q.CODES_GEMM_OPERAND_E4M3, mask_mode=None, dequant=None)
    check_codes_operand(res["codes"], o)


def test_e4m3_operand_codes_reject_wide_codes(cuda_device):
    x = inputs.activations(4, 256, seed=1).to("cuda")
    with pytest.raises(q.QuestError):
        q.quantize_fwd(x, 5, code_mode=q.CODES_GEMM_OPERAND_E4M3, mask_mode=None)

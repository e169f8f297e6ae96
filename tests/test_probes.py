"""The benchmark's tensor-core rate probes (libquest_probe.so): each runs to completion
with its bounded wait satisfied, and reports a rate between a tenth of and twice the
part's nominal dense figure for its kind (so a probe that skipped its MMAs, or timed
nothing, fails)."""
import pytest
import torch

from bit_quantization_aware_blockwise_b200 import _binding as b

NOMINAL_TOPS = {"i8": 4500.0, "bf16": 2250.0, "fp4": 9000.0, "sp_i8": 9000.0, "i8_pair": 4500.0}
K_PER_MMA = {"i8": 32, "bf16": 16, "fp4": 64, "sp_i8": 64, "i8_pair": 32}
M_PER_MMA = {"i8_pair": 256}   # the pair probe: M = 256 per pair of CTAs; the others M = 128 per CTA


def _rate(kind, iters=4000, cp_every=0):
    s = torch.cuda.current_stream()
    launch = {"i8": b.probe_mma_i8, "bf16": b.probe_mma_bf16, "fp4": b.probe_mma_fp4,
              "sp_i8": lambda n, st: b.probe_mma_sp_i8(n, cp_every, st), "i8_pair": b.probe_mma_i8_pair}[kind]
    launch(iters, s.cuda_stream)   # warm-up
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(s)
    ctas = launch(iters, s.cuda_stream)
    t1.record(s)
    torch.cuda.synchronize()
    b.probe_status(s.cuda_stream)   # raises if a completion wait gave up
    ms = t0.elapsed_time(t1)
    units = ctas // 2 if kind == "i8_pair" else ctas
    return 2.0 * M_PER_MMA.get(kind, 128) * 256 * K_PER_MMA[kind] * iters * units / (ms * 1e-3) / 1e12


@pytest.mark.gpu
@pytest.mark.parametrize("kind", ["i8", "bf16", "fp4", "sp_i8", "i8_pair"])
def test_probe_rate_is_plausible(cuda_device, kind):
    tops = _rate(kind)
    assert 0.1 * NOMINAL_TOPS[kind] < tops < 2.0 * NOMINAL_TOPS[kind], f"{kind}: {tops:.0f} TOPS"


@pytest.mark.gpu
def test_sparse_probe_metadata_copies_cost_time(cuda_device):
    # a metadata copy before every MMA can only slow the MMA stream down
    resident = _rate("sp_i8", cp_every=0)
    copied = _rate("sp_i8", cp_every=1)
    assert copied < resident * 1.02, (copied, resident)

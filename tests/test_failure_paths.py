"""The library's error paths, exercised without faulting a GPU.

The library's own failure handling: every entry point reports a status; a launch
failure maps to QUEST_ECUDA with the outputs untouched; a bounded device-side
wait that runs out leaves QUEST_ETIMEOUT for quest_device_status. The faults are
armed on the host (include/quest_debug.h): a simulated launch failure launches
nothing, and the injected timeout makes the integer layer's producer withhold
every operand copy, so its pipeline waits run out after 1 ms with nothing in
flight. The pages define no failure handling; these tests have no passage.
"""
import ctypes

import numpy as np
import pytest
import torch

import bit_quantization_aware_blockwise_b200 as q
import oracle

FAKE = 1 << 20   # an aligned address that is never dereferenced (no launch happens)


def test_injected_launch_failure_on_the_host():
    # No GPU needed: with the fault armed, a call that passes its checks returns
    # QUEST_ECUDA before any CUDA call.
    lib = q.load_library()
    assert lib.quest_debug_inject_fault(7) == 1                      # unknown fault
    assert lib.quest_debug_inject_fault(q.FAULT_LAUNCH) == 0
    # a rejected call (N not a multiple of 8) leaves the fault armed
    assert lib.quest_w4a4_linear(FAKE, FAKE, FAKE, FAKE, 4, 12, 64, FAKE, None, None) == 1
    assert lib.quest_w4a4_linear(FAKE, FAKE, FAKE, FAKE, 4, 16, 64, FAKE, None, None) == 3
    assert b"injected" in lib.quest_last_error_message()
    # every launching entry point honours it
    calls = [
        lambda: lib.quest_quantize_fwd(FAKE, 0, 4, 256, 256, 4, 128, 128, 1.0, 0, FAKE, FAKE, 0, FAKE, None, 0, None),
        lambda: lib.quest_trust_bwd(FAKE, FAKE, 0, 4, 256, 128, FAKE + (1 << 16), None),
        lambda: lib.quest_quantize_operands(FAKE, 4, FAKE + (1 << 16), 8, 256, 0, 4, 128, 2, FAKE + (2 << 16),
                                            FAKE + (3 << 16), FAKE + (4 << 16), FAKE + (5 << 16), None),
        lambda: lib.quest_fp4_linear(FAKE, FAKE, FAKE, FAKE, 4, 16, 64, FAKE, None, None),
        lambda: lib.quest_w4a4_linear_grouped(FAKE, FAKE, FAKE, FAKE, 4, 16, 128, 128, FAKE, None, None),
        lambda: lib.quest_linear_bf16(FAKE, FAKE + (1 << 16), 4, 16, 64, FAKE + (2 << 16), None),
        lambda: lib.quest_transpose_bf16(FAKE, 4, 16, FAKE + (1 << 16), None),
        lambda: lib.quest_trust_bwd_linear(FAKE, FAKE + (1 << 16), FAKE + (2 << 16), 4, 64, 256, 128,
                                           FAKE + (3 << 16), None),
    ]
    for call in calls:
        assert lib.quest_debug_inject_fault(q.FAULT_LAUNCH) == 0
        assert call() == 3
        assert b"injected" in lib.quest_last_error_message()
    assert lib.quest_debug_inject_fault(q.FAULT_NONE) == 0


def _codes(g, rows, K):
    return (2 * g.integers(-8, 8, (rows, K)) + 1).astype(np.int8)


@pytest.mark.gpu
def test_injected_launch_failure_leaves_outputs_untouched(cuda_device):
    g = np.random.default_rng(3)
    M, N, K = 96, 256, 384
    a, w = _codes(g, M, K), _codes(g, N, K)
    sa = g.uniform(0.5, 2, M).astype(np.float32)
    sw = g.uniform(0.5, 2, N).astype(np.float32)
    da, dw = torch.from_numpy(a).cuda(), torch.from_numpy(w).cuda()
    dsa, dsw = torch.from_numpy(sa).cuda(), torch.from_numpy(sw).cuda()
    y = torch.full((M, N), 7.0, dtype=torch.bfloat16, device="cuda")
    acc = torch.full((M, N), -5, dtype=torch.int32, device="cuda")
    q.debug_inject_fault(q.FAULT_LAUNCH)
    with pytest.raises(q.QuestError) as err:
        q.w4a4_linear_raw(da.data_ptr(), dsa.data_ptr(), dw.data_ptr(), dsw.data_ptr(), M, N, K,
                          y.data_ptr(), acc.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert err.value.status == 3 and "injected" in str(err.value)
    torch.cuda.synchronize()
    assert torch.all(y == 7.0) and torch.all(acc == -5)
    q.device_status(torch.cuda.current_stream().cuda_stream)        # nothing ran, nothing set
    # the next call runs normally and is exact
    q.w4a4_linear_raw(da.data_ptr(), dsa.data_ptr(), dw.data_ptr(), dsw.data_ptr(), M, N, K,
                      y.data_ptr(), acc.data_ptr(), torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert np.array_equal(acc.cpu().numpy(), oracle.gemm_i8(a, w))


@pytest.mark.gpu
@pytest.mark.parametrize("M", [64, 300])
def test_injected_wait_timeout_reports_and_recovers(cuda_device, M):
    # The producer withholds its copies: the MMA thread's wait for the first stage
    # runs out after 1 ms, sets the device status word and the CTA's abort flag;
    # the epilogue leaves on the flag; TMEM is freed; the context stays usable.
    g = np.random.default_rng(4)
    N, K = 512, 256
    a, w = _codes(g, M, K), _codes(g, N, K)
    sa = np.ones(M, np.float32)
    sw = np.ones(N, np.float32)
    da, dw = torch.from_numpy(a).cuda(), torch.from_numpy(w).cuda()
    dsa, dsw = torch.from_numpy(sa).cuda(), torch.from_numpy(sw).cuda()
    y = torch.zeros((M, N), dtype=torch.bfloat16, device="cuda")
    acc = torch.zeros((M, N), dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    lib = q.load_library()
    q.debug_inject_fault(q.FAULT_WAIT_TIMEOUT)
    q.w4a4_linear_raw(da.data_ptr(), dsa.data_ptr(), dw.data_ptr(), dsw.data_ptr(), M, N, K,
                      y.data_ptr(), acc.data_ptr(), stream)          # the launch itself succeeds
    assert lib.quest_device_status(ctypes.c_void_p(stream)) == 4     # QUEST_ETIMEOUT
    assert b"gave up" in lib.quest_last_error_message()
    assert lib.quest_device_status(ctypes.c_void_p(stream)) == 0     # read and cleared
    # nothing was accumulated: the epilogue left before reading TMEM
    assert torch.all(acc == 0)
    # the next normal call is exact, and leaves no status behind
    q.w4a4_linear_raw(da.data_ptr(), dsa.data_ptr(), dw.data_ptr(), dsw.data_ptr(), M, N, K,
                      y.data_ptr(), acc.data_ptr(), stream)
    assert lib.quest_device_status(ctypes.c_void_p(stream)) == 0
    assert np.array_equal(acc.cpu().numpy(), oracle.gemm_i8(a, w))

"""Host-side logic of bench.py that needs no GPU: the algorithmic byte counts, the
max-over-ranks timing on a world-size-2 gloo group, and the CPU reference arm."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_part_bytes_by_hand():
    e = 16384 * 2048
    p = bench.part_bytes()
    assert p["quantize_fwd"] == 2 * e + e // 2 + e // 8 + 4 * (e // 128)
    assert p["trust_bwd"] == int(4.125 * e)
    assert p["quantize_operands"] == 3 * e + 4 * 16384 + 3 * 5632 * 2048 + 4 * 5632
    assert p["w4a4_linear"] == 16384 * 2048 + 5632 * 2048 + 4 * (16384 + 5632) + 2 * 16384 * 5632
    assert bench.GEMM_OPS == 2 * 16384 * 5632 * 2048
    assert 590e6 < sum(p.values()) < 595e6


def test_traffic_is_reported_only_for_the_captured_sources(monkeypatch):
    rec = bench.NCU_TRAFFIC["w4a4_linear"]
    # the record's hash is of the sources as they stand, so its bytes are reported
    assert bench.ncu_traffic("w4a4_linear") == rec["dram_read"] + rec["dram_write"]
    assert 200e6 < bench.ncu_traffic("w4a4_linear") < 240e6      # about the 229.7 MB algorithmic
    # any change to the kernel's sources withdraws it
    monkeypatch.setitem(bench.NCU_TRAFFIC, "w4a4_linear", dict(rec, sha256="0" * 64))
    assert bench.ncu_traffic("w4a4_linear") is None
    monkeypatch.setitem(bench.NCU_TRAFFIC, "w4a4_linear", dict(rec, sources=rec["sources"] + ["missing.cu"]))
    assert bench.ncu_traffic("w4a4_linear") is None
    assert bench.ncu_traffic("quantize_fwd") is None


class _FakeNvml:
    """The NVML names the clock sampler reads, with the bit values NVML defines."""
    NVML_CLOCK_SM = 1
    nvmlClocksEventReasonGpuIdle = 0x1
    nvmlClocksEventReasonApplicationsClocksSetting = 0x2
    nvmlClocksEventReasonSwPowerCap = 0x4
    nvmlClocksEventReasonHwSlowdown = 0x8
    nvmlClocksEventReasonSyncBoost = 0x10
    nvmlClocksEventReasonSwThermalSlowdown = 0x20
    nvmlClocksEventReasonHwThermalSlowdown = 0x40
    nvmlClocksEventReasonHwPowerBrakeSlowdown = 0x80

    def __init__(self, seq):
        self.seq = list(seq)

    def nvmlDeviceGetClockInfo(self, h, which):
        return self.seq[0][0]

    def nvmlDeviceGetCurrentClocksEventReasons(self, h):
        return self.seq.pop(0)[1]


def test_clock_summary_from_samples():
    cs = bench.ClockSampler.__new__(bench.ClockSampler)
    cs.ok, cs.samples, cs.max_mhz, cs.h = True, [], 1965, None
    cs.nv = _FakeNvml([(1965, 0x1), (1875, 0x4), (1852, 0x4), (1965, 0x0), (1900, 0x4 | 0x1)])
    for _ in range(5):
        cs.sample_now()
    out = cs.summary()
    assert out == {"sm_mhz": 1900, "sm_max_mhz": 1965, "reasons": ["sw_power_cap"], "samples": 5}
    cs.nv.seq = [(1500, 0x40 | 0x8)]
    cs.sample_now()
    # reasons are the union over the timed region: one throttled sample marks the run
    assert cs.summary()["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_power_cap"]
    # without NVML the line says so instead of guessing a clock
    cs.ok = False
    assert cs.summary()["sm_mhz"] is None and "NVML" in cs.summary()["note"]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.dist_barrier(world)
        ms = bench.dist_max(1.0 + rank * 0.5, world, device="cpu")
        q.put((rank, ms, bench.aggregate_throughput(1e9, world, ms)))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=5) for _ in range(2))
    # both ranks agree on the slowest rank's time; throughput counts both ranks' work
    assert [r[1] for r in res] == [1.5, 1.5]
    assert res[0][2] == pytest.approx(2e9 / 1.5e-3 / 1e9)


def test_reference_arm_runs_on_cpu():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "1", "--warmup", "0"], capture_output=True, text=True,
                         timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr
    line = json.loads(out.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0 and line["unit"] == "GB/s"
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] == 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "1", "--warmup", "0"], capture_output=True, text=True,
                         timeout=120, cwd=ROOT, env=env)
    assert out.returncode == 0 and out.stdout.strip() == ""

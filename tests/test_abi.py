"""C-ABI checks that need no GPU: the library loads, exports every function the
header declares, computes alpha_b on the host, and rejects invalid arguments
before touching the device."""
import ctypes
import math
import os
import re

import pytest

import oracle
import bit_quantization_aware_blockwise_b200 as q
from bit_quantization_aware_blockwise_b200 import _binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


PROBE_HEADER = "quest_probe.h"   # the benchmark's own library, libquest_probe.so


def _declared_functions(probe=False):
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h") and (fn == PROBE_HEADER) == probe:
            with open(os.path.join(ROOT, "include", fn)) as f:
                text = f.read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(quest_\w+)\s*\(", text))
    return names


def test_library_exports_every_declared_symbol():
    lib = q.load_library()
    declared = _declared_functions()
    assert "quest_quantize_fwd" in declared and "quest_w4a4_linear" in declared
    assert "quest_debug_inject_fault" in declared
    for name in sorted(declared):
        assert hasattr(lib, name), name
    # and the binding knows the signature of each
    assert declared == set(_binding.SIGNATURES)


def test_probe_library_is_separate():
    declared = _declared_functions(probe=True)
    assert declared == set(_binding.PROBE_SIGNATURES) and declared
    probe = _binding.load_probe_library()
    for name in sorted(declared):
        assert hasattr(probe, name), name
    # the product library exports only the method's calls (and the debug hook)
    lib = q.load_library()
    for name in sorted(declared):
        assert not hasattr(lib, name), name


def test_version_and_status_strings():
    lib = q.load_library()
    assert lib.quest_version() >= 10000
    for s in range(5):
        assert lib.quest_status_string(s)


@pytest.mark.parametrize("bits", range(1, 9))
def test_alpha_table_matches_oracle(bits):
    # The library finds alpha_b by bisection on the stationarity condition; the
    # oracle by golden-section search on the MSE itself. The golden section only
    # locates a flat minimum to ~sqrt(eps) of its argument.
    a_lib = q.alpha(bits)
    a_ref, _, _ = oracle.alpha(bits)
    assert a_lib == pytest.approx(a_ref, rel=3e-7)


def test_alpha_sparse24_matches_oracle():
    # library: closed-form cell masses, Gauss-Legendre first moments and bisection on
    # the stationarity condition; oracle: Simpson quadrature of the MSE and a
    # golden-section search, which resolves the argmin of a flat minimum to about
    # sqrt(machine epsilon)
    for bits in range(1, 9):
        assert q.alpha_sparse24(bits) == pytest.approx(oracle.alpha_sparse24(bits)[0], rel=1e-7)
    assert math.isnan(q.alpha_sparse24(0)) and math.isnan(q.alpha_sparse24(9))


def test_quantize_sparse24_rejects_invalid_arguments():
    lib = q.load_library()
    ok = dict(x=FAKE, rows=4, cols=256, bits=4, had=128, rg=128, trust=1.0, codes=FAKE, meta=FAKE, scales=FAKE)

    def call(**kw):
        a = dict(ok)
        a.update(kw)
        return lib.quest_quantize_sparse24(a["x"], a["rows"], a["cols"], a["bits"], a["had"], a["rg"], a["trust"],
                                           a["codes"], a["meta"], a["scales"], None, None, None)
    for kw, st in [(dict(bits=8), 1), (dict(bits=0), 1), (dict(had=64), 2), (dict(had=100), 1), (dict(cols=200), 1),
                   (dict(rg=512), 1), (dict(cols=384, rg=384), 2), (dict(trust=0.0), 1), (dict(x=None), 1),
                   (dict(meta=None), 1), (dict(x=FAKE + 8), 1), (dict(codes=FAKE + 4), 1), (dict(rows=-1), 1)]:
        assert call(**kw) == st, kw
    assert call(rows=0, x=None, codes=None, meta=None, scales=None) == 0


def test_alpha_fp4_matches_oracle():
    # library: bisection on the stationarity condition of the E2M1 grid; oracle:
    # golden section on its closed-form Gaussian MSE
    s_ref, _ = oracle.alpha_fp4()
    assert q.alpha_fp4() == pytest.approx(s_ref, rel=3e-7)


def test_alpha_one_bit_exact():
    assert q.alpha(1) == pytest.approx(2 * math.sqrt(2 / math.pi), rel=1e-14)
    assert math.isnan(q.alpha(0)) and math.isnan(q.alpha(9))


def test_sizes():
    assert [q.container_bits(b) for b in range(1, 9)] == [1, 2, 4, 4, 8, 8, 8, 8]
    assert q.codes_bytes(16384, 2048, 4) == 16384 * 2048 // 2
    assert q.codes_bytes(3, 128, 1) == 3 * 16
    assert q.codes_bytes(3, 128, 4, q.CODES_GEMM_OPERAND) == 3 * 128
    assert q.mask_bytes(16384, 2048, q.MASK_BITS) == 16384 * 2048 // 8
    assert q.mask_bytes(2, 128, q.MASK_BYTES) == 256
    assert q.codes_bytes(1, 128, 0) == 0 and q.mask_bytes(1, 12, q.MASK_BITS) == 0
    assert q.codes_bytes(3, 256, 4, q.CODES_FP4_PACKED) == 3 * 128
    assert q.codes_bytes(3, 256, 4, q.CODES_FP4_OPERAND) == 3 * 256
    assert q.codes_bytes(3, 256, 3, q.CODES_FP4_PACKED) == 0


# Invalid calls: the library must return QUEST_EINVAL / EUNSUPPORTED before any
# CUDA call, so these run without a GPU. The pointers are never dereferenced.
FAKE = 1 << 20  # 16-byte aligned, never touched


def _qf(**kw):
    args = dict(x=FAKE, x_dtype=0, rows=4, cols=256, ld_x=256, bits=4, had_block=128,
                rms_group=128, trust=1.0, code_mode=0, codes=FAKE, scales=FAKE, mask_mode=0,
                mask=FAKE, dequant=None, dequant_dtype=0, stream=None)
    args.update(kw)
    lib = q.load_library()
    return lib.quest_quantize_fwd(*args.values())


@pytest.mark.parametrize("kw,status", [
    (dict(bits=0), 1), (dict(bits=9), 1), (dict(had_block=100), 1), (dict(had_block=512), 1),
    (dict(cols=200), 1), (dict(ld_x=128), 1), (dict(rms_group=64), 1), (dict(trust=0.0), 1),
    (dict(trust=-1.0), 1), (dict(trust=float("inf")), 1), (dict(code_mode=7), 1),
    (dict(code_mode=2, bits=8), 1), (dict(x=None), 1), (dict(codes=None), 1),
    (dict(scales=None), 1), (dict(x=FAKE + 4), 1), (dict(ld_x=260), 1),
    (dict(codes=FAKE + 2), 1), (dict(x_dtype=5), 1), (dict(mask_mode=3), 1),
    (dict(dequant=FAKE + 8), 1), (dict(rows=-1), 1),
    (dict(cols=16384 * 2, ld_x=16384 * 2, rms_group=16384 * 2), 2),
    (dict(code_mode=4, bits=3), 1), (dict(code_mode=5, bits=8), 1),
    # the FP4 grid runs only on the slab layouts: rows of 96 columns are not whole slabs
    (dict(code_mode=4, cols=96, ld_x=96, had_block=32, rms_group=32), 2),
    (dict(code_mode=5, cols=96, ld_x=96, had_block=32, rms_group=32), 2),
])
def test_quantize_rejects_invalid_arguments(kw, status):
    assert _qf(**kw) == status
    assert q.load_library().quest_last_error_message()


def test_quantize_zero_rows_is_a_noop():
    assert _qf(rows=0, x=None, codes=None, scales=None, mask=None) == 0


def test_trust_bwd_rejects_invalid_arguments():
    lib = q.load_library()
    ok = dict(g=FAKE, m=FAKE, mm=0, rows=4, cols=256, hb=128, out=FAKE * 4, s=None)
    def call(**kw):
        a = dict(ok); a.update(kw)
        return lib.quest_trust_bwd(*a.values())
    assert call(hb=100) == 1
    assert call(cols=100) == 1
    assert call(mm=2) == 1
    assert call(g=None) == 1
    assert call(out=FAKE + 2) == 1
    assert call(out=FAKE) == 1            # aliasing grad_out
    assert call(mm=1, m=FAKE + 4) == 1    # byte mask misaligned
    assert call(rows=0, g=None, m=None, out=None) == 0


def test_w4a4_rejects_invalid_arguments():
    lib = q.load_library()
    ok = dict(a=FAKE, sa=FAKE, w=FAKE, sw=FAKE, M=128, N=256, K=2048, y=FAKE, acc=None, s=None)
    def call(**kw):
        a = dict(ok); a.update(kw)
        return lib.quest_w4a4_linear(*a.values())
    assert call(K=100) == 1
    assert call(N=100) == 1
    assert call(K=131072) == 1
    assert call(M=-1) == 1
    assert call(a=FAKE + 8) == 1
    assert call(y=None) == 1
    assert call(sa=FAKE + 2) == 1
    assert call(M=0) == 0 and call(N=0) == 0   # empty output: nothing to do


def test_probe_rejects_invalid_arguments():
    lib = _binding.load_probe_library()
    n = ctypes.c_int(0)
    for fn in (lib.quest_probe_mma_i8, lib.quest_probe_mma_fp4, lib.quest_probe_mma_bf16, lib.quest_probe_mma_i8_pair):
        assert fn(0, ctypes.byref(n), None) == 1
        assert fn((1 << 16) + 1, ctypes.byref(n), None) == 1   # cap: far inside the 2 s wait
        assert fn(100, None, None) == 1
    sp = lib.quest_probe_mma_sp_i8
    assert sp(0, 0, ctypes.byref(n), None) == 1
    assert sp((1 << 16) + 1, 2, ctypes.byref(n), None) == 1
    assert sp(100, -1, ctypes.byref(n), None) == 1 and sp(100, 65, ctypes.byref(n), None) == 1
    assert sp(100, 2, None, None) == 1


def test_trust_bwd_linear_rejects_invalid_arguments():
    lib = q.load_library()
    ok = dict(gy=FAKE, wt=FAKE, mask=FAKE, M=4, N=64, K=256, had=128, gx=FAKE)

    def call(**kw):
        a = dict(ok)
        a.update(kw)
        return lib.quest_trust_bwd_linear(a["gy"], a["wt"], a["mask"], a["M"], a["N"], a["K"], a["had"],
                                          a["gx"], None)
    for kw, st in [(dict(M=-1), 1), (dict(K=200), 1), (dict(N=12), 1), (dict(had=64), 2), (dict(had=100), 1),
                   (dict(gx=None), 1), (dict(mask=None), 1), (dict(gy=None), 1), (dict(gy=FAKE + 8), 1),
                   (dict(mask=FAKE + 4), 1), (dict(M=1 << 31), 1),
                   (dict(gx=FAKE + 64), 1)]:                                  # grad_x overlapping grad_y
        assert call(**kw) == st, kw
    assert call(M=0, gy=None, wt=None, mask=None, gx=None) == 0
    assert lib.quest_transpose_bf16(FAKE, -1, 4, FAKE, None) == 1
    assert lib.quest_transpose_bf16(FAKE, 4, 4, FAKE + 8, None) == 1      # overlapping
    assert lib.quest_transpose_bf16(None, 0, 4, None, None) == 0


def test_quantize_operands_rejects_invalid_arguments():
    lib = q.load_library()
    ok = dict(x=FAKE, M=4, w=FAKE, N=8, K=256, dt=0, bits=4, had=128, mode=2, cx=FAKE, sx=FAKE, cw=FAKE, sw=FAKE)

    def call(**kw):
        a = dict(ok)
        a.update(kw)
        return lib.quest_quantize_operands(*a.values(), None)
    for kw in [dict(bits=9), dict(K=200), dict(had=100), dict(mode=7), dict(x=None), dict(cw=None),
               dict(sw=None), dict(w=FAKE + 4), dict(mode=5, bits=3), dict(dt=4)]:
        assert call(**kw) == 1, kw
    assert call(M=0, N=0, x=None, w=None, cx=None, sx=None, cw=None, sw=None) == 0


def test_linear_bf16_rejects_invalid_arguments():
    lib = q.load_library()

    def call(x=FAKE, w=FAKE + (1 << 24), M=4, N=16, K=64, y=FAKE + (1 << 25)):
        return lib.quest_linear_bf16(x, w, M, N, K, y, None)
    for kw in [dict(M=-1), dict(K=12), dict(N=12), dict(y=None), dict(x=None), dict(w=FAKE + 8),
               dict(y=FAKE + 64), dict(M=1 << 31)]:
        assert call(**kw) == 1, kw
    assert call(M=0, x=None, w=None, y=None) == 0


def test_fp4_linear_rejects_invalid_arguments():
    lib = q.load_library()

    def call(a=FAKE, sa=FAKE + (1 << 20), w=FAKE + (1 << 24), sw=FAKE + (1 << 21), M=4, N=16, K=64,
             y=FAKE + (1 << 25), acc=None):
        return lib.quest_fp4_linear(a, sa, w, sw, M, N, K, y, acc, None)
    for kw in [dict(M=-1), dict(K=48), dict(K=16416), dict(N=12), dict(y=None), dict(a=None), dict(sw=None),
               dict(w=FAKE + 8), dict(sa=FAKE + 2), dict(acc=FAKE + 6), dict(y=FAKE + 8), dict(M=1 << 31)]:
        assert call(**kw) == 1, kw
    assert call(M=0, a=None, w=None, sa=None, sw=None, y=None) == 0


def test_grouped_linear_rejects_invalid_arguments():
    lib = q.load_library()

    def call(a=FAKE, sa=FAKE + (1 << 20), w=FAKE + (1 << 24), sw=FAKE + (1 << 21), M=4, N=16, K=256, group=128,
             y=FAKE + (1 << 25), y32=None):
        return lib.quest_w4a4_linear_grouped(a, sa, w, sw, M, N, K, group, y, y32, None)
    for kw in [dict(M=-1), dict(K=200), dict(K=1 << 24), dict(N=12), dict(y=None), dict(a=None), dict(sw=None),
               dict(w=FAKE + 8), dict(sa=FAKE + 2), dict(y32=FAKE + 6), dict(y=FAKE + 8), dict(M=1 << 31)]:
        assert call(**kw) == 1, kw
    assert call(group=64) == 2 and call(group=256) == 2      # the layer takes 128-value groups only
    assert call(M=0, a=None, w=None, sa=None, sw=None, y=None) == 0


def test_sparse24_linear_rejects_invalid_arguments():
    lib = q.load_library()

    def call(x=FAKE, sx=FAKE + (1 << 20), w=FAKE + (1 << 24), meta=FAKE + (1 << 23), sw=FAKE + (1 << 21), M=4,
             N=16, K=256, y=FAKE + (1 << 25), acc=None):
        return lib.quest_w4a4_linear_sparse24(x, sx, w, meta, sw, M, N, K, y, acc, None)
    for kw in [dict(M=-1), dict(K=192), dict(K=131072), dict(N=12), dict(y=None), dict(x=None), dict(meta=None),
               dict(sw=None), dict(w=FAKE + 8), dict(meta=FAKE + 4), dict(sx=FAKE + 2), dict(acc=FAKE + 6),
               dict(y=FAKE + 8), dict(N=1 << 31)]:
        assert call(**kw) == 1, kw
    assert call(N=0, x=None, w=None, meta=None, sx=None, sw=None, y=None) == 0

"""Parity of the 2:4-sparse quantizer (quest_quantize_sparse24) with the oracle.

The format (the pages' 2:4-sparse INT4: atlas.scime.ai summary, ablation table;
pith.science review, results list and Figure 4a; the reading is spelled out in
include/quest.h): transform and RMS as the dense quantizer, keep the two largest
magnitudes of each run of four, quantize the survivors with the step fitted to
surviving values of an N(0,1) input, half-interval trust mask on each value's
total error. Integer outputs must match bit for bit except where the oracle's
pre-round value lies within 1e-5 relative of a decision: a code boundary, a mask
flip point, or (for the choice of survivors) the gap between the 2nd and 3rd
largest magnitude of the run.
"""
import numpy as np
import pytest
import torch

import bit_quantization_aware_blockwise_b200 as q
import oracle
from bit_quantization_aware_blockwise_b200 import inputs
from parity import EXEMPT_REL, check_bf16, check_f32, unpack_mask_bits

pytestmark = pytest.mark.gpu

SCALE_REL = 1e-5


def decompress(codes, meta, rows, cols):
    """Dense c [rows, cols] (0 where pruned) and the kept pattern from the compressed
    codes [rows, cols/2] and the metadata nibbles [rows, cols/8]."""
    codes = np.asarray(codes, dtype=np.int8).reshape(rows, cols // 2).astype(np.int32)
    meta = np.asarray(meta, dtype=np.uint8).reshape(rows, cols // 8).astype(np.int32)
    runs = cols // 4
    nib = np.stack([meta & 0xF, meta >> 4], axis=-1).reshape(rows, runs)
    i0, i1 = nib & 3, nib >> 2
    assert np.all(i0 < i1), "metadata: the kept indices of a run must be increasing"
    dense = np.zeros((rows, runs, 4), dtype=np.int32)
    kept = np.zeros((rows, runs, 4), dtype=np.uint8)
    r_idx, k_idx = np.meshgrid(np.arange(rows), np.arange(runs), indexing="ij")
    dense[r_idx, k_idx, i0] = codes[:, 0::2]
    dense[r_idx, k_idx, i1] = codes[:, 1::2]
    kept[r_idx, k_idx, i0] = 1
    kept[r_idx, k_idx, i1] = 1
    return dense.reshape(rows, cols), kept.reshape(rows, cols)


def check_sparse(res, o, rows, cols, trust=1.0, bits=4):
    dense, kept = decompress(res["codes"], res["meta"], rows, cols)
    t = o["t"]
    # a run is exempt when its 2nd and 3rd largest |t| are within the band
    runmax = np.repeat(np.abs(t).reshape(rows, -1, 4).max(axis=-1), 4, axis=1)
    ex_run = o["d_prune"] <= EXEMPT_REL * np.maximum(runmax, 1.0)
    bad = (kept != o["kept"]) & ~ex_run
    assert not bad.any(), f"kept pattern: {int(bad.sum())} mismatches, first {np.argwhere(bad)[:5].tolist()}"
    # codes of survivors (c = 2q + 1), exact outside the code-boundary band
    ex_code = o["d_round"] <= EXEMPT_REL * np.maximum(np.abs(t), 1.0)
    surv = o["kept"].astype(bool) & ~ex_run
    q_gpu = (dense - 1) // 2
    bad = surv & (q_gpu != o["q"]) & ~ex_code
    assert not bad.any(), f"codes: {int(bad.sum())} mismatches, first {np.argwhere(bad)[:5].tolist()}"
    assert np.all(np.abs(q_gpu - o["q"])[surv & ex_code] <= 1)
    assert np.all(dense[kept == 0] == 0) and np.all(np.abs(dense[kept == 1]) % 2 == 1)
    check_f32(res["scales"], o["scale"], SCALE_REL, what="scales")
    # exempt codes: the band is 2e-5 |t| wide at every integer, and the spread of t
    # grows as 2^(b-1) / alpha_b, so the allowance does too
    n_code = int((surv & ex_code).sum())
    assert n_code <= max(1e-4, 5e-5 * 2 ** (bits - 1)) * rows * cols + 2, f"{n_code} exempt codes"
    n_ex = 0
    if res.get("mask") is not None:
        m = unpack_mask_bits(res["mask"], rows, cols)
        ex_mask = o["d_mask"] <= EXEMPT_REL * np.maximum(np.abs(t), 1.0)
        bad = (m != o["mask"]) & ~ex_mask & ~ex_run
        assert not bad.any(), f"mask: {int(bad.sum())} mismatches, first {np.argwhere(bad)[:5].tolist()}"
        n_ex += int((ex_mask & ~ex_run).sum())
    if res.get("deq_bits") is not None:
        skip = ex_run | (surv & ex_code)
        check_bf16(res["deq_bits"], o["yhat"], skip=skip, what="dequant bf16")
    # exempt mask bits outside exempt runs, as for the dense quantizer; and exempt runs
    # (a prune tie exempts its four values) at most 1e-4 of the runs
    frac = 1e-4 if trust >= 1 else 5e-4
    assert n_ex <= frac * rows * cols + 2, f"{n_ex} exempt mask bits of {rows * cols}"
    n_runs = int(ex_run.sum()) // 4
    assert n_runs <= 1e-4 * rows * cols / 4 + 2, f"{n_runs} exempt runs of {rows * cols // 4}"
    return n_code + n_ex + 4 * n_runs


def run(x, bits, rms_group=128, trust=1.0, dequant=True):
    out = q.quantize_sparse24(x.to("cuda"), bits, rms_group=rms_group, trust=trust, dequant=dequant)
    torch.cuda.synchronize()
    res = {"codes": out["codes"].cpu().numpy(), "meta": out["meta"].cpu().numpy(),
           "scales": out["scales"].cpu().numpy(), "mask": out["mask"].cpu().numpy().view(np.uint8)}
    if dequant:
        res["deq_bits"] = out["dequant"].cpu().view(torch.int16).numpy().view(np.uint16)
    return res


@pytest.mark.parametrize("bits,trust", [(4, 1.0), (2, 0.7), (1, 1.3), (7, 1.0), (3, 2.0)])
def test_activations_group_rms(cuda_device, bits, trust):
    # Student-t(3) activations with outlier channels; 37 rows x 768 (ragged last warp step)
    x = inputs.activations(37, 768, seed=40 + bits)
    o = oracle.quantize_sparse24(inputs.to_f64(x), bits=bits, had=128, trust=trust)
    check_sparse(run(x, bits, trust=trust), o, 37, 768, trust, bits)


@pytest.mark.parametrize("spr", [1, 2, 4, 8, 16])
def test_row_rms_all_slab_counts(cuda_device, spr):
    cols = 128 * spr
    x = inputs.weights(45, cols, seed=spr)
    o = oracle.quantize_sparse24(inputs.to_f64(x), bits=4, had=128, rms_group=cols)
    check_sparse(run(x, 4, rms_group=cols), o, 45, cols)


@pytest.mark.parametrize("rms", ["group", 1, 2, 4, 8, 16])
def test_codes_and_metadata_only(cuda_device, rms):
    # without mask and dequant the kernels run with the optional outputs compiled out;
    # codes, metadata and scales must match the oracle and, bit for bit, the run that
    # writes every output
    cols = 768 if rms == "group" else 128 * rms
    rg = 128 if rms == "group" else cols
    x = inputs.activations(45, cols, seed=50 + cols)
    o = oracle.quantize_sparse24(inputs.to_f64(x), bits=4, had=128, rms_group=rg)
    lean = q.quantize_sparse24(x.cuda(), 4, rms_group=rg, mask=False, dequant=False)
    full = q.quantize_sparse24(x.cuda(), 4, rms_group=rg, mask=True, dequant=True)
    torch.cuda.synchronize()
    assert lean["mask"] is None and lean["dequant"] is None
    for k in ("codes", "meta", "scales"):
        assert torch.equal(lean[k], full[k]), k
    check_sparse({"codes": lean["codes"].cpu().numpy(), "meta": lean["meta"].cpu().numpy(),
                  "scales": lean["scales"].cpu().numpy()}, o, 45, cols)


def test_activation_slice_full_width(cuda_device):
    # 512 rows of the 16384 x 2048 activation workload
    x = inputs.activations(512, 2048, seed=1)
    o = oracle.quantize_sparse24(inputs.to_f64(x), bits=4, had=128)
    check_sparse(run(x, 4), o, 512, 2048)


def test_zero_group_and_zero_rows(cuda_device):
    x = inputs.activations(5, 512, seed=3)
    x[2, 128:256] = 0
    o = oracle.quantize_sparse24(inputs.to_f64(x), bits=4, had=128)
    res = run(x, 4)
    check_sparse(res, o, 5, 512)
    _, kept = decompress(res["codes"], res["meta"], 5, 512)
    assert np.array_equal(kept[2, 128:256], np.tile([1, 1, 0, 0], 32))
    out = q.quantize_sparse24(torch.empty((0, 512), dtype=torch.bfloat16, device="cuda"), 4)
    assert out["codes"].numel() == 0


def test_weight_up_full_size(cuda_device):
    # the 5632 x 2048 up-projection, one RMS per row: the operand of the sparse layer
    x = inputs.weight_up()
    o = oracle.quantize_sparse24(inputs.to_f64(x), bits=4, had=128, rms_group=2048)
    check_sparse(run(x, 4, rms_group=2048, dequant=False), o, 5632, 2048)


# ---------------------------------------------------------------------------
# The layer on the sparse tensor cores
# ---------------------------------------------------------------------------

def compress(dense_c, kept):
    """Test-side compression of dense codes with exactly two survivors per run of four:
    the survivors' codes in index order and the metadata nibbles."""
    rows, cols = dense_c.shape
    runs = cols // 4
    kp = kept.reshape(rows, runs, 4).astype(bool)
    assert np.all(kp.sum(axis=-1) == 2)
    idx = np.argsort(~kp, axis=-1, kind="stable")[..., :2]          # the kept indices, increasing
    vals = np.take_along_axis(dense_c.reshape(rows, runs, 4), idx, axis=-1)
    nib = (idx[..., 0] | (idx[..., 1] << 2)).astype(np.uint8)
    meta = (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)
    return vals.reshape(rows, cols // 2).astype(np.int8), meta


def random_sparse_codes(rows, cols, seed, lim=15):
    g = np.random.default_rng(seed)
    dense = (2 * g.integers(-(lim + 1) // 2, (lim + 1) // 2, (rows, cols)) + 1).astype(np.int32)
    kept = np.zeros((rows, cols // 4, 4), dtype=np.uint8)
    choice = np.array([[0, 1], [0, 2], [0, 3], [1, 2], [1, 3], [2, 3]])
    pick = choice[g.integers(0, 6, (rows, cols // 4))]
    np.put_along_axis(kept, pick, 1, axis=-1)
    kept = kept.reshape(rows, cols)
    return dense * kept, kept


def run_sparse_layer(xc, sx, wc, meta, sw):
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    y, acc = q.w4a4_linear_sparse24(t(xc), t(sx), t(wc), t(meta), t(sw), acc=True)
    torch.cuda.synchronize()
    q.device_status()
    return y.cpu().view(torch.int16).numpy().view(np.uint16), acc.cpu().numpy()


@pytest.mark.parametrize("M,N,K", [(224, 128, 128), (300, 136, 384), (17, 8, 128), (450, 264, 1024),
                                   (1000, 520, 2048), (300, 264, 2304), (600, 520, 4096), (256, 264, 16384),
                                   (40, 64, 8192)])
def test_sparse_layer_accumulator_exact(cuda_device, M, N, K):
    # ragged tiles in both directions, several waves, K of one to sixteen stages (the
    # metadata resident in TMEM) and beyond (2304 to 16384: the metadata staged per
    # stage, in the CTA-pair and the one-CTA kernel)
    g = np.random.default_rng(M + N + K)
    xc = (2 * g.integers(-8, 8, (M, K)) + 1).astype(np.int8)
    wd, kept = random_sparse_codes(N, K, seed=K)
    wc, meta = compress(wd, kept)
    sx = g.uniform(0.5, 2.0, M).astype(np.float32)
    sw = g.uniform(0.5, 2.0, N).astype(np.float32)
    y, acc = run_sparse_layer(xc, sx, wc, meta, sw)
    ref = oracle.gemm_i8(xc, wd.astype(np.int8))
    assert np.array_equal(acc, ref)
    check_bf16(y, oracle.dequant_linear(ref, sx.astype(np.float64), sw.astype(np.float64)), what="y")


@pytest.mark.parametrize("M,N,K", [(4000, 1288, 640), (3600, 1096, 2048)])
def test_sparse_layer_weight_tile_changes(cuda_device, M, N, K):
    # more tiles than CTA pairs: each pair walks a run of tiles in weight-major order
    # and reloads the resident metadata where the run crosses into the next 256 weight
    # rows; rows sampled from every token tile, against the exact product
    g = np.random.default_rng(M + K)
    xc = (2 * g.integers(-8, 8, (M, K)) + 1).astype(np.int8)
    wd, kept = random_sparse_codes(N, K, seed=K + 1)
    wc, meta = compress(wd, kept)
    sx = g.uniform(0.5, 2.0, M).astype(np.float32)
    sw = g.uniform(0.5, 2.0, N).astype(np.float32)
    y, acc = run_sparse_layer(xc, sx, wc, meta, sw)
    rows = np.unique(np.concatenate([np.arange(0, M, 224), np.arange(223, M, 224), g.integers(0, M, 64), [M - 1]]))
    ref = oracle.gemm_i8(np.ascontiguousarray(xc[rows]), wd.astype(np.int8))
    assert np.array_equal(acc[rows], ref)
    check_bf16(y[rows], oracle.dequant_linear(ref, sx[rows].astype(np.float64), sw.astype(np.float64)), what="y")


def test_sparse_layer_full_shape_sampled(cuda_device):
    # 16384 x 5632 x 2048, the launch the configs time: seeded b = 4 activation codes and
    # random 2:4-sparse weight codes; the oracle recomputes a 24 x 24 grid of outputs
    M, N, K = inputs.TOKENS, inputs.MLP_WIDTH, inputs.HIDDEN
    xc = inputs.gemm_codes(M, K, seed=41)
    wd, kept = random_sparse_codes(N, K, seed=42)
    wc, meta = compress(wd, kept)
    sx, sw = inputs.positive_scales(M, 43), inputs.positive_scales(N, 44)
    y, acc = run_sparse_layer(xc, sx, wc, meta, sw)
    g = np.random.default_rng(45)
    rows = np.unique(np.concatenate([[0, M - 1], g.choice(M, 22, replace=False)]))
    cols = np.unique(np.concatenate([[0, N - 1], g.choice(N, 22, replace=False)]))
    ref = oracle.gemm_i8(np.ascontiguousarray(xc[rows]), np.ascontiguousarray(wd[cols].astype(np.int8)))
    assert np.array_equal(acc[np.ix_(rows, cols)].astype(np.int64), ref)
    check_bf16(y[np.ix_(rows, cols)], oracle.dequant_linear(ref, sx[rows].astype(np.float64),
                                                            sw[cols].astype(np.float64)), what="y (sampled)")


def test_sparse_layer_extreme_codes(cuda_device):
    # every survivor +-127 against +-127: |acc| = 127^2 K / 2 at K = 2048 (no overflow)
    M, N, K = 256, 128, 2048
    g = np.random.default_rng(5)
    xc = np.where(g.random((M, K)) < 0.5, 127, -127).astype(np.int8)
    wd, kept = random_sparse_codes(N, K, seed=6)
    wd = np.where(kept == 1, np.where(g.random((N, K)) < 0.5, 127, -127), 0).astype(np.int32)
    xc[0] = 127
    wd[0] = 127 * kept[0]
    wc, meta = compress(wd, kept)
    y, acc = run_sparse_layer(xc, np.ones(M, np.float32), wc, meta, np.ones(N, np.float32))
    assert np.array_equal(acc, oracle.gemm_i8(xc, wd.astype(np.int8)))
    assert acc[0, 0] == 127 * 127 * K // 2


def test_sparse_layer_end_to_end(cuda_device):
    # activations through quest_quantize_operands (one RMS per row, c = 2q + 1), the
    # up-projection slice through quest_quantize_sparse24 (one RMS per row); the layer
    # against the oracle's product on the oracle's own codes
    x = inputs.activations(512, 2048, seed=1)
    w = inputs.weight_up()[:768]
    ox = oracle.quantize(inputs.to_f64(x), bits=4, had=128, rms_group=2048)
    ow = oracle.quantize_sparse24(inputs.to_f64(w), bits=4, had=128, rms_group=2048)
    opx, _ = q.quantize_operands(x.cuda(), w.cuda()[:0], 4, 128, q.CODES_GEMM_OPERAND)
    xcodes_t = opx["codes"][: 512 * 2048].view(torch.int8).view(512, 2048)
    sw = q.quantize_sparse24(w.cuda(), 4, rms_group=2048, mask=False)
    y, acc = q.w4a4_linear_sparse24(xcodes_t, opx["scales"], sw["codes"], sw["meta"], sw["scales"], acc=True)
    torch.cuda.synchronize()
    # the GPU's own codes must match the oracle's (outside the exemption bands)...
    dense, kept = decompress(sw["codes"].cpu().numpy(), sw["meta"].cpu().numpy(), 768, 2048)
    check_sparse({"codes": sw["codes"].cpu().numpy(), "meta": sw["meta"].cpu().numpy(),
                  "scales": sw["scales"].cpu().numpy()}, ow, 768, 2048)
    # ...and the layer on those codes is the exact integer product
    xcodes = xcodes_t.cpu().numpy()
    assert np.array_equal(acc.cpu().numpy(), oracle.gemm_i8(xcodes, dense.astype(np.int8)))
    ref = oracle.dequant_linear(oracle.gemm_i8(xcodes, dense.astype(np.int8)),
                                opx["scales"].cpu().numpy().astype(np.float64),
                                sw["scales"].cpu().numpy().reshape(-1).astype(np.float64))
    check_bf16(y.cpu().view(torch.int16).numpy().view(np.uint16), ref, what="y")

"""Seeded synthetic inputs shaped like the QuEST pages' workloads.

This module is the one piece shared by the product's benchmark and the oracle
tests. It draws random numbers and lays them out; it holds none of the method's
arithmetic (no transform, no RMS, no grid, no mask rule).

The pages measure on a Llama-family model trained on C4 (atlas.scime.ai summary,
"Experimental setup"; pith.science review, Figure 5 caption); neither the trained
weights nor the data are available, so these tensors stand in for them:
Gaussian weights, heavy-tailed activations with a few outlier channels, and
small Gaussian upstream gradients, at the Llama MLP shapes that follow the
"8/3 of the hidden size, padded to 256" rule (hidden 2048 -> 5632).

All tensors are drawn in fp32 with numpy's PCG64 ``default_rng(seed)`` and, for
bf16 inputs, rounded to bfloat16 by torch (round-to-nearest-even), so every
consumer sees identical bits.
"""
from __future__ import annotations

import numpy as np
import torch

HIDDEN = 2048
MLP_WIDTH = 5632      # 8/3 * 2048 = 5461.3, padded up to a multiple of 256
TOKENS = 16384


def rng(seed: int) -> np.random.Generator:
    return np.random.default_rng(seed)


def as_dtype(a32: np.ndarray, dtype: str) -> torch.Tensor:
    """fp32 numpy -> CPU torch tensor of ``dtype`` ("bf16" or "fp32")."""
    t = torch.from_numpy(np.ascontiguousarray(a32, dtype=np.float32))
    if dtype == "bf16":
        return t.to(torch.bfloat16)
    if dtype == "fp32":
        return t.clone()
    raise ValueError(f"unknown dtype {dtype!r}")


def to_f64(t: torch.Tensor) -> np.ndarray:
    """Exact fp64 values of a bf16/fp32 CPU tensor."""
    return t.detach().to("cpu", torch.float64).numpy()


def gaussian(rows: int, cols: int, seed: int, std: float = 1.0, dtype: str = "bf16") -> torch.Tensor:
    """iid N(0, std^2) entries."""
    a = rng(seed).standard_normal((rows, cols), dtype=np.float32) * np.float32(std)
    return as_dtype(a, dtype)


def activations(rows: int, cols: int, seed: int, nu: float = 3.0, n_outliers: int = 16,
                outlier_scale: float = 20.0, dtype: str = "bf16") -> torch.Tensor:
    """Student-t(nu) entries (unscaled), with ``n_outliers`` distinct random channels
    (columns) multiplied by ``outlier_scale``: heavy-tailed LLM-like activations."""
    g = rng(seed)
    a = g.standard_t(nu, size=(rows, cols)).astype(np.float32)
    k = min(n_outliers, cols)
    if k > 0:
        cols_sel = g.choice(cols, k, replace=False)
        a[:, cols_sel] *= np.float32(outlier_scale)
    return as_dtype(a, dtype)


def weights(rows: int, cols: int, seed: int, std: float = 0.02, dtype: str = "bf16") -> torch.Tensor:
    """Random-init linear weights, N(0, std^2)."""
    return gaussian(rows, cols, seed, std, dtype)


def upstream_grad(rows: int, cols: int, seed: int, std: float = 1e-3) -> torch.Tensor:
    """Upstream gradient in the Hadamard domain, N(0, std^2), bf16."""
    return gaussian(rows, cols, seed, std, "bf16")


def random_mask(rows: int, cols: int, seed: int, keep_prob: float) -> np.ndarray:
    """0/1 uint8 mask, 1 with probability ``keep_prob`` independently."""
    return (rng(seed).random((rows, cols)) < keep_prob).astype(np.uint8)


def pack_mask_bits(mask01: np.ndarray) -> np.ndarray:
    """Lay a 0/1 [rows, cols] mask out as uint32 words [rows, cols/32]:
    bit j of word w holds column 32*w + j."""
    m = np.ascontiguousarray(mask01, dtype=np.uint8)
    rows, cols = m.shape
    if cols % 32:
        raise ValueError("cols must be a multiple of 32")
    by = np.packbits(m.reshape(rows, cols // 8, 8), axis=-1, bitorder="little")
    return by.reshape(rows, cols // 8).view(np.uint32).reshape(rows, cols // 32).copy()


def gemm_codes(rows: int, cols: int, seed: int, bits: int = 4) -> np.ndarray:
    """Odd integer operands c in [-(2^bits - 1), 2^bits - 1], uniform: the value set
    of the c = 2q+1 operand form of a b-bit code, at its full range."""
    half = 1 << (bits - 1)
    q = rng(seed).integers(-half, half, size=(rows, cols))
    return (2 * q + 1).astype(np.int8)


def fp4_codes(rows: int, cols: int, seed: int) -> np.ndarray:
    """Packed 4-bit codes [rows, cols/2] bytes, every nibble uniform over its 16 values
    (two per byte, element 2j in the low nibble)."""
    return rng(seed).integers(0, 256, size=(rows, cols // 2)).astype(np.uint8)


def positive_scales(n: int, seed: int, lo: float = 1e-3, hi: float = 5e-2) -> np.ndarray:
    """Positive fp32 per-row scale factors, log-uniform in [lo, hi]."""
    u = rng(seed).random(n)
    return np.exp(np.log(lo) + u * (np.log(hi) - np.log(lo))).astype(np.float32)


# ---------------------------------------------------------------------------
# The workloads, by name. Sizes default to the full Llama-style shapes; tests
# pass smaller row counts to keep the oracle fast.
# ---------------------------------------------------------------------------

def smoke_input(rows: int = 256, cols: int = 512) -> torch.Tensor:
    """fp32 [256, 512] iid N(0,1), seed 0."""
    return gaussian(rows, cols, seed=0, dtype="fp32")


def activation_input(rows: int = TOKENS, cols: int = HIDDEN) -> torch.Tensor:
    """bf16 [16384, 2048] Student-t(3) activations with 16 outlier channels x20, seed 1."""
    return activations(rows, cols, seed=1)


def weight_up(rows: int = MLP_WIDTH, cols: int = HIDDEN) -> torch.Tensor:
    """bf16 [5632, 2048] up-projection weights N(0, 0.02^2), seed 2."""
    return weights(rows, cols, seed=2)


def weight_down(rows: int = HIDDEN, cols: int = MLP_WIDTH) -> torch.Tensor:
    """bf16 [2048, 5632] down-projection weights N(0, 0.02^2), seed 3."""
    return weights(rows, cols, seed=3)


def grad_input(rows: int = TOKENS, cols: int = HIDDEN) -> torch.Tensor:
    """bf16 [16384, 2048] upstream gradient N(0, 1e-3^2), seed 4."""
    return upstream_grad(rows, cols, seed=4)


def layer_output_grad(rows: int = TOKENS, cols: int = MLP_WIDTH) -> torch.Tensor:
    """bf16 [16384, 5632] gradient of the up-projection's output, N(0, 1e-3^2), seed 5."""
    return upstream_grad(rows, cols, seed=5)

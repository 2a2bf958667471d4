"""NVFP4 storage of the first moment (momentum) for Q-Root, step by step.

TEST INFRASTRUCTURE ONLY: imported by tests and by the smoke check; never by the
product path.  (The CPU-baseline leg of bench.py times the C++ restatement of the
same steps, oracle/cpp/fs4_oracle.cpp, which the tests pin to this module bit for bit.)

Source: "Full-Stack FP4" (arXiv 2607.04422), Section 3.3 "Quantized-State AdamW": for
the first moment, Hadamard mixing smooths the distribution before stochastic rounding
(SR) and adaptive 4/6 quantisation; Section 3.4: Q-Root's first-order momentum follows
that storage recipe.

Readings taken where the pages are silent:
  * Update: m_t = fp32(fp32(beta * m_prev) + fp32(fp32(1 - beta) * g)), m_prev the
    decoded previous state (zero on the first step).
  * Storage: y = m_t H16^r (the FP32 butterfly of nvfp4.hadamard_rows with the caller's
    sign mask), quantised in 1x16 row blocks with the adaptive 4/6 rule of
    nvfp4.quantize_rows (tensor scale by the 1792 rule, block scales round to nearest,
    M = 4 kept only when its FP32 squared error is strictly smaller), except that every
    element code is rounded stochastically: for v = fp32(|y| / den) below 6, with lo
    and hi the E2M1 magnitudes around v, the code is hi when u < (v - lo) / (hi - lo)
    and lo otherwise (the fraction is exact in FP32: hi - lo is a power of two and
    v - lo is exact); v >= 6 gives 6.  Both 4/6 candidates use the same u.
  * Decoding: the FP32 dequantised state (fp32(fp32(code * s_b) * s_g)) times the inverse
    transform (H16^r)^-1 = H16 D / 4: the same butterfly, the exact * 0.25, then the signs.
  * u for element i (row-major index in the m x n matrix) is the top 24 bits of
    SplitMix64 (Steele, Lea and Flood, "Fast splittable pseudorandom number generators",
    OOPSLA 2014): z = seed + (i + 1) * 0x9E3779B97F4A7C15 (mod 2^64), mixed by
    z ^= z >> 30, z *= 0xBF58476D1CE4E5B9, z ^= z >> 27, z *= 0x94D049BB133111EB,
    z ^= z >> 31; u = (z >> 40) * 2^-24.
"""
from __future__ import annotations

import numpy as np

from . import nvfp4
from .nvfp4 import BLOCK, E2M1_MAGNITUDES, E4M3_VALUES

GOLDEN_GAMMA = np.uint64(0x9E3779B97F4A7C15)


def splitmix64(seed: int, idx: np.ndarray) -> np.ndarray:
    """SplitMix64 output for counter values idx (the (idx + 1)-th output of a generator
    started at `seed`), uint64."""
    with np.errstate(over="ignore"):
        z = np.uint64(seed) + (np.asarray(idx, dtype=np.uint64) + np.uint64(1)) * GOLDEN_GAMMA
        z = (z ^ (z >> np.uint64(30))) * np.uint64(0xBF58476D1CE4E5B9)
        z = (z ^ (z >> np.uint64(27))) * np.uint64(0x94D049BB133111EB)
        z = z ^ (z >> np.uint64(31))
    return z


def uniform24(seed: int, idx: np.ndarray) -> np.ndarray:
    """FP32 u in [0, 1): the top 24 bits of splitmix64 times 2^-24 (exact)."""
    return ((splitmix64(seed, idx) >> np.uint64(40)).astype(np.float64) * 2.0 ** -24).astype(np.float32)


def sr_encode_magnitude(v: np.ndarray, u: np.ndarray) -> np.ndarray:
    """Stochastic rounding of FP32 v >= 0 onto E2M1 codes 0..7 with FP32 u in [0, 1)."""
    v = np.asarray(v, dtype=np.float32)
    u = np.asarray(u, dtype=np.float32)
    if not np.all(np.isfinite(v)) or np.any(v < 0):
        raise ValueError("SR encode expects finite non-negative inputs")
    grid = E2M1_MAGNITUDES
    lo = np.clip(np.searchsorted(grid, v.astype(np.float64), side="right") - 1, 0, 7)
    hi = np.minimum(lo + 1, 7)
    gap = (grid[hi] - grid[lo]).astype(np.float32)
    frac = np.where(gap > 0, (v - grid[lo].astype(np.float32)) / np.where(gap > 0, gap, 1), 0)
    up = (u < frac.astype(np.float32)) & (lo < 7)
    return np.where(v >= np.float32(6.0), 7, np.where(up, hi, lo)).astype(np.uint8)


def _quantize_blocks_sr(blocks, s_g, M, u):
    """As nvfp4._quantize_blocks, with stochastically rounded element codes."""
    amax_b = np.max(np.abs(blocks), axis=2)
    v = amax_b / (np.float32(M) * s_g)                       # FP32 division
    scales = nvfp4.e4m3_encode(v)
    den = E4M3_VALUES[scales].astype(np.float32) * s_g       # FP32 product
    safe = np.where(den > 0, den, np.float32(1.0)).astype(np.float32)
    q = np.abs(blocks) / safe[:, :, None]                    # FP32 division
    mag = sr_encode_magnitude(q, u)
    sign = np.signbit(blocks).astype(np.uint8) << 3
    nib = np.where((den > 0)[:, :, None], mag | sign, 0).astype(np.uint8)
    deq = (nvfp4.code_values(nib) * den[:, :, None]).astype(np.float32)
    return nib, scales, deq


def store(m_t: np.ndarray, mask: int, seed: int):
    """NVFP4 state of the FP32 momentum m_t: (codes, scales, s_g) of Q(m_t H16^r) with
    SR element codes and adaptive 4/6 block scales (1x16 row blocks, plain layout)."""
    m_t = np.asarray(m_t, dtype=np.float32)
    rows, cols = m_t.shape
    y = nvfp4.hadamard_rows(m_t, mask)
    amax = float(np.max(np.abs(y))) if y.size else 0.0
    s_g = nvfp4.global_scale(amax, "pow2", nvfp4.SG_DENOM_46)
    blocks = y.reshape(rows, cols // BLOCK, BLOCK)
    u = uniform24(seed, np.arange(rows * cols, dtype=np.uint64)).reshape(blocks.shape)
    nib6, sc6, deq6 = _quantize_blocks_sr(blocks, s_g, 6.0, u)
    nib4, sc4, deq4 = _quantize_blocks_sr(blocks, s_g, 4.0, u)
    use4 = nvfp4._block_sq_error_f32(blocks, deq4) < nvfp4._block_sq_error_f32(blocks, deq6)
    nib = np.where(use4[:, :, None], nib4, nib6).reshape(rows, cols)
    scales = np.where(use4, sc4, sc6).astype(np.uint8)
    codes = (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)
    return codes, scales, s_g


def inverse_hadamard_rows(y: np.ndarray, mask: int) -> np.ndarray:
    """FP32 y (H16^r)^-1 = y H16 D / 4 on every 16-element block: the butterfly of
    nvfp4.hadamard_rows without its leading signs, the exact * 0.25, then the signs."""
    y = np.asarray(y, dtype=np.float32)
    rows, cols = y.shape
    t = nvfp4.hadamard_rows(y, 0)              # butterfly then * 0.25 (mask 0: no signs)
    t = t.reshape(rows, cols // BLOCK, BLOCK) * nvfp4.mask_signs(mask).astype(np.float32)
    return t.astype(np.float32).reshape(rows, cols)


def load(codes, scales, s_g, mask: int) -> np.ndarray:
    """FP32 momentum decoded from a state written by store()."""
    return inverse_hadamard_rows(nvfp4.dequantize_rows(codes, scales, s_g, dtype=np.float32), mask)


def update(g: np.ndarray, beta: float, state=None, mask_prev: int = 0, mask_next: int = 0,
           seed: int = 0):
    """One momentum step: returns (m_t FP32, new state (codes, scales, s_g))."""
    g = np.asarray(g, dtype=np.float32)
    m_prev = np.zeros_like(g) if state is None else load(*state, mask_prev)
    b = np.float32(beta)
    omb = np.float32(np.float32(1.0) - b)
    m_t = ((b * m_prev).astype(np.float32) + (omb * g).astype(np.float32)).astype(np.float32)
    return m_t, store(m_t, mask_next, seed)

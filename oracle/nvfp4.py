"""NVFP4 codecs and 1x16 block quantisation, written out from the format definition.

TEST INFRASTRUCTURE ONLY: imported by tests, by the smoke check and by the
CPU-baseline leg of bench.py; never by the product path.

Source: "Full-Stack FP4" (arXiv 2607.04422), Section 2 "Preliminaries",
paragraph "NVFP4 format": E2M1 elements (1 sign, 2 exponent, 1 mantissa bit),
one FP8 E4M3 scale per block of 1x16 elements, one FP32 tensor scale s_g, and
x_hat = x_E2M1 * s * s_g.  Section 3.4 and the "Others" paragraph of Section 2:
all quantisations round to nearest (RTN).

Readings taken where the pages are silent:
  * RTN is IEEE round-to-nearest, ties to the even code, saturating at the
    largest finite value (E2M1: 6, E4M3: 448).
  * Block scale s_b = RN_e4m3( fp32( amax_b / fp32(6 * s_g) ) ); element code
    = sign | RN_e2m1( fp32( |x| / fp32(dec(s_b) * s_g) ) ).  Both divisions are
    IEEE FP32 divisions: the decision is taken in the precision of the tensors
    being quantised (FP32).  A block whose scale rounds to 0 gets all codes 0.
  * Tensor scale s_g (default "pow2"): the smallest power of two 2^e with
    6 * 448 * 2^e >= amax, e clamped to [-116, 118]; s_g = 1 for an all-zero
    tensor.  The "amax" mode is the common s_g = fp32(amax / 2688).
  * Packing: byte j of a block row holds element 2j in its low nibble and
    element 2j+1 in its high nibble; a nibble is (sign, e1, e0, m).

Everything here is plain numpy: nearest-value searches over the full code
tables, no bit tricks, so it can be checked against the definition by eye.
"""
from __future__ import annotations

import math

import numpy as np

E2M1_MAX = 6.0
E4M3_MAX = 448.0
SG_DENOM = E2M1_MAX * E4M3_MAX  # 2688: largest |x| one tensor scale unit covers
SG_EXP_MIN = -116
SG_EXP_MAX = 118
BLOCK = 16

# |value| of the 8 non-negative E2M1 codes 0..7 (code bit 3 is the sign).
E2M1_MAGNITUDES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], dtype=np.float64)


def e4m3_value(byte: int) -> float:
    """Value of one FP8 E4M3 (OCP 'FN' variant) byte: bias 7, no infinities,
    S.1111.111 is NaN, exponent field 0 holds subnormals m/8 * 2^-6."""
    sign = -1.0 if byte & 0x80 else 1.0
    e = (byte >> 3) & 0xF
    m = byte & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        return sign * (m / 8.0) * 2.0 ** -6
    return sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)


E4M3_VALUES = np.array([e4m3_value(b) for b in range(256)], dtype=np.float64)
# Non-negative finite E4M3 values in byte order 0x00..0x7E; increasing with the byte.
_E4M3_POS = E4M3_VALUES[:0x7F].copy()


def _nearest_even(q: np.ndarray, grid: np.ndarray) -> np.ndarray:
    """Index of the grid value nearest to each q >= 0 (grid ascending, indices
    are the codes); an exact tie goes to the even index; q above the grid
    saturates to the last index."""
    q = np.asarray(q, dtype=np.float64)
    if not np.all(np.isfinite(q)) or np.any(q < 0):
        raise ValueError("RN encode expects finite non-negative inputs")
    top = len(grid) - 1
    hi = np.clip(np.searchsorted(grid, q, side="left"), 0, top)
    lo = np.clip(hi - 1, 0, top)
    d_lo = q - grid[lo]
    d_hi = grid[hi] - q
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    idx = np.where(pick_hi, hi, lo)
    return np.where(q >= grid[top], top, idx).astype(np.uint8)


def e2m1_encode_magnitude(q: np.ndarray) -> np.ndarray:
    """RN (ties to even code), saturating, of non-negative q onto E2M1 codes 0..7."""
    return _nearest_even(q, E2M1_MAGNITUDES)


def e4m3_encode(v: np.ndarray) -> np.ndarray:
    """RN (ties to even byte), saturating at 448, of non-negative v onto E4M3 bytes."""
    return _nearest_even(v, _E4M3_POS)


SG_DENOM_46 = 4.0 * E4M3_MAX  # 1792: under adaptive 4/6 the M = 4 candidate must fit too


def global_scale(amax: float, mode: str = "pow2", denom: float = SG_DENOM) -> np.float32:
    """FP32 tensor scale s_g for a tensor whose largest |element| is ``amax``.

    denom: 2688 = 6 * 448 (a block's amax mapped to 6 fits the largest E4M3 scale);
    SG_DENOM_46 = 1792 under adaptive 4/6.  Reading (the pages do not say): with
    4/6 the tensor scale also covers the M = 4 candidate, so neither candidate's
    block scale saturates."""
    amax = float(np.float32(amax))
    if not math.isfinite(amax) or amax < 0:
        raise ValueError("amax must be finite and non-negative")
    if amax == 0.0:
        return np.float32(1.0)
    if mode == "amax":
        return np.float32(np.float32(amax) / np.float32(denom))
    if mode != "pow2":
        raise ValueError(f"unknown tensor-scale mode {mode!r}")
    # smallest integer e with denom * 2^e >= amax (exact float64 comparisons)
    e = math.frexp(amax)[1] - 12
    while math.ldexp(denom, e) < amax:
        e += 1
    while math.ldexp(denom, e - 1) >= amax:
        e -= 1
    e = min(max(e, SG_EXP_MIN), SG_EXP_MAX)
    return np.float32(math.ldexp(1.0, e))


def _quantize_blocks(blocks: np.ndarray, s_g: np.float32, M: float):
    """Codes (4-bit, sign included), E4M3 scale bytes and FP32 dequantised values of
    (rows, nb, 16) FP32 blocks with block scale RN_e4m3(amax / fp32(M * s_g))."""
    amax_b = np.max(np.abs(blocks), axis=2)                      # exact
    v = amax_b / (np.float32(M) * s_g)                           # FP32 division
    scales = e4m3_encode(v)
    den = E4M3_VALUES[scales].astype(np.float32) * s_g           # FP32 product
    safe = np.where(den > 0, den, np.float32(1.0)).astype(np.float32)
    q = np.abs(blocks) / safe[:, :, None]                        # FP32 division
    mag = e2m1_encode_magnitude(q)
    sign = np.signbit(blocks).astype(np.uint8) << 3
    nib = np.where((den > 0)[:, :, None], mag | sign, 0).astype(np.uint8)
    deq = (code_values(nib) * den[:, :, None]).astype(np.float32)   # exact in FP32
    return nib, scales, deq


def _block_sq_error_f32(blocks: np.ndarray, deq: np.ndarray) -> np.ndarray:
    """sum_i (x_i - deq_i)^2 of each block, in FP32 with one rounding per operation,
    summed in element order 0..15 (the order fixes the result bit for bit)."""
    err = np.zeros(blocks.shape[:2], dtype=np.float32)
    for i in range(BLOCK):
        d = (blocks[:, :, i] - deq[:, :, i]).astype(np.float32)
        err = (err + (d * d).astype(np.float32)).astype(np.float32)
    return err


def quantize_rows(x: np.ndarray, s_g: float | None = None, mode: str = "pow2",
                  adaptive46: bool = False):
    """Q_1x16: quantise an FP32 matrix in blocks of 16 consecutive elements of a row.

    Returns (codes, scales, s_g): codes uint8 [rows, cols/2] (two elements per
    byte, low nibble first), scales uint8 [rows, cols/16] (E4M3 bytes), s_g
    float32.  ``s_g`` may be given (the value another implementation used);
    otherwise it is derived from the exact amax of ``x``.

    adaptive46: the adaptive 4/6 block scaling named in Section 3.4 ("All
    quantizations use RTN and adaptive 4/6 scaling"; Four Over Six, Section 2
    "Others"): each block is quantised with its largest magnitude mapped to
    M = 6 (the plain rule) and to M = 4, and keeps M = 4 only when that
    candidate's squared error is strictly smaller (ties keep M = 6).  Reading:
    the same tensor scale s_g serves both candidates; the error is the FP32
    sum of _block_sq_error_f32.
    """
    x = np.asarray(x)
    if x.dtype != np.float32:
        raise TypeError("quantize_rows expects float32 input")
    if x.ndim != 2 or x.shape[1] % BLOCK:
        raise ValueError("expected a 2-D array whose row length is a multiple of 16")
    if not np.all(np.isfinite(x)):
        raise ValueError("non-finite input")
    rows, cols = x.shape
    if s_g is None:
        amax = float(np.max(np.abs(x))) if x.size else 0.0
        s_g = global_scale(amax, mode, SG_DENOM_46 if adaptive46 else SG_DENOM)
    s_g = np.float32(s_g)
    blocks = x.reshape(rows, cols // BLOCK, BLOCK)
    nib, scales, deq6 = _quantize_blocks(blocks, s_g, 6.0)
    if adaptive46:
        nib4, scales4, deq4 = _quantize_blocks(blocks, s_g, 4.0)
        use4 = _block_sq_error_f32(blocks, deq4) < _block_sq_error_f32(blocks, deq6)
        nib = np.where(use4[:, :, None], nib4, nib)
        scales = np.where(use4, scales4, scales).astype(np.uint8)
    nib = nib.reshape(rows, cols)
    codes = (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)
    return codes, scales, s_g


def quantize_cols(x: np.ndarray, s_g: float | None = None, mode: str = "pow2",
                  adaptive46: bool = False):
    """Q_16x1: blocks of 16 consecutive elements of a column.  The result is
    laid out as the 1x16 quantisation of x^T (a cols x rows matrix)."""
    return quantize_rows(np.ascontiguousarray(np.asarray(x).T), s_g, mode, adaptive46)


# ---------------------------------------------------------------- random Hadamard transform
# Section 3.4 applies H16^r, "a fresh 16x16 random Hadamard transform", along the
# K dimension of every quantised operand: qX = Q1x16(X H), qX16x1 = Q16x1(H^T X), so
# that each product of two quantised operands carries H H^T = I.  Readings:
#   * H16^r = D H16 / 4, with H16 the Sylvester Hadamard matrix (H16[i, j] =
#     (-1)^popcount(i & j)) and D = diag of 16 random signs, given as a 16-bit mask
#     (bit i set: element i of every block is negated before the transform).
#   * One mask per product, shared by both of its operands and by every block.
#   * In FP32 the transform is the in-place butterfly with strides 1, 2, 4, 8
#     ((u, v) -> (u + v, u - v), one rounding per addition), then the exact * 0.25.

def sylvester16() -> np.ndarray:
    """H16 with entries (-1)^popcount(i & j) (float64)."""
    i = np.arange(BLOCK)
    pc = np.vectorize(lambda t: bin(int(t)).count("1"))(i[:, None] & i[None, :])
    return np.where(pc % 2 == 0, 1.0, -1.0)


def mask_signs(mask: int) -> np.ndarray:
    """The 16 signs (+-1.0) of D for a sign mask."""
    return np.array([-1.0 if (mask >> i) & 1 else 1.0 for i in range(BLOCK)])


def hadamard_rows(x: np.ndarray, mask: int) -> np.ndarray:
    """FP32 x H16^r on every 16-element block of each row (the butterfly reading)."""
    x = np.asarray(x, dtype=np.float32)
    rows, cols = x.shape
    y = (x.reshape(rows, cols // BLOCK, BLOCK) * mask_signs(mask).astype(np.float32)).astype(np.float32)
    y = y.copy()
    h = 1
    while h < BLOCK:
        for i in range(0, BLOCK, 2 * h):
            for j in range(i, i + h):
                u, v = y[:, :, j].copy(), y[:, :, j + h].copy()
                y[:, :, j] = (u + v).astype(np.float32)
                y[:, :, j + h] = (u - v).astype(np.float32)
        h *= 2
    return (y * np.float32(0.25)).astype(np.float32).reshape(rows, cols)


def hadamard_cols(x: np.ndarray, mask: int) -> np.ndarray:
    """FP32 (H16^r)^T x on every 16-element block of each column."""
    return np.ascontiguousarray(hadamard_rows(np.ascontiguousarray(np.asarray(x).T), mask).T)


def hadamard_rows_f64(x: np.ndarray, mask: int) -> np.ndarray:
    """x H16^r in float64 from the matrix definition (reference for the butterfly)."""
    x = np.asarray(x, dtype=np.float64)
    rows, cols = x.shape
    Hr = np.diag(mask_signs(mask)) @ sylvester16() / 4.0
    return (x.reshape(rows, cols // BLOCK, BLOCK) @ Hr).reshape(rows, cols)


def unpack_codes(codes: np.ndarray) -> np.ndarray:
    """uint8 [rows, cols/2] -> 4-bit codes uint8 [rows, cols]."""
    codes = np.asarray(codes, dtype=np.uint8)
    out = np.empty((codes.shape[0], codes.shape[1] * 2), dtype=np.uint8)
    out[:, 0::2] = codes & 0xF
    out[:, 1::2] = codes >> 4
    return out


def code_values(nib: np.ndarray) -> np.ndarray:
    """Signed E2M1 values of 4-bit codes (float64)."""
    nib = np.asarray(nib, dtype=np.uint8)
    mag = E2M1_MAGNITUDES[nib & 7]
    return np.where(nib & 8, -mag, mag)


def dequantize_rows(codes, scales, s_g, dtype=np.float64) -> np.ndarray:
    """Inverse of quantize_rows.  float64: the exact value code * s_b * s_g.
    float32: fp32(fp32(code * s_b) * s_g), the rounding order of the FP32 API."""
    nib = unpack_codes(codes)
    rows, cols = nib.shape
    vals = code_values(nib).reshape(rows, cols // BLOCK, BLOCK)
    sb = E4M3_VALUES[np.asarray(scales, dtype=np.uint8)]
    if dtype == np.float64:
        out = vals * sb[:, :, None] * float(np.float32(s_g))
    elif dtype == np.float32:
        prod = (vals * sb[:, :, None]).astype(np.float32)        # exact: <= 6 significant bits
        out = prod * np.float32(s_g)
    else:
        raise TypeError("dtype must be float32 or float64")
    return out.reshape(rows, cols)


def dequantize_cols(codes, scales, s_g, dtype=np.float64) -> np.ndarray:
    """Inverse of quantize_cols: returns the rows x cols matrix."""
    return dequantize_rows(codes, scales, s_g, dtype).T


def product_f64(a_codes, a_scales, a_sg, b_codes, b_scales, b_sg) -> np.ndarray:
    """D = deq(A) . deq(B)^T in float64, A [M, K] and B [N, K] both 1x16-blocked
    along K: the textbook product of the dequantised operands."""
    return dequantize_rows(a_codes, a_scales, a_sg) @ dequantize_rows(b_codes, b_scales, b_sg).T

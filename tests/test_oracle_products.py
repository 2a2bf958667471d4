"""Pins of the oracle's product and measurement helpers ("Full-Stack FP4", Section 3.4:
the Gram and update products of the NVFP4 Newton-Schulz step are products of
block-scaled NVFP4 operands; Section 2 "Root optimizer": the iteration drives X X^T
towards I).

Every expected value here is written down by hand from the definition of the
format (E2M1 code values, E4M3 block scales, FP32 tensor scale) or from a closed
form, not by calling the oracle's own arithmetic a second time.
"""
import numpy as np
import pytest

from oracle import nvfp4 as Q
from oracle import root_ns as R

# E2M1 codes (sign bit 8) and E4M3 bytes used below, decoded by hand:
# code 0x2 = 1.0, 0x4 = 2.0, 0x5 = 3.0, 0x7 = 6.0, 0xB = -1.5;
# E4M3 byte (e << 3) | m = 2^(e - 7) (1 + m / 8): 0x38 = 1.0, 0x40 = 2.0, 0x44 = 3.0.
CODE_VAL = {0x2: 1.0, 0x4: 2.0, 0x5: 3.0, 0x7: 6.0, 0xB: -1.5, 0x0: 0.0}
SCALE_VAL = {0x38: 1.0, 0x40: 2.0, 0x44: 3.0}


def pack(nibbles):
    """One row of 4-bit codes -> bytes, element 2j in the low nibble of byte j."""
    nibbles = list(nibbles)
    return [nibbles[2 * j] | (nibbles[2 * j + 1] << 4) for j in range(len(nibbles) // 2)]


def operand(rows_spec):
    """rows_spec: per row, a list of (code, scale byte) per 16-element block."""
    codes, scales = [], []
    for blocks in rows_spec:
        nib = [c for c, _ in blocks for _ in range(16)]
        codes.append(pack(nib))
        scales.append([s for _, s in blocks])
    return np.array(codes, np.uint8), np.array(scales, np.uint8)


def test_product_f64_is_a_times_b_transposed_with_every_scale_applied():
    """A is 2 x 32 and B is 3 x 32, both blocked along K = 32 (two blocks per row);
    D[i, j] = sum_k a_ik b_jk must come out 2 x 3 with each block's own scale and
    each operand's own tensor scale."""
    a_spec = [[(0x2, 0x38), (0x4, 0x40)],       # row 0: 16 x 1.0*1, then 16 x 2.0*2
              [(0xB, 0x44), (0x0, 0x38)]]       # row 1: 16 x -1.5*3, then zeros
    b_spec = [[(0x2, 0x38), (0x2, 0x38)],       # row 0: 32 x 1
              [(0x5, 0x40), (0x7, 0x38)],       # row 1: 16 x 6, then 16 x 6
              [(0x0, 0x38), (0x4, 0x44)]]       # row 2: zeros, then 16 x 6
    a_codes, a_scales = operand(a_spec)
    b_codes, b_scales = operand(b_spec)
    a_sg, b_sg = np.float32(0.5), np.float32(0.25)

    def rowvals(spec, sg):
        return [[CODE_VAL[c] * SCALE_VAL[s] * float(sg) for c, s in blocks for _ in range(16)]
                for blocks in spec]

    A, B = rowvals(a_spec, a_sg), rowvals(b_spec, b_sg)
    want = np.zeros((2, 3))
    for i in range(2):
        for j in range(3):
            want[i, j] = sum(A[i][k] * B[j][k] for k in range(32))
    # the same numbers by hand: a0 = [0.5]*16 + [2]*16, a1 = [-2.25]*16 + [0]*16,
    # b0 = [0.25]*32, b1 = [1.5]*32, b2 = [0]*16 + [1.5]*16
    hand = np.array([[16 * 0.5 * 0.25 + 16 * 2 * 0.25, 16 * 0.5 * 1.5 + 16 * 2 * 1.5, 16 * 2 * 1.5],
                     [16 * -2.25 * 0.25, 16 * -2.25 * 1.5, 0.0]])
    assert np.array_equal(want, hand)
    got = Q.product_f64(a_codes, a_scales, a_sg, b_codes, b_scales, b_sg)
    assert got.shape == (2, 3)
    assert np.array_equal(got, hand)


def test_product_f64_brute_force_on_random_tiny_operands():
    """Random codes and scales: the product equals a triple loop over hand-decoded
    values (E2M1 magnitudes {0, .5, 1, 1.5, 2, 3, 4, 6}, E4M3 from its bit fields)."""
    rng = np.random.default_rng(5)
    M, N, K = 3, 5, 48
    mags = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]

    def e4m3(byte):
        e, m = (byte >> 3) & 0xF, byte & 7
        return (m / 8) * 2.0 ** -6 if e == 0 else (1 + m / 8) * 2.0 ** (e - 7)

    def draw(rows):
        nib = rng.integers(0, 16, size=(rows, K)).astype(np.uint8)
        sc = rng.integers(0x20, 0x50, size=(rows, K // 16)).astype(np.uint8)
        codes = (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)
        vals = [[(-1 if nib[r, k] & 8 else 1) * mags[nib[r, k] & 7] * e4m3(int(sc[r, k // 16]))
                 for k in range(K)] for r in range(rows)]
        return codes, sc, vals

    ac, asc, av = draw(M)
    bc, bsc, bv = draw(N)
    a_sg, b_sg = np.float32(2.0 ** -3), np.float32(2.0 ** 5)
    want = np.array([[sum(av[i][k] * bv[j][k] for k in range(K)) * float(a_sg) * float(b_sg)
                      for j in range(N)] for i in range(M)])
    got = Q.product_f64(ac, asc, a_sg, bc, bsc, b_sg)
    assert got.shape == (M, N)
    np.testing.assert_allclose(got, want, rtol=1e-14, atol=0)


def test_orthogonality_error_closed_forms():
    """||X X^T - I||_F / sqrt(m): zero on orthonormal rows; for X = diag(d) [I 0] it is
    sqrt(sum (d_i^2 - 1)^2 / m); a tall input is measured as its transpose."""
    rng = np.random.default_rng(2)
    Qm, _ = np.linalg.qr(rng.standard_normal((40, 40)))
    X = Qm[:12]                                   # 12 orthonormal rows of length 40
    assert R.orthogonality_error(X) == pytest.approx(0.0, abs=1e-14)
    d = np.array([1.0, 2.0, 0.5, 3.0])
    X = np.zeros((4, 9))
    X[np.arange(4), np.arange(4)] = d
    want = np.sqrt(((d ** 2 - 1) ** 2).sum() / 4)
    assert R.orthogonality_error(X) == pytest.approx(want, rel=1e-15)
    assert R.orthogonality_error(X.T) == pytest.approx(want, rel=1e-15)


def test_symmetric_from_upper_mirrors_entry_by_entry():
    rng = np.random.default_rng(4)
    U = rng.standard_normal((5, 5))
    S = R.symmetric_from_upper(U)
    for i in range(5):
        for j in range(5):
            assert S[i, j] == U[min(i, j), max(i, j)]

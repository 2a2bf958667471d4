"""Pins for the oracle's BF16 Newton-Schulz route (the BF16 baseline the pages compare
Q-Root against; "Full-Stack FP4", Section 4.4 and Table 6), CPU only.

The BF16 rounding is checked against torch's float32 -> bfloat16 conversion and hand
ties; the iteration against a case where every BF16 rounding is exact (so it must equal
the float64 polynomial step), a hand-worked case that tells which tensors are rounded,
and the float64 iteration it approximates.
"""
import numpy as np
import pytest
import torch

from oracle import root_ns as R

MUON = (3.4445, -4.7750, 2.0315)
QUINTIC = (15 / 8, -10 / 8, 3 / 8)


def test_bf16_round_matches_torch_and_hand_ties():
    rng = np.random.default_rng(0)
    bits = rng.integers(0, 0x7F7F0000, 200000, dtype=np.uint64).astype(np.uint32)
    x = np.concatenate([bits.view(np.float32), -bits.view(np.float32),
                        np.float32([0.0, -0.0, 1.0, 3.0e38, 1e-40, -1e-45])])
    want = torch.from_numpy(x.copy()).bfloat16().float().numpy()
    got = R.bf16_round(x)
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32))
    # ties: 1 + 2^-8 is halfway between 1 and 1 + 2^-7 -> even (1); 1 + 3 * 2^-8 -> 1 + 2^-6
    t = np.float32([1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, 1 + 2.0 ** -8 + 2.0 ** -20])
    assert R.bf16_round(t).tolist() == [1.0, 1 + 2.0 ** -6, 1 + 2.0 ** -7]


def test_bf16_iteration_equals_float64_when_every_rounding_is_exact():
    """X0 = t S, S = 16 rows of a 32 x 32 Sylvester Hadamard matrix, t = 2^-5:
    A = 32 t^2 I = 2^-5 I, P = A^2 and B = -A + 16 A^2 = -2^-6 I are BF16 numbers, so
    one BF16 step must equal the float64 polynomial step."""
    H = np.array([[1.0]])
    while H.shape[0] < 32:
        H = np.block([[H, H], [H, -H]])
    X0 = (2.0 ** -5 * H[:16, :]).astype(np.float32)
    a, b, c = 1.875, -1.0, 16.0
    got = R.ns_iterations_bf16(X0, 1, a, b, c)
    A = X0.astype(np.float64) @ X0.T.astype(np.float64)
    want = a * X0 + (b * A + c * A @ A) @ X0
    assert np.array_equal(got.astype(np.float64), want)
    assert not np.allclose(want, a * X0)


def test_bf16_iteration_rounds_the_operands_not_the_fp32_term_by_hand():
    """X0 = 16 x 16 with X0[0, 0] = 1 + 2^-10 (not a BF16 number: it rounds to 1) and
    nothing else.  Then by hand: Xb[0, 0] = 1, A[0, 0] = 1, bf16(A) = A, P[0, 0] = 1,
    B[0, 0] = -0.5 + 0.25 = -0.25 (a BF16 number), and
    X1[0, 0] = 1 * (1 + 2^-10) + (-0.25) * 1 = 0.75 + 2^-10: the a X term keeps the
    FP32 X while the product uses the BF16 view.  Squaring the FP32 X would give
    A[0, 0] = (1 + 2^-10)^2 instead."""
    X0 = np.zeros((16, 16), np.float32)
    X0[0, 0] = np.float32(1 + 2.0 ** -10)
    trace = []
    got = R.ns_iterations_bf16(X0, 1, 1.0, -0.5, 0.25, trace=trace)
    assert trace[0]["A"][0, 0] == 1.0 and trace[0]["P"][0, 0] == 1.0
    assert trace[0]["B"][0, 0] == -0.25
    assert got[0, 0] == np.float32(0.75 + 2.0 ** -10)
    assert np.count_nonzero(got) == 1


@pytest.mark.parametrize("coef,tol", [(MUON, 4e-2), (QUINTIC, 5e-3)])
def test_bf16_route_stays_close_to_float64(coef, tol):
    rng = np.random.default_rng(3)
    G = (rng.standard_normal((256, 768)) * 0.02).astype(np.float32)
    yb = R.root_ns(G, 5, *coef, bf16=True)
    yf = R.root_ns(G, 5, *coef, quantized=False)
    assert np.linalg.norm(yb - yf) / np.linalg.norm(yf) < tol
    eb, ef = R.orthogonality_error(yb), R.orthogonality_error(yf)
    assert abs(eb - ef) <= 0.02 * ef


def test_bf16_route_transpose_symmetry():
    rng = np.random.default_rng(5)
    G = (rng.standard_normal((64, 160)) * 0.02).astype(np.float32)
    assert np.array_equal(R.root_ns(G.T, 3, bf16=True), R.root_ns(G, 3, bf16=True).T)

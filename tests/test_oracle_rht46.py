"""Pins of the oracle's random Hadamard transform and adaptive 4/6 block scaling
("Full-Stack FP4", Section 3.4: qX = Q1x16(X H16^r), qX16x1 = Q16x1(H16^r^T X), and
"all quantizations use RTN and adaptive 4/6 scaling").  The transform is checked
against an independently built Sylvester matrix, its orthogonality and its
cancellation inside a product; the 4/6 choice against hand-worked blocks and
exact float64 error comparisons."""
import json
import os

import numpy as np
import pytest

from oracle import nvfp4 as Q
from oracle import root_ns as R

pytestmark = pytest.mark.filterwarnings("ignore")


def _sylvester_kron(n):
    """Sylvester Hadamard by the doubling construction H_2n = [[H, H], [H, -H]]."""
    H = np.array([[1.0]])
    while H.shape[0] < n:
        H = np.block([[H, H], [H, -H]])
    return H


@pytest.mark.parametrize("mask", [0x0000, 0xFFFF, 0x5A3C, 0x8001])
def test_unit_vectors_give_exact_scaled_hadamard_rows(mask):
    """Row j of I16 H16^r is s_j * H16[j, :] / 4 exactly (one nonzero per butterfly)."""
    H = _sylvester_kron(16)
    s = np.array([-1.0 if (mask >> i) & 1 else 1.0 for i in range(16)])
    got = Q.hadamard_rows(np.eye(16, dtype=np.float32), mask)
    want = (s[:, None] * H / 4.0).astype(np.float32)
    assert np.array_equal(got, want)


def test_butterfly_matches_matrix_definition():
    rng = np.random.default_rng(1)
    X = rng.standard_normal((64, 256)).astype(np.float32)
    H = _sylvester_kron(16)
    for mask in (0, 0x1234, 0xBEEF):
        s = np.array([-1.0 if (mask >> i) & 1 else 1.0 for i in range(16)])
        want = (X.astype(np.float64).reshape(64, 16, 16) @ (np.diag(s) @ H / 4.0)).reshape(64, 256)
        got = Q.hadamard_rows(X, mask).astype(np.float64)
        # four FP32 additions per output: within a few ulps of the block's magnitude
        assert np.max(np.abs(got - want)) <= 4 * 2.0 ** -23 * np.max(np.abs(X)) * 4
        assert np.allclose(Q.hadamard_rows_f64(X, mask), want, rtol=0, atol=1e-12)


def test_transform_is_orthogonal_and_invertible():
    rng = np.random.default_rng(2)
    X = rng.standard_normal((32, 128)).astype(np.float32)
    mask = 0x6B2D
    Y = Q.hadamard_rows(X, mask)
    blocks = lambda t: t.astype(np.float64).reshape(32, 8, 16)
    assert np.allclose(np.sum(blocks(Y) ** 2, axis=2), np.sum(blocks(X) ** 2, axis=2), rtol=1e-5)
    # inverse of x D H / 4 is y H D / 4 (H symmetric, H H = 16 I)
    H = _sylvester_kron(16)
    s = np.array([-1.0 if (mask >> i) & 1 else 1.0 for i in range(16)])
    back = (blocks(Y) @ (H @ np.diag(s) / 4.0)).reshape(32, 128)
    assert np.allclose(back, X, rtol=0, atol=1e-5)


def test_transforms_cancel_inside_products():
    """(X H)(Y H)^T = X Y^T and (X H)(H^T Z) = X Z: the reason one mask serves both operands."""
    rng = np.random.default_rng(3)
    X = rng.standard_normal((48, 64)).astype(np.float32)
    Y = rng.standard_normal((40, 64)).astype(np.float32)
    Z = rng.standard_normal((64, 24)).astype(np.float32)
    m = 0x0F0F
    lhs = Q.hadamard_rows(X, m).astype(np.float64) @ Q.hadamard_rows(Y, m).astype(np.float64).T
    ref = X.astype(np.float64) @ Y.astype(np.float64).T
    assert np.linalg.norm(lhs - ref) <= 1e-6 * np.linalg.norm(ref)
    lhs2 = Q.hadamard_rows(X, m).astype(np.float64) @ Q.hadamard_cols(Z, m).astype(np.float64)
    ref2 = X.astype(np.float64) @ Z.astype(np.float64)
    assert np.linalg.norm(lhs2 - ref2) <= 1e-6 * np.linalg.norm(ref2)


def test_adaptive46_hand_worked_blocks(golden_dir):
    with open(os.path.join(golden_dir, "adaptive46_blocks.json")) as f:
        data = json.load(f)
    for case in data["cases"]:
        x = np.array(case["x"], dtype=np.float32).reshape(1, -1)
        codes, scales, sg = Q.quantize_rows(x, s_g=case["s_g"], adaptive46=True)
        assert scales.tobytes().hex() == "".join(case["scales_hex"]), case["name"]
        assert codes.tobytes().hex() == "".join(case["codes_hex"]), case["name"]


def _exact_error(x, codes, scales, s_g):
    d = Q.dequantize_rows(codes, scales, s_g)          # float64, exact values
    return np.sum((x.astype(np.float64) - d).reshape(x.shape[0], -1, 16) ** 2, axis=2)


def test_adaptive46_choice_is_the_smaller_exact_error():
    """Wherever the two candidates' exact squared errors differ by more than the FP32
    decision's rounding, the kept candidate is the one with the smaller error; it is
    never worse than plain M = 6 beyond that margin."""
    rng = np.random.default_rng(4)
    x = (rng.standard_normal((64, 512)) * rng.lognormal(0, 1, (64, 1))).astype(np.float32)
    x[:, :64] = np.round(x[:, :64] * 2) / 2          # blocks with exactly representable values
    sg = Q.global_scale(float(np.max(np.abs(x))))
    c6, s6, _ = Q.quantize_rows(x, s_g=sg)
    c46, s46, _ = Q.quantize_rows(x, s_g=sg, adaptive46=True)
    e6 = _exact_error(x, c6, s6, sg)
    e46 = _exact_error(x, c46, s46, sg)
    # candidate M = 4 alone: quantise with the block max mapped to 4
    blocks = x.reshape(64, 32, 16)
    nib4, sc4, deq4 = Q._quantize_blocks(blocks, np.float32(sg), 4.0)
    e4 = np.sum((blocks.astype(np.float64) - deq4.astype(np.float64)) ** 2, axis=2)
    margin = 1e-5 * np.maximum(e4, e6) + 1e-30
    clear4 = e4 < e6 - margin
    clear6 = e6 < e4 - margin
    assert np.array_equal(e46[clear4], e4[clear4])
    assert np.array_equal(e46[clear6], e6[clear6])
    assert np.all(e46 <= e6 + margin)
    assert clear4.any() and clear6.any()


def test_rht46_route_stays_close_to_float64_for_contractive_quintic():
    """The full Section 3.4 route (transform on every quantised operand, one mask per
    product, adaptive 4/6) stays within a few percent of the float64 iteration."""
    rng = np.random.default_rng(9)
    G = (rng.standard_normal((128, 384)) * 0.02).astype(np.float32)
    quintic = (15 / 8, -10 / 8, 3 / 8)
    masks = [int(v) for v in rng.integers(0, 1 << 16, 15)]
    yq = R.root_ns(G, 5, *quintic, rht_masks=masks, adaptive46=True)
    yf = R.root_ns(G, 5, *quintic, quantized=False)
    assert np.linalg.norm(yq - yf) / np.linalg.norm(yf) < 0.1


@pytest.mark.parametrize("amax", [1e-30, 3e-5, 0.02, 1.0, 1.5, 1791.9, 1792.0, 1792.1, 3.0e30])
def test_adaptive46_tensor_scale_covers_the_m4_candidate(amax):
    """Under 4/6 the power-of-two s_g is the smallest with 4 * 448 * s_g >= amax, so the
    largest block's M = 4 scale amax / (4 s_g) never exceeds the largest E4M3 value."""
    sg = float(Q.global_scale(amax, denom=Q.SG_DENOM_46))
    assert 1792.0 * sg >= float(np.float32(amax)) and 1792.0 * sg / 2 < float(np.float32(amax))
    assert sg == 2.0 ** round(np.log2(sg))
    x = np.zeros((1, 16), np.float32)
    x[0, 0] = amax
    codes, scales, got = Q.quantize_rows(x, adaptive46=True)
    assert got == sg and Q.E4M3_VALUES[scales[0, 0]] * float(sg) * 6 >= float(np.float32(amax)) * 0.9

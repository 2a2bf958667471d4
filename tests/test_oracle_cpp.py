"""Pins for the C++ oracle (oracle/cpp/fs4_oracle.cpp), CPU only.

The C++ oracle restates the same pages ("Full-Stack FP4", arXiv 2607.04422,
Section 2 "NVFP4 format" and Section 3.4) in plain loops without BLAS.  It is
tied to things other than itself: the code-point values of the format, the
hand-worked blocks under tests/golden/, the hand-worked combine step, brute-force
products on tiny operands, the closed form of the float64 iteration, and (as an
independent second implementation) the numpy oracle, bit for bit where the
arithmetic is exact and within the float64 summation-order noise elsewhere.
"""
import json
import os

import numpy as np
import pytest

from oracle import cpp_oracle as C
from oracle import nvfp4 as Q
from oracle import root_ns as R

MUON = (3.4445, -4.7750, 2.0315)
QUINTIC = (15 / 8, -10 / 8, 3 / 8)
CUBIC = (1.5, -0.5, 0.0)


def test_e2m1_code_points_are_the_format_values():
    want = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    L = C.lib()
    for code in range(16):
        v = L.fs4o_e2m1_value(code)
        assert abs(v) == want[code & 7]
        assert np.signbit(v) == bool(code & 8)
    for code in range(8):
        assert L.fs4o_e2m1_encode(want[code]) == code


def test_e4m3_every_byte_matches_the_numpy_codec():
    L = C.lib()
    for b in range(256):
        v, w = L.fs4o_e4m3_value(b), Q.E4M3_VALUES[b]
        assert (np.isnan(v) and np.isnan(w)) or v == w


def test_encoders_agree_with_the_numpy_oracle_on_ties_and_random_values():
    rng = np.random.default_rng(0)
    L = C.lib()
    ties = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0, 6.5, 100.0]
    q = np.concatenate([rng.uniform(0, 7, 3000), ties,
                        np.nextafter(ties, 0.0), np.nextafter(ties, 9.0)])
    assert [L.fs4o_e2m1_encode(float(v)) for v in q] == Q.e2m1_encode_magnitude(q).tolist()
    grid = Q.E4M3_VALUES[:0x7F]
    mids = (grid[1:] + grid[:-1]) / 2          # every E4M3 tie
    v = np.concatenate([rng.uniform(0, 500, 3000), 2.0 ** rng.uniform(-12, 9, 3000), mids,
                        np.nextafter(mids, 0.0), np.nextafter(mids, 1e9), [448.0, 460.0, 1e6, 0.0]])
    assert [L.fs4o_e4m3_encode(float(x)) for x in v] == Q.e4m3_encode(v).tolist()


def test_tensor_scale_matches_the_numpy_oracle():
    rng = np.random.default_rng(1)
    L = C.lib()
    amax = np.concatenate([np.float32(2.0) ** rng.uniform(-120, 120, 500).astype(np.float32),
                           np.float32([0.0, 2688.0, 2688.0 * 2 ** -10, 6.0, 12.0, 3e38, 1e-40])])
    for a in amax.astype(np.float32):
        for mode, name in ((0, "pow2"), (1, "amax")):
            assert L.fs4o_tensor_scale(float(a), mode) == Q.global_scale(float(a), name)


def test_hand_blocks(golden_dir):
    with open(os.path.join(golden_dir, "hand_blocks.json")) as f:
        cases = json.load(f)["cases"]
    for case in cases:
        x = np.array(case["x"], np.float32)[None, :]
        codes, scales, sg = C.quantize_rows(x)
        assert sg == np.float32(case["s_g"]), case["name"]
        assert [f"{b:02x}" for b in scales[0]] == case["scales_hex"], case["name"]
        assert [f"{b:02x}" for b in codes[0]] == case["codes_hex"], case["name"]
        deq = C.dequantize_rows(codes, scales, sg)[0]
        want = np.array(case["dequantized"], np.float64)
        assert np.array_equal(deq, want) and np.array_equal(np.signbit(deq), np.signbit(want))


@pytest.mark.parametrize("kind", ["gauss", "outliers", "student", "zeros_and_signed_zeros", "tiny"])
@pytest.mark.parametrize("mode", ["pow2", "amax"])
def test_quantise_bit_exact_against_the_numpy_oracle(kind, mode):
    rng = np.random.default_rng(2)
    x = rng.standard_normal((48, 160)) * 0.02
    if kind == "outliers":
        x[rng.random(x.shape) < 0.01] *= 50
    elif kind == "student":
        x = rng.standard_t(3, x.shape)
    elif kind == "zeros_and_signed_zeros":
        x[rng.random(x.shape) < 0.3] = -0.0
        x[rng.random(x.shape) < 0.2] = 0.0
        x[:, 16:32] = 0.0
    elif kind == "tiny":
        x = x * 1e-30
    x = x.astype(np.float32)
    for fc, fn in ((C.quantize_rows, Q.quantize_rows), (C.quantize_cols, Q.quantize_cols)):
        c1, s1, g1 = fc(x, mode=mode)
        c2, s2, g2 = fn(x, mode=mode)
        assert g1 == g2 and np.array_equal(s1, s2) and np.array_equal(c1, c2)
        assert np.array_equal(C.dequantize_rows(c1, s1, g1), Q.dequantize_rows(c2, s2, g2))


def test_product_against_brute_force():
    rng = np.random.default_rng(3)
    L = rng.standard_normal((5, 7))
    Rm = rng.standard_normal((7, 3))
    got = C.product(L, Rm)
    for i in range(5):
        for j in range(3):
            s = 0.0
            for k in range(7):
                s += L[i, k] * Rm[k, j]
            assert got[i, j] == s        # the same summation order: bit-equal


def test_normalise_and_clip_matches_the_numpy_oracle():
    rng = np.random.default_rng(4)
    G = (rng.standard_normal((64, 96)) * 0.02).astype(np.float32)
    G[3, 5] = 5.0
    for clip in (3.0, None):
        X1, inv1, tau1, n1 = C.normalise_and_clip(G, clip)
        X2, inv2, tau2, n2 = R.normalise_and_clip(G, clip)
        assert inv1 == inv2 and tau1 == tau2 and abs(n1 - n2) <= 1e-12 * n2
        assert np.array_equal(X1.view(np.uint32), X2.view(np.uint32))


def test_combine_step_by_hand():
    """The 16 x 16 iteration worked out by hand in tests/test_oracle_ns.py."""
    X0 = np.zeros((16, 16), np.float32)
    X0[0, 0] = 6.0
    X0[1, 0], X0[1, 1] = 1.0, 1.5
    got = C.ns_iterations_nvfp4(X0, 1, 1.0, -0.5, 0.25)
    want = np.zeros((16, 16))
    want[:2, :2] = [[1930.0, 78.0], [334.0, 15.0]]
    assert np.array_equal(got.astype(np.float64), want)


@pytest.mark.parametrize("coef", [MUON, CUBIC, QUINTIC])
def test_float64_route_matches_the_closed_form(coef):
    from tests.test_oracle_ns import built_from_svd, poly_iterate
    rng = np.random.default_rng(3)
    m, n, K = 24, 40, 5
    sigma = np.sort(rng.uniform(0.05, 2.0, m))[::-1]
    U, V, G = built_from_svd(m, n, sigma, rng)
    s0 = sigma / (np.linalg.norm(sigma) + R.NS_EPS)
    want = U @ np.diag(poly_iterate(s0, K, *coef)) @ V.T
    got = C.root_ns(G.astype(np.float32), K, *coef, clip_k=None, quantized=False)
    # G was rounded to FP32 on the way in: compare with the closed form of that input
    Gf = G.astype(np.float32).astype(np.float64)
    u, s, vt = np.linalg.svd(Gf, full_matrices=False)
    want = u @ np.diag(poly_iterate(s / (np.linalg.norm(s) + R.NS_EPS), K, *coef)) @ vt
    assert np.linalg.norm(got - want) <= 1e-10 * max(1.0, np.linalg.norm(want))


@pytest.mark.parametrize("shape,K,coef", [((64, 160), 3, MUON), ((160, 64), 2, MUON),
                                          ((96, 320), 5, QUINTIC), ((48, 48), 5, CUBIC)])
def test_quantised_route_matches_the_numpy_oracle(shape, K, coef):
    """Two independent implementations of the same steps.  Their products differ only
    in float64 summation order (BLAS blocking versus k order), which changes an FP32
    iterate by at most one rounding in rare entries."""
    rng = np.random.default_rng(5)
    G = (rng.standard_normal(shape) * 0.02).astype(np.float32)
    got = C.root_ns(G, K, *coef, clip_k=3.0)
    want = R.root_ns(G, K, *coef, clip_k=3.0)
    assert got.shape == want.shape
    assert np.linalg.norm(got - want) <= 1e-6 * np.linalg.norm(want)


def test_nonfinite_input_is_refused():
    G = np.zeros((16, 16), np.float32)
    G[2, 3] = np.nan
    with pytest.raises(ValueError):
        C.root_ns(G, 1)


@pytest.mark.parametrize("shape,K,coef", [((64, 160), 3, MUON), ((96, 320), 2, QUINTIC),
                                          ((48, 48), 2, CUBIC)])
def test_numpy_iteration_with_the_cpp_codec_is_bit_identical(shape, K, coef):
    """The large-size GPU tests run the numpy oracle's iteration with the C++ codec
    (codec=cpp_oracle) for speed; it must give the numpy codec's result bit for bit."""
    rng = np.random.default_rng(6)
    X0 = R.normalise_and_clip((rng.standard_normal(shape) * 0.02).astype(np.float32), 3.0)[0]
    a = R.ns_iterations_nvfp4(X0, K, *coef)
    b = R.ns_iterations_nvfp4(X0, K, *coef, codec=C)
    assert np.array_equal(a.view(np.uint32), b.view(np.uint32))

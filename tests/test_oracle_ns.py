"""Pins for the oracle's Newton-Schulz iteration (CPU only).

"Full-Stack FP4" (arXiv 2607.04422): Section 2, paragraph "Root optimizer"
(the polynomial X_{k+1} = a X + b X(X^T X) + c X(X^T X)^2) and Section 3.4
(the NVFP4 iteration).  The pins come from the mathematics: the closed form of
the polynomial iteration on a matrix built from its SVD, convergence of the
cubic and quintic iterations to the polar factor (numpy SVD), a case where
every NVFP4 quantisation is exact so the quantised iteration must equal the
float64 one, the transpose symmetry, and the shrinking singular-value spread.
"""
import numpy as np
import pytest

from oracle import nvfp4 as Q
from oracle import root_ns as R

MUON = (3.4445, -4.7750, 2.0315)
CUBIC = (1.5, -0.5, 0.0)
QUINTIC = (15 / 8, -10 / 8, 3 / 8)


def householder_orthogonal(n, rng, reflections=6):
    """A random n x n orthogonal matrix as a product of Householder reflections."""
    Qm = np.eye(n)
    for _ in range(reflections):
        v = rng.standard_normal(n)
        v /= np.linalg.norm(v)
        Qm = Qm - 2.0 * np.outer(Qm @ v, v)
    return Qm


def built_from_svd(m, n, sigma, rng):
    U = householder_orthogonal(m, rng)
    V = householder_orthogonal(n, rng)[:, :m]
    return U, V, U @ np.diag(sigma) @ V.T


def poly_iterate(s, K, a, b, c):
    for _ in range(K):
        s = a * s + b * s ** 3 + c * s ** 5
    return s


@pytest.mark.parametrize("coef", [MUON, CUBIC, QUINTIC])
@pytest.mark.parametrize("tall", [False, True])
def test_float64_iteration_matches_closed_form_on_svd_input(coef, tall):
    rng = np.random.default_rng(3)
    m, n, K = 24, 40, 5
    sigma = np.sort(rng.uniform(0.05, 2.0, m))[::-1]
    U, V, G = built_from_svd(m, n, sigma, rng)
    eps = R.NS_EPS
    s0 = sigma / (np.linalg.norm(sigma) + eps)
    want = U @ np.diag(poly_iterate(s0, K, *coef)) @ V.T
    if tall:
        got = R.root_ns(G.T, K, *coef, clip_k=None, quantized=False).T
    else:
        got = R.root_ns(G, K, *coef, clip_k=None, quantized=False)
    assert np.linalg.norm(got - want) <= 1e-12 * max(1.0, np.linalg.norm(want))


@pytest.mark.parametrize("coef,K", [(CUBIC, 40), (QUINTIC, 30)])
def test_convergent_iterations_reach_polar_factor(coef, K):
    rng = np.random.default_rng(4)
    m, n = 20, 36
    sigma = np.linspace(0.2, 1.0, m)
    _, _, G = built_from_svd(m, n, sigma, rng)
    u, _, vt = np.linalg.svd(G, full_matrices=False)
    got = R.root_ns(G, K, *coef, clip_k=None, quantized=False)
    assert np.linalg.norm(got - u @ vt) < 1e-9


def test_quantised_iteration_equals_float64_when_every_quantisation_is_exact():
    """X0 = t*S with S = 16 rows of a 32x32 Sylvester Hadamard matrix and
    t = 1.5*2^-5: X0, A = 32 t^2 I, P = A^2 and B = b A + c A^2 with (b, c) =
    (-1, 16) are all exactly representable in NVFP4, so one quantised step must
    reproduce the float64 polynomial step exactly."""
    H = np.array([[1.0]])
    while H.shape[0] < 32:
        H = np.block([[H, H], [H, -H]])
    t = 1.5 * 2.0 ** -5
    X0 = (t * H[:16, :]).astype(np.float32)
    a, b, c = 1.875, -1.0, 16.0
    got = R.ns_iterations_nvfp4(X0, 1, a, b, c)
    A = X0.astype(np.float64) @ X0.T.astype(np.float64)
    want = a * X0 + (b * A + c * A @ A) @ X0
    assert np.array_equal(got.astype(np.float64), want)
    # the premise: B is not a multiple of the identity that happens to vanish
    assert not np.allclose(want, a * X0)


def test_quantised_transpose_symmetry():
    rng = np.random.default_rng(5)
    G = (rng.standard_normal((64, 160)) * 0.02).astype(np.float32)
    assert np.array_equal(R.root_ns(G.T, 3), R.root_ns(G, 3).T)


def _spread(X):
    s = np.linalg.svd(X.astype(np.float64), compute_uv=False)
    return s[0] / s[-1]


@pytest.mark.parametrize("quantized,coef,kmax", [(False, MUON, 5), (True, QUINTIC, 5), (True, MUON, 2)])
def test_singular_value_spread_shrinks(quantized, coef, kmax):
    """Rectangular Gaussian input: sigma_max / sigma_min decreases every iteration
    until it is within the polynomial's fixed band."""
    rng = np.random.default_rng(6)
    G = (rng.standard_normal((96, 320)) * 0.02).astype(np.float32)
    X0, _, _, _ = R.normalise_and_clip(G, 3.0)
    prev = _spread(X0)
    X = X0
    band = 1.25 / 0.68 if coef is MUON else 1.05
    for _ in range(kmax):
        X = (R.ns_iterations_nvfp4(X, 1, *coef) if quantized
             else R.ns_iterations_f64(X, 1, *coef))
        cur = _spread(X)
        assert cur <= prev or cur <= band
        prev = cur
    assert prev < _spread(X0)


def test_normalisation_and_clip():
    rng = np.random.default_rng(7)
    G = (rng.standard_normal((32, 64)) * 0.02).astype(np.float32)
    G[3, 5] = 5.0   # an outlier far beyond 3 RMS
    X0, inv, tau, norm = R.normalise_and_clip(G, 3.0)
    assert np.isclose(norm, np.linalg.norm(G.astype(np.float64)))
    assert inv == np.float32(1.0 / (norm + R.NS_EPS))
    rms = norm * float(inv) / np.sqrt(G.size)
    assert np.isclose(float(tau), 3.0 * rms, rtol=1e-6)
    assert X0[3, 5] == tau
    assert np.max(np.abs(X0)) == tau
    inside = np.abs(G * inv) < tau
    assert np.array_equal(X0[inside], (G * inv)[inside])


def test_scale_invariance():
    rng = np.random.default_rng(8)
    G = (rng.standard_normal((64, 192)) * 0.02).astype(np.float32)
    y1 = R.root_ns(G, 5, *QUINTIC)
    y2 = R.root_ns(G * np.float32(8.0), 5, *QUINTIC)
    assert np.linalg.norm(y1 - y2) / np.linalg.norm(y1) < 1e-3


def test_zero_input_gives_zero_output():
    y = R.root_ns(np.zeros((32, 48), np.float32), 5)
    assert not y.any() and np.all(np.isfinite(y))


def test_nonfinite_input_is_refused():
    G = np.zeros((16, 16), np.float32)
    G[0, 0] = np.inf
    with pytest.raises(ValueError):
        R.root_ns(G, 1)


def test_quantised_route_stays_close_to_float64_for_contractive_quintic():
    """Sanity of the whole route: with the stable quintic the NVFP4 iterate
    stays within a few percent of the float64 one on a rectangular input."""
    rng = np.random.default_rng(9)
    G = (rng.standard_normal((128, 384)) * 0.02).astype(np.float32)
    yq = R.root_ns(G, 5, *QUINTIC)
    yf = R.root_ns(G, 5, *QUINTIC, quantized=False)
    assert np.linalg.norm(yq - yf) / np.linalg.norm(yf) < 0.1


def _signs(m, n, rng):
    return rng.choice([-1.0, 1.0], (m, n))


def test_gram_uses_the_row_blocked_view():
    """Rows of constant magnitude 1.5*2^j (j varying by row): the 1x16 view of
    X is exact, the 16x1 view is not.  The Gram matrix must therefore be the
    exact X X^T (rounded once to FP32)."""
    rng = np.random.default_rng(21)
    m, n = 32, 64
    w = 1.5 * 2.0 ** (-5 - rng.integers(0, 6, m))
    X0 = (w[:, None] * _signs(m, n, rng)).astype(np.float32)
    c16, s16, g16 = Q.quantize_cols(X0)
    assert not np.array_equal(Q.dequantize_cols(c16, s16, g16), X0)   # premise
    trace = []
    R.ns_iterations_nvfp4(X0, 1, *MUON, trace=trace)
    exact = X0.astype(np.float64) @ X0.T.astype(np.float64)
    assert np.array_equal(trace[0]["A"], exact.astype(np.float32))


def test_update_uses_the_column_blocked_view():
    """Columns of constant magnitude: the 16x1 view of X is exact, the 1x16
    view is not.  The update X_1 - a X_0 must be qB times the exact X_0."""
    rng = np.random.default_rng(22)
    m, n = 32, 64
    w = 1.5 * 2.0 ** (-5 - rng.integers(0, 6, n))
    X0 = (_signs(m, n, rng) * w[None, :]).astype(np.float32)
    c1, s1, g1 = Q.quantize_rows(X0)
    assert not np.array_equal(Q.dequantize_rows(c1, s1, g1), X0)       # premise
    trace = []
    a = MUON[0]
    R.ns_iterations_nvfp4(X0, 1, *MUON, trace=trace)
    qb = Q.dequantize_rows(*trace[0]["qB"])
    want = (a * X0.astype(np.float64) + qb @ X0.astype(np.float64)).astype(np.float32)
    assert np.array_equal(trace[0]["X_next"], want)


def test_combine_step_uses_the_quantised_square_and_the_fp32_gram_by_hand():
    """One iteration worked out by hand (Section 3.4, second line of the iteration:
    B = b A + c qA qA16x1).  X_0 is 16 x 16 with two non-zero rows, [6, 0, ...] and
    [1, 1.5, 0, ...]; both of its NVFP4 views are exact (s_g = 2^-8, block scales
    256 and 64).  Then, by hand:
      A = X X^T:   A00 = 36, A01 = 6, A11 = 3.25 (FP32-exact, not NVFP4-exact);
      qA:  s_g = 2^-6; row 0 [36, 6]: scale 384, den 6, codes 6, 1 (exact);
           row 1 [6, 3.25]: scale 64, den 1, 3.25 rounds to the E2M1 value 3;
           the 16x1 view of the symmetric A has the same values;
      P = deq(qA) deq(qA16) = [[36, 6], [6, 3]]^2 = [[1332, 234], [234, 45]];
      B = -0.5 A + 0.25 P = [[315, 55.5], [55.5, 9.625]];
      qB:  s_g = 2^-3; row 0: 315 / 0.75 = 420 -> scale 416, den 52, codes 6 (312),
           1 (52); row 1: 55.5 / 0.75 = 74 -> scale 72, den 9, codes 6 (54), 1 (9);
      X_1 = 1 * X + deq(qB) X = [[1930, 78], [334, 15]] in the top-left corner.
    The two plausible misreadings give different B: squaring the FP32 A
    (P = A A: B01 = 55.875, B11 = 10.015625) and using deq(qA) in the b A term
    (B11 = 9.75)."""
    X0 = np.zeros((16, 16), np.float32)
    X0[0, 0] = 6.0
    X0[1, 0], X0[1, 1] = 1.0, 1.5
    a, b, c = 1.0, -0.5, 0.25
    trace = []
    R.ns_iterations_nvfp4(X0, 1, a, b, c, trace=trace)
    t = trace[0]

    def corner(M, vals):
        want = np.zeros((16, 16))
        want[:2, :2] = vals
        return np.array_equal(np.asarray(M, np.float64), want)

    assert corner(t["A"], [[36.0, 6.0], [6.0, 3.25]])
    assert corner(Q.dequantize_rows(*t["qA"]), [[36.0, 6.0], [6.0, 3.0]])
    assert corner(t["P"], [[1332.0, 234.0], [234.0, 45.0]])
    assert corner(t["B"], [[315.0, 55.5], [55.5, 9.625]])
    assert corner(Q.dequantize_rows(*t["qB"]), [[312.0, 52.0], [54.0, 9.0]])
    want_x1 = np.zeros((16, 16))
    want_x1[:2, :2] = [[1930.0, 78.0], [334.0, 15.0]]
    assert np.array_equal(t["X_next"].astype(np.float64), want_x1)
    # the misreadings are distinguishable on this input
    A = np.asarray(t["A"], np.float64)
    assert not corner(b * A + c * (A @ A), [[315.0, 55.5], [55.5, 9.625]])
    dqa = Q.dequantize_rows(*t["qA"])
    assert not corner(b * dqa + c * np.asarray(t["P"]), [[315.0, 55.5], [55.5, 9.625]])

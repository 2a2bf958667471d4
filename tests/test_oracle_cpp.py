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
from oracle import momentum as M
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


# ---------------------------------------------------------------- options of Section 3.4
# H16^r ("a fresh 16x16 random Hadamard transform"), adaptive 4/6 block scaling and the
# nearest-rank quantile clip ("p99 outlier clipping", Table 8 "Root quantile ratio").

MASKS = [0x0000, 0x0001, 0x8000, 0xA5C3, 0x3A5C, 0xFFFF]


def _awkward(shape, seed):
    """Heavy-tailed values with signed zeros, an all-zero block and a few outliers."""
    rng = np.random.default_rng(seed)
    x = rng.standard_t(3, shape) * 0.02
    x[rng.random(shape) < 0.02] *= 300.0
    x[rng.random(shape) < 0.05] = -0.0
    x[:, 16:32] = 0.0
    return x.astype(np.float32)


@pytest.mark.parametrize("mask", MASKS)
def test_hadamard_bit_exact_against_the_numpy_oracle(mask):
    x = _awkward((48, 96), 11)
    for fc, fn in ((C.hadamard_rows, Q.hadamard_rows), (C.hadamard_cols, Q.hadamard_cols)):
        got, want = fc(x, mask), fn(x, mask)
        assert np.array_equal(got.view(np.uint32), want.view(np.uint32))


@pytest.mark.parametrize("mask", MASKS)
def test_hadamard_matches_the_matrix_definition(mask):
    """y = x D H16 / 4 from the Sylvester matrix: each FP32 output is four levels of
    additions of the block's 16 inputs, so it lies within 4 * 2^-24 * sum|x_block|
    (before the exact / 4) of the float64 value.  A block of unit vectors gives
    the rows of D H16 / 4 exactly."""
    x = _awkward((24, 64), 12)
    got = C.hadamard_rows(x, mask).astype(np.float64)
    want = Q.hadamard_rows_f64(x, mask)
    bound = 4 * 2.0 ** -24 * np.abs(x.astype(np.float64)).reshape(24, 4, 16).sum(axis=2) / 4
    assert np.all(np.abs(got - want).reshape(24, 4, 16) <= bound[:, :, None] + 1e-45)
    eye = np.eye(16, dtype=np.float32)
    Hr = np.diag(Q.mask_signs(mask)) @ Q.sylvester16() / 4.0
    assert np.array_equal(C.hadamard_rows(eye, mask).astype(np.float64), Hr)


def test_hadamard_refuses_a_bad_mask_or_shape():
    with pytest.raises(ValueError):
        C.hadamard_rows(np.zeros((2, 24), np.float32), 0)
    with pytest.raises(ValueError):
        C.hadamard_rows(np.zeros((2, 16), np.float32), 0x10000)


def test_adaptive46_hand_worked_blocks(golden_dir):
    with open(os.path.join(golden_dir, "adaptive46_blocks.json")) as f:
        data = json.load(f)
    for case in data["cases"]:
        x = np.array(case["x"], dtype=np.float32).reshape(1, -1)
        codes, scales, sg = C.quantize_rows(x, s_g=case["s_g"], adaptive46=True)
        assert scales.tobytes().hex() == "".join(case["scales_hex"]), case["name"]
        assert codes.tobytes().hex() == "".join(case["codes_hex"]), case["name"]


@pytest.mark.parametrize("kind", ["gauss", "awkward", "half_steps", "tiny"])
@pytest.mark.parametrize("mode", ["pow2", "amax"])
def test_quantise_adaptive46_bit_exact_against_the_numpy_oracle(kind, mode):
    rng = np.random.default_rng(13)
    if kind == "gauss":
        x = (rng.standard_normal((48, 192)) * rng.lognormal(0, 1, (48, 1))).astype(np.float32)
    elif kind == "awkward":
        x = _awkward((48, 192), 14)
    elif kind == "half_steps":       # many blocks that one of the candidates holds exactly
        x = (np.round(rng.standard_normal((48, 192)) * 4) / 2).astype(np.float32)
    else:
        x = (rng.standard_normal((48, 192)) * 1e-30).astype(np.float32)
    for fc, fn in ((C.quantize_rows, Q.quantize_rows), (C.quantize_cols, Q.quantize_cols)):
        c1, s1, g1 = fc(x, mode=mode, adaptive46=True)
        c2, s2, g2 = fn(x, mode=mode, adaptive46=True)
        assert g1 == g2 and np.array_equal(s1, s2) and np.array_equal(c1, c2)
    # 4/6 changes some blocks, and keeps M = 6 on others
    _, s46, g46 = C.quantize_rows(x, mode=mode, adaptive46=True)
    _, s6, _ = C.quantize_rows(x, s_g=g46, mode=mode)
    if kind != "tiny":
        assert np.any(s6 != s46) and np.any(s6 == s46)


def test_quantile_clip_hand_worked_vector():
    # |G| = {5, 1, 3, 2, 4}; q = 0.5 -> rank 3 -> tau = fp32(3 inv); -5 and 4 clamp to -+tau
    G = np.array([[-5.0, 1.0, 3.0, -2.0, 4.0]], np.float32)
    X0, inv, tau, norm = C.normalise_and_clip(G, None, clip_quantile=0.5)
    assert norm == pytest.approx(np.sqrt(55.0), rel=1e-15)
    assert tau == np.float32(3.0) * inv
    assert np.array_equal(X0, np.array([[-tau, 1.0 * inv, tau, -2.0 * inv, tau]], np.float32))


@pytest.mark.parametrize("q", [0.99, 0.5, 0.999, 1.0, 1e-9])
def test_quantile_clip_matches_the_numpy_oracle(q):
    G = _awkward((64, 96), 15)
    X1, inv1, tau1, n1 = C.normalise_and_clip(G, 3.0, clip_quantile=q)   # the quantile wins
    X2, inv2, tau2, n2 = R.normalise_and_clip(G, 3.0, clip_quantile=q)
    assert inv1 == inv2 and tau1 == tau2 and abs(n1 - n2) <= 1e-12 * n2
    assert np.array_equal(X1.view(np.uint32), X2.view(np.uint32))


OPTIONS = [dict(), dict(adaptive46=True), dict(rht=True), dict(rht=True, adaptive46=True),
           dict(rht=True, adaptive46=True, mode="amax")]


def _opts(o, K, seed):
    o = dict(o)
    masks = None
    if o.pop("rht", False):
        masks = [int(v) for v in np.random.default_rng(seed).integers(0, 1 << 16, 3 * K)]
    return dict(o, rht_masks=masks)


@pytest.mark.parametrize("opts", OPTIONS, ids=lambda o: "+".join(sorted(o)) or "plain")
@pytest.mark.parametrize("shape,K,coef", [((48, 112), 3, MUON), ((32, 32), 2, QUINTIC)])
def test_iteration_options_bit_identical_to_the_numpy_steps(opts, shape, K, coef):
    """The numpy iteration with its own codec, H16^r and 4/6 and the C++ product in
    place of BLAS (so that both sum every product in k order) gives the C++
    iteration's FP32 iterate bit for bit: every quantisation, transform, mask
    index and combine agrees."""
    rng = np.random.default_rng(16)
    X0 = R.normalise_and_clip((rng.standard_t(4, shape) * 0.02).astype(np.float32), 3.0)[0]
    o = _opts(opts, K, 17)
    got = C.ns_iterations_nvfp4(X0, K, *coef, **o)
    want = R.ns_iterations_nvfp4(X0, K, *coef, matmul=C.product, **o)
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32))


@pytest.mark.parametrize("opts", OPTIONS[1:4], ids=lambda o: "+".join(sorted(o)))
@pytest.mark.parametrize("shape", [(64, 160), (160, 64)])
def test_root_ns_options_match_the_numpy_oracle(opts, shape):
    """The whole step with each option (and the 0.99 quantile clip) against the numpy
    oracle with BLAS products: equal up to float64 summation order."""
    K = 3
    rng = np.random.default_rng(18)
    G = (rng.standard_t(3, shape) * 0.02).astype(np.float32)
    o = _opts(opts, K, 19)
    for clip in (dict(clip_k=3.0), dict(clip_k=None, clip_quantile=0.99)):
        got = C.root_ns(G, K, *MUON, **clip, **o)
        want = R.root_ns(G, K, *MUON, **clip, **o)
        assert got.shape == want.shape
        assert np.linalg.norm(got - want) <= 1e-6 * np.linalg.norm(want)


def test_float64_route_quantile_clip_matches_the_numpy_oracle():
    """Both float64 routes with the 0.99 quantile clip agree; q = 1 clips nothing, so
    that route equals the unclipped one, whose closed form is pinned above."""
    rng = np.random.default_rng(20)
    G = (rng.standard_t(3, (48, 80)) * 0.02).astype(np.float32)
    for impl in (C, R):
        got = impl.root_ns(G, 3, *MUON, clip_k=None, clip_quantile=0.99, quantized=False)
        assert np.all(np.isfinite(got)) and got.shape == G.shape
        q1 = impl.root_ns(G, 3, *MUON, clip_k=None, clip_quantile=1.0, quantized=False)
        none = impl.root_ns(G, 3, *MUON, clip_k=None, quantized=False)
        assert np.array_equal(q1, none)
    got = C.root_ns(G, 3, *MUON, clip_k=None, clip_quantile=0.99, quantized=False)
    want = R.root_ns(G, 3, *MUON, clip_k=None, clip_quantile=0.99, quantized=False)
    assert np.linalg.norm(got - want) <= 1e-12 * np.linalg.norm(want)
    assert np.linalg.norm(got - C.root_ns(G, 3, *MUON, clip_k=None, quantized=False)) > 0


def test_too_few_masks_are_refused():
    X0 = np.zeros((16, 16), np.float32)
    with pytest.raises(ValueError):
        C.ns_iterations_nvfp4(X0, 2, *MUON, rht_masks=[1, 2, 3, 4, 5])
    with pytest.raises(ValueError):
        C.root_ns(X0, 1, *MUON, rht_masks=[1, 2, 0x10000])


# ---------------------------------------------------------------- BF16 route and NVFP4 momentum
# The BF16 comparison step (Section 4.4, Table 6) and the NVFP4 first moment (Section 3.3,
# which Section 3.4's momentum follows), restated in C++ and pinned to the same things as
# the numpy oracle: the published SplitMix64 outputs, hand-checkable roundings, and the
# numpy oracle bit for bit.

def test_splitmix64_reference_outputs_and_draws():
    z = C.splitmix64(0, np.arange(3, dtype=np.uint64))
    assert [int(v) for v in z] == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]
    idx = np.arange(1 << 12, dtype=np.uint64)
    for seed in (0, 1, 12345, 2 ** 63 + 5, 2 ** 64 - 1):
        assert np.array_equal(C.splitmix64(seed, idx), M.splitmix64(seed, idx))
        u = C.uniform24(seed, idx)
        assert np.array_equal(u, M.uniform24(seed, idx))
        assert u.min() >= 0.0 and u.max() < 1.0


def test_stochastic_rounding_against_the_numpy_oracle_and_by_hand():
    grid = Q.E2M1_MAGNITUDES.astype(np.float32)
    for code, g in enumerate(grid):                 # grid points never move
        for u in (0.0, 0.5, 1 - 2 ** -24):
            assert C.sr_encode_magnitude([g], [u])[0] == code
    # v = 2.5 lies halfway between 2 (code 4) and 3 (code 5): up exactly when u < 0.5
    assert list(C.sr_encode_magnitude([2.5, 2.5, 2.5], [0.0, 0.4999999, 0.5])) == [5, 5, 4]
    assert list(C.sr_encode_magnitude([6.0, 7.5, 1e30], [0.0, 0.0, 0.9])) == [7, 7, 7]
    rng = np.random.default_rng(21)
    v = np.concatenate([rng.uniform(0, 7, 3000), [0.25, 0.75, 5.999, 1e-30]]).astype(np.float32)
    u = rng.uniform(0, 1, v.size).astype(np.float32)
    assert np.array_equal(C.sr_encode_magnitude(v, u), M.sr_encode_magnitude(v, u))


@pytest.mark.parametrize("masks,seeds", [((0x0000, 0x5A5A), (1, 2)), ((0xA5C3, 0xFFFF), (99, 2 ** 40 + 3))])
def test_momentum_steps_bit_exact_against_the_numpy_oracle(masks, seeds):
    rng = np.random.default_rng(22)
    g1 = (rng.standard_t(3, (64, 96)) * 0.02).astype(np.float32)
    g2 = (rng.standard_t(3, (64, 96)) * 0.02).astype(np.float32)
    g1[:, 32:48] = 0.0                                # an all-zero block
    state_c = state_n = None
    mask_prev = 0
    for g, mask, seed, beta in ((g1, masks[0], seeds[0], 0.9), (g2, masks[1], seeds[1], 0.95)):
        mc, state_c = C.momentum_update(g, beta, state_c, mask_prev, mask, seed)
        mn, state_n = M.update(g, beta, state_n, mask_prev, mask, seed)
        assert np.array_equal(mc.view(np.uint32), mn.view(np.uint32))
        assert state_c[2] == state_n[2]
        assert np.array_equal(state_c[0], state_n[0]) and np.array_equal(state_c[1], state_n[1])
        dc, dn = C.momentum_load(*state_c, mask), M.load(*state_n, mask)
        assert np.array_equal(dc.view(np.uint32), dn.view(np.uint32))
        mask_prev = mask


def test_momentum_beta_zero_stores_the_gradient():
    """beta = 0: m_t = g exactly.  Decoding the state undoes H16^r, which is orthogonal, so
    each block's error has the L2 norm of its error in the transformed domain: at most
    sqrt(16) elements x the widest E2M1 gap (2) x the block's scale s_b s_g (plus FP32
    rounding of the two transforms)."""
    rng = np.random.default_rng(23)
    g = (rng.standard_normal((16, 64)) * 0.02).astype(np.float32)
    m, st = C.momentum_update(g, 0.0, None, 0, 0x3C3C, 5)
    assert np.array_equal(m, g)
    back = C.momentum_load(*st, 0x3C3C).astype(np.float64)
    den = Q.E4M3_VALUES[st[1]].astype(np.float64) * float(st[2])          # 16 x 4 blocks
    err = np.linalg.norm((back - g).reshape(16, 4, 16), axis=2)
    gb = np.linalg.norm(g.astype(np.float64).reshape(16, 4, 16), axis=2)
    assert np.all(err <= 4 * 2 * den + 1e-5 * gb)
    assert np.all(err > 0)                                                  # SR moved every block


def test_bf16_round_against_the_numpy_oracle_and_by_hand():
    # 1 + 2^-8 is a tie between 1 and 1 + 2^-7: it goes to the even mantissa (1);
    # 1 + 3 * 2^-8 is a tie between 1 + 2^-7 and 1 + 2^-6: it goes to 1 + 2^-6
    x = np.float32([1 + 2 ** -8, 1 + 3 * 2 ** -8, 1 + 2 ** -8 + 2 ** -20, -2.0, 0.0, -0.0])
    want = np.float32([1.0, 1 + 2 ** -6, 1 + 2 ** -7, -2.0, 0.0, -0.0])
    got = C.bf16_round(x)
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32))
    y = (np.random.default_rng(24).standard_normal((40, 64)) * 10.0 ** np.arange(-20, 20, 0.625)).astype(np.float32)
    assert np.array_equal(C.bf16_round(y).view(np.uint32), R.bf16_round(y).view(np.uint32))


@pytest.mark.parametrize("shape,K,coef", [((48, 112), 3, MUON), ((32, 32), 2, QUINTIC), ((16, 40), 5, CUBIC)])
def test_bf16_iteration_bit_identical_to_the_numpy_steps(shape, K, coef):
    rng = np.random.default_rng(25)
    X0 = R.normalise_and_clip((rng.standard_t(4, shape) * 0.02).astype(np.float32), 3.0)[0]
    got = C.ns_iterations_bf16(X0, K, *coef)
    want = R.ns_iterations_bf16(X0, K, *coef, matmul=C.product)
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32))


@pytest.mark.parametrize("shape", [(64, 160), (160, 64)])
def test_bf16_route_matches_the_numpy_oracle(shape):
    rng = np.random.default_rng(26)
    G = (rng.standard_t(3, shape) * 0.02).astype(np.float32)
    got = C.root_ns(G, 3, *MUON, clip_k=3.0, bf16=True)
    want = R.root_ns(G, 3, *MUON, clip_k=3.0, bf16=True)
    assert got.shape == want.shape
    assert np.linalg.norm(got - want) <= 1e-6 * np.linalg.norm(want)

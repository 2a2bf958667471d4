"""Pins of the oracle's NVFP4 momentum store ("Full-Stack FP4" Section 3.3: Hadamard
mixing before stochastic rounding and adaptive 4/6 quantisation; Section 3.4: Q-Root's
first-order momentum follows that recipe).

What fixes each part independently of the oracle's own code:
  * the generator: SplitMix64's published reference outputs for seed 0;
  * stochastic rounding: exact expectations over a dense grid of u, grid points and
    saturation, and the bracket property;
  * the inverse transform: the float64 matrix inverse (H16^r)^-1 = H16 D / 4, exact
    round trips on small integers;
  * the update and the store: beta = 0, the zero state, the 4/6 choice (the kept
    candidate never has the larger error), and unbiasedness of SR over seeds.
"""
import numpy as np
import pytest

from oracle import momentum as M
from oracle import nvfp4 as Q


def test_splitmix64_reference_outputs():
    # the first three outputs of SplitMix64 started at 0 (reference implementation)
    z = M.splitmix64(0, np.arange(3, dtype=np.uint64))
    assert [int(v) for v in z] == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_uniform24_is_exact_and_spread():
    u = M.uniform24(12345, np.arange(1 << 18, dtype=np.uint64))
    assert u.dtype == np.float32 and u.min() >= 0.0 and u.max() < 1.0
    assert np.all((u.astype(np.float64) * 2 ** 24) % 1 == 0)          # multiples of 2^-24
    hist = np.bincount((u * 64).astype(int), minlength=64)
    expect = u.size / 64
    chi2 = float(np.sum((hist - expect) ** 2 / expect))
    assert chi2 < 130            # 63 degrees of freedom: far above the 99.99th percentile would fail
    assert abs(float(u.mean()) - 0.5) < 0.005


def test_sr_on_grid_points_and_saturation():
    grid = Q.E2M1_MAGNITUDES.astype(np.float32)
    for code, g in enumerate(grid):
        for u in (0.0, 0.5, 1 - 2 ** -24):
            assert M.sr_encode_magnitude(np.array([g]), np.array([u], np.float32))[0] == code
    v = np.array([6.0, 7.5, 1e30], np.float32)
    assert np.all(M.sr_encode_magnitude(v, np.zeros(3, np.float32)) == 7)


def test_sr_expectation_over_dense_u_grid():
    # over u = k / 2^14 the expected value of the SR result equals v to 2^-14 of the gap
    u = (np.arange(1 << 14, dtype=np.float64) / (1 << 14)).astype(np.float32)
    rng = np.random.default_rng(0)
    for v in np.concatenate([rng.uniform(0, 6, 40), [0.25, 0.75, 1.25, 2.5, 5.0, 5.999]]).astype(np.float32):
        codes = M.sr_encode_magnitude(np.full(u.shape, v, np.float32), u)
        vals = Q.E2M1_MAGNITUDES[codes]
        lo = Q.E2M1_MAGNITUDES[Q.E2M1_MAGNITUDES <= v].max()
        hi = Q.E2M1_MAGNITUDES[Q.E2M1_MAGNITUDES >= v].min()
        assert set(np.unique(vals)) <= {lo, hi}
        assert abs(vals.mean() - float(v)) <= (hi - lo) * 2 ** -14 + 1e-12


def test_inverse_transform_matches_the_matrix_inverse():
    rng = np.random.default_rng(1)
    y = rng.standard_normal((8, 64)).astype(np.float32)
    for mask in (0, 0xBEEF, 0xFFFF):
        Hr = np.diag(Q.mask_signs(mask)) @ Q.sylvester16() / 4.0
        want = (y.astype(np.float64).reshape(8, 4, 16) @ np.linalg.inv(Hr)).reshape(8, 64)
        got = M.inverse_hadamard_rows(y, mask).astype(np.float64)
        assert np.max(np.abs(got - want)) <= 4e-6 * np.max(np.abs(want))
        # small integers: every butterfly sum is exact, so the round trip is exact
        x = rng.integers(-8, 9, (4, 32)).astype(np.float32)
        assert np.array_equal(M.inverse_hadamard_rows(Q.hadamard_rows(x, mask), mask), x)


def test_update_with_beta_zero_and_zero_state():
    rng = np.random.default_rng(2)
    g = (rng.standard_normal((16, 64)) * 1e-3).astype(np.float32)
    m_t, _ = M.update(g, 0.0, None)
    assert np.array_equal(m_t, g)
    m_t, _ = M.update(g, 0.9, None)
    assert np.array_equal(m_t, (np.float32(np.float32(1) - np.float32(0.9)) * g).astype(np.float32))


def test_store_keeps_the_smaller_error_candidate_and_round_trips():
    rng = np.random.default_rng(3)
    m = (rng.standard_t(3, (32, 256)) * 1e-3).astype(np.float32)
    codes, scales, s_g = M.store(m, 0x1234, seed=7)
    y = Q.hadamard_rows(m, 0x1234)
    blocks = y.reshape(32, 16, 16)
    deq = Q.dequantize_rows(codes, scales, s_g, dtype=np.float32).reshape(32, 16, 16)
    u = M.uniform24(7, np.arange(m.size, dtype=np.uint64)).reshape(blocks.shape)
    _, _, d6 = M._quantize_blocks_sr(blocks, s_g, 6.0, u)
    _, _, d4 = M._quantize_blocks_sr(blocks, s_g, 4.0, u)
    e = lambda d: np.sum((blocks.astype(np.float64) - d) ** 2, axis=2)
    chosen = e(deq)
    assert np.all(chosen <= np.minimum(e(d6), e(d4)) * (1 + 1e-5) + 1e-30)
    back = M.load(codes, scales, s_g, 0x1234)
    rel = np.linalg.norm(back - m) / np.linalg.norm(m)
    assert rel < 0.2


def test_stochastic_rounding_is_unbiased_over_seeds():
    rng = np.random.default_rng(4)
    m = (rng.standard_normal((16, 64)) * 1e-3).astype(np.float32)
    acc = np.zeros(m.shape)
    n = 200
    for seed in range(n):
        acc += M.load(*M.store(m, 0x0F0F, seed), 0x0F0F)
    single = np.linalg.norm(M.load(*M.store(m, 0x0F0F, 0), 0x0F0F) - m)
    mean_err = np.linalg.norm(acc / n - m)
    assert mean_err < 0.25 * single       # averaging cancels the rounding noise

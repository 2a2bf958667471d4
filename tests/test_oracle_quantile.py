"""Pins of the oracle's quantile clip ("Full-Stack FP4" Section 3.4: "p99 outlier
clipping"; Table 8: "Root quantile ratio 0.99").

Reading (the pages do not define the quantile): tau is the nearest-rank q-quantile of
|X_0|, the k-th smallest |x| with k = ceil(fl64(q32) * N), and X_0 is clamped to
[-tau, tau] after normalisation.  The pins check the rank arithmetic on hand-worked
values, the order statistic through counts (not by sorting), the degenerate ratios,
a hand example, and the identity the GPU path relies on (the quantile of fp32(G inv)
is fp32(quantile of |G| * inv)).
"""
import numpy as np
import pytest

from oracle import root_ns as R


def test_rank_follows_the_fp32_ratio():
    # fl32(0.6) = 0.600000023841857910156250 > 0.6, so 0.6 * 5 rounds up to rank 4
    assert R.quantile_rank(0.6, 5) == 4
    # 0.5 is exact: ceil(2.5) = 3
    assert R.quantile_rank(0.5, 5) == 3
    # fl32(0.99) = 0.990000009536743164062500: 99.000001 -> the largest of 100 values
    assert R.quantile_rank(0.99, 100) == 100
    # ... and rank 990 of 1000 needs the product 990.00001 -> 991
    assert R.quantile_rank(0.99, 1000) == 991
    assert R.quantile_rank(1.0, 12345) == 12345
    assert R.quantile_rank(1e-12, 12345) == 1


@pytest.mark.parametrize("seed", range(6))
def test_threshold_is_the_kth_smallest_by_counting(seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(1, 3000))
    kind = seed % 3
    if kind == 0:
        x = rng.standard_normal(n)
    elif kind == 1:                       # heavy ties
        x = rng.choice([-3.0, -1.0, 0.0, 0.5, 2.0, 7.0], n)
    else:
        x = rng.standard_t(3, n) * np.exp(rng.uniform(-20, 5, n))
    x = x.astype(np.float32)
    for q in (0.99, 0.5, 0.9, 1.0, 0.01):
        tau = R.quantile_clip_threshold(x, q)
        k = R.quantile_rank(q, n)
        a = np.abs(x)
        assert np.count_nonzero(a < tau) < k <= np.count_nonzero(a <= tau)
        assert np.any(a == tau)


def test_ratio_one_clips_nothing_and_tiny_ratio_gives_the_minimum():
    rng = np.random.default_rng(7)
    G = (rng.standard_normal((48, 80)) * 0.02).astype(np.float32)
    X_none, inv, _, _ = R.normalise_and_clip(G, None)
    X_q1, inv1, tau1, _ = R.normalise_and_clip(G, None, clip_quantile=1.0)
    assert inv == inv1
    assert tau1 == np.abs(X_none).max()
    assert np.array_equal(X_q1, X_none)
    _, _, tau0, _ = R.normalise_and_clip(G, None, clip_quantile=1e-9)
    assert tau0 == np.abs(X_none).min()


def test_hand_worked_vector():
    # |G| = {5, 1, 3, 2, 4}; q = 0.5 -> k = 3 -> the third smallest |G| is 3, so
    # tau = fp32(3 * inv) and the entries -5 and 4 are clamped to -tau and +tau
    G = np.array([[-5.0, 1.0, 3.0, -2.0, 4.0]], np.float32)
    X0, inv, tau, norm = R.normalise_and_clip(G, None, clip_quantile=0.5)
    assert norm == pytest.approx(np.sqrt(55.0), rel=1e-15)
    assert tau == np.float32(3.0) * inv
    want = np.array([[-tau, 1.0 * inv, tau, -2.0 * inv, tau]], np.float32)
    assert np.array_equal(X0, want)


@pytest.mark.parametrize("seed", range(4))
def test_quantile_of_scaled_matrix_is_scaled_quantile_of_raw_magnitudes(seed):
    # X_0 = fp32(G * inv) with inv > 0 is a monotone map of |G|, so its k-th smallest
    # magnitude is fp32(k-th smallest |G| * inv): the quantile can be selected on |G|
    rng = np.random.default_rng(100 + seed)
    G = (rng.standard_t(3, (64, 96)) * 0.02).astype(np.float32)
    _, inv, tau, _ = R.normalise_and_clip(G, None, clip_quantile=0.99)
    k = R.quantile_rank(0.99, G.size)
    raw = np.sort(np.abs(G).ravel())[k - 1]
    assert tau == np.float32(raw) * inv


def test_root_ns_with_quantile_clip_runs_and_q1_matches_no_clip():
    rng = np.random.default_rng(3)
    G = (rng.standard_normal((64, 160)) * 0.02).astype(np.float32)
    a, b, c = 15 / 8, -10 / 8, 3 / 8
    y_q1 = R.root_ns(G, 2, a, b, c, clip_k=0.0, clip_quantile=1.0)
    y_none = R.root_ns(G, 2, a, b, c, clip_k=0.0)
    assert np.array_equal(y_q1, y_none)
    y = R.root_ns(G, 2, a, b, c, clip_quantile=0.99)
    assert np.all(np.isfinite(y)) and not np.array_equal(y, y_none)

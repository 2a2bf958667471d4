"""How sensitive the NVFP4 Newton-Schulz iteration is to FP32 rounding (CPU only).

"Full-Stack FP4" (arXiv 2607.04422), Section 3.4: the iteration stores A_k, B_k and
X_k as FP32 tensors and quantises them to NVFP4 before each product.  Two facts
about the method decide which end-to-end tolerance is attainable:

  * accumulating the products in FP32 instead of float64 changes nothing that
    matters: the dequantised operands carry few significant bits, so the sums are
    nearly always exact in FP32 (checked here at K = 1..5);
  * one FP32 rounding of B_k = b A_k + c qA_k qA16_k taken differently (a +-1 ulp
    change, as an FMA-based evaluation of the combine gives) is amplified by the
    Muon coefficients (3.4445, -4.7750, 2.0315): the outputs of two such
    evaluations agree within 2e-2 up to K = 3 and differ by more than 2e-2 at K = 5.
    The contractive quintic (15/8, -10/8, 3/8) does not amplify it.

So a product within the 1e-5 per-GEMM tolerance cannot promise the 2e-2 end-to-end
tolerance at K = 5 with the Muon coefficients; the GPU tests assert 2e-2 where this
test shows it is attainable (K <= 3 with Muon, K = 5 with the quintic) and, at K = 5
with Muon, one oracle iteration from the GPU's own iterate at every k.
"""
import numpy as np
import pytest

from oracle import root_ns as R

MUON = (3.4445, -4.7750, 2.0315)
QUINTIC = (15 / 8, -10 / 8, 3 / 8)


def _x0(seed=3, shape=(512, 1536)):
    rng = np.random.default_rng(seed)
    G = (rng.standard_normal(shape) * 0.02).astype(np.float32)
    return R.normalise_and_clip(G, 3.0)[0]


def _one_ulp_noise_on_b(seed):
    """A perturbation hook: every entry of B_k moves by one ulp up or down (random,
    kept symmetric), i.e. another valid FP32 rounding of the same combine."""
    rng = np.random.default_rng(seed)

    def hook(k, name, T):
        if name != "B":
            return T
        s = rng.choice([-1, 1], T.shape)
        s = np.triu(s) + np.triu(s, 1).T
        up = np.nextafter(T, np.float32(np.inf))
        down = np.nextafter(T, np.float32(-np.inf))
        return np.where(s > 0, up, down).astype(np.float32)

    return hook


def _fp32_products(left, right):
    return (left.astype(np.float32) @ right.astype(np.float32)).astype(np.float64)


def _trajectories(coef, K, **kw):
    X0 = _x0()
    base, other = [], []
    xb, xo = X0, X0
    hook = kw.get("perturb")
    for k in range(K):
        xb = R.ns_iterations_nvfp4(xb, 1, *coef)
        extra = dict(kw)
        if hook is not None:
            extra["perturb"] = (lambda kk, name, T, k=k: hook(k, name, T))
        xo = R.ns_iterations_nvfp4(xo, 1, *coef, **extra)
        base.append(xb)
        other.append(xo)
    return [float(np.linalg.norm(o - b) / np.linalg.norm(b)) for b, o in zip(base, other)]


def test_fp32_accumulation_of_the_products_changes_nothing_that_matters():
    for coef in (MUON, QUINTIC):
        gaps = _trajectories(coef, 5, matmul=_fp32_products)
        assert max(gaps) <= 1e-6, gaps


def test_one_ulp_in_the_combine_is_amplified_by_the_muon_coefficients():
    gaps = _trajectories(MUON, 5, perturb=_one_ulp_noise_on_b(1))
    assert max(gaps[:3]) <= 2e-2, gaps       # K <= 3: within the end-to-end tolerance
    assert gaps[4] > 2e-2, gaps              # K = 5: beyond it
    assert gaps[4] > 10 * max(gaps[2], 1e-6), gaps


def test_one_ulp_in_the_combine_is_not_amplified_by_the_quintic():
    gaps = _trajectories(QUINTIC, 5, perturb=_one_ulp_noise_on_b(1))
    assert max(gaps) <= 2e-2, gaps

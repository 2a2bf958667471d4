"""GPU parity of the tcgen05 block-scaled NVFP4 GEMM.

Operands are quantised by the oracle from seeded inputs, laid out in the
TILED layout and handed to the kernel; the expected value is the oracle's
float64 product of the same dequantised operands.  Tolerance: relative
Frobenius error 1e-5 (FP32 accumulation in TMEM).
"""
import numpy as np
import pytest
import torch

from oracle import nvfp4 as Q
from tests.helpers import plain_to_tiled, rel_frob

pytestmark = pytest.mark.gpu


def _operand(x, mode="pow2"):
    codes, scales, sg = Q.quantize_rows(x, mode=mode)
    ct, st = plain_to_tiled(codes, scales, x.shape[0], x.shape[1])
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    return (codes, scales, sg), (dev(ct), dev(st), dev(np.array([sg], np.float32)))


@pytest.mark.parametrize("M,N,K", [
    (128, 256, 256), (256, 256, 1024), (200, 300, 528), (16, 16, 16), (128, 128, 256),
    (384, 640, 768), (1024, 1024, 4096), (2048, 2304, 2048),
])
def test_gemm_matches_float64_product_of_identical_operands(fs4, M, N, K):
    rng = np.random.default_rng(M * 7 + N * 3 + K)
    a = (rng.standard_normal((M, K)) * 0.02).astype(np.float32)
    b = rng.standard_t(3, (N, K)).astype(np.float32)
    (ac, as_, ag), A = _operand(a)
    (bc, bs, bg), B = _operand(b)
    want = Q.product_f64(ac, as_, ag, bc, bs, bg)
    got = fs4.gemm(A, B, M, N, K).cpu().numpy()
    assert rel_frob(got, want) <= 1e-5


def test_gemm_textbook_scale_and_strided_output(fs4):
    rng = np.random.default_rng(5)
    M, N, K = 256, 512, 512
    a = rng.standard_normal((M, K)).astype(np.float32)
    b = rng.standard_normal((N, K)).astype(np.float32)
    (ac, as_, ag), A = _operand(a, "amax")
    (bc, bs, bg), B = _operand(b, "amax")
    out = torch.full((M, N + 40), 7.0, device="cuda")
    fs4.gemm(A, B, M, N, K, out=out[:, :N])
    got = out.cpu().numpy()
    want = Q.product_f64(ac, as_, ag, bc, bs, bg)
    assert rel_frob(got[:, :N], want) <= 1e-5
    assert np.all(got[:, N:] == 7.0)


def test_gemm_exact_on_exactly_representable_operands(fs4):
    """Small-integer operands: every product and partial sum is exact in FP32."""
    rng = np.random.default_rng(6)
    M, N, K = 128, 256, 512
    a = rng.choice([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], (M, K)) * rng.choice([-1, 1], (M, K))
    b = rng.choice([0.0, 0.5, 1.0, 2.0, 6.0], (N, K)) * rng.choice([-1, 1], (N, K))
    a[:, ::16] = 6.0          # every block's amax is 6: s_g = 2^-8, every scale decodes to 256
    b[:, ::16] = 6.0
    (ac, as_, ag), A = _operand(a.astype(np.float32))
    (bc, bs, bg), B = _operand(b.astype(np.float32))
    want = Q.product_f64(ac, as_, ag, bc, bs, bg)
    got = fs4.gemm(A, B, M, N, K).cpu().numpy()
    assert np.array_equal(got.astype(np.float64), want)

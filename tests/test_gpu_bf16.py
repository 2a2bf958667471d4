"""GPU parity of the BF16 comparison step (fs4_root_ns_bf16_batched): the same
Newton-Schulz plan with BF16 operands on tcgen05 kind::f16, the optimized BF16
baseline that "Full-Stack FP4" (Section 4.4, Table 6) compares Q-Root against.

Expected values come from oracle.root_ns.ns_iterations_bf16 / root_ns(bf16=True).
Tolerances: every BF16 view bit-exact (the oracle's round-to-nearest-even of the
GPU's own FP32 tensor); each product within 5e-5 of the float64 product of the GPU's
own BF16 operands (a BF16 x BF16 product has a 16-bit significand, so unlike the NVFP4
products the FP32 sum over K terms is not exact: its rounding error grows like
sqrt(K) u to K u, u = 2^-24, i.e. up to 2.4e-4 at K = 4096; measured 1.3e-5); end to end within 2e-2 of the BF16 oracle and, against the float64
iteration, within 4e-2 (Muon, K = 5; the BF16 route itself is 1.4-2.2% from float64
there) with the orthogonality error within 10%.
"""
import numpy as np
import pytest
import torch

from oracle import root_ns as R
from tests.helpers import rel_frob, tiled_bf16_to_plain, ws_f32
from tests.test_gpu_ns import momentum, working

pytestmark = pytest.mark.gpu

MUON = (3.4445, -4.7750, 2.0315)
QUINTIC = (15 / 8, -10 / 8, 3 / 8)
CUBIC = (1.5, -0.5, 0.0)
TOL_PRODUCT = 5e-5


def run_bf16(F, G, K, coef, clip_k=3.0, flags=0):
    Gt = torch.from_numpy(G).cuda()
    need = F.ns_bf16_batched_workspace_size([G.shape])
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    out = F.root_ns_bf16_batched([Gt], K, [coef], clip_k=clip_k, workspace=ws, flags=flags)[0]
    assert F.device_status(ws) == 0
    return out.cpu().numpy(), ws.cpu().numpy()


def bview(ws, off, rows, cols):
    return tiled_bf16_to_plain(ws[off:off + 2 * rows * cols], rows, cols)


def upper(mp):
    t = np.arange(mp) // 256
    return t[:, None] <= t[None, :]


def sym(M, mp):
    return np.where(upper(mp), M, M.T)


@pytest.mark.parametrize("shape,kind", [((256, 256), "gauss"), ((48, 80), "gauss"),
                                        ((1024, 4096), "outliers"), ((320, 96), "student")])
def test_bf16_preamble_views_bit_exact(fs4, shape, kind):
    G = momentum(*shape, kind=kind, seed=21)
    _, ws = run_bf16(fs4, G, 1, MUON, flags=fs4.stop_after(0))
    lay = fs4.ns_bf16_layout([shape], 0)
    mp, np_ = lay.mp, lay.np
    X0 = R.normalise_and_clip(working(G), 3.0)[0]
    m, n = X0.shape
    Xg = ws_f32(ws, lay.X, mp * np_).reshape(mp, np_)
    assert np.array_equal(Xg[:m, :n].view(np.uint32), X0.view(np.uint32))
    Xp = np.zeros((mp, np_), np.float32)
    Xp[:m, :n] = X0
    assert np.array_equal(bview(ws, lay.qX_codes[0], mp, np_).view(np.uint32),
                          R.bf16_round(Xp).view(np.uint32))
    assert np.array_equal(bview(ws, lay.qXT_codes[0], np_, mp).view(np.uint32),
                          R.bf16_round(np.ascontiguousarray(Xp.T)).view(np.uint32))


@pytest.mark.parametrize("shape,kind", [((256, 256), "gauss"), ((1024, 4096), "outliers"),
                                        ((4096, 1024), "student"), ((768, 1280), "gauss"),
                                        ((48, 80), "gauss")])
@pytest.mark.parametrize("coef", [(0.0, 0.0, 1.0), MUON])
def test_bf16_products_against_float64_and_views_bit_exact(fs4, shape, kind, coef):
    """The three products of the first iteration, each against the float64 product of
    the GPU's own BF16 operands (TOL_PRODUCT), and every BF16 view the epilogues write
    (A, B and both views of X_1) bit for bit."""
    G = momentum(*shape, kind=kind, seed=22)
    lay = fs4.ns_bf16_layout([shape], 0)
    mp, np_ = lay.mp, lay.np
    m, n = min(shape), max(shape)
    b32, c32, a32 = (np.float64(np.float32(v)) for v in (coef[1], coef[2], coef[0]))
    _, w0 = run_bf16(fs4, G, 2, coef, flags=fs4.stop_after(0))
    _, w1 = run_bf16(fs4, G, 2, coef, flags=fs4.stop_after(1))
    _, w2 = run_bf16(fs4, G, 2, coef, flags=fs4.stop_after(2))
    _, w3 = run_bf16(fs4, G, 2, coef, flags=fs4.stop_after(3))
    up = upper(mp)
    # product 1: A = Xb Xb^T
    Xb = bview(w0, lay.qX_codes[0], mp, np_).astype(np.float64)
    A = np.where(up, ws_f32(w1, lay.A, mp * mp).reshape(mp, mp), np.float32(0))
    Aw = Xb @ Xb.T
    assert rel_frob(A[up], Aw[up]) <= TOL_PRODUCT
    Ab = bview(w1, lay.qA_codes, mp, mp)
    assert np.array_equal(Ab.view(np.uint32), R.bf16_round(sym(A, mp)).view(np.uint32))
    # product 2: B = b A + c Ab Ab^T (written over A by the debug stop)
    B = np.where(up, ws_f32(w2, lay.A, mp * mp).reshape(mp, mp), np.float32(0))
    Ab64 = Ab.astype(np.float64)
    Bw = b32 * sym(A, mp).astype(np.float64) + c32 * (Ab64 @ Ab64.T)
    assert rel_frob(B[up], Bw[up]) <= TOL_PRODUCT
    Bb = bview(w2, lay.qB_codes, mp, mp)
    assert np.array_equal(Bb.view(np.uint32), R.bf16_round(sym(B, mp)).view(np.uint32))
    # product 3: X1 = a X0 + Bb Xb^T-view (the update operand is the BF16 copy of X^T)
    X0 = ws_f32(w2, lay.X, mp * np_).reshape(mp, np_).astype(np.float64)
    XbT = bview(w2, lay.qXT_codes[0], np_, mp).astype(np.float64)
    X1w = a32 * X0 + Bb.astype(np.float64) @ XbT.T
    X1 = ws_f32(w3, lay.X, mp * np_).reshape(mp, np_)
    assert rel_frob(X1[:m, :n], X1w[:m, :n]) <= TOL_PRODUCT
    assert np.array_equal(bview(w3, lay.qX_codes[1], mp, np_).view(np.uint32),
                          R.bf16_round(X1).view(np.uint32))
    assert np.array_equal(bview(w3, lay.qXT_codes[1], np_, mp).view(np.uint32),
                          R.bf16_round(np.ascontiguousarray(X1.T)).view(np.uint32))


@pytest.mark.parametrize("shape,kind,K,coef", [
    ((256, 256), "gauss", 5, MUON), ((1024, 4096), "outliers", 5, MUON),
    ((4096, 1024), "student", 5, MUON), ((512, 1536), "gauss", 5, QUINTIC),
    ((48, 80), "gauss", 3, CUBIC), ((272, 528), "outliers", 5, QUINTIC),
])
def test_bf16_end_to_end_against_the_bf16_oracle_and_float64(fs4, shape, kind, K, coef):
    G = momentum(*shape, kind=kind, seed=23)
    got, _ = run_bf16(fs4, G, K, coef)
    want = R.root_ns(G, K, *coef, clip_k=3.0, bf16=True)
    assert got.shape == G.shape and np.all(np.isfinite(got))
    assert rel_frob(got, want) <= 2e-2
    f64 = R.root_ns(G, K, *coef, clip_k=3.0, quantized=False)
    assert rel_frob(got, f64) <= 4e-2
    eo, eg = R.orthogonality_error(f64), R.orthogonality_error(got)
    assert abs(eg - eo) <= 0.1 * eo


def test_bf16_batch_of_mixed_shapes_and_coefficients(fs4):
    rng = np.random.default_rng(78)
    specs = []
    for i in range(7):
        m, n = (int(v) * 16 for v in rng.integers(1, 40, 2))
        specs.append(((m, n), (MUON, QUINTIC, CUBIC)[i % 3]))
    Gs = [momentum(*s, kind=("gauss", "student", "outliers")[i % 3], seed=300 + i)
          for i, (s, _) in enumerate(specs)]
    coeffs = [c for _, c in specs]
    outs = fs4.root_ns_bf16_batched([torch.from_numpy(G).cuda() for G in Gs], K=3, coeffs=coeffs)
    torch.cuda.synchronize()
    for G, o, coef in zip(Gs, outs, coeffs):
        got = o.cpu().numpy()
        assert rel_frob(got, R.root_ns(G, 3, *coef, clip_k=3.0, bf16=True)) <= 2e-2, G.shape


def test_bf16_full_size_one_block_every_shape_class(fs4):
    """The seven matrices of one 3B-class block in one batched call (the bench's launch
    configuration), K = 5 Muon: one matrix of each shape class against the BF16 oracle."""
    from nvfp4_precision_optimizer_b200.workloads import BASE_SEED, WORKLOADS, matrices
    w = WORKLOADS["3b_1block_gauss"]
    Gs = matrices(w, device="cuda", seed=BASE_SEED)
    outs = fs4.root_ns_bf16_batched(Gs, K=w.K, coeffs=w.coeffs, clip_k=w.clip_k)
    torch.cuda.synchronize()
    shapes = [tuple(G.shape) for G in Gs]
    for i in sorted({s: i for i, s in enumerate(shapes)}.values()):
        got = outs[i].cpu().numpy()
        want = R.root_ns(Gs[i].cpu().numpy(), w.K, *w.coeffs[i], clip_k=w.clip_k, bf16=True)
        assert rel_frob(got, want) <= 2e-2, shapes[i]


def test_bf16_rejects_the_nvfp4_quantiser_options(fs4):
    G = torch.zeros((64, 64), device="cuda")
    with pytest.raises(fs4.Fs4Error):
        fs4.root_ns_bf16_batched([G], 1, flags=fs4.FS4_NS_RHT)

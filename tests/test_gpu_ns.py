"""GPU parity of the direct NVFP4 Newton-Schulz step (fs4_root_ns / _batched).

Inputs are seeded synthetic momenta; expected values come from oracle/ on the
same FP32 input.  Tolerances:
  * preamble (normalise, clip, both NVFP4 views): bit-exact;
  * each product of an iteration (A = qX qX^T, B = b A + c qA qA16x1,
    X' = a X + qB qX16x1): relative Frobenius <= 1e-5 against the float64
    product of the GPU's own dequantised operands, and every NVFP4 view an
    epilogue writes is the oracle's quantisation of the GPU's FP32 result,
    byte for byte;
  * end-to-end: relative Frobenius <= 2e-2 and orthogonality error within 10%
    of the oracle's wherever that is attainable: K <= 3 with the Muon
    coefficients and K = 5 with the contractive quintic and cubic.  At K = 5 with
    the Muon coefficients a one-ulp change in the FP32 rounding of B moves the
    oracle's own output by about 10% (tests/test_oracle_sensitivity.py), so
    there the orthogonality error within 10% and the singular-value spectrum
    within 5% are asserted, and every iteration is checked on its own: one oracle
    iteration from the GPU's X_k against the GPU's X_{k+1}, within 2e-2.
"""
import numpy as np
import pytest
import torch

from oracle import nvfp4 as Q
from oracle import root_ns as R
from tests.helpers import rel_frob, tiled_to_plain, ws_f32


def view(ws, codes_off, scales_off, rows, cols):
    """PLAIN codes/scales of a rows x cols TILED view stored in the workspace."""
    nc, ns = rows * cols // 2, rows * cols // 16
    c, s, _, _ = tiled_to_plain(ws[codes_off:codes_off + nc], ws[scales_off:scales_off + ns], rows, cols)
    return c, s

pytestmark = pytest.mark.gpu

MUON = (3.4445, -4.7750, 2.0315)
QUINTIC = (15 / 8, -10 / 8, 3 / 8)
CUBIC = (1.5, -0.5, 0.0)


def momentum(m, n, kind="gauss", seed=0):
    rng = np.random.default_rng(seed)
    if kind == "gauss":
        g = rng.standard_normal((m, n)) * 0.02
    elif kind == "outliers":
        g = rng.standard_normal((m, n)) * 0.02
        g[rng.random((m, n)) < 0.001] *= 50
    elif kind == "student":
        t = rng.standard_t(3, (m, n))
        g = t * (0.02 / np.sqrt(np.mean(t * t)))
    else:
        raise ValueError(kind)
    return g.astype(np.float32)


def run_gpu(F, G, K, coef, clip_k=3.0, flags=0):
    Gt = torch.from_numpy(G).cuda()
    ws = torch.zeros(F.ns_workspace_size(*G.shape), dtype=torch.uint8, device="cuda")
    out = F.root_ns(Gt, K, *coef, clip_k=clip_k, workspace=ws, flags=flags)
    assert F.device_status(ws) == 0
    return out.cpu().numpy(), ws.cpu().numpy()


def working(G):
    return G.T if G.shape[0] > G.shape[1] else G


@pytest.mark.parametrize("shape,kind", [((256, 256), "gauss"), ((48, 80), "gauss"),
                                        ((1024, 4096), "outliers"), ((320, 96), "student"),
                                        ((512, 272), "gauss")])
def test_preamble_bit_exact(fs4, shape, kind):
    G = momentum(*shape, kind=kind, seed=1)
    _, ws = run_gpu(fs4, G, 1, MUON, flags=fs4.stop_after(0))
    lay = fs4.ns_layout([shape], 0)
    mp, np_ = lay.mp, lay.np
    X0, inv, tau, _ = R.normalise_and_clip(working(G), 3.0)
    m, n = X0.shape
    Xg = ws_f32(ws, lay.X, mp * np_).reshape(mp, np_)
    assert np.array_equal(Xg[:m, :n].view(np.uint32), X0.view(np.uint32))
    assert not Xg[m:].any() and not Xg[:, n:].any()
    sg = ws_f32(ws, lay.scalars, 192)
    c, s, g = Q.quantize_rows(X0)
    assert sg[0] == g
    gc, gs = view(ws, lay.qX_codes[0], lay.qX_scales[0], mp, np_)
    assert np.array_equal(gs[:m, :n // 16], s) and np.array_equal(gc[:m, :n // 2], c)
    ct, st, gt = Q.quantize_cols(X0)
    assert gt == g
    gc, gs = view(ws, lay.qXT_codes[0], lay.qXT_scales[0], np_, mp)
    assert np.array_equal(gs[:n, :m // 16], st) and np.array_equal(gc[:n, :m // 2], ct)


@pytest.mark.parametrize("shape,kind", [((256, 256), "gauss"), ((1024, 4096), "outliers"),
                                        ((512, 768), "student"), ((48, 80), "gauss")])
def test_first_gram_product_and_its_requantisation(fs4, shape, kind):
    G = momentum(*shape, kind=kind, seed=2)
    _, ws = run_gpu(fs4, G, 1, MUON, flags=fs4.stop_after(1))
    lay = fs4.ns_layout([shape], 0)
    mp = lay.mp
    X0, _, _, _ = R.normalise_and_clip(working(G), 3.0)
    m = X0.shape[0]
    c, s, g = Q.quantize_rows(X0)
    dX = Q.dequantize_rows(c, s, g)
    A = dX @ dX.T
    Ag = ws_f32(ws, lay.A, mp * mp).reshape(mp, mp).astype(np.float64)
    upper = (np.arange(mp)[:, None] // 256) <= (np.arange(mp)[None, :] // 256)
    Aw = np.zeros((mp, mp))
    Aw[:m, :m] = A
    assert rel_frob(Ag[upper], Aw[upper]) <= 1e-5
    assert not Ag[upper & ((np.arange(mp)[:, None] >= m) | (np.arange(mp)[None, :] >= m))].any()
    # the GPU's tensor scale of A is a power of two that covers amax(A)
    sga = ws_f32(ws, lay.scalars, 192)[64]
    assert 2688 * sga >= np.abs(A).max() and np.log2(sga) == int(np.log2(sga))
    # requantised A (both triangles, from the 1x16 view and the mirrored 16x1 view)
    A32 = R.symmetric_from_upper(A).astype(np.float32)
    oc, os_, og = Q.quantize_rows(A32)
    want = Q.dequantize_rows(oc, os_, og)
    gc, gs = view(ws, lay.qA_codes, lay.qA_scales, mp, mp)
    got = Q.dequantize_rows(gc[:m, :m // 2], gs[:m, :m // 16], sga)
    diff = got != want
    assert diff.mean() <= 2e-3
    # where they differ, the FP32 inputs straddled a rounding boundary: one grid step apart
    assert np.all(np.abs(got - want)[diff] <= 0.51 * np.maximum(np.abs(got), np.abs(want))[diff] + 1e-30)


def _upper_tiles_to_full(Ag, mp):
    """Symmetric mp x mp matrix from the 256 x 256 tiles on and above the diagonal."""
    t = np.arange(mp) // 256
    upper = t[:, None] <= t[None, :]
    return np.where(upper, Ag, Ag.T)


@pytest.mark.parametrize("shape,kind", [((256, 256), "gauss"), ((48, 80), "gauss"),
                                        ((1024, 4096), "outliers"), ((4096, 1024), "student"),
                                        ((768, 1280), "gauss")])
def test_epilogue_requantisation_bit_exact(fs4, shape, kind):
    """The fused GEMM epilogues quantise their own FP32 results exactly as Q1x16 and
    Q16x1 do (Section 3.4): the GPU's FP32 A_0 and X_1, quantised by the oracle with
    the GPU's tensor scales, give the GPU's codes and scales byte for byte, on both
    triangles of A (the lower one comes from the mirrored 16x1 view) and on both views
    of X_1, padding included."""
    G = momentum(*shape, kind=kind, seed=5)
    lay = fs4.ns_layout([shape], 0)
    mp, np_ = lay.mp, lay.np
    # A_0 after the first Gram product
    _, ws = run_gpu(fs4, G, 2, MUON, flags=fs4.stop_after(1))
    A = _upper_tiles_to_full(ws_f32(ws, lay.A, mp * mp).reshape(mp, mp), mp)
    sga = ws_f32(ws, lay.scalars, 192)[64]
    oc, os_, _ = Q.quantize_rows(np.ascontiguousarray(A, dtype=np.float32), s_g=sga)
    gc, gs = view(ws, lay.qA_codes, lay.qA_scales, mp, mp)
    assert np.array_equal(gs, os_) and np.array_equal(gc, oc)
    # X_1 after the first update (K = 2, so it is requantised for iteration 1)
    _, ws = run_gpu(fs4, G, 2, MUON, flags=fs4.stop_after(3))
    X1 = ws_f32(ws, lay.X, mp * np_).reshape(mp, np_)
    sgx = ws_f32(ws, lay.scalars, 192)[1]
    assert 2688 * sgx >= np.abs(X1).max()
    oc, os_, _ = Q.quantize_rows(X1, s_g=sgx)
    gc, gs = view(ws, lay.qX_codes[1], lay.qX_scales[1], mp, np_)
    assert np.array_equal(gs, os_) and np.array_equal(gc, oc)
    oc, os_, _ = Q.quantize_rows(np.ascontiguousarray(X1.T), s_g=sgx)
    gc, gs = view(ws, lay.qXT_codes[1], lay.qXT_scales[1], np_, mp)
    assert np.array_equal(gs, os_) and np.array_equal(gc, oc)


def _spectrum_rel(a, b):
    sa = np.linalg.svd(working(a).astype(np.float64), compute_uv=False)
    sb = np.linalg.svd(working(b).astype(np.float64), compute_uv=False)
    return float(np.linalg.norm(sa - sb) / np.linalg.norm(sb))


@pytest.mark.parametrize("shape,kind,K,coef", [
    ((256, 256), "gauss", 1, MUON), ((256, 256), "gauss", 3, MUON),
    ((1024, 4096), "outliers", 2, MUON), ((1024, 4096), "outliers", 3, MUON),
    ((48, 80), "gauss", 3, MUON), ((4096, 1024), "student", 2, MUON),
    ((512, 1536), "gauss", 5, QUINTIC), ((1536, 512), "student", 5, QUINTIC),
    ((272, 528), "outliers", 5, QUINTIC), ((256, 768), "gauss", 5, CUBIC),
])
def test_end_to_end_parity(fs4, shape, kind, K, coef):
    G = momentum(*shape, kind=kind, seed=3)
    got, _ = run_gpu(fs4, G, K, coef)
    want = R.root_ns(G, K, *coef, clip_k=3.0)
    assert got.shape == G.shape
    assert rel_frob(got, want) <= 2e-2
    eo, eg = R.orthogonality_error(want), R.orthogonality_error(got)
    assert abs(eg - eo) <= 0.1 * eo


@pytest.mark.parametrize("shape,kind", [((256, 256), "gauss"), ((1024, 4096), "outliers")])
def test_five_muon_steps_orthogonality_and_spectrum(fs4, shape, kind):
    G = momentum(*shape, kind=kind, seed=4)
    got, _ = run_gpu(fs4, G, 5, MUON)
    want = R.root_ns(G, 5, *MUON, clip_k=3.0)
    eo, eg = R.orthogonality_error(want), R.orthogonality_error(got)
    assert abs(eg - eo) <= 0.1 * eo
    assert _spectrum_rel(got, want) <= 5e-2
    assert np.all(np.isfinite(got))


def test_batched_matches_single_calls_and_oracle(fs4):
    specs = [((256, 256), "gauss", MUON), ((128, 384), "gauss", QUINTIC),
             ((384, 128), "student", CUBIC), ((48, 80), "outliers", MUON),
             ((512, 1024), "gauss", QUINTIC)]
    Gs = [momentum(*s, kind=k, seed=10 + i) for i, (s, k, _) in enumerate(specs)]
    coeffs = [c for _, _, c in specs]
    Gt = [torch.from_numpy(G).cuda() for G in Gs]
    outs = fs4.root_ns_batched(Gt, K=3, coeffs=coeffs, clip_k=3.0)
    torch.cuda.synchronize()
    for G, Gd, o, coef in zip(Gs, Gt, outs, coeffs):
        single = fs4.root_ns(Gd, 3, *coef, clip_k=3.0).cpu().numpy()
        got = o.cpu().numpy()
        assert np.array_equal(got, single)
        assert rel_frob(got, R.root_ns(G, 3, *coef, clip_k=3.0)) <= 2e-2


def test_strided_input_and_output(fs4):
    G = momentum(96, 160, seed=5)
    big = torch.zeros((96, 200), device="cuda")
    big[:, :160] = torch.from_numpy(G).cuda()
    out = torch.full((96, 176), -1.0, device="cuda")
    fs4.root_ns(big[:, :160], 3, *QUINTIC, out=out[:, :160])
    got = out.cpu().numpy()
    assert np.all(got[:, 160:] == -1.0)
    assert rel_frob(got[:, :160], R.root_ns(G, 3, *QUINTIC)) <= 2e-2


def test_no_clip(fs4):
    G = momentum(128, 256, kind="outliers", seed=6)
    got, _ = run_gpu(fs4, G, 3, QUINTIC, clip_k=0.0)
    assert rel_frob(got, R.root_ns(G, 3, *QUINTIC, clip_k=None)) <= 2e-2


def test_zero_input(fs4):
    got, _ = run_gpu(fs4, np.zeros((64, 128), np.float32), 5, MUON)
    assert not got.any()


def test_nonfinite_input_reports_status_and_zero_output(fs4):
    G = momentum(64, 128, seed=7)
    G[5, 9] = np.inf
    Gt = torch.from_numpy(G).cuda()
    ws = torch.zeros(fs4.ns_workspace_size(64, 128), dtype=torch.uint8, device="cuda")
    out = fs4.root_ns(Gt, 3, workspace=ws)
    assert fs4.device_status(ws) == -7
    assert not out.cpu().numpy().any()


def test_bounded_wait_timeout_reports_status_and_context_survives(fs4):
    """A device wait that runs out (FS4_TEST_STALL: the first Gram product's MMA issuer
    waits on a barrier nothing arrives on) ends the call with FS4_ERR_TIMEOUT in the
    status word within a few seconds, with no fault; the next call on the same stream
    is correct."""
    import time
    G = momentum(256, 256, seed=11)
    Gt = torch.from_numpy(G).cuda()
    ws = torch.zeros(fs4.ns_workspace_size(256, 256), dtype=torch.uint8, device="cuda")
    t0 = time.time()
    fs4.root_ns(Gt, 2, *MUON, workspace=ws, flags=fs4.FS4_TEST_STALL)
    torch.cuda.synchronize()
    assert time.time() - t0 < 30.0
    assert fs4.device_status(ws) == -8          # FS4_ERR_TIMEOUT
    got, ws2 = run_gpu(fs4, G, 2, MUON)         # fresh workspace, same context
    want = R.root_ns(G, 2, *MUON, clip_k=3.0)
    assert rel_frob(got, want) <= 2e-2


@pytest.mark.parametrize("shape,kind,K,coef", [
    ((16, 16), "gauss", 3, QUINTIC),          # the smallest legal matrix: one padded tile
    ((16, 4096), "gauss", 3, QUINTIC),        # m = 16: a 16 x 16 Gram inside one 256 x 256 tile
    ((4096, 16), "student", 3, QUINTIC),      # tall: processed as its 16 x 4096 transpose
    ((272, 272), "outliers", 3, QUINTIC),     # one row and column past a 256 boundary
    ((2064, 256), "gauss", 2, CUBIC),         # tall: working 256 x 2064, n padded to 2304
])
def test_extreme_shapes_parity(fs4, shape, kind, K, coef):
    G = momentum(*shape, kind=kind, seed=6)
    got, _ = run_gpu(fs4, G, K, coef)
    want = R.root_ns(G, K, *coef, clip_k=3.0)
    assert got.shape == G.shape and np.all(np.isfinite(got))
    assert rel_frob(got, want) <= 2e-2


def test_batch_of_random_shapes_matches_oracle(fs4):
    """A batch of random multiple-of-16 shapes (both orientations, different paddings)
    with per-matrix coefficients, against the oracle one by one."""
    rng = np.random.default_rng(77)
    specs = []
    for i in range(9):
        m, n = (int(v) * 16 for v in rng.integers(1, 40, 2))
        coef = (QUINTIC, CUBIC)[i % 2]
        specs.append(((m, n), coef))
    Gs = [momentum(*s, kind=("gauss", "student", "outliers")[i % 3], seed=200 + i)
          for i, (s, _) in enumerate(specs)]
    coeffs = [c for _, c in specs]
    Gt = [torch.from_numpy(G).cuda() for G in Gs]
    outs = fs4.root_ns_batched(Gt, K=2, coeffs=coeffs, clip_k=3.0)
    torch.cuda.synchronize()
    for G, o, coef in zip(Gs, outs, coeffs):
        got = o.cpu().numpy()
        assert got.shape == G.shape
        assert rel_frob(got, R.root_ns(G, 2, *coef, clip_k=3.0)) <= 2e-2, G.shape


def test_preamble_keeps_the_sign_of_negative_zeros(fs4):
    """Exact -0.0 entries of G give -0.0 in X_0 and the sign code 0x8 in both views."""
    G = momentum(64, 96, kind="gauss", seed=8)
    rng = np.random.default_rng(8)
    G[rng.random(G.shape) < 0.1] = -0.0
    G[rng.random(G.shape) < 0.05] = 0.0
    _, ws = run_gpu(fs4, G, 1, MUON, flags=fs4.stop_after(0))
    lay = fs4.ns_layout([G.shape], 0)
    X0, _, _, _ = R.normalise_and_clip(G, 3.0)
    Xg = ws_f32(ws, lay.X, lay.mp * lay.np).reshape(lay.mp, lay.np)
    assert np.array_equal(Xg[:64, :96].view(np.uint32), X0.view(np.uint32))
    c, s, _ = Q.quantize_rows(X0)
    gc, gs = view(ws, lay.qX_codes[0], lay.qX_scales[0], lay.mp, lay.np)
    assert np.array_equal(gc[:64, :48], c) and np.array_equal(gs[:64, :6], s)
    ct, st, _ = Q.quantize_cols(X0)
    gc, gs = view(ws, lay.qXT_codes[0], lay.qXT_scales[0], lay.np, lay.mp)
    assert np.array_equal(gc[:96, :32], ct) and np.array_equal(gs[:96, :4], st)


def _ws_runs(fs4, G, K, coef, stops):
    """One call per debug stop on the same input; returns a grab(off, n) per stop."""
    out = {}
    for s in stops:
        _, ws = run_gpu(fs4, G, K, coef, flags=fs4.stop_after(s))
        out[s] = (lambda w: (lambda off, n: w[off:off + n]))(ws)
    return out


@pytest.mark.parametrize("shape,kind", [((256, 256), "gauss"), ((48, 80), "gauss"),
                                        ((1024, 4096), "outliers"), ((4096, 1024), "student"),
                                        ((768, 1280), "gauss")])
@pytest.mark.parametrize("coef", [(0.0, 0.0, 1.0), MUON])
def test_second_and_third_products_against_float64(fs4, shape, kind, coef):
    """Products 2 and 3 of the first iteration (Section 3.4: B = b A + c qA qA16x1 and
    X_1 = a X_0 + qB qX16x1), each against the float64 product of the GPU's own
    dequantised operands, within 1e-5; the epilogues' NVFP4 views of B and X_1 are
    the oracle's quantisation of the GPU's FP32 results, byte for byte.  With
    (a, b, c) = (0, 0, 1) the results are the bare products B = qA qA^T and
    X_1 = qB qX16x1; with the Muon coefficients the fused combines are included."""
    from tests import gemm_checks as GC
    G = momentum(*shape, kind=kind, seed=12)
    lay = fs4.ns_layout([shape], 0)
    m, n = min(shape), max(shape)
    g = _ws_runs(fs4, G, 2, coef, [1, 2, 3])
    err_b, qb_ok = GC.check_second_product(g[1], g[2], lay, 0, coef[1], coef[2])
    assert err_b <= 1e-5, err_b
    assert qb_ok
    err_x = GC.check_third_product(g[2], g[3], lay, 0, coef[0], m, n)
    assert err_x <= 1e-5, err_x
    assert GC.check_first_product_views(g[3], lay, 0, m, n)


@pytest.mark.parametrize("shape,kind", [((256, 256), "gauss"), ((1024, 4096), "outliers"),
                                        ((4096, 1024), "student"), ((512, 1536), "gauss")])
def test_every_muon_iteration_from_the_gpu_iterate(fs4, shape, kind):
    """K = 5 with the Muon coefficients, one iteration at a time: the oracle's NVFP4
    iteration from the GPU's X_k against the GPU's X_{k+1} (the caller's output for
    k = 4), within 2e-2 (Section 3.4)."""
    G = momentum(*shape, kind=kind, seed=13)
    lay = fs4.ns_layout([shape], 0)
    m, n = min(shape), max(shape)
    xs = []
    for k in range(5):
        _, ws = run_gpu(fs4, G, 5, MUON, flags=fs4.stop_after(3 * k))
        xs.append(np.ascontiguousarray(ws_f32(ws, lay.X, lay.mp * lay.np).reshape(lay.mp, lay.np)[:m, :n]))
    out, _ = run_gpu(fs4, G, 5, MUON)
    xs.append(np.ascontiguousarray(working(out)))
    X0 = R.normalise_and_clip(working(G), 3.0)[0]
    assert np.array_equal(xs[0].view(np.uint32), X0.view(np.uint32))
    for k in range(5):
        want = R.ns_iterations_nvfp4(xs[k], 1, *MUON).astype(np.float64)
        assert rel_frob(xs[k + 1], want) <= 2e-2, (k, rel_frob(xs[k + 1], want))

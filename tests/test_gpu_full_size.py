"""Parity at the benchmark's full sizes, in the launch configuration bench.py times
(one batched call over all matrices of a workload).

  * every matrix's preamble is bit-exact for sampled matrices, and sampled entries
    of the first Gram product are within 1e-5 of the oracle's float64 products;
  * each of the three products of an iteration, on every full-size shape class
    (3072 x 3072, tall 8192 x 3072, wide 3072 x 8192, 8192 x 8192), is within 1e-5
    of the float64 product of the GPU's own dequantised operands, and the NVFP4
    views its epilogue writes are the oracle's quantisation of its FP32 result;
  * every iteration k = 0 .. 4 on the 196-matrix 28-block set (all seven roles of
    blocks 0 and 27, with different coefficient triples per matrix) and on the
    8192 x 8192 Student-t matrix: one oracle iteration from the GPU's X_k against
    the GPU's X_{k+1} (the caller's output for the last one), within 2e-2;
  * the output is finite and has the input's shape everywhere.
The oracle runs its numpy iteration with the C++ codec (bit-identical to the numpy
codec, pinned in tests/test_oracle_cpp.py) so that full-size iterations take seconds.
"""
import numpy as np
import pytest
import torch

from nvfp4_precision_optimizer_b200.workloads import BASE_SEED, WORKLOADS, matrices
from oracle import nvfp4 as Q
from oracle import root_ns as R
from tests.helpers import ws_f32
from tests.test_gpu_ns import view, working

pytestmark = pytest.mark.gpu


def _run(fs4, Gs, w, flags=0, coeffs=None, outs=None, ws=None):
    coeffs = w.coeffs if coeffs is None else coeffs
    outs = [torch.empty_like(G) for G in Gs] if outs is None else outs
    if ws is None:
        arr = fs4._descs(Gs, outs, coeffs)
        need = int(fs4._lib.lib().fs4_root_ns_batched_workspace_size(len(Gs), arr))
        ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    fs4.root_ns_batched(Gs, K=w.K, coeffs=coeffs, clip_k=w.clip_k, outs=outs, workspace=ws, flags=flags)
    assert fs4.device_status(ws) == 0
    return outs, ws


def _grabber(ws):
    return lambda off, n: ws[off:off + n].cpu().numpy()


@pytest.mark.parametrize("name", ["3b_4blocks_gauss", "single_8192x8192_student"])
def test_full_size_preamble_and_first_gram_sampled(fs4, name):
    w = WORKLOADS[name]
    Gs = matrices(w, device="cuda", seed=BASE_SEED)
    _, ws = _run(fs4, Gs, w, flags=fs4.stop_after(1))
    shapes = [tuple(G.shape) for G in Gs]
    # one matrix of each shape class
    picks = sorted({s: i for i, s in enumerate(shapes)}.values())
    rng = np.random.default_rng(0)
    wsn = None
    for i in picks:
        lay = fs4.ns_layout(shapes, i)
        mp, np_ = lay.mp, lay.np
        G = Gs[i].cpu().numpy()
        X0, _, _, _ = R.normalise_and_clip(working(G), w.clip_k)
        m, n = X0.shape
        c, s, g = Q.quantize_rows(X0)
        # slice only this matrix's regions out of the (large) workspace
        def grab(off, nbytes):
            return ws[off:off + nbytes].cpu().numpy()
        Xg = grab(lay.X, 4 * mp * np_).view(np.float32).reshape(mp, np_)
        assert np.array_equal(Xg[:m, :n].view(np.uint32), X0.view(np.uint32))
        sg = grab(lay.scalars, 4 * 192).view(np.float32)
        assert sg[0] == g
        nc, ns = mp * np_ // 2, mp * np_ // 16
        from tests.helpers import tiled_to_plain
        gc, gs, _, _ = tiled_to_plain(grab(lay.qX_codes[0], nc), grab(lay.qX_scales[0], ns), mp, np_)
        assert np.array_equal(gc[:m, :n // 2], c) and np.array_equal(gs[:m, :n // 16], s)
        # sampled entries of A_0 = qX qX^T on and above the 256-tile diagonal
        dX = Q.dequantize_rows(c, s, g)
        Ag = grab(lay.A, 4 * mp * mp).view(np.float32).reshape(mp, mp)
        ii = rng.integers(0, m, 400)
        jj = rng.integers(0, m, 400)
        up = (ii // 256) <= (jj // 256)
        ii, jj = ii[up], jj[up]
        want = np.einsum("kj,kj->k", dX[ii], dX[jj])
        got = Ag[ii, jj].astype(np.float64)
        assert np.linalg.norm(got - want) <= 1e-5 * np.linalg.norm(want)


def test_full_size_batched_step_properties(fs4):
    w = WORKLOADS["3b_4blocks_gauss"]
    Gs = matrices(w, device="cuda", seed=BASE_SEED)
    outs, _ = _run(fs4, Gs, w)
    for G, o in zip(Gs, outs):
        assert o.shape == G.shape
        assert torch.isfinite(o).all()
    # full oracle run on the smallest shape class (3072 x 3072): orthogonality within 10%
    i = 0
    got = outs[i].cpu().numpy()
    want = R.root_ns(Gs[i].cpu().numpy(), w.K, *w.coeffs[i], clip_k=w.clip_k)
    eo, eg = R.orthogonality_error(want), R.orthogonality_error(got)
    assert abs(eg - eo) <= 0.1 * eo


def test_full_size_first_iteration_per_shape_class(fs4):
    """One complete iteration (GramX, GramA, Update) inside the full 3b_4blocks_gauss
    batched call (bench.py's launch configuration), stopped after the first update:
    X_1 of one matrix of each shape class (3072^2, tall 8192 x 3072, wide 3072 x 8192)
    against the oracle's NVFP4 iteration from the same X_0.  One step is not chaotic,
    so the relative Frobenius error is held to 2e-2."""
    w = WORKLOADS["3b_4blocks_gauss"]
    Gs = matrices(w, device="cuda", seed=BASE_SEED)
    _, ws = _run(fs4, Gs, w, flags=fs4.stop_after(3))
    shapes = [tuple(G.shape) for G in Gs]
    picks = sorted({s: i for i, s in enumerate(shapes)}.values())
    assert len(picks) == 3
    for i in picks:
        lay = fs4.ns_layout(shapes, i)
        X0, _, _, _ = R.normalise_and_clip(working(Gs[i].cpu().numpy()), w.clip_k)
        m, n = X0.shape
        want = R.ns_iterations_nvfp4(X0, 1, *w.coeffs[i]).astype(np.float64)
        Xg = ws[lay.X:lay.X + 4 * lay.mp * lay.np].cpu().numpy().view(np.float32)
        got = Xg.reshape(lay.mp, lay.np)[:m, :n].astype(np.float64)
        err = np.linalg.norm(got - want) / np.linalg.norm(want)
        assert err <= 2e-2, (shapes[i], err)


@pytest.mark.parametrize("axis", [0, 1])
def test_full_size_standalone_quantise_bit_exact(fs4, axis):
    """fs4_nvfp4_quantize on a whole 8192 x 3072 workload matrix (the bench's --op
    quantize call), every code and scale against the oracle."""
    w = WORKLOADS["3b_1block_gauss"]
    G = matrices(w, device="cuda", seed=BASE_SEED)[4]
    assert tuple(G.shape) == (8192, 3072)
    x = G.cpu().numpy()
    want_c, want_s, want_g = Q.quantize_rows(x) if axis == 0 else Q.quantize_cols(x)
    c, s, g = fs4.quantize(G, axis=axis)
    torch.cuda.synchronize()
    assert np.float32(g.cpu().numpy()[0]) == want_g
    assert np.array_equal(s.cpu().numpy(), want_s)
    assert np.array_equal(c.cpu().numpy(), want_c)


QUINTIC = (15 / 8, -10 / 8, 3 / 8)
CUBIC = (1.5, -0.5, 0.0)


@pytest.mark.parametrize("name", ["3b_1block_gauss", "single_8192x8192_student"])
@pytest.mark.parametrize("coef", [(0.0, 0.0, 1.0), (3.4445, -4.7750, 2.0315)])
def test_full_size_products_against_float64_per_shape_class(fs4, name, coef):
    """Products 2 and 3 (and the views of X_1) of the first iteration for one matrix of
    every shape class, inside the batched call: within 1e-5 of the float64 product of
    the GPU's own operands, views byte for byte.  Product 1 at full size is the
    sampled check above; (a, b, c) = (0, 0, 1) isolates the bare products."""
    from tests import gemm_checks as GC
    w = WORKLOADS[name]
    Gs = matrices(w, device="cuda", seed=BASE_SEED)
    coeffs = [coef] * len(Gs)
    shapes = [tuple(G.shape) for G in Gs]
    picks = sorted({s: i for i, s in enumerate(shapes)}.values())
    grabs = {}
    outs, ws = None, None
    for stop in (1, 2, 3):
        outs, ws = _run(fs4, Gs, w, flags=fs4.stop_after(stop), coeffs=coeffs, outs=outs, ws=ws)
        grabs[stop] = {i: _snapshot(fs4, ws, shapes, i) for i in picks}
    for i in picks:
        lay = fs4.ns_layout(shapes, i)
        m, n = min(shapes[i]), max(shapes[i])
        err_b, qb_ok = GC.check_second_product(grabs[1][i], grabs[2][i], lay, 0, coef[1], coef[2])
        assert err_b <= 1e-5 and qb_ok, (shapes[i], err_b, qb_ok)
        err_x = GC.check_third_product(grabs[2][i], grabs[3][i], lay, 0, coef[0], m, n)
        assert err_x <= 1e-5, (shapes[i], err_x)
        assert GC.check_first_product_views(grabs[3][i], lay, 0, m, n), shapes[i]


def _snapshot(fs4, ws, shapes, i):
    """Host copies of matrix i's state block (tensor scales) and of its big buffers
    (X, A and every NVFP4 view), served through the grab(off, n) interface with
    workspace offsets."""
    lay = fs4.ns_layout(shapes, i)
    s_lo = lay.scalars
    state = ws[s_lo:s_lo + 4 * 192].cpu().numpy()
    lo = lay.X
    hi = lay.qB_scales + lay.mp * lay.mp // 16
    big = ws[lo:hi].cpu().numpy()

    def grab(off, n):
        if s_lo <= off < s_lo + 4 * 192:
            return state[off - s_lo:off - s_lo + n]
        assert lo <= off and off + n <= hi
        return big[off - lo:off - lo + n]

    return grab


def _per_iteration_errors(fs4, Gs, w, coeffs, picks):
    """One oracle iteration from the GPU's X_k against the GPU's X_{k+1}, k = 0..K-1,
    for the matrices in picks; the GPU iterates come from calls stopped after each
    update (X_K is the caller's output)."""
    from oracle import cpp_oracle as C
    shapes = [tuple(G.shape) for G in Gs]
    iters = {i: [] for i in picks}
    outs, ws = None, None
    for k in range(w.K):
        outs, ws = _run(fs4, Gs, w, flags=fs4.stop_after(3 * k), coeffs=coeffs, outs=outs, ws=ws)
        for i in picks:
            lay = fs4.ns_layout(shapes, i)
            m, n = min(shapes[i]), max(shapes[i])
            X = ws[lay.X:lay.X + 4 * lay.mp * lay.np].cpu().numpy().view(np.float32)
            iters[i].append(np.ascontiguousarray(X.reshape(lay.mp, lay.np)[:m, :n]))
    outs, ws = _run(fs4, Gs, w, coeffs=coeffs, outs=outs, ws=ws)
    errs = {}
    for i in picks:
        out = outs[i].cpu().numpy()
        assert np.all(np.isfinite(out)) and out.shape == shapes[i]
        iters[i].append(np.ascontiguousarray(working(out)))
        for k in range(w.K):
            want = R.ns_iterations_nvfp4(iters[i][k], 1, *coeffs[i], codec=C).astype(np.float64)
            got = iters[i][k + 1].astype(np.float64)
            errs[(i, k)] = float(np.linalg.norm(got - want) / np.linalg.norm(want))
    return errs


def test_full_size_every_iteration_28_blocks(fs4):
    """The 196-matrix 28-block Student-t set in one batched call, with the coefficient
    triple changing from matrix to matrix (Muon, quintic, cubic in turn): all seven
    roles of the first and the last block, every iteration."""
    w = WORKLOADS["3b_28blocks_student"]
    Gs = matrices(w, device="cuda", seed=BASE_SEED)
    coeffs = [(MUON_T, QUINTIC, CUBIC)[i % 3] for i in range(len(Gs))]
    picks = list(range(7)) + list(range(len(Gs) - 7, len(Gs)))
    errs = _per_iteration_errors(fs4, Gs, w, coeffs, picks)
    worst = max(errs.values())
    assert worst <= 2e-2, sorted(errs.items(), key=lambda kv: -kv[1])[:5]


def test_full_size_every_iteration_8192_student(fs4):
    w = WORKLOADS["single_8192x8192_student"]
    Gs = matrices(w, device="cuda", seed=BASE_SEED)
    errs = _per_iteration_errors(fs4, Gs, w, w.coeffs, [0])
    assert max(errs.values()) <= 2e-2, errs


MUON_T = (3.4445, -4.7750, 2.0315)

"""Parity at the benchmark's full sizes, in the launch configuration bench.py times
(one batched call over all matrices of a workload).

The oracle cannot redo a whole 3B-class step in seconds, so these tests check
(1) every matrix's preamble bit-exactly for sampled matrices, (2) sampled
entries of the first Gram product, which the oracle computes one by one from
the (bit-identical) quantised rows, within 1e-5, and (3) properties that hold at
any size: the output is finite, has the input's shape, and its orthogonality
error matches a full oracle run on one sampled matrix of each shape class
within 10% (K = 5, Muon coefficients; see tests/test_gpu_ns.py for why the
elementwise comparison is not meaningful there).
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


def _run(fs4, Gs, w, flags=0):
    outs = [torch.empty_like(G) for G in Gs]
    arr = fs4._descs(Gs, outs, w.coeffs)
    need = int(fs4._lib.lib().fs4_root_ns_batched_workspace_size(len(Gs), arr))
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    fs4.root_ns_batched(Gs, K=w.K, coeffs=w.coeffs, clip_k=w.clip_k, outs=outs, workspace=ws, flags=flags)
    assert fs4.device_status(ws) == 0
    return outs, ws


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

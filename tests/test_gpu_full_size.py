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

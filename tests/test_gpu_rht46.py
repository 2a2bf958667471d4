"""GPU parity of the Section 3.4 quantiser options of the Newton-Schulz step:
the random Hadamard transform H16^r on every quantised operand and adaptive 4/6
block scaling ("Full-Stack FP4", Section 3.4).  Expected values come from the
oracle on the same FP32 inputs and the same sign masks:
  * preamble views of X_0: bit-exact (the GPU's tensor scale, which covers
    4 x amax(X_0) under the transform, is checked against that rule);
  * the epilogues' requantisation of the GPU's own FP32 A_0 and X_1: bit-exact;
  * end to end: relative Frobenius <= 2e-2 and orthogonality within 10% on the
    non-chaotic settings, as for the plain route."""
import numpy as np
import pytest
import torch

from oracle import nvfp4 as Q
from oracle import root_ns as R
from tests.helpers import rel_frob, ws_f32
from tests.test_gpu_ns import MUON, QUINTIC, momentum, view, working

pytestmark = pytest.mark.gpu

OPTS = [(True, True), (True, False), (False, True)]   # (rht, adaptive46)


def _masks(K, seed):
    rng = np.random.default_rng(seed)
    return [int(v) for v in rng.integers(0, 1 << 16, 3 * K)]


def _run(fs4, G, K, coef, masks, a46, flags=0):
    Gt = torch.from_numpy(G).cuda()
    ws = torch.zeros(fs4.ns_workspace_size(*G.shape), dtype=torch.uint8, device="cuda")
    out = fs4.root_ns(Gt, K, *coef, workspace=ws, flags=flags, rht_masks=masks, adaptive46=a46)
    assert fs4.device_status(ws) == 0
    return out.cpu().numpy(), ws.cpu().numpy()


def _hr(x, masks, j):
    return x if masks is None else Q.hadamard_rows(x, masks[j])


@pytest.mark.parametrize("rht,a46", OPTS)
@pytest.mark.parametrize("shape,kind", [((256, 256), "gauss"), ((48, 80), "gauss"),
                                        ((1024, 4096), "outliers"), ((320, 96), "student")])
def test_preamble_views_bit_exact(fs4, shape, kind, rht, a46):
    G = momentum(*shape, kind=kind, seed=21)
    masks = _masks(2, 7) if rht else None
    _, ws = _run(fs4, G, 2, MUON, masks, a46, flags=fs4.stop_after(0))
    lay = fs4.ns_layout([shape], 0)
    mp, np_ = lay.mp, lay.np
    X0, _, _, _ = R.normalise_and_clip(working(G), 3.0)
    m, n = X0.shape
    sg = ws_f32(ws, lay.scalars, 192)[0]
    assert sg == Q.global_scale(float(np.max(np.abs(X0))) * (4.0 if rht else 1.0),
                                denom=Q.SG_DENOM_46 if a46 else Q.SG_DENOM)
    c, s, _ = Q.quantize_rows(_hr(X0, masks, 0), s_g=sg, adaptive46=a46)
    gc, gs = view(ws, lay.qX_codes[0], lay.qX_scales[0], mp, np_)
    assert np.array_equal(gs[:m, :n // 16], s) and np.array_equal(gc[:m, :n // 2], c)
    XT = np.ascontiguousarray(X0.T)
    ct, st, _ = Q.quantize_rows(_hr(XT, masks, 2), s_g=sg, adaptive46=a46)
    gc, gs = view(ws, lay.qXT_codes[0], lay.qXT_scales[0], np_, mp)
    assert np.array_equal(gs[:n, :m // 16], st) and np.array_equal(gc[:n, :m // 2], ct)


def _upper_tiles_to_full(Ag, mp):
    t = np.arange(mp) // 256
    return np.where(t[:, None] <= t[None, :], Ag, Ag.T)


@pytest.mark.parametrize("rht,a46", OPTS)
@pytest.mark.parametrize("shape,kind", [((256, 256), "gauss"), ((1024, 4096), "outliers"),
                                        ((4096, 1024), "student"), ((768, 1280), "gauss")])
def test_epilogue_requantisation_bit_exact(fs4, shape, kind, rht, a46):
    G = momentum(*shape, kind=kind, seed=22)
    masks = _masks(2, 8) if rht else None
    lay = fs4.ns_layout([shape], 0)
    mp, np_ = lay.mp, lay.np
    _, ws = _run(fs4, G, 2, MUON, masks, a46, flags=fs4.stop_after(1))
    A = np.ascontiguousarray(_upper_tiles_to_full(ws_f32(ws, lay.A, mp * mp).reshape(mp, mp), mp),
                             dtype=np.float32)
    sga = ws_f32(ws, lay.scalars, 192)[64]
    oc, os_, _ = Q.quantize_rows(_hr(A, masks, 1), s_g=sga, adaptive46=a46)
    gc, gs = view(ws, lay.qA_codes, lay.qA_scales, mp, mp)
    assert np.array_equal(gs, os_) and np.array_equal(gc, oc)
    _, ws = _run(fs4, G, 2, MUON, masks, a46, flags=fs4.stop_after(3))
    X1 = ws_f32(ws, lay.X, mp * np_).reshape(mp, np_)
    sgx = ws_f32(ws, lay.scalars, 192)[1]
    assert (1792 if a46 else 2688) * sgx >= np.abs(X1).max() * (4.0 if rht else 1.0)
    oc, os_, _ = Q.quantize_rows(_hr(X1, masks, 3), s_g=sgx, adaptive46=a46)
    gc, gs = view(ws, lay.qX_codes[1], lay.qX_scales[1], mp, np_)
    assert np.array_equal(gs, os_) and np.array_equal(gc, oc)
    oc, os_, _ = Q.quantize_rows(_hr(np.ascontiguousarray(X1.T), masks, 5), s_g=sgx, adaptive46=a46)
    gc, gs = view(ws, lay.qXT_codes[1], lay.qXT_scales[1], np_, mp)
    assert np.array_equal(gs, os_) and np.array_equal(gc, oc)


@pytest.mark.parametrize("rht,a46", OPTS)
@pytest.mark.parametrize("shape,kind,K,coef", [
    ((256, 256), "gauss", 2, MUON), ((1024, 4096), "outliers", 2, MUON),
    ((512, 1536), "gauss", 5, QUINTIC), ((1536, 512), "student", 5, QUINTIC),
])
def test_end_to_end_parity(fs4, shape, kind, K, coef, rht, a46):
    G = momentum(*shape, kind=kind, seed=23)
    masks = _masks(K, 9) if rht else None
    got, _ = _run(fs4, G, K, coef, masks, a46)
    want = R.root_ns(G, K, *coef, clip_k=3.0, rht_masks=masks, adaptive46=a46)
    assert rel_frob(got, want) <= 2e-2
    eo, eg = R.orthogonality_error(want), R.orthogonality_error(got)
    assert abs(eg - eo) <= 0.1 * eo

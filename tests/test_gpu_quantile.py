"""GPU parity of the quantile clip of the Newton-Schulz preamble (FS4_NS_CLIP_QUANTILE;
"Full-Stack FP4" Section 3.4 "p99 outlier clipping", Table 8 "Root quantile ratio 0.99").

tau is the nearest-rank q-quantile of |X_0|; the GPU selects it exactly, so the clamped
X_0 and both of its NVFP4 views must match the oracle bit for bit.  End to end (the
contractive quintic, two steps) the usual 2e-2 relative Frobenius bound applies.
"""
import numpy as np
import pytest
import torch

from oracle import nvfp4 as Q
from oracle import root_ns as R
from tests.helpers import rel_frob, ws_f32
from tests.test_gpu_ns import QUINTIC, momentum, view, working

pytestmark = pytest.mark.gpu


def run_quantile(F, G, K, coef, q, extra_flags=0, Gt=None):
    if Gt is None:
        Gt = torch.from_numpy(G).cuda()
    ws = torch.zeros(F.ns_workspace_size(*G.shape), dtype=torch.uint8, device="cuda")
    out = F.root_ns(Gt, K, *coef, workspace=ws, flags=extra_flags, clip_quantile=q)
    status = F.device_status(ws)
    return out.cpu().numpy(), ws.cpu().numpy(), status


def check_preamble(F, G, ws, q):
    shape = G.shape
    lay = F.ns_layout([shape], 0)
    mp, np_ = lay.mp, lay.np
    X0, inv, tau, _ = R.normalise_and_clip(working(G), None, clip_quantile=q)
    m, n = X0.shape
    Xg = ws_f32(ws, lay.X, mp * np_).reshape(mp, np_)
    assert np.array_equal(Xg[:m, :n].view(np.uint32), X0.view(np.uint32)), (shape, q)
    assert not Xg[m:].any() and not Xg[:, n:].any()
    sg = ws_f32(ws, lay.scalars, 192)
    c, s, g = Q.quantize_rows(X0)
    assert sg[0] == g
    gc, gs = view(ws, lay.qX_codes[0], lay.qX_scales[0], mp, np_)
    assert np.array_equal(gs[:m, :n // 16], s) and np.array_equal(gc[:m, :n // 2], c)
    ct, st, _ = Q.quantize_cols(X0)
    gc, gs = view(ws, lay.qXT_codes[0], lay.qXT_scales[0], np_, mp)
    assert np.array_equal(gs[:n, :m // 16], st) and np.array_equal(gc[:n, :m // 2], ct)
    return X0, tau


@pytest.mark.parametrize("shape,kind,q", [((256, 256), "gauss", 0.99), ((48, 80), "gauss", 0.5),
                                          ((1024, 4096), "outliers", 0.99),
                                          ((320, 96), "student", 0.99),
                                          ((512, 272), "gauss", 0.9999), ((64, 64), "gauss", 1.0),
                                          ((16, 16), "gauss", 0.01), ((208, 1040), "student", 0.9)])
def test_quantile_preamble_bit_exact(fs4, shape, kind, q):
    G = momentum(*shape, kind=kind, seed=11)
    _, ws, status = run_quantile(fs4, G, 1, QUINTIC, q, fs4.stop_after(0))
    assert status == 0
    X0, tau = check_preamble(fs4, G, ws, q)
    # every entry of rank k and above (N - k + 1 of them) sits at |tau| after the clamp
    k = R.quantile_rank(q, G.size)
    assert np.count_nonzero(np.abs(X0) == tau) >= G.size - k + 1


def test_quantile_with_ties_and_equal_magnitudes(fs4):
    rng = np.random.default_rng(5)
    # many exactly equal magnitudes around the quantile, and a matrix of one magnitude
    # (every key lands in the selected bin: the gather holds all m n keys)
    G1 = (rng.choice([-3.0, -1.0, 0.5, 1.0, 2.0, 4.0], (96, 160)) * 0.01).astype(np.float32)
    G2 = np.where(rng.random((64, 128)) < 0.5, -0.02, 0.02).astype(np.float32)
    # 16 x 1024 = 16384 hits per 16-row unit: the gather's staging buffer fills and flushes
    G3 = np.where(rng.random((64, 1024)) < 0.5, -0.02, 0.02).astype(np.float32)
    for G in (G1, G2, G3):
        for q in (0.99, 0.5, 0.001):
            _, ws, status = run_quantile(fs4, G, 1, QUINTIC, q, fs4.stop_after(0))
            assert status == 0
            check_preamble(fs4, G, ws, q)


def test_quantile_strided_input(fs4):
    G = momentum(208, 304, kind="gauss", seed=21)
    big = torch.zeros((208, 320), dtype=torch.float32, device="cuda")
    big[:, 7:7 + 304] = torch.from_numpy(G).cuda()
    Gt = big[:, 7:7 + 304]
    _, ws, status = run_quantile(fs4, G, 1, QUINTIC, 0.99, fs4.stop_after(0), Gt=Gt)
    assert status == 0
    check_preamble(fs4, G, ws, 0.99)


@pytest.mark.parametrize("shape,kind", [((256, 512), "gauss"), ((384, 128), "student")])
def test_quantile_end_to_end(fs4, shape, kind):
    G = momentum(*shape, kind=kind, seed=31)
    got, _, status = run_quantile(fs4, G, 2, QUINTIC, 0.99)
    assert status == 0
    want = R.root_ns(G, 2, *QUINTIC, clip_quantile=0.99)
    assert rel_frob(got, want) <= 2e-2
    eo, eg = R.orthogonality_error(want), R.orthogonality_error(got)
    assert abs(eg - eo) <= 0.1 * eo + 1e-6


def test_quantile_batched_matches_oracle_per_matrix(fs4):
    shapes = [(256, 256), (128, 384), (400, 144), (64, 64)]
    Gs = [momentum(*s, kind="student", seed=40 + i) for i, s in enumerate(shapes)]
    Gt = [torch.from_numpy(G).cuda() for G in Gs]
    outs = [torch.empty_like(g) for g in Gt]
    arr = fs4._descs(Gt, outs, [QUINTIC] * len(Gt))
    need = int(fs4._lib.lib().fs4_root_ns_batched_workspace_size(len(Gt), arr))
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    fs4.root_ns_batched(Gt, K=1, coeffs=[QUINTIC] * len(Gt), outs=outs, workspace=ws,
                        flags=fs4.stop_after(0), clip_quantile=0.99)
    assert fs4.device_status(ws) == 0
    wsn = ws.cpu().numpy()
    for i, G in enumerate(Gs):
        lay = fs4.ns_layout(shapes, i)
        X0, _, _, _ = R.normalise_and_clip(working(G), None, clip_quantile=0.99)
        m, n = X0.shape
        Xg = ws_f32(wsn, lay.X, lay.mp * lay.np).reshape(lay.mp, lay.np)
        assert np.array_equal(Xg[:m, :n].view(np.uint32), X0.view(np.uint32)), shapes[i]


def test_quantile_nonfinite_input_reports_status_and_zero_output(fs4):
    G = momentum(64, 96, seed=3)
    G[5, 9] = np.inf
    got, _, status = run_quantile(fs4, G, 2, QUINTIC, 0.99)
    assert status == -7
    assert not got.any()

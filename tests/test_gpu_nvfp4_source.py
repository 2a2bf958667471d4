"""GPU parity of the Newton-Schulz step reading its input as an NVFP4 first-moment state
(fs4_root_ns_batched_nvfp4; "Full-Stack FP4" Section 3.4: the first-order momentum follows
the storage recipe of Section 3.3, and the step consumes it).

The decoded matrix is fp32(fp32(code * s) * s_g) then (H16^r)^-1, exactly as the oracle's
momentum.load computes it, so the step from the state must equal, bit for bit, the step
from that FP32 matrix; and its preamble must match the oracle bit for bit.
"""
import numpy as np
import pytest
import torch

from oracle import momentum as M
from oracle import nvfp4 as Q
from oracle import root_ns as R
from tests.helpers import rel_frob, ws_f32
from tests.test_gpu_ns import QUINTIC, momentum, view, working

pytestmark = pytest.mark.gpu


def _state(fs4, shape, kind, seed, mask):
    g = momentum(*shape, kind=kind, seed=seed)
    _, st = fs4.momentum_nvfp4(torch.from_numpy(g).cuda(), 0.9, None, mask=mask, seed=seed)
    torch.cuda.synchronize()
    host = (st[0].cpu().numpy(), st[1].cpu().numpy(), np.float32(st[2].cpu().numpy()[0]))
    return st + (mask,), M.load(*host, mask)


@pytest.mark.parametrize("shape,kind", [((256, 256), "gauss"), ((128, 400), "student"),
                                        ((400, 144), "outliers"), ((48, 1040), "gauss")])
def test_preamble_from_state_bit_exact(fs4, shape, kind):
    st, G = _state(fs4, shape, kind, 31, 0x6B2D)
    ws = torch.zeros(fs4.ns_batched_workspace_size([shape]), dtype=torch.uint8, device="cuda")
    fs4.root_ns_batched_nvfp4([st], K=1, coeffs=[QUINTIC], workspace=ws, flags=fs4.stop_after(0))
    assert fs4.device_status(ws) == 0
    wsn = ws.cpu().numpy()
    lay = fs4.ns_layout([shape], 0)
    X0, _, _, _ = R.normalise_and_clip(working(G), 3.0)
    m, n = X0.shape
    Xg = ws_f32(wsn, lay.X, lay.mp * lay.np).reshape(lay.mp, lay.np)
    assert np.array_equal(Xg[:m, :n].view(np.uint32), X0.view(np.uint32))
    c, s, g = Q.quantize_rows(X0)
    gc, gs = view(wsn, lay.qX_codes[0], lay.qX_scales[0], lay.mp, lay.np)
    assert np.array_equal(gs[:m, :n // 16], s) and np.array_equal(gc[:m, :n // 2], c)
    ct, st_, _ = Q.quantize_cols(X0)
    gc, gs = view(wsn, lay.qXT_codes[0], lay.qXT_scales[0], lay.np, lay.mp)
    assert np.array_equal(gs[:n, :m // 16], st_) and np.array_equal(gc[:n, :m // 2], ct)


@pytest.mark.parametrize("clip_quantile", [None, 0.99])
def test_step_from_state_equals_step_from_its_fp32_decode(fs4, clip_quantile):
    shapes = [(256, 256), (128, 384), (384, 128), (64, 1024)]
    pairs = [_state(fs4, s, ("gauss", "student")[i % 2], 50 + i, (0x1F2E * (i + 1)) & 0xFFFF)
             for i, s in enumerate(shapes)]
    states = [p[0] for p in pairs]
    Gs = [torch.from_numpy(np.ascontiguousarray(p[1])).cuda() for p in pairs]
    coeffs = [QUINTIC] * len(shapes)
    out_q = fs4.root_ns_batched_nvfp4(states, K=3, coeffs=coeffs, clip_quantile=clip_quantile)
    out_f = fs4.root_ns_batched(Gs, K=3, coeffs=coeffs, clip_quantile=clip_quantile)
    torch.cuda.synchronize()
    for a, b, G in zip(out_q, out_f, pairs):
        assert torch.equal(a, b)
        want = R.root_ns(G[1], 3, *QUINTIC, clip_k=3.0, clip_quantile=clip_quantile)
        assert rel_frob(a.cpu().numpy(), want) <= 2e-2

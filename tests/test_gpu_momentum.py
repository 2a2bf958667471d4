"""GPU parity of the NVFP4 first-moment store (fs4_momentum_nvfp4; "Full-Stack FP4"
Section 3.3 first-moment recipe, Section 3.4).

Every decision is taken in FP32 with the same operations on both sides and the random
numbers come from the same counter-based generator, so m_t, the codes, the scales and
the tensor scale must match the oracle bit for bit, step after step.
"""
import numpy as np
import pytest
import torch

from oracle import momentum as M

pytestmark = pytest.mark.gpu


def _grad(rows, cols, kind, seed):
    rng = np.random.default_rng(seed)
    if kind == "gauss":
        g = rng.standard_normal((rows, cols)) * 1e-3
    elif kind == "student":
        g = rng.standard_t(3, (rows, cols)) * 1e-3
    elif kind == "outliers":
        g = rng.standard_normal((rows, cols)) * 1e-3
        g[rng.random((rows, cols)) < 0.001] *= 50
    else:
        g = np.exp(rng.uniform(-20, 2, (rows, 1))) * rng.standard_normal((rows, cols))
    return g.astype(np.float32)


def _gpu_state(st):
    return tuple(t.cpu().numpy() for t in st[:2]) + (np.float32(st[2].cpu().numpy()[0]),)


def _assert_same(gpu_m, gpu_state, want_m, want_state):
    assert np.array_equal(gpu_m.view(np.uint32), want_m.view(np.uint32))
    gc, gs, gg = gpu_state
    wc, ws_, wg = want_state
    assert gg == wg
    assert np.array_equal(gs, ws_), np.argwhere(gs != ws_)[:5]
    assert np.array_equal(gc, wc), np.argwhere(gc != wc)[:5]


@pytest.mark.parametrize("shape,kind", [((64, 256), "gauss"), ((100, 272), "student"),
                                        ((1, 16), "gauss"), ((257, 1024), "outliers"),
                                        ((48, 4096), "wide")])
def test_three_steps_bit_exact(fs4, shape, kind):
    beta = 0.95
    masks = [0x0000, 0xA5C3, 0x1234, 0xFFFF]
    seeds = [11, 12, 13]
    state_o = None
    state_g = None
    for t in range(3):
        g = _grad(*shape, kind, 100 + t)
        want_m, state_o = M.update(g, beta, state_o, masks[t], masks[t + 1], seeds[t])
        m, st = fs4.momentum_nvfp4(torch.from_numpy(g).cuda(), beta, state_g, prev_mask=masks[t],
                                   mask=masks[t + 1], seed=seeds[t])
        torch.cuda.synchronize()
        state_g = st
        _assert_same(m.cpu().numpy(), _gpu_state(st), want_m, state_o)


def test_in_place_step_matches_out_of_place(fs4):
    g0 = _grad(128, 512, "student", 1)
    g1 = _grad(128, 512, "student", 2)
    _, st = fs4.momentum_nvfp4(torch.from_numpy(g0).cuda(), 0.9, None, mask=0x5555, seed=5)
    copy = tuple(t.clone() for t in st)
    m_a, out_a = fs4.momentum_nvfp4(torch.from_numpy(g1).cuda(), 0.9, st, prev_mask=0x5555,
                                    mask=0x00FF, seed=6)
    m_b, out_b = fs4.momentum_nvfp4(torch.from_numpy(g1).cuda(), 0.9, copy, prev_mask=0x5555,
                                    mask=0x00FF, seed=6, out_state=copy)
    torch.cuda.synchronize()
    assert torch.equal(m_a, m_b)
    for a, b in zip(out_a, out_b):
        assert torch.equal(a, b)


def test_strided_unaligned_gradient_and_beta_zero(fs4):
    g = _grad(96, 320, "gauss", 7)
    big = torch.zeros((96, 333), dtype=torch.float32, device="cuda")
    big[:, 3:3 + 320] = torch.from_numpy(g).cuda()
    view = big[:, 3:3 + 320]
    m, st = fs4.momentum_nvfp4(view, 0.0, None, mask=0x0F0F, seed=99)
    torch.cuda.synchronize()
    want_m, want_state = M.update(g, 0.0, None, 0, 0x0F0F, 99)
    _assert_same(m.cpu().numpy(), _gpu_state(st), want_m, want_state)
    assert np.array_equal(m.cpu().numpy(), g)


def test_nonfinite_gradient_reports_status(fs4):
    g = _grad(32, 64, "gauss", 8)
    g[3, 5] = np.nan
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    fs4.momentum_nvfp4(torch.from_numpy(g).cuda(), 0.9, None, workspace=ws)
    assert fs4.device_status(ws) == -7


def test_momentum_feeds_the_newton_schulz_step(fs4):
    # the FP32 m_t is an ordinary input of the Newton-Schulz step
    g = _grad(256, 512, "gauss", 9)
    m, _ = fs4.momentum_nvfp4(torch.from_numpy(g).cuda(), 0.9, None, mask=0x3C3C, seed=1)
    out = fs4.root_ns(m, 2, 15 / 8, -10 / 8, 3 / 8)
    torch.cuda.synchronize()
    assert torch.isfinite(out).all() and out.abs().max() > 0

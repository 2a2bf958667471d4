"""GPU parity of the standalone NVFP4 quantiser and dequantiser (bit-exact).

Inputs are seeded; expected codes, scales and tensor scales come from the
oracle (oracle/nvfp4.py) applied to the same FP32 input.
"""
import json
import os

import numpy as np
import pytest
import torch

from oracle import nvfp4 as Q
from tests.helpers import tiled_to_plain

pytestmark = pytest.mark.gpu


def _inputs():
    rng = np.random.default_rng(2026)
    cases = {
        "gauss_64x64": rng.standard_normal((64, 64)) * 0.02,
        "gauss_ragged_100x272": rng.standard_normal((100, 272)),
        "student_t_257x1024": rng.standard_t(3, (257, 1024)) * 0.02,
        "outliers_48x4096": rng.standard_normal((48, 4096)) * 0.02 * np.where(rng.random((48, 4096)) < 0.001, 50, 1),
        "one_block_1x16": rng.standard_normal((1, 16)),
        "wide_range_32x512": rng.standard_normal((32, 512)) * np.exp(rng.uniform(-14, 4, (32, 1))),
        "ties_16x64": rng.choice([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0], (16, 64)) * rng.choice([-1, 1], (16, 64)),
        "zeros_32x32": np.zeros((32, 32)),
        "tiny_negative_16x32": -np.abs(rng.standard_normal((16, 32))) * np.where(rng.random((16, 32)) < 0.5, 1e-3, 1.0),
        "large_2048x2048": rng.standard_normal((2048, 2048)),
        # exact -0.0 entries keep their sign code (0x8); +0.0 gives 0x0
        "signed_zeros_32x64": rng.choice([-0.0, 0.0, 1.0, -1.0, 5e-4, -5e-4], (32, 64)),
    }
    return {k: v.astype(np.float32) for k, v in cases.items()}


CASES = _inputs()


def _gpu_quant(F, x, axis, tiled, mode):
    xt = torch.from_numpy(x).cuda()
    codes, scales, sg = F.quantize(xt, axis=axis, tiled=tiled, sg_mode=mode)
    torch.cuda.synchronize()
    return codes.cpu().numpy(), scales.cpu().numpy(), sg.cpu().numpy()[0]


@pytest.mark.parametrize("name", sorted(CASES))
@pytest.mark.parametrize("axis", [0, 1])
@pytest.mark.parametrize("tiled", [False, True])
def test_quantize_bit_exact(fs4, name, axis, tiled):
    x = CASES[name]
    if axis == 1 and x.shape[0] % 16:
        pytest.skip("column blocks need rows % 16 == 0")
    for mode in ("pow2", "amax"):
        want_c, want_s, want_g = (Q.quantize_rows(x, mode=mode) if axis == 0
                                  else Q.quantize_cols(x, mode=mode))
        c, s, g = _gpu_quant(fs4, x, axis, tiled, mode)
        R, C = (x.shape if axis == 0 else x.shape[::-1])
        if tiled:
            c, s, cpad, spad = tiled_to_plain(c, s, R, C)
            assert not cpad[R:].any() and not cpad[:, C // 2:].any()
            assert not spad[R:].any() and not spad[:, C // 16:].any()
        assert np.float32(g) == want_g, (name, mode)
        assert np.array_equal(s, want_s), (name, mode, np.argwhere(s != want_s)[:5])
        assert np.array_equal(c, want_c), (name, mode, np.argwhere(c != want_c)[:5])


def test_hand_worked_blocks_on_gpu(fs4, golden_dir):
    with open(os.path.join(golden_dir, "hand_blocks.json")) as f:
        cases = json.load(f)["cases"]
    for case in cases:
        x = np.array(case["x"], np.float32)[None, :]
        c, s, g = _gpu_quant(fs4, x, 0, False, "pow2")
        assert float(g) == case["s_g"]
        assert [f"{b:02x}" for b in s[0]] == case["scales_hex"]
        assert [f"{b:02x}" for b in c[0]] == case["codes_hex"]


@pytest.mark.parametrize("name", ["gauss_ragged_100x272", "wide_range_32x512", "student_t_257x1024"])
@pytest.mark.parametrize("tiled", [False, True])
def test_dequantize_bit_exact(fs4, name, tiled):
    x = CASES[name]
    xt = torch.from_numpy(x).cuda()
    for mode in ("pow2", "amax"):
        codes, scales, sg = fs4.quantize(xt, tiled=tiled, sg_mode=mode)
        y = fs4.dequantize(codes, scales, sg, x.shape[0], x.shape[1], tiled=tiled).cpu().numpy()
        wc, ws, wg = Q.quantize_rows(x, mode=mode)
        want = Q.dequantize_rows(wc, ws, wg, dtype=np.float32)
        assert np.array_equal(y.view(np.uint32), want.view(np.uint32))


def test_nonfinite_input_sets_device_status(fs4):
    x = torch.zeros((16, 32), device="cuda")
    x[3, 7] = float("nan")
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    fs4.quantize(x, workspace=ws)
    assert fs4.device_status(ws) == -7
    fs4.quantize(torch.ones((16, 32), device="cuda"), workspace=ws)
    assert fs4.device_status(ws) == 0


def test_quantize_barrier_timeout_reports_status_and_context_survives(fs4):
    """The quantise call's grid barrier (between its amax pass and its quantise pass)
    is a bounded wait: with FS4_TEST_STALL it waits for one CTA more than the launch
    has, gives up after about 2 s and records FS4_ERR_TIMEOUT, with no fault; the next
    call on the same stream and workspace is bit-exact."""
    import time
    rng = np.random.default_rng(3)
    x = (rng.standard_normal((512, 1024)) * 0.02).astype(np.float32)
    xd = torch.from_numpy(x).cuda()
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    t0 = time.time()
    fs4.quantize(xd, workspace=ws, flags=fs4.FS4_TEST_STALL)
    torch.cuda.synchronize()
    assert time.time() - t0 < 30.0
    assert fs4.device_status(ws) == -8          # FS4_ERR_TIMEOUT
    codes, scales, sg = fs4.quantize(xd, workspace=ws)
    assert fs4.device_status(ws) == 0
    wc, wsc, wg = Q.quantize_rows(x)
    assert np.array_equal(codes.cpu().numpy(), wc) and np.array_equal(scales.cpu().numpy(), wsc)
    assert float(sg.item()) == float(wg)


def _threshold_sweep():
    """Blocks whose scale decodes to each E4M3 mantissa 1 + m/8 and whose other
    15 elements sweep 2^14 consecutive FP32 values on both sides of every E2M1
    decision threshold (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5) times the decoded
    scale.  The first element of each block is 6 * 2^-8 * (1 + m/8) * 256 /
    256, which makes amax_b / (6 s_g) land exactly on that E4M3 value."""
    rows = []
    s_g = 2.0 ** -8
    for m in range(8):
        dec = (1 + m / 8) * 128                      # E4M3 value in [128, 256)
        den = np.float32(dec * s_g)
        head = np.float32(6.0 * dec * s_g)           # block amax -> scale exactly dec
        for t in (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0):
            centre = np.float32(t * den)
            bits = centre.view(np.uint32).astype(np.int64)
            vals = (np.arange(bits - 8190, bits + 8190)).astype(np.uint32).view(np.float32)
            vals = vals.reshape(-1, 15)
            blk = np.concatenate([np.full((vals.shape[0], 1), head, np.float32), vals], axis=1)
            blk[1::2, 1:] *= -1
            rows.append(blk)
    x = np.concatenate(rows)
    x = x[: x.shape[0] // 4 * 4].reshape(-1, 64)
    # a whole-tensor amax equal to the block heads keeps s_g = 2^-8 (6 * 255 * 2^-8 < 2688 * 2^-8)
    return x.astype(np.float32)


def test_quantize_decisions_next_to_every_threshold(fs4):
    x = _threshold_sweep()
    want_c, want_s, want_g = Q.quantize_rows(x)
    assert want_g == 2.0 ** -8
    for tiled in (False, True):
        c, s, g = _gpu_quant(fs4, x, 0, tiled, "pow2")
        if tiled:
            c, s, _, _ = tiled_to_plain(c, s, x.shape[0], x.shape[1])
        assert g == want_g
        assert np.array_equal(s, want_s)
        assert np.array_equal(c, want_c), np.argwhere(c != want_c)[:5]


@pytest.mark.parametrize("shape,axis", [((100, 272), 0), ((96, 200), 1), ((130, 1040), 0), ((272, 130), 1)])
@pytest.mark.parametrize("tiled", [False, True])
def test_quantize_strided_unaligned_input(fs4, shape, axis, tiled):
    """x as a column-offset view of a wider matrix: its base is 4 bytes past a
    16-byte boundary and its row stride is not a multiple of 4 floats, so the
    quantiser takes its scalar staging path on every tile."""
    R0, C0 = shape
    rng = np.random.default_rng(17 + R0 + C0)
    big = (rng.standard_normal((R0, C0 + 7)) * 0.05).astype(np.float32)
    xt = torch.from_numpy(big).cuda()[:, 1:C0 + 1]
    assert xt.stride(0) % 4 != 0 and (xt.data_ptr() % 16) != 0
    x = np.ascontiguousarray(big[:, 1:C0 + 1])
    want_c, want_s, want_g = Q.quantize_rows(x) if axis == 0 else Q.quantize_cols(x)
    c, s, g = fs4.quantize(xt, axis=axis, tiled=tiled)
    torch.cuda.synchronize()
    c, s, g = c.cpu().numpy(), s.cpu().numpy(), s_g_value(g)
    R, C = (R0, C0) if axis == 0 else (C0, R0)
    if tiled:
        c, s, _, _ = tiled_to_plain(c, s, R, C)
    assert np.float32(g) == want_g
    assert np.array_equal(s, want_s)
    assert np.array_equal(c, want_c)


def s_g_value(g):
    return g.cpu().numpy()[0]


@pytest.mark.parametrize("tiled", [False, True])
def test_dequantize_into_strided_unaligned_view(fs4, tiled):
    """Dequantise into a column-offset view (scalar store path): every element
    matches the oracle bit for bit and the columns around the view keep their
    sentinel."""
    x = CASES["gauss_ragged_100x272"]
    R, C = x.shape
    codes, scales, sg = fs4.quantize(torch.from_numpy(x).cuda(), tiled=tiled)
    big = torch.full((R, C + 5), 7.0, dtype=torch.float32, device="cuda")
    view = big[:, 1:C + 1]
    fs4.dequantize(codes, scales, sg, R, C, tiled=tiled, out=view)
    got = big.cpu().numpy()
    wc, ws, wg = Q.quantize_rows(x)
    want = Q.dequantize_rows(wc, ws, wg, dtype=np.float32)
    assert np.array_equal(got[:, 1:C + 1].view(np.uint32), want.view(np.uint32))
    assert (got[:, 0] == 7.0).all() and (got[:, C + 1:] == 7.0).all()


@pytest.mark.parametrize("shape", [(4096, 4096), (1000, 2064)])
def test_dequantize_large_grid_stride(fs4, shape):
    """Shapes with more 4-element groups than one persistent wave holds, so the
    grid-stride loop wraps rows several times (including a ragged last row)."""
    rng = np.random.default_rng(shape[0])
    x = rng.standard_normal(shape).astype(np.float32)
    codes, scales, sg = fs4.quantize(torch.from_numpy(x).cuda())
    y = fs4.dequantize(codes, scales, sg, *shape).cpu().numpy()
    wc, ws, wg = Q.quantize_rows(x)
    want = Q.dequantize_rows(wc, ws, wg, dtype=np.float32)
    assert np.array_equal(y.view(np.uint32), want.view(np.uint32))


# ---------------------------------------------------------------- batched quantise

def _batch_inputs():
    """Every case of CASES whose shape suits the axis, in one batch."""
    return {name: x for name, x in CASES.items()}


@pytest.mark.parametrize("axis", [0, 1])
@pytest.mark.parametrize("tiled", [False, True])
@pytest.mark.parametrize("sg_mode", ["pow2", "amax"])
def test_quantize_batched_matches_single_calls_and_oracle(fs4, axis, tiled, sg_mode):
    """fs4_nvfp4_quantize_batched over a batch of mixed shapes (every case above whose
    blocked dimension is a multiple of 16), each matrix byte for byte equal to its
    single-matrix fs4_nvfp4_quantize result and to the oracle's quantisation with its own
    tensor scale."""
    names = [n for n, x in _batch_inputs().items() if (x.shape[1] if axis == 0 else x.shape[0]) % 16 == 0]
    xs = [torch.from_numpy(CASES[n]).cuda() for n in names]
    outs = fs4.quantize_batched(xs, axis=axis, tiled=tiled, sg_mode=sg_mode)
    torch.cuda.synchronize()
    for n, x, (c, s, g) in zip(names, xs, outs):
        c1, s1, g1 = fs4.quantize(x, axis=axis, tiled=tiled, sg_mode=sg_mode)
        assert torch.equal(c, c1) and torch.equal(s, s1) and torch.equal(g, g1), n
        if not tiled:
            xn = CASES[n]
            wc, ws_, wg = (Q.quantize_rows if axis == 0 else Q.quantize_cols)(xn, mode=sg_mode)
            assert np.float32(g.item()) == wg, n
            assert np.array_equal(c.cpu().numpy(), wc) and np.array_equal(s.cpu().numpy(), ws_), n


def test_quantize_batched_strided_and_unaligned_views(fs4):
    rng = np.random.default_rng(41)
    big = torch.from_numpy((rng.standard_normal((300, 1200)) * 0.02).astype(np.float32)).cuda()
    xs = [big[:100, 1:273], big[10:150, 4:516], big[:, 16:16 + 1024]]   # odd offsets and strides
    outs = fs4.quantize_batched(xs, axis=0)
    for x, (c, s, g) in zip(xs, outs):
        wc, ws_, wg = Q.quantize_rows(x.cpu().numpy())
        assert np.float32(g.item()) == wg
        assert np.array_equal(c.cpu().numpy(), wc) and np.array_equal(s.cpu().numpy(), ws_)


def test_quantize_batched_full_size_3b_block(fs4):
    """One 3B-class block (the bench's --op quantize workload unit): seven 3072 x 3072,
    8192 x 3072 and 3072 x 8192 matrices in one launch, every byte against the single
    calls, and two matrices against the C++ oracle."""
    from nvfp4_precision_optimizer_b200.workloads import BASE_SEED, WORKLOADS, matrices
    from oracle import cpp_oracle as C
    Gs = matrices(WORKLOADS["3b_1block_gauss"], device="cuda", seed=BASE_SEED)
    outs = fs4.quantize_batched(Gs, axis=0)
    torch.cuda.synchronize()
    for i, (G, (c, s, g)) in enumerate(zip(Gs, outs)):
        c1, s1, g1 = fs4.quantize(G, axis=0)
        assert torch.equal(c, c1) and torch.equal(s, s1) and torch.equal(g, g1)
        if i in (0, 4):
            wc, ws_, wg = C.quantize_rows(G.cpu().numpy())
            assert np.float32(g.item()) == wg
            assert np.array_equal(c.cpu().numpy(), wc) and np.array_equal(s.cpu().numpy(), ws_)


def test_quantize_batched_nonfinite_and_timeout_status(fs4):
    x = torch.zeros((32, 64), device="cuda")
    y = torch.ones((16, 32), device="cuda")
    x[3, 5] = float("nan")
    ws = torch.zeros(fs4._lib.lib().fs4_nvfp4_quantize_batched_workspace_size(2), dtype=torch.uint8,
                     device="cuda")
    fs4.quantize_batched([x, y], workspace=ws)
    assert fs4.device_status(ws) == -7
    import time
    t0 = time.time()
    fs4.quantize_batched([y, y], workspace=ws, flags=fs4.FS4_TEST_STALL)
    torch.cuda.synchronize()
    assert time.time() - t0 < 30.0
    assert fs4.device_status(ws) == -8
    (c, s, g), = fs4.quantize_batched([y])
    wc, ws_, wg = Q.quantize_rows(y.cpu().numpy())
    assert np.array_equal(c.cpu().numpy(), wc) and np.float32(g.item()) == wg

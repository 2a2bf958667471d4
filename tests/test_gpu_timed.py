"""GPU: the phase-timed entry points (fs4_root_ns_batched_timed, fs4_root_ns_batched_nvfp4_timed,
fs4_root_ns_bf16_batched_timed) run the same step as the untimed calls ("Full-Stack FP4",
Section 3.4) and only add CUDA events between its phases: their results equal the untimed
calls' bit for bit, the 3 + 3K events complete in order, and a call given fewer events than
that is rejected before it launches anything.
"""

import numpy as np
import pytest
import torch

from tests.test_gpu_ns import QUINTIC, momentum

pytestmark = pytest.mark.gpu

SHAPES = [(256, 256), (128, 384), (384, 128)]
K = 3
INVALID_ARG = -1


def _inputs():
    return [torch.from_numpy(momentum(*s, kind=("gauss", "student")[i % 2], seed=70 + i)).cuda()
            for i, s in enumerate(SHAPES)]


def _events(fs4, n):
    # torch creates an event's CUDA handle at its first record
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
    for e in evs:
        e.record()
    torch.cuda.synchronize()
    assert all(e.cuda_event for e in evs)
    return evs, (fs4._lib.c_vp * n)(*[e.cuda_event for e in evs])


def _check_events(evs):
    torch.cuda.synchronize()
    gaps = [evs[i].elapsed_time(evs[i + 1]) for i in range(len(evs) - 1)]
    assert all(g >= 0.0 for g in gaps)
    assert sum(gaps) > 0.0


def test_timed_fp32_step_equals_untimed(fs4):
    Gs = _inputs()
    coeffs = [QUINTIC] * len(Gs)
    want = fs4.root_ns_batched(Gs, K=K, coeffs=coeffs)
    outs = [torch.empty_like(G) for G in Gs]
    arr = fs4._descs(Gs, outs, coeffs)
    lib = fs4._lib.lib()
    need = int(lib.fs4_root_ns_batched_workspace_size(len(Gs), arr))
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    evs, ev_arr = _events(fs4, 3 + 3 * K)
    # too few events: refused before any launch (the outputs stay untouched)
    for o in outs:
        o.fill_(7.0)
    assert lib.fs4_root_ns_batched_timed(len(Gs), arr, K, 3.0, 0, None, ws.data_ptr(), need, stream,
                                         ev_arr, 2 + 3 * K) == INVALID_ARG
    torch.cuda.synchronize()
    assert all(bool((o == 7.0).all()) for o in outs)
    fs4.check(lib.fs4_root_ns_batched_timed(len(Gs), arr, K, 3.0, 0, None, ws.data_ptr(), need, stream,
                                            ev_arr, len(evs)), "fs4_root_ns_batched_timed")
    _check_events(evs)
    for a, b in zip(outs, want):
        assert torch.equal(a, b)


def test_timed_nvfp4_state_step_equals_untimed(fs4):
    states = []
    for i, G in enumerate(_inputs()):
        _, st = fs4.momentum_nvfp4(G, 0.9, None, mask=(0x3A5C * (i + 1)) & 0xFFFF, seed=80 + i)
        states.append(st + ((0x3A5C * (i + 1)) & 0xFFFF,))
    coeffs = [QUINTIC] * len(states)
    want = fs4.root_ns_batched_nvfp4(states, K=K, coeffs=coeffs)
    outs = [torch.empty_like(w) for w in want]
    arr = (fs4.NsDesc * len(states))()
    sts = (fs4._lib.Nvfp4State * len(states))()
    for i, (st, o) in enumerate(zip(states, outs)):
        m, n = o.shape
        arr[i] = fs4.NsDesc(None, o.data_ptr(), m, n, n, n, *coeffs[i])
        sts[i] = fs4._lib.Nvfp4State(st[0].data_ptr(), st[1].data_ptr(), st[2].data_ptr(), int(st[3]))
    lib = fs4._lib.lib()
    need = int(lib.fs4_root_ns_batched_workspace_size(len(states), arr))
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    evs, ev_arr = _events(fs4, 3 + 3 * K)
    assert lib.fs4_root_ns_batched_nvfp4_timed(len(states), arr, sts, K, 3.0, 0, None, ws.data_ptr(),
                                               need, stream, None, len(evs)) == INVALID_ARG
    fs4.check(lib.fs4_root_ns_batched_nvfp4_timed(len(states), arr, sts, K, 3.0, 0, None, ws.data_ptr(),
                                                  need, stream, ev_arr, len(evs)),
              "fs4_root_ns_batched_nvfp4_timed")
    _check_events(evs)
    for a, b in zip(outs, want):
        assert torch.equal(a, b)


def test_timed_bf16_step_equals_untimed(fs4):
    Gs = _inputs()
    coeffs = [QUINTIC] * len(Gs)
    want = fs4.root_ns_bf16_batched(Gs, K=K, coeffs=coeffs)
    outs = [torch.empty_like(G) for G in Gs]
    arr = fs4._descs(Gs, outs, coeffs)
    lib = fs4._lib.lib()
    need = int(lib.fs4_root_ns_bf16_batched_workspace_size(len(Gs), arr))
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    evs, ev_arr = _events(fs4, 3 + 3 * K)
    fs4.check(lib.fs4_root_ns_bf16_batched_timed(len(Gs), arr, K, 3.0, 0, ws.data_ptr(), need, stream,
                                                 ev_arr, len(evs)), "fs4_root_ns_bf16_batched_timed")
    _check_events(evs)
    for a, b in zip(outs, want):
        assert torch.equal(a, b)
    # the per-phase events bracket the work: the products take longer than the reset
    times = np.array([evs[i].elapsed_time(evs[i + 1]) for i in range(len(evs) - 1)])
    assert times[2:].sum() > times[0]

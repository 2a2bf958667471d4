"""A Newton-Schulz call captured in a CUDA graph replays like the same call issued
on a stream.

The library allocates nothing, never synchronises inside a call and reads every
input through the pointers it is given, so a launch-bound caller (small
matrices, where the host's launch rate sets the step time) can capture one
grouped call and replay it each step.  The replay reads whatever the captured
buffers hold at replay time; these tests check that, and that the replayed
result is the method's (oracle parity), on a batch of small matrices with tall,
wide and square members.
"""
import numpy as np
import pytest
import torch

import nvfp4_precision_optimizer_b200 as F
from oracle import root_ns as R
from tests.helpers import rel_frob

pytestmark = pytest.mark.gpu

SHAPES = [(256, 256), (256, 512), (768, 256)]
K = 3   # Muon coefficients: K <= 3 stays inside the 2e-2 parity regime


def draw(rng):
    return [(rng.standard_normal(s) * 0.02).astype(np.float32) for s in SHAPES]


def test_graph_replay_matches_stream_call_and_oracle():
    rng = np.random.default_rng(20260705)
    host = draw(rng)
    Gs = [torch.from_numpy(h).cuda() for h in host]
    outs = [torch.empty_like(G) for G in Gs]
    ws = torch.empty(F.ns_batched_workspace_size(SHAPES), dtype=torch.uint8, device="cuda")
    F.root_ns_batched(Gs, K=K, outs=outs, workspace=ws)   # first call outside any capture
    torch.cuda.synchronize()
    assert F.device_status(ws) == 0

    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        F.root_ns_batched(Gs, K=K, outs=outs, workspace=ws)

    for step in range(2):
        if step == 1:   # new contents in the captured buffers: the replay must read them
            host = draw(rng)
            for G, h in zip(Gs, host):
                G.copy_(torch.from_numpy(h))
        for o in outs:
            o.fill_(float("nan"))
        graph.replay()
        torch.cuda.synchronize()
        assert F.device_status(ws) == 0
        stream_outs = F.root_ns_batched(Gs, K=K)
        for o, s, h in zip(outs, stream_outs, host):
            got = o.cpu().numpy()
            assert np.all(np.isfinite(got))
            # the same kernels on the same data; float atomics in the row/column sums
            # may only move a bound by an ulp, which leaves the power-of-two scales alone
            assert rel_frob(got, s.cpu().numpy()) <= 1e-6
            assert rel_frob(got, R.root_ns(h, K=K, clip_k=3.0)) <= 2e-2


def test_graph_replay_is_repeatable():
    """Several replays of one captured call on unchanged inputs agree with each other
    (each call clears the state it accumulates into before using it)."""
    rng = np.random.default_rng(7)
    Gs = [torch.from_numpy(h).cuda() for h in draw(rng)]
    outs = [torch.empty_like(G) for G in Gs]
    ws = torch.empty(F.ns_batched_workspace_size(SHAPES), dtype=torch.uint8, device="cuda")
    F.root_ns_batched(Gs, K=K, outs=outs, workspace=ws)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        F.root_ns_batched(Gs, K=K, outs=outs, workspace=ws)
    graph.replay()
    torch.cuda.synchronize()
    first = [o.cpu().numpy().copy() for o in outs]
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    assert F.device_status(ws) == 0
    for o, f in zip(outs, first):
        assert rel_frob(o.cpu().numpy(), f) <= 1e-6

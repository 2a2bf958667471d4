"""Sharding one model's Newton-Schulz steps across ranks (nvfp4_precision_optimizer_b200.shard),
on CPU: the LPT plan against hand-worked and brute-force cases, the buffer layout, and
the all-gather path on two gloo ranks with a CPU stand-in for the step (the CUDA path is
not run here; only the host logic and the collective are).
"""
import datetime
import itertools
import json
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from nvfp4_precision_optimizer_b200 import shard
from nvfp4_precision_optimizer_b200.workloads import WORKLOADS


def test_ns_flops_by_hand():
    # m = 2, n = 3 (either orientation), K = 1: 2*3*3 + 2*3*2 + 2*4*3 = 18 + 12 + 24
    assert shard.ns_flops((2, 3), 1) == 54
    assert shard.ns_flops((3, 2), 1) == 54
    assert shard.ns_flops((3072, 8192), 5) == 5 * (3072 * 3073 * 8192 + 3072 * 3073 * 3072
                                                    + 2 * 3072 * 3072 * 8192)


def test_lpt_hand_worked():
    # decreasing costs 7, 5, 4, 3, 3, 2 over 2 ranks:
    # 7 -> r0 (7, 0); 5 -> r1 (7, 5); 4 -> r1 (7, 9); 3 -> r0 (10, 9); 3 -> r1 (10, 12); 2 -> r0 (12, 12)
    assert shard.lpt_owners([7, 5, 4, 3, 3, 2], 2) == [0, 1, 1, 0, 1, 0]
    # ties: equal costs go in index order to the least-loaded, lowest rank
    assert shard.lpt_owners([1, 1, 1, 1], 3) == [0, 1, 2, 0]
    assert shard.lpt_owners([], 4) == []
    with pytest.raises(ValueError):
        shard.lpt_owners([1], 0)


@pytest.mark.parametrize("seed", range(20))
def test_lpt_within_grahams_bound_of_the_brute_force_optimum(seed):
    """LPT's makespan is at most (4/3 - 1/(3w)) of the optimum (Graham, 1969)."""
    rng = np.random.default_rng(seed)
    world = int(rng.integers(2, 4))
    costs = [int(v) for v in rng.integers(1, 50, int(rng.integers(1, 8)))]
    owners = shard.lpt_owners(costs, world)
    load = [sum(c for c, o in zip(costs, owners) if o == r) for r in range(world)]
    best = min(max(sum(c for c, o in zip(costs, a) if o == r) for r in range(world))
               for a in itertools.product(range(world), repeat=len(costs)))
    assert max(load) <= (4 / 3 - 1 / (3 * world)) * best + 1e-9
    assert sorted(set(owners)) == list(range(min(world, len(costs))))   # no rank idles early


@pytest.mark.parametrize("world", [1, 2, 3, 8])
def test_plan_layout(world):
    w = WORKLOADS["3b_4blocks_gauss"]
    p = shard.plan(w.shapes, w.K, world)
    assert len(p.owners) == len(w.shapes)
    assert sorted(sum((p.local(r) for r in range(world)), [])) == list(range(len(w.shapes)))
    assert sum(p.loads) == sum(shard.ns_flops(s, w.K) for s in w.shapes)
    for r in range(world):
        spans = sorted((p.offsets[i], p.offsets[i] + p.shapes[i][0] * p.shapes[i][1]) for i in p.local(r))
        for (a0, a1), (b0, _) in zip(spans, spans[1:]):
            assert a1 <= b0                                      # disjoint
        assert all(a % shard.ALIGN_ELEMS == 0 for a, _ in spans)   # 256-byte aligned
        assert all(b <= p.chunk for _, b in spans)                 # inside the send buffer


def test_bench_workload_balance():
    """The 196-matrix 3B workload splits evenly: every rank's load is within 5% of the mean."""
    w = WORKLOADS["3b_28blocks_student"]
    for world in (2, 4, 8):
        assert shard.plan(w.shapes, w.K, world).imbalance < 1.05


def _double(Gs, outs, scale=2.0):
    for G, o in zip(Gs, outs):
        o.copy_(scale * G)


def test_call_options_reach_the_step():
    shapes = [(32, 48), (16, 16)]
    Gs = [torch.randn(s) for s in shapes]
    S = shard.ShardedRootNS(shapes, K=3, rank=0, world=1, device="cpu", compute=_double)
    outs = S(Gs, scale=3.0)
    assert all(torch.equal(o, 3.0 * G) for o, G in zip(outs, Gs))


def test_one_rank_needs_no_collective():
    shapes = [(32, 48), (16, 16), (64, 32)]
    Gs = [torch.randn(s) for s in shapes]
    S = shard.ShardedRootNS(shapes, K=3, rank=0, world=1, device="cpu", compute=_double)
    outs = S(Gs)
    assert all(torch.equal(o, 2.0 * G) for o, G in zip(outs, Gs))
    assert all(o.data_ptr() >= S.send.data_ptr() for o in outs)
    with pytest.raises(ValueError):
        S(Gs[:2])
    with pytest.raises(ValueError):
        S([Gs[0], None, Gs[2]])


WORLD = 2


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, outdir: str) -> None:
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        shapes = [(48, 32), (16, 64), (96, 96), (32, 32), (16, 16), (64, 48), (128, 16)]
        gen = torch.Generator().manual_seed(5)
        Gs = [torch.randn(s, generator=gen) for s in shapes]          # every rank: the same model
        S = shard.ShardedRootNS(shapes, K=5, rank=rank, world=world, device="cpu", compute=_double)
        mine = set(S.local)
        seen = [G if i in mine else None for i, G in enumerate(Gs)]   # others' momenta not needed
        res = {"local": S.local, "ok": [], "ok2": []}
        outs = S(seen)
        res["ok"] = [bool(torch.equal(o, 2.0 * G)) for o, G in zip(outs, Gs)]
        # a second call overwrites the same views
        Gs2 = [G + 1.0 for G in Gs]
        outs2 = S([G if i in mine else None for i, G in enumerate(Gs2)])
        res["ok2"] = [bool(torch.equal(o, 2.0 * G)) for o, G in zip(outs2, Gs2)]
        res["same_views"] = all(a.data_ptr() == b.data_ptr() for a, b in zip(outs, outs2))
        # a model with fewer matrices than ranks: one rank owns nothing
        T = shard.ShardedRootNS([(32, 16)], K=5, rank=rank, world=world, device="cpu", compute=_double)
        g = torch.arange(512, dtype=torch.float32).view(32, 16)
        res["single"] = bool(torch.equal(T([g if rank == 0 else None])[0], 2.0 * g))
        res["single_local"] = T.local
        with open(os.path.join(outdir, f"rank{rank}.json"), "w") as f:
            json.dump(res, f)
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.fixture(scope="module")
def rank_results(tmp_path_factory):
    outdir = tmp_path_factory.mktemp("shard")
    mp.spawn(_rank_main, args=(WORLD, _free_port(), str(outdir)), nprocs=WORLD, join=True)
    out = []
    for r in range(WORLD):
        with open(outdir / f"rank{r}.json") as f:
            out.append(json.load(f))
    return out


def test_every_rank_gets_every_update(rank_results):
    for res in rank_results:
        assert all(res["ok"]) and all(res["ok2"]) and res["same_views"]
        assert res["single"]


def test_the_ranks_split_the_work(rank_results):
    locs = [set(r["local"]) for r in rank_results]
    assert locs[0] and locs[1] and not (locs[0] & locs[1])
    assert locs[0] | locs[1] == set(range(7))
    assert rank_results[0]["single_local"] == [0] and rank_results[1]["single_local"] == []

"""bench.py --shard lpt on two gloo ranks (CPU): the measurement and reporting logic of the
sharded step, with CPU stand-ins for CUDA events, the device and the step itself (each
update is 2 G).  What this checks is the host side: every rank times the same sequence of
phases, the maxima over ranks are taken in the same order everywhere, every rank ends with
every update, and rank 0 prints one strong-scaling line whose value is the model's matrices
over the slowest rank's step time.
"""
import datetime
import json
import os
import socket
import time
import types

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

WORLD = 2
SHAPES = [(64, 128), (128, 64), (32, 32), (96, 96), (48, 16)]


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class _Event:
    def __init__(self, enable_timing=False):
        self.t = None

    def record(self, stream=None):
        self.t = time.perf_counter()

    def elapsed_time(self, other):
        return 1000.0 * (other.t - self.t)


class _Clocks:
    def __init__(self, gpu):
        pass

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        pass

    def summary(self):
        return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}


def _rank_main(rank, world, port, outdir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import contextlib
    import io

    import bench
    from nvfp4_precision_optimizer_b200 import shard
    from nvfp4_precision_optimizer_b200 import workloads as W
    # CPU stand-ins (this process only)
    torch.cuda.Event = _Event
    torch.cuda.current_stream = lambda: None
    torch.cuda.synchronize = lambda: None
    torch.cuda.get_device_properties = lambda i: types.SimpleNamespace(L2_cache_size=1 << 10)
    bench.ClockSampler = _Clocks
    made = []
    real = shard.ShardedRootNS

    def on_cpu(shapes, **kw):
        kw["device"] = "cpu"
        kw.pop("clip_k", None)
        S = real(shapes, compute=lambda Gs, outs: [o.copy_(2.0 * g) for g, o in zip(Gs, outs)], **kw)
        made.append(S)
        return S
    shard.ShardedRootNS = on_cpu
    gen = W.generate
    W.generate = lambda s, d, seed, device: gen(s, d, seed, "cpu")
    try:
        w = W.Workload("five_small_gauss", SHAPES, "gauss")
        args = types.SimpleNamespace(quant="plain", clip="rms", source="fp32", graph=False,
                                     warmup=3, steps=2)
        out = io.StringIO()
        with contextlib.redirect_stdout(out):
            bench.run_sharded(args, w, rank, world, 0, dist.barrier,
                              lambda v: bench.max_over_ranks(v, world, "cpu"))
        S = made[0]
        want = [2.0 * gen(s, w.dist, W.BASE_SEED + i, "cpu") for i, s in enumerate(SHAPES)]
        res = {"stdout": out.getvalue(), "local": S.local,
               "all_updates": all(bool(torch.equal(o, g)) for o, g in zip(S.outs, want))}
        with open(os.path.join(outdir, f"rank{rank}.json"), "w") as f:
            json.dump(res, f)
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.fixture(scope="module")
def ranks(tmp_path_factory):
    outdir = tmp_path_factory.mktemp("bench_shard")
    mp.spawn(_rank_main, args=(WORLD, _free_port(), str(outdir)), nprocs=WORLD, join=True)
    res = []
    for r in range(WORLD):
        with open(outdir / f"rank{r}.json") as f:
            res.append(json.load(f))
    return res


def test_every_rank_ends_with_every_update(ranks):
    assert all(r["all_updates"] for r in ranks)
    assert set(ranks[0]["local"]).isdisjoint(ranks[1]["local"])
    assert sorted(ranks[0]["local"] + ranks[1]["local"]) == list(range(len(SHAPES)))


def test_rank0_prints_one_strong_scaling_line(ranks):
    assert ranks[1]["stdout"] == ""
    lines = [ln for ln in ranks[0]["stdout"].splitlines() if ln.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["n_gpus"] == WORLD and line["scaling"] == "strong" and line["steps"] == 2
    assert line["value"] == pytest.approx(len(SHAPES) / (line["ms_per_step"] * 1e-3), rel=1e-12)
    split = line["split_ms"]
    assert split["share_step_max_over_ranks"] >= 0 and split["all_gather_max_over_ranks"] >= 0
    assert line["config"]["parallelism"].startswith("lpt x2")
    assert line["config"]["load_imbalance"] >= 1.0
    assert line["all_gather_recv_bytes_per_rank"] > 0
    assert line["gpu_launches"] == 2 * (2 + 6 * 5)

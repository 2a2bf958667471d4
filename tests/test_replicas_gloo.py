"""Multi-rank host logic of bench.py on CPU: two gloo ranks (no GPU).

Across GPUs the Newton-Schulz step runs as replicas: every rank runs the whole workload
on its own seeded matrices (the matrices are independent, so no collective touches the
data path), the step time is the maximum over ranks, and the reported throughput is
world_size x the units of one rank over that time ("scaling": "weak").
"""
import datetime
import json
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

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
        import bench
        from nvfp4_precision_optimizer_b200.workloads import BASE_SEED, WORKLOADS, matrices
        w = WORKLOADS["3b_1block_gauss"]
        Gs = matrices(WORKLOADS["single_256x256_gauss"], device="cpu",
                      seed=bench.rank_seed(BASE_SEED, rank))
        step_ms = 10.0 + 5.0 * rank            # this rank's (synthetic) step time
        slowest = bench.max_over_ranks(step_ms, world, "cpu")
        result = {
            "rank": rank,
            "slowest": slowest,
            "checksum": float(Gs[0].double().abs().sum()),
            "rate": bench.job_rate(world, len(w.shapes), slowest),
        }
        with open(os.path.join(outdir, f"rank{rank}.json"), "w") as f:
            json.dump(result, f)
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.fixture(scope="module")
def rank_results(tmp_path_factory):
    outdir = tmp_path_factory.mktemp("gloo")
    mp.spawn(_rank_main, args=(WORLD, _free_port(), str(outdir)), nprocs=WORLD, join=True)
    out = []
    for r in range(WORLD):
        with open(outdir / f"rank{r}.json") as f:
            out.append(json.load(f))
    return out


def test_every_rank_sees_the_slowest_step(rank_results):
    assert [r["slowest"] for r in rank_results] == [15.0, 15.0]


def test_ranks_run_distinct_matrices(rank_results):
    sums = [r["checksum"] for r in rank_results]
    assert sums[0] > 0 and sums[1] > 0 and sums[0] != sums[1]


def test_whole_job_rate_counts_every_rank(rank_results):
    # 7 matrices per rank and step, 2 ranks, slowest step 15 ms
    for r in rank_results:
        assert r["rate"] == pytest.approx(2 * 7 / 15e-3)


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.job_rate(1, 28, 12.5) == pytest.approx(28 / 12.5e-3)
    assert bench.rank_seed(100, 0) == 100 and bench.rank_seed(100, 3) == 3100

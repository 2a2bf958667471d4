"""CPU checks of bench.py's JSON contract on the arm that needs no GPU.

`bench.py --impl reference` times the oracle on the host cores and prints one JSON
line with the same metric, unit and workload description as the GPU arm.  Run on the
smallest workload, so that the sample takes seconds.
"""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def run_bench(*args):
    r = subprocess.run([sys.executable, "bench.py", *args], cwd=ROOT, capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    return json.loads(r.stdout.strip().splitlines()[-1])


@pytest.mark.parametrize("variant", [[], ["--quant", "rht46", "--clip", "p99"]])
def test_reference_arm_line(variant):
    import bench
    from nvfp4_precision_optimizer_b200.workloads import WORKLOADS

    line = run_bench("--impl", "reference", "--workload", "single_256x256_gauss",
                     "--steps", "1", "--warmup", "0", *variant)
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference"
    assert line["metric"] == bench.METRIC and line["unit"] == bench.UNIT
    assert line["higher_is_better"] is True and line["vs_baseline"] is None
    assert line["value"] > 0 and line["steps"] == 1
    quant = variant[1] if variant else "plain"
    clip = variant[3] if variant else "rms"
    # the workload keys are those the GPU arm prints for the same flags
    want = bench.ns_config(WORKLOADS["single_256x256_gauss"], quant, clip, 1)
    assert line["config"] == json.loads(json.dumps(want))
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"] and cb["sample"]
    e2e = line["e2e"]
    assert e2e["value"] == line["value"] and e2e["unit"] == line["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0
    # a step is one bounded oracle sample: ms_per_step is the time that sample took,
    # and the workload time it extrapolates to is stated beside it
    assert line["ms_per_workload_extrapolated"] == pytest.approx(
        1000.0 * line["config"]["matrices"] / line["value"])
    assert 0 < line["ms_per_step"] <= 1000.0 * line["steps"] * 600


def test_reference_arm_other_ranks_exit_quietly():
    """Under torchrun only rank 0 runs the reference arm; the others exit 0 without work."""
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload",
                        "single_256x256_gauss", "--steps", "1", "--warmup", "0"],
                       cwd=ROOT, capture_output=True, text=True, timeout=300, env=env)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_committed_traffic_is_close_to_the_algorithmic_bytes():
    """profiles/traffic.json holds each launch's measured DRAM bytes (ncu, scaled to the
    workload by its units).  A product or element-wise phase that re-read its operands from
    DRAM would show well above its algorithmic bytes; a capture of the wrong launch would
    show far off either way.  Writes still in L2 when a kernel ends make the measurement a
    little lower."""
    import bench
    from nvfp4_precision_optimizer_b200.workloads import WORKLOADS

    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        traffic = json.load(f)
    assert "3b_28blocks_student" in traffic
    for workload, kinds in traffic.items():
        for kind in ("reduce", "preamble", "gram_x", "gram_a", "update"):
            ent = kinds[kind]
            ratio = ent["bytes_per_launch"] / bench.bytes_per_launch(WORKLOADS[workload], kind)
            assert 0.6 <= ratio <= 1.25, (workload, kind, ratio)
            assert len(ent["source_sha"]) == 16 and ent["how"]


def test_roofline_helpers_by_hand():
    """bench.py's per-launch algorithmic work, for one m x n matrix (m <= n) in working
    orientation: the update is 2 m^2 n FLOPs over 0.5625 m^2 + 0.5625 mn + 8 mn + 1.125 mn
    bytes, the Gram products m (m + 1) n and m (m + 1) m FLOPs (symmetric halves).  With
    the measured peaks' ratio (about 992 FLOPs per byte for dense FP4) the update of a
    3072-row matrix is HBM-bound and that of an 8192-row matrix tensor-bound."""
    import bench
    from nvfp4_precision_optimizer_b200.workloads import Workload

    m, n = 3072, 8192
    w = Workload("hand", [(n, m)], "gauss")          # a tall matrix, transposed to m x n
    assert bench.flops_per_launch(w, "update") == 2 * m * m * n
    assert bench.flops_per_launch(w, "gram_x") == m * (m + 1) * n
    assert bench.flops_per_launch(w, "gram_a") == m * (m + 1) * m
    e = m * n
    assert bench.bytes_per_launch(w, "update") == pytest.approx(0.5625 * m * m + 0.5625 * e + 8 * e + 1.125 * e)
    assert bench.bytes_per_launch(w, "reduce") == 4 * e
    assert bench.bytes_per_launch(w, "preamble") == pytest.approx(9.125 * e)

    fp4, hbm = 4.0 * 1622.9e12, 6540.8e9             # peaks of the machine's B200s
    for side, bound in ((3072, "hbm"), (8192, "tensor")):
        wm = Workload("hand", [(side, side)], "gauss")
        t_flop = bench.flops_per_launch(wm, "update") / fp4
        t_byte = bench.bytes_per_launch(wm, "update") / hbm
        assert ("hbm" if t_byte > t_flop else "tensor") == bound, side


def test_committed_register_report_matches_the_sources():
    """profiles/ptxas_resources_all_kernels.md was made from the current CUDA sources (its
    digest), lists one row per kernel, and records no spill on the default or 8192-class
    GEMM variants."""
    import re

    from nvfp4_precision_optimizer_b200 import build
    text = open(os.path.join(ROOT, "profiles", "ptxas_resources_all_kernels.md")).read()
    m = re.search(r"(\d+) kernels; CUDA source digest ([0-9a-f]{16})", text)
    assert m, "the report carries its kernel count and source digest"
    assert m.group(2) == build.source_digest(), \
        "CUDA sources changed: rerun python -m nvfp4_precision_optimizer_b200.build --ptxas-table"
    rows = re.findall(r"^\| `([^`]+)` \| (\d+) \| (\d+) / (\d+) \|", text, re.M)
    assert len(rows) == int(m.group(1))
    for name, regs, st, ld in rows:
        if name.startswith("nvfp4_gemm_kernel") and name.split()[-1] in ("plain", "wide-K"):
            assert int(regs) == 168 and int(st) == 0 and int(ld) == 0, name

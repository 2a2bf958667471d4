"""GPU: one model's Newton-Schulz step through the sharded driver
(nvfp4_precision_optimizer_b200.shard.ShardedRootNS) on a single rank.  Every matrix is
local, no collective runs, and the updates (views of one flat buffer at 256-byte aligned
offsets) equal fs4_root_ns_batched's outputs on the same inputs bit for bit.
"""
import pytest
import torch

from nvfp4_precision_optimizer_b200 import shard
from tests.test_gpu_ns import QUINTIC, momentum

pytestmark = pytest.mark.gpu

SHAPES = [(256, 512), (384, 128), (128, 128), (512, 256)]


def test_one_rank_sharded_step_equals_the_batched_call(fs4):
    Gs = [torch.from_numpy(momentum(*s, kind=("gauss", "student")[i % 2], seed=90 + i)).cuda()
          for i, s in enumerate(SHAPES)]
    coeffs = [QUINTIC] * len(Gs)
    want = fs4.root_ns_batched(Gs, K=3, coeffs=coeffs)
    S = shard.ShardedRootNS(SHAPES, K=3, coeffs=coeffs, device="cuda")
    assert S.local == list(range(len(SHAPES)))
    for _ in range(2):                   # the second call overwrites the same views
        got = S(Gs)
        torch.cuda.synchronize()
        assert fs4.device_status(S.workspace) == 0
        for a, b in zip(got, want):
            assert a.shape == b.shape and torch.equal(a, b)
        assert all(o.data_ptr() % 256 == 0 for o in got)

"""The Newton-Schulz entry point for callers that cannot allocate device memory
(fs4_root_ns_noalloc), called through the C ABI.

Some callers have no way to hand the library a workspace: a plugin inside a host
framework that owns every device allocation and lends none, or a loop that is not
allowed to allocate at run time.  This entry point takes its workspace from a fixed
array inside the library instead.  Its results must be those of the
workspace-taking entry point fs4_root_ns on the same input, bit for bit, call after
call, although every call reuses the same array; and they must match the oracle.
This file is collected last on purpose.
"""
import numpy as np
import pytest
import torch

from oracle import root_ns as R
from tests.helpers import rel_frob

pytestmark = pytest.mark.gpu

QUINTIC = (15 / 8, -10 / 8, 3 / 8)
MUON = (3.4445, -4.7750, 2.0315)


def _noalloc(fs4, G, K, coef, clip_k=3.0):
    out = torch.full_like(G, float("nan"))
    st = fs4._lib.lib().fs4_root_ns_noalloc(G.data_ptr(), G.shape[0], G.shape[1], G.stride(0),
                                            out.data_ptr(), out.stride(0), K, *coef, clip_k,
                                            torch.cuda.current_stream().cuda_stream)
    assert st == 0, fs4._lib.STATUS_NAMES.get(st, st)
    return out


def test_noalloc_matches_workspace_entry_point_on_two_calls_in_a_row(fs4):
    """Two calls in a row share the built-in array; the second, smaller one must not see
    anything the first left behind (row and column sums, maxima, tensor scales)."""
    rng = np.random.default_rng(31)
    cases = [((512, 768), 3, MUON, 1.0), ((256, 128), 5, QUINTIC, 8.0)]
    for (m, n), K, coef, scale in cases:
        G = torch.from_numpy((rng.standard_normal((m, n)) * 0.02 * scale).astype(np.float32)).cuda()
        got = _noalloc(fs4, G, K, coef).cpu().numpy()
        want = fs4.root_ns(G, K, *coef, clip_k=3.0).cpu().numpy()
        assert np.all(np.isfinite(got))
        assert np.array_equal(got.view(np.uint32), want.view(np.uint32))
        oracle = R.root_ns(G.cpu().numpy(), K, *coef, clip_k=3.0)
        assert rel_frob(got, oracle) <= 2e-2


def test_noalloc_rejects_matrices_beyond_the_built_in_scratch(fs4):
    G = torch.zeros((1024, 2048), device="cuda")
    out = torch.zeros_like(G)
    st = fs4._lib.lib().fs4_root_ns_noalloc(G.data_ptr(), 1024, 2048, 2048, out.data_ptr(), 2048, 5,
                                            *MUON, 3.0, torch.cuda.current_stream().cuda_stream)
    assert st == -4   # FS4_ERR_WORKSPACE, nothing launched
    assert not out.any()

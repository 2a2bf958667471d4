"""CPU-only checks of the C ABI: the library loads, exports every entry point
declared in include/fs4.h, and its host-side validation and planning work
without a GPU (no compute call is made here)."""
import ctypes
import os
import re

import numpy as np
import pytest

from tests.helpers import plain_to_tiled, tiled_to_plain

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def F():
    import nvfp4_precision_optimizer_b200 as F
    F._lib.lib()
    return F


def header_functions():
    src = open(os.path.join(ROOT, "include", "fs4.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(fs4_[a-z0-9_]+)\s*\(", src)) - {"fs4_status"})


def test_library_exports_every_declared_entry_point(F):
    names = header_functions()
    assert len(names) >= 11
    lib = F._lib.lib()
    for name in names:
        assert hasattr(lib, name), name
    assert set(names) == set(F._lib.SIGNATURES)


def test_status_strings(F):
    lib = F._lib.lib()
    for code, name in F._lib.STATUS_NAMES.items():
        assert lib.fs4_status_string(code).decode() == name
    assert lib.fs4_status_string(-99).decode() == "FS4_ERR_UNKNOWN"


def test_quantize_rejects_bad_arguments_before_touching_the_device(F):
    lib = F._lib.lib()
    ws = ctypes.create_string_buffer(512)
    wsp = (ctypes.addressof(ws) + 255) // 256 * 256
    fake = 1 << 20
    q = lib.fs4_nvfp4_quantize
    assert q(None, 4, 16, 16, 0, fake, fake, fake, 0, wsp, 256, None) == -1       # null x
    assert q(fake, 4, 17, 17, 0, fake, fake, fake, 0, wsp, 256, None) == -2       # cols % 16
    assert q(fake, 17, 16, 16, 1, fake, fake, fake, 0, wsp, 256, None) == -2      # column axis: rows % 16
    assert q(fake, 0, 16, 16, 0, fake, fake, fake, 0, wsp, 256, None) == -2       # empty
    assert q(fake, 4, 16, 8, 0, fake, fake, fake, 0, wsp, 256, None) == -1        # ld < cols
    assert q(fake, 4, 16, 16, 2, fake, fake, fake, 0, wsp, 256, None) == -1       # bad axis
    assert q(fake, 4, 16, 16, 0, fake + 8, fake, fake, 0, wsp, 256, None) == -1   # misaligned codes
    assert q(fake, 4, 16, 16, 0, fake, fake, fake, 1 << 7, wsp, 256, None) == -1  # unknown flag
    # the test-only stall flag does not excuse another unknown bit
    assert q(fake, 4, 16, 16, 0, fake, fake, fake, F.FS4_TEST_STALL | (1 << 7), wsp, 256, None) == -1
    assert q(fake, 4, 16, 16, 0, fake, fake, fake, 0, wsp, 100, None) == -4       # workspace too small
    assert q(fake, 4, 16, 16, 0, fake, fake, fake, 0, wsp + 8, 256, None) == -4   # misaligned workspace


def test_gemm_and_dequantize_reject_bad_arguments(F):
    lib = F._lib.lib()
    fake = 1 << 20
    assert lib.fs4_nvfp4_gemm(fake, fake, fake, fake, fake, fake, 0, 8, 8, fake, 8, fake, 256, None) == -2
    assert lib.fs4_nvfp4_gemm(fake, fake, fake, fake, fake, fake, 8, 8, 8, fake, 4, fake, 256, None) == -1
    assert lib.fs4_nvfp4_gemm(fake, fake, fake, fake, fake, fake, 8, 8, 8, fake, 8, fake, 16, None) == -4
    assert lib.fs4_nvfp4_gemm(None, fake, fake, fake, fake, fake, 8, 8, 8, fake, 8, fake, 256, None) == -1
    assert lib.fs4_nvfp4_dequantize(fake, fake, fake, 4, 24, fake, 24, 0, None) == -2
    assert lib.fs4_nvfp4_dequantize(fake, fake, fake, 4, 32, fake, 16, 0, None) == -1


def _desc(F, G, out, m, n, ld=None, ld_out=None, abc=(3.4445, -4.775, 2.0315)):
    return F._lib.NsDesc(G, out, m, n, ld or n, ld_out or n, *abc)


def test_root_ns_rejects_bad_arguments(F):
    lib = F._lib.lib()
    G, O, W = 1 << 30, 1 << 34, 1 << 38
    ok = lib.fs4_root_ns_workspace_size(64, 96)
    assert ok > 0
    ns = lib.fs4_root_ns
    assert ns(G, 64, 96, 96, O, 96, 5, 1.0, 0.0, 0.0, 3.0, 0, W, ok - 1, None) == -4   # small workspace
    assert ns(G, 64, 96, 96, O, 96, 0, 1.0, 0.0, 0.0, 3.0, 0, W, ok, None) == -2       # K = 0
    assert ns(G, 64, 96, 96, O, 96, 33, 1.0, 0.0, 0.0, 3.0, 0, W, ok, None) == -2      # K too large
    assert ns(G, 64, 90, 90, O, 90, 5, 1.0, 0.0, 0.0, 3.0, 0, W, ok, None) == -2       # n % 16
    assert ns(G, 8, 96, 96, O, 96, 5, 1.0, 0.0, 0.0, 3.0, 0, W, ok, None) == -2        # m < 16
    assert ns(G, 64, 96, 64, O, 96, 5, 1.0, 0.0, 0.0, 3.0, 0, W, ok, None) == -1       # ld < n
    assert ns(None, 64, 96, 96, O, 96, 5, 1.0, 0.0, 0.0, 3.0, 0, W, ok, None) == -1
    assert ns(G, 64, 96, 96, O, 96, 5, float("nan"), 0.0, 0.0, 3.0, 0, W, ok, None) == -1
    assert ns(G, 64, 96, 96, O, 96, 5, 1.0, 0.0, 0.0, float("inf"), 0, W, ok, None) == -1
    assert ns(G, 64, 96, 96, G + 1024, 96, 5, 1.0, 0.0, 0.0, 3.0, 0, W, ok, None) == -3  # out overlaps G
    assert ns(G, 64, 96, 96, O, 96, 5, 1.0, 0.0, 0.0, 3.0, 0, G, ok, None) == -3         # ws overlaps G
    assert ns(G, 64, 96, 96, O, 96, 5, 1.0, 0.0, 0.0, 3.0, 0, W + 4, ok, None) == -4     # misaligned ws
    assert ns(G, 64, 96, 96, O, 96, 5, 1.0, 0.0, 0.0, 3.0, 1 << 5, W, ok, None) == -1    # unknown flag
    # the Hadamard option needs the masks only the _ex entry point takes
    assert ns(G, 64, 96, 96, O, 96, 5, 1.0, 0.0, 0.0, 3.0, F.FS4_NS_RHT, W, ok, None) == -1
    desc = (F.NsDesc * 1)()
    desc[0].G, desc[0].out, desc[0].m, desc[0].n, desc[0].ld, desc[0].ld_out = G, O, 64, 96, 96, 96
    desc[0].a, desc[0].b, desc[0].c = 1.0, 0.0, 0.0
    ex = lib.fs4_root_ns_batched_ex
    assert ex(1, desc, 5, 3.0, F.FS4_NS_RHT, None, W, ok, None) == -1                    # no masks
    masks = (ctypes.c_uint16 * 15)(*range(15))
    assert ex(1, desc, 5, 3.0, F.FS4_NS_RHT | F.FS4_NS_ADAPTIVE46, masks, W, ok - 1, None) == -4
    assert ns(G, 64, 96, 96, O, 96, 5, 1.0, 0.0, 0.0, 3.0, 1 << 29, W, ok, None) == -1   # unknown flag
    # the test-only stall flag is accepted (the call then fails on the workspace size)
    assert ns(G, 64, 96, 96, O, 96, 5, 1.0, 0.0, 0.0, 3.0, F.FS4_TEST_STALL, W, ok - 1, None) == -4
    # the quantile clip takes clip_k as a ratio in (0, 1]
    qf = F.FS4_NS_CLIP_QUANTILE
    assert ns(G, 64, 96, 96, O, 96, 5, 1.0, 0.0, 0.0, 0.0, qf, W, ok, None) == -1
    assert ns(G, 64, 96, 96, O, 96, 5, 1.0, 0.0, 0.0, 3.0, qf, W, ok, None) == -1
    assert ns(G, 64, 96, 96, O, 96, 5, 1.0, 0.0, 0.0, -0.5, qf, W, ok, None) == -1
    assert ns(G, 64, 96, 96, O, 96, 5, 1.0, 0.0, 0.0, 0.99, qf, W, ok - 1, None) == -4   # accepted
    assert ns(G, 64, 96, 96, O, 96, 5, 1.0, 0.0, 0.0, 1.0, qf, W, ok - 1, None) == -4


def test_batched_rejects_overlapping_outputs_and_bad_counts(F):
    lib = F._lib.lib()
    arr = (F._lib.NsDesc * 2)()
    arr[0] = _desc(F, 1 << 30, 1 << 34, 32, 32)
    arr[1] = _desc(F, 1 << 31, (1 << 34) + 64, 32, 32)
    # the size query looks at shapes only; the call itself rejects the overlapping outputs
    need = lib.fs4_root_ns_batched_workspace_size(2, arr)
    assert need > 0 and need == F.ns_batched_workspace_size([(32, 32), (32, 32)])
    assert lib.fs4_root_ns_batched(2, arr, 5, 3.0, 0, 1 << 40, 1 << 30, None) == -3
    assert lib.fs4_root_ns_batched(0, arr, 5, 3.0, 0, 1 << 40, 1 << 30, None) == -2
    assert lib.fs4_root_ns_batched(225, arr, 5, 3.0, 0, 1 << 40, 1 << 30, None) == -2


def test_workspace_plan_and_layout(F):
    shapes = [(256, 256), (4096, 1024), (48, 80)]
    need = F.ns_batched_workspace_size(shapes)
    assert need > 0 and need % 1024 == 0
    prev_end = 0
    for i, (m, n) in enumerate(shapes):
        lay = F.ns_layout(shapes, i)
        mm, nn = min(m, n), max(m, n)
        assert lay.mp == round_up(mm) and lay.np == round_up(nn)
        offs = [lay.X, lay.A, lay.qX_codes[0], lay.qX_scales[0], lay.qX_codes[1], lay.qX_scales[1],
                lay.qXT_codes[0], lay.qXT_scales[0], lay.qXT_codes[1], lay.qXT_scales[1],
                lay.qA_codes, lay.qA_scales, lay.qB_codes, lay.qB_scales]
        assert offs == sorted(offs) and offs[0] >= prev_end
        assert all(o % 1024 == 0 for o in offs)
        prev_end = lay.qB_scales + lay.mp * lay.mp // 16
        assert lay.scalars > 0 and lay.scalars < lay.X
    assert prev_end <= need
    single = F.ns_workspace_size(48, 80)
    assert single == F.ns_batched_workspace_size([(48, 80)])
    assert F.ns_workspace_size(48, 81) == 0


def round_up(v, a=256):
    return (v + a - 1) // a * a


def test_tiled_layout_helpers_round_trip():
    rng = np.random.default_rng(0)
    for rows, cols in [(1, 16), (128, 256), (200, 48), (300, 520)]:
        codes = rng.integers(0, 256, (rows, cols // 2), dtype=np.uint8)
        scales = rng.integers(0, 256, (rows, cols // 16), dtype=np.uint8)
        ct, st = plain_to_tiled(codes, scales, rows, cols)
        c2, s2, cp, sp = tiled_to_plain(ct, st, rows, cols)
        assert np.array_equal(c2, codes) and np.array_equal(s2, scales)
        assert not cp[rows:].any() and not cp[:, cols // 2:].any()


def test_tiled_layout_matches_header_formula():
    """Spot-check the documented byte formulas of the TILED layout."""
    rows, cols = 256, 512
    codes = np.zeros((rows, cols // 2), np.uint8)
    scales = np.zeros((rows, cols // 16), np.uint8)
    r, c = 133, 300                   # element (r, c); chunk j = (c % 256) // 32
    codes[r, c // 2] = 0xAB
    scales[r, c // 16] = 0xCD
    ct, st = plain_to_tiled(codes, scales, rows, cols)
    Cp = 512
    tile = (r // 128) * (Cp // 256) + c // 256
    j = (c % 256) // 32
    off = tile * 16384 + 128 * (r % 128) + 16 * (j ^ (r % 8)) + (c % 32) // 2
    assert ct[off] == 0xAB and np.count_nonzero(ct) == 1
    atom = (r // 128) * (Cp // 64) + c // 64
    soff = atom * 512 + 16 * (r % 32) + 4 * ((r % 128) // 32) + (c // 16) % 4
    assert st[soff] == 0xCD and np.count_nonzero(st) == 1


def test_momentum_argument_errors(F):
    """fs4_momentum_nvfp4 rejects bad arguments on the host, before any launch."""
    lib = F._lib.lib()
    mo = lib.fs4_momentum_nvfp4
    g, c, s, sg, W, mout = 1 << 20, 2 << 20, 3 << 20, 4 << 20, 5 << 20, 6 << 20   # fake aligned pointers
    wsz = lib.fs4_momentum_workspace_size()
    ok = (g, 32, 64, 64, 0.9, None, None, None, 0, c, s, sg, 0, 1, mout, 64, W, wsz, None)
    def call(**kw):
        args = list(ok)
        names = ["g", "rows", "cols", "ld", "beta", "pc", "ps", "psg", "pmask", "c", "s", "sg",
                 "mask", "seed", "m", "ldo", "ws", "wsb", "st"]
        for k, v in kw.items():
            args[names.index(k)] = v
        return mo(*args)
    assert call(cols=72) == -2                       # cols % 16
    assert call(rows=0) == -2
    assert call(g=None) == -1
    assert call(c=None) == -1
    assert call(beta=float("nan")) == -1
    assert call(ld=48) == -1                         # ld < cols
    assert call(ldo=48) == -1
    assert call(pc=c) == -1                          # partial previous state
    assert call(mask=1 << 16) == -1
    assert call(c=c + 8) == -1                       # codes not 16-byte aligned
    assert call(m=g + 1024) == -3                    # m_out overlaps g
    assert call(ws=W + 4) == -4
    assert call(wsb=wsz - 1) == -4


def test_nvfp4_source_argument_errors(F):
    """fs4_root_ns_batched_nvfp4 checks its states on the host, before any launch."""
    lib = F._lib.lib()
    nv = lib.fs4_root_ns_batched_nvfp4
    arr = (F._lib.NsDesc * 1)()
    arr[0] = F._lib.NsDesc(None, 1 << 34, 64, 96, 96, 96, 1.0, 0.0, 0.0)
    st = (F._lib.Nvfp4State * 1)()
    st[0] = F._lib.Nvfp4State(1 << 30, 1 << 31, 1 << 32, 0x1234)
    need = lib.fs4_root_ns_batched_workspace_size(1, arr)   # a null G is fine for sizing
    assert need > 0
    W = 1 << 40
    assert nv(1, arr, st, 5, 3.0, 0, None, W, need - 1, None) == -4       # accepted up to the size
    assert nv(1, arr, None, 5, 3.0, 0, None, W, need, None) == -1         # no states
    bad = (F._lib.Nvfp4State * 1)()
    bad[0] = F._lib.Nvfp4State(1 << 30, (1 << 31) + 8, 1 << 32, 0)       # scales misaligned
    assert nv(1, arr, bad, 5, 3.0, 0, None, W, need, None) == -1
    bad[0] = F._lib.Nvfp4State(1 << 30, 1 << 31, 1 << 32, 1 << 16)       # mask too wide
    assert nv(1, arr, bad, 5, 3.0, 0, None, W, need, None) == -1
    arr[0] = F._lib.NsDesc(1 << 33, 1 << 34, 64, 96, 96, 96, 1.0, 0.0, 0.0)   # G must be null
    assert nv(1, arr, st, 5, 3.0, 0, None, W, need, None) == -1
    arr[0] = F._lib.NsDesc(None, (1 << 30) + 64, 64, 96, 96, 96, 1.0, 0.0, 0.0)  # out over the codes
    assert nv(1, arr, st, 5, 3.0, 0, None, W, need, None) == -3


def test_timed_entry_points_check_their_events_on_the_host(F):
    """The phase-timed calls (fs4_root_ns_batched_timed, fs4_root_ns_batched_nvfp4_timed,
    fs4_root_ns_bf16_batched_timed) refuse a missing event array, fewer than 3 + 3K events or
    a null event handle before anything is launched (the handles are not touched here)."""
    lib = F._lib.lib()
    K = 2
    n = 3 + 3 * K
    arr = (F._lib.NsDesc * 1)()
    arr[0] = F._lib.NsDesc(1 << 33, 1 << 34, 64, 96, 96, 96, 1.0, 0.0, 0.0)
    W = 1 << 40
    ev = (F._lib.c_vp * n)(*([1 << 20] * n))
    ev_null = (F._lib.c_vp * n)(*([1 << 20] * (n - 1) + [None]))
    need = lib.fs4_root_ns_batched_workspace_size(1, arr)
    t = lib.fs4_root_ns_batched_timed
    assert t(1, arr, K, 3.0, 0, None, W, need, None, None, n) == -1      # no event array
    assert t(1, arr, K, 3.0, 0, None, W, need, None, ev, n - 1) == -1    # one event short
    assert t(1, arr, K, 3.0, 0, None, W, need, None, ev_null, n) == -1   # a null handle
    assert t(1, arr, K, 3.0, 0, None, W, need - 1, None, ev, n) == -4    # workspace first
    need_b = lib.fs4_root_ns_bf16_batched_workspace_size(1, arr)
    assert need_b > need                                                   # 2 B per view element
    tb = lib.fs4_root_ns_bf16_batched_timed
    assert tb(1, arr, K, 3.0, 0, W, need_b, None, None, n) == -1
    assert tb(1, arr, K, 3.0, 0, W, need_b, None, ev, n - 1) == -1
    st = (F._lib.Nvfp4State * 1)()
    st[0] = F._lib.Nvfp4State(1 << 30, 1 << 31, 1 << 32, 0x1234)
    arr[0] = F._lib.NsDesc(None, 1 << 34, 64, 96, 96, 96, 1.0, 0.0, 0.0)
    tn = lib.fs4_root_ns_batched_nvfp4_timed
    assert tn(1, arr, st, K, 3.0, 0, None, W, need, None, None, n) == -1
    assert tn(1, arr, None, K, 3.0, 0, None, W, need, None, ev, n) == -1
    assert tn(1, arr, st, K, 3.0, 0, None, W, need, None, ev, n - 1) == -1


def test_missing_library_fails_loudly():
    """Without libfs4.so every call raises ImportError: there is no CPU or library
    fallback.  Checked in a fresh interpreter whose loader points at a missing path."""
    import subprocess
    import sys
    code = (
        "import nvfp4_precision_optimizer_b200 as F\n"
        "F._lib.LIB_PATH = '/nonexistent/libfs4.so'\n"
        "F._lib._lib = None\n"
        "import torch\n"
        "# calls that reach the library first: ImportError\n"
        "for call in (F._lib.lib, lambda: F.ns_workspace_size(256, 256),\n"
        "             lambda: F.ns_batched_workspace_size([(256, 512)])):\n"
        "    try:\n"
        "        call()\n"
        "    except ImportError:\n"
        "        continue\n"
        "    except Exception as e:\n"
        "        raise SystemExit('wrong error: %r' % (e,))\n"
        "    raise SystemExit('no error')\n"
        "# compute calls on host tensors are refused before anything runs (no CPU path)\n"
        "for call in (lambda: F.quantize(torch.zeros(16, 16)),\n"
        "             lambda: F.root_ns(torch.zeros(16, 16))):\n"
        "    try:\n"
        "        call()\n"
        "    except (ImportError, ValueError):\n"
        "        continue\n"
        "    raise SystemExit('a host tensor was accepted')\n"
        "print('ok')\n")
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip().endswith("ok"), r.stdout + r.stderr

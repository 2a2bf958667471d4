"""Per-product parity checks of one Newton-Schulz iteration read out of a workspace.

"Full-Stack FP4" (arXiv 2607.04422), Section 3.4, iteration k:
  product 1  A   = qX qX^T
  product 2  B   = b A + c qA qA16x1         (qA16x1 = qA^T: A is symmetric)
  product 3  X'  = a X + qB qX16x1
Each GPU product is compared with the float64 product of the GPU's own dequantised
operands (the operands are read from the workspace, so only the product and its
epilogue are under test), and every NVFP4 view the epilogue writes is compared byte
for byte with the oracle's quantisation of the GPU's own FP32 result at the GPU's
tensor scale.  `grab(off, nbytes)` returns workspace bytes as a numpy uint8 array.
"""
from __future__ import annotations

import numpy as np

from oracle import cpp_oracle as C
from tests.helpers import rel_frob, tiled_to_plain


def f32(grab, off, rows, cols):
    return grab(off, 4 * rows * cols).view(np.float32).reshape(rows, cols)


def view(grab, codes_off, scales_off, rows, cols):
    """PLAIN (codes, scales) of a rows x cols TILED view, padding included."""
    nc, ns = rows * cols // 2, rows * cols // 16
    _, _, c, s = tiled_to_plain(grab(codes_off, nc), grab(scales_off, ns), rows, cols)
    return c, s


def scalars(grab, lay):
    return grab(lay.scalars, 4 * 192).view(np.float32)


def upper_mask(mp):
    t = np.arange(mp) // 256
    return t[:, None] <= t[None, :]


def symmetric_from_tiles(M, mp):
    """The symmetric mp x mp matrix whose 256 x 256 tiles on and above the diagonal
    are those of M (diagonal tiles kept as computed)."""
    up = upper_mask(mp)
    return np.where(up, M, M.T)


def check_second_product(grab_after_1, grab_after_2, lay, k, b, c):
    """Product 2 of iteration k.  grab_after_1: workspace after product 1 (A, qA);
    grab_after_2: after product 2 with the debug stop (B written over A, qB).
    Returns (relative Frobenius error of B over the computed tiles, qB bit-exact)."""
    mp = lay.mp
    up = upper_mask(mp)
    # only the tiles on and above the diagonal are ever written: mask the rest
    A = np.where(up, f32(grab_after_1, lay.A, mp, mp), np.float32(0)).astype(np.float64)
    qa_c, qa_s = view(grab_after_1, lay.qA_codes, lay.qA_scales, mp, mp)
    sg_a = scalars(grab_after_1, lay)[64 + k]
    dA = C.dequantize_rows(qa_c, qa_s, sg_a)
    P = dA @ dA.T
    want = np.float64(np.float32(b)) * symmetric_from_tiles(A, mp) + np.float64(np.float32(c)) * P
    Bg = np.where(up, f32(grab_after_2, lay.A, mp, mp), np.float32(0))
    err = rel_frob(Bg.astype(np.float64)[up], want[up])
    sg_b = scalars(grab_after_2, lay)[128 + k]
    oc, os_, _ = C.quantize_rows(np.ascontiguousarray(symmetric_from_tiles(Bg, mp), np.float32), s_g=sg_b)
    gc, gs = view(grab_after_2, lay.qB_codes, lay.qB_scales, mp, mp)
    return err, bool(np.array_equal(gc, oc) and np.array_equal(gs, os_))


def check_third_product(grab_after_2, grab_after_3, lay, k, a, m, n):
    """Product 3 of iteration k.  grab_after_2: workspace after product 2 (X_k, qB,
    the 16x1 view of X_k in slot k % 2); grab_after_3: after product 3 (X_{k+1}).
    Returns the relative Frobenius error of X_{k+1} against a X_k + deq(qB) deq(qX16)."""
    mp, np_ = lay.mp, lay.np
    X = f32(grab_after_2, lay.X, mp, np_).astype(np.float64)
    qb_c, qb_s = view(grab_after_2, lay.qB_codes, lay.qB_scales, mp, mp)
    sc = scalars(grab_after_2, lay)
    dB = C.dequantize_rows(qb_c, qb_s, sc[128 + k])
    slot = k % 2
    qt_c, qt_s = view(grab_after_2, lay.qXT_codes[slot], lay.qXT_scales[slot], np_, mp)
    dXT = C.dequantize_rows(qt_c, qt_s, sc[k])           # n x m: the 16x1 view of X_k, transposed
    want = np.float64(np.float32(a)) * X + dB @ dXT.T
    got = f32(grab_after_3, lay.X, mp, np_).astype(np.float64)
    return rel_frob(got[:m, :n], want[:m, :n])


def check_first_product_views(grab_after_3, lay, k, m, n):
    """The two NVFP4 views of X_{k+1} written by product 3 (slot (k + 1) % 2) against
    the oracle's quantisation of the GPU's X_{k+1} at the GPU's tensor scale."""
    mp, np_ = lay.mp, lay.np
    X1 = np.ascontiguousarray(f32(grab_after_3, lay.X, mp, np_))
    sg = scalars(grab_after_3, lay)[k + 1]
    slot = (k + 1) % 2
    oc, os_, _ = C.quantize_rows(X1, s_g=sg)
    gc, gs = view(grab_after_3, lay.qX_codes[slot], lay.qX_scales[slot], mp, np_)
    ok_rows = np.array_equal(gc, oc) and np.array_equal(gs, os_)
    oc, os_, _ = C.quantize_rows(np.ascontiguousarray(X1.T), s_g=sg)
    gc, gs = view(grab_after_3, lay.qXT_codes[slot], lay.qXT_scales[slot], np_, mp)
    return bool(ok_rows and np.array_equal(gc, oc) and np.array_equal(gs, os_))

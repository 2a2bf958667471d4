"""Test utilities: TILED <-> PLAIN layout permutations and workspace readers.

These are index permutations of the documented TILED layout (include/fs4.h);
they hold none of the method's arithmetic.
"""
from __future__ import annotations

import numpy as np


def round_up(v: int, a: int) -> int:
    return (v + a - 1) // a * a


def _chunk_index():
    r = np.arange(128)
    j = np.arange(8)
    return r, (j[None, :] ^ (r[:, None] % 8))          # physical chunk of logical chunk j in row r


def _scale_index():
    r = np.arange(128)[:, None]
    kb = np.arange(4)[None, :]
    return 16 * (r % 32) + 4 * (r // 32) + kb          # [128, 4] byte inside a 512-byte atom


def tiled_to_plain(codes_t, scales_t, rows: int, cols: int):
    """TILED codes/scales of a rows x cols NVFP4 matrix -> (codes [rows, cols/2],
    scales [rows, cols/16]) in the PLAIN layout, plus the padded arrays."""
    Rp, Cp = round_up(rows, 128), round_up(cols, 256)
    ct = np.asarray(codes_t, dtype=np.uint8).reshape(Rp // 128, Cp // 256, 128, 8, 16)
    r, pos = _chunk_index()
    ct = ct[:, :, r[:, None], pos, :]                  # logical chunk order
    plain = ct.transpose(0, 2, 1, 3, 4).reshape(Rp, Cp // 2)
    st = np.asarray(scales_t, dtype=np.uint8).reshape(Rp // 128, Cp // 64, 512)
    sp = st[:, :, _scale_index()].transpose(0, 2, 1, 3).reshape(Rp, Cp // 16)
    return plain[:rows, :cols // 2], sp[:rows, :cols // 16], plain, sp


def plain_to_tiled(codes, scales, rows: int, cols: int):
    """PLAIN codes/scales -> TILED byte arrays (zero padded)."""
    Rp, Cp = round_up(rows, 128), round_up(cols, 256)
    pc = np.zeros((Rp, Cp // 2), np.uint8)
    pc[:rows, :cols // 2] = codes
    ps = np.zeros((Rp, Cp // 16), np.uint8)
    ps[:rows, :cols // 16] = scales
    ct = pc.reshape(Rp // 128, 128, Cp // 256, 8, 16).transpose(0, 2, 1, 3, 4).copy()
    out = np.zeros_like(ct)
    r, pos = _chunk_index()
    out[:, :, r[:, None], pos, :] = ct
    st = ps.reshape(Rp // 128, 128, Cp // 64, 4).transpose(0, 2, 1, 3)
    so = np.zeros((Rp // 128, Cp // 64, 512), np.uint8)
    so[:, :, _scale_index()] = st
    return out.reshape(-1), so.reshape(-1)


def rel_frob(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    den = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (den if den > 0 else 1.0))


def ws_f32(ws_np: np.ndarray, off: int, count: int) -> np.ndarray:
    return ws_np[off:off + 4 * count].view(np.float32)


def ws_bytes(ws_np: np.ndarray, off: int, count: int) -> np.ndarray:
    return ws_np[off:off + count]


def tiled_bf16_to_plain(buf, rows: int, cols: int) -> np.ndarray:
    """The TILED BF16 layout (tiles of 128 rows x 64 elements, 16-byte chunk j of row r
    at position j ^ (r % 8)) of a rows x cols matrix -> its FP32 values, padding
    included (shape Rp x Cp)."""
    Rp, Cp = round_up(rows, 128), round_up(cols, 64)
    t = np.asarray(buf, dtype=np.uint8).reshape(Rp // 128, Cp // 64, 128, 8, 16)
    r, pos = _chunk_index()
    t = t[:, :, r[:, None], pos, :]                    # logical chunk order
    plain = np.ascontiguousarray(t.transpose(0, 2, 1, 3, 4)).reshape(Rp, Cp * 2)
    u16 = plain.view(np.uint16)
    return (u16.astype(np.uint32) << 16).view(np.float32)

"""Direct NVFP4 Newton-Schulz orthogonalisation (the Q-Root step of "Full-Stack
FP4", arXiv 2607.04422, Section 3.4) on NVIDIA B200.

Every step runs in the sm_100a kernels of libfs4.so behind the C ABI declared
in include/fs4.h; this module only marshals torch tensors (device memory and
streams) into those calls.  There is no CPU or fallback path.
"""
from __future__ import annotations

import ctypes
from typing import Sequence

import torch

from . import _lib
from ._lib import (FS4_AXIS_COL, FS4_AXIS_ROW, FS4_LAYOUT_TILED, FS4_NS_ADAPTIVE46, FS4_NS_CLIP_QUANTILE, FS4_NS_RHT,
                   FS4_SG_AMAX, FS4_TEST_STALL, Fs4Error, NsDesc, NsLayout, check, stop_after)

MUON_COEFFS = (3.4445, -4.7750, 2.0315)

__all__ = [
    "quantize", "quantize_batched", "dequantize", "gemm", "root_ns", "root_ns_batched", "ns_workspace_size",
    "ns_batched_workspace_size", "ns_layout", "device_status", "tiled_shape", "Fs4Error",
    "momentum_nvfp4", "root_ns_batched_nvfp4", "root_ns_bf16_batched", "ns_bf16_batched_workspace_size",
    "ns_bf16_layout",
    "MUON_COEFFS", "stop_after", "FS4_AXIS_ROW", "FS4_AXIS_COL", "FS4_TEST_STALL",
    "FS4_NS_RHT", "FS4_NS_ADAPTIVE46", "FS4_NS_CLIP_QUANTILE",
]


def _ptr(t: torch.Tensor | None) -> int | None:
    return None if t is None else t.data_ptr()


def _stream(stream) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _check_f32_matrix(x: torch.Tensor, name: str) -> None:
    if not x.is_cuda or x.dtype != torch.float32 or x.dim() != 2 or x.stride(1) != 1:
        raise ValueError(f"{name} must be a CUDA float32 matrix with unit column stride")


def _round_up(v: int, a: int) -> int:
    return (v + a - 1) // a * a


def tiled_shape(rows: int, cols: int) -> tuple[int, int]:
    """(codes bytes, scales bytes) of a rows x cols matrix in the TILED layout."""
    rp, cp = _round_up(rows, 128), _round_up(cols, 256)
    return rp * cp // 2, rp * cp // 16


def quantize(x: torch.Tensor, axis: int = FS4_AXIS_ROW, tiled: bool = False,
             sg_mode: str = "pow2", workspace: torch.Tensor | None = None, stream=None,
             flags: int = 0):
    """NVFP4-quantise x (fs4_nvfp4_quantize).  Returns (codes, scales, s_g).
    flags: extra call flags (FS4_TEST_STALL for the timeout test)."""
    _check_f32_matrix(x, "x")
    rows, cols = x.shape
    R, C = (rows, cols) if axis == FS4_AXIS_ROW else (cols, rows)
    if tiled:
        ncode, nscale = tiled_shape(R, C)
        codes = torch.empty(ncode, dtype=torch.uint8, device=x.device)
        scales = torch.empty(nscale, dtype=torch.uint8, device=x.device)
    else:
        codes = torch.empty((R, C // 2), dtype=torch.uint8, device=x.device)
        scales = torch.empty((R, max(C // 16, 1)), dtype=torch.uint8, device=x.device)
    s_g = torch.empty(1, dtype=torch.float32, device=x.device)
    ws_bytes = _lib.lib().fs4_nvfp4_quantize_workspace_size()
    if workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=x.device)
    flags |= (FS4_LAYOUT_TILED if tiled else 0) | (FS4_SG_AMAX if sg_mode == "amax" else 0)
    ld = x.stride(0) if rows > 1 else cols
    check(_lib.lib().fs4_nvfp4_quantize(x.data_ptr(), rows, cols, ld, axis,
                                        codes.data_ptr(), scales.data_ptr(), s_g.data_ptr(), flags,
                                        workspace.data_ptr(), workspace.numel(), _stream(stream)),
          "fs4_nvfp4_quantize")
    return codes, scales, s_g


def quantize_batched(xs: Sequence[torch.Tensor], axis: int = FS4_AXIS_ROW, tiled: bool = False,
                     sg_mode: str = "pow2", workspace: torch.Tensor | None = None, stream=None,
                     flags: int = 0):
    """fs4_nvfp4_quantize on every matrix of xs in one launch
    (fs4_nvfp4_quantize_batched).  Returns a list of (codes, scales, s_g)."""
    outs = []
    arr = (_lib.QuantDesc * len(xs))()
    for i, x in enumerate(xs):
        _check_f32_matrix(x, "x")
        rows, cols = x.shape
        R, C = (rows, cols) if axis == FS4_AXIS_ROW else (cols, rows)
        if tiled:
            ncode, nscale = tiled_shape(R, C)
            codes = torch.empty(ncode, dtype=torch.uint8, device=x.device)
            scales = torch.empty(nscale, dtype=torch.uint8, device=x.device)
        else:
            codes = torch.empty((R, C // 2), dtype=torch.uint8, device=x.device)
            scales = torch.empty((R, max(C // 16, 1)), dtype=torch.uint8, device=x.device)
        s_g = torch.empty(1, dtype=torch.float32, device=x.device)
        ld = x.stride(0) if rows > 1 else cols
        arr[i] = _lib.QuantDesc(x.data_ptr(), rows, cols, ld, axis, codes.data_ptr(), scales.data_ptr(),
                                s_g.data_ptr())
        outs.append((codes, scales, s_g))
    need = int(_lib.lib().fs4_nvfp4_quantize_batched_workspace_size(len(xs)))
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=xs[0].device)
    flags |= (FS4_LAYOUT_TILED if tiled else 0) | (FS4_SG_AMAX if sg_mode == "amax" else 0)
    check(_lib.lib().fs4_nvfp4_quantize_batched(len(xs), arr, flags, workspace.data_ptr(),
                                                workspace.numel(), _stream(stream)),
          "fs4_nvfp4_quantize_batched")
    return outs


def dequantize(codes: torch.Tensor, scales: torch.Tensor, s_g: torch.Tensor, rows: int, cols: int,
               tiled: bool = False, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """FP32 rows x cols matrix from an NVFP4 one (fs4_nvfp4_dequantize); `out`, if
    given, is a rows x cols FP32 view with unit column stride (any row stride)."""
    if out is None:
        y = torch.empty((rows, cols), dtype=torch.float32, device=codes.device)
    else:
        _check_f32_matrix(out, "out")
        if tuple(out.shape) != (rows, cols):
            raise ValueError(f"out must be {rows} x {cols}, got {tuple(out.shape)}")
        y = out
    check(_lib.lib().fs4_nvfp4_dequantize(codes.data_ptr(), scales.data_ptr(), s_g.data_ptr(),
                                          rows, cols, y.data_ptr(), _ld(y),
                                          FS4_LAYOUT_TILED if tiled else 0, _stream(stream)),
          "fs4_nvfp4_dequantize")
    return y


def momentum_nvfp4(g: torch.Tensor, beta: float, state=None, prev_mask: int = 0, mask: int = 0,
                   seed: int = 0, want_m: bool = True, out_state=None,
                   workspace: torch.Tensor | None = None, stream=None):
    """One step of the NVFP4-stored first moment (fs4_momentum_nvfp4).  state / out_state
    are (codes, scales, s_g) triples in the PLAIN layout (out_state may be `state` for an
    in-place step).  Returns (m_t FP32 or None, new state)."""
    _check_f32_matrix(g, "g")
    rows, cols = g.shape
    dev = g.device
    if out_state is None:
        out_state = (torch.empty((rows, cols // 2), dtype=torch.uint8, device=dev),
                     torch.empty((rows, cols // 16), dtype=torch.uint8, device=dev),
                     torch.empty(1, dtype=torch.float32, device=dev))
    m_out = torch.empty_like(g) if want_m else None
    if workspace is None:
        workspace = torch.empty(_lib.lib().fs4_momentum_workspace_size(), dtype=torch.uint8, device=dev)
    prev = (None, None, None) if state is None else tuple(t.data_ptr() for t in state)
    check(_lib.lib().fs4_momentum_nvfp4(g.data_ptr(), rows, cols, _ld(g), beta, prev[0], prev[1],
                                        prev[2], prev_mask, out_state[0].data_ptr(),
                                        out_state[1].data_ptr(), out_state[2].data_ptr(), mask,
                                        seed, _ptr(m_out), _ld(m_out) if want_m else cols,
                                        workspace.data_ptr(), workspace.numel(), _stream(stream)),
          "fs4_momentum_nvfp4")
    return m_out, out_state


def gemm(a, b, M: int, N: int, K: int, out: torch.Tensor | None = None,
         workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """D = deq(A) deq(B)^T on the tensor cores (fs4_nvfp4_gemm); a, b are
    (codes, scales, s_g) triples in the TILED layout, A M x K and B N x K."""
    dev = a[0].device
    if out is None:
        out = torch.empty((M, N), dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = torch.empty(256, dtype=torch.uint8, device=dev)
    check(_lib.lib().fs4_nvfp4_gemm(a[0].data_ptr(), a[1].data_ptr(), a[2].data_ptr(),
                                    b[0].data_ptr(), b[1].data_ptr(), b[2].data_ptr(), M, N, K,
                                    out.data_ptr(), _ld(out), workspace.data_ptr(),
                                    workspace.numel(), _stream(stream)),
          "fs4_nvfp4_gemm")
    return out


def _ld(t: torch.Tensor) -> int:
    return t.stride(0) if t.shape[0] > 1 else t.shape[1]


def _descs(Gs: Sequence[torch.Tensor], outs: Sequence[torch.Tensor], coeffs) -> ctypes.Array:
    arr = (NsDesc * len(Gs))()
    for i, (G, o) in enumerate(zip(Gs, outs)):
        a, b, c = coeffs[i]
        arr[i] = NsDesc(G.data_ptr(), o.data_ptr(), G.shape[0], G.shape[1], _ld(G), _ld(o), a, b, c)
    return arr


def ns_workspace_size(m: int, n: int) -> int:
    return int(_lib.lib().fs4_root_ns_workspace_size(m, n))


def _shape_descs(shapes: Sequence[tuple[int, int]]) -> ctypes.Array:
    """Descriptors for size/layout queries: disjoint placeholder address ranges
    (never dereferenced) so that the overlap checks pass."""
    arr = (NsDesc * len(shapes))()
    for i, (m, n) in enumerate(shapes):
        arr[i] = NsDesc((2 * i + 1) << 36, (2 * i + 2) << 36, m, n, n, n, 1.0, 0.0, 0.0)
    return arr


def ns_batched_workspace_size(shapes: Sequence[tuple[int, int]]) -> int:
    return int(_lib.lib().fs4_root_ns_batched_workspace_size(len(shapes), _shape_descs(shapes)))


def _masks(rht_masks, K):
    """Host uint16 array of the 3K H16^r sign masks (or None)."""
    if rht_masks is None:
        return None
    masks = [int(v) & 0xFFFF for v in rht_masks]
    if len(masks) < 3 * K:
        raise ValueError(f"need 3K = {3 * K} sign masks, got {len(masks)}")
    return (ctypes.c_uint16 * len(masks))(*masks)


def root_ns(G: torch.Tensor, K: int = 5, a: float = MUON_COEFFS[0], b: float = MUON_COEFFS[1],
            c: float = MUON_COEFFS[2], clip_k: float = 3.0, out: torch.Tensor | None = None,
            workspace: torch.Tensor | None = None, flags: int = 0, stream=None,
            rht_masks=None, adaptive46: bool = False,
            clip_quantile: float | None = None) -> torch.Tensor:
    """Direct NVFP4 Newton-Schulz step on one FP32 matrix (fs4_root_ns; with
    rht_masks (3K sign masks of H16^r) or adaptive46, fs4_root_ns_batched_ex).
    clip_quantile = q clips at the q-quantile of |X_0| (FS4_NS_CLIP_QUANTILE)
    instead of clip_k * RMS."""
    _check_f32_matrix(G, "G")
    if clip_quantile is not None:
        flags |= FS4_NS_CLIP_QUANTILE
        clip_k = clip_quantile
    if out is None:
        out = torch.empty_like(G)
    m, n = G.shape
    if workspace is None:
        workspace = torch.empty(ns_workspace_size(m, n), dtype=torch.uint8, device=G.device)
    if rht_masks is None and not adaptive46:
        check(_lib.lib().fs4_root_ns(G.data_ptr(), m, n, _ld(G), out.data_ptr(), _ld(out), K,
                                     a, b, c, clip_k, flags, workspace.data_ptr(), workspace.numel(),
                                     _stream(stream)),
              "fs4_root_ns")
        return out
    root_ns_batched([G], K, [(a, b, c)], clip_k, [out], workspace, flags, stream, rht_masks,
                    adaptive46)
    return out


def root_ns_batched(Gs: Sequence[torch.Tensor], K: int = 5, coeffs=None, clip_k: float = 3.0,
                    outs: Sequence[torch.Tensor] | None = None,
                    workspace: torch.Tensor | None = None, flags: int = 0, stream=None,
                    rht_masks=None, adaptive46: bool = False,
                    clip_quantile: float | None = None):
    """Direct NVFP4 Newton-Schulz step on a list of matrices in one grouped call
    (fs4_root_ns_batched); coeffs is a list of per-matrix (a, b, c).  rht_masks
    (3K sign masks of H16^r) and adaptive46 select the Section 3.4 quantiser
    options (fs4_root_ns_batched_ex); clip_quantile = q clips at the q-quantile
    of |X_0| (FS4_NS_CLIP_QUANTILE) instead of clip_k * RMS."""
    if clip_quantile is not None:
        flags |= FS4_NS_CLIP_QUANTILE
        clip_k = clip_quantile
    for G in Gs:
        _check_f32_matrix(G, "G")
    if coeffs is None:
        coeffs = [MUON_COEFFS] * len(Gs)
    if outs is None:
        outs = [torch.empty_like(G) for G in Gs]
    arr = _descs(Gs, outs, coeffs)
    need = int(_lib.lib().fs4_root_ns_batched_workspace_size(len(Gs), arr))
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=Gs[0].device)
    if rht_masks is None and not adaptive46:
        check(_lib.lib().fs4_root_ns_batched(len(Gs), arr, K, clip_k, flags, workspace.data_ptr(),
                                             workspace.numel(), _stream(stream)),
              "fs4_root_ns_batched")
        return outs
    flags |= (FS4_NS_RHT if rht_masks is not None else 0) | (FS4_NS_ADAPTIVE46 if adaptive46 else 0)
    masks = _masks(rht_masks, K)
    check(_lib.lib().fs4_root_ns_batched_ex(len(Gs), arr, K, clip_k, flags,
                                            ctypes.cast(masks, ctypes.c_void_p) if masks else None,
                                            workspace.data_ptr(), workspace.numel(),
                                            _stream(stream)),
          "fs4_root_ns_batched_ex")
    return outs


def root_ns_batched_nvfp4(states, K: int = 5, coeffs=None, clip_k: float = 3.0,
                          outs: Sequence[torch.Tensor] | None = None,
                          workspace: torch.Tensor | None = None, flags: int = 0, stream=None,
                          rht_masks=None, adaptive46: bool = False,
                          clip_quantile: float | None = None):
    """The Newton-Schulz step on matrices given as NVFP4 first-moment states
    (fs4_root_ns_batched_nvfp4): each state is (codes, scales, s_g, mask) as
    momentum_nvfp4 returns it (plus the mask it was stored with); the matrix is
    codes.shape[0] x 2 * codes.shape[1].  Other arguments as root_ns_batched."""
    if clip_quantile is not None:
        flags |= FS4_NS_CLIP_QUANTILE
        clip_k = clip_quantile
    shapes = [(int(st[0].shape[0]), int(st[0].shape[1]) * 2) for st in states]
    dev = states[0][0].device
    if coeffs is None:
        coeffs = [MUON_COEFFS] * len(states)
    if outs is None:
        outs = [torch.empty(sh, dtype=torch.float32, device=dev) for sh in shapes]
    arr = (NsDesc * len(states))()
    sts = (_lib.Nvfp4State * len(states))()
    for i, (st, o, sh) in enumerate(zip(states, outs, shapes)):
        a, b, c = coeffs[i]
        arr[i] = NsDesc(None, o.data_ptr(), sh[0], sh[1], sh[1], _ld(o), a, b, c)
        sts[i] = _lib.Nvfp4State(st[0].data_ptr(), st[1].data_ptr(), st[2].data_ptr(), int(st[3]))
    need = int(_lib.lib().fs4_root_ns_batched_workspace_size(len(states), arr))
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    flags |= (FS4_NS_RHT if rht_masks is not None else 0) | (FS4_NS_ADAPTIVE46 if adaptive46 else 0)
    masks = _masks(rht_masks, K)
    check(_lib.lib().fs4_root_ns_batched_nvfp4(len(states), arr, sts, K, clip_k, flags,
                                               ctypes.cast(masks, ctypes.c_void_p) if masks else None,
                                               workspace.data_ptr(), workspace.numel(),
                                               _stream(stream)),
          "fs4_root_ns_batched_nvfp4")
    return outs


def root_ns_bf16_batched(Gs: Sequence[torch.Tensor], K: int = 5, coeffs=None, clip_k: float = 3.0,
                         outs: Sequence[torch.Tensor] | None = None,
                         workspace: torch.Tensor | None = None, flags: int = 0, stream=None,
                         clip_quantile: float | None = None):
    """The BF16 comparison step (fs4_root_ns_bf16_batched): the same Newton-Schulz
    iteration with BF16 operands on the tensor cores instead of NVFP4.  Arguments as
    root_ns_batched (no quantiser options)."""
    if clip_quantile is not None:
        flags |= FS4_NS_CLIP_QUANTILE
        clip_k = clip_quantile
    for G in Gs:
        _check_f32_matrix(G, "G")
    if coeffs is None:
        coeffs = [MUON_COEFFS] * len(Gs)
    if outs is None:
        outs = [torch.empty_like(G) for G in Gs]
    arr = _descs(Gs, outs, coeffs)
    need = int(_lib.lib().fs4_root_ns_bf16_batched_workspace_size(len(Gs), arr))
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=Gs[0].device)
    check(_lib.lib().fs4_root_ns_bf16_batched(len(Gs), arr, K, clip_k, flags, workspace.data_ptr(),
                                              workspace.numel(), _stream(stream)),
          "fs4_root_ns_bf16_batched")
    return outs


def ns_bf16_batched_workspace_size(shapes: Sequence[tuple[int, int]]) -> int:
    return int(_lib.lib().fs4_root_ns_bf16_batched_workspace_size(len(shapes), _shape_descs(shapes)))


def ns_bf16_layout(shapes: Sequence[tuple[int, int]], index: int = 0) -> NsLayout:
    """Workspace offsets of matrix `index` of a BF16 step on matrices of these shapes."""
    arr = _shape_descs(shapes)
    lay = NsLayout()
    check(_lib.lib().fs4_root_ns_bf16_layout(len(shapes), arr, index, ctypes.byref(lay)),
          "fs4_root_ns_bf16_layout")
    return lay


def ns_layout(shapes: Sequence[tuple[int, int]], index: int = 0) -> NsLayout:
    """Offsets of the internal tensors of matrix `index` (of a batched call on
    matrices of these shapes) in the workspace."""
    arr = _shape_descs(shapes)
    lay = NsLayout()
    check(_lib.lib().fs4_root_ns_layout(len(shapes), arr, index, ctypes.byref(lay)),
          "fs4_root_ns_layout")
    return lay


def device_status(workspace: torch.Tensor, stream=None) -> int:
    """Synchronise and return the device status word of the last call (0 = FS4_OK)."""
    return int(_lib.lib().fs4_device_status(workspace.data_ptr(), _stream(stream)))


GEMM_SOURCES = ("gemm.cu", "fs4_device.cuh", "fs4_internal.h")
ELEMENTWISE_SOURCES = ("kernels.cu", "fs4_device.cuh", "fs4_internal.h")


def _source_digest(files=GEMM_SOURCES) -> str:
    """Short hash of the CUDA sources that define a kernel (ties stored ncu counters
    to the code they measured)."""
    import hashlib
    import os
    csrc = os.path.join(os.path.dirname(os.path.abspath(__file__)), "csrc")
    h = hashlib.sha256()
    for name in sorted(files):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]

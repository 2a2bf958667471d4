"""ctypes declarations of the C ABI in include/fs4.h.

Loading fails loudly (ImportError) when libfs4.so has not been built: there is
no fallback implementation of any step.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "lib", "libfs4.so")

c_i32, c_i64, c_u32, c_f32, c_sz, c_vp = (ctypes.c_int32, ctypes.c_int64, ctypes.c_uint32,
                                          ctypes.c_float, ctypes.c_size_t, ctypes.c_void_p)

FS4_OK = 0
STATUS_NAMES = {
    0: "FS4_OK", -1: "FS4_ERR_INVALID_ARG", -2: "FS4_ERR_SHAPE", -3: "FS4_ERR_ALIAS",
    -4: "FS4_ERR_WORKSPACE", -5: "FS4_ERR_ARCH", -6: "FS4_ERR_CUDA", -7: "FS4_ERR_NONFINITE",
    -8: "FS4_ERR_TIMEOUT",
}
FS4_AXIS_ROW, FS4_AXIS_COL = 0, 1
FS4_SG_AMAX, FS4_LAYOUT_TILED = 1, 2
FS4_TEST_STALL = 1 << 30   # test only: a device wait that runs out (see include/fs4.h)
FS4_NS_RHT, FS4_NS_ADAPTIVE46, FS4_NS_CLIP_QUANTILE = 1 << 2, 1 << 3, 1 << 4
MAX_BATCH = 224
MAX_ITERS = 32


def stop_after(phase: int) -> int:
    """Flag bits of FS4_STOP_AFTER(phase)."""
    return ((phase + 1) & 0xFF) << 8


class NsDesc(ctypes.Structure):
    _fields_ = [("G", c_vp), ("out", c_vp), ("m", c_i64), ("n", c_i64), ("ld", c_i64),
                ("ld_out", c_i64), ("a", c_f32), ("b", c_f32), ("c", c_f32)]


class Nvfp4State(ctypes.Structure):
    _fields_ = [("codes", c_vp), ("scales", c_vp), ("s_g", c_vp), ("mask", c_u32)]


class QuantDesc(ctypes.Structure):
    _fields_ = [("x", c_vp), ("rows", c_i64), ("cols", c_i64), ("ld", c_i64), ("axis", c_i32),
                ("codes", c_vp), ("scales", c_vp), ("s_g", c_vp)]


class NsLayout(ctypes.Structure):
    _fields_ = [("mp", c_i64), ("np", c_i64), ("X", c_i64), ("A", c_i64),
                ("qX_codes", c_i64 * 2), ("qX_scales", c_i64 * 2),
                ("qXT_codes", c_i64 * 2), ("qXT_scales", c_i64 * 2),
                ("qA_codes", c_i64), ("qA_scales", c_i64), ("qB_codes", c_i64),
                ("qB_scales", c_i64), ("scalars", c_i64)]


# name -> (restype, argtypes); the order follows include/fs4.h
SIGNATURES = {
    "fs4_nvfp4_quantize_workspace_size": (c_sz, []),
    "fs4_momentum_workspace_size": (c_sz, []),
    "fs4_momentum_nvfp4": (c_i32, [c_vp, c_i64, c_i64, c_i64, c_f32, c_vp, c_vp, c_vp, c_u32,
                                   c_vp, c_vp, c_vp, c_u32, ctypes.c_uint64, c_vp, c_i64, c_vp,
                                   c_sz, c_vp]),
    "fs4_nvfp4_quantize": (c_i32, [c_vp, c_i64, c_i64, c_i64, c_i32, c_vp, c_vp, c_vp, c_u32,
                                   c_vp, c_sz, c_vp]),
    "fs4_nvfp4_quantize_batched_workspace_size": (c_sz, [c_i32]),
    "fs4_nvfp4_quantize_batched": (c_i32, [c_i32, ctypes.POINTER(QuantDesc), c_u32, c_vp, c_sz, c_vp]),
    "fs4_nvfp4_dequantize": (c_i32, [c_vp, c_vp, c_vp, c_i64, c_i64, c_vp, c_i64, c_u32, c_vp]),
    "fs4_nvfp4_gemm": (c_i32, [c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_i64, c_i64, c_i64, c_vp,
                               c_i64, c_vp, c_sz, c_vp]),
    "fs4_root_ns_workspace_size": (c_sz, [c_i64, c_i64]),
    "fs4_root_ns_batched_workspace_size": (c_sz, [c_i32, ctypes.POINTER(NsDesc)]),
    "fs4_root_ns": (c_i32, [c_vp, c_i64, c_i64, c_i64, c_vp, c_i64, c_i32, c_f32, c_f32, c_f32,
                            c_f32, c_u32, c_vp, c_sz, c_vp]),
    "fs4_root_ns_batched": (c_i32, [c_i32, ctypes.POINTER(NsDesc), c_i32, c_f32, c_u32, c_vp,
                                    c_sz, c_vp]),
    "fs4_root_ns_batched_ex": (c_i32, [c_i32, ctypes.POINTER(NsDesc), c_i32, c_f32, c_u32, c_vp,
                                       c_vp, c_sz, c_vp]),
    "fs4_root_ns_batched_nvfp4": (c_i32, [c_i32, ctypes.POINTER(NsDesc), ctypes.POINTER(Nvfp4State),
                                          c_i32, c_f32, c_u32, c_vp, c_vp, c_sz, c_vp]),
    "fs4_root_ns_batched_nvfp4_timed": (c_i32, [c_i32, ctypes.POINTER(NsDesc), ctypes.POINTER(Nvfp4State),
                                                c_i32, c_f32, c_u32, c_vp, c_vp, c_sz, c_vp,
                                                ctypes.POINTER(c_vp), c_i32]),
    "fs4_root_ns_batched_timed": (c_i32, [c_i32, ctypes.POINTER(NsDesc), c_i32, c_f32, c_u32,
                                          c_vp, c_vp, c_sz, c_vp, ctypes.POINTER(c_vp), c_i32]),
    "fs4_root_ns_bf16_batched_workspace_size": (c_sz, [c_i32, ctypes.POINTER(NsDesc)]),
    "fs4_root_ns_bf16_batched": (c_i32, [c_i32, ctypes.POINTER(NsDesc), c_i32, c_f32, c_u32, c_vp,
                                         c_sz, c_vp]),
    "fs4_root_ns_bf16_batched_timed": (c_i32, [c_i32, ctypes.POINTER(NsDesc), c_i32, c_f32, c_u32,
                                               c_vp, c_sz, c_vp, ctypes.POINTER(c_vp), c_i32]),
    "fs4_root_ns_noalloc": (c_i32, [c_vp, c_i64, c_i64, c_i64, c_vp, c_i64, c_i32, c_f32, c_f32,
                                    c_f32, c_f32, c_vp]),
    "fs4_device_status": (c_i32, [c_vp, c_vp]),
    "fs4_status_string": (ctypes.c_char_p, [c_i32]),
    "fs4_root_ns_layout": (c_i32, [c_i32, ctypes.POINTER(NsDesc), c_i32, ctypes.POINTER(NsLayout)]),
    "fs4_root_ns_bf16_layout": (c_i32, [c_i32, ctypes.POINTER(NsDesc), c_i32,
                                        ctypes.POINTER(NsLayout)]),
}

_lib = None


def lib() -> ctypes.CDLL:
    """The loaded libfs4 (raises ImportError if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libfs4.so not found at {LIB_PATH}; run "
                              "`python -m nvfp4_precision_optimizer_b200.build` first")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


class Fs4Error(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS_NAMES.get(status, status)}")


def check(status: int, what: str) -> None:
    if status != FS4_OK:
        raise Fs4Error(status, what)

"""ctypes binding of the C++ oracle (oracle/cpp/fs4_oracle.cpp).

TEST INFRASTRUCTURE ONLY: loaded by the tests, by the smoke check and by the
CPU-baseline / reference legs of bench.py; never by the product path.

The C++ oracle is the plain, slow restatement of the direct NVFP4 Newton-Schulz
step ("Full-Stack FP4", arXiv 2607.04422, Section 3.4): no BLAS, float64 triple
loops over dequantised operands, nearest-value searches over the code tables,
OpenMP over independent rows.  `build()` compiles it with g++ (no fast-math, no
floating-point contraction); `lib()` builds it on first use if it is missing.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "cpp", "fs4_oracle.cpp")
LIB_PATH = os.path.join(HERE, "cpp", "libfs4_oracle.so")

_lib = None
_c = ctypes
_fp = _c.POINTER(_c.c_float)
_dp = _c.POINTER(_c.c_double)
_up = _c.POINTER(_c.c_uint8)
_u16p = _c.POINTER(_c.c_uint16)
_u64p = _c.POINTER(_c.c_uint64)

AMAX_MODE = 1      # quantiser flags of the C ABI: s_g = amax / denom
ADAPTIVE46 = 2     #                               adaptive 4/6 blocks


def build(force: bool = False) -> str:
    """Compile the oracle into oracle/cpp/libfs4_oracle.so (skipped when up to date)."""
    if (not force and os.path.exists(LIB_PATH)
            and os.path.getmtime(LIB_PATH) >= os.path.getmtime(SRC)):
        return LIB_PATH
    cmd = ["g++", "-std=c++17", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
           "-fPIC", "-shared", "-o", LIB_PATH + ".tmp", SRC]
    subprocess.run(cmd, check=True)
    os.replace(LIB_PATH + ".tmp", LIB_PATH)
    return LIB_PATH


def lib():
    global _lib
    if _lib is None:
        build()
        L = _c.CDLL(LIB_PATH)
        L.fs4o_threads.restype = _c.c_int
        L.fs4o_e2m1_value.restype = _c.c_double
        L.fs4o_e2m1_value.argtypes = [_c.c_int]
        L.fs4o_e4m3_value.restype = _c.c_double
        L.fs4o_e4m3_value.argtypes = [_c.c_int]
        L.fs4o_e2m1_encode.restype = _c.c_int
        L.fs4o_e2m1_encode.argtypes = [_c.c_double]
        L.fs4o_e4m3_encode.restype = _c.c_int
        L.fs4o_e4m3_encode.argtypes = [_c.c_double]
        L.fs4o_tensor_scale.restype = _c.c_float
        L.fs4o_tensor_scale.argtypes = [_c.c_float, _c.c_int]
        L.fs4o_quantize_rows.restype = _c.c_int
        L.fs4o_quantize_rows.argtypes = [_fp, _c.c_int64, _c.c_int64, _c.c_float, _c.c_int, _up, _up,
                                         _fp, _c.c_int]
        L.fs4o_dequantize_rows.restype = _c.c_int
        L.fs4o_dequantize_rows.argtypes = [_up, _up, _c.c_float, _c.c_int64, _c.c_int64, _dp, _c.c_int]
        L.fs4o_product.restype = _c.c_int
        L.fs4o_product.argtypes = [_dp, _dp, _c.c_int64, _c.c_int64, _c.c_int64, _dp, _c.c_int]
        L.fs4o_hadamard_rows.restype = _c.c_int
        L.fs4o_hadamard_rows.argtypes = [_fp, _c.c_int64, _c.c_int64, _c.c_int, _fp]
        L.fs4o_normalise_and_clip.restype = _c.c_double
        L.fs4o_normalise_and_clip.argtypes = [_fp, _c.c_int64, _c.c_int64, _c.c_double, _c.c_double,
                                              _fp, _fp, _fp]
        L.fs4o_ns_iterations_nvfp4.restype = _c.c_int
        L.fs4o_ns_iterations_nvfp4.argtypes = [_fp, _c.c_int64, _c.c_int64, _c.c_int, _c.c_double,
                                               _c.c_double, _c.c_double, _u16p, _c.c_int, _c.c_int]
        L.fs4o_bf16_round.restype = None
        L.fs4o_bf16_round.argtypes = [_fp, _c.c_int64, _fp]
        L.fs4o_ns_iterations_bf16.restype = _c.c_int
        L.fs4o_ns_iterations_bf16.argtypes = [_fp, _c.c_int64, _c.c_int64, _c.c_int, _c.c_double,
                                              _c.c_double, _c.c_double, _c.c_int]
        L.fs4o_splitmix64.restype = None
        L.fs4o_splitmix64.argtypes = [_c.c_uint64, _u64p, _c.c_int64, _u64p]
        L.fs4o_uniform24.restype = None
        L.fs4o_uniform24.argtypes = [_c.c_uint64, _u64p, _c.c_int64, _fp]
        L.fs4o_e2m1_encode_sr.restype = _c.c_int
        L.fs4o_e2m1_encode_sr.argtypes = [_c.c_float, _c.c_float]
        L.fs4o_momentum_update.restype = _c.c_int
        L.fs4o_momentum_update.argtypes = [_fp, _c.c_int64, _c.c_int64, _c.c_double, _up, _up, _c.c_float,
                                           _c.c_int, _c.c_int, _c.c_uint64, _fp, _up, _up, _fp, _c.c_int]
        L.fs4o_momentum_load.restype = _c.c_int
        L.fs4o_momentum_load.argtypes = [_up, _up, _c.c_float, _c.c_int, _c.c_int64, _c.c_int64, _fp]
        L.fs4o_root_ns.restype = _c.c_int
        L.fs4o_root_ns.argtypes = [_fp, _c.c_int64, _c.c_int64, _c.c_int, _c.c_double, _c.c_double,
                                   _c.c_double, _c.c_double, _c.c_double, _c.c_int, _u16p, _c.c_int,
                                   _fp, _dp, _c.c_int]
        _lib = L
    return _lib


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


def _ptr(a, t):
    return a.ctypes.data_as(t)


def threads() -> int:
    return int(lib().fs4o_threads())


def _flags(mode, adaptive46):
    if mode not in ("pow2", "amax"):
        raise ValueError(f"unknown tensor-scale mode {mode!r}")
    return (AMAX_MODE if mode == "amax" else 0) | (ADAPTIVE46 if adaptive46 else 0)


def _masks(rht_masks, K):
    """The 3K sign masks of H16^r as a uint16 array (None: H = I)."""
    if rht_masks is None:
        return None
    m = np.ascontiguousarray([int(v) for v in rht_masks], dtype=np.int64)
    if m.size < 3 * K or np.any(m < 0) or np.any(m > 0xFFFF):
        raise ValueError("rht_masks needs 3K masks in 0 .. 0xFFFF")
    return m.astype(np.uint16)


def quantize_rows(x, s_g=None, mode="pow2", adaptive46=False, threads=0):
    """Q1x16 of an FP32 matrix: (codes [rows, cols/2], scales [rows, cols/16], s_g).
    The same signature and result as oracle.nvfp4.quantize_rows."""
    x = _f32(x)
    rows, cols = x.shape
    codes = np.zeros((rows, cols // 2), np.uint8)
    scales = np.zeros((rows, cols // 16), np.uint8)
    sg = np.zeros(1, np.float32)
    st = lib().fs4o_quantize_rows(_ptr(x, _fp), rows, cols, float(s_g) if s_g is not None else -1.0,
                                  _flags(mode, adaptive46), _ptr(codes, _up), _ptr(scales, _up),
                                  _ptr(sg, _fp), threads)
    if st != 0:
        raise ValueError("bad shape")
    return codes, scales, np.float32(sg[0])


def quantize_cols(x, s_g=None, mode="pow2", adaptive46=False, threads=0):
    """Q16x1, laid out as the Q1x16 of x^T."""
    return quantize_rows(np.ascontiguousarray(np.asarray(x, np.float32).T), s_g, mode, adaptive46,
                         threads)


def dequantize_rows(codes, scales, s_g, threads=0):
    codes = np.ascontiguousarray(codes, np.uint8)
    scales = np.ascontiguousarray(scales, np.uint8)
    rows, cols = codes.shape[0], codes.shape[1] * 2
    out = np.zeros((rows, cols), np.float64)
    if lib().fs4o_dequantize_rows(_ptr(codes, _up), _ptr(scales, _up), float(s_g), rows, cols,
                                  _ptr(out, _dp), threads) != 0:
        raise ValueError("bad shape")
    return out


def dequantize_cols(codes, scales, s_g, threads=0):
    """Inverse of quantize_cols: the rows x cols matrix (float64, exact)."""
    return dequantize_rows(codes, scales, s_g, threads).T


def product(L, R, threads=0):
    L = np.ascontiguousarray(L, np.float64)
    R = np.ascontiguousarray(R, np.float64)
    out = np.zeros((L.shape[0], R.shape[1]), np.float64)
    if lib().fs4o_product(_ptr(L, _dp), _ptr(R, _dp), L.shape[0], L.shape[1], R.shape[1],
                          _ptr(out, _dp), threads) != 0:
        raise ValueError("bad shape")
    return out


def hadamard_rows(x, mask):
    """FP32 x H16^r on every 16-element block of each row (oracle.nvfp4.hadamard_rows)."""
    x = _f32(x)
    y = np.zeros_like(x)
    if lib().fs4o_hadamard_rows(_ptr(x, _fp), x.shape[0], x.shape[1], int(mask), _ptr(y, _fp)) != 0:
        raise ValueError("bad shape or mask")
    return y


def hadamard_cols(x, mask):
    """FP32 (H16^r)^T x on every 16-element block of each column."""
    return np.ascontiguousarray(hadamard_rows(np.ascontiguousarray(np.asarray(x, np.float32).T), mask).T)


def normalise_and_clip(G, clip_k, clip_quantile=None):
    """(X0, inv, tau, norm) of an FP32 matrix already in working orientation;
    clip_quantile = q replaces the clip_k * RMS threshold by the q-quantile of |X0|."""
    G = _f32(G)
    X0 = np.zeros_like(G)
    inv = np.zeros(1, np.float32)
    tau = np.zeros(1, np.float32)
    q = float(clip_quantile) if clip_quantile is not None else 0.0
    norm = lib().fs4o_normalise_and_clip(_ptr(G, _fp), G.shape[0], G.shape[1],
                                         float(clip_k) if clip_k else 0.0, q, _ptr(X0, _fp),
                                         _ptr(inv, _fp), _ptr(tau, _fp))
    clipped = clip_quantile is not None or bool(clip_k)
    return X0, np.float32(inv[0]), (np.float32(tau[0]) if clipped else None), float(norm)


def ns_iterations_nvfp4(X0, K, a, b, c, mode="pow2", rht_masks=None, adaptive46=False, threads=0):
    """K NVFP4 iterations (oracle.root_ns.ns_iterations_nvfp4 with the same options)."""
    X = _f32(X0).copy()
    masks = _masks(rht_masks, K)
    mp = _ptr(masks, _u16p) if masks is not None else None
    if lib().fs4o_ns_iterations_nvfp4(_ptr(X, _fp), X.shape[0], X.shape[1], int(K), float(a), float(b),
                                      float(c), mp, _flags(mode, adaptive46), threads) != 0:
        raise ValueError("bad shape")
    return X


def root_ns(G, K=5, a=3.4445, b=-4.7750, c=2.0315, clip_k=3.0, quantized=True, mode="pow2",
            rht_masks=None, adaptive46=False, clip_quantile=None, bf16=False, threads=0):
    """The whole step (normalise, clip, K iterations) on an FP32 matrix of any orientation,
    with the options of oracle.root_ns.root_ns (bf16=True: the BF16 route)."""
    G = _f32(G)
    out32 = np.zeros(G.shape, np.float32)
    out64 = np.zeros(G.shape, np.float64)
    masks = _masks(rht_masks, K) if quantized and not bf16 else None
    mp = _ptr(masks, _u16p) if masks is not None else None
    route = (2 if bf16 else 1) if quantized else 0
    st = lib().fs4o_root_ns(_ptr(G, _fp), G.shape[0], G.shape[1], int(K), float(a), float(b), float(c),
                            float(clip_k) if clip_k else 0.0,
                            float(clip_quantile) if clip_quantile is not None else 0.0,
                            route, mp, _flags(mode, adaptive46), _ptr(out32, _fp),
                            _ptr(out64, _dp), threads)
    if st != 0:
        raise ValueError("bad shape or non-finite input")
    return out32 if quantized else out64


def bf16_round(x):
    """FP32 -> BF16 (round to nearest, ties to even) as FP32 values (oracle.root_ns.bf16_round)."""
    x = _f32(x)
    y = np.zeros_like(x)
    lib().fs4o_bf16_round(_ptr(x, _fp), x.size, _ptr(y, _fp))
    return y


def ns_iterations_bf16(X0, K, a, b, c, threads=0):
    """K BF16 iterations (oracle.root_ns.ns_iterations_bf16)."""
    X = _f32(X0).copy()
    if lib().fs4o_ns_iterations_bf16(_ptr(X, _fp), X.shape[0], X.shape[1], int(K), float(a), float(b),
                                     float(c), threads) != 0:
        raise ValueError("bad shape")
    return X


def splitmix64(seed, idx):
    idx = np.ascontiguousarray(idx, dtype=np.uint64)
    out = np.zeros(idx.shape, np.uint64)
    lib().fs4o_splitmix64(int(seed) & (2 ** 64 - 1), _ptr(idx, _u64p), idx.size, _ptr(out, _u64p))
    return out


def uniform24(seed, idx):
    idx = np.ascontiguousarray(idx, dtype=np.uint64)
    out = np.zeros(idx.shape, np.float32)
    lib().fs4o_uniform24(int(seed) & (2 ** 64 - 1), _ptr(idx, _u64p), idx.size, _ptr(out, _fp))
    return out


def sr_encode_magnitude(v, u):
    """Stochastic rounding of FP32 v >= 0 onto E2M1 codes 0..7 (oracle.momentum.sr_encode_magnitude)."""
    v = np.asarray(v, np.float32).ravel()
    u = np.asarray(u, np.float32).ravel()
    if not np.all(np.isfinite(v)) or np.any(v < 0):
        raise ValueError("SR encode expects finite non-negative inputs")
    return np.array([lib().fs4o_e2m1_encode_sr(float(a), float(b)) for a, b in zip(v, u)], np.uint8)


def momentum_update(g, beta, state=None, mask_prev=0, mask_next=0, seed=0, threads=0):
    """One NVFP4 first-moment step (oracle.momentum.update): (m_t, (codes, scales, s_g))."""
    g = _f32(g)
    rows, cols = g.shape
    m_t = np.zeros_like(g)
    codes = np.zeros((rows, cols // 2), np.uint8)
    scales = np.zeros((rows, cols // 16), np.uint8)
    sg = np.zeros(1, np.float32)
    if state is None:
        pc = ps = None
        psg = 0.0
    else:
        pcodes = np.ascontiguousarray(state[0], np.uint8)
        pscales = np.ascontiguousarray(state[1], np.uint8)
        pc, ps, psg = _ptr(pcodes, _up), _ptr(pscales, _up), float(state[2])
    if lib().fs4o_momentum_update(_ptr(g, _fp), rows, cols, float(beta), pc, ps, psg, int(mask_prev),
                                  int(mask_next), int(seed) & (2 ** 64 - 1), _ptr(m_t, _fp),
                                  _ptr(codes, _up), _ptr(scales, _up), _ptr(sg, _fp), threads) != 0:
        raise ValueError("bad shape or mask")
    return m_t, (codes, scales, np.float32(sg[0]))


def momentum_load(codes, scales, s_g, mask):
    """FP32 momentum decoded from a state (oracle.momentum.load)."""
    codes = np.ascontiguousarray(codes, np.uint8)
    scales = np.ascontiguousarray(scales, np.uint8)
    rows, cols = codes.shape[0], codes.shape[1] * 2
    out = np.zeros((rows, cols), np.float32)
    if lib().fs4o_momentum_load(_ptr(codes, _up), _ptr(scales, _up), float(s_g), int(mask), rows, cols,
                                _ptr(out, _fp)) != 0:
        raise ValueError("bad shape or mask")
    return out

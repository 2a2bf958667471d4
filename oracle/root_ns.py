"""Direct NVFP4 Newton-Schulz orthogonalisation (Q-Root), step by step.

TEST INFRASTRUCTURE ONLY: imported by tests, by the smoke check and by the
CPU-baseline leg of bench.py; never by the product path.

Source: "Full-Stack FP4" (arXiv 2607.04422).
  * Section 2, paragraph "Root optimizer": X_{k+1} = a X_k + b X_k (X_k^T X_k)
    + c X_k (X_k^T X_k)^2, typically 5 iterations.  Written in the Gram-left
    form used by Section 3.4, X (X^T X) = (X X^T) X, the Gram matrix is m x m
    on the short side when X is m x n with m <= n.
  * Section 3.4 "NVFP4 Root Optimizer", the iteration (by default with the
    random Hadamard transform taken as the identity and plain M = 6 block
    scaling; rht_masks / adaptive46 select the transform and the adaptive 4/6
    scaling the section also names):
        qX_k  = Q1x16(X_k),            A_k = qX_k qX_k^T
        qA_k  = Q1x16(A_k),  qA16_k = Q16x1(A_k),  B_k = b A_k + c qA_k qA16_k
        qB_k  = Q1x16(B_k),  qX16_k = Q16x1(X_k),  X_{k+1} = a X_k + qB_k qX16_k
  * Section 3.4 also clips outliers before the iteration ("p99 outlier clipping";
    Table 8: "Root quantile ratio 0.99").  Two clip rules are provided: a hard
    clamp at clip_k * RMS of the normalised matrix (the default), and a hard clamp
    at the q-quantile of |X_0| (clip_quantile = q).

Readings taken where the pages are silent:
  * Frobenius normalisation X_0 = G / (||G||_F + eps), eps = 1e-7, ||G||_F
    accumulated in float64; inv = fp32(1 / (||G||_F + eps)) and X_0 = fp32(G * inv).
  * Clip: tau = fp32(clip_k * ||G||_F * inv / sqrt(m n)), X_0 = clamp(X_0, -tau, tau).
  * Quantile clip: tau = the nearest-rank q-quantile of |X_0|, i.e. its k-th smallest
    entry with k = ceil(fl64(q) * N) (1-based, clamped to [1, N]; N = m n; q is the
    FP32 value the caller passes and the product is one IEEE float64 multiply), then
    X_0 = clamp(X_0, -tau, tau).
  * Iterates X_k, A_k and B_k are FP32 tensors (the precision the quantiser
    reads); every matrix product is taken in float64 on dequantised operands
    and rounded once to FP32.  A_k is made exactly symmetric (upper triangle
    mirrored), as the Gram matrix is by definition.
  * A tall input (m0 > n0) is processed as its transpose and the result is
    transposed back, so the Gram matrix is always min(m0, n0) square.
"""
from __future__ import annotations

import numpy as np

from . import nvfp4
from . import nvfp4 as _nvfp4

NS_EPS = 1e-7


def quantile_rank(q: float, N: int) -> int:
    """1-based rank of the nearest-rank q-quantile of N values: ceil(fl64(q32) * N),
    clamped to [1, N] (q32 = the FP32 value of q)."""
    k = int(np.ceil(np.float64(np.float32(q)) * np.float64(N)))
    return min(max(k, 1), N)


def quantile_clip_threshold(X0: np.ndarray, q: float) -> np.float32:
    """The nearest-rank q-quantile of |X0| (Section 3.4 "p99 outlier clipping", Table 8
    "Root quantile ratio 0.99"): its k-th smallest entry, k = quantile_rank(q, N)."""
    a = np.abs(np.asarray(X0, dtype=np.float32)).ravel()
    k = quantile_rank(q, a.size)
    return np.float32(np.partition(a, k - 1)[k - 1])


def normalise_and_clip(X: np.ndarray, clip_k: float | None, eps: float = NS_EPS,
                       clip_quantile: float | None = None):
    """FP32 X_0 = clamp(fp32(X * inv), +-tau).  Returns (X0, inv, tau, norm).
    clip_quantile = q: tau is the q-quantile of |fp32(X * inv)| instead of clip_k * RMS."""
    X = np.asarray(X, dtype=np.float32)
    m, n = X.shape
    norm = float(np.sqrt(np.sum(X.astype(np.float64) ** 2)))
    inv = np.float32(1.0 / (norm + eps))
    X0 = X * inv
    tau = None
    if clip_quantile is not None:
        tau = quantile_clip_threshold(X0, clip_quantile)
        X0 = np.clip(X0, -tau, tau).astype(np.float32)
    elif clip_k is not None and clip_k > 0:
        tau = np.float32(clip_k * norm * float(inv) / np.sqrt(float(m) * float(n)))
        X0 = np.clip(X0, -tau, tau).astype(np.float32)
    return X0, inv, tau, norm


def symmetric_from_upper(A: np.ndarray) -> np.ndarray:
    """Mirror the upper triangle (diagonal included) into the lower one."""
    return np.triu(A) + np.triu(A, 1).T


def ns_iterations_nvfp4(X0, K, a, b, c, mode="pow2", trace=None, rht_masks=None,
                        adaptive46=False, perturb=None, matmul=None, codec=None):
    """K NVFP4 Newton-Schulz iterations (Section 3.4) from the FP32 m x n X0 (m <= n).

    rht_masks: None (H = I) or 3K sign masks of H16^r (see nvfp4.hadamard_rows), one
    per product: 3k for A_k = qX_k qX_k^T, 3k + 1 for qA_k qA16_k, 3k + 2 for
    qB_k qX16_k.  adaptive46: adaptive 4/6 block scaling in every quantisation.
    perturb: None, or a function (k, name, T) -> T' applied to each FP32 tensor
    ("A", "B", "X") right after it is formed; it lets a test study how the iteration
    responds to other, equally valid FP32 roundings of the same values.  matmul: None
    (float64 products), or a function (L, R) -> L R used for the three products
    instead, e.g. one accumulating in FP32.  None for both leaves the arithmetic
    above untouched.  codec: None (this package's numpy codec, oracle.nvfp4) or
    another module with the same quantize_rows / quantize_cols / dequantize_rows /
    dequantize_cols, such as oracle.cpp_oracle (bit-identical, much faster on
    large matrices).
    """
    nvfp4 = _nvfp4 if codec is None else codec
    pert = (lambda k, name, t: t) if perturb is None else perturb
    mm = (lambda l, r: l @ r) if matmul is None else matmul
    X = np.asarray(X0, dtype=np.float32)
    hr = (lambda t, j: t) if rht_masks is None else (lambda t, j: _nvfp4.hadamard_rows(t, rht_masks[j]))
    hc = (lambda t, j: t) if rht_masks is None else (lambda t, j: _nvfp4.hadamard_cols(t, rht_masks[j]))
    a46 = adaptive46
    for k in range(K):
        # qX_k = Q1x16(X_k H); qX16_k = Q16x1(H'^T X_k) (held as the 1x16 quantisation of
        # its transpose); H belongs to the Gram product, H' to the update product
        qx, sx, gx = nvfp4.quantize_rows(hr(X, 3 * k), mode=mode, adaptive46=a46)
        qxt, sxt, gxt = nvfp4.quantize_cols(hc(X, 3 * k + 2), mode=mode, adaptive46=a46)
        dX = nvfp4.dequantize_rows(qx, sx, gx)                     # m x n
        dX16 = nvfp4.dequantize_cols(qxt, sxt, gxt)                # m x n, 16x1 blocks
        # A_k = qX_k qX_k^T
        A = pert(k, "A", symmetric_from_upper(mm(dX, dX.T)).astype(np.float32))
        # qA_k = Q1x16(A_k H), qA16_k = Q16x1(H^T A_k), B_k = b A_k + c qA_k qA16_k
        qa, sa, ga = nvfp4.quantize_rows(hr(A, 3 * k + 1), mode=mode, adaptive46=a46)
        qa16, sa16, ga16 = nvfp4.quantize_cols(hc(A, 3 * k + 1), mode=mode, adaptive46=a46)
        P = mm(nvfp4.dequantize_rows(qa, sa, ga), nvfp4.dequantize_cols(qa16, sa16, ga16))
        B = pert(k, "B", (b * A.astype(np.float64) + c * P).astype(np.float32))
        # qB_k = Q1x16(B_k H'), X_{k+1} = a X_k + qB_k qX16_k
        qb, sb, gb = nvfp4.quantize_rows(hr(B, 3 * k + 2), mode=mode, adaptive46=a46)
        Xn = (a * X.astype(np.float64) + mm(nvfp4.dequantize_rows(qb, sb, gb), dX16)).astype(np.float32)
        Xn = pert(k, "X", Xn)
        if trace is not None:
            trace.append(dict(X=X, qX=(qx, sx, gx), qXT=(qxt, sxt, gxt), A=A,
                              qA=(qa, sa, ga), P=P, B=B, qB=(qb, sb, gb), X_next=Xn))
        X = Xn
    return X


def bf16_round(x) -> np.ndarray:
    """FP32 -> BF16 by round-to-nearest, ties to even, returned as the FP32 numbers
    those BF16 values are.  BF16 keeps the sign, the 8 exponent bits and the top 7
    mantissa bits of an FP32 number: the lower 16 bits are rounded away.  Finite
    inputs only."""
    x = np.asarray(x, dtype=np.float32)
    bits = x.view(np.uint32).astype(np.uint64)
    keep = bits >> 16
    rest = bits & 0xFFFF
    up = (rest > 0x8000) | ((rest == 0x8000) & ((keep & 1) == 1))
    return ((keep + up.astype(np.uint64)) << 16).astype(np.uint32).view(np.float32)


def ns_iterations_bf16(X0, K, a, b, c, trace=None, matmul=None):
    """K Newton-Schulz iterations with BF16 operands (the optimized BF16 baseline the
    pages compare Q-Root against, Section 4.4 and Table 6), from the FP32 m x n X0
    (m <= n).  Same plan as the NVFP4 route with bf16() in place of each
    quantisation: Xb = bf16(X), A = Xb Xb^T, B = b A + c bf16(A) bf16(A)^T,
    X_{k+1} = a X + bf16(B) Xb.  Products in float64 on the BF16 values, rounded once
    to FP32; A made exactly symmetric from its upper triangle; X, A, B FP32.
    matmul: None (float64 products), or a function (L, R) -> L R used for the three
    products instead (as in ns_iterations_nvfp4)."""
    mm = (lambda l, r: l @ r) if matmul is None else matmul
    X = np.asarray(X0, dtype=np.float32)
    for _ in range(K):
        Xb = bf16_round(X).astype(np.float64)
        A = symmetric_from_upper(mm(Xb, Xb.T)).astype(np.float32)
        Ab = bf16_round(A).astype(np.float64)
        P = mm(Ab, Ab.T)
        B = (b * A.astype(np.float64) + c * P).astype(np.float32)
        Bb = bf16_round(B).astype(np.float64)
        Xn = (a * X.astype(np.float64) + mm(Bb, Xb)).astype(np.float32)
        if trace is not None:
            trace.append(dict(X=X, A=A, P=P, B=B, X_next=Xn))
        X = Xn
    return X


def ns_iterations_f64(X0, K, a, b, c):
    """K Newton-Schulz iterations in float64, no quantisation (Section 2)."""
    X = np.asarray(X0, dtype=np.float64)
    for _ in range(K):
        A = X @ X.T
        X = a * X + (b * A + c * (A @ A)) @ X
    return X


def root_ns(G, K=5, a=3.4445, b=-4.7750, c=2.0315, clip_k=3.0, eps=NS_EPS,
            quantized=True, mode="pow2", trace=None, rht_masks=None, adaptive46=False,
            clip_quantile=None, bf16=False):
    """Normalise, clip and run K Newton-Schulz iterations on the FP32 matrix G.

    quantized=True: the NVFP4 route of Section 3.4 (FP32 result); with bf16=True
    the same plan with BF16 operands (ns_iterations_bf16) instead.
    quantized=False: the plain float64 iteration of Section 2 (float64 result;
    normalisation and clip done in float64).
    """
    G = np.asarray(G)
    if G.ndim != 2:
        raise ValueError("G must be a matrix")
    if not np.all(np.isfinite(G)):
        raise ValueError("non-finite input")
    tall = G.shape[0] > G.shape[1]
    X = G.T if tall else G
    if quantized:
        X0, inv, tau, norm = normalise_and_clip(X.astype(np.float32), clip_k, eps,
                                                clip_quantile=clip_quantile)
        if trace is not None:
            trace.append(dict(X0=X0, inv=inv, tau=tau, norm=norm))
        if bf16:
            Y = ns_iterations_bf16(X0, K, a, b, c, trace=trace)
        else:
            Y = ns_iterations_nvfp4(X0, K, a, b, c, mode=mode, trace=trace, rht_masks=rht_masks,
                                    adaptive46=adaptive46)
    else:
        X64 = np.asarray(X, dtype=np.float64)
        norm = float(np.sqrt(np.sum(X64 ** 2)))
        X0 = X64 / (norm + eps)
        if clip_quantile is not None:
            mag = np.abs(X0).ravel()
            k = quantile_rank(clip_quantile, mag.size)
            tau = np.partition(mag, k - 1)[k - 1]
            X0 = np.clip(X0, -tau, tau)
        elif clip_k is not None and clip_k > 0:
            tau = clip_k * np.sqrt(np.sum(X0 ** 2)) / np.sqrt(X0.size)
            X0 = np.clip(X0, -tau, tau)
        Y = ns_iterations_f64(X0, K, a, b, c)
    return np.ascontiguousarray(Y.T if tall else Y)


def orthogonality_error(X) -> float:
    """||X X^T - I||_F / sqrt(m) for m x n X (m <= n, else X^T)."""
    X = np.asarray(X, dtype=np.float64)
    if X.shape[0] > X.shape[1]:
        X = X.T
    m = X.shape[0]
    return float(np.linalg.norm(X @ X.T - np.eye(m)) / np.sqrt(m))

"""CPU oracle for the direct NVFP4 Newton-Schulz step (test infrastructure only).

This package is the slow, plainly written reference that the CUDA path is
checked against.  It is TEST INFRASTRUCTURE: only the test-suite, the smoke
check of ``__graft_entry__`` and the CPU-baseline leg of ``bench.py`` may
import it.  The product path (``nvfp4_precision_optimizer_b200``) never calls
into it and shares no code, tables or helpers with it.

Source of the method: "Full-Stack FP4: Stable LLM Pretraining with Quantized
Projections, Optimizers, and Attention" (arXiv 2607.04422):
  * Section 2 "Preliminaries", paragraph "NVFP4 format": E2M1 values in 1x16
    blocks, one FP8 E4M3 scale per block, one FP32 tensor scale s_g, and
    x_hat = x_E2M1 * s * s_g.
  * Section 2, paragraph "Root optimizer": the Newton-Schulz polynomial
    X_{k+1} = a X_k + b X_k (X_k^T X_k) + c X_k (X_k^T X_k)^2.
  * Section 3.4 "NVFP4 Root Optimizer": the NVFP4 iteration
    A = qX qX^T, B = b A + c qA qA^{16x1}, X_{k+1} = a X_k + qB qX^{16x1},
    with round-to-nearest quantisation.

Modules:
  * ``oracle.nvfp4``   -- E2M1/E4M3 codecs, tensor scale, 1x16 quantise and
                          dequantise (numpy, exact emulation).
  * ``oracle.root_ns`` -- normalise + clip + K NVFP4 Newton-Schulz iterations,
                          products in float64 on dequantised operands.
  * ``oracle.cpp_oracle`` -- ctypes binding of ``oracle/cpp/fs4_oracle.cpp``, the
                          same steps restated in plain C++17 (OpenMP over rows,
                          float64 triple loops, no BLAS), options included
                          (H16^r, adaptive 4/6, quantile clip), with the BF16
                          route and the NVFP4 first moment; a second,
                          independent implementation, and the one the CPU
                          baseline times.
"""

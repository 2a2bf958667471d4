/*
 * fs4.h -- C ABI of libfs4: direct NVFP4 Newton-Schulz orthogonalisation on
 * NVIDIA B200 (sm_100a).
 *
 * The method is the "NVFP4 Root Optimizer" of "Full-Stack FP4: Stable LLM
 * Pretraining with Quantized Projections, Optimizers, and Attention"
 * (arXiv 2607.04422):
 *   - Section 2, paragraph "NVFP4 format": E2M1 values in 1x16 blocks, one
 *     FP8 E4M3 scale s per block and one FP32 tensor scale s_g, with
 *     x_hat = x_E2M1 * s * s_g.
 *   - Section 2, paragraph "Root optimizer": the Newton-Schulz polynomial
 *     X_{k+1} = a X + b X (X^T X) + c X (X^T X)^2, typically 5 iterations.
 *   - Section 3.4, "NVFP4 Root Optimizer": outlier clipping, then the
 *     iteration A = qX qX^T, B = b A + c qA qA^{16x1},
 *     X_{k+1} = a X + qB qX^{16x1}, all quantisations round to nearest.
 *
 * Conventions shared by every entry point
 *   - Pointers are DEVICE pointers unless a parameter says "host".  The caller
 *     owns every buffer, including the workspace; the library never allocates
 *     device memory and never synchronises, except fs4_device_status().
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  All work is enqueued asynchronously on it.
 *   - Matrices are row-major FP32 with a leading dimension `ld` (elements)
 *     >= the number of columns.
 *   - Argument errors are detected on the host, returned synchronously, and
 *     nothing is enqueued.  Conditions only the device can see (non-finite
 *     input, a bounded device-side wait that gave up) are recorded in a status
 *     word inside the workspace; read it with fs4_device_status().  Device
 *     code never traps.
 *   - Functions are thread-safe; the only global state is a per-device cache
 *     of the SM count and architecture check.
 *
 * NVFP4 storage
 *   - Codes: 4-bit E2M1, (sign, e1, e0, m), element 2j of a block row in the
 *     LOW nibble of byte j and element 2j+1 in the high nibble.
 *   - Scales: one E4M3 byte per 16 consecutive elements of a row.
 *   - Tensor scale: one FP32 (device) per tensor.  Default: the smallest power
 *     of two s_g with 6 * 448 * s_g >= amax (s_g = 1 for an all-zero tensor).
 *   - PLAIN layout (default): codes[r * (cols/2) + c/2], scales[r * (cols/16) + c/16].
 *   - TILED layout (FS4_LAYOUT_TILED), the tensor-core operand layout: rows
 *     padded to Rp = roundup(rows,128), columns to Cp = roundup(cols,256),
 *     padding is zero.  Codes: tile (r/128, c/256) of 16384 bytes at
 *     ((r/128)*(Cp/256) + c/256) * 16384; inside it row r%128 starts at byte
 *     128*(r%128) and its 16-byte chunk j = (c%256)/32 is stored at chunk
 *     position j ^ (r%8).  Scales: atom (r/128, c/64) of 512 bytes at
 *     ((r/128)*(Cp/64) + c/64) * 512; inside it the scale of rows r and of
 *     column block (c/16)%4 is byte 16*(r%32) + 4*((r%128)/32) + (c/16)%4.
 *     Sizes: codes Rp*Cp/2 bytes, scales Rp*Cp/16 bytes.
 */
#ifndef FS4_H
#define FS4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int32_t fs4_status;

enum {
  FS4_OK = 0,
  FS4_ERR_INVALID_ARG = -1, /* null pointer, bad leading dimension, misaligned buffer, bad flag */
  FS4_ERR_SHAPE = -2,       /* a size is zero, negative, too large, or not a multiple of 16 */
  FS4_ERR_ALIAS = -3,       /* an output overlaps an input */
  FS4_ERR_WORKSPACE = -4,   /* workspace null, misaligned (256 B) or smaller than required */
  FS4_ERR_ARCH = -5,        /* current device is not compute capability 10.0 */
  FS4_ERR_CUDA = -6,        /* a CUDA runtime call or kernel launch failed */
  FS4_ERR_NONFINITE = -7,   /* (device status) NaN or Inf in the input matrix */
  FS4_ERR_TIMEOUT = -8      /* (device status) a bounded device-side wait gave up */
};

enum { FS4_AXIS_ROW = 0, /* 1x16 blocks along each row */
       FS4_AXIS_COL = 1  /* 16x1 blocks along each column; stored as the quantisation of x^T */ };

enum {
  FS4_SG_AMAX = 1u << 0,      /* quantize only: s_g = fp32(amax / 2688) instead of a power of two */
  FS4_LAYOUT_TILED = 1u << 1  /* quantize/dequantize: codes and scales in the TILED layout */
};

/* Debug stop for fs4_root_ns / fs4_root_ns_batched: run only the phases up to
 * and including `phase` and return (the workspace then holds that state).
 * phase 0 = preamble (normalise, clip, quantise X_0); phase 1 + 3k + j is the
 * j-th product of iteration k (j = 0: A = qX qX^T, 1: P = qA qA^T and
 * B = b A + c P, 2: X_{k+1} = a X_k + qB qX^{16x1}).  Encoded in flag bits 8..15
 * as (phase + 1); 0 means run everything.  A stop right after product 1 of an
 * iteration also writes that product's B (FP32) over the upper 256 x 256 tiles
 * of A in the workspace (fs4_ns_layout.A), where B is otherwise never stored in
 * FP32; without the stop the kernels never write it. */
#define FS4_STOP_AFTER(phase) ((uint32_t)(((phase) + 1) & 0xFF) << 8)

/* Quantiser options of the Newton-Schulz step (Section 3.4: "qX_k =
 * Q1x16(X H16^r)" ... "All quantizations use RTN and adaptive 4/6 scaling").
 * Off by default: the default step quantises plainly (H = I, M = 6).
 * FS4_NS_ADAPTIVE46: every block is quantised with its amax mapped to 6 and to
 *   4 and keeps the M = 4 candidate only if its squared error (FP32, summed in
 *   element order) is strictly smaller; the tensor scale is shared.
 * FS4_NS_RHT: every quantised operand is transformed along its K dimension by
 *   H16^r = D H16 / 4 (H16 the Sylvester Hadamard matrix, D the diagonal of
 *   signs of a 16-bit mask, bit i negating element i of each 16-element block;
 *   FP32 butterfly with strides 1, 2, 4, 8, then * 0.25) before quantisation.
 *   Both operands of a product carry the same mask, so the products are those
 *   of the untransformed tensors.  Tensor scales then cover 4x the amax bound
 *   (|x H| <= 4 amax).  Only fs4_root_ns_batched_ex takes the masks. */
#define FS4_NS_ADAPTIVE46 (1u << 3)
#define FS4_NS_RHT (1u << 2)

/* Quantile clip of the Newton-Schulz step (Section 3.4: "p99 outlier clipping";
 * Table 8: "Root quantile ratio 0.99").  With this flag clip_k is the quantile
 * ratio q, 0 < q <= 1 (else FS4_ERR_INVALID_ARG), and tau is the nearest-rank
 * q-quantile of |X_0|: the k-th smallest |x| of the normalised matrix with
 * k = ceil(q * m * n) (q widened to double, one IEEE double multiply, k clamped to
 * [1, m n]).  X_0 is clamped to [-tau, tau] as with the default rule.  The
 * selection is exact (three radix digits of the 31-bit magnitude key) and adds
 * three launches after the reduction; it uses the matrix's X buffer as scratch
 * before the preamble writes X_0 there. */
#define FS4_NS_CLIP_QUANTILE (1u << 4)

/* Test-only flag for fs4_root_ns / fs4_root_ns_batched and fs4_nvfp4_quantize
 * (no counterpart in the paper).  Newton-Schulz: the MMA issuer of the first
 * Gram product waits on a barrier that nothing arrives on.  Quantise: the grid
 * barrier between the amax pass and the quantise pass waits for one CTA more
 * than the launch has.  The bounded wait gives up after about 2 s, records the
 * timeout in the status word, and the rest of the call's work is skipped;
 * fs4_device_status then returns FS4_ERR_TIMEOUT and the outputs are undefined.
 * The CUDA context stays usable: no trap, fault or unbounded wait is involved.
 * It exists so that the device-side timeout path can be exercised on a GPU. */
#define FS4_TEST_STALL (1u << 30)

/* Upper limits checked on the host. */
#define FS4_MAX_DIM 65536       /* m, n of one Newton-Schulz matrix */
#define FS4_MAX_ITERS 32        /* K */
#define FS4_MAX_BATCH 224       /* matrices per fs4_root_ns_batched call */

/* ------------------------------------------------------------------ quantise */

/* Bytes of workspace fs4_nvfp4_quantize needs (at least 256-byte aligned). */
size_t fs4_nvfp4_quantize_workspace_size(void);

/* NVFP4-quantise an FP32 matrix x (rows x cols, leading dimension ld).
 * Source: Section 2 "NVFP4 format" (block scale per 16 elements, FP32 tensor
 * scale) with round-to-nearest (Section 3.4).
 *   axis FS4_AXIS_ROW: 1x16 blocks along rows; the result is rows x cols
 *     (cols % 16 == 0 for the PLAIN layout).
 *   axis FS4_AXIS_COL: 16x1 blocks along columns; the result is the
 *     quantisation of x^T, a cols x rows matrix (rows % 16 == 0 for PLAIN).
 *   codes, scales: outputs in the PLAIN or TILED layout (flags); s_g: output,
 *   one device float.  Rule for each block: s = RN_e4m3(fp32(amax_b /
 *   fp32(6 s_g))) saturating at 448; code = sign | RN_e2m1(fp32(|x| /
 *   fp32(dec(s) * s_g))) saturating at 6, ties to the even code; a block whose
 *   scale rounds to 0 gets all-zero codes.
 *   Errors: FS4_ERR_SHAPE for empty or unaligned shapes; FS4_ERR_INVALID_ARG
 *   for null pointers, ld < cols, codes/scales not 16-byte aligned (TILED);
 *   FS4_ERR_WORKSPACE.  Non-finite input is recorded as FS4_ERR_NONFINITE in
 *   the workspace status word (outputs then undefined).
 *   One cooperative launch: a pass for the tensor amax, a grid-wide barrier
 *   (a bounded wait: FS4_ERR_TIMEOUT in the status word if it runs out), then
 *   the quantise pass.  The workspace holds the call's amax and barrier count,
 *   so calls whose work may overlap on the GPU need separate workspaces. */
fs4_status fs4_nvfp4_quantize(const float* x, int64_t rows, int64_t cols, int64_t ld,
                              int32_t axis, uint8_t* codes, uint8_t* scales, float* s_g,
                              uint32_t flags, void* workspace, size_t workspace_bytes,
                              void* stream);

/* One matrix of a batched quantise: x (device, rows x cols, leading dimension ld),
 * axis (FS4_AXIS_ROW or FS4_AXIS_COL) and its outputs codes, scales, s_g, each as
 * for fs4_nvfp4_quantize. */
typedef struct {
  const float* x;
  int64_t rows, cols, ld;
  int32_t axis;
  uint8_t* codes;
  uint8_t* scales;
  float* s_g;
} fs4_quant_desc;

/* Bytes of workspace fs4_nvfp4_quantize_batched needs for `count` matrices (0 if
 * count is outside [1, FS4_MAX_BATCH]). */
size_t fs4_nvfp4_quantize_batched_workspace_size(int32_t count);

/* fs4_nvfp4_quantize on `count` matrices (descs: HOST array) in one launch: each matrix
 * gets its own tensor scale from its own amax and is quantised exactly as by
 * fs4_nvfp4_quantize with the same axis and flags (Section 2 "NVFP4 format").  One
 * cooperative launch covers every matrix: an amax pass, a grid-wide barrier (bounded:
 * FS4_ERR_TIMEOUT in the status word if it runs out), then the quantise pass over the
 * tiles of all matrices.  flags: FS4_SG_AMAX, FS4_LAYOUT_TILED (for all matrices),
 * FS4_TEST_STALL.  Errors as fs4_nvfp4_quantize for each descriptor, plus
 * FS4_ERR_SHAPE for count outside [1, FS4_MAX_BATCH]; a non-finite input anywhere is
 * recorded as FS4_ERR_NONFINITE in the status word.  Outputs of different matrices
 * must not overlap; calls whose work overlaps on the GPU need separate workspaces. */
fs4_status fs4_nvfp4_quantize_batched(int32_t count, const fs4_quant_desc* descs, uint32_t flags,
                                      void* workspace, size_t workspace_bytes, void* stream);

/* Dequantise a row-blocked NVFP4 matrix (rows x cols, as written by/* Dequantise a row-blocked NVFP4 matrix (rows x cols, as written by
 * fs4_nvfp4_quantize in the layout given by flags) into FP32 y (leading
 * dimension ld): y = fp32(fp32(code * s) * s_g).
 * Source: Section 2 "NVFP4 format": an element's value is its E2M1 value times
 * its block's E4M3 scale times the FP32 tensor scale.
 *   codes, scales: device, PLAIN (rows x cols/2 bytes, low nibble first;
 *   rows x cols/16 bytes) or TILED (FS4_LAYOUT_TILED), 16-byte aligned; s_g:
 *   one device float; y: device, caller-owned, rows x cols with ld >= cols, not
 *   overlapping the inputs.  One launch, no workspace.
 *   Errors: FS4_ERR_SHAPE (empty, or cols % 16 != 0), FS4_ERR_INVALID_ARG (null
 *   pointers, unknown flags, ld < cols, misaligned pointers), FS4_ERR_ARCH,
 *   FS4_ERR_CUDA. */
fs4_status fs4_nvfp4_dequantize(const uint8_t* codes, const uint8_t* scales, const float* s_g,
                                int64_t rows, int64_t cols, float* y, int64_t ld,
                                uint32_t flags, void* stream);

/* ------------------------------------------------------- momentum (first moment) */

/* Bytes of workspace fs4_momentum_nvfp4 needs (at least 256-byte aligned). */
size_t fs4_momentum_workspace_size(void);

/* One step of the NVFP4-stored first moment of Q-Root (Section 3.3: "Hadamard mixing
 * smooths the distribution before SR and adaptive 4/6 quantization"; Section 3.4: the
 * first-order momentum follows that storage recipe).  Per element of the FP32 gradient
 * g (rows x cols, leading dimension ld, cols % 16 == 0):
 *   m_prev = 0, or the previous state decoded: fp32(fp32(code * s) * s_g) on each 1x16
 *            block, then (H16^r)^-1 = H16 D / 4 with D the signs of prev_mask;
 *   m_t    = fp32(fp32(beta * m_prev) + fp32(fp32(1 - beta) * g));
 *   state  = NVFP4 of y = m_t H16^r (signs of `mask`, FP32 butterfly, * 0.25) in
 *            PLAIN 1x16 row blocks: tensor scale the smallest power of two with
 *            4 * 448 * s_g >= max |y|; per block the M = 6 and M = 4 candidates
 *            (scale RN_e4m3(amax_b / (M s_g))) with stochastically rounded codes,
 *            M = 4 kept only when its FP32 squared error (summed in element order)
 *            is strictly smaller.  A code is rounded up from the E2M1 value lo below
 *            v = fp32(|y| / den) to the next one, hi, when u < (v - lo) / (hi - lo);
 *            v >= 6 gives 6.  u for element (i, j) is the top 24 bits of SplitMix64
 *            at counter i * cols + j: z = seed + (i * cols + j + 1) * 0x9E3779B97F4A7C15,
 *            z ^= z >> 30, z *= 0xBF58476D1CE4E5B9, z ^= z >> 27,
 *            z *= 0x94D049BB133111EB, z ^= z >> 31; u = (z >> 40) * 2^-24.
 * prev_codes, prev_scales, prev_sg: the previous state (all null on the first step);
 * they may be the same buffers as codes, scales, s_g (in-place update).  m_out (may be
 * null; leading dimension ld_out) receives m_t in FP32, the matrix the Newton-Schulz
 * step consumes; it must not overlap g.  codes: rows x cols/2 bytes, scales:
 * rows x cols/16 bytes (16-byte aligned), s_g: one device float.  Two launches.
 * Errors: FS4_ERR_SHAPE, FS4_ERR_INVALID_ARG (null outputs, a partial previous state,
 * non-finite beta, ld or ld_out too small, misalignment), FS4_ERR_ALIAS (m_out
 * overlaps g), FS4_ERR_WORKSPACE; non-finite g is reported as FS4_ERR_NONFINITE
 * through fs4_device_status. */
fs4_status fs4_momentum_nvfp4(const float* g, int64_t rows, int64_t cols, int64_t ld,
                              float beta, const uint8_t* prev_codes,
                              const uint8_t* prev_scales, const float* prev_sg,
                              uint32_t prev_mask, uint8_t* codes, uint8_t* scales, float* s_g,
                              uint32_t mask, uint64_t seed, float* m_out, int64_t ld_out,
                              void* workspace, size_t workspace_bytes, void* stream);

/* --------------------------------------------------------------------- GEMM */

/* D = deq(A) * deq(B)^T on the tcgen05 block-scaled tensor cores
 * (kind::mxf4nvf4, UE4M3 scales per 16 elements, FP32 accumulation in TMEM).
 * The product is the one every step of Section 3.4 takes on NVFP4 operands.
 * A is M x K and B is N x K, both row-blocked along K and in the TILED layout
 * (as fs4_nvfp4_quantize writes with FS4_LAYOUT_TILED); a_sg, b_sg are their
 * device tensor scales.  D is M x N FP32 with leading dimension ldd.
 * K is rounded up to 256 with the zero padding of the TILED layout.
 * Errors: FS4_ERR_SHAPE (M, N, K < 1 or > FS4_MAX_DIM), FS4_ERR_INVALID_ARG
 * (null or non-16-byte-aligned operand, ldd < N), FS4_ERR_WORKSPACE (status
 * word: workspace of fs4_nvfp4_quantize_workspace_size() bytes). */
fs4_status fs4_nvfp4_gemm(const uint8_t* a_codes, const uint8_t* a_scales, const float* a_sg,
                          const uint8_t* b_codes, const uint8_t* b_scales, const float* b_sg,
                          int64_t M, int64_t N, int64_t K, float* d, int64_t ldd,
                          void* workspace, size_t workspace_bytes, void* stream);

/* ----------------------------------------------------------- Newton-Schulz */

/* One matrix of a batched call.  G (input) and out (output) are m x n FP32
 * device matrices with leading dimensions ld and ld_out; out must not overlap
 * G.  (a, b, c) are this matrix's polynomial coefficients (Section 3.4:
 * Root's shape-dependent coefficients are passed per matrix). */
typedef struct {
  const float* G;
  float* out;
  int64_t m, n, ld, ld_out;
  float a, b, c;
} fs4_ns_desc;

/* Workspace bytes fs4_root_ns needs for one m x n matrix. */
size_t fs4_root_ns_workspace_size(int64_t m, int64_t n);

/* Workspace bytes fs4_root_ns_batched (and _ex, _nvfp4) needs for `count` matrices
 * (host array); it depends on the shapes only (pointers may be null or overlap). */
size_t fs4_root_ns_batched_workspace_size(int32_t count, const fs4_ns_desc* descs);

/* Direct NVFP4 Newton-Schulz step (Section 3.4) on one FP32 momentum matrix.
 *   X_0 = clamp(G / (||G||_F + 1e-7), +-tau), tau = clip_k * RMS of the
 *   normalised matrix (clip_k <= 0 disables the clamp), or with
 *   FS4_NS_CLIP_QUANTILE the clip_k-quantile of |X_0|; then K iterations of
 *   qX = Q1x16(X), A = qX qX^T, B = b A + c Q1x16(A) Q16x1(A),
 *   X <- a X + Q1x16(B) Q16x1(X).  A tall matrix (m > n) is processed as its
 *   transpose so the Gram matrix is min(m,n) square; out has G's shape.
 *   m, n multiples of 16 in [16, FS4_MAX_DIM]; 1 <= K <= FS4_MAX_ITERS;
 *   a, b, c, clip_k finite.  Errors: FS4_ERR_SHAPE, FS4_ERR_INVALID_ARG,
 *   FS4_ERR_ALIAS (out overlaps G), FS4_ERR_WORKSPACE, FS4_ERR_ARCH,
 *   FS4_ERR_CUDA; device-side FS4_ERR_NONFINITE / FS4_ERR_TIMEOUT via
 *   fs4_device_status (out is then zero or undefined-but-finite). */
fs4_status fs4_root_ns(const float* G, int64_t m, int64_t n, int64_t ld, float* out,
                       int64_t ld_out, int32_t K, float a, float b, float c, float clip_k,
                       uint32_t flags, void* workspace, size_t workspace_bytes, void* stream);

/* The same step on `count` independent matrices (descs is a HOST array),
 * grouped so that each phase of the iteration is one launch over the tiles
 * of all matrices, each GEMM followed by a small bounds kernel (2 + 6K launches per call).
 * Source: Section 3.4 (the step of fs4_root_ns); the per-matrix (a, b, c) of each
 * descriptor carry the shape-dependent coefficients of Section 2 "Root optimizer".
 *   descs[i]: G (device, m x n, leading dimension ld), out (device, caller-owned,
 *   same shape, leading dimension ld_out), a, b, c.  The workspace
 *   (fs4_root_ns_batched_workspace_size, 256-byte aligned, caller-owned) holds
 *   every matrix's iterates and views; it must not overlap any G or out, and no
 *   out may overlap another out or any G.
 *   Errors: FS4_ERR_SHAPE (count outside [1, FS4_MAX_BATCH], a shape as for
 *   fs4_root_ns, K outside [1, FS4_MAX_ITERS]), FS4_ERR_INVALID_ARG (null
 *   pointers, ld or ld_out < n, pointers not 4-byte aligned, non-finite
 *   coefficients or clip_k, unknown flags),
 *   FS4_ERR_ALIAS, FS4_ERR_WORKSPACE, FS4_ERR_ARCH, FS4_ERR_CUDA; device-side
 *   conditions as for fs4_root_ns. */
fs4_status fs4_root_ns_batched(int32_t count, const fs4_ns_desc* descs, int32_t K, float clip_k,
                               uint32_t flags, void* workspace, size_t workspace_bytes,
                               void* stream);

/* fs4_root_ns_batched with the quantiser options above.  rht_masks: HOST
 * array of 3K sign masks when flags has FS4_NS_RHT (else ignored, may be
 * NULL): entry 3k + j is the mask of product j of iteration k (j = 0:
 * A = qX qX^T; 1: qA qA^T; 2: qB qX16x1), shared by both of its operands and
 * drawn fresh by the caller (Section 3.4: "a fresh 16x16 random Hadamard
 * transform").  Errors as fs4_root_ns_batched; FS4_ERR_INVALID_ARG also for
 * FS4_NS_RHT without masks. */
fs4_status fs4_root_ns_batched_ex(int32_t count, const fs4_ns_desc* descs, int32_t K, float clip_k,
                                  uint32_t flags, const uint16_t* rht_masks, void* workspace,
                                  size_t workspace_bytes, void* stream);

/* An NVFP4 first-moment state, as fs4_momentum_nvfp4 writes it: PLAIN 1x16 row blocks
 * (codes m x n/2 bytes, scales m x n/16 bytes, both 16-byte aligned; s_g one device
 * float) of m_t H16^r, with `mask` the sign mask of its H16^r. */
typedef struct {
  const uint8_t* codes;
  const uint8_t* scales;
  const float* s_g;
  uint32_t mask;
} fs4_nvfp4_state;

/* fs4_root_ns_batched_ex on matrices given as NVFP4 first-moment states instead of FP32
 * (the Newton-Schulz step consumes the stored momentum directly; Section 3.4: "The
 * first-order momentum follows the first-moment storage recipe in Section 3.3").
 * descs[i].G must be null and descs[i].ld is ignored; matrix i is the state states[i],
 * decoded as fs4_momentum_nvfp4 decodes its previous state (fp32(fp32(code * s) * s_g)
 * on each block, then (H16^r)^-1 = H16 D / 4), read by the reduction and the preamble in
 * place of G.  Everything else (shapes, flags, masks, workspace, outputs) is as for
 * fs4_root_ns_batched_ex; the workspace size and layout queries accept descriptors
 * with a null G.  Errors as there; also FS4_ERR_INVALID_ARG for a null states array, a
 * non-null G, or a state with null or misaligned pointers or mask > 0xFFFF. */
fs4_status fs4_root_ns_batched_nvfp4(int32_t count, const fs4_ns_desc* descs,
                                     const fs4_nvfp4_state* states, int32_t K, float clip_k,
                                     uint32_t flags, const uint16_t* rht_masks, void* workspace,
                                     size_t workspace_bytes, void* stream);


/* fs4_root_ns_batched_nvfp4, with CUDA events recorded on `stream` around each
 * phase at the 3 + 3K positions of fs4_root_ns_batched_timed (phase_events: HOST
 * array of n_events >= 3 + 3K cudaEvent_t handles created by the caller with timing
 * enabled).  Arguments, layouts and errors as fs4_root_ns_batched_nvfp4, plus
 * FS4_ERR_INVALID_ARG for a missing event array or too few events, checked before
 * anything is launched. */
fs4_status fs4_root_ns_batched_nvfp4_timed(int32_t count, const fs4_ns_desc* descs,
                                           const fs4_nvfp4_state* states, int32_t K, float clip_k,
                                           uint32_t flags, const uint16_t* rht_masks,
                                           void* workspace, size_t workspace_bytes, void* stream,
                                           void* const* phase_events, int32_t n_events);

/* fs4_root_ns_batched_ex, with CUDA events recorded on `stream` around each
 * phase so a caller can time the kernels on the launching stream.
 * phase_events: HOST array of n_events >= 3 + 3K cudaEvent_t handles (created
 * by the caller with timing enabled).  Event 0 is recorded before the
 * workspace reset and the reduction kernel, event 1 after it, event 2 after
 * the preamble kernels, and event 3 + 3k + j after product j (0: A = qX qX^T,
 * 1: B, 2: update) of iteration k and its bounds kernel.  Errors as
 * fs4_root_ns_batched_ex, plus FS4_ERR_INVALID_ARG for a missing event. */
fs4_status fs4_root_ns_batched_timed(int32_t count, const fs4_ns_desc* descs, int32_t K,
                                     float clip_k, uint32_t flags, const uint16_t* rht_masks,
                                     void* workspace, size_t workspace_bytes, void* stream,
                                     void* const* phase_events, int32_t n_events);

/* -------------------------------------------------- BF16 comparison step */

/* The same Newton-Schulz step with BF16 operands instead of NVFP4: the step of
 * Section 2 "Root optimizer" as an optimized BF16 implementation takes it, the
 * baseline that Section 4.4 and Table 6 (Root rows: BF16 344.55 ms, NVFP4
 * 109.80 ms at d = 4096) compare the NVFP4 step against.  X_0 is normalised and
 * clipped exactly as in fs4_root_ns; then K iterations of
 *   Xb = bf16(X), A = Xb Xb^T, B = b A + c bf16(A) bf16(A)^T,
 *   X <- a X + bf16(B) Xb,
 * with bf16() rounding to nearest (ties to even), BF16 x BF16 products on the
 * tensor cores (tcgen05 kind::f16) accumulated in FP32, and X, A, B held in FP32.
 * Tall matrices are transposed as in fs4_root_ns.  There are no tensor scales, so
 * a call launches 2 + 3K kernels.  Arguments, layouts, ownership, aliasing rules
 * and errors as fs4_root_ns_batched; flags may hold FS4_STOP_AFTER,
 * FS4_NS_CLIP_QUANTILE and FS4_TEST_STALL (FS4_NS_RHT and FS4_NS_ADAPTIVE46 give
 * FS4_ERR_INVALID_ARG).  A stop after product 1 writes B (FP32) over A as in the
 * NVFP4 step.  The workspace (larger than the NVFP4 step's: 2 bytes per element
 * for each BF16 view) is sized by fs4_root_ns_bf16_batched_workspace_size. */
size_t fs4_root_ns_bf16_batched_workspace_size(int32_t count, const fs4_ns_desc* descs);

fs4_status fs4_root_ns_bf16_batched(int32_t count, const fs4_ns_desc* descs, int32_t K,
                                    float clip_k, uint32_t flags, void* workspace,
                                    size_t workspace_bytes, void* stream);

/* fs4_root_ns_bf16_batched with CUDA events recorded around each phase, at the
 * same 3 + 3K positions as fs4_root_ns_batched_timed. */
fs4_status fs4_root_ns_bf16_batched_timed(int32_t count, const fs4_ns_desc* descs, int32_t K,
                                          float clip_k, uint32_t flags, void* workspace,
                                          size_t workspace_bytes, void* stream,
                                          void* const* phase_events, int32_t n_events);



/* ------------------------------------------------------------ no-alloc variant */

/* Bytes of the workspace array built into the library for fs4_root_ns_noalloc. */
#define FS4_NOALLOC_SCRATCH_BYTES (16u << 20)

/* fs4_root_ns for callers that cannot allocate device memory (no counterpart in
 * the paper; an interface addition).  Examples: plugins inside a host framework
 * that owns all device memory and lends none; loops in which a run-time
 * allocation is forbidden.  Same arguments and result as fs4_root_ns
 * with flags = 0, but the workspace is a fixed 16 MiB array compiled into the
 * library (every device that loads the library holds it until the process
 * exits).  Matrices whose fs4_root_ns_workspace_size(m, n) exceeds
 * FS4_NOALLOC_SCRATCH_BYTES are rejected with FS4_ERR_WORKSPACE before anything
 * is launched (1024 x 1024 needs 11.4 MiB and fits; 1024 x 2048 needs 17.6 MiB); other errors as fs4_root_ns.  The first call
 * on each device looks up the array's device address with that device current
 * (make it before any stream capture).  Every call shares the array and it keeps
 * the last call's contents; each call clears what must start at zero, but calls
 * whose work overlaps on the GPU race on it.  Device-side conditions (non-finite
 * input: zero output) cannot be queried through fs4_device_status.  Allocates
 * nothing. */
fs4_status fs4_root_ns_noalloc(const float* G, int64_t m, int64_t n, int64_t ld, float* out,
                               int64_t ld_out, int32_t K, float a, float b, float c,
                               float clip_k, void* stream);

/* Synchronise `stream` and return the device status recorded in `workspace`
 * by the last call that used it (FS4_OK, FS4_ERR_NONFINITE, FS4_ERR_TIMEOUT). */
fs4_status fs4_device_status(const void* workspace, void* stream);

/* Human-readable name of a status code (static string). */
const char* fs4_status_string(fs4_status status);

/* Byte offsets (from the workspace base) of the internal tensors of matrix
 * `index` of a batched call, for inspection after an FS4_STOP_AFTER run.
 * mp, np: working dimensions padded to 256 (m <= n after the tall transpose).
 * X: FP32 mp x np.  A: FP32 mp x mp (upper 256x256 tiles written).
 * qX/qXT/qA/qB: TILED codes + scales of X (mp x np), X^T (np x mp, the 16x1
 * view of X), A and B (mp x mp); qX and qXT alternate between two buffers by
 * iteration parity (slot k%2 holds the view of X_k).  scalars: a float array
 * with s_g of X_k at [k], of A_k at [64+k], of B_k at [128+k]. */
typedef struct {
  int64_t mp, np;
  int64_t X, A;
  int64_t qX_codes[2], qX_scales[2], qXT_codes[2], qXT_scales[2];
  int64_t qA_codes, qA_scales, qB_codes, qB_scales;
  int64_t scalars;
} fs4_ns_layout;

fs4_status fs4_root_ns_layout(int32_t count, const fs4_ns_desc* descs, int32_t index,
                              fs4_ns_layout* layout);

/* Workspace offsets of matrix `index` of a BF16 step (see fs4_root_ns_layout).  The
 * *_codes fields locate the BF16 views in the TILED BF16 layout: tiles of 128 rows x
 * 64 elements (16384 bytes), tile (r/128, c/64) at ((r/128)*(Cp/64) + c/64)*16384,
 * row r%128 at byte 128*(r%128), its 16-byte chunk j = (c%64)/8 at chunk position
 * j ^ (r%8); the *_scales fields are unused. */
fs4_status fs4_root_ns_bf16_layout(int32_t count, const fs4_ns_desc* descs, int32_t index,
                                   fs4_ns_layout* layout);

#ifdef __cplusplus
}
#endif
#endif /* FS4_H */

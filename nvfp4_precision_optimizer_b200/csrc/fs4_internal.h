// Internal definitions shared by libfs4's kernels and its host-side planner.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

namespace fs4 {

constexpr int kMaxBatch = 224;   // matrices per batched call (kernel-parameter table size)
constexpr int kMaxIters = 32;
constexpr int kPad = 256;        // working dimensions are padded to multiples of 256

// ---------------------------------------------------------------- workspace header
// Byte 0 of every workspace: the 32-bit device status word (kStatus* bits).
// Bytes 4..7 of the quantize workspace: max |x| as float bits.
constexpr size_t kHeaderBytes = 256;

// ---------------------------------------------------------------- per-matrix state
// One 4 KB block per matrix, zeroed at the start of every Newton-Schulz call.
struct NsState {
  double sumsq;            // sum of G^2 (float64)
  uint32_t amaxG;          // max |G| as float bits
  uint32_t nonfinite;      // G holds NaN or Inf
  uint32_t done[8];        // finished work units per phase kind (preamble, G1, G2, G3, reduce)
  float inv0, tau0;        // fp32(1 / (||G|| + eps)) and the clip threshold (set after the reduction)
  uint32_t q_bin1;         // quantile clip: top 11 key bits of the selected |G| (select pass 1)
  uint32_t q_pad;
  uint64_t q_rank1;        // quantile clip: rank of the selected key within that bin (1-based)
  unsigned long long q_count;   // quantile clip: candidates gathered (keys in bin q_bin1)
  uint32_t pad0[44];
  float sg[192];           // tensor scales: X_k at [k], A_k at [64+k], B_k at [128+k]
  float u_rowX[64];        // max_i sum_j deq(qX_k)_ij^2
  float u_colX[64];        // max_j sum_i deq(qX16_k)_ij^2
  float u_rowA[64];        // max_i sum_j deq(qA_k)_ij^2
  float u_rowB[64];        // max_i sum_j deq(qB_k)_ij^2
  uint32_t amaxX[64];      // max |X_k| as float bits
  uint32_t pad1[448];
};
static_assert(sizeof(NsState) == 4096, "NsState must stay 4 KB");
constexpr int kSgX = 0, kSgA = 64, kSgB = 128;

// Quantile clip: the 31-bit key of |g| (its float bits without the sign) is selected
// in three digits of 11, 11 and 9 bits; the first digit's histogram lives in the
// zeroed state block.
constexpr int kQBins1 = 2048, kQBins2 = 2048, kQBins3 = 512;

// Offsets (bytes, from the workspace base) of one matrix's buffers.
struct MatLayout {
  int64_t state;                                 // NsState
  int64_t rowsumX, colsumX, rowsumA, rowsumB;    // float [mp], [np], [mp], [mp]
  int64_t qhist;                                 // uint32 [kQBins1] (quantile clip)
  int64_t X, A;                                  // float [mp*np], [mp*mp]
  int64_t qX[2], sX[2], qXT[2], sXT[2];          // TILED codes/scales of X (mp x np), X^T (np x mp)
  int64_t qA, sA, qB, sB;                        // TILED codes/scales of A, B (mp x mp)
};

__host__ __device__ inline int64_t align_up(int64_t v, int64_t a) { return (v + a - 1) / a * a; }

// Bytes of the zero-initialised block (state + sums) of an mp x np matrix.
__host__ __device__ inline int64_t state_block_bytes(int64_t mp, int64_t np) {
  return align_up(4096 + 4 * (3 * mp + np) + 4 * kQBins1, 256);
}

// Bytes per element of one operand view: NVFP4 (codes 1/2 B + scales 1/16 B) or BF16 (2 B).
// Returned as sixteenths of a byte so that both are integers.
__host__ __device__ inline int64_t view_sixteenths(bool bf16) { return bf16 ? 32 : 9; }

// Bytes of the large buffers of an mp x np matrix (bf16: the BF16 comparison step,
// whose operand views are BF16 instead of NVFP4).
__host__ __device__ inline int64_t big_block_bytes(int64_t mp, int64_t np, bool bf16 = false) {
  const int64_t xn = mp * np, aa = mp * mp, v = view_sixteenths(bf16);
  return 4 * xn + 4 * aa + 4 * (xn * v / 16) + 2 * (aa * v / 16);
}

__host__ __device__ inline MatLayout mat_layout(int64_t mp, int64_t np, int64_t state_off,
                                                int64_t big_off, bool bf16 = false) {
  MatLayout L;
  L.state = state_off;
  L.rowsumX = state_off + 4096;
  L.colsumX = L.rowsumX + 4 * mp;
  L.rowsumA = L.colsumX + 4 * np;
  L.rowsumB = L.rowsumA + 4 * mp;
  L.qhist = L.rowsumB + 4 * mp;
  const int64_t xn = mp * np, aa = mp * mp;
  // NVFP4: codes (1/2 B per element) then scales (1/16 B); BF16: 2 B per element, no scales
  const int64_t cx = bf16 ? 2 * xn : xn / 2, sx = bf16 ? 0 : xn / 16;
  const int64_t ca = bf16 ? 2 * aa : aa / 2, sa = bf16 ? 0 : aa / 16;
  int64_t o = big_off;
  L.X = o; o += 4 * xn;
  L.A = o; o += 4 * aa;
  for (int s = 0; s < 2; ++s) { L.qX[s] = o; o += cx; L.sX[s] = o; o += sx; }
  for (int s = 0; s < 2; ++s) { L.qXT[s] = o; o += cx; L.sXT[s] = o; o += sx; }
  L.qA = o; o += ca; L.sA = o; o += sa;
  L.qB = o; o += ca; L.sB = o; o += sa;
  return L;
}

// One matrix of a Newton-Schulz launch (kernel parameter, by value).
struct MatDesc {
  const float* G;          // caller's input, m0 x n0, leading dimension ldg
  float* out;              // caller's output, m0 x n0, leading dimension ldo
  int64_t ldg, ldo;
  int64_t state_off, big_off;
  int32_t m, n;            // working orientation, m <= n
  int32_t mp, np;          // padded to multiples of 256
  int32_t tall;            // 1: working X = G^T
  float a, b, c;
  // NVFP4 source (G given as an NVFP4 state: PLAIN 1x16 row blocks of G H16^r, as the
  // first-moment step stores it) or null (G is the FP32 matrix above)
  const uint8_t* qcodes;
  const uint8_t* qscales;
  const float* qsg;
  uint32_t qmask;
};

// Kernel parameters of one Newton-Schulz phase over a batch of matrices.
constexpr uint32_t kOptRht = 1u, kOpt46 = 2u;   // NsParams::opts
constexpr uint32_t kOptQuantile = 4u;            // clip at the clip_k-quantile of |X_0|
constexpr uint32_t kOptNvSrc = 8u;               // every G is an NVFP4 state (MatDesc::qcodes)
constexpr uint32_t kOptBf16 = 16u;               // BF16 operand views and kind::f16 products
constexpr uint32_t kOptWideK = 32u;              // NVFP4 products of 8192-class matrices: their
                                                 // mainloops set the time (two scale copiers each)

struct NsParams {
  int32_t count;
  int32_t iter;            // k of the current iteration
  int32_t last;            // 1 on the final update product (writes `out`)
  int32_t stall;           // test only: the MMA issuer waits on a barrier nothing arrives on
  int32_t dbg_b;           // debug stop after the second product: also write B (FP32) over A
  uint32_t opts;           // kOptRht | kOpt46 | kOptQuantile
  float clip_k;            // clip_k * RMS, or with kOptQuantile the quantile ratio q in (0, 1]
  uint32_t* status;
  uint8_t* ws;             // workspace base
  uint16_t rht[3 * kMaxIters];   // H16^r sign mask of product j of iteration k at 3k + j
  int32_t prefix[kMaxBatch + 1];   // prefix sums of this phase's work units per matrix
  MatDesc mat[kMaxBatch];
};
static_assert(sizeof(NsParams) <= 32000, "kernel parameter block too large");

// Parameters of the standalone block-scaled GEMM.
struct GemmPlainArgs {
  const uint8_t* a_codes; const uint8_t* a_scales; const float* a_sg;
  const uint8_t* b_codes; const uint8_t* b_scales; const float* b_sg;
  int32_t M, N, Kp;        // Kp: K padded to 256
  int32_t Mp, Np;          // rows padded to 128
  float* d;
  int64_t ldd;
  uint32_t* status;
};

enum class Epi : int { Plain = 0, GramX = 1, GramA = 2, Update = 3 };

// One matrix of a batched standalone quantise (host side; mirrors fs4_quant_desc).
struct QuantDesc {
  const float* x;
  int64_t rows, cols, ld;
  int32_t axis;
  uint8_t* codes;
  uint8_t* scales;
  float* s_g;
};

// ---------------------------------------------------------------- launchers (kernels.cu / gemm.cu)
size_t quantize_batched_workspace_bytes(int32_t count);
cudaError_t launch_quantize_batched(int32_t count, const QuantDesc* descs, uint32_t flags, uint8_t* ws,
                                    cudaStream_t st, int num_sms);
cudaError_t launch_quantize(const float* x, int64_t rows, int64_t cols, int64_t ld, int axis,
                            uint8_t* codes, uint8_t* scales, float* s_g, uint32_t flags,
                            uint8_t* ws, cudaStream_t st, int num_sms);
cudaError_t launch_dequantize(const uint8_t* codes, const uint8_t* scales, const float* s_g,
                              int64_t rows, int64_t cols, float* y, int64_t ld, uint32_t flags,
                              cudaStream_t st, int num_sms);
cudaError_t launch_ns_reduce(const NsParams& p, cudaStream_t st, int num_sms);
cudaError_t launch_ns_quantile(const NsParams& p, cudaStream_t st, int num_sms);
cudaError_t launch_momentum(const float* g, int64_t rows, int64_t cols, int64_t ld, float beta,
                            const uint8_t* prev_codes, const uint8_t* prev_scales,
                            const float* prev_sg, uint32_t prev_mask, uint8_t* codes,
                            uint8_t* scales, float* s_g, uint32_t mask, uint64_t seed,
                            float* m_out, int64_t ld_out, uint8_t* ws, cudaStream_t st,
                            int num_sms);
cudaError_t launch_ns_preamble(const NsParams& p, cudaStream_t st, int num_sms);
cudaError_t launch_gemm_plain(const GemmPlainArgs& a, cudaStream_t st, int num_sms);
cudaError_t launch_gemm_ns(Epi epi, const NsParams& p, cudaStream_t st, int num_sms);

}  // namespace fs4

// Plain, slow C++17 oracle of the direct NVFP4 Newton-Schulz step.
//
// TEST INFRASTRUCTURE ONLY.  Only the test-suite, the smoke check and the
// CPU-baseline / reference legs of bench.py load this library (through
// oracle/cpp_oracle.py).  It shares no code, table or helper with the CUDA path,
// and it uses no BLAS: every product is a triple loop in float64 over
// dequantised operands, and every NVFP4 decision is a nearest-value search over
// the code tables.  Loops over independent rows run in parallel (OpenMP); no
// loop is blocked, fused or reordered beyond that.
//
// Source: "Full-Stack FP4: Stable LLM Pretraining with Quantized Projections,
// Optimizers, and Attention" (arXiv 2607.04422).
//   * Section 2 "Preliminaries", paragraph "NVFP4 format": E2M1 elements in
//     blocks of 16 with one E4M3 scale per block and one FP32 tensor scale s_g;
//     x_hat = x_E2M1 * s * s_g.
//   * Section 2, paragraph "Root optimizer": X_{k+1} = a X + b X (X^T X)
//     + c X (X^T X)^2, typically five iterations.
//   * Section 3.4 "NVFP4 Root Optimizer": the quantised iteration
//       qX = Q1x16(X), A = qX qX^T, B = b A + c Q1x16(A) Q16x1(A),
//       X_{k+1} = a X + Q1x16(B) Q16x1(X), round-to-nearest throughout.
//
// Readings where the pages are silent (the same ones the numpy oracle takes):
//   * RTN = IEEE round-to-nearest, ties to the even code, saturating (E2M1 at 6,
//     E4M3 at 448).  Codes are sign-magnitude; the sign bit is the element's.
//   * s_g: the smallest power of two with 6 * 448 * s_g >= amax (clamped to
//     2^-116 .. 2^118, 1 for an all-zero tensor), or fp32(amax / 2688).
//   * block scale s = RN_e4m3(fp32(amax_b / fp32(6 s_g))); code =
//     sign | RN_e2m1(fp32(|x| / fp32(dec(s) s_g))); scale 0 gives all-zero codes.
//   * X_0 = clamp(fp32(G * inv), +-tau), inv = fp32(1 / (||G||_F + 1e-7)) with
//     ||G||_F summed in float64, tau = fp32(clip_k ||G|| inv / sqrt(m n)).
//   * A, B and X are FP32 tensors; products are float64 sums over dequantised
//     operands, rounded once to FP32 (B and X' after the combine).  A is made
//     exactly symmetric from its upper triangle.  Tall inputs are transposed.
//
// Options of Section 3.4 (off by default; the same readings as the numpy oracle):
//   * Adaptive 4/6 ("All quantizations use RTN and adaptive 4/6 scaling"; Four
//     Over Six): every block is quantised twice, with its amax mapped to M = 6 and
//     to M = 4, and keeps M = 4 only when that candidate's squared error, summed
//     in FP32 in element order, is strictly smaller.  Both candidates share s_g,
//     whose denominator becomes 4 * 448 = 1792.
//   * H16^r ("a fresh 16x16 random Hadamard transform" along K of every quantised
//     operand): H16^r = D H16 / 4 with D the diagonal of 16 signs given by a 16-bit
//     mask (bit i set: element i negated), one mask per product (3k: A_k, 3k + 1:
//     qA qA16, 3k + 2: qB qX16), applied in FP32 as the butterfly with strides 1, 2,
//     4, 8 ((u, v) -> (u + v, u - v)) and a final exact * 0.25.
//   * Quantile clip ("p99 outlier clipping", Table 8 "Root quantile ratio 0.99"):
//     tau is the k-th smallest |fp32(G inv)|, k = ceil(fl64(fp32(q)) N) clamped to
//     [1, N] (the nearest-rank quantile), in place of clip_k * RMS.
//
// The BF16 route (the optimized BF16 baseline of Section 4.4 and Table 6): the same
// plan with bf16() in place of every quantisation, bf16() = round to nearest, ties
// to even, of the low 16 bits of the FP32 word.
//
// The NVFP4 first moment (Section 3.3 "Quantized-State AdamW", which Section 3.4's
// momentum follows: Hadamard mixing, stochastic rounding, adaptive 4/6):
//   * m_t = fp32(fp32(beta m_prev) + fp32(fp32(1 - beta) g)), m_prev the decoded
//     previous state (zero on the first step);
//   * state = Q(m_t H16^r) in 1x16 row blocks with 4/6 block scales (s_g by the 1792
//     rule), every element code rounded stochastically: v = fp32(|y| / den) below 6
//     goes to the upper of its two neighbouring E2M1 magnitudes when u < fp32((v - lo)
//     / (hi - lo)), else to the lower; v >= 6 gives 6; both 4/6 candidates use the
//     same u;
//   * u of element i (row-major) = top 24 bits of SplitMix64 (Steele, Lea and Flood,
//     OOPSLA 2014) at counter i + 1 from the seed, times 2^-24;
//   * decode: fp32(fp32(code s_b) s_g), then (H16^r)^-1 = H16 D / 4 (the butterfly,
//     the exact * 0.25, then the signs).
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

#ifdef _OPENMP
#include <omp.h>
#endif

namespace {

constexpr int kBlock = 16;
constexpr double kE2m1Mag[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
constexpr double kSgDenom = 6.0 * 448.0;   // 2688
constexpr double kSgDenom46 = 4.0 * 448.0; // 1792: the M = 4 candidate fits too
constexpr int kAmaxMode = 1;               // quantiser flags: s_g = amax / denom
constexpr int kAdaptive46 = 2;             //                  adaptive 4/6 blocks
constexpr double kEps = 1e-7;

// Value of an FP8 E4M3 byte (bias 7, no infinities, S.1111.111 = NaN, exponent
// field 0 = subnormal m/8 * 2^-6).
double e4m3_value(int byte) {
  const double sign = (byte & 0x80) ? -1.0 : 1.0;
  const int e = (byte >> 3) & 0xF, m = byte & 0x7;
  if (e == 0xF && m == 0x7) return NAN;
  if (e == 0) return sign * (m / 8.0) * std::ldexp(1.0, -6);
  return sign * (1.0 + m / 8.0) * std::ldexp(1.0, e - 7);
}

// Signed value of a 4-bit E2M1 code (bit 3 = sign).
double e2m1_value(int code) {
  const double mag = kE2m1Mag[code & 7];
  return (code & 8) ? -mag : mag;
}

// Index of the grid value nearest to q >= 0 (grid ascending); a tie goes to the
// even index; q at or above the last value saturates to it.
int nearest_even(double q, const double* grid, int n) {
  if (q >= grid[n - 1]) return n - 1;
  int best = 0;
  double best_d = std::fabs(q - grid[0]);
  for (int i = 1; i < n; ++i) {
    const double d = std::fabs(q - grid[i]);
    if (d < best_d || (d == best_d && i % 2 == 0)) {
      best = i;
      best_d = d;
    }
  }
  return best;
}

struct E4m3Grid {
  double v[127];   // bytes 0x00 .. 0x7E, increasing
  E4m3Grid() {
    for (int b = 0; b < 127; ++b) v[b] = e4m3_value(b);
  }
};
const E4m3Grid& e4m3_grid() {
  static const E4m3Grid g;
  return g;
}

int e2m1_encode(double q) { return nearest_even(q, kE2m1Mag, 8); }
int e4m3_encode(double v) { return nearest_even(v, e4m3_grid().v, 127); }

float tensor_scale(float amax, int amax_mode, double denom = kSgDenom) {
  if (!(amax > 0.0f)) return 1.0f;
  if (amax_mode) return amax / (float)denom;
  int e = std::ilogb((double)amax) - 12;
  while (std::ldexp(denom, e) < (double)amax) ++e;
  while (std::ldexp(denom, e - 1) >= (double)amax) --e;
  if (e < -116) e = -116;
  if (e > 118) e = 118;
  return (float)std::ldexp(1.0, e);
}

// One block of 16 FP32 values with its amax mapped to M: the E4M3 scale byte, the
// 4-bit codes and the FP32 dequantised values.
struct Block {
  int scale;
  uint8_t code[kBlock];
  float deq[kBlock];
};

// Stochastic rounding of FP32 v >= 0 onto an E2M1 magnitude code with FP32 u in
// [0, 1): lo = the largest magnitude <= v, hi the next; up when u < (v - lo) / (hi - lo).
int e2m1_encode_sr(float v, float u) {
  if (v >= 6.0f) return 7;
  int lo = 0;
  while (lo < 7 && kE2m1Mag[lo + 1] <= (double)v) ++lo;
  const float gap = (float)(kE2m1Mag[lo + 1] - kE2m1Mag[lo]);
  const float frac = (v - (float)kE2m1Mag[lo]) / gap;
  return u < frac ? lo + 1 : lo;
}

// u: null for round to nearest, else the block's 16 stochastic-rounding draws.
Block quantize_block(const float* xb, float s_g, float M, const float* u = nullptr) {
  Block q;
  float amax = 0.0f;
  for (int i = 0; i < kBlock; ++i) amax = std::fmax(amax, std::fabs(xb[i]));
  const float v = amax / (M * s_g);
  q.scale = e4m3_encode((double)v);
  const float den = (float)e4m3_value(q.scale) * s_g;
  for (int i = 0; i < kBlock; ++i) {
    uint8_t code = 0;
    if (den > 0.0f) {
      const float r = std::fabs(xb[i]) / den;
      const int mag = u ? e2m1_encode_sr(r, u[i]) : e2m1_encode((double)r);
      code = (uint8_t)(mag | (std::signbit(xb[i]) ? 8 : 0));
    }
    q.code[i] = code;
    q.deq[i] = (float)(e2m1_value(code) * (double)den);
  }
  return q;
}

// sum_i (x_i - deq_i)^2 in FP32, one rounding per operation, i = 0 .. 15 in order.
float block_sq_error(const float* xb, const Block& q) {
  float e = 0.0f;
  for (int i = 0; i < kBlock; ++i) {
    const float d = xb[i] - q.deq[i];
    const float d2 = d * d;
    e = e + d2;
  }
  return e;
}

// Q1x16 of an FP32 rows x cols matrix (cols % 16 == 0) with tensor scale s_g:
// 4-bit codes (one per element, unpacked) and E4M3 scale bytes.  adaptive46: each
// block keeps the M = 4 candidate when its squared error is strictly smaller.
void quantize_rows(const float* x, int64_t rows, int64_t cols, float s_g, bool adaptive46,
                   uint8_t* nib, uint8_t* scales) {
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t jb = 0; jb < cols / kBlock; ++jb) {
      const float* xb = x + r * cols + jb * kBlock;
      Block q = quantize_block(xb, s_g, 6.0f);
      if (adaptive46) {
        const Block q4 = quantize_block(xb, s_g, 4.0f);
        if (block_sq_error(xb, q4) < block_sq_error(xb, q)) q = q4;
      }
      scales[r * (cols / kBlock) + jb] = (uint8_t)q.scale;
      for (int i = 0; i < kBlock; ++i) nib[r * cols + jb * kBlock + i] = q.code[i];
    }
  }
}

// Exact float64 values code * s * s_g of a Q1x16 matrix.
void dequantize_rows(const uint8_t* nib, const uint8_t* scales, float s_g, int64_t rows,
                     int64_t cols, double* out) {
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t c = 0; c < cols; ++c)
      out[r * cols + c] =
          e2m1_value(nib[r * cols + c]) * e4m3_value(scales[r * (cols / kBlock) + c / kBlock]) * (double)s_g;
}

float amax_of(const float* x, int64_t count) {
  float m = 0.0f;
  for (int64_t i = 0; i < count; ++i) m = std::fmax(m, std::fabs(x[i]));
  return m;
}

void transpose(const float* x, int64_t rows, int64_t cols, float* y) {
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t c = 0; c < cols; ++c) y[c * rows + r] = x[r * cols + c];
}

// Quantiser options of one NS iteration: quantiser flags (kAmaxMode, kAdaptive46)
// and the 3K sign masks of H16^r (null: H = I).
struct Opts {
  int flags = 0;
  const uint16_t* masks = nullptr;
};

// x H16^r on every 16-element block of each row, in FP32 (rows x cols, in place):
// signs of D, then the butterfly with strides 1, 2, 4, 8, then * 0.25.
void hadamard_rows(float* x, int64_t rows, int64_t cols, uint16_t mask) {
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t jb = 0; jb < cols / kBlock; ++jb) {
      float* y = x + r * cols + jb * kBlock;
      for (int i = 0; i < kBlock; ++i)
        if ((mask >> i) & 1) y[i] = -y[i];
      for (int h = 1; h < kBlock; h *= 2)
        for (int i = 0; i < kBlock; i += 2 * h)
          for (int j = i; j < i + h; ++j) {
            const float u = y[j], v = y[j + h];
            y[j] = u + v;
            y[j + h] = u - v;
          }
      for (int i = 0; i < kBlock; ++i) y[i] = y[i] * 0.25f;
    }
  }
}

// Dequantised Q1x16(x H) (s_g from the exact amax of x H) as a rows x cols float64
// matrix; mask < 0: H = I.
void q1x16(const float* x, int64_t rows, int64_t cols, int flags, int mask, double* out,
           float* sg_out) {
  std::vector<float> xh;
  if (mask >= 0) {
    xh.assign(x, x + rows * cols);
    hadamard_rows(xh.data(), rows, cols, (uint16_t)mask);
    x = xh.data();
  }
  std::vector<uint8_t> nib((size_t)(rows * cols)), sc((size_t)(rows * cols / kBlock));
  const bool a46 = flags & kAdaptive46;
  const float sg = tensor_scale(amax_of(x, rows * cols), flags & kAmaxMode, a46 ? kSgDenom46 : kSgDenom);
  quantize_rows(x, rows, cols, sg, a46, nib.data(), sc.data());
  dequantize_rows(nib.data(), sc.data(), sg, rows, cols, out);
  if (sg_out) *sg_out = sg;
}

// Dequantised Q16x1(H^T x): blocks of 16 down each column, returned as the rows x
// cols matrix.  Held as the Q1x16 of (H^T x)^T = x^T H, transposed back.
void q16x1(const float* x, int64_t rows, int64_t cols, int flags, int mask, double* out) {
  std::vector<float> xt((size_t)(rows * cols));
  transpose(x, rows, cols, xt.data());
  std::vector<double> dt((size_t)(rows * cols));
  q1x16(xt.data(), cols, rows, flags, mask, dt.data(), nullptr);
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t c = 0; c < cols; ++c) out[r * cols + c] = dt[c * rows + r];
}

// out = L R in float64 (L is M x K, R is K x N), summed in k order.
void product(const double* L, const double* R, int64_t M, int64_t K, int64_t N, double* out) {
#pragma omp parallel for schedule(dynamic, 4)
  for (int64_t i = 0; i < M; ++i) {
    double* o = out + i * N;
    for (int64_t j = 0; j < N; ++j) o[j] = 0.0;
    for (int64_t k = 0; k < K; ++k) {
      const double l = L[i * K + k];
      const double* r = R + k * N;
      for (int64_t j = 0; j < N; ++j) o[j] += l * r[j];
    }
  }
}

// 1-based rank of the nearest-rank q-quantile of N values: ceil(fl64(fp32(q)) N),
// clamped to [1, N].
int64_t quantile_rank(double q, int64_t N) {
  int64_t k = (int64_t)std::ceil((double)(float)q * (double)N);
  return k < 1 ? 1 : (k > N ? N : k);
}

// The k-th smallest of a[0 .. N) (1-based k): sort a copy and index it.
template <class T>
T kth_smallest(const T* a, int64_t N, int64_t k) {
  std::vector<T> s(a, a + N);
  std::sort(s.begin(), s.end());
  return s[(size_t)(k - 1)];
}

// X_0 from G (m x n, working orientation): returns ||G||_F.  clip_quantile > 0:
// tau is that quantile of |fp32(G inv)|; else clip_k > 0: tau = clip_k * RMS;
// else no clip.
double normalise_and_clip(const float* G, int64_t m, int64_t n, double clip_k,
                          double clip_quantile, float* X0, float* inv_out, float* tau_out) {
  double s = 0.0;
  for (int64_t i = 0; i < m * n; ++i) s += (double)G[i] * (double)G[i];
  const double norm = std::sqrt(s);
  const float inv = (float)(1.0 / (norm + kEps));
  for (int64_t i = 0; i < m * n; ++i) X0[i] = G[i] * inv;
  float tau = 0.0f;
  bool clip = false;
  if (clip_quantile > 0.0) {
    std::vector<float> a((size_t)(m * n));
    for (int64_t i = 0; i < m * n; ++i) a[i] = std::fabs(X0[i]);
    tau = kth_smallest(a.data(), m * n, quantile_rank(clip_quantile, m * n));
    clip = true;
  } else if (clip_k > 0.0) {
    tau = (float)(clip_k * norm * (double)inv / std::sqrt((double)m * (double)n));
    clip = true;
  }
  if (clip)
    for (int64_t i = 0; i < m * n; ++i) X0[i] = X0[i] > tau ? tau : (X0[i] < -tau ? -tau : X0[i]);
  if (inv_out) *inv_out = inv;
  if (tau_out) *tau_out = tau;
  return norm;
}

// One NVFP4 Newton-Schulz iteration k on the FP32 m x n X (m <= n), in place.
void nvfp4_iteration(float* X, int64_t m, int64_t n, double a, double b, double c, int k,
                     const Opts& o) {
  const int hX = o.masks ? o.masks[3 * k] : -1;       // H of A_k = qX qX^T
  const int hA = o.masks ? o.masks[3 * k + 1] : -1;   // H of qA qA16
  const int hU = o.masks ? o.masks[3 * k + 2] : -1;   // H' of qB qX16
  std::vector<double> dX((size_t)(m * n)), dX16((size_t)(m * n));
  q1x16(X, m, n, o.flags, hX, dX.data(), nullptr);       // qX = Q1x16(X H)
  q16x1(X, m, n, o.flags, hU, dX16.data());              // qX16x1 = Q16x1(H'^T X)
  // A = qX qX^T (upper triangle, mirrored), FP32
  std::vector<double> dXt((size_t)(m * n));
  for (int64_t r = 0; r < m; ++r)
    for (int64_t kk = 0; kk < n; ++kk) dXt[kk * m + r] = dX[r * n + kk];
  std::vector<double> A64((size_t)(m * m));
  product(dX.data(), dXt.data(), m, n, m, A64.data());
  std::vector<float> A((size_t)(m * m));
  for (int64_t i = 0; i < m; ++i)
    for (int64_t j = i; j < m; ++j) A[i * m + j] = A[j * m + i] = (float)A64[i * m + j];
  // B = b A + c qA qA16x1 with qA = Q1x16(A H), qA16x1 = Q16x1(H^T A), FP32
  std::vector<double> dA((size_t)(m * m)), dA16((size_t)(m * m)), P((size_t)(m * m));
  q1x16(A.data(), m, m, o.flags, hA, dA.data(), nullptr);
  q16x1(A.data(), m, m, o.flags, hA, dA16.data());
  product(dA.data(), dA16.data(), m, m, m, P.data());
  std::vector<float> B((size_t)(m * m));
  for (int64_t i = 0; i < m * m; ++i) B[i] = (float)(b * (double)A[i] + c * P[i]);
  // X' = a X + qB qX16x1 with qB = Q1x16(B H'), FP32
  std::vector<double> dB((size_t)(m * m)), U((size_t)(m * n));
  q1x16(B.data(), m, m, o.flags, hU, dB.data(), nullptr);
  product(dB.data(), dX16.data(), m, m, n, U.data());
  for (int64_t i = 0; i < m * n; ++i) X[i] = (float)(a * (double)X[i] + U[i]);
}

// FP32 -> BF16 (round to nearest, ties to even, on the low 16 bits), returned as the
// FP32 number that BF16 value is.  Finite inputs.
float bf16_round(float x) {
  uint32_t bits;
  std::memcpy(&bits, &x, 4);
  const uint32_t keep = bits >> 16, rest = bits & 0xFFFFu;
  const uint32_t up = (rest > 0x8000u || (rest == 0x8000u && (keep & 1u))) ? 1u : 0u;
  bits = (keep + up) << 16;
  float y;
  std::memcpy(&y, &bits, 4);
  return y;
}

// One BF16 Newton-Schulz iteration on the FP32 m x n X (m <= n), in place:
// Xb = bf16(X), A = Xb Xb^T, B = b A + c bf16(A) bf16(A)^T, X' = a X + bf16(B) Xb.
void bf16_iteration(float* X, int64_t m, int64_t n, double a, double b, double c) {
  std::vector<double> Xb((size_t)(m * n)), Xbt((size_t)(m * n));
  for (int64_t r = 0; r < m; ++r)
    for (int64_t k = 0; k < n; ++k) {
      Xb[r * n + k] = (double)bf16_round(X[r * n + k]);
      Xbt[k * m + r] = Xb[r * n + k];
    }
  std::vector<double> A64((size_t)(m * m));
  product(Xb.data(), Xbt.data(), m, n, m, A64.data());
  std::vector<float> A((size_t)(m * m));
  for (int64_t i = 0; i < m; ++i)
    for (int64_t j = i; j < m; ++j) A[i * m + j] = A[j * m + i] = (float)A64[i * m + j];
  std::vector<double> Ab((size_t)(m * m)), Abt((size_t)(m * m)), P((size_t)(m * m));
  for (int64_t i = 0; i < m; ++i)
    for (int64_t j = 0; j < m; ++j) {
      Ab[i * m + j] = (double)bf16_round(A[i * m + j]);
      Abt[j * m + i] = Ab[i * m + j];
    }
  product(Ab.data(), Abt.data(), m, m, m, P.data());
  std::vector<double> Bb((size_t)(m * m)), U((size_t)(m * n));
  for (int64_t i = 0; i < m * m; ++i)
    Bb[i] = (double)bf16_round((float)(b * (double)A[i] + c * P[i]));
  product(Bb.data(), Xb.data(), m, m, n, U.data());
  for (int64_t i = 0; i < m * n; ++i) X[i] = (float)(a * (double)X[i] + U[i]);
}

// SplitMix64 output at counter idx + 1 from seed (Steele, Lea and Flood, OOPSLA 2014).
uint64_t splitmix64(uint64_t seed, uint64_t idx) {
  uint64_t z = seed + (idx + 1) * 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

// FP32 u in [0, 1): the top 24 bits of splitmix64 times 2^-24 (exact).
float uniform24(uint64_t seed, uint64_t idx) {
  return (float)std::ldexp((double)(splitmix64(seed, idx) >> 40), -24);
}

// NVFP4 state of the FP32 rows x cols momentum m_t: Q(m_t H16^r) with stochastically
// rounded element codes and adaptive 4/6 block scales (1x16 row blocks, unpacked codes).
void store_state(const float* m_t, int64_t rows, int64_t cols, uint16_t mask, uint64_t seed,
                 uint8_t* nib, uint8_t* scales, float* s_g_out) {
  std::vector<float> y(m_t, m_t + rows * cols);
  hadamard_rows(y.data(), rows, cols, mask);
  const float sg = tensor_scale(amax_of(y.data(), rows * cols), 0, kSgDenom46);
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t jb = 0; jb < cols / kBlock; ++jb) {
      const float* xb = y.data() + r * cols + jb * kBlock;
      float u[kBlock];
      for (int i = 0; i < kBlock; ++i) u[i] = uniform24(seed, (uint64_t)(r * cols + jb * kBlock + i));
      Block q = quantize_block(xb, sg, 6.0f, u);
      const Block q4 = quantize_block(xb, sg, 4.0f, u);
      if (block_sq_error(xb, q4) < block_sq_error(xb, q)) q = q4;
      scales[r * (cols / kBlock) + jb] = (uint8_t)q.scale;
      for (int i = 0; i < kBlock; ++i) nib[r * cols + jb * kBlock + i] = q.code[i];
    }
  }
  *s_g_out = sg;
}

// FP32 momentum decoded from a state: fp32(fp32(code s_b) s_g), then (H16^r)^-1.
void load_state(const uint8_t* nib, const uint8_t* scales, float s_g, uint16_t mask, int64_t rows,
                int64_t cols, float* out) {
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t c = 0; c < cols; ++c) {
      const float cs = (float)(e2m1_value(nib[r * cols + c]) *
                               e4m3_value(scales[r * (cols / kBlock) + c / kBlock]));   // exact
      out[r * cols + c] = cs * s_g;
    }
  hadamard_rows(out, rows, cols, 0);   // the butterfly and * 0.25, no signs
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t c = 0; c < cols; ++c)
      if ((mask >> (c % kBlock)) & 1) out[r * cols + c] = -out[r * cols + c];
}

// One float64 Newton-Schulz iteration (Section 2), in place.
void f64_iteration(double* X, int64_t m, int64_t n, double a, double b, double c) {
  std::vector<double> Xt((size_t)(m * n)), A((size_t)(m * m)), A2((size_t)(m * m)),
      U((size_t)(m * n));
  for (int64_t r = 0; r < m; ++r)
    for (int64_t k = 0; k < n; ++k) Xt[k * m + r] = X[r * n + k];
  product(X, Xt.data(), m, n, m, A.data());
  product(A.data(), A.data(), m, m, m, A2.data());
  for (int64_t i = 0; i < m * m; ++i) A2[i] = b * A[i] + c * A2[i];
  product(A2.data(), X, m, m, n, U.data());
  for (int64_t i = 0; i < m * n; ++i) X[i] = a * X[i] + U[i];
}

void set_threads(int threads) {
#ifdef _OPENMP
  if (threads > 0) omp_set_num_threads(threads);
#else
  (void)threads;
#endif
}

}  // namespace

extern "C" {

// Threads the parallel loops use (OpenMP's current setting).
int fs4o_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

double fs4o_e2m1_value(int code) { return e2m1_value(code); }
double fs4o_e4m3_value(int byte) { return e4m3_value(byte); }
int fs4o_e2m1_encode(double q) { return e2m1_encode(q); }
int fs4o_e4m3_encode(double v) { return e4m3_encode(v); }
float fs4o_tensor_scale(float amax, int amax_mode) { return tensor_scale(amax, amax_mode); }

// Q1x16 of x (rows x cols, cols % 16 == 0): packed codes (element 2j in the low
// nibble of byte j), scale bytes, tensor scale.  s_g_in > 0 uses that tensor scale,
// otherwise it is derived from the exact amax.  flags: bit 0 (1) s_g = amax / denom
// instead of a power of two; bit 1 (2) adaptive 4/6 blocks (denom 1792, else 2688).
// Returns 0, or -1 for a bad shape.
int fs4o_quantize_rows(const float* x, int64_t rows, int64_t cols, float s_g_in, int flags,
                       uint8_t* codes, uint8_t* scales, float* s_g_out, int threads) {
  if (rows < 1 || cols < kBlock || cols % kBlock) return -1;
  set_threads(threads);
  const bool a46 = flags & kAdaptive46;
  const float sg = s_g_in > 0.0f ? s_g_in
                                 : tensor_scale(amax_of(x, rows * cols), flags & kAmaxMode,
                                                a46 ? kSgDenom46 : kSgDenom);
  std::vector<uint8_t> nib((size_t)(rows * cols));
  quantize_rows(x, rows, cols, sg, a46, nib.data(), scales);
  for (int64_t i = 0; i < rows * cols / 2; ++i)
    codes[i] = (uint8_t)(nib[2 * i] | (nib[2 * i + 1] << 4));
  *s_g_out = sg;
  return 0;
}

// y = x H16^r (FP32, every 16-element block of each row; x and y rows x cols, may
// alias), H16^r = D H16 / 4 with D from the sign mask.  Returns 0, or -1 for a bad
// shape.
int fs4o_hadamard_rows(const float* x, int64_t rows, int64_t cols, int mask, float* y) {
  if (rows < 1 || cols < kBlock || cols % kBlock || mask < 0 || mask > 0xFFFF) return -1;
  if (y != x) std::memcpy(y, x, sizeof(float) * (size_t)(rows * cols));
  hadamard_rows(y, rows, cols, (uint16_t)mask);
  return 0;
}

// Exact float64 dequantisation of packed Q1x16 codes.
int fs4o_dequantize_rows(const uint8_t* codes, const uint8_t* scales, float s_g, int64_t rows,
                         int64_t cols, double* out, int threads) {
  if (rows < 1 || cols < kBlock || cols % kBlock) return -1;
  set_threads(threads);
  std::vector<uint8_t> nib((size_t)(rows * cols));
  for (int64_t i = 0; i < rows * cols / 2; ++i) {
    nib[2 * i] = codes[i] & 0xF;
    nib[2 * i + 1] = codes[i] >> 4;
  }
  dequantize_rows(nib.data(), scales, s_g, rows, cols, out);
  return 0;
}

// out (M x N) = L (M x K) R (K x N) in float64.
int fs4o_product(const double* L, const double* R, int64_t M, int64_t K, int64_t N, double* out,
                 int threads) {
  if (M < 1 || K < 1 || N < 1) return -1;
  set_threads(threads);
  product(L, R, M, K, N, out);
  return 0;
}

// X_0 of an m x n FP32 matrix (already in working orientation).  clip_quantile > 0:
// nearest-rank quantile clip; else clip_k > 0: clip_k * RMS; else no clip.
double fs4o_normalise_and_clip(const float* G, int64_t m, int64_t n, double clip_k,
                               double clip_quantile, float* X0, float* inv, float* tau) {
  return normalise_and_clip(G, m, n, clip_k, clip_quantile, X0, inv, tau);
}

// K NVFP4 iterations from an FP32 working-orientation X_0 (m <= n), in place.
// masks: null (H = I) or 3K sign masks of H16^r; flags: as fs4o_quantize_rows,
// applied to every quantisation.
int fs4o_ns_iterations_nvfp4(float* X, int64_t m, int64_t n, int K, double a, double b, double c,
                             const uint16_t* masks, int flags, int threads) {
  if (m < 1 || n < 1 || m % kBlock || n % kBlock || K < 0) return -1;
  set_threads(threads);
  Opts o;
  o.flags = flags;
  o.masks = masks;
  for (int k = 0; k < K; ++k) nvfp4_iteration(X, m, n, a, b, c, k, o);
  return 0;
}

// The whole step on an FP32 m0 x n0 matrix G: normalise, clip, K iterations.
// quantized = 1: the NVFP4 route, result in out32 (m0 x n0 FP32), with the masks
// and flags of fs4o_ns_iterations_nvfp4.  quantized = 2: the BF16 route (masks and
// flags ignored), result in out32.
// quantized = 0: the float64 route of Section 2 (normalisation and clip in float64),
// result in out64.  clip_quantile > 0 replaces the clip_k * RMS clip on both routes.
// Returns 0, or -1 for a bad shape or non-finite input.
int fs4o_root_ns(const float* G, int64_t m0, int64_t n0, int K, double a, double b, double c,
                 double clip_k, double clip_quantile, int quantized, const uint16_t* masks,
                 int flags, float* out32, double* out64, int threads) {
  if (m0 < 1 || n0 < 1 || K < 0) return -1;
  for (int64_t i = 0; i < m0 * n0; ++i)
    if (!std::isfinite(G[i])) return -1;
  set_threads(threads);
  const bool tall = m0 > n0;
  const int64_t m = tall ? n0 : m0, n = tall ? m0 : n0;
  std::vector<float> W((size_t)(m * n));
  if (tall) transpose(G, m0, n0, W.data());
  else std::memcpy(W.data(), G, sizeof(float) * (size_t)(m * n));
  if (quantized) {
    if (m % kBlock || n % kBlock) return -1;
    std::vector<float> X((size_t)(m * n));
    normalise_and_clip(W.data(), m, n, clip_k, clip_quantile, X.data(), nullptr, nullptr);
    Opts o;
    o.flags = flags;
    o.masks = masks;
    for (int k = 0; k < K; ++k) {
      if (quantized == 2) bf16_iteration(X.data(), m, n, a, b, c);
      else nvfp4_iteration(X.data(), m, n, a, b, c, k, o);
    }
    if (tall) transpose(X.data(), m, n, out32);
    else std::memcpy(out32, X.data(), sizeof(float) * (size_t)(m * n));
  } else {
    std::vector<double> X((size_t)(m * n));
    double s = 0.0;
    for (int64_t i = 0; i < m * n; ++i) s += (double)W[i] * (double)W[i];
    const double norm = std::sqrt(s);
    for (int64_t i = 0; i < m * n; ++i) X[i] = (double)W[i] / (norm + kEps);
    double tau = -1.0;
    if (clip_quantile > 0.0) {
      std::vector<double> a0((size_t)(m * n));
      for (int64_t i = 0; i < m * n; ++i) a0[i] = std::fabs(X[i]);
      tau = kth_smallest(a0.data(), m * n, quantile_rank(clip_quantile, m * n));
    } else if (clip_k > 0.0) {
      double s0 = 0.0;
      for (int64_t i = 0; i < m * n; ++i) s0 += X[i] * X[i];
      tau = clip_k * std::sqrt(s0) / std::sqrt((double)(m * n));
    }
    if (tau >= 0.0)
      for (int64_t i = 0; i < m * n; ++i) X[i] = X[i] > tau ? tau : (X[i] < -tau ? -tau : X[i]);
    for (int k = 0; k < K; ++k) f64_iteration(X.data(), m, n, a, b, c);
    for (int64_t r = 0; r < m; ++r)
      for (int64_t cc = 0; cc < n; ++cc) {
        const double v = X[r * n + cc];
        if (tall) out64[cc * m + r] = v;
        else out64[r * n + cc] = v;
      }
  }
  return 0;
}

// FP32 -> BF16 -> FP32 of n values (round to nearest, ties to even).
void fs4o_bf16_round(const float* x, int64_t n, float* y) {
  for (int64_t i = 0; i < n; ++i) y[i] = bf16_round(x[i]);
}

// K BF16 iterations from an FP32 working-orientation X_0 (m <= n), in place.
int fs4o_ns_iterations_bf16(float* X, int64_t m, int64_t n, int K, double a, double b, double c,
                            int threads) {
  if (m < 1 || n < 1 || K < 0) return -1;
  set_threads(threads);
  for (int k = 0; k < K; ++k) bf16_iteration(X, m, n, a, b, c);
  return 0;
}

// SplitMix64 outputs at counters idx[0 .. count) + 1, and the u24 draws.
void fs4o_splitmix64(uint64_t seed, const uint64_t* idx, int64_t count, uint64_t* out) {
  for (int64_t i = 0; i < count; ++i) out[i] = splitmix64(seed, idx[i]);
}
void fs4o_uniform24(uint64_t seed, const uint64_t* idx, int64_t count, float* out) {
  for (int64_t i = 0; i < count; ++i) out[i] = uniform24(seed, idx[i]);
}

// Stochastic rounding of FP32 v >= 0 (finite) onto an E2M1 magnitude code 0..7.
int fs4o_e2m1_encode_sr(float v, float u) { return e2m1_encode_sr(v, u); }

// One NVFP4 first-moment step on a rows x cols FP32 gradient g (cols % 16 == 0):
// m_t (FP32) and the new state (packed codes, scale bytes, s_g).  The previous state is
// given by prev_codes / prev_scales / prev_sg with sign mask mask_prev, or
// prev_codes = null for a zero previous moment.  Returns 0, or -1 for a bad shape.
int fs4o_momentum_update(const float* g, int64_t rows, int64_t cols, double beta,
                         const uint8_t* prev_codes, const uint8_t* prev_scales, float prev_sg,
                         int mask_prev, int mask_next, uint64_t seed, float* m_t, uint8_t* codes,
                         uint8_t* scales, float* s_g, int threads) {
  if (rows < 1 || cols < kBlock || cols % kBlock) return -1;
  if (mask_prev < 0 || mask_prev > 0xFFFF || mask_next < 0 || mask_next > 0xFFFF) return -1;
  set_threads(threads);
  std::vector<float> mp((size_t)(rows * cols), 0.0f);
  if (prev_codes) {
    std::vector<uint8_t> nib((size_t)(rows * cols));
    for (int64_t i = 0; i < rows * cols / 2; ++i) {
      nib[2 * i] = prev_codes[i] & 0xF;
      nib[2 * i + 1] = prev_codes[i] >> 4;
    }
    load_state(nib.data(), prev_scales, prev_sg, (uint16_t)mask_prev, rows, cols, mp.data());
  }
  const float b = (float)beta;
  const float omb = 1.0f - b;
  for (int64_t i = 0; i < rows * cols; ++i) {
    const float t1 = b * mp[i];
    const float t2 = omb * g[i];
    m_t[i] = t1 + t2;
  }
  std::vector<uint8_t> nib((size_t)(rows * cols));
  store_state(m_t, rows, cols, (uint16_t)mask_next, seed, nib.data(), scales, s_g);
  for (int64_t i = 0; i < rows * cols / 2; ++i)
    codes[i] = (uint8_t)(nib[2 * i] | (nib[2 * i + 1] << 4));
  return 0;
}

// FP32 momentum decoded from a state (packed codes).
int fs4o_momentum_load(const uint8_t* codes, const uint8_t* scales, float s_g, int mask,
                       int64_t rows, int64_t cols, float* out) {
  if (rows < 1 || cols < kBlock || cols % kBlock || mask < 0 || mask > 0xFFFF) return -1;
  std::vector<uint8_t> nib((size_t)(rows * cols));
  for (int64_t i = 0; i < rows * cols / 2; ++i) {
    nib[2 * i] = codes[i] & 0xF;
    nib[2 * i + 1] = codes[i] >> 4;
  }
  load_state(nib.data(), scales, s_g, (uint16_t)mask, rows, cols, out);
  return 0;
}

}  // extern "C"

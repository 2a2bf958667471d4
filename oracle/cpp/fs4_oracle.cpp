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

float tensor_scale(float amax, int amax_mode) {
  if (!(amax > 0.0f)) return 1.0f;
  if (amax_mode) return amax / 2688.0f;
  int e = std::ilogb((double)amax) - 12;
  while (std::ldexp(kSgDenom, e) < (double)amax) ++e;
  while (std::ldexp(kSgDenom, e - 1) >= (double)amax) --e;
  if (e < -116) e = -116;
  if (e > 118) e = 118;
  return (float)std::ldexp(1.0, e);
}

// Q1x16 of an FP32 rows x cols matrix (cols % 16 == 0) with tensor scale s_g:
// 4-bit codes (one per element, unpacked) and E4M3 scale bytes.
void quantize_rows(const float* x, int64_t rows, int64_t cols, float s_g, uint8_t* nib,
                   uint8_t* scales) {
  const float six_sg = 6.0f * s_g;
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t jb = 0; jb < cols / kBlock; ++jb) {
      const float* xb = x + r * cols + jb * kBlock;
      float amax = 0.0f;
      for (int i = 0; i < kBlock; ++i) amax = std::fmax(amax, std::fabs(xb[i]));
      const float v = amax / six_sg;
      const int s = e4m3_encode((double)v);
      scales[r * (cols / kBlock) + jb] = (uint8_t)s;
      const float den = (float)e4m3_value(s) * s_g;
      for (int i = 0; i < kBlock; ++i) {
        uint8_t code = 0;
        if (den > 0.0f) {
          const float q = std::fabs(xb[i]) / den;
          code = (uint8_t)(e2m1_encode((double)q) | (std::signbit(xb[i]) ? 8 : 0));
        }
        nib[r * cols + jb * kBlock + i] = code;
      }
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

// Dequantised Q1x16(x) (s_g from the exact amax) as a rows x cols float64 matrix.
void q1x16(const float* x, int64_t rows, int64_t cols, double* out, float* sg_out) {
  std::vector<uint8_t> nib((size_t)(rows * cols)), sc((size_t)(rows * cols / kBlock));
  const float sg = tensor_scale(amax_of(x, rows * cols), 0);
  quantize_rows(x, rows, cols, sg, nib.data(), sc.data());
  dequantize_rows(nib.data(), sc.data(), sg, rows, cols, out);
  if (sg_out) *sg_out = sg;
}

// Dequantised Q16x1(x): blocks of 16 down each column, returned as the rows x cols
// matrix (the quantisation of x^T, transposed back).
void q16x1(const float* x, int64_t rows, int64_t cols, double* out) {
  std::vector<float> xt((size_t)(rows * cols));
  transpose(x, rows, cols, xt.data());
  std::vector<double> dt((size_t)(rows * cols));
  q1x16(xt.data(), cols, rows, dt.data(), nullptr);
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

// X_0 from G (m x n, working orientation): returns ||G||_F.
double normalise_and_clip(const float* G, int64_t m, int64_t n, double clip_k, float* X0,
                          float* inv_out, float* tau_out) {
  double s = 0.0;
  for (int64_t i = 0; i < m * n; ++i) s += (double)G[i] * (double)G[i];
  const double norm = std::sqrt(s);
  const float inv = (float)(1.0 / (norm + kEps));
  for (int64_t i = 0; i < m * n; ++i) X0[i] = G[i] * inv;
  float tau = 0.0f;
  if (clip_k > 0.0) {
    tau = (float)(clip_k * norm * (double)inv / std::sqrt((double)m * (double)n));
    for (int64_t i = 0; i < m * n; ++i) X0[i] = X0[i] > tau ? tau : (X0[i] < -tau ? -tau : X0[i]);
  }
  if (inv_out) *inv_out = inv;
  if (tau_out) *tau_out = tau;
  return norm;
}

// One NVFP4 Newton-Schulz iteration on the FP32 m x n X (m <= n), in place.
void nvfp4_iteration(float* X, int64_t m, int64_t n, double a, double b, double c) {
  std::vector<double> dX((size_t)(m * n)), dX16((size_t)(m * n));
  q1x16(X, m, n, dX.data(), nullptr);       // qX
  q16x1(X, m, n, dX16.data());              // qX16x1
  // A = qX qX^T (upper triangle, mirrored), FP32
  std::vector<double> dXt((size_t)(m * n));
  for (int64_t r = 0; r < m; ++r)
    for (int64_t k = 0; k < n; ++k) dXt[k * m + r] = dX[r * n + k];
  std::vector<double> A64((size_t)(m * m));
  product(dX.data(), dXt.data(), m, n, m, A64.data());
  std::vector<float> A((size_t)(m * m));
  for (int64_t i = 0; i < m; ++i)
    for (int64_t j = i; j < m; ++j) A[i * m + j] = A[j * m + i] = (float)A64[i * m + j];
  // B = b A + c qA qA16x1, FP32
  std::vector<double> dA((size_t)(m * m)), dA16((size_t)(m * m)), P((size_t)(m * m));
  q1x16(A.data(), m, m, dA.data(), nullptr);
  q16x1(A.data(), m, m, dA16.data());
  product(dA.data(), dA16.data(), m, m, m, P.data());
  std::vector<float> B((size_t)(m * m));
  for (int64_t i = 0; i < m * m; ++i) B[i] = (float)(b * (double)A[i] + c * P[i]);
  // X' = a X + qB qX16x1, FP32
  std::vector<double> dB((size_t)(m * m)), U((size_t)(m * n));
  q1x16(B.data(), m, m, dB.data(), nullptr);
  product(dB.data(), dX16.data(), m, m, n, U.data());
  for (int64_t i = 0; i < m * n; ++i) X[i] = (float)(a * (double)X[i] + U[i]);
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
// otherwise it is derived from the exact amax (amax_mode: 0 power of two,
// 1 amax / 2688).  Returns 0, or -1 for a bad shape.
int fs4o_quantize_rows(const float* x, int64_t rows, int64_t cols, float s_g_in, int amax_mode,
                       uint8_t* codes, uint8_t* scales, float* s_g_out, int threads) {
  if (rows < 1 || cols < kBlock || cols % kBlock) return -1;
  set_threads(threads);
  const float sg = s_g_in > 0.0f ? s_g_in : tensor_scale(amax_of(x, rows * cols), amax_mode);
  std::vector<uint8_t> nib((size_t)(rows * cols));
  quantize_rows(x, rows, cols, sg, nib.data(), scales);
  for (int64_t i = 0; i < rows * cols / 2; ++i)
    codes[i] = (uint8_t)(nib[2 * i] | (nib[2 * i + 1] << 4));
  *s_g_out = sg;
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

// X_0 of an m x n FP32 matrix (already in working orientation); clip_k <= 0: no clip.
double fs4o_normalise_and_clip(const float* G, int64_t m, int64_t n, double clip_k, float* X0,
                               float* inv, float* tau) {
  return normalise_and_clip(G, m, n, clip_k, X0, inv, tau);
}

// K NVFP4 iterations from an FP32 working-orientation X_0 (m <= n), in place.
int fs4o_ns_iterations_nvfp4(float* X, int64_t m, int64_t n, int K, double a, double b, double c,
                             int threads) {
  if (m < 1 || n < 1 || m % kBlock || n % kBlock || K < 0) return -1;
  set_threads(threads);
  for (int k = 0; k < K; ++k) nvfp4_iteration(X, m, n, a, b, c);
  return 0;
}

// The whole step on an FP32 m0 x n0 matrix G: normalise, clip, K iterations.
// quantized = 1: the NVFP4 route, result in out32 (m0 x n0 FP32).
// quantized = 0: the float64 route of Section 2 (normalisation and clip in float64),
// result in out64.  Returns 0, or -1 for a bad shape or non-finite input.
int fs4o_root_ns(const float* G, int64_t m0, int64_t n0, int K, double a, double b, double c,
                 double clip_k, int quantized, float* out32, double* out64, int threads) {
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
    normalise_and_clip(W.data(), m, n, clip_k, X.data(), nullptr, nullptr);
    for (int k = 0; k < K; ++k) nvfp4_iteration(X.data(), m, n, a, b, c);
    if (tall) transpose(X.data(), m, n, out32);
    else std::memcpy(out32, X.data(), sizeof(float) * (size_t)(m * n));
  } else {
    std::vector<double> X((size_t)(m * n));
    double s = 0.0;
    for (int64_t i = 0; i < m * n; ++i) s += (double)W[i] * (double)W[i];
    const double norm = std::sqrt(s);
    for (int64_t i = 0; i < m * n; ++i) X[i] = (double)W[i] / (norm + kEps);
    if (clip_k > 0.0) {
      double s0 = 0.0;
      for (int64_t i = 0; i < m * n; ++i) s0 += X[i] * X[i];
      const double tau = clip_k * std::sqrt(s0) / std::sqrt((double)(m * n));
      for (int64_t i = 0; i < m * n; ++i) X[i] = X[i] > tau ? tau : (X[i] < -tau ? -tau : X[i]);
    }
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

}  // extern "C"
